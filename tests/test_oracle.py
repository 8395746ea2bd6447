"""Pins for the CPU oracle (runs without a GPU).

The oracle is the plain direct convolution the three MLX pull requests check
their kernels against ("CPU reference" / "CPU convolution").  None of these
tests re-types its formula with the oracle's own code: each one checks it
against something independent --

* brute force in exact integer arithmetic (pure-Python loops, a different
  code path) on tiny inputs over every stride/pad/dilation combination;
* closed forms: a 1x1 convolution is a matrix product, a delta kernel is the
  identity or a known shift, an all-ones kernel counts in-bounds neighbours;
* textbook identities: linearity, stride = subsampled stride-1 output,
  dilation = zero-inserted kernel, conv3d with KD = 1 = per-frame conv2d and
  conv3d = the sum of its depth taps ("Decompose small kernel-depth 3D convs
  into 2D convs", section Change);
* a library routine: torch.nn.functional.conv2d/conv3d in float64 on CPU;
* the exact decoding of every fp16 and bf16 bit pattern.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from dense_convolution_nhwc_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# Independent brute force: exact Python integers, nested lists
# ---------------------------------------------------------------------------

def brute_conv2d(x, w, stride, pad, dil):
    """x: nested list [N][H][W][C] of ints, w: [O][KH][KW][C] of ints."""
    N, H, W, C = len(x), len(x[0]), len(x[0][0]), len(x[0][0][0])
    O, KH, KW = len(w), len(w[0]), len(w[0][0])
    OH = (H + 2 * pad[0] - dil[0] * (KH - 1) - 1) // stride[0] + 1
    OW = (W + 2 * pad[1] - dil[1] * (KW - 1) - 1) // stride[1] + 1
    out = [[[[0] * O for _ in range(OW)] for _ in range(OH)] for _ in range(N)]
    for n in range(N):
        for oy in range(OH):
            for ox in range(OW):
                for o in range(O):
                    s = 0
                    for ky in range(KH):
                        for kx in range(KW):
                            iy = oy * stride[0] - pad[0] + ky * dil[0]
                            ix = ox * stride[1] - pad[1] + kx * dil[1]
                            if 0 <= iy < H and 0 <= ix < W:
                                for c in range(C):
                                    s += x[n][iy][ix][c] * w[o][ky][kx][c]
                    out[n][oy][ox][o] = s
    return out


def brute_conv3d(x, w, stride, pad, dil):
    N, D, H, W, C = len(x), len(x[0]), len(x[0][0]), len(x[0][0][0]), len(x[0][0][0][0])
    O, KD, KH, KW = len(w), len(w[0]), len(w[0][0]), len(w[0][0][0])
    dims = [(D, KD), (H, KH), (W, KW)]
    OD, OH, OW = [(i + 2 * pad[a] - dil[a] * (k - 1) - 1) // stride[a] + 1 for a, (i, k) in enumerate(dims)]
    out = np.zeros((N, OD, OH, OW, O), dtype=object)
    for n, oz, oy, ox, o in itertools.product(range(N), range(OD), range(OH), range(OW), range(O)):
        s = 0
        for kz, ky, kx in itertools.product(range(KD), range(KH), range(KW)):
            iz = oz * stride[0] - pad[0] + kz * dil[0]
            iy = oy * stride[1] - pad[1] + ky * dil[1]
            ix = ox * stride[2] - pad[2] + kx * dil[2]
            if 0 <= iz < D and 0 <= iy < H and 0 <= ix < W:
                for c in range(C):
                    s += x[n][iz][iy][ix][c] * w[o][kz][ky][kx][c]
        out[n, oz, oy, ox, o] = s
    return out


def rand_int(rng, shape, lo=-4, hi=4):
    return rng.integers(lo, hi + 1, size=shape)


def as_storage(a_int, dtype):
    if dtype == "f32":
        return a_int.astype(np.float32)
    t = torch.from_numpy(a_int.astype(np.float32)).to(synth.TORCH_DTYPES[dtype])
    return t


# ---------------------------------------------------------------------------
# Brute force on tiny integer inputs: bit-exact
# ---------------------------------------------------------------------------

CASES_2D = []
for (kh, kw) in [(1, 1), (3, 3), (2, 3), (3, 1)]:
    for s in [(1, 1), (2, 2), (1, 3)]:
        for p in [(0, 0), (1, 1), (2, 1)]:
            for d in [(1, 1), (2, 2), (1, 2)]:
                CASES_2D.append(((kh, kw), s, p, d))


@pytest.mark.parametrize("k,s,p,d", CASES_2D)
def test_conv2d_brute_force_exact(k, s, p, d):
    rng = np.random.default_rng(hash((k, s, p, d)) % (2 ** 32))
    N, H, W, C, O = 2, 7, 6, 3, 2
    if H + 2 * p[0] - d[0] * (k[0] - 1) - 1 < 0 or W + 2 * p[1] - d[1] * (k[1] - 1) - 1 < 0:
        pytest.skip("empty output")
    x = rand_int(rng, (N, H, W, C))
    w = rand_int(rng, (O, k[0], k[1], C))
    want = np.array(brute_conv2d(x.tolist(), w.tolist(), s, p, d), dtype=np.float64)
    for dtype in ("f32", "f16", "bf16"):
        got = oracle.conv2d(as_storage(x, dtype), as_storage(w, dtype), dtype, s, p, d)
        assert got.shape == want.shape
        assert np.array_equal(got, want), dtype


@pytest.mark.parametrize("stride,pad,dil", [((1, 1, 1), (0, 0, 0), (1, 1, 1)),
                                            ((2, 1, 2), (1, 1, 0), (1, 2, 1)),
                                            ((1, 2, 1), (0, 1, 1), (2, 1, 1))])
def test_conv3d_brute_force_exact(stride, pad, dil):
    rng = np.random.default_rng(7)
    N, D, H, W, C, O = 2, 5, 5, 4, 2, 3
    x = rand_int(rng, (N, D, H, W, C))
    w = rand_int(rng, (O, 2, 3, 2, C))
    want = brute_conv3d(x.tolist(), w.tolist(), stride, pad, dil).astype(np.float64)
    got = oracle.conv3d(x.astype(np.float32), w.astype(np.float32), "f32", stride, pad, dil)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------------------
# Closed forms
# ---------------------------------------------------------------------------

def test_1x1_is_matmul_exact_on_integers():
    rng = np.random.default_rng(1)
    N, H, W, C, O = 3, 5, 4, 17, 9
    x = rand_int(rng, (N, H, W, C)).astype(np.float32)
    w = rand_int(rng, (O, 1, 1, C)).astype(np.float32)
    got = oracle.conv2d(x, w, "f32")
    want = x.reshape(-1, C).astype(np.float64) @ w.reshape(O, C).T.astype(np.float64)
    assert np.array_equal(got.reshape(-1, O), want)


def test_1x1_is_matmul_random_floats():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2, 6, 7, 33)).astype(np.float32)
    w = rng.standard_normal((5, 1, 1, 33)).astype(np.float32)
    got = oracle.conv2d(x, w, "f32").reshape(-1, 5)
    want = x.reshape(-1, 33).astype(np.float64) @ w.reshape(5, 33).T.astype(np.float64)
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("k,d", [(3, 1), (3, 2), (5, 1), (5, 2)])
def test_centre_delta_is_identity(k, d):
    rng = np.random.default_rng(3)
    C = 4
    x = rng.standard_normal((2, 9, 8, C)).astype(np.float32)
    w = np.zeros((C, k, k, C), np.float32)
    for c in range(C):
        w[c, k // 2, k // 2, c] = 1.0
    p = d * (k - 1) // 2
    got = oracle.conv2d(x, w, "f32", (1, 1), (p, p), (d, d))
    assert np.array_equal(got, x.astype(np.float64))


def test_offcentre_delta_is_a_shift():
    """w[o,0,0,c] = delta_oc with pad 1 and a 3x3 kernel reads in[oh-1, ow-1]:
    this pins the orientation (cross-correlation, no flip)."""
    rng = np.random.default_rng(4)
    C = 3
    x = rng.standard_normal((1, 6, 7, C)).astype(np.float32)
    w = np.zeros((C, 3, 3, C), np.float32)
    for c in range(C):
        w[c, 0, 0, c] = 1.0
    got = oracle.conv2d(x, w, "f32", (1, 1), (1, 1), (1, 1))
    want = np.zeros((1, 6, 7, C))
    want[:, 1:, 1:, :] = x[:, :-1, :-1, :]
    assert np.array_equal(got, want)
    # the bottom-right tap reads in[oh+1, ow+1]
    w2 = np.zeros((C, 3, 3, C), np.float32)
    for c in range(C):
        w2[c, 2, 2, c] = 1.0
    got2 = oracle.conv2d(x, w2, "f32", (1, 1), (1, 1), (1, 1))
    want2 = np.zeros((1, 6, 7, C))
    want2[:, :-1, :-1, :] = x[:, 1:, 1:, :]
    assert np.array_equal(got2, want2)


def test_golden_fixtures():
    """Hand-derived closed forms stored under tests/golden (each file states
    its derivation)."""
    files = sorted(f for f in os.listdir(GOLDEN) if f.endswith(".json"))
    assert files
    for f in files:
        with open(os.path.join(GOLDEN, f)) as fh:
            g = json.load(fh)
        x = np.array(g["x"], np.float32)
        w = np.array(g["w"], np.float32)
        got = oracle.conv2d(x, w, "f32", tuple(g["stride"]), tuple(g["pad"]), tuple(g["dilation"]))
        assert np.array_equal(got, np.array(g["out"], np.float64)), f


# ---------------------------------------------------------------------------
# Textbook identities
# ---------------------------------------------------------------------------

def test_linearity_exact():
    rng = np.random.default_rng(5)
    x1, x2 = rand_int(rng, (2, 6, 6, 3)), rand_int(rng, (2, 6, 6, 3))
    w1, w2 = rand_int(rng, (4, 3, 3, 3)), rand_int(rng, (4, 3, 3, 3))
    a, b = 3, -2
    f = lambda x, w: oracle.conv2d(x.astype(np.float32), w.astype(np.float32), "f32", (2, 1), (1, 2), (1, 2))
    assert np.array_equal(f(a * x1 + b * x2, w1), a * f(x1, w1) + b * f(x2, w1))
    assert np.array_equal(f(x1, a * w1 + b * w2), a * f(x1, w1) + b * f(x1, w2))


@pytest.mark.parametrize("s", [2, 3])
def test_stride_is_subsampled_stride1(s):
    rng = np.random.default_rng(6)
    x = rand_int(rng, (2, 11, 10, 3)).astype(np.float32)
    w = rand_int(rng, (2, 3, 3, 3)).astype(np.float32)
    full = oracle.conv2d(x, w, "f32", (1, 1), (1, 1), (1, 1))
    sub = oracle.conv2d(x, w, "f32", (s, s), (1, 1), (1, 1))
    assert np.array_equal(sub, full[:, ::s, ::s, :])


def test_dilation_is_zero_inserted_kernel():
    rng = np.random.default_rng(8)
    x = rand_int(rng, (1, 12, 11, 2)).astype(np.float32)
    w = rand_int(rng, (3, 3, 3, 2)).astype(np.float32)
    d = 2
    wz = np.zeros((3, 5, 5, 2), np.float32)
    wz[:, ::d, ::d, :] = w
    a = oracle.conv2d(x, w, "f32", (1, 1), (2, 2), (d, d))
    b = oracle.conv2d(x, wz, "f32", (1, 1), (2, 2), (1, 1))
    assert np.array_equal(a, b)


def test_conv3d_kd1_is_per_frame_conv2d():
    rng = np.random.default_rng(9)
    x = rand_int(rng, (2, 4, 6, 5, 3)).astype(np.float32)
    w = rand_int(rng, (4, 1, 3, 3, 3)).astype(np.float32)
    got = oracle.conv3d(x, w, "f32", (1, 1, 1), (0, 1, 1), (1, 1, 1))
    frames = x.reshape(8, 6, 5, 3)
    want = oracle.conv2d(frames, w[:, 0], "f32", (1, 1), (1, 1), (1, 1)).reshape(got.shape)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("KD", [2, 3, 5])
def test_conv3d_is_sum_of_depth_taps(KD):
    """conv3d = sum over kd of conv2d(frame view at depth offset kd, w[:, kd])."""
    rng = np.random.default_rng(10 + KD)
    T, H, W, C, O = 7, 5, 6, 3, 2
    x = rand_int(rng, (1, T, H, W, C)).astype(np.float32)
    w = rand_int(rng, (O, KD, 3, 3, C)).astype(np.float32)
    got = oracle.conv3d(x, w, "f32", (1, 1, 1), (0, 1, 1), (1, 1, 1))
    OD = T - KD + 1
    acc = np.zeros((OD, H, W, O))
    for kd in range(KD):
        view = np.ascontiguousarray(x[0, kd:kd + OD])
        acc += oracle.conv2d(view, np.ascontiguousarray(w[:, kd]), "f32", (1, 1), (1, 1), (1, 1))
    assert np.array_equal(got[0], acc)


# ---------------------------------------------------------------------------
# Library routine: torch float64 on CPU
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(6))
def test_matches_torch_conv2d_f64(seed):
    rng = np.random.default_rng(100 + seed)
    N, H, W = rng.integers(1, 3), rng.integers(5, 13), rng.integers(5, 13)
    C, O = rng.integers(1, 9), rng.integers(1, 9)
    KH, KW = rng.integers(1, 5), rng.integers(1, 5)
    s = tuple(int(v) for v in rng.integers(1, 4, 2))
    d = tuple(int(v) for v in rng.integers(1, 3, 2))
    p = tuple(int(v) for v in rng.integers(0, 3, 2))
    if H + 2 * p[0] - d[0] * (KH - 1) - 1 < 0 or W + 2 * p[1] - d[1] * (KW - 1) - 1 < 0:
        pytest.skip("empty")
    x = rng.standard_normal((N, H, W, C)).astype(np.float32)
    w = rng.standard_normal((O, KH, KW, C)).astype(np.float32)
    got = oracle.conv2d(x, w, "f32", s, p, d)
    ref = F.conv2d(torch.from_numpy(x).double().permute(0, 3, 1, 2),
                   torch.from_numpy(w).double().permute(0, 3, 1, 2), stride=s, padding=p, dilation=d)
    ref = ref.permute(0, 2, 3, 1).numpy()
    assert got.shape == ref.shape
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_matches_torch_conv3d_f64():
    rng = np.random.default_rng(200)
    x = rng.standard_normal((2, 6, 7, 5, 3)).astype(np.float32)
    w = rng.standard_normal((4, 3, 2, 3, 3)).astype(np.float32)
    s, p, d = (2, 1, 1), (1, 0, 1), (1, 2, 1)
    got = oracle.conv3d(x, w, "f32", s, p, d)
    ref = F.conv3d(torch.from_numpy(x).double().permute(0, 4, 1, 2, 3),
                   torch.from_numpy(w).double().permute(0, 4, 1, 2, 3), stride=s, padding=p, dilation=d)
    ref = ref.permute(0, 2, 3, 4, 1).numpy()
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Decoding of 16-bit storage, every bit pattern
# ---------------------------------------------------------------------------

def test_decode_every_f16_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits, "f16")
    want = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert oracle.decode(np.array([0x3C00, 0x0001, 0x7BFF, 0xC000], np.uint16), "f16").tolist() == \
        [1.0, 2.0 ** -24, 65504.0, -2.0]


def test_decode_every_bf16_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits, "bf16")
    want = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert oracle.decode(np.array([0x3F80, 0xC040, 0x0001], np.uint16), "bf16").tolist() == \
        [1.0, -3.0, 2.0 ** -133]


def test_f32_values_are_exact():
    x = np.array([1 + 2 ** -23, -3.0e38, 1e-45], np.float32)
    assert np.array_equal(oracle.decode(x, "f32"), x.astype(np.float64))


# ---------------------------------------------------------------------------
# Modes and edge cases
# ---------------------------------------------------------------------------

def test_sampled_pixels_match_full_tensor():
    x, w = synth.conv2d_inputs(synth.Conv2dShape(3, 9, 11, 5, 6, 3, 3, (2, 1), (1, 1), (1, 2)), "bf16", "normal")
    full = oracle.conv2d(x, w, "bf16", (2, 1), (1, 1), (1, 2))
    pix = synth.sample_pixels(3, full.shape[1], full.shape[2], count=20, seed=3)
    samp = oracle.conv2d(x, w, "bf16", (2, 1), (1, 1), (1, 2), pixels=pix.numpy())
    for i, (n, y, xx) in enumerate(pix.tolist()):
        assert np.array_equal(samp[i], full[n, y, xx])


def test_sampled_pixels_match_full_tensor_3d():
    """The 3D sampled mode reads (n, od, oh, ow) quadruples: each sampled row
    equals the full tensor at that position, with N > 1, OD > 1 and stride,
    padding and dilation that differ per axis (depth padding included), on
    pixels that include the first and last output frame of both images."""
    s = synth.Conv3dShape(2, 9, 8, 10, 3, 5, 3, 2, 3, (2, 1, 2), (2, 1, 1), (2, 1, 1))
    x, w = synth.conv3d_inputs(s, "f16", "normal", 4)
    full = oracle.conv3d(x, w, "f16", s.stride, s.pad, s.dilation)
    assert full.shape == (2, s.od, s.oh, s.ow, 5) and s.od > 2
    pix = synth.sample_pixels(2, s.oh, s.ow, count=40, seed=5, od=s.od)
    quads = {tuple(p) for p in pix.tolist()}
    for n in (0, 1):
        for f in (0, s.od - 1):
            assert (n, f, 0, 0) in quads and (n, f, s.oh - 1, s.ow - 1) in quads
    assert {p[1] for p in quads} >= {0, s.od - 1} and len({p[1] for p in quads}) > 2
    samp = oracle.conv3d(x, w, "f16", s.stride, s.pad, s.dilation, pixels=pix.numpy())
    assert samp.shape == (pix.shape[0], 5)
    for i, (n, f, y, xx) in enumerate(pix.tolist()):
        assert np.array_equal(samp[i], full[n, f, y, xx]), (n, f, y, xx)


def test_empty_batch_is_empty():
    x = np.zeros((0, 5, 5, 2), np.float32)
    w = np.ones((3, 3, 3, 2), np.float32)
    assert oracle.conv2d(x, w, "f32", pad=(1, 1)).shape == (0, 5, 5, 3)


def test_invalid_shapes_rejected():
    x = np.zeros((1, 2, 2, 1), np.float32)
    w = np.ones((1, 5, 5, 1), np.float32)
    with pytest.raises(ValueError):
        oracle.conv2d(x, w, "f32")        # OH <= 0


def test_sample_pixels_cover_edges():
    pix = synth.sample_pixels(4, 10, 12, count=16, seed=1)
    s = {tuple(p) for p in pix.tolist()}
    for n in (0, 3):
        for (y, xx) in [(0, 0), (0, 11), (9, 0), (9, 11)]:
            assert (n, y, xx) in s
    assert len(s) == pix.shape[0]
