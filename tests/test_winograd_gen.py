"""The Winograd F(m x m, 3 x 3) transforms the GPU path uses (CPU-only checks).

* The exact Cook-Toom matrices reproduce direct correlation in rational
  arithmetic, 1D and 2D: A^T[(G g) . (B^T d)] = sum_k g_k d_{i+k} and
  A^T[(G g G^T) . (B^T d B)]A = the 3x3 correlation of the tile (the method of
  "Fast Algorithms for Convolutional Neural Networks", Lavin and Gray).
* The same matrices nested along three axes reproduce the 3x3x3 correlation
  of an alpha^3 cube exactly (the native 3D Winograd's transforms).
* The committed header is exactly what the generator writes.
* The generated straight-line code (paired even/odd sums) computes those
  matrices: it is compiled with g++ as C++ and compared with the exact
  products on random inputs.
"""
import ctypes
import os
import random
import subprocess
import sys
import tempfile
from fractions import Fraction as Fr

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "dense_convolution_nhwc_b200", "csrc")
sys.path.insert(0, CSRC)
import gen_winograd  # noqa: E402


@pytest.mark.parametrize("m", [2, 4, 6])
def test_matrices_reproduce_1d_correlation_exactly(m):
    AT, G, BT = gen_winograd.matrices(m)
    a = m + 2
    rng = random.Random(m)
    for _ in range(20):
        g = [Fr(rng.randint(-9, 9)) for _ in range(3)]
        d = [Fr(rng.randint(-9, 9), rng.randint(1, 4)) for _ in range(a)]
        Gg = [sum(G[j][k] * g[k] for k in range(3)) for j in range(a)]
        Bd = [sum(BT[j][n] * d[n] for n in range(a)) for j in range(a)]
        y = [sum(AT[i][j] * Gg[j] * Bd[j] for j in range(a)) for i in range(m)]
        assert y == [sum(g[k] * d[i + k] for k in range(3)) for i in range(m)]


@pytest.mark.parametrize("m", [2, 4, 6])
def test_matrices_reproduce_2d_correlation_exactly(m):
    AT, G, BT = gen_winograd.matrices(m)
    a = m + 2
    rng = random.Random(10 + m)
    mm = lambda X, Y: [[sum(X[i][k] * Y[k][j] for k in range(len(Y))) for j in range(len(Y[0]))] for i in range(len(X))]
    tr = lambda X: [list(r) for r in zip(*X)]
    g = [[Fr(rng.randint(-5, 5)) for _ in range(3)] for _ in range(3)]
    d = [[Fr(rng.randint(-5, 5)) for _ in range(a)] for _ in range(a)]
    U = mm(mm(G, g), tr(G))
    V = mm(mm(BT, d), tr(BT))
    Y = mm(mm(AT, [[U[i][j] * V[i][j] for j in range(a)] for i in range(a)]), tr(AT))
    want = [[sum(g[u][v] * d[i + u][j + v] for u in range(3) for v in range(3)) for j in range(m)] for i in range(m)]
    assert Y == want


@pytest.mark.parametrize("m", [2, 4])
def test_matrices_reproduce_3d_correlation_exactly(m):
    """(A^T (x) A^T (x) A^T)[(G (x) G (x) G) g . (B^T (x) B^T (x) B^T) d] is the
    3x3x3 correlation of the alpha^3 cube d, each 1D matrix applied along one
    axis in turn (depth, height, width)."""
    AT, G, BT = gen_winograd.matrices(m)
    a = m + 2
    rng = random.Random(20 + m)

    def along(M, X, axis):
        """Apply the matrix M along one axis of the nested-list cube X."""
        n0, n1, n2 = len(X), len(X[0]), len(X[0][0])
        if axis == 0:
            return [[[sum(M[i][k] * X[k][y][z] for k in range(n0)) for z in range(n2)] for y in range(n1)]
                    for i in range(len(M))]
        if axis == 1:
            return [[[sum(M[i][k] * X[x][k][z] for k in range(n1)) for z in range(n2)] for i in range(len(M))]
                    for x in range(n0)]
        return [[[sum(M[i][k] * X[x][y][k] for k in range(n2)) for i in range(len(M))] for y in range(n1)]
                for x in range(n0)]

    def cube3(M, X):
        return along(M, along(M, along(M, X, 0), 1), 2)

    g = [[[Fr(rng.randint(-4, 4)) for _ in range(3)] for _ in range(3)] for _ in range(3)]
    d = [[[Fr(rng.randint(-4, 4)) for _ in range(a)] for _ in range(a)] for _ in range(a)]
    U, V = cube3(G, g), cube3(BT, d)
    P = [[[U[i][j][k] * V[i][j][k] for k in range(a)] for j in range(a)] for i in range(a)]
    Y = cube3(AT, P)
    want = [[[sum(g[u][v][w] * d[i + u][j + v][k + w] for u in range(3) for v in range(3) for w in range(3))
              for k in range(m)] for j in range(m)] for i in range(m)]
    assert Y == want


def test_committed_header_is_generated():
    with open(os.path.join(CSRC, "winograd_gen.cuh")) as f:
        assert f.read() == gen_winograd.emit()


@pytest.fixture(scope="module")
def compiled_transforms():
    src = r"""
#define __device__
#define __forceinline__ inline
#include "winograd_gen.cuh"
extern "C" void run(int m, int which, const float* x, float* y) {
  if (m == 2) { if (which == 0) wino2_bt(x, y); else if (which == 1) wino2_g(x, y); else wino2_at(x, y); }
  if (m == 4) { if (which == 0) wino4_bt(x, y); else if (which == 1) wino4_g(x, y); else wino4_at(x, y); }
  if (m == 6) { if (which == 0) wino6_bt(x, y); else if (which == 1) wino6_g(x, y); else wino6_at(x, y); }
}
"""
    d = tempfile.mkdtemp()
    cpp, so = os.path.join(d, "t.cpp"), os.path.join(d, "t.so")
    with open(cpp, "w") as f:
        f.write(src)
    subprocess.check_call(["g++", "-O1", "-ffp-contract=off", "-shared", "-fPIC", "-I", CSRC, cpp, "-o", so])
    lib = ctypes.CDLL(so)
    lib.run.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    return lib


@pytest.mark.parametrize("m", [2, 4, 6])
def test_generated_code_computes_the_matrices(compiled_transforms, m):
    AT, G, BT = gen_winograd.matrices(m)
    a = m + 2
    rng = np.random.default_rng(m)
    for which, M in ((0, BT), (1, G), (2, AT)):
        Mf = np.array([[float(v) for v in row] for row in M])
        n_in, n_out = Mf.shape[1], Mf.shape[0]
        for _ in range(50):
            x = rng.standard_normal(n_in).astype(np.float32)
            y = np.zeros(max(n_out, 8), np.float32)
            compiled_transforms.run(m, which, x.ctypes.data, y.ctypes.data)
            want = Mf @ x.astype(np.float64)
            scale = np.abs(Mf).sum(axis=1) * np.abs(x).max() + 1e-30
            assert np.all(np.abs(y[:n_out] - want) <= 4e-7 * scale), (m, which)
