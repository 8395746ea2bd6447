// winograd.cu -- Winograd F(m x m, 3 x 3) transforms for 3x3 stride-1 convs.
//
// The Winograd path of "Bound winograd conv2d working set by tiling the batch"
// (Problem, Fix): input transform, batched GEMM, output transform.  With
// alpha = m + 2 and T = N * ceil(OH/m) * ceil(OW/m) tiles,
//   U[xi][o][c] = (G g_oc G^T)[xi]                      filter transform
//   V[xi][t][c] = (B^T d_tc B)[xi]                      input transform
//   M[xi][t][o] = sum_c V[xi][t][c] * U[xi][o][c]        batched GEMM (elsewhere)
//   y_to        = A^T M[.][t][o] A  (m x m, cropped)     output transform
// where d_tc is the alpha x alpha input patch of tile t (origin
// (ty*m - ph, tx*m - pw)), zero outside the image: padding is applied by
// bounds, not by a padded copy of the input.  All transform arithmetic is
// fp32; U and V are stored in the GEMM's operand dtype, M is fp32.
//
// Every thread owns one (tile, channel) pair and every tile is transformed
// independently, so the result for an image does not depend on which batch
// tile it was processed in (batch tiling stays bit-identical).
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "wino_1d.cuh"
#include "wino_tile.cuh"

namespace b200conv {
namespace {

// ---------------------------------------------------------------------------
// Filter transform: one thread per (o, c).
// ---------------------------------------------------------------------------
template <int M, typename Tin, typename Tst>
__global__ void wino_filter_kernel(const Tin* __restrict__ w, long long w_row_stride, int O, int C,
                                   Tst* __restrict__ u) {
  constexpr int A = Wino<M>::A;
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)O * C) return;
  int o = (int)(idx / C), c = (int)(idx - (long long)o * C);
  const Tin* wp = w + (long long)o * w_row_stride + c;
  float g[3][3];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int j = 0; j < 3; ++j) g[i][j] = Store<Tin>::to_f32(wp[(long long)(i * 3 + j) * C]);
  // t = G g (A x 3), then U = t G^T (A x A)
  float t[A][3];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    float col[3] = {g[0][j], g[1][j], g[2][j]}, r[A];
    Wino<M>::g(col, r);
#pragma unroll
    for (int i = 0; i < A; ++i) t[i][j] = r[i];
  }
  const long long plane = (long long)O * C;
#pragma unroll
  for (int i = 0; i < A; ++i) {
    float r[A];
    Wino<M>::g(t[i], r);
#pragma unroll
    for (int j = 0; j < A; ++j) u[(long long)(i * A + j) * plane + idx] = Store<Tst>::from_f32(r[j]);
  }
}

// Filter transform for the split-bf16 fp32 GEMM: U'[xi][o][3C] bf16, the three
// C-wide segments holding the parts (b0, b1, b2) of the fp32 value.
template <int M, typename Tin>
__global__ void wino_filter_split_kernel(const Tin* __restrict__ w, long long w_row_stride, int O, int C,
                                         __nv_bfloat16* __restrict__ u) {
  constexpr int A = Wino<M>::A;
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)O * C) return;
  int o = (int)(idx / C), c = (int)(idx - (long long)o * C);
  const Tin* wp = w + (long long)o * w_row_stride + c;
  float g[3][3];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int j = 0; j < 3; ++j) g[i][j] = Store<Tin>::to_f32(wp[(long long)(i * 3 + j) * C]);
  float t[A][3];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    float col[3] = {g[0][j], g[1][j], g[2][j]}, r[A];
    Wino<M>::g(col, r);
#pragma unroll
    for (int i = 0; i < A; ++i) t[i][j] = r[i];
  }
  const long long plane = (long long)O * 3 * C;
  __nv_bfloat16* up = u + (long long)o * 3 * C + c;
#pragma unroll
  for (int i = 0; i < A; ++i) {
    float r[A];
    Wino<M>::g(t[i], r);
#pragma unroll
    for (int j = 0; j < A; ++j) {
      __nv_bfloat16 b[3];
      split_bf16x3(r[j], b[0], b[1], b[2]);
      __nv_bfloat16* q = up + (long long)(i * A + j) * plane;
      q[0] = b[0];
      q[C] = b[1];
      q[2 * C] = b[2];
    }
  }
}

template <int M, typename Idx>
__global__ void __launch_bounds__(256)
wino_input_split_kernel(const float* __restrict__ in, const WinoInArgs a, __nv_bfloat16* __restrict__ v) {
  wino_input_block<M, float, __nv_bfloat16, Idx, 1>(in, a, v, blockIdx.x, threadIdx.x, threadIdx.y, blockDim.x,
                                                    blockDim.y);
}

// Input transform: one thread per (tile, channel); threadIdx.x runs over
// channels so loads and stores are coalesced.
template <int M, typename Tin, typename Tst, typename Idx>
__global__ void __launch_bounds__(256)
wino_input_kernel(const Tin* __restrict__ in, const WinoInArgs a, Tst* __restrict__ v) {
  wino_input_block<M, Tin, Tst, Idx>(in, a, v, blockIdx.x, threadIdx.x, threadIdx.y, blockDim.x, blockDim.y);
}

// Output transform: one thread per (tile, output channel).
template <int M, typename TM, typename Tout, typename Idx>
__global__ void __launch_bounds__(256)
wino_output_kernel(const TM* __restrict__ mb, const WinoOutArgs a, Tout* __restrict__ out) {
  wino_output_block<M, TM, Tout, Idx>(mb, a, out, blockIdx.x, blockIdx.y, threadIdx.x, threadIdx.y, blockDim.x,
                                      blockDim.y);
}

// One pass of the chunked fp32 Winograd pipeline: the output transform of
// chunk i-1 and the input transform of chunk i in one launch (1D grid of
// 256-thread blocks, the input blocks first).  The output blocks wait for the
// previous kernel in the stream (the GEMM of chunk i-1) before reading M; the
// input blocks do not wait: they read only the conv's input and write the V
// buffer that the GEMM of chunk i-2 read, which had finished before that
// previous GEMM could start.  They therefore run in the SMs the previous GEMM
// frees as it drains.  Every block releases the next launch (the GEMM of
// chunk i), whose own wait covers this whole grid.
template <int M, typename Tin, typename Idx>
__global__ void __launch_bounds__(256)
wino_pass_kernel(const Tin* __restrict__ in, const WinoInArgs ai, float* __restrict__ v, long long in_blocks, int ibx,
                 const float* __restrict__ mb, const WinoOutArgs ao, Tin* __restrict__ out, unsigned ogx, int obx) {
  const long long b = blockIdx.x;
  if (b < in_blocks) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    wino_input_block<M, Tin, float, Idx>(in, ai, v, b, threadIdx.x % ibx, threadIdx.x / ibx, ibx, 256 / ibx);
  } else {
    pdl_wait_then_release();
    const long long ob = b - in_blocks;
    wino_output_block<M, float, Tin, Idx>(mb, ao, out, ob % ogx, (int)(ob / ogx), threadIdx.x % obx,
                                          threadIdx.x / obx, obx, 256 / obx);
  }
}


// ---------------------------------------------------------------------------
// 16-bit transforms on channel pairs: a thread owns channels (2p, 2p+1) of one
// tile, so each load and store moves 32 bits (the arithmetic per channel is
// that of the kernels above, bit for bit).
// ---------------------------------------------------------------------------
template <int M, typename T, typename Idx>
__global__ void __launch_bounds__(256)
wino_input_pair_kernel(const T* __restrict__ in, const WinoInArgs a, T* __restrict__ v) {
  using P = Pair<T>;
  using PT = typename P::type;
  constexpr int A = Wino<M>::A;
  const int cp = a.c >> 1;
  const int cgroups = (cp + blockDim.x - 1) / blockDim.x;
  const int cg = (int)(blockIdx.x % cgroups);
  const long long tg = blockIdx.x / cgroups;
  const int c2 = cg * blockDim.x + threadIdx.x;
  const long long t = tg * blockDim.y + threadIdx.y;
  if (c2 >= cp || t >= a.t_count) return;
  const int per_img = a.tiles_h * a.tiles_w;
  const long long tglob = a.t_base + t;
  const int nl = (int)(tglob / per_img);
  const int r = (int)(tglob - (long long)nl * per_img);
  const int ty = r / a.tiles_w, tx = r - (r / a.tiles_w) * a.tiles_w;
  const int y0 = ty * M - a.ph, x0 = tx * M - a.pw;
  const PT* base = reinterpret_cast<const PT*>(in + (long long)(a.n0 + nl) * a.in_img_stride) + c2;
  const Idx cs = cp, wc = (Idx)a.w * cp;

  float d[2][A][A];
  auto put = [&](int i, int j, PT pv) {
    const float2 f = P::to_f32(pv);
    d[0][i][j] = f.x;
    d[1][i][j] = f.y;
  };
  if (y0 >= 0 && x0 >= 0 && y0 + A <= a.h && x0 + A <= a.w) {
    const PT* p = base + ((Idx)y0 * wc + (Idx)x0 * cs);
#pragma unroll
    for (int i = 0; i < A; ++i)
#pragma unroll
      for (int j = 0; j < A; ++j) put(i, j, p[(Idx)i * wc + (Idx)j * cs]);
  } else {
    unsigned xm = 0;
#pragma unroll
    for (int j = 0; j < A; ++j)
      if (x0 + j >= 0 && x0 + j < a.w) xm |= 1u << j;
#pragma unroll
    for (int i = 0; i < A; ++i) {
      const int y = y0 + i;
      const bool yok = y >= 0 && y < a.h;
      const Idx ro = yok ? (Idx)y * wc + (Idx)x0 * cs : (Idx)0;
#pragma unroll
      for (int j = 0; j < A; ++j) {
        if (yok && ((xm >> j) & 1u)) {
          put(i, j, base[ro + (Idx)j * cs]);
        } else {
          d[0][i][j] = 0.0f;
          d[1][i][j] = 0.0f;
        }
      }
    }
  }
  float res[2][A][A];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float tt[A][A];
#pragma unroll
    for (int j = 0; j < A; ++j) {
      float col[A], rr[A];
#pragma unroll
      for (int i = 0; i < A; ++i) col[i] = d[h][i][j];
      Wino<M>::bt(col, rr);
#pragma unroll
      for (int i = 0; i < A; ++i) tt[i][j] = rr[i];
    }
#pragma unroll
    for (int i = 0; i < A; ++i) Wino<M>::bt(tt[i], res[h][i]);
  }
  const Idx plane = (Idx)(a.t_stride * cp);
  PT* vp = reinterpret_cast<PT*>(v + t * a.c) + c2;
#pragma unroll
  for (int i = 0; i < A; ++i)
#pragma unroll
    for (int j = 0; j < A; ++j) vp[(Idx)(i * A + j) * plane] = P::from_f32(res[0][i][j], res[1][i][j]);
}

template <int M, typename T, typename Idx>
__global__ void __launch_bounds__(256)
wino_output_pair_kernel(const T* __restrict__ mb, const WinoOutArgs a, T* __restrict__ out) {
  using P = Pair<T>;
  using PT = typename P::type;
  constexpr int A = Wino<M>::A;
  const int op = a.o >> 1;
  const int o2 = blockIdx.y * blockDim.x + threadIdx.x;
  const long long t = (long long)blockIdx.x * blockDim.y + threadIdx.y;
  if (o2 >= op || t >= a.t_count) return;
  const int per_img = a.tiles_h * a.tiles_w;
  const long long tglob = a.t_base + t;
  const int nl = (int)(tglob / per_img);
  const int r = (int)(tglob - (long long)nl * per_img);
  const int ty = r / a.tiles_w, tx = r - (r / a.tiles_w) * a.tiles_w;

  const Idx plane = (Idx)(a.t_stride * op);
  const PT* mp = reinterpret_cast<const PT*>(mb + t * a.o) + o2;
  float x[2][A][A];
#pragma unroll
  for (int i = 0; i < A; ++i)
#pragma unroll
    for (int j = 0; j < A; ++j) {
      const float2 f = P::to_f32(mp[(Idx)(i * A + j) * plane]);
      x[0][i][j] = f.x;
      x[1][i][j] = f.y;
    }
  float y[2][M][M];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float tt[M][A];
#pragma unroll
    for (int j = 0; j < A; ++j) {
      float col[A], rr[M];
#pragma unroll
      for (int i = 0; i < A; ++i) col[i] = x[h][i][j];
      Wino<M>::at(col, rr);
#pragma unroll
      for (int i = 0; i < M; ++i) tt[i][j] = rr[i];
    }
#pragma unroll
    for (int i = 0; i < M; ++i) Wino<M>::at(tt[i], y[h][i]);
  }
  PT* opp = reinterpret_cast<PT*>(out + (long long)(a.n0 + nl) * a.out_img_stride) + o2;
  const Idx os = op, wo = (Idx)a.ow * op;
  const bool whole = ty * M + M <= a.oh && tx * M + M <= a.ow;
#pragma unroll
  for (int i = 0; i < M; ++i) {
    const int yy = ty * M + i;
    if (!whole && yy >= a.oh) continue;
    PT* rp = opp + ((Idx)yy * wo + (Idx)(tx * M) * os);
#pragma unroll
    for (int j = 0; j < M; ++j) {
      if (!whole && tx * M + j >= a.ow) continue;
      float v0 = y[0][i][j], v1 = y[1][i][j];
      if (a.accumulate) {
        const float2 old = P::to_f32(rp[(Idx)j * os]);
        const float2 tap = P::to_f32(P::from_f32(v0, v1));
        v0 = old.x + tap.x;
        v1 = old.y + tap.y;
      }
      rp[(Idx)j * os] = P::from_f32(v0, v1);
    }
  }
}

// ---------------------------------------------------------------------------
// Channel-major variants for the FFMA GEMM: U[xi][c][o] (row stride O_pad) and
// V[xi][c][t] (row stride T_pad), fp32.  Rows of both are contiguous in the
// GEMM's m / n direction, so the GEMM stages them with 16-byte copies.
// ---------------------------------------------------------------------------
template <int M, typename Tin>
__global__ void wino_filter_cmajor_kernel(const Tin* __restrict__ w, long long w_row_stride, int O, int C,
                                          long long o_pad, float* __restrict__ u) {
  constexpr int A = Wino<M>::A;
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)O * C) return;
  const int c = (int)(idx / O), o = (int)(idx - (long long)c * O);    // o fastest: coalesced stores
  const Tin* wp = w + (long long)o * w_row_stride + c;
  float g[3][3];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int j = 0; j < 3; ++j) g[i][j] = Store<Tin>::to_f32(wp[(long long)(i * 3 + j) * C]);
  float t[A][3];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    float col[3] = {g[0][j], g[1][j], g[2][j]}, r[A];
    Wino<M>::g(col, r);
#pragma unroll
    for (int i = 0; i < A; ++i) t[i][j] = r[i];
  }
  const long long plane = (long long)C * o_pad;
  float* up = u + (long long)c * o_pad + o;
#pragma unroll
  for (int i = 0; i < A; ++i) {
    float r[A];
    Wino<M>::g(t[i], r);
#pragma unroll
    for (int j = 0; j < A; ++j) up[(long long)(i * A + j) * plane] = r[j];
  }
}

// Input transform, channel-major output.  A block transforms a strip of
// kStripTiles consecutive tiles of one tile row, for kStripChans channels:
// the strip's alpha rows x (kStripTiles*m + 2) columns x channels are staged
// in shared memory ([c][y][x]) with sector-sized global reads, then thread
// (tile, channel) transforms its alpha x alpha patch and writes V[xi][c][t]
// with consecutive threads on consecutive tiles (128-byte rows).
constexpr int kStripTiles = 32;
constexpr int kStripChans = 8;

template <int M>
struct Strip {
  static constexpr int A = M + 2;
  static constexpr int W = kStripTiles * M + 2;               // staged columns
  static constexpr int WP = W + ((1 - W) % 4 + 4) % 4;        // padded row: WP = 1 (mod 4)
  static constexpr int BYTES = kStripChans * A * WP * 4;
};

struct WinoInCArgs {
  int h, w, c, ph, pw, tiles_h, tiles_w, strips_w;
  long long in_img_stride;
  int n0;
  long long t_stride;     // row stride of V (T_pad)
};

template <int M, typename Tin>
__global__ void __launch_bounds__(256)
wino_input_cmajor_kernel(const Tin* __restrict__ in, const WinoInCArgs a, float* __restrict__ v) {
  constexpr int A = Wino<M>::A;
  using S = Strip<M>;
  extern __shared__ float sm[];     // [kStripChans][A][S::WP]
  const int tid = threadIdx.x;
  // blockIdx.x -> (image, tile row, strip, channel group), channel group fastest so
  // that concurrently running blocks together read whole pixels (C contiguous).
  const int cgroups = (a.c + kStripChans - 1) / kStripChans;
  const long long bid = blockIdx.x;
  const int cg = (int)(bid % cgroups);
  const long long strip = bid / cgroups;
  const int strips_per_img = a.tiles_h * a.strips_w;
  const int nl = (int)(strip / strips_per_img);
  const int r = (int)(strip - (long long)nl * strips_per_img);
  const int ty = r / a.strips_w, sx = r - (r / a.strips_w) * a.strips_w;
  const int c0 = cg * kStripChans;
  const int y0 = ty * M - a.ph, x0 = sx * kStripTiles * M - a.pw;
  const Tin* base = in + (long long)(a.n0 + nl) * a.in_img_stride;

  // Stage: 4 channels per load (16 bytes for fp32) when the rows allow it.
  const bool vec4 = (a.c % 4 == 0) && ((reinterpret_cast<uintptr_t>(in) & (4 * sizeof(Tin) - 1)) == 0) &&
                    (a.in_img_stride % 4 == 0);
  constexpr int Q = kStripChans / 4;
  for (int idx = tid; idx < A * S::W * Q; idx += 256) {
    const int q = idx % Q;
    const int rest = idx / Q;
    const int x = rest % S::W, y = rest / S::W;
    const int gy = y0 + y, gx = x0 + x, c = c0 + 4 * q;
    float val[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (gy >= 0 && gy < a.h && gx >= 0 && gx < a.w && c < a.c) {
      const Tin* p = base + ((long long)gy * a.w + gx) * a.c + c;
      if (vec4) {
        if constexpr (sizeof(Tin) == 4) {
          const float4 f = __ldg(reinterpret_cast<const float4*>(p));
          val[0] = f.x; val[1] = f.y; val[2] = f.z; val[3] = f.w;
        } else {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
          const Tin* e = reinterpret_cast<const Tin*>(&u);
#pragma unroll
          for (int k = 0; k < 4; ++k) val[k] = Store<Tin>::to_f32(e[k]);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (c + k < a.c) val[k] = Store<Tin>::to_f32(p[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) sm[((4 * q + k) * A + y) * S::WP + x] = val[k];
  }
  __syncthreads();

  const int txl = tid % kStripTiles, cl = tid / kStripTiles;
  const int tx = sx * kStripTiles + txl;
  const int c = c0 + cl;
  if (tx >= a.tiles_w || c >= a.c) return;
  const float* sp = sm + cl * A * S::WP + txl * M;
  float tt[A][A];
#pragma unroll
  for (int j = 0; j < A; ++j) {
    float col[A], res[A];
#pragma unroll
    for (int i = 0; i < A; ++i) col[i] = sp[i * S::WP + j];
    Wino<M>::bt(col, res);
#pragma unroll
    for (int i = 0; i < A; ++i) tt[i][j] = res[i];
  }
  const long long t = (long long)nl * a.tiles_h * a.tiles_w + (long long)ty * a.tiles_w + tx;
  const long long plane = (long long)a.c * a.t_stride;
  float* vp = v + (long long)c * a.t_stride + t;
#pragma unroll
  for (int i = 0; i < A; ++i) {
    float res[A];
    Wino<M>::bt(tt[i], res);
#pragma unroll
    for (int j = 0; j < A; ++j) vp[(long long)(i * A + j) * plane] = res[j];
  }
}

}  // namespace

cudaError_t launch_wino_filter(const void* w, long long w_row_stride, int o, int c, int m,
                               conv_dtype_t in_dt, conv_dtype_t store_dt, void* u, cudaStream_t s) {
  long long n = (long long)o * c;
  if (n == 0) return cudaSuccess;
  unsigned blocks = (unsigned)((n + 255) / 256);
  return wino_by_m(m, [&](auto mc) {
    constexpr int M = decltype(mc)::value;
    return wino_by_dt(in_dt, [&](auto ti) {
      using Tin = decltype(ti);
      return wino_by_dt(store_dt, [&](auto ts) {
        using Tst = decltype(ts);
        wino_filter_kernel<M, Tin, Tst><<<blocks, 256, 0, s>>>(
            static_cast<const Tin*>(w), w_row_stride, o, c, static_cast<Tst*>(u));
        return cudaGetLastError();
      });
    });
  });
}

cudaError_t launch_wino_filter_split(const float* w, long long w_row_stride, int o, int c, void* u,
                                     cudaStream_t s) {
  long long n = (long long)o * c;
  if (n == 0) return cudaSuccess;
  wino_filter_split_kernel<6, float><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
      w, w_row_stride, o, c, static_cast<__nv_bfloat16*>(u));
  return cudaGetLastError();
}

cudaError_t launch_wino_input_split(const float* in, const Geom& g, int n0, long long t_count, void* v,
                                    long long t_tile, cudaStream_t s) {
  constexpr int m = 6;
  WinoInArgs a{};
  a.h = g.h; a.w = g.w; a.c = g.c; a.ph = g.ph; a.pw = g.pw;
  a.tiles_h = (g.oh + m - 1) / m;
  a.tiles_w = (g.ow + m - 1) / m;
  a.in_img_stride = g.in_img_stride;
  a.n0 = n0;
  a.t_base = 0;
  a.t_count = t_count;
  a.t_stride = t_tile;
  if (a.t_count == 0) return cudaSuccess;
  const int bx = g.c >= 64 ? 64 : 32;
  dim3 block(bx, 256 / bx);
  const long long blocks = ((a.t_count + block.y - 1) / block.y) * ((g.c + bx - 1) / bx);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  // int input offsets whenever one image (with a row of slack for the
  // padding) stays below 2^31 elements; the V offsets are 64-bit in this form
  const bool idx32 = g.in_img_stride + 4LL * g.w * g.c < (1LL << 31);
  if (idx32)
    wino_input_split_kernel<m, int><<<(unsigned)blocks, block, 0, s>>>(in, a, static_cast<__nv_bfloat16*>(v));
  else
    wino_input_split_kernel<m, long long><<<(unsigned)blocks, block, 0, s>>>(in, a, static_cast<__nv_bfloat16*>(v));
  return cudaGetLastError();
}

cudaError_t launch_wino_input(const void* in, const Geom& g, int n0, long long t_base, long long t_count, int m,
                              conv_dtype_t in_dt, conv_dtype_t store_dt, void* v, long long t_tile,
                              cudaStream_t s) {
  WinoInArgs a{};
  a.h = g.h; a.w = g.w; a.c = g.c; a.ph = g.ph; a.pw = g.pw;
  a.tiles_h = (g.oh + m - 1) / m;
  a.tiles_w = (g.ow + m - 1) / m;
  a.in_img_stride = g.in_img_stride;
  a.n0 = n0;
  a.t_base = t_base;
  a.t_count = t_count;
  a.t_stride = t_tile;
  if (a.t_count == 0) return cudaSuccess;
  int bx = g.c >= 64 ? 64 : 32;
  dim3 block(bx, 256 / bx);
  const long long blocks = ((a.t_count + block.y - 1) / block.y) * ((g.c + bx - 1) / bx);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  dim3 grid((unsigned)blocks);
  // 32-bit offsets when one image (with a row of slack for the padding) and the
  // whole V plane set stay below 2^31 elements
  const int a2 = (m + 2) * (m + 2);
  const bool idx32 = g.in_img_stride + 4LL * g.w * g.c < (1LL << 31) && (long long)a2 * t_tile * g.c < (1LL << 31);
  // 16-bit in and out, F(2,3): channel pairs
  if (m == 2 && in_dt != CONV_F32 && store_dt == in_dt && g.c % 2 == 0 && g.in_img_stride % 2 == 0 &&
      (reinterpret_cast<uintptr_t>(in) & 3) == 0 && (reinterpret_cast<uintptr_t>(v) & 3) == 0) {
    const int cp = g.c / 2;
    const int pbx = cp >= 64 ? 64 : 32;
    dim3 pblock(pbx, 256 / pbx);
    const long long pblocks = ((a.t_count + pblock.y - 1) / pblock.y) * ((cp + pbx - 1) / pbx);
    if (pblocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    auto go = [&](auto tv) {
      using T = decltype(tv);
      if (idx32)
        wino_input_pair_kernel<2, T, int><<<(unsigned)pblocks, pblock, 0, s>>>(static_cast<const T*>(in), a,
                                                                              static_cast<T*>(v));
      else
        wino_input_pair_kernel<2, T, long long><<<(unsigned)pblocks, pblock, 0, s>>>(static_cast<const T*>(in), a,
                                                                                    static_cast<T*>(v));
      return cudaGetLastError();
    };
    return in_dt == CONV_BF16 ? go(__nv_bfloat16{}) : go(__half{});
  }
  return wino_by_m(m, [&](auto mc) {
    constexpr int M = decltype(mc)::value;
    return wino_by_dt(in_dt, [&](auto ti) {
      using Tin = decltype(ti);
      return wino_by_dt(store_dt, [&](auto ts) {
        using Tst = decltype(ts);
        if (idx32)
          wino_input_kernel<M, Tin, Tst, int><<<grid, block, 0, s>>>(static_cast<const Tin*>(in), a,
                                                                     static_cast<Tst*>(v));
        else
          wino_input_kernel<M, Tin, Tst, long long><<<grid, block, 0, s>>>(static_cast<const Tin*>(in), a,
                                                                           static_cast<Tst*>(v));
        return cudaGetLastError();
      });
    });
  });
}

cudaError_t launch_wino_pass(const void* in, const Geom& g, int m, conv_dtype_t dt, int n0, long long in_t_base,
                             long long in_t_count, float* v, long long out_t_base, long long out_t_count,
                             const float* mb, void* out, bool accumulate, bool pdl, cudaStream_t s) {
  if (in_t_count == 0 && out_t_count == 0) return cudaSuccess;
  const int tiles_h = (g.oh + m - 1) / m, tiles_w = (g.ow + m - 1) / m;
  WinoInArgs ai{};
  ai.h = g.h; ai.w = g.w; ai.c = g.c; ai.ph = g.ph; ai.pw = g.pw;
  ai.tiles_h = tiles_h; ai.tiles_w = tiles_w;
  ai.in_img_stride = g.in_img_stride;
  ai.n0 = n0;
  ai.t_base = in_t_base;
  ai.t_count = in_t_count;
  ai.t_stride = in_t_count;
  WinoOutArgs ao{};
  ao.oh = g.oh; ao.ow = g.ow; ao.o = g.o;
  ao.tiles_h = tiles_h; ao.tiles_w = tiles_w;
  ao.out_img_stride = g.out_img_stride;
  ao.n0 = n0;
  ao.t_base = out_t_base;
  ao.t_count = out_t_count;
  ao.t_stride = out_t_count;
  ao.accumulate = accumulate ? 1 : 0;
  const int ibx = g.c >= 64 ? 64 : 32, iby = 256 / ibx;
  const int obx = g.o >= 64 ? 64 : 32, oby = 256 / obx;
  const long long in_blocks = ((in_t_count + iby - 1) / iby) * ((g.c + ibx - 1) / ibx);
  const long long ogx = (out_t_count + oby - 1) / oby, ogy = (g.o + obx - 1) / obx;
  const long long blocks = in_blocks + ogx * ogy;
  if (blocks > 0x7fffffffLL || ogx > 0xffffffffLL) return cudaErrorInvalidValue;
  const int a2 = (m + 2) * (m + 2);
  const bool idx32 = g.in_img_stride + 4LL * g.w * g.c < (1LL << 31) &&
                     (long long)a2 * in_t_count * g.c < (1LL << 31) && g.out_img_stride < (1LL << 31) &&
                     (long long)a2 * out_t_count * g.o < (1LL << 31);
  return wino_by_m(m, [&](auto mc) {
    constexpr int M = decltype(mc)::value;
    return wino_by_dt(dt, [&](auto ti) {
      using Tin = decltype(ti);
      auto run = [&](auto kernel) {
        const Tin* ip = static_cast<const Tin*>(in);
        Tin* op = static_cast<Tin*>(out);
        if (pdl)
          return launch_pdl(kernel, dim3((unsigned)blocks), dim3(256), 0, s, ip, ai, v, in_blocks, ibx, mb, ao, op,
                            (unsigned)ogx, obx);
        kernel<<<(unsigned)blocks, 256, 0, s>>>(ip, ai, v, in_blocks, ibx, mb, ao, op, (unsigned)ogx, obx);
        return cudaGetLastError();
      };
      return idx32 ? run(wino_pass_kernel<M, Tin, int>) : run(wino_pass_kernel<M, Tin, long long>);
    });
  });
}

cudaError_t launch_wino_filter_cmajor(const void* w, long long w_row_stride, int o, int c, int m,
                                      conv_dtype_t in_dt, long long o_pad, float* u, cudaStream_t s) {
  long long n = (long long)o * c;
  if (n == 0) return cudaSuccess;
  unsigned blocks = (unsigned)((n + 255) / 256);
  return wino_by_m(m, [&](auto mc) {
    constexpr int M = decltype(mc)::value;
    return wino_by_dt(in_dt, [&](auto ti) {
      using Tin = decltype(ti);
      wino_filter_cmajor_kernel<M, Tin><<<blocks, 256, 0, s>>>(static_cast<const Tin*>(w), w_row_stride, o, c,
                                                                o_pad, u);
      return cudaGetLastError();
    });
  });
}

cudaError_t launch_wino_input_cmajor(const void* in, const Geom& g, int n0, int nb, int m, conv_dtype_t in_dt,
                                     float* v, long long t_stride, cudaStream_t s) {
  WinoInCArgs a{};
  a.h = g.h; a.w = g.w; a.c = g.c; a.ph = g.ph; a.pw = g.pw;
  a.tiles_h = (g.oh + m - 1) / m;
  a.tiles_w = (g.ow + m - 1) / m;
  a.strips_w = (a.tiles_w + kStripTiles - 1) / kStripTiles;
  a.in_img_stride = g.in_img_stride;
  a.n0 = n0;
  a.t_stride = t_stride;
  const long long blocks = (long long)nb * a.tiles_h * a.strips_w * ((g.c + kStripChans - 1) / kStripChans);
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  dim3 grid((unsigned)blocks);
  return wino_by_m(m, [&](auto mc) {
    constexpr int M = decltype(mc)::value;
    return wino_by_dt(in_dt, [&](auto ti) {
      using Tin = decltype(ti);
      auto k = wino_input_cmajor_kernel<M, Tin>;
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Strip<M>::BYTES);
      if (e != cudaSuccess) return e;
      k<<<grid, 256, Strip<M>::BYTES, s>>>(static_cast<const Tin*>(in), a, v);
      return cudaGetLastError();
    });
  });
}

cudaError_t launch_wino_output(const void* mbuf, conv_dtype_t m_dt, const Geom& g, int n0, long long t_base,
                               long long t_count, int m, long long t_tile, conv_dtype_t out_dt, void* out,
                               bool accumulate, cudaStream_t s) {
  WinoOutArgs a{};
  a.oh = g.oh; a.ow = g.ow; a.o = g.o;
  a.tiles_h = (g.oh + m - 1) / m;
  a.tiles_w = (g.ow + m - 1) / m;
  a.out_img_stride = g.out_img_stride;
  a.n0 = n0;
  a.t_base = t_base;
  a.t_count = t_count;
  a.t_stride = t_tile;
  a.accumulate = accumulate ? 1 : 0;
  if (a.t_count == 0) return cudaSuccess;
  int bx = g.o >= 64 ? 64 : 32;
  dim3 block(bx, 256 / bx);
  dim3 grid((unsigned)((a.t_count + block.y - 1) / block.y), (g.o + bx - 1) / bx);
  if (grid.y > 65535) return cudaErrorInvalidValue;
  const int a2 = (m + 2) * (m + 2);
  const bool idx32 = g.out_img_stride < (1LL << 31) && (long long)a2 * t_tile * g.o < (1LL << 31);
  // 16-bit M and out, F(2,3): channel pairs
  if (m == 2 && out_dt != CONV_F32 && m_dt == out_dt && g.o % 2 == 0 && g.out_img_stride % 2 == 0 &&
      (reinterpret_cast<uintptr_t>(out) & 3) == 0 && (reinterpret_cast<uintptr_t>(mbuf) & 3) == 0) {
    const int op = g.o / 2;
    const int pbx = op >= 64 ? 64 : 32;
    dim3 pblock(pbx, 256 / pbx);
    dim3 pgrid((unsigned)((a.t_count + pblock.y - 1) / pblock.y), (op + pbx - 1) / pbx);
    if (pgrid.y > 65535) return cudaErrorInvalidValue;
    auto go = [&](auto tv) {
      using T = decltype(tv);
      if (idx32)
        wino_output_pair_kernel<2, T, int><<<pgrid, pblock, 0, s>>>(static_cast<const T*>(mbuf), a,
                                                                    static_cast<T*>(out));
      else
        wino_output_pair_kernel<2, T, long long><<<pgrid, pblock, 0, s>>>(static_cast<const T*>(mbuf), a,
                                                                          static_cast<T*>(out));
      return cudaGetLastError();
    };
    return out_dt == CONV_BF16 ? go(__nv_bfloat16{}) : go(__half{});
  }
  return wino_by_m(m, [&](auto mc) {
    constexpr int M = decltype(mc)::value;
    return wino_by_dt(out_dt, [&](auto to) {
      using Tout = decltype(to);
      auto go = [&](auto tm) {
        using TM = decltype(tm);
        const TM* mp = static_cast<const TM*>(mbuf);
        if (idx32)
          wino_output_kernel<M, TM, Tout, int><<<grid, block, 0, s>>>(mp, a, static_cast<Tout*>(out));
        else
          wino_output_kernel<M, TM, Tout, long long><<<grid, block, 0, s>>>(mp, a, static_cast<Tout*>(out));
        return cudaGetLastError();
      };
      // M is fp32, or the output's own 16-bit type
      if (m_dt == CONV_F32) return go(float{});
      if (m_dt != out_dt) return cudaErrorInvalidValue;
      return go(Tout{});
    });
  });
}

}  // namespace b200conv
