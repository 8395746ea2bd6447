// simt_conv.cu -- implicit-GEMM convolution on the CUDA cores (FFMA, fp32).
//
// GEMM view (the implicit GEMM of "Use the explicit gemm for wide convs on
// neural accelerators", description): rows m = (n, oh, ow) of the output,
// columns o, reduction k = (kh, kw, c) in the OHWI weight order.  A[m][k] is
// gathered from the NHWC input on the fly (zero outside the image), never
// materialised; B[o][k] is the weight row.  Every product and sum is an fp32
// FFMA (true fp32: no TF32 anywhere), and each output's reduction runs over k
// in ascending order inside one thread, so its result does not depend on how
// many rows the problem has (the Winograd batch-tiling bit-identity relies on
// this).
//
// Tiling: 128 x BN output tile per 256-thread block, 16-wide k chunks staged
// through double-buffered shared memory (transposed, k-major), 8 x BN/16
// outputs per thread, multiplied as packed fp32 FMAs on column pairs (two
// lanes per instruction, each exactly fmaf).  k chunks never straddle a
// filter tap, so each A row resolves its input pixel once per tap.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace b200conv {
namespace {

constexpr int BM = 128;
constexpr int BK = 16;
constexpr int THREADS = 256;
constexpr int LDA = BM + 2;   // conflict-free transposed stores, 8-byte aligned pairs

struct SimtArgs {
  const void* in;
  const void* w;
  void* out;
  int h, w_, c, o, kh, kw, sh, sw, ph, pw, dh, dw, oh, ow;
  long long m;               // rows per batch: n * oh * ow
  long long in_img_stride;   // elements between images
  long long w_row_stride;    // elements between weight rows
  long long a_batch, b_batch, d_batch;   // batch strides (grid.z), elements
  int accumulate;
  int ksplit;                // > 1: blockIdx.z splits the K range; fp32 partials go to `partial`
  float* partial;            // [ksplit][m][o] when ksplit > 1
};

// Loads 4 consecutive channels starting at p (all < C when full) as fp32.
template <typename T, bool VEC>
__device__ __forceinline__ void load4(const T* p, int valid, float* v) {
  if (VEC && valid == 4) {
    if constexpr (sizeof(T) == 4) {
      float4 q = __ldg(reinterpret_cast<const float4*>(p));
      v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
      uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
      const T* e = reinterpret_cast<const T*>(&q);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = Store<T>::to_f32(e[i]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = (i < valid) ? Store<T>::to_f32(p[i]) : 0.0f;
  }
}

template <typename T, int BN, bool VEC>
__global__ void __launch_bounds__(THREADS)
simt_conv_kernel(const SimtArgs a) {
  constexpr int TN = BN / 16;        // columns per thread
  constexpr int LDB = BN + 2;
  constexpr int B_CHUNKS = BN * 4;   // 4-channel chunks in a BN x 16 tile
  constexpr int B_PER_T = (B_CHUNKS + THREADS - 1) / THREADS;

  __shared__ __align__(16) float As[2][BK][LDA];
  __shared__ __align__(16) float Bs[2][BK][LDB];

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const long long m0 = (long long)blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const int bz = a.ksplit > 1 ? 0 : blockIdx.z;
  const int split = a.ksplit > 1 ? blockIdx.z : 0;

  const T* __restrict__ in = static_cast<const T*>(a.in) + (long long)bz * a.a_batch;
  const T* __restrict__ wt = static_cast<const T*>(a.w) + (long long)bz * a.b_batch;
  T* __restrict__ out = static_cast<T*>(a.out) + (long long)bz * a.d_batch;

  // The two A rows this thread loads: resolve (n, oh, ow) once.
  const int kq = (tid & 3) * 4;
  int a_ih0[2], a_iw0[2];
  long long a_base[2];
  bool a_row_ok[2];
  const long long ohw = (long long)a.oh * a.ow;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    long long m = m0 + (tid >> 2) + 64 * r;
    a_row_ok[r] = m < a.m;
    long long mm = a_row_ok[r] ? m : 0;
    long long n = mm / ohw;
    int rem = (int)(mm - n * ohw);
    int oy = rem / a.ow, ox = rem - (rem / a.ow) * a.ow;
    a_ih0[r] = oy * a.sh - a.ph;
    a_iw0[r] = ox * a.sw - a.pw;
    a_base[r] = n * a.in_img_stride;
  }

  const int cchunks = (a.c + BK - 1) / BK;
  const int steps_all = a.kh * a.kw * cchunks;
  // K range of this block: all of it, or split `split` of ksplit
  const int step_lo = (int)((long long)steps_all * split / a.ksplit);
  const int step_hi = (int)((long long)steps_all * (split + 1) / a.ksplit);
  const int steps = step_hi - step_lo;

  float ra[2][4];
  float rb[B_PER_T][4];

  auto load_tiles = [&](int step_rel) {
    const int step = step_lo + step_rel;
    const int tap = step / cchunks;
    const int c0 = (step - tap * cchunks) * BK;
    const int ky = tap / a.kw, kx = tap - (tap / a.kw) * a.kw;
    const int cc = c0 + kq;
    const int valid = max(0, min(4, a.c - cc));
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      int ih = a_ih0[r] + ky * a.dh, iw = a_iw0[r] + kx * a.dw;
      bool ok = a_row_ok[r] && ih >= 0 && ih < a.h && iw >= 0 && iw < a.w_ && valid > 0;
      if (ok) {
        const T* p = in + a_base[r] + ((long long)ih * a.w_ + iw) * a.c + cc;
        load4<T, VEC>(p, valid, ra[r]);
      } else {
        ra[r][0] = ra[r][1] = ra[r][2] = ra[r][3] = 0.0f;
      }
    }
#pragma unroll
    for (int r = 0; r < B_PER_T; ++r) {
      int q = tid + r * THREADS;
      int row = q >> 2, kk = (q & 3) * 4;
      int o = n0 + row;
      int ccb = c0 + kk;
      int vb = max(0, min(4, a.c - ccb));
      if (q < B_CHUNKS && o < a.o && vb > 0) {
        const T* p = wt + (long long)o * a.w_row_stride + (long long)tap * a.c + ccb;
        load4<T, VEC>(p, vb, rb[r]);
      } else {
        rb[r][0] = rb[r][1] = rb[r][2] = rb[r][3] = 0.0f;
      }
    }
  };

  auto store_tiles = [&](int buf) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      int row = (tid >> 2) + 64 * r;
#pragma unroll
      for (int e = 0; e < 4; ++e) As[buf][kq + e][row] = ra[r][e];
    }
#pragma unroll
    for (int r = 0; r < B_PER_T; ++r) {
      int q = tid + r * THREADS;
      if (q < B_CHUNKS) {
        int row = q >> 2, kk = (q & 3) * 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) Bs[buf][kk + e][row] = rb[r][e];
      }
    }
  };

  // column pairs for the packed fp32 FMA (each lane exactly fmaf)
  float2 acc[8][TN / 2];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < TN / 2; ++j) acc[i][j] = make_float2(0.0f, 0.0f);

  if (steps > 0) load_tiles(0);
  else ra[0][0] = ra[0][1] = ra[0][2] = ra[0][3] = ra[1][0] = ra[1][1] = ra[1][2] = ra[1][3] = 0.0f;
  if (steps <= 0) {
#pragma unroll
    for (int r = 0; r < B_PER_T; ++r) rb[r][0] = rb[r][1] = rb[r][2] = rb[r][3] = 0.0f;
  }
  store_tiles(0);
  __syncthreads();

  for (int step = 0; step < steps; ++step) {
    const int buf = step & 1;
    if (step + 1 < steps) load_tiles(step + 1);
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float av[8];
      float2 bv[TN / 2];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 t = *reinterpret_cast<const float2*>(&As[buf][k][32 * i + ty * 2]);
        av[2 * i] = t.x; av[2 * i + 1] = t.y;
      }
#pragma unroll
      for (int j = 0; j < TN / 2; ++j) bv[j] = *reinterpret_cast<const float2*>(&Bs[buf][k][32 * j + tx * 2]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 a2 = make_float2(av[i], av[i]);
#pragma unroll
        for (int j = 0; j < TN / 2; ++j) acc[i][j] = __ffma2_rn(a2, bv[j], acc[i][j]);
      }
    }
    if (step + 1 < steps) store_tiles(buf ^ 1);
    __syncthreads();
  }

  // Epilogue: rows m0 + 32i + 2ty + e, columns n0 + 32j + 2tx + f.
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    long long m = m0 + 32 * (i >> 1) + ty * 2 + (i & 1);
    if (m >= a.m) continue;
    if (a.ksplit > 1) {
      float* prow = a.partial + (long long)split * a.m * a.o + m * a.o;
#pragma unroll
      for (int j = 0; j < TN; ++j) {
        int o = n0 + 32 * (j >> 1) + tx * 2 + (j & 1);
        if (o < a.o) prow[o] = (j & 1) ? acc[i][j >> 1].y : acc[i][j >> 1].x;
      }
      continue;
    }
    T* orow = out + m * a.o;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      int o = n0 + 32 * (j >> 1) + tx * 2 + (j & 1);
      if (o < a.o) {
        float v = (j & 1) ? acc[i][j >> 1].y : acc[i][j >> 1].x;
        if (a.accumulate) v = Store<T>::to_f32(orow[o]) + Store<T>::to_f32(Store<T>::from_f32(v));
        orow[o] = Store<T>::from_f32(v);
      }
    }
  }
}

template <typename T, bool VEC>
cudaError_t launch_typed(const SimtArgs& a, int batches, cudaStream_t s) {
  const long long mblocks = (a.m + BM - 1) / BM;
  if (mblocks > 0x7fffffffLL || batches > 65535) return cudaErrorInvalidValue;
  int bn = a.o <= 64 ? 64 : (a.o <= 96 ? 96 : 128);
  dim3 grid((unsigned)mblocks, (a.o + bn - 1) / bn, batches);
  if (grid.y > 65535) return cudaErrorInvalidValue;
  if (bn == 64)
    simt_conv_kernel<T, 64, VEC><<<grid, THREADS, 0, s>>>(a);
  else if (bn == 96)
    simt_conv_kernel<T, 96, VEC><<<grid, THREADS, 0, s>>>(a);
  else
    simt_conv_kernel<T, 128, VEC><<<grid, THREADS, 0, s>>>(a);
  return cudaGetLastError();
}

template <bool VEC>
cudaError_t launch_dt(const SimtArgs& a, conv_dtype_t dt, int batches, cudaStream_t s) {
  switch (dt) {
    case CONV_F32: return launch_typed<float, VEC>(a, batches, s);
    case CONV_F16: return launch_typed<__half, VEC>(a, batches, s);
    case CONV_BF16: return launch_typed<__nv_bfloat16, VEC>(a, batches, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_simt_conv(const void* in, const void* w, void* out, const Geom& g,
                             conv_dtype_t dt, bool vec, bool accumulate, cudaStream_t s, int ksplit,
                             float* partial) {
  if (g.out_img_stride != (long long)g.oh * g.ow * g.o) return cudaErrorInvalidValue;
  SimtArgs a{};
  a.in = in; a.w = w; a.out = out;
  a.h = g.h; a.w_ = g.w; a.c = g.c; a.o = g.o; a.kh = g.kh; a.kw = g.kw;
  a.sh = g.sh; a.sw = g.sw; a.ph = g.ph; a.pw = g.pw; a.dh = g.dh; a.dw = g.dw;
  a.oh = g.oh; a.ow = g.ow;
  a.m = (long long)g.n * g.oh * g.ow;
  a.in_img_stride = g.in_img_stride;
  a.w_row_stride = g.w_row_stride;
  a.a_batch = a.b_batch = a.d_batch = 0;
  a.accumulate = accumulate ? 1 : 0;
  a.ksplit = ksplit > 1 ? ksplit : 1;
  a.partial = partial;
  if (a.m == 0) return cudaSuccess;
  if (a.ksplit > 1 && !partial) return cudaErrorInvalidValue;
  return vec ? launch_dt<true>(a, dt, a.ksplit, s) : launch_dt<false>(a, dt, a.ksplit, s);
}


}  // namespace b200conv
