// wino_gemm_f32.cu -- the Winograd batched GEMM in true fp32 (FFMA).
//
// The batched GEMM step of the Winograd path ("Bound winograd conv2d working
// set by tiling the batch", Problem: input transform, GEMMs, output
// transform):
//
//   D[xi][t][o] = sum_c A[xi][c][t] * B[xi][c][o]      xi < alpha^2
//
// with A = V stored channel-major ([xi][C][T_pad], T_pad = T rounded up to 4)
// and B = U stored [xi][C][O_pad] by the transforms, so that every k-slice of
// both operands is a contiguous row: tiles move global -> shared memory with
// 16-byte cp.async (zero-filled past T, C and O) in a 3-stage ring, with no
// register staging and no transposes.  Each of the 128 threads owns an
// 8 x BN/8 block of D and reads its operand fragments with 128-bit shared
// loads.  The products run as packed fp32 FMAs on column pairs (sm_100's
// two-lane FMA; each lane is exactly fmaf), which halves the FMA issue slots
// of a kernel that is otherwise issue-bound.  Every output's reduction runs
// over c in ascending order inside one thread, so the result does not depend
// on T (batch-tiled Winograd stays bit-identical to untiled).
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace b200conv {
namespace {

constexpr int BM = 128;
constexpr int BK = 16;
constexpr int STAGES = 3;
constexpr int THREADS = 128;

struct WgArgs {
  const float* a;
  const float* b;
  float* d;
  int t, c, o;
  long long lda, ldb;              // row strides of A ([C][T_pad]) and B ([C][O_pad])
  long long a_batch, b_batch, d_batch;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// A_TMAJOR = false: A is [C][T_pad] (row = one channel, contiguous in t);
// A_TMAJOR = true:  A is [T][C]     (row = one tile, contiguous in c), staged
// into shared memory as [t][BK c] rows whose 16-byte chunks are XOR-swizzled
// by (t / 4) % 4, so the per-k column reads of four rows 4 apart hit four
// different banks.
template <int BN, bool A_TMAJOR>
__global__ void __launch_bounds__(THREADS, 2)
wino_gemm_f32_kernel(const WgArgs p) {
  constexpr int TN = BN / 8;                 // columns per thread (8, 12 or 16)
  constexpr int A_CHUNKS = BK * BM / 4;      // 16-byte chunks per stage
  constexpr int B_CHUNKS = BK * BN / 4;
  extern __shared__ __align__(16) float smem[];
  float* As = smem;                          // [STAGES][BK][BM]
  float* Bs = smem + STAGES * BK * BM;       // [STAGES][BK][BN]

  const int tid = threadIdx.x;
  const int tc = tid & 7, tr = tid >> 3;     // 8 thread-columns x 16 thread-rows
  const long long t0 = (long long)blockIdx.x * BM;
  const int o0 = blockIdx.y * BN;
  const int bz = blockIdx.z;
  const float* __restrict__ A = p.a + bz * p.a_batch;
  const float* __restrict__ B = p.b + bz * p.b_batch;
  float* __restrict__ D = p.d + bz * p.d_batch;
  const int ktiles = (p.c + BK - 1) / BK;

  // Launched with programmatic stream serialization: everything above is
  // address arithmetic; wait here for the kernel that wrote A (and for the one
  // that last read D) before the first global access.
  pdl_wait_then_release();

  // Per-thread copy descriptors, fixed across k-tiles (only the k offset moves).
  constexpr int A_PER = (A_CHUNKS + THREADS - 1) / THREADS;
  constexpr int B_PER = (B_CHUNKS + THREADS - 1) / THREADS;
  static_assert(!A_TMAJOR || A_CHUNKS % THREADS == 0, "A copies");
  // A tile-major: copy i moves row (tid >> 2) + 32 i, chunk tid & 3.
  const int a_chunk = tid & 3;
  const int a_row0 = tid >> 2;
  const float* a_src0 = A + (t0 + a_row0) * p.lda + a_chunk * 4;
  const long long a_step = 32 * p.lda;
  const uint32_t a_dst0 = (uint32_t)__cvta_generic_to_shared(As) +
                          (uint32_t)(a_row0 * BK + ((a_chunk ^ ((a_row0 >> 2) & 3)) * 4)) * 4u;
  unsigned a_valid = 0;
#pragma unroll
  for (int i = 0; i < A_PER; ++i)
    if (t0 + a_row0 + 32 * i < p.t) a_valid |= 1u << i;
  int b_off[B_PER], b_k[B_PER], b_bytes[B_PER];
  uint32_t b_dst[B_PER];
#pragma unroll
  for (int i = 0; i < B_PER; ++i) {
    const int q = tid + i * THREADS;
    const int k = q / (BN / 4), col = (q % (BN / 4)) * 4;
    const int oo = o0 + col;
    b_k[i] = q < B_CHUNKS ? k : BK;          // BK: never copies
    b_off[i] = (int)(k * p.ldb) + oo;
    b_bytes[i] = oo < p.o ? min(16, (p.o - oo) * 4) : 0;
    b_dst[i] = (uint32_t)__cvta_generic_to_shared(Bs) + (uint32_t)(k * BN + col) * 4u;
  }

  auto load_stage = [&](int stage, int kt) {
    const int c0 = kt * BK;
    if (A_TMAJOR) {
      const int cc = c0 + a_chunk * 4;
      const int cbytes = cc < p.c ? min(16, (p.c - cc) * 4) : 0;
      const uint32_t dst = a_dst0 + (uint32_t)(stage * BK * BM) * 4u;
#pragma unroll
      for (int i = 0; i < A_PER; ++i) {
        const int bytes = (a_valid >> i) & 1 ? cbytes : 0;
        const float* src = bytes ? a_src0 + c0 + i * a_step : A;
        cp_async16(dst + (uint32_t)(i * 32 * BK) * 4u, src, bytes);
      }
    } else {
      float* as = As + stage * BK * BM;
#pragma unroll
      for (int i = 0; i < (A_CHUNKS + THREADS - 1) / THREADS; ++i) {
        const int q = tid + i * THREADS;
        if (q < A_CHUNKS) {
          const int k = q / (BM / 4), col = (q % (BM / 4)) * 4;
          const long long tt = t0 + col;
          int bytes = 0;
          const float* src = A;
          if (c0 + k < p.c && tt < p.t) {
            bytes = (int)min(16LL, (p.t - tt) * 4);
            src = A + (long long)(c0 + k) * p.lda + tt;
          }
          cp_async16((uint32_t)__cvta_generic_to_shared(as + k * BM + col), src, bytes);
        }
      }
    }
    const float* bbase = B + (long long)c0 * p.ldb;
    const uint32_t bstage = (uint32_t)(stage * BK * BN) * 4u;
#pragma unroll
    for (int i = 0; i < B_PER; ++i) {
      if (b_k[i] < BK) {
        const int bytes = c0 + b_k[i] < p.c ? b_bytes[i] : 0;
        cp_async16(b_dst[i] + bstage, bytes ? bbase + b_off[i] : B, bytes);
      }
    }
  };

  // accumulators in column pairs: the packed fp32 FMA (two lanes per
  // instruction, each lane exactly fmaf) halves the FMA issue slots
  float2 acc[8][TN / 2];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < TN / 2; ++j) acc[i][j] = make_float2(0.0f, 0.0f);

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < ktiles) load_stage(s, s);
    cp_commit();
  }

  for (int kt = 0; kt < ktiles; ++kt) {
    cp_wait<STAGES - 2>();
    __syncthreads();
    const int pre = kt + STAGES - 1;
    if (pre < ktiles) load_stage(pre % STAGES, pre);
    cp_commit();
    const float* as = As + (kt % STAGES) * BK * BM;
    const float* bs = Bs + (kt % STAGES) * BK * BN;
    if constexpr (A_TMAJOR) {
      // one 128-bit load per A row covers 4 k-steps (rows are contiguous in k)
#pragma unroll
      for (int k4 = 0; k4 < BK / 4; ++k4) {
        float4 a4[8];
        const int off = (k4 ^ (tr & 3)) << 2;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a4[i] = *reinterpret_cast<const float4*>(as + (tr * 4 + i) * BK + off);
          a4[4 + i] = *reinterpret_cast<const float4*>(as + (64 + tr * 4 + i) * BK + off);
        }
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const int k = 4 * k4 + kq;
          float2 bv[TN / 2];
#pragma unroll
          for (int j = 0; j < TN / 4; ++j) {
            const float4 b = *reinterpret_cast<const float4*>(bs + k * BN + 32 * j + tc * 4);
            bv[2 * j] = make_float2(b.x, b.y);
            bv[2 * j + 1] = make_float2(b.z, b.w);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float av = kq == 0 ? a4[i].x : kq == 1 ? a4[i].y : kq == 2 ? a4[i].z : a4[i].w;
            const float2 a2 = make_float2(av, av);
#pragma unroll
            for (int j = 0; j < TN / 2; ++j) acc[i][j] = __ffma2_rn(a2, bv[j], acc[i][j]);
          }
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < BK; ++k) {
        float av[8];
        float2 bv[TN / 2];
        const float4 a0 = *reinterpret_cast<const float4*>(as + k * BM + tr * 4);
        const float4 a1 = *reinterpret_cast<const float4*>(as + k * BM + 64 + tr * 4);
        av[0] = a0.x; av[1] = a0.y; av[2] = a0.z; av[3] = a0.w;
        av[4] = a1.x; av[5] = a1.y; av[6] = a1.z; av[7] = a1.w;
#pragma unroll
        for (int j = 0; j < TN / 4; ++j) {
          const float4 b = *reinterpret_cast<const float4*>(bs + k * BN + 32 * j + tc * 4);
          bv[2 * j] = make_float2(b.x, b.y);
          bv[2 * j + 1] = make_float2(b.z, b.w);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 a2 = make_float2(av[i], av[i]);
#pragma unroll
          for (int j = 0; j < TN / 2; ++j) acc[i][j] = __ffma2_rn(a2, bv[j], acc[i][j]);
        }
      }
    }
  }
  cp_wait<0>();

  // rows t0 + tr*4 + i (i < 4) and t0 + 64 + tr*4 + (i - 4); columns o0 + 32j + 4tc + e
  const bool vec = (p.o & 3) == 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long long t = t0 + (i < 4 ? tr * 4 + i : 64 + tr * 4 + i - 4);
    if (t >= p.t) continue;
    float* drow = D + t * p.o;
#pragma unroll
    for (int j = 0; j < TN / 4; ++j) {
      const int o = o0 + 32 * j + tc * 4;
      const float4 v4 = make_float4(acc[i][2 * j].x, acc[i][2 * j].y, acc[i][2 * j + 1].x, acc[i][2 * j + 1].y);
      if (vec && o + 3 < p.o) {
        *reinterpret_cast<float4*>(drow + o) = v4;
      } else {
        const float ve[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (o + e < p.o) drow[o + e] = ve[e];
      }
    }
  }
}

template <int BN, bool A_TMAJOR>
cudaError_t launch_bn(const WgArgs& p, int batches, cudaStream_t s) {
  const int smem = STAGES * BK * (BM + BN) * (int)sizeof(float);
  static int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(wino_gemm_f32_kernel<BN, A_TMAJOR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured_dev = dev;
  }
  const long long mblocks = (p.t + BM - 1) / BM;
  dim3 grid((unsigned)mblocks, (p.o + BN - 1) / BN, batches);
  return launch_pdl(wino_gemm_f32_kernel<BN, A_TMAJOR>, grid, dim3(THREADS), smem, s, p);
}

}  // namespace

int wino_gemm_f32_tile_n(int o) { return o <= 64 ? 64 : (o <= 96 ? 96 : 128); }

cudaError_t launch_wino_gemm_f32(const float* a, const float* b, float* d, int batches, int t, int c, int o,
                                 long long lda, long long ldb, bool a_tmajor, cudaStream_t s) {
  if (t == 0 || batches == 0) return cudaSuccess;
  if ((lda & 3) || (ldb & 3) || (reinterpret_cast<uintptr_t>(a) & 15) || (reinterpret_cast<uintptr_t>(b) & 15))
    return cudaErrorInvalidValue;
  if (batches > 65535 || (t + BM - 1) / BM > 0x7fffffffLL) return cudaErrorInvalidValue;
  const long long a_batch = a_tmajor ? (long long)t * lda : (long long)c * lda;
  WgArgs p{a, b, d, t, c, o, lda, ldb, a_batch, (long long)c * ldb, (long long)t * o};
  const int bn = wino_gemm_f32_tile_n(o);
  if (a_tmajor)
    return bn == 64 ? launch_bn<64, true>(p, batches, s)
                    : bn == 96 ? launch_bn<96, true>(p, batches, s) : launch_bn<128, true>(p, batches, s);
  return bn == 64 ? launch_bn<64, false>(p, batches, s)
                  : bn == 96 ? launch_bn<96, false>(p, batches, s) : launch_bn<128, false>(p, batches, s);
}

}  // namespace b200conv
