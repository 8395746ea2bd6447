// tc_conv.cu -- implicit-GEMM convolution on the sm_100a tensor cores.
//
// The implicit GEMM of "Use the explicit gemm for wide convs on neural
// accelerators" (description: im2col is never materialised), B200-first:
//
//   rows m = (n, oh, ow), columns o, reduction k = (kh, kw, c);
//   A tile (128 pixels x 64 channels) of tap (kh, kw) is fetched by one TMA
//   load in im2col mode: the tensor map walks 128 consecutive output pixels
//   (stride sh/sw, wrapping rows and images inside the padded bounding box)
//   and the per-tap offset (kw*dw, kh*dh) selects the filter tap; out-of-image
//   pixels read as zero, so padding costs nothing.  The gather happens on the
//   way into shared memory, in the 128-byte-swizzled K-major layout the MMA
//   reads directly.
//   B tile (BN weight rows x 64 channels) is a tiled TMA load of the OHWI
//   weights viewed as [O][taps][C] (row stride = a conv3d slice's stride).
//   tcgen05.mma (kind::f16, M = 128, N = BN, K = 16) accumulates in fp32 in
//   tensor memory, double-buffered so the epilogue of one tile overlaps the
//   main loop of the next.
//
// Warp roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0     TMA producer (one thread), multi-stage mbarrier ring
//   warp 1     TMEM allocator + MMA issuer (one thread)
//   warps 2-5  epilogue: tcgen05.ld -> round to the out dtype -> global
//
// Every mbarrier wait is bounded (about 2 s of %globaltimer); a wait that runs
// out records a code in the device error word, raises a CTA-wide abort flag,
// drains its own in-flight copies / MMAs (again bounded), frees TMEM and
// returns, so a fault in the pipeline can never hang the GPU.
//
// The same kernel runs the Winograd batched GEMM (tiled TMA for A, fp32 D).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace b200conv {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 x 16-bit = one 128-byte swizzle row
constexpr int THREADS = 192;
#ifndef TC_EPI_COLS
#define TC_EPI_COLS 128        // accumulator columns an epilogue thread reads per TMEM wait
#endif

template <int BN> struct Cfg {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;           // two fp32 accumulators
  static constexpr int BAR_BYTES = 256;
  // The epilogue stages each warp's output chunk for a TMA store: 32 rows of
  // 128 bytes (32 fp32 or 64 16-bit columns), 4 warps x 2 buffers, 128-byte swizzled
  static constexpr int STORE_BYTES = 4 * 2 * 32 * 128;
  template <typename TOut>
  static constexpr int smem() {
    return 1024 + STAGES * STAGE_BYTES + STORE_BYTES + BAR_BYTES;
  }
};

struct TcArgs {
  int m_tiles, n_tiles, batches;
  int kb_per_tap, taps;
  int kw, dh, dw;
  int oh, ow, sh, sw, ph, pw;
  int kh, od, sd, pd, dd;      // depth axis of the native 3D mode (kh splits a tap into kd, kh, kw)
  long long m_rows;            // rows per batch
  int ocols;                   // output columns (O)
  void* out;
  long long ldo;               // elements between output rows
  long long out_batch;         // elements between batches
  int accumulate;              // out = round(out + round(acc)) instead of out = round(acc)
  int ksplit;                  // conv modes: > 1 splits the K range, the split index in the batch slot
  int tma_store;               // write 32-row x 128-byte chunks with TMA stores through tmD
  int* err;
};

// --------------------------------- kernel -----------------------------------

// MODE 0: batched GEMM (tiled A); 1: conv2d (4D im2col A); 2: conv3d (5D im2col A).
template <int BN, int MODE, typename TIn, typename TOut>
__global__ void __launch_bounds__(THREADS, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmD, const TcArgs a) {
  using C = Cfg<BN>;
  constexpr int STORE_BYTES = C::STORE_BYTES;
  constexpr uint32_t IDESC = make_idesc<BN>(std::is_same<TIn, __nv_bfloat16>::value ? 1u : 0u);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint8_t* sStore = sB + C::STAGES * C::B_BYTES;        // fp32 output staging (1024-aligned)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStore + STORE_BYTES);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto tfull_bar = [&](int i) { return bar0 + 8u * (2 * C::STAGES + i); };
  auto tempty_bar = [&](int i) { return bar0 + 8u * (2 * C::STAGES + 2 + i); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::STAGES + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 128);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (a.tma_store) prefetch_tensormap(&tmD);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_then_release();

  const long long total_tiles = (long long)a.batches * a.m_tiles * a.n_tiles;
  const int ksteps = a.taps * a.kb_per_tap;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const int nt = (int)(tile % a.n_tiles);
        const long long rest = tile / a.n_tiles;
        const int mt = (int)(rest % a.m_tiles);
        const int b = (int)(rest / a.m_tiles);
        int img = 0, wx = 0, hy = 0, dz = 0;
        if (MODE != 0) {
          // first output pixel of the tile -> its window's corner in the input
          const long long m0 = (long long)mt * BM;
          const long long ohw = (long long)a.oh * a.ow;
          long long fr = m0 / ohw;                   // image (2D) or image*OD + od (3D)
          const int rem = (int)(m0 - fr * ohw);
          const int oy = rem / a.ow, ox = rem - (rem / a.ow) * a.ow;
          wx = ox * a.sw - a.pw;
          hy = oy * a.sh - a.ph;
          if (MODE == 2) {
            const int odz = (int)(fr % a.od);
            fr /= a.od;
            dz = odz * a.sd - a.pd;
          }
          img = (int)fr;
        }
        int ks_lo = 0, ks_hi = ksteps;
        if (MODE != 0 && a.ksplit > 1) {
          ks_lo = (int)((long long)ksteps * b / a.ksplit);
          ks_hi = (int)((long long)ksteps * (b + 1) / a.ksplit);
        }
        for (int ks = ks_lo; ks < ks_hi; ++ks) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.err, DEVERR_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          const int tap = ks / a.kb_per_tap;
          const int kb = ks - tap * a.kb_per_tap;
          const uint32_t fb = full_bar(stage);
          mbar_expect_tx(fb, C::STAGE_BYTES);
          const uint32_t dA = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t dB = smem_u32(sB + stage * C::B_BYTES);
          if (MODE == 1) {
            const int ky = tap / a.kw, kx = tap - (tap / a.kw) * a.kw;
            tma_load_im2col_4d(dA, &tmA, fb, kb * BK, wx, hy, img, (uint16_t)(kx * a.dw),
                               (uint16_t)(ky * a.dh));
            tma_load_3d(dB, &tmB, fb, kb * BK, tap, nt * BN);
          } else if (MODE == 2) {
            const int khw = a.kh * a.kw;
            const int kz = tap / khw, r2 = tap - kz * khw;
            const int ky = r2 / a.kw, kx = r2 - (r2 / a.kw) * a.kw;
            tma_load_im2col_5d(dA, &tmA, fb, kb * BK, wx, hy, dz, img, (uint16_t)(kx * a.dw),
                               (uint16_t)(ky * a.dh), (uint16_t)(kz * a.dd));
            tma_load_3d(dB, &tmB, fb, kb * BK, tap, nt * BN);
          } else {
            tma_load_3d(dA, &tmA, fb, kb * BK, mt * BM, b);
            tma_load_3d(dB, &tmB, fb, kb * BK, nt * BN, b);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: wait (bounded) until the last loads in flight have landed.
      const int pending = issued < C::STAGES ? (int)issued : C::STAGES;
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < pending; ++i) {
        if (--s < 0) {
          s = C::STAGES - 1;
          ph ^= 1u;
        }
        volatile int never = 0;
        mbar_wait(full_bar(s), ph, &never, a.err, 0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------- MMA issuer -------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, a.err, DEVERR_TIMEOUT_MMA_TMEM)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        int nks = ksteps;
        if (MODE != 0 && a.ksplit > 1) {
          const int b = (int)(tile / a.n_tiles / a.m_tiles);
          nks = (int)((long long)ksteps * (b + 1) / a.ksplit) - (int)((long long)ksteps * b / a.ksplit);
        }
        for (int ks = 0; ks < nks; ++ks) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, a.err, DEVERR_TIMEOUT_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t aa = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t bb = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            tc_mma(d_tmem, sdesc(aa + 32u * k), sdesc(bb + 32u * k), IDESC, (ks | k) != 0 ? 1u : 0u);
          tc_commit(empty_bar(stage));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit(tfull_bar(acc));
      }
      // Drain: all MMAs this thread issued have completed once this arrives.
      tc_commit(drain_bar);
      volatile int never = 0;
      mbar_wait(drain_bar, 0, &never, a.err, 0);
    }
    __syncwarp();
  } else {
    // -------------------------------- epilogue --------------------------------
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    int it = 0;
    int store_count = 0;                    // TMA-stored chunks of this warp (staging double buffer)
    for (long long tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag, a.err, DEVERR_TIMEOUT_EPILOGUE)) break;
      tc_fence_after();
      const int nt = (int)(tile % a.n_tiles);
      const long long rest = tile / a.n_tiles;
      const int mt = (int)(rest % a.m_tiles);
      const int b = (int)(rest / a.m_tiles);
      const long long m = (long long)mt * BM + row;
      const bool row_ok = m < a.m_rows;
      TOut* orow = static_cast<TOut*>(a.out) + (long long)b * a.out_batch + (row_ok ? m : 0) * a.ldo;
      const int n0 = nt * BN;
      // EPI columns per round: EPI/32 TMEM loads in flight behind one wait
      constexpr int EPI = BN < TC_EPI_COLS ? BN : TC_EPI_COLS;
#pragma unroll 1
      for (int cg = 0; cg < BN; cg += EPI) {
        uint32_t rr[EPI / 32][32];
#pragma unroll
        for (int h = 0; h < EPI / 32; ++h) {
          const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + cg + 32 * h);
          TMEM_LD32(taddr, rr[h]);
        }
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if constexpr (sizeof(TOut) == 4) {
          if (a.tma_store) {
            // stage row `lane` of this warp's 32 x 32 chunk (16-byte chunks XOR-swizzled by
            // lane % 8, the TMA 128-byte swizzle), then one lane stores it; rows past the
            // batch's last row and columns past O are clipped by the tensor map
#pragma unroll
            for (int h = 0; h < EPI / 32; ++h) {
              const int c0 = n0 + cg + 32 * h;
              if (c0 >= a.ocols) continue;
              float* sb = reinterpret_cast<float*>(sStore + (q * 2 + (store_count & 1)) * 4096);
              if (store_count >= 2) {
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
              }
              float4* rowp = reinterpret_cast<float4*>(sb + lane * 32);
#pragma unroll
              for (int k = 0; k < 8; ++k)
                rowp[k ^ (lane & 7)] = make_float4(__uint_as_float(rr[h][4 * k]), __uint_as_float(rr[h][4 * k + 1]),
                                                   __uint_as_float(rr[h][4 * k + 2]), __uint_as_float(rr[h][4 * k + 3]));
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              __syncwarp();
              if (lane == 0) {
                tma_store_3d(&tmD, smem_u32(sb), c0, mt * BM + q * 32, b);
                bulk_commit();
              }
              ++store_count;
            }
            continue;
          }
        } else {
          if (a.tma_store) {
            // 16-bit: stage row `lane` of a 32 x 64 chunk (two 32-column groups, 128 bytes
            // per row, 16-byte chunks XOR-swizzled by lane % 8), then one lane stores it
#pragma unroll
            for (int h = 0; h < EPI / 32; h += 2) {
              const int c0 = n0 + cg + 32 * h;
              if (c0 >= a.ocols) continue;
              uint4* sb = reinterpret_cast<uint4*>(sStore + (q * 2 + (store_count & 1)) * 4096);
              if (store_count >= 2) {
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
              }
              uint4* rowp = sb + lane * 8;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const uint32_t* r = rr[h + (k >> 2)] + (k & 3) * 8;
                uint4 u;
                u.x = pack2<TOut>(__uint_as_float(r[0]), __uint_as_float(r[1]));
                u.y = pack2<TOut>(__uint_as_float(r[2]), __uint_as_float(r[3]));
                u.z = pack2<TOut>(__uint_as_float(r[4]), __uint_as_float(r[5]));
                u.w = pack2<TOut>(__uint_as_float(r[6]), __uint_as_float(r[7]));
                rowp[k ^ (lane & 7)] = u;
              }
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              __syncwarp();
              if (lane == 0) {
                tma_store_3d(&tmD, smem_u32(sb), c0, mt * BM + q * 32, b);
                bulk_commit();
              }
              ++store_count;
            }
            continue;
          }
        }
        if (!row_ok) continue;
#pragma unroll
        for (int h = 0; h < EPI / 32; ++h) {
        const uint32_t* r = rr[h];
        const int cc = cg + 32 * h;
        const int c0 = n0 + cc;
        if (c0 >= a.ocols) continue;
        TOut* p = orow + c0;
        const bool full = c0 + 32 <= a.ocols;
        if (a.accumulate) {
          // depth-tap accumulate: round the tap to the storage type, add in fp32, round again
          constexpr int E = 16 / sizeof(TOut);                 // elements per 16-byte vector
          if (full && ((reinterpret_cast<uintptr_t>(p) & 15) == 0)) {
            uint4 old[32 / E];
#pragma unroll
            for (int v = 0; v < 32 / E; ++v) old[v] = reinterpret_cast<const uint4*>(p)[v];
#pragma unroll
            for (int v = 0; v < 32 / E; ++v) {
              TOut* e = reinterpret_cast<TOut*>(&old[v]);
#pragma unroll
              for (int k = 0; k < E; ++k) {
                const float tap = Store<TOut>::to_f32(Store<TOut>::from_f32(__uint_as_float(r[v * E + k])));
                e[k] = Store<TOut>::from_f32(Store<TOut>::to_f32(e[k]) + tap);
              }
              reinterpret_cast<uint4*>(p)[v] = old[v];
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (c0 + j < a.ocols) {
                const float tap = Store<TOut>::to_f32(Store<TOut>::from_f32(__uint_as_float(r[j])));
                p[j] = Store<TOut>::from_f32(Store<TOut>::to_f32(p[j]) + tap);
              }
            }
          }
        } else if constexpr (sizeof(TOut) == 4) {
          if (full && ((reinterpret_cast<uintptr_t>(p) & 15) == 0)) {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              float4 f = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                     __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
              reinterpret_cast<float4*>(p)[v] = f;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c0 + j < a.ocols) p[j] = Store<TOut>::from_f32(__uint_as_float(r[j]));
          }
        } else {
          if (full && ((reinterpret_cast<uintptr_t>(p) & 15) == 0)) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 u;
              u.x = pack2<TOut>(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
              u.y = pack2<TOut>(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
              u.z = pack2<TOut>(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
              u.w = pack2<TOut>(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
              reinterpret_cast<uint4*>(p)[v] = u;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c0 + j < a.ocols) p[j] = Store<TOut>::from_f32(__uint_as_float(r[j]));
          }
        }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
    }
    if (a.tma_store && lane == 0) bulk_wait_all();   // the last stores have landed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

// Watchdog self-test: wait on an mbarrier phase that nothing completes, with a
// short limit, so the timeout path (error word, abort, return) is exercised
// without any risk of a hang.
__global__ void wait_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait(smem_u32(&bar), 0, reinterpret_cast<volatile int*>(&abort_flag), err, DEVERR_TIMEOUT_SELFTEST,
              limit_ns);
}

// ------------------------------- host side ----------------------------------

template <int BN, int MODE, typename TIn, typename TOut>
cudaError_t launch_kernel(const CUtensorMap& A, const CUtensorMap& B, const TcArgs& a, int sm_count,
                          cudaStream_t s, const CUtensorMap* D = nullptr) {
  auto k = tc_gemm_kernel<BN, MODE, TIn, TOut>;
  constexpr int smem = Cfg<BN>::template smem<TOut>();
  static_assert(smem <= 232448, "shared memory budget");
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  long long tiles = (long long)a.batches * a.m_tiles * a.n_tiles;
  if (tiles == 0) return cudaSuccess;
  int grid = (int)(tiles < sm_count ? tiles : sm_count);
  CUtensorMap none;
  memset(&none, 0, sizeof(none));
  return launch_pdl(k, dim3(grid), dim3(THREADS), smem, s, A, B, D ? *D : none, a);
}

// 3D map over D [batches][rows][cols] (fp32 or 16-bit) for the epilogue's TMA stores: boxes of
// 32 rows x 128 bytes (32 fp32 or 64 16-bit columns), 128-byte swizzle.  Rows must be 16-byte
// multiples and D 16-byte aligned; rows and columns past the ends are clipped by the map.
bool encode_store_map(CUtensorMap* m, const void* d, conv_dtype_t dt, long long cols, long long rows,
                      long long batches) {
  const int esz = dtype_size(dt);
  if ((cols * esz) % 16 != 0 || (reinterpret_cast<uintptr_t>(d) & 15)) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batches};
  cuuint64_t strides[2] = {(cuuint64_t)cols * esz, (cuuint64_t)rows * cols * esz};
  cuuint32_t box[3] = {(cuuint32_t)(128 / esz), 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapDataType t = dt == CONV_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : tmap_dtype(dt);
  return g_encode_tiled(m, t, 3, const_cast<void*>(d), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_wait_selftest(int* err_word, long long limit_ns, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(err_word, (unsigned long long)limit_ns);
  return cudaGetLastError();
}

bool tc_conv_supported(const Geom& g, conv_dtype_t dt, const void* in, const void* w) {
  if (dt == CONV_F32) return false;
  if (!driver_fns()) return false;
  if (g.c % 8 != 0) return false;                               // 16-byte row strides
  if ((reinterpret_cast<uintptr_t>(in) & 15) || (reinterpret_cast<uintptr_t>(w) & 15)) return false;
  if ((g.in_img_stride * 2) % 16 || (g.w_row_stride * 2) % 16) return false;
  if (g.sh > 8 || g.sw > 8) return false;                       // im2col traversal stride
  const int lw = -g.pw, lh = -g.ph;
  const int uw = g.pw - g.dw * (g.kw - 1), uh = g.ph - g.dh * (g.kh - 1);
  if (lw < -128 || lh < -128 || uw < -128 || uw > 127 || uh < -128 || uh > 127) return false;
  if ((long long)g.dw * (g.kw - 1) > 65535 || (long long)g.dh * (g.kh - 1) > 65535) return false;
  if (g.n <= 0 || g.oh <= 0 || g.ow <= 0) return false;
  if (g.out_img_stride != (long long)g.oh * g.ow * g.o) return false;
  return true;
}

cudaError_t launch_tc_conv(const void* in, const void* w, void* out, const Geom& g, conv_dtype_t dt,
                           int tile_n, int sm_count, int* err_word, bool accumulate, cudaStream_t s, int ksplit,
                           float* partial) {
  if (!tc_conv_supported(g, dt, in, w)) return cudaErrorNotSupported;
  const long long M = (long long)g.n * g.oh * g.ow;
  if (M == 0) return cudaSuccess;
  // A: im2col view of the NHWC input (C, W, H, N).
  CUtensorMap tA, tB;
  {
    cuuint64_t dims[4] = {(cuuint64_t)g.c, (cuuint64_t)g.w, (cuuint64_t)g.h, (cuuint64_t)g.n};
    cuuint64_t strides[3] = {(cuuint64_t)g.c * 2, (cuuint64_t)g.w * g.c * 2, (cuuint64_t)g.in_img_stride * 2};
    int lower[2] = {-g.pw, -g.ph};
    int upper[2] = {g.pw - g.dw * (g.kw - 1), g.ph - g.dh * (g.kh - 1)};
    cuuint32_t es[4] = {1, (cuuint32_t)g.sw, (cuuint32_t)g.sh, 1};
    CUresult r = g_encode_im2col(&tA, tmap_dtype(dt), 4, const_cast<void*>(in), dims, strides, lower, upper,
                                 BK, BM, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  // B: weights as (C, taps, O), row stride w_row_stride.
  const int taps = g.kh * g.kw;
  if (!encode_3d(&tB, dt, w, g.c, taps, g.o, (uint64_t)g.c * 2, (uint64_t)g.w_row_stride * 2, BK, 1,
                 tile_n))
    return cudaErrorInvalidValue;

  TcArgs a{};
  a.m_tiles = (int)((M + BM - 1) / BM);
  a.n_tiles = (g.o + tile_n - 1) / tile_n;
  a.batches = 1;
  a.kb_per_tap = (g.c + BK - 1) / BK;
  a.taps = taps;
  a.kw = g.kw; a.dh = g.dh; a.dw = g.dw;
  a.oh = g.oh; a.ow = g.ow; a.sh = g.sh; a.sw = g.sw; a.ph = g.ph; a.pw = g.pw;
  a.m_rows = M;
  a.ocols = g.o;
  a.out = out;
  a.ldo = g.o;
  a.out_batch = 0;
  a.accumulate = accumulate ? 1 : 0;
  a.ksplit = 1;
  a.err = err_word;
  if (ksplit > 1) {
    // split-K: ksplit partial fp32 results [ksplit][M][O], reduced by launch_splitk_reduce
    if (!partial || ksplit > taps * a.kb_per_tap) return cudaErrorInvalidValue;
    a.ksplit = ksplit;
    a.batches = ksplit;
    a.out = partial;
    a.out_batch = M * g.o;
    a.accumulate = 0;
    CUtensorMap tD;
    a.tma_store = encode_store_map(&tD, partial, CONV_F32, g.o, M, ksplit) ? 1 : 0;
    if (dt == CONV_BF16)
      return tile_n == 256 ? launch_kernel<256, 1, __nv_bfloat16, float>(tA, tB, a, sm_count, s, &tD)
                           : launch_kernel<128, 1, __nv_bfloat16, float>(tA, tB, a, sm_count, s, &tD);
    return tile_n == 256 ? launch_kernel<256, 1, __half, float>(tA, tB, a, sm_count, s, &tD)
                         : launch_kernel<128, 1, __half, float>(tA, tB, a, sm_count, s, &tD);
  }
  CUtensorMap tD;
  a.tma_store = !accumulate && encode_store_map(&tD, out, dt, g.o, M, 1) ? 1 : 0;
  if (dt == CONV_BF16)
    return tile_n == 256 ? launch_kernel<256, 1, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD)
                         : launch_kernel<128, 1, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD);
  return tile_n == 256 ? launch_kernel<256, 1, __half, __half>(tA, tB, a, sm_count, s, &tD)
                       : launch_kernel<128, 1, __half, __half>(tA, tB, a, sm_count, s, &tD);
}

bool tc_conv3d_supported(const Geom3& g, conv_dtype_t dt, const void* in, const void* w) {
  if (dt == CONV_F32) return false;
  if (!driver_fns()) return false;
  if (g.c % 8 != 0) return false;
  if ((reinterpret_cast<uintptr_t>(in) & 15) || (reinterpret_cast<uintptr_t>(w) & 15)) return false;
  if (g.sd > 8 || g.sh > 8 || g.sw > 8) return false;
  // 5D im2col bounding-box corners are limited to [-16, 15] per axis
  const int lo[3] = {-g.pw, -g.ph, -g.pd};
  const int up[3] = {g.pw - g.dw * (g.kw - 1), g.ph - g.dh * (g.kh - 1), g.pd - g.dd * (g.kd - 1)};
  for (int i = 0; i < 3; ++i)
    if (lo[i] < -16 || lo[i] > 15 || up[i] < -16 || up[i] > 15) return false;
  if ((long long)g.dw * (g.kw - 1) > 65535 || (long long)g.dh * (g.kh - 1) > 65535 ||
      (long long)g.dd * (g.kd - 1) > 65535)
    return false;
  return g.n > 0 && g.od > 0 && g.oh > 0 && g.ow > 0;
}

cudaError_t launch_tc_conv3d(const void* in, const void* w, void* out, const Geom3& g, conv_dtype_t dt, int tile_n,
                             int sm_count, int* err_word, cudaStream_t s) {
  if (!tc_conv3d_supported(g, dt, in, w)) return cudaErrorNotSupported;
  const long long M = (long long)g.n * g.od * g.oh * g.ow;
  if (M == 0) return cudaSuccess;
  CUtensorMap tA, tB;
  {
    // A: im2col view of the NDHWC input (C, W, H, D, N)
    cuuint64_t dims[5] = {(cuuint64_t)g.c, (cuuint64_t)g.w, (cuuint64_t)g.h, (cuuint64_t)g.d, (cuuint64_t)g.n};
    cuuint64_t strides[4] = {(cuuint64_t)g.c * 2, (cuuint64_t)g.w * g.c * 2, (cuuint64_t)g.h * g.w * g.c * 2,
                             (cuuint64_t)g.d * g.h * g.w * g.c * 2};
    int lower[3] = {-g.pw, -g.ph, -g.pd};
    int upper[3] = {g.pw - g.dw * (g.kw - 1), g.ph - g.dh * (g.kh - 1), g.pd - g.dd * (g.kd - 1)};
    cuuint32_t es[5] = {1, (cuuint32_t)g.sw, (cuuint32_t)g.sh, (cuuint32_t)g.sd, 1};
    CUresult r = g_encode_im2col(&tA, tmap_dtype(dt), 5, const_cast<void*>(in), dims, strides, lower, upper, BK, BM,
                                 es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  const int taps = g.kd * g.kh * g.kw;
  if (!encode_3d(&tB, dt, w, g.c, taps, g.o, (uint64_t)g.c * 2, (uint64_t)taps * g.c * 2, BK, 1, tile_n))
    return cudaErrorInvalidValue;
  TcArgs a{};
  a.m_tiles = (int)((M + BM - 1) / BM);
  a.n_tiles = (g.o + tile_n - 1) / tile_n;
  a.batches = 1;
  a.kb_per_tap = (g.c + BK - 1) / BK;
  a.taps = taps;
  a.kw = g.kw; a.dh = g.dh; a.dw = g.dw;
  a.oh = g.oh; a.ow = g.ow; a.sh = g.sh; a.sw = g.sw; a.ph = g.ph; a.pw = g.pw;
  a.kh = g.kh; a.od = g.od; a.sd = g.sd; a.pd = g.pd; a.dd = g.dd;
  a.ksplit = 1;
  a.m_rows = M;
  a.ocols = g.o;
  a.out = out;
  a.ldo = g.o;
  a.out_batch = 0;
  a.accumulate = 0;
  a.err = err_word;
  CUtensorMap tD;
  a.tma_store = encode_store_map(&tD, out, dt, g.o, M, 1) ? 1 : 0;
  if (dt == CONV_BF16)
    return tile_n == 256 ? launch_kernel<256, 2, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD)
                         : launch_kernel<128, 2, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD);
  return tile_n == 256 ? launch_kernel<256, 2, __half, __half>(tA, tB, a, sm_count, s, &tD)
                       : launch_kernel<128, 2, __half, __half>(tA, tB, a, sm_count, s, &tD);
}

cudaError_t launch_tc_batched_gemm(const BatchedGemm& bg, conv_dtype_t dt, int tile_n, int sm_count,
                                   int* err_word, cudaStream_t s) {
  if (dt == CONV_F32 || !driver_fns()) return cudaErrorNotSupported;
  if (bg.c % 8 != 0 || (reinterpret_cast<uintptr_t>(bg.a) & 15) || (reinterpret_cast<uintptr_t>(bg.b) & 15))
    return cudaErrorNotSupported;
  if (bg.t == 0 || bg.batches == 0) return cudaSuccess;
  CUtensorMap tA, tB;
  if (!encode_3d(&tA, dt, bg.a, bg.c, bg.t, bg.batches, (uint64_t)bg.c * 2, (uint64_t)bg.t * bg.c * 2, BK,
                 BM, 1))
    return cudaErrorInvalidValue;
  if (!encode_3d(&tB, dt, bg.b, bg.c, bg.o, bg.batches, (uint64_t)bg.c * 2, (uint64_t)bg.o * bg.c * 2, BK,
                 tile_n, 1))
    return cudaErrorInvalidValue;
  TcArgs a{};
  a.m_tiles = (bg.t + BM - 1) / BM;
  a.n_tiles = (bg.o + tile_n - 1) / tile_n;
  a.batches = bg.batches;
  a.kb_per_tap = (bg.c + BK - 1) / BK;
  a.taps = 1;
  a.kw = 1; a.dh = 1; a.dw = 1;
  a.oh = 1; a.ow = bg.t; a.sh = 1; a.sw = 1; a.ph = 0; a.pw = 0;
  a.m_rows = bg.t;
  a.ocols = bg.o;
  a.out = bg.d;
  a.ldo = bg.o;
  a.out_batch = (long long)bg.t * bg.o;
  a.ksplit = 1;
  a.err = err_word;
  if (bg.d_dt != CONV_F32) {
    // D in the operand type: the vectorised 16-bit epilogue
    if (bg.d_dt != dt) return cudaErrorInvalidValue;
    CUtensorMap tD16;
    a.tma_store = encode_store_map(&tD16, bg.d, dt, bg.o, bg.t, bg.batches) ? 1 : 0;
    if (dt == CONV_BF16)
      return tile_n == 256 ? launch_kernel<256, 0, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD16)
                           : launch_kernel<128, 0, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD16);
    return tile_n == 256 ? launch_kernel<256, 0, __half, __half>(tA, tB, a, sm_count, s, &tD16)
                         : launch_kernel<128, 0, __half, __half>(tA, tB, a, sm_count, s, &tD16);
  }
  CUtensorMap tD;
  a.tma_store = encode_store_map(&tD, bg.d, CONV_F32, bg.o, bg.t, bg.batches) ? 1 : 0;
  if (dt == CONV_BF16)
    return tile_n == 256 ? launch_kernel<256, 0, __nv_bfloat16, float>(tA, tB, a, sm_count, s, &tD)
                         : launch_kernel<128, 0, __nv_bfloat16, float>(tA, tB, a, sm_count, s, &tD);
  return tile_n == 256 ? launch_kernel<256, 0, __half, float>(tA, tB, a, sm_count, s, &tD)
                       : launch_kernel<128, 0, __half, float>(tA, tB, a, sm_count, s, &tD);
}

}  // namespace b200conv
