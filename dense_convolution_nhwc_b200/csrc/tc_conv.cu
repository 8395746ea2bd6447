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

// CG = 1: one CTA computes a 128 x BN tile.  CG = 2: a CTA pair computes a
// 256 x BN tile, each CTA holding 128 rows of A and BN/2 rows of B per stage.
// PARTS = 3: the split-bf16 batched GEMM, whose stage holds the three bf16
// parts of one 64-wide K block of A and of B.
template <int BN, int CG = 1, int PARTS = 1> struct Cfg {
  static constexpr int STAGES = PARTS == 3 ? 2 : (CG == 2 ? (BN == 256 ? 6 : 8) : (BN == 256 ? 4 : 6));
  static constexpr int A_PART = BM * BK * 2;
  static constexpr int B_PART = (BN / CG) * BK * 2;
  static constexpr int A_BYTES = PARTS * A_PART;
  static constexpr int B_BYTES = PARTS * B_PART;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // two fp32 accumulators, ACC_COLS apart; the allocation is a power of two
  // columns (BN = 96: 256 columns, the accumulators at 0 and 128)
  static constexpr int TMEM_COLS = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
  static constexpr int ACC_COLS = TMEM_COLS / 2;
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
  int cluster_reduce;          // split-K whose ksplit CTAs of a tile form a cluster: rank 0 sums the
                               // others' fp32 partials from their shared memory and writes out
  int split_cb;                // MODE 3 (split-bf16 batched GEMM): 64-wide K blocks per part; A and B
                               // rows hold three parts of C side by side
  int serial_reduce;           // split-K whose last-arriving split of a tile sums the fp32 partials
  float* partial;              // serial_reduce: [ksplit][m_rows][ocols] fp32 partials
  long long part_batch;        // serial_reduce: elements between splits' partials
  int* tile_cnt;               // serial_reduce: m_tiles * n_tiles * 4 arrival counters (one per tile and
                               // epilogue warp), zero on entry
  int* err;
};

// --------------------------------- kernel -----------------------------------

// MODE 0: batched GEMM (tiled A); 1: conv2d (4D im2col A); 2: conv3d (5D im2col A);
// 3: batched GEMM over split-bf16 operands (each stage the three parts of a K
// block of A and of B; the six products a_i b_j with i + j <= 2 per stage).
// CG = 2: CTA pairs (clusters of 2) on 256-row tiles, a.m_tiles counting 256-row tiles.
template <int BN, int MODE, typename TIn, typename TOut, int CG = 1>
__global__ void __launch_bounds__(THREADS, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmD, const TcArgs a) {
  using C = Cfg<BN, CG, MODE == 3 ? 3 : 1>;
  static_assert(MODE != 3 || CG == 1, "split-bf16 GEMM on single CTAs");
  constexpr int STORE_BYTES = C::STORE_BYTES;
  constexpr uint32_t IDESC = make_idesc<BN, BM * CG>(std::is_same<TIn, __nv_bfloat16>::value ? 1u : 0u);
  static_assert(CG == 1 || CG == 2, "CTA group");

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
  static_assert(BM * BN * 4 <= C::STAGES * C::STAGE_BYTES, "split partial fits the stage ring");
  const bool cl = CG == 1 && MODE == 1 && a.cluster_reduce;
  const bool sr = CG == 1 && MODE == 1 && a.serial_reduce && !a.cluster_reduce;
  const uint32_t crank = cl ? cluster_rank() : 0u;
  // CTA pair: rank 0 issues the MMAs; both load and drain their own halves.
  const uint32_t prank = CG == 2 ? cluster_rank() : 0u;
  const long long tile0 = CG == 2 ? (long long)(blockIdx.x >> 1) : (long long)blockIdx.x;
  const long long tile_step = CG == 2 ? (long long)(gridDim.x >> 1) : (long long)gridDim.x;
  // In cluster mode the grid holds one CTA per (tile, split), the splits of a
  // tile adjacent (the cluster); map to the tile order of the other modes.
  auto tile_of = [&](long long lt) {
    if (!cl) return lt;
    return (lt % a.ksplit) * ((long long)a.m_tiles * a.n_tiles) + lt / a.ksplit;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 128 * CG);     // CTA pair: both CTAs' epilogue threads, on rank 0's barrier
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      // the same warp of both CTAs allocates, with the same destination offset
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"((uint32_t)C::TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"((uint32_t)C::TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  if (threadIdx.x == 32) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (a.tma_store) prefetch_tensormap(&tmD);
  }
  tc_fence_before();
  if (cl || CG == 2)
    cluster_sync_all();     // every CTA's barriers are initialised before any remote arrive
  else
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
      for (long long lt = tile0; lt < total_tiles && ok; lt += tile_step) {
        const long long tile = tile_of(lt);
        const int nt = (int)(tile % a.n_tiles);
        const long long rest = tile / a.n_tiles;
        const int mt = (int)(rest % a.m_tiles);
        const int b = (int)(rest / a.m_tiles);
        // this CTA's 128 rows of the tile (the second half of a pair's 256)
        const long long row0 = (long long)mt * (BM * CG) + (long long)prank * BM;
        int img = 0, wx = 0, hy = 0, dz = 0;
        if (MODE == 1 || MODE == 2) {
          // first output pixel of the tile -> its window's corner in the input
          const long long m0 = row0;
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
        if ((MODE == 1 || MODE == 2) && a.ksplit > 1) {
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
          const uint32_t dA = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t dB = smem_u32(sB + stage * C::B_BYTES);
          if constexpr (CG == 2) {
            // both CTAs' loads complete on rank 0's full barrier, which expects both halves
            if (prank == 0) mbar_expect_tx(full_bar(stage), 2 * C::STAGE_BYTES);
            const uint32_t fb0 = mapa_shared(full_bar(stage), 0);
            const int ncol = nt * BN + (int)prank * (BN / 2);
            if (MODE == 1) {
              const int ky = tap / a.kw, kx = tap - (tap / a.kw) * a.kw;
              tma_load_im2col_4d_pair(dA, &tmA, fb0, kb * BK, wx, hy, img, (uint16_t)(kx * a.dw),
                                      (uint16_t)(ky * a.dh));
              tma_load_3d_pair(dB, &tmB, fb0, kb * BK, tap, ncol);
            } else if (MODE == 2) {
              const int khw = a.kh * a.kw;
              const int kz = tap / khw, r2 = tap - kz * khw;
              const int ky = r2 / a.kw, kx = r2 - (r2 / a.kw) * a.kw;
              tma_load_im2col_5d_pair(dA, &tmA, fb0, kb * BK, wx, hy, dz, img, (uint16_t)(kx * a.dw),
                                      (uint16_t)(ky * a.dh), (uint16_t)(kz * a.dd));
              tma_load_3d_pair(dB, &tmB, fb0, kb * BK, tap, ncol);
            } else {
              tma_load_3d_pair(dA, &tmA, fb0, kb * BK, (int)row0, b);
              tma_load_3d_pair(dB, &tmB, fb0, kb * BK, ncol, b);
            }
            ++issued;
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          const uint32_t fb = full_bar(stage);
          mbar_expect_tx(fb, C::STAGE_BYTES);
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
          } else if (MODE == 3) {
            // the three parts of K block kb of A and of B, one barrier for all six
#pragma unroll
            for (int pt = 0; pt < 3; ++pt) {
              tma_load_3d(dA + pt * C::A_PART, &tmA, fb, (pt * a.split_cb + kb) * BK, (int)row0, b);
              tma_load_3d(dB + pt * C::B_PART, &tmB, fb, (pt * a.split_cb + kb) * BK, nt * BN, b);
            }
          } else {
            tma_load_3d(dA, &tmA, fb, kb * BK, (int)row0, b);
            tma_load_3d(dB, &tmB, fb, kb * BK, nt * BN, b);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: wait (bounded) until the last loads in flight have landed.  A pair's
      // loads land on rank 0's barriers, so rank 0 drains for both.
      const int pending = (CG == 2 && prank != 0) ? 0 : (issued < C::STAGES ? (int)issued : C::STAGES);
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
    // (a CTA pair's MMAs are issued by rank 0 alone, for both CTAs)
    if (lane == 0 && (CG == 1 || prank == 0)) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (long long lt = tile0; lt < total_tiles && ok; lt += tile_step, ++it) {
        const long long tile = tile_of(lt);
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, a.err, DEVERR_TIMEOUT_MMA_TMEM)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * C::ACC_COLS);
        int nks = ksteps;
        if ((MODE == 1 || MODE == 2) && a.ksplit > 1) {
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
          if constexpr (CG == 2) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              tc_mma_pair(d_tmem, sdesc(aa + 32u * k), sdesc(bb + 32u * k), IDESC, (ks | k) != 0 ? 1u : 0u);
            tc_commit_pair_both(empty_bar(stage));      // frees the stage in both CTAs
          } else if constexpr (MODE == 3) {
            // products a_i b_j, i + j <= 2: A parts (0,0,1,0,1,2) against B parts (0,1,0,2,1,0)
#pragma unroll
            for (int term = 0; term < 6; ++term) {
              const uint32_t ai = (0x210100u >> (4 * term)) & 0xFu, bj = (0x012010u >> (4 * term)) & 0xFu;
#pragma unroll
              for (int k = 0; k < BK / 16; ++k)
                tc_mma(d_tmem, sdesc(aa + ai * C::A_PART + 32u * k), sdesc(bb + bj * C::B_PART + 32u * k), IDESC,
                       (ks | term | k) != 0 ? 1u : 0u);
            }
            tc_commit(empty_bar(stage));
          } else {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              tc_mma(d_tmem, sdesc(aa + 32u * k), sdesc(bb + 32u * k), IDESC, (ks | k) != 0 ? 1u : 0u);
            tc_commit(empty_bar(stage));
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) {
          if constexpr (CG == 2)
            tc_commit_pair_both(tfull_bar(acc));       // both CTAs' accumulator halves are ready
          else
            tc_commit(tfull_bar(acc));
        }
      }
      // Drain: all MMAs this thread issued have completed once this arrives.
      if constexpr (CG == 2)
        tc_commit_pair_self(drain_bar);
      else
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
    for (long long lt = tile0; lt < total_tiles; lt += tile_step, ++it) {
      const long long tile = tile_of(lt);
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag, a.err, DEVERR_TIMEOUT_EPILOGUE)) break;
      tc_fence_after();
      if (cl) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the ring is reused for the partial
      const int nt = (int)(tile % a.n_tiles);
      const long long rest = tile / a.n_tiles;
      const int mt = (int)(rest % a.m_tiles);
      const int b = (int)(rest / a.m_tiles);
      const long long trow0 = (long long)mt * (BM * CG) + (long long)prank * BM;   // this CTA's first row
      const long long m = trow0 + row;
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
          const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_COLS + cg + 32 * h);
          TMEM_LD32(taddr, rr[h]);
        }
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (cl) {
          // split-K in a cluster: this split's fp32 partial goes to the (drained) stage
          // ring as [128 rows][BN/4 float4], the float4 column XOR-swizzled by the row so
          // that both this row-per-lane write and the column-per-lane reads of the
          // reduction below are free of bank conflicts
#pragma unroll
          for (int h = 0; h < EPI / 32; ++h)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int col4 = (cg + 32 * h) / 4 + k;
              *reinterpret_cast<float4*>(sA + ((size_t)row * (BN / 4) + (col4 ^ (row & (BN / 4 - 1)))) * 16) =
                  make_float4(__uint_as_float(rr[h][4 * k]), __uint_as_float(rr[h][4 * k + 1]),
                              __uint_as_float(rr[h][4 * k + 2]), __uint_as_float(rr[h][4 * k + 3]));
            }
          continue;
        }
        if (sr) {
          // serial split-K: this split's fp32 partial rows (the output comes later)
          if (row_ok) {
            float* prow = a.partial + (long long)b * a.part_batch + m * a.ocols;
            const bool vec4 = (a.ocols & 3) == 0;
#pragma unroll
            for (int h = 0; h < EPI / 32; ++h) {
              const int c0 = n0 + cg + 32 * h;
              if (c0 >= a.ocols) continue;
              if (vec4 && c0 + 32 <= a.ocols) {
#pragma unroll
                for (int v = 0; v < 8; ++v)
                  reinterpret_cast<float4*>(prow + c0)[v] =
                      make_float4(__uint_as_float(rr[h][4 * v]), __uint_as_float(rr[h][4 * v + 1]),
                                  __uint_as_float(rr[h][4 * v + 2]), __uint_as_float(rr[h][4 * v + 3]));
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (c0 + j < a.ocols) prow[c0 + j] = __uint_as_float(rr[h][j]);
              }
            }
          }
          continue;
        }
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
                tma_store_3d(&tmD, smem_u32(sb), c0, (int)trow0 + q * 32, b);
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
                tma_store_3d(&tmD, smem_u32(sb), c0, (int)trow0 + q * 32, b);
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
      if (CG == 2 && prank != 0)
        mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));   // the pair's accumulator lives on in rank 0's count
      else
        mbar_arrive(tempty_bar(acc));
      if (sr) {
        // Serial split-K, per epilogue warp (its 32 rows): publish this split's
        // partial rows, count the arrivals at (tile, warp); the split that arrives
        // last sums all partials in split order (the order of the reduce kernel)
        // and writes those output rows.  No warp or split waits for another.
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          int* cnt = a.tile_cnt + (((long long)mt * a.n_tiles + nt) * 4 + q);
          last = atomicAdd(cnt, 1) == a.ksplit - 1;
          if (last) *cnt = 0;              // ready for the next call on this workspace
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          // warp q sums its 32 rows, 8 at a time, lane = 4 columns: the 8 rows'
          // loads of one split are in flight together
          TOut* obase = static_cast<TOut*>(a.out);
          const bool vec4 = (a.ocols & 3) == 0;
          for (int c4 = lane; c4 < BN / 4; c4 += 32) {
            const int col = n0 + 4 * c4;
            if (col >= a.ocols) continue;
            const int nv = a.ocols - col < 4 ? a.ocols - col : 4;
            for (int i0 = 0; i0 < 32; i0 += 8) {
              float4 acc[8];
              bool rok[8];
#pragma unroll
              for (int r = 0; r < 8; ++r) {
                const long long mr = trow0 + q * 32 + i0 + r;
                rok[r] = mr < a.m_rows;
                acc[r] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (rok[r] && vec4) acc[r] = __ldcg(reinterpret_cast<const float4*>(a.partial + mr * a.ocols + col));
              }
              if (vec4) {
#pragma unroll 2
                for (int sp = 1; sp < a.ksplit; ++sp) {
                  float4 t[8];
#pragma unroll
                  for (int r = 0; r < 8; ++r) {
                    const long long mr = trow0 + q * 32 + i0 + r;
                    t[r] = rok[r] ? __ldcg(reinterpret_cast<const float4*>(a.partial + sp * a.part_batch +
                                                                            mr * a.ocols + col))
                                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                  }
#pragma unroll
                  for (int r = 0; r < 8; ++r) {
                    acc[r].x += t[r].x; acc[r].y += t[r].y; acc[r].z += t[r].z; acc[r].w += t[r].w;
                  }
                }
              } else {
                // O not a multiple of 4: element by element, in split order from 0
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                  if (!rok[r]) continue;
                  const long long mr = trow0 + q * 32 + i0 + r;
                  float e4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                  for (int e = 0; e < nv; ++e) {
                    float sum = 0.0f;
                    for (int sp = 0; sp < a.ksplit; ++sp) sum += __ldcg(a.partial + sp * a.part_batch + mr * a.ocols + col + e);
                    e4[e] = sum;
                  }
                  acc[r] = make_float4(e4[0], e4[1], e4[2], e4[3]);
                }
              }
#pragma unroll
              for (int r = 0; r < 8; ++r) {
                if (!rok[r]) continue;
                const long long mr = trow0 + q * 32 + i0 + r;
                TOut* po = obase + mr * a.ldo + col;
                const float v[4] = {acc[r].x, acc[r].y, acc[r].z, acc[r].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  if (e < nv) {
                    float rv = v[e];
                    if (a.accumulate) rv = Store<TOut>::to_f32(po[e]) + Store<TOut>::to_f32(Store<TOut>::from_f32(v[e]));
                    po[e] = Store<TOut>::from_f32(rv);
                  }
                }
              }
            }
          }
        }
      }
    }
    if (a.tma_store && lane == 0) bulk_wait_all();   // the last stores have landed
    __syncwarp();
  }

  tc_fence_before();
  if (cl) {
    // Split-K reduction, shared by the cluster: once every split's partial is in
    // (the barrier), CTA r sums rows [128 r / ks, 128 (r + 1) / ks) of the tile
    // over the splits in split order (the order of the separate reduce kernel)
    // from the CTAs' shared memory, and writes those output rows.
    cluster_sync_all();
    if (warp >= 2 && !*abort_flag) {
      const int ks = a.ksplit;
      const long long tile = tile_of(blockIdx.x);
      const int nt = (int)(tile % a.n_tiles);
      const int mt = (int)((tile / a.n_tiles) % a.m_tiles);
      const int ew = warp - 2;
      const int r_lo = (int)((long long)BM * crank / ks), r_hi = (int)((long long)BM * (crank + 1) / ks);
      const uint32_t pbase = smem_u32(sA);
      TOut* obase = static_cast<TOut*>(a.out);
      for (int rr = r_lo + ew; rr < r_hi; rr += 4) {
        const long long m = (long long)mt * BM + rr;
        if (m >= a.m_rows) break;
        for (int c4 = lane; c4 < BN / 4; c4 += 32) {
          const int col = nt * BN + 4 * c4;
          if (col >= a.ocols) continue;
          const uint32_t off = (uint32_t)(((size_t)rr * (BN / 4) + (c4 ^ (rr & (BN / 4 - 1)))) * 16);
          float4 sum = ld_cluster_f4(mapa_shared(pbase, 0) + off);
          for (int sp = 1; sp < ks; ++sp) {
            const float4 pv = ld_cluster_f4(mapa_shared(pbase, (uint32_t)sp) + off);
            sum.x += pv.x; sum.y += pv.y; sum.z += pv.z; sum.w += pv.w;
          }
          TOut* p = obase + m * a.ldo + col;
          float v[4] = {sum.x, sum.y, sum.z, sum.w};
          const int nv = a.ocols - col < 4 ? a.ocols - col : 4;
          if (a.accumulate) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < nv)
                v[e] = Store<TOut>::to_f32(p[e]) + Store<TOut>::to_f32(Store<TOut>::from_f32(v[e]));
          }
          if (nv == 4 && (reinterpret_cast<uintptr_t>(p) & (4 * sizeof(TOut) - 1)) == 0) {
            if constexpr (sizeof(TOut) == 4) {
              *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
            } else {
              uint2 u;
              u.x = pack2<TOut>(v[0], v[1]);
              u.y = pack2<TOut>(v[2], v[3]);
              *reinterpret_cast<uint2*>(p) = u;
            }
          } else {
            for (int e = 0; e < nv; ++e) p[e] = Store<TOut>::from_f32(v[e]);
          }
        }
      }
    }
  }
  // In cluster mode no CTA leaves while another may still read its shared
  // memory: every wait above is bounded, so every thread of the cluster
  // reaches this barrier.
  if (cl || CG == 2)
    cluster_sync_all();
  else
    __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (CG == 2)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"((uint32_t)C::TMEM_COLS)
                   : "memory");
    else
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
  constexpr int smem = Cfg<BN, 1, MODE == 3 ? 3 : 1>::template smem<TOut>();
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

// CTA pairs: clusters of 2 on 256-row tiles, persistent over the tiles (one
// pair per two SMs).  Sets *launched = false and launches nothing when the
// device cannot hold such a pair (the caller then runs the 1-CTA kernel).
template <int BN, int MODE, typename TIn, typename TOut>
cudaError_t launch_kernel_pair(const CUtensorMap& A, const CUtensorMap& B, const TcArgs& a, int sm_count,
                               cudaStream_t s, const CUtensorMap* D, bool* launched) {
  *launched = false;
  auto k = tc_gemm_kernel<BN, MODE, TIn, TOut, 2>;
  constexpr int smem = Cfg<BN, 2>::template smem<TOut>();
  static_assert(smem <= 232448, "shared memory budget");
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)a.batches * a.m_tiles * a.n_tiles;
  if (tiles == 0) return cudaSuccess;
  const long long pairs = tiles < sm_count / 2 ? tiles : sm_count / 2;
  if (pairs < 1) return cudaSuccess;
  static std::mutex mu;
  static int ok_dev[64];          // 0 unknown, 1 yes, -1 no
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return cudaSuccess;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (ok_dev[dev] == 0) {
      cfg.numAttrs = 1;
      int n = 0;
      const cudaError_t qe = cudaOccupancyMaxActiveClusters(&n, k, &cfg);
      if (qe != cudaSuccess) cudaGetLastError();
      ok_dev[dev] = (qe == cudaSuccess && n >= 1) ? 1 : -1;
    }
    if (ok_dev[dev] < 0) return cudaSuccess;
  }
  cfg.numAttrs = 2;
  CUtensorMap none;
  memset(&none, 0, sizeof(none));
  e = cudaLaunchKernelEx(&cfg, k, A, B, D ? *D : none, a);
  if (e == cudaSuccess) *launched = true;
  return e;
}

// Run the 1-CTA kernel, or (tile_m == 256) the CTA-pair kernel when the device
// can hold a pair.  `a.m_tiles` counts rows in units of tile_m; the caller
// encodes B with a box of BN / (tile_m / 128) rows.
template <int BN, int MODE, typename TIn, typename TOut>
cudaError_t launch_tiles(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& Bpair, const TcArgs& a,
                         int tile_m, int sm_count, cudaStream_t s, const CUtensorMap* D) {
  if (tile_m == 256) {
    bool launched = false;
    cudaError_t e = launch_kernel_pair<BN, MODE, TIn, TOut>(A, Bpair, a, sm_count, s, D, &launched);
    if (e != cudaSuccess || launched) return e;
  }
  TcArgs one = a;
  one.m_tiles = (int)((a.m_rows + BM - 1) / BM);
  return launch_kernel<BN, MODE, TIn, TOut>(A, B, one, sm_count, s, D);
}

// Split-K with the splits of each tile as one thread-block cluster of ks CTAs
// (grid = tiles x ks, one (tile, split) per CTA).  Sets *launched = false and
// launches nothing when the device cannot hold such a cluster (the caller then
// takes the partials-and-reduce route).
template <int BN, int MODE, typename TIn, typename TOut>
cudaError_t launch_kernel_cluster(const CUtensorMap& A, const CUtensorMap& B, const TcArgs& a, int ks,
                                  cudaStream_t s, const CUtensorMap* D, bool* launched) {
  *launched = false;
  auto k = tc_gemm_kernel<BN, MODE, TIn, TOut>;
  constexpr int smem = Cfg<BN>::template smem<TOut>();
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)a.batches * a.m_tiles * a.n_tiles;
  if (tiles == 0 || tiles % ks != 0 || tiles > 0x7fffffffLL) return cudaSuccess;
  // How many clusters of ks such CTAs can be resident at once?  Asked once per
  // (kernel, ks, device).  Clusters need ks SMs of one GPC each, so fewer fit
  // than 148 / ks; unless all of this launch's clusters fit in one wave the
  // partials-and-reduce route is faster, and the caller takes it.
  static std::mutex mu;
  static int cache[64][17];      // [device][ks]: 0 unknown, -1 none, else the resident cluster count
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64 || ks > 16) return cudaSuccess;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev][ks] == 0) {
      if (ks > 8) cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3((unsigned)tiles);
      q.blockDim = dim3(THREADS);
      q.dynamicSmemBytes = smem;
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = ks;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      q.attrs = qa;
      q.numAttrs = 1;
      int n = 0;
      const cudaError_t qe = cudaOccupancyMaxActiveClusters(&n, k, &q);
      if (qe != cudaSuccess) cudaGetLastError();      // clear it: the answer is "no"
      cache[dev][ks] = (qe == cudaSuccess && n >= 1) ? n : -1;
    }
    if (cache[dev][ks] < 0 || tiles / ks > cache[dev][ks]) return cudaSuccess;
  }
  CUtensorMap none;
  memset(&none, 0, sizeof(none));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)tiles);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, k, A, B, D ? *D : none, a);
  if (e == cudaSuccess) *launched = true;
  return e;
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
                           float* partial, bool* reduced, int tile_m, int* tile_cnt) {
  if (reduced) *reduced = false;
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
  if (ksplit > 1 && reduced && tile_cnt && partial && ksplit <= taps * a.kb_per_tap) {
    // split-K inside the kernel, serially: the last split of each (tile, epilogue
    // warp) sums the fp32 partials in split order and writes the output
    TcArgs c = a;
    c.ksplit = ksplit;
    c.batches = ksplit;
    c.serial_reduce = 1;
    c.partial = partial;
    c.part_batch = M * g.o;
    c.tile_cnt = tile_cnt;
    c.tma_store = 0;
    cudaError_t e;
    if (dt == CONV_BF16)
      e = tile_n == 256 ? launch_kernel<256, 1, __nv_bfloat16, __nv_bfloat16>(tA, tB, c, sm_count, s)
                        : launch_kernel<128, 1, __nv_bfloat16, __nv_bfloat16>(tA, tB, c, sm_count, s);
    else
      e = tile_n == 256 ? launch_kernel<256, 1, __half, __half>(tA, tB, c, sm_count, s)
                        : launch_kernel<128, 1, __half, __half>(tA, tB, c, sm_count, s);
    if (e == cudaSuccess) *reduced = true;
    return e;
  }
  if (ksplit > 1 && reduced && !tile_cnt && ksplit <= 16 && ksplit <= taps * a.kb_per_tap) {
    // split-K inside the kernel: the ksplit CTAs of a tile form a cluster and
    // rank 0 adds the others' partials (in split order) from their shared memory
    TcArgs c = a;
    c.ksplit = ksplit;
    c.batches = ksplit;
    c.cluster_reduce = 1;
    CUtensorMap tD;
    c.tma_store = !accumulate && encode_store_map(&tD, out, dt, g.o, M, 1) ? 1 : 0;
    bool launched = false;
    cudaError_t e;
    if (dt == CONV_BF16)
      e = tile_n == 256 ? launch_kernel_cluster<256, 1, __nv_bfloat16, __nv_bfloat16>(tA, tB, c, ksplit, s, &tD, &launched)
                        : launch_kernel_cluster<128, 1, __nv_bfloat16, __nv_bfloat16>(tA, tB, c, ksplit, s, &tD, &launched);
    else
      e = tile_n == 256 ? launch_kernel_cluster<256, 1, __half, __half>(tA, tB, c, ksplit, s, &tD, &launched)
                        : launch_kernel_cluster<128, 1, __half, __half>(tA, tB, c, ksplit, s, &tD, &launched);
    if (e != cudaSuccess) return e;
    if (launched) {
      *reduced = true;
      return cudaSuccess;
    }
  }
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
  if (tile_n == 256 && tile_m == 256) {
    // CTA pairs: each CTA loads 128 weight rows of the 256-column tile
    CUtensorMap tBp;
    if (!encode_3d(&tBp, dt, w, g.c, taps, g.o, (uint64_t)g.c * 2, (uint64_t)g.w_row_stride * 2, BK, 1, 128))
      return cudaErrorInvalidValue;
    TcArgs p = a;
    p.m_tiles = (int)((M + 255) / 256);
    if (dt == CONV_BF16)
      return launch_tiles<256, 1, __nv_bfloat16, __nv_bfloat16>(tA, tB, tBp, p, 256, sm_count, s, &tD);
    return launch_tiles<256, 1, __half, __half>(tA, tB, tBp, p, 256, sm_count, s, &tD);
  }
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
                             int sm_count, int* err_word, cudaStream_t s, int tile_m) {
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
  if (tile_n == 256 && tile_m == 256) {
    CUtensorMap tBp;
    if (!encode_3d(&tBp, dt, w, g.c, taps, g.o, (uint64_t)g.c * 2, (uint64_t)taps * g.c * 2, BK, 1, 128))
      return cudaErrorInvalidValue;
    TcArgs p = a;
    p.m_tiles = (int)((M + 255) / 256);
    if (dt == CONV_BF16)
      return launch_tiles<256, 2, __nv_bfloat16, __nv_bfloat16>(tA, tB, tBp, p, 256, sm_count, s, &tD);
    return launch_tiles<256, 2, __half, __half>(tA, tB, tBp, p, 256, sm_count, s, &tD);
  }
  if (dt == CONV_BF16)
    return tile_n == 256 ? launch_kernel<256, 2, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD)
                         : launch_kernel<128, 2, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD);
  return tile_n == 256 ? launch_kernel<256, 2, __half, __half>(tA, tB, a, sm_count, s, &tD)
                       : launch_kernel<128, 2, __half, __half>(tA, tB, a, sm_count, s, &tD);
}

cudaError_t launch_tc_batched_gemm(const BatchedGemm& bg, conv_dtype_t dt, int tile_n, int sm_count,
                                   int* err_word, cudaStream_t s, int tile_m) {
  if (dt == CONV_F32 || !driver_fns()) return cudaErrorNotSupported;
  if (bg.c % 8 != 0 || (reinterpret_cast<uintptr_t>(bg.a) & 15) || (reinterpret_cast<uintptr_t>(bg.b) & 15))
    return cudaErrorNotSupported;
  if (bg.split_bf16 && (dt != CONV_BF16 || bg.c % BK != 0 || bg.d_dt != CONV_F32)) return cudaErrorNotSupported;
  if (bg.t == 0 || bg.batches == 0) return cudaSuccess;
  // K extents of A and B (the split-bf16 GEMM: rows of three C-wide parts)
  const long long ka = bg.split_bf16 ? 3LL * bg.c : bg.c, kb_ = ka;
  CUtensorMap tA, tB;
  if (!encode_3d(&tA, dt, bg.a, ka, bg.t, bg.batches, (uint64_t)ka * 2, (uint64_t)bg.t * ka * 2, BK, BM, 1))
    return cudaErrorInvalidValue;
  if (!encode_3d(&tB, dt, bg.b, kb_, bg.o, bg.batches, (uint64_t)kb_ * 2, (uint64_t)bg.o * kb_ * 2, BK, tile_n, 1))
    return cudaErrorInvalidValue;
  TcArgs a{};
  a.m_tiles = (bg.t + BM - 1) / BM;
  a.n_tiles = (bg.o + tile_n - 1) / tile_n;
  a.batches = bg.batches;
  a.kb_per_tap = bg.split_bf16 ? bg.c / BK : (int)((kb_ + BK - 1) / BK);
  a.split_cb = bg.split_bf16 ? bg.c / BK : 0;
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
    if (tile_n == 256 && tile_m == 256) {
      CUtensorMap tBp;
      if (!encode_3d(&tBp, dt, bg.b, bg.c, bg.o, bg.batches, (uint64_t)bg.c * 2, (uint64_t)bg.o * bg.c * 2, BK, 128,
                     1))
        return cudaErrorInvalidValue;
      TcArgs p = a;
      p.m_tiles = (bg.t + 255) / 256;
      if (dt == CONV_BF16)
        return launch_tiles<256, 0, __nv_bfloat16, __nv_bfloat16>(tA, tB, tBp, p, 256, sm_count, s, &tD16);
      return launch_tiles<256, 0, __half, __half>(tA, tB, tBp, p, 256, sm_count, s, &tD16);
    }
    if (dt == CONV_BF16)
      return tile_n == 256 ? launch_kernel<256, 0, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD16)
                           : launch_kernel<128, 0, __nv_bfloat16, __nv_bfloat16>(tA, tB, a, sm_count, s, &tD16);
    return tile_n == 256 ? launch_kernel<256, 0, __half, __half>(tA, tB, a, sm_count, s, &tD16)
                         : launch_kernel<128, 0, __half, __half>(tA, tB, a, sm_count, s, &tD16);
  }
  CUtensorMap tD;
  a.tma_store = encode_store_map(&tD, bg.d, CONV_F32, bg.o, bg.t, bg.batches) ? 1 : 0;
  if (bg.split_bf16) {
    if (tile_n != 96 && tile_n != 128) return cudaErrorInvalidValue;
    return tile_n == 96 ? launch_kernel<96, 3, __nv_bfloat16, float>(tA, tB, a, sm_count, s, &tD)
                        : launch_kernel<128, 3, __nv_bfloat16, float>(tA, tB, a, sm_count, s, &tD);
  }
  if (dt == CONV_BF16)
    return tile_n == 256 ? launch_kernel<256, 0, __nv_bfloat16, float>(tA, tB, a, sm_count, s, &tD)
                         : launch_kernel<128, 0, __nv_bfloat16, float>(tA, tB, a, sm_count, s, &tD);
  return tile_n == 256 ? launch_kernel<256, 0, __half, float>(tA, tB, a, sm_count, s, &tD)
                       : launch_kernel<128, 0, __half, float>(tA, tB, a, sm_count, s, &tD);
}

}  // namespace b200conv
