// wino_fused_f32.cu -- the fp32 Winograd F(6x6,3x3) conv as one persistent
// kernel that overlaps the transforms with the batched GEMM.
//
// The Winograd path of "Bound winograd conv2d working set by tiling the batch"
// (Problem, Fix) runs as three launches: the input transform and the output
// transform are HBM-bound, the FFMA GEMM between them is ALU-bound, and each
// waits for the one before.  Here one CTA per SM runs all three on its own
// blocks of 128 tiles:
//   - two GEMM units of four warps compute the 64 point GEMMs of block j,
//       M[xi][t][o] = sum_c V[xi][t][c] * U[xi][c][o]     (xi < 64, t < 128)
//     each unit taking every other (point, column block) item;
//   - a transform warpgroup meanwhile writes V of block j+1 (input transform)
//     and turns M of block j-1 into output pixels (output transform).
// The roles are warpgroups (384 threads): launched at 168 registers a thread,
// the GEMM warpgroups raise theirs to 200 and the transform warpgroup lowers
// its own to 104 (setmaxnreg), 2 x 128 x 200 + 128 x 104 = 384 x 168.
// V and M of a block live in two per-CTA scratch buffers each (global memory,
// 2 x 64 x 128 x (C + O) floats per CTA).  The roles hand the buffers over
// through four mbarriers (V ready, V free, M ready, M free) with bounded waits,
// so no CTA waits on another and the grid needs no co-residency.
//
// Every output is computed by the same chain of operations as in the
// three-launch path: the transform bodies are shared (wino_tile.cuh) and every
// GEMM output is an fmaf chain over c ascending from 0.0f inside one thread.
// Results therefore equal that path bit for bit, for any grid size.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "mbar.cuh"
#include "wino_tile.cuh"

namespace b200conv {
namespace {

constexpr int FM = 6;                        // F(6x6, 3x3)
constexpr int FA2 = (FM + 2) * (FM + 2);     // 64 transform points
constexpr int FBM = 128;                     // tiles per block (GEMM rows)
constexpr int FBK = 16;                      // channels per k-slice
constexpr int FSTAGES = 3;                   // cp.async ring depth of a GEMM unit
constexpr int UNIT = 128;                    // threads of one GEMM unit (a warpgroup)
constexpr int XF = 128;                      // transform threads (a warpgroup)
constexpr int FTHREADS = 2 * UNIT + XF;
constexpr int REG_LAUNCH = 168, REG_GEMM = 200, REG_XFORM = 104;
static_assert(2 * UNIT * REG_GEMM + XF * REG_XFORM <= FTHREADS * REG_LAUNCH, "register split");

struct FusedArgs {
  const float* in;
  const float* u;            // transformed filter [64][C][ldb]
  float* out;
  float* scratch;            // per CTA: V[2][64][128][C], then M[2][64][128][O]
  long long cta_floats;      // floats of one CTA's scratch
  long long tiles;           // N * tiles_h * tiles_w
  long long blocks;          // ceil(tiles / 128)
  int ldb;                   // row stride of U (O rounded up to 4)
  WinoInArgs ai;             // t_base / t_count / t_stride are set per block
  WinoOutArgs ao;
  int* err;
};

__device__ __forceinline__ void fcp16(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void fcp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void fcp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// Named barriers: 1 + u for GEMM unit u, 3 for the transform warpgroup.
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int BN>
__global__ void __launch_bounds__(FTHREADS, 1)
wino_fused_f32_kernel(const FusedArgs p) {
  constexpr int TN = BN / 8;                 // columns per thread
  constexpr int A_PER = FBK * FBM / 4 / UNIT;
  constexpr int B_CHUNKS = FBK * BN / 4;
  constexpr int B_PER = (B_CHUNKS + UNIT - 1) / UNIT;
  static_assert(A_PER * UNIT * 4 == FBK * FBM, "A copies");
  extern __shared__ __align__(16) float fsm[];
  // vready[2], vfree[2], mready[2], mfree[2]
  __shared__ __align__(8) uint64_t bars[8];
  __shared__ int abort_flag;
  __shared__ int role_ok[3];

  const int tid = threadIdx.x;
  const uint32_t b0 = smem_u32(bars);
  auto vready = [&](int b) { return b0 + 8u * b; };
  auto vfree = [&](int b) { return b0 + 8u * (2 + b); };
  auto mready = [&](int b) { return b0 + 8u * (4 + b); };
  auto mfree = [&](int b) { return b0 + 8u * (6 + b); };
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(vready(b), XF);
      mbar_init(vfree(b), 2 * UNIT);
      mbar_init(mready(b), 2 * UNIT);
      mbar_init(mfree(b), XF);
    }
    abort_flag = 0;
  }
  __syncthreads();

  const int C = p.ai.c, O = p.ao.o;
  const long long vfl = (long long)FA2 * FBM * C, mfl = (long long)FA2 * FBM * O;
  float* sc = p.scratch + (long long)blockIdx.x * p.cta_floats;
  auto vbuf = [&](int b) { return sc + (b ? vfl : 0); };
  auto mbuf = [&](int b) { return sc + 2 * vfl + (b ? mfl : 0); };

  if (tid < 2 * UNIT) {
    // ------------------------------ GEMM unit ------------------------------
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_GEMM));
    const int u = tid / UNIT;
    const int lt = tid % UNIT;
    float* As = fsm + u * FSTAGES * FBK * (FBM + BN);     // [FSTAGES][FBK][FBM]
    float* Bs = As + FSTAGES * FBK * FBM;                 // [FSTAGES][FBK][BN]
    const int tc = lt & 7, tr = lt >> 3;                  // 8 thread-columns x 16 thread-rows
    const int nob = (O + BN - 1) / BN;
    const int items = FA2 * nob;                          // (point, column block) pairs
    const int my_items = (items - u + 1) / 2;             // this unit takes items u, u + 2, ...
    const int ktiles = (C + FBK - 1) / FBK;
    const int steps = my_items * ktiles;
    // A (V rows, one tile each, contiguous in c): copy i moves row (lt >> 2) + 32 i,
    // 16-byte chunk lt & 3, XOR-swizzled by (row / 4) % 4 in shared memory
    const int a_chunk = lt & 3, a_row0 = lt >> 2;
    const uint32_t a_dst0 = smem_u32(As) + (uint32_t)(a_row0 * FBK + ((a_chunk ^ ((a_row0 >> 2) & 3)) * 4)) * 4u;
    int sblk = 0;
    for (long long blk = blockIdx.x; blk < p.blocks; blk += gridDim.x, ++sblk) {
      const int buf = sblk & 1;
      const uint32_t ph = (uint32_t)(sblk >> 1) & 1u;
      if (lt == 0) {
        bool ok = mbar_wait_inl(vready(buf), ph, &abort_flag, p.err, DEVERR_TIMEOUT_FUSED_GEMM);
        if (ok && sblk >= 2) ok = mbar_wait_inl(mfree(buf), ph ^ 1u, &abort_flag, p.err, DEVERR_TIMEOUT_FUSED_GEMM);
        role_ok[u] = ok ? 1 : 0;
      }
      named_sync(1 + u, UNIT);
      if (!role_ok[u]) break;
      (void)mbar_try(vready(buf), ph);           // every thread's own acquire of the completed phase
      const long long t0 = blk * FBM;
      const int tcount = (int)(p.tiles - t0 < FBM ? p.tiles - t0 : FBM);
      const float* __restrict__ V = vbuf(buf);
      float* __restrict__ Mo = mbuf(buf);
      unsigned a_valid = 0;
#pragma unroll
      for (int i = 0; i < A_PER; ++i)
        if (a_row0 + 32 * i < tcount) a_valid |= 1u << i;

      // the prefetch position (point, column block, k-slice), stepped per stage
      int pf_xi = u / nob, pf_ob = u - (u / nob) * nob, pf_kt = 0;
      auto load_stage = [&](int stage) {
        const int xi = pf_xi, ob = pf_ob;
        const int c0 = pf_kt * FBK;
        if (++pf_kt == ktiles) {
          pf_kt = 0;
          pf_ob += 2;
          while (pf_ob >= nob) {
            pf_ob -= nob;
            ++pf_xi;
          }
        }
        const int cc = c0 + a_chunk * 4;
        const int cbytes = cc < C ? min(16, (C - cc) * 4) : 0;
        const float* asrc = V + (long long)xi * FBM * C + (long long)a_row0 * C + cc;
        const uint32_t adst = a_dst0 + (uint32_t)(stage * FBK * FBM) * 4u;
#pragma unroll
        for (int i = 0; i < A_PER; ++i) {
          const int bytes = (a_valid >> i) & 1 ? cbytes : 0;
          fcp16(adst + (uint32_t)(i * 32 * FBK) * 4u, bytes ? asrc + (long long)i * 32 * C : V, bytes);
        }
        const float* bbase = p.u + ((long long)xi * C + c0) * p.ldb;
        const uint32_t bdst = smem_u32(Bs) + (uint32_t)(stage * FBK * BN) * 4u;
#pragma unroll
        for (int i = 0; i < B_PER; ++i) {
          const int q = lt + i * UNIT;
          if (q < B_CHUNKS) {
            const int k = q / (BN / 4), col = (q % (BN / 4)) * 4;
            const int oo = ob * BN + col;
            const int bytes = (c0 + k < C && oo < O) ? min(16, (O - oo) * 4) : 0;
            fcp16(bdst + (uint32_t)(k * BN + col) * 4u, bytes ? bbase + (long long)k * p.ldb + oo : p.u, bytes);
          }
        }
      };

      float2 acc[8][TN / 2];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < TN / 2; ++j) acc[i][j] = make_float2(0.0f, 0.0f);

#pragma unroll
      for (int s = 0; s < FSTAGES - 1; ++s) {
        if (s < steps) load_stage(s);
        fcp_commit();
      }
      int kt = 0, it = 0;
      for (int step = 0; step < steps; ++step) {
        fcp_wait<FSTAGES - 2>();
        named_sync(1 + u, UNIT);
        const int pre = step + FSTAGES - 1;
        if (pre < steps) load_stage(pre % FSTAGES);
        fcp_commit();
        const float* as = As + (step % FSTAGES) * FBK * FBM;
        const float* bs = Bs + (step % FSTAGES) * FBK * BN;
        // one 128-bit load per A row covers 4 k-steps (rows are contiguous in c)
#pragma unroll
        for (int k4 = 0; k4 < FBK / 4; ++k4) {
          float4 a4[8];
          const int off = (k4 ^ (tr & 3)) << 2;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            a4[i] = *reinterpret_cast<const float4*>(as + (tr * 4 + i) * FBK + off);
            a4[4 + i] = *reinterpret_cast<const float4*>(as + (64 + tr * 4 + i) * FBK + off);
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
        if (++kt == ktiles) {
          // item done: its 128 x BN block of M_xi, then fresh accumulators
          const int item = u + 2 * it;
          const int xi = item / nob, ob = item - (item / nob) * nob;
          float* mp = Mo + (long long)xi * FBM * O;
          const bool vec = (O & 3) == 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int t = i < 4 ? tr * 4 + i : 64 + tr * 4 + i - 4;
            if (t < tcount) {
              float* drow = mp + (long long)t * O;
#pragma unroll
              for (int j = 0; j < TN / 4; ++j) {
                const int o = ob * BN + 32 * j + tc * 4;
                const float4 v4 =
                    make_float4(acc[i][2 * j].x, acc[i][2 * j].y, acc[i][2 * j + 1].x, acc[i][2 * j + 1].y);
                if (vec && o + 3 < O) {
                  *reinterpret_cast<float4*>(drow + o) = v4;
                } else {
                  const float ve[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                  for (int e = 0; e < 4; ++e)
                    if (o + e < O) drow[o + e] = ve[e];
                }
              }
            }
#pragma unroll
            for (int j = 0; j < TN / 2; ++j) acc[i][j] = make_float2(0.0f, 0.0f);
          }
          kt = 0;
          ++it;
        }
      }
      fcp_wait<0>();
      named_sync(1 + u, UNIT);                   // the ring is free for the next block's prologue
      mbar_arrive(mready(buf));                  // this thread's M stores are done
      mbar_arrive(vfree(buf));                   // and its V reads
    }
  } else {
    // -------------------------- transform warpgroup --------------------------
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_XFORM));
    const int xt = tid - 2 * UNIT;
    const int lane = xt & 31, wx = xt >> 5;
    // input transform: blocks of ibx channels x (XF / ibx) tiles
    const int ibx = C % 64 == 0 ? 64 : 32, iby = XF / ibx;
    const long long nmy = (long long)blockIdx.x < p.blocks ? (p.blocks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    for (long long s = 0; s <= nmy; ++s) {
      if (s < nmy) {
        // input transform of this CTA's block s into V buffer s % 2
        const int buf = (int)(s & 1);
        if (s >= 2) {
          if (xt == 0)
            role_ok[2] = mbar_wait_inl(vfree(buf), (uint32_t)((s - 2) >> 1) & 1u, &abort_flag, p.err,
                                   DEVERR_TIMEOUT_FUSED_XFORM) ? 1 : 0;
          named_sync(3, XF);
          if (!role_ok[2]) break;
        }
        WinoInArgs ai = p.ai;
        ai.n0 = 0;
        ai.t_base = ((long long)blockIdx.x + s * gridDim.x) * FBM;
        ai.t_count = p.tiles - ai.t_base < FBM ? p.tiles - ai.t_base : FBM;
        ai.t_stride = FBM;
        const int cgroups = (C + ibx - 1) / ibx;
        const long long nb = ((ai.t_count + iby - 1) / iby) * cgroups;
        for (long long bid = 0; bid < nb; ++bid)
          wino_input_block<FM, float, float, int>(p.in, ai, vbuf(buf), bid, xt % ibx, xt / ibx, ibx, iby);
        mbar_arrive(vready(buf));                // this thread's V stores are done
      }
      if (s >= 1) {
        // output transform of block s - 1 from M buffer (s - 1) % 2
        const long long sp = s - 1;
        const int buf = (int)(sp & 1);
        if (xt == 0)
          role_ok[2] = mbar_wait_inl(mready(buf), (uint32_t)(sp >> 1) & 1u, &abort_flag, p.err,
                                 DEVERR_TIMEOUT_FUSED_XFORM) ? 1 : 0;
        named_sync(3, XF);
        if (!role_ok[2]) break;
        (void)mbar_try(mready(buf), (uint32_t)(sp >> 1) & 1u);
        WinoOutArgs ao = p.ao;
        ao.n0 = 0;
        ao.t_base = ((long long)blockIdx.x + sp * gridDim.x) * FBM;
        ao.t_count = p.tiles - ao.t_base < FBM ? p.tiles - ao.t_base : FBM;
        ao.t_stride = FBM;
        const int ogroups = (O + 31) / 32;
        const long long tquads = (ao.t_count + 3) / 4;
        for (long long bx = 0; bx < tquads; ++bx)
          for (int by = 0; by < ogroups; ++by)
            wino_output_block<FM, float, float, int>(mbuf(buf), ao, p.out, bx, by, lane, wx, 32, 4);
        mbar_arrive(mfree(buf));                 // this thread's M reads are done
      }
    }
  }
}

template <int BN>
cudaError_t launch_bn(const FusedArgs& p, int grid, cudaStream_t s) {
  const int smem = 2 * FSTAGES * FBK * (FBM + BN) * (int)sizeof(float);
  static int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    // The warpgroups' setmaxnreg split draws on the registers the block is
    // launched with; with fewer than REG_LAUNCH a thread the raise would never
    // be granted, so such a build is refused here rather than launched.
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, wino_fused_f32_kernel<BN>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < REG_LAUNCH) return cudaErrorInvalidDeviceFunction;
    e = cudaFuncSetAttribute(wino_fused_f32_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured_dev = dev;
  }
  wino_fused_f32_kernel<BN><<<grid, FTHREADS, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t wino_fused_f32_cta_bytes(int c, int o) { return (size_t)2 * FA2 * FBM * ((size_t)c + o) * sizeof(float); }

long long wino_fused_f32_blocks(long long tiles) { return (tiles + FBM - 1) / FBM; }

bool wino_fused_f32_shape_ok(const Geom& g) {
  if (g.kh != 3 || g.kw != 3 || g.sh != 1 || g.sw != 1 || g.dh != 1 || g.dw != 1) return false;
  if (g.c % 4 != 0 || g.c <= 0 || g.o <= 0) return false;
  // 32-bit offsets inside one image (with a row of slack for the padding) and one block's planes
  if (g.in_img_stride + 4LL * g.w * g.c >= (1LL << 31) || g.out_img_stride >= (1LL << 31)) return false;
  if ((long long)FA2 * FBM * g.c >= (1LL << 31) || (long long)FA2 * FBM * g.o >= (1LL << 31)) return false;
  // a block's GEMM stays far inside the 2 s bound of the transform warps' wait
  if ((long long)g.c * g.o > (1LL << 22)) return false;
  return true;
}

cudaError_t launch_wino_fused_f32(const float* in, const Geom& g, const float* u, long long ldb, float* out,
                                  float* scratch, int grid, bool accumulate, int* err_word, cudaStream_t s) {
  if (!wino_fused_f32_shape_ok(g) || (ldb & 3) || (reinterpret_cast<uintptr_t>(u) & 15) ||
      (reinterpret_cast<uintptr_t>(scratch) & 15))
    return cudaErrorInvalidValue;
  const int m = FM;
  FusedArgs p{};
  p.in = in;
  p.u = u;
  p.out = out;
  p.scratch = scratch;
  p.cta_floats = (long long)(wino_fused_f32_cta_bytes(g.c, g.o) / sizeof(float));
  const int th = (g.oh + m - 1) / m, tw = (g.ow + m - 1) / m;
  p.tiles = (long long)g.n * th * tw;
  p.blocks = wino_fused_f32_blocks(p.tiles);
  p.ldb = (int)ldb;
  p.ai.h = g.h; p.ai.w = g.w; p.ai.c = g.c; p.ai.ph = g.ph; p.ai.pw = g.pw;
  p.ai.tiles_h = th; p.ai.tiles_w = tw;
  p.ai.in_img_stride = g.in_img_stride;
  p.ao.oh = g.oh; p.ao.ow = g.ow; p.ao.o = g.o;
  p.ao.tiles_h = th; p.ao.tiles_w = tw;
  p.ao.out_img_stride = g.out_img_stride;
  p.ao.accumulate = accumulate ? 1 : 0;
  p.err = err_word;
  if (p.tiles == 0) return cudaSuccess;
  if (grid <= 0) return cudaErrorInvalidValue;
  if (grid > p.blocks) grid = (int)p.blocks;
  const int bn = wino_gemm_f32_tile_n(g.o);
  return bn == 64 ? launch_bn<64>(p, grid, s) : bn == 96 ? launch_bn<96>(p, grid, s) : launch_bn<128>(p, grid, s);
}

}  // namespace b200conv
