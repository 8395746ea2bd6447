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
#include "tc_ptx.cuh"
#include "wino_tile.cuh"

namespace b200conv {
namespace {

constexpr int FM = 6;                        // F(6x6, 3x3)
constexpr int FA2 = (FM + 2) * (FM + 2);     // 64 transform points
constexpr int FBM = 128;                     // tiles per block (GEMM rows)
constexpr int FBK = 16;                      // channels per k-slice
constexpr int FSTAGES = 4;                   // cp.async ring depth of a GEMM unit
constexpr int UNIT = 128;                    // threads of one GEMM unit (a warpgroup)
constexpr int XF = 128;                      // transform threads (a warpgroup)
constexpr int FTHREADS = 2 * UNIT + XF;
constexpr int REG_LAUNCH = 168, REG_GEMM = 192, REG_XFORM = 120;
static_assert(2 * UNIT * REG_GEMM + XF * REG_XFORM <= FTHREADS * REG_LAUNCH, "register split");
// Input staging of the transform warpgroup: TMA boxes of IC channels x IW
// columns x 8 rows of one image, the input patches of a strip of up to IS
// tiles of one tile row (padding comes from the tensor map's zero fill).
constexpr int IS = 6;
constexpr int IW = FM * IS + 2;
constexpr int IC = 32;
constexpr int IBOX = 8 * IW * IC;            // floats per staged box
constexpr int NIBUF = 2;                     // staged boxes in the ring (one in flight ahead of the current)

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
  int tma_in;                // the input is read through tmIn (else by per-thread loads)
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

// A strip of the input transform: `len` tiles from global tile t of one tile
// row, channel group cg.
struct Strip {
  long long t;
  int n, ty, tx, len, cg;
};
__device__ __forceinline__ Strip strip_at(long long t, long long t_end, int tiles_w, int per_img) {
  Strip st;
  st.t = t;
  st.n = (int)(t / per_img);
  const int r = (int)(t - (long long)st.n * per_img);
  st.ty = r / tiles_w;
  st.tx = r - st.ty * tiles_w;
  const long long left = t_end - t;
  st.len = min(IS, tiles_w - st.tx);
  if (left < st.len) st.len = (int)left;
  st.cg = 0;
  return st;
}

template <int BN>
__global__ void __launch_bounds__(FTHREADS, 1)
wino_fused_f32_kernel(const __grid_constant__ CUtensorMap tmIn, const FusedArgs p) {
  constexpr int TN = BN / 8;                 // columns per thread
  constexpr int A_PER = FBK * FBM / 4 / UNIT;
  constexpr int B_CHUNKS = FBK * BN / 4;
  constexpr int B_PER = (B_CHUNKS + UNIT - 1) / UNIT;
  static_assert(A_PER * UNIT * 4 == FBK * FBM, "A copies");
  // the dynamic region, aligned by hand to 128 bytes (TMA box destinations)
  extern __shared__ __align__(16) unsigned char fsm_raw[];
  float* fsm = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(fsm_raw) + 127) & ~uintptr_t(127));
  // vready[2], vfree[2], mready[2], mfree[2], input box full[NIBUF]
  __shared__ __align__(8) uint64_t bars[8 + NIBUF];
  __shared__ int abort_flag;
  __shared__ int role_ok[3];

  const int tid = threadIdx.x;
  const uint32_t b0 = smem_u32(bars);
  auto vready = [&](int b) { return b0 + 8u * b; };
  auto vfree = [&](int b) { return b0 + 8u * (2 + b); };
  auto mready = [&](int b) { return b0 + 8u * (4 + b); };
  auto mfree = [&](int b) { return b0 + 8u * (6 + b); };
  auto infull = [&](int b) { return b0 + 8u * (8 + b); };
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(vready(b), XF);
      mbar_init(vfree(b), 2 * UNIT);
      mbar_init(mready(b), 2 * UNIT);
      mbar_init(mfree(b), XF);
    }
    for (int b = 0; b < NIBUF; ++b) mbar_init(infull(b), 1);
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
    // B (U rows, contiguous in o): copy i moves k-row b_k[i] (FBK: none), columns b_col[i] .. + 3
    int b_k[B_PER], b_col[B_PER], b_off[B_PER];
    uint32_t b_dst[B_PER];
#pragma unroll
    for (int i = 0; i < B_PER; ++i) {
      const int q = lt + i * UNIT;
      const int k = q / (BN / 4), col = (q % (BN / 4)) * 4;
      b_k[i] = q < B_CHUNKS ? k : FBK;
      b_col[i] = col;
      b_off[i] = k * p.ldb + col;
      b_dst[i] = smem_u32(Bs) + (uint32_t)(k * BN + col) * 4u;
    }
    int sblk = 0;
    for (long long blk = blockIdx.x; blk < p.blocks; blk += gridDim.x, ++sblk) {
      const int buf = sblk & 1;
      const uint32_t ph = (uint32_t)(sblk >> 1) & 1u;
      if (lt == 0) {
        bool ok = mbar_wait_sleep(vready(buf), ph, &abort_flag, p.err, DEVERR_TIMEOUT_FUSED_GEMM);
        if (ok && sblk >= 2) ok = mbar_wait_sleep(mfree(buf), ph ^ 1u, &abort_flag, p.err, DEVERR_TIMEOUT_FUSED_GEMM);
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

      // The prefetch position (point, column block, k-slice), stepped per stage;
      // the per-thread copy offsets are fixed, only the bases move.
      int pf_xi = u / nob, pf_ob = u - (u / nob) * nob, pf_kt = 0;
      const float* a_base = V + (long long)a_row0 * C + a_chunk * 4;
      const long long a_step = 32LL * C;
      long long pf_aoff = (long long)pf_xi * FBM * C;
      const float* pf_b = p.u + (long long)pf_xi * C * p.ldb + pf_ob * BN;
      int b_bytes[B_PER];
      auto set_b_bytes = [&]() {
#pragma unroll
        for (int i = 0; i < B_PER; ++i) {
          const int oo = pf_ob * BN + b_col[i];
          b_bytes[i] = oo < O ? min(16, (O - oo) * 4) : 0;
        }
      };
      set_b_bytes();
      auto load_stage = [&](int stage) {
        const int c0 = pf_kt * FBK;
        const int cc = c0 + a_chunk * 4;
        const int cbytes = cc < C ? min(16, (C - cc) * 4) : 0;
        const float* asrc = a_base + pf_aoff + c0;
        const uint32_t adst = a_dst0 + (uint32_t)(stage * FBK * FBM) * 4u;
#pragma unroll
        for (int i = 0; i < A_PER; ++i) {
          const int bytes = (a_valid >> i) & 1 ? cbytes : 0;
          fcp16(adst + (uint32_t)(i * 32 * FBK) * 4u, bytes ? asrc + i * a_step : V, bytes);
        }
        const float* bsrc = pf_b + c0 * p.ldb;
        const uint32_t bstage = (uint32_t)(stage * FBK * BN) * 4u;
#pragma unroll
        for (int i = 0; i < B_PER; ++i) {
          if (b_k[i] < FBK) {
            const int bytes = c0 + b_k[i] < C ? b_bytes[i] : 0;
            fcp16(b_dst[i] + bstage, bytes ? bsrc + b_off[i] : p.u, bytes);
          }
        }
        if (++pf_kt == ktiles) {
          pf_kt = 0;
          pf_ob += 2;
          while (pf_ob >= nob) {
            pf_ob -= nob;
            ++pf_xi;
          }
          pf_aoff = (long long)pf_xi * FBM * C;
          pf_b = p.u + (long long)pf_xi * C * p.ldb + pf_ob * BN;
          if (nob > 1) set_b_bytes();
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
      // items outer, k-slices inner (the ring runs on across items)
      int step = 0;
      for (int it = 0; it < my_items; ++it) {
        for (int kt = 0; kt < ktiles; ++kt, ++step) {
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
        }
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
    float* ibuf = fsm + 2 * FSTAGES * FBK * (FBM + BN);   // two staged input boxes
    static_assert((2 * FSTAGES * FBK * (FBM + BN) * 4) % 128 == 0 && (IBOX * 4) % 128 == 0, "box alignment");
    static_assert(IW <= 256 && IC <= 256, "TMA box dimensions");
    uint32_t kin = 0;                                     // staged boxes so far (their barrier phases)
    const bool tma_in = p.tma_in && (smem_u32(ibuf) & 127u) == 0;
    if (p.tma_in && !tma_in && xt == 0) atomicCAS(p.err, 0, DEVERR_FUSED_SMEM_ALIGN);
    const long long nmy = (long long)blockIdx.x < p.blocks ? (p.blocks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    for (long long s = 0; s <= nmy; ++s) {
      if (s < nmy) {
        // input transform of this CTA's block s into V buffer s % 2
        const int buf = (int)(s & 1);
        if (s >= 2) {
          if (xt == 0)
            role_ok[2] = mbar_wait_sleep(vfree(buf), (uint32_t)((s - 2) >> 1) & 1u, &abort_flag, p.err,
                                   DEVERR_TIMEOUT_FUSED_XFORM) ? 1 : 0;
          named_sync(3, XF);
          if (!role_ok[2]) break;
        }
        WinoInArgs ai = p.ai;
        ai.n0 = 0;
        ai.t_base = ((long long)blockIdx.x + s * gridDim.x) * FBM;
        ai.t_count = p.tiles - ai.t_base < FBM ? p.tiles - ai.t_base : FBM;
        ai.t_stride = FBM;
        if (tma_in) {
          // strips x channel groups through a ring of NIBUF staged boxes, one thread
          // issuing up to NIBUF ahead while the warpgroup transforms the current
          // box (lane = channel).  Box k sits in buffer k % NIBUF, the (k / NIBUF)-th
          // use of that buffer's barrier.
          const long long t_end = ai.t_base + ai.t_count;
          const int per_img = ai.tiles_h * ai.tiles_w;
          const int icg = (C + IC - 1) / IC;
          float* vb = vbuf(buf);
          auto next = [&](Strip st) {
            if (++st.cg < icg) return st;
            return strip_at(st.t + st.len, t_end, ai.tiles_w, per_img);
          };
          Strip ahead = strip_at(ai.t_base, t_end, ai.tiles_w, per_img);
          uint32_t kissue = kin;
          auto issue_more = [&]() {
            while (ahead.t < t_end && kissue < kin + NIBUF) {
              if (xt == 0) {
                const int b = (int)(kissue % NIBUF);
                mbar_expect_tx(infull(b), IBOX * 4);
                tma_load_4d(smem_u32(ibuf + b * IBOX), &tmIn, infull(b), ahead.cg * IC, ahead.tx * FM - ai.pw,
                            ahead.ty * FM - ai.ph, ahead.n);
              }
              ahead = next(ahead);
              ++kissue;
            }
          };
          issue_more();
          Strip cur = strip_at(ai.t_base, t_end, ai.tiles_w, per_img);
          bool fail = false;
          while (true) {
            const Strip nx = next(cur);
            const bool more = nx.t < t_end;
            if (!mbar_wait_sleep(infull((int)(kin % NIBUF)), (kin / NIBUF) & 1u, &abort_flag, p.err,
                                 DEVERR_TIMEOUT_FUSED_XFORM))
              fail = true;
            const float* box = ibuf + (kin % NIBUF) * IBOX;
            const int c = cur.cg * IC + lane;
            if (!fail && c < C) {
              for (int j = wx; j < cur.len; j += XF / 32) {
                // columns: t = B^T d, then rows: V = t B (the order of the shared transform body)
                const float* pt = box + j * FM * IC + lane;
                float tt[8][8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                  float col[8], res[8];
#pragma unroll
                  for (int i = 0; i < 8; ++i) col[i] = pt[(i * IW + jj) * IC];
                  Wino<FM>::bt(col, res);
#pragma unroll
                  for (int i = 0; i < 8; ++i) tt[i][jj] = res[i];
                }
                float* vp = vb + (cur.t - ai.t_base + j) * C + c;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  float res[8];
                  Wino<FM>::bt(tt[i], res);
#pragma unroll
                  for (int jj = 0; jj < 8; ++jj) vp[(long long)(i * 8 + jj) * FBM * C] = res[jj];
                }
              }
            }
            named_sync(3, XF);                   // box kin's buffer is free again
            ++kin;
            if (abort_flag || !more) break;
            issue_more();
            cur = nx;
          }
          if (abort_flag) {
            // leave no box in flight into this CTA's shared memory (bounded waits)
            if (xt == 0) {
              volatile int never = 0;
              for (uint32_t k = kin; k < kissue; ++k)
                mbar_wait_sleep(infull((int)(k % NIBUF)), (k / NIBUF) & 1u, &never, p.err, 0, 100000000ull);
            }
            break;
          }
        } else {
          const int cgroups = (C + ibx - 1) / ibx;
          const long long nb = ((ai.t_count + iby - 1) / iby) * cgroups;
          for (long long bid = 0; bid < nb; ++bid)
            wino_input_block<FM, float, float, int>(p.in, ai, vbuf(buf), bid, xt % ibx, xt / ibx, ibx, iby);
        }
        mbar_arrive(vready(buf));                // this thread's V stores are done
      }
      if (s >= 1) {
        // output transform of block s - 1 from M buffer (s - 1) % 2
        const long long sp = s - 1;
        const int buf = (int)(sp & 1);
        if (xt == 0)
          role_ok[2] = mbar_wait_sleep(mready(buf), (uint32_t)(sp >> 1) & 1u, &abort_flag, p.err,
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
cudaError_t launch_bn(const CUtensorMap& tm, const FusedArgs& p, int grid, cudaStream_t s) {
  const int smem = (2 * FSTAGES * FBK * (FBM + BN) + NIBUF * IBOX) * (int)sizeof(float) + 128;
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
  wino_fused_f32_kernel<BN><<<grid, FTHREADS, smem, s>>>(tm, p);
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
  // The input as a 4D (C, W, H, N) map whose boxes are the staged strips; an
  // input that is not 16-byte aligned is read by per-thread loads instead.
  CUtensorMap tm;
  memset(&tm, 0, sizeof(tm));
  p.tma_in = 0;
  if (driver_fns() && (reinterpret_cast<uintptr_t>(in) & 15) == 0 && g.in_img_stride % 4 == 0) {
    cuuint64_t dims[4] = {(cuuint64_t)g.c, (cuuint64_t)g.w, (cuuint64_t)g.h, (cuuint64_t)g.n};
    cuuint64_t strides[3] = {(cuuint64_t)g.c * 4, (cuuint64_t)g.w * g.c * 4, (cuuint64_t)g.in_img_stride * 4};
    cuuint32_t box[4] = {IC, IW, 8, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    p.tma_in = g_encode_tiled(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(in), dims, strides, box,
                              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  const int bn = wino_gemm_f32_tile_n(g.o);
  return bn == 64 ? launch_bn<64>(tm, p, grid, s)
                  : bn == 96 ? launch_bn<96>(tm, p, grid, s) : launch_bn<128>(tm, p, grid, s);
}

}  // namespace b200conv
