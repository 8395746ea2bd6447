// wino_tile.cuh -- the per-(tile, channel) bodies of the Winograd
// F(m x m, 3 x 3) input and output transforms, shared by the transform
// kernels and by the persistent fp32 Winograd kernel.
//
// Every thread owns one (tile, channel) pair and every tile is transformed
// independently, so a tile's result does not depend on which launch or block
// transformed it.
#pragma once

#include <cuda_runtime.h>

#include <type_traits>

#include "common.cuh"
#include "wino_1d.cuh"

namespace b200conv {
namespace {

// ---------------------------------------------------------------------------
// Input transform: one thread per (tile, channel); threadIdx.x runs over
// channels so loads and stores are coalesced.
// ---------------------------------------------------------------------------
struct WinoInArgs {
  int h, w, c, ph, pw, tiles_h, tiles_w;
  long long in_img_stride;
  int n0;                 // first image of this batch tile
  long long t_base;       // first tile of this call, counted from image n0's first tile
  long long t_count;      // tiles in this call (V rows 0 .. t_count-1)
  long long t_stride;     // row count of V's planes (the workspace's tile capacity)
};

// Idx is the type of the offsets inside one image and one V plane set: int
// when the host has checked that they fit (fewer address instructions per
// element), long long otherwise.  Tiles wholly inside the image skip the
// bounds tests.
// The body of one input-transform block: block `bid` of a 1D grid, thread
// (tx, ty) of a bx x by block.
// An fp32 value as three bf16 parts whose sum is the value (each part the
// round-to-nearest bf16 of what the parts before it leave; the residuals are
// exact in fp32): the operand split of the split-bf16 fp32 GEMM.
__device__ __forceinline__ void split_bf16x3(float x, __nv_bfloat16& p0, __nv_bfloat16& p1, __nv_bfloat16& p2) {
  p0 = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(p0);
  p1 = __float2bfloat16_rn(r1);
  p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
}

// SPLIT = 1: Tst is bf16 and every V row holds the three bf16 parts of the fp32
// values side by side ([t][3C]: part 0 at c, part 1 at C + c, part 2 at 2C + c).
template <int M, typename Tin, typename Tst, typename Idx, int SPLIT = 0>
__device__ __forceinline__ void wino_input_block(const Tin* __restrict__ in, const WinoInArgs& a,
                                                 Tst* __restrict__ v, long long bid, int lx, int ly, int bx,
                                                 int by) {
  constexpr int A = Wino<M>::A;
  // channel group fastest across blocks, so one tile's V rows are written by
  // blocks that run together
  const int cgroups = (a.c + bx - 1) / bx;
  const int cg = (int)(bid % cgroups);
  const long long tg = bid / cgroups;
  const int c = cg * bx + lx;
  const long long t = tg * by + ly;
  if (c >= a.c || t >= a.t_count) return;
  const int per_img = a.tiles_h * a.tiles_w;
  const long long tglob = a.t_base + t;
  const int nl = (int)(tglob / per_img);
  const int r = (int)(tglob - (long long)nl * per_img);
  const int ty = r / a.tiles_w, tx = r - (r / a.tiles_w) * a.tiles_w;
  const int y0 = ty * M - a.ph, x0 = tx * M - a.pw;
  const Tin* base = in + (long long)(a.n0 + nl) * a.in_img_stride + c;
  const Idx cs = a.c, wc = (Idx)a.w * a.c;

  float d[A][A];
  if (y0 >= 0 && x0 >= 0 && y0 + A <= a.h && x0 + A <= a.w) {
    const Tin* p = base + ((Idx)y0 * wc + (Idx)x0 * cs);
#pragma unroll
    for (int i = 0; i < A; ++i)
#pragma unroll
      for (int j = 0; j < A; ++j) d[i][j] = Store<Tin>::to_f32(p[(Idx)i * wc + (Idx)j * cs]);
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
      for (int j = 0; j < A; ++j)
        d[i][j] = (yok && ((xm >> j) & 1u)) ? Store<Tin>::to_f32(base[ro + (Idx)j * cs]) : 0.0f;
    }
  }
  // columns: t = B^T d, then rows: V = t B
  float tt[A][A];
#pragma unroll
  for (int j = 0; j < A; ++j) {
    float col[A], res[A];
#pragma unroll
    for (int i = 0; i < A; ++i) col[i] = d[i][j];
    Wino<M>::bt(col, res);
#pragma unroll
    for (int i = 0; i < A; ++i) tt[i][j] = res[i];
  }
  // V offsets: Idx, except in the split form, whose three-part rows make the
  // plane set 3x larger; there they are 64-bit so that Idx (int for every
  // image below 2^31 elements) bounds only the input offsets
  using VIdx = typename std::conditional<SPLIT != 0, long long, Idx>::type;
  const VIdx rowc = SPLIT ? (VIdx)3 * a.c : (VIdx)a.c;
  const VIdx plane = (VIdx)(a.t_stride * rowc);
  Tst* vp = v + t * rowc + c;
#pragma unroll
  for (int i = 0; i < A; ++i) {
    float res[A];
    Wino<M>::bt(tt[i], res);
#pragma unroll
    for (int j = 0; j < A; ++j) {
      if constexpr (SPLIT) {
        __nv_bfloat16 p0, p1, p2;
        split_bf16x3(res[j], p0, p1, p2);
        Tst* q = vp + (VIdx)(i * A + j) * plane;
        q[0] = p0;
        q[a.c] = p1;
        q[2 * a.c] = p2;
      } else {
        vp[(VIdx)(i * A + j) * plane] = Store<Tst>::from_f32(res[j]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Output transform: one thread per (tile, output channel).
// ---------------------------------------------------------------------------
struct WinoOutArgs {
  int oh, ow, o, tiles_h, tiles_w;
  long long out_img_stride;
  int n0;
  long long t_base;       // first tile of this call, counted from image n0's first tile
  long long t_count, t_stride;
  int accumulate;
};

// TM: the element type of M (fp32, or the 16-bit operand type of the
// tensor-core path).
// The body of one output-transform block: block (bidx, bidy) of the grid,
// thread (tx, ty) of a bx x by block.
template <int M, typename TM, typename Tout, typename Idx>
__device__ __forceinline__ void wino_output_block(const TM* __restrict__ mb, const WinoOutArgs& a,
                                                  Tout* __restrict__ out, long long bidx, int bidy, int lx, int ly,
                                                  int bx, int by) {
  constexpr int A = Wino<M>::A;
  const int o = bidy * bx + lx;
  const long long t = bidx * by + ly;
  if (o >= a.o || t >= a.t_count) return;
  const int per_img = a.tiles_h * a.tiles_w;
  const long long tglob = a.t_base + t;
  const int nl = (int)(tglob / per_img);
  const int r = (int)(tglob - (long long)nl * per_img);
  const int ty = r / a.tiles_w, tx = r - (r / a.tiles_w) * a.tiles_w;

  const Idx plane = (Idx)(a.t_stride * a.o);
  const TM* mp = mb + t * a.o + o;
  float x[A][A];
#pragma unroll
  for (int i = 0; i < A; ++i)
#pragma unroll
    for (int j = 0; j < A; ++j) x[i][j] = Store<TM>::to_f32(mp[(Idx)(i * A + j) * plane]);
  // columns: t = A^T x (M x A), then rows: y = t A (M x M)
  float tt[M][A];
#pragma unroll
  for (int j = 0; j < A; ++j) {
    float col[A], res[M];
#pragma unroll
    for (int i = 0; i < A; ++i) col[i] = x[i][j];
    Wino<M>::at(col, res);
#pragma unroll
    for (int i = 0; i < M; ++i) tt[i][j] = res[i];
  }
  Tout* op = out + (long long)(a.n0 + nl) * a.out_img_stride + o;
  const Idx os = a.o, wo = (Idx)a.ow * a.o;
  const bool whole = ty * M + M <= a.oh && tx * M + M <= a.ow;
#pragma unroll
  for (int i = 0; i < M; ++i) {
    float res[M];
    Wino<M>::at(tt[i], res);
    const int y = ty * M + i;
    if (!whole && y >= a.oh) continue;
    Tout* rp = op + ((Idx)y * wo + (Idx)(tx * M) * os);
    if (a.accumulate) {
      // the row's old values first, so the loads are not ordered behind the stores
      float old[M];
#pragma unroll
      for (int j = 0; j < M; ++j)
        old[j] = (whole || tx * M + j < a.ow) ? Store<Tout>::to_f32(rp[(Idx)j * os]) : 0.0f;
#pragma unroll
      for (int j = 0; j < M; ++j) res[j] = old[j] + Store<Tout>::to_f32(Store<Tout>::from_f32(res[j]));
    }
#pragma unroll
    for (int j = 0; j < M; ++j)
      if (whole || tx * M + j < a.ow) rp[(Idx)j * os] = Store<Tout>::from_f32(res[j]);
  }
}

}  // namespace
}  // namespace b200conv
