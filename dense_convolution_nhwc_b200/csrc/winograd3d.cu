// winograd3d.cu -- native 3D Winograd F(m x m x m, 3 x 3 x 3) transforms.
//
// The native 3D Winograd that "Decompose small kernel-depth 3D convs into 2D
// convs" (Open questions, item 3) leaves open: the 2D algorithm of "Bound
// winograd conv2d working set by tiling the batch" with the 1D transforms
// applied along depth, height and width.  With alpha = m + 2, a tile is an
// m x m x m block of outputs and its alpha x alpha x alpha input patch; with
// xi = (xi_z * alpha + xi_y) * alpha + xi_x,
//   U[xi][.][.] = (G (x) G (x) G) g_oc                  filter transform
//   V[xi][t][c] = (B^T (x) B^T (x) B^T) d_tc            input transform
//   M[xi][t][o] = sum_c V[xi][t][c] * U[xi][.][.]       batched GEMM (elsewhere)
//   y_to        = (A^T (x) A^T (x) A^T) M[.][t][o]       output transform (cropped)
// where (x) applies a 1D transform along one axis of the cube.  The input
// patch of tile (n, tz, ty, tx) starts at (tz*m - pd, ty*m - ph, tx*m - pw)
// and reads zero outside the volume.  Transform arithmetic is fp32; U and V
// are stored in the GEMM's operand dtype, M is fp32.
//
// Tiles are numbered unit-major: a unit is one (image, depth-tile) slab of
// tiles_h * tiles_w tiles, and a batch tile of the workspace is a run of
// consecutive units.  Every tile is transformed on its own, so the result
// does not depend on how the units are grouped (tiling stays bit-identical).
//
// The input and output kernels give one block to a (tile, 32-channel group):
// warp j owns the x = j slice of the cube for the depth and height transforms,
// the slices meet in shared memory, and each warp then runs the width
// transform of alpha (z, y) lines.  Lanes run over channels, so every global
// access of a warp is one contiguous row segment.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "wino_1d.cuh"

namespace b200conv {
namespace {

// ---------------------------------------------------------------------------
// Filter transform: one thread per (o, c).  CMAJOR stores U[xi][c][o_pad]
// (the FFMA GEMM's B), else U[xi][o][c] (the tcgen05 GEMM's K-major B).
// ---------------------------------------------------------------------------
template <int M, typename Tin, typename Tst, bool CMAJOR>
__global__ void __launch_bounds__(256)
wino3d_filter_kernel(const Tin* __restrict__ w, int O, int C, long long o_pad, Tst* __restrict__ u) {
  constexpr int A = Wino<M>::A;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)O * C) return;
  int o, c;
  if (CMAJOR) {
    c = (int)(idx / O);
    o = (int)(idx - (long long)c * O);      // o fastest: coalesced stores
  } else {
    o = (int)(idx / C);
    c = (int)(idx - (long long)o * C);
  }
  const Tin* wp = w + (long long)o * 27 * C + c;
  // along x: t1[kz][ky][xi_x]
  float t1[3][3][A];
#pragma unroll
  for (int kz = 0; kz < 3; ++kz)
#pragma unroll
    for (int ky = 0; ky < 3; ++ky) {
      float row[3];
#pragma unroll
      for (int kx = 0; kx < 3; ++kx) row[kx] = Store<Tin>::to_f32(wp[(long long)((kz * 3 + ky) * 3 + kx) * C]);
      Wino<M>::g(row, t1[kz][ky]);
    }
  // along y: t2[kz][xi_y][xi_x]
  float t2[3][A][A];
#pragma unroll
  for (int kz = 0; kz < 3; ++kz)
#pragma unroll
    for (int xx = 0; xx < A; ++xx) {
      float col[3] = {t1[kz][0][xx], t1[kz][1][xx], t1[kz][2][xx]}, r[A];
      Wino<M>::g(col, r);
#pragma unroll
      for (int yy = 0; yy < A; ++yy) t2[kz][yy][xx] = r[yy];
    }
  // along z, stored as computed
  const long long plane = CMAJOR ? (long long)C * o_pad : (long long)O * C;
  Tst* up = CMAJOR ? u + (long long)c * o_pad + o : u + idx;
#pragma unroll
  for (int yy = 0; yy < A; ++yy)
#pragma unroll
    for (int xx = 0; xx < A; ++xx) {
      float col[3] = {t2[0][yy][xx], t2[1][yy][xx], t2[2][yy][xx]}, r[A];
      Wino<M>::g(col, r);
#pragma unroll
      for (int zz = 0; zz < A; ++zz) up[(long long)((zz * A + yy) * A + xx) * plane] = Store<Tst>::from_f32(r[zz]);
    }
}

// Tile numbering shared by the input and output kernels.
struct TileIdx {
  int n, tz, ty, tx;
};

__device__ __forceinline__ TileIdx tile_of(long long u0, long long t, int tiles_d, int tiles_h, int tiles_w) {
  const long long per_unit = (long long)tiles_h * tiles_w;
  const long long unit = u0 + t / per_unit;
  const int r = (int)(t % per_unit);
  TileIdx ti;
  ti.n = (int)(unit / tiles_d);
  ti.tz = (int)(unit - (long long)ti.n * tiles_d);
  ti.ty = r / tiles_w;
  ti.tx = r - ti.ty * tiles_w;
  return ti;
}

// ---------------------------------------------------------------------------
// Input transform.
// ---------------------------------------------------------------------------
struct Wino3InArgs {
  int d, h, w, c, pd, ph, pw;
  int tiles_d, tiles_h, tiles_w;
  long long in_img_stride;   // D*H*W*C
  long long u0;              // first unit of this batch tile
  long long t_count;         // tiles in this batch tile
  long long t_stride;        // rows of each V plane
};

// Idx: the offset type inside one image and one V plane set (int when the host
// has checked that they fit, long long otherwise).
template <int M, typename Tin, typename Tst, typename Idx>
__global__ void __launch_bounds__(32 * (M + 2))
wino3d_input_kernel(const Tin* __restrict__ in, const Wino3InArgs a, Tst* __restrict__ v) {
  constexpr int A = Wino<M>::A;
  __shared__ float sm[A * A][A][32];      // [xi_z * A + xi_y][x][lane]
  const int lane = threadIdx.x & 31, j = threadIdx.x >> 5;
  const int cgroups = (a.c + 31) >> 5;
  const int cg = (int)(blockIdx.x % cgroups);     // channel group fastest: whole pixels read together
  const long long t = blockIdx.x / cgroups;
  const int c = cg * 32 + lane;
  const bool cok = c < a.c;
  const TileIdx ti = tile_of(a.u0, t, a.tiles_d, a.tiles_h, a.tiles_w);
  const int z0 = ti.tz * M - a.pd, y0 = ti.ty * M - a.ph, x = ti.tx * M - a.pw + j;
  const bool xok = cok && x >= 0 && x < a.w;
  const Tin* base = in + (long long)ti.n * a.in_img_stride + (long long)x * a.c + c;

  // Slice x = j: depth then height transforms of its alpha x alpha values.
  const Idx wc = (Idx)a.w * a.c, hwc = (Idx)a.h * wc;
  float d[A][A];
  if (xok && z0 >= 0 && y0 >= 0 && z0 + A <= a.d && y0 + A <= a.h) {
    const Tin* p = base + ((Idx)z0 * hwc + (Idx)y0 * wc);
#pragma unroll
    for (int zz = 0; zz < A; ++zz)
#pragma unroll
      for (int yy = 0; yy < A; ++yy) d[zz][yy] = Store<Tin>::to_f32(p[(Idx)zz * hwc + (Idx)yy * wc]);
  } else {
    unsigned ym = 0;
#pragma unroll
    for (int yy = 0; yy < A; ++yy)
      if (y0 + yy >= 0 && y0 + yy < a.h) ym |= 1u << yy;
#pragma unroll
    for (int zz = 0; zz < A; ++zz) {
      const int z = z0 + zz;
      const bool zok = xok && z >= 0 && z < a.d;
      const Idx ro = zok ? (Idx)z * hwc + (Idx)y0 * wc : (Idx)0;
#pragma unroll
      for (int yy = 0; yy < A; ++yy)
        d[zz][yy] = (zok && ((ym >> yy) & 1u)) ? Store<Tin>::to_f32(base[ro + (Idx)yy * wc]) : 0.0f;
    }
  }
  float tz[A][A];     // [xi_z][y]
#pragma unroll
  for (int yy = 0; yy < A; ++yy) {
    float col[A], r[A];
#pragma unroll
    for (int zz = 0; zz < A; ++zz) col[zz] = d[zz][yy];
    Wino<M>::bt(col, r);
#pragma unroll
    for (int zz = 0; zz < A; ++zz) tz[zz][yy] = r[zz];
  }
#pragma unroll
  for (int zz = 0; zz < A; ++zz) {
    float r[A];
    Wino<M>::bt(tz[zz], r);
#pragma unroll
    for (int yy = 0; yy < A; ++yy) sm[zz * A + yy][j][lane] = r[yy];
  }
  __syncthreads();

  // Width transform of lines l = j, j + A, ... (all A*A (xi_z, xi_y) lines).
  if (!cok) return;
  const Idx plane = (Idx)(a.t_stride * a.c);
  Tst* vp = v + t * a.c + c + (long long)(j * A) * (a.t_stride * a.c);
#pragma unroll
  for (int k = 0; k < A; ++k) {
    const int l = j + k * A;
    float row[A], r[A];
#pragma unroll
    for (int xx = 0; xx < A; ++xx) row[xx] = sm[l][xx][lane];
    Wino<M>::bt(row, r);
#pragma unroll
    for (int xx = 0; xx < A; ++xx) vp[(Idx)(k * A * A + xx) * plane] = Store<Tst>::from_f32(r[xx]);
  }
}

// ---------------------------------------------------------------------------
// Output transform.
// ---------------------------------------------------------------------------
struct Wino3OutArgs {
  int od, oh, ow, o;
  int tiles_d, tiles_h, tiles_w;
  long long out_img_stride;  // OD*OH*OW*O
  long long u0, t_count, t_stride;
};

template <int M, typename Tout, typename Idx>
__global__ void __launch_bounds__(32 * (M + 2))
wino3d_output_kernel(const float* __restrict__ mb, const Wino3OutArgs a, Tout* __restrict__ out) {
  constexpr int A = Wino<M>::A;
  __shared__ float sm[M * M][A][32];      // [oz * M + oy][xi_x][lane]
  const int lane = threadIdx.x & 31, j = threadIdx.x >> 5;
  const int ogroups = (a.o + 31) >> 5;
  const int og = (int)(blockIdx.x % ogroups);
  const long long t = blockIdx.x / ogroups;
  const int o = og * 32 + lane;
  const bool ook = o < a.o;

  // Slice xi_x = j: depth then height transforms.
  const Idx plane = (Idx)(a.t_stride * a.o);
  const float* mp = mb + t * a.o + o + (long long)j * (a.t_stride * a.o);
  float x[A][A];      // [xi_z][xi_y]
#pragma unroll
  for (int zz = 0; zz < A; ++zz)
#pragma unroll
    for (int yy = 0; yy < A; ++yy) x[zz][yy] = ook ? __ldg(mp + (Idx)((zz * A + yy) * A) * plane) : 0.0f;
  float tz[M][A];     // [oz][xi_y]
#pragma unroll
  for (int yy = 0; yy < A; ++yy) {
    float col[A], r[M];
#pragma unroll
    for (int zz = 0; zz < A; ++zz) col[zz] = x[zz][yy];
    Wino<M>::at(col, r);
#pragma unroll
    for (int zz = 0; zz < M; ++zz) tz[zz][yy] = r[zz];
  }
#pragma unroll
  for (int zz = 0; zz < M; ++zz) {
    float r[M];
    Wino<M>::at(tz[zz], r);
#pragma unroll
    for (int yy = 0; yy < M; ++yy) sm[zz * M + yy][j][lane] = r[yy];
  }
  __syncthreads();

  if (!ook) return;
  const TileIdx ti = tile_of(a.u0, t, a.tiles_d, a.tiles_h, a.tiles_w);
  Tout* op = out + (long long)ti.n * a.out_img_stride + o;
  const Idx os = a.o, wo = (Idx)a.ow * a.o;
  const bool xwhole = ti.tx * M + M <= a.ow;
  for (int l = j; l < M * M; l += A) {
    const int z = ti.tz * M + l / M, y = ti.ty * M + l % M;
    if (z >= a.od || y >= a.oh) continue;
    float row[A], r[M];
#pragma unroll
    for (int xx = 0; xx < A; ++xx) row[xx] = sm[l][xx][lane];
    Wino<M>::at(row, r);
    Tout* rp = op + (((Idx)z * a.oh + y) * wo + (Idx)(ti.tx * M) * os);
#pragma unroll
    for (int xx = 0; xx < M; ++xx)
      if (xwhole || ti.tx * M + xx < a.ow) rp[(Idx)xx * os] = Store<Tout>::from_f32(r[xx]);
  }
}

// The 3D transforms exist for F(2,3) (alpha^3 = 64) and F(4,3) (216).
template <typename F>
cudaError_t by_m3(int m, F&& f) {
  switch (m) {
    case 2: return f(std::integral_constant<int, 2>{});
    case 4: return f(std::integral_constant<int, 4>{});
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_wino3d_filter(const void* w, int o, int c, int m, conv_dtype_t in_dt, conv_dtype_t store_dt,
                                 bool cmajor, long long o_pad, void* u, cudaStream_t s) {
  const long long n = (long long)o * c;
  if (n == 0) return cudaSuccess;
  if (cmajor && store_dt != CONV_F32) return cudaErrorInvalidValue;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  return by_m3(m, [&](auto mc) {
    constexpr int M = decltype(mc)::value;
    return wino_by_dt(in_dt, [&](auto ti) {
      using Tin = decltype(ti);
      return wino_by_dt(store_dt, [&](auto ts) {
        using Tst = decltype(ts);
        if (cmajor)
          wino3d_filter_kernel<M, Tin, Tst, true><<<blocks, 256, 0, s>>>(static_cast<const Tin*>(w), o, c, o_pad,
                                                                         static_cast<Tst*>(u));
        else
          wino3d_filter_kernel<M, Tin, Tst, false><<<blocks, 256, 0, s>>>(static_cast<const Tin*>(w), o, c, o_pad,
                                                                          static_cast<Tst*>(u));
        return cudaGetLastError();
      });
    });
  });
}

cudaError_t launch_wino3d_input(const void* in, const Geom3& g, long long u0, long long nu, int m,
                                conv_dtype_t in_dt, conv_dtype_t store_dt, void* v, long long t_stride,
                                cudaStream_t s) {
  Wino3InArgs a{};
  a.d = g.d; a.h = g.h; a.w = g.w; a.c = g.c;
  a.pd = g.pd; a.ph = g.ph; a.pw = g.pw;
  a.tiles_d = (g.od + m - 1) / m;
  a.tiles_h = (g.oh + m - 1) / m;
  a.tiles_w = (g.ow + m - 1) / m;
  a.in_img_stride = (long long)g.d * g.h * g.w * g.c;
  a.u0 = u0;
  a.t_count = nu * a.tiles_h * a.tiles_w;
  a.t_stride = t_stride;
  if (a.t_count == 0) return cudaSuccess;
  const long long blocks = a.t_count * ((g.c + 31) / 32);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  // 32-bit offsets when one image (with slack for the padding) and the whole V
  // plane set stay below 2^31 elements
  const long long a3 = (long long)(m + 2) * (m + 2) * (m + 2);
  const bool idx32 = a.in_img_stride + 4LL * g.w * g.c < (1LL << 31) && a3 * t_stride * g.c < (1LL << 31);
  return by_m3(m, [&](auto mc) {
    constexpr int M = decltype(mc)::value;
    return wino_by_dt(in_dt, [&](auto ti) {
      using Tin = decltype(ti);
      return wino_by_dt(store_dt, [&](auto ts) {
        using Tst = decltype(ts);
        if (idx32)
          wino3d_input_kernel<M, Tin, Tst, int><<<(unsigned)blocks, 32 * (M + 2), 0, s>>>(
              static_cast<const Tin*>(in), a, static_cast<Tst*>(v));
        else
          wino3d_input_kernel<M, Tin, Tst, long long><<<(unsigned)blocks, 32 * (M + 2), 0, s>>>(
              static_cast<const Tin*>(in), a, static_cast<Tst*>(v));
        return cudaGetLastError();
      });
    });
  });
}

cudaError_t launch_wino3d_output(const float* mbuf, const Geom3& g, long long u0, long long nu, int m,
                                 long long t_stride, conv_dtype_t out_dt, void* out, cudaStream_t s) {
  Wino3OutArgs a{};
  a.od = g.od; a.oh = g.oh; a.ow = g.ow; a.o = g.o;
  a.tiles_d = (g.od + m - 1) / m;
  a.tiles_h = (g.oh + m - 1) / m;
  a.tiles_w = (g.ow + m - 1) / m;
  a.out_img_stride = (long long)g.od * g.oh * g.ow * g.o;
  a.u0 = u0;
  a.t_count = nu * a.tiles_h * a.tiles_w;
  a.t_stride = t_stride;
  if (a.t_count == 0) return cudaSuccess;
  const long long blocks = a.t_count * ((g.o + 31) / 32);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const long long a3 = (long long)(m + 2) * (m + 2) * (m + 2);
  const bool idx32 = a.out_img_stride < (1LL << 31) && a3 * t_stride * g.o < (1LL << 31);
  return by_m3(m, [&](auto mc) {
    constexpr int M = decltype(mc)::value;
    return wino_by_dt(out_dt, [&](auto to) {
      using Tout = decltype(to);
      if (idx32)
        wino3d_output_kernel<M, Tout, int><<<(unsigned)blocks, 32 * (M + 2), 0, s>>>(mbuf, a,
                                                                                     static_cast<Tout*>(out));
      else
        wino3d_output_kernel<M, Tout, long long><<<(unsigned)blocks, 32 * (M + 2), 0, s>>>(mbuf, a,
                                                                                           static_cast<Tout*>(out));
      return cudaGetLastError();
    });
  });
}

}  // namespace b200conv
