// elementwise.cu -- bandwidth-bound helpers around the GEMM cores.
//
//  * accumulate: out[i] = round(out[i] + tap[i]), the in-place add that sums a
//    conv3d's depth taps ("Decompose small kernel-depth 3D convs into 2D
//    convs", Change and Open questions 1).  fp32 add, one rounding to the
//    storage dtype; 16-byte vector accesses when both pointers allow it.
//  * channel pad: copies NHWC (or OHWI) rows of C channels into rows of Cp
//    channels with zeros after C, so that rows meet the tensor-memory-access
//    16-byte stride rule.
//  * tap packing: for a few channels (a 3-channel stem), folds the KW taps of
//    each output column into channels so the tensor cores see a KH x 1 conv
//    over KW*C packed channels instead of KH*KW mostly-empty 64-channel steps.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace b200conv {
namespace {

template <typename T>
__global__ void accumulate_vec_kernel(T* __restrict__ out, const T* __restrict__ tap, size_t nvec) {
  constexpr int E = 16 / sizeof(T);
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (; i < nvec; i += stride) {
    uint4 a = reinterpret_cast<const uint4*>(out)[i];
    uint4 b = __ldg(reinterpret_cast<const uint4*>(tap) + i);
    T* pa = reinterpret_cast<T*>(&a);
    const T* pb = reinterpret_cast<const T*>(&b);
#pragma unroll
    for (int e = 0; e < E; ++e)
      pa[e] = Store<T>::from_f32(Store<T>::to_f32(pa[e]) + Store<T>::to_f32(pb[e]));
    reinterpret_cast<uint4*>(out)[i] = a;
  }
}

template <typename T>
__global__ void accumulate_scalar_kernel(T* __restrict__ out, const T* __restrict__ tap, size_t n) {
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (; i < n; i += stride)
    out[i] = Store<T>::from_f32(Store<T>::to_f32(out[i]) + Store<T>::to_f32(tap[i]));
}

template <typename T>
cudaError_t accumulate_typed(void* out, const void* tap, size_t count, cudaStream_t s) {
  constexpr int E = 16 / sizeof(T);
  T* o = static_cast<T*>(out);
  const T* t = static_cast<const T*>(tap);
  const bool aligned = ((reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(tap)) & 15) == 0;
  size_t nvec = aligned ? count / E : 0;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned cap = (unsigned)sms * 8;
  if (nvec > 0) {
    unsigned blocks = (unsigned)((nvec + 255) / 256 < cap ? (nvec + 255) / 256 : cap);
    accumulate_vec_kernel<T><<<blocks, 256, 0, s>>>(o, t, nvec);
  }
  size_t done = nvec * E;
  if (done < count) {
    size_t rest = count - done;
    unsigned blocks = (unsigned)((rest + 255) / 256 < cap ? (rest + 255) / 256 : cap);
    accumulate_scalar_kernel<T><<<blocks, 256, 0, s>>>(o + done, t + done, rest);
  }
  return cudaGetLastError();
}

template <typename T>
__global__ void channel_pad_kernel(const T* __restrict__ src, long long outer, long long inner, int c,
                                   long long src_outer_stride, T* __restrict__ dst, int cp) {
  const long long total = outer * inner * cp;
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (; i < total; i += stride) {
    long long row = i / cp;
    int ch = (int)(i - row * cp);
    long long a = row / inner, b = row - a * inner;
    dst[i] = ch < c ? src[a * src_outer_stride + b * c + ch] : Store<T>::from_f32(0.0f);
  }
}

// Tap packing for small C: P[n][h][ow][kw*C + c] = in[n][h][ow*sw - pw + kw*dw][c]
// (zero outside the row and for channels >= KW*C), so the conv becomes KH x 1
// over Cp = KW*C rounded up packed channels.
template <typename T>
__global__ void wpack_kernel(const T* __restrict__ src, long long pixels /* n*h*ow */, int w, int c, int kw, int sw,
                             int pw, int dw, int ow, long long in_row_stride, long long in_img_stride, int h,
                             T* __restrict__ dst, int cp) {
  // one thread per output pixel (n, y, x); its cp packed channels are written in
  // 8-element vectors (cp is a multiple of 8, rows 16-byte aligned).  Packed
  // channel ch = k*c + cc is walked incrementally (no division per element).
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const int kc = kw * c;
  for (; i < pixels; i += stride) {
    long long nh;
    int x;
    if (pixels < (1LL << 31)) {        // 32-bit division when the pixel count allows it
      const int ii = (int)i;
      nh = ii / ow;
      x = ii - (int)nh * ow;
    } else {
      nh = i / ow;
      x = (int)(i - nh * ow);
    }
    const long long n = nh / h, y = nh - n * h;
    const T* row = src + n * in_img_stride + y * in_row_stride;
    T* out = dst + i * cp;
    int ix = x * sw - pw, cc = 0, ch = 0;
    for (int ch0 = 0; ch0 < cp; ch0 += 8) {
      __align__(16) T v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float f = 0.0f;
        if (ch < kc && ix >= 0 && ix < w) f = Store<T>::to_f32(row[(long long)ix * c + cc]);
        v[e] = Store<T>::from_f32(f);
        ++ch;
        if (++cc == c) {
          cc = 0;
          ix += dw;
        }
      }
      if constexpr (sizeof(T) == 2) {
        *reinterpret_cast<uint4*>(out + ch0) = *reinterpret_cast<const uint4*>(v);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) out[ch0 + e] = v[e];
      }
    }
  }
}

// Four elements per thread (count % 4 == 0, 16-byte aligned partials); the
// partial sums are added in split order 0..ksplit-1 for every element.
template <typename T>
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int ksplit, size_t count, T* __restrict__ out,
                                     int accumulate) {
  pdl_wait_then_release();     // the partials come from the conv launched just before
  const size_t n4 = count / 4;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (; i < n4; i += stride) {
    float4 sum = __ldg(reinterpret_cast<const float4*>(partial) + i);
    for (int k = 1; k < ksplit; ++k) {
      const float4 p = __ldg(reinterpret_cast<const float4*>(partial + (size_t)k * count) + i);
      sum.x += p.x; sum.y += p.y; sum.z += p.z; sum.w += p.w;
    }
    float v[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      T* o = out + 4 * i + e;
      float r = v[e];
      if (accumulate) r = Store<T>::to_f32(*o) + Store<T>::to_f32(Store<T>::from_f32(v[e]));
      *o = Store<T>::from_f32(r);
    }
  }
}

template <typename T>
__global__ void splitk_reduce_scalar_kernel(const float* __restrict__ partial, int ksplit, size_t count,
                                            T* __restrict__ out, int accumulate) {
  pdl_wait_then_release();
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (; i < count; i += stride) {
    float sum = 0.0f;
    for (int k = 0; k < ksplit; ++k) sum += __ldg(partial + (size_t)k * count + i);   // fixed order
    float v = sum;
    if (accumulate) v = Store<T>::to_f32(out[i]) + Store<T>::to_f32(Store<T>::from_f32(sum));
    out[i] = Store<T>::from_f32(v);
  }
}

}  // namespace

// The small kernels that run between tensor-core convs ask for the same
// shared-memory carveout as those (the maximum), so the SM is not
// reconfigured between a conv and its reduce or pre-pass.  A preference only;
// set once per kernel (the attribute is per function).
template <typename K>
bool prefer_max_shared(K kernel) {
  cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  return true;
}

cudaError_t launch_splitk_reduce(const float* partial, int ksplit, size_t count, void* out, conv_dtype_t dt,
                                 bool accumulate, cudaStream_t s) {
  if (count == 0) return cudaSuccess;
  const int acc = accumulate ? 1 : 0;
  const bool vec = count % 4 == 0 && (reinterpret_cast<uintptr_t>(partial) & 15) == 0;
  const size_t items = vec ? count / 4 : count;
  unsigned blocks = (unsigned)((items + 255) / 256 < 148 * 16 ? (items + 255) / 256 : 148 * 16);
  auto run = [&](auto tag) {
    using T = decltype(tag);
    static const bool pv = prefer_max_shared(splitk_reduce_kernel<T>);
    static const bool ps = prefer_max_shared(splitk_reduce_scalar_kernel<T>);
    (void)pv;
    (void)ps;
    T* o = static_cast<T*>(out);
    if (vec) return launch_pdl(splitk_reduce_kernel<T>, dim3(blocks), dim3(256), 0, s, partial, ksplit, count, o, acc);
    return launch_pdl(splitk_reduce_scalar_kernel<T>, dim3(blocks), dim3(256), 0, s, partial, ksplit, count, o, acc);
  };
  switch (dt) {
    case CONV_F32: return run(float{});
    case CONV_F16: return run(__half{});
    case CONV_BF16: return run(__nv_bfloat16{});
  }
  return cudaErrorInvalidValue;
}

// Full tap packing for a few-channel input (the ResNet stem): the conv becomes a
// 1x1 conv over cp = KH*KW*C rounded up to 8 packed channels, packed channel
// k = (kh*KW + kw)*C + c of output pixel (n, oy, ox) holding
// src[n][oy*sh - ph + kh*dh][ox*sw - pw + kw*dw][c] (zero outside the image and
// for k >= KH*KW*C).  One thread writes 8 consecutive packed channels (16 bytes
// for 16-bit types) of one pixel, so neighbouring threads write neighbouring
// bytes; (kh, kw, c) are decoded once per thread and then stepped.
template <typename T, typename Idx>
__global__ void __launch_bounds__(256)
fullpack_kernel(const T* __restrict__ src, Idx chunks, int chunks_per_px, int oh, int ow, int h, int w, int c,
                int kh, int kw, int sh, int sw, int ph, int pw, int dh, int dw, long long in_img_stride,
                T* __restrict__ dst, int cp) {
  const int ktot = kh * kw * c;
  const int kwc = kw * c;
  const Idx ohw = (Idx)oh * ow;
  for (Idx i = (Idx)blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += (Idx)gridDim.x * blockDim.x) {
    const Idx px = i / chunks_per_px;
    const int chunk = (int)(i - px * chunks_per_px);
    const Idx nimg = px / ohw;
    const int r = (int)(px - nimg * ohw);
    const int oy = r / ow, ox = r - (r / ow) * ow;
    const T* img = src + (long long)nimg * in_img_stride;
    int k = chunk * 8;
    int ky = k / kwc;
    int rem = k - ky * kwc;
    int kx = rem / c, cc = rem - kx * c;
    const int y0 = oy * sh - ph, x0 = ox * sw - pw;
    __align__(16) T v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int y = y0 + ky * dh, x = x0 + kx * dw;
      const bool ok = k < ktot && y >= 0 && y < h && x >= 0 && x < w;
      v[e] = ok ? img[((Idx)y * w + x) * c + cc] : Store<T>::from_f32(0.0f);
      ++k;
      if (++cc == c) {
        cc = 0;
        if (++kx == kw) {
          kx = 0;
          ++ky;
        }
      }
    }
    T* out = dst + (long long)px * cp + chunk * 8;
    if constexpr (sizeof(T) == 2) {
      *reinterpret_cast<uint4*>(out) = *reinterpret_cast<const uint4*>(v);
    } else {
      *reinterpret_cast<float4*>(out) = *reinterpret_cast<const float4*>(v);
      *reinterpret_cast<float4*>(out + 4) = *reinterpret_cast<const float4*>(v + 4);
    }
  }
}

// The same packing, staged: one block takes up to P consecutive output pixels of
// one output row.  It first copies the KH input rows those pixels read (the
// span of columns they reach, zero outside the image) into shared memory, and a
// table mapping packed channel k to its offset in that staged span; every packed
// value of pixel p is then tile[p*sw*C + tab[k]], so no packed value needs an
// index decode of its own.
template <typename T>
__global__ void __launch_bounds__(256, 8)
fullpack_rows_kernel(const T* __restrict__ src, int oh, int ow, int h, int w, int c, int kh, int kw, int sh,
                     int sw, int ph, int pw, int dh, int dw, long long in_img_stride, T* __restrict__ dst, int cp,
                     int P, int xtiles) {
  extern __shared__ __align__(16) unsigned char fp_smem[];
  int* tab = reinterpret_cast<int*>(fp_smem);
  T* tile = reinterpret_cast<T*>(fp_smem + (size_t)cp * sizeof(int));
  const T zero = Store<T>::from_f32(0.0f);
  const int bd = blockDim.x;
  const int b = blockIdx.x;
  const int xt = b % xtiles;
  const int rest = b / xtiles;
  const int oy = rest % oh;
  const long long nimg = rest / oh;
  const int ox0 = xt * P;
  const int np = min(P, ow - ox0);
  const int L = ((np - 1) * sw + (kw - 1) * dw + 1) * c;   // staged elements per input row
  const int xs = ox0 * sw - pw;                             // first staged input column
  const int kwc = kw * c, ktot = kh * kwc;
  for (int k = threadIdx.x; k < cp; k += bd) {
    int t = -1;
    if (k < ktot) {
      const int ky = k / kwc, r = k - ky * kwc;
      const int kx = r / c, cc = r - kx * c;
      t = ky * L + kx * dw * c + cc;
    }
    tab[k] = t;
  }
  const T* img = src + nimg * in_img_stride;
  // staged elements e in [lo, hi) of a row lie inside the image columns
  const int lo = max(0, -xs * c), hi = min(L, (w - xs) * c);
  for (int ky = 0; ky < kh; ++ky) {
    const int y = oy * sh - ph + ky * dh;
    T* trow = tile + ky * L;
    if (y < 0 || y >= h) {
      for (int e = threadIdx.x; e < L; e += bd) trow[e] = zero;
      continue;
    }
    const T* row = img + ((long long)y * w + xs) * c;
#pragma unroll 4
    for (int e = threadIdx.x; e < L; e += bd) trow[e] = (e >= lo && e < hi) ? row[e] : zero;
  }
  __syncthreads();
  // The block is a whole number R of rows of cp/2 threads: each thread owns one
  // pair of adjacent packed channels (its two tap offsets held in registers) and
  // steps through pixels p, p + R, ...; a warp writes contiguous bytes.
  struct alignas(2 * sizeof(T)) V2 {
    T x, y;
  };
  const int cph = cp / 2;
  const int R = bd / cph;
  if (threadIdx.x >= R * cph) return;
  const int k2 = threadIdx.x % cph;
  int p = threadIdx.x / cph;
  const int2 t = reinterpret_cast<const int2*>(tab)[k2];
  const bool v0 = t.x >= 0, v1 = t.y >= 0;
  const T* b0 = tile + p * sw * c + (v0 ? t.x : 0);
  const T* b1 = tile + p * sw * c + (v1 ? t.y : 0);
  const int pstep = R * sw * c;
  T* o = dst + (((nimg * oh + oy) * ow + ox0 + p) * (long long)cp + 2 * k2);
  const long long ostep = (long long)R * cp;
  for (; p < np; p += R) {
    V2 v;
    v.x = v0 ? *b0 : zero;
    v.y = v1 ? *b1 : zero;
    *reinterpret_cast<V2*>(o) = v;
    b0 += pstep;
    b1 += pstep;
    o += ostep;
  }
}

cudaError_t launch_fullpack(const void* src, const Geom& g, void* dst, int cp, conv_dtype_t dt, int sm_count,
                            cudaStream_t s) {
  if (cp % 8 != 0) return cudaErrorInvalidValue;
  const long long px = (long long)g.n * g.oh * g.ow;
  const long long chunks = px * (cp / 8);
  if (chunks == 0) return cudaSuccess;
  // Staged form: the widest row segment (at most 128 pixels) whose staged input
  // rows and tap table fit 48 KB of shared memory, narrowed (to no less than 16
  // pixels) while that leaves fewer than eight blocks per SM.  The block is the
  // largest whole number of cp/2-thread rows within 256 threads.
  const int esz = dt == CONV_F32 ? 4 : 2;
  auto smem_for = [&](long long P) {
    return (long long)cp * 4 + (long long)g.kh * ((P - 1) * g.sw + (long long)(g.kw - 1) * g.dw + 1) * g.c * esz;
  };
  long long P = g.ow < 128 ? g.ow : 128;
  while (P > 1 && smem_for(P) > 48 * 1024) P /= 2;
  while (P >= 32 && (long long)g.n * g.oh * ((g.ow + P - 1) / P) < 8LL * sm_count) P = (P + 1) / 2;
  const long long xtiles = (g.ow + P - 1) / P;
  const long long row_blocks = (long long)g.n * g.oh * xtiles;
  if (cp <= 512 && smem_for(P) <= 48 * 1024 && row_blocks < (1LL << 31)) {
    const size_t smem = (size_t)smem_for(P);
    auto staged = [&](auto tag) {
      using T = decltype(tag);
      fullpack_rows_kernel<T><<<(unsigned)row_blocks, (cp / 2) * (256 / (cp / 2)), smem, s>>>(
          static_cast<const T*>(src), g.oh, g.ow, g.h, g.w, g.c, g.kh, g.kw, g.sh, g.sw, g.ph, g.pw, g.dh, g.dw,
          g.in_img_stride, static_cast<T*>(dst), cp, (int)P, (int)xtiles);
      return cudaGetLastError();
    };
    switch (dt) {
      case CONV_F32: return staged(float{});
      case CONV_F16: return staged(__half{});
      case CONV_BF16: return staged(__nv_bfloat16{});
    }
    return cudaErrorInvalidValue;
  }
  unsigned blocks = (unsigned)((chunks + 255) / 256 < 148 * 32 ? (chunks + 255) / 256 : 148 * 32);
  // 32-bit index arithmetic when the chunk count and one image fit
  const bool idx32 = chunks < (1LL << 31) && g.in_img_stride < (1LL << 31);
  auto go = [&](auto tag) {
    using T = decltype(tag);
    if (idx32)
      fullpack_kernel<T, int><<<blocks, 256, 0, s>>>(static_cast<const T*>(src), (int)chunks, cp / 8, g.oh, g.ow,
                                                     g.h, g.w, g.c, g.kh, g.kw, g.sh, g.sw, g.ph, g.pw, g.dh, g.dw,
                                                     g.in_img_stride, static_cast<T*>(dst), cp);
    else
      fullpack_kernel<T, long long><<<blocks, 256, 0, s>>>(static_cast<const T*>(src), chunks, cp / 8, g.oh, g.ow,
                                                           g.h, g.w, g.c, g.kh, g.kw, g.sh, g.sw, g.ph, g.pw, g.dh,
                                                           g.dw, g.in_img_stride, static_cast<T*>(dst), cp);
    return cudaGetLastError();
  };
  switch (dt) {
    case CONV_F32: return go(float{});
    case CONV_F16: return go(__half{});
    case CONV_BF16: return go(__nv_bfloat16{});
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_wpack(const void* src, long long n, int h, int w, int c, int kw, int sw, int pw, int dw, int ow,
                         long long in_img_stride, void* dst, int cp, conv_dtype_t dt, cudaStream_t s) {
  if (cp % 8 != 0) return cudaErrorInvalidValue;
  const long long total = n * h * (long long)ow;     // output pixels
  if (total == 0) return cudaSuccess;
  unsigned blocks = (unsigned)((total + 255) / 256 < 148 * 32 ? (total + 255) / 256 : 148 * 32);
  const long long rs = (long long)w * c;
  switch (dt) {
    case CONV_F32:
      wpack_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(src), total, w, c, kw, sw, pw, dw, ow, rs,
                                                 in_img_stride, h, static_cast<float*>(dst), cp);
      break;
    case CONV_F16:
      wpack_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(src), total, w, c, kw, sw, pw, dw, ow, rs,
                                                  in_img_stride, h, static_cast<__half*>(dst), cp);
      break;
    case CONV_BF16:
      wpack_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src), total, w, c, kw, sw,
                                                         pw, dw, ow, rs, in_img_stride, h,
                                                         static_cast<__nv_bfloat16*>(dst), cp);
      break;
  }
  return cudaGetLastError();
}

cudaError_t launch_accumulate(void* out, const void* tap, size_t count, conv_dtype_t dt,
                              cudaStream_t s) {
  if (count == 0) return cudaSuccess;
  switch (dt) {
    case CONV_F32: return accumulate_typed<float>(out, tap, count, s);
    case CONV_F16: return accumulate_typed<__half>(out, tap, count, s);
    case CONV_BF16: return accumulate_typed<__nv_bfloat16>(out, tap, count, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_fill_zero(void* out, size_t bytes, cudaStream_t s) {
  if (bytes == 0) return cudaSuccess;
  return cudaMemsetAsync(out, 0, bytes, s);
}

cudaError_t launch_channel_pad(const void* src, long long outer, long long inner, int c,
                               long long src_outer_stride, void* dst, int cp, conv_dtype_t dt,
                               cudaStream_t s) {
  long long total = outer * inner * cp;
  if (total == 0) return cudaSuccess;
  unsigned blocks = (unsigned)((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16);
  switch (dt) {
    case CONV_F32:
      channel_pad_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(src), outer, inner, c,
                                                       src_outer_stride, static_cast<float*>(dst), cp);
      break;
    case CONV_F16:
      channel_pad_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(src), outer, inner, c,
                                                        src_outer_stride, static_cast<__half*>(dst), cp);
      break;
    case CONV_BF16:
      channel_pad_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(src), outer, inner, c, src_outer_stride,
          static_cast<__nv_bfloat16*>(dst), cp);
      break;
  }
  return cudaGetLastError();
}

}  // namespace b200conv
