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
