// common.cuh -- helpers shared by the kernels: storage-type traits,
// round-to-nearest-even conversions from the fp32 accumulators, and
// programmatic dependent launch.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>
#include <utility>

#include <cuda_runtime.h>

namespace b200conv {

template <typename T> struct Store;

template <> struct Store<float> {
  static __device__ __forceinline__ float to_f32(float v) { return v; }
  static __device__ __forceinline__ float from_f32(float v) { return v; }
};
template <> struct Store<__half> {
  static __device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }
  static __device__ __forceinline__ __half from_f32(float v) { return __float2half_rn(v); }
};
template <> struct Store<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float v) { return __float2bfloat16_rn(v); }
};

// Two adjacent 16-bit values as one 32-bit word, converted per component with
// the same round-to-nearest-even as Store<T>.
template <typename T> struct Pair;
template <> struct Pair<__half> {
  using type = __half2;
  static __device__ __forceinline__ float2 to_f32(type v) { return __half22float2(v); }
  static __device__ __forceinline__ type from_f32(float a, float b) { return __floats2half2_rn(a, b); }
};
template <> struct Pair<__nv_bfloat16> {
  using type = __nv_bfloat162;
  static __device__ __forceinline__ float2 to_f32(type v) { return __bfloat1622float2(v); }
  static __device__ __forceinline__ type from_f32(float a, float b) { return __floats2bfloat162_rn(a, b); }
};

template <typename T>
__device__ __forceinline__ float ld_f32(const T* p) { return Store<T>::to_f32(*p); }
template <typename T>
__device__ __forceinline__ void st_f32(T* p, float v) { *p = Store<T>::from_f32(v); }

// Pack two fp32 values into one 32-bit word of two 16-bit values (low = a).
template <typename T> __device__ __forceinline__ uint32_t pack2(float a, float b);
template <> __device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialization attribute may start while the previous kernel in the
// stream finishes; it runs its prologue (barriers, TMEM, tensor-map prefetch),
// then waits here for the previous kernel's results before touching global
// memory, and lets the next kernel start launching.  Both are no-ops for a
// normal launch.
__device__ __forceinline__ void pdl_wait_then_release() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch with programmatic stream serialization (the kernel calls
// pdl_wait_then_release before its first global access).
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, int smem, cudaStream_t s, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

}  // namespace b200conv
