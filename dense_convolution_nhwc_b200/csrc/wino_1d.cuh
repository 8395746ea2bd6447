// wino_1d.cuh -- the 1D Winograd F(m, 3) transforms as a compile-time family,
// shared by the 2D and 3D transform kernels.  Multi-dimensional transforms are
// these applied along each axis in turn ("Fast Algorithms for Convolutional
// Neural Networks", Lavin and Gray, 2016: the nested form of the 1D algorithm).
#pragma once

#include <cuda_runtime.h>

#include <type_traits>

#include "../../include/b200conv.h"
#include "winograd_gen.cuh"

namespace b200conv {

template <int M> struct Wino;
template <> struct Wino<2> {
  static constexpr int A = 4;
  static __device__ __forceinline__ void bt(const float* x, float* y) { wino2_bt(x, y); }
  static __device__ __forceinline__ void g(const float* x, float* y) { wino2_g(x, y); }
  static __device__ __forceinline__ void at(const float* x, float* y) { wino2_at(x, y); }
};
template <> struct Wino<4> {
  static constexpr int A = 6;
  static __device__ __forceinline__ void bt(const float* x, float* y) { wino4_bt(x, y); }
  static __device__ __forceinline__ void g(const float* x, float* y) { wino4_g(x, y); }
  static __device__ __forceinline__ void at(const float* x, float* y) { wino4_at(x, y); }
};
template <> struct Wino<6> {
  static constexpr int A = 8;
  static __device__ __forceinline__ void bt(const float* x, float* y) { wino6_bt(x, y); }
  static __device__ __forceinline__ void g(const float* x, float* y) { wino6_g(x, y); }
  static __device__ __forceinline__ void at(const float* x, float* y) { wino6_at(x, y); }
};

// Host-side dispatch of a runtime m / dtype onto the templates.
template <typename F>
cudaError_t wino_by_m(int m, F&& f) {
  switch (m) {
    case 2: return f(std::integral_constant<int, 2>{});
    case 4: return f(std::integral_constant<int, 4>{});
    case 6: return f(std::integral_constant<int, 6>{});
  }
  return cudaErrorInvalidValue;
}

template <typename F>
cudaError_t wino_by_dt(conv_dtype_t dt, F&& f) {
  switch (dt) {
    case CONV_F32: return f(float{});
    case CONV_F16: return f(__half{});
    case CONV_BF16: return f(__nv_bfloat16{});
  }
  return cudaErrorInvalidValue;
}

}  // namespace b200conv
