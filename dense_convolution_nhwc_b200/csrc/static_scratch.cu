// static_scratch.cu -- a Winograd conv2d entry point that allocates nothing.
//
// conv2d_forward needs a caller-provided workspace for the Winograd path (the
// transformed filter, and the transformed input and GEMM output of one batch
// tile).  Some callers cannot provide one: code that runs inside another
// runtime's hooks with no access to an allocator, code that must not
// allocate once it is running (real-time or fixed-footprint services), and
// callers that receive only borrowed input/output pointers.  For them this file
// holds the scratch in a fixed device array compiled into the library, and the
// entry point below runs the Winograd path with it.
//
// The array is 64 MiB.  Every GPU that loads the library holds it until the
// process exits.  All calls share it and it keeps the last call's contents;
// the Winograd path writes every scratch element it reads, so nothing needs
// clearing between calls.  Two calls whose work overlaps on the GPU (on
// different streams, or from several host threads) race on the array.
//
// The batch is tiled so that the transformed filter plus one batch tile fit in
// the array, exactly as the budgeted Winograd path tiles it, so results equal
// conv2d_forward's Winograd results bit for bit.  A conv whose transformed
// filter plus a single image's transform buffers do not fit is rejected with
// CONV_ERR_WORKSPACE before anything is launched.
#include <cuda_runtime.h>

#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;

// Host code must never use this name as a device address: it is a host-side
// stand-in.  The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// The array's device address in the current device's context.  It is looked
// up on every call rather than cached: a context torn down and re-created
// (cudaDeviceReset) places the array at a new address, and a cached one would
// hand the kernels memory the device no longer maps.  The lookup allocates
// nothing; the first one on a device loads the library's device code there.
conv_status_t scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return CONV_ERR_CUDA;
  *out = p;
  return CONV_OK;
}

}  // namespace

extern "C" conv_status_t conv2d_forward_winograd_static(const void* in, const void* w, void* out,
                                                        const conv2d_desc_t* desc, conv_dtype_t dtype,
                                                        void* stream) {
  if (!desc) return CONV_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CONV_ERR_CUDA;
  void* scratch = nullptr;
  conv_status_t st = scratch_address(&scratch);
  if (st != CONV_OK) return st;

  // Is the shape one the Winograd path runs at all (3x3, stride 1, dilation 1)?
  conv_options_t o{CONV_ALGO_WINOGRAD, 1LL << 60, 1};
  conv_plan_t plan{};
  st = conv2d_plan(desc, dtype, dev, &o, &plan);
  if (st != CONV_OK) return st;
  if (desc->n == 0) return CONV_OK;

  // The largest batch tile whose scratch (transformed filter + the tile's
  // transform buffers) fits the array, by bisection over the forced tile size
  // (the scratch grows with the tile).  Forcing the tile keeps small tiles on
  // the Winograd path.
  o.winograd_budget_bytes = (long long)kStaticScratchBytes;
  auto fits = [&](int tile, conv_plan_t* p) {
    o.winograd_tile_batch = tile;
    return conv2d_plan(desc, dtype, dev, &o, p) == CONV_OK && p->algo == CONV_ALGO_WINOGRAD &&
           p->workspace_bytes <= kStaticScratchBytes;
  };
  if (!fits(1, &plan)) return CONV_ERR_WORKSPACE;   // not even one image fits
  int lo = 1, hi = desc->n;                          // fits(lo) holds
  while (lo < hi) {
    const int mid = lo + (hi - lo + 1) / 2;
    conv_plan_t p{};
    if (fits(mid, &p)) lo = mid;
    else hi = mid - 1;
  }
  if (!fits(lo, &plan)) return CONV_ERR_WORKSPACE;
  return conv2d_forward(in, w, out, desc, dtype, &o, scratch, kStaticScratchBytes, stream);
}
