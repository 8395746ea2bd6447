// api.cu -- the C ABI: validation, the algorithm selector, and dispatch.
//
// Selector ("Bound winograd conv2d working set by tiling the batch", Problem
// and Fix; maintainer review: dispatch never depends on current memory):
//   * Winograd is considered for 3x3, stride 1, dilation 1 convs that meet
//     the page's channel rule C % 32 == 0 && O % 32 == 0 && C + O >= 256, for
//     fp32 inputs, and for 16-bit inputs only with deep, wide GEMMs (C >= 1024
//     and O >= 1024, or C >= 512 and O >= 2048): below that the transforms'
//     HBM traffic costs more than the tensor cores save.
//   * The batch is cut into tiles of nb images, nb = floor(budget /
//     per-image scratch), budget = min(3/4 * total device memory - (input +
//     output + transformed filter), 8 GiB).  nb = 0, or tiles carrying fewer
//     GEMM rows than one wave of 128-row tiles per SM, fall back to the
//     scratch-free implicit GEMM.  A forced tile size is capped by nb.
//   * Everything is a pure function of (shape, dtype, constant device
//     properties, options); the environment hooks are read before selection.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace b200conv {
namespace {

__device__ int g_error_word;

constexpr long long kWinogradCap = 8LL << 30;   // 8 GiB: the GPU is shared
constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  conv_device_props_t props{};
  int* err_word = nullptr;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Constant properties are cached per device.  The error word's device address
// is looked up again on every call made with that device current: a context
// torn down and re-created (cudaDeviceReset) gives the word a new address, and
// a cached one would then point at memory the device no longer maps.  The
// lookup allocates nothing.
conv_status_t device_state(int dev, DeviceState** out) {
  if (dev < 0 || dev >= kMaxDevices) return CONV_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceState& d = g_dev[dev];
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return CONV_ERR_CUDA;
  if (!d.ready) {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return CONV_ERR_CUDA;
    d.props.sm_count = p.multiProcessorCount;
    d.props.cc_major = p.major;
    d.props.cc_minor = p.minor;
    d.props.total_global_mem = (unsigned long long)p.totalGlobalMem;
    d.ready = true;
  }
  if (cur == dev || !d.err_word) {
    if (cur != dev && cudaSetDevice(dev) != cudaSuccess) return CONV_ERR_CUDA;
    void* addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_error_word);
    if (e == cudaSuccess && addr != d.err_word) e = cudaMemset(addr, 0, sizeof(int));   // a new context
    if (cur != dev) cudaSetDevice(cur);
    if (e != cudaSuccess) return CONV_ERR_CUDA;
    d.err_word = static_cast<int*>(addr);
  }
  *out = &d;
  return CONV_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

long long out_extent(long long in, int k, int s, int p, int d) {
  return (in + 2LL * p - (long long)d * (k - 1) - 1) / s + 1;
}

// ------------------------------ profiling ------------------------------------
// Opt-in: each kernel launch is bracketed by two events on its stream.

enum Kind { K_TC_CONV, K_TC_CONV3D, K_SIMT_CONV, K_SPLITK_REDUCE, K_WINO_FILTER, K_WINO_INPUT, K_WINO_GEMM_TC, K_WINO_GEMM_SIMT,
            K_WINO_OUTPUT, K_WINO3D_FILTER, K_WINO3D_INPUT, K_WINO3D_GEMM_TC, K_WINO3D_GEMM_SIMT, K_WINO3D_OUTPUT,
            K_ACCUMULATE, K_CHANNEL_PAD, K_FILL, K_WINO_PASS, K_WINO_FUSED, K_COUNT };
const char* const kKindName[K_COUNT] = {"tc_conv", "tc_conv3d", "simt_conv", "splitk_reduce", "wino_filter", "wino_input", "wino_gemm_tc",
                                        "wino_gemm_simt", "wino_output", "wino3d_filter", "wino3d_input", "wino3d_gemm_tc",
                                        "wino3d_gemm_simt", "wino3d_output", "accumulate", "channel_pad", "fill",
                                        "wino_pass", "wino_fused"};

struct ProfRecord {
  int kind;
  cudaEvent_t a, b;
};
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<ProfRecord> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
} g_prof;

struct ProfScope {
  cudaStream_t s;
  bool active = false;
  ProfRecord r{};
  ProfScope(int kind, cudaStream_t st) : s(st) {
    if (!g_prof.on) return;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    r.kind = kind;
    r.a = g_prof.get();
    r.b = g_prof.get();
    if (r.a && r.b && cudaEventRecord(r.a, s) == cudaSuccess) active = true;
  }
  ~ProfScope() {
    if (!active) return;
    cudaEventRecord(r.b, s);
    std::lock_guard<std::mutex> lk(g_prof.mu);
    g_prof.recs.push_back(r);
  }
};

// ----------------------------- options ---------------------------------------

conv_options_t effective_options(const conv_options_t* opts) {
  if (opts) return *opts;
  conv_options_t o{CONV_ALGO_AUTO, -1, 0};
  if (const char* a = std::getenv("B200CONV_ALGO")) {
    std::string s(a);
    if (s == "implicit") o.algo = CONV_ALGO_IMPLICIT_GEMM;
    else if (s == "winograd") o.algo = CONV_ALGO_WINOGRAD;
    else if (s == "direct") o.algo = CONV_ALGO_DIRECT;
  }
  if (const char* b = std::getenv("B200CONV_WINOGRAD_WORKSPACE_BYTES")) o.winograd_budget_bytes = std::atoll(b);
  if (const char* t = std::getenv("B200CONV_WINOGRAD_TILE_BATCH")) o.winograd_tile_batch = std::atoi(t);
  return o;
}

// ----------------------------- validation ------------------------------------

bool valid_dtype(conv_dtype_t t) { return t == CONV_F32 || t == CONV_F16 || t == CONV_BF16; }

conv_status_t geom2d(const conv2d_desc_t* d, Geom* g) {
  if (!d) return CONV_ERR_INVALID;
  if (d->n < 0 || d->h <= 0 || d->w <= 0 || d->c <= 0 || d->o <= 0 || d->kh <= 0 || d->kw <= 0)
    return CONV_ERR_INVALID;
  for (int i = 0; i < 2; ++i)
    if (d->stride[i] <= 0 || d->dilation[i] <= 0 || d->pad[i] < 0) return CONV_ERR_INVALID;
  long long oh = out_extent(d->h, d->kh, d->stride[0], d->pad[0], d->dilation[0]);
  long long ow = out_extent(d->w, d->kw, d->stride[1], d->pad[1], d->dilation[1]);
  if (oh <= 0 || ow <= 0 || oh > (1 << 30) || ow > (1 << 30)) return CONV_ERR_INVALID;
  g->n = d->n; g->h = d->h; g->w = d->w; g->c = d->c; g->o = d->o; g->kh = d->kh; g->kw = d->kw;
  g->sh = d->stride[0]; g->sw = d->stride[1];
  g->ph = d->pad[0]; g->pw = d->pad[1];
  g->dh = d->dilation[0]; g->dw = d->dilation[1];
  g->oh = (int)oh; g->ow = (int)ow;
  g->in_img_stride = (long long)d->h * d->w * d->c;
  g->w_row_stride = (long long)d->kh * d->kw * d->c;
  g->out_img_stride = oh * ow * d->o;
  return CONV_OK;
}

// ------------------------------- selector ------------------------------------

struct Sel {
  conv_algo_t algo = CONV_ALGO_IMPLICIT_GEMM;
  conv_engine_t engine = CONV_ENGINE_SIMT;
  int tile_m = 128, tile_n = 128;
  int wino_m = 0, nb = 0, ntiles = 0, cpad = 0;
  bool wpack = false;      // KW taps folded into cpad channels (a few-channel input)
  bool fpack = false;      // all KH*KW taps folded into cpad channels: a 1x1 conv over them
  int ksplit = 1;          // implicit GEMM: K range split over ksplit CTAs, fp32 partials reduced after
  size_t split_off = 0;    // workspace offset of the partials
  conv_dtype_t wino_store = CONV_F32;
  long long chunk = 0;     // Winograd: tiles per transform -> GEMM -> transform pass (0: the whole batch tile)
  bool fused = false;      // fp32 Winograd as one persistent kernel (transforms overlapped with the GEMM)
  bool split_bf16 = false; // fp32 Winograd whose GEMM runs on tcgen05 over split-bf16 operands
  int fused_grid = 0;      // its CTAs (one per SM)
  size_t ws = 0;
};

bool winograd_shape(const Geom& g) {
  return g.kh == 3 && g.kw == 3 && g.sh == 1 && g.sw == 1 && g.dh == 1 && g.dw == 1;
}
bool winograd_channel_rule(const Geom& g) {
  return g.c % 32 == 0 && g.o % 32 == 0 && g.c + g.o >= 256;
}
// 16-bit inputs: F(2x2,3x3) on the tensor cores against the implicit GEMM.
// Winograd saves 2.25x of the tensor work but moves V and M through HBM; on
// B200 it is the faster of the two once the GEMMs are deep and wide enough
// (measured on the wide 3x3 set: C >= 1024 with O >= 1024, C >= 512 with O >= 2048).
bool winograd_16bit_wins(const Geom& g) {
  return (g.c >= 1024 && g.o >= 1024) || (g.c >= 512 && g.o >= 2048);
}
int winograd_m_for(conv_dtype_t dt) { return dt == CONV_F32 ? 6 : 2; }

// The tensor-core engine can express this shape (pointer alignment is checked at launch).
bool tc_shape_ok(const Geom& g, conv_dtype_t dt, const conv_device_props_t& p) {
  if (dt == CONV_F32 || p.cc_major != 10) return false;
  if (g.sh > 8 || g.sw > 8) return false;
  const int uw = g.pw - g.dw * (g.kw - 1), uh = g.ph - g.dh * (g.kh - 1);
  if (g.pw > 128 || g.ph > 128 || uw < -128 || uw > 127 || uh < -128 || uh > 127) return false;
  if ((long long)g.dw * (g.kw - 1) > 65535 || (long long)g.dh * (g.kh - 1) > 65535) return false;
  return true;
}

int tc_tile_n(const Geom& g, const conv_device_props_t& p) {
  if (g.o <= 128) return 128;
  long long m_tiles = ((long long)g.n * g.oh * g.ow + 127) / 128;
  long long tiles256 = m_tiles * ((g.o + 255) / 256);
  return tiles256 < p.sm_count ? 128 : 256;
}

long long round4(long long x) { return (x + 3) & ~3LL; }

// CTA pairs (tile_m = 256, two SMs per tile sharing the weight tile) for
// 256-wide column tiles with a K loop of at least 8 steps of 64 when there are
// enough 256-row tiles to give every SM pair one.  With a shorter K loop the
// pair's shared accumulator handshake makes every tile wait for the slower of
// its two epilogues, and the 128-row tiles are faster (measured on the 16-bit
// Winograd GEMM: pairs slower at C = 128 and 256, faster at C = 512 and 1024).
// B200CONV_TC_PAIR=0 (a test hook, read on every call) keeps 128-row tiles.
bool tc_pair_tiles(long long rows, long long batches, int o, int tile_n, long long ksteps,
                   const conv_device_props_t& p) {
  if (tile_n != 256 || ksteps < 8) return false;
  if (const char* e = std::getenv("B200CONV_TC_PAIR"))
    if (std::strcmp(e, "0") == 0) return false;
  const long long tiles = batches * ((rows + 255) / 256) * ((o + 255) / 256);
  return tiles >= p.sm_count / 2;
}

// V layout of the fp32 (FFMA) Winograd path: tile-major [a2][T][C] lets the
// input transform write whole pixels' channels contiguously; the GEMM stages
// it through swizzled shared rows.
#ifndef B200CONV_F32_V_TILE_MAJOR
#define B200CONV_F32_V_TILE_MAJOR 1
#endif
constexpr bool kF32VTileMajor = B200CONV_F32_V_TILE_MAJOR != 0;

// Workspace layout of the Winograd path for batch tiles of nb images.
//   tensor-core GEMM (16-bit operands): U [a2][O][C], V [a2][T][C], M [a2][T][O], all in the
//                                       operand type (M accumulated in fp32, stored rounded)
//   FFMA GEMM (fp32 operands):          U [a2][C][O4], V [a2][T][C] (tile-major) or
//                                       [a2][C][T4] (channel-major), M [a2][T][O] fp32
// (O4, T4 = O, T rounded up to 4 so rows start 16-byte aligned).
struct WinoLayout {
  size_t u_bytes = 0, v_bytes = 0, m_bytes = 0;
  long long tiles_per_img = 0;
  size_t per_img = 0;   // V + M bytes per image (the budget unit)
};

// chunk > 0: the batch tile's tiles pass through V and M in chunks of at most
// `chunk` tiles, so V and M hold one chunk.
// split: the split-bf16 fp32 GEMM's operands, U [a2][O][3C] and V [a2][T][3C]
// in bf16, M [a2][T][O] fp32.
WinoLayout winograd_layout(const Geom& g, conv_dtype_t store, bool cmajor, int m, long long nb, long long chunk = 0,
                           bool split = false) {
  WinoLayout L;
  const long long a2 = (long long)(m + 2) * (m + 2);
  L.tiles_per_img = (long long)((g.oh + m - 1) / m) * ((g.ow + m - 1) / m);
  if (split) {
    const long long t = nb * L.tiles_per_img;
    L.per_img = (size_t)(a2 * L.tiles_per_img) * ((size_t)g.c * 6 + (size_t)g.o * 4);
    L.u_bytes = align256((size_t)(a2 * g.o * g.c) * 6);
    L.v_bytes = align256((size_t)(a2 * t * g.c) * 6);
    L.m_bytes = align256((size_t)(a2 * t * g.o) * 4);
    return L;
  }
  const int esz = dtype_size(store);
  L.per_img = (size_t)(a2 * L.tiles_per_img) * ((size_t)g.c * esz + (size_t)g.o * (cmajor ? 4 : esz));
  const long long t = chunk > 0 ? std::min(nb * L.tiles_per_img, chunk) : nb * L.tiles_per_img;
  if (cmajor) {
    L.u_bytes = align256((size_t)(a2 * g.c * round4(g.o)) * esz);
    L.v_bytes = align256((size_t)(a2 * g.c * ((kF32VTileMajor && g.c % 4 == 0) ? t : round4(t))) * esz);
    if (chunk > 0) L.v_bytes *= 2;   // two V buffers: chunk i+1 is transformed while chunk i's GEMM drains
  } else {
    L.u_bytes = align256((size_t)(a2 * g.o * g.c) * esz);
    L.v_bytes = align256((size_t)(a2 * t * g.c) * esz);
  }
  L.m_bytes = align256((size_t)(a2 * t * g.o) * (cmajor ? 4 : esz));
  return L;
}

// The persistent fp32 Winograd kernel (transforms overlapped with the FFMA
// GEMM inside each CTA) against the three-launch path: it needs F(6x6,3x3)
// with fp32 input and tile-major V.  On the 40 x 512 x 512, 192 -> 96 case it
// measured 18.2 against 18.4 ms for the three launches (one run each on one
// B200), a gain inside run-to-run spread for 2.8 GB of per-CTA scratch, so
// it runs only when B200CONV_WINOGRAD_FUSED=1 (a test hook, read on every
// call; =0 or unset keeps the three launches).  kFusedMinBlocksPerSm is the
// rule it would take by default: enough 128-tile blocks that every SM gets at
// least eight (its first input transform and last output transform are not
// overlapped).
constexpr bool kFusedByDefault = false;
constexpr long long kFusedMinBlocksPerSm = 8;
bool winograd_fused_wanted(const Geom& g, conv_dtype_t dt, int m, long long tiles, const conv_device_props_t& p) {
  if (dt != CONV_F32 || m != 6 || !kF32VTileMajor || !wino_fused_f32_shape_ok(g)) return false;
  if (const char* e = std::getenv("B200CONV_WINOGRAD_FUSED")) {
    if (std::strcmp(e, "0") == 0) return false;
    if (std::strcmp(e, "1") == 0) return true;
  }
  return kFusedByDefault && wino_fused_f32_blocks(tiles) >= kFusedMinBlocksPerSm * p.sm_count;
}

// Tiles per chunk of the fp32 Winograd pass (FFMA GEMM, tile-major V).  0
// keeps the whole batch tile in one pass.  B200CONV_WINOGRAD_CHUNK_TILES
// overrides it (a test hook, read on every call).
long long winograd_chunk_tiles(const Geom& g, int m, const conv_device_props_t& p) {
  (void)g; (void)m; (void)p;
  if (const char* e = std::getenv("B200CONV_WINOGRAD_CHUNK_TILES")) return std::max(0LL, std::atoll(e));
  return 0;
}

// The fp32 Winograd GEMM on the tensor cores over split-bf16 operands: each fp32
// value is the exact sum of three bf16 parts, and the six products a_i b_j with
// i + j <= 2 are accumulated in fp32 (TMEM), which keeps fp32 accuracy (the
// dropped products are below 2^-24 of the result).
// It needs F(6x6,3x3), a tcgen05 device, C a multiple of 64 and O of 4.
// B200CONV_WINOGRAD_SPLIT_BF16=1 turns it on (a test hook read on every call).
bool winograd_split_wanted(const Geom& g, conv_dtype_t dt, int m, const conv_device_props_t& p) {
  if (dt != CONV_F32 || m != 6 || p.cc_major != 10 || g.c % 64 != 0 || g.o % 4 != 0) return false;
  if (const char* f = std::getenv("B200CONV_WINOGRAD_FUSED"))
    if (std::strcmp(f, "1") == 0) return false;
  const char* e = std::getenv("B200CONV_WINOGRAD_SPLIT_BF16");
  return e && std::strcmp(e, "1") == 0;
}

conv_status_t select2d(const Geom& g, conv_dtype_t dt, const conv_device_props_t& p,
                       const conv_options_t& o, Sel* s) {
  const int esz = dtype_size(dt);
  const bool wshape = winograd_shape(g);
  bool want_wino = false;
  if (o.algo == CONV_ALGO_WINOGRAD) {
    if (!wshape) return CONV_ERR_UNSUPPORTED;
    want_wino = true;
  } else if (o.algo == CONV_ALGO_AUTO) {
    want_wino = wshape && winograd_channel_rule(g) && (dt == CONV_F32 || winograd_16bit_wins(g));
  } else if (o.algo != CONV_ALGO_IMPLICIT_GEMM && o.algo != CONV_ALGO_DIRECT) {
    return CONV_ERR_INVALID;
  }

  if (want_wino && g.n > 0) {
    const int m = winograd_m_for(dt);
    // 16-bit operands go to the tensor cores when their rows meet the
    // 16-byte rule, else the transforms store fp32 for the FFMA engine.
    const bool split = winograd_split_wanted(g, dt, m, p);
    const bool tc_gemm = split || (dt != CONV_F32 && p.cc_major == 10 && g.c % 8 == 0);
    const conv_dtype_t store = split ? CONV_BF16 : ((dt == CONV_F32 || !tc_gemm) ? CONV_F32 : dt);
    const WinoLayout L1 = winograd_layout(g, store, !tc_gemm, m, 1, 0, split);
    const size_t u_bytes = L1.u_bytes, per_img = L1.per_img;
    const long long tiles_per_img = L1.tiles_per_img;
    long long budget;
    if (o.winograd_budget_bytes >= 0) {
      budget = o.winograd_budget_bytes;
    } else {
      const long long own = (long long)g.n * g.h * g.w * g.c * esz + (long long)g.n * g.oh * g.ow * g.o * esz +
                            (long long)u_bytes;
      budget = std::min((long long)(p.total_global_mem / 4 * 3) - own, kWinogradCap);
    }
    long long nb = budget > 0 ? budget / (long long)per_img : 0;
    nb = std::min<long long>(nb, g.n);
    const bool forced_tile = o.winograd_tile_batch > 0;
    if (forced_tile) nb = std::min<long long>(nb, o.winograd_tile_batch);
    // The persistent fp32 kernel: per-CTA scratch in place of the batch tile's V and M
    if (!forced_tile && !tc_gemm && winograd_fused_wanted(g, dt, m, (long long)g.n * tiles_per_img, p)) {
      const long long blocks = wino_fused_f32_blocks((long long)g.n * tiles_per_img);
      int grid = (int)std::min<long long>(p.sm_count, blocks);
      // B200CONV_WINOGRAD_FUSED_GRID=<ctas> (a test hook) runs fewer CTAs, each taking more blocks
      if (const char* e = std::getenv("B200CONV_WINOGRAD_FUSED_GRID"))
        if (std::atoi(e) > 0) grid = (int)std::min<long long>(std::atoi(e), blocks);
      const size_t scratch = align256((size_t)grid * wino_fused_f32_cta_bytes(g.c, g.o));
      if ((long long)scratch <= budget) {
        s->algo = CONV_ALGO_WINOGRAD;
        s->engine = CONV_ENGINE_SIMT;
        s->wino_m = m;
        s->wino_store = store;
        s->nb = g.n;
        s->ntiles = 1;
        s->tile_n = wino_gemm_f32_tile_n(g.o);
        s->tile_m = 128;
        s->chunk = 0;
        s->fused = true;
        s->fused_grid = grid;
        s->ws = u_bytes + scratch;
        s->cpad = 0;
        return CONV_OK;
      }
    }
    // Batch-tiled, each tile's point GEMMs run as one batched launch of
    // alpha^2 GEMMs.  On the FFMA engine a few full 128-row tiles per point are
    // enough, since its alternative (the FFMA implicit GEMM) is far slower: on
    // 40 x 512 x 512, 192 -> 96, 1-image tiles took 19.5 ms against 18.6
    // untiled and 76.9 ms for the implicit GEMM.  The tensor-core path keeps a
    // full wave of rows per point before it prefers Winograd over its implicit GEMM.
    const long long r_min = (tc_gemm && !split) ? (long long)p.sm_count * 128 : 4 * 128;
    bool fallback = nb <= 0 || (!forced_tile && nb < g.n && nb * tiles_per_img < r_min);
    if (fallback && o.algo == CONV_ALGO_WINOGRAD) return CONV_ERR_UNSUPPORTED;
    if (!fallback) {
      s->algo = CONV_ALGO_WINOGRAD;
      s->engine = tc_gemm ? CONV_ENGINE_TCGEN05 : CONV_ENGINE_SIMT;
      s->wino_m = m;
      s->wino_store = store;
      s->nb = (int)nb;
      s->ntiles = (int)((g.n + nb - 1) / nb);
      s->tile_n = split ? (g.o <= 96 ? 96 : 128)
                  : tc_gemm ? (g.o <= 128 ? 128 : 256) : wino_gemm_f32_tile_n(g.o);
      s->tile_m = tc_gemm && !split && tc_pair_tiles(nb * tiles_per_img, (long long)(m + 2) * (m + 2), g.o,
                                                     s->tile_n, (g.c + 63) / 64, p) ? 256 : 128;
      s->chunk = (!tc_gemm && kF32VTileMajor && g.c % 4 == 0) ? winograd_chunk_tiles(g, m, p) : 0;
      s->split_bf16 = split;
      const WinoLayout L = winograd_layout(g, store, !tc_gemm, m, nb, s->chunk, split);
      s->ws = L.u_bytes + L.v_bytes + L.m_bytes;
      s->cpad = 0;
      return CONV_OK;
    }
  }

  // Implicit GEMM (or the direct SIMT path).
  s->algo = o.algo == CONV_ALGO_DIRECT ? CONV_ALGO_DIRECT : CONV_ALGO_IMPLICIT_GEMM;
  s->wino_m = 0;
  s->nb = g.n;
  s->ntiles = 1;
  s->cpad = 0;
  s->ws = 0;
  if (s->algo == CONV_ALGO_IMPLICIT_GEMM && tc_shape_ok(g, dt, p)) {
    s->engine = CONV_ENGINE_TCGEN05;
    s->tile_m = 128;
    s->tile_n = tc_tile_n(g, p);
    s->wpack = false;
    s->fpack = false;
    if (g.c % 8 != 0 && g.kh * g.kw > 1 && g.kh * g.kw * g.c <= 192) {
      // a few channels and a small window: fold every tap into channels, the
      // conv becoming a 1x1 conv over at most 3 full K steps (the ResNet stem's
      // 7x7x3 = 147 -> 152 channels), instead of KH K steps of mostly padding
      const int cp = (g.kh * g.kw * g.c + 7) / 8 * 8;
      s->cpad = cp;
      s->fpack = true;
      s->ws = align256((size_t)g.n * g.oh * g.ow * cp * esz) + align256((size_t)g.o * cp * esz);
    } else if (g.c % 8 != 0 && g.kw > 1 && g.kw * g.c <= 64) {
      // a few channels: fold the KW taps into channels (KH x 1 conv over KW*C)
      const int cp = (g.kw * g.c + 7) / 8 * 8;
      s->cpad = cp;
      s->wpack = true;
      s->ws = align256((size_t)g.n * g.h * g.ow * cp * esz) + align256((size_t)g.o * g.kh * cp * esz);
    } else if (g.c % 8 != 0) {
      const int cp = (g.c + 7) / 8 * 8;
      s->cpad = cp;
      s->ws = align256((size_t)g.n * g.h * g.w * cp * esz) + align256((size_t)g.o * g.kh * g.kw * cp * esz);
    }
  } else {
    s->engine = CONV_ENGINE_SIMT;
    s->tile_m = 128;
    s->tile_n = g.o <= 64 ? 64 : (g.o <= 96 ? 96 : 128);
    s->wpack = false;
    if (s->algo == CONV_ALGO_IMPLICIT_GEMM && g.c <= 8 && g.kw > 1 && g.kw * g.c <= 64) {
      // a few channels: fold the KW taps into channels for the 16-wide k chunks too
      const int cp = (g.kw * g.c + 7) / 8 * 8;
      s->cpad = cp;
      s->wpack = true;
      s->ws = align256((size_t)g.n * g.h * g.ow * cp * esz) + align256((size_t)g.o * g.kh * cp * esz);
    }
  }
  // Split-K for grids under half a wave with a long K loop: each split writes
  // fp32 partials, reduced in a fixed order (deterministic for a given plan).
  const long long M = (long long)g.n * g.oh * g.ow;
  if (s->algo == CONV_ALGO_IMPLICIT_GEMM && M > 0) {
    const int c_eff = s->cpad ? s->cpad : g.c;
    const long long taps = s->fpack ? 1 : (s->wpack ? g.kh : (long long)g.kh * g.kw);
    long long ks = 1;
    if (s->engine == CONV_ENGINE_TCGEN05) {
      const long long ksteps = taps * ((c_eff + 63) / 64);
      const long long tiles = ((M + 127) / 128) * ((g.o + s->tile_n - 1) / s->tile_n);
      if (tiles * 2 <= p.sm_count && ksteps >= 16) ks = std::min({(long long)p.sm_count / tiles, ksteps / 4, 16LL});
    } else {
      const long long steps = taps * ((c_eff + 15) / 16);
      const long long blocks = ((M + 127) / 128) * ((g.o + s->tile_n - 1) / s->tile_n);
      if (blocks * 2 <= p.sm_count && steps >= 16) ks = std::min({(long long)p.sm_count / blocks, steps / 8, 16LL});
    }
    if (ks >= 2) {
      s->ksplit = (int)ks;
      s->split_off = s->ws;
      s->ws += align256((size_t)ks * M * g.o * 4);
      // arrival counters of the serial in-kernel reduction: one per (128-row tile,
      // column tile, epilogue warp)
      if (s->engine == CONV_ENGINE_TCGEN05)
        s->ws += align256((size_t)((M + 127) / 128) * ((g.o + s->tile_n - 1) / s->tile_n) * 4 * sizeof(int));
    }
    if (s->engine == CONV_ENGINE_TCGEN05 && s->ksplit == 1 && !s->wpack && !s->fpack &&
        tc_pair_tiles(M, 1, g.o, s->tile_n, taps * ((c_eff + 63) / 64), p))
      s->tile_m = 256;
  }
  return CONV_OK;
}

void fill_plan(const Sel& s, conv_plan_t* plan, int taps, size_t ws) {
  plan->algo = s.algo;
  plan->engine = s.engine;
  plan->tile_m = s.tile_m;
  plan->tile_n = s.tile_n;
  plan->winograd_m = s.wino_m;
  plan->batch_tile = s.nb;
  plan->num_batch_tiles = s.ntiles;
  plan->channel_pad = s.cpad;
  plan->packed_taps = s.fpack ? 2 : (s.wpack ? 1 : 0);
  plan->k_split = s.ksplit;
  plan->taps = taps;
  plan->winograd_fused = s.fused ? 1 : 0;
  plan->winograd_split_bf16 = s.split_bf16 ? 1 : 0;
  plan->workspace_bytes = ws;
}

// B200CONV_LOG=1: one line per forward call on stderr with the plan that runs
// (read on every call, like the other environment hooks).
bool log_enabled() {
  const char* v = std::getenv("B200CONV_LOG");
  return v && v[0] && std::strcmp(v, "0") != 0;
}

const char* dtype_name(conv_dtype_t t) { return t == CONV_F32 ? "f32" : (t == CONV_F16 ? "f16" : "bf16"); }
const char* algo_name(conv_algo_t a) {
  switch (a) {
    case CONV_ALGO_IMPLICIT_GEMM: return "implicit";
    case CONV_ALGO_WINOGRAD: return "winograd";
    case CONV_ALGO_DIRECT: return "direct";
    default: return "auto";
  }
}

void log_plan(const char* op, const char* shape, conv_dtype_t dt, const Sel& s, const char* path, size_t ws) {
  std::fprintf(stderr,
               "b200conv: %s %s %s -> algo=%s engine=%s path=%s tile=%dx%d winograd_m=%d batch_tile=%d "
               "batch_tiles=%d channel_pad=%d packed_taps=%d k_split=%d fused=%d split_bf16=%d workspace=%zu\n",
               op, shape, dtype_name(dt), algo_name(s.algo), s.engine == CONV_ENGINE_TCGEN05 ? "tcgen05" : "simt",
               path, s.tile_m, s.tile_n, s.wino_m, s.nb, s.ntiles, s.cpad, s.fpack ? 2 : (s.wpack ? 1 : 0), s.ksplit,
               s.fused ? 1 : 0, s.split_bf16 ? 1 : 0, ws);
}

// ------------------------------- execution -----------------------------------

conv_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? CONV_OK : CONV_ERR_CUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
// The workspace's sub-buffers sit at 256-byte offsets from its base and are
// read by TMA and 16-byte copies, so the base itself must be 256-byte aligned.
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

// Run one planned 2D conv.  ws holds at least s.ws bytes.  accumulate: add the
// result into out (out = round(out + round(result))), the depth-tap sum fused
// into the conv's output stage.
conv_status_t run2d(const void* in, const void* w, void* out, const Geom& g, conv_dtype_t dt, const Sel& s,
                    void* ws, const DeviceState& d, cudaStream_t st, bool accumulate = false) {
  if (g.n == 0) return CONV_OK;
  if (s.algo == CONV_ALGO_WINOGRAD) {
    const int m = s.wino_m, a2 = (m + 2) * (m + 2);
    const bool cmajor = s.engine == CONV_ENGINE_SIMT;
    const WinoLayout L = winograd_layout(g, s.wino_store, cmajor, m, s.nb, s.chunk, s.split_bf16);
    uint8_t* base = static_cast<uint8_t*>(ws);
    void* u = base;
    void* v = base + L.u_bytes;
    void* mb = base + L.u_bytes + L.v_bytes;
    const conv_dtype_t m_dt = (cmajor || s.split_bf16) ? CONV_F32 : s.wino_store;
    cudaError_t e;
    {
      ProfScope ps(K_WINO_FILTER, st);
      e = s.split_bf16 ? launch_wino_filter_split(static_cast<const float*>(w), g.w_row_stride, g.o, g.c, u, st)
          : cmajor ? launch_wino_filter_cmajor(w, g.w_row_stride, g.o, g.c, m, dt, round4(g.o), static_cast<float*>(u), st)
                   : launch_wino_filter(w, g.w_row_stride, g.o, g.c, m, dt, s.wino_store, u, st);
    }
    if (e != cudaSuccess) return CONV_ERR_CUDA;
    if (s.fused) {
      // one persistent launch: per-CTA V and M scratch right after U
      ProfScope ps(K_WINO_FUSED, st);
      e = launch_wino_fused_f32(static_cast<const float*>(in), g, static_cast<const float*>(u), round4(g.o),
                                static_cast<float*>(out), reinterpret_cast<float*>(base + L.u_bytes), s.fused_grid,
                                accumulate, d.err_word, st);
      return e == cudaSuccess ? CONV_OK : CONV_ERR_CUDA;
    }
    const bool tmajor = kF32VTileMajor && g.c % 4 == 0;
    if (s.chunk > 0) {
      // Chunked pipeline: per batch tile, chunks of at most s.chunk tiles, so V
      // and M stay in L2 between the kernels.  Pass k transforms the output of
      // chunk k-1 and the input of chunk k in one launch; the GEMM of chunk k
      // sits between passes k and k+1.  V alternates between two buffers.
      struct Chunk { long long t0, t; };
      std::vector<Chunk> chunks;
      for (int n0 = 0; n0 < g.n; n0 += s.nb) {
        const long long t_all = (long long)std::min(s.nb, g.n - n0) * L.tiles_per_img;
        for (long long tb = 0; tb < t_all; tb += s.chunk)
          chunks.push_back({(long long)n0 * L.tiles_per_img + tb, std::min(s.chunk, t_all - tb)});
      }
      float* vbuf[2] = {static_cast<float*>(v), static_cast<float*>(v) + L.v_bytes / 2 / sizeof(float)};
      const size_t nc = chunks.size();
      for (size_t k = 0; k <= nc; ++k) {
        const Chunk in_c = k < nc ? chunks[k] : Chunk{0, 0};
        const Chunk out_c = k > 0 ? chunks[k - 1] : Chunk{0, 0};
        {
          ProfScope ps(K_WINO_PASS, st);
          // the first pass waits for everything before it in the stream
          e = launch_wino_pass(in, g, m, dt, 0, in_c.t0, in_c.t, vbuf[k & 1], out_c.t0, out_c.t,
                               static_cast<const float*>(mb), out, accumulate, k > 0, st);
        }
        if (e != cudaSuccess) return CONV_ERR_CUDA;
        if (k < nc) {
          ProfScope ps(K_WINO_GEMM_SIMT, st);
          e = launch_wino_gemm_f32(vbuf[k & 1], static_cast<const float*>(u), static_cast<float*>(mb), a2,
                                   (int)in_c.t, g.c, g.o, g.c, round4(g.o), true, st);
          if (e != cudaSuccess) return CONV_ERR_CUDA;
        }
      }
      return CONV_OK;
    }
    for (int n0 = 0; n0 < g.n; n0 += s.nb) {
      const int nbi = std::min(s.nb, g.n - n0);
      const long long t_all = (long long)nbi * L.tiles_per_img;
      {
        const long long tb = 0, t = t_all;
        {
          ProfScope ps(K_WINO_INPUT, st);
          if (s.split_bf16)
            e = launch_wino_input_split(static_cast<const float*>(in), g, n0, t, v, t, st);
          else if (cmajor && !tmajor)
            e = launch_wino_input_cmajor(in, g, n0, nbi, m, dt, static_cast<float*>(v), round4(t), st);
          else
            e = launch_wino_input(in, g, n0, tb, t, m, dt, s.wino_store, v, t, st);
        }
        if (e != cudaSuccess) return CONV_ERR_CUDA;
        if (cmajor) {
          ProfScope ps(K_WINO_GEMM_SIMT, st);
          e = launch_wino_gemm_f32(static_cast<const float*>(v), static_cast<const float*>(u), static_cast<float*>(mb),
                                   a2, (int)t, g.c, g.o, tmajor ? g.c : round4(t), round4(g.o), tmajor, st);
        } else {
          BatchedGemm bg{a2, (int)t, g.c, g.o, v, u, mb, m_dt};
          bg.split_bf16 = s.split_bf16;
          ProfScope ps(K_WINO_GEMM_TC, st);
          e = launch_tc_batched_gemm(bg, s.wino_store, s.tile_n, d.props.sm_count, d.err_word, st, s.tile_m);
        }
        if (e != cudaSuccess) return CONV_ERR_CUDA;
        {
          ProfScope ps(K_WINO_OUTPUT, st);
          e = launch_wino_output(mb, m_dt, g, n0, tb, t, m, t, dt, out, accumulate, st);
        }
        if (e != cudaSuccess) return CONV_ERR_CUDA;
      }
    }
    return CONV_OK;
  }
  // Implicit GEMM / direct: optional pre-pass (tap packing or channel pad),
  // the GEMM engine, and the split-K reduction.
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int esz = dtype_size(dt);
  const void* cin = in;
  const void* cw = w;
  Geom gg = g;
  if (s.fpack) {
    void* pin = base;
    void* pw = base + align256((size_t)g.n * g.oh * g.ow * s.cpad * esz);
    cudaError_t e;
    {
      ProfScope ps(K_CHANNEL_PAD, st);
      e = launch_fullpack(in, g, pin, s.cpad, dt, d.props.sm_count, st);
    }
    if (e == cudaSuccess) {
      // w[o][kh][kw][c]: rows of KH*KW*C values -> [o][cp]
      ProfScope ps(K_CHANNEL_PAD, st);
      e = launch_channel_pad(w, g.o, 1, g.kh * g.kw * g.c, g.w_row_stride, pw, s.cpad, dt, st);
    }
    if (e != cudaSuccess) return CONV_ERR_CUDA;
    cin = pin;
    cw = pw;
    gg.h = g.oh;
    gg.w = g.ow;
    gg.c = s.cpad;
    gg.kh = gg.kw = 1;
    gg.sh = gg.sw = 1;
    gg.ph = gg.pw = 0;
    gg.dh = gg.dw = 1;
    gg.in_img_stride = (long long)g.oh * g.ow * s.cpad;
    gg.w_row_stride = s.cpad;
  } else if (s.wpack) {
    void* pin = base;
    void* pw = base + align256((size_t)g.n * g.h * g.ow * s.cpad * esz);
    cudaError_t e;
    {
      ProfScope ps(K_CHANNEL_PAD, st);
      e = launch_wpack(in, g.n, g.h, g.w, g.c, g.kw, g.sw, g.pw, g.dw, g.ow, g.in_img_stride, pin, s.cpad, dt, st);
    }
    if (e == cudaSuccess) {
      // w[o][kh][kw][c] rows of KW*C channels -> [o][kh][cp]
      ProfScope ps(K_CHANNEL_PAD, st);
      e = launch_channel_pad(w, g.o, g.kh, g.kw * g.c, g.w_row_stride, pw, s.cpad, dt, st);
    }
    if (e != cudaSuccess) return CONV_ERR_CUDA;
    cin = pin;
    cw = pw;
    gg.w = g.ow;
    gg.c = s.cpad;
    gg.kw = 1;
    gg.sw = 1;
    gg.pw = 0;
    gg.dw = 1;
    gg.in_img_stride = (long long)g.h * g.ow * s.cpad;
    gg.w_row_stride = (long long)g.kh * s.cpad;
  } else if (s.cpad) {
    void* pin = base;
    void* pw = base + align256((size_t)g.n * g.h * g.w * s.cpad * esz);
    cudaError_t e;
    {
      ProfScope ps(K_CHANNEL_PAD, st);
      e = launch_channel_pad(in, g.n, (long long)g.h * g.w, g.c, g.in_img_stride, pin, s.cpad, dt, st);
    }
    if (e == cudaSuccess) {
      ProfScope ps(K_CHANNEL_PAD, st);
      e = launch_channel_pad(w, g.o, (long long)g.kh * g.kw, g.c, g.w_row_stride, pw, s.cpad, dt, st);
    }
    if (e != cudaSuccess) return CONV_ERR_CUDA;
    cin = pin;
    cw = pw;
    gg.c = s.cpad;
    gg.in_img_stride = (long long)g.h * g.w * s.cpad;
    gg.w_row_stride = (long long)g.kh * g.kw * s.cpad;
  }
  float* partial = s.ksplit > 1 ? reinterpret_cast<float*>(base + s.split_off) : nullptr;
  bool done = false, reduced = false;
  if (s.engine == CONV_ENGINE_TCGEN05 && tc_conv_supported(gg, dt, cin, cw)) {
    // Split-K partials go through the workspace to the reduce kernel.  The
    // in-kernel cluster reduction (B200CONV_SPLITK_CLUSTER=1, a test hook read
    // on every call) gives the same bits but measured 4-7 % slower on the
    // ResNet-50 layer set: the small split tiles finish faster than a cluster
    // barrier plus distributed-shared-memory sums.
    const char* sc = std::getenv("B200CONV_SPLITK_CLUSTER");
    const bool cluster_ok = sc && std::strcmp(sc, "1") == 0;
    // The serial in-kernel reduction (B200CONV_SPLITK_SERIAL=1, a test hook read
    // on every call): the last-arriving split of each tile sums the partials;
    // its counters are cleared before the launch.
    const char* ss = std::getenv("B200CONV_SPLITK_SERIAL");
    int* counters = nullptr;
    if (s.ksplit > 1 && ss && std::strcmp(ss, "1") == 0) {
      const long long Mr = (long long)g.n * g.oh * g.ow;
      const size_t n_cnt = (size_t)((Mr + 127) / 128) * ((g.o + s.tile_n - 1) / s.tile_n) * 4;
      counters = reinterpret_cast<int*>(base + s.split_off + align256((size_t)s.ksplit * Mr * g.o * 4));
      if (cudaMemsetAsync(counters, 0, n_cnt * sizeof(int), st) != cudaSuccess) return CONV_ERR_CUDA;
    }
    ProfScope ps(K_TC_CONV, st);
    if (launch_tc_conv(cin, cw, out, gg, dt, s.tile_n, d.props.sm_count, d.err_word, accumulate, st, s.ksplit,
                       partial, (cluster_ok || counters) ? &reduced : nullptr, s.tile_m, counters) != cudaSuccess)
      return CONV_ERR_CUDA;
    done = true;
  }
  if (!done) {
    // FFMA engine, or misaligned pointers on the tensor-core plan: the any-alignment path
    const bool vec = s.algo != CONV_ALGO_DIRECT && gg.c % 4 == 0 && (gg.in_img_stride % 4 == 0) &&
                     (gg.w_row_stride % 4 == 0) && aligned16(cin) && aligned16(cw);
    ProfScope ps(K_SIMT_CONV, st);
    if (launch_simt_conv(cin, cw, out, gg, dt, vec, accumulate, st, s.ksplit, partial) != cudaSuccess)
      return CONV_ERR_CUDA;
  }
  if (s.ksplit > 1 && !reduced) {
    ProfScope ps(K_SPLITK_REDUCE, st);
    if (launch_splitk_reduce(partial, s.ksplit, (size_t)g.n * g.oh * g.ow * g.o, out, dt, accumulate, st) !=
        cudaSuccess)
      return CONV_ERR_CUDA;
  }
  return CONV_OK;
}

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  if (!a || !b || an == 0 || bn == 0) return false;
  uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + bn && y < x + an;
}

// ------------------------------- conv3d --------------------------------------

struct Tap {
  int kd, od_lo, od_hi, id_lo;   // output frames od_lo..od_hi read input frame id_lo + (od - od_lo) * sd
};

conv_status_t geom3d(const conv3d_desc_t* d, long long* od, Geom* g2) {
  if (!d) return CONV_ERR_INVALID;
  if (d->n < 0 || d->d <= 0 || d->h <= 0 || d->w <= 0 || d->c <= 0 || d->o <= 0 || d->kd <= 0 || d->kh <= 0 ||
      d->kw <= 0)
    return CONV_ERR_INVALID;
  for (int i = 0; i < 3; ++i)
    if (d->stride[i] <= 0 || d->dilation[i] <= 0 || d->pad[i] < 0) return CONV_ERR_INVALID;
  *od = out_extent(d->d, d->kd, d->stride[0], d->pad[0], d->dilation[0]);
  if (*od <= 0 || *od > (1 << 30)) return CONV_ERR_INVALID;
  // The 2D problem of one depth tap: "images" are output frames.
  conv2d_desc_t d2{};
  d2.n = (int)*od; d2.h = d->h; d2.w = d->w; d2.c = d->c; d2.o = d->o; d2.kh = d->kh; d2.kw = d->kw;
  d2.stride[0] = d->stride[1]; d2.stride[1] = d->stride[2];
  d2.pad[0] = d->pad[1]; d2.pad[1] = d->pad[2];
  d2.dilation[0] = d->dilation[1]; d2.dilation[1] = d->dilation[2];
  conv_status_t st = geom2d(&d2, g2);
  if (st != CONV_OK) return st;
  g2->in_img_stride = (long long)d->stride[0] * d->h * d->w * d->c;            // frame view stride
  g2->w_row_stride = (long long)d->kd * d->kh * d->kw * d->c;                  // weight slice rows
  return CONV_OK;
}

int taps3d(const conv3d_desc_t* d, long long od, Tap* taps) {
  int n = 0;
  for (int kd = 0; kd < d->kd; ++kd) {
    const long long off = (long long)kd * d->dilation[0] - d->pad[0];   // id = od*sd + off
    long long lo = off >= 0 ? 0 : (-off + d->stride[0] - 1) / d->stride[0];
    long long hi = (d->d - 1 - off) >= 0 ? (d->d - 1 - off) / d->stride[0] : -1;
    hi = std::min(hi, od - 1);
    if (lo > hi) continue;
    taps[n++] = Tap{kd, (int)lo, (int)hi, (int)(lo * d->stride[0] + off)};
  }
  return n;
}

Geom3 geom3_of(const conv3d_desc_t* d, long long od, const Geom& g2) {
  Geom3 g{};
  g.n = d->n; g.d = d->d; g.h = d->h; g.w = d->w; g.c = d->c; g.o = d->o;
  g.kd = d->kd; g.kh = d->kh; g.kw = d->kw;
  g.sd = d->stride[0]; g.sh = d->stride[1]; g.sw = d->stride[2];
  g.pd = d->pad[0]; g.ph = d->pad[1]; g.pw = d->pad[2];
  g.dd = d->dilation[0]; g.dh = d->dilation[1]; g.dw = d->dilation[2];
  g.od = (int)od; g.oh = g2.oh; g.ow = g2.ow;
  return g;
}

// The depth-tap page's guard ("Decompose small kernel-depth 3D convs into 2D
// convs", Change): N == 1, KD <= 7, depth stride 1, kernel dilation 1, no depth
// padding, channel counts that are multiples of 16.
bool depth_tap_guard(const conv3d_desc_t* d) {
  return d->n == 1 && d->kd <= 7 && d->stride[0] == 1 && d->dilation[0] == 1 && d->dilation[1] == 1 &&
         d->dilation[2] == 1 && d->pad[0] == 0 && d->c % 16 == 0 && d->o % 16 == 0;
}

// The native 3D implicit GEMM can express this shape (pointers are checked at launch).
bool native3d_shape_ok(const Geom3& g, conv_dtype_t dt, const conv_device_props_t& p) {
  if (dt == CONV_F32 || p.cc_major != 10 || g.c % 8 != 0) return false;
  if (g.sd > 8 || g.sh > 8 || g.sw > 8) return false;
  const int lo[3] = {-g.pw, -g.ph, -g.pd};
  const int up[3] = {g.pw - g.dw * (g.kw - 1), g.ph - g.dh * (g.kh - 1), g.pd - g.dd * (g.kd - 1)};
  for (int i = 0; i < 3; ++i)
    if (lo[i] < -16 || lo[i] > 15 || up[i] < -16 || up[i] > 15) return false;
  return (long long)g.dw * (g.kw - 1) <= 65535 && (long long)g.dh * (g.kh - 1) <= 65535 &&
         (long long)g.dd * (g.kd - 1) <= 65535;
}

// Native 3D Winograd F(m^3, 3^3): 3x3x3 kernels, stride 1, dilation 1, any
// padding.  fp32 takes F(4,3) along each axis (alpha^3 = 216); 16-bit takes
// F(2,3) (alpha^3 = 64), whose transforms keep bf16 inside its tolerance.
bool wino3d_shape(const conv3d_desc_t* d) {
  for (int i = 0; i < 3; ++i)
    if (d->stride[i] != 1 || d->dilation[i] != 1) return false;
  return d->kd == 3 && d->kh == 3 && d->kw == 3;
}
int wino3d_m_for(conv_dtype_t dt) { return dt == CONV_F32 ? 4 : 2; }

// Workspace of the 3D Winograd path for batch tiles of nu units, a unit being
// one (image, depth tile) slab of tiles_hw tiles:
//   tensor-core GEMM (16-bit operands): U [a3][O][C], V [a3][T][C], M [a3][T][O] fp32
//   FFMA GEMM (fp32 operands):          U [a3][C][O4], V [a3][T][C], M [a3][T][O] fp32
struct Wino3Layout {
  size_t u_bytes = 0, v_bytes = 0, m_bytes = 0;
  long long tiles_hw = 0, units = 0;
  size_t per_unit = 0;   // V + M bytes per unit (the budget unit)
};

Wino3Layout wino3d_layout(const Geom3& g, conv_dtype_t store, bool ffma, int m, long long nu) {
  Wino3Layout L;
  const long long a3 = (long long)(m + 2) * (m + 2) * (m + 2);
  L.tiles_hw = (long long)((g.oh + m - 1) / m) * ((g.ow + m - 1) / m);
  L.units = (long long)g.n * ((g.od + m - 1) / m);
  const int esz = dtype_size(store);
  L.per_unit = (size_t)(a3 * L.tiles_hw) * ((size_t)g.c * esz + (size_t)g.o * 4);
  const long long t = nu * L.tiles_hw;
  L.u_bytes = align256((size_t)(a3 * g.c * (ffma ? round4(g.o) : g.o)) * esz);
  L.v_bytes = align256((size_t)(a3 * t * g.c) * esz);
  L.m_bytes = align256((size_t)(a3 * t * g.o) * 4);
  return L;
}

// The Winograd selection of select2d with units in place of images.  Returns
// true and fills s when the 3D Winograd runs.
bool select_wino3d(const conv3d_desc_t* d, const Geom3& g, conv_dtype_t dt, const conv_device_props_t& p,
                   const conv_options_t& o, Sel* s) {
  if (!wino3d_shape(d) || g.n == 0 || g.c % 4 != 0) return false;
  if (o.algo == CONV_ALGO_AUTO) {
    if (dt != CONV_F32 || g.c % 32 != 0 || g.o % 32 != 0 || g.c + g.o < 256) return false;
  } else if (o.algo != CONV_ALGO_WINOGRAD) {
    return false;
  }
  const int m = wino3d_m_for(dt);
  const bool tc_gemm = dt != CONV_F32 && p.cc_major == 10 && g.c % 8 == 0;
  const conv_dtype_t store = tc_gemm ? dt : CONV_F32;
  const Wino3Layout L1 = wino3d_layout(g, store, !tc_gemm, m, 1);
  const int esz = dtype_size(dt);
  long long budget;
  if (o.winograd_budget_bytes >= 0) {
    budget = o.winograd_budget_bytes;
  } else {
    const long long own = (long long)g.n * g.d * g.h * g.w * g.c * esz +
                          (long long)g.n * g.od * g.oh * g.ow * g.o * esz + (long long)L1.u_bytes;
    budget = std::min((long long)(p.total_global_mem / 4 * 3) - own, kWinogradCap);
  }
  long long nu = budget > 0 ? budget / (long long)L1.per_unit : 0;
  nu = std::min<long long>(nu, L1.units);
  const bool forced_tile = o.winograd_tile_batch > 0;
  if (forced_tile) nu = std::min<long long>(nu, o.winograd_tile_batch);
  // A batch tile of nu units runs its alpha^3 point GEMMs in one batched launch
  // of nu * tiles_hw rows each, so the tile needs only a few full 128-row GEMM
  // tiles per point to fill the GPU (the 2D rule's full wave of rows per point
  // undercounts the launch by alpha^3).  Measured on 1 x 41 x 120 x 208,
  // 512 -> 512, fp32 under the 8 GiB cap: 6-unit tiles (9,360 rows) 35.2 ms
  // against 55.5 ms for its depth taps.
  const long long rows_min = 4 * 128;
  if (nu <= 0 || (!forced_tile && nu < L1.units && nu * L1.tiles_hw < rows_min)) return false;
  // the same number of tiles, evened out (5 + 5 units measured 34.7 ms against
  // 35.2 for 6 + 4 on that case)
  if (!forced_tile && nu < L1.units) {
    const long long nt = (L1.units + nu - 1) / nu;
    nu = (L1.units + nt - 1) / nt;
  }
  s->algo = CONV_ALGO_WINOGRAD;
  s->engine = tc_gemm ? CONV_ENGINE_TCGEN05 : CONV_ENGINE_SIMT;
  s->wino_m = m;
  s->wino_store = store;
  s->nb = (int)nu;
  s->ntiles = (int)((L1.units + nu - 1) / nu);
  s->tile_m = 128;
  s->tile_n = tc_gemm ? (g.o <= 128 ? 128 : 256) : wino_gemm_f32_tile_n(g.o);
  s->cpad = 0;
  s->wpack = false;
  s->ksplit = 1;
  const Wino3Layout L = wino3d_layout(g, store, !tc_gemm, m, nu);
  s->ws = L.u_bytes + L.v_bytes + L.m_bytes;
  return true;
}

enum Path3d { P3_TAPS, P3_NATIVE, P3_WINO3D };

conv_status_t plan3d_impl(const conv3d_desc_t* d, conv_dtype_t dt, const conv_device_props_t& p,
                          const conv_options_t& o, Sel* s, Geom* g2, long long* od, size_t* ws_total,
                          Path3d* path) {
  if (!valid_dtype(dt)) return CONV_ERR_INVALID;
  conv_status_t st = geom3d(d, od, g2);
  if (st != CONV_OK) return st;
  const Geom3 g3 = geom3_of(d, *od, *g2);
  // fp32 3x3x3 stride-1 convs under the channel rule (or any dtype, forced):
  // the native 3D Winograd, when its workspace budget allows a full wave.
  if (select_wino3d(d, g3, dt, p, o, s)) {
    *path = P3_WINO3D;
    *ws_total = s->ws;
    return CONV_OK;
  }
  const bool can_native = native3d_shape_ok(g3, dt, p);
  // Auto: the page's guard keeps the depth taps; the cases it sends to a native
  // 3D kernel go to the K-fused tcgen05 implicit GEMM.  Forcing the implicit
  // GEMM asks for the native kernel whenever it can run the shape.
  const bool native = can_native && ((o.algo == CONV_ALGO_AUTO && !depth_tap_guard(d)) || o.algo == CONV_ALGO_IMPLICIT_GEMM);
  *path = native ? P3_NATIVE : P3_TAPS;
  if (native) {
    s->algo = CONV_ALGO_IMPLICIT_GEMM;
    s->engine = CONV_ENGINE_TCGEN05;
    s->tile_m = 128;
    const long long m_tiles = ((long long)d->n * *od * g2->oh * g2->ow + 127) / 128;
    s->tile_n = d->o <= 128 || m_tiles * ((d->o + 255) / 256) < p.sm_count ? 128 : 256;
    s->tile_m = tc_pair_tiles((long long)d->n * *od * g2->oh * g2->ow, 1, d->o, s->tile_n,
                              (long long)d->kd * d->kh * d->kw * ((d->c + 63) / 64), p) ? 256 : 128;
    s->wino_m = 0;
    s->nb = d->n;
    s->ntiles = 1;
    s->cpad = 0;
    s->ws = 0;
    *ws_total = 0;
    return CONV_OK;
  }
  st = select2d(*g2, dt, p, o, s);
  if (st != CONV_OK) return st;
  // Taps after the first add into out inside their own output stage: no tap scratch.
  *ws_total = s->ws;
  return CONV_OK;
}

// Run the planned 3D Winograd: the filter transform once, then per batch tile
// of s.nb units the input transform, the alpha^3 batched GEMMs and the output
// transform, all through one reused workspace.
conv_status_t run3d_winograd(const void* in, const void* w, void* out, const Geom3& g, conv_dtype_t dt, const Sel& s,
                             void* ws, const DeviceState& d, cudaStream_t st) {
  const int m = s.wino_m, a3 = (m + 2) * (m + 2) * (m + 2);
  const bool ffma = s.engine == CONV_ENGINE_SIMT;
  const Wino3Layout L = wino3d_layout(g, s.wino_store, ffma, m, s.nb);
  uint8_t* base = static_cast<uint8_t*>(ws);
  void* u = base;
  void* v = base + L.u_bytes;
  float* mb = reinterpret_cast<float*>(base + L.u_bytes + L.v_bytes);
  cudaError_t e;
  {
    ProfScope ps(K_WINO3D_FILTER, st);
    e = launch_wino3d_filter(w, g.o, g.c, m, dt, s.wino_store, ffma, round4(g.o), u, st);
  }
  if (e != cudaSuccess) return CONV_ERR_CUDA;
  for (long long u0 = 0; u0 < L.units; u0 += s.nb) {
    const long long nu = std::min<long long>(s.nb, L.units - u0);
    const long long t = nu * L.tiles_hw;
    if (t > 0x7fffffffLL) return CONV_ERR_UNSUPPORTED;
    {
      ProfScope ps(K_WINO3D_INPUT, st);
      e = launch_wino3d_input(in, g, u0, nu, m, dt, s.wino_store, v, t, st);
    }
    if (e != cudaSuccess) return CONV_ERR_CUDA;
    if (ffma) {
      ProfScope ps(K_WINO3D_GEMM_SIMT, st);
      e = launch_wino_gemm_f32(static_cast<const float*>(v), static_cast<const float*>(u), mb, a3, (int)t, g.c, g.o,
                               g.c, round4(g.o), true, st);
    } else {
      BatchedGemm bg{a3, (int)t, g.c, g.o, v, u, mb, CONV_F32};
      ProfScope ps(K_WINO3D_GEMM_TC, st);
      e = launch_tc_batched_gemm(bg, s.wino_store, s.tile_n, d.props.sm_count, d.err_word, st);
    }
    if (e != cudaSuccess) return CONV_ERR_CUDA;
    {
      ProfScope ps(K_WINO3D_OUTPUT, st);
      e = launch_wino3d_output(mb, g, u0, nu, m, t, dt, out, st);
    }
    if (e != cudaSuccess) return CONV_ERR_CUDA;
  }
  return CONV_OK;
}

}  // namespace
}  // namespace b200conv

using namespace b200conv;

extern "C" {

const char* conv_status_string(conv_status_t s) {
  switch (s) {
    case CONV_OK: return "ok";
    case CONV_ERR_INVALID: return "invalid argument";
    case CONV_ERR_UNSUPPORTED: return "unsupported by the requested algorithm";
    case CONV_ERR_ALIGNMENT: return "misaligned pointer";
    case CONV_ERR_WORKSPACE: return "workspace too small";
    case CONV_ERR_CUDA: return "CUDA error";
    case CONV_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

conv_status_t conv_device_props(int device, conv_device_props_t* props) {
  if (!props) return CONV_ERR_INVALID;
  DeviceState* d = nullptr;
  conv_status_t st = device_state(device, &d);
  if (st != CONV_OK) return st;
  *props = d->props;
  return CONV_OK;
}

conv_status_t conv2d_plan_for_props(const conv2d_desc_t* desc, conv_dtype_t dtype, const conv_device_props_t* props,
                                    const conv_options_t* opts, conv_plan_t* plan) {
  if (!props || !plan || !valid_dtype(dtype)) return CONV_ERR_INVALID;
  Geom g;
  conv_status_t st = geom2d(desc, &g);
  if (st != CONV_OK) return st;
  Sel s;
  st = select2d(g, dtype, *props, effective_options(opts), &s);
  if (st != CONV_OK) return st;
  fill_plan(s, plan, 1, s.ws);
  return CONV_OK;
}

conv_status_t conv2d_plan(const conv2d_desc_t* desc, conv_dtype_t dtype, int device, const conv_options_t* opts,
                          conv_plan_t* plan) {
  DeviceState* d = nullptr;
  conv_status_t st = device_state(device, &d);
  if (st != CONV_OK) return st;
  return conv2d_plan_for_props(desc, dtype, &d->props, opts, plan);
}

size_t conv2d_workspace_size(const conv2d_desc_t* desc, conv_dtype_t dtype, int device, const conv_options_t* opts) {
  conv_plan_t p;
  return conv2d_plan(desc, dtype, device, opts, &p) == CONV_OK ? p.workspace_bytes : 0;
}

conv_status_t conv2d_forward(const void* in, const void* w, void* out, const conv2d_desc_t* desc, conv_dtype_t dtype,
                             const conv_options_t* opts, void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_dtype(dtype)) return CONV_ERR_INVALID;
  Geom g;
  conv_status_t st = geom2d(desc, &g);
  if (st != CONV_OK) return st;
  if (g.n == 0) return CONV_OK;
  if (!in || !w || !out) return CONV_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CONV_ERR_CUDA;
  DeviceState* d = nullptr;
  st = device_state(dev, &d);
  if (st != CONV_OK) return st;
  Sel s;
  st = select2d(g, dtype, d->props, effective_options(opts), &s);
  if (st != CONV_OK) return st;
  const int esz = dtype_size(dtype);
  const size_t out_bytes = (size_t)g.n * g.out_img_stride * esz;
  if (overlaps(out, out_bytes, in, (size_t)g.n * g.in_img_stride * esz) ||
      overlaps(out, out_bytes, w, (size_t)g.o * g.w_row_stride * esz))
    return CONV_ERR_INVALID;
  if (workspace_bytes < s.ws || (s.ws > 0 && !workspace)) return CONV_ERR_WORKSPACE;
  if (s.ws > 0 && !aligned256(workspace)) return CONV_ERR_ALIGNMENT;
  if (overlaps(out, out_bytes, workspace, s.ws)) return CONV_ERR_INVALID;
  if (log_enabled()) {
    char shape[192];
    std::snprintf(shape, sizeof shape, "n%d %dx%d %d->%d k%dx%d s%d,%d p%d,%d d%d,%d", g.n, g.h, g.w, g.c, g.o, g.kh,
                  g.kw, g.sh, g.sw, g.ph, g.pw, g.dh, g.dw);
    log_plan("conv2d", shape, dtype, s, "2d", s.ws);
  }
  return run2d(in, w, out, g, dtype, s, workspace, *d, static_cast<cudaStream_t>(stream));
}

static bool desc2d_of(const conv1d_desc_t* d, conv2d_desc_t* d2) {
  if (!d) return false;
  *d2 = conv2d_desc_t{};
  d2->n = d->n; d2->h = 1; d2->w = d->l; d2->c = d->c; d2->o = d->o; d2->kh = 1; d2->kw = d->k;
  d2->stride[0] = 1; d2->stride[1] = d->stride;
  d2->pad[0] = 0; d2->pad[1] = d->pad;
  d2->dilation[0] = 1; d2->dilation[1] = d->dilation;
  return true;
}

conv_status_t conv1d_plan(const conv1d_desc_t* desc, conv_dtype_t dtype, int device, const conv_options_t* opts,
                          conv_plan_t* plan) {
  conv2d_desc_t d2;
  if (!desc2d_of(desc, &d2)) return CONV_ERR_INVALID;
  return conv2d_plan(&d2, dtype, device, opts, plan);
}

size_t conv1d_workspace_size(const conv1d_desc_t* desc, conv_dtype_t dtype, int device, const conv_options_t* opts) {
  conv2d_desc_t d2;
  if (!desc2d_of(desc, &d2)) return 0;
  return conv2d_workspace_size(&d2, dtype, device, opts);
}

conv_status_t conv1d_forward(const void* in, const void* w, void* out, const conv1d_desc_t* desc, conv_dtype_t dtype,
                             const conv_options_t* opts, void* workspace, size_t workspace_bytes, void* stream) {
  conv2d_desc_t d2;
  if (!desc2d_of(desc, &d2)) return CONV_ERR_INVALID;
  return conv2d_forward(in, w, out, &d2, dtype, opts, workspace, workspace_bytes, stream);
}

conv_status_t conv3d_plan_for_props(const conv3d_desc_t* desc, conv_dtype_t dtype, const conv_device_props_t* props,
                                    const conv_options_t* opts, conv_plan_t* plan) {
  if (!props || !plan) return CONV_ERR_INVALID;
  Sel s;
  Geom g2;
  long long od;
  size_t ws;
  Path3d path = P3_TAPS;
  conv_status_t st = plan3d_impl(desc, dtype, *props, effective_options(opts), &s, &g2, &od, &ws, &path);
  if (st != CONV_OK) return st;
  fill_plan(s, plan, path == P3_TAPS ? desc->kd : 1, ws);
  return CONV_OK;
}

conv_status_t conv3d_plan(const conv3d_desc_t* desc, conv_dtype_t dtype, int device, const conv_options_t* opts,
                          conv_plan_t* plan) {
  DeviceState* d = nullptr;
  conv_status_t st = device_state(device, &d);
  if (st != CONV_OK) return st;
  return conv3d_plan_for_props(desc, dtype, &d->props, opts, plan);
}

size_t conv3d_workspace_size(const conv3d_desc_t* desc, conv_dtype_t dtype, int device, const conv_options_t* opts) {
  conv_plan_t p;
  return conv3d_plan(desc, dtype, device, opts, &p) == CONV_OK ? p.workspace_bytes : 0;
}

conv_status_t conv3d_forward(const void* in, const void* w, void* out, const conv3d_desc_t* desc, conv_dtype_t dtype,
                             const conv_options_t* opts, void* workspace, size_t workspace_bytes, void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CONV_ERR_CUDA;
  DeviceState* d = nullptr;
  conv_status_t st = device_state(dev, &d);
  if (st != CONV_OK) return st;
  Sel s;
  Geom g2;
  long long od;
  size_t ws;
  Path3d path = P3_TAPS;
  st = plan3d_impl(desc, dtype, d->props, effective_options(opts), &s, &g2, &od, &ws, &path);
  if (st != CONV_OK) return st;
  if (desc->n == 0) return CONV_OK;
  if (!in || !w || !out) return CONV_ERR_INVALID;
  if (workspace_bytes < ws || (ws > 0 && !workspace)) return CONV_ERR_WORKSPACE;
  if (ws > 0 && !aligned256(workspace)) return CONV_ERR_ALIGNMENT;
  const int esz = dtype_size(dtype);
  const long long frame_in = (long long)desc->h * desc->w * desc->c;
  const long long frame_out = (long long)g2.oh * g2.ow * g2.o;
  const size_t out_bytes = (size_t)desc->n * od * frame_out * esz;
  if (overlaps(out, out_bytes, in, (size_t)desc->n * desc->d * frame_in * esz) ||
      overlaps(out, out_bytes, w, (size_t)desc->o * g2.w_row_stride * esz) ||
      overlaps(out, out_bytes, workspace, ws))
    return CONV_ERR_INVALID;

  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  const Geom3 g3 = geom3_of(desc, od, g2);
  const char* path_name = path == P3_WINO3D ? "winograd3d" : "depth_taps";
  if (path == P3_NATIVE) {
    if (tc_conv3d_supported(g3, dtype, in, w)) {
      path_name = "native3d";
    } else {
      // misaligned pointers: depth taps on the any-alignment path
      conv_options_t o2 = effective_options(opts);
      o2.algo = CONV_ALGO_DIRECT;
      st = select2d(g2, dtype, d->props, o2, &s);
      if (st != CONV_OK) return st;
      path = P3_TAPS;
    }
  }
  if (log_enabled()) {
    char shape[224];
    std::snprintf(shape, sizeof shape, "n%d %dx%dx%d %d->%d k%dx%dx%d s%d,%d,%d p%d,%d,%d d%d,%d,%d", desc->n, desc->d,
                  desc->h, desc->w, desc->c, desc->o, desc->kd, desc->kh, desc->kw, desc->stride[0], desc->stride[1],
                  desc->stride[2], desc->pad[0], desc->pad[1], desc->pad[2], desc->dilation[0], desc->dilation[1],
                  desc->dilation[2]);
    log_plan("conv3d", shape, dtype, s, path_name, ws);
  }
  if (path == P3_WINO3D) return run3d_winograd(in, w, out, g3, dtype, s, workspace, *d, st_);
  if (path == P3_NATIVE) {
    ProfScope ps(K_TC_CONV3D, st_);
    return cuda_status(launch_tc_conv3d(in, w, out, g3, dtype, s.tile_n, d->props.sm_count, d->err_word, st_, s.tile_m));
  }
  Tap taps[1024];
  if (desc->kd > 1024) return CONV_ERR_UNSUPPORTED;
  const int ntaps = taps3d(desc, od, taps);
  const bool first_covers_all = ntaps > 0 && taps[0].od_lo == 0 && taps[0].od_hi == od - 1;

  for (int n = 0; n < desc->n; ++n) {
    const uint8_t* in_n = static_cast<const uint8_t*>(in) + (size_t)n * desc->d * frame_in * esz;
    uint8_t* out_n = static_cast<uint8_t*>(out) + (size_t)n * od * frame_out * esz;
    if (!first_covers_all) {
      ProfScope ps(K_FILL, st_);
      if (launch_fill_zero(out_n, (size_t)od * frame_out * esz, st_) != cudaSuccess) return CONV_ERR_CUDA;
    }
    for (int i = 0; i < ntaps; ++i) {
      const Tap& t = taps[i];
      Geom g = g2;
      g.n = t.od_hi - t.od_lo + 1;
      const void* in_view = in_n + (size_t)t.id_lo * frame_in * esz;
      const void* w_slice = static_cast<const uint8_t*>(w) + (size_t)t.kd * desc->kh * desc->kw * desc->c * esz;
      uint8_t* out_view = out_n + (size_t)t.od_lo * frame_out * esz;
      // tap 0 writes (when it covers every frame); the others add in ascending kd order
      const bool accumulate = !(i == 0 && first_covers_all);
      st = run2d(in_view, w_slice, out_view, g, dtype, s, workspace, *d, st_, accumulate);
      if (st != CONV_OK) return st;
    }
  }
  return CONV_OK;
}

conv_status_t conv_accumulate(void* out, const void* tap, size_t count, conv_dtype_t dtype, void* stream) {
  if (!valid_dtype(dtype)) return CONV_ERR_INVALID;
  if (count == 0) return CONV_OK;
  if (!out || !tap) return CONV_ERR_INVALID;
  const size_t bytes = count * dtype_size(dtype);
  if (overlaps(out, bytes, tap, bytes)) return CONV_ERR_INVALID;
  ProfScope ps(K_ACCUMULATE, static_cast<cudaStream_t>(stream));
  return cuda_status(launch_accumulate(out, tap, count, dtype, static_cast<cudaStream_t>(stream)));
}

conv_status_t conv_selftest_timeout(long long limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 100000000LL) return CONV_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CONV_ERR_CUDA;
  DeviceState* d = nullptr;
  conv_status_t st = device_state(dev, &d);
  if (st != CONV_OK) return st;
  return cuda_status(launch_wait_selftest(d->err_word, limit_ns, static_cast<cudaStream_t>(stream)));
}

conv_status_t conv_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  for (auto& r : g_prof.recs) {
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.recs.clear();
  g_prof.on = true;
  return CONV_OK;
}

int conv_profile_end(conv_kernel_time_t* out, int max_entries) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.on = false;
  int launches[K_COUNT] = {0};
  double ms[K_COUNT] = {0};
  bool failed = false;
  for (auto& r : g_prof.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      failed = true;
    launches[r.kind] += 1;
    ms[r.kind] += t;
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.recs.clear();
  if (failed) return -1;
  int n = 0;
  for (int k = 0; k < K_COUNT; ++k) {
    if (!launches[k]) continue;
    if (out && n < max_entries) out[n] = conv_kernel_time_t{kKindName[k], launches[k], ms[k]};
    ++n;
  }
  return std::min(n, max_entries);
}

conv_status_t conv_check(void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CONV_ERR_CUDA;
  DeviceState* d = nullptr;
  conv_status_t st = device_state(dev, &d);
  if (st != CONV_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CONV_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, d->err_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return CONV_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    if (cudaMemcpy(d->err_word, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return CONV_ERR_CUDA;
    return CONV_ERR_TIMEOUT;
  }
  return CONV_OK;
}

}  // extern "C"
