/*
 * b200conv.h -- C ABI of the B200 (sm_100a) NHWC convolution forward library.
 *
 * The operation (all entry points): a cross-correlation with zero padding,
 * groups = 1,
 *
 *   out[n,oh,ow,o] = sum_{kh,kw,c} in[n, oh*sh - ph + kh*dh, ow*sw - pw + kw*dw, c] * w[o,kh,kw,c]
 *   OH = floor((H + 2*ph - dh*(KH-1) - 1) / sh) + 1            (same for OW)
 *
 * over NHWC activations and OHWI weights, accumulated in fp32 and rounded
 * once (round-to-nearest-even) to the storage dtype.  fp32 inputs are
 * computed in true fp32 (FFMA; never TF32).  This is the operation the MLX pull
 * requests "Bound winograd conv2d working set by tiling the batch" (Problem,
 * Fix), "Use the explicit gemm for wide convs on neural accelerators"
 * (description) and "Decompose small kernel-depth 3D convs into 2D convs"
 * (Change) dispatch to their GPU kernels.
 *
 * Two algorithms sit behind one deterministic selector (conv2d_plan):
 *  - implicit GEMM: A = im2col(in) is never materialised; 16-bit inputs run on
 *    tcgen05 tensor cores with TMEM accumulators and TMA im2col staging, fp32
 *    inputs on an FFMA core;
 *  - Winograd F(m x m, 3 x 3) for 3x3 stride-1 convs: filter, input and output
 *    transforms around a batched GEMM, with the batch tiled over one reused
 *    workspace so that the scratch working set is bounded; tiled output is
 *    bit-identical to untiled ("Bound winograd conv2d working set by tiling
 *    the batch", Fix and Testing).
 * conv3d runs as KD depth-tap 2D convs over zero-copy frame views whose results
 * are accumulated in place ("Decompose small kernel-depth 3D convs into 2D
 * convs", Change), as a native 3D implicit GEMM, or, for 3x3x3 stride-1
 * convs, as a native 3D Winograd F(m x m x m, 3 x 3 x 3) (that page's Open
 * questions, item 3).
 *
 * Conventions shared by every entry point:
 *  - Pointers named in/w/out/workspace are DEVICE pointers owned by the caller;
 *    the library never allocates or frees device memory in a forward call and
 *    holds no state except a per-device cache of constant device properties.
 *  - in, w and out share one dtype.  in is NHWC (NDHWC for 3D) contiguous,
 *    w is OHWI (O,KD,KH,KW,I for 3D) contiguous, out is NHWC (NDHWC) contiguous.
 *  - Work is enqueued asynchronously on `stream` (0 = the legacy default
 *    stream).  A returned CONV_OK means the work was validated and enqueued;
 *    device-side failures (a bounded wait that ran out) are reported by
 *    conv_check().
 *  - out must not overlap in, w or workspace (CONV_ERR_INVALID).
 *  - N = 0 is a valid no-op.  An empty output (OH <= 0, ...) or a non-positive
 *    size, stride or dilation, or a negative pad, is CONV_ERR_INVALID.
 *  - The selector is a pure function of (shape, dtype, device properties,
 *    options); it never looks at the device's current free memory ("Bound
 *    winograd conv2d working set by tiling the batch", maintainer review).
 */
#ifndef B200CONV_H
#define B200CONV_H

#include <stddef.h>

#if defined(__GNUC__)
#define B200CONV_API __attribute__((visibility("default")))
#else
#define B200CONV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { CONV_F32 = 0, CONV_F16 = 1, CONV_BF16 = 2 } conv_dtype_t;

typedef enum {
    CONV_OK = 0,
    CONV_ERR_INVALID = 1,      /* bad shape, pointer, overlap or argument */
    CONV_ERR_UNSUPPORTED = 2,  /* forced algorithm cannot run this shape */
    CONV_ERR_ALIGNMENT = 3,    /* a workspace that is not 256-byte aligned; nothing was launched
                                  (misaligned in / w / out take the any-alignment path instead) */
    CONV_ERR_WORKSPACE = 4,    /* workspace smaller than the plan needs; nothing was launched */
    CONV_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    CONV_ERR_TIMEOUT = 6       /* a kernel's bounded wait ran out (reported by conv_check) */
} conv_status_t;

typedef enum {
    CONV_ALGO_AUTO = 0,
    CONV_ALGO_IMPLICIT_GEMM = 1,
    CONV_ALGO_WINOGRAD = 2,
    CONV_ALGO_DIRECT = 3      /* SIMT implicit GEMM with scalar loads: any alignment */
} conv_algo_t;

typedef enum {
    CONV_ENGINE_NONE = 0,
    CONV_ENGINE_TCGEN05 = 1,  /* tcgen05.mma, TMEM accumulators, TMA staging (16-bit) */
    CONV_ENGINE_SIMT = 2      /* FFMA in fp32 registers */
} conv_engine_t;

/* 2D problem.  stride/pad/dilation are {H, W}. */
typedef struct {
    int n, h, w, c, o, kh, kw;
    int stride[2], pad[2], dilation[2];
} conv2d_desc_t;

/* 3D problem.  stride/pad/dilation are {D, H, W}. */
typedef struct {
    int n, d, h, w, c, o, kd, kh, kw;
    int stride[3], pad[3], dilation[3];
} conv3d_desc_t;

/* 1D problem: in [N, L, C] (channels last), w [O, K, C], out [N, OL, O]. */
typedef struct {
    int n, l, c, o, k;
    int stride, pad, dilation;
} conv1d_desc_t;

/* Constant device properties the selector may depend on. */
typedef struct {
    int sm_count;
    int cc_major, cc_minor;
    unsigned long long total_global_mem;   /* bytes; a constant, never free memory */
} conv_device_props_t;

/*
 * Options.  Pass NULL for the defaults, which are read from the environment
 * (test hooks, read on every call before selection):
 *   B200CONV_ALGO=auto|implicit|winograd|direct
 *   B200CONV_WINOGRAD_WORKSPACE_BYTES=<bytes>   replaces the Winograd scratch budget
 *   B200CONV_WINOGRAD_TILE_BATCH=<images>       forces the batch-tile size (capped by the budget)
 * A non-NULL options struct ignores the environment.  Independently of the
 * options, B200CONV_LOG=1 makes every conv*_forward call print the plan it
 * runs (algorithm, engine, path, tile, Winograd m and batch tile, channel pad,
 * K split, workspace bytes) as one line on stderr.  Further test hooks, also
 * read on every call, select between execution routes that give the same
 * result: B200CONV_TC_PAIR=0 keeps the tensor-core kernels on 128-row tiles
 * (no CTA pairs); B200CONV_SPLITK_CLUSTER=1 sums split-K partials inside the
 * conv kernel (thread-block clusters) instead of the reduce kernel;
 * B200CONV_SPLITK_SERIAL=1 has the last-arriving split of each tile sum them;
 * B200CONV_WINOGRAD_CHUNK_TILES=<tiles> runs the fp32 Winograd path in chunks
 * of that many tiles (pipelined transform / GEMM passes; 0 or unset: off);
 * B200CONV_WINOGRAD_FUSED=1 runs the fp32 Winograd F(6x6,3x3) path as one
 * persistent kernel whenever the shape allows (=0 or unset: three launches);
 * B200CONV_WINOGRAD_FUSED_GRID=<ctas> runs that kernel on fewer CTAs;
 * B200CONV_WINOGRAD_SPLIT_BF16=1 runs the fp32 Winograd GEMM on the tensor
 * cores over split-bf16 operands (fp32 accuracy; C a multiple of 64, O of 4).
 */
typedef struct {
    conv_algo_t algo;                     /* CONV_ALGO_AUTO: let the selector choose */
    long long winograd_budget_bytes;      /* < 0: the device default budget */
    int winograd_tile_batch;              /* <= 0: derived from the budget */
} conv_options_t;

typedef struct {
    conv_algo_t algo;          /* the algorithm that will run */
    conv_engine_t engine;      /* the GEMM engine under it */
    int tile_m, tile_n;        /* GEMM tile (rows x output channels) */
    int winograd_m;            /* m of F(m x m, 3 x 3) (F(m^3, 3^3) for the 3D Winograd); 0 unless Winograd */
    int batch_tile;            /* images per Winograd batch tile (= n when untiled); for the
                                  3D Winograd, units per tile, a unit being one (image, depth
                                  tile of m output frames) slab */
    int num_batch_tiles;       /* number of batch tiles */
    int channel_pad;           /* padded channel count of the pre-pass, 0 if none */
    int packed_taps;           /* few-channel inputs: 1 if the KW taps are folded into channel_pad channels
                                  (a KH x 1 conv over them), 2 if all KH*KW taps are (a 1 x 1 conv); else 0 */
    int k_split;               /* implicit GEMM: K range split over this many CTAs (fp32 partials), 1 if none */
    int taps;                  /* conv3d: number of depth taps (KD); 1 for conv2d */
    int winograd_fused;        /* 1 if the fp32 Winograd F(6x6,3x3) runs as one persistent kernel (input
                                  transform, FFMA GEMM and output transform overlapped inside each CTA,
                                  per-CTA scratch in the workspace); else 0 */
    int winograd_split_bf16;   /* 1 if the fp32 Winograd GEMM runs on the tensor cores over split-bf16
                                  operands (each fp32 value the exact sum of three bf16 parts, the six
                                  products a_i b_j with i + j <= 2 accumulated in fp32); else 0 */
    size_t workspace_bytes;    /* bytes the caller must pass to *_forward */
} conv_plan_t;

/* Fill props for CUDA device `device`.  CONV_ERR_CUDA if there is none. */
B200CONV_API conv_status_t conv_device_props(int device, conv_device_props_t *props);

/*
 * Plan a conv2d: validate, compute the output shape, pick the algorithm, the
 * tile configuration and the Winograd batch tile, and size the workspace.
 * Pure: the same arguments give the same plan in any process at any time.
 * Winograd (auto) needs 3x3, stride 1, dilation 1 and the page's channel rule
 * (C % 32 == 0, O % 32 == 0, C + O >= 256); 16-bit inputs take it only for deep,
 * wide GEMMs (C >= 1024 and O >= 1024, or C >= 512 and O >= 2048), else the
 * tensor-core implicit GEMM.
 * The Winograd budget is 3/4 of the device's total memory minus the conv's own
 * tensors (input, output, transformed filter), capped at 8 GiB because the GPU
 * is shared ("Bound winograd conv2d working set by tiling the batch", Fix).
 * plan->tile_m == 256 means the tensor-core kernel runs CTA pairs: two SMs
 * per 256 x 256 output tile (cta_group::2), each holding half of the input
 * and half of the weight tile.
 */
B200CONV_API conv_status_t conv2d_plan(const conv2d_desc_t *desc, conv_dtype_t dtype, int device,
                          const conv_options_t *opts, conv_plan_t *plan);
/* Same selector for explicit device properties (usable without a GPU). */
B200CONV_API conv_status_t conv2d_plan_for_props(const conv2d_desc_t *desc, conv_dtype_t dtype,
                                    const conv_device_props_t *props,
                                    const conv_options_t *opts, conv_plan_t *plan);
/* Workspace bytes conv2d_forward needs with these options; 0 if invalid. */
B200CONV_API size_t conv2d_workspace_size(const conv2d_desc_t *desc, conv_dtype_t dtype, int device,
                             const conv_options_t *opts);

/*
 * Run a conv2d on `stream`.  in [N,H,W,C], w [O,KH,KW,C], out [N,OH,OW,O],
 * all of `dtype`, on the current CUDA device.  workspace may be NULL when the
 * plan needs 0 bytes; a workspace_bytes smaller than the plan's is
 * CONV_ERR_WORKSPACE and launches nothing (never a partial or zeroed result).
 * A non-empty workspace must start on a 256-byte boundary (cudaMalloc and
 * torch allocations do), else CONV_ERR_ALIGNMENT and nothing is launched.
 */
B200CONV_API conv_status_t conv2d_forward(const void *in, const void *w, void *out,
                             const conv2d_desc_t *desc, conv_dtype_t dtype,
                             const conv_options_t *opts,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * conv1d through the 2D path, as the implicit-GEMM page's conv_1D_gpu routes
 * 1D convolutions into the 2D dispatch ("Use the explicit gemm for wide convs
 * on neural accelerators", the Whisper follow-up): a [N, L, C] input is the
 * [N, 1, L, C] image of a 1 x K conv2d with stride (1, s), padding (0, p) and
 * dilation (1, d).  Same selector, kernels, ownership and error behaviour as
 * conv2d_*.
 */
B200CONV_API conv_status_t conv1d_plan(const conv1d_desc_t *desc, conv_dtype_t dtype, int device,
                                       const conv_options_t *opts, conv_plan_t *plan);
B200CONV_API size_t conv1d_workspace_size(const conv1d_desc_t *desc, conv_dtype_t dtype, int device,
                                          const conv_options_t *opts);
B200CONV_API conv_status_t conv1d_forward(const void *in, const void *w, void *out,
                                          const conv1d_desc_t *desc, conv_dtype_t dtype,
                                          const conv_options_t *opts,
                                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * conv3d, in[N,D,H,W,C], w[O,KD,KH,KW,C], out[N,OD,OH,OW,O].  Three algorithms:
 *  - depth taps ("Decompose small kernel-depth 3D convs into 2D convs",
 *    Change): for each kd, a 2D conv over the zero-copy view of the input
 *    frames at depth offset kd*dd (frame stride sd*H*W*C) with the weight slice
 *    w[:, kd] (row stride KD*KH*KW*C); tap 0 writes out and taps 1..KD-1 add in
 *    ascending order inside their own output stage (round the tap, add in
 *    fp32, round).  Depth padding, depth stride/dilation, N > 1 and any KD are
 *    handled by restricting each tap to the output frames whose input frame
 *    exists.
 *  - a native 3D implicit GEMM (16-bit, tensor cores): K = KD*KH*KW*C in one
 *    main loop, A tiles gathered by a 5D TMA im2col map; output written once.
 *  - a native 3D Winograd for KD = KH = KW = 3, all strides and dilations 1,
 *    any padding, C % 4 == 0: the 1D F(m, 3) transforms applied along depth,
 *    height and width around alpha^3 batched GEMMs (F(4,3), alpha^3 = 216, for
 *    fp32; F(2,3), alpha^3 = 64, for 16-bit).  Its workspace is tiled over
 *    units (image, depth tile of m output frames) under the conv2d Winograd
 *    budget rule, tiled output bit-identical to untiled.
 * With CONV_ALGO_AUTO, fp32 shapes of the 3D Winograd that meet the conv2d
 * channel rule (C % 32 == 0, O % 32 == 0, C + O >= 256) take it when the
 * budget allows (the same fallback rule as conv2d).  Otherwise the page's
 * guard (N == 1, KD <= 7, depth stride 1, kernel dilation 1, no depth padding,
 * C and O multiples of 16) selects the depth taps, and the other shapes take
 * the native GEMM when it can express them (16-bit, C % 8 == 0, 5D box corners
 * within [-16, 15]), else the depth taps.
 * CONV_ALGO_IMPLICIT_GEMM asks for the native GEMM whenever it can run;
 * CONV_ALGO_WINOGRAD asks for the 3D Winograd on its shapes (any dtype, no
 * channel rule) and otherwise for depth taps with the 2D Winograd;
 * CONV_ALGO_DIRECT picks the depth taps' any-alignment 2D path.
 * plan->taps is KD for depth taps and 1 for the native GEMM and the 3D Winograd.
 */
B200CONV_API conv_status_t conv3d_plan(const conv3d_desc_t *desc, conv_dtype_t dtype, int device,
                          const conv_options_t *opts, conv_plan_t *plan);
B200CONV_API conv_status_t conv3d_plan_for_props(const conv3d_desc_t *desc, conv_dtype_t dtype,
                                    const conv_device_props_t *props,
                                    const conv_options_t *opts, conv_plan_t *plan);
B200CONV_API size_t conv3d_workspace_size(const conv3d_desc_t *desc, conv_dtype_t dtype, int device,
                             const conv_options_t *opts);
B200CONV_API conv_status_t conv3d_forward(const void *in, const void *w, void *out,
                             const conv3d_desc_t *desc, conv_dtype_t dtype,
                             const conv_options_t *opts,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * In-place depth-tap accumulate, out[i] = round(out[i] + tap[i]) for i < count
 * (fp32 add, one rounding to dtype): the step the depth-tap page performs with
 * an in-place binary add ("Decompose small kernel-depth 3D convs into 2D
 * convs", Open questions 1).  Device pointers; out and tap must not overlap.
 */
B200CONV_API conv_status_t conv_accumulate(void *out, const void *tap, size_t count, conv_dtype_t dtype,
                              void *stream);

/*
 * Diagnostic: measure the CUDA-core fp32 FMA rate of the current device in
 * TFLOP/s (2 FLOP per lane per FMA), scalar FFMA (packed = 0) or sm_100's
 * packed two-lane FMA (packed = 1), the denominator of the fp32 kernels'
 * roofline.  Runs a few short FMA-chain kernels on `stream` and synchronizes
 * it; allocates no device memory.  CONV_ERR_CUDA if the device cannot run it.
 */
B200CONV_API conv_status_t conv_fp32_fma_rate(int packed, double *tflops, void *stream);

/*
 * Synchronise `stream`, then read and clear the current device's error word.
 * Returns CONV_ERR_TIMEOUT if a kernel's bounded wait ran out since the last
 * check, CONV_ERR_CUDA if the synchronisation failed, else CONV_OK.
 */
B200CONV_API conv_status_t conv_check(void *stream);

/*
 * Winograd conv2d that allocates nothing.  The pages have no counterpart of
 * this entry point; it serves callers that cannot allocate device memory or
 * hand the library a workspace (code running inside another runtime's hooks
 * with no allocator, services that must not allocate once running, callers
 * that hold only borrowed input/output pointers).  Its scratch is a 64 MiB
 * device array compiled into the library, held by every GPU that loads it
 * until the process exits.  in/w/out and their layouts are as for
 * conv2d_forward.  The shape must be 3x3, stride 1, dilation 1
 * (CONV_ERR_UNSUPPORTED otherwise).  The batch is tiled so that the transformed
 * filter and one batch tile fit in the array; a conv whose filter plus one
 * image's transform buffers exceed 64 MiB is rejected with CONV_ERR_WORKSPACE
 * and nothing is launched.  Output equals conv2d_forward with
 * CONV_ALGO_WINOGRAD at the same tile size.  No cudaMalloc or cudaFree is
 * called.  Every call looks up the array's address in the current device's
 * context (a lookup, not an allocation), so a context re-created after
 * cudaDeviceReset is followed; the first call on a device also loads the
 * library's device code there, so make that first call before any stream
 * capture.  All calls share the array and
 * it keeps the last call's contents (nothing needs clearing); calls whose work
 * overlaps on the GPU race on it.
 */
B200CONV_API conv_status_t conv2d_forward_winograd_static(const void *in, const void *w, void *out,
                                                          const conv2d_desc_t *desc, conv_dtype_t dtype,
                                                          void *stream);

/*
 * Opt-in kernel timing, for benchmarks.  Between conv_profile_begin() and
 * conv_profile_end() every kernel the library launches on the current device
 * is bracketed by a pair of CUDA events recorded on its launch stream.
 * conv_profile_end() waits for those events, stops recording and writes up to
 * max_entries per-kernel summaries (one per kernel kind that ran: its name,
 * launch count and summed event time), returning how many it wrote (or -1 on
 * a CUDA error).  Recording is process-wide and not meant for concurrent use
 * from several threads.
 */
typedef struct {
    const char *name;       /* static string, e.g. "tc_conv" */
    int launches;
    double total_ms;
} conv_kernel_time_t;
B200CONV_API conv_status_t conv_profile_begin(void);
B200CONV_API int conv_profile_end(conv_kernel_time_t *out, int max_entries);

/*
 * Watchdog self-test.  Launches one tiny kernel that waits, through the same
 * bounded-wait routine the tensor-core pipeline uses, on an mbarrier phase that
 * nothing completes; after limit_ns nanoseconds (1 us .. 100 ms, else
 * CONV_ERR_INVALID) the wait gives up, records a timeout in the device error
 * word and the kernel returns.  The next conv_check() then reports
 * CONV_ERR_TIMEOUT (and clears it).  Used by the tests to show that a stuck
 * pipeline ends with a status instead of a hang.
 */
B200CONV_API conv_status_t conv_selftest_timeout(long long limit_ns, void *stream);

/* Static description of a status code. */
B200CONV_API const char *conv_status_string(conv_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* B200CONV_H */
