// internal.h -- declarations shared by the library's translation units.
// Nothing here is part of the C ABI (include/b200conv.h is).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/b200conv.h"

namespace b200conv {

// Device-side error codes written to the per-device error word.
enum DevErr : int {
  DEVERR_NONE = 0,
  DEVERR_TIMEOUT_PRODUCER = 0x101,   // TMA producer waited too long for a free stage
  DEVERR_TIMEOUT_MMA_FULL = 0x102,   // MMA issuer waited too long for a loaded stage
  DEVERR_TIMEOUT_MMA_TMEM = 0x103,   // MMA issuer waited too long for a drained accumulator
  DEVERR_TIMEOUT_EPILOGUE = 0x104,   // epilogue waited too long for a finished accumulator
  DEVERR_TIMEOUT_FUSED_GEMM = 0x105,   // persistent fp32 Winograd: a GEMM unit waited too long for V or a free M
  DEVERR_TIMEOUT_FUSED_XFORM = 0x106,  // persistent fp32 Winograd: the transform warps waited too long for the GEMM
  DEVERR_FUSED_SMEM_ALIGN = 0x107,     // persistent fp32 Winograd: input boxes not 128-byte aligned (read without TMA)
  DEVERR_TIMEOUT_SELFTEST = 0x1ff,   // the watchdog self-test's deliberate wait
};

inline int dtype_size(conv_dtype_t t) { return t == CONV_F32 ? 4 : 2; }

// One 2D convolution as the kernels see it.  The "batch" of a 2D conv is
// n images whose starts are in_img_stride elements apart (a conv3d depth tap
// passes frame views with stride sd*H*W*C); the weights are O rows of
// KH*KW*C elements, w_row_stride apart (KD*KH*KW*C for a depth-tap slice).
struct Geom {
  int n, h, w, c, o, kh, kw;
  int sh, sw, ph, pw, dh, dw;
  int oh, ow;
  long long in_img_stride;    // elements
  long long w_row_stride;     // elements
  long long out_img_stride;   // elements (OH*OW*O for a dense NHWC output)
};

// One 3D convolution (NDHWC input, O,KD,KH,KW,I weights, dense NDHWC output).
struct Geom3 {
  int n, d, h, w, c, o, kd, kh, kw;
  int sd, sh, sw, pd, ph, pw, dd, dh, dw;
  int od, oh, ow;
};

// Batched GEMM view used by the Winograd path: for b < batches,
//   D_b[t][o] = sum_c A_b[t][c] * B_b[o][c]   (A: [batches][T][C], B: [batches][O][C])
// accumulated in fp32 and stored in d_dt (fp32, or the 16-bit operand type).
struct BatchedGemm {
  int batches, t, c, o;
  const void* a;        // [batches][T][C] in the input dtype (fp32 for the SIMT engine)
  const void* b;        // [batches][O][C]
  void* d;              // [batches][T][O] in d_dt
  conv_dtype_t d_dt;
  // split-bf16 fp32 GEMM: a is [batches][T][3C] and b is [batches][O][3C] (the
  // three bf16 parts of each value side by side), d is fp32
  bool split_bf16 = false;
};

// ---- kernel launchers (return a CUDA error; never synchronise) ----

// SIMT implicit GEMM (FFMA, fp32 accumulate): any dtype, any alignment when
// vec == false.  accumulate: out = round(out + round(result)).
// ksplit > 1: the K range is split over ksplit blocks that write fp32 partials
// [ksplit][M][O] to `partial` (then launch_splitk_reduce).
cudaError_t launch_simt_conv(const void* in, const void* w, void* out, const Geom& g,
                             conv_dtype_t dt, bool vec, bool accumulate, cudaStream_t s, int ksplit = 1,
                             float* partial = nullptr);
// out[i] = round(sum_s partial[s][i]) (s ascending), or with accumulate
// out[i] = round(out[i] + round(sum)), for i < count.
cudaError_t launch_splitk_reduce(const float* partial, int ksplit, size_t count, void* out, conv_dtype_t dt,
                                 bool accumulate, cudaStream_t s);

// tcgen05 implicit GEMM for 16-bit dtypes (TMA im2col staging, TMEM accumulators).
// Returns cudaErrorNotSupported if the shape cannot be encoded as TMA maps.
bool tc_conv_supported(const Geom& g, conv_dtype_t dt, const void* in, const void* w);
// accumulate: out = round(out + round(result)), the unfused depth-tap add's arithmetic.
// ksplit > 1: the K range is split over ksplit CTAs per tile.  With `reduced`
// and `tile_cnt` given (M/128 x O/tile_n x 4 zeroed counters), each split writes
// fp32 partials [ksplit][M][O] to `partial` and the last split of each (tile,
// epilogue warp) sums them in split order and writes the output (*reduced set).
// With `reduced` alone, the splits of a tile run as one thread-block cluster
// that sums the partials from shared memory (*reduced set unless the device
// cannot hold the cluster).  Otherwise the caller runs launch_splitk_reduce on
// `partial` (the same sums in the same order on every route).
cudaError_t launch_tc_conv(const void* in, const void* w, void* out, const Geom& g,
                           conv_dtype_t dt, int tile_n, int sm_count, int* err_word,
                           bool accumulate, cudaStream_t s, int ksplit = 1, float* partial = nullptr,
                           bool* reduced = nullptr, int tile_m = 128, int* tile_cnt = nullptr);
// Native 3D implicit GEMM on tcgen05: K = KD*KH*KW*C in one main loop, the A
// tiles gathered by a 5D TMA im2col map (corners limited to [-16, 15]).
bool tc_conv3d_supported(const Geom3& g, conv_dtype_t dt, const void* in, const void* w);
// tile_m == 256 (with tile_n == 256): CTA pairs on 256-row tiles where the device can hold them.
cudaError_t launch_tc_conv3d(const void* in, const void* w, void* out, const Geom3& g, conv_dtype_t dt, int tile_n,
                             int sm_count, int* err_word, cudaStream_t s, int tile_m = 128);
// tcgen05 batched GEMM for 16-bit operands with fp32 D (Winograd 16-bit path).
cudaError_t launch_tc_batched_gemm(const BatchedGemm& bg, conv_dtype_t dt, int tile_n,
                                   int sm_count, int* err_word, cudaStream_t s, int tile_m = 128);

// Watchdog self-test: one bounded wait on a barrier nothing arrives on.
cudaError_t launch_wait_selftest(int* err_word, long long limit_ns, cudaStream_t s);

// Winograd transforms (fp32 arithmetic; V/U stored in `store_dt`).
cudaError_t launch_wino_filter(const void* w, long long w_row_stride, int o, int c, int m,
                               conv_dtype_t in_dt, conv_dtype_t store_dt, void* u, cudaStream_t s);
// A call covers tiles [t_base, t_base + t_count) counted from image n0's first
// tile (tile t of an image at t / (tiles_h*tiles_w) images past n0); V and M
// rows are numbered from 0 within the call, t_tile rows per plane.
cudaError_t launch_wino_input(const void* in, const Geom& g, int n0, long long t_base, long long t_count, int m,
                              conv_dtype_t in_dt, conv_dtype_t store_dt, void* v, long long t_tile,
                              cudaStream_t s);
// One pass of the chunked fp32-store Winograd pipeline: the input transform of
// tiles [in_t_base, +in_t_count) into V (fp32, rows packed: in_t_count per
// plane) and the output transform of tiles [out_t_base, +out_t_count) from M
// (fp32, out_t_count rows per plane), tiles counted from image n0's first
// tile, in one launch.  Either count may be 0.  pdl: launched with
// programmatic stream serialization, the output part waiting for the previous
// kernel (the GEMM that wrote M) and the input part not waiting, which is
// correct only when V was last read by the kernel before that one.
cudaError_t launch_wino_pass(const void* in, const Geom& g, int m, conv_dtype_t dt, int n0, long long in_t_base,
                             long long in_t_count, float* v, long long out_t_base, long long out_t_count,
                             const float* mb, void* out, bool accumulate, bool pdl, cudaStream_t s);
// Channel-major fp32 variants for the FFMA GEMM: U[xi][c][o_pad], V[xi][c][t_stride].
cudaError_t launch_wino_filter_cmajor(const void* w, long long w_row_stride, int o, int c, int m,
                                      conv_dtype_t in_dt, long long o_pad, float* u, cudaStream_t s);
cudaError_t launch_wino_input_cmajor(const void* in, const Geom& g, int n0, int nb, int m, conv_dtype_t in_dt,
                                     float* v, long long t_stride, cudaStream_t s);
// Batched FFMA GEMM D[b][t][o] = sum_c A[b][.][.] * B[b][c][o]; A is [C][lda] (channel-major)
// or, with a_tmajor, [T][lda] (tile-major); B row stride ldb.
cudaError_t launch_wino_gemm_f32(const float* a, const float* b, float* d, int batches, int t, int c, int o,
                                 long long lda, long long ldb, bool a_tmajor, cudaStream_t s);
int wino_gemm_f32_tile_n(int o);

// Split-bf16 fp32 Winograd F(6x6,3x3): the filter transform as U'[64][O][3C]
// bf16 and the input transform as V'[64][t_tile][3C] bf16 (fp32 input).
cudaError_t launch_wino_filter_split(const float* w, long long w_row_stride, int o, int c, void* u,
                                     cudaStream_t s);
cudaError_t launch_wino_input_split(const float* in, const Geom& g, int n0, long long t_count, void* v,
                                    long long t_tile, cudaStream_t s);

// The fp32 Winograd F(6x6,3x3) conv as one persistent kernel (input transform,
// FFMA GEMM and output transform overlapped inside each CTA, blocks of 128
// tiles).  u: the transformed filter [64][C][ldb] (ldb = O rounded up to 4);
// scratch: grid x wino_fused_f32_cta_bytes(C, O) bytes, 16-byte aligned.
bool wino_fused_f32_shape_ok(const Geom& g);
size_t wino_fused_f32_cta_bytes(int c, int o);
long long wino_fused_f32_blocks(long long tiles);
cudaError_t launch_wino_fused_f32(const float* in, const Geom& g, const float* u, long long ldb, float* out,
                                  float* scratch, int grid, bool accumulate, int* err_word, cudaStream_t s);
// M [a2][t_tile][O] in m_dt (fp32, or the 16-bit operand type of the tensor-core path).
cudaError_t launch_wino_output(const void* mbuf, conv_dtype_t m_dt, const Geom& g, int n0, long long t_base,
                               long long t_count, int m, long long t_tile, conv_dtype_t out_dt, void* out,
                               bool accumulate, cudaStream_t s);

// Native 3D Winograd F(m^3, 3^3) transforms, m in {2, 4}, for 3x3x3 stride-1
// dilation-1 convs.  Tiles are numbered unit-major, a unit being one (image,
// depth tile) slab of ceil(OH/m)*ceil(OW/m) tiles; a call covers units
// [u0, u0 + nu).  U: [a3][C][o_pad] fp32 (cmajor) or [a3][O][C] in store_dt;
// V: [a3][t_stride][C] in store_dt; M: [a3][t_stride][O] fp32.
cudaError_t launch_wino3d_filter(const void* w, int o, int c, int m, conv_dtype_t in_dt, conv_dtype_t store_dt,
                                 bool cmajor, long long o_pad, void* u, cudaStream_t s);
cudaError_t launch_wino3d_input(const void* in, const Geom3& g, long long u0, long long nu, int m,
                                conv_dtype_t in_dt, conv_dtype_t store_dt, void* v, long long t_stride,
                                cudaStream_t s);
cudaError_t launch_wino3d_output(const float* mbuf, const Geom3& g, long long u0, long long nu, int m,
                                 long long t_stride, conv_dtype_t out_dt, void* out, cudaStream_t s);

// Elementwise helpers.
cudaError_t launch_accumulate(void* out, const void* tap, size_t count, conv_dtype_t dt,
                              cudaStream_t s);
cudaError_t launch_fill_zero(void* out, size_t bytes, cudaStream_t s);
// Tap packing: dst[n][y][x][k*c + ch] = src[n][y][x*sw - pw + k*dw][ch] (zero outside the row and
// for channels >= kw*c); dst is dense [n][h][ow][cp].
cudaError_t launch_wpack(const void* src, long long n, int h, int w, int c, int kw, int sw, int pw, int dw, int ow,
                         long long in_img_stride, void* dst, int cp, conv_dtype_t dt, cudaStream_t s);
// Full tap packing: dst[n][oy][ox][k] for k < cp (a multiple of 8) holds the input
// value under tap (kh, kw) and channel c, k = (kh*KW + kw)*C + c (zero outside the
// image and for k >= KH*KW*C); the conv then runs as a 1x1 conv over cp channels.
cudaError_t launch_fullpack(const void* src, const Geom& g, void* dst, int cp, conv_dtype_t dt, int sm_count,
                            cudaStream_t s);
// Channel pad: dst[a][b][c'] = c' < c ? src[a*src_outer_stride + b*c + c'] : 0 for a < outer,
// b < inner, c' < cp; dst is dense [outer][inner][cp].  Element strides.
cudaError_t launch_channel_pad(const void* src, long long outer, long long inner, int c,
                               long long src_outer_stride, void* dst, int cp, conv_dtype_t dt,
                               cudaStream_t s);

}  // namespace b200conv
