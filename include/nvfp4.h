/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 linear-layer library (libnvfp4.so).
 *
 * The format (sources: "NVFP4 Is a Scaling System, Not Just a 4-Bit Number",
 * section "The smallest example: the same payload, two real values";
 * "MXFP4 和 NVFP4 的区别", sections "数据格式:极简的 E2M1" and
 * "精度核心:两级分层缩放"; "Melatih model dalam 4 bit: pengaman numerik di
 * balik NVFP4", section "Anatomi NVFP4: empat bit dengan dua tingkat skala"):
 *   x = x_e2m1 * s_block * s_global
 *   - x_e2m1: 4-bit E2M1 code (1 sign, 2 exponent, 1 mantissa bit), magnitudes
 *     {0, 0.5, 1, 1.5, 2, 3, 4, 6}; code bits b3 = sign, b2..b1 = exponent,
 *     b0 = mantissa; two codes per byte, element 2j in the low nibble of byte j.
 *   - s_block: E4M3 (FN, max 448) scale shared by 16 consecutive elements
 *     along K (1D) or by a 16x16 tile (2D, weights).
 *   - s_global: one FP32 scale per tensor, amax / (448 * 6).
 *
 * Conventions (all entry points):
 *   - Every pointer argument except the host-side ones named in a comment is a
 *     DEVICE pointer owned by the caller.  The library allocates no memory and
 *     keeps no per-call state; the only library state is a device error word
 *     (see nvfp4_get_error) and a per-device attribute cache.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     stream-ordered and asynchronous: a call returns after enqueueing.
 *   - Input tensors are bf16, row-major with a row stride `ld` in elements.
 *     Inputs must be finite; non-finite input does not fault or hang, but the
 *     outputs are then unspecified.
 *   - Validation happens on the host, before any launch.  On error nothing is
 *     enqueued and the status says why:
 *       NVFP4_ERR_INVALID_ARG       null pointer, negative size, bad enum,
 *       NVFP4_ERR_UNSUPPORTED_SHAPE a size the kernels do not handle (below),
 *       NVFP4_ERR_MISALIGNED        a pointer or stride breaks the 16-byte rule,
 *       NVFP4_ERR_WORKSPACE         workspace missing or smaller than required,
 *       NVFP4_ERR_CUDA              a CUDA launch or driver call failed,
 *       NVFP4_ERR_TIMEOUT           (from nvfp4_get_error) a device-side wait ran
 *                                   out of its bound; the kernel returned early.
 *   - Alignment: x, codes, scales and scales_mma base pointers 16-byte aligned;
 *     `ld` a multiple of 8 elements.
 *
 * Scale layouts:
 *   - Plain ("scales"): row-major, one byte per block: 1D [rows x K/16],
 *     2D [rows/16 x cols/16].  This is the layout the CPU oracle produces.
 *   - MMA ("scales_mma"): the tiled layout the block-scaled tensor-core GEMM
 *     reads (one 512-byte chunk per 128 rows x 4 consecutive 16-blocks along K,
 *     so a chunk is copied to tensor memory as is).  For an operand with R rows
 *     and K elements per row, Kb = K/16 blocks, chunks_k = ceil(Kb / 4):
 *       offset(r, b) = ((r / 128) * chunks_k + b / 4) * 512
 *                      + (r % 32) * 16 + ((r / 32) % 4) * 4 + (b % 4)
 *     Size: nvfp4_mma_scale_bytes(R, K) = ceil(R/128) * chunks_k * 512.
 *     Entries past R rows or past Kb blocks are written as 0.
 *     2D scales are expanded per row: row r, block b holds the tile scale of
 *     (r/16, b).
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2,
    NVFP4_ERR_MISALIGNED = 3,
    NVFP4_ERR_CUDA = 4,
    NVFP4_ERR_TIMEOUT = 5,
    NVFP4_ERR_WORKSPACE = 6
} nvfp4_status;

enum { NVFP4_RNE = 0, NVFP4_SR = 1 };            /* rounding of element codes */
enum { NVFP4_SCALE_1D = 0, NVFP4_SCALE_2D = 1 };  /* 16 along K | 16x16 tile */
enum { NVFP4_OUT_F32 = 0, NVFP4_OUT_BF16 = 1 };   /* GEMM / dequantize output type */

/* Library ABI version (major * 100 + minor): 101 = 1.1, the 1.0 entry points
 * plus the dual, from-amax, GEMM-amax, MXFP4 and RHT-order ones. */
int nvfp4_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* nvfp4_status_string(nvfp4_status s);

/* Bytes of device workspace a quantize call on a [rows x cols] input needs
 * (scratch for the tensor-amax partial maxima).  The caller allocates it; the
 * call overwrites it; it holds nothing between calls. */
size_t nvfp4_workspace_size(int64_t rows, int64_t cols);

/* Bytes of an MMA-layout scale array for an operand of `rows` rows and K
 * elements per row (K a multiple of 16). */
size_t nvfp4_mma_scale_bytes(int64_t rows, int64_t k);

/* 1D quantization [two-level scaling of "精度核心:两级分层缩放"; rounding per
 * "随机舍入" -- RNE for weights/activations, SR for gradients].
 *   x          bf16 [rows x cols], row stride ld.
 *   transpose  0: quantize Q = x ([rows x cols], blocks along cols);
 *              1: quantize Q = x^T ([cols x rows], blocks along rows).
 *   rounding   NVFP4_RNE or NVFP4_SR.  SR draws 16 bits per element from
 *              Philox4x32-10 keyed by sr_seed at counter (i/8, 0) where i is
 *              the element's index in Q (row-major); word (i%8)/2, low half
 *              for even i.  Between the neighbouring codes lo <= |v| < hi,
 *              p = (|v| - lo) / (hi - lo): round up iff floor(p * 65536) + bits
 *              >= 65536 (the carry of the random bits added below the kept
 *              precision; up-rate within 2^-16 of p).
 *   Outputs for Q of shape [Qr x Qc] (Qc % 16 == 0):
 *     codes        [Qr x Qc/2] packed E2M1 (required),
 *     scales       [Qr x Qc/16] E4M3, plain layout (nullable),
 *     scales_mma   MMA layout of Q's scales, nvfp4_mma_scale_bytes(Qr, Qc) (nullable),
 *     global_scale one float, s_global = amax(Q) / 2688 (required).
 *   At least one of scales / scales_mma must be non-NULL.
 *   Computation: s_global = RN(amax / 2688); per block t = RN(6 s_global),
 *   s = e4m3_rne_satfinite(RN(block_amax / t)) (0 when t == 0); per element
 *   v = RN(x * RN(1 / RN(s * s_global))), code = E2M1(v) saturating at +-6,
 *   sign of x kept; s == 0 or x == 0 gives a signed zero.
 *   Shapes: Qc a multiple of 16; rows, cols >= 1.
 *   Workspace: >= nvfp4_workspace_size(rows, cols) bytes, 16-byte aligned. */
nvfp4_status nvfp4_quantize_1d(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                               int rounding, uint64_t sr_seed, uint8_t* codes, uint8_t* scales,
                               uint8_t* scales_mma, float* global_scale, void* workspace,
                               size_t ws_bytes, void* stream);

/* nvfp4_quantize_1d for callers that cannot allocate device memory.  The
 * paper has no counterpart to this entry point.
 * Who needs it: a process whose device memory is all owned by another
 * allocator (a framework's caching allocator, or an inference engine that
 * reserves the whole HBM at start-up), and plug-ins or callbacks that are not
 * allowed to allocate -- they can hand over inputs and outputs but have no
 * way to provide a scratch buffer.  This entry point takes the arguments of
 * nvfp4_quantize_1d minus the workspace and allocates nothing: the tensor-
 * amax scratch (one partial maximum per CTA of the amax pass) is a static
 * 4 KiB array inside the library (1024 partials), which every GPU that loads
 * the library holds until the process exits.
 *   - The first call on a device looks up that array's device address (with
 *     that device current) and keeps it for later calls; make this first
 *     call before any stream capture.  The address belongs to the CUDA
 *     context current at the lookup: when a call finds another context
 *     current (after cudaDeviceReset, or once the primary context was
 *     released and created again), it looks the address up again, so a
 *     context reset leaves no stale address behind; the first call after the
 *     reset is again a set-up call.
 *   - The amax pass launches at most 4 CTAs per SM, one partial each; on a
 *     device with more than 256 SMs a call that would need more than 1024
 *     partials is refused with NVFP4_ERR_WORKSPACE before anything is
 *     enqueued (the environment variable NVFP4_SM_COUNT, a positive integer,
 *     replaces the device's SM count in all grid sizing of the quantizers;
 *     results do not depend on it, this capacity check does).
 *   - All calls on a device share the array, which keeps the last call's
 *     contents; each call's amax pass overwrites every entry its encode pass
 *     reads, so nothing needs clearing between calls.  Calls that overlap on
 *     the GPU (other streams, or other host threads on the same device) race
 *     on the array: serialize them.
 *   Outputs are bit-identical to nvfp4_quantize_1d's. */
nvfp4_status nvfp4_quantize_1d_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                                       int rounding, uint64_t sr_seed, uint8_t* codes, uint8_t* scales,
                                       uint8_t* scales_mma, float* global_scale, void* stream);

/* Random Hadamard transform + quantization of a wgrad operand ["随机 Hadamard
 * 变换" -- an orthogonal rotation with a random sign diagonal applied before
 * quantization, only on the weight-gradient GEMM inputs; "构造 Hadamard 矩阵的
 * 方法" -- Sylvester construction; "Empat pengaman" -- RHT on the column-
 * quantized wgrad operand, BF16 inputs].
 *   Same arguments as nvfp4_quantize_1d plus rht_seed.  Every 16-chunk of a Q
 *   row is replaced by y = (1/4) H16 (d . chunk) before amax and encoding,
 *   H16 the +-1 Sylvester matrix (H[i][j] = (-1)^popcount(i & j)), computed
 *   by butterflies h = 1, 2, 4, 8 (y_i, y_{i+h}) <- (y_i + y_{i+h},
 *   y_i - y_{i+h}) then a multiply by 0.25; d_j = -1 iff bit j of word 0 of
 *   Philox4x32-10(key = rht_seed, counter = (0, 0, 1, 0)).  Use the same
 *   rht_seed for both operands of one wgrad GEMM: the rotation cancels in the
 *   dot product along K.  Typical use: transpose = 1 (K = tokens innermost),
 *   rounding = NVFP4_SR for the gradient, NVFP4_RNE for the activation. */
nvfp4_status nvfp4_rht_quantize_sr(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                                   uint64_t rht_seed, int rounding, uint64_t sr_seed, uint8_t* codes,
                                   uint8_t* scales, uint8_t* scales_mma, float* global_scale,
                                   void* workspace, size_t ws_bytes, void* stream);

/* The same with an RHT of larger order ["MXFP4 和 NVFP4 的区别", "构造
 * Hadamard 矩阵的方法" -- the Sylvester recursion gives H for every power of
 * two; "为什么不用 Conference 矩阵,而用 Hadamard" -- the fast transform is
 * butterflies of additions and subtractions].
 *   rht_order      n = 16, 32, 64 or 128 (16 is nvfp4_rht_quantize_sr).
 *                  Every n-chunk of a Q row is replaced by
 *                  y = c_n H_n (d . chunk): butterflies h = 1, 2, ..., n/2 as
 *                  above, then one binary32 multiply by c_n = RN(1/sqrt(n))
 *                  (1/4, RN(sqrt 2)/8, 1/8, RN(sqrt 2)/16); d_j = -1 iff bit
 *                  j % 32 of word j / 32 of the same Philox output (the
 *                  16-point signs are its first 16).  Blocks stay 16
 *                  elements, n/16 per chunk.
 *   The length of a Q row (cols, or rows when transpose = 1) must be a
 *   multiple of n: NVFP4_ERR_UNSUPPORTED_SHAPE otherwise; another order is
 *   NVFP4_ERR_INVALID_ARG.  Other arguments, layouts and errors as
 *   nvfp4_rht_quantize_sr. */
nvfp4_status nvfp4_rht_quantize_n(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                                  int rht_order, uint64_t rht_seed, int rounding, uint64_t sr_seed,
                                  uint8_t* codes, uint8_t* scales, uint8_t* scales_mma, float* global_scale,
                                  void* workspace, size_t ws_bytes, void* stream);

/* Both GEMM roles of one tensor in one call ["Empat pengaman" -- the
 * gradient and the activation are each needed row-wise (fprop/dgrad) and,
 * rotated, column-wise (wgrad); "NVFP4 Is a Scaling System", "Where speed and
 * accuracy claims can fail" -- quantization work counts]:
 *   Q1 = x, 1D along cols (as nvfp4_quantize_1d with transpose = 0, sr_seed),
 *   Q2 = RHT(x^T), 1D along rows (as nvfp4_rht_quantize_sr with transpose = 1,
 *        rht_seed, sr_seed_t),
 *   both with `rounding`.  Outputs are bit-identical to the two separate
 *   calls.  The two amax passes share one read of x (the rotated and the
 *   plain maxima are reduced together), so x is read three times instead of
 *   four.  rows and cols multiples of 16; workspace >= 2 *
 *   nvfp4_workspace_size(rows, cols) bytes; codes [rows x cols/2], codes_t
 *   [cols x rows/2], scales / scales_mma as the single calls. */
nvfp4_status nvfp4_quantize_dual(const void* x, int64_t rows, int64_t cols, int64_t ld, int rounding,
                                 uint64_t sr_seed, uint8_t* codes, uint8_t* scales, uint8_t* scales_mma,
                                 float* global_scale, uint64_t rht_seed, uint64_t sr_seed_t, uint8_t* codes_t,
                                 uint8_t* scales_t, uint8_t* scales_mma_t, float* global_scale_t, void* workspace,
                                 size_t ws_bytes, void* stream);

/* 2D (16x16 tile) quantization of a weight, RNE ["2D block scaling for
 * weights" (How does MVFP4 make 4-bit AI training work?); "Empat pengaman" --
 * one scale per 16x16 block makes rowwise and columnwise quantization
 * numerically identical].
 *   w              bf16 [rows x cols], row stride ld; rows, cols multiples of 16.
 *   codes_row      [rows x cols/2] codes of W (required).
 *   codes_col      [cols x rows/2] codes of W^T (nullable) -- the same codes,
 *                  transposed (dgrad operand).
 *   scales         [rows/16 x cols/16] plain tile scales (nullable).
 *   scales_mma_row MMA layout for W as a GEMM operand (R = rows, K = cols),
 *                  nvfp4_mma_scale_bytes(rows, cols) (nullable).
 *   scales_mma_col MMA layout for W^T (R = cols, K = rows) (nullable).
 *   global_scale   one float (required).  One of the scale outputs required. */
nvfp4_status nvfp4_quantize_2d(const void* w, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes_row,
                               uint8_t* codes_col, uint8_t* scales, uint8_t* scales_mma_row,
                               uint8_t* scales_mma_col, float* global_scale, void* workspace,
                               size_t ws_bytes, void* stream);

/* Quantization with the tensor amax already known ["NVFP4 Is a Scaling
 * System, Not Just a 4-Bit Number", "Where speed and accuracy claims can
 * fail" -- quantization and scale handling consume work]: the amax pass,
 * i.e. the first full read of the input, is skipped.  The amax typically comes
 * from the kernel that produced the input (nvfp4_gemm_amax).
 *   amax  device pointer to max |x| over the tensor as it will be quantized
 *         (finite, >= 0).  The result is bit-identical to nvfp4_quantize_1d /
 *         nvfp4_quantize_2d when amax is exact; a larger value gives a valid
 *         but coarser quantization, a smaller one saturates codes at +-6.
 *   No workspace.  Other arguments and outputs as nvfp4_quantize_1d /
 *   nvfp4_quantize_2d (there is no RHT variant: the amax of the rotated
 *   tensor is not known to a producer). */
nvfp4_status nvfp4_quantize_1d_from_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                                         int rounding, uint64_t sr_seed, const float* amax, uint8_t* codes,
                                         uint8_t* scales, uint8_t* scales_mma, float* global_scale, void* stream);
nvfp4_status nvfp4_quantize_2d_from_amax(const void* w, int64_t rows, int64_t cols, int64_t ld, const float* amax,
                                         uint8_t* codes_row, uint8_t* codes_col, uint8_t* scales,
                                         uint8_t* scales_mma_row, uint8_t* scales_mma_col, float* global_scale,
                                         void* stream);

/* Reconstruction x = value(code) * s_block * s_global ["The smallest example:
 * the same payload, two real values"]: out = RN(RN(value * s_block) *
 * s_global) in binary32 (the inner product is exact); NVFP4_OUT_BF16 rounds
 * that to bf16 (nearest even).
 *   codes [rows x cols/2]; scales plain layout (scale_mode 1D: [rows x cols/16],
 *   2D: [rows/16 x cols/16]); global_scale device pointer to one float;
 *   out [rows x cols] (row stride cols).  cols % 16 == 0 (2D: rows % 16 == 0). */
nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int scale_mode,
                              const float* global_scale, int64_t rows, int64_t cols, int out_dtype,
                              void* out, void* stream);

/* Block-scaled NVFP4 GEMM with FP32 accumulation, C = A . B^T (both operands
 * K-major, "TN") ["Presisi sebagai tombol throughput" -- most step time is in
 * the matmuls; "Hardware support still needs a full sentence" -- native
 * block-scaled matrix operations on Blackwell tensor cores]:
 *   C[i][j] = alpha * sum_k (a_ik * sa_i,k/16) * (b_jk * sb_j,k/16),
 *   the sum accumulated in FP32 in tensor memory, then C = RN(sum * alpha)
 *   with alpha = RN(s_global_A * s_global_B).  When that alpha is not a
 *   normal binary32 number (both global scales tiny, product subnormal or
 *   zero; or both huge, product overflowing), the scales are applied one
 *   after the other, C = RN(RN(sum * s_global_A) * s_global_B), so that C
 *   keeps its precision wherever C itself is a normal number.
 *   a_codes [M x K/2], a_scales_mma (MMA layout, R = M), a_gs device float;
 *   b_codes [N x K/2], b_scales_mma (MMA layout, R = N), b_gs device float;
 *   c [M x ldc] FP32 or bf16 (row-major), ldc >= N.
 *   Shapes: M, N >= 1; K a multiple of 64 (K/2 bytes per code row, 16-byte
 *   aligned); ragged M and N tails are handled.  c 16-byte aligned and ldc a
 *   multiple of 8 elements.
 *   Kernel: pairs of CTAs on two SMs computing 256 x 256 tiles (tcgen05
 *   cta_group::2); the environment variable NVFP4_GEMM_PAIR=0 selects the
 *   single-SM kernel (128 x 256 tiles), which meets the same tolerance. */
nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales_mma, const float* a_gs,
                        const uint8_t* b_codes, const uint8_t* b_scales_mma, const float* b_gs, int64_t M,
                        int64_t N, int64_t K, int out_dtype, void* c, int64_t ldc, void* stream);

/* nvfp4_gemm that also produces the tensor amax of its output, so that the
 * next layer can quantize C in one read (nvfp4_quantize_1d_from_amax) ["NVFP4
 * Is a Scaling System, Not Just a 4-Bit Number", "Where speed and accuracy
 * claims can fail"]: c_amax (device float, 4-byte aligned) receives max |C|
 * over the M x N stored values (after the bf16 rounding for a bf16 C).  The
 * library zeroes it first, then every epilogue warp folds its maximum in with
 * one atomic. */
nvfp4_status nvfp4_gemm_amax(const uint8_t* a_codes, const uint8_t* a_scales_mma, const float* a_gs,
                             const uint8_t* b_codes, const uint8_t* b_scales_mma, const float* b_gs, int64_t M,
                             int64_t N, int64_t K, int out_dtype, void* c, int64_t ldc, float* c_amax,
                             void* stream);

/* Re-layout plain scales into the MMA layout (for callers that kept only the
 * plain layout).  scale_mode 1D: scales [rows x k/16]; 2D: [rows/16 x k/16],
 * expanded per row.  scales_mma: nvfp4_mma_scale_bytes(rows, k) bytes. */
nvfp4_status nvfp4_scales_to_mma(const uint8_t* scales, int scale_mode, int64_t rows, int64_t k,
                                 uint8_t* scales_mma, void* stream);

/* MXFP4 ["MXFP4 和 NVFP4 的区别", "MXFP4:开放标准,但精度较粗" -- 32 values
 * share one scale restricted to powers of two, stored as E8M0; "NVFP4 Is a
 * Scaling System, Not Just a 4-Bit Number", "Generic FP4, MXFP4, and NVFP4"
 * -- E2M1 payloads, no tensor-level scale; "Melatih model dalam 4 bit",
 * "Anatomi NVFP4" -- 4.25 bits per element].  The library's MXFP4 variant
 * of the path, for comparison with NVFP4 on the same kernels.
 *
 * Quantize (RNE, one pass: no tensor amax is needed):
 *   per 32-block along K, e = clamp(floor(log2(block amax)) - 2, -127, 127)
 *   (-127 for an all-zero block), scale code = e + 127 (E8M0), element code =
 *   E2M1 nearest-even of x / 2^e, saturating at +-6, sign kept.
 *   x bf16 [rows x cols] (row stride ld); cols % 32 == 0.
 *   codes [rows x cols/2]; scales [rows x cols/32] E8M0 codes (nullable);
 *   scales_mma (nullable, one of the two required): the NVFP4 MMA layout of
 *   nvfp4_mma_scale_bytes(rows, cols) bytes, in which the 4-byte entry of a
 *   row and 64-wide K step holds the step's two E8M0 codes in bytes 0 and 1
 *   and zeros in bytes 2 and 3. */
nvfp4_status nvfp4_mxfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes,
                                  uint8_t* scales, uint8_t* scales_mma, void* stream);

/* MXFP4 reconstruction: out = RN(value(code) * 2^e) in binary32 (exact unless
 * it underflows), NVFP4_OUT_BF16 then rounds to bf16.  codes [rows x cols/2],
 * scales [rows x cols/32] (plain), out [rows x cols]; cols % 32 == 0. */
nvfp4_status nvfp4_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                    int out_dtype, void* out, void* stream);

/* MXFP4 GEMM, C = A . B^T with FP32 accumulation (no global scales, alpha 1):
 * the NVFP4 GEMM kernels with tcgen05.mma block_scale.scale_vec::2X and UE8M0
 * scales.  Operands as nvfp4_gemm (codes K-major, MMA-layout scales from
 * nvfp4_mxfp4_quantize); same shape, alignment and output rules. */
nvfp4_status nvfp4_mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales_mma, const uint8_t* b_codes,
                              const uint8_t* b_scales_mma, int64_t M, int64_t N, int64_t K, int out_dtype, void* c,
                              int64_t ldc, void* stream);

/* Number of kernels (and memset nodes excluded) this library has enqueued in
 * this process; instrumentation for benchmarks. */
long long nvfp4_kernel_launches(void);

/* Synchronizes `stream`, then reads and clears the device error word set by a
 * kernel whose bounded wait ran out (NVFP4_ERR_TIMEOUT) -- no kernel of this
 * library traps or spins without bound.  Returns NVFP4_ERR_CUDA if the stream
 * itself reports an error. */
nvfp4_status nvfp4_get_error(void* stream);

/* Self-test of the failure path (no counterpart on the pages): enqueues one
 * small kernel in which a thread waits, bounded by `limit_ns` nanoseconds, on
 * a barrier that nothing arrives on -- the same bounded wait every pipeline
 * barrier of the GEMM uses.  When the limit runs out the kernel raises the
 * device error word and returns normally, so the next nvfp4_get_error on the
 * stream reports NVFP4_ERR_TIMEOUT and clears it; the context stays usable.
 * No fault, trap or unbounded spin is involved.
 *   limit_ns in [1000, 2e9], else NVFP4_ERR_INVALID_ARG. */
nvfp4_status nvfp4_selftest_wait_timeout(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
