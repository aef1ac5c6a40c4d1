// api.cu -- the C ABI (include/nvfp4.h): argument validation on the host, then
// stream-ordered kernel launches.  Nothing here allocates device memory.
#include <atomic>
#include <cstdint>

#include "../../include/nvfp4.h"
#include "internal.h"

using namespace nvfp4;

namespace {

std::atomic<long long> g_launches{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

constexpr size_t kWorkspaceBytes = (size_t)kMaxPartials * sizeof(uint32_t);
constexpr int64_t kMaxDim = (int64_t)1 << 31;   // TMA and index arithmetic bound per dimension

nvfp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

nvfp4_status check_quant_common(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                                int rounding, const uint8_t* codes, const uint8_t* scales,
                                const uint8_t* scales_mma, const float* gs, const void* ws, size_t ws_bytes) {
    if (!x || !codes || !gs || (!scales && !scales_mma)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 1 || cols < 1 || ld < cols || rows >= kMaxDim || cols >= kMaxDim) return NVFP4_ERR_INVALID_ARG;
    if ((transpose != 0 && transpose != 1) || (rounding != NVFP4_RNE && rounding != NVFP4_SR))
        return NVFP4_ERR_INVALID_ARG;
    const int64_t qc = transpose ? rows : cols;
    if (qc % 16 != 0 || cols % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ld % 8 != 0 || !aligned16(x) || !aligned16(codes) || (scales && !aligned16(scales)) ||
        (scales_mma && !aligned16(scales_mma)) || !aligned4(gs))
        return NVFP4_ERR_MISALIGNED;
    if (!ws || ws_bytes < kWorkspaceBytes || !aligned16(ws)) return NVFP4_ERR_WORKSPACE;
    return NVFP4_OK;
}

}  // namespace

extern "C" {

int nvfp4_version(void) { return 101; }

const char* nvfp4_status_string(nvfp4_status s) {
    switch (s) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case NVFP4_ERR_MISALIGNED: return "misaligned pointer or stride";
        case NVFP4_ERR_CUDA: return "CUDA error";
        case NVFP4_ERR_TIMEOUT: return "device wait timed out";
        case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

size_t nvfp4_workspace_size(int64_t rows, int64_t cols) {
    (void)rows;
    (void)cols;
    return kWorkspaceBytes;
}

size_t nvfp4_mma_scale_bytes(int64_t rows, int64_t k) {
    if (rows < 1 || k < 16 || k % 16) return 0;
    return mma_scale_bytes(rows, k);
}

long long nvfp4_kernel_launches(void) { return g_launches.load(); }

static nvfp4_status quantize_1d_impl(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose, int rht,
                                     uint64_t rht_seed, int rounding, uint64_t sr_seed, uint8_t* codes,
                                     uint8_t* scales, uint8_t* scales_mma, float* global_scale, void* workspace,
                                     size_t ws_bytes, void* stream, const float* given_amax = nullptr,
                                     int rht_order = 16) {
    nvfp4_status st = check_quant_common(x, rows, cols, ld, transpose, rounding, codes, scales, scales_mma,
                                         global_scale, workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    if (rht) {
        if (rht_order != 16 && rht_order != 32 && rht_order != 64 && rht_order != 128) return NVFP4_ERR_INVALID_ARG;
        if ((transpose ? rows : cols) % rht_order) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    }
    QuantArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.transpose = transpose;
    a.rht = rht;
    a.rht_order = rht_order;
    a.rht_seed = rht_seed;
    a.rounding = rounding;
    a.sr_seed = sr_seed;
    a.codes = codes;
    a.scales = scales;
    a.scales_mma = scales_mma;
    a.global_scale = global_scale;
    a.partials = static_cast<uint32_t*>(workspace);
    a.given_amax = given_amax;
    int n = 0;
    cudaError_t e = launch_quantize_1d(a, static_cast<cudaStream_t>(stream), &n);
    g_launches += n;
    return from_cuda(e);
}

nvfp4_status nvfp4_quantize_1d(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose, int rounding,
                               uint64_t sr_seed, uint8_t* codes, uint8_t* scales, uint8_t* scales_mma,
                               float* global_scale, void* workspace, size_t ws_bytes, void* stream) {
    return quantize_1d_impl(x, rows, cols, ld, transpose, 0, 0, rounding, sr_seed, codes, scales, scales_mma,
                            global_scale, workspace, ws_bytes, stream);
}

nvfp4_status nvfp4_quantize_1d_from_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                                         int rounding, uint64_t sr_seed, const float* amax, uint8_t* codes,
                                         uint8_t* scales, uint8_t* scales_mma, float* global_scale, void* stream) {
    if (!amax) return NVFP4_ERR_INVALID_ARG;
    if (!aligned4(amax)) return NVFP4_ERR_MISALIGNED;
    // no amax pass, so no workspace: the check gets a placeholder it only compares
    return quantize_1d_impl(x, rows, cols, ld, transpose, 0, 0, rounding, sr_seed, codes, scales, scales_mma,
                            global_scale, reinterpret_cast<void*>(uintptr_t(256)), kWorkspaceBytes, stream, amax);
}

nvfp4_status nvfp4_quantize_1d_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                                       int rounding, uint64_t sr_seed, uint8_t* codes, uint8_t* scales,
                                       uint8_t* scales_mma, float* global_scale, void* stream) {
    // The argument checks of nvfp4_quantize_1d.  There is no caller workspace
    // here (the scratch is the library's static array), so the workspace check
    // is given a placeholder that is only compared, never dereferenced.
    nvfp4_status st = check_quant_common(x, rows, cols, ld, transpose, rounding, codes, scales, scales_mma,
                                         global_scale, reinterpret_cast<const void*>(uintptr_t(256)),
                                         kWorkspaceBytes);
    if (st != NVFP4_OK) return st;
    QuantArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.transpose = transpose;
    a.rounding = rounding;
    a.sr_seed = sr_seed;
    a.codes = codes;
    a.scales = scales;
    a.scales_mma = scales_mma;
    a.global_scale = global_scale;
    int n = 0;
    bool too_big = false;
    cudaError_t e = launch_quantize_1d_noalloc(a, static_cast<cudaStream_t>(stream), &n, &too_big);
    if (too_big) return NVFP4_ERR_WORKSPACE;
    g_launches += n;
    return from_cuda(e);
}

nvfp4_status nvfp4_rht_quantize_sr(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                                   uint64_t rht_seed, int rounding, uint64_t sr_seed, uint8_t* codes,
                                   uint8_t* scales, uint8_t* scales_mma, float* global_scale, void* workspace,
                                   size_t ws_bytes, void* stream) {
    return quantize_1d_impl(x, rows, cols, ld, transpose, 1, rht_seed, rounding, sr_seed, codes, scales,
                            scales_mma, global_scale, workspace, ws_bytes, stream);
}

nvfp4_status nvfp4_rht_quantize_n(const void* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                                  int rht_order, uint64_t rht_seed, int rounding, uint64_t sr_seed, uint8_t* codes,
                                  uint8_t* scales, uint8_t* scales_mma, float* global_scale, void* workspace,
                                  size_t ws_bytes, void* stream) {
    return quantize_1d_impl(x, rows, cols, ld, transpose, 1, rht_seed, rounding, sr_seed, codes, scales,
                            scales_mma, global_scale, workspace, ws_bytes, stream, nullptr, rht_order);
}

static nvfp4_status quantize_2d_impl(const void* w, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes_row,
                                     uint8_t* codes_col, uint8_t* scales, uint8_t* scales_mma_row,
                                     uint8_t* scales_mma_col, float* global_scale, void* workspace,
                                     size_t ws_bytes, void* stream, const float* given_amax) {
    if (!w || !codes_row || !global_scale || (!scales && !scales_mma_row && !scales_mma_col))
        return NVFP4_ERR_INVALID_ARG;
    if (rows < 1 || cols < 1 || ld < cols || rows >= kMaxDim || cols >= kMaxDim) return NVFP4_ERR_INVALID_ARG;
    if (rows % 16 || cols % 16) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ld % 8 || !aligned16(w) || !aligned16(codes_row) || (codes_col && !aligned16(codes_col)) ||
        (scales && !aligned16(scales)) || (scales_mma_row && !aligned16(scales_mma_row)) ||
        (scales_mma_col && !aligned16(scales_mma_col)) || !aligned4(global_scale))
        return NVFP4_ERR_MISALIGNED;
    if (!workspace || ws_bytes < kWorkspaceBytes || !aligned16(workspace)) return NVFP4_ERR_WORKSPACE;
    Quant2dArgs a{};
    a.w = static_cast<const uint16_t*>(w);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.codes_row = codes_row;
    a.codes_col = codes_col;
    a.scales = scales;
    a.scales_mma_row = scales_mma_row;
    a.scales_mma_col = scales_mma_col;
    a.global_scale = global_scale;
    a.partials = static_cast<uint32_t*>(workspace);
    a.given_amax = given_amax;
    int n = 0;
    cudaError_t e = launch_quantize_2d(a, static_cast<cudaStream_t>(stream), &n);
    g_launches += n;
    return from_cuda(e);
}

nvfp4_status nvfp4_quantize_dual(const void* x, int64_t rows, int64_t cols, int64_t ld, int rounding,
                                 uint64_t sr_seed, uint8_t* codes, uint8_t* scales, uint8_t* scales_mma,
                                 float* global_scale, uint64_t rht_seed, uint64_t sr_seed_t, uint8_t* codes_t,
                                 uint8_t* scales_t, uint8_t* scales_mma_t, float* global_scale_t, void* workspace,
                                 size_t ws_bytes, void* stream) {
    // both halves must pass the single-call checks; the workspace holds two sets of partials
    nvfp4_status st = check_quant_common(x, rows, cols, ld, 0, rounding, codes, scales, scales_mma, global_scale,
                                         workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    st = check_quant_common(x, rows, cols, ld, 1, rounding, codes_t, scales_t, scales_mma_t, global_scale_t,
                            workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    if (ws_bytes < 2 * kWorkspaceBytes) return NVFP4_ERR_WORKSPACE;
    QuantArgs r{}, t{};
    r.x = t.x = static_cast<const uint16_t*>(x);
    r.rows = t.rows = rows;
    r.cols = t.cols = cols;
    r.ld = t.ld = ld;
    r.rounding = t.rounding = rounding;
    r.sr_seed = sr_seed;
    r.codes = codes;
    r.scales = scales;
    r.scales_mma = scales_mma;
    r.global_scale = global_scale;
    r.partials = static_cast<uint32_t*>(workspace) + kMaxPartials;
    t.transpose = 1;
    t.rht = 1;
    t.rht_seed = rht_seed;
    t.sr_seed = sr_seed_t;
    t.codes = codes_t;
    t.scales = scales_t;
    t.scales_mma = scales_mma_t;
    t.global_scale = global_scale_t;
    t.partials = static_cast<uint32_t*>(workspace);
    int n = 0;
    cudaError_t e = launch_quantize_dual(r, t, static_cast<cudaStream_t>(stream), &n);
    g_launches += n;
    return from_cuda(e);
}

nvfp4_status nvfp4_quantize_2d(const void* w, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes_row,
                               uint8_t* codes_col, uint8_t* scales, uint8_t* scales_mma_row,
                               uint8_t* scales_mma_col, float* global_scale, void* workspace, size_t ws_bytes,
                               void* stream) {
    return quantize_2d_impl(w, rows, cols, ld, codes_row, codes_col, scales, scales_mma_row, scales_mma_col,
                            global_scale, workspace, ws_bytes, stream, nullptr);
}

nvfp4_status nvfp4_quantize_2d_from_amax(const void* w, int64_t rows, int64_t cols, int64_t ld, const float* amax,
                                         uint8_t* codes_row, uint8_t* codes_col, uint8_t* scales,
                                         uint8_t* scales_mma_row, uint8_t* scales_mma_col, float* global_scale,
                                         void* stream) {
    if (!amax) return NVFP4_ERR_INVALID_ARG;
    if (!aligned4(amax)) return NVFP4_ERR_MISALIGNED;
    return quantize_2d_impl(w, rows, cols, ld, codes_row, codes_col, scales, scales_mma_row, scales_mma_col,
                            global_scale, reinterpret_cast<void*>(uintptr_t(256)), kWorkspaceBytes, stream, amax);
}

nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int scale_mode,
                              const float* global_scale, int64_t rows, int64_t cols, int out_dtype, void* out,
                              void* stream) {
    if (!codes || !scales || !global_scale || !out) return NVFP4_ERR_INVALID_ARG;
    if (scale_mode != NVFP4_SCALE_1D && scale_mode != NVFP4_SCALE_2D) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
    if (rows < 1 || cols < 1 || rows >= kMaxDim || cols >= kMaxDim) return NVFP4_ERR_INVALID_ARG;
    if (cols % 16 || (scale_mode == NVFP4_SCALE_2D && rows % 16)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(codes) || !aligned16(out) || !aligned4(global_scale)) return NVFP4_ERR_MISALIGNED;
    cudaError_t e = launch_dequantize(codes, scales, scale_mode, global_scale, rows, cols,
                                      out_dtype == NVFP4_OUT_BF16, out, static_cast<cudaStream_t>(stream));
    g_launches += 1;
    return from_cuda(e);
}

static nvfp4_status gemm_impl(const uint8_t* a_codes, const uint8_t* a_scales_mma, const float* a_gs,
                              const uint8_t* b_codes, const uint8_t* b_scales_mma, const float* b_gs, int64_t M,
                              int64_t N, int64_t K, int out_dtype, void* c, int64_t ldc, float* c_amax,
                              void* stream, int mx = 0) {
    if (!a_codes || !a_scales_mma || !b_codes || !b_scales_mma || !c) return NVFP4_ERR_INVALID_ARG;
    if (!mx && (!a_gs || !b_gs)) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 1 || ldc < N || M >= kMaxDim || N >= kMaxDim || K >= kMaxDim)
        return NVFP4_ERR_INVALID_ARG;
    if (K % 64) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales_mma) || !aligned16(b_scales_mma) ||
        !aligned16(c) || ldc % 8 || (!mx && (!aligned4(a_gs) || !aligned4(b_gs))))
        return NVFP4_ERR_MISALIGNED;
    GemmArgs g{};
    g.a = a_codes;
    g.sfa = a_scales_mma;
    g.a_gs = a_gs;
    g.b = b_codes;
    g.sfb = b_scales_mma;
    g.b_gs = b_gs;
    g.M = M;
    g.N = N;
    g.K = K;
    g.out_bf16 = out_dtype == NVFP4_OUT_BF16;
    g.c = c;
    g.ldc = ldc;
    g.c_amax = c_amax;
    g.mx = mx;
    if (c_amax) {
        cudaError_t z = cudaMemsetAsync(c_amax, 0, sizeof(float), static_cast<cudaStream_t>(stream));
        if (z != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    cudaError_t e = launch_gemm(g, static_cast<cudaStream_t>(stream));
    g_launches += 1;
    return from_cuda(e);
}

nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales_mma, const float* a_gs,
                        const uint8_t* b_codes, const uint8_t* b_scales_mma, const float* b_gs, int64_t M,
                        int64_t N, int64_t K, int out_dtype, void* c, int64_t ldc, void* stream) {
    return gemm_impl(a_codes, a_scales_mma, a_gs, b_codes, b_scales_mma, b_gs, M, N, K, out_dtype, c, ldc, nullptr,
                     stream);
}

nvfp4_status nvfp4_gemm_amax(const uint8_t* a_codes, const uint8_t* a_scales_mma, const float* a_gs,
                             const uint8_t* b_codes, const uint8_t* b_scales_mma, const float* b_gs, int64_t M,
                             int64_t N, int64_t K, int out_dtype, void* c, int64_t ldc, float* c_amax,
                             void* stream) {
    if (!c_amax) return NVFP4_ERR_INVALID_ARG;
    if (!aligned4(c_amax)) return NVFP4_ERR_MISALIGNED;
    return gemm_impl(a_codes, a_scales_mma, a_gs, b_codes, b_scales_mma, b_gs, M, N, K, out_dtype, c, ldc, c_amax,
                     stream);
}

nvfp4_status nvfp4_mxfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes,
                                  uint8_t* scales, uint8_t* scales_mma, void* stream) {
    if (!x || !codes || (!scales && !scales_mma)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 1 || cols < 1 || ld < cols || rows >= kMaxDim || cols >= kMaxDim) return NVFP4_ERR_INVALID_ARG;
    if (cols % 32) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ld % 8 || !aligned16(x) || !aligned16(codes) || (scales_mma && !aligned16(scales_mma)))
        return NVFP4_ERR_MISALIGNED;
    cudaError_t e = launch_mx_quantize(static_cast<const uint16_t*>(x), rows, cols, ld, codes, scales, scales_mma,
                                       static_cast<cudaStream_t>(stream));
    g_launches += 1;
    return from_cuda(e);
}

nvfp4_status nvfp4_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                    int out_dtype, void* out, void* stream) {
    if (!codes || !scales || !out) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
    if (rows < 1 || cols < 1 || rows >= kMaxDim || cols >= kMaxDim) return NVFP4_ERR_INVALID_ARG;
    if (cols % 32) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(codes) || !aligned16(out)) return NVFP4_ERR_MISALIGNED;
    cudaError_t e = launch_mx_dequantize(codes, scales, rows, cols, out_dtype == NVFP4_OUT_BF16, out,
                                         static_cast<cudaStream_t>(stream));
    g_launches += 1;
    return from_cuda(e);
}

nvfp4_status nvfp4_mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales_mma, const uint8_t* b_codes,
                              const uint8_t* b_scales_mma, int64_t M, int64_t N, int64_t K, int out_dtype, void* c,
                              int64_t ldc, void* stream) {
    return gemm_impl(a_codes, a_scales_mma, nullptr, b_codes, b_scales_mma, nullptr, M, N, K, out_dtype, c, ldc,
                     nullptr, stream, 1);
}

nvfp4_status nvfp4_scales_to_mma(const uint8_t* scales, int scale_mode, int64_t rows, int64_t k,
                                 uint8_t* scales_mma, void* stream) {
    if (!scales || !scales_mma) return NVFP4_ERR_INVALID_ARG;
    if (scale_mode != NVFP4_SCALE_1D && scale_mode != NVFP4_SCALE_2D) return NVFP4_ERR_INVALID_ARG;
    if (rows < 1 || k < 16 || rows >= kMaxDim || k >= kMaxDim) return NVFP4_ERR_INVALID_ARG;
    if (k % 16 || (scale_mode == NVFP4_SCALE_2D && rows % 16)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    cudaError_t e = launch_scales_to_mma(scales, scale_mode, rows, k, scales_mma, static_cast<cudaStream_t>(stream));
    g_launches += 1;
    return from_cuda(e);
}

nvfp4_status nvfp4_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1000 || limit_ns > 2000000000ull) return NVFP4_ERR_INVALID_ARG;
    g_launches.fetch_add(1);
    return launch_wait_selftest((unsigned long long)limit_ns, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? NVFP4_OK
               : NVFP4_ERR_CUDA;
}

nvfp4_status nvfp4_get_error(void* stream) {
    cudaError_t err = cudaSuccess;
    const unsigned int w = read_and_clear_error_word(static_cast<cudaStream_t>(stream), &err);
    if (err != cudaSuccess) return NVFP4_ERR_CUDA;
    return w ? NVFP4_ERR_TIMEOUT : NVFP4_OK;
}

}  // extern "C"
