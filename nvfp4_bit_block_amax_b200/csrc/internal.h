// internal.h -- host-side launchers shared between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

// Grid of the amax pass: one partial maximum per CTA, reduced by every CTA of
// the quantize pass that follows on the same stream.
constexpr int kMaxPartials = 4096;

struct QuantArgs {
    const uint16_t* x;
    int64_t rows, cols, ld;       // input [rows x cols], row stride ld (elements)
    int transpose;                // Q = x (0) or x^T (1)
    int rht;                      // RHT along Q rows
    int rht_order;                // its order: 16 (0 also means 16), 32, 64 or 128
    uint64_t rht_seed;
    int rounding;                 // 0 RNE, 1 SR
    uint64_t sr_seed;
    uint8_t* codes;               // [Qr x Qc/2]
    uint8_t* scales;              // [Qr x Qc/16] or nullptr
    uint8_t* scales_mma;          // MMA layout or nullptr
    float* global_scale;
    uint32_t* partials;           // workspace
    const float* given_amax;      // non-null: the tensor amax is known, skip the amax pass
};

struct Quant2dArgs {
    const uint16_t* w;
    int64_t rows, cols, ld;
    uint8_t* codes_row;
    uint8_t* codes_col;           // nullable
    uint8_t* scales;              // nullable
    uint8_t* scales_mma_row;      // nullable
    uint8_t* scales_mma_col;      // nullable
    float* global_scale;
    uint32_t* partials;
    const float* given_amax;      // non-null: the tensor amax is known, skip the amax pass
};

cudaError_t launch_quantize_1d(const QuantArgs& a, cudaStream_t s, int* launches);
cudaError_t launch_quantize_2d(const Quant2dArgs& a, cudaStream_t s, int* launches);
cudaError_t launch_quantize_dual(const QuantArgs& r, const QuantArgs& t, cudaStream_t s, int* launches);
cudaError_t launch_quantize_1d_noalloc(const QuantArgs& a, cudaStream_t s, int* launches, bool* too_big);
int noalloc_capacity();
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, int scale_mode, const float* gs,
                              int64_t rows, int64_t cols, int out_bf16, void* out, cudaStream_t s);
cudaError_t launch_scales_to_mma(const uint8_t* scales, int scale_mode, int64_t rows, int64_t k,
                                 uint8_t* scales_mma, cudaStream_t s);

struct GemmArgs {
    const uint8_t* a;
    const uint8_t* sfa;
    const float* a_gs;
    const uint8_t* b;
    const uint8_t* sfb;
    const float* b_gs;
    int64_t M, N, K;
    int out_bf16;
    void* c;
    int64_t ldc;
    float* c_amax;                // non-null: also max |C| over the stored values (zeroed by the caller)
    int mx;                       // MXFP4 operands (UE8M0 per 32, a_gs = b_gs = nullptr, alpha = 1)
};
cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s);

unsigned int read_and_clear_error_word(cudaStream_t s, cudaError_t* err);
cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t s);
cudaError_t launch_mx_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes,
                               uint8_t* scales, uint8_t* scales_mma, cudaStream_t s);
cudaError_t launch_mx_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                 int out_bf16, void* out, cudaStream_t s);

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t mma_chunks_k(int64_t k) { return ceil_div(k / 16, 4); }
inline size_t mma_scale_bytes(int64_t rows, int64_t k) {
    return (size_t)(ceil_div(rows, 128) * mma_chunks_k(k) * 512);
}

}  // namespace nvfp4
