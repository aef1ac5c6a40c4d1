// mxfp4.cu -- MXFP4 quantize and dequantize kernels for sm_100a.
//
// MXFP4 ("MXFP4 和 NVFP4 的区别", section "MXFP4:开放标准,但精度较粗";
// "NVFP4 Is a Scaling System, Not Just a 4-Bit Number", section "Generic
// FP4, MXFP4, and NVFP4"): E2M1 payloads, 32 consecutive values along K share
// one E8M0 scale -- a power of two -- and there is no tensor-level scale.
// The power of two is X = 2^(floor(log2(block amax)) - 2), clamped to
// [2^-127, 2^127] (2^-127 for an all-zero block): the block maximum lands in
// [4, 8), values above 6 saturate.  Element code = E2M1 nearest-even of
// x / X; the division is a multiply by an exact power of two.
// One pass: no global amax is needed, so the input is read once.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace nvfp4 {

namespace {

constexpr int kMxThreads = 256;

// E8M0 scale code of a block from the binary32 bits of its amax (>= 0):
// floor(log2(amax)) = biased exponent - 127 for normal values; below 2^-125
// the clamp at 2^-127 applies, so subnormal amaxes need no special care.
__device__ __forceinline__ uint32_t mx_scale_code(uint32_t amax_bits) {
    const int ebiased = (int)(amax_bits >> 23);
    return (uint32_t)max(ebiased - 2, 0);       // (floor(log2) - 2) + 127, clamped at -127 + 127
}
// 2^-e as binary32 for the scale code c (e = c - 127): bits (254 - c) << 23.
__device__ __forceinline__ float mx_inverse_scale(uint32_t code) { return __uint_as_float((254u - code) << 23); }
// 2^e as binary32 (subnormal for e < -126; exact in every case e <= 127).
__device__ __forceinline__ float mx_scale_value(uint32_t code) {
    return code == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(code << 23);
}

// One thread per 32-block: a warp covers 1024 consecutive columns of a row.
__global__ void __launch_bounds__(kMxThreads) mx_rows_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                             int64_t cols, int64_t ld, uint8_t* __restrict__ codes,
                                                             uint8_t* __restrict__ scales,
                                                             uint8_t* __restrict__ scales_mma, int64_t chunks_k) {
    const int lane = threadIdx.x & 31;
    const int64_t upr = (cols + 1023) >> 10;
    const int64_t total = rows * upr;
    const int64_t nwarps = (int64_t)gridDim.x * (kMxThreads / 32);
    const int64_t kb = cols >> 5;
    for (int64_t u = (int64_t)blockIdx.x * (kMxThreads / 32) + (threadIdx.x >> 5); u < total; u += nwarps) {
        const int64_t row = u / upr;
        const int64_t c0 = (u - row * upr) * 1024 + lane * 32;
        const bool ok = c0 < cols;
        uint32_t w[16];
        if (ok) {
            const uint4* src = reinterpret_cast<const uint4*>(x + row * ld + c0);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint4 v = ldg_stream(reinterpret_cast<const uint16_t*>(src + k));
                w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) w[k] = 0u;
        }
        uint32_t acc = 0;
#pragma unroll
        for (int k = 0; k < 16; ++k) acc = absmax2(acc, w[k]);
        const uint32_t code = mx_scale_code(absmax2_fold(acc));
        const float r = mx_inverse_scale(code);
        const float2 r2 = make_float2(r, r);
        uint32_t out[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 q[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                q[j] = __fmul2_rn(make_float2(bf16_lo(w[4 * k + j]), bf16_hi(w[4 * k + j])), r2);
            out[k] = e2m1x8(q[0].x, q[0].y, q[1].x, q[1].y, q[2].x, q[2].y, q[3].x, q[3].y);
        }
        const int64_t b = c0 >> 5;
        if (ok) {
            *reinterpret_cast<uint4*>(codes + row * (cols >> 1) + (c0 >> 1)) = make_uint4(out[0], out[1], out[2], out[3]);
            if (scales) scales[row * kb + b] = (uint8_t)code;
        }
        if (scales_mma) {
            // blocks 2g, 2g+1 of a row share the 4-byte entry of one 64-wide K
            // step: bytes 0 and 1, bytes 2 and 3 zero
            const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, ok ? code : 0u, 1);
            if (ok && (lane & 1) == 0)
                *reinterpret_cast<uint32_t*>(scales_mma + mma_scale_offset(row, b * 2, chunks_k)) =
                    code | (other << 8);
        }
    }
}

// One thread per 32-block: out = value(code) * 2^e.
__global__ void __launch_bounds__(kMxThreads) mx_dequant_kernel(const uint8_t* __restrict__ codes,
                                                                const uint8_t* __restrict__ scales, int64_t rows,
                                                                int64_t cols, int out_bf16, void* __restrict__ out) {
    const int64_t kb = cols >> 5;
    const int64_t total = rows * kb;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * blockDim.x) {
        const uint4 cw = __ldg(reinterpret_cast<const uint4*>(codes) + u);
        const float s = mx_scale_value(__ldg(scales + u));
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
        float o[32];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t h[4];
            e2m1x8_decode(words[k], h);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 val = __half22float2(*reinterpret_cast<const __half2*>(&h[j]));
                o[8 * k + 2 * j] = __fmul_rn(val.x, s);
                o[8 * k + 2 * j + 1] = __fmul_rn(val.y, s);
            }
        }
        if (out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + u * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint32_t wv[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(o[8 * k + 2 * j], o[8 * k + 2 * j + 1]);
                    wv[j] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                dst[k] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
        } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + u * 32);
#pragma unroll
            for (int k = 0; k < 8; ++k) dst[k] = make_float4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
        }
    }
}

int mx_grid(int64_t work) {
    static int sms = 0;
    if (!sms) {
        int dev = 0, n = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        sms = n > 0 ? n : 148;
    }
    const int64_t g = std::min<int64_t>((int64_t)sms * 8, work);
    return (int)std::max<int64_t>(g, 1);
}

}  // namespace

cudaError_t launch_mx_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes,
                               uint8_t* scales, uint8_t* scales_mma, cudaStream_t s) {
    const int64_t chunks_k = mma_chunks_k(cols);
    if (scales_mma && ((rows % 128) || (cols % 64))) {
        cudaError_t e = cudaMemsetAsync(scales_mma, 0, mma_scale_bytes(rows, cols), s);
        if (e != cudaSuccess) return e;
    }
    const int64_t warps = rows * ((cols + 1023) >> 10);
    mx_rows_kernel<<<mx_grid((warps + 7) / 8), kMxThreads, 0, s>>>(x, rows, cols, ld, codes, scales, scales_mma,
                                                                  chunks_k);
    return cudaGetLastError();
}

cudaError_t launch_mx_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                 int out_bf16, void* out, cudaStream_t s) {
    const int64_t blocks = rows * (cols >> 5);
    mx_dequant_kernel<<<mx_grid((blocks + kMxThreads - 1) / kMxThreads), kMxThreads, 0, s>>>(codes, scales, rows,
                                                                                             cols, out_bf16, out);
    return cudaGetLastError();
}

}  // namespace nvfp4
