// quant.cu -- NVFP4 quantizer kernels for sm_100a.  The round-to-nearest
// passes are bound by HBM bandwidth; the stochastic-rounding and RHT passes
// by instruction issue (16 Philox bits per element, the butterflies).
//
// Steps (sources: "Melatih model dalam 4 bit: pengaman numerik di balik NVFP4",
// "Anatomi NVFP4" and "Empat pengaman"; "MXFP4 和 NVFP4 的区别", "精度核心:
// 两级分层缩放", "随机舍入", "随机 Hadamard 变换", "构造 Hadamard 矩阵的方法";
// "NVFP4 Is a Scaling System, Not Just a 4-Bit Number", "Why two levels":
// the global scale comes from the tensor amax before the block maxima):
//   pass 1 (amax):  A = max |Q| over the tensor (Q rotated when RHT is on;
//                   the 16-point transform's 1/4 is applied to the maximum,
//                   see kRht16Norm); one partial maximum per CTA into the
//                   caller's workspace.
//   pass 2 (encode): every CTA folds the partials into A, s_global =
//                   RN(A / 2688); per 16-block: block amax, E4M3 scale, E2M1
//                   codes (RNE or stochastic rounding), packed two per byte.
// All floating-point steps are single IEEE binary32 operations in the order
// stated in nvfp4.h (this file is built with --fmad=false).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <mutex>

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// SM count of the current device, cached per device.  NVFP4_SM_COUNT, when
// set to a positive integer, replaces it in the grid sizing (the kernels'
// results do not depend on the grid; the allocation-free entry point's
// capacity check does, which is how that check is exercised without a GPU).
int sm_count() {
    if (const char* o = getenv("NVFP4_SM_COUNT")) {
        const int n = atoi(o);
        if (n > 0) return n;
    }
    static std::atomic<int> cached[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (!n) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// ------------------------------------------------------------ amax (plain) --
// Tensor amax of a bf16 tensor without rotation: transposing does not change
// it.  16-byte streaming loads, 16-bit integer magnitude maxima.
template <bool CONTIG>
__global__ void __launch_bounds__(kThreads) amax_plain_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                              int64_t cols, int64_t ld,
                                                              uint32_t* __restrict__ partials) {
    const int64_t cpr = cols >> 3;
    const int64_t nvec = rows * cpr;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    auto addr = [&](int64_t i) -> const uint16_t* {
        if (CONTIG) return x + (i << 3);
        const int64_t r = i / cpr;
        return x + r * ld + ((i - r * cpr) << 3);
    };
    uint32_t acc = 0;
    for (; v + (kUnroll - 1) * stride < nvec; v += kUnroll * stride) {
        uint4 a[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) a[u] = ldg_stream(addr(v + u * stride));
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            acc = absmax2(absmax2(absmax2(absmax2(acc, a[u].x), a[u].y), a[u].z), a[u].w);
    }
    for (; v < nvec; v += stride) {
        const uint4 a = ldg_stream(addr(v));
        acc = absmax2(absmax2(absmax2(absmax2(acc, a.x), a.y), a.z), a.w);
    }
    __shared__ uint32_t s_red[kThreads / 32];
    uint32_t m = __reduce_max_sync(0xFFFFFFFFu, absmax2_fold(acc));
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < (kThreads / 32) ? s_red[threadIdx.x] : 0u;
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        if (threadIdx.x == 0) partials[blockIdx.x] = m;
    }
}

// Block-level max of non-negative float bits, written as this CTA's partial.
__device__ __forceinline__ void write_partial(uint32_t m, uint32_t* partials) {
    __shared__ uint32_t s_red[kThreads / 32];
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < (kThreads / 32) ? s_red[threadIdx.x] : 0u;
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        if (threadIdx.x == 0) partials[blockIdx.x] = m;
    }
}

struct Params {
    const uint16_t* x;
    int64_t rows, cols, ld;
    uint64_t rht_seed, sr_seed;
    PhiloxKeys sr_keys;           // round keys of sr_seed
    SignWords rht_sign;           // RHT signs of the 16 positions of a chunk, as unpack masks
    uint8_t* codes;
    uint8_t* scales;
    uint8_t* scales_mma;
    int64_t chunks_k;
    float* global_scale;
    uint32_t* partials;
    int n_partials;
    uint32_t* partials2;          // amax pass of the dual quantizer: plain |x| maxima here too
};

// Global scale from the amax partials; block 0 publishes it.
__device__ __forceinline__ void global_scales(const Params& p, float& sg, float& t) {
    const float A = reduce_partials(p.partials, p.n_partials);
    sg = __fdiv_rn(A, kGlobalDiv);
    t = __fmul_rn(6.0f, sg);
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.global_scale = sg;
}

// 32-byte load of 16 bf16 values (one block).  A single 256-bit load when the
// address is 32-byte aligned, else two 16-byte loads.
__device__ __forceinline__ void load_block(const uint16_t* p, bool a32, uint32_t w[8]) {
    if (a32) {
        asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
                       "=r"(w[7])
                     : "l"(p));
    } else {
        const uint4 a = ldg_stream(p), b = ldg_stream(p + 8);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
}

// Butterflies h = 1, 2, 4, 8 of a 16-point RHT chunk held by one thread
// (pairs of independent butterflies packed into f32x2 adds); the signs are
// applied by the caller.
__device__ __forceinline__ void rht16_butterflies(float y[16]) {
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
        int idx[8];
        int n = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (!(i & h)) idx[n++] = i;
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
            const int i0 = idx[k], i1 = idx[k + 1];
            const float2 a = make_float2(y[i0], y[i1]);
            const float2 b = make_float2(y[i0 + h], y[i1 + h]);
            const float2 sum = __fadd2_rn(a, b);
            const float2 dif = __fadd2_rn(a, make_float2(-b.x, -b.y));
            y[i0] = sum.x;
            y[i1] = sum.y;
            y[i0 + h] = dif.x;
            y[i1 + h] = dif.y;
        }
    }
}

__device__ __forceinline__ void scale_regs(float y[16], float c) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        const float2 v = __fmul2_rn(make_float2(y[i], y[i + 1]), make_float2(c, c));
        y[i] = v.x;
        y[i + 1] = v.y;
    }
}

// The butterflies h = 16, 32, .. of a (16 << LOGM)-point RHT whose 16-point
// pieces sit in 2^LOGM consecutive lanes (piece index = lane bits 0..LOGM-1):
// the lane with bit s clear keeps a + b, its partner a - b, a being the
// lower piece's value -- the order and rounding of the sequential butterflies.
template <int LOGM>
__device__ __forceinline__ void rht_cross_lanes(float y[16], int lane) {
#pragma unroll
    for (int s = 0; s < LOGM; ++s) {
        // upper: o + (-y) = a - b; lower: o + y = a + b (addition commutes,
        // the sign flip is exact)
        const float sg = ((lane >> s) & 1) ? -1.0f : 1.0f;
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const float2 o = make_float2(__shfl_xor_sync(0xFFFFFFFFu, y[i], 1 << s),
                                         __shfl_xor_sync(0xFFFFFFFFu, y[i + 1], 1 << s));
            const float2 v = __fadd2_rn(o, __fmul2_rn(make_float2(y[i], y[i + 1]), make_float2(sg, sg)));
            y[i] = v.x;
            y[i + 1] = v.y;
        }
    }
}

// Encode one 16-block held by one thread: codes for elements 0..7 (lo) and
// 8..15 (hi).  SR draws its bits for output elements 8g .. 8g+15.
template <bool SR>
__device__ __forceinline__ void encode16(const float y[16], const BlockScale& bs, const PhiloxKeys& sr_keys,
                                         uint64_t g, uint32_t& lo, uint32_t& hi) {
    float q[16];
    if (!isinf(bs.r)) {
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const float2 v = __fmul2_rn(make_float2(y[i], y[i + 1]), make_float2(bs.r, bs.r));
            q[i] = v.x;
            q[i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = scaled_inf(y[i]);
    }
    if (SR) {
        const uint4 r0 = sr_bits8(sr_keys, g);
        const uint4 r1 = sr_bits8(sr_keys, g + 1);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            sr_grid2(q[i], q[i + 1], sr_u16(r0, i), sr_u16(r0, i + 1));
            sr_grid2(q[i + 8], q[i + 9], sr_u16(r1, i), sr_u16(r1, i + 1));
        }
    }
    lo = e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
    hi = e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
}

// ------------------------------------------------- rowwise 1D (Q = x) --------
// One thread per 16-block: a warp takes 512 consecutive columns of a Q row
// (32 blocks) per unit, consecutive units per warp, 2 units in flight.
// RHT of order 16 << LOGM: a chunk is 2^LOGM consecutive lanes (Q rows hold
// a multiple of the order, so a chunk never straddles the end of a row).
template <bool RHT, bool SR, bool AMAX_ONLY, int LOGM = 0>
__global__ void __launch_bounds__(kThreads) rows_kernel(Params p) {
    __shared__ float s_rtab[128];
    ScaleCtx ctx{};
    if (!AMAX_ONLY) {
        float sg, t;
        global_scales(p, sg, t);
        ctx = make_scale_ctx(sg, t, s_rtab);
    }
    const int lane = threadIdx.x & 31;
    uint32_t sw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (RHT) {
        const uint32_t d = LOGM == 0 ? rht_sign_mask(p.rht_seed)
                                     : rht_sign_mask_at(p.rht_seed, 16 * (lane & ((1 << LOGM) - 1)));
#pragma unroll
        for (int k = 0; k < 8; ++k)
            sw[k] = (((d >> (2 * k)) & 1u) ? 0x8000u : 0u) | (((d >> (2 * k + 1)) & 1u) ? 0x80000000u : 0u);
    }
    const int64_t upr = (p.cols + 511) >> 9;
    const int64_t total = p.rows * upr;
    const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t wid = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    // Groups of U consecutive units, interleaved over the warps (group g goes
    // to warp g mod nwarps): at any moment the grid works on a narrow window of
    // the tensor, which keeps the address translations it needs few.
    constexpr int U = 2;
    const int64_t step = nwarps * U;                   // units between a warp's groups
    const int64_t step_rows = step / upr, step_uc = step - step_rows * upr;
    int64_t u = wid * U;
    const int64_t uend = total;
    const int64_t kb = p.cols >> 4;
    const int64_t chunks512 = p.chunks_k << 9;         // bytes per 128-row band of the GEMM scale layout
    const bool a32 = ((reinterpret_cast<uintptr_t>(p.x) & 31u) == 0) && ((p.ld & 15) == 0);
    uint32_t amax_bits = 0;
    if (u < uend) {
        int64_t row0 = u / upr;
        int64_t uc0 = u - row0 * upr;
        for (; u < uend; u += step) {
            uint32_t w[U][8];
            int64_t rr[U], cc[U];
            bool ok[U];
            int64_t row = row0, uc = uc0;
#pragma unroll
            for (int k = 0; k < U; ++k) {
                rr[k] = row;
                cc[k] = uc * 512 + lane * 16;
                ok[k] = (u + k < uend) && (cc[k] < p.cols);
                if (ok[k]) {
                    load_block(p.x + row * p.ld + cc[k], a32, w[k]);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) w[k][j] = 0u;
                }
                if (++uc == upr) {
                    uc = 0;
                    ++row;
                }
            }
            // the next group of this warp
            row0 += step_rows;
            uc0 += step_uc;
            if (uc0 >= upr) {
                uc0 -= upr;
                ++row0;
            }
#pragma unroll
            for (int k = 0; k < U; ++k) {
                float y[16];
                float bmax;
                if (RHT) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t ww = w[k][j] ^ sw[j];
                        y[2 * j] = bf16_lo(ww);
                        y[2 * j + 1] = bf16_hi(ww);
                    }
                    rht16_butterflies(y);
                    if (LOGM > 0) rht_cross_lanes<LOGM>(y, lane);
                    // the 16-point amax pass applies the 1/4 to its maximum (kRht16Norm)
                    if (!(AMAX_ONLY && LOGM == 0)) scale_regs(y, rht_norm<LOGM>());
                    bmax = 0.0f;
#pragma unroll
                    for (int j = 0; j < 16; j += 2) bmax = max3f(bmax, fabsf(y[j]), fabsf(y[j + 1]));
                } else {
                    uint32_t acc = 0;
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc = absmax2(acc, w[k][j]);
                    bmax = __uint_as_float(absmax2_fold(acc));
                }
                if (AMAX_ONLY) {
                    if (ok[k]) amax_bits = max(amax_bits, __float_as_uint(bmax));
                    continue;
                }
                if (u + k >= uend) continue;   // the same for the whole warp
                if (!RHT) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        y[2 * j] = bf16_lo(w[k][j]);
                        y[2 * j + 1] = bf16_hi(w[k][j]);
                    }
                }
                // Lanes past the end of the row hold zeros and encode zero
                // scales, which is what the padded GEMM scale layout holds.
                const BlockScale bs = block_scale(bmax, ctx);
                uint32_t lo, hi;
                encode16<SR>(y, bs, p.sr_keys, (uint64_t)(rr[k] * p.cols + cc[k]) >> 3, lo, hi);
                const int64_t b = cc[k] >> 4;
                if (ok[k]) {
                    *reinterpret_cast<uint2*>(p.codes + rr[k] * (p.cols >> 1) + (cc[k] >> 1)) = make_uint2(lo, hi);
                    if (p.scales) p.scales[rr[k] * kb + b] = (uint8_t)bs.code;
                }
                if (p.scales_mma && ok[k]) {
                    // Blocks 4g .. 4g+3 of a row are 4 consecutive bytes of the
                    // GEMM layout, so lanes 4g .. 4g+3 each store their own byte
                    // (the four land in one sector; gathering them into a word
                    // first cost two shuffles and the full offset arithmetic in
                    // every lane).  This is mma_scale_offset(r, b) with the row
                    // part in 32 bits (r < 2^31) and b & 3 = lane & 3.  Bytes of
                    // a group past the row's end stay as the launch zeroed them.
                    const uint32_t r32 = (uint32_t)rr[k];
                    const int64_t off = (int64_t)(r32 >> 7) * chunks512 + ((cc[k] >> 6) << 9) +
                                        (int64_t)(((r32 & 31u) << 4) | (((r32 >> 5) & 3u) << 2) | (uint32_t)(lane & 3));
                    p.scales_mma[off] = (uint8_t)bs.code;
                }
            }
        }
    }
    if (AMAX_ONLY) {
        if (RHT && LOGM == 0) amax_bits = __float_as_uint(__uint_as_float(amax_bits) * kRht16Norm);
        write_partial(amax_bits, p.partials);
    }
}

// ------------------------------------- rowwise 1D, stochastic rounding ------
// Stochastic rounding needs 16 Philox bits per element, which makes the
// encode pass instruction-bound: this kernel keeps the per-block bookkeeping
// small by giving each thread 64 consecutive elements of a Q row (4 blocks,
// one 128-byte span): one Philox counter base, one 32-byte code store pair,
// and the 4 block scales of a row are exactly one 32-bit word of the GEMM
// scale layout.  A warp takes 32 such units (2048 columns) of one row at a
// time; segments are dealt to the warps in order.  RHT (16-point): the signs
// are folded into the bf16 unpack (sign words from the parameter bank).
template <bool RHT>
__global__ void __launch_bounds__(kThreads) rows_sr_kernel(Params p) {
    __shared__ float s_rtab[128];
    float sg, t;
    global_scales(p, sg, t);
    const ScaleCtx ctx = make_scale_ctx(sg, t, s_rtab);
    const int lane = threadIdx.x & 31;
    const int64_t C = p.cols;
    const int64_t upr = (C + 63) >> 6;                   // 64-element units per row
    const int64_t spr = (upr + 31) >> 5;                 // 32-unit warp segments per row
    const int64_t items = p.rows * spr;
    const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
    int64_t item = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    if (item >= items) return;                           // (no block-wide barrier below)
    int64_t row = item / spr, seg = item - row * spr;
    const int64_t step_rows = nwarps / spr, step_seg = nwarps - step_rows * spr;
    const bool a32 = ((reinterpret_cast<uintptr_t>(p.x) & 31u) == 0) && ((p.ld & 15) == 0);
    const bool c16 = ((C & 63) == 0) && ((reinterpret_cast<uintptr_t>(p.codes) & 15u) == 0);
    const int64_t chunks512 = p.chunks_k << 9;         // bytes per 128-row band of the GEMM scale layout
    for (; item < items; item += nwarps) {
        const int64_t col0 = ((seg << 5) + lane) << 6;
        const int nb = col0 < C ? (int)min((int64_t)4, (C - col0) >> 4) : 0;   // blocks of this unit inside the row
        uint32_t w[4][8];
        const uint16_t* src = p.x + row * p.ld + col0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            if (b < nb) load_block(src + 16 * b, a32, w[b]);
            else {
#pragma unroll
                for (int j = 0; j < 8; ++j) w[b][j] = 0u;
            }
        }
        const uint64_t g0 = (uint64_t)(row * C + col0) >> 3;   // Philox counter of the unit's first 8 elements
        uint32_t cw[8];
        uint32_t sword = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float y[16];
            float bmax;
            if (RHT) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    y[2 * j] = bf16_lo_signed(w[b][j], p.rht_sign.m[2 * j]);
                    y[2 * j + 1] = bf16_hi_signed(w[b][j], p.rht_sign.m[2 * j + 1]);
                }
                rht16_butterflies(y);
                scale_regs(y, 0.25f);
                bmax = 0.0f;
#pragma unroll
                for (int j = 0; j < 16; j += 2) bmax = max3f(bmax, fabsf(y[j]), fabsf(y[j + 1]));
            } else {
                uint32_t acc = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) acc = absmax2(acc, w[b][j]);
                bmax = __uint_as_float(absmax2_fold(acc));
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    y[2 * j] = bf16_lo(w[b][j]);
                    y[2 * j + 1] = bf16_hi(w[b][j]);
                }
            }
            // blocks past the row's end hold zeros: zero scale, codes not stored
            const BlockScale bs = block_scale(bmax, ctx);
            encode16<true>(y, bs, p.sr_keys, g0 + 2 * b, cw[2 * b], cw[2 * b + 1]);
            if (b < nb) sword |= bs.code << (8 * b);
        }
        if (nb > 0) {
            uint8_t* cp = p.codes + row * (C >> 1) + (col0 >> 1);
            if (nb == 4 && c16) {
                *reinterpret_cast<uint4*>(cp) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                *reinterpret_cast<uint4*>(cp + 16) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
            } else {
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    if (b < nb) *reinterpret_cast<uint2*>(cp + 8 * b) = make_uint2(cw[2 * b], cw[2 * b + 1]);
            }
            if (p.scales) {
                uint8_t* sp = p.scales + row * (C >> 4) + (col0 >> 4);
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    if (b < nb) sp[b] = (uint8_t)(sword >> (8 * b));
            }
            // blocks 4g .. 4g+3 of the row: one word of the GEMM layout (zeros past the row's end)
            if (p.scales_mma) {
                // mma_scale_offset(row, col0 / 16) with the row part in 32 bits
                // (row < 2^31) and col0 / 16 a multiple of 4
                const uint32_t r32 = (uint32_t)row;
                const int64_t off = (int64_t)(r32 >> 7) * chunks512 + ((col0 >> 6) << 9) +
                                    (int64_t)(((r32 & 31u) << 4) | (((r32 >> 5) & 3u) << 2));
                *reinterpret_cast<uint32_t*>(p.scales_mma + off) = sword;
            }
        }
        row += step_rows;
        seg += step_seg;
        if (seg >= spr) {
            seg -= spr;
            ++row;
        }
    }
}

// ---------------------------------------------- transposed 1D (Q = x^T) -------
// x is [T x F] (tokens x features); Q = x^T is [F x T] with 16-blocks along
// tokens.  CTA tile: 128 tokens x 256 features; warp w: tokens 16w..16w+15,
// lane: 8 features, so a thread holds 8 whole blocks (one per feature) and
// the RHT runs in registers.  Codes are staged in shared memory and written
// as 8-byte row segments of Q.
// RHT of order 16 << LOGM (LOGM <= 3): the same tile, mapped so that the
// pieces of a chunk share a warp -- warp w: features 32w .. 32w+31; lane:
// 16-token piece lane >> 2, 8 features from 8 * (lane & 3) -- and the
// butterflies h >= 16 are shuffles between lanes lane ^ 4, ^ 8, ^ 16.
// The 16-point stochastic-rounding encode stores each thread's 8-byte code
// segments straight from registers instead (the four warps of a tile fill
// each 32-byte sector between them): that pass is bound by instruction issue,
// and the staging copy's shared-memory traffic and barrier cost more than the
// narrower global stores.  With round-to-nearest the staged store is faster.
template <bool RHT, bool SR, bool AMAX_ONLY, int LOGM = 0>
__global__ void __launch_bounds__(kThreads, 2) cols_kernel(Params p) {
    constexpr bool kDirect = RHT && SR && !AMAX_ONLY && LOGM == 0;
    __shared__ __align__(16) uint8_t s_codes[(AMAX_ONLY || kDirect) ? 16 : 256 * 64];
    __shared__ __align__(16) uint8_t s_sc[AMAX_ONLY ? 1 : 256][8];   // [feature in tile][token block in tile]
    __shared__ float s_rtab[128];
    ScaleCtx ctx{};
    if (!AMAX_ONLY) {
        float sg, t;
        global_scales(p, sg, t);
        ctx = make_scale_ctx(sg, t, s_rtab);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int piece = LOGM == 0 ? warp : (lane >> 2);                     // 16-token block in the tile
    const int fl0 = LOGM == 0 ? lane * 8 : warp * 32 + (lane & 3) * 8;    // first of 8 features in the tile
    const uint32_t dmask = !RHT ? 0u
                           : LOGM == 0 ? rht_sign_mask(p.rht_seed)
                                       : rht_sign_mask_at(p.rht_seed, 16 * (piece & ((1 << LOGM) - 1)));
    const int64_t T = p.rows, F = p.cols;
    const int64_t ntt = (T + 127) >> 7, nft = (F + 255) >> 8;
    const int64_t ntiles = ntt * nft;
    const int64_t kb = T >> 4;
    uint32_t amax_bits = 0, plain_acc = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t tt = tile / nft, ft = tile - tt * nft;
        const int64_t t0 = tt * 128 + piece * 16;
        const int64_t f0 = ft * 256 + fl0;
        const bool ok = (t0 < T) && (f0 < F);
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            v[i] = ok ? ldg_stream(p.x + (t0 + i) * p.ld + f0) : make_uint4(0u, 0u, 0u, 0u);
        if (AMAX_ONLY && p.partials2) {   // the un-rotated amax from the same read
#pragma unroll
            for (int i = 0; i < 16; ++i)
                plain_acc = absmax2(absmax2(absmax2(absmax2(plain_acc, v[i].x), v[i].y), v[i].z), v[i].w);
        }
#pragma unroll
        for (int jp = 0; jp < 4; ++jp) {
            float2 y[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                uint32_t w = jp == 0 ? v[i].x : jp == 1 ? v[i].y : jp == 2 ? v[i].z : v[i].w;
                if (RHT && LOGM == 0) {   // signs folded into the unpack (sign words from the parameter bank)
                    y[i] = make_float2(bf16_lo_signed(w, p.rht_sign.m[i]), bf16_hi_signed(w, p.rht_sign.m[i]));
                    continue;
                }
                if (RHT && ((dmask >> i) & 1u)) w ^= 0x80008000u;
                y[i] = make_float2(bf16_lo(w), bf16_hi(w));
            }
            if (RHT) {
#pragma unroll
                for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (i & h) continue;
                        const float2 a = y[i], b = y[i + h];
                        y[i] = __fadd2_rn(a, b);
                        y[i + h] = __fadd2_rn(a, make_float2(-b.x, -b.y));
                    }
                }
#pragma unroll
                for (int s = 0; s < LOGM; ++s) {
                    // lower piece: o + y = a + b; upper: o + (-y) = a - b
                    // (addition commutes, the sign flip is exact)
                    const float sg = ((piece >> s) & 1) ? -1.0f : 1.0f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 o = make_float2(__shfl_xor_sync(0xFFFFFFFFu, y[i].x, 4 << s),
                                                     __shfl_xor_sync(0xFFFFFFFFu, y[i].y, 4 << s));
                        y[i] = __fadd2_rn(o, __fmul2_rn(y[i], make_float2(sg, sg)));
                    }
                }
                // The 16-point amax pass leaves out the 1/4 here and applies it
                // once to the maximum (kRht16Norm).
                if (!(AMAX_ONLY && LOGM == 0)) {
                    constexpr float c = rht_norm<LOGM>();
#pragma unroll
                    for (int i = 0; i < 16; ++i) y[i] = __fmul2_rn(y[i], make_float2(c, c));
                }
            }
            float bm0 = 0.0f, bm1 = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                bm0 = max3f(bm0, fabsf(y[i].x), fabsf(y[i + 1].x));
                bm1 = max3f(bm1, fabsf(y[i].y), fabsf(y[i + 1].y));
            }
            if (AMAX_ONLY) {
                if (ok) amax_bits = max(amax_bits, __float_as_uint(fmaxf(bm0, bm1)));
                continue;
            }
            // Features 2jp and 2jp+1: two blocks, scaled together in f32x2.
            const BlockScale bs0 = block_scale(bm0, ctx), bs1 = block_scale(bm1, ctx);
            float q[2][16];
            if (!isinf(bs0.r) && !isinf(bs1.r)) {
                const float2 r2 = make_float2(bs0.r, bs1.r);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 v2 = __fmul2_rn(y[i], r2);
                    q[0][i] = v2.x;
                    q[1][i] = v2.y;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    q[0][i] = isinf(bs0.r) ? scaled_inf(y[i].x) : scaled(y[i].x, bs0.r);
                    q[1][i] = isinf(bs1.r) ? scaled_inf(y[i].y) : scaled(y[i].y, bs1.r);
                }
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int j = 2 * jp + c;
                const uint32_t code = c ? bs1.code : bs0.code;
                if (SR) {
                    const uint64_t g = (uint64_t)((f0 + j) * T + t0) >> 3;
                    const uint4 r0 = sr_bits8(p.sr_keys, g);
                    const uint4 r1 = sr_bits8(p.sr_keys, g + 1);
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        sr_grid2(q[c][i], q[c][i + 1], sr_u16(r0, i), sr_u16(r0, i + 1));
                        sr_grid2(q[c][i + 8], q[c][i + 9], sr_u16(r1, i), sr_u16(r1, i + 1));
                    }
                }
                const uint32_t lo = e2m1x8(q[c][0], q[c][1], q[c][2], q[c][3], q[c][4], q[c][5], q[c][6], q[c][7]);
                const uint32_t hi =
                    e2m1x8(q[c][8], q[c][9], q[c][10], q[c][11], q[c][12], q[c][13], q[c][14], q[c][15]);
                const int srow = fl0 + j;
                if (kDirect) {
                    if (ok) *reinterpret_cast<uint2*>(p.codes + (f0 + j) * (T >> 1) + (t0 >> 1)) = make_uint2(lo, hi);
                } else {
                    const int key = LOGM == 0 ? (lane & 7) : ((srow >> 3) & 7);   // = (srow >> 3) & 7
                    *reinterpret_cast<uint2*>(s_codes + srow * 64 + ((piece ^ key) * 8)) = make_uint2(lo, hi);
                }
                s_sc[srow][piece] = ok ? (uint8_t)code : (uint8_t)0;
                if (ok && p.scales) p.scales[(f0 + j) * kb + (t0 >> 4)] = (uint8_t)code;
            }
        }
        if (AMAX_ONLY) continue;
        __syncthreads();
        const int64_t fbase = ft * 256, tbyte = tt * 64;
        if (p.scales_mma) {
            // GEMM scale layout: blocks 4g .. 4g+3 of a Q row are one word.
            for (int k = threadIdx.x; k < 256 * 2; k += kThreads) {
                const int fl = k >> 1, g = k & 1;
                const int64_t f = fbase + fl, blk = tt * 8 + g * 4;
                if (f < F && blk < kb)
                    *reinterpret_cast<uint32_t*>(p.scales_mma + mma_scale_offset(f, blk, p.chunks_k)) =
                        *reinterpret_cast<const uint32_t*>(&s_sc[fl][g * 4]);
            }
        }
        const int64_t row_bytes = min((int64_t)64, (T >> 1) - tbyte);
        for (int k = threadIdx.x; !kDirect && k < 256 * 8; k += kThreads) {
            const int r = k >> 3, c8 = k & 7;
            if (fbase + r < F && c8 * 8 < row_bytes) {
                const uint2 val = *reinterpret_cast<const uint2*>(s_codes + r * 64 + ((c8 ^ ((r >> 3) & 7)) * 8));
                *reinterpret_cast<uint2*>(p.codes + (fbase + r) * (T >> 1) + tbyte + c8 * 8) = val;
            }
        }
        __syncthreads();
    }
    if (AMAX_ONLY) {
        if (RHT && LOGM == 0) amax_bits = __float_as_uint(__uint_as_float(amax_bits) * kRht16Norm);
        write_partial(amax_bits, p.partials);
        if (p.partials2) {
            __syncthreads();   // write_partial's shared scratch is reused
            write_partial(absmax2_fold(plain_acc), p.partials2);
        }
    }
}

// ------------------------------------------------------------ 2D (16x16) ---
struct Params2d {
    const uint16_t* w;
    int64_t rows, cols, ld;
    uint8_t* codes_row;
    uint8_t* codes_col;
    uint8_t* scales;
    uint8_t* mma_row;
    uint8_t* mma_col;
    int64_t chunks_row, chunks_col;
    float* global_scale;
    uint32_t* partials;
    int n_partials;
};

// Transpose of an 8x8 matrix of nibbles held as 8 words (word i = row i,
// nibble j = column j): afterwards word j holds column j, row i in nibble i.
// Swaps of 4x4 blocks (16-bit halves), then 2x2 blocks (bytes), then single
// nibbles; the three levels commute.
__device__ __forceinline__ void transpose_nibbles8(uint32_t a[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t x = a[i], y = a[i + 4];
        a[i] = __byte_perm(x, y, 0x5410);
        a[i + 4] = __byte_perm(x, y, 0x7632);
    }
#pragma unroll
    for (int i = 0; i < 8; i += (i & 1) ? 3 : 1) {   // i = 0, 1, 4, 5
        const uint32_t x = a[i], y = a[i + 2];
        a[i] = __byte_perm(x, y, 0x6240);
        a[i + 2] = __byte_perm(x, y, 0x7351);
    }
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const uint32_t t = ((a[i] >> 4) ^ a[i + 1]) & 0x0F0F0F0Fu;
        a[i + 1] ^= t;
        a[i] ^= t << 4;
    }
}

// CTA tile: 128 rows x 256 columns; warp w: rows 16w..16w+15, lane: 8 columns,
// a lane pair: one 16x16 tile.  Each lane encodes its 16 x 8 elements once
// (row codes, one word per row); the columnwise codes (of W^T) are the same
// nibbles transposed in registers and staged in shared memory.  The tile's
// 128 block-scale codes are staged too, so both GEMM scale layouts are
// written as whole 32-bit words (4 consecutive blocks of one row).
template <bool COLS>
__global__ void __launch_bounds__(kThreads, 2) q2d_kernel(Params2d p) {
    __shared__ __align__(16) uint8_t s_col[COLS ? 256 * 64 : 16];
    __shared__ __align__(16) uint8_t s_sc[8][16];   // [row tile in CTA][column tile in CTA]
    __shared__ float s_rtab[128];
    ScaleCtx ctx;
    {
        const float A = reduce_partials(p.partials, p.n_partials);
        const float sg = __fdiv_rn(A, kGlobalDiv);
        if (blockIdx.x == 0 && threadIdx.x == 0) *p.global_scale = sg;
        ctx = make_scale_ctx(sg, __fmul_rn(6.0f, sg), s_rtab);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t R = p.rows, C = p.cols;
    const int64_t ntr = (R + 127) >> 7, ntc = (C + 255) >> 8;
    const int64_t ntiles = ntr * ntc;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t tr = tile / ntc, tc = tile - tr * ntc;
        const int64_t r0 = tr * 128 + warp * 16;
        const int64_t c0 = tc * 256 + lane * 8;
        const bool ok = (r0 < R) && (c0 < C);
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = ok ? ldg_stream(p.w + (r0 + i) * p.ld + c0) : make_uint4(0u, 0u, 0u, 0u);
        // While this tile is encoded and its outputs staged (two block-wide
        // barriers, during which no load of this CTA is in flight), pull the
        // CTA's next tile into L2: thread r < 128 takes row r (512 bytes).
        {
            const int64_t nt = tile + gridDim.x;
            if (nt < ntiles && threadIdx.x < 128) {
                const int64_t ntr_ = nt / ntc, ntc_ = nt - ntr_ * ntc;
                const int64_t pr = ntr_ * 128 + threadIdx.x, pc = ntc_ * 256;
                if (pr < R) prefetch_l2(p.w + pr * p.ld + pc, (uint32_t)(min((int64_t)256, C - pc) * 2));
            }
        }
        uint32_t acc = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) acc = absmax2(absmax2(absmax2(absmax2(acc, v[i].x), v[i].y), v[i].z), v[i].w);
        float b = __uint_as_float(absmax2_fold(acc));
        b = fmaxf(b, __shfl_xor_sync(0xFFFFFFFFu, b, 1));
        const BlockScale bs = block_scale(b, ctx);
        uint32_t rc[16];
        if (!isinf(bs.r)) {
            const float2 r2 = make_float2(bs.r, bs.r);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float2 q0 = __fmul2_rn(make_float2(bf16_lo(v[i].x), bf16_hi(v[i].x)), r2);
                const float2 q1 = __fmul2_rn(make_float2(bf16_lo(v[i].y), bf16_hi(v[i].y)), r2);
                const float2 q2 = __fmul2_rn(make_float2(bf16_lo(v[i].z), bf16_hi(v[i].z)), r2);
                const float2 q3 = __fmul2_rn(make_float2(bf16_lo(v[i].w), bf16_hi(v[i].w)), r2);
                rc[i] = e2m1x8(q0.x, q0.y, q1.x, q1.y, q2.x, q2.y, q3.x, q3.y);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                rc[i] = e2m1x8(scaled_inf(bf16_lo(v[i].x)), scaled_inf(bf16_hi(v[i].x)), scaled_inf(bf16_lo(v[i].y)),
                               scaled_inf(bf16_hi(v[i].y)), scaled_inf(bf16_lo(v[i].z)), scaled_inf(bf16_hi(v[i].z)),
                               scaled_inf(bf16_lo(v[i].w)), scaled_inf(bf16_hi(v[i].w)));
        }
        if (ok) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                *reinterpret_cast<uint32_t*>(p.codes_row + (r0 + i) * (C >> 1) + (c0 >> 1)) = rc[i];
            if ((lane & 1) == 0 && p.scales) p.scales[(r0 >> 4) * (C >> 4) + (c0 >> 4)] = (uint8_t)bs.code;
        }
        if ((lane & 1) == 0) s_sc[warp][lane >> 1] = ok ? (uint8_t)bs.code : (uint8_t)0;
        if (COLS) {
            transpose_nibbles8(rc);
            transpose_nibbles8(rc + 8);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint2*>(s_col + (lane * 8 + j) * 64 + ((warp ^ (lane & 7)) * 8)) =
                    make_uint2(rc[j], rc[8 + j]);
        }
        __syncthreads();
        // GEMM scale layouts: word = scales of blocks 4g .. 4g+3 of one row.
        if (p.mma_row) {
            for (int k = threadIdx.x; k < 128 * 4; k += kThreads) {
                const int rr = k >> 2, g = k & 3;
                const int64_t r = tr * 128 + rr, blk = tc * 16 + g * 4;
                if (r < R && blk < (C >> 4))
                    *reinterpret_cast<uint32_t*>(p.mma_row + mma_scale_offset(r, blk, p.chunks_row)) =
                        *reinterpret_cast<const uint32_t*>(&s_sc[rr >> 4][g * 4]);
            }
        }
        if (p.mma_col) {
            for (int k = threadIdx.x; k < 256 * 2; k += kThreads) {
                const int cc = k >> 1, g = k & 1;
                const int64_t c = tc * 256 + cc, blk = tr * 8 + g * 4;
                if (c < C && blk < (R >> 4)) {
                    const int cb = cc >> 4;
                    const uint32_t word = (uint32_t)s_sc[g * 4][cb] | ((uint32_t)s_sc[g * 4 + 1][cb] << 8) |
                                          ((uint32_t)s_sc[g * 4 + 2][cb] << 16) | ((uint32_t)s_sc[g * 4 + 3][cb] << 24);
                    *reinterpret_cast<uint32_t*>(p.mma_col + mma_scale_offset(c, blk, p.chunks_col)) = word;
                }
            }
        }
        if (COLS) {
            const int64_t cbase = tc * 256, rbyte = tr * 64;
            const int64_t row_bytes = min((int64_t)64, (R >> 1) - rbyte);
            for (int k = threadIdx.x; k < 256 * 8; k += kThreads) {
                const int r = k >> 3, c8 = k & 7;
                if (cbase + r < C && c8 * 8 < row_bytes) {
                    const uint2 val = *reinterpret_cast<const uint2*>(s_col + r * 64 + ((c8 ^ ((r >> 3) & 7)) * 8));
                    *reinterpret_cast<uint2*>(p.codes_col + (cbase + r) * (R >> 1) + rbyte + c8 * 8) = val;
                }
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------- dequantize ---
// One thread per 16-block: out = RN(RN(value * s_dec) * s_global).
__global__ void __launch_bounds__(kThreads) dequant_kernel(const uint8_t* __restrict__ codes,
                                                          const uint8_t* __restrict__ scales, int mode2d,
                                                          const float* __restrict__ gs, int64_t rows,
                                                          int64_t cols, int out_bf16, void* __restrict__ out) {
    const float sg = __ldg(gs);
    const int64_t kb = cols >> 4;
    const int64_t total = rows * kb;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * blockDim.x) {
        const uint2 cw = __ldg(reinterpret_cast<const uint2*>(codes) + u);
        int64_t si = u;
        if (mode2d) {
            const int64_t r = u / kb;
            si = (r >> 4) * kb + (u - r * kb);
        }
        const float s = e4m3_decode(__ldg(scales + si));
        float o[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t h[4];
            e2m1x8_decode(half ? cw.y : cw.x, h);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 val = __half22float2(*reinterpret_cast<const __half2*>(&h[k]));
                o[8 * half + 2 * k] = __fmul_rn(__fmul_rn(val.x, s), sg);
                o[8 * half + 2 * k + 1] = __fmul_rn(__fmul_rn(val.y, s), sg);
            }
        }
        if (out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + u * 16);
            uint32_t wv[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * k], o[2 * k + 1]);
                wv[k] = *reinterpret_cast<const uint32_t*>(&h);
            }
            dst[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            dst[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
        } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + u * 16);
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = make_float4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
        }
    }
}

// ------------------------------------------------------------ scale layout ---
__global__ void __launch_bounds__(kThreads) scales_to_mma_kernel(const uint8_t* __restrict__ scales, int mode2d,
                                                                int64_t rows, int64_t kb, int64_t chunks_k,
                                                                int64_t total, uint8_t* __restrict__ dst) {
    for (int64_t d = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; d < total;
         d += (int64_t)gridDim.x * blockDim.x) {
        const int64_t chunk = d >> 9, within = d & 511;
        const int64_t rc = chunk / chunks_k, kc = chunk - rc * chunks_k;
        const int64_t r = rc * 128 + ((within >> 2) & 3) * 32 + (within >> 4);
        const int64_t b = kc * 4 + (within & 3);
        uint8_t val = 0;
        if (r < rows && b < kb) val = mode2d ? scales[(r >> 4) * kb + b] : scales[r * kb + b];
        dst[d] = val;
    }
}

template <typename K>
int grid_for(K kernel, int64_t work_items) {
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0);
    if (per_sm < 1) per_sm = 1;
    int64_t g = (int64_t)sm_count() * per_sm;
    if (g > work_items) g = work_items;
    if (g < 1) g = 1;
    if (g > kMaxPartials) g = kMaxPartials;
    return (int)g;
}

// CTA count of the plain amax pass: up to kAmaxPerSm CTAs per SM, each with
// kUnroll 16-byte loads per thread in flight.
constexpr int kAmaxPerSm = 4;
int plain_amax_grid(int64_t rows, int64_t cols) {
    const int64_t vecs = rows * (cols >> 3);
    const int64_t want = (vecs + (int64_t)kThreads * kUnroll - 1) / ((int64_t)kThreads * kUnroll);
    int64_t g = std::min<int64_t>((int64_t)sm_count() * kAmaxPerSm, want);
    g = std::max<int64_t>(g, 1);
    return (int)std::min<int64_t>(g, kMaxPartials);
}

// Launches the plain amax pass; returns the number of partials it writes.
int launch_amax_plain(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t* partials,
                      cudaStream_t s) {
    const int g = plain_amax_grid(rows, cols);
    if (ld == cols) amax_plain_kernel<true><<<g, kThreads, 0, s>>>(x, rows, cols, ld, partials);
    else amax_plain_kernel<false><<<g, kThreads, 0, s>>>(x, rows, cols, ld, partials);
    return g;
}

// Grid of the SR row-wise encode pass: every resident CTA of the device,
// no more than there are warp segments to hand out.
template <bool RHT>
int rows_sr_grid(const Params& p) {
    const int64_t segs = p.rows * ((((p.cols + 63) >> 6) + 31) >> 5);
    return grid_for(rows_sr_kernel<RHT>, (segs + 7) / 8);
}

template <bool RHT, bool SR, int LOGM = 0>
cudaError_t run_rows(Params p, const float* given, cudaStream_t s, int* launches) {
    const int64_t units = p.rows * ((p.cols + 511) >> 9);
    const int64_t warps_needed = (units + 1) / 2;
    const int g = grid_for(rows_kernel<RHT, SR, false, LOGM>, (warps_needed + 7) / 8);
    if (given) {   // the tensor amax is known: it is the single partial
        p.partials = const_cast<uint32_t*>(reinterpret_cast<const uint32_t*>(given));
        p.n_partials = 1;
        *launches -= 1;
    } else if (RHT) {
        p.n_partials = g;
        rows_kernel<true, false, true, LOGM><<<g, kThreads, 0, s>>>(p);
    } else {
        p.n_partials = launch_amax_plain(p.x, p.rows, p.cols, p.ld, p.partials, s);
    }
    if (SR && LOGM == 0) rows_sr_kernel<RHT><<<rows_sr_grid<RHT>(p), kThreads, 0, s>>>(p);
    else rows_kernel<RHT, SR, false, LOGM><<<g, kThreads, 0, s>>>(p);
    *launches += 2;
    return cudaGetLastError();
}

template <bool RHT, bool SR, int LOGM = 0>
cudaError_t run_cols(Params p, const float* given, cudaStream_t s, int* launches) {
    const int64_t tiles = ((p.rows + 127) >> 7) * ((p.cols + 255) >> 8);
    const int g = grid_for(cols_kernel<RHT, SR, false, LOGM>, tiles);
    if (given) {
        p.partials = const_cast<uint32_t*>(reinterpret_cast<const uint32_t*>(given));
        p.n_partials = 1;
        *launches -= 1;
    } else if (RHT) {
        p.n_partials = g;
        cols_kernel<true, false, true, LOGM><<<g, kThreads, 0, s>>>(p);
    } else {
        p.n_partials = launch_amax_plain(p.x, p.rows, p.cols, p.ld, p.partials, s);
    }
    cols_kernel<RHT, SR, false, LOGM><<<g, kThreads, 0, s>>>(p);
    *launches += 2;
    return cudaGetLastError();
}

// RHT quantizers by order: log2(order / 16) as a template argument.
template <int LOGM>
cudaError_t run_rht(const QuantArgs& a, const Params& p, cudaStream_t s, int* launches) {
    const bool sr = a.rounding == 1;
    const float* g = a.given_amax;
    if (!a.transpose)
        return sr ? run_rows<true, true, LOGM>(p, g, s, launches) : run_rows<true, false, LOGM>(p, g, s, launches);
    return sr ? run_cols<true, true, LOGM>(p, g, s, launches) : run_cols<true, false, LOGM>(p, g, s, launches);
}

}  // namespace

cudaError_t launch_quantize_1d(const QuantArgs& a, cudaStream_t s, int* launches) {
    Params p{};
    p.x = a.x;
    p.rows = a.rows;
    p.cols = a.cols;
    p.ld = a.ld;
    p.rht_seed = a.rht_seed;
    p.sr_seed = a.sr_seed;
    p.sr_keys = philox_round_keys(a.sr_seed);
    p.rht_sign = rht_sign_words_host(a.rht_seed);
    p.codes = a.codes;
    p.scales = a.scales;
    p.scales_mma = a.scales_mma;
    p.global_scale = a.global_scale;
    p.partials = a.partials;
    const int64_t qr = a.transpose ? a.cols : a.rows;
    const int64_t qc = a.transpose ? a.rows : a.cols;
    p.chunks_k = mma_chunks_k(qc);
    if (a.scales_mma && ((qr % 128) || ((qc / 16) % 4))) {
        cudaError_t e = cudaMemsetAsync(a.scales_mma, 0, mma_scale_bytes(qr, qc), s);
        if (e != cudaSuccess) return e;
    }
    const bool sr = a.rounding == 1;
    const float* g = a.given_amax;
    if (a.rht) {
        switch (a.rht_order) {
            case 32: return run_rht<1>(a, p, s, launches);
            case 64: return run_rht<2>(a, p, s, launches);
            case 128: return run_rht<3>(a, p, s, launches);
            default: return run_rht<0>(a, p, s, launches);
        }
    }
    if (!a.transpose)
        return sr ? run_rows<false, true>(p, g, s, launches) : run_rows<false, false>(p, g, s, launches);
    return sr ? run_cols<false, true>(p, g, s, launches) : run_cols<false, false>(p, g, s, launches);
}

// Both GEMM roles of one tensor from one amax read: Q = x (1D along the
// rows, args r) and Q = RHT(x^T) (args t).  The transposed amax pass also
// reduces the plain |x| maxima (second half of the workspace), which the
// row-wise encode pass then folds; the transposed encode pass folds the
// rotated ones.  Three launches instead of four, one full read saved.
cudaError_t launch_quantize_dual(const QuantArgs& r, const QuantArgs& t, cudaStream_t s, int* launches) {
    Params pt{};
    pt.x = t.x;
    pt.rows = t.rows;
    pt.cols = t.cols;
    pt.ld = t.ld;
    pt.rht_seed = t.rht_seed;
    pt.sr_seed = t.sr_seed;
    pt.sr_keys = philox_round_keys(t.sr_seed);
    pt.rht_sign = rht_sign_words_host(t.rht_seed);
    pt.codes = t.codes;
    pt.scales = t.scales;
    pt.scales_mma = t.scales_mma;
    pt.chunks_k = mma_chunks_k(t.rows);
    pt.global_scale = t.global_scale;
    pt.partials = t.partials;
    pt.partials2 = r.partials;
    Params pr{};
    pr.x = r.x;
    pr.rows = r.rows;
    pr.cols = r.cols;
    pr.ld = r.ld;
    pr.sr_seed = r.sr_seed;
    pr.sr_keys = philox_round_keys(r.sr_seed);
    pr.codes = r.codes;
    pr.scales = r.scales;
    pr.scales_mma = r.scales_mma;
    pr.chunks_k = mma_chunks_k(r.cols);
    pr.global_scale = r.global_scale;
    pr.partials = r.partials;
    if (r.scales_mma && ((r.rows % 128) || ((r.cols / 16) % 4))) {
        cudaError_t e = cudaMemsetAsync(r.scales_mma, 0, mma_scale_bytes(r.rows, r.cols), s);
        if (e != cudaSuccess) return e;
    }
    if (t.scales_mma && ((t.cols % 128) || ((t.rows / 16) % 4))) {
        cudaError_t e = cudaMemsetAsync(t.scales_mma, 0, mma_scale_bytes(t.cols, t.rows), s);
        if (e != cudaSuccess) return e;
    }
    const bool sr_r = r.rounding == 1, sr_t = t.rounding == 1;
    const int64_t tiles = ((t.rows + 127) >> 7) * ((t.cols + 255) >> 8);
    const int gc = sr_t ? grid_for(cols_kernel<true, true, false>, tiles) : grid_for(cols_kernel<true, false, false>, tiles);
    cols_kernel<true, false, true><<<gc, kThreads, 0, s>>>(pt);
    pt.n_partials = gc;
    pr.n_partials = gc;
    pt.partials2 = nullptr;
    const int64_t units = r.rows * ((r.cols + 511) >> 9);
    const int64_t wneed = (units + 1) / 2;
    if (sr_r) rows_sr_kernel<false><<<rows_sr_grid<false>(pr), kThreads, 0, s>>>(pr);
    else rows_kernel<false, false, false><<<grid_for(rows_kernel<false, false, false>, (wneed + 7) / 8), kThreads, 0, s>>>(pr);
    if (sr_t) cols_kernel<true, true, false><<<gc, kThreads, 0, s>>>(pt);
    else cols_kernel<true, false, false><<<gc, kThreads, 0, s>>>(pt);
    *launches += 3;
    return cudaGetLastError();
}

cudaError_t launch_quantize_2d(const Quant2dArgs& a, cudaStream_t s, int* launches) {
    Params2d p{};
    p.w = a.w;
    p.rows = a.rows;
    p.cols = a.cols;
    p.ld = a.ld;
    p.codes_row = a.codes_row;
    p.codes_col = a.codes_col;
    p.scales = a.scales;
    p.mma_row = a.scales_mma_row;
    p.mma_col = a.scales_mma_col;
    p.chunks_row = mma_chunks_k(a.cols);
    p.chunks_col = mma_chunks_k(a.rows);
    p.global_scale = a.global_scale;
    p.partials = a.partials;
    if (a.scales_mma_row && ((a.rows % 128) || ((a.cols / 16) % 4))) {
        cudaError_t e = cudaMemsetAsync(a.scales_mma_row, 0, mma_scale_bytes(a.rows, a.cols), s);
        if (e != cudaSuccess) return e;
    }
    if (a.scales_mma_col && ((a.cols % 128) || ((a.rows / 16) % 4))) {
        cudaError_t e = cudaMemsetAsync(a.scales_mma_col, 0, mma_scale_bytes(a.cols, a.rows), s);
        if (e != cudaSuccess) return e;
    }
    const int64_t tiles = ((a.rows + 127) >> 7) * ((a.cols + 255) >> 8);
    const int g = a.codes_col ? grid_for(q2d_kernel<true>, tiles) : grid_for(q2d_kernel<false>, tiles);
    if (a.given_amax) {   // the tensor amax is known: it is the single partial
        p.partials = const_cast<uint32_t*>(reinterpret_cast<const uint32_t*>(a.given_amax));
        p.n_partials = 1;
        *launches -= 1;
    } else {
        p.n_partials = launch_amax_plain(a.w, a.rows, a.cols, a.ld, a.partials, s);
    }
    if (a.codes_col) q2d_kernel<true><<<g, kThreads, 0, s>>>(p);
    else q2d_kernel<false><<<g, kThreads, 0, s>>>(p);
    *launches += 2;
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, int scale_mode, const float* gs,
                              int64_t rows, int64_t cols, int out_bf16, void* out, cudaStream_t s) {
    const int64_t total = rows * (cols >> 4);
    const int g = grid_for(dequant_kernel, (total + kThreads - 1) / kThreads);
    dequant_kernel<<<g, kThreads, 0, s>>>(codes, scales, scale_mode, gs, rows, cols, out_bf16, out);
    return cudaGetLastError();
}

cudaError_t launch_scales_to_mma(const uint8_t* scales, int scale_mode, int64_t rows, int64_t k,
                                 uint8_t* scales_mma, cudaStream_t s) {
    const int64_t total = (int64_t)mma_scale_bytes(rows, k);
    const int g = grid_for(scales_to_mma_kernel, (total + kThreads - 1) / kThreads);
    scales_to_mma_kernel<<<g, kThreads, 0, s>>>(scales, scale_mode, rows, k >> 4, mma_chunks_k(k), total,
                                                scales_mma);
    return cudaGetLastError();
}


// ------------------------------------------------------ no-allocation path ---
// Scratch for callers that cannot allocate device memory (see
// nvfp4_quantize_1d_noalloc in nvfp4.h).  The amax pass writes one partial
// maximum per CTA here and the encode pass reads them back.  The array lives
// in the library's device image: every GPU that loads the library holds it
// until the process exits, and all calls on a device share it.
constexpr int kNoAllocPartials = 1024;   // 4 KiB
static __device__ __align__(256) uint32_t g_noalloc_partials[kNoAllocPartials];

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Identity of the CUDA context current on this thread (0 when none is, or
// when the driver cannot tell).  A context that is destroyed and created
// again (cudaDeviceReset, a primary context released and retained) gets a
// new identity, and the library's device image -- the scratch array with it
// -- may then sit at another address.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

std::mutex g_noalloc_mutex;
struct ScratchSlot {
    unsigned long long ctx_id;
    void* ptr;
};
ScratchSlot g_noalloc_slot[64] = {};

// Device address of the static scratch in the current context (host code
// only sees a stand-in symbol, never a device address).  Looked up with the
// device current the first time a context uses it, and again whenever the
// current context is not the one the cached address belongs to.
cudaError_t noalloc_scratch(uint32_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    ScratchSlot& slot = g_noalloc_slot[dev];
    const unsigned long long id = current_context_id();
    if (!slot.ptr || id == 0 || id != slot.ctx_id) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_partials);   // also makes the device's context current
        if (e != cudaSuccess) return e;
        slot.ptr = ptr;
        slot.ctx_id = current_context_id();
    }
    *out = static_cast<uint32_t*>(slot.ptr);
    return cudaSuccess;
}
}  // namespace

int noalloc_capacity() { return kNoAllocPartials; }

// Same launches as launch_quantize_1d, with the partial maxima in the static
// scratch.  The amax pass writes one partial per CTA (plain_amax_grid); a
// configuration that would need more partials than the scratch holds is
// refused (*too_big = true) before anything is enqueued.
cudaError_t launch_quantize_1d_noalloc(const QuantArgs& a, cudaStream_t s, int* launches, bool* too_big) {
    *too_big = false;
    const int g = plain_amax_grid(a.rows, a.cols);
    if (g > kNoAllocPartials) {
        *too_big = true;
        return cudaSuccess;
    }
    uint32_t* scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return e;
    QuantArgs b = a;
    b.rht = 0;
    b.given_amax = nullptr;
    b.partials = scratch;
    return launch_quantize_1d(b, s, launches);
}

}  // namespace nvfp4
