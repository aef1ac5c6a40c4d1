// common.cuh -- device helpers shared by the NVFP4 kernels (sm_100a only).
//
// Format (sources: "NVFP4 Is a Scaling System, Not Just a 4-Bit Number",
// "The smallest example"; "MXFP4 和 NVFP4 的区别", "数据格式:极简的 E2M1" and
// "精度核心:两级分层缩放"; "Melatih model dalam 4 bit", "Anatomi NVFP4"):
// x = e2m1 * e4m3_block_scale * fp32_global_scale, global = amax / (448 * 6).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library is built for sm_100a only"
#endif

namespace nvfp4 {

constexpr float kGlobalDiv = 2688.0f;   // 448 (E4M3 max) * 6 (E2M1 max)

// ---------------------------------------------------------------- loads ----
// Streaming 16-byte load that does not allocate in L1 (each byte is read once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Bring `bytes` (a multiple of 16) from a 16-byte-aligned global address
// into L2 without waiting for it (bulk prefetch; nothing tracks completion).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// bf16 halves of a packed word -> binary32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Largest |bf16| of a packed pair, accumulated lane-wise: max.xorsign.abs
// keeps max(|acc|, |w|) in each half (its sign bit, the xor of the operands'
// signs, is dropped by absmax2_fold).  Exact, subnormals included.
__device__ __forceinline__ uint32_t absmax2(uint32_t acc, uint32_t w) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(acc), "r"(w));
    return d;
}
__device__ __forceinline__ uint32_t absmax2_fold(uint32_t acc) {   // -> binary32 bits of the max
    const uint32_t lo = acc & 0x7FFFu, hi = (acc >> 16) & 0x7FFFu;
    return (lo > hi ? lo : hi) << 16;
}

// ------------------------------------------------------- format conversion --
// E4M3 (FN) encode of s >= 0: round to nearest even, saturating to 448.
__device__ __forceinline__ uint32_t e4m3_encode(float s) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(s));
    return out & 0xFFu;
}
// E4M3 -> binary32 (exact, through f16).
__device__ __forceinline__ float e4m3_decode(uint32_t code) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)code));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// E2M1 encode (nearest even, saturating to +-6, sign kept) of 8 values into
// 8 nibbles, value 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5,
                                           float v6, float v7) {
    uint32_t out;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(out)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return out;
}

// Eight E2M1 codes (a 32-bit word, code 2j in the low nibble of byte j) ->
// four f16x2 words (exact); half 0 of word k is element 2k.
__device__ __forceinline__ void e2m1x8_decode(uint32_t word, uint32_t h[4]) {
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "mov.b32 {q0, q1, q2, q3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, q1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, q2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, q3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(word));
}

// -------------------------------------------------------------- Philox ----
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): multipliers 0xD2511F53
// (word 0) and 0xCD9E8D57 (word 2), Weyl key increments 0x9E3779B9 and
// 0xBB67AE85 between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    }
    return c;
}

// The ten round keys of Philox4x32-10 for one key (k0, k1): (k0 + r *
// 0x9E3779B9, k1 + r * 0xBB67AE85), r = 0..9.  Computed once on the host and
// passed as kernel parameters, so every round reads its key from the
// parameter bank instead of recomputing it.
struct PhiloxKeys {
    uint32_t k[20];
};
inline PhiloxKeys philox_round_keys(uint64_t key) {
    PhiloxKeys r;
    uint32_t k0 = (uint32_t)key, k1 = (uint32_t)(key >> 32);
    for (int i = 0; i < 10; ++i) {
        r.k[2 * i] = k0;
        r.k[2 * i + 1] = k1;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return r;
}
// The same generator on the host: word 0 of Philox4x32-10 at counter
// (0, 0, 1, 0) under key `key` -- the RHT sign word (bit j set <=> d_j = -1).
inline uint32_t rht_sign_word_host(uint64_t key) {
    const PhiloxKeys k = philox_round_keys(key);
    uint32_t c0 = 0u, c1 = 0u, c2 = 1u, c3 = 0u;
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k.k[2 * r];
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k.k[2 * r + 1];
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = n0;
        c2 = n2;
    }
    return c0;
}

// Sign of each of the 16 positions of a chunk as a word to fold into the
// bf16 -> binary32 unpack: 0x80000000 where d_j = -1, else 0.
struct SignWords {
    uint32_t m[16];
};
inline SignWords rht_sign_words_host(uint64_t rht_seed) {
    const uint32_t d = rht_sign_word_host(rht_seed) & 0xFFFFu;
    SignWords s;
    for (int j = 0; j < 16; ++j) s.m[j] = ((d >> j) & 1u) ? 0x80000000u : 0u;
    return s;
}
// bf16 halves of a packed word -> binary32 with a sign word applied: the low
// half as w * 2^16 + m (adding 2^31 flips the sign bit, nothing else), the
// high half as (w & 0xFFFF0000) ^ m -- one instruction each.
__device__ __forceinline__ float bf16_lo_signed(uint32_t w, uint32_t m) {
    uint32_t d;
    asm("mad.lo.u32 %0, %1, 65536, %2;" : "=r"(d) : "r"(w), "r"(m));
    return __uint_as_float(d);
}
__device__ __forceinline__ float bf16_hi_signed(uint32_t w, uint32_t m) {
    return __uint_as_float((w & 0xFFFF0000u) ^ m);
}

__device__ __forceinline__ uint4 philox4x32_10_keys(uint4 c, const PhiloxKeys& keys) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        // one 32 x 32 -> 64-bit multiply per word gives both halves
        const uint64_t p0 = (uint64_t)0xD2511F53u * c.x;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c.z;
        c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ keys.k[2 * r], (uint32_t)p1,
                       (uint32_t)(p0 >> 32) ^ c.w ^ keys.k[2 * r + 1], (uint32_t)p0);
    }
    return c;
}

// 16 random bits for the 8 output elements 8g .. 8g+7 (element e: word e/2,
// low half for even e), Philox keyed by the seed whose round keys are given.
__device__ __forceinline__ uint4 sr_bits8(const PhiloxKeys& keys, uint64_t g) {
    return philox4x32_10_keys(make_uint4((uint32_t)g, (uint32_t)(g >> 32), 0u, 0u), keys);
}
// The 16 random bits u of element e: word e/2, low half for even e.
__device__ __forceinline__ uint32_t sr_u16(const uint4& w, int e) {
    const uint32_t word = (e >> 1) == 0 ? w.x : (e >> 1) == 1 ? w.y : (e >> 1) == 2 ? w.z : w.w;
    return (e & 1) ? (word >> 16) : (word & 0xFFFFu);
}

// RHT sign mask ("随机 Hadamard 变换": a random diagonal of signs): bit j set
// <=> d_j = -1; word 0 of Philox4x32-10 at counter (0, 0, 1, 0), key rht_seed.
__device__ __forceinline__ uint32_t rht_sign_mask(uint64_t rht_seed) {
    return philox4x32_10(make_uint4(0u, 0u, 1u, 0u), (uint32_t)rht_seed, (uint32_t)(rht_seed >> 32)).x & 0xFFFFu;
}

// Signs of an n-point RHT, n <= 128 ("构造 Hadamard 矩阵的方法": the Sylvester
// recursion continues to any power of two): d_j = -1 <=> bit j % 32 of word
// j / 32 of the same Philox output, so the 16-point signs are its first 16.
// Returns the 16-bit mask of positions base .. base+15 (base a multiple of 16).
__device__ __forceinline__ uint32_t rht_sign_mask_at(uint64_t rht_seed, int base) {
    const uint4 w = philox4x32_10(make_uint4(0u, 0u, 1u, 0u), (uint32_t)rht_seed, (uint32_t)(rht_seed >> 32));
    const int k = base >> 5;
    const uint32_t word = k == 0 ? w.x : k == 1 ? w.y : k == 2 ? w.z : w.w;
    return (word >> (base & 31)) & 0xFFFFu;
}

// Normalisation of the (16 << LOGM)-point transform: RN(1/sqrt(n)) in binary32
// (1/4, RN(sqrt 2)/8, 1/8, RN(sqrt 2)/16), applied once after the butterflies.
template <int LOGM>
__device__ __forceinline__ constexpr float rht_norm() {
    return LOGM == 0 ? 0.25f : LOGM == 1 ? 0x1.6a09e6p-3f : LOGM == 2 ? 0.125f : 0x1.6a09e6p-4f;
}
// The 16-point factor 1/4 commutes exactly with the maximum: every butterfly
// value is a sum of +-bf16 values, so a multiple of 2^-133 (bf16's smallest
// subnormal), and a quarter of it is representable in binary32 (2^-135 is a
// multiple of binary32's subnormal step 2^-149).  So max |y / 4| = (max |y|) / 4
// bit for bit, and an amax pass may scale its maximum once instead of every
// element.
constexpr float kRht16Norm = 0.25f;

// Stochastic rounding onto the E2M1 grid of one scaled value v (finite):
// between neighbours lo <= |v| < hi, f = floor(p * 2^16) with
// p = (|v| - lo) / (hi - lo), round up iff f + u >= 2^16; results above 6
// are left for the saturating E2M1 conversion.
// E2M1 is a float with one mantissa bit and subnormals, and binary32 scaled by
// 2^-126 lines up with it: |v| in [1, 8) becomes a normal number whose
// mantissa bit 22 is the E2M1 mantissa bit, |v| < 1 a subnormal whose bit 22
// is the E2M1 subnormal bit (0.5), so in both the 22 bits below bit 22 hold
// p * 2^22, cut towards zero to an integer.  Adding u * 2^6 carries into bit
// 22 iff floor(p * 2^22) + u * 2^6 >= 2^22, i.e. iff f + u >= 2^16 (the
// floors nest); the carry walks into the exponent where the step doubles
// (subnormal 0.5 -> 1, 1.5 -> 2, 3 -> 4).  Rounding towards zero keeps the
// sign out of it, and the scaling back is exact.
__device__ __forceinline__ float sr_grid(float v, uint32_t u) {
    const uint32_t t = __float_as_uint(__fmul_rz(v, 0x1p-126f)) + (u << 6);
    return __fmul_rn(__uint_as_float(t & 0xFFC00000u), 0x1p126f);
}
// sr_grid of two values with the two scalings done as f32x2 multiplies.
__device__ __forceinline__ void sr_grid2(float& v0, float& v1, uint32_t u0, uint32_t u1) {
    float s0, s1;
    asm("{\n\t.reg .b64 a, b, d;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 b, {%4, %4};\n\t"
        "mul.rz.f32x2 d, a, b;\n\t"
        "mov.b64 {%0, %1}, d;\n\t}"
        : "=f"(s0), "=f"(s1)
        : "f"(v0), "f"(v1), "f"(0x1p-126f));
    const float r0 = __uint_as_float((__float_as_uint(s0) + (u0 << 6)) & 0xFFC00000u);
    const float r1 = __uint_as_float((__float_as_uint(s1) + (u1 << 6)) & 0xFFC00000u);
    const float2 q = __fmul2_rn(make_float2(r0, r1), make_float2(0x1p126f, 0x1p126f));
    v0 = q.x;
    v1 = q.y;
}

// Per-block scale derived from the block amax ("精度核心:两级分层缩放";
// "Anatomi NVFP4"): s = e4m3(RN(bmax / t)), t = RN(6 s_global) (s = 0 when
// t == 0); multiplier r = RN(1 / RN(s * s_global)).  r == 0 marks a zero
// scale (every element encodes a signed zero); r == +inf marks a product that
// underflowed or a reciprocal that overflowed (nonzero elements saturate).
//
// Per tensor, everything after the quotient depends on the 8-bit code alone,
// so each CTA tabulates r for the 128 non-negative codes once (ScaleCtx) and
// a block costs one quotient, one E4M3 conversion and one shared-memory load.
// The quotient bmax / t: with y = RN(1/t), q0 = RN(bmax * y) and the exact
// residual e = bmax - q0 * t (one FMA), RN(q0 + e * y) (one FMA) is the
// correctly rounded quotient (Markstein's FMA division theorem) as long as
// nothing underflows: used for t >= 2^-60, where every quotient that can
// reach a nonzero E4M3 code (>= 2^-11) keeps e normal; IEEE division
// otherwise.
struct BlockScale {
    uint32_t code;
    float r;
};
struct ScaleCtx {
    float t, inv_t;
    bool fast;
    const float* rtab;   // shared memory, 128 entries
};
__device__ __forceinline__ ScaleCtx make_scale_ctx(float sg, float t, float* s_rtab) {
    for (int c = threadIdx.x; c < 128; c += blockDim.x) {
        const float sdec = e4m3_decode((uint32_t)c);
        s_rtab[c] = (sdec == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(sdec, sg));
    }
    __syncthreads();
    ScaleCtx c;
    c.t = t;
    c.fast = t >= 0x1p-60f;
    c.inv_t = c.fast ? __frcp_rn(t) : 0.0f;
    c.rtab = s_rtab;
    return c;
}
__device__ __forceinline__ BlockScale block_scale(float bmax, const ScaleCtx& c) {
    float sf;
    if (c.fast) {
        const float q0 = __fmul_rn(bmax, c.inv_t);
        sf = __fmaf_rn(__fmaf_rn(-q0, c.t, bmax), c.inv_t, q0);
    } else {
        sf = (c.t == 0.0f) ? 0.0f : __fdiv_rn(bmax, c.t);
    }
    BlockScale b;
    b.code = e4m3_encode(sf);
    b.r = c.rtab[b.code & 127u];
    return b;
}

// Scaled value of one element: RN(x * r); the r == +inf case maps nonzero x to
// +-6 (saturation) and zero x to a signed zero, as the unrounded products do.
__device__ __forceinline__ float scaled(float x, float r) {
    return __fmul_rn(x, r);
}
__device__ __forceinline__ float scaled_inf(float x) {
    return x == 0.0f ? x : copysignf(6.0f, x);
}

// Offset of scale (row r, block b) in the MMA scale layout (see nvfp4.h).
__host__ __device__ __forceinline__ int64_t mma_scale_offset(int64_t r, int64_t b, int64_t chunks_k) {
    return ((r >> 7) * chunks_k + (b >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Reduce the per-CTA amax partials (binary32 bits of non-negative maxima) to
// the tensor amax; every thread of the block gets it.
__device__ __forceinline__ float reduce_partials(const uint32_t* __restrict__ partials, int n) {
    __shared__ uint32_t s_red[32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) m = max(m, __ldg(partials + i));
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        uint32_t v = lane < (int)(blockDim.x >> 5) ? s_red[lane] : 0u;
        v = __reduce_max_sync(0xFFFFFFFFu, v);
        if (lane == 0) s_red[0] = v;
    }
    __syncthreads();
    return __uint_as_float(s_red[0]);
}

}  // namespace nvfp4
