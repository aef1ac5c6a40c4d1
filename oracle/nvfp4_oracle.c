/*
 * nvfp4_oracle.c -- plain, slow, scalar CPU oracle for the NVFP4 quantize path.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and
 * the bench's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant generator with the CUDA library: every value here
 * is computed from the definitions below, one element at a time, in IEEE
 * binary32 (C `float`, built with -ffp-contract=off, no fast-math, no FTZ).
 *
 * Sources (page title, section):
 *  [P2] "MXFP4 和 NVFP4 的区别" (blog.daoxuan.cc): sections
 *       "数据格式:极简的 E2M1", "精度核心:两级分层缩放", "随机舍入",
 *       "随机 Hadamard 变换", "构造 Hadamard 矩阵的方法",
 *       "为什么不用 Conference 矩阵,而用 Hadamard" (fast transform, butterflies).
 *  [P3] "Melatih model dalam 4 bit: pengaman numerik di balik NVFP4"
 *       (iohtechco.com): "Anatomi NVFP4: empat bit dengan dua tingkat skala",
 *       "Empat pengaman yang membuat 4 bit bisa konvergen".
 *  [P4] "how numbers are stored in computers" (number.rest/format/fp4).
 *  [P5] "NVFP4 Is a Scaling System, Not Just a 4-Bit Number"
 *       (nakranivaibhav.github.io): "Four bits do not provide many choices",
 *       "The smallest example: the same payload, two real values",
 *       "A format is not a training recipe".
 *  Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
 *       Easy as 1, 2, 3", SC'11 -- the published round function and constants.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - E2M1 code bits: b3 sign, b2..b1 exponent e, b0 mantissa m; magnitude
 *    m/2 when e == 0, else 2^(e-1) * (1 + m/2).  Bias 1 is the only bias that
 *    gives the listed magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 in code order.
 *  - All 16 E2M1 codes are finite (the NaN claim on [P4] is not followed).
 *  - Nibble order: element 2j goes to the low nibble of byte j.
 *  - E4M3 block scales are the FN variant (max 448), round to nearest even,
 *    saturating to 448; block scales are >= 0 so the sign bit is 0.
 *  - s_global = amax / (448 * 6); the block scale is block_amax / (6 * s_global)
 *    with the multiply and the divide each rounded; the element multiplier is
 *    the rounded reciprocal of the rounded product s_block * s_global.
 *  - Zero handling: amax 0 gives s_global 0; a zero block scale, or a zero
 *    element, encodes a signed zero.
 *  - The RHT is 16 points, y = (1/4) * H16 * (d . x), H16 the Sylvester
 *    matrix in natural order, applied per 16-chunk along the quantized axis,
 *    d a +-1 vector drawn from Philox; amax is taken of the rotated values.
 *    Larger orders n = 32, 64, 128 (the Sylvester recursion goes on to any
 *    power of two): the same butterflies for h = 1 .. n/2, then one multiply
 *    by RN(1/sqrt(n)); the 16-element quantization blocks stay as they are,
 *    n/16 of them per chunk.
 *  - Stochastic rounding uses 16 random bits per element from Philox keyed by
 *    (seed, element index in the quantized output layout).
 *  NOTE: nothing here calls, links or includes the CUDA library.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bf16 input: a bf16 value is the top 16 bits of a binary32 (exact widening) */
static float bf16_to_float(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------ */
/* E2M1 element format [P2 "数据格式:极简的 E2M1"], [P5 "Four bits ..."].     */
double nvfp4o_e2m1_value(int code) {
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Nearest magnitude code (0..7) to a >= 0, ties to the even mantissa; a >= 6
 * (and +inf) saturates to code 7 = 6.0.  Distances are exact in double. */
static int e2m1_mag_rne(double a) {
    if (!(a < 6.0)) return 7;            /* >= 6, +inf (and NaN: outside the contract) */
    int best = 0;
    double bestd = a;                    /* distance to magnitude 0 */
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - nvfp4o_e2m1_value(c));
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* Round-to-nearest-even encode of one binary32 value; the sign bit is always
 * the sign of v, so -0 and tiny negatives give code 0x8. */
int nvfp4o_e2m1_rne(float v) {
    int sign = signbit(v) ? 8 : 0;
    return sign | e2m1_mag_rne(fabs((double)v));
}

/* Stochastic rounding [P2 "随机舍入"], [P3 "Empat pengaman"]: between the two
 * neighbouring magnitudes lo <= |v| < hi, p = (|v| - lo) / (hi - lo) is cut
 * to 16 fraction bits, f = floor(p * 2^16), the element's 16 random bits u
 * are added, and the carry decides: up iff f + u >= 2^16 (probability
 * f / 2^16, within 2^-16 of p).  Representable |v| never moves; |v| >= 6
 * saturates to 6. */
int nvfp4o_e2m1_sr(float v, uint32_t u16) {
    int sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    if (!(a < 6.0)) return sign | 7;
    int lo = 0;
    for (int c = 1; c < 8; ++c)
        if (nvfp4o_e2m1_value(c) <= a) lo = c;
    double lov = nvfp4o_e2m1_value(lo);
    if (a == lov) return sign | lo;
    double hiv = nvfp4o_e2m1_value(lo + 1);
    double p = (a - lov) / (hiv - lov);          /* exact: the gap is a power of two */
    double f = floor(p * 65536.0);               /* exact: p has at most 24 significant bits */
    return sign | ((f + (double)u16 >= 65536.0) ? lo + 1 : lo);
}

/* ------------------------------------------------------------------------ */
/* E4M3 (FN) block scale [P2 "精度核心:两级分层缩放"], [P3 "Anatomi NVFP4"]:
 * 4 exponent bits (bias 7), 3 mantissa bits, max 448, S.1111.111 is NaN.    */
double nvfp4o_e4m3_value(int code) {
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest non-negative finite E4M3 code to s >= 0, ties to even mantissa,
 * values above 448 saturate to 448 (code 0x7E). */
int nvfp4o_e4m3_rne_satfinite(float s) {
    double a = (double)s;
    if (!(a <= 448.0)) return 0x7E;
    int best = 0;
    double bestd = fabs(a);
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs(a - nvfp4o_e4m3_value(c));
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon et al., SC'11): ten rounds of the 4x32 S-box with
 * multipliers 0xD2511F53 (word 0) and 0xCD9E8D57 (word 2); the key is bumped
 * by the Weyl constants 0x9E3779B9 / 0xBB67AE85 between rounds. */
void nvfp4o_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        uint32_t n1 = (uint32_t)p1;
        uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        uint32_t n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* 16 random bits of output element i: counter (lo32(i/8), hi32(i/8), 0, 0),
 * key (lo32(seed), hi32(seed)); word (i%8)/2, low half when i is even. */
uint32_t nvfp4o_sr_bits(uint64_t seed, uint64_t i) {
    uint64_t g = i / 8;
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), 0u, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    nvfp4o_philox4x32_10(ctr, key, out);
    uint32_t w = out[(i % 8) / 2];
    return (i % 2 == 0) ? (w & 0xFFFFu) : (w >> 16);
}

/* RHT sign vector [P2 "随机 Hadamard 变换" -- a random diagonal of signs]:
 * Philox at counter (0, 0, 1, 0), key from rht_seed; d_j = -1 iff bit
 * (j mod 32) of output word floor(j / 32) is set.  Writes n entries of +-1,
 * n <= 128 (one Philox call gives 128 bits); the first 16 entries do not
 * depend on n. */
void nvfp4o_rht_signs_n(uint64_t rht_seed, int n, float* d) {
    uint32_t ctr[4] = {0u, 0u, 1u, 0u};
    uint32_t key[2] = {(uint32_t)rht_seed, (uint32_t)(rht_seed >> 32)};
    uint32_t out[4];
    nvfp4o_philox4x32_10(ctr, key, out);
    for (int j = 0; j < n; ++j) d[j] = ((out[j / 32] >> (j % 32)) & 1u) ? -1.0f : 1.0f;
}

/* The 16-point sign vector (word 0, bits 0..15). */
void nvfp4o_rht_signs(uint64_t rht_seed, float d[16]) { nvfp4o_rht_signs_n(rht_seed, 16, d); }

/* Normalisation of the n-point transform: 1/sqrt(n) rounded to binary32
 * (a power of two for n = 16, 64; RN(sqrt(2)) * 2^-3 and * 2^-4 for n = 32
 * and 128), so that RN(1/sqrt(n)) * H_n * D is orthogonal up to one
 * rounding of the factor. */
float nvfp4o_rht_norm(int n) { return (float)(1.0 / sqrt((double)n)); }

/* n-point random Hadamard transform of one chunk, n a power of two in
 * [16, 128] [P2 "构造 Hadamard 矩阵的方法" (Sylvester recursion: four H_n
 * blocks, lower-right negated, so H_n[i][j] = (-1)^popcount(i & j)) and
 * "为什么不用 Conference 矩阵" (fast transform by butterflies, additions and
 * subtractions only)]: y = d . x; for h = 1, 2, 4, ..., n/2 replace each pair
 * (y_i, y_{i+h}) with i & h == 0 by (y_i + y_{i+h}, y_i - y_{i+h}); then
 * multiply every entry by nvfp4o_rht_norm(n). */
void nvfp4o_rht_n(const float* x, const float* d, int n, float* y) {
    float t[128];
    for (int j = 0; j < n; ++j) t[j] = d[j] * x[j];
    for (int h = 1; h < n; h <<= 1) {
        for (int i = 0; i < n; ++i) {
            if (i & h) continue;
            float a = t[i], b = t[i + h];
            t[i] = a + b;
            t[i + h] = a - b;
        }
    }
    float c = nvfp4o_rht_norm(n);
    for (int j = 0; j < n; ++j) y[j] = t[j] * c;
}

/* The 16-point transform, y = (1/4) H16 (d . x). */
void nvfp4o_rht16(const float x[16], const float d[16], float y[16]) { nvfp4o_rht_n(x, d, 16, y); }

/* ------------------------------------------------------------------------ */
/* Global (tensor) scale [P3 "Anatomi NVFP4"]: amax / (448 * 6). */
float nvfp4o_global_scale(float amax) {
    const float emax_prod = 2688.0f;   /* 448 (E4M3 max) * 6 (E2M1 max), exact */
    return amax / emax_prod;
}

/* Block scale [P2 "精度核心:两级分层缩放"], [P5 "The smallest example"]:
 * s = e4m3(block_amax / (6 * s_global)); returns the code. */
int nvfp4o_block_scale_code(float block_amax, float s_global) {
    float t = 6.0f * s_global;
    float sf = (t == 0.0f) ? 0.0f : block_amax / t;
    return nvfp4o_e4m3_rne_satfinite(sf);
}

/* Encode one element given its block's decoded scale and the global scale.
 * rounding 0 = RNE, 1 = SR (u16 = the element's random bits). */
int nvfp4o_encode_element(float y, float s_dec, float s_global, int rounding, uint32_t u16) {
    if (s_dec == 0.0f || y == 0.0f) return signbit(y) ? 8 : 0;
    float prod = s_dec * s_global;
    float r = (prod == 0.0f) ? INFINITY : 1.0f / prod;
    float v = y * r;
    return rounding ? nvfp4o_e2m1_sr(v, u16) : nvfp4o_e2m1_rne(v);
}

/* ------------------------------------------------------------------------ */
/* The quantized tensor Q of a bf16 input x [rows x cols] (row stride ld):
 * Q = x when transpose == 0 ([rows x cols]); Q = x^T when transpose == 1
 * ([cols x rows]).  Q(r, c) as binary32. */
static float q_at(const uint16_t* x, int64_t ld, int transpose, int64_t r, int64_t c) {
    return transpose ? bf16_to_float(x[c * ld + r]) : bf16_to_float(x[r * ld + c]);
}

/* Row r of Q, columns c0 .. c0+n-1, after the n-point RHT when rht_n != 0
 * (n = rht_n, c0 a multiple of it); without RHT, n = 16. */
static void q_chunk(const uint16_t* x, int64_t ld, int transpose, int rht_n, const float* d,
                    int64_t r, int64_t c0, float* y) {
    int n = rht_n ? rht_n : 16;
    float t[128];
    for (int j = 0; j < n; ++j) t[j] = q_at(x, ld, transpose, r, c0 + j);
    if (rht_n) nvfp4o_rht_n(t, d, rht_n, y);
    else memcpy(y, t, sizeof(float) * (size_t)n);
}

/* Tensor amax [P3 "Anatomi NVFP4"; P5 "Why two levels" -- the global scale
 * comes from the tensor's maximum absolute value before the block maxima],
 * over Q (rotated by the rht_n-point transform when rht_n != 0; the length of
 * a Q row must then be a multiple of rht_n). */
float nvfp4o_amax_n(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                    int rht_n, uint64_t rht_seed) {
    int64_t qr = transpose ? cols : rows, qc = transpose ? rows : cols;
    int n = rht_n ? rht_n : 16;
    float d[128];
    float a = 0.0f;
    if (rht_n) nvfp4o_rht_signs_n(rht_seed, rht_n, d);
    for (int64_t r = 0; r < qr; ++r) {
        for (int64_t c0 = 0; c0 + n <= qc; c0 += n) {
            float y[128];
            q_chunk(x, ld, transpose, rht_n, d, r, c0, y);
            for (int j = 0; j < n; ++j) {
                float m = fabsf(y[j]);
                if (m > a) a = m;
            }
        }
    }
    return a;
}

float nvfp4o_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                  int rht, uint64_t rht_seed) {
    return nvfp4o_amax_n(x, rows, cols, ld, transpose, rht ? 16 : 0, rht_seed);
}

/* 1D quantization (16 consecutive elements of a Q row share one E4M3 scale)
 * of Q rows [r_begin, r_end), given the tensor's global scale.  codes points
 * at the codes of row r_begin ([r_end - r_begin] x Q_cols/2), scales at its
 * scales ([r_end - r_begin] x Q_cols/16).  rounding 0 = RNE (weights and
 * activations), 1 = SR (gradients) [P2 "随机舍入:为什么只用在梯度上"].
 * rht_n != 0: Q rows are first rotated chunk by chunk (rht_n points, a
 * multiple of 16); each chunk then holds rht_n/16 blocks. */
void nvfp4o_quantize_1d_rows_n(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                               int transpose, int rht_n, uint64_t rht_seed, int rounding,
                               uint64_t sr_seed, float s_global, int64_t r_begin, int64_t r_end,
                               uint8_t* codes, uint8_t* scales) {
    int64_t qc = transpose ? rows : cols;
    int n = rht_n ? rht_n : 16;
    float d[128];
    if (rht_n) nvfp4o_rht_signs_n(rht_seed, rht_n, d);
    for (int64_t r = r_begin; r < r_end; ++r) {
        for (int64_t c0 = 0; c0 + n <= qc; c0 += n) {
            float ychunk[128];
            q_chunk(x, ld, transpose, rht_n, d, r, c0, ychunk);
            for (int b0 = 0; b0 < n; b0 += 16) {
                const float* y = ychunk + b0;
                int64_t cb = c0 + b0;
                float b = 0.0f;
                for (int j = 0; j < 16; ++j) {
                    float m = fabsf(y[j]);
                    if (m > b) b = m;
                }
                int sc = nvfp4o_block_scale_code(b, s_global);
                float s_dec = (float)nvfp4o_e4m3_value(sc);
                scales[(r - r_begin) * (qc / 16) + cb / 16] = (uint8_t)sc;
                for (int j = 0; j < 16; ++j) {
                    uint64_t idx = (uint64_t)(r * qc + cb + j);
                    uint32_t u = rounding ? nvfp4o_sr_bits(sr_seed, idx) : 0u;
                    int code = nvfp4o_encode_element(y[j], s_dec, s_global, rounding, u);
                    uint8_t* byte = &codes[(r - r_begin) * (qc / 2) + (cb + j) / 2];
                    if (((cb + j) & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | code);
                    else *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
                }
            }
        }
    }
}

void nvfp4o_quantize_1d_rows(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                             int transpose, int rht, uint64_t rht_seed, int rounding,
                             uint64_t sr_seed, float s_global, int64_t r_begin, int64_t r_end,
                             uint8_t* codes, uint8_t* scales) {
    nvfp4o_quantize_1d_rows_n(x, rows, cols, ld, transpose, rht ? 16 : 0, rht_seed, rounding, sr_seed,
                              s_global, r_begin, r_end, codes, scales);
}

/* Whole-tensor 1D quantization: amax, global scale, then every row. */
void nvfp4o_quantize_1d_n(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                          int rht_n, uint64_t rht_seed, int rounding, uint64_t sr_seed,
                          uint8_t* codes, uint8_t* scales, float* global_scale) {
    float a = nvfp4o_amax_n(x, rows, cols, ld, transpose, rht_n, rht_seed);
    float sg = nvfp4o_global_scale(a);
    int64_t qr = transpose ? cols : rows;
    nvfp4o_quantize_1d_rows_n(x, rows, cols, ld, transpose, rht_n, rht_seed, rounding, sr_seed, sg, 0, qr,
                              codes, scales);
    *global_scale = sg;
}

void nvfp4o_quantize_1d(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int transpose,
                        int rht, uint64_t rht_seed, int rounding, uint64_t sr_seed,
                        uint8_t* codes, uint8_t* scales, float* global_scale) {
    nvfp4o_quantize_1d_n(x, rows, cols, ld, transpose, rht ? 16 : 0, rht_seed, rounding, sr_seed, codes, scales,
                         global_scale);
}

/* 2D quantization of a weight [P1 "2D block scaling for weights"; P3 "Empat
 * pengaman" -- one E4M3 scale per 16x16 tile, so rowwise and columnwise
 * quantization agree], round to nearest even.  Tile rows [tr_begin, tr_end)
 * (units of 16 rows).  codes_row points at the codes of row 16*tr_begin,
 * scales at the scales of tile row tr_begin; codes_col (may be NULL) is the
 * whole code array of W^T, [cols x rows/2]. */
void nvfp4o_quantize_2d_tiles(const uint16_t* w, int64_t rows, int64_t cols, int64_t ld,
                              float s_global, int64_t tr_begin, int64_t tr_end,
                              uint8_t* codes_row, uint8_t* codes_col, uint8_t* scales) {
    for (int64_t tr = tr_begin; tr < tr_end; ++tr) {
        for (int64_t tc = 0; tc < cols / 16; ++tc) {
            float b = 0.0f;
            for (int i = 0; i < 16; ++i)
                for (int j = 0; j < 16; ++j) {
                    float m = fabsf(bf16_to_float(w[(tr * 16 + i) * ld + tc * 16 + j]));
                    if (m > b) b = m;
                }
            int sc = nvfp4o_block_scale_code(b, s_global);
            float s_dec = (float)nvfp4o_e4m3_value(sc);
            scales[(tr - tr_begin) * (cols / 16) + tc] = (uint8_t)sc;
            for (int i = 0; i < 16; ++i)
                for (int j = 0; j < 16; ++j) {
                    int64_t r = tr * 16 + i, c = tc * 16 + j;
                    int code = nvfp4o_encode_element(bf16_to_float(w[r * ld + c]), s_dec, s_global, 0, 0u);
                    uint8_t* br = &codes_row[(r - tr_begin * 16) * (cols / 2) + c / 2];
                    if ((c & 1) == 0) *br = (uint8_t)((*br & 0xF0) | code);
                    else *br = (uint8_t)((*br & 0x0F) | (code << 4));
                    if (codes_col) {
                        uint8_t* bc = &codes_col[c * (rows / 2) + r / 2];
                        if ((r & 1) == 0) *bc = (uint8_t)((*bc & 0xF0) | code);
                        else *bc = (uint8_t)((*bc & 0x0F) | (code << 4));
                    }
                }
        }
    }
}

void nvfp4o_quantize_2d(const uint16_t* w, int64_t rows, int64_t cols, int64_t ld,
                        uint8_t* codes_row, uint8_t* codes_col, uint8_t* scales, float* global_scale) {
    float a = nvfp4o_amax(w, rows, cols, ld, 0, 0, 0);
    float sg = nvfp4o_global_scale(a);
    nvfp4o_quantize_2d_tiles(w, rows, cols, ld, sg, 0, rows / 16, codes_row, codes_col, scales);
    *global_scale = sg;
}

/* ------------------------------------------------------------------------ */
/* Reconstruction [P5 "The smallest example": x = x_e2m1 * s_block * s_global;
 * P2 "精度核心"]: out = RN(RN(value(code) * s_dec) * s_global), binary32.
 * scale_mode 0: scales [rows x cols/16]; 1: scales [rows/16 x cols/16]. */
void nvfp4o_dequantize(const uint8_t* codes, const uint8_t* scales, int scale_mode, float s_global,
                       int64_t rows, int64_t cols, float* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 0xF);
            int sc = scale_mode ? scales[(r / 16) * (cols / 16) + c / 16] : scales[r * (cols / 16) + c / 16];
            float s_dec = (float)nvfp4o_e4m3_value(sc);
            float v = (float)nvfp4o_e2m1_value(code);
            float t = v * s_dec;
            out[r * cols + c] = t * s_global;
        }
}

/* ------------------------------------------------------------------------ */
/* Element-wise batch forms of the scalar encoders above (plain loops; they
 * exist only so that exhaustive tests do not pay one foreign call per value). */
void nvfp4o_e2m1_rne_batch(const float* v, int64_t n, uint8_t* codes) {
    for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)nvfp4o_e2m1_rne(v[i]);
}

/* SR of v[i] with the random bits of output index first_index + i. */
void nvfp4o_e2m1_sr_batch(const float* v, int64_t n, uint64_t seed, uint64_t first_index, uint8_t* codes) {
    for (int64_t i = 0; i < n; ++i)
        codes[i] = (uint8_t)nvfp4o_e2m1_sr(v[i], nvfp4o_sr_bits(seed, first_index + (uint64_t)i));
}

void nvfp4o_e4m3_batch(const float* s, int64_t n, uint8_t* codes) {
    for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)nvfp4o_e4m3_rne_satfinite(s[i]);
}

/* ------------------------------------------------------------------------ */
/* MXFP4 [P2 "MXFP4:开放标准,但精度较粗" -- 32 values share one scale that can
 * only be a power of two, stored as E8M0; P5 "Generic FP4, MXFP4, and NVFP4"
 * -- E2M1 payloads, one E8M0 scale per 32 values, no tensor-level scale].
 * The pages do not say how the power of two is chosen; reading: the OCP
 * microscaling rule the format is named after -- X = 2^(floor(log2(amax)) -
 * 2), 2 being the exponent of the largest E2M1 value (6 = 1.5 * 2^2), so the
 * block maximum lands in [4, 8) and values above 6 saturate.  The exponent is
 * clamped to the E8M0 range [-127, 127]; an all-zero block gets -127.
 * E8M0 code = exponent + 127 (255, NaN, is never produced). */
int nvfp4o_mx_scale_exp(float block_amax) {
    if (!(block_amax > 0.0f)) return -127;
    int e2;
    (void)frexp((double)block_amax, &e2);        /* amax = f * 2^e2, f in [0.5, 1) */
    int e = (e2 - 1) - 2;                        /* floor(log2(amax)) - 2 */
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

double nvfp4o_e8m0_value(int code) { return ldexp(1.0, code - 127); }

/* One element: v = x / 2^e (exact in double), E2M1 by nearest-even with
 * saturation at +-6, sign kept. */
int nvfp4o_mx_encode_element(float x, int e) {
    double v = ldexp((double)x, -e);
    int sign = signbit(x) ? 8 : 0;
    return sign | e2m1_mag_rne(fabs(v));
}

/* MXFP4 quantization of bf16 x [rows x cols] (cols % 32 == 0), blocks of 32
 * along each row: codes [rows x cols/2], scales (E8M0 codes) [rows x cols/32]. */
void nvfp4o_mx_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes,
                        uint8_t* scales) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 32; ++b) {
            float amax = 0.0f;
            for (int j = 0; j < 32; ++j) {
                float a = fabsf(bf16_to_float(x[r * ld + 32 * b + j]));
                if (a > amax) amax = a;
            }
            int e = nvfp4o_mx_scale_exp(amax);
            scales[r * (cols / 32) + b] = (uint8_t)(e + 127);
            for (int j = 0; j < 32; j += 2) {
                int lo = nvfp4o_mx_encode_element(bf16_to_float(x[r * ld + 32 * b + j]), e);
                int hi = nvfp4o_mx_encode_element(bf16_to_float(x[r * ld + 32 * b + j + 1]), e);
                codes[r * (cols / 2) + 16 * b + j / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
}

/* Reconstruction x = value(code) * 2^e, in binary32 (exact unless it underflows). */
void nvfp4o_mx_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, float* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 0xF);
            double s = nvfp4o_e8m0_value(scales[r * (cols / 32) + c / 32]);
            out[r * cols + c] = (float)(nvfp4o_e2m1_value(code) * s);
        }
}
