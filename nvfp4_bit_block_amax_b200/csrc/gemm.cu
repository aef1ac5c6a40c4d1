// gemm.cu -- block-scaled NVFP4 GEMM on the sm_100a tensor cores.
//
// C = alpha * A . B^T, A [M x K] and B [N x K] as packed E2M1 codes (K-major,
// "TN"), one UE4M3 scale per 16 elements along K for each row, FP32
// accumulation in tensor memory, alpha = s_global_A * s_global_B.
// Sources: "Melatih model dalam 4 bit: pengaman numerik di balik NVFP4",
// "Presisi sebagai tombol throughput" (the matmuls dominate the step);
// "NVFP4 Is a Scaling System, Not Just a 4-Bit Number", "Hardware support
// still needs a full sentence" (native block-scaled matrix operations on
// Blackwell tensor cores) and "“4-bit” is a payload count" (TN-only GEMM
// layout, padded/swizzled scale layout).
//
// Design (one CTA per SM, persistent over 128 x 256 output tiles; tiles are
// taken in groups of M-tiles so that the concurrently active A and B panels
// stay resident in L2):
//   warp 0      TMA producer: A tile 128 x 256 codes, B tile 256 x 256 codes
//               (128-byte swizzled), scale chunks by bulk copy; 4 stages.
//   warp 1      TMEM allocator and MMA issuer: tcgen05.mma kind::mxf4nvf4
//               block_scale scale_vec::4X, M = 128, N = 256, K = 64; commits
//               free smem stages, scale buffers and signal the accumulator.
//               Nothing but MMAs goes down its tensor pipe: a scale copy
//               (tcgen05.cp) issued in the same pipe costs about half an MMA.
//   warps 2..5  one warp per TMEM lane quarter.  (a) Block scales smem ->
//               registers -> TMEM (tcgen05.st), up to 4 K-blocks ahead of
//               the MMAs.  (b) The epilogue of columns 0..127 of a finished
//               tile, started the moment its accumulator is complete (the
//               waits for scale data poll for it).
//   warps 6..9  epilogue of columns 128..255.  Epilogue: TMEM -> registers
//               (128 columns per thread, packed to bf16), free the
//               accumulator for the next tile, then scale by alpha and store.
// Every mbarrier wait is bounded in time: on expiry the kernel raises the
// device error word, lets in-flight copies and MMAs land, frees TMEM and
// returns (nvfp4_get_error reports NVFP4_ERR_TIMEOUT).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace nvfp4 {

__device__ unsigned int g_error_word = 0;

namespace {

constexpr int BM = 128, BN = 256, BK = 256;          // elements
constexpr int BKB = BK / 2;                          // bytes of codes per row per stage
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BKB;                    // 16 KB
constexpr int B_STAGE = BN * BKB;                    // 32 KB
constexpr int SFA_STAGE = 4 * 512;                   // 4 K-steps x (128 rows x 4 scales)
constexpr int SFB_STAGE = 2 * 4 * 512;               // 2 row chunks x 4 K-steps
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_SFA = OFF_B + STAGES * B_STAGE;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_STAGE;
// Block scales of stage s live in tensor-memory buffer s: a stage's data can
// only land after the MMAs that read the buffer's previous contents have
// completed (the producer waits for them), so the buffer needs no barrier of
// its own to be freed.
constexpr int NUM_BARS = 3 * STAGES + 3;             // full, empty, sf_full per stage; tmem_full/empty, drain
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;     // + alignment slack
constexpr int NUM_THREADS = 320;                     // 10 warps (at most 3 per SM sub-partition)
constexpr int EPI_WARPS = 8;                         // warps 2..5: scales -> TMEM + epilogue columns 0..127;
                                                     // warps 6..9: epilogue columns 128..255
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t SF_COL = 256;                     // one buffer of 48 columns (16 SFA + 32 SFB) per stage
constexpr unsigned long long kWaitLimitNs = 4000000000ull;
static_assert(SF_COL + STAGES * 48 <= TMEM_COLS, "scale buffers must fit in tensor memory");

// ------------------------------------------------------------- PTX wrappers --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Non-blocking probe of a barrier phase.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false when the limit ran out (the error word and the CTA's
// abort flag are then set) or another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicExch(&g_error_word, 1u);
            return false;
        }
    }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// NVFP4: one UE4M3 scale per 16 elements (scale_vec::4X).  MXFP4: one UE8M0
// scale per 32 elements (scale_vec::2X), in bytes 0-1 of the same 4-byte
// scale entry per row and 64-wide K step.
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa, uint32_t sfb, uint32_t accumulate, bool mx) {
    if (mx)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
            : "memory");
}
__device__ __forceinline__ void tc_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}


// --------------------------------------------------- CTA-pair (2-SM) helpers --
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on the barrier at the same shared-memory offset in CTA `rank` of the
// cluster.  Relaxed: what the peer waits for is tensor-memory traffic that
// this thread has already waited out (tcgen05.wait::st / wait::ld, then
// tcgen05.fence::before_thread_sync); a release at cluster scope would also
// wait for every global store the warp has in flight (the epilogue's), which
// measured above 1000 cycles per arrive.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar, uint32_t rank) {
    asm volatile(
        "{\n\t.reg .b32 ra;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
        "mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [ra];\n\t}"
        ::"r"(bar), "r"(rank)
        : "memory");
}
__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_test_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_cluster(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicExch(&g_error_word, 1u);
            return false;
        }
    }
}
// Completion of the CTA pair's prior tcgen05 operations arrives on the barrier
// at this offset in both CTAs.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(bar), "h"((uint16_t)3)
        : "memory");
}
__device__ __forceinline__ void tc_mma_nvf4_pair(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t sfa, uint32_t sfb, uint32_t accumulate, bool mx) {
    if (mx)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
            : "memory");
}

// Shared-memory matrix descriptor: K-major operand tile of rows x 128 bytes,
// 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1), K-major,
// UE4M3 scales, dense K = 64, M = 128, N = 256.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t kIdescUe8m0 = 1u << 23;   // scale type UE8M0 (MXFP4) instead of UE4M3

struct KParams {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* a_gs;
    const float* b_gs;
    int M, N, K;
    int chunks_k;
    int out_bf16;
    void* c;
    int64_t ldc;
    int tiles_m, tiles_n;
    int group_m;   // tile rasterization: groups of group_m M-tiles, M fastest inside a group
    unsigned int* c_amax;   // nullable: atomic max of |C| (binary32 bits of the stored values)
    int mx;                 // MXFP4 operands: UE8M0 scales per 32 elements, no global scales (alpha = 1)
};

// Fold this thread's maximum |C| (binary32 bits, non-negative) into c_amax:
// one atomic per warp, once per kernel (the epilogue roles keep a running
// maximum over all the tiles they drain).
__device__ __forceinline__ void amax_publish(unsigned int* c_amax, uint32_t m) {
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if ((threadIdx.x & 31) == 0 && m) atomicMax(c_amax, m);
}
// Largest |bf16| among the packed pairs of one epilogue row: columns at or
// past ncols (and rows at or past M) do not count.
__device__ __forceinline__ uint32_t packed_row_amax(const uint32_t (&packed)[64], int ncols, bool row_ok) {
    uint32_t acc = 0;
    if (row_ok) {
#pragma unroll
        for (int g = 0; g < 64; ++g) {
            uint32_t w = packed[g];
            if (2 * g + 1 >= ncols) w = (2 * g < ncols) ? (w & 0xFFFFu) : 0u;
            acc = absmax2(acc, w);
        }
    }
    return absmax2_fold(acc);
}

// Output scale factors (a1, a2): C = RN(RN(acc * a1) * a2).  Normally a1 =
// alpha = RN(s_global_A * s_global_B) and a2 = 1 (the second multiply is
// exact).  When alpha is not a normal binary32 number -- both global scales
// tiny, so that their product is subnormal or zero, or both huge, so that it
// overflows -- the two global scales are applied one after the other
// (a1 = s_global_A, a2 = s_global_B): the accumulator times one scale stays
// in range wherever C itself does.  MXFP4 operands have no global scale.
__device__ __forceinline__ float2 out_scales(const KParams& p) {
    if (!p.a_gs) return make_float2(1.0f, 1.0f);
    const float sa = __ldg(p.a_gs), sb = __ldg(p.b_gs);
    const float alpha = __fmul_rn(sa, sb);
    if (alpha >= 0x1p-126f && alpha <= 0x1.fffffep127f) return make_float2(alpha, 1.0f);
    return make_float2(sa, sb);
}
// Two accumulator values scaled by (a1, a2), in f32x2 multiplies.
__device__ __forceinline__ float2 scale_out2(uint32_t u0, uint32_t u1, float2 al) {
    const float2 v = __fmul2_rn(make_float2(__uint_as_float(u0), __uint_as_float(u1)), make_float2(al.x, al.x));
    return __fmul2_rn(v, make_float2(al.y, al.y));
}

// Tile t -> (tm, tn).  Tiles are taken in groups of group_m M-tiles; inside a
// group M runs fastest, then N, and odd groups walk N backwards.  The CTAs
// working at the same time then share group_m A panels and a few B panels,
// which stay resident in L2, and a group starts on the B panels its
// predecessor used last (measured: dgrad DRAM reads 3.2 -> 2.6 GB per launch).
__device__ __forceinline__ void tile_coords(int t, const KParams& p, int& tm, int& tn) {
    const int per_group = p.group_m * p.tiles_n;
    const int g = t / per_group;
    const int r = t - g * per_group;
    const int first = g * p.group_m;
    const int gm = min(p.group_m, p.tiles_m - first);
    tm = first + r % gm;
    tn = r / gm;
    if (g & 1) tn = p.tiles_n - 1 - tn;   // serpentine: a group starts on the B panels the previous one ended on
}

// Epilogue of one column half (128 columns) of a finished tile for the
// calling warp's TMEM lane quarter: TMEM -> registers (bf16 output: packed
// pairs, 64 registers), arrive on tmem_empty, then store.  False when the
// bounded wait for the accumulator ran out.
__device__ __forceinline__ bool epilogue_half(const KParams& p, int tile, int half, int q, int lane, uint32_t tmem,
                                              float2 alpha, uint32_t bar_tfull, uint32_t bar_tempty,
                                              uint32_t& acc_phase, volatile int* abort_flag, uint32_t& amax_acc) {
    if (!mbar_wait(bar_tfull, acc_phase, abort_flag)) return false;
    tc_fence_after();
    int tm, tn;
    tile_coords(tile, p, tm, tn);
    const int row = tm * BM + q * 32 + lane;
    const int col0 = tn * BN + half * 128;
    const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + ACC_COL + half * 128;
    const int ncols = p.N - col0;   // columns of this half inside C
    if (p.out_bf16) {
        // Two rounds of 64 columns: both loads of a round are in flight
        // before the one wait, so the accumulator is read with two TMEM
        // round trips instead of eight.
        uint32_t packed[64];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint32_t v0[32], v1[32];
            tc_ld_32x32b_x32(taddr + 64 * i, v0);
            tc_ld_32x32b_x32(taddr + 64 * i + 32, v1);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float2 f0 = scale_out2(v0[2 * e], v0[2 * e + 1], alpha);
                const float2 f1 = scale_out2(v1[2 * e], v1[2 * e + 1], alpha);
                const __nv_bfloat162 h0 = __floats2bfloat162_rn(f0.x, f0.y);
                const __nv_bfloat162 h1 = __floats2bfloat162_rn(f1.x, f1.y);
                packed[32 * i + e] = *reinterpret_cast<const uint32_t*>(&h0);
                packed[32 * i + 16 + e] = *reinterpret_cast<const uint32_t*>(&h1);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_tempty);
        acc_phase ^= 1;
        if (p.c_amax) amax_acc = max(amax_acc, packed_row_amax(packed, ncols, row < p.M));
        if (row < p.M && ncols > 0) {
            __nv_bfloat16* crow = reinterpret_cast<__nv_bfloat16*>(p.c) + (int64_t)row * p.ldc + col0;
            if (ncols >= 128) {
#pragma unroll
                for (int g = 0; g < 16; ++g)
                    *reinterpret_cast<uint4*>(crow + 8 * g) =
                        make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
            } else {
#pragma unroll
                for (int g = 0; g < 64; ++g) {
                    if (2 * g + 1 < ncols) reinterpret_cast<uint32_t*>(crow)[g] = packed[g];
                    else if (2 * g < ncols) reinterpret_cast<uint16_t*>(crow)[2 * g] = (uint16_t)(packed[g] & 0xFFFFu);
                }
            }
        }
    } else {
        float* crow = reinterpret_cast<float*>(p.c) + (int64_t)row * p.ldc + col0;
        float fmax = 0.0f;
#pragma unroll 1
        for (int i = 0; i < 4; ++i) {
            uint32_t v[32];
            tc_ld_32x32b_x32(taddr + 32 * i, v);
            tc_wait_ld();
            if (row < p.M) {
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const int cc = 32 * i + 4 * g;
                    const float2 f01 = scale_out2(v[4 * g], v[4 * g + 1], alpha);
                    const float2 f23 = scale_out2(v[4 * g + 2], v[4 * g + 3], alpha);
                    const float4 f = make_float4(f01.x, f01.y, f23.x, f23.y);
                    if (cc + 4 <= ncols) {
                        *reinterpret_cast<float4*>(crow + cc) = f;
                        fmax = fmaxf(fmaxf(fmaxf(fmax, fabsf(f.x)), fmaxf(fabsf(f.y), fabsf(f.z))), fabsf(f.w));
                    } else {
                        const float ff[4] = {f.x, f.y, f.z, f.w};
                        for (int e = 0; e < 4; ++e)
                            if (cc + e < ncols) {
                                crow[cc + e] = ff[e];
                                fmax = fmaxf(fmax, fabsf(ff[e]));
                            }
                    }
                }
            }
        }
        amax_acc = max(amax_acc, __float_as_uint(fmax));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_tempty);
        acc_phase ^= 1;
    }
    return true;
}

// MX: MXFP4 operands (scale_vec::2X, UE8M0); a compile-time choice, so the
// MMA issue loop carries no branch for it.
template <bool MX>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_nvf4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b, KParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + OFF_BAR;
    const uint32_t bar_empty = bar_full + STAGES * 8;
    const uint32_t bar_sf_full = bar_empty + STAGES * 8;
    const uint32_t bar_tfull = bar_sf_full + STAGES * 8;
    const uint32_t bar_tempty = bar_tfull + 8;
    const uint32_t bar_drain = bar_tempty + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = p.tiles_m * p.tiles_n;
    const int k_blocks = (p.K + BK - 1) / BK;
    const int k_steps = p.K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
            mbar_init(bar_sf_full + 8 * s, 4);
        }
        mbar_init(bar_tfull, 1);
        mbar_init(bar_tempty, EPI_WARPS);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ producer ----
        if (lane == 0) {
            int s = 0;
            uint32_t phase = 0;
            uint32_t issued_parity = 0;   // bit s: parity of the last phase issued on stage s
            uint32_t issued_any = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                int tm, tn;
                tile_coords(tile, p, tm, tn);
                const int m0 = tm * BM, n0 = tn * BN;
                const int rc_a = m0 >> 7, rc_b = n0 >> 7;
                const int rc_b_max = (p.N + 127) >> 7;
                const int nh = (rc_b + 1 < rc_b_max) ? 2 : 1;
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * s, phase ^ 1, abort_flag)) { ok = false; break; }
                    const int nk = min(4, k_steps - kb * 4);
                    const uint32_t full = bar_full + 8 * s;
                    mbar_expect_tx(full, (uint32_t)(A_STAGE + B_STAGE + nk * 512 * (1 + nh)));
                    tma_load_2d(sbase + OFF_A + s * A_STAGE, &map_a, full, kb * BKB, m0);
                    tma_load_2d(sbase + OFF_B + s * B_STAGE, &map_b, full, kb * BKB, n0);
                    bulk_load(sbase + OFF_SFA + s * SFA_STAGE,
                              p.sfa + ((int64_t)rc_a * p.chunks_k + kb * 4) * 512, nk * 512, full);
                    for (int h = 0; h < nh; ++h)
                        bulk_load(sbase + OFF_SFB + s * SFB_STAGE + h * 2048,
                                  p.sfb + ((int64_t)(rc_b + h) * p.chunks_k + kb * 4) * 512, nk * 512, full);
                    issued_any |= 1u << s;
                    issued_parity = (issued_parity & ~(1u << s)) | (phase << s);
                    if (++s == STAGES) { s = 0; phase ^= 1; }
                }
            }
            // let every issued copy land before the CTA can exit
            for (int st = 0; st < STAGES; ++st)
                if (issued_any & (1u << st)) {
                    const uint32_t par = (issued_parity >> st) & 1u;
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try(bar_full + 8 * st, par) && globaltimer() - t0 < kWaitLimitNs) {}
                }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------- MMA ----
        // Only MMAs go down the tensor pipe: the block scales are already in
        // tensor memory, written by the scale warps.
        if (lane == 0) {
            int s = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            const uint32_t idesc = kIdesc | (MX ? kIdescUe8m0 : 0u);
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait(bar_tempty, acc_phase ^ 1, abort_flag)) break;
                tc_fence_after();
                for (int kb = 0; kb < k_blocks; ++kb) {
                    // sf_full[s] is raised by the scale warps after they saw
                    // full[s]: the stage's codes have landed too.
                    if (!mbar_wait(bar_sf_full + 8 * s, phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const int nk = min(4, k_steps - kb * 4);
                    const uint32_t a_addr = sbase + OFF_A + s * A_STAGE;
                    const uint32_t b_addr = sbase + OFF_B + s * B_STAGE;
                    const uint32_t sfa_col = tmem + SF_COL + s * 48;
                    const uint32_t sfb_col = sfa_col + 16;
                    for (int j = 0; j < nk; ++j)
                        tc_mma_nvf4(tmem + ACC_COL, desc_sw128(a_addr + j * 32), desc_sw128(b_addr + j * 32), idesc,
                                    sfa_col + 4 * j, sfb_col + 8 * j, (kb | j) != 0, MX);
                    tc_commit(bar_empty + 8 * s);
                    if (++s == STAGES) { s = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(bar_tfull);
                acc_phase ^= 1;
            }
            // all MMAs of this CTA complete before TMEM can be freed
            tc_commit(bar_drain);
            const unsigned long long t0 = globaltimer();
            while (!mbar_try(bar_drain, 0) && globaltimer() - t0 < kWaitLimitNs) {}
        }
    } else if (warp < 6) {
        // ------------------------------- scales -> TMEM, and the epilogue ----
        // Warp q of this group owns TMEM lanes 32q..32q+31.  Per 64-wide K
        // step j the MMA reads 4 SFA columns (128 rows; every lane quarter a
        // copy) and 8 SFB columns (256 rows); lane l of every quarter holds
        // the 16 bytes at offset 16 l of the step's 512-byte scale chunks.
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const float2 alpha = out_scales(p);
        int s = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        int prev_tile = -1;
        uint32_t amax_acc = 0;   // max |C| of this thread's drained rows (binary32 bits)

        auto epilogue = [&](int tile) -> bool {
            return epilogue_half(p, tile, 0, q, lane, tmem, alpha, bar_tfull, bar_tempty, acc_phase, abort_flag, amax_acc);
        };

        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            for (int kb = 0; kb < k_blocks; ++kb) {
                // Wait for the stage (its scale buffer is free by then);
                // meanwhile, the moment the previous tile's accumulator is
                // complete, drain this warp's half of it, so that the MMAs of
                // this tile never wait on the arrival of this tile's data to
                // get it back.
                {
                    const unsigned long long t0 = globaltimer();
                    while (true) {
                        if (prev_tile >= 0 && mbar_test(bar_tfull, acc_phase)) {
                            if (!epilogue(prev_tile)) { ok = false; break; }
                            prev_tile = -1;
                        }
                        if (mbar_test(bar_full + 8 * s, phase)) break;
                        if (*abort_flag) { ok = false; break; }
                        if (globaltimer() - t0 > kWaitLimitNs) {
                            *abort_flag = 1;
                            atomicExch(&g_error_word, 1u);
                            ok = false;
                            break;
                        }
                    }
                    if (!ok) break;
                }
                const uint32_t sfa_s = sbase + OFF_SFA + s * SFA_STAGE + 16 * lane;
                const uint32_t sfb_s = sbase + OFF_SFB + s * SFB_STAGE + 16 * lane;
                uint32_t ra[16], rb0[16], rb1[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 va = lds128(sfa_s + j * 512);
                    ra[4 * j] = va.x; ra[4 * j + 1] = va.y; ra[4 * j + 2] = va.z; ra[4 * j + 3] = va.w;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint4 vb = lds128(sfb_s + h * 2048 + j * 512);
                        uint32_t* rb = j < 2 ? rb0 : rb1;
                        const int o = 8 * (j & 1) + 4 * h;
                        rb[o] = vb.x; rb[o + 1] = vb.y; rb[o + 2] = vb.z; rb[o + 3] = vb.w;
                    }
                }
                const uint32_t col = tmem + lane_base + SF_COL + s * 48;
                tc_st_32x32b_x16(col, ra);
                tc_st_32x32b_x16(col + 16, rb0);
                tc_st_32x32b_x16(col + 32, rb1);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_sf_full + 8 * s);
                if (++s == STAGES) { s = 0; phase ^= 1; }
            }
            if (ok && prev_tile >= 0) {   // fewer K-blocks than it took the accumulator to complete
                if (!epilogue(prev_tile)) ok = false;
                prev_tile = -1;
            }
            if (ok) prev_tile = tile;
        }
        if (ok && prev_tile >= 0) epilogue(prev_tile);
        __syncwarp();
        if (p.c_amax) amax_publish(p.c_amax, amax_acc);
    } else {
        // ---------------------------------------- epilogue, columns 128..255 ----
        const int q = warp & 3;
        const float2 alpha = out_scales(p);
        uint32_t acc_phase = 0;
        uint32_t amax_acc = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x)
            if (!epilogue_half(p, tile, 1, q, lane, tmem, alpha, bar_tfull, bar_tempty, acc_phase, abort_flag,
                               amax_acc)) break;
        __syncwarp();
        if (p.c_amax) amax_publish(p.c_amax, amax_acc);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}


// ===================================================================== 2-SM ===
// CTA-pair variant: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64).  CTA r loads A rows
// 128r..128r+127 and B rows 128r..128r+127 of the tile (its halves), its own
// 128 rows of A scales and all 256 rows of B scales; its TMEM holds rows
// 128r.. of the accumulator.  Only CTA 0 issues MMAs; their completion is
// committed to the barriers of both CTAs.  The other CTA signals CTA 0 when
// its scales are in TMEM (which implies its stage has landed) and when its
// epilogue has drained the accumulator.  Per SM this moves 38 KB per 64 K
// columns instead of 54 KB: the single-SM tile is L2-bandwidth bound.
// Per CTA 14 warps: warp 0 the TMA producer, warp 1 the MMA issuer (CTA 0),
// warps 2..5 copy block scales to tensor memory and nothing else (one per
// TMEM lane quarter), warps 6..13 the epilogue (two per lane quarter, one
// per 128-column half).  Keeping the scale copies off the epilogue warps
// means the scales of the next stages are in place while a finished tile is
// drained and stored.  The epilogue stores C through the TMA: each warp
// stages 32 rows x 64 bytes in shared memory and issues one bulk tensor
// store per chunk, so C is written in whole lines and the hardware drops the
// rows and columns past the edges of a ragged tile.
constexpr int P_STAGES = 5;
static_assert(SF_COL + P_STAGES * 48 <= TMEM_COLS, "scale buffers must fit in tensor memory");
constexpr int P_A_STAGE = 128 * BKB;                 // 16 KB
constexpr int P_B_STAGE = 128 * BKB;                 // 16 KB
constexpr int P_OFF_A = 0;
constexpr int P_OFF_B = P_OFF_A + P_STAGES * P_A_STAGE;
constexpr int P_OFF_SFA = P_OFF_B + P_STAGES * P_B_STAGE;
constexpr int P_OFF_SFB = P_OFF_SFA + P_STAGES * SFA_STAGE;
constexpr int P_OFF_BAR = P_OFF_SFB + P_STAGES * SFB_STAGE;
constexpr int P_NUM_BARS = 3 * P_STAGES + 3;   // full, empty, sf_full per stage; tmem_full/empty, drain
constexpr int P_OFF_MISC = P_OFF_BAR + P_NUM_BARS * 8;
constexpr int P_OFF_EPI = (P_OFF_MISC + 16 + 1023) / 1024 * 1024;   // output staging, one 2 KB buffer per epilogue warp
constexpr int EPI_BUF = 2048;                                      // 32 rows x 64 bytes, 64-byte swizzle
constexpr int P_SMEM_BYTES = P_OFF_EPI + 8 * EPI_BUF + 1024;
constexpr int P_NUM_THREADS = 448;                  // 14 warps: producer, MMA, 4 scale warps, 8 epilogue warps
// M = 256 (pair), N = 256, E2M1 x E2M1, UE4M3 scales, K-major.
constexpr uint32_t kIdescPair = (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

// Output store through the tensor-memory-access unit: a 32-row x 64-byte
// chunk staged in shared memory (64-byte swizzle: 16-byte unit u of row r
// sits at unit u ^ ((r >> 1) & 3)) is written to C by one bulk tensor store;
// rows and columns past the tensor's edge are dropped by the hardware.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Stage one 32-row x 64-byte chunk (this lane's row: 16 words) and store it.
__device__ __forceinline__ void store_chunk(const CUtensorMap* map_c, uint32_t buf, int lane, const uint32_t* w, int col,
                                            int row0, bool first) {
    if (!first) {
        if (lane == 0) bulk_wait_read0();   // the buffer's previous chunk has been read out
        __syncwarp();
    }
    const uint32_t rowaddr = buf + lane * 64;
    const uint32_t sw = (lane >> 1) & 3;
#pragma unroll
    for (int u = 0; u < 4; ++u) sts128(rowaddr + ((u ^ sw) << 4), w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(map_c, buf, col, row0);
        bulk_commit();
    }
}

__device__ __forceinline__ bool epilogue_half_pair(const KParams& p, int tile, int half, int q, int lane, uint32_t rank,
                                                   uint32_t tmem, float2 alpha, uint32_t bar_tfull, uint32_t bar_tempty,
                                                   uint32_t& acc_phase, volatile int* abort_flag, uint32_t& amax_acc,
                                                   const CUtensorMap* map_c, uint32_t buf, bool& first) {
    if (!mbar_wait_cluster(bar_tfull, acc_phase, abort_flag)) return false;
    tc_fence_after();
    int tm, tn;
    tile_coords(tile, p, tm, tn);
    const int row = tm * 256 + (int)rank * 128 + q * 32 + lane;
    const int col0 = tn * BN + half * 128;
    const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + ACC_COL + half * 128;
    const int ncols = p.N - col0;
    auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            if (rank == 0) mbar_arrive(bar_tempty);
            else mbar_arrive_cluster(bar_tempty, 0);
        }
        acc_phase ^= 1;
    };
    if (p.out_bf16) {
        uint32_t packed[64];
#pragma unroll
        for (int i = 0; i < 2; ++i) {   // two TMEM round trips of 64 columns
            uint32_t v0[32], v1[32];
            tc_ld_32x32b_x32(taddr + 64 * i, v0);
            tc_ld_32x32b_x32(taddr + 64 * i + 32, v1);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float2 f0 = scale_out2(v0[2 * e], v0[2 * e + 1], alpha);
                const float2 f1 = scale_out2(v1[2 * e], v1[2 * e + 1], alpha);
                const __nv_bfloat162 h0 = __floats2bfloat162_rn(f0.x, f0.y);
                const __nv_bfloat162 h1 = __floats2bfloat162_rn(f1.x, f1.y);
                packed[32 * i + e] = *reinterpret_cast<const uint32_t*>(&h0);
                packed[32 * i + 16 + e] = *reinterpret_cast<const uint32_t*>(&h1);
            }
        }
        release();
        if (p.c_amax) amax_acc = max(amax_acc, packed_row_amax(packed, ncols, row < p.M));
        const int row0 = tm * 256 + (int)rank * 128 + q * 32;
        if (row0 < p.M && ncols > 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (32 * k < ncols) store_chunk(map_c, buf, lane, packed + 16 * k, col0 + 32 * k, row0, first);
                first = false;
            }
        }
    } else {
        // fp32: 8 chunks of 16 columns (64 bytes per row), two chunks per TMEM load of 32 columns
        const int row0 = tm * 256 + (int)rank * 128 + q * 32;
        const bool live = row0 < p.M && ncols > 0;
        float fmax = 0.0f;
#pragma unroll 1
        for (int i = 0; i < 4; ++i) {
            uint32_t v[32];
            tc_ld_32x32b_x32(taddr + 32 * i, v);
            tc_wait_ld();
            if (i == 3) release();
            uint32_t f[32];
#pragma unroll
            for (int g = 0; g < 16; ++g) {
                const float2 o = scale_out2(v[2 * g], v[2 * g + 1], alpha);
                f[2 * g] = __float_as_uint(o.x);
                f[2 * g + 1] = __float_as_uint(o.y);
                if (row < p.M) {
                    if (32 * i + 2 * g < ncols) fmax = fmaxf(fmax, fabsf(o.x));
                    if (32 * i + 2 * g + 1 < ncols) fmax = fmaxf(fmax, fabsf(o.y));
                }
            }
            if (live) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (32 * i + 16 * h < ncols) store_chunk(map_c, buf, lane, f + 16 * h, col0 + 32 * i + 16 * h, row0, first);
                    first = false;
                }
            }
        }
        amax_acc = max(amax_acc, __float_as_uint(fmax));
    }
    return true;
}

template <bool MX>
__global__ void __launch_bounds__(P_NUM_THREADS, 1)
gemm_nvf4_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_c, KParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + P_OFF_BAR;
    const uint32_t bar_empty = bar_full + P_STAGES * 8;
    const uint32_t bar_sf_full = bar_empty + P_STAGES * 8;
    const uint32_t bar_tfull = bar_sf_full + P_STAGES * 8;
    const uint32_t bar_tempty = bar_tfull + 8;
    const uint32_t bar_drain = bar_tempty + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + P_OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + P_OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const int num_tiles = p.tiles_m * p.tiles_n;
    const int k_blocks = (p.K + BK - 1) / BK;
    const int k_steps = p.K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < P_STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
            mbar_init(bar_sf_full + 8 * s, 8);       // 4 scale warps in each CTA
        }
        mbar_init(bar_tfull, 1);
        mbar_init(bar_tempty, 2 * EPI_WARPS);        // epilogue warps of both CTAs
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ producer ----
        if (lane == 0) {
            int s = 0;
            uint32_t phase = 0, issued_parity = 0, issued_any = 0;
            bool ok = true;
            const int rc_a_max = (p.M + 127) >> 7, rc_b_max = (p.N + 127) >> 7;
            for (int tile = cluster; tile < num_tiles && ok; tile += n_clusters) {
                int tm, tn;
                tile_coords(tile, p, tm, tn);
                const int m0 = tm * 256 + (int)rank * 128, n0 = tn * 256 + (int)rank * 128;
                const int rc_a = m0 >> 7, rc_b = (tn * 256) >> 7;
                const int has_a = rc_a < rc_a_max ? 1 : 0;
                const int nh = (rc_b + 1 < rc_b_max) ? 2 : 1;
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait_cluster(bar_empty + 8 * s, phase ^ 1, abort_flag)) { ok = false; break; }
                    const int nk = min(4, k_steps - kb * 4);
                    const uint32_t full = bar_full + 8 * s;
                    mbar_expect_tx(full, (uint32_t)(P_A_STAGE + P_B_STAGE + nk * 512 * (has_a + nh)));
                    tma_load_2d(sbase + P_OFF_A + s * P_A_STAGE, &map_a, full, kb * BKB, m0);
                    tma_load_2d(sbase + P_OFF_B + s * P_B_STAGE, &map_b, full, kb * BKB, n0);
                    if (has_a)
                        bulk_load(sbase + P_OFF_SFA + s * SFA_STAGE,
                                  p.sfa + ((int64_t)rc_a * p.chunks_k + kb * 4) * 512, nk * 512, full);
                    for (int h = 0; h < nh; ++h)
                        bulk_load(sbase + P_OFF_SFB + s * SFB_STAGE + h * 2048,
                                  p.sfb + ((int64_t)(rc_b + h) * p.chunks_k + kb * 4) * 512, nk * 512, full);
                    issued_any |= 1u << s;
                    issued_parity = (issued_parity & ~(1u << s)) | (phase << s);
                    if (++s == P_STAGES) { s = 0; phase ^= 1; }
                }
            }
            for (int st = 0; st < P_STAGES; ++st)
                if (issued_any & (1u << st)) {
                    const uint32_t par = (issued_parity >> st) & 1u;
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try(bar_full + 8 * st, par) && globaltimer() - t0 < kWaitLimitNs) {}
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA (CTA 0 of the pair) ----
        if (lane == 0 && rank == 0) {
            int s = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            const uint32_t idesc = kIdescPair | (MX ? kIdescUe8m0 : 0u);
            for (int tile = cluster; tile < num_tiles && ok; tile += n_clusters) {
                if (!mbar_wait_cluster(bar_tempty, acc_phase ^ 1, abort_flag)) break;
                tc_fence_after();
                for (int kb = 0; kb < k_blocks; ++kb) {
                    // raised by the scale warps of both CTAs once their own
                    // stage s had landed
                    if (!mbar_wait_cluster(bar_sf_full + 8 * s, phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const int nk = min(4, k_steps - kb * 4);
                    const uint32_t a_addr = sbase + P_OFF_A + s * P_A_STAGE;
                    const uint32_t b_addr = sbase + P_OFF_B + s * P_B_STAGE;
                    const uint32_t sfa_col = tmem + SF_COL + s * 48;
                    const uint32_t sfb_col = sfa_col + 16;
                    for (int j = 0; j < nk; ++j)
                        tc_mma_nvf4_pair(tmem + ACC_COL, desc_sw128(a_addr + j * 32), desc_sw128(b_addr + j * 32),
                                         idesc, sfa_col + 4 * j, sfb_col + 8 * j, (kb | j) != 0, MX);
                    tc_commit_pair(bar_empty + 8 * s);
                    if (++s == P_STAGES) { s = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit_pair(bar_tfull);
                acc_phase ^= 1;
            }
            tc_commit_pair(bar_drain);
        }
        // both CTAs, also after an abort: every MMA of the pair -- and with it
        // every commit CTA 0 multicasts to this CTA's barriers -- has completed
        // before shared memory and TMEM can be released
        if (lane == 0) {
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_cluster(bar_drain, 0) && globaltimer() - t0 < kWaitLimitNs) {}
        }
    } else if (warp < 6) {
        // -------------------------------------------------- scales -> TMEM ----
        // Warp q of this group owns TMEM lanes 32q..32q+31 (q = warp % 4) and
        // does nothing else, so the block scales of the next stages are in
        // tensor memory while the epilogue warps drain and store.
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        int s = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = cluster; tile < num_tiles && ok; tile += n_clusters) {
            for (int kb = 0; kb < k_blocks; ++kb) {
                if (!mbar_wait(bar_full + 8 * s, phase, abort_flag)) { ok = false; break; }
                const uint32_t sfa_s = sbase + P_OFF_SFA + s * SFA_STAGE + 16 * lane;
                const uint32_t sfb_s = sbase + P_OFF_SFB + s * SFB_STAGE + 16 * lane;
                uint32_t ra[16], rb0[16], rb1[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 va = lds128(sfa_s + j * 512);
                    ra[4 * j] = va.x; ra[4 * j + 1] = va.y; ra[4 * j + 2] = va.z; ra[4 * j + 3] = va.w;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint4 vb = lds128(sfb_s + h * 2048 + j * 512);
                        uint32_t* rb = j < 2 ? rb0 : rb1;
                        const int o = 8 * (j & 1) + 4 * h;
                        rb[o] = vb.x; rb[o + 1] = vb.y; rb[o + 2] = vb.z; rb[o + 3] = vb.w;
                    }
                }
                const uint32_t col = tmem + lane_base + SF_COL + s * 48;
                tc_st_32x32b_x16(col, ra);
                tc_st_32x32b_x16(col + 16, rb0);
                tc_st_32x32b_x16(col + 32, rb1);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0) mbar_arrive(bar_sf_full + 8 * s);
                    else mbar_arrive_cluster(bar_sf_full + 8 * s, 0);
                }
                if (++s == P_STAGES) { s = 0; phase ^= 1; }
            }
        }
    } else {
        // ----------------------------------------------------------- epilogue ----
        // warps 6..9: columns 0..127, warps 10..13: columns 128..255, of the
        // TMEM lane quarter warp % 4
        const int q = warp & 3, half = (warp - 6) >> 2;
        const float2 alpha = out_scales(p);
        const uint32_t buf = sbase + P_OFF_EPI + (warp - 6) * EPI_BUF;
        uint32_t acc_phase = 0;
        uint32_t amax_acc = 0;
        bool first = true;
        for (int tile = cluster; tile < num_tiles; tile += n_clusters)
            if (!epilogue_half_pair(p, tile, half, q, lane, rank, tmem, alpha, bar_tfull, bar_tempty, acc_phase,
                                    abort_flag, amax_acc, &map_c, buf, first)) break;
        if (lane == 0) bulk_wait0();    // every store of this warp has completed
        __syncwarp();
        if (p.c_amax) amax_publish(p.c_amax, amax_acc);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

// ------------------------------------------------------- wait self-test ----
// The failure path of every bounded wait, exercised without a fault: one
// thread waits on a barrier that nothing arrives on, with the caller's limit;
// when it runs out the kernel raises the device error word and returns.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns);
}

// ----------------------------------------------------------- host side -----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

bool make_code_map(CUtensorMap* m, const uint8_t* base, int64_t rows, int64_t k, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
    cuuint32_t box[2] = {(cuuint32_t)BKB, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_out_map(CUtensorMap* m, void* base, int64_t rows, int64_t cols, int64_t ldc, bool bf16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int esz = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ldc * esz)};
    cuuint32_t box[2] = {(cuuint32_t)(64 / esz), 32};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceInfo {
    int sms = 0;
    int pair_clusters = 0;   // co-resident CTA pairs of the 2-SM kernel
};

DeviceInfo device_info() {
    static DeviceInfo cached[64];
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    std::lock_guard<std::mutex> lock(mu);
    DeviceInfo& d = cached[dev];
    if (!d.sms) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        for (auto k : {gemm_nvf4_kernel<false>, gemm_nvf4_kernel<true>})
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        for (auto k : {gemm_nvf4_pair_kernel<false>, gemm_nvf4_pair_kernel<true>}) {
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_BYTES);
            cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (n / 2));
        cfg.blockDim = dim3(P_NUM_THREADS);
        cfg.dynamicSmemBytes = P_SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, gemm_nvf4_pair_kernel<false>, &cfg) != cudaSuccess ||
            clusters < 1) {
            cudaGetLastError();
            clusters = n / 2;
        }
        d.pair_clusters = clusters;
        d.sms = n > 0 ? n : 148;
    }
    return d;
}

int group_for(int64_t rows_per_tile, int64_t K, int tiles_m) {
    // group as many A panels (rows_per_tile x K/2 bytes each) as fit in ~24 MB of L2
    const int64_t panel = rows_per_tile * (K / 2);
    int64_t gm = (24ll << 20) / (panel > 0 ? panel : 1);
    if (gm < 1) gm = 1;
    if (gm > tiles_m) gm = tiles_m;
    return (int)gm;
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s) {
    const DeviceInfo dev = device_info();
    KParams p{};
    p.sfa = g.sfa;
    p.sfb = g.sfb;
    p.a_gs = g.a_gs;
    p.b_gs = g.b_gs;
    p.M = (int)g.M;
    p.N = (int)g.N;
    p.K = (int)g.K;
    p.chunks_k = (int)mma_chunks_k(g.K);
    p.out_bf16 = g.out_bf16;
    p.c = g.c;
    p.ldc = g.ldc;
    p.c_amax = reinterpret_cast<unsigned int*>(g.c_amax);
    p.mx = g.mx;
    p.tiles_n = (int)ceil_div(g.N, BN);
    // The CTA-pair kernel is the default: per SM it moves 38 KB instead of
    // 54 KB from L2 per 256-wide K block.  NVFP4_GEMM_PAIR=0 selects the
    // single-SM kernel, as does a device on which no pair can be co-resident.
    const char* pair = getenv("NVFP4_GEMM_PAIR");
    if ((pair && pair[0] == '0') || dev.pair_clusters < 1) {
        CUtensorMap ma, mb;
        if (!make_code_map(&ma, g.a, g.M, g.K, BM) || !make_code_map(&mb, g.b, g.N, g.K, BN))
            return cudaErrorInvalidValue;
        p.tiles_m = (int)ceil_div(g.M, BM);
        p.group_m = group_for(BM, g.K, p.tiles_m);
        const int tiles = p.tiles_m * p.tiles_n;
        const int grid = tiles < dev.sms ? tiles : dev.sms;
        if (p.mx) gemm_nvf4_kernel<true><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ma, mb, p);
        else gemm_nvf4_kernel<false><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ma, mb, p);
        return cudaGetLastError();
    }
    // CTA pairs: 256 x 256 tiles, each CTA loads 128-row boxes of A and B
    CUtensorMap ma, mb, mc;
    if (!make_code_map(&ma, g.a, g.M, g.K, 128) || !make_code_map(&mb, g.b, g.N, g.K, 128) ||
        !make_out_map(&mc, g.c, g.M, g.N, g.ldc, g.out_bf16 != 0))
        return cudaErrorInvalidValue;
    p.tiles_m = (int)ceil_div(g.M, 256);
    p.group_m = group_for(256, g.K, p.tiles_m);
    const int tiles = p.tiles_m * p.tiles_n;
    const int clusters = tiles < dev.pair_clusters ? tiles : dev.pair_clusters;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(P_NUM_THREADS);
    cfg.dynamicSmemBytes = P_SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return p.mx ? cudaLaunchKernelEx(&cfg, gemm_nvf4_pair_kernel<true>, ma, mb, mc, p)
                : cudaLaunchKernelEx(&cfg, gemm_nvf4_pair_kernel<false>, ma, mb, mc, p);
}

unsigned int read_and_clear_error_word(cudaStream_t s, cudaError_t* err) {
    *err = cudaStreamSynchronize(s);
    if (*err != cudaSuccess) return 0;
    unsigned int w = 0;
    *err = cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w));
    if (*err != cudaSuccess) return 0;
    const unsigned int zero = 0;
    *err = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    return w;
}

cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t s) {
    wait_selftest_kernel<<<1, 32, 0, s>>>(limit_ns);
    return cudaGetLastError();
}

}  // namespace nvfp4
