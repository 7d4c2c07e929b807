// coli_prefill.cuh -- expert phases for prefill batches: int4-dequant grouped GEMM
// on the 5th-generation tensor cores (tcgen05.mma, operands and accumulators in TMEM).
//
// The pages compute batched prefill with an int4 kernel and single-token
// decode in f32 ("Colibri 完全ガイド", section 詳細解説 step 3); with hundreds of
// tokens per expert the expert FFN is a dense contraction, so it runs on the
// tensor cores here.  Weights are int4 with one fp32 scale per 64 along K
// ("gs64 build", "colibri: 744B MoEをストレージから推論するCエンジン").
//
// Work item = one weight tile (128 rows) x one token tile (a union group of
// <= kPfMaxN pairs of one expert, N padded to 16):  D[128, N] = W[128, K] . X[N, K]^T.
// Persistent CTAs (one per SM) walk the items; inside a CTA, warp roles:
//   warp 0     TMA producer: int4 bytes + scales of the weight tile, 256 K at a
//              time (3-deep ring), and the token rows (bf16), 64 K at a time
//              (6-deep ring), straight into the 128-byte-swizzled layouts;
//   warps 6..  dequantise: each thread owns one weight row (= TMEM lane) and
//              a part of a 64-K step; q * s is formed in bf16 and written into a
//              4-deep ring of A operands in TMEM with tcgen05.st;
//   warp 1     one thread issues tcgen05.mma (A from TMEM, B from shared memory,
//              M 128, K 16, fp32 accumulate) into one of two TMEM accumulators;
//   warps 2-5  epilogue: tcgen05.ld of the finished accumulator while the next
//              item accumulates into the other one.  The gate/up GEMM applies
//              SwiGLU (tile rows 0-63 are gate rows, 64-127 the matching up
//              rows); the down GEMM scales by the routing weight and writes one
//              bf16 row per (token, slot), summed later in slot order.
//
// K order inside the MMA.  A dequantised register holds the nibbles m and m + 4
// of a 32-bit word of int4 (bits 4m and 4m + 16), so MMA K position p of each
// group of 8 carries k = sigma(p), sigma = (0, 4, 1, 5, 2, 6, 3, 7).  The token
// rows (gathered activations, and the SwiGLU output h that the down GEMM reads)
// are stored in the same permuted order, so every dot product is unchanged.
//
// Every wait on an mbarrier is bounded in time; a timeout sets an error word and
// every role winds down (in-flight copies land, TMEM is freed) instead of hanging.
#pragma once

#include <cuda.h>  // CUtensorMap (type only; maps are encoded on the host)

#include "coli_common.cuh"

namespace coli {

constexpr int kPfMaxN = 192;      // tokens per tile (union group size on this path)
constexpr int kPfKStep = 64;      // K per MMA stage = one scale group
constexpr int kPfRawK = 256;      // K per int4 stage
constexpr int kPfRawStages = 3;
constexpr int kPfBStages = 6;
constexpr int kPfAStages = 4;     // dequantised weight stages in TMEM, 32 columns each
constexpr int kPfTmemCols = 512;
constexpr int kPfACol = 2 * kPfMaxN;  // columns [0, 2 N_max): two accumulators; then the A ring
constexpr int kPfBRows = 32;          // token rows per TMA box
constexpr int kPfBStageBytes = kPfMaxN * 128;
constexpr int kPfRawHalfBytes = 64 * kPfRawK / 2;             // int4 bytes of 64 rows
constexpr int kPfRawScaleOff = 2 * kPfRawHalfBytes;          // then 2 x 64 rows x 4 scales
constexpr int kPfRawStageBytes = kPfRawScaleOff + 2 * 64 * 16;
constexpr int kPfXchFloats = 64 * 17;                        // gate/up exchange, one buffer
#ifndef COLI_PF_DEQ_WARPS
#define COLI_PF_DEQ_WARPS 8
#endif
constexpr int kPfDeqWarps = COLI_PF_DEQ_WARPS;   // 8 or 16: each takes 64 / (warps / 4) K of a step
constexpr int kPfDeqParts = kPfDeqWarps / 4;     // warps per TMEM lane quadrant
constexpr int kPfDeqK = kPfKStep / kPfDeqParts;  // K values per dequant thread per step
constexpr int kPfWarpMma = 1, kPfWarpEpi = 2, kPfWarpDeq = 6, kPfWarpEnd = 6 + kPfDeqWarps;
constexpr int kPfThreads = kPfWarpEnd * 32;
constexpr size_t kPfSmemBytes = 1024 /*alignment slack*/ + (size_t)kPfBStages * kPfBStageBytes +
                                (size_t)kPfRawStages * kPfRawStageBytes + 2 * kPfXchFloats * 4 + 2 * kPfMaxN * 4;
constexpr unsigned long long kPfWaitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait
constexpr unsigned long long kPfDrainNs = 100000000ull;  // teardown waits

static_assert(kPfACol + kPfAStages * 32 <= kPfTmemCols, "TMEM budget");
static_assert(kPfDeqWarps == 8 || kPfDeqWarps == 16, "dequant split");
static_assert(kPfMaxN % kPfBRows == 0 && kPfMaxN % 16 == 0 && kPfMaxN <= 256, "tile width");
static_assert(kPfBStageBytes % 1024 == 0 && kPfRawStageBytes % 1024 == 0, "swizzled stages stay 1024-aligned");

// ---------------------------------------------------------------------------
// PTX wrappers


__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Arrive once and add `bytes` to the transaction count of the current phase.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Same, but the thread may be suspended (issuing nothing) until the phase
// completes or about `hint_ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false after the
// deadline (error word set).  Waiting threads sleep in the barrier instead of
// spinning, so they take no issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned long long deadline, int* err)
{
    if (mbar_try_wait(bar, parity)) return true;
    while (!mbar_try_wait_sleep(bar, parity, 1000000u)) {
        if (global_ns() > deadline) {
            atomicExch(err, 1);
            return false;
        }
    }
    return true;
}

// 2-D tiled TMA load into this CTA's shared memory; completion is counted in
// bytes on the mbarrier.  x is the innermost coordinate (elements).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Named barrier 1 over the 4 epilogue warps; returns the AND of `pred` over them.
__device__ __forceinline__ bool epi_bar_and(bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void epi_bar() { asm volatile("barrier.cta.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[tmem] . B[smem descriptor]^T
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Store NC (8 or 16) consecutive 32-bit TMEM columns of this thread's lane
// (asynchronous: tmem_wait_st() waits for all of this thread's stores).
template <int NC>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&r)[NC])
{
    if constexpr (NC == 16) {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::
                "r"(taddr),
            "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
            "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
            : "memory");
    } else {
        static_assert(NC == 8, "8 or 16 columns");
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                     "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                     : "memory");
    }
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128 bytes,
// 8-row groups 1024 bytes apart (tcgen05 descriptor version 1).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);  // start address
    d |= (uint64_t)1 << 16;                  // leading byte offset (16 B units; unused when swizzled)
    d |= (uint64_t)(1024 >> 4) << 32;        // stride byte offset
    d |= (uint64_t)1 << 46;                  // version
    d |= (uint64_t)2 << 61;                  // SWIZZLE_128B
    return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, both K-major, M = 128.
__device__ __forceinline__ uint32_t idesc_bf16(int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

// 8 * NW int4 weights (NW 32-bit words, low nibble first) of one row -> 4 * NW
// bf16x2 words of q * s.  Word 4i + m holds (nibble m, nibble m + 4) of 32-bit
// word i: the mask picks bits 0-3 and 16-19 after a shift by 4m, and the xor
// makes each half the bf16 number 128 + (nibble ^ 8) = 136 + q (exponent 2^7:
// one unit per step).  q = v - 136 is exact; q * bf16(s) is rounded once to bf16.
template <int NW>
__device__ __forceinline__ void dequant_words(const uint32_t (&words)[NW], float s, uint32_t (&o)[4 * NW])
{
    const __nv_bfloat162 s2 = __float2bfloat162_rn(s);
    const __nv_bfloat162 c136 = __float2bfloat162_rn(136.f);
#pragma unroll
    for (int i = 0; i < NW; ++i) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint32_t v;
            asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(v) : "r"(words[i] >> (4 * m)), "r"(0x000F000Fu), "r"(0x43084308u));
            const __nv_bfloat162 q = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&v), c136);
            o[4 * i + m] = bf16x2_bits(__hmul2(q, s2));
        }
    }
}

// Stored position of feature f in a permuted token row: inverse of sigma inside
// each group of 8.
__host__ __device__ __forceinline__ int pf_store_pos(int f)
{
    const int m = f & 7;
    return (f & ~7) | (m < 4 ? 2 * m : 2 * (m - 4) + 1);
}

struct PrefillArgs {
    int NW;        // weight rows of one matrix: F (gate/up) or H (down)
    int K;         // reduction length: H (gate/up) or F (down)
    int k, P;      // top-k, routed pairs T * k
    int n_mtiles;  // weight tiles per token tile: F / 64 (gate/up) or H / 128 (down)
    const int32_t* ctl;       // ctl[0] = number of token tiles
    const int32_t* g_expert;  // token tiles (union groups of <= kPfMaxN pairs)
    const int32_t* g_start;
    const int32_t* g_count;
    const int32_t* perm;      // pair id of each sorted position (slot = id % k)
    const float* pair_w;      // routing weight of each sorted position (1 for shared)
    uint16_t* h;              // gate/up out: bf16 [P + T, F], permuted rows
    uint16_t* ys;             // down out: bf16 [T, k + 1, H]
    int* err;
    unsigned long long wait_ns;  // limit of every pipeline wait (teardown drains keep their own)
};

// tq0 / tq1: int4 bytes of tile rows 0-63 / 64-127 (box 128 B x 64 rows, 128-byte
// swizzle); ts0 / ts1: their scales (box 4 x 64); tb: token rows, bf16 [P + T, K]
// permuted (box 64 x 32, 128-byte swizzle).
template <bool kGemm1>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_gemm_kernel(const __grid_constant__ CUtensorMap tq0, const __grid_constant__ CUtensorMap tq1,
                    const __grid_constant__ CUtensorMap ts0, const __grid_constant__ CUtensorMap ts1,
                    const __grid_constant__ CUtensorMap tb, const PrefillArgs a)
{
    extern __shared__ __align__(16) unsigned char pf_smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(pf_smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char* bring = smem;
    unsigned char* rring = bring + (size_t)kPfBStages * kPfBStageBytes;
    float* xch = reinterpret_cast<float*>(rring + (size_t)kPfRawStages * kPfRawStageBytes);
    int* s_dst = reinterpret_cast<int*>(xch + 2 * kPfXchFloats);
    float* s_w = reinterpret_cast<float*>(s_dst + kPfMaxN);

    __shared__ uint64_t raw_full[kPfRawStages], raw_empty[kPfRawStages], b_full[kPfBStages], b_empty[kPfBStages];
    __shared__ uint64_t a_full[kPfAStages], a_empty[kPfAStages], acc_full[2], acc_empty[2], done_bar;
    __shared__ uint32_t tmem_base;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = a.ctl[0] * a.n_mtiles;
    const int ksteps = a.K / kPfKStep;
    const int rsteps = a.K / kPfRawK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kPfRawStages; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], kPfDeqWarps);  // one arrival per dequant warp
        }
        for (int i = 0; i < kPfBStages; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], 1);
        }
        for (int i = 0; i < kPfAStages; ++i) {
            mbar_init(&a_full[i], kPfDeqWarps);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);  // one arrival per epilogue warp
        }
        mbar_init(&done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kPfWarpMma) tmem_alloc(&tmem_base, kPfTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const unsigned long long deadline = global_ns() + a.wait_ns;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            tma_prefetch_map(&tq0);
            tma_prefetch_map(&tq1);
            tma_prefetch_map(&ts0);
            tma_prefetch_map(&ts1);
            tma_prefetch_map(&tb);
            int kb = 0, kr = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                const int tile = it / a.n_mtiles, mt = it - tile * a.n_mtiles;
                const int e = a.g_expert[tile], start = a.g_start[tile], count = a.g_count[tile];
                const int nbox = (count + kPfBRows - 1) / kPfBRows;
                const int r0 = kGemm1 ? e * a.NW + mt * 64 : e * a.NW + mt * 128;
                const int r1 = kGemm1 ? r0 : r0 + 64;
                for (int j = 0; j < rsteps && ok; ++j) {
                    const int sr = kr % kPfRawStages;
                    if (kr >= kPfRawStages) ok = mbar_wait(&raw_empty[sr], ((kr / kPfRawStages) - 1) & 1, deadline, a.err);
                    if (!ok) break;
                    unsigned char* st = rring + (size_t)sr * kPfRawStageBytes;
                    mbar_expect_tx(&raw_full[sr], kPfRawStageBytes);
                    tma_load_2d(st, &tq0, j * (kPfRawK / 2), r0, &raw_full[sr]);
                    tma_load_2d(st + kPfRawHalfBytes, &tq1, j * (kPfRawK / 2), r1, &raw_full[sr]);
                    tma_load_2d(st + kPfRawScaleOff, &ts0, j * (kPfRawK / kGroup), r0, &raw_full[sr]);
                    tma_load_2d(st + kPfRawScaleOff + 64 * 16, &ts1, j * (kPfRawK / kGroup), r1, &raw_full[sr]);
                    ++kr;
                    for (int s = 0; s < kPfRawK / kPfKStep; ++s) {
                        const int sb = kb % kPfBStages;
                        if (kb >= kPfBStages) ok = mbar_wait(&b_empty[sb], ((kb / kPfBStages) - 1) & 1, deadline, a.err);
                        if (!ok) break;
                        unsigned char* bs = bring + (size_t)sb * kPfBStageBytes;
                        mbar_expect_tx(&b_full[sb], nbox * kPfBRows * 128);
                        const int kx = (j * (kPfRawK / kPfKStep) + s) * kPfKStep;
                        for (int i = 0; i < nbox; ++i)
                            tma_load_2d(bs + i * kPfBRows * 128, &tb, kx, start + kPfBRows * i, &b_full[sb]);
                        ++kb;
                    }
                }
            }
            // Let every issued copy land before the CTA can retire (normally long done).
            const unsigned long long drain = global_ns() + kPfDrainNs;
            for (int s = 0; s < kPfBStages && s < kb; ++s) {
                const int last = kb - 1 - ((kb - 1 - s) % kPfBStages);
                mbar_wait(&b_full[s], (last / kPfBStages) & 1, drain, a.err);
            }
            for (int s = 0; s < kPfRawStages && s < kr; ++s) {
                const int last = kr - 1 - ((kr - 1 - s) % kPfRawStages);
                mbar_wait(&raw_full[s], (last / kPfRawStages) & 1, drain, a.err);
            }
        }
    } else if (warp == kPfWarpMma) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int kg = 0, kb = 0, local = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++local) {
                const int tile = it / a.n_mtiles;
                const int N = (a.g_count[tile] + 15) & ~15;
                const uint32_t idesc = idesc_bf16(N);
                const int ab = local & 1, use = local >> 1;
                if (use > 0) {
                    ok = mbar_wait(&acc_empty[ab], (use - 1) & 1, deadline, a.err);
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t d = tmem + (uint32_t)(ab * kPfMaxN);
                for (int ks = 0; ks < ksteps; ++ks) {
                    const int sa = kg % kPfAStages, sb = kb % kPfBStages;
                    ok = mbar_wait(&a_full[sa], (kg / kPfAStages) & 1, deadline, a.err) &&
                         mbar_wait(&b_full[sb], (kb / kPfBStages) & 1, deadline, a.err);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t bbase = smem_u32(bring + (size_t)sb * kPfBStageBytes);
                    const uint32_t acol = tmem + (uint32_t)(kPfACol + sa * 32);
#pragma unroll
                    for (int kk = 0; kk < kPfKStep / 16; ++kk)
                        tc_mma_ts(d, acol + kk * 8, smem_desc_sw128(bbase + kk * 32), idesc, (ks | kk) != 0);
                    tc_commit(&a_empty[sa]);
                    tc_commit(&b_empty[sb]);
                    ++kg;
                    ++kb;
                }
                if (!ok) break;
                tc_commit(&acc_full[ab]);
            }
            tc_commit(&done_bar);  // every MMA issued above completes before TMEM is freed
        }
    } else if (warp < kPfWarpDeq) {
        // ---------------- epilogue (warps 2-5: TMEM lane quadrants 2, 3, 0, 1) ----------------
        const int qd = warp & 3, row = qd * 32 + lane, et = threadIdx.x - kPfWarpEpi * 32;
        int local = 0;
        for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++local) {
            const int tile = it / a.n_mtiles, mt = it - tile * a.n_mtiles;
            const int start = a.g_start[tile], count = a.g_count[tile];
            const int ab = local & 1;
            if (!kGemm1) {
                epi_bar();  // the previous item's readers are done with s_dst / s_w
                for (int c = et; c < count; c += 128) {
                    const int pos = start + c;
                    int t, slot;
                    if (pos < a.P) {
                        const int pid = a.perm[pos];
                        t = pid / a.k;
                        slot = pid - t * a.k;
                    } else {
                        t = pos - a.P;
                        slot = a.k;
                    }
                    // destination row of ys [T, k+1, H]; the bounds-checked build parks a bad one on row 0
                    const int dst = t * (a.k + 1) + slot;
                    s_dst[c] = COLI_IN_BOUNDS(t >= 0 && slot >= 0 && slot <= a.k && (pos >= a.P || t < a.P / a.k),
                                              a.err) ? dst : 0;
                    s_w[c] = a.pair_w[pos];
                }
            }
            const bool got = mbar_wait(&acc_full[ab], (local >> 1) & 1, deadline, a.err);
            if (!epi_bar_and(__all_sync(0xFFFFFFFFu, got))) break;  // uniform over the 4 warps
            tc_fence_after();
            const uint32_t tacc = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(ab * kPfMaxN);
            const int n16 = (count + 15) & ~15;
            for (int c0 = 0, ch = 0; c0 < n16; c0 += 16, ++ch) {
                float v[16];
                tmem_ld16(tacc + c0, v);
                if (kGemm1) {
                    float* xb = xch + (ch & 1) * kPfXchFloats;
                    if (qd >= 2) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) xb[(row - 64) * 17 + i] = v[i];
                    }
                    epi_bar();
                    if (qd < 2) {
                        const int fs = pf_store_pos(mt * 64 + row);
                        uint16_t* hp = a.h + (size_t)(start + c0) * a.NW + fs;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            if (c0 + i < count) {
                                const float g = v[i], u = xb[row * 17 + i];
                                hp[(size_t)i * a.NW] = float_to_bf16_bits(g / (1.0f + expf(-g)) * u);
                            }
                        }
                    }
                } else {
                    uint16_t* yp = a.ys + mt * 128 + row;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (c0 + i < count)
                            yp[(size_t)s_dst[c0 + i] * a.NW] = float_to_bf16_bits(s_w[c0 + i] * v[i]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
    } else if (warp < kPfWarpEnd) {
        // ---------------- dequantise (warps 6 ..) ----------------
        // One flat sequence over this CTA's k-steps (K is a multiple of the int4
        // stage, so stage boundaries line up with items).  Software-pipelined:
        // the TMEM store of step n is in flight while step n + 1 is read and
        // dequantised.
        constexpr int kWords = kPfDeqK / 8;  // 32-bit words of int4 per thread and step
        constexpr int kSubs = kPfRawK / kPfKStep;
        const int qd = warp & 3, part = (warp - kPfWarpDeq) >> 2;
        const int row = qd * 32 + lane, box = row >> 6, rr = row & 63;
        const uint32_t tlane = (uint32_t)(qd * 32) << 16;
        const int my_items = n_items > (int)blockIdx.x ? (n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
        const int total = my_items * ksteps;
        uint32_t words[kWords];
        float scale = 0.f;
        // int4 words and scale of step n (waits for its stage; frees the stage after its last step)
        auto load = [&](int n) -> bool {
            const int sub = n % kSubs, kr = n / kSubs, sr = kr % kPfRawStages;
            bool ok = true;
            if (sub == 0) ok = mbar_wait(&raw_full[sr], (kr / kPfRawStages) & 1, deadline, a.err);
            if (!__all_sync(0xFFFFFFFFu, ok)) return false;
            const unsigned char* st = rring + (size_t)sr * kPfRawStageBytes;
            // this thread's bytes: K [sub * 64 + part * kPfDeqK, + kPfDeqK) of the stage
            const int byte0 = sub * 32 + part * (kPfDeqK / 2);
            const int c = byte0 >> 4;  // 16-byte chunk of the 128-byte row
            const unsigned char* src = st + box * kPfRawHalfBytes + rr * 128 + ((c ^ (rr & 7)) << 4) + (byte0 & 15);
            if constexpr (kWords == 4) {
                const uint4 w = *reinterpret_cast<const uint4*>(src);
                words[0] = w.x, words[1] = w.y, words[2] = w.z, words[3] = w.w;
            } else {
                const uint2 w = *reinterpret_cast<const uint2*>(src);
                words[0] = w.x, words[1] = w.y;
            }
            scale = *reinterpret_cast<const float*>(st + kPfRawScaleOff + box * 64 * 16 + rr * 16 + sub * 4);
            if (sub == kSubs - 1) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&raw_empty[sr]);
            }
            return true;
        };
        uint32_t o[4 * kWords];
        bool ok = total > 0 && load(0);
        if (ok) dequant_words<kWords>(words, scale, o);
        for (int n = 0; n < total && ok; ++n) {
            const int sa = n % kPfAStages;
            bool got = true;
            if (n >= kPfAStages) got = mbar_wait(&a_empty[sa], ((n / kPfAStages) - 1) & 1, deadline, a.err);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            tc_fence_after();
            tmem_st<4 * kWords>(tmem + tlane + (uint32_t)(kPfACol + sa * 32 + part * (kPfDeqK / 2)), o);
            if (n + 1 < total) {
                ok = load(n + 1);
                if (ok) dequant_words<kWords>(words, scale, o);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[sa]);
        }
    }

    __syncthreads();
    if (warp == kPfWarpMma) {
        if (lane == 0) mbar_wait(&done_bar, 0, global_ns() + kPfDrainNs, a.err);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kPfTmemCols);
    }
}

// Token rows of every sorted position, bf16, in the permuted K order:
// xg[pos, 8g + p] = x[pair_token[pos], 8g + sigma(p)].
template <bool kXBf16>
__global__ void prefill_gather_kernel(const void* __restrict__ x, const int32_t* __restrict__ pair_token, int Q,
                                      int T, int H, uint16_t* __restrict__ xg)
{
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int g8 = H / 8;
    if (i >= (size_t)Q * g8) return;
    const int pos = (int)(i / g8), g = (int)(i - (size_t)pos * g8);
    int t = pair_token[pos];
    if (!COLI_IN_BOUNDS(t >= 0 && t < T, nullptr)) t = 0;
    float v[8];
    if constexpr (kXBf16) {
        const uint4 r = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + (size_t)t * H + 8 * g);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[2 * j] = bf16_bits_to_float(w[j] & 0xFFFFu);
            v[2 * j + 1] = bf16_bits_to_float(w[j] >> 16);
        }
    } else {
        const float* src = static_cast<const float*>(x) + (size_t)t * H + 8 * g;
        const float4 a0 = *reinterpret_cast<const float4*>(src), a1 = *reinterpret_cast<const float4*>(src + 4);
        v[0] = a0.x, v[1] = a0.y, v[2] = a0.z, v[3] = a0.w, v[4] = a1.x, v[5] = a1.y, v[6] = a1.z, v[7] = a1.w;
    }
    uint32_t o[4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
        o[m] = (uint32_t)float_to_bf16_bits(v[m]) | ((uint32_t)float_to_bf16_bits(v[m + 4]) << 16);
    *reinterpret_cast<uint4*>(xg + (size_t)pos * H + 8 * g) = make_uint4(o[0], o[1], o[2], o[3]);
}

// out[t, n] = sum over slots j (routed in slot order, shared last) of ys[t, j, n].
// Slots whose routing index is -1 (dropped by adaptive top-p) were never written and are skipped.
template <bool kOutBf16>
__global__ void slot_reduce_kernel(const uint16_t* __restrict__ ys, int T, int S, int H,
                                   const int32_t* __restrict__ topk_idx, void* __restrict__ out)
{
    const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;  // 8 outputs per thread
    if (i >= (size_t)T * H) return;
    const size_t t = i / H, n = i - t * H;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < S; ++j) {
        if (j < S - 1 && topk_idx[t * (S - 1) + j] < 0) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(ys + ((size_t)t * S + j) * H + n);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            acc[2 * p] += bf16_bits_to_float(w[p] & 0xFFFFu);
            acc[2 * p + 1] += bf16_bits_to_float(w[p] >> 16);
        }
    }
    if constexpr (kOutBf16) {
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p)
            o[p] = (uint32_t)float_to_bf16_bits(acc[2 * p]) | ((uint32_t)float_to_bf16_bits(acc[2 * p + 1]) << 16);
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + i) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
        float* o = static_cast<float*>(out) + i;
        *reinterpret_cast<float4*>(o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(o + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

}  // namespace coli
