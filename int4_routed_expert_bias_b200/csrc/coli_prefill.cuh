// coli_prefill.cuh -- expert phases for prefill batches: int4-dequant grouped GEMM
// on the 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM).
//
// The pages compute batched prefill with an int4 kernel and single-token
// decode in f32 ("Colibri 完全ガイド", section 詳細解説 step 3); with hundreds of
// tokens per expert the expert FFN is a dense contraction, so it runs on the
// tensor cores here.  Weights are int4 with one fp32 scale per 64 along K
// ("gs64 build", "colibri: 744B MoEをストレージから推論するCエンジン").
//
// One CTA computes one tile D[128 weight rows, N tokens] = W[128, K] . X[N, K]^T
// for one token tile of one expert (a union group of <= 256 tokens, N padded
// to a multiple of 16):
//   - 8 producer warps stage, per K-step of 64, the int4 bytes and scales of the
//     128 weight rows and the N token rows (bf16) with cp.async, S stages ahead;
//     the token rows land directly in the 128-byte-swizzled K-major layout the
//     MMA reads; the int4 bytes are dequantised to bf16 (q * scale) into the
//     same layout;
//   - one thread of a 9th warp issues tcgen05.mma (M 128, N, K 16, bf16 in,
//     fp32 accumulate in TMEM) and tcgen05.commit frees each stage;
//   - after the last K-step the first four warps read the accumulator with
//     tcgen05.ld and write the tile: the gate/up GEMM applies SwiGLU (gate and
//     up rows are interleaved in 32-row blocks of the weight tile); the down
//     GEMM multiplies by the routing weight and writes one bf16 row per (token,
//     slot), summed later in slot order (deterministic combine).
// Every wait on an mbarrier is bounded in time; a timeout sets an error word
// and the CTA winds down (frees its TMEM) instead of hanging.
#pragma once

#include "coli_common.cuh"
#include "coli_int4.cuh"

namespace coli {

constexpr int kPfStages = 3;    // MMA stages (bf16 weights + token rows)
constexpr int kPfRawStages = 8; // int4 byte stages (issued kPfRawStages - 1 k-steps ahead)
constexpr int kPfProducers = 256;            // 8 producer warps
constexpr int kPfThreads = kPfProducers + 32;  // + the MMA warp
constexpr int kPfMaxN = 256;                 // tokens per tile
constexpr int kPfTmemCols = 256;
constexpr int kPfKStep = 64;                 // = one scale group
constexpr int kPfABytes = 128 * 128;         // 128 rows x 64 bf16
constexpr int kPfBBytes = kPfMaxN * 128;     // 256 rows x 64 bf16
constexpr int kPfRawBytes = 128 * 32 + 128 * 2 * 4;  // int4 bytes + two copies of the scale per row
constexpr int kPfStageBytes = kPfABytes + kPfBBytes;
constexpr size_t kPfSmemBytes =
    1024 /*alignment slack*/ + (size_t)kPfStages * kPfStageBytes + (size_t)kPfRawStages * kPfRawBytes + 256;
constexpr unsigned long long kPfWaitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait

// ---------------------------------------------------------------------------
// PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

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

// Wait for the given phase parity; false after the deadline (error word set).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned long long deadline, int* err)
{
    if (mbar_try_wait(bar, parity)) return true;
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() > deadline) {
            atomicExch(err, 1);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// The mbarrier receives one arrival when all earlier cp.async of this thread land.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
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

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128 bytes,
// 8-row groups 1024 bytes apart (tcgen05 descriptor version 1).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);  // start address
    d |= (uint64_t)1 << 16;                  // leading byte offset (16 B units)
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

// bf16 bit pattern of q * s for 32 nibbles (16 bytes) of one row.
__device__ __forceinline__ uint32_t bf16x2_of(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

struct PrefillArgs {
    const uint8_t* q0;  // gate (GEMM1) or down (GEMM2) bytes [E+1, N_w, K/2]
    const float* s0;
    const uint8_t* q1;  // up bytes (GEMM1)
    const float* s1;
    int NW;             // weight rows of one matrix: F (GEMM1: gate and up each) or H (GEMM2)
    int K;              // H (GEMM1) or F (GEMM2)
    int E, k, T, P;
    const void* act;    // GEMM1: x [T, H] (fp32 or bf16); GEMM2: h bf16 [P+T, F]
    const int32_t* ctl;       // ctl[0] = number of token tiles
    const int32_t* g_expert;  // token tiles (union groups of <= 256 pairs)
    const int32_t* g_start;
    const int32_t* g_count;
    const int32_t* pair_token;
    const float* pair_w;
    const int32_t* perm;      // pair id of each sorted position (slot = id % k)
    uint16_t* h;              // GEMM1 out: h bf16 [P+T, F]
    uint16_t* ys;             // GEMM2 out: bf16 [T, k+1, H]
    int* err;
};

template <bool kGemm1, bool kXBf16>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_gemm_kernel(PrefillArgs a)
{
    extern __shared__ __align__(16) unsigned char pf_smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(pf_smem_raw) + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full_bar[kPfStages], empty_bar[kPfStages], acc_bar;
    __shared__ uint32_t tmem_base;
    __shared__ int s_tok[kPfMaxN];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_mtiles = kGemm1 ? (2 * a.NW) / 128 : a.NW / 128;
    const int tile = blockIdx.x / n_mtiles, mt = blockIdx.x - tile * n_mtiles;
    if (tile >= a.ctl[0]) return;  // uniform across the CTA
    const int e = a.g_expert[tile], start = a.g_start[tile], count = a.g_count[tile];
    const int N = (count + 15) & ~15;
    const int ksteps = a.K / kPfKStep;

    if (tid < kPfMaxN) s_tok[tid] = tid < count ? (kGemm1 ? a.pair_token[start + tid] : start + tid) : -1;
    if (tid == 0) {
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(&full_bar[s], 2 * kPfProducers);  // per producer: A arrive + B arrive
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&acc_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 8) tmem_alloc(&tmem_base, kPfTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const unsigned long long deadline = global_ns() + kPfWaitNs;

    auto stage_a = [&](int s) { return smem + (size_t)s * kPfStageBytes; };
    auto stage_b = [&](int s) { return smem + (size_t)s * kPfStageBytes + kPfABytes; };
    auto stage_raw = [&](int r) { return smem + (size_t)kPfStages * kPfStageBytes + (size_t)r * kPfRawBytes; };

    if (warp < 8) {
        // ---------------- producers ----------------
        const int row = tid >> 1, half = tid & 1;  // A: one 16-byte half-row of int4 per thread
        // weight row of this thread in the tile
        const uint8_t* qrow;
        const float* srow;
        if (kGemm1) {
            // rows 0-31 gate n0.., 32-63 up n0.., 64-95 gate n0+32.., 96-127 up n0+32..
            const int n = mt * 64 + (row >> 6) * 32 + (row & 31);
            const bool up = (row >> 5) & 1;
            const size_t r = (size_t)e * a.NW + n;
            qrow = (up ? a.q1 : a.q0) + r * (a.K / 2);
            srow = (up ? a.s1 : a.s0) + r * (a.K / kGroup);
        } else {
            const size_t r = (size_t)e * a.NW + mt * 128 + row;
            qrow = a.q0 + r * (a.K / 2);
            srow = a.s0 + r * (a.K / kGroup);
        }
        const size_t act_row_bytes = (size_t)a.K * ((kGemm1 && !kXBf16) ? 4 : 2);
        bool ok = true;

        // int4 bytes and scales of k-step ks -> raw ring slot ks % kPfRawStages (own data of this thread)
        auto issue_raw = [&](int ks) {
            unsigned char* raw = stage_raw(ks % kPfRawStages);
            cp_async16(raw + row * 32 + half * 16, qrow + (size_t)ks * 32 + half * 16);
            cp_async4(raw + 128 * 32 + (row * 2 + half) * 4, srow + ks);
        };
        // token rows of k-step ks -> MMA stage ks % kPfStages; the stage's full barrier gets
        // this thread's arrival when its copies (and all earlier ones) have landed
        auto issue_b = [&](int ks) {
            const int s = ks % kPfStages;
            if (kGemm1 && !kXBf16) return;  // fp32 activations: converted while storing, below
            unsigned char* b = stage_b(s);
            for (int i = tid; i < N * 8; i += kPfProducers) {
                const int r = i >> 3, c = i & 7;
                const int src_row = s_tok[r] >= 0 ? s_tok[r] : s_tok[0];
                const unsigned char* src = static_cast<const unsigned char*>(a.act) + (size_t)src_row * act_row_bytes +
                                           (size_t)ks * 128 + c * 16;
                cp_async16(b + r * 128 + ((c ^ (r & 7)) * 16), src);
            }
        };

        // prologue: int4 bytes kPfRawStages - 1 k-steps ahead, token rows kPfStages - 1 ahead
        for (int ks = 0; ks < kPfRawStages - 1; ++ks) {
            if (ks < ksteps) issue_raw(ks);
            cp_async_commit();
        }
        for (int ks = 0; ks < kPfStages - 1 && ks < ksteps; ++ks) {
            issue_b(ks);
            if (kGemm1 && !kXBf16) mbar_arrive(&full_bar[ks % kPfStages]);
            else cp_async_arrive_noinc(&full_bar[ks % kPfStages]);
        }
        for (int ks = 0; ks < ksteps && ok; ++ks) {
            const int s = ks % kPfStages;
            // token rows for k-step ks + S - 1, once the MMA has released that stage
            const int kb = ks + kPfStages - 1;
            if (kb < ksteps) {
                const int sb = kb % kPfStages, fill = kb / kPfStages;
                if (fill > 0) ok = mbar_wait(&empty_bar[sb], (fill - 1) & 1, deadline, a.err);
                if (!ok) break;
                issue_b(kb);
                if (kGemm1 && !kXBf16) mbar_arrive(&full_bar[sb]);
                else cp_async_arrive_noinc(&full_bar[sb]);
            }
            // int4 bytes for k-step ks + R - 1 (its ring slot was consumed at k-step ks - 1)
            if (ks + kPfRawStages - 1 < ksteps) issue_raw(ks + kPfRawStages - 1);
            cp_async_commit();
            cp_async_wait<kPfRawStages - 1>();  // the group of k-step ks has landed
            unsigned char* raw = stage_raw(ks % kPfRawStages);
            const uint4 w = *reinterpret_cast<const uint4*>(raw + row * 32 + half * 16);
            const float sc = *reinterpret_cast<const float*>(raw + 128 * 32 + (row * 2 + half) * 4);
            unsigned char* A = stage_a(s);
            // q * s from the two mantissa windows (exact q; one fp32 rounding, then bf16)
            const float s16 = 16.f * sc, m24 = -24.f * sc, s256 = 256.f * sc, m264 = -264.f * sc;
            const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {  // 8 values per 16-byte chunk of the bf16 row
                const uint32_t wd = words[c4], tt = wd >> 12;
                const uint32_t sh[4] = {wd << 15, wd << 7, tt << 11, tt << 3};
                uint32_t o[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 f = nib_pair(sh[p]);  // (odd k, even k) of the pair
                    o[p] = bf16x2_of(fmaf(f.y, s256, m264), fmaf(f.x, s16, m24));
                }
                const int c = half * 4 + c4;
                *reinterpret_cast<uint4*>(A + row * 128 + ((c ^ (row & 7)) * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            if (kGemm1 && !kXBf16) {
                unsigned char* b = stage_b(s);
                for (int i = tid; i < N * 8; i += kPfProducers) {
                    const int r = i >> 3, c = i & 7;
                    const int src_row = s_tok[r] >= 0 ? s_tok[r] : s_tok[0];
                    const float* src = reinterpret_cast<const float*>(static_cast<const unsigned char*>(a.act) +
                                                                      (size_t)src_row * act_row_bytes) +
                                       (size_t)ks * 64 + c * 8;
                    const float4 v0 = *reinterpret_cast<const float4*>(src);
                    const float4 v1 = *reinterpret_cast<const float4*>(src + 4);
                    *reinterpret_cast<uint4*>(b + r * 128 + ((c ^ (r & 7)) * 16)) =
                        make_uint4(bf16x2_of(v0.x, v0.y), bf16x2_of(v0.z, v0.w), bf16x2_of(v1.x, v1.y),
                                   bf16x2_of(v1.z, v1.w));
                }
            }
            fence_proxy_async();
            mbar_arrive(&full_bar[s]);
        }
        cp_async_wait<0>();

        // ---------------- epilogue (warps 0-3: TMEM lane quadrants 0-3) ----------------
        if (warp < 4) {
            if (ok) ok = mbar_wait(&acc_bar, 0, deadline, a.err);
            ok = __all_sync(0xFFFFFFFFu, ok);  // tcgen05.ld is warp-collective
            tc_fence_after();
            float* stg = reinterpret_cast<float*>(stage_b(0));  // [128 rows][16 cols] fp32
            for (int c0 = 0; c0 < N; c0 += 16) {
                float v[16];
                if (ok) tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) stg[(warp * 32 + lane) * 17 + i] = ok ? v[i] : 0.f;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (kGemm1) {
                    // 64 outputs n x 16 tokens: thread -> (token c, 8 consecutive n)
                    const int c = tid >> 3, nb = (tid & 7) * 8;
                    if (c0 + c < count) {
                        uint32_t o[4];
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            float hv[2];
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                const int nl = nb + 2 * p + q;                    // 0..63
                                const int gr = (nl >> 5) * 64 + (nl & 31);        // gate row in the tile
                                const float gv = stg[gr * 17 + c], uv = stg[(gr + 32) * 17 + c];
                                hv[q] = gv / (1.0f + expf(-gv)) * uv;
                            }
                            o[p] = bf16x2_of(hv[0], hv[1]);
                        }
                        const int pos = start + c0 + c;
                        *reinterpret_cast<uint4*>(a.h + (size_t)pos * a.NW + mt * 64 + nb) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                } else {
                    // 128 outputs n x 16 tokens: thread -> (token c of 8, 16 consecutive n), two passes
#pragma unroll
                    for (int pass = 0; pass < 2; ++pass) {
                        const int c = pass * 8 + (tid >> 4), nb = (tid & 15) * 8;
                        if (c0 + c < count) {
                            const int pos = start + c0 + c;
                            int t, slot;
                            if (pos < a.P) {
                                const int pid = a.perm[pos];
                                t = pid / a.k;
                                slot = pid - t * a.k;
                            } else {
                                t = pos - a.P;
                                slot = a.k;
                            }
                            const float wgt = a.pair_w[pos];
                            uint32_t o[4];
#pragma unroll
                            for (int p = 0; p < 4; ++p)
                                o[p] = bf16x2_of(wgt * stg[(nb + 2 * p) * 17 + c], wgt * stg[(nb + 2 * p + 1) * 17 + c]);
                            *reinterpret_cast<uint4*>(a.ys + ((size_t)t * (a.k + 1) + slot) * a.NW + mt * 128 + nb) =
                                make_uint4(o[0], o[1], o[2], o[3]);
                        }
                    }
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
            }
            tc_fence_before();
        }
    } else if (lane == 0) {
        // ---------------- MMA issuer ----------------
        const uint32_t idesc = idesc_bf16(N);
        bool ok = true;
        for (int ks = 0; ks < ksteps; ++ks) {
            const int s = ks % kPfStages;
            ok = mbar_wait(&full_bar[s], (ks / kPfStages) & 1, deadline, a.err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t abase = smem_u32(stage_a(s)), bbase = smem_u32(stage_b(s));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc_mma(tmem, smem_desc_sw128(abase + kk * 32), smem_desc_sw128(bbase + kk * 32), idesc,
                       (ks | kk) != 0);
            tc_commit(&empty_bar[s]);
        }
        tc_commit(&acc_bar);  // also on a timeout: every issued MMA completes before TMEM is freed
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 8) {
        if (lane == 0) mbar_wait(&acc_bar, 0, deadline, a.err);
        __syncwarp();
        tmem_dealloc(tmem, kPfTmemCols);
    }
}

// out[t, n] = sum over slots j (routed in slot order, shared last) of ys[t, j, n].
template <bool kOutBf16>
__global__ void slot_reduce_kernel(const uint16_t* __restrict__ ys, int T, int S, int H, void* __restrict__ out)
{
    const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;  // 8 outputs per thread
    if (i >= (size_t)T * H) return;
    const size_t t = i / H, n = i - t * H;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < S; ++j) {
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
