// coli_layer.cuh -- the whole MoE layer for decode batches (1..64 tokens) in one
// cooperative launch: Route, Union, gate/up + SwiGLU, down and the weighted
// combine, separated by grid-wide barriers.
//
// The pages' per-token path is Route -> Union -> expert compute (Korean
// getting-started page, section 토큰당 처리 경로); the router is DeepSeek-V3's
// sigmoid router with a selection bias ("Colibri 完全ガイド", section コア技術の
// ハイライト) and the experts are int4 with one scale per 64 ("colibri: 744B MoE
// …", section はじめにとソースが語らないこと); decode runs in fp32 (完全ガイド,
// section 詳細解説 step 3).
//
// One CTA per SM, every CTA resident (cooperative launch).  Phases:
//   A  router partial scores (fp32 weights x staged activations) and the
//      shared expert's gate/up rows, which need no routing;
//   -- grid barrier --
//   B  every CTA takes the top-k of every token and the batch union (a stable
//      counting sort in shared memory: the same result in every CTA); then the
//      routed experts' gate/up rows.  With several tokens, also the shared
//      expert's down rows.  One token: the shared expert's down rows for this
//      CTA's output rows run while warp 0 takes the top-k;
//   -- grid barrier --
//   C  one token: this CTA's output rows of every selected down matrix, summed
//      in slot order into out (no partial buffer, no further barrier).
//      Several tokens: the routed down rows, one partial output per pair;
//   -- grid barrier (several tokens) --
//   D  several tokens: out[t] = sum over the token's slots (slot order) of the
//      partial outputs, plus the shared expert's.
//
// Work inside a phase is a flat list of items (a gate/up row pair of one token
// group, a down row pair, a router row piece) cut into contiguous, equally
// costly ranges, one per CTA, and dealt to the CTA's warps round-robin; each
// warp streams its items' int4 rows through a rolling register pipeline (the
// loads of the next P chunk-steps are in flight while one is computed).  Each
// int4 word is decoded once and applied to every token of the group.
//
// The only waits are the grid barriers; each gives up after a time limit,
// records an error in the status word and lets the kernel finish.
#pragma once

#include <cooperative_groups.h>

#include "coli_int4.cuh"
#include "coli_router.cuh"

namespace coli {

// Threads per block: 16 warps (one CTA per SM, at most 128 registers a thread).
__host__ __device__ constexpr int layer_threads(int) { return 512; }
constexpr int kLayerMaxT = 64;      // tokens (64-bit token masks in the union)
constexpr unsigned long long kBarrierNs = 2000000000ull;  // 2 s: far beyond any legitimate wait

// ---------------------------------------------------------------------------
// grid barrier

__device__ __forceinline__ unsigned long long layer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Barrier over all CTAs of a cooperative launch, on the launch's own barrier
// word (zero-based, provided by the driver for cooperative launches).  CTA 0
// adds 2^31 - (G - 1) and every other CTA 1, so bit 31 of the word flips
// exactly when the last CTA arrives and the low bits return to where they
// were.  Thread 0 of each CTA keeps the bit it expects before its next arrival
// (read once at kernel start: it cannot flip before this CTA arrives), so an
// arrival is a fire-and-forget release reduction and only the poll waits.  The
// poll acquires at GPU scope, so writes before the barrier are visible after
// it.  Gives up after the deadline (error word set) instead of waiting forever.
struct GridBar {
    unsigned int* word;
    unsigned int phase;  // bit 31 of the word before this CTA's next arrival (thread 0)
};

__device__ __forceinline__ GridBar grid_bar_open(unsigned int* word)
{
    GridBar b{word, 0u};
    if (threadIdx.x == 0) {
        unsigned int cur;
        asm volatile("ld.relaxed.gpu.u32 %0, [%1];" : "=r"(cur) : "l"(word) : "memory");
        b.phase = cur;  // only bit 31 is compared; the value is first needed at the first barrier
    }
    return b;
}

__device__ __forceinline__ void grid_barrier(GridBar& b, unsigned long long deadline, int* err)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned int add = blockIdx.x == 0 ? 0x80000000u - (gridDim.x - 1) : 1u;
        asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(b.word), "r"(add) : "memory");
        unsigned int cur;
        while (true) {
            asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(cur) : "l"(b.word) : "memory");
            if ((cur ^ b.phase) & 0x80000000u) break;
            if (layer_ns() > deadline) {
                atomicExch(err, 2);
                break;
            }
        }
        b.phase ^= 0x80000000u;
    }
    __syncthreads();
}

// Warp sums of four values: the sum of a lands on lanes 0-7 (read on lane 0),
// of b on lane 8, of c on lane 16, of d on lane 24; six shuffles.
__device__ __forceinline__ float warp_sum4(float a, float b, float c, float d)
{
    const bool h16 = (threadIdx.x & 16) != 0, h8 = (threadIdx.x & 8) != 0;
    const float v1 = (h16 ? c : a) + __shfl_xor_sync(0xFFFFFFFFu, h16 ? a : c, 16);
    const float v2 = (h16 ? d : b) + __shfl_xor_sync(0xFFFFFFFFu, h16 ? b : d, 16);
    float v = (h8 ? v2 : v1) + __shfl_xor_sync(0xFFFFFFFFu, h8 ? v1 : v2, 8);
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// the rolling int4 row-pair engine

// The int4 rows (bytes and scales) that one item streams, RW of them.
template <int RW>
struct Rows {
    const uint8_t* q[RW];
    const float* s[RW];
};

// The staged vectors that one item multiplies its rows with (indices into the
// staged set: vector i's digit planes start i * vstride 16-byte units in, its
// per-chunk (scale, corr) entries i * nch entries in).
template <int MT>
struct VecSet {
    int m;       // vectors used (<= MT)
    int vi[MT];  // staged-vector index of vector t
};

// One 16-byte chunk of each of the RW rows against up to MT digit-staged
// vectors of ND digits (see coli_int4.cuh): each word of each row is decoded
// once into biased bytes and applied to every vector with dp4a; every
// activation load serves all RW rows.  xd = this lane's plane 0 of the chunk
// in vector 0's frame; cc = this lane's chunk entry in vector 0's frame.
template <int MT, int RW, int ND>
__device__ __forceinline__ void chunk_rows_digit_vectors(const uint4 (&w)[RW], const uint4* xd, const float2* cc,
                                                         const VecSet<MT>& v, int vstride, int nch,
                                                         const float (&sc)[RW], float (&tot)[RW][MT])
{
    uint32_t lo[RW][4], hi[RW][4];
#pragma unroll
    for (int r = 0; r < RW; ++r) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t a = q == 0 ? w[r].x : q == 1 ? w[r].y : q == 2 ? w[r].z : w[r].w;
            lo[r][q] = nib_lo_u8(a);
            hi[r][q] = nib_hi_u8(a);
        }
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        if (t < v.m) {
            const uint4* x = xd + v.vi[t] * vstride;
            int acc[RW][ND];
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int d = 0; d < ND; ++d) acc[r][d] = 0;
#pragma unroll
            for (int d = 0; d < ND; ++d) {
                const uint4 xl = x[(2 * d) * 32], xh = x[(2 * d + 1) * 32];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t l = q == 0 ? xl.x : q == 1 ? xl.y : q == 2 ? xl.z : xl.w;
                    const uint32_t h = q == 0 ? xh.x : q == 1 ? xh.y : q == 2 ? xh.z : xh.w;
#pragma unroll
                    for (int r = 0; r < RW; ++r) {
                        acc[r][d] = dp4a_us(lo[r][q], l, acc[r][d]);
                        acc[r][d] = dp4a_us(hi[r][q], h, acc[r][d]);
                    }
                }
            }
            const float2 c = cc[v.vi[t] * nch];
            const uint32_t corr = (uint32_t)__float_as_int(c.y);
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                // X = 16384 d0 + 128 d1 + d2 (three digits), 128 d0 + d1 (two), d0 (one)
                uint32_t D = (uint32_t)acc[r][0];
#pragma unroll
                for (int d = 1; d < ND; ++d) D = D * 128u + (uint32_t)acc[r][d];
                D -= corr;
                tot[r][t] = fmaf(sc[r] * c.x, (float)(int)D, tot[r][t]);
            }
        }
    }
}

struct NoHook {
    __device__ void operator()() const {}
};

// Bytes of one ring slot (one step of a warp): RW 16-byte chunks and RW scales per lane.
__host__ __device__ constexpr int slot_bytes(int RW) { return 32 * RW * (16 + 4); }

// hook(): called by every thread once the first R - 1 steps are in flight and
// before the first one is consumed (e.g. a barrier and the staging of the
// vectors), also by warps that have no items.
// The streamed weights are read once per call: they are copied with an
// evict-first L2 policy, so that the stream (far larger than L2) does not push
// the kernel's instructions and the call's small shared data (activations,
// router partials, h) out of L2 between and within calls.
__device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// Asks the L2 cache for the bytes [p, p + n) (p and n multiples of 16); no completion to wait for.
__device__ __forceinline__ void l2_prefetch_bulk(const void* p, uint32_t n)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(n) : "memory");
}

__device__ __forceinline__ void cp_async16_s(uint32_t smem, const void* gmem, uint64_t pol)
{
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem), "l"(gmem), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async4_s(uint32_t smem, const void* gmem, uint64_t pol)
{
    asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 4, %2;" ::"r"(smem), "l"(gmem), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ float4 ldg_stream4(const float4* p, uint64_t pol)
{
    float4 v;
    asm("ld.global.nc.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t smem)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(smem));
    return r;
}
__device__ __forceinline__ float lds32(uint32_t smem)
{
    float r;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(r) : "r"(smem));
    return r;
}

// Streams items j0, j0 + js, ... (nj of them) of a row list: item j has RW
// int4 rows of K = 32 * nch values (rows_of(j, Rows<RW>&)) and up to MT staged
// vectors of ND digits (vecs_of(j, VecSet&)).  The lane takes chunks
// c = lane + 32 i, i < per_lane; a step is one chunk of every row (16 bytes of
// each and their scales).  The steps' bytes travel through this warp's ring of
// R slots in shared memory, filled by cp.async R - 1 steps ahead of the one
// being computed, so the bytes in flight do not cost registers and the loop
// stays small (the slot index is an address, not a register name).  At the
// end of item j, finish(j, VecSet, tot) gets the lane's partial sums
// tot[row][vector] (to be summed over the warp).  xs: staged digit planes;
// corr: staged chunk entries; ring: this warp's R * slot_bytes(RW) bytes.
template <int MT, int RW, int R, int ND, typename RowsOf, typename VecsOf, typename Finish, typename Hook = NoHook>
__device__ __forceinline__ void stream_rows(int j0, int js, int nj, int per_lane, int nch, const float4* xs,
                                            const void* corr, unsigned char* ring, RowsOf rows_of, VecsOf vecs_of,
                                            Finish finish, Hook hook = Hook())
{
    if (nj <= 0) {
        hook();
        return;
    }
    constexpr uint32_t kSlot = slot_bytes(RW);
    const int lane = threadIdx.x & 31;
    const bool whole = (nch & 31) == 0;  // every lane has a chunk at every step
    // this lane's bytes of ring slot 0: the 16-byte chunk of row r at +512 r, its scale at sc_off + 128 r
    const uint32_t ring_lane = smem_u32(ring) + lane * 16;
    const uint32_t ring_end = ring_lane + R * kSlot;
    const uint32_t sc_off = 512 * RW - 12 * lane;
    const uint64_t pol = l2_evict_first();
    // load cursor: item lj (0-based among mine), chunk step lci, this lane's slot address and source pointers
    int lj = 0, lci = 0;
    uint32_t lsl = ring_lane;
    const uint8_t* pq[RW];
    const float* ps[RW];
    auto set_rows = [&](int j) {
        Rows<RW> r;
        rows_of(j, r);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            pq[i] = r.q[i] + lane * 16;
            ps[i] = r.s[i] + (lane >> 1);
        }
    };
    set_rows(j0);
    auto issue = [&]() {
        if (lj < nj && (whole || lane + 32 * lci < nch)) {
#pragma unroll
            for (int i = 0; i < RW; ++i) cp_async16_s(lsl + 512 * i, pq[i], pol);
#pragma unroll
            for (int i = 0; i < RW; ++i) cp_async4_s(lsl + sc_off + 128 * i, ps[i], pol);
        }
        cp_async_commit();  // one group per step (empty past the end)
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            pq[i] += 512;  // this lane's next chunk: 32 chunks on
            ps[i] += 16;
        }
        lsl += kSlot;
        if (lsl == ring_end) lsl = ring_lane;
        if (++lci == per_lane) {
            lci = 0;
            if (++lj < nj) set_rows(j0 + lj * js);
        }
    };
#pragma unroll 1
    for (int u = 0; u < R - 1; ++u) issue();
    hook();

    int cj = 0, cci = 0;
    uint32_t csl = ring_lane;
    VecSet<MT> v;
    vecs_of(j0, v);
    float tot[RW][MT];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int t = 0; t < MT; ++t) tot[r][t] = 0.f;
    // staged vectors: 2 ND planes of 32 units of 16 bytes per chunk step; a float2 entry per chunk
    constexpr int kXStep = digit_planes(ND) * 32;
    const int vstride = per_lane * kXStep;  // 16-byte units per staged vector
    const uint4* xrow = reinterpret_cast<const uint4*>(xs) + lane;
    const float2* crow = static_cast<const float2*>(corr) + lane;
    const int S = nj * per_lane;
#pragma unroll 1
    for (int s = 0; s < S; ++s) {
        issue();                   // step s + R - 1 into the slot consumed last iteration
        cp_async_wait<R - 1>();    // step s has landed (this lane's own bytes)
        if (whole || lane + 32 * cci < nch) {
            uint4 w[RW];
            float sc[RW];
#pragma unroll
            for (int i = 0; i < RW; ++i) {
                w[i] = lds128(csl + 512 * i);
                sc[i] = lds32(csl + sc_off + 128 * i);
            }
            chunk_rows_digit_vectors<MT, RW, ND>(w, xrow, crow, v, vstride, nch, sc, tot);
        }
        csl += kSlot;
        if (csl == ring_end) csl = ring_lane;
        xrow += kXStep;
        crow += 32;
        if (++cci == per_lane) {
            cci = 0;
            xrow = reinterpret_cast<const uint4*>(xs) + lane;
            crow = static_cast<const float2*>(corr) + lane;
            finish(j0 + cj * js, v, tot);
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int t = 0; t < MT; ++t) tot[r][t] = 0.f;
            if (++cj < nj) vecs_of(j0 + cj * js, v);
        }
    }
    cp_async_wait<0>();  // the trailing (empty) groups: nothing is left in flight into the ring
}

// ---------------------------------------------------------------------------
// layer arguments and shared-memory layout

constexpr int kMaxPrefetch = 8;  // router weights, selection bias, the shared expert's 3 matrices and 3 scale arrays

struct LayerArgs {
    const float* w_router;  // [E, H]
    const float* sel_bias;  // [E]
    const uint8_t* gate_q;
    const float* gate_s;
    const uint8_t* up_q;
    const float* up_s;
    const uint8_t* down_q;
    const float* down_s;
    int H, F, E, k, T;
    float routed_scale;
    const void* x;          // [T, H] fp32 or bf16
    void* out;              // [T, H] fp32 or bf16
    float* logit_part;      // [n_pieces, T, E] router partial scores (n_pieces = 1: computed before the launch)
    int n_pieces;           // 0: the kernel computes the router (pieces of 1024 K); else precomputed pieces
    int32_t* idx_out;       // [T, k]
    float* w_out;           // [T, k]
    float* h;               // [T*k + T, F] SwiGLU outputs, sorted pair order, shared expert at T*k + t
    float* y;               // [T*k + T, H] partial outputs (several tokens)
    int* err;               // status word
    unsigned long long wait_ns;  // limit of each grid-barrier wait
    float top_p;            // adaptive expert top-p (0: plain top-k)
    unsigned long long* stamps;  // optional [gridDim.x, kStamps] globaltimer stamps per CTA (test hook)
    // router lookahead: byte ranges of the next layer to bring into L2 (pf_n of them, one token only)
    const unsigned char* pf_base[kMaxPrefetch];
    unsigned long long pf_bytes[kMaxPrefetch];
    int pf_n;
};

constexpr int kStamps = 16;

// Test hook: thread `by` (default 0) of each CTA records the time it reached point i.
__device__ __forceinline__ void stamp(const LayerArgs& a, int i, int by = 0)
{
    if (a.stamps && threadIdx.x == by) a.stamps[blockIdx.x * kStamps + i] = layer_ns();
}

// Shared-memory plan of one launch (host and device compute the same one).
// The union tables' offsets are kernel parameters, so their addresses are one
// add away and need no registers across the kernel.
struct LayerSmem {
    int nx;       // activation vectors staged (all tokens when T <= MT, else MT)
    int nh;       // h vectors staged
    size_t x_off, h_off, u_off, y_off, bytes;
    // union tables (byte offsets from the start of shared memory)
    uint32_t mask, cnt, off, gpre, idx, w, perm, ipos, gexp, gpos, seg_c, seg_i, seg_cost, tmp;
    uint32_t logit;  // router scores [T, E] of the tokens (when the kernel scores them itself)
    uint32_t ring;   // the warps' cp.async rings, warps x ring_slots x slot_bytes(layer_rows(MT, nd))
    int ring_slots;
};

// Rows per engine step: four (each activation load then serves four rows),
// except for groups of several tokens of three-digit activations, whose four
// staged vectors leave no room for the four-row ring.
__host__ __device__ constexpr int layer_rows(int MT, int nd) { return MT == 1 || nd <= 2 ? 4 : 2; }

// Ring slots per warp (steps in flight + 1): deeper when fewer activation
// vectors are staged, shallower for the four-row slots.
__host__ __device__ constexpr int layer_ring_slots(int MT, int nd)
{
    return layer_rows(MT, nd) == 4 ? 3 : MT == 1 ? 5 : 4;
}

// rows_per_cta: output rows of one CTA in the one-token output-row mode; nd:
// digits per staged activation (3 for fp32 inputs, 2 for bf16, 1 for int8).
__host__ __device__ inline LayerSmem layer_smem(int T, int H, int F, int E, int k, int MT, bool out_rows,
                                                int rows_per_cta, int nd)
{
    LayerSmem s{};
    s.nx = T <= MT ? T : MT;
    s.nh = out_rows ? k + 1 : MT;
    size_t off = 0;
    s.x_off = off;
    off += align_up(digit_smem_bytes(H, s.nx, nd), 16);
    s.h_off = off;
    off += align_up(digit_smem_bytes(F, s.nh, nd), 16);
    s.u_off = off;
    {
        const size_t P = (size_t)T * k;
        size_t o = off;
        auto take = [&](size_t bytes) {
            const uint32_t r = (uint32_t)o;
            o += align_up(bytes, 16);
            return r;
        };
        s.mask = take((size_t)E * 8);
        s.cnt = take((size_t)E * 4);
        s.off = take(((size_t)E + 1) * 4);
        s.gpre = take(((size_t)E + 1) * 4);
        s.idx = take(P * 4);
        s.w = take(P * 4);
        s.perm = take(P * 4);
        s.ipos = take(P * 4);
        s.gexp = take((P + 64) * 4);
        s.gpos = take((P + 64) * 4);
        s.seg_c = take((P + (size_t)E + 70) * 8);
        s.seg_i = take((P + (size_t)E + 70) * 4);
        s.seg_cost = take((P + (size_t)E + 70) * 4);
        s.tmp = take(32 * 8);
        s.logit = take(T <= MT ? (size_t)T * E * 4 : 16);
        s.ring_slots = layer_ring_slots(MT, nd);
        s.ring = take((size_t)(layer_threads(MT) / 32) * s.ring_slots * slot_bytes(layer_rows(MT, nd)));
        off = o;
    }
    s.y_off = off;
    off += out_rows ? align_up((size_t)rows_per_cta * (k + 1) * 4, 16) : 0;
    s.bytes = off;
    return s;
}

}  // namespace coli

namespace coli {

// ---------------------------------------------------------------------------
// top-k of one token from register-held scores

// Top-k of one token by one warp; lane l holds the router scores of experts
// e = l + 32 i in l[i] (E <= 32 kPer).  Same rule as the layer's other top-k:
// order by c = sigmoid(logit) + bias descending (NaN -> -inf, -0 -> +0), ties
// to the lower expert index.  c is mapped to an order-preserving 32-bit key
// (never 0 for an expert; 0 marks an empty or taken entry).  Each round every
// lane offers its best remaining entry (lowest index among equal keys), a warp
// max-reduction picks the key and a min-reduction over the lanes offering it
// picks the lowest expert index; the owner marks it taken.  Lane j < k returns
// the j-th expert and its weight routed_scale * s_j / sum s.
template <int kPer>
__device__ __forceinline__ void topk_regs(const float (&l)[kPer], int E, int k, const float* __restrict__ sel_bias,
                                          float routed_scale, float top_p, int& my_e, float& my_w)
{
    const int lane = threadIdx.x & 31;
    uint32_t key[kPer];
    float sg[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        key[i] = 0u;
        sg[i] = 0.f;
        if (e < E) {
            const float s = 1.0f / (1.0f + expf(-l[i]));
            const float ci = s + sel_bias[e];
            const float c = (ci == ci) ? ci + 0.0f : -INFINITY;
            const uint32_t u = __float_as_uint(c);
            key[i] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
            sg[i] = s;
        }
    }
    my_e = -1;
    float my_s = 0.f;
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u;
        int bi = 0;
        float bs = 0.f;
#pragma unroll
        for (int i = 0; i < kPer; ++i)
            if (key[i] > bk) {
                bk = key[i];
                bi = i;
                bs = sg[i];
            }
        const uint32_t top = __reduce_max_sync(0xFFFFFFFFu, bk);
        const uint32_t e = __reduce_min_sync(0xFFFFFFFFu, bk == top ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu);
        const float s = __shfl_sync(0xFFFFFFFFu, bs, e & 31);
        if (lane == (int)(e & 31)) {
#pragma unroll
            for (int i = 0; i < kPer; ++i)
                if (i == (int)(e >> 5)) key[i] = 0u;
        }
        if (lane == j) {
            my_e = (int)e;
            my_s = s;
        }
    }
    topk_weights(k, top_p, routed_scale, my_e, my_s, my_w);
}

// Top-k of one token by one warp from per-expert selection keys in shared
// memory (key as in topk_regs, 0 = taken).  Each round every lane offers its
// best remaining expert (lowest index among equal keys), a max-reduction picks
// the key, a min-reduction the lowest index offering it, and lane 0 clears it.
// Lane j < k returns the j-th expert and its sigmoid; the loops are rolled (the
// code runs once per call).
__device__ __forceinline__ void topk_smem(uint32_t* key, const float* sig, int E, int k, int& my_e, float& my_s)
{
    const int lane = threadIdx.x & 31;
    my_e = -1;
    my_s = 0.f;
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u;
        int be = 0;
#pragma unroll 4
        for (int e = lane; e < E; e += 32) {
            const uint32_t kv = key[e];
            if (kv > bk) {
                bk = kv;
                be = e;
            }
        }
        const uint32_t top = __reduce_max_sync(0xFFFFFFFFu, bk);
        const uint32_t e = __reduce_min_sync(0xFFFFFFFFu, bk == top ? (uint32_t)be : 0xFFFFFFFFu);
        if (e < (uint32_t)E) {
            if (lane == 0) key[e] = 0u;
            if (lane == j) {
                my_e = (int)e;
                my_s = sig[e];
            }
        }
        __syncwarp();
    }
}

// Top-k of token t for more than 256 experts (same rule and result as
// topk_regs), with few registers: k rounds of a warp arg-max over the scores,
// re-read from global memory each round; taken experts are marked in a
// per-lane bit mask (expert lane + 32 i <-> bit i).
__device__ __noinline__ void topk_rounds_global(const float* __restrict__ part, int npc, int T, int t, int E, int k,
                                                const float* __restrict__ sel_bias, float routed_scale, float top_p,
                                                int& my_e, float& my_w)
{
    const int lane = threadIdx.x & 31;
    unsigned int taken = 0u;
    my_e = -1;
    float my_s = 0.f;
    for (int j = 0; j < k; ++j) {
        unsigned long long best = 0ull;
        float best_s = 0.f;
        for (int i = 0; 32 * i < E; ++i) {
            const int e = lane + 32 * i;
            if (e >= E || ((taken >> i) & 1u)) continue;
            float l = 0.f;
            for (int p = 0; p < npc; ++p) l += part[((size_t)p * T + t) * E + e];
            const float s = 1.0f / (1.0f + expf(-l));
            const float ci = s + sel_bias[e];
            const float c = (ci == ci) ? ci + 0.0f : -INFINITY;
            const uint32_t uu = __float_as_uint(c);
            const uint32_t m = (uu & 0x80000000u) ? ~uu : (uu | 0x80000000u);
            const unsigned long long key = ((unsigned long long)m << 32) | (uint32_t)(0xFFFFu - e);
            if (key > best) {
                best = key;
                best_s = s;
            }
        }
        unsigned long long w = best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xFFFFFFFFu, w, o);
            w = other > w ? other : w;
        }
        const int e = (int)(0xFFFFu - (uint32_t)(w & 0xFFFFu));
        const float s = __shfl_sync(0xFFFFFFFFu, best_s, e & 31);
        if (lane == (e & 31)) taken |= 1u << (e >> 5);
        if (lane == j) {
            my_e = e;
            my_s = s;
        }
    }
    topk_weights(k, top_p, routed_scale, my_e, my_s, my_w);
}

// ---------------------------------------------------------------------------
// the kernel

// Work-list segments of one phase: segment s holds n items of cost c each.
// Once built (seg_build_warp), ipre[s] / cpre[s] are the item / cost offsets of segment s
// (ipre[nseg], cpre[nseg] the totals).
struct SegTable {
    int* ipre;        // [nseg + 1]
    long long* cpre;  // [nseg + 1]
    int* cost;        // [nseg]
    long long* tmp;   // [32]
    int nseg;
};

// Largest s in [0, n] with a[s] <= x (a ascending, a[0] <= x).
template <typename V>
__device__ __forceinline__ int last_le(const V* a, int n, long long x)
{
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((long long)a[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// This CTA's items of the phase: those whose start cost lies in
// [C b / G, C (b + 1) / G).  The quotients are taken in double precision,
// exact here (the costs stay far below 2^53 / G, and a ceiling quotient that
// is not an integer is at least 1 / cost from one), without the slow 64-bit
// integer division; a boundary shared by two CTAs is the same expression in
// both.
__device__ __forceinline__ void seg_cta_range(const SegTable& st, int& lo, int& hi)
{
    const long long C = st.cpre[st.nseg];
    auto first = [&](long long x) -> int {
        const int s = last_le(st.cpre, st.nseg, x);
        if (s >= st.nseg) return st.ipre[st.nseg];
        const int c = st.cost[s] > 0 ? st.cost[s] : 1;
        const long long r = (long long)ceil((double)(x - st.cpre[s]) / (double)c);
        const long long n = st.ipre[s + 1] - st.ipre[s];
        return st.ipre[s] + (int)(r < n ? r : n);
    };
    const double G = (double)gridDim.x;
    lo = first((long long)floor((double)C * blockIdx.x / G));
    hi = first((long long)floor((double)C * (blockIdx.x + 1) / G));
}

// Union tables in shared memory (every CTA computes the same ones).
struct UnionSmem {
    unsigned long long* mask;  // [E] tokens that chose expert e
    int* cnt;                  // [E]
    int* off;                  // [E + 1] first sorted position of expert e
    int* gpre;                 // [E + 1] first group of expert e
    int* idx;                  // [P] routing (token-major)
    float* w;                  // [P]
    int* perm;                 // [P] pair id at each sorted position
    int* ipos;                 // [P] sorted position of each pair
    int* gexp;                 // [P + 64] expert of each routed group
    int* gpos;                 // [P + 64] first sorted position of each routed group
    int* seg_i;                // segment table storage
    long long* seg_c;
    int* seg_cost;
    long long* tmp;            // [32]
};

__device__ __forceinline__ UnionSmem union_smem(unsigned char* base, const LayerSmem& ls)
{
    UnionSmem u;
    u.mask = reinterpret_cast<unsigned long long*>(base + ls.mask);
    u.cnt = reinterpret_cast<int*>(base + ls.cnt);
    u.off = reinterpret_cast<int*>(base + ls.off);
    u.gpre = reinterpret_cast<int*>(base + ls.gpre);
    u.idx = reinterpret_cast<int*>(base + ls.idx);
    u.w = reinterpret_cast<float*>(base + ls.w);
    u.perm = reinterpret_cast<int*>(base + ls.perm);
    u.ipos = reinterpret_cast<int*>(base + ls.ipos);
    u.gexp = reinterpret_cast<int*>(base + ls.gexp);
    u.gpos = reinterpret_cast<int*>(base + ls.gpos);
    u.seg_c = reinterpret_cast<long long*>(base + ls.seg_c);
    u.seg_i = reinterpret_cast<int*>(base + ls.seg_i);
    u.seg_cost = reinterpret_cast<int*>(base + ls.seg_cost);
    u.tmp = reinterpret_cast<long long*>(base + ls.tmp);
    return u;
}


// A segment table built by one warp: segment s < nseg has items_of(s) items
// of cost_of(s) each; ipre / cpre get the item / cost offsets of s = 0..nseg
// (exclusive prefix sums, the totals at nseg) and cost the per-item costs.
// Each lane takes a contiguous run of segments; two warp scans join them.  The
// caller synchronises the block before the table is read.
template <typename ItemsOf, typename CostOf>
__device__ __forceinline__ void seg_build_warp(const UnionSmem& u, int nseg, ItemsOf items_of, CostOf cost_of)
{
    const int lane = threadIdx.x & 31;
    const int per = (nseg + 1 + 31) / 32;
    const int s_lo = min(nseg + 1, lane * per), s_hi = min(nseg + 1, s_lo + per);
    int isum = 0;
    long long csum = 0;
    for (int s = s_lo; s < s_hi && s < nseg; ++s) {
        const int n = items_of(s);
        isum += n;
        csum += (long long)n * cost_of(s);
    }
    int iinc = isum;
    long long cinc = csum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, iinc, o);
        const long long yc = __shfl_up_sync(0xFFFFFFFFu, cinc, o);
        if (lane >= o) {
            iinc += y;
            cinc += yc;
        }
    }
    int ip = iinc - isum;
    long long cp = cinc - csum;
    for (int s = s_lo; s < s_hi; ++s) {
        u.seg_i[s] = ip;
        u.seg_c[s] = cp;
        if (s < nseg) {
            const int n = items_of(s), c = cost_of(s);
            u.seg_cost[s] = c;
            ip += n;
            cp += (long long)n * c;
        }
    }
}

// The batch union by one warp (T <= 64 tokens, their k slots in idx, dropped
// slots -1): per expert the token mask, count, first sorted position (off) and
// first group (gpre, groups of up to MT pairs), the sorted pair list perm and
// each pair's position ipos (experts ascending, pairs ascending within an
// expert), and per group its expert and first position.  Each lane takes a
// contiguous run of experts; warp scans give the offsets.  Returns the number
// of groups (also at gpre[E]).  The caller synchronises the block afterwards.
template <int MT>
__device__ __forceinline__ int union_warp(const UnionSmem& u, int T, int k, int E, int* err)
{
    const int lane = threadIdx.x & 31;
    const int P = T * k;
    for (int e = lane; e < E; e += 32) u.mask[e] = 0ull;
    __syncwarp();
    for (int p = lane; p < P; p += 32) {
        const int e = u.idx[p];
        if (e >= 0 && COLI_IN_BOUNDS(e < E, err)) atomicOr(&u.mask[e], 1ull << (p / k));  // dropped slots: none
    }
    __syncwarp();
    const int per = (E + 31) / 32;
    const int e_lo = min(E, lane * per), e_hi = min(E, e_lo + per);
    int cs = 0, gs = 0;
    for (int e = e_lo; e < e_hi; ++e) {
        const int c = __popcll(u.mask[e]);
        cs += c;
        gs += (c + MT - 1) / MT;
    }
    int ci = cs, gi = gs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, ci, o);
        const int yg = __shfl_up_sync(0xFFFFFFFFu, gi, o);
        if (lane >= o) {
            ci += y;
            gi += yg;
        }
    }
    const int n_pairs = __shfl_sync(0xFFFFFFFFu, ci, 31), n_groups = __shfl_sync(0xFFFFFFFFu, gi, 31);
    int oc = ci - cs, og = gi - gs;
    for (int e = e_lo; e < e_hi; ++e) {
        const int c = __popcll(u.mask[e]);
        u.cnt[e] = c;
        u.off[e] = oc;
        u.gpre[e] = og;
        for (int i = 0; i * MT < c; ++i, ++og) {
            u.gexp[og] = e;
            u.gpos[og] = oc + i * MT;
        }
        oc += c;
    }
    if (lane == 0) {
        u.off[E] = n_pairs;
        u.gpre[E] = n_groups;
    }
    __syncwarp();
    for (int p = lane; p < P; p += 32) {
        const int t = p / k, e = u.idx[p];
        int pos = -1;
        if (e >= 0 && e < E) {
            const unsigned long long below = t == 0 ? 0ull : (u.mask[e] & ((1ull << t) - 1ull));
            pos = u.off[e] + __popcll(below);
            if (COLI_IN_BOUNDS(pos < P, err)) u.perm[pos] = p;
            else pos = -1;
        }
        u.ipos[p] = pos;
    }
    return n_groups;
}

}  // namespace coli

namespace coli {

// Grid-barrier word of this cooperative launch (nullptr if the launch was not cooperative).
__device__ __forceinline__ unsigned int* launch_barrier_word()
{
    cooperative_groups::details::grid_workspace* ws = cooperative_groups::details::get_grid_workspace();
    return ws ? &ws->barrier : nullptr;
}

// Partial router scores of one piece: chunks c = lane + 32 (PC p + q), q < PC,
// of router row e (32 fp32 weights each) against the nt tokens' activations,
// read in fp32 from global memory (L2); the warp's sums go to
// logit_part[p][t][e].  All the piece's weight loads are issued together.
template <int NT, bool kBf16, int PC>
__device__ __forceinline__ void router_piece(const LayerArgs& a, int e, int p, int nt, const StageGeom& g)
{
    const int lane = threadIdx.x & 31;
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.f;
    const uint64_t pol = l2_evict_first();
    float4 wv[PC][8];
#pragma unroll
    for (int q = 0; q < PC; ++q) {
        const int c = lane + 32 * (PC * p + q);
        const float4* wrow = reinterpret_cast<const float4*>(a.w_router + (size_t)e * a.H) + (size_t)c * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) wv[q][j] = c < g.nch ? ldg_stream4(wrow + j, pol) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < PC; ++q) {
        const int c = lane + 32 * (PC * p + q);
        if (c < g.nch) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (t < nt) {
                    const char* xr = static_cast<const char*>(a.x) + (size_t)t * a.H * (kBf16 ? 2 : 4);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 xv = load_act4<kBf16>(xr, c * kChunkK + 4 * j);
                        acc[t] = fmaf(wv[q][j].x, xv.x, acc[t]);
                        acc[t] = fmaf(wv[q][j].y, xv.y, acc[t]);
                        acc[t] = fmaf(wv[q][j].z, xv.z, acc[t]);
                        acc[t] = fmaf(wv[q][j].w, xv.w, acc[t]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (t < nt) {
            const float v = warp_sum(acc[t]);
            if (lane == 0) a.logit_part[((size_t)p * a.T + t) * a.E + e] = v;
        }
    }
}

// Cost of an item of RW rows (RW / 2 row pairs) against m vectors of ND
// digits: bytes of the rows (in 256-byte units) times (c + m), the int4 decode
// and the copies being shared by the vectors and the multiply-adds not; c, the
// per-byte share, measured best at 2 for two-digit vectors (four rows a step)
// and 3 otherwise.
template <int RW, int ND>
__device__ __forceinline__ int item_cost(int K, int m)
{
    return max(1, (K + K / 8) / 256) * ((ND == 2 ? 2 : 3) + m) * (RW / 2);
}

// The layer, T <= 64 tokens.  MT = tokens per group (vectors per item);
// kOutRows: one token, down and combine by output rows; kI8: the
// integer-activation variant (int8 activations, one digit plane).
template <int MT, bool kBf16, bool kOutBf16, bool kOutRows, bool kI8>
__global__ void __launch_bounds__(layer_threads(MT), 1)
moe_layer_kernel(const LayerArgs a, const LayerSmem ls)
{
    constexpr int kLayerThreads = layer_threads(MT);
    constexpr int kLayerWarps = kLayerThreads / 32;
    extern __shared__ __align__(16) unsigned char lsm[];
    // digits per staged activation: fp32 activations three (21-bit), bf16 two (14-bit), the int8 variant one
    constexpr int nd = kI8 ? 1 : kBf16 ? 2 : 3;
    // rows per step of the several-token streams (item = kRW rows: kHP gate/up row pairs, or kRW down rows);
    // the one-token streams take two
    constexpr int kRW = layer_rows(MT, nd), kHP = kRW / 2;
    constexpr int P_GU = layer_ring_slots(MT, nd);  // ring slots (steps in flight + 1) of the streams
    constexpr int P_DN = P_GU;
    const int H = a.H, F = a.F, E = a.E, k = a.k, T = a.T;
    const int P = T * k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const StageGeom gH = stage_geom(H), gF = stage_geom(F);
    float4* xs = reinterpret_cast<float4*>(lsm + ls.x_off);
    constexpr int kPieceChunks = 2;  // router chunks per lane per piece
    // staged vectors as digit planes (16-byte units per vector)
    const int xvs = digit_vec_units(H, nd);
    const int hvs = digit_vec_units(F, nd);
    unsigned char* xcorr = lsm + ls.x_off + (size_t)ls.nx * xvs * 16;
    float4* hs = reinterpret_cast<float4*>(lsm + ls.h_off);
    unsigned char* hcorr = lsm + ls.h_off + (size_t)ls.nh * hvs * 16;
    const UnionSmem u = union_smem(lsm, ls);
    float* ypart = reinterpret_cast<float*>(lsm + ls.y_off);
    unsigned char* ring = lsm + ls.ring + (size_t)(threadIdx.x >> 5) * P_GU * slot_bytes(kRW);  // this warp's ring

    unsigned int* bar_word = launch_barrier_word();
    if (!bar_word) {  // not a cooperative launch: nothing can be synchronised (same answer in every CTA)
        if (blockIdx.x == 0 && threadIdx.x == 0) *a.err = 3;
        return;
    }
    GridBar bar = grid_bar_open(bar_word);
    const unsigned long long deadline = layer_ns() + a.wait_ns;
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.err = 0;
    stamp(a, 0);
    const bool all_x = T <= MT;  // every token's activations staged once for the whole call
    const int n_sg = (T + MT - 1) / MT;  // shared-expert groups

    // activations / SwiGLU outputs into shared memory: vector t = row row0 + t (or tbl[t] / tdiv)
    auto stage_vecs = [&](const void* src, int bf16, int K, int n, int row0, const int* tbl, int tdiv, float4* dst,
                          unsigned char* dcorr, int tid, int nthr) {
        if constexpr (kI8)
            stage_rows_int8(src, bf16, K, n, row0, tbl, tdiv, reinterpret_cast<uint4*>(dst),
                            reinterpret_cast<float2*>(dcorr), tid, nthr);
        else if constexpr (kBf16)
            stage_rows_digits2(src, bf16, K, n, row0, tbl, tdiv, reinterpret_cast<uint4*>(dst),
                               reinterpret_cast<float2*>(dcorr), tid, nthr);
        else
            stage_rows_digits(src, bf16, K, n, row0, tbl, tdiv, reinterpret_cast<uint4*>(dst),
                              reinterpret_cast<float2*>(dcorr), tid, nthr);
    };
    auto stage_x = [&](int n, int row0, const int* tbl = nullptr, int tdiv = 1) {
        stage_vecs(a.x, kBf16 ? 1 : 0, H, n, row0, tbl, tdiv, xs, xcorr, (int)threadIdx.x, kLayerThreads);
    };
    auto stage_h = [&](int n, int row0) {
        stage_vecs(a.h, 0, F, n, row0, nullptr, 1, hs, hcorr, (int)threadIdx.x, kLayerThreads);
    };

    // Sums of an item's rows over the warp, for each of its vectors: out(r, t, value) runs on one
    // lane per row r and vector t.  tot is float[RW][MT] (RW = 2 or 4 rows).
    auto rows_out = [&](const VecSet<MT>& v, const auto& tot, auto out) {
        constexpr int RW = sizeof(tot) / sizeof(tot[0]);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            if (t < v.m) {
                if constexpr (RW == 2) {
                    const float y = warp_sum2(tot[0][t], tot[1][t]);  // lane 0: row 0, lane 16: row 1
                    if ((lane & 15) == 0) out(lane >> 4, t, y);
                } else {
                    const float y = warp_sum4(tot[0][t], tot[1][t], tot[2][t], tot[3][t]);  // row r on lane 8 r
                    if ((lane & 7) == 0) out(lane >> 3, t, y);
                }
            }
        }
    };
    // gate/up item finisher: the item's rows are (gate n0, up n0, gate n0 + 1, up n0 + 1, ...);
    // h[pos0 + t, n] = silu(gate) * up for the group's vectors
    auto gateup_finish = [&](int n0, int pos0, const VecSet<MT>& v, const auto& tot) {
        constexpr int RW = sizeof(tot) / sizeof(tot[0]);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            if (t < v.m) {
                float gv, uv;
                int n;
                bool mine;
                if constexpr (RW == 2) {
                    gv = warp_sum2(tot[0][t], tot[1][t]);  // lane 0: gate, lane 16: up
                    uv = __shfl_sync(0xFFFFFFFFu, gv, 16);
                    n = n0;
                    mine = lane == 0;
                } else {
                    gv = warp_sum4(tot[0][t], tot[1][t], tot[2][t], tot[3][t]);  // gate/up of n0 on lanes 0/8, of n0 + 1 on 16/24
                    uv = __shfl_down_sync(0xFFFFFFFFu, gv, 8);
                    n = n0 + (lane >> 4);
                    mine = (lane & 15) == 0;
                }
                const int pos = pos0 + t;
                if (mine && COLI_IN_BOUNDS(pos >= 0 && pos < P + T && n >= 0 && n < F, a.err))
                    a.h[(size_t)pos * F + n] = gv / (1.0f + expf(-gv)) * uv;
            }
        }
    };
    // an item's rows: gate/up rows row0 .. row0 + RW / 2 - 1 of the stacked [E + 1, F] rows, as
    // (gate, up) pairs; down rows row0 .. row0 + RW - 1 of the stacked [E + 1, H] rows
    auto gateup_rows = [&](auto& r, size_t row0) {
        constexpr int RW = sizeof(r.q) / sizeof(r.q[0]);
#pragma unroll
        for (int p = 0; p < RW / 2; ++p) {
            const size_t row = row0 + p;
            r.q[2 * p] = a.gate_q + row * (H / 2);
            r.q[2 * p + 1] = a.up_q + row * (H / 2);
            r.s[2 * p] = a.gate_s + row * (H / kGroup);
            r.s[2 * p + 1] = a.up_s + row * (H / kGroup);
        }
    };
    auto down_rows = [&](auto& r, size_t row0) {
        constexpr int RW = sizeof(r.q) / sizeof(r.q[0]);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            r.q[i] = a.down_q + (row0 + i) * (F / 2);
            r.s[i] = a.down_s + (row0 + i) * (F / kGroup);
        }
    };

    // The CTA's items j = lo, lo + 1, ... go to its warps round-robin, continued across segments: the
    // first item of a segment that starts d items into the CTA's range belongs to warp d mod warps,
    // and this warp's first item of the segment is deal(d) items into it.
    auto deal = [&](int d) { return ((warp - d) % kLayerWarps + kLayerWarps) % kLayerWarps; };

    // ======================= phase A: router pieces, shared gate/up =======================
    {
        // Tokens scored here (one token group): the activations are staged and the router pieces
        // (block b takes pieces b, b + G, ...; about the same number per block) computed side by side;
        // the shared expert streams in phases B (gate/up, beside the routing) and C (down).
        // Larger batches (scored before the launch): the shared expert's gate/up rows of every token
        // group, cut into equal-cost ranges, each group's activations staged in the stream's hook.
        const int nrp = a.n_pieces == 0 ? (gH.per_lane + kPieceChunks - 1) / kPieceChunks : 0;  // pieces per row
        const int nseg = all_x ? 0 : n_sg;
        if (nseg > 0) {
            const SegTable st{u.seg_i, u.seg_c, u.seg_cost, u.tmp, nseg};
            if (warp == 0)
                seg_build_warp(
                    u, nseg, [&](int) { return F / kHP; }, [&](int s) { return item_cost<kRW, nd>(H, min(MT, T - s * MT)); });
            __syncthreads();
            int lo, hi;
            seg_cta_range(st, lo, hi);
            stamp(a, 10);
            for (int s = 0; s < nseg; ++s) {
                const int s_lo = max(lo, st.ipre[s]), s_hi = min(hi, st.ipre[s + 1]);
                if (s_lo >= s_hi) continue;
                const int t0 = s * MT, m = min(MT, T - t0);
                const int base = st.ipre[s];
                auto rows_of = [&](int j, Rows<kRW>& r) { gateup_rows(r, (size_t)E * F + kHP * (j - base)); };
                auto vecs_of = [&](int, VecSet<MT>& v) {
                    v.m = m;
#pragma unroll
                    for (int t = 0; t < MT; ++t) v.vi[t] = t;
                };
                auto fin = [&](int j, const VecSet<MT>& v, const float (&tot)[kRW][MT]) {
                    gateup_finish(kHP * (j - base), P + t0, v, tot);
                };
                auto hook = [&]() {  // this group's tokens
                    __syncthreads();
                    stage_x(m, t0);
                    __syncthreads();
                };
                const int first = s_lo + deal(s_lo - lo);
                const int nj = first < s_hi ? (s_hi - first + kLayerWarps - 1) / kLayerWarps : 0;
                stream_rows<MT, kRW, P_GU, nd>(first, kLayerWarps, nj, gH.per_lane, gH.nch, xs, xcorr, ring, rows_of,
                                               vecs_of, fin, hook);
            }
        }
        stamp(a, 15);
        if (all_x) {
            // nothing streams in this phase: the router pieces (their weight loads the longest latency
            // here) run on the last rw warps beside the staging of x on the others
            const int per_cta = (E * nrp + (int)gridDim.x - 1) / (int)gridDim.x;
            const int rw = max(1, min(kLayerWarps - (T > 1 ? 8 : 4), per_cta));
            const int xw = kLayerWarps - rw;
            if (warp < xw) {
                stage_vecs(a.x, kBf16 ? 1 : 0, H, T, 0, nullptr, 1, xs, xcorr, (int)threadIdx.x, xw * 32);
            } else {
                const int total = E * nrp;
                for (int i = blockIdx.x + gridDim.x * (warp - xw); i < total; i += gridDim.x * rw)
                    router_piece<MT, kBf16, kPieceChunks>(a, i / nrp, i % nrp, T, gH);
            }
            __syncthreads();
            stamp(a, 1);
        }
    }
    stamp(a, 2);
    grid_barrier(bar, deadline, a.err);
    stamp(a, 3);

    // ======================= phase B: top-k, union, routed gate/up =======================
    const int S1 = k + 1;  // one token: slots (routed in order, shared last)
    // one token: this CTA's output rows, units pr_lo .. pr_lo + npr - 1 of kRW rows each
    const int pr_lo = (int)((long long)(H / kRW) * blockIdx.x / gridDim.x);
    const int npr = (int)((long long)(H / kRW) * (blockIdx.x + 1) / gridDim.x) - pr_lo;
    const int npc = a.n_pieces == 0 ? (gH.per_lane + kPieceChunks - 1) / kPieceChunks : a.n_pieces;
    float* s_logit = reinterpret_cast<float*>(lsm + ls.logit);
    if constexpr (kOutRows) {
        // The shared expert's gate/up rows need no routing: this CTA's share of them (an even split)
        // has its first loads issued, then (hook) the token is scored and routed while no warp
        // streams; then the shared rows, then the routed experts' rows.
        auto route_hook = [&]() {
            // the token's router scores (sums of the pieces), sigmoids and selection keys
            uint32_t* s_key = reinterpret_cast<uint32_t*>(u.mask);  // the union's token masks are not used here
            float* s_sig = reinterpret_cast<float*>(u.mask) + E;
            for (int e = threadIdx.x; e < E; e += kLayerThreads) {
                float v = 0.f;
#pragma unroll
                for (int p = 0; p < 16; ++p)
                    if (p < npc) v += a.logit_part[(size_t)p * E + e];
                const float sg = 1.0f / (1.0f + expf(-v));
                const float ci = sg + a.sel_bias[e];
                const float c = (ci == ci) ? ci + 0.0f : -INFINITY;
                const uint32_t cu = __float_as_uint(c);
                s_key[e] = (cu & 0x80000000u) ? ~cu : (cu | 0x80000000u);
                s_sig[e] = sg;
            }
            __syncthreads();
            stamp(a, 11);
            if (warp == 0) {
                // the token's top-k, then the union of its k experts: ascending expert order
                int my_e;
                float my_s, my_w;
                topk_smem(s_key, s_sig, E, k, my_e, my_s);
                topk_weights(k, a.top_p, a.routed_scale, my_e, my_s, my_w);
                // kept experts (top-p may drop slots: expert -1) in ascending order
                int rank = 0;
                for (int i = 0; i < k; ++i) {
                    const int ei = __shfl_sync(0xFFFFFFFFu, my_e, i);
                    rank += (ei >= 0 && ei < my_e) ? 1 : 0;
                }
                const int n_kept = __popc(__ballot_sync(0xFFFFFFFFu, lane < k && my_e >= 0));
                if (lane < k) {
                    u.idx[lane] = my_e;
                    u.w[lane] = my_w;
                    u.ipos[lane] = my_e >= 0 ? rank : -1;
                    if (my_e >= 0) {
                        u.perm[rank] = lane;
                        u.gexp[rank] = my_e;
                        u.gpos[rank] = rank;
                    }
                    if (blockIdx.x == 0) {
                        a.idx_out[lane] = my_e;
                        a.w_out[lane] = my_w;
                    }
                }
                if (lane == 0) reinterpret_cast<int*>(u.tmp)[0] = n_kept;
                stamp(a, 12);
            }
            __syncthreads();
        };
        {
            const int s_lo = (int)((long long)(F / kHP) * blockIdx.x / gridDim.x);
            const int s_hi = (int)((long long)(F / kHP) * (blockIdx.x + 1) / gridDim.x);
            auto rows_of = [&](int j, Rows<kRW>& r) { gateup_rows(r, (size_t)E * F + kHP * j); };
            auto vecs_of = [&](int, VecSet<MT>& v) {
                v.m = 1;
#pragma unroll
                for (int t = 0; t < MT; ++t) v.vi[t] = 0;
            };
            auto fin = [&](int j, const VecSet<MT>& v, const float (&tot)[kRW][MT]) { gateup_finish(kHP * j, P, v, tot); };
            const int first = s_lo + warp;
            const int nj = first < s_hi ? (s_hi - first + kLayerWarps - 1) / kLayerWarps : 0;
            stream_rows<MT, kRW, P_GU, nd>(first, kLayerWarps, nj, gH.per_lane, gH.nch, xs, xcorr, ring, rows_of, vecs_of,
                                           fin, route_hook);
        }
        stamp(a, 14);
        stamp(a, 4);
        // routed gate/up: the kept experts x F / kHP items, equal cost, an even split
        const int n_kept = reinterpret_cast<const int*>(u.tmp)[0];
        const int fi = F / kHP;  // items per expert
        const int total = n_kept * fi;
        const int lo = (int)((long long)total * blockIdx.x / gridDim.x);
        const int hi = (int)((long long)total * (blockIdx.x + 1) / gridDim.x);
        const FastDiv div_f(fi, total);
        auto rows_of = [&](int j, Rows<kRW>& r) {
            const int g = div_f(j);
            int e = u.gexp[g];
            if (!COLI_IN_BOUNDS(e >= 0 && e < E, a.err)) e = 0;
            gateup_rows(r, (size_t)e * F + kHP * (j - g * fi));
        };
        auto vecs_of = [&](int, VecSet<MT>& v) {
            v.m = 1;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                v.vi[t] = 0;
            }
        };
        auto fin = [&](int j, const VecSet<MT>& v, const float (&tot)[kRW][MT]) {
            const int g = div_f(j);
            gateup_finish(kHP * (j - g * fi), g, v, tot);
        };
        const int first = lo + warp;
        const int nj = first < hi ? (hi - first + kLayerWarps - 1) / kLayerWarps : 0;
        stream_rows<MT, kRW, P_GU, nd>(first, kLayerWarps, nj, gH.per_lane, gH.nch, xs, xcorr, ring, rows_of, vecs_of,
                                       fin);
    } else {
        const bool scored_here = all_x;  // the kernel scored the tokens (npc partial pieces per score)
        if (scored_here) {
            // the scores: sums of the pieces (independent loads, every thread), into shared memory
            for (int i = threadIdx.x; i < T * E; i += kLayerThreads) {
                float v = 0.f;
#pragma unroll
                for (int p = 0; p < 16; ++p)
                    if (p < npc) v += a.logit_part[(size_t)p * T * E + i];
                s_logit[i] = v;
            }
            __syncthreads();
        }
        // top-k: one warp per token
        for (int t = warp; t < T; t += kLayerWarps) {
            int my_e;
            float my_w;
            if (E <= 256) {
                float l[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int e = lane + 32 * i;
                    l[i] = e >= E ? 0.f : scored_here ? s_logit[t * E + e] : a.logit_part[(size_t)t * E + e];
                }
                topk_regs<8>(l, E, k, a.sel_bias, a.routed_scale, a.top_p, my_e, my_w);
            } else {
                topk_rounds_global(a.logit_part, npc, T, t, E, k, a.sel_bias, a.routed_scale, a.top_p, my_e, my_w);
            }
            if (lane < k) {
                u.idx[t * k + lane] = my_e;
                u.w[t * k + lane] = my_w;
                if (blockIdx.x == 0) {
                    a.idx_out[t * k + lane] = my_e;
                    a.w_out[t * k + lane] = my_w;
                }
            }
        }
        stamp(a, 11);
        __syncthreads();
        // union and the segment table of this phase by warp 0:
        // [shared down groups (several token groups)] + routed gate/up groups
        const int n_sd = all_x ? 0 : n_sg;
        if (warp == 0) {
            const int n_rg = union_warp<MT>(u, T, k, E, a.err);
            __syncwarp();
            seg_build_warp(
                u, n_sd + n_rg, [&](int s) { return s < n_sd ? H / kRW : F / kHP; },
                [&](int s) {
                    if (s < n_sd) return item_cost<kRW, nd>(F, min(MT, T - s * MT));
                    const int g = s - n_sd, e = u.gexp[g];
                    return item_cost<kRW, nd>(H, min(MT, u.off[e] + u.cnt[e] - u.gpos[g]));
                });
        } else if (all_x) {
            // one token group: the shared expert's gate/up for the staged tokens, on the other warps
            // beside the routing (this CTA's even share of the F row pairs, two rows a step through a
            // ring of twice the slots: a warp holds about one item, its steps nearly all in flight)
            constexpr int R2 = P_GU * kRW / 2;
            const int s_lo = (int)((long long)F * blockIdx.x / gridDim.x);
            const int s_hi = (int)((long long)F * (blockIdx.x + 1) / gridDim.x);
            auto rows_of = [&](int j, Rows<2>& r) { gateup_rows(r, (size_t)E * F + j); };
            auto vecs_of = [&](int, VecSet<MT>& v) {
                v.m = T;
#pragma unroll
                for (int t = 0; t < MT; ++t) v.vi[t] = t;
            };
            auto fin = [&](int j, const VecSet<MT>& v, const float (&tot)[2][MT]) { gateup_finish(j, P, v, tot); };
            const int first = s_lo + warp - 1;
            const int nj = first < s_hi ? (s_hi - first + kLayerWarps - 2) / (kLayerWarps - 1) : 0;
            stream_rows<MT, 2, R2, nd>(first, kLayerWarps - 1, nj, gH.per_lane, gH.nch, xs, xcorr, ring, rows_of,
                                       vecs_of, fin);
        }
        __syncthreads();
        stamp(a, 12);
        const int nseg = n_sd + u.gpre[E];
        const SegTable st{u.seg_i, u.seg_c, u.seg_cost, u.tmp, nseg};
        int lo, hi;
        seg_cta_range(st, lo, hi);

        stamp(a, 13);
        // shared expert's down rows (several tokens), one run per shared group
        for (int s = 0; s < n_sd; ++s) {
            const int s_lo = max(lo, st.ipre[s]), s_hi = min(hi, st.ipre[s + 1]);
            if (s_lo >= s_hi) continue;
            const int t0 = s * MT, m = min(MT, T - t0);
            __syncthreads();
            stage_h(m, P + t0);
            __syncthreads();
            const int base = st.ipre[s];
            auto rows_of = [&](int j, Rows<kRW>& r) { down_rows(r, (size_t)E * H + kRW * (j - base)); };
            auto vecs_of = [&](int, VecSet<MT>& v) {
                v.m = m;
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    v.vi[t] = t;
                }
            };
            auto fin = [&](int j, const VecSet<MT>& v, const float (&tot)[kRW][MT]) {
                const int n0 = kRW * (j - base);
                rows_out(v, tot, [&](int r, int t, float y) {
                    if (COLI_IN_BOUNDS(n0 + r < H, a.err)) a.y[(size_t)(P + t0 + t) * H + n0 + r] = y;
                });
            };
            const int first = s_lo + deal(s_lo - lo);
            const int nj = first < s_hi ? (s_hi - first + kLayerWarps - 1) / kLayerWarps : 0;
            stream_rows<MT, kRW, P_DN, nd>(first, kLayerWarps, nj, gF.per_lane, gF.nch, hs, hcorr, ring, rows_of, vecs_of,
                                           fin);
        }

        stamp(a, 14);
        // routed gate/up: one run over all routed groups when every token is staged,
        // else one run per group (its tokens staged)
        const int r_lo = max(lo, st.ipre[n_sd]), r_hi = hi;
        for (int s = n_sd; s < nseg && r_lo < r_hi; ++s) {
            int s_lo, s_hi;
            if (all_x) {
                if (s != n_sd) break;
                s_lo = r_lo;
                s_hi = r_hi;
            } else {
                s_lo = max(r_lo, st.ipre[s]);
                s_hi = min(r_hi, st.ipre[s + 1]);
                if (s_lo >= s_hi) continue;
                const int g = s - n_sd, e = u.gexp[g], p0 = u.gpos[g];
                const int m = min(MT, u.off[e] + u.cnt[e] - p0);
                __syncthreads();
                stage_x(m, 0, u.perm + p0, k);
                __syncthreads();
            }
            auto seg_of = [&](int j) { return all_x ? last_le(st.ipre, nseg - 1, j) : s; };
            auto rows_of = [&](int j, Rows<kRW>& r) {
                const int sj = seg_of(j);
                int e = u.gexp[sj - n_sd];
                if (!COLI_IN_BOUNDS(e >= 0 && e < E && j - st.ipre[sj] < F / kHP, a.err)) e = 0;
                gateup_rows(r, (size_t)e * F + kHP * (j - st.ipre[sj]));
            };
            auto vecs_of = [&](int j, VecSet<MT>& v) {
                const int g = seg_of(j) - n_sd, e = u.gexp[g], p0 = u.gpos[g];
                v.m = min(MT, u.off[e] + u.cnt[e] - p0);
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    const int vi = all_x ? (t < v.m ? u.perm[p0 + t] / k : 0) : t;
                    v.vi[t] = vi;
                }
            };
            auto fin = [&](int j, const VecSet<MT>& v, const float (&tot)[kRW][MT]) {
                const int sj = seg_of(j);
                gateup_finish(kHP * (j - st.ipre[sj]), u.gpos[sj - n_sd], v, tot);
            };
            const int first = s_lo + deal(s_lo - lo);
            const int nj = first < s_hi ? (s_hi - first + kLayerWarps - 1) / kLayerWarps : 0;
            stream_rows<MT, kRW, P_GU, nd>(first, kLayerWarps, nj, gH.per_lane, gH.nch, xs, xcorr, ring, rows_of, vecs_of,
                                           fin);
        }
    }
    stamp(a, 5);
    if constexpr (!kOutRows) {
        grid_barrier(bar, deadline, a.err);
        stamp(a, 6);
    }

    // ======================= phase C: down =======================
    if constexpr (kOutRows) {
        // one token: this CTA's output row pairs of the kept routed experts and the shared expert;
        // the loads of the first rows are issued before the grid barrier (the weights do not
        // depend on it), the h vectors are staged after it
        const int S = S1;
        // item j = (slot g = j / npr: the g-th kept expert in ascending order, the shared expert
        // at g = n_kept; unit of kRW output rows)
        const int n_kept = reinterpret_cast<const int*>(u.tmp)[0];
        const int n_slots = n_kept + 1;
        const FastDiv div_pr(npr, (long long)npr * n_slots);
        auto rows_of = [&](int j, Rows<kRW>& r) {
            const int slot = div_pr(j), pr = pr_lo + (j - slot * npr);
            int e = slot < n_kept ? u.gexp[slot] : E;
            if (!COLI_IN_BOUNDS(e >= 0 && e <= E && kRW * pr + kRW - 1 < H, a.err)) e = 0;
            down_rows(r, (size_t)e * H + kRW * pr);
        };
        auto vecs_of = [&](int j, VecSet<MT>& v) {
            const int slot = div_pr(j);
            v.m = 1;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                v.vi[t] = slot;
            }
        };
        auto fin = [&](int j, const VecSet<MT>& v, const float (&tot)[kRW][MT]) {
            const int slot = div_pr(j), pl = j - slot * npr;
            const int col = slot < n_kept ? slot : k;  // the shared expert's column is k
            rows_out(v, tot, [&](int r, int, float y) { ypart[(kRW * pl + r) * S + col] = y; });
        };
        auto hook = [&]() {
            if (a.pf_n > 0 && warp == kLayerWarps - 1) {
                // router lookahead, while the blocks meet and stage h (the memory is otherwise idle then):
                // this CTA's share of each range of the next layer, up to 4 KB per lane request
                for (int r = 0; r < a.pf_n && r < kMaxPrefetch; ++r) {
                    const unsigned long long B = a.pf_bytes[r];
                    const unsigned long long lo = (B * blockIdx.x / gridDim.x) & ~15ull;
                    const unsigned long long hi = (B * (blockIdx.x + 1) / gridDim.x) & ~15ull;
                    for (unsigned long long off = lo + 4096ull * lane; off < hi; off += 32ull * 4096)
                        l2_prefetch_bulk(a.pf_base[r] + off, (uint32_t)(hi - off < 4096ull ? hi - off : 4096ull));
                }
            }
            grid_barrier(bar, deadline, a.err);
            stamp(a, 6);
            // h of the g-th kept expert sits at position g, the shared expert's at P (= k)
            if (n_kept == P) {
                stage_h(n_kept + 1, 0);
            } else {
                stage_h(n_kept, 0);
                stage_vecs(a.h, 0, F, 1, P, nullptr, 1, hs + (size_t)n_kept * hvs, hcorr + (size_t)n_kept * gF.nch * 8,
                           (int)threadIdx.x, kLayerThreads);
            }
            __syncthreads();
            stamp(a, 7);
        };
        const int total = npr * n_slots;
        const int first = warp;
        const int nj = first < total ? (total - first + kLayerWarps - 1) / kLayerWarps : 0;
        stream_rows<MT, kRW, P_DN, nd>(first, kLayerWarps, nj, gF.per_lane, gF.nch, hs, hcorr, ring, rows_of, vecs_of,
                                       fin, hook);
        __syncthreads();
        stamp(a, 8);
        for (int i = threadIdx.x; i < kRW * npr; i += kLayerThreads) {
            float acc = 0.f;
            for (int j = 0; j < k; ++j)
                if (u.ipos[j] >= 0) acc = fmaf(u.w[j], ypart[i * S + u.ipos[j]], acc);
            acc += ypart[i * S + k];
            const int n = kRW * pr_lo + i;
            if constexpr (kOutBf16) static_cast<uint16_t*>(a.out)[n] = float_to_bf16_bits(acc);
            else static_cast<float*>(a.out)[n] = acc;
        }
    } else {
        // several tokens: routed down rows, one partial output row per pair (routing weight applied);
        // for one token group first the shared expert's down rows (its h at P + t, weight 1)
        const int n_sdc = all_x ? 1 : 0;
        const int nseg = n_sdc + u.gpre[E];
        auto seg_e = [&](int s) { return s < n_sdc ? E : u.gexp[s - n_sdc]; };
        auto seg_p0 = [&](int s) { return s < n_sdc ? P : u.gpos[s - n_sdc]; };
        auto seg_m = [&](int s) { return s < n_sdc ? T : min(MT, u.off[seg_e(s)] + u.cnt[seg_e(s)] - seg_p0(s)); };
        if (warp == 0)
            seg_build_warp(
                u, nseg, [&](int) { return H / kRW; }, [&](int s) { return item_cost<kRW, nd>(F, seg_m(s)); });
        __syncthreads();
        const SegTable st{u.seg_i, u.seg_c, u.seg_cost, u.tmp, nseg};
        int lo, hi;
        seg_cta_range(st, lo, hi);
        for (int s = 0; s < nseg; ++s) {
            const int s_lo = max(lo, st.ipre[s]), s_hi = min(hi, st.ipre[s + 1]);
            if (s_lo >= s_hi) continue;
            const bool shared = s < n_sdc;
            const int e = seg_e(s), p0 = seg_p0(s);
            const int m = seg_m(s);
            __syncthreads();
            stage_h(m, p0);
            __syncthreads();
            const int base = st.ipre[s];
            auto rows_of = [&](int j, Rows<kRW>& r) { down_rows(r, (size_t)e * H + kRW * (j - base)); };
            auto vecs_of = [&](int, VecSet<MT>& v) {
                v.m = m;
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    v.vi[t] = t;
                }
            };
            auto fin = [&](int j, const VecSet<MT>& v, const float (&tot)[kRW][MT]) {
                const int n0 = kRW * (j - base);
                rows_out(v, tot, [&](int r, int t, float y) {
                    if (COLI_IN_BOUNDS(p0 + t < (shared ? P + T : P) && n0 + r < H, a.err)) {
                        const float wt = shared ? 1.0f : u.w[u.perm[p0 + t]];
                        a.y[(size_t)(p0 + t) * H + n0 + r] = wt * y;
                    }
                });
            };
            const int first = s_lo + deal(s_lo - lo);
            const int nj = first < s_hi ? (s_hi - first + kLayerWarps - 1) / kLayerWarps : 0;
            stream_rows<MT, kRW, P_DN, nd>(first, kLayerWarps, nj, gF.per_lane, gF.nch, hs, hcorr, ring, rows_of, vecs_of,
                                           fin);
        }
        stamp(a, 7);
        grid_barrier(bar, deadline, a.err);
        stamp(a, 8);

        // ======================= phase D: combine =======================
        const int per_row = H / 4;
        const int total = T * per_row;
        const int stride = gridDim.x * kLayerThreads;
        for (int i = blockIdx.x * kLayerThreads + threadIdx.x; i < total; i += stride) {
            const int t = i / per_row, n = (i - t * per_row) * 4;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j <= k; ++j) {
                const int pos = j < k ? u.ipos[t * k + j] : P + t;
                if (pos < 0) continue;  // a slot dropped by top-p
                if (!COLI_IN_BOUNDS(pos < P + T, a.err)) continue;
                const float4 v = *reinterpret_cast<const float4*>(a.y + (size_t)pos * H + n);
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            }
            if constexpr (kOutBf16) {
                uint2 o;
                o.x = (uint32_t)float_to_bf16_bits(acc.x) | ((uint32_t)float_to_bf16_bits(acc.y) << 16);
                o.y = (uint32_t)float_to_bf16_bits(acc.z) | ((uint32_t)float_to_bf16_bits(acc.w) << 16);
                *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + (size_t)t * H + n) = o;
            } else {
                *reinterpret_cast<float4*>(static_cast<float*>(a.out) + (size_t)t * H + n) = acc;
            }
        }
    }
    stamp(a, 9);
}

}  // namespace coli
