// coli_union.cuh -- Union: stable counting sort of (token, slot) pairs by expert.
//
// Korean getting-started page, section 토큰당 처리 경로 ("Union"): experts that
// several tokens of a batch select are de-duplicated, so each expert's weights
// are streamed once per batch for all the tokens routed to it.
#pragma once

#include "coli_common.cuh"
#include "coli_router.cuh"

namespace coli {

constexpr int kUnionThreads = 1024;
constexpr int kUnionWarps = kUnionThreads / 32;

// Work lists for the expert phases of the layer (optional outputs of the union).
struct WorkLists {
    int32_t* pair_token;  // [P + T]: token of each sorted pair; pairs P..P+T-1 = shared expert
    float* pair_w;        // [P + T]: routing weight of each sorted pair (1 for shared)
    int32_t* ctl;         // [4]: n_groups, gate/up task counter, down task counter, unused
    int32_t* g_expert;    // [G]: expert of each token group
    int32_t* g_start;     // [G]: first sorted pair of the group
    int32_t* g_count;     // [G]: pairs in the group (<= group_tokens)
    const float* topk_w;  // [P]
    int group_tokens;     // tokens per group
};

// Optional fused top-k in front of the union (small batches): the router
// scores are in logits [T, E]; topk_idx / topk_w receive the routing.
struct TopkArgs {
    const float* logits;
    const float* sel_bias;
    float routed_scale;
    float* topk_w;
    float top_p;  // adaptive expert top-p (0: plain top-k)
};

// Inclusive scan of one value per thread over the block (kUnionThreads threads).
__device__ __forceinline__ int block_incl_scan(int v, int* warp_tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += n;
        }
        warp_tot[lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    const int add = warp > 0 ? warp_tot[warp - 1] : 0;
    const int r = v + add;
    __syncthreads();  // warp_tot may be reused by the caller
    return r;
}

// Single block.  Pairs are processed in chunks of kUnionThreads in ascending p;
// inside a chunk a pair's rank among equal experts is its rank inside its warp
// (match_any) plus the counts of that expert in earlier warps, so the order is
// the stable (expert, p) order whatever the thread timing.
template <bool kLists, bool kTopk>
__global__ void __launch_bounds__(kUnionThreads)
union_kernel(int32_t* topk_idx, int T, int k, int E,
             int32_t* __restrict__ count, int32_t* __restrict__ offset,
             int32_t* __restrict__ active, int32_t* __restrict__ n_active,
             int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm, WorkLists wl, TopkArgs tk)
{
    if constexpr (kTopk) {
        // Route first: one warp per token, written to topk_idx / topk_w
        for (int t = threadIdx.x >> 5; t < T; t += kUnionWarps)
            topk_warp_t<8>(tk.logits + (size_t)t * E, E, k, tk.sel_bias, tk.routed_scale, tk.top_p,
                           topk_idx + (size_t)t * k, tk.topk_w + (size_t)t * k);  // E <= 256 here
        __syncthreads();
    }
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_cursor[kMaxExperts];
    __shared__ uint8_t s_wcnt[kUnionWarps][kMaxExperts];
    __shared__ int s_scan[32];
    __shared__ int s_total[3];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int P = T * k;

    for (int e = tid; e < E; e += kUnionThreads) s_cnt[e] = 0;
    __syncthreads();
    for (int p = tid; p < P; p += kUnionThreads) {
        const int e = topk_idx[p];
        if ((unsigned)e < (unsigned)E) atomicAdd(&s_cnt[e], 1);  // out-of-range ids are skipped
    }
    __syncthreads();

    // offsets and the active list (E <= kUnionThreads: one expert per thread)
    const int v = tid < E ? s_cnt[tid] : 0;
    const int incl = block_incl_scan(v, s_scan);
    if (tid < E) {
        count[tid] = v;
        offset[tid] = incl - v;
        s_cursor[tid] = incl - v;
    }
    if (tid == E - 1) {
        offset[E] = incl;
        s_total[2] = incl;  // pairs with an expert (dropped slots have none)
    }
    const int f = (tid < E && v > 0) ? 1 : 0;
    const int fincl = block_incl_scan(f, s_scan);
    if (tid == E - 1) s_total[0] = fincl;
    int ng = 0;
    if (kLists && tid < E && v > 0) ng = (v + wl.group_tokens - 1) / wl.group_tokens;
    const int gincl = kLists ? block_incl_scan(ng, s_scan) : 0;
    if (kLists && tid == E - 1) s_total[1] = gincl;
    __syncthreads();
    const int na = s_total[0];
    if (f) active[fincl - 1] = tid;
    if (tid < E && tid >= na) active[tid] = -1;
    if (tid == 0) n_active[0] = na;

    // stable scatter
    for (int base = 0; base < P; base += kUnionThreads) {
        for (int i = tid; i < kUnionWarps * E; i += kUnionThreads) s_wcnt[i / E][i % E] = 0;
        __syncthreads();
        const int p = base + tid;
        int e = p < P ? topk_idx[p] : -1;
        if ((unsigned)e >= (unsigned)E) e = -1;
        const unsigned m = __match_any_sync(0xFFFFFFFFu, e);
        const int rank = __popc(m & ((1u << lane) - 1u));
        const int cw = __popc(m);
        if (e >= 0 && rank == 0) s_wcnt[warp][e] = (uint8_t)cw;
        __syncthreads();
        int pos = 0;
        if (e >= 0) {
            int pre = 0;
            for (int w = 0; w < warp; ++w) pre += s_wcnt[w][e];
            pos = s_cursor[e] + pre + rank;
            perm[pos] = p;
            inv_perm[p] = pos;
        }
        __syncthreads();
        if (e >= 0 && rank == cw - 1) {
            int later = 0;
            for (int w = warp + 1; w < kUnionWarps; ++w) later += s_wcnt[w][e];
            if (later == 0) s_cursor[e] = pos + 1;
        }
        __syncthreads();
    }

    if constexpr (kLists) {
        // sorted-pair tables (perm/inv_perm are complete: same block, after a barrier)
        __threadfence_block();
        const int valid = s_total[2];
        for (int pos = tid; pos < P; pos += kUnionThreads) {
            if (pos < valid) {
                const int p = perm[pos];
                wl.pair_token[pos] = p / k;
                wl.pair_w[pos] = wl.topk_w[p];
            } else {  // positions of dropped slots: a valid token, no weight
                wl.pair_token[pos] = 0;
                wl.pair_w[pos] = 0.f;
            }
        }
        for (int t = tid; t < T; t += kUnionThreads) {
            wl.pair_token[P + t] = t;
            wl.pair_w[P + t] = 1.0f;
        }
        // token groups: routed experts in ascending order, then the shared expert
        const int G = wl.group_tokens;
        const int routed_groups = s_total[1];
        if (tid < E && v > 0) {
            int gi = gincl - ng;
            const int off = incl - v;
            for (int i = 0; i < ng; ++i, ++gi) {
                wl.g_expert[gi] = tid;
                wl.g_start[gi] = off + i * G;
                wl.g_count[gi] = min(G, v - i * G);
            }
        }
        const int shared_groups = (T + G - 1) / G;
        for (int i = tid; i < shared_groups; i += kUnionThreads) {
            wl.g_expert[routed_groups + i] = E;
            wl.g_start[routed_groups + i] = P + i * G;
            wl.g_count[routed_groups + i] = min(G, T - i * G);
        }
        if (tid == 0) {
            wl.ctl[0] = routed_groups + shared_groups;
            wl.ctl[1] = 0;
            wl.ctl[2] = 0;
            wl.ctl[3] = 0;
        }
    }
}

}  // namespace coli

namespace coli {

// ---------------------------------------------------------------------------
// Union of large batches on the whole GPU: the same stable counting sort in
// three launches.  The pairs are cut into chunks of kUnionChunk;
//   union_chunk_kernel   (one CTA per chunk): per-expert counts of the chunk and
//                        each pair's rank among the chunk's pairs of its expert
//                        (warp match_any ranks plus the counts of earlier warps);
//   union_scan_kernel    (one CTA): per-expert totals and offsets, the start of
//                        every (chunk, expert) bucket, the active list and the
//                        token groups of the expert phases;
//   union_scatter_kernel (one thread per pair): position = bucket start + rank.
// Positions equal the single-CTA kernel's: experts ascending, pairs ascending
// within an expert.

constexpr int kUnionChunk = 256;  // pairs per chunk = threads of union_chunk_kernel

__global__ void __launch_bounds__(kUnionChunk)
union_chunk_kernel(const int32_t* __restrict__ topk_idx, int P, int E, int32_t* __restrict__ chunk_cnt,
                   int32_t* __restrict__ rank)
{
    constexpr int kWarps = kUnionChunk / 32;
    __shared__ int s_cnt[kMaxExperts];
    __shared__ uint16_t s_wcnt[kWarps][kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int p = blockIdx.x * kUnionChunk + tid;
    for (int e = tid; e < E; e += kUnionChunk) s_cnt[e] = 0;
    for (int i = tid; i < kWarps * E; i += kUnionChunk) s_wcnt[i / E][i % E] = 0;
    __syncthreads();
    int e = p < P ? topk_idx[p] : -1;
    if ((unsigned)e >= (unsigned)E) e = -1;  // out-of-range ids take no position
    const unsigned m = __match_any_sync(0xFFFFFFFFu, e);
    const int r = __popc(m & ((1u << lane) - 1u));
    if (e >= 0 && r == 0) {
        s_wcnt[warp][e] = (uint16_t)__popc(m);
        atomicAdd(&s_cnt[e], __popc(m));
    }
    __syncthreads();
    if (e >= 0) {
        int pre = 0;
        for (int w = 0; w < warp; ++w) pre += s_wcnt[w][e];
        rank[p] = pre + r;
    }
    for (int i = tid; i < E; i += kUnionChunk) chunk_cnt[(size_t)blockIdx.x * E + i] = s_cnt[i];
}

// chunk_cnt [n_chunks, E] becomes the bucket starts in place.
template <bool kLists>
__global__ void __launch_bounds__(kUnionThreads)
union_scan_kernel(int32_t* __restrict__ chunk_cnt, int n_chunks, int T, int k, int E, int32_t* __restrict__ count,
                  int32_t* __restrict__ offset, int32_t* __restrict__ active, int32_t* __restrict__ n_active,
                  WorkLists wl)
{
    __shared__ int s_scan[32];
    __shared__ int s_total[2];
    const int tid = threadIdx.x;
    int v = 0;
    if (tid < E)
        for (int c = 0; c < n_chunks; ++c) v += chunk_cnt[(size_t)c * E + tid];
    const int incl = block_incl_scan(v, s_scan);
    const int base = incl - v;
    if (tid < E) {
        count[tid] = v;
        offset[tid] = base;
        int run = base;
        for (int c = 0; c < n_chunks; ++c) {
            int32_t* q = chunk_cnt + (size_t)c * E + tid;
            const int n = *q;
            *q = run;
            run += n;
        }
    }
    if (tid == E - 1) {
        offset[E] = incl;
        s_total[2] = incl;  // pairs with an expert (dropped slots have none)
    }
    const int f = (tid < E && v > 0) ? 1 : 0;
    const int fincl = block_incl_scan(f, s_scan);
    if (tid == E - 1) s_total[0] = fincl;
    int ng = 0;
    if (kLists && tid < E && v > 0) ng = (v + wl.group_tokens - 1) / wl.group_tokens;
    const int gincl = kLists ? block_incl_scan(ng, s_scan) : 0;
    if (kLists && tid == E - 1) s_total[1] = gincl;
    __syncthreads();
    const int na = s_total[0];
    if (f) active[fincl - 1] = tid;
    if (tid < E && tid >= na) active[tid] = -1;
    if (tid == 0) n_active[0] = na;
    if constexpr (kLists) {
        const int G = wl.group_tokens, P = T * k;
        const int routed_groups = s_total[1];
        if (tid < E && v > 0) {
            int gi = gincl - ng;
            for (int i = 0; i < ng; ++i, ++gi) {
                wl.g_expert[gi] = tid;
                wl.g_start[gi] = base + i * G;
                wl.g_count[gi] = min(G, v - i * G);
            }
        }
        const int shared_groups = (T + G - 1) / G;
        for (int i = tid; i < shared_groups; i += kUnionThreads) {
            wl.g_expert[routed_groups + i] = E;
            wl.g_start[routed_groups + i] = P + i * G;
            wl.g_count[routed_groups + i] = min(G, T - i * G);
        }
        if (tid == 0) {
            wl.ctl[0] = routed_groups + shared_groups;
            wl.ctl[1] = 0;
            wl.ctl[2] = 0;
            wl.ctl[3] = 0;
        }
    }
}

template <bool kLists>
__global__ void union_scatter_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E,
                                     const int32_t* __restrict__ bucket, const int32_t* __restrict__ rank,
                                     const int32_t* __restrict__ offset, int32_t* __restrict__ perm,
                                     int32_t* __restrict__ inv_perm, WorkLists wl)
{
    const int P = T * k;
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if constexpr (kLists) {
        if (p >= offset[E] && p < P) {  // positions of dropped slots: a valid token, no weight
            wl.pair_token[p] = 0;
            wl.pair_w[p] = 0.f;
        }
    }
    if (p < P) {
        const int e = topk_idx[p];
        if ((unsigned)e < (unsigned)E) {
            const int pos = bucket[(size_t)(p / kUnionChunk) * E + e] + rank[p];
            perm[pos] = p;
            inv_perm[p] = pos;
            if constexpr (kLists) {
                wl.pair_token[pos] = p / k;
                wl.pair_w[pos] = wl.topk_w[p];
            }
        }
    }
    if constexpr (kLists) {
        if (p < T) {
            wl.pair_token[P + p] = p;
            wl.pair_w[P + p] = 1.0f;
        }
    }
}

}  // namespace coli
