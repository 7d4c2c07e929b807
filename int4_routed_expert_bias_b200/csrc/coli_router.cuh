// coli_router.cuh -- Route: router scores (fp32 GEMV) and bias-corrected top-k.
//
// DeepSeek-V3-style sigmoid router ("Colibri 完全ガイド", section コア技術のハイライト):
//   logit_e = x . w_router[e], s_e = sigmoid(logit_e), c_e = s_e + bias_e,
//   idx = top-k of c (descending, equal c -> lower e), w_j = alpha * s_j / sum s.
#pragma once

#include <cooperative_groups.h>

#include "coli_common.cuh"

namespace coli {

constexpr int kRouterTokens = 4;     // tokens per router block
constexpr int kRouterThreads = 256;

// logits[t, e] for one expert row e (blockIdx.x) and up to kRouterTokens tokens
// (blockIdx.y); optionally zeroes n_zero counters used by the next kernels.  The row of w_router is read once per token group with 16-byte
// loads; the per-thread partial sums are reduced in a fixed order, so the
// result is deterministic.
template <bool kBf16>
__global__ void __launch_bounds__(kRouterThreads)
router_logits_kernel(const void* __restrict__ x, int T, int H, const float* __restrict__ w_router,
                     int E, float* __restrict__ logits, int32_t* __restrict__ zero_ctr, int n_zero)
{
    if (zero_ctr && blockIdx.x == 0 && blockIdx.y == 0)
        for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero_ctr[i] = 0;
    const int e = blockIdx.x;
    const int t0 = blockIdx.y * kRouterTokens;
    const int nt = min(kRouterTokens, T - t0);
    const float* wrow = w_router + (size_t)e * H;
    const size_t xrow_bytes = (size_t)H * (kBf16 ? 2 : 4);
    const char* xb = static_cast<const char*>(x) + (size_t)t0 * xrow_bytes;

    float acc[kRouterTokens];
#pragma unroll
    for (int t = 0; t < kRouterTokens; ++t) acc[t] = 0.f;

    // Issue every weight load of a pass before the first FMA: up to kUnroll
    // 16-byte loads in flight per thread (H = 6144 needs 6).
    constexpr int kUnroll = 8;
    for (int base = threadIdx.x * 4; base < H; base += kUnroll * kRouterThreads * 4) {
        float4 wv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = base + u * kRouterThreads * 4;
            wv[u] = i < H ? *reinterpret_cast<const float4*>(wrow + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int t = 0; t < kRouterTokens; ++t) {
            if (t < nt) {
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int i = base + u * kRouterThreads * 4;
                    if (i < H) {
                        const float4 v = load_act4<kBf16>(xb + t * xrow_bytes, i);
                        acc[t] = fmaf(wv[u].x, v.x, acc[t]);
                        acc[t] = fmaf(wv[u].y, v.y, acc[t]);
                        acc[t] = fmaf(wv[u].z, v.z, acc[t]);
                        acc[t] = fmaf(wv[u].w, v.w, acc[t]);
                    }
                }
            }
        }
    }
    __shared__ float red[kRouterThreads / 32][kRouterTokens];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int t = 0; t < kRouterTokens; ++t) {
        const float v = warp_sum(acc[t]);
        if (lane == 0) red[warp][t] = v;
    }
    __syncthreads();
    if (threadIdx.x < nt) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kRouterThreads / 32; ++w) v += red[w][threadIdx.x];
        logits[(size_t)(t0 + threadIdx.x) * E + e] = v;
    }
}

// logits[t, e] for large batches: a 64-token x 64-expert tile per block,
// K-steps of 32 staged in shared memory, 4 x 4 outputs per thread, fp32.
constexpr int kRtTile = 64;
constexpr int kRtK = 32;

template <bool kBf16>
__global__ void __launch_bounds__(256)
router_logits_tiled_kernel(const void* __restrict__ x, int T, int H, const float* __restrict__ w_router, int E,
                           float* __restrict__ logits)
{
    __shared__ float xs[kRtK][kRtTile + 4];
    __shared__ float ws[kRtK][kRtTile + 4];
    const int t0 = blockIdx.x * kRtTile, e0 = blockIdx.y * kRtTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // outputs (t0 + ty*4 + i, e0 + tx*4 + j)
    float acc[4][4] = {};
    for (int k0 = 0; k0 < H; k0 += kRtK) {
        // stage 64 x 32 of x and of w_router, transposed to [k][row]
        for (int i = threadIdx.x; i < kRtTile * kRtK / 4; i += 256) {
            const int r = i / (kRtK / 4), c = (i % (kRtK / 4)) * 4;
            float4 xv = make_float4(0.f, 0.f, 0.f, 0.f), wv = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t0 + r < T) xv = load_act4<kBf16>(static_cast<const char*>(x) + (size_t)(t0 + r) * H * (kBf16 ? 2 : 4), k0 + c);
            if (e0 + r < E) wv = *reinterpret_cast<const float4*>(w_router + (size_t)(e0 + r) * H + k0 + c);
            xs[c][r] = xv.x; xs[c + 1][r] = xv.y; xs[c + 2][r] = xv.z; xs[c + 3][r] = xv.w;
            ws[c][r] = wv.x; ws[c + 1][r] = wv.y; ws[c + 2][r] = wv.z; ws[c + 3][r] = wv.w;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kRtK; ++kk) {
            const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
            const float4 b = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = t0 + ty * 4 + i, e = e0 + tx * 4 + j;
            if (t < T && e < E) logits[(size_t)t * E + e] = acc[i][j];
        }
}

// Top-k of one token by one warp: sigmoid, bias, k rounds of warp arg-max,
// renormalised weights.  Lane j keeps the j-th selection.  The arg-max key is
// (c desc, index asc); a non-finite score can never make the warp pick an index
// twice or out of range.
// kPer = experts held per lane (E <= 32 * kPer).
template <int kPer>
__device__ __forceinline__ void topk_warp_rounds(const float* lrow, int E, int k, const float* __restrict__ sel_bias,
                                            float routed_scale, int32_t* idx_row, float* w_row)
{
    const int lane = threadIdx.x & 31;
    float s[kPer], c[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            const float l = lrow[e];
            s[i] = 1.0f / (1.0f + expf(-l));
            const float ci = s[i] + sel_bias[e];
            c[i] = (ci == ci) ? ci : -INFINITY;  // NaN ranks last: keeps the order total
        } else {
            s[i] = 0.f;
            c[i] = 0.f;
        }
    }
    uint32_t taken = 0;
    int my_idx = 0;
    float my_s = 0.f;
    for (int j = 0; j < k; ++j) {
        float bv = 0.f;
        int bi = -1;
        float bs = 0.f;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && (bi < 0 || c[i] > bv)) {
                bv = c[i];
                bi = e;
                bs = s[i];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
            const float os = __shfl_xor_sync(0xFFFFFFFFu, bs, o);
            if (oi >= 0 && (bi < 0 || ov > bv || (ov == bv && oi < bi))) {
                bv = ov;
                bi = oi;
                bs = os;
            }
        }
        if (lane == (bi & 31)) taken |= 1u << (bi >> 5);
        if (lane == j) {
            my_idx = bi;
            my_s = bs;
        }
    }
    float total = 0.f;
    for (int j = 0; j < k; ++j) total += __shfl_sync(0xFFFFFFFFu, my_s, j);
    if (lane < k) {
        idx_row[lane] = my_idx;
        w_row[lane] = routed_scale * my_s / total;
    }
}

// Top-k of one token by one warp for E <= 32 * kPer (same result as
// topk_warp_rounds, shorter dependency chain): every candidate gets one 64-bit
// key, high word an order-preserving image of c = sigmoid(logit) + bias (NaN ->
// -inf, -0 -> +0), low word the complement of the expert index, so a larger key
// means (c desc, index asc) and keys are unique.  Each lane sorts its kPer keys;
// then k rounds take the warp-wide maximum of the lanes' heads, and the lane
// that owns it pops its head.
template <int kPer>
__device__ __forceinline__ void topk_warp_heads(const float* lrow, int E, int k, const float* __restrict__ sel_bias,
                                                float routed_scale, int32_t* idx_row, float* w_row)
{
    const int lane = threadIdx.x & 31;
    unsigned long long key[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        key[i] = 0ull;  // no expert: below every real key
        if (e < E) {
            const float s = 1.0f / (1.0f + expf(-lrow[e]));
            const float ci = s + sel_bias[e];
            const float c = (ci == ci) ? ci + 0.0f : -INFINITY;
            const uint32_t u = __float_as_uint(c);
            const uint32_t m = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
            key[i] = ((unsigned long long)m << 32) | (uint32_t)(0xFFFFu - e);
        }
    }
    // descending sort of the lane's keys (odd-even transposition; kPer is small)
#pragma unroll
    for (int r = 0; r < kPer; ++r)
#pragma unroll
        for (int i = r & 1; i + 1 < kPer; i += 2) {
            const unsigned long long a = key[i], b = key[i + 1];
            key[i] = a > b ? a : b;
            key[i + 1] = a > b ? b : a;
        }
    unsigned long long mine = 0ull;  // lane j: the j-th winner
    for (int j = 0; j < k; ++j) {
        unsigned long long best = key[0];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xFFFFFFFFu, best, o);
            best = other > best ? other : best;
        }
        if (key[0] == best) {  // unique owner pops its head
#pragma unroll
            for (int i = 0; i + 1 < kPer; ++i) key[i] = key[i + 1];
            key[kPer - 1] = 0ull;
        }
        if (lane == j) mine = best;
    }
    const int my_e = (int)(0xFFFFu - (uint32_t)(mine & 0xFFFFu));
    const float my_s = lane < k ? 1.0f / (1.0f + expf(-lrow[my_e])) : 0.f;
    float total = 0.f;
    for (int j = 0; j < k; ++j) total += __shfl_sync(0xFFFFFFFFu, my_s, j);
    if (lane < k) {
        idx_row[lane] = my_e;
        w_row[lane] = routed_scale * my_s / total;
    }
}

// Default warp top-k: the tournament of sorted heads for up to 8 experts per
// lane, rounds of arg-max above that.
template <int kPer>
__device__ __forceinline__ void topk_warp_t(const float* lrow, int E, int k, const float* __restrict__ sel_bias,
                                            float routed_scale, int32_t* idx_row, float* w_row)
{
    if constexpr (kPer <= 8) topk_warp_heads<kPer>(lrow, E, k, sel_bias, routed_scale, idx_row, w_row);
    else topk_warp_rounds<kPer>(lrow, E, k, sel_bias, routed_scale, idx_row, w_row);
}

__device__ __forceinline__ void topk_warp(const float* lrow, int E, int k, const float* __restrict__ sel_bias,
                                          float routed_scale, int32_t* idx_row, float* w_row)
{
    if (E <= 256) topk_warp_t<8>(lrow, E, k, sel_bias, routed_scale, idx_row, w_row);
    else topk_warp_t<kMaxExperts / 32>(lrow, E, k, sel_bias, routed_scale, idx_row, w_row);
}

// One warp per token, logits from global memory (layer path).  When launched as
// a programmatic dependent it waits for the router scores, and lets its own
// dependent launch at once (that kernel waits for this one's results).
__global__ void __launch_bounds__(256)
router_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                   const float* __restrict__ sel_bias, float routed_scale,
                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w)
{
    griddep_wait();
    griddep_launch_dependents();
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;  // whole warp leaves together
    topk_warp(logits + (size_t)t * E, E, k, sel_bias, routed_scale, topk_idx + (size_t)t * k,
              topk_w + (size_t)t * k);
}

// Scratch-free router for the stand-alone entry point.  A cluster of
// kRouterCluster CTAs owns kRouterTokens tokens; CTA r scores experts
// e = r, r + kRouterCluster, ... (one warp per expert row, lanes split H) and
// writes the logits into CTA 0's shared memory through distributed shared
// memory; after a cluster barrier CTA 0 takes the top-k, one warp per token.
constexpr int kRouterCluster = 8;
constexpr int kRouterClusterThreads = 512;

template <bool kBf16>
__global__ void __cluster_dims__(kRouterCluster, 1, 1) __launch_bounds__(kRouterClusterThreads)
router_cluster_kernel(const void* __restrict__ x, int T, int H, const float* __restrict__ w_router,
                      const float* __restrict__ sel_bias, int E, int k, float routed_scale,
                      int32_t* __restrict__ topk_idx, float* __restrict__ topk_w)
{
    __shared__ float s_logits[kRouterTokens][kMaxExperts];
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int t0 = (blockIdx.x / kRouterCluster) * kRouterTokens;
    const int nt = min(kRouterTokens, T - t0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kWarps = kRouterClusterThreads / 32;
    float* dst = cluster.map_shared_rank(&s_logits[0][0], 0);
    const size_t xrow_bytes = (size_t)H * (kBf16 ? 2 : 4);
    const char* xb = static_cast<const char*>(x) + (size_t)t0 * xrow_bytes;

    for (int e = rank + kRouterCluster * warp; e < E; e += kRouterCluster * kWarps) {
        const float* wrow = w_router + (size_t)e * H;
        float acc[kRouterTokens];
#pragma unroll
        for (int t = 0; t < kRouterTokens; ++t) acc[t] = 0.f;
        for (int i = lane * 4; i < H; i += 32 * 4) {
            const float4 wv = *reinterpret_cast<const float4*>(wrow + i);
#pragma unroll
            for (int t = 0; t < kRouterTokens; ++t) {
                if (t < nt) {
                    const float4 v = load_act4<kBf16>(xb + t * xrow_bytes, i);
                    acc[t] = fmaf(wv.x, v.x, acc[t]);
                    acc[t] = fmaf(wv.y, v.y, acc[t]);
                    acc[t] = fmaf(wv.z, v.z, acc[t]);
                    acc[t] = fmaf(wv.w, v.w, acc[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < kRouterTokens; ++t) {
            const float v = warp_sum(acc[t]);
            if (lane == 0 && t < nt) dst[t * kMaxExperts + e] = v;
        }
    }
    cluster.sync();
    if (rank == 0 && warp < nt)
        topk_warp(&s_logits[warp][0], E, k, sel_bias, routed_scale, topk_idx + (size_t)(t0 + warp) * k,
                  topk_w + (size_t)(t0 + warp) * k);
}

}  // namespace coli
