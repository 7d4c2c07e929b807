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

// logits[t, e] for large batches: a 128-token x 64-expert tile per block of
// 256 threads, 8 tokens x 4 experts per thread (packed fp32x2 multiply-adds
// over expert pairs), K-steps of 16 staged in shared memory transposed to
// [k][row] and double-buffered: the next step's global loads are in registers
// while the current step is multiplied.  fp32 throughout; every output is one
// sequential sum over k, as in the oracle's definition up to rounding order.
constexpr int kRtT = 128, kRtE = 64, kRtK = 16;
constexpr int kRtThreads = 256;

template <bool kBf16>
__global__ void __launch_bounds__(kRtThreads)
router_logits_tiled_kernel(const void* __restrict__ x, int T, int H, const float* __restrict__ w_router, int E,
                           float* __restrict__ logits)
{
    __shared__ __align__(16) float xs[2][kRtK][kRtT + 4];
    __shared__ __align__(16) float ws[2][kRtK][kRtE + 4];
    const int t0 = blockIdx.x * kRtT, e0 = blockIdx.y * kRtE;
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;  // outputs (t0 + ty*8 + i, e0 + tx*4 + j)
    // global -> register staging: x rows (tid & 127), k chunks of 4; w rows (tid & 63)
    const int xr = tid & 127, xk = (tid >> 7) * 4;   // x: k = xk + 8 q, q < 2
    const int wr = tid & 63, wk = (tid >> 6) * 4;    // w: k = wk
    const size_t xrow_bytes = (size_t)H * (kBf16 ? 2 : 4);
    const bool xin = t0 + xr < T, win = e0 + wr < E;
    const char* xp = static_cast<const char*>(x) + (size_t)(xin ? t0 + xr : 0) * xrow_bytes;
    const float* wp = w_router + (size_t)(win ? e0 + wr : 0) * H;
    float4 xv[2], wv;
    auto fetch = [&](int k0) {
#pragma unroll
        for (int q = 0; q < 2; ++q)
            xv[q] = xin ? load_act4<kBf16>(xp, k0 + xk + 8 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
        wv = win ? *reinterpret_cast<const float4*>(wp + k0 + wk) : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int k = xk + 8 * q;
            xs[buf][k][xr] = xv[q].x;
            xs[buf][k + 1][xr] = xv[q].y;
            xs[buf][k + 2][xr] = xv[q].z;
            xs[buf][k + 3][xr] = xv[q].w;
        }
        ws[buf][wk][wr] = wv.x;
        ws[buf][wk + 1][wr] = wv.y;
        ws[buf][wk + 2][wr] = wv.z;
        ws[buf][wk + 3][wr] = wv.w;
    };
    float2 acc[8][2];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = make_float2(0.f, 0.f);
    fetch(0);
    store(0);
    __syncthreads();
    const int nk = H / kRtK;
    for (int ks = 0; ks < nk; ++ks) {
        const int buf = ks & 1;
        if (ks + 1 < nk) fetch((ks + 1) * kRtK);
#pragma unroll
        for (int kk = 0; kk < kRtK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&xs[buf][kk][ty * 8]);
            const float4 a1 = *reinterpret_cast<const float4*>(&xs[buf][kk][ty * 8 + 4]);
            const float4 bw = *reinterpret_cast<const float4*>(&ws[buf][kk][tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float2 b01 = make_float2(bw.x, bw.y), b23 = make_float2(bw.z, bw.w);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float2 ai = make_float2(av[i], av[i]);
                acc[i][0] = __ffma2_rn(ai, b01, acc[i][0]);
                acc[i][1] = __ffma2_rn(ai, b23, acc[i][1]);
            }
        }
        if (ks + 1 < nk) store(buf ^ 1);
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = t0 + ty * 8 + i;
        if (t >= T) continue;
        const float o[4] = {acc[i][0].x, acc[i][0].y, acc[i][1].x, acc[i][1].y};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + tx * 4 + j;
            if (e < E) logits[(size_t)t * E + e] = o[j];
        }
    }
}

// Routing weights of a warp's top-k: lane j < k holds slot j's expert my_e and
// its unbiased sigmoid my_s.  w_j = routed_scale * s_j / sum s.  With adaptive
// expert top-p (0 < top_p < 1; "colibri解説", section 速度を稼ぐ実用ノブ, --topp):
// the slots are ranked by share s_j / sum s (descending, lower expert first), a
// slot is kept while the share of the slots ranked ahead of it is below top_p
// (the shortest prefix that reaches top_p), the kept weights are renormalised
// over the kept slots and a dropped slot gets expert -1 and weight 0.  Every
// sum runs in slot order; without top-p the result is the plain weights.
__device__ __forceinline__ void topk_weights(int k, float top_p, float routed_scale, int& my_e, float my_s,
                                             float& my_w)
{
    const int lane = threadIdx.x & 31;
    float total = 0.f;
    for (int j = 0; j < k; ++j) total += __shfl_sync(0xFFFFFFFFu, my_s, j);
    bool keep = lane < k;
    if (top_p > 0.f && top_p < 1.f) {
        float ahead = 0.f;
        for (int j = 0; j < k; ++j) {
            const float sj = __shfl_sync(0xFFFFFFFFu, my_s, j);
            const int ej = __shfl_sync(0xFFFFFFFFu, my_e, j);
            if (j != lane && (sj > my_s || (sj == my_s && ej < my_e))) ahead += sj;
        }
        keep = keep && ahead / total < top_p;
    }
    float kept = 0.f;
    for (int j = 0; j < k; ++j) kept += __shfl_sync(0xFFFFFFFFu, keep ? my_s : 0.f, j);
    my_w = keep ? routed_scale * my_s / kept : 0.f;
    if (lane < k && !keep) my_e = -1;
}

// Top-k of one token by one warp: sigmoid, bias, k rounds of warp arg-max,
// renormalised weights.  Lane j keeps the j-th selection.  The arg-max key is
// (c desc, index asc); a non-finite score can never make the warp pick an index
// twice or out of range.
// kPer = experts held per lane (E <= 32 * kPer).
template <int kPer>
__device__ __forceinline__ void topk_warp_rounds(const float* lrow, int E, int k, const float* __restrict__ sel_bias,
                                            float routed_scale, float top_p, int32_t* idx_row, float* w_row)
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
    float my_w;
    topk_weights(k, top_p, routed_scale, my_idx, my_s, my_w);
    if (lane < k) {
        idx_row[lane] = my_idx;
        w_row[lane] = my_w;
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
                                                float routed_scale, float top_p, int32_t* idx_row, float* w_row)
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
    int my_e = (int)(0xFFFFu - (uint32_t)(mine & 0xFFFFu));
    const float my_s = lane < k ? 1.0f / (1.0f + expf(-lrow[my_e])) : 0.f;
    float my_w;
    topk_weights(k, top_p, routed_scale, my_e, my_s, my_w);
    if (lane < k) {
        idx_row[lane] = my_e;
        w_row[lane] = my_w;
    }
}

// Default warp top-k: the tournament of sorted heads for up to 8 experts per
// lane, rounds of arg-max above that.
template <int kPer>
__device__ __forceinline__ void topk_warp_t(const float* lrow, int E, int k, const float* __restrict__ sel_bias,
                                            float routed_scale, float top_p, int32_t* idx_row, float* w_row)
{
    if constexpr (kPer <= 8) topk_warp_heads<kPer>(lrow, E, k, sel_bias, routed_scale, top_p, idx_row, w_row);
    else topk_warp_rounds<kPer>(lrow, E, k, sel_bias, routed_scale, top_p, idx_row, w_row);
}

__device__ __forceinline__ void topk_warp(const float* lrow, int E, int k, const float* __restrict__ sel_bias,
                                          float routed_scale, float top_p, int32_t* idx_row, float* w_row)
{
    if (E <= 256) topk_warp_t<8>(lrow, E, k, sel_bias, routed_scale, top_p, idx_row, w_row);
    else topk_warp_t<kMaxExperts / 32>(lrow, E, k, sel_bias, routed_scale, top_p, idx_row, w_row);
}

// One warp per token, logits from global memory (layer path).  When launched as
// a programmatic dependent it waits for the router scores, and lets its own
// dependent launch at once (that kernel waits for this one's results).
__global__ void __launch_bounds__(256)
router_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                   const float* __restrict__ sel_bias, float routed_scale, float top_p,
                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w)
{
    griddep_wait();
    griddep_launch_dependents();
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;  // whole warp leaves together
    topk_warp(logits + (size_t)t * E, E, k, sel_bias, routed_scale, top_p, topk_idx + (size_t)t * k,
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
        topk_warp(&s_logits[warp][0], E, k, sel_bias, routed_scale, 0.f, topk_idx + (size_t)(t0 + warp) * k,
                  topk_w + (size_t)(t0 + warp) * k);
}

}  // namespace coli
