// coli_decode1.cuh -- the layer for one token (batch-1 decode), four launches:
//   router scores (router_logits_kernel, also zeroes the work counters)
//   gateup_single_kernel:  top-k (every CTA, from the router scores), then
//                          h_j = silu(W_gate,e_j x) * (W_up,e_j x) for the k
//                          selected experts and the shared expert
//   down_single_kernel:    partial_j = w_j W_down,e_j h_j (w = 1 for shared)
//   combine_single_kernel: out = sum_j partial_j in slot order (deterministic)
// The last three are launched as programmatic dependents of their predecessor,
// so their launch overlaps its tail; they wait (griddepcontrol.wait) before
// reading its results.
//
// Work units are warp-sized and dealt out statically over a persistent grid
// (one wave); each unit issues all of its weight loads before its first multiply.  Route/Union as on the Korean
// getting-started page (토큰당 처리 경로); with one token the union of the
// batch is the token's own k experts.
#pragma once

#include "coli_int4.cuh"
#include "coli_router.cuh"

namespace coli {

constexpr int kSingleThreads = 512;  // one CTA per SM
constexpr int kSingleWarps = kSingleThreads / 32;
constexpr int kHalf = 3;             // chunks per lane per half-row batch (a 6144-wide row is 2 halves)

struct SingleArgs {
    const uint8_t* gate_q;
    const float* gate_s;
    const uint8_t* up_q;
    const float* up_s;
    const uint8_t* down_q;
    const float* down_s;
    int H, F, E, k;
    float routed_scale;
    const float* logits;    // [E] router scores of the token
    const float* sel_bias;  // [E]
    const void* x;          // [H] fp32 or bf16
    int32_t* idx;           // [k] written by CTA 0 of the gate/up kernel
    float* w;               // [k]
    float* h;               // [k+1, F] SwiGLU activations, slot order, shared expert last
    float* partial;         // [k+1, H] weighted down projections
    void* out;              // [H] fp32 or bf16
};

// Half of a gate/up unit's loads: chunks b0 .. b0+kHalf-1 (c = lane + 32 b) of
// the gate row and of the up row.
struct HalfRegs {
    uint4 w[kHalf][2];
    float sc[kHalf][2];
};

__device__ __forceinline__ void half_load(const SingleArgs& a, const StageGeom& g, int e, int n, int b0,
                                          int lane, HalfRegs& r)
{
    const size_t row = (size_t)e * a.F + n;
    const uint8_t* gq = a.gate_q + row * ((size_t)a.H / 2);
    const uint8_t* uq = a.up_q + row * ((size_t)a.H / 2);
    const float* gs = a.gate_s + row * ((size_t)a.H / kGroup);
    const float* us = a.up_s + row * ((size_t)a.H / kGroup);
#pragma unroll
    for (int b = 0; b < kHalf; ++b) {
        const int c = lane + 32 * (b0 + b);
        if (b0 + b < g.per_lane && c < g.nch) {
            r.w[b][0] = ldg_stream(gq + (size_t)c * 16);
            r.w[b][1] = ldg_stream(uq + (size_t)c * 16);
            r.sc[b][0] = ldg_f32(gs + (c >> 1));
            r.sc[b][1] = ldg_f32(us + (c >> 1));
        }
    }
}

__device__ __forceinline__ void half_compute(const StageGeom& g, const float4* xs, const float* corr, int b0,
                                             int lane, const HalfRegs& r, float& tg, float& tu)
{
#pragma unroll
    for (int b = 0; b < kHalf; ++b) {
        const int c = lane + 32 * (b0 + b);
        if (b0 + b < g.per_lane && c < g.nch) {
            float2 acc[2];
            chunk_acc_rows<2>(r.w[b], xs + (b0 + b) * 256, lane, acc);
            const float cr = corr[c];
            tg = chunk_finish(acc[0], cr, r.sc[b][0], tg);
            tu = chunk_finish(acc[1], cr, r.sc[b][1], tu);
        }
    }
}

// One work unit = (slot, row n): gu[slot][0][n] = (W_gate,e x)[n] and
// gu[slot][1][n] = (W_up,e x)[n]; SwiGLU is applied when the down kernel stages
// h.  The gate and up rows share every staged x load.  Units are numbered
// shared expert first, then routed slots, rows fastest, and dealt out
// statically (warp gw of W takes gw, gw + W, ...): all units cost the same.
// The multiply-adds of the int4 decode keep the integer pipe busy, so the kernel
// relies on occupancy (32 warps per SM at <= 64 registers) to keep enough
// loads in flight; each half-row's loads are issued together.  A warp whose
// first unit is a shared-expert row issues its loads before the router's top-k
// is known; warp 0's top-k and the staging of x overlap them.
template <bool kBf16>
__global__ void __launch_bounds__(kSingleThreads, 2)
gateup_single_kernel(SingleArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_e[kMaxTopK + 1];
    __shared__ int32_t s_idx[kMaxTopK];
    __shared__ float s_w[kMaxTopK];
    const StageGeom g = stage_geom(a.H);
    float4* xs = reinterpret_cast<float4*>(smem);
    float* corr = reinterpret_cast<float*>(smem + (size_t)g.f4 * 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = gridDim.x * kSingleWarps;

    int u = blockIdx.x * kSingleWarps + warp;
    HalfRegs A;
    const bool first_shared = u < a.F;
    if (first_shared) half_load(a, g, a.E, u, 0, lane, A);  // shared expert: no routing needed
    stage_vectors<kBf16>(a.x, a.H, 1, [](int) { return 0; }, g, xs, corr);  // x is this call's input
    griddep_wait();  // router scores of this call are complete
    if (warp == 0) {
        topk_warp_t<8>(a.logits, a.E, a.k, a.sel_bias, a.routed_scale, s_idx, s_w);  // E <= 256 on this path
        __syncwarp();
        if (lane < a.k) {
            s_e[lane] = s_idx[lane];
            if (blockIdx.x == 0) {
                a.idx[lane] = s_idx[lane];
                a.w[lane] = s_w[lane];
            }
        }
    }
    __syncthreads();

    bool loaded = first_shared;
    int sl = u / a.F, n = u - sl * a.F;  // slot index (0 = shared) and row of unit u
    while (sl <= a.k) {
        const int e = sl == 0 ? a.E : s_e[sl - 1];
        float tg = 0.f, tu = 0.f;
        if (!loaded) half_load(a, g, e, n, 0, lane, A);
        loaded = false;
        half_compute(g, xs, corr, 0, lane, A, tg, tu);
        if (g.per_lane > kHalf) {
            half_load(a, g, e, n, kHalf, lane, A);
            half_compute(g, xs, corr, kHalf, lane, A, tg, tu);
        }
        tg = warp_sum(tg);
        tu = warp_sum(tu);
        if (lane == 0) {
            const int j = sl == 0 ? a.k : sl - 1;  // slot in h (shared last)
            a.h[(size_t)j * a.F + n] = tg / (1.0f + expf(-tg)) * tu;
        }
        n += W;
        while (n >= a.F) {
            n -= a.F;
            ++sl;
        }
    }
    griddep_launch_dependents();
}

// Loads of one down item: rows n, n+1 of expert e's down matrix, the lane's
// chunks c = lane + 32 i (i < per_lane <= 2).
struct DownRegs {
    uint4 w[2][2];  // [row][i]
    float sc[2][2];
};

__device__ __forceinline__ void down_load(const SingleArgs& a, const StageGeom& g, int e, int n, int lane,
                                          DownRegs& r)
{
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const size_t row = (size_t)e * a.H + n + rr;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int c = lane + 32 * i;
            if (i < g.per_lane && c < g.nch) {
                r.w[rr][i] = ldg_stream(a.down_q + row * ((size_t)a.F / 2) + (size_t)c * 16);
                r.sc[rr][i] = ldg_f32(a.down_s + row * ((size_t)a.F / kGroup) + (c >> 1));
            }
        }
    }
}

__device__ __forceinline__ void down_compute(const StageGeom& g, const float4* hs, const float* corr, int j,
                                             float wj, int lane, const DownRegs& r, float& o0, float& o1)
{
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = lane + 32 * i;
        if (i < g.per_lane && c < g.nch) {
            float2 acc[2];
            const uint4 w2[2] = {r.w[0][i], r.w[1][i]};
            chunk_acc_rows<2>(w2, hs + (size_t)j * g.f4 + i * 256, lane, acc);
            const float cr = corr[j * g.nch + c];
            o0 = fmaf(wj, chunk_finish(acc[0], cr, r.sc[0][i], 0.f), o0);
            o1 = fmaf(wj, chunk_finish(acc[1], cr, r.sc[1][i], 0.f), o1);
        }
    }
}

// One work unit = (slot j, output rows n, n+1): partial[j][n..n+1] =
// w_j * (W_down,e_j h_j)[n..n+1] (w = 1 for the shared expert).  The two rows
// share every staged h load.  Units run row-pair-major (the k+1 slots of a row
// pair are neighbours) and are dealt out statically; the next unit's loads are
// issued before this unit's reduction.  combine_single_kernel then sums the
// partials in slot order (deterministic).
template <int kUnused = 0>
__global__ void __launch_bounds__(kSingleThreads, 2)
down_single_kernel(SingleArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_e[kMaxTopK + 1];
    __shared__ float s_w[kMaxTopK + 1];
    const int S = a.k + 1;  // slots: k routed + shared
    const StageGeom g = stage_geom(a.F);
    float4* hs = reinterpret_cast<float4*>(smem);
    float* corr = reinterpret_cast<float*>(smem + (size_t)S * g.f4 * 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = gridDim.x * kSingleWarps;
    const int units = (a.H / 2) * S;

    griddep_wait();  // routing and h of this call are complete
    if (threadIdx.x < S) {
        s_e[threadIdx.x] = threadIdx.x < a.k ? a.idx[threadIdx.x] : a.E;
        s_w[threadIdx.x] = threadIdx.x < a.k ? a.w[threadIdx.x] : 1.0f;
    }
    __syncthreads();
    int u = blockIdx.x * kSingleWarps + warp;
    int j = u % S, rp = u / S;  // slot and row pair of unit u
    DownRegs X;
    if (u < units) down_load(a, g, s_e[j], 2 * rp, lane, X);
    stage_vectors<false>(a.h, a.F, S, [](int t) { return t; }, g, hs, corr);
    __syncthreads();

    const int dj = W % S, drp = W / S;  // unit stride W as (slot, row pair) steps
    for (; u < units; u += W) {
        float o0 = 0.f, o1 = 0.f;
        down_compute(g, hs, corr, j, s_w[j], lane, X, o0, o1);
        const int jc = j, nc = 2 * rp;
        j += dj;
        rp += drp;
        if (j >= S) {
            j -= S;
            ++rp;
        }
        if (u + W < units) down_load(a, g, s_e[j], 2 * rp, lane, X);
        o0 = warp_sum(o0);
        o1 = warp_sum(o1);
        if (lane == 0) {
            a.partial[(size_t)jc * a.H + nc] = o0;
            a.partial[(size_t)jc * a.H + nc + 1] = o1;
        }
    }
    griddep_launch_dependents();
}

// out[n] = sum over slots j (routed in order, shared last) of partial[j][n].
template <bool kOutBf16>
__global__ void combine_single_kernel(const float* __restrict__ partial, int S, int H, void* __restrict__ out)
{
    griddep_wait();
    const int n = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (n >= H) return;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < S; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(partial + (size_t)j * H + n);
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    if constexpr (kOutBf16) {
        uint2 o;
        o.x = (uint32_t)float_to_bf16_bits(s.x) | ((uint32_t)float_to_bf16_bits(s.y) << 16);
        o.y = (uint32_t)float_to_bf16_bits(s.z) | ((uint32_t)float_to_bf16_bits(s.w) << 16);
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + n) = o;
    } else {
        *reinterpret_cast<float4*>(static_cast<float*>(out) + n) = s;
    }
}

}  // namespace coli
