// coli_decode1.cuh -- the layer for one token (batch-1 decode), five launches:
//   router scores (router_logits_kernel)
//   router_topk_kernel:    top-k of the scores, one warp
//   gateup_single_kernel:  h_j = silu(W_gate,e_j x) * (W_up,e_j x) for the k
//                          selected experts and the shared expert
//   down_single_kernel:    partial_j = w_j W_down,e_j h_j (w = 1 for shared)
//   combine_single_kernel: out = sum_j partial_j in slot order (deterministic)
// The last four are launched as programmatic dependents of their predecessor,
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

// Half of a gate/up unit: chunks c = lane + 32 b for b in [b0, b0 + kHalf) of the
// gate row and of the up row (kPL chunks per lane in all).
struct HalfRegs {
    uint4 w[kHalf][2];
    float sc[kHalf][2];
};

template <int b0>
__device__ __forceinline__ void half_load(const uint8_t* gq, const uint8_t* uq, const float* gs, const float* us,
                                          HalfRegs& r)
{
    // gq/uq point at this lane's first chunk (lane * 16), gs/us at the row's scales + lane / 2
#pragma unroll
    for (int b = 0; b < kHalf; ++b) {
        r.w[b][0] = ldg_stream(gq + (b0 + b) * 512);
        r.w[b][1] = ldg_stream(uq + (b0 + b) * 512);
        r.sc[b][0] = ldg_f32(gs + (b0 + b) * 16);
        r.sc[b][1] = ldg_f32(us + (b0 + b) * 16);
    }
}

template <int b0>
__device__ __forceinline__ void half_compute(const float4* xs, const float* corr, const int (&off)[8],
                                             const HalfRegs& r, float& tg, float& tu)
{
    // xs: staged x; corr: this lane's chunk corrections (corr + lane)
#pragma unroll
    for (int b = 0; b < kHalf; ++b) {
        float2 acc[2];
        chunk_acc_rows_off<2>(r.w[b], xs + (b0 + b) * 256, off, acc);
        const float cr = corr[(b0 + b) * 32];
        tg = chunk_finish(acc[0], cr, r.sc[b][0], tg);
        tu = chunk_finish(acc[1], cr, r.sc[b][1], tu);
    }
}

// One work unit = (slot, row n): h[slot][n] = silu((W_gate,e x)[n]) * (W_up,e x)[n];
// the gate and up rows share every staged x load.  Units are numbered shared
// expert first, then routed slots, rows fastest, and dealt out statically (warp
// gw of W takes gw, gw + W, ...): all units cost the same.  The int4 decode
// keeps the integer pipe busy, so the kernel relies on occupancy (32 warps per
// SM at <= 64 registers) to keep loads in flight; each half-row's loads are
// issued together.  A warp whose first unit is a shared-expert row issues its
// loads before the routing is known; the staging of x and the wait for the
// routing overlap them.  kPL = chunks per lane = H / 1024 (two halves of kHalf).
template <bool kBf16>
__global__ void __launch_bounds__(kSingleThreads, 2)
gateup_single_kernel(SingleArgs a)
{
    constexpr int kPL = 2 * kHalf;
    extern __shared__ __align__(16) unsigned char smem[];
    const StageGeom g = stage_geom(a.H);  // g.per_lane == kPL on this path
    float4* xs = reinterpret_cast<float4*>(smem);
    float* corr = reinterpret_cast<float*>(smem + (size_t)g.f4 * 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = gridDim.x * kSingleWarps;
    int off[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) off[j] = j * 32 + (lane ^ j);
    const size_t qrow = (size_t)a.H / 2, srow = (size_t)a.H / kGroup;
    auto rows = [&](int e, int n, const uint8_t*& gq, const uint8_t*& uq, const float*& gs, const float*& us) {
        const size_t row = (size_t)e * a.F + n;
        gq = a.gate_q + row * qrow + lane * 16;
        uq = a.up_q + row * qrow + lane * 16;
        gs = a.gate_s + row * srow + (lane >> 1);
        us = a.up_s + row * srow + (lane >> 1);
    };

    int u = blockIdx.x * kSingleWarps + warp;
    HalfRegs A;
    const bool first_shared = u < a.F;
    if (first_shared) {  // shared expert: no routing needed
        const uint8_t *gq, *uq;
        const float *gs, *us;
        rows(a.E, u, gq, uq, gs, us);
        half_load<0>(gq, uq, gs, us, A);
    }
    stage_vectors<kBf16>(a.x, a.H, 1, [](int) { return 0; }, g, xs, corr);  // x is this call's input
    __syncthreads();
    griddep_wait();  // the routing of this call (router_topk_kernel) is complete
    const int my_e = lane < a.k ? a.idx[lane] : a.E;  // expert of routed slot j + 1 in lane j

    bool loaded = first_shared;
    int sl = u / a.F, n = u - sl * a.F;  // slot index (0 = shared) and row of unit u
    const float* cl = corr + lane;
    while (sl <= a.k) {
        const uint8_t *gq, *uq;
        const float *gs, *us;
        const int er = __shfl_sync(0xFFFFFFFFu, my_e, sl > 0 ? sl - 1 : 0);  // sl is warp-uniform
        rows(sl == 0 ? a.E : er, n, gq, uq, gs, us);
        float tg = 0.f, tu = 0.f;
        if (!loaded) half_load<0>(gq, uq, gs, us, A);
        loaded = false;
        half_compute<0>(xs, cl, off, A, tg, tu);
        half_load<kHalf>(gq, uq, gs, us, A);
        half_compute<kHalf>(xs, cl, off, A, tg, tu);
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
// chunks c = lane + 32 i (i < 2: F = 2048 on this path).
struct DownRegs {
    uint4 w[2][2];  // [row][i]
    float sc[2][2];
};

__device__ __forceinline__ void down_load(const SingleArgs& a, int e, int n, int lane, DownRegs& r)
{
    const size_t row = (size_t)e * a.H + n;
    const uint8_t* q = a.down_q + row * ((size_t)a.F / 2) + lane * 16;
    const float* s = a.down_s + row * ((size_t)a.F / kGroup) + (lane >> 1);
    const size_t qr = (size_t)a.F / 2, sr = (size_t)a.F / kGroup;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            r.w[rr][i] = ldg_stream(q + rr * qr + i * 512);
            r.sc[rr][i] = ldg_f32(s + rr * sr + i * 16);
        }
}

__device__ __forceinline__ void down_compute(const float4* hs_j, const float* corr_j, const int (&off)[8], float wj,
                                             const DownRegs& r, float& o0, float& o1)
{
    // hs_j: staged h of slot j; corr_j: its chunk corrections + lane
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float2 acc[2];
        const uint4 w2[2] = {r.w[0][i], r.w[1][i]};
        chunk_acc_rows_off<2>(w2, hs_j + i * 256, off, acc);
        const float cr = corr_j[i * 32];
        o0 = fmaf(wj, chunk_finish(acc[0], cr, r.sc[0][i], 0.f), o0);
        o1 = fmaf(wj, chunk_finish(acc[1], cr, r.sc[1][i], 0.f), o1);
    }
}

// One work unit = (slot j, output rows n, n+1): partial[j][n..n+1] =
// w_j * (W_down,e_j h_j)[n..n+1] (w = 1 for the shared expert).  The two rows
// share every staged h load.  Each CTA serves one slot (CTA b takes slot
// b mod (k+1)), so it stages only that slot's h after the gate/up kernel is
// done; the slot's row pairs are dealt out statically over its CTAs' warps, and
// the next unit's loads are issued before this unit's reduction.
// combine_single_kernel then sums the partials in slot order (deterministic).
template <int kUnused = 0>
__global__ void __launch_bounds__(kSingleThreads, 2)
down_single_kernel(SingleArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int S = a.k + 1;  // slots: k routed + shared
    const StageGeom g = stage_geom(a.F);  // g.per_lane == 2 on this path
    float4* hs = reinterpret_cast<float4*>(smem);
    float* corr = reinterpret_cast<float*>(smem + (size_t)g.f4 * 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x % S;                           // this CTA's slot
    const int nc = ((int)gridDim.x - j + S - 1) / S;        // CTAs serving slot j
    const int Wj = nc * kSingleWarps;                        // their warps
    const int pairs = a.H / 2;
    int off[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) off[jj] = jj * 32 + (lane ^ jj);

    griddep_wait();  // routing and h of this call are complete
    const int e = j < a.k ? a.idx[j] : a.E;
    const float wj = j < a.k ? a.w[j] : 1.0f;
    int rp = (int)(blockIdx.x / S) * kSingleWarps + warp;  // first row pair of this warp
    DownRegs X;
    if (rp < pairs) down_load(a, e, 2 * rp, lane, X);
    stage_vectors<false>(a.h, a.F, 1, [j](int) { return j; }, g, hs, corr);
    __syncthreads();

    for (; rp < pairs; rp += Wj) {
        float o0 = 0.f, o1 = 0.f;
        down_compute(hs, corr + lane, off, wj, X, o0, o1);
        const int nc0 = 2 * rp;
        if (rp + Wj < pairs) down_load(a, e, 2 * (rp + Wj), lane, X);
        o0 = warp_sum(o0);
        o1 = warp_sum(o1);
        if (lane == 0) {
            a.partial[(size_t)j * a.H + nc0] = o0;
            a.partial[(size_t)j * a.H + nc0 + 1] = o1;
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
