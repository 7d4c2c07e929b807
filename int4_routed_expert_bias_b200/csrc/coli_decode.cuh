// coli_decode.cuh -- expert phases for decode batches: int4-gs64 GEMV on CUDA cores.
//
// The routed and shared experts are SwiGLU FFNs on int4 weights with one fp32
// scale per 64 along K ("colibri: 744B MoE…", section はじめにとソースが語らないこと,
// "gs64"; "Colibri 完全ガイド", section 詳細解説 step 3: single-token decode runs in f32).
//
// Work unit: one token group (<= TG pairs of one expert, from the union's work
// lists) times one block of rows.  Persistent CTAs take work units from a
// device counter, so the grid stays one wave regardless of the batch union.
// Each warp streams R rows of each matrix with 16-byte non-caching loads (one
// 16-byte chunk = 32 nibbles = half a scale group per lane), turns nibbles into
// floats in registers and takes the dot products with activations staged in
// shared memory, in fp32.
#pragma once

#include "coli_int4.cuh"

namespace coli {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kGateUpRows = 2;   // rows per warp of each of gate and up
constexpr int kDownRows = 4;     // rows per warp of down

// Dot products of NS int4 rows (qrow[r]: packed bytes, srow[r]: scales) with
// ntok staged vectors, reduced over the warp: every lane returns the totals.
// The loads of the next chunk are issued before the current one is consumed.
template <int NS, int TG>
__device__ __forceinline__ void rows_dot(const uint8_t* const (&qrow)[NS], const float* const (&srow)[NS],
                                         const StageGeom& g, const float4* xs, const float* corr,
                                         int ntok, float (&acc)[NS][TG])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int r = 0; r < NS; ++r)
#pragma unroll
        for (int t = 0; t < TG; ++t) acc[r][t] = 0.f;

    uint4 w[NS], wn[NS];
    float sc[NS], scn[NS];
#pragma unroll
    for (int r = 0; r < NS; ++r) {
        w[r] = wn[r] = make_uint4(0u, 0u, 0u, 0u);
        sc[r] = scn[r] = 0.f;
    }
    int c = lane;
    if (c < g.nch) {
#pragma unroll
        for (int r = 0; r < NS; ++r) {
            w[r] = ldg_stream(qrow[r] + (size_t)c * 16);
            sc[r] = ldg_f32(srow[r] + (c >> 1));
        }
    }
#pragma unroll 1
    for (int i = 0; i < g.per_lane; ++i, c += 32) {
        const int cn = c + 32;
        if (cn < g.nch) {
#pragma unroll
            for (int r = 0; r < NS; ++r) {
                wn[r] = ldg_stream(qrow[r] + (size_t)cn * 16);
                scn[r] = ldg_f32(srow[r] + (cn >> 1));
            }
        }
        if (c < g.nch) {
#pragma unroll
            for (int t = 0; t < TG; ++t) {
                if (t < ntok) {
                    float2 a[NS];
                    chunk_acc_rows<NS>(w, xs + (size_t)t * g.f4 + i * 256, lane, a);
                    const float cr = corr[t * g.nch + c];
#pragma unroll
                    for (int r = 0; r < NS; ++r) acc[r][t] = chunk_finish(a[r], cr, sc[r], acc[r][t]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < NS; ++r) {
            w[r] = wn[r];
            sc[r] = scn[r];
        }
    }
#pragma unroll
    for (int r = 0; r < NS; ++r)
#pragma unroll
        for (int t = 0; t < TG; ++t) acc[r][t] = warp_sum(acc[r][t]);
}

struct PhaseArgs {
    const uint8_t* q0;  // gate (or down) bytes, [E+1, N, K/2]
    const float* s0;    // its scales, [E+1, N, K/64]
    const uint8_t* q1;  // up bytes (gate/up phase only)
    const float* s1;
    int N, K;           // rows and columns of one expert matrix
    const void* act;    // gate/up: x [T, H]; down: h [P+T, F] fp32
    const int32_t* ctl;      // ctl[0] = number of token groups
    int32_t* task_ctr;       // work-unit counter (zeroed by the union kernel)
    const int32_t* g_expert;
    const int32_t* g_start;
    const int32_t* g_count;
    const int32_t* pair_token;
    const float* pair_w;
    float* out;         // gate/up: h [P+T, F]; down: partial [P+T, H]
};

// Shared part of both phases: the persistent task loop and the staging cache.
// kGateUp: out[pos, n] = silu(g) * u; else out[pos, n] = pair_w[pos] * y.
template <bool kGateUp, bool kBf16, int TG>
__global__ void __launch_bounds__(kDecThreads)
expert_phase_kernel(PhaseArgs a)
{
    constexpr int R = kGateUp ? kGateUpRows : kDownRows;
    constexpr int NS = kGateUp ? 2 * R : R;
    constexpr int RW = kDecWarps * R;  // rows per work unit

    extern __shared__ __align__(16) unsigned char smem[];
    const StageGeom g = stage_geom(a.K);
    float4* xs = reinterpret_cast<float4*>(smem);
    float* corr = reinterpret_cast<float*>(smem + (size_t)TG * g.f4 * 16);
    __shared__ int s_tok[TG];
    __shared__ int s_ntok;
    __shared__ int s_next;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int RB = a.N / RW;
    const int n_units = a.ctl[0] * RB;
    if (threadIdx.x == 0) {
        s_ntok = -1;
        s_next = atomicAdd(a.task_ctr, 1);
    }
    __syncthreads();
    int unit = s_next;
    while (unit < n_units) {
        __syncthreads();  // everyone has read s_next
        if (threadIdx.x == 0) s_next = atomicAdd(a.task_ctr, 1);

        const int grp = unit / RB;
        const int rb = unit - grp * RB;
        const int e = a.g_expert[grp];
        const int start = a.g_start[grp];
        const int n = a.g_count[grp];
        int tok[TG];
        bool same = (n == s_ntok);
#pragma unroll
        for (int t = 0; t < TG; ++t) {
            tok[t] = t < n ? (kGateUp ? a.pair_token[start + t] : start + t) : 0;
            if (t < n && tok[t] != s_tok[t]) same = false;
        }
        if (!same) {  // uniform across the block
            __syncthreads();
            auto rows = [&](int t) { return tok[t]; };
            if (kGateUp) stage_vectors<kBf16>(a.act, a.K, n, rows, g, xs, corr);
            else stage_vectors<false>(a.act, a.K, n, rows, g, xs, corr);
            if (threadIdx.x == 0) {
                s_ntok = n;
#pragma unroll
                for (int t = 0; t < TG; ++t) s_tok[t] = tok[t];
            }
            __syncthreads();
        }

        const int row0 = rb * RW + warp * R;
        const uint8_t* qrow[NS];
        const float* srow[NS];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const size_t row = (size_t)e * a.N + row0 + r;
            qrow[r] = a.q0 + row * (a.K / 2);
            srow[r] = a.s0 + row * (a.K / kGroup);
            if constexpr (kGateUp) {
                qrow[R + r] = a.q1 + row * (a.K / 2);
                srow[R + r] = a.s1 + row * (a.K / kGroup);
            }
        }
        float acc[NS][TG];
        rows_dot<NS, TG>(qrow, srow, g, xs, corr, n, acc);

        // lane (r * TG + t) writes one result
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < TG; ++t) {
                if (lane == r * TG + t && t < n) {
                    const int pos = start + t;
                    float v;
                    if constexpr (kGateUp) {
                        const float gv = acc[r][t];
                        v = gv / (1.0f + expf(-gv)) * acc[R + r][t];
                        a.out[(size_t)pos * a.N + row0 + r] = v;
                    } else {
                        v = a.pair_w[pos] * acc[r][t];
                        a.out[(size_t)pos * a.N + row0 + r] = v;
                    }
                }
            }
        __syncthreads();
        unit = s_next;
    }
}

// out[t, n] = sum_j partial[inv_perm[t*k + j], n] + partial[P + t, n], in slot
// order j = 0..k-1, then the shared expert.  4 outputs per thread.
// Slots whose routing index is -1 (dropped by adaptive top-p) are skipped.
template <bool kOutBf16>
__global__ void combine_kernel(const float* __restrict__ partial, const int32_t* __restrict__ inv_perm,
                               const int32_t* __restrict__ topk_idx, int T, int k, int H, void* __restrict__ out)
{
    const int P = T * k;
    const int per_row = H / 4;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * per_row) return;
    const int t = i / per_row;
    const int n = (i - t * per_row) * 4;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        if (topk_idx[(size_t)t * k + j] < 0) continue;
        const int pos = inv_perm[(size_t)t * k + j];
        const float4 v = *reinterpret_cast<const float4*>(partial + (size_t)pos * H + n);
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    const float4 v = *reinterpret_cast<const float4*>(partial + (size_t)(P + t) * H + n);
    s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    if constexpr (kOutBf16) {
        uint2 o;
        o.x = (uint32_t)float_to_bf16_bits(s.x) | ((uint32_t)float_to_bf16_bits(s.y) << 16);
        o.y = (uint32_t)float_to_bf16_bits(s.z) | ((uint32_t)float_to_bf16_bits(s.w) << 16);
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + (size_t)t * H + n) = o;
    } else {
        *reinterpret_cast<float4*>(static_cast<float*>(out) + (size_t)t * H + n) = s;
    }
}

}  // namespace coli
