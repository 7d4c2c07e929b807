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

#include "coli_common.cuh"

namespace coli {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kGateUpRows = 2;   // rows per warp of each of gate and up
constexpr int kDownRows = 4;     // rows per warp of down

// Shared-memory image of TG activation vectors of length K, laid out so that
// lane l reading chunk c = l + 32 i, float4 j finds it at ((i * 8 + j) * 32 + l):
// conflict-free 16-byte loads.  m24[t][c] = -24 * (sum of the 32 values of chunk c).
struct StageGeom {
    int nch;       // chunks (32 values) per vector = K / 32
    int per_lane;  // ceil(nch / 32)
    int f4;        // float4 slots per vector = per_lane * 32 * 8
};

__host__ __device__ inline StageGeom stage_geom(int K)
{
    StageGeom g;
    g.nch = K / kChunkK;
    g.per_lane = (g.nch + 31) / 32;
    g.f4 = g.per_lane * 32 * 8;
    return g;
}

__host__ __device__ inline size_t stage_smem_bytes(int K, int TG)
{
    const StageGeom g = stage_geom(K);
    return (size_t)TG * g.f4 * 16 + (size_t)TG * g.nch * 4;
}

// Stage n vectors (rows tok[0..n) of src, K values each, fp32 or bf16) into xs/m24.
template <bool kBf16>
__device__ __forceinline__ void stage_vectors(const void* __restrict__ src, size_t row_elems,
                                              const int* tok, int n, const StageGeom& g,
                                              float4* xs, float* m24)
{
    const int total = n * g.nch * 8;
    const size_t esz = kBf16 ? 2 : 4;
    for (int base = 0; base < total; base += blockDim.x) {
        const int idx = base + threadIdx.x;
        const bool valid = idx < total;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        int t = 0, c = 0, j = 0;
        if (valid) {
            t = idx / (g.nch * 8);
            const int rem = idx - t * g.nch * 8;
            c = rem >> 3;
            j = rem & 7;
            const char* row = static_cast<const char*>(src) + (size_t)tok[t] * row_elems * esz;
            v = load_act4<kBf16>(row, c * kChunkK + j * 4);
            xs[(size_t)t * g.f4 + ((c >> 5) * 8 + j) * 32 + (c & 31)] = v;
        }
        float part = (v.x + v.y) + (v.z + v.w);
        part += __shfl_xor_sync(0xFFFFFFFFu, part, 1);
        part += __shfl_xor_sync(0xFFFFFFFFu, part, 2);
        part += __shfl_xor_sync(0xFFFFFFFFu, part, 4);
        if (valid && j == 0) m24[t * g.nch + c] = -24.f * part;
    }
}

template <int q>
__device__ __forceinline__ uint32_t word_of(const uint4& w)
{
    if constexpr (q == 0) return w.x;
    else if constexpr (q == 1) return w.y;
    else if constexpr (q == 2) return w.z;
    else return w.w;
}

// Accumulate, for NS row streams and up to TG staged vectors, the dot product of
// one 16-byte chunk (32 nibbles, k = 32c..32c+31) with the vectors:
//   sum_k q_k x_k = 16 * sum_k (1.5 + q_k/16) x_k - 24 * sum_k x_k,
// then scale by the row's group scale.
template <int NS, int TG>
__device__ __forceinline__ void chunk_dot(const uint4 (&w)[NS], const float (&sc)[NS],
                                          const float4* xs_i, int f4, const float* m24c, int nch,
                                          int ntok, float (&acc)[NS][TG])
{
#pragma unroll
    for (int t = 0; t < TG; ++t) {
        if (t < ntok) {
            float a[NS];
#pragma unroll
            for (int r = 0; r < NS; ++r) a[r] = 0.f;
            const float4* xt = xs_i + (size_t)t * f4;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const float4 xv = xt[jj * 32];
#pragma unroll
                for (int r = 0; r < NS; ++r) {
                    uint32_t wd;
                    if ((jj >> 1) == 0) wd = word_of<0>(w[r]);
                    else if ((jj >> 1) == 1) wd = word_of<1>(w[r]);
                    else if ((jj >> 1) == 2) wd = word_of<2>(w[r]);
                    else wd = word_of<3>(w[r]);
                    if (jj & 1) {
                        a[r] = fmaf(nib_as_float<4>(wd), xv.x, a[r]);
                        a[r] = fmaf(nib_as_float<5>(wd), xv.y, a[r]);
                        a[r] = fmaf(nib_as_float<6>(wd), xv.z, a[r]);
                        a[r] = fmaf(nib_as_float<7>(wd), xv.w, a[r]);
                    } else {
                        a[r] = fmaf(nib_as_float<0>(wd), xv.x, a[r]);
                        a[r] = fmaf(nib_as_float<1>(wd), xv.y, a[r]);
                        a[r] = fmaf(nib_as_float<2>(wd), xv.z, a[r]);
                        a[r] = fmaf(nib_as_float<3>(wd), xv.w, a[r]);
                    }
                }
            }
            const float m = m24c[t * nch];
#pragma unroll
            for (int r = 0; r < NS; ++r) acc[r][t] = fmaf(sc[r], fmaf(a[r], 16.f, m), acc[r][t]);
        }
    }
}

// Dot products of NS int4 rows (qrow[r]: packed bytes, srow[r]: scales) with
// ntok staged vectors, reduced over the warp: every lane returns the totals.
template <int NS, int TG>
__device__ __forceinline__ void rows_dot(const uint8_t* const (&qrow)[NS], const float* const (&srow)[NS],
                                         const StageGeom& g, const float4* xs, const float* m24,
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
        if (cn < g.nch) {  // prefetch the next chunk while this one is consumed
#pragma unroll
            for (int r = 0; r < NS; ++r) {
                wn[r] = ldg_stream(qrow[r] + (size_t)cn * 16);
                scn[r] = ldg_f32(srow[r] + (cn >> 1));
            }
        }
        if (c < g.nch)
            chunk_dot<NS, TG>(w, sc, xs + i * 256 + lane, g.f4, m24 + c, g.nch, ntok, acc);
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
    float* m24 = reinterpret_cast<float*>(smem + (size_t)TG * g.f4 * 16);
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
            if (kGateUp) stage_vectors<kBf16>(a.act, (size_t)a.K, tok, n, g, xs, m24);
            else stage_vectors<false>(a.act, (size_t)a.K, tok, n, g, xs, m24);
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
        rows_dot<NS, TG>(qrow, srow, g, xs, m24, n, acc);

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
template <bool kOutBf16>
__global__ void combine_kernel(const float* __restrict__ partial, const int32_t* __restrict__ inv_perm,
                               int T, int k, int H, void* __restrict__ out)
{
    const int P = T * k;
    const int per_row = H / 4;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * per_row) return;
    const int t = i / per_row;
    const int n = (i - t * per_row) * 4;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
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
