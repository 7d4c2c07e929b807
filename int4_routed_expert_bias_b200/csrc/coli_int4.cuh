// coli_int4.cuh -- int4-gs64 dot products on CUDA cores (decode path building blocks).
//
// Weights are stored as int4 with one fp32 scale per 64 along K ("gs64 build",
// "colibri: 744B MoEをストレージから推論するCエンジン", section はじめにとソースが語らないこと);
// decode keeps the arithmetic in fp32 ("Colibri 完全ガイド", section 詳細解説 step 3).
//
// Nibble -> float without an int->float conversion.  One shift of a packed
// word w puts two neighbouring nibbles into two mantissa windows of 1.0f:
//   window A, bits 19..22:  fa = 1 + (q_a + 8) / 16
//   window B, bits 15..18:  fb = 1 + (q_b + 8) / 256
// (the nibble's top bit is flipped, so q + 8 = nibble ^ 8 for two's complement).
// The four shifts w<<15, w<<7, w>>1 and w>>9 place nibbles (1,0), (3,2), (5,4)
// and (7,6) into (A,B); each float is one lop3, so a word costs 4 shifts and
// 8 lop3 on the integer pipe.  A packed fp32x2 FMA then takes one odd-k and
// one even-k product.  Over a chunk of 32 k values:
//   sum_k q_k x_k = 16 * sum_odd fa x + 256 * sum_even fb x
//                   - 24 * sum_odd x - 264 * sum_even x,
// the last two terms coming from the staged activations.  Window B keeps every
// product exact to 2^-16 of |x|, far inside fp32-accumulate tolerances.
#pragma once

#include "coli_common.cuh"

namespace coli {

// (a & b) ^ c in one instruction
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ float2 nib_pair(uint32_t s)
{
    return make_float2(__uint_as_float(and_xor(s, 0x00780000u, 0x3FC00000u)),
                       __uint_as_float(and_xor(s, 0x00078000u, 0x3F840000u)));
}

// Accumulate one packed word (k = 8q .. 8q+7 of a chunk) against activations
// staged as swapped pairs: x01 = (x[8q+1], x[8q]), x23 = (x[8q+3], x[8q+2]), ...
__device__ __forceinline__ float2 word_dot(uint32_t w, float4 xlo, float4 xhi, float2 acc)
{
    acc = __ffma2_rn(nib_pair(w << 15), make_float2(xlo.x, xlo.y), acc);
    acc = __ffma2_rn(nib_pair(w << 7), make_float2(xlo.z, xlo.w), acc);
    acc = __ffma2_rn(nib_pair(w >> 1), make_float2(xhi.x, xhi.y), acc);
    acc = __ffma2_rn(nib_pair(w >> 9), make_float2(xhi.z, xhi.w), acc);
    return acc;
}

// total += scale * (sum_k q_k x_k) for one chunk, given its accumulators and the
// chunk's correction corr = -24 * sum_odd x - 264 * sum_even x.
__device__ __forceinline__ float chunk_finish(float2 acc, float corr, float scale, float total)
{
    return fmaf(scale, fmaf(acc.x, 16.f, fmaf(acc.y, 256.f, corr)), total);
}

// Per-lane accumulation of NS rows' chunks against one staged chunk; each x
// slot is loaded once and used for every row.  xrow = the staged vector's
// float4 row block of this lane's chunk (xs + i * 256), slot j at
// xrow[j * 32 + (lane ^ j)].
template <int NS>
__device__ __forceinline__ void chunk_acc_rows(const uint4 (&w)[NS], const float4* xrow, int lane,
                                               float2 (&acc)[NS])
{
#pragma unroll
    for (int r = 0; r < NS; ++r) acc[r] = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 xlo = xrow[(2 * q) * 32 + (lane ^ (2 * q))];
        const float4 xhi = xrow[(2 * q + 1) * 32 + (lane ^ (2 * q + 1))];
#pragma unroll
        for (int r = 0; r < NS; ++r) {
            const uint32_t wd = q == 0 ? w[r].x : q == 1 ? w[r].y : q == 2 ? w[r].z : w[r].w;
            acc[r] = word_dot(wd, xlo, xhi, acc[r]);
        }
    }
}

// Same, with the lane's 8 swizzled slot offsets (slot j of row block 0 at
// xrow[off[j]], off[j] = j * 32 + (lane ^ j)) computed once by the caller.
template <int NS>
__device__ __forceinline__ void chunk_acc_rows_off(const uint4 (&w)[NS], const float4* xrow, const int (&off)[8],
                                                   float2 (&acc)[NS])
{
#pragma unroll
    for (int r = 0; r < NS; ++r) acc[r] = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 xlo = xrow[off[2 * q]];
        const float4 xhi = xrow[off[2 * q + 1]];
#pragma unroll
        for (int r = 0; r < NS; ++r) {
            const uint32_t wd = q == 0 ? w[r].x : q == 1 ? w[r].y : q == 2 ? w[r].z : w[r].w;
            acc[r] = word_dot(wd, xlo, xhi, acc[r]);
        }
    }
}

// ---------------------------------------------------------------------------
// Staging of activation vectors in shared memory.
//
// One vector of K values becomes K/4 float4 slots: chunk c (32 values), slot
// j (values 4j..4j+3 of the chunk) lives at ((c / 32) * 8 + j) * 32 + ((c % 32) ^ j).
// Lane l reading chunk c = l + 32 i, slot j touches 32 distinct 16-byte words of
// one 512-byte row, and the staging threads (8 consecutive threads per chunk,
// one per slot) write distinct banks: both directions are conflict-free.
// Each slot holds the swapped pairs (x1, x0, x3, x2).
// corr[c] = -24 * (odd-k sum) - 264 * (even-k sum) of chunk c.

struct StageGeom {
    int nch;       // chunks per vector = K / 32
    int per_lane;  // ceil(nch / 32)
    int f4;        // float4 slots per vector = per_lane * 256
};

__host__ __device__ inline StageGeom stage_geom(int K)
{
    StageGeom g;
    g.nch = K / kChunkK;
    g.per_lane = (g.nch + 31) / 32;
    g.f4 = g.per_lane * 256;
    return g;
}

__host__ __device__ inline size_t stage_smem_bytes(int K, int n_vectors)
{
    const StageGeom g = stage_geom(K);
    return (size_t)n_vectors * g.f4 * 16 + (size_t)n_vectors * g.nch * 4;
}

// Stage n vectors; load(t, i) returns values i..i+3 of vector t (fp32).
// Threads tid = 0 .. nthr-1 (whole warps) share the work; each has kU loads in
// flight before it stores.  All nthr threads must call this (it uses warp
// shuffles).
template <typename Load4>
__device__ __forceinline__ void stage_vectors_part(int n, Load4 load, const StageGeom& g, float4* xs, float* corr,
                                                   int tid, int nthr)
{
    constexpr int kU = 8;
    const int total = n * g.nch * 8;
    for (int base = 0; base < total; base += kU * nthr) {
        float4 v[kU];
#pragma unroll
        for (int r = 0; r < kU; ++r) {
            const int idx = base + r * nthr + tid;
            v[r] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (idx < total) {
                const int t = idx / (g.nch * 8);
                const int rem = idx - t * g.nch * 8;
                v[r] = load(t, (rem >> 3) * kChunkK + (rem & 7) * 4);
            }
        }
#pragma unroll
        for (int r = 0; r < kU; ++r) {
            const int idx = base + r * nthr + tid;
            const bool valid = idx < total;
            int t = 0, c = 0, j = 0;
            if (valid) {
                t = idx / (g.nch * 8);
                const int rem = idx - t * g.nch * 8;
                c = rem >> 3;
                j = rem & 7;
                xs[(size_t)t * g.f4 + ((c >> 5) * 8 + j) * 32 + ((c & 31) ^ j)] =
                    make_float4(v[r].y, v[r].x, v[r].w, v[r].z);
            }
            float odd = v[r].y + v[r].w, even = v[r].x + v[r].z;
            odd += __shfl_xor_sync(0xFFFFFFFFu, odd, 1);
            even += __shfl_xor_sync(0xFFFFFFFFu, even, 1);
            odd += __shfl_xor_sync(0xFFFFFFFFu, odd, 2);
            even += __shfl_xor_sync(0xFFFFFFFFu, even, 2);
            odd += __shfl_xor_sync(0xFFFFFFFFu, odd, 4);
            even += __shfl_xor_sync(0xFFFFFFFFu, even, 4);
            if (valid && j == 0) corr[t * g.nch + c] = fmaf(-24.f, odd, -264.f * even);
        }
    }
}

// ---------------------------------------------------------------------------
// Integer-dot form of the one-vector products.
//
// An activation chunk of 32 values is held as 21-bit fixed point over one
// power-of-two chunk scale: with m = max |x| < 2^e,
//   X = round(x * 2^(21 - e)),  |X| < 2^21,   x_hat = 2^(e - 21) X,
// so |x - x_hat| <= 2^(e - 22) <= 2^-21 m.  X is stored as three 8-bit digit
// planes, its two's-complement bit slices X = 16384 d0 + 128 d1 + d2 (d0 the
// signed top byte, d1 and d2 seven unsigned bits each).  An int4 word becomes
// biased bytes n = q + 8 in [0, 15] with three integer operations (lo:
// nibbles 0, 2, 4, 6; hi: nibbles 1, 3, 5, 7), and dp4a sums n * d exactly in
// int32 per plane.  Per chunk and row:
//   sum_k q_k x_hat_k = 2^(e - 21) * (D - corr),
//   D = sum_k n_k X_k = 16384 D0 + 128 D1 + D2,  corr = 8 * sum_k X_k,
// an exact integer below 2^29 in magnitude, converted to fp32 once.  The
// integer products leave the float pipes free and take far fewer issue slots
// than decoding nibbles to floats.
//
// The integer-activation variant (int8 activations) uses the first plane pair
// only: d0 = round(x * 127 / m), scale m / 127 (the pages' integer dot-product
// kernel, "Colibri 完全ガイド", section コア技術のハイライト).
//
// Shared-memory layout of one staged vector with nd digits (np = 2 nd planes):
// chunk c = l + 32 i, plane p = 2 * digit + (0: lo, 1: hi), as uint4 at
// ((i * np + p) * 32 + l); word w of the uint4 covers k = 8 w .. 8 w + 7 of
// the chunk, byte b of a lo (hi) word holds the digit of k = 8 w + 2 b (+ 1).
// Per chunk one float2: (2^(e - 21), corr as int bits).
__host__ __device__ constexpr int digit_planes(int nd) { return 2 * nd; }

__host__ __device__ inline int digit_vec_units(int K, int nd)  // 16-byte units per staged vector
{
    return stage_geom(K).per_lane * digit_planes(nd) * 32;
}

__host__ __device__ inline size_t digit_smem_bytes(int K, int n_vectors, int nd)
{
    return (size_t)n_vectors * digit_vec_units(K, nd) * 16 + (size_t)n_vectors * (K / kChunkK) * 8;
}

// biased bytes q + 8 of nibbles 0, 2, 4, 6 (lo) and 1, 3, 5, 7 (hi) of a word
__device__ __forceinline__ uint32_t nib_lo_u8(uint32_t w)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(w), "r"(0x0F0F0F0Fu), "r"(0x08080808u));
    return d;
}
__device__ __forceinline__ uint32_t nib_hi_u8(uint32_t w) { return nib_lo_u8(w >> 4); }

// c + sum of the four products of unsigned bytes of a and signed bytes of b
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// low bytes of a, b, c, d as one word (a in byte 0)
__device__ __forceinline__ uint32_t pack_lo_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Stage n vectors of K values (rows of src, fp32 or bf16) as digit planes: vector
// t is row row0 + t of src, or row tbl[t] / tdiv when tbl is given.  One thread
// encodes one chunk.  Threads tid = 0 .. nthr-1 share the work.  Not inlined:
// one copy of the code serves every call site.
static __device__ __noinline__ void stage_rows_digits(const void* __restrict__ src, int bf16, int K, int n, int row0,
                                                      const int* tbl, int tdiv, uint4* xd, float2* xc, int tid,
                                                      int nthr)
{
    constexpr int ND = 3;  // digits per value
    const int nch = K / kChunkK;
    const int vunits = digit_vec_units(K, ND);
    const size_t row_bytes = (size_t)K * (bf16 ? 2 : 4);
    for (int idx = tid; idx < n * nch; idx += nthr) {
        const int t = idx / nch, c = idx - t * nch;
        const int row = tbl ? tbl[t] / tdiv : row0 + t;
        const char* rp = static_cast<const char*>(src) + (size_t)row * row_bytes;
        float x[32];
        if (bf16) {
            const uint4* p4 = reinterpret_cast<const uint4*>(rp + (size_t)c * kChunkK * 2);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v = p4[j];
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    x[8 * j + 2 * h] = bf16_bits_to_float(u[h] & 0xFFFFu);
                    x[8 * j + 2 * h + 1] = bf16_bits_to_float(u[h] >> 16);
                }
            }
        } else {
            const float4* p4 = reinterpret_cast<const float4*>(rp + (size_t)c * kChunkK * 4);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 v = p4[j];
                x[4 * j] = v.x;
                x[4 * j + 1] = v.y;
                x[4 * j + 2] = v.z;
                x[4 * j + 3] = v.w;
            }
        }
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(x[j]));
        const bool finite = m <= 3.402823466e38f;  // false for inf and NaN
        const int ex = (int)(__float_as_uint(m) >> 23);
        // chunks whose largest magnitude is below 2^-100 contribute nothing (their products are far below any
        // fp32 rounding of the result); e = ex - 126 gives m < 2^e
        const bool live = finite && ex >= 26;
        const int e = live ? ex - 126 : 0;
        const float mult = live ? __uint_as_float((uint32_t)(148 - e) << 23) : 0.f;  // 2^(21 - e)
        uint32_t X[32];
        int csum = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            // round(x * 2^(21 - e)) by the 1.5 * 2^23 addition (|product| < 2^21 + 1 keeps it exact)
            const int v = __float_as_int(fmaf(x[j], mult, 12582912.0f)) - 0x4B400000;
            const int vc = min(v, (1 << 21) - 1);  // a value rounding up to 2^21 is held at the top code
            X[j] = (uint32_t)vc;
            csum += vc;
        }
        uint4* base = xd + (size_t)t * vunits + (size_t)(c >> 5) * digit_planes(ND) * 32 + (c & 31);
        uint32_t lo[4], hi[4];
        // plane d2: bits 0-6; d1: bits 7-13; d0: bits 14-21 (signed)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            lo[w] = pack_lo_bytes(X[8 * w], X[8 * w + 2], X[8 * w + 4], X[8 * w + 6]) & 0x7F7F7F7Fu;
            hi[w] = pack_lo_bytes(X[8 * w + 1], X[8 * w + 3], X[8 * w + 5], X[8 * w + 7]) & 0x7F7F7F7Fu;
        }
        base[4 * 32] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        base[5 * 32] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            lo[w] = pack_lo_bytes(X[8 * w] >> 7, X[8 * w + 2] >> 7, X[8 * w + 4] >> 7, X[8 * w + 6] >> 7) & 0x7F7F7F7Fu;
            hi[w] = pack_lo_bytes(X[8 * w + 1] >> 7, X[8 * w + 3] >> 7, X[8 * w + 5] >> 7, X[8 * w + 7] >> 7) &
                    0x7F7F7F7Fu;
        }
        base[2 * 32] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        base[3 * 32] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            lo[w] = pack_lo_bytes(X[8 * w] >> 14, X[8 * w + 2] >> 14, X[8 * w + 4] >> 14, X[8 * w + 6] >> 14);
            hi[w] = pack_lo_bytes(X[8 * w + 1] >> 14, X[8 * w + 3] >> 14, X[8 * w + 5] >> 14, X[8 * w + 7] >> 14);
        }
        base[0 * 32] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        base[1 * 32] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        const float scale = !finite ? __int_as_float(0x7FC00000) : live ? __uint_as_float((uint32_t)(106 + e) << 23)
                                                                          : 0.f;
        xc[(size_t)t * nch + c] = make_float2(scale, __int_as_float(8 * csum));
    }
}

// Two-digit staging for bf16 activations: 14-bit fixed point plus sign over the
// chunk's power-of-two scale, X = round(x * 2^(14 - e)) held at 2^14 - 1, as
// X = 128 d0 + d1 (d0 the signed top byte, d1 seven unsigned bits) in the
// first two plane pairs, and a float2 (2^(e - 14), 8 * sum X) per chunk.  The
// rounding error, at most 2^-15 m per value, stays far below the bf16 rounding
// (up to 2^-9 |x|) that the activations already carry, and it takes two dp4a
// planes instead of three.  Chunk rules as in stage_rows_digits.
static __device__ __noinline__ void stage_rows_digits2(const void* __restrict__ src, int bf16, int K, int n, int row0,
                                                       const int* tbl, int tdiv, uint4* xd, float2* xc, int tid,
                                                       int nthr)
{
    constexpr int ND = 2;  // digits per value
    const int nch = K / kChunkK;
    const int vunits = digit_vec_units(K, ND);
    const size_t row_bytes = (size_t)K * (bf16 ? 2 : 4);
    for (int idx = tid; idx < n * nch; idx += nthr) {
        const int t = idx / nch, c = idx - t * nch;
        const int row = tbl ? tbl[t] / tdiv : row0 + t;
        const char* rp = static_cast<const char*>(src) + (size_t)row * row_bytes;
        float x[32];
        if (bf16) {
            const uint4* p4 = reinterpret_cast<const uint4*>(rp + (size_t)c * kChunkK * 2);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v = p4[j];
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    x[8 * j + 2 * h] = bf16_bits_to_float(u[h] & 0xFFFFu);
                    x[8 * j + 2 * h + 1] = bf16_bits_to_float(u[h] >> 16);
                }
            }
        } else {
            const float4* p4 = reinterpret_cast<const float4*>(rp + (size_t)c * kChunkK * 4);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 v = p4[j];
                x[4 * j] = v.x;
                x[4 * j + 1] = v.y;
                x[4 * j + 2] = v.z;
                x[4 * j + 3] = v.w;
            }
        }
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(x[j]));
        const bool finite = m <= 3.402823466e38f;  // false for inf and NaN
        const int ex = (int)(__float_as_uint(m) >> 23);
        const bool live = finite && ex >= 26;  // m >= 2^-100, as in stage_rows_digits
        const int e = live ? ex - 126 : 0;     // m < 2^e
        const float mult = live ? __uint_as_float((uint32_t)(141 - e) << 23) : 0.f;  // 2^(14 - e)
        uint32_t X[32];
        int csum = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int v = __float_as_int(fmaf(x[j], mult, 12582912.0f)) - 0x4B400000;
            const int vc = min(v, (1 << 14) - 1);
            X[j] = (uint32_t)vc;
            csum += vc;
        }
        uint4* base = xd + (size_t)t * vunits + (size_t)(c >> 5) * digit_planes(ND) * 32 + (c & 31);
        uint32_t lo[4], hi[4];
        // plane d1: bits 0-6; d0: bits 7-14 (signed)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            lo[w] = pack_lo_bytes(X[8 * w], X[8 * w + 2], X[8 * w + 4], X[8 * w + 6]) & 0x7F7F7F7Fu;
            hi[w] = pack_lo_bytes(X[8 * w + 1], X[8 * w + 3], X[8 * w + 5], X[8 * w + 7]) & 0x7F7F7F7Fu;
        }
        base[2 * 32] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        base[3 * 32] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            lo[w] = pack_lo_bytes(X[8 * w] >> 7, X[8 * w + 2] >> 7, X[8 * w + 4] >> 7, X[8 * w + 6] >> 7);
            hi[w] = pack_lo_bytes(X[8 * w + 1] >> 7, X[8 * w + 3] >> 7, X[8 * w + 5] >> 7, X[8 * w + 7] >> 7);
        }
        base[0 * 32] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        base[1 * 32] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        const float scale = !finite ? __int_as_float(0x7FC00000) : live ? __uint_as_float((uint32_t)(113 + e) << 23)
                                                                          : 0.f;
        xc[(size_t)t * nch + c] = make_float2(scale, __int_as_float(8 * csum));
    }
}

// The integer-activation variant's staging: one plane pair of symmetric int8
// codes per chunk, code = rint(x * (127 / m)) with m = max |x| of the chunk,
// scale m / 127 (a chunk whose 127 / m overflows fp32 is zero; one holding inf
// or NaN gets scale NaN).  Same layout as stage_rows_digits (first plane pair,
// a float2 (scale, 8 * sum of codes) per chunk).
static __device__ __noinline__ void stage_rows_int8(const void* __restrict__ src, int bf16, int K, int n, int row0,
                                                    const int* tbl, int tdiv, uint4* xd, float2* xc, int tid,
                                                    int nthr)
{
    constexpr int ND = 1;  // digits per value
    const int nch = K / kChunkK;
    const int vunits = digit_vec_units(K, ND);
    const size_t row_bytes = (size_t)K * (bf16 ? 2 : 4);
    for (int idx = tid; idx < n * nch; idx += nthr) {
        const int t = idx / nch, c = idx - t * nch;
        const int row = tbl ? tbl[t] / tdiv : row0 + t;
        const char* rp = static_cast<const char*>(src) + (size_t)row * row_bytes;
        float x[32];
        if (bf16) {
            const uint4* p4 = reinterpret_cast<const uint4*>(rp + (size_t)c * kChunkK * 2);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v = p4[j];
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    x[8 * j + 2 * h] = bf16_bits_to_float(u[h] & 0xFFFFu);
                    x[8 * j + 2 * h + 1] = bf16_bits_to_float(u[h] >> 16);
                }
            }
        } else {
            const float4* p4 = reinterpret_cast<const float4*>(rp + (size_t)c * kChunkK * 4);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 v = p4[j];
                x[4 * j] = v.x;
                x[4 * j + 1] = v.y;
                x[4 * j + 2] = v.z;
                x[4 * j + 3] = v.w;
            }
        }
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(x[j]));
        const bool finite = m <= 3.402823466e38f;  // false for inf and NaN
        const float inv = finite && m > 0.f ? 127.0f / m : 0.f;
        const bool live = inv > 0.f && inv <= 3.402823466e38f;
        uint32_t X[32];
        int csum = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int v = live ? (int)fminf(fmaxf(rintf(x[j] * inv), -127.f), 127.f) : 0;
            X[j] = (uint32_t)v;
            csum += v;
        }
        uint4* base = xd + (size_t)t * vunits + (size_t)(c >> 5) * digit_planes(ND) * 32 + (c & 31);
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            lo[w] = pack_lo_bytes(X[8 * w], X[8 * w + 2], X[8 * w + 4], X[8 * w + 6]);
            hi[w] = pack_lo_bytes(X[8 * w + 1], X[8 * w + 3], X[8 * w + 5], X[8 * w + 7]);
        }
        base[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        base[32] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        const float scale = !finite ? __int_as_float(0x7FC00000) : live ? m / 127.0f : 0.f;
        xc[(size_t)t * nch + c] = make_float2(scale, __int_as_float(8 * csum));
    }
}

// The same with every thread of the block.
template <typename Load4>
__device__ __forceinline__ void stage_vectors_fn(int n, Load4 load, const StageGeom& g, float4* xs, float* corr)
{
    stage_vectors_part(n, load, g, xs, corr, (int)threadIdx.x, (int)blockDim.x);
}

// Stage n vectors; vector v is row rows(v) of src (K values each, fp32 or bf16).
template <bool kBf16, typename RowOf>
__device__ __forceinline__ void stage_vectors(const void* __restrict__ src, int K, int n, RowOf rows,
                                              const StageGeom& g, float4* xs, float* corr, int tid = -1,
                                              int nthr = 0)
{
    const size_t row_bytes = (size_t)K * (kBf16 ? 2 : 4);
    auto load = [&](int t, int i) {
        return load_act4<kBf16>(static_cast<const char*>(src) + (size_t)rows(t) * row_bytes, i);
    };
    if (tid < 0) stage_vectors_fn(n, load, g, xs, corr);
    else stage_vectors_part(n, load, g, xs, corr, tid, nthr);
}

}  // namespace coli
