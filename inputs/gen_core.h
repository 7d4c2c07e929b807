/*
 * gen_core.h -- counter-based generator of synthetic int4-gs64 expert weights.
 *
 * Input generation only: this header encodes random bytes in the storage
 * format and performs none of the layer's arithmetic.  It compiles as plain C
 * for the host and as CUDA for the device, so both sides produce bit-identical
 * weights from (seed, layer, expert, tensor, index) without copying them.
 *
 * Hash: the SplitMix64 output function of Steele, Lea & Flood, "Fast
 * splittable pseudorandom number generators" (OOPSLA 2014), applied to a
 * counter advanced by the 64-bit golden-ratio increment.
 *
 * Nibbles: each 64-bit hash yields four 16-bit uniforms u; a nibble value is
 * -8 + #{i : u >= COLI_GEN_CDF[i]}, i.e. rint(2.9 * Z) for Z ~ N(0,1) clamped
 * to [-8, 7] (thresholds = round(65536 * Phi((m + 0.5) / 2.9)), m = -8..6).
 * Scales: s = (3072 + (h mod 1024)) * 2^-19, exact in fp32, so the weight
 * standard deviation is about 2.9 * 0.0068 = 0.02.
 */
#ifndef COLI_GEN_CORE_H
#define COLI_GEN_CORE_H

#include <stdint.h>

#if defined(__CUDACC__)
#define COLI_GEN_HD __host__ __device__ __forceinline__
#else
#define COLI_GEN_HD static inline
#endif

#define COLI_GEN_GOLDEN 0x9E3779B97F4A7C15ULL

/* tensor ids inside one expert */
enum { COLI_GEN_GATE_Q = 0, COLI_GEN_GATE_S = 1, COLI_GEN_UP_Q = 2, COLI_GEN_UP_S = 3,
       COLI_GEN_DOWN_Q = 4, COLI_GEN_DOWN_S = 5 };

COLI_GEN_HD uint64_t coli_gen_mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Stream key of one tensor. */
COLI_GEN_HD uint64_t coli_gen_key(uint64_t seed, uint32_t layer, uint32_t expert, uint32_t tensor)
{
    uint64_t k = coli_gen_mix64(seed + COLI_GEN_GOLDEN);
    k = coli_gen_mix64(k ^ ((uint64_t)layer << 32 | (uint64_t)expert));
    return coli_gen_mix64(k + (uint64_t)(tensor + 1) * COLI_GEN_GOLDEN);
}

/* i-th 64-bit draw of a stream. */
COLI_GEN_HD uint64_t coli_gen_draw(uint64_t key, uint64_t i)
{
    return coli_gen_mix64(key + (i + 1) * COLI_GEN_GOLDEN);
}

/* 16-bit uniform -> nibble value in [-8, 7] (two's-complement low 4 bits returned). */
COLI_GEN_HD uint32_t coli_gen_nibble(uint32_t u)
{
    int v = -8;
    v += (u >= 318u);   v += (u >= 819u);   v += (u >= 1897u);  v += (u >= 3956u);
    v += (u >= 7454u);  v += (u >= 12735u); v += (u >= 19824u); v += (u >= 28282u);
    v += (u >= 37254u); v += (u >= 45712u); v += (u >= 52801u); v += (u >= 58082u);
    v += (u >= 61580u); v += (u >= 63639u); v += (u >= 64717u);
    return (uint32_t)v & 0xFu;
}

/* Two packed bytes (nibbles 4j..4j+3, low nibble first) from draw j. */
COLI_GEN_HD uint32_t coli_gen_bytes2(uint64_t key, uint64_t j)
{
    uint64_t h = coli_gen_draw(key, j);
    uint32_t n0 = coli_gen_nibble((uint32_t)(h & 0xFFFF));
    uint32_t n1 = coli_gen_nibble((uint32_t)((h >> 16) & 0xFFFF));
    uint32_t n2 = coli_gen_nibble((uint32_t)((h >> 32) & 0xFFFF));
    uint32_t n3 = coli_gen_nibble((uint32_t)((h >> 48) & 0xFFFF));
    return (n0 | (n1 << 4)) | ((n2 | (n3 << 4)) << 8);
}

/* Scale number i of a stream: (3072 + (h mod 1024)) * 2^-19, exact in fp32. */
COLI_GEN_HD float coli_gen_scale(uint64_t key, uint64_t i)
{
    uint64_t h = coli_gen_draw(key, i);
    return (float)(3072u + (uint32_t)(h & 1023u)) * (1.0f / 524288.0f);
}

#endif /* COLI_GEN_CORE_H */
