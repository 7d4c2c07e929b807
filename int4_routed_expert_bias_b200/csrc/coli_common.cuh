// coli_common.cuh -- small device helpers shared by the layer's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace coli {

constexpr int kGroup = 64;       // int4 scale group along K
constexpr int kChunkK = 32;      // K values in one 16-byte chunk of packed nibbles
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Sums of a and b over the warp in five exchanges: lane 0 ends with the sum of
// a, lane 16 with the sum of b.
__device__ __forceinline__ float warp_sum2(float a, float b)
{
    const bool hi = (threadIdx.x & 16) != 0;
    float v = (hi ? b : a) + __shfl_xor_sync(0xFFFFFFFFu, hi ? a : b, 16);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// floor(j / d) for 0 <= j <= j_max by a divisor fixed for the call: the high
// word of j * ceil(2^32 / d), exact while j_max * d < 2^32 (else a plain
// division is used).
struct FastDiv {
    uint32_t m;  // ceil(2^32 / d) (0 when d == 1)
    int d;
    bool exact;
    __device__ __forceinline__ FastDiv(int d_, long long j_max)
        : m(d_ > 1 ? (uint32_t)((0x100000000ull + (unsigned long long)d_ - 1ull) / (unsigned long long)d_) : 0u),
          d(d_), exact((unsigned long long)j_max * (unsigned long long)d_ < 0x100000000ull)
    {
    }
    __device__ __forceinline__ int operator()(int j) const
    {
        return !exact ? j / d : m ? (int)__umulhi((uint32_t)j, m) : j;
    }
};

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) { return __uint_as_float(b16 << 16); }

// fp32 -> bf16 bits, round to nearest even (inputs here are finite).
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Load 4 consecutive activations starting at element i of a row (fp32 or bf16),
// widened exactly to fp32.  i is a multiple of 4 and the row is 16-byte aligned.
template <bool kBf16>
__device__ __forceinline__ float4 load_act4(const void* row, int i)
{
    if constexpr (kBf16) {
        const uint2 v = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(row) + i);
        return make_float4(bf16_bits_to_float(v.x & 0xFFFFu), bf16_bits_to_float(v.x >> 16),
                           bf16_bits_to_float(v.y & 0xFFFFu), bf16_bits_to_float(v.y >> 16));
    } else {
        return *reinterpret_cast<const float4*>(static_cast<const float*>(row) + i);
    }
}

// Nibble m (bits 4m..4m+3) of a packed word as the float 1.5 + q/16, where q is
// the nibble read as a two's-complement integer in [-8, 7].  The nibble is moved
// to mantissa bits 19..22 of 1.0f with its top bit flipped (q + 8 = nibble ^ 8),
// giving 1 + (q + 8)/16 exactly.  So q = 16 * v - 24.
template <int m>
__device__ __forceinline__ float nib_as_float(uint32_t w)
{
    uint32_t t;
    if constexpr (4 * m <= 19) t = w << (19 - 4 * m);
    else t = w >> (4 * m - 19);
    return __uint_as_float((t & 0x00780000u) ^ 0x3FC00000u);
}

// Non-caching 16-byte load for weights streamed once from HBM.
__device__ __forceinline__ uint4 ldg_stream(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float ldg_f32(const float* p) { return __ldg(p); }

// Programmatic dependent launch: a kernel launched as a programmatic dependent
// waits here until its predecessor grid has completed and flushed its writes
// (a no-op when launched without the attribute); the predecessor may signal
// early that dependents can start launching.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__host__ __device__ __forceinline__ size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Index checks of the bounds-checked build (libcoli_bounds.so, compiled with
// COLI_DEBUG_BOUNDS): a failed check records status 4 in the call's status word
// and the caller skips the access; nothing traps.  In the normal build the
// check is the constant true and costs nothing.
#ifdef COLI_DEBUG_BOUNDS
__device__ __forceinline__ bool coli_in_bounds(bool ok, int* status)
{
    if (!ok && status) atomicExch(status, 4);
    return ok;
}
#define COLI_IN_BOUNDS(cond, status) ::coli::coli_in_bounds((cond), (status))
#else
#define COLI_IN_BOUNDS(cond, status) true
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Asynchronous global -> shared copies (cp.async): 16 bytes bypassing L1, 4 bytes
// through L1; completion is tracked per thread in commit groups.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's most recent commit groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace coli
