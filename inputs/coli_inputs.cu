// coli_inputs.cu -- host and device entry points of the synthetic weight generator.
//
// Input generation only (no layer arithmetic).  Both sides evaluate the same
// counter-based hash from gen_core.h, so a weight tensor generated on the GPU
// is bit-identical to the one generated on the host for the same
// (seed, layer, expert, tensor).  Layouts are the library's storage layout:
// q bytes [N, K/2] (low nibble = even k), scales fp32 [N, K/64].
#include <cuda_runtime.h>
#include <stdint.h>

#include "gen_core.h"

namespace {

__global__ void gen_q_kernel(uint64_t seed, uint32_t layer, uint32_t expert0, uint32_t tensor,
                             int64_t bytes_per_expert, uint32_t n_experts, uint8_t* q)
{
    const int64_t units_per_expert = bytes_per_expert / 16;
    const int64_t total = units_per_expert * n_experts;
    for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t e = (uint32_t)(u / units_per_expert);
        const int64_t local = u - (int64_t)e * units_per_expert;
        const uint64_t key = coli_gen_key(seed, layer, expert0 + e, tensor);
        const uint64_t j0 = (uint64_t)local * 8;  // 8 draws of 2 bytes each
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = coli_gen_bytes2(key, j0 + 2 * i) | (coli_gen_bytes2(key, j0 + 2 * i + 1) << 16);
        reinterpret_cast<uint4*>(q)[u] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__global__ void gen_s_kernel(uint64_t seed, uint32_t layer, uint32_t expert0, uint32_t tensor,
                             int64_t scales_per_expert, uint32_t n_experts, float* s)
{
    const int64_t total = scales_per_expert * n_experts;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t e = (uint32_t)(i / scales_per_expert);
        const int64_t local = i - (int64_t)e * scales_per_expert;
        s[i] = coli_gen_scale(coli_gen_key(seed, layer, expert0 + e, tensor), (uint64_t)local);
    }
}

}  // namespace

extern "C" {

// One matrix of one expert on the host.  which: 0 gate [N=F,K=H], 1 up, 2 down [N=H,K=F].
int coli_inputs_gen_matrix_host(uint64_t seed, uint32_t layer, uint32_t expert, uint32_t which,
                                int64_t N, int64_t K, uint8_t* q, float* s)
{
    if (!q || !s || which > 2 || N <= 0 || K <= 0 || K % 64 != 0) return -1;
    const uint64_t kq = coli_gen_key(seed, layer, expert, 2 * which);
    const uint64_t ks = coli_gen_key(seed, layer, expert, 2 * which + 1);
    const int64_t nbytes = N * K / 2;
    for (int64_t j = 0; j < nbytes / 2; ++j) {
        uint32_t b = coli_gen_bytes2(kq, (uint64_t)j);
        q[2 * j] = (uint8_t)(b & 0xFF);
        q[2 * j + 1] = (uint8_t)(b >> 8);
    }
    const int64_t nscales = N * K / 64;
    for (int64_t i = 0; i < nscales; ++i) s[i] = coli_gen_scale(ks, (uint64_t)i);
    return 0;
}

// The same matrix for experts [expert0, expert0 + n_experts) on the device, written
// contiguously (expert-major) into q [n_experts, N, K/2] and s [n_experts, N, K/64].
int coli_inputs_gen_matrix_device(uint64_t seed, uint32_t layer, uint32_t expert0,
                                  uint32_t n_experts, uint32_t which, int64_t N, int64_t K,
                                  uint8_t* q, float* s, void* stream)
{
    if (!q || !s || which > 2 || N <= 0 || K <= 0 || K % 64 != 0 || n_experts == 0) return -1;
    if (((uintptr_t)q & 15) != 0) return -1;
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t bpe = N * K / 2;
    const int64_t spe = N * K / 64;
    const int threads = 256;
    const int64_t qunits = bpe / 16 * n_experts;
    const int64_t sunits = spe * n_experts;
    const int qblocks = (int)((qunits + threads - 1) / threads < 148 * 64 ? (qunits + threads - 1) / threads : 148 * 64);
    const int sblocks = (int)((sunits + threads - 1) / threads < 148 * 64 ? (sunits + threads - 1) / threads : 148 * 64);
    gen_q_kernel<<<qblocks, threads, 0, st>>>(seed, layer, expert0, 2 * which, bpe, n_experts, q);
    gen_s_kernel<<<sblocks, threads, 0, st>>>(seed, layer, expert0, 2 * which + 1, spe, n_experts, s);
    return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

}  // extern "C"
