// coli.cu -- C ABI of the routed-expert MoE layer (see include/coli.h).
//
// Host side: argument checks (before anything is enqueued), workspace layout,
// kernel selection and launch order.  Every step of the layer runs in the
// kernels of this library; there is no CPU fallback.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "coli.h"
#include "coli_common.cuh"
#include "coli_decode.cuh"
#include "coli_layer.cuh"
#include "coli_prefill.cuh"
#include "coli_router.cuh"
#include "coli_union.cuh"

using namespace coli;

namespace {

thread_local char g_err[512] = "";

// Test hook: device buffer for the decode kernel's per-CTA phase stamps (null = off).
std::atomic<unsigned long long*> g_stamps{nullptr};

// Test hook: limit of the kernels' bounded waits (0 = the built-in limits).
std::atomic<unsigned long long> g_wait_ns{0};
unsigned long long wait_limit(unsigned long long dflt)
{
    const unsigned long long v = g_wait_ns.load(std::memory_order_relaxed);
    return v ? v : dflt;
}
thread_local cudaEvent_t* g_prof_events = nullptr;
thread_local int g_prof_n = 0;

coli_status fail(coli_status st, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

coli_status cuda_fail(cudaError_t e, const char* what)
{
    return fail(COLI_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

constexpr int kMaxTokens = 65536;

// Batches above this size take the tensor-core prefill path.
constexpr int kDecodeMaxT = 64;

coli_status check_sizes(int T, int H, int E, int k)
{
    if (T < 0 || T > kMaxTokens) return fail(COLI_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, kMaxTokens);
    if (H <= 0 || H % kGroup != 0) return fail(COLI_ERR_INVALID_ARG, "hidden=%d is not a positive multiple of 64", H);
    if (k < 1 || k > kMaxTopK) return fail(COLI_ERR_INVALID_ARG, "top_k=%d outside [1, %d]", k, kMaxTopK);
    if (E < k || E > kMaxExperts) return fail(COLI_ERR_INVALID_ARG, "n_experts=%d outside [top_k=%d, %d]", E, k, kMaxExperts);
    return COLI_OK;
}

// Per-device launch facts, filled on first use: SM count, and the dynamic
// shared-memory limit that every staged-activation kernel is opted in to.
struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int smem_optin = 0;
    // decode-kernel residency already checked on this device: (kernel, dynamic shared memory) pairs
    static constexpr int kFitSlots = 64;
    const void* fit_kern[kFitSlots] = {};
    size_t fit_bytes[kFitSlots] = {};
    int n_fit = 0;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

constexpr int kMaxStageK = 16384;  // largest hidden / ffn width accepted

// Dynamic shared memory the decode-layer kernel may use (it has no static shared
// memory): sm_100's 227 KB per block, less 1 KB of slack.
constexpr int kSmemBudget = 232448 - 1024;
size_t gateup_smem(int H, int TG) { return stage_smem_bytes(H, TG); }
size_t down_smem(int F, int TG) { return stage_smem_bytes(F, TG); }

template <typename Kern>
cudaError_t allow_smem(Kern k, int bytes)
{
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// The fused decode-layer kernel, one instantiation per (tokens per group,
// activation dtype, output dtype, one-token output-row mode, int8 activations).
using LayerKernel = void (*)(const LayerArgs, const LayerSmem);
template <int MT, bool kRows, bool kI8>
LayerKernel layer_kernel_dtypes(bool bf16, bool out_bf16)
{
    if (bf16)
        return out_bf16 ? moe_layer_kernel<MT, true, true, kRows, kI8> : moe_layer_kernel<MT, true, false, kRows, kI8>;
    return out_bf16 ? moe_layer_kernel<MT, false, true, kRows, kI8> : moe_layer_kernel<MT, false, false, kRows, kI8>;
}

LayerKernel layer_kernel(int MT, bool bf16, bool out_bf16, bool out_rows, bool i8)
{
    if (MT == 4)
        return i8 ? layer_kernel_dtypes<4, false, true>(bf16, out_bf16) : layer_kernel_dtypes<4, false, false>(bf16, out_bf16);
    if (out_rows)
        return i8 ? layer_kernel_dtypes<1, true, true>(bf16, out_bf16) : layer_kernel_dtypes<1, true, false>(bf16, out_bf16);
    return i8 ? layer_kernel_dtypes<1, false, true>(bf16, out_bf16) : layer_kernel_dtypes<1, false, false>(bf16, out_bf16);
}

cudaError_t allow_layer_kernels(int bytes)
{
    const int mts[2] = {1, 4};
    for (int mt : mts)
        for (int rows = 0; rows < 2; ++rows)
            for (int b = 0; b < 8; ++b) {
                if (mt == 4 && rows) continue;
                const cudaError_t e = cudaFuncSetAttribute(layer_kernel(mt, b & 1, b & 2, rows, b & 4),
                                                           cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
                if (e != cudaSuccess) return e;
            }
    return cudaSuccess;
}

coli_status device_info(DeviceInfo** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(COLI_ERR_UNSUPPORTED, "device %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        const int lim = d.smem_optin - 8192;  // room for the kernels' static shared memory
        if ((e = allow_smem(expert_phase_kernel<true, false, 1>, lim)) != cudaSuccess ||
            (e = allow_smem(expert_phase_kernel<true, false, 4>, lim)) != cudaSuccess ||
            (e = allow_smem(expert_phase_kernel<true, true, 1>, lim)) != cudaSuccess ||
            (e = allow_smem(expert_phase_kernel<true, true, 4>, lim)) != cudaSuccess ||
            (e = allow_smem(expert_phase_kernel<false, false, 1>, lim)) != cudaSuccess ||
            (e = allow_smem(expert_phase_kernel<false, false, 4>, lim)) != cudaSuccess ||
            (e = allow_layer_kernels(std::min(d.smem_optin, kSmemBudget))) != cudaSuccess ||  // no static smem
            (kPfSmemBytes <= (size_t)lim &&
             ((e = allow_smem(prefill_gemm_kernel<true>, (int)kPfSmemBytes)) != cudaSuccess ||
              (e = allow_smem(prefill_gemm_kernel<false>, (int)kPfSmemBytes)) != cudaSuccess)))
            return cuda_fail(e, "kernel attribute setup");
        d.smem_optin = lim;
        d.ready = true;
    }
    *out = &d;
    return COLI_OK;
}

// Resident blocks per SM for the actual dynamic smem of one launch.
template <typename Kern>
int blocks_per_sm(Kern k, size_t smem, int threads = kDecThreads)
{
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, threads, smem) != cudaSuccess) return 1;
    return occ > 0 ? occ : 1;
}

// Tokens per group of the expert phases: 4 when the staged activations fit.
int group_tokens(int T, int H, int F, int smem_limit)
{
    if (T == 1) return 1;
    if (gateup_smem(H, 4) <= (size_t)smem_limit && down_smem(F, 4) <= (size_t)smem_limit) return 4;
    return 1;
}

// ---------------------------------------------------------------------------
// workspace layout

struct Workspace {
    float* logits;      // [T, E]
    int32_t* idx;       // [P]
    float* w;           // [P]
    int32_t* count;     // [E]
    int32_t* offset;    // [E+1]
    int32_t* active;    // [E]
    int32_t* n_active;  // [1]
    int32_t* perm;      // [P]
    int32_t* inv_perm;  // [P]
    int32_t* pair_token;  // [P+T]
    float* pair_w;        // [P+T]
    int32_t* ctl;         // [4]
    int32_t* g_expert;    // [G]
    int32_t* g_start;
    int32_t* g_count;
    float* h;             // [P+T, F]
    float* partial;       // [P+T, H]
    int32_t* chunk;       // [ceil(P / kUnionChunk), E] union bucket counts / starts (large batches)
    int32_t* rank;        // [P] rank of each pair in its (chunk, expert) bucket
    size_t bytes;
};

Workspace layout(void* base, int T, int H, int F, int E, int k)
{
    Workspace w{};
    const size_t P = (size_t)T * k, Q = P + T, G = P + (size_t)E + T + 1;
    size_t off = 0;
    auto take = [&](size_t bytes) -> char* {
        char* p = base ? static_cast<char*>(base) + off : nullptr;
        off += align_up(bytes, 256);
        return p;
    };
    // router scores [T, E]; up to 4 tokens the decode kernel writes per-piece partials [pieces, T, E]
    w.logits = (float*)take((size_t)(T <= 4 ? stage_geom(H).per_lane : 1) * T * E * 4);
    w.idx = (int32_t*)take(P * 4);
    w.w = (float*)take(P * 4);
    w.count = (int32_t*)take((size_t)E * 4);
    w.offset = (int32_t*)take(((size_t)E + 1) * 4);
    w.active = (int32_t*)take((size_t)E * 4);
    w.n_active = (int32_t*)take(4);
    w.perm = (int32_t*)take(P * 4);
    w.inv_perm = (int32_t*)take(P * 4);
    w.pair_token = (int32_t*)take(Q * 4);
    w.pair_w = (float*)take(Q * 4);
    w.ctl = (int32_t*)take(16);
    w.g_expert = (int32_t*)take(G * 4);
    w.g_start = (int32_t*)take(G * 4);
    w.g_count = (int32_t*)take(G * 4);
    w.h = (float*)take(Q * F * 4);
    w.partial = (float*)take(Q * H * 4);
    const bool big = T > kDecodeMaxT;  // the chunked union of large batches
    w.chunk = (int32_t*)take(big ? (P + kUnionChunk - 1) / kUnionChunk * (size_t)E * 4 : 0);
    w.rank = (int32_t*)take(big ? P * 4 : 0);
    w.bytes = off;
    return w;
}

coli_status check_layer_fields(const coli_moe_layer* L, int T)
{
    if (!L) return fail(COLI_ERR_INVALID_ARG, "layer is NULL");
    coli_status st = check_sizes(T, L->hidden, L->n_experts, L->top_k);
    if (st != COLI_OK) return st;
    if (L->ffn <= 0 || L->ffn % kGroup != 0) return fail(COLI_ERR_INVALID_ARG, "ffn=%d is not a positive multiple of 64", L->ffn);
    if (L->group != kGroup) return fail(COLI_ERR_UNSUPPORTED, "group=%d (only 64 is supported)", L->group);
    if (L->hidden > kMaxStageK || L->ffn > kMaxStageK)
        return fail(COLI_ERR_UNSUPPORTED, "hidden=%d / ffn=%d above %d", L->hidden, L->ffn, kMaxStageK);
    if (!std::isfinite(L->routed_scale)) return fail(COLI_ERR_INVALID_ARG, "routed_scale is not finite");
    if (!(L->top_p >= 0.f) || !std::isfinite(L->top_p)) return fail(COLI_ERR_INVALID_ARG, "top_p is negative or not finite");
    if (L->act_int8 != 0 && L->act_int8 != 1) return fail(COLI_ERR_INVALID_ARG, "act_int8=%d (0 or 1)", L->act_int8);
    const void* ptrs[] = {L->w_router, L->sel_bias, L->gate_q, L->up_q, L->down_q, L->gate_s, L->up_s, L->down_s};
    const char* names[] = {"w_router", "sel_bias", "gate_q", "up_q", "down_q", "gate_s", "up_s", "down_s"};
    for (int i = 0; i < 8; ++i) {
        if (!ptrs[i]) return fail(COLI_ERR_INVALID_ARG, "layer.%s is NULL", names[i]);
        if (!aligned(ptrs[i], i == 1 ? 4 : 16)) return fail(COLI_ERR_INVALID_ARG, "layer.%s is not 16-byte aligned", names[i]);
    }
    return COLI_OK;
}

// The layer's fields, and those of the layer named for the router-lookahead prefetch (not followed further).
coli_status check_layer(const coli_moe_layer* L, int T)
{
    coli_status st = check_layer_fields(L, T);
    if (st != COLI_OK || !L->prefetch_next) return st;
    if ((st = check_layer_fields(L->prefetch_next, 1)) != COLI_OK) {
        char why[256];
        snprintf(why, sizeof why, "%s", coli_last_error());
        return fail(st, "prefetch_next: %s", why);
    }
    return COLI_OK;
}

// Byte ranges of layer N that the router-lookahead prefetch asks L2 for: its router weights and
// selection bias, and its shared expert's three matrices and their scales (16-byte aligned inside).
int lookahead_ranges(const coli_moe_layer* N, const unsigned char** base, unsigned long long* bytes)
{
    const size_t H = N->hidden, F = N->ffn, E = N->n_experts;
    const struct {
        const void* p;
        size_t off, n;
    } r[] = {{N->w_router, 0, E * H * 4},
             {N->sel_bias, 0, E * 4},
             {N->gate_q, E * F * (H / 2), F * (H / 2)},
             {N->up_q, E * F * (H / 2), F * (H / 2)},
             {N->down_q, E * H * (F / 2), H * (F / 2)},
             {N->gate_s, E * F * (H / kGroup) * 4, F * (H / kGroup) * 4},
             {N->up_s, E * F * (H / kGroup) * 4, F * (H / kGroup) * 4},
             {N->down_s, E * H * (F / kGroup) * 4, H * (F / kGroup) * 4}};
    int n = 0;
    for (const auto& x : r) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(x.p) + x.off;
        const uintptr_t lo = (a + 15) & ~(uintptr_t)15, hi = (a + x.n) & ~(uintptr_t)15;
        if (hi <= lo || n == kMaxPrefetch) continue;
        base[n] = reinterpret_cast<const unsigned char*>(lo);
        bytes[n] = hi - lo;
        ++n;
    }
    return n;
}

// Argument checks of a layer call other than its workspace (host only).
int choose_path(const coli_moe_layer* L, int T);

coli_status check_call(const coli_moe_layer* L, const void* x, coli_dtype xt, int T, const void* out, coli_dtype ot,
                       const int32_t* topk_idx_out, const float* topk_w_out)
{
    coli_status st = check_layer(L, T);
    if (st != COLI_OK) return st;
    if (xt != COLI_F32 && xt != COLI_BF16) return fail(COLI_ERR_INVALID_ARG, "unknown activation dtype %d", (int)xt);
    if (ot != COLI_F32 && ot != COLI_BF16) return fail(COLI_ERR_INVALID_ARG, "unknown output dtype %d", (int)ot);
    if (T == 0) return COLI_OK;
    if (L->act_int8) {
        const int p = choose_path(L, T);
        if (p != COLI_PATH_SINGLE && p != COLI_PATH_DECODE)
            return fail(COLI_ERR_UNSUPPORTED, "act_int8: the integer-activation variant runs in the fused decode kernel "
                                              "(batches of up to %d tokens)", kDecodeMaxT);
    }
    if (!x || !out) return fail(COLI_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(x, 16) || !aligned(out, 16)) return fail(COLI_ERR_INVALID_ARG, "x / out not 16-byte aligned");
    if ((topk_idx_out && !aligned(topk_idx_out, 4)) || (topk_w_out && !aligned(topk_w_out, 4)))
        return fail(COLI_ERR_INVALID_ARG, "routing outputs not 4-byte aligned");
    return COLI_OK;
}

struct StageTimer {
    cudaEvent_t* ev = nullptr;
    int n = 0;
    bool capturing = false;
    cudaStream_t s = nullptr;
    cudaError_t rec(int stage, int end)
    {
        const int i = 2 * stage + end;
        if (!ev || i >= n) return cudaSuccess;
        return capturing ? cudaEventRecordWithFlags(ev[i], s, cudaEventRecordExternal) : cudaEventRecord(ev[i], s);
    }
};

coli_status launch_logits(const void* x, coli_dtype xt, int T, int H, const float* w_router, int E,
                          float* logits, int32_t* zero_ctr, int n_zero, cudaStream_t s)
{
    dim3 grid(E, (T + kRouterTokens - 1) / kRouterTokens);
    if (xt == COLI_BF16)
        router_logits_kernel<true><<<grid, kRouterThreads, 0, s>>>(x, T, H, w_router, E, logits, zero_ctr, n_zero);
    else
        router_logits_kernel<false><<<grid, kRouterThreads, 0, s>>>(x, T, H, w_router, E, logits, zero_ctr, n_zero);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? COLI_OK : cuda_fail(e, "router launch");
}

// Launch as a programmatic dependent of the previous kernel on the stream: its
// launch may overlap the predecessor's tail; the kernel calls griddep_wait()
// before it reads anything the predecessor wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// cuTensorMapEncodeTiled from the CUDA driver, looked up once (the library links
// only the runtime).  nullptr when the CUDA driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Row-major 2-D tensor [rows, inner] of esize-byte elements, read in boxes of
// box_inner x box_rows.
bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, size_t esize, const void* base, uint64_t inner,
               uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * esize};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Maps of one expert matrix set: int4 bytes [(E+1) NW, K/2] and scales [(E+1) NW, K/64].
bool encode_weight_maps(CUtensorMap* q, CUtensorMap* s, const uint8_t* qp, const float* sp, int E, int NW, int K)
{
    const uint64_t rows = (uint64_t)(E + 1) * NW;
    return encode_2d(q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, qp, (uint64_t)K / 2, rows, kPfRawK / 2, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B) &&
           encode_2d(s, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, sp, (uint64_t)K / kGroup, rows, kPfRawK / kGroup, 64,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
}


// Batches up to this size take the top-k inside the union block.
constexpr int kFusedTopkMaxT = 256;

// The kernel chain a valid call of T tokens runs (coli_moe_path), from the
// shapes alone: every path's shared-memory needs fit the 227 KB per block of
// sm_100, which the device set-up checks once.
// The one-token output-row mode sizes its row buffer for GPUs of at least this many SMs.
constexpr int kMinLayerSms = 64;

// How the fused decode-layer kernel runs a batch: tokens per group (MT), the
// one-token output-row mode, and its shared memory; ok = false if it does not fit.
struct LayerPlan {
    bool ok = false;
    int MT = 1;
    bool out_rows = false;
    LayerSmem ls{};
};

// nd: digits per staged activation (3: fp32 activations, 2: bf16, 1: the int8 variant).
LayerPlan layer_plan(int T, int H, int F, int E, int k, int nd)
{
    LayerPlan p;
    if (T < 1 || T > kLayerMaxT) return p;
    const int ru = layer_rows(1, nd);  // one token: output rows are split in units of ru rows
    const int rows_per_cta = ru * ((H / ru + kMinLayerSms - 1) / kMinLayerSms);
    auto fits = [&](int MT, bool rows) {
        const LayerSmem ls = layer_smem(T, H, F, E, k, MT, rows, rows_per_cta, nd);
        if (ls.bytes > (size_t)kSmemBudget) return false;
        p.ok = true;
        p.MT = MT;
        p.out_rows = rows;
        p.ls = ls;
        return true;
    };
    if (T == 1) {
        if (fits(1, true) || fits(1, false)) return p;
        return p;
    }
    if (fits(4, false) || fits(1, false)) return p;
    return p;
}

int choose_path(const coli_moe_layer* L, int T)
{
    if (T == 0) return COLI_PATH_NONE;
    if (T <= kDecodeMaxT) {
        // the path does not depend on the activations' type: plan with the largest staging (fp32)
        const LayerPlan pl = layer_plan(T, L->hidden, L->ffn, L->n_experts, L->top_k, L->act_int8 ? 1 : 3);
        if (pl.ok) return pl.out_rows ? COLI_PATH_SINGLE : COLI_PATH_DECODE;
    }
    if (T > kDecodeMaxT && L->hidden % kPfRawK == 0 && L->ffn % kPfRawK == 0) return COLI_PATH_PREFILL;
    return COLI_PATH_WIDE;
}

}  // namespace

extern "C" {

const char* coli_status_string(coli_status st)
{
    switch (st) {
        case COLI_OK: return "COLI_OK";
        case COLI_ERR_INVALID_ARG: return "COLI_ERR_INVALID_ARG";
        case COLI_ERR_UNSUPPORTED: return "COLI_ERR_UNSUPPORTED";
        case COLI_ERR_WORKSPACE: return "COLI_ERR_WORKSPACE";
        case COLI_ERR_CUDA: return "COLI_ERR_CUDA";
    }
    return "COLI_ERR_UNKNOWN";
}

const char* coli_last_error(void) { return g_err; }

void coli_debug_set_wait_ns(unsigned long long ns) { g_wait_ns.store(ns, std::memory_order_relaxed); }

void coli_debug_phase_stamps(unsigned long long* device_buffer) { g_stamps.store(device_buffer); }

coli_status coli_moe_profile_next(cudaEvent_t* events, int n_events)
{
    if (events && n_events < 0) return fail(COLI_ERR_INVALID_ARG, "n_events < 0");
    g_prof_events = events;
    g_prof_n = events ? n_events : 0;
    return COLI_OK;
}

coli_status coli_router_topk(const void* x, coli_dtype xt, int T, int H, const float* w_router,
                             const float* sel_bias, int E, int k, float routed_scale,
                             int32_t* topk_idx, float* topk_w, cudaStream_t stream)
{
    coli_status st = check_sizes(T, H, E, k);
    if (st != COLI_OK) return st;
    if (xt != COLI_F32 && xt != COLI_BF16) return fail(COLI_ERR_INVALID_ARG, "unknown activation dtype %d", (int)xt);
    if (T == 0) return COLI_OK;
    if (!x || !w_router || !sel_bias || !topk_idx || !topk_w) return fail(COLI_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(x, 16) || !aligned(w_router, 16)) return fail(COLI_ERR_INVALID_ARG, "x / w_router not 16-byte aligned");
    if (!std::isfinite(routed_scale)) return fail(COLI_ERR_INVALID_ARG, "routed_scale is not finite");
    dim3 grid(kRouterCluster * ((T + kRouterTokens - 1) / kRouterTokens));
    if (xt == COLI_BF16)
        router_cluster_kernel<true><<<grid, kRouterClusterThreads, 0, stream>>>(
            x, T, H, w_router, sel_bias, E, k, routed_scale, topk_idx, topk_w);
    else
        router_cluster_kernel<false><<<grid, kRouterClusterThreads, 0, stream>>>(
            x, T, H, w_router, sel_bias, E, k, routed_scale, topk_idx, topk_w);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? COLI_OK : cuda_fail(e, "router launch");
}

coli_status coli_expert_union(const int32_t* topk_idx, int T, int k, int E, int32_t* count,
                              int32_t* offset, int32_t* active, int32_t* n_active, int32_t* perm,
                              int32_t* inv_perm, cudaStream_t stream)
{
    if (T < 0 || T > kMaxTokens) return fail(COLI_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, kMaxTokens);
    if (k < 1 || k > kMaxTopK) return fail(COLI_ERR_INVALID_ARG, "top_k=%d outside [1, %d]", k, kMaxTopK);
    if (E < k || E > kMaxExperts) return fail(COLI_ERR_INVALID_ARG, "n_experts=%d outside [top_k, %d]", E, kMaxExperts);
    if (!count || !offset || !active || !n_active || (T > 0 && (!topk_idx || !perm || !inv_perm)))
        return fail(COLI_ERR_INVALID_ARG, "NULL pointer argument");
    WorkLists wl{};
    TopkArgs tk{};
    union_kernel<false, false><<<1, kUnionThreads, 0, stream>>>(const_cast<int32_t*>(topk_idx), T, k, E, count,
                                                                offset, active, n_active, perm, inv_perm, wl, tk);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? COLI_OK : cuda_fail(e, "union launch");
}

size_t coli_moe_workspace_size(const coli_moe_layer* L, int T)
{
    if (check_layer(L, T) != COLI_OK) return 0;
    return layout(nullptr, T, L->hidden, L->ffn, L->n_experts, L->top_k).bytes;
}

int coli_moe_path(const coli_moe_layer* L, int T)
{
    if (check_layer(L, T) != COLI_OK) return COLI_PATH_NONE;
    return choose_path(L, T);
}

size_t coli_moe_status_word_offset(const coli_moe_layer* L, int T)
{
    if (check_layer(L, T) != COLI_OK || T == 0) return SIZE_MAX;
    char* const base = reinterpret_cast<char*>(256);  // any aligned base: only differences are used
    const Workspace w = layout(base, T, L->hidden, L->ffn, L->n_experts, L->top_k);
    return (size_t)(reinterpret_cast<char*>(w.ctl + 3) - base);
}

coli_status coli_moe_forward(const coli_moe_layer* L, const void* x, coli_dtype xt, int T, void* out,
                             coli_dtype ot, void* workspace, size_t ws_bytes, int32_t* topk_idx_out,
                             float* topk_w_out, cudaStream_t stream)
{
    StageTimer tm;
    tm.ev = g_prof_events;
    tm.n = g_prof_n;
    g_prof_events = nullptr;  // one-shot
    g_prof_n = 0;

    coli_status st = check_call(L, x, xt, T, out, ot, topk_idx_out, topk_w_out);
    if (st != COLI_OK || T == 0) return st;
    if (!workspace) return fail(COLI_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(workspace, 256)) return fail(COLI_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    const int H = L->hidden, F = L->ffn, E = L->n_experts, k = L->top_k;
    Workspace w = layout(workspace, T, H, F, E, k);
    if (ws_bytes < w.bytes)
        return fail(COLI_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, w.bytes);

    DeviceInfo* dev = nullptr;
    if ((st = device_info(&dev)) != COLI_OK) return st;
    cudaError_t e = cudaSuccess;
    if (tm.ev) {  // stage events requested (test hook): recorded differently inside a graph capture
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if ((e = cudaStreamIsCapturing(stream, &cs)) != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
        tm.capturing = (cs == cudaStreamCaptureStatusActive);
    }
    tm.s = stream;

    int32_t* idx = topk_idx_out ? topk_idx_out : w.idx;
    float* wt = topk_w_out ? topk_w_out : w.w;
    const bool bf16 = (xt == COLI_BF16);

    // One token: router scores, top-k, gate/up, down, combine; the union of a
    // one-token batch is its k experts.
    const int path = choose_path(L, T);

    // Up to 64 tokens: the fused decode-layer kernel, one cooperative launch
    // (after the router-score kernel when the batch is larger than one token group).
    if (path == COLI_PATH_SINGLE || path == COLI_PATH_DECODE) {
        const LayerPlan pl = layer_plan(T, H, F, E, k, L->act_int8 ? 1 : bf16 ? 2 : 3);
        if (dev->sms < kMinLayerSms) return fail(COLI_ERR_UNSUPPORTED, "%d SMs: the decode kernel needs %d", dev->sms, kMinLayerSms);
        const LayerKernel kern = layer_kernel(pl.MT, bf16, ot == COLI_BF16, pl.out_rows, L->act_int8 != 0);
        {  // one block per SM must be resident (a cooperative launch); the answer is cached per (kernel, bytes)
            bool known = false;
            {
                std::lock_guard<std::mutex> lock(g_dev_mu);
                for (int i = 0; i < dev->n_fit && !known; ++i)
                    known = dev->fit_kern[i] == (const void*)kern && dev->fit_bytes[i] == pl.ls.bytes;
            }
            if (!known) {
                int occ = 0;
                if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, layer_threads(pl.MT), pl.ls.bytes)) !=
                    cudaSuccess)
                    return cuda_fail(e, "occupancy query");
                if (occ < 1)
                    return fail(COLI_ERR_UNSUPPORTED, "the decode kernel does not fit on an SM (%zu B shared memory)",
                                pl.ls.bytes);
                std::lock_guard<std::mutex> lock(g_dev_mu);
                if (dev->n_fit < DeviceInfo::kFitSlots) {
                    dev->fit_kern[dev->n_fit] = (const void*)kern;
                    dev->fit_bytes[dev->n_fit] = pl.ls.bytes;
                    ++dev->n_fit;
                }
            }
        }
        const bool fused_router = T <= pl.MT;
        if ((e = tm.rec(COLI_STAGE_ROUTE, 0)) != cudaSuccess) return cuda_fail(e, "event record");
        if (!fused_router) {
            st = launch_logits(x, xt, T, H, L->w_router, E, w.logits, nullptr, 0, stream);
            if (st != COLI_OK) return st;
        }
        if ((e = tm.rec(COLI_STAGE_ROUTE, 1)) != cudaSuccess || (e = tm.rec(COLI_STAGE_UNION, 0)) != cudaSuccess ||
            (e = tm.rec(COLI_STAGE_UNION, 1)) != cudaSuccess || (e = tm.rec(COLI_STAGE_GATEUP, 0)) != cudaSuccess)
            return cuda_fail(e, "event record");
        LayerArgs la{L->w_router, L->sel_bias, L->gate_q, L->gate_s, L->up_q, L->up_s, L->down_q, L->down_s,
                     H, F, E, k, T, L->routed_scale, x, out, w.logits, fused_router ? 0 : 1, idx, wt, w.h,
                     w.partial, w.ctl + 3, wait_limit(kBarrierNs), L->top_p, g_stamps.load()};
        if (pl.out_rows && L->prefetch_next) la.pf_n = lookahead_ranges(L->prefetch_next, la.pf_base, la.pf_bytes);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(dev->sms);
        cfg.blockDim = dim3(layer_threads(pl.MT));
        cfg.dynamicSmemBytes = pl.ls.bytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if ((e = cudaLaunchKernelEx(&cfg, kern, la, pl.ls)) != cudaSuccess) return cuda_fail(e, "decode-layer launch");
        // the layer kernel fuses gate/up, down and the combine
        if ((e = tm.rec(COLI_STAGE_GATEUP, 1)) != cudaSuccess || (e = tm.rec(COLI_STAGE_DOWN, 0)) != cudaSuccess ||
            (e = tm.rec(COLI_STAGE_DOWN, 1)) != cudaSuccess || (e = tm.rec(COLI_STAGE_COMBINE, 0)) != cudaSuccess ||
            (e = tm.rec(COLI_STAGE_COMBINE, 1)) != cudaSuccess)
            return cuda_fail(e, "event record");
        e = cudaGetLastError();
        return e == cudaSuccess ? COLI_OK : cuda_fail(e, "layer launch");
    }

    // Prefill: tensor-core grouped GEMMs over token tiles of <= kPfMaxN pairs per expert.
    // The TMA maps need K a multiple of 256 (scale rows of whole 16-byte boxes).
    CUtensorMap m_gq, m_gs, m_uq, m_us, m_dq, m_ds, m_x, m_h;
    const size_t Q = (size_t)T * k + T;
    uint16_t* xg = reinterpret_cast<uint16_t*>(w.partial);  // gathered rows; later reused for ys
    uint16_t* hb = reinterpret_cast<uint16_t*>(w.h);
    if (path == COLI_PATH_PREFILL && (size_t)dev->smem_optin < kPfSmemBytes)
        return fail(COLI_ERR_UNSUPPORTED, "the device offers %d bytes of shared memory per block; the prefill GEMM needs %zu",
                    dev->smem_optin, kPfSmemBytes);
    if (path == COLI_PATH_PREFILL && !tensor_map_encoder())
        return fail(COLI_ERR_UNSUPPORTED, "the CUDA driver provides no cuTensorMapEncodeTiled (tensor-core prefill path)");
    if (path == COLI_PATH_PREFILL &&
        !(encode_weight_maps(&m_gq, &m_gs, L->gate_q, L->gate_s, E, F, H) &&
                         encode_weight_maps(&m_uq, &m_us, L->up_q, L->up_s, E, F, H) &&
                         encode_weight_maps(&m_dq, &m_ds, L->down_q, L->down_s, E, H, F) &&
                         encode_2d(&m_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, xg, (uint64_t)H, Q, kPfKStep, kPfBRows,
                                   CU_TENSOR_MAP_SWIZZLE_128B) &&
                         encode_2d(&m_h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, hb, (uint64_t)F, Q, kPfKStep, kPfBRows,
                                   CU_TENSOR_MAP_SWIZZLE_128B)))
        return fail(COLI_ERR_CUDA, "cuTensorMapEncodeTiled rejected a prefill tensor map");
    if (path == COLI_PATH_PREFILL) {
        if ((e = tm.rec(COLI_STAGE_ROUTE, 0)) != cudaSuccess) return cuda_fail(e, "event record");
        {
            dim3 grid((T + kRtT - 1) / kRtT, (E + kRtE - 1) / kRtE);
            if (bf16) router_logits_tiled_kernel<true><<<grid, kRtThreads, 0, stream>>>(x, T, H, L->w_router, E, w.logits);
            else router_logits_tiled_kernel<false><<<grid, kRtThreads, 0, stream>>>(x, T, H, L->w_router, E, w.logits);
        }
        const bool fused = T <= kFusedTopkMaxT && E <= 256;
        if (!fused)
            router_topk_kernel<<<(T + 7) / 8, 256, 0, stream>>>(w.logits, T, E, k, L->sel_bias, L->routed_scale, L->top_p, idx, wt);
        if ((e = tm.rec(COLI_STAGE_ROUTE, 1)) != cudaSuccess || (e = tm.rec(COLI_STAGE_UNION, 0)) != cudaSuccess)
            return cuda_fail(e, "event record");
        WorkLists wl{w.pair_token, w.pair_w, w.ctl, w.g_expert, w.g_start, w.g_count, wt, kPfMaxN};
        TopkArgs tk{w.logits, L->sel_bias, L->routed_scale, wt, L->top_p};
        const int P = T * k;
        if (fused) {
            union_kernel<true, true><<<1, kUnionThreads, 0, stream>>>(idx, T, k, E, w.count, w.offset, w.active,
                                                                      w.n_active, w.perm, w.inv_perm, wl, tk);
        } else {  // the whole GPU: per-chunk ranks, bucket starts, scatter
            const int n_chunks = (P + kUnionChunk - 1) / kUnionChunk;
            union_chunk_kernel<<<n_chunks, kUnionChunk, 0, stream>>>(idx, P, E, w.chunk, w.rank);
            union_scan_kernel<true><<<1, kUnionThreads, 0, stream>>>(w.chunk, n_chunks, T, k, E, w.count, w.offset,
                                                                     w.active, w.n_active, wl);
            union_scatter_kernel<true><<<(std::max(P, T) + 255) / 256, 256, 0, stream>>>(
                idx, T, k, E, w.chunk, w.rank, w.offset, w.perm, w.inv_perm, wl);
        }
        if ((e = tm.rec(COLI_STAGE_UNION, 1)) != cudaSuccess || (e = tm.rec(COLI_STAGE_GATEUP, 0)) != cudaSuccess)
            return cuda_fail(e, "event record");
        const int max_tiles = P / kPfMaxN + E + (T + kPfMaxN - 1) / kPfMaxN + 1;  // >= number of union groups
        {
            const size_t n = Q * (size_t)(H / 8);
            const int blocks = (int)((n + 255) / 256);
            if (bf16) prefill_gather_kernel<true><<<blocks, 256, 0, stream>>>(x, w.pair_token, (int)Q, T, H, xg);
            else prefill_gather_kernel<false><<<blocks, 256, 0, stream>>>(x, w.pair_token, (int)Q, T, H, xg);
        }
        PrefillArgs pa{F, H, k, P, F / 64, w.ctl, w.g_expert, w.g_start, w.g_count, w.perm, w.pair_w, hb, xg, w.ctl + 3, wait_limit(kPfWaitNs)};
        const int grid1 = std::min(dev->sms, max_tiles * (F / 64));
        prefill_gemm_kernel<true><<<grid1, kPfThreads, kPfSmemBytes, stream>>>(m_gq, m_uq, m_gs, m_us, m_x, pa);
        if ((e = tm.rec(COLI_STAGE_GATEUP, 1)) != cudaSuccess || (e = tm.rec(COLI_STAGE_DOWN, 0)) != cudaSuccess)
            return cuda_fail(e, "event record");
        uint16_t* ys = xg;  // the gathered rows are dead once gate/up is done
        PrefillArgs pd{H, F, k, P, H / 128, w.ctl, w.g_expert, w.g_start, w.g_count, w.perm, w.pair_w, hb, ys, w.ctl + 3, wait_limit(kPfWaitNs)};
        const int grid2 = std::min(dev->sms, max_tiles * (H / 128));
        prefill_gemm_kernel<false><<<grid2, kPfThreads, kPfSmemBytes, stream>>>(m_dq, m_dq, m_ds, m_ds, m_h, pd);
        if ((e = tm.rec(COLI_STAGE_DOWN, 1)) != cudaSuccess || (e = tm.rec(COLI_STAGE_COMBINE, 0)) != cudaSuccess)
            return cuda_fail(e, "event record");
        {
            const size_t n8 = (size_t)T * H / 8;
            const int blocks = (int)((n8 + 255) / 256);
            if (ot == COLI_BF16) slot_reduce_kernel<true><<<blocks, 256, 0, stream>>>(ys, T, k + 1, H, idx, out);
            else slot_reduce_kernel<false><<<blocks, 256, 0, stream>>>(ys, T, k + 1, H, idx, out);
        }
        if ((e = tm.rec(COLI_STAGE_COMBINE, 1)) != cudaSuccess) return cuda_fail(e, "event record");
        e = cudaGetLastError();
        return e == cudaSuccess ? COLI_OK : cuda_fail(e, "layer launch");
    }

    const int TG = group_tokens(T, H, F, dev->smem_optin);

    // Route (router scores; the top-k runs in the union block for small batches)
    if ((e = tm.rec(COLI_STAGE_ROUTE, 0)) != cudaSuccess) return cuda_fail(e, "event record");
    st = launch_logits(x, xt, T, H, L->w_router, E, w.logits, nullptr, 0, stream);
    if (st != COLI_OK) return st;
    const bool fused_topk = T <= kFusedTopkMaxT && E <= 256;
    if (!fused_topk)
        router_topk_kernel<<<(T + 7) / 8, 256, 0, stream>>>(w.logits, T, E, k, L->sel_bias, L->routed_scale, L->top_p, idx, wt);
    if ((e = tm.rec(COLI_STAGE_ROUTE, 1)) != cudaSuccess) return cuda_fail(e, "event record");

    // Union and work lists
    if ((e = tm.rec(COLI_STAGE_UNION, 0)) != cudaSuccess) return cuda_fail(e, "event record");
    WorkLists wl{w.pair_token, w.pair_w, w.ctl, w.g_expert, w.g_start, w.g_count, wt, TG};
    TopkArgs tk{w.logits, L->sel_bias, L->routed_scale, wt, L->top_p};
    if (fused_topk)
        union_kernel<true, true><<<1, kUnionThreads, 0, stream>>>(idx, T, k, E, w.count, w.offset, w.active,
                                                                  w.n_active, w.perm, w.inv_perm, wl, tk);
    else
        union_kernel<true, false><<<1, kUnionThreads, 0, stream>>>(idx, T, k, E, w.count, w.offset, w.active,
                                                                   w.n_active, w.perm, w.inv_perm, wl, tk);
    if ((e = tm.rec(COLI_STAGE_UNION, 1)) != cudaSuccess) return cuda_fail(e, "event record");

    // Gate/up + SwiGLU for every token group (routed experts, then the shared expert)
    PhaseArgs ga{L->gate_q, L->gate_s, L->up_q, L->up_s, F, H, x, w.ctl, w.ctl + 1,
                 w.g_expert, w.g_start, w.g_count, w.pair_token, w.pair_w, w.h};
    const size_t gsm = gateup_smem(H, TG);
    if ((e = tm.rec(COLI_STAGE_GATEUP, 0)) != cudaSuccess) return cuda_fail(e, "event record");
    {
        auto kern = bf16 ? (TG == 1 ? expert_phase_kernel<true, true, 1> : expert_phase_kernel<true, true, 4>)
                         : (TG == 1 ? expert_phase_kernel<true, false, 1> : expert_phase_kernel<true, false, 4>);
        const int grid = dev->sms * blocks_per_sm(kern, gsm);
        kern<<<grid, kDecThreads, gsm, stream>>>(ga);
    }
    if ((e = tm.rec(COLI_STAGE_GATEUP, 1)) != cudaSuccess) return cuda_fail(e, "event record");

    // Down projection with the routing weight, one partial row per pair
    PhaseArgs da{L->down_q, L->down_s, nullptr, nullptr, H, F, w.h, w.ctl, w.ctl + 2,
                 w.g_expert, w.g_start, w.g_count, w.pair_token, w.pair_w, w.partial};
    const size_t dsm = down_smem(F, TG);
    if ((e = tm.rec(COLI_STAGE_DOWN, 0)) != cudaSuccess) return cuda_fail(e, "event record");
    {
        auto kern = TG == 1 ? expert_phase_kernel<false, false, 1> : expert_phase_kernel<false, false, 4>;
        const int grid = dev->sms * blocks_per_sm(kern, dsm);
        kern<<<grid, kDecThreads, dsm, stream>>>(da);
    }
    if ((e = tm.rec(COLI_STAGE_DOWN, 1)) != cudaSuccess) return cuda_fail(e, "event record");

    // Combine
    if ((e = tm.rec(COLI_STAGE_COMBINE, 0)) != cudaSuccess) return cuda_fail(e, "event record");
    {
        const int n = T * (H / 4);
        const int blocks = (n + 255) / 256;
        if (ot == COLI_BF16) combine_kernel<true><<<blocks, 256, 0, stream>>>(w.partial, w.inv_perm, idx, T, k, H, out);
        else combine_kernel<false><<<blocks, 256, 0, stream>>>(w.partial, w.inv_perm, idx, T, k, H, out);
    }
    if ((e = tm.rec(COLI_STAGE_COMBINE, 1)) != cudaSuccess) return cuda_fail(e, "event record");

    e = cudaGetLastError();
    return e == cudaSuccess ? COLI_OK : cuda_fail(e, "layer launch");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of coli_moe_forward: the workspace is a file-scope
// __device__ array compiled into the library (COLI_NOALLOC_SCRATCH_BYTES per
// device, resident until the process exits), for callers that cannot allocate
// device memory themselves.  Host code never passes the array's name to a
// kernel (on the host it names a host-side stand-in); it passes the device
// address looked up once per device with cudaGetSymbolAddress.

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[COLI_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on the
// first call per device, with that device current).
coli_status noalloc_scratch(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(COLI_ERR_UNSUPPORTED, "device %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return COLI_OK;
}

}  // namespace

extern "C" coli_status coli_moe_forward_host(const coli_moe_layer* L, const void* x_host, void* x_dev, coli_dtype xt,
                                             int T, void* out_host, void* out_dev, coli_dtype ot, void* workspace,
                                             size_t ws_bytes, cudaStream_t stream)
{
    coli_status st = check_call(L, x_dev, xt, T, out_dev, ot, nullptr, nullptr);
    if (st != COLI_OK || T == 0) return st;
    if (!x_host || !out_host || !workspace) return fail(COLI_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(workspace, 256)) return fail(COLI_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    const size_t need = coli_moe_workspace_size(L, T);
    if (ws_bytes < need) return fail(COLI_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, need);
    const size_t n = (size_t)T * L->hidden;
    const size_t xb = n * (xt == COLI_BF16 ? 2 : 4), ob = n * (ot == COLI_BF16 ? 2 : 4);
    cudaError_t e = cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail(e, "input copy");
    if ((st = coli_moe_forward(L, x_dev, xt, T, out_dev, ot, workspace, ws_bytes, nullptr, nullptr, stream)) != COLI_OK)
        return st;
    e = cudaMemcpyAsync(out_host, out_dev, ob, cudaMemcpyDeviceToHost, stream);
    return e == cudaSuccess ? COLI_OK : cuda_fail(e, "output copy");
}

extern "C" coli_status coli_moe_forward_noalloc(const coli_moe_layer* L, const void* x, coli_dtype xt, int T,
                                                void* out, coli_dtype ot, int32_t* topk_idx_out,
                                                float* topk_w_out, cudaStream_t stream)
{
    // Every argument is checked before any CUDA call; a refused or empty call
    // consumes an armed stage-timing hook, as coli_moe_forward would.
    coli_status st0 = check_call(L, x, xt, T, out, ot, topk_idx_out, topk_w_out);
    const size_t need = st0 == COLI_OK ? coli_moe_workspace_size(L, T) : 0;
    if (st0 != COLI_OK || T == 0 || need > (size_t)COLI_NOALLOC_SCRATCH_BYTES) {
        g_prof_events = nullptr;
        g_prof_n = 0;
    }
    if (st0 != COLI_OK || T == 0) return st0;
    if (need > (size_t)COLI_NOALLOC_SCRATCH_BYTES) {
        return fail(COLI_ERR_WORKSPACE,
                    "T=%d needs %zu bytes of scratch; the static scratch holds %zu bytes (use coli_moe_forward)",
                    T, need, (size_t)COLI_NOALLOC_SCRATCH_BYTES);
    }
    void* ws = nullptr;
    coli_status st = noalloc_scratch(&ws);
    if (st != COLI_OK) return st;
    return coli_moe_forward(L, x, xt, T, out, ot, ws, (size_t)COLI_NOALLOC_SCRATCH_BYTES, topk_idx_out,
                            topk_w_out, stream);
}
