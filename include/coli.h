/*
 * coli.h -- C ABI of the B200 routed-expert MoE layer library (libcoli.so).
 *
 * The calls follow the colibri pages' per-token path: Route, then Union, then
 * the expert compute with its combine (Korean getting-started page, section
 * 토큰당 처리 경로 "The Per-Token Path"; "colibri: 744B MoEをストレージから推論する
 * Cエンジン", section トークンごとの5ステップパスとデュアルSSDミラー).  The two
 * steps of that path about storage (Place, Learn) have no counterpart here:
 * every expert is resident in HBM.
 *
 * Conventions for every call:
 *   - Every tensor pointer is a caller-owned DEVICE pointer, row-major and
 *     densely packed.  The library allocates no device memory and keeps no
 *     device state between calls; scratch memory is the caller's workspace.
 *   - All work is enqueued on the given stream; calls are asynchronous and
 *     never synchronise the device.  Argument checks run on the host before
 *     anything is enqueued: a call that returns an error has launched nothing.
 *   - Nothing is thrown across the ABI.  Every call returns a coli_status;
 *     coli_last_error() returns a description of the calling thread's most
 *     recent failure.
 *   - Sizes: hidden H and expert width F are multiples of 64 (the int4 group),
 *     H and F <= 16384; 1 <= top_k <= 32; top_k <= n_experts <= 1024;
 *     0 <= T <= 65536.  T == 0 is a valid empty call: coli_router_topk and
 *     coli_moe_forward launch nothing, coli_expert_union still writes its
 *     per-expert outputs (all counts zero).
 *   - Alignment: activations, outputs and weight/scale pointers 16-byte
 *     aligned; workspace 256-byte aligned.
 *
 * int4-gs64 storage of one matrix [N, K] ("gs64 build" of the int4 container,
 * "colibri: 744B MoE…", section はじめにとソースが語らないこと): bytes [N, K/2],
 * two values per byte, even k in the low nibble, each nibble a two's-complement
 * integer in [-8, 7] with no zero point; fp32 scales [N, K/64];
 * W[n, k] = q[n, k] * scale[n, k / 64].
 */
#ifndef COLI_H
#define COLI_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define COLI_API __attribute__((visibility("default")))
#else
#define COLI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    COLI_OK = 0,
    COLI_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or dtype */
    COLI_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement */
    COLI_ERR_WORKSPACE = 3,    /* workspace smaller than coli_moe_workspace_size() */
    COLI_ERR_CUDA = 4          /* a CUDA runtime call failed; see coli_last_error() */
} coli_status;

typedef enum { COLI_F32 = 0, COLI_BF16 = 1 } coli_dtype;

/* One MoE layer.  Expert index n_experts is the shared expert, so every
 * expert array holds n_experts + 1 experts, expert-major. */
typedef struct coli_moe_layer {
    int hidden;            /* H, e.g. 6144 */
    int ffn;               /* F, expert width, e.g. 2048 */
    int n_experts;         /* E routed experts, e.g. 256 */
    int top_k;             /* k, e.g. 8 */
    int group;             /* scale group along K; must be 64 */
    float routed_scale;    /* factor applied to the renormalised routed weights, e.g. 2.5 */
    const float* w_router; /* [E, H] fp32 */
    const float* sel_bias; /* [E] fp32, selection-only bias */
    const uint8_t* gate_q; /* [E+1, F, H/2] */
    const uint8_t* up_q;   /* [E+1, F, H/2] */
    const uint8_t* down_q; /* [E+1, H, F/2] */
    const float* gate_s;   /* [E+1, F, H/64] */
    const float* up_s;     /* [E+1, F, H/64] */
    const float* down_s;   /* [E+1, H, F/64] */
    float top_p;           /* adaptive expert top-p: 0 (or >= 1) = plain top-k; see coli_moe_forward */
    int act_int8;          /* 1: integer-activation variant (int8 activations per 32); 0: default; see coli_moe_forward */
    const struct coli_moe_layer* prefetch_next; /* the layer the next call runs, for the router-lookahead
                                                   prefetch, or NULL; see coli_moe_forward */
} coli_moe_layer;

/*
 * Route ("Colibri 完全ガイド", section コア技術のハイライト: DeepSeek-V3-style
 * sigmoid router).  For each token t of x [T, H] (dtype xt):
 *   logit_e = x_t . w_router[e];  s_e = 1/(1+exp(-logit_e));  c_e = s_e + sel_bias[e]
 *   topk_idx[t, :] = the k experts of largest c_e, in descending c_e
 *                    (equal c_e: lower expert index first)
 *   topk_w[t, j]   = routed_scale * s_idx[j] / sum_j' s_idx[j']
 * The bias selects experts but does not enter the weights.  Computed in fp32.
 * Outputs: topk_idx int32 [T, k], topk_w fp32 [T, k] (device).
 */
COLI_API coli_status coli_router_topk(const void* x, coli_dtype xt, int T, int H,
                             const float* w_router, const float* sel_bias, int E, int k,
                             float routed_scale, int32_t* topk_idx, float* topk_w,
                             cudaStream_t stream);

/*
 * Union (Korean getting-started page, section 토큰당 처리 경로, "Union": experts
 * chosen by several tokens of the batch are de-duplicated).  A stable counting
 * sort of the T*k pairs p = t*k + j by expert topk_idx[p]:
 *   count[E]      pairs per expert
 *   offset[E+1]   exclusive prefix sum of count (offset[E] = T*k)
 *   active[E]     experts with count > 0 in ascending order, tail filled with -1
 *   n_active[1]   number of active experts (the batch union size U)
 *   perm[T*k]     pair ids in (expert, token, slot) order
 *   inv_perm[T*k] inv_perm[perm[i]] = i
 * All outputs are int32 device arrays; results are deterministic (bit-exact).
 * Every topk_idx entry must lie in [0, E); this is not checked on the device.
 */
COLI_API coli_status coli_expert_union(const int32_t* topk_idx, int T, int k, int E,
                              int32_t* count, int32_t* offset, int32_t* active,
                              int32_t* n_active, int32_t* perm, int32_t* inv_perm,
                              cudaStream_t stream);

/* Bytes of workspace coli_moe_forward needs for T tokens of this layer
 * (0 if the layer description is invalid). */
COLI_API size_t coli_moe_workspace_size(const coli_moe_layer* layer, int T);

/* Device status of a coli_moe_forward call (no counterpart on the pages: it
 * reports on this library's own kernels).  Kernels whose warps or blocks wait
 * on one another inside a launch bound every wait in time; a wait that runs out
 * (a fault or stall elsewhere on the GPU) leaves the outputs undefined and sets
 * a 32-bit status word in the workspace, which is 0 after a normal call
 * (1: a prefill GEMM pipeline wait ran out; 2: a decode-kernel grid barrier
 * did; 3: the decode kernel was not launched cooperatively).  This returns the
 * byte offset of that word inside the workspace of a call with T tokens of this
 * layer: read the 4 bytes after the call has completed (e.g. with cudaMemcpy).
 * Returns SIZE_MAX if the sizes are invalid or T == 0.  Host arithmetic only:
 * launches nothing, touches no device memory. */
COLI_API size_t coli_moe_status_word_offset(const coli_moe_layer* layer, int T);

/*
 * The whole layer: Route, Union, the expert FFNs and the weighted combine.
 *   out_t = sum_j topk_w[t,j] * FFN_{topk_idx[t,j]}(x_t) + FFN_shared(x_t)
 *   FFN_e(x) = W_down,e (silu(W_gate,e x) * (W_up,e x)),  silu(z) = z/(1+exp(-z))
 * The pages name the routed experts, the shared expert ("Colibri 完全ガイド",
 * DeepSeek-V3 router row) and int4 weights with one scale per 64; the SwiGLU
 * form of the expert and the unscaled, always-on shared expert are this
 * library's reading of them.
 * Adaptive expert top-p (layer->top_p in (0, 1); "colibri解説", section 速度を稼ぐ
 * 実用ノブ, the --topp knob, which the page credits with 30-40 % fewer expert
 * reads): of the k selected experts, ranked by share s_j / sum s (descending,
 * lower expert first), only the shortest prefix whose cumulative share reaches
 * top_p is kept; the kept weights are renormalised to routed_scale over the
 * kept experts, dropped slots are reported as index -1 with weight 0 and cost
 * no expert reads.  The rule is this library's reading: the page names the
 * knob and its effect only.  The router is fp32.  Batches of up to 64 tokens
 * compute the experts with fp32 accumulation; the activations (and the SwiGLU
 * output h) enter the expert products as fixed point per block of 32 values
 * over a power-of-two block scale, multiplied exactly in integers: 21 bits for
 * fp32 activations (each value within 2^-21 of its block's largest magnitude,
 * an error of the order of fp32 arithmetic), 14 bits plus sign for bf16
 * activations (within 2^-15 of the block's largest magnitude, well below the
 * up to 2^-9 relative rounding the bf16 inputs carry).  Larger batches run the experts on the tensor cores with
 * bf16 operands (weights q * scale, activations and the SwiGLU output rounded
 * to bf16) and fp32 accumulation.
 * Integer-activation variant (layer->act_int8 = 1; "Colibri 完全ガイド", section
 * コア技術のハイライト, row 整数ドット積カーネル, int8 activations times packed
 * int4 weights): x before gate/up and h before down are quantised to
 * symmetric int8 per block of 32 (scale max|v| / 127, codes rint(v * 127 /
 * max|v|) in fp32) and multiplied exactly in integers; routing is unchanged.
 * The quantisation rule is this library's reading.  Batches of up to 64 tokens
 * only: a larger batch with act_int8 set returns COLI_ERR_UNSUPPORTED.  out is
 * written as fp32 or bf16 (round to nearest even).
 * Router-lookahead prefetch ("Colibri 完全ガイド", section Router-Lookahead
 * プリフェッチ: the next layer's experts are fetched while the current layer
 * computes): when layer->prefetch_next is set (checked like layer itself), a
 * one-token call asks the L2 cache for that layer's router weights, selection
 * bias and shared expert (weights and scales) while it routes its own token,
 * when the memory is otherwise idle, so that the next call finds them in L2.
 * The next layer's routed experts are not predicted: their router input is the
 * next layer's activations, which this call does not have (this library's
 * reading).  The results are unchanged; batches of more than one token ignore
 * the field.
 * x [T, H] dtype xt; out [T, H] dtype ot; workspace of at least
 * coli_moe_workspace_size(layer, T) bytes, contents undefined on entry and on
 * exit apart from the status word (coli_moe_status_word_offset), not shared by
 * calls that may run concurrently.  topk_idx_out [T, k] and topk_w_out [T, k]
 * are optional copies of the routing (NULL to skip).
 */
COLI_API coli_status coli_moe_forward(const coli_moe_layer* layer, const void* x, coli_dtype xt, int T,
                             void* out, coli_dtype ot, void* workspace, size_t ws_bytes,
                             int32_t* topk_idx_out, float* topk_w_out, cudaStream_t stream);

/* Kernel chains of coli_moe_forward (coli_moe_path). */
enum {
    COLI_PATH_NONE = 0,     /* empty batch or invalid arguments: nothing runs */
    COLI_PATH_SINGLE = 1,   /* one token: the fused decode-layer kernel, down summed by output rows */
    COLI_PATH_DECODE = 2,   /* 1-64 tokens: the fused decode-layer kernel (CUDA cores, fp32) */
    COLI_PATH_PREFILL = 3,  /* > 64 tokens: tcgen05 tensor-core grouped GEMMs (bf16 operands, fp32 accumulation) */
    COLI_PATH_WIDE = 4      /* batches neither kernel takes: CUDA-core expert-phase kernels (fp32) */
};

/*
 * Which kernel chain coli_moe_forward runs for a batch of T tokens of this
 * layer.  Decided by the shapes alone.  Batches of up to 64 tokens run the
 * fused decode-layer kernel (one cooperative launch; with more than one token
 * group it is preceded by the router-score kernel) when its shared memory
 * (activations, union tables) fits in 227 KB; batches of more than 64 tokens
 * with hidden and ffn multiples of 256 take the tensor-core path (a device
 * without cuTensorMapEncodeTiled in its driver then gets COLI_ERR_UNSUPPORTED
 * from coli_moe_forward, never another path); every other valid batch runs the
 * CUDA-core expert-phase kernels in fp32.  Host-only, launches nothing.
 */
COLI_API int coli_moe_path(const coli_moe_layer* layer, int T);

/* Stages of coli_moe_forward, for coli_moe_profile_next(). */
enum {
    COLI_STAGE_ROUTE = 0,   /* router scores and top-k */
    COLI_STAGE_UNION = 1,   /* batch union and work lists */
    COLI_STAGE_GATEUP = 2,  /* gate/up projections with SwiGLU */
    COLI_STAGE_DOWN = 3,    /* down projections, routing weight applied */
    COLI_STAGE_COMBINE = 4, /* per-token sum of expert outputs into out */
    COLI_N_STAGES = 5
};

/*
 * Optional stage timing.  Arms a one-shot hook for the calling host thread:
 * the next coli_moe_forward on this thread records events[2*s] on its stream
 * just before stage s and events[2*s+1] just after it, for s < n_events/2,
 * then disarms.  Stages that a path fuses into another are recorded
 * back-to-back.  events are caller-created cudaEvent_t handles (host objects);
 * pass events = NULL to disarm.  Inside stream capture the records become
 * external event-record nodes of the graph.
 */
COLI_API coli_status coli_moe_profile_next(cudaEvent_t* events, int n_events);

/*
 * Allocation-free variant of coli_moe_forward (the colibri pages have no
 * counterpart: it exists for callers of this library, not for the method).
 *
 * Some callers cannot hand the library a workspace.  cudaMalloc and cudaFree
 * synchronise the whole device, so a latency-bound decode loop that must not
 * stall the GPU cannot call them between tokens; and a library embedded in a
 * host framework that owns every device allocation (its own pool, its own
 * accounting) may not be allowed to allocate on its own at all.  This entry
 * point takes the same arguments as coli_moe_forward minus the workspace and
 * uses instead a scratch array compiled into libcoli.so as a file-scope
 * __device__ array of COLI_NOALLOC_SCRATCH_BYTES bytes.  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 * Limits and behaviour:
 *   - A batch is accepted when coli_moe_workspace_size(layer, T) is at most
 *     COLI_NOALLOC_SCRATCH_BYTES (8 MiB: up to 28 tokens at hidden 6144, ffn
 *     2048, 256 experts, top-8); larger batches return COLI_ERR_WORKSPACE
 *     with the sizes in coli_last_error() and launch nothing.
 *   - Every GPU that loads the library holds the 8 MiB array until the process
 *     exits.  The first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current; make that first
 *     call before any stream capture.  The address is kept for the life of
 *     the process: do not call this entry point on a device after
 *     cudaDeviceReset() (the array may then sit elsewhere).
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (nothing in it needs to start at zero: every call writes what it
 *     reads).  Calls whose work may overlap on the GPU (different streams, or
 *     different host threads without ordering) race on it and give wrong
 *     results; order them on one stream.
 */
#define COLI_NOALLOC_SCRATCH_BYTES (8u << 20)
COLI_API coli_status coli_moe_forward_noalloc(const coli_moe_layer* layer, const void* x, coli_dtype xt,
                                              int T, void* out, coli_dtype ot, int32_t* topk_idx_out,
                                              float* topk_w_out, cudaStream_t stream);

/*
 * The layer end to end from host memory: the per-token path of
 * coli_moe_forward (Korean getting-started page, section 토큰당 처리 경로)
 * with the activations read from and the output written to host buffers, the
 * way an engine that keeps its token state on the host would call it.  Three
 * steps are enqueued on stream, in order: x_host [T, H] (dtype xt) is copied
 * into the caller's device buffer x_dev [T, H]; coli_moe_forward runs on
 * x_dev into the caller's device buffer out_dev [T, H] (dtype ot) with the
 * given workspace; out_dev is copied to out_host [T, H].  Host buffers should
 * be page-locked (cudaHostAlloc / cudaHostRegister) for the copies to be
 * asynchronous; the caller owns all five buffers, and out_host holds the
 * result once the stream has reached the end of the call (e.g. after
 * cudaStreamSynchronize).  Every argument (those of coli_moe_forward, the two
 * host pointers and the workspace size) is checked before anything is
 * enqueued; COLI_ERR_CUDA if a copy cannot be enqueued.  T == 0 enqueues
 * nothing.
 */
COLI_API coli_status coli_moe_forward_host(const coli_moe_layer* layer, const void* x_host, void* x_dev,
                                           coli_dtype xt, int T, void* out_host, void* out_dev, coli_dtype ot,
                                           void* workspace, size_t ws_bytes, cudaStream_t stream);

COLI_API const char* coli_status_string(coli_status status);
COLI_API const char* coli_last_error(void);

/*
 * Test hook, not part of the layer's interface.  Every wait inside the kernels
 * (the decode kernel's grid barriers, the prefill GEMMs' pipeline waits) gives
 * up after a time limit (2 s), records a non-zero status word
 * (coli_moe_status_word_offset) and lets the kernel finish, so a stuck wait
 * never hangs the GPU.  This call sets that limit for the launches that follow
 * (ns = 0 restores the built-in limit), so that tests can make waits run out on
 * purpose and check the status word; the outputs of such a call are undefined.
 * Process-wide; teardown drains keep their own limits.
 */
COLI_API void coli_debug_set_wait_ns(unsigned long long ns);

/*
 * Test hook, not part of the layer's interface: the fused decode kernel runs
 * its phases (router, union, gate/up, down, combine) inside one launch, where
 * stream events cannot see them.  With a device buffer of at least
 * (number of SMs) x 16 uint64 set here, the decode launches that follow record
 * in it, per block, the GPU global timer (ns) at 16 fixed points of the kernel
 * (0 start, 1 activations staged, 2 phase A done, 3 after the first grid
 * barrier, 4 routing known, 5 gate/up done, 6 after the second barrier,
 * 7 h staged, 8 down done, 9 end; unused points are left unwritten).  NULL
 * turns it off.  Process-wide.
 */
COLI_API void coli_debug_phase_stamps(unsigned long long* device_buffer);

#ifdef __cplusplus
}
#endif
#endif /* COLI_H */
