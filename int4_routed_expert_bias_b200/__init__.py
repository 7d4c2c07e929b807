"""B200 routed-expert MoE layer: thin Python binding of libcoli.so (include/coli.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (torch is used for device memory and
streams).  The names mirror the C ABI: router_topk, expert_union,
moe_workspace_size, moe_forward.  If the compiled library is missing, importing
this package raises: there is no fallback path.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
# COLI_LIB=bounds loads the bounds-checked build (index checks write status 4 instead of trapping)
LIB_PATH = os.path.join(PKG, "libcoli_bounds.so" if os.environ.get("COLI_LIB") == "bounds" else "libcoli.so")

F32, BF16 = 0, 1
STATUS = {0: "COLI_OK", 1: "COLI_ERR_INVALID_ARG", 2: "COLI_ERR_UNSUPPORTED", 3: "COLI_ERR_WORKSPACE",
          4: "COLI_ERR_CUDA"}
STAGES = ("route", "union", "gateup", "down", "combine")
PATHS = {0: "none", 1: "single", 2: "decode", 3: "prefill", 4: "wide"}

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                      "(python int4_routed_expert_bias_b200/_build.py)")

_lib = ctypes.CDLL(LIB_PATH)
_p = ctypes.c_void_p
_i = ctypes.c_int
_lib.coli_router_topk.restype = _i
_lib.coli_router_topk.argtypes = [_p, _i, _i, _i, _p, _p, _i, _i, ctypes.c_float, _p, _p, _p]
_lib.coli_expert_union.restype = _i
_lib.coli_expert_union.argtypes = [_p, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p]
_lib.coli_moe_workspace_size.restype = ctypes.c_size_t
_lib.coli_moe_workspace_size.argtypes = [_p, _i]
_lib.coli_moe_status_word_offset.restype = ctypes.c_size_t
_lib.coli_moe_status_word_offset.argtypes = [_p, _i]
_lib.coli_moe_path.restype = _i
_lib.coli_moe_path.argtypes = [_p, _i]
_lib.coli_moe_forward.restype = _i
_lib.coli_moe_forward.argtypes = [_p, _p, _i, _i, _p, _i, _p, ctypes.c_size_t, _p, _p, _p]
_lib.coli_moe_forward_noalloc.restype = _i
_lib.coli_moe_forward_noalloc.argtypes = [_p, _p, _i, _i, _p, _i, _p, _p, _p]
_lib.coli_moe_forward_host.restype = _i
_lib.coli_moe_forward_host.argtypes = [_p, _p, _p, _i, _i, _p, _p, _i, _p, ctypes.c_size_t, _p]
_lib.coli_moe_profile_next.restype = _i
_lib.coli_moe_profile_next.argtypes = [_p, _i]
_lib.coli_status_string.restype = ctypes.c_char_p
_lib.coli_status_string.argtypes = [_i]
_lib.coli_last_error.restype = ctypes.c_char_p
_lib.coli_last_error.argtypes = []
_lib.coli_debug_set_wait_ns.restype = None
_lib.coli_debug_set_wait_ns.argtypes = [ctypes.c_ulonglong]
_lib.coli_debug_phase_stamps.restype = None
_lib.coli_debug_phase_stamps.argtypes = [_p]


class ColiError(RuntimeError):
    def __init__(self, status):
        self.status = status
        super().__init__(f"{STATUS.get(status, status)}: {last_error()}")


class _LayerStruct(ctypes.Structure):
    _fields_ = [("hidden", _i), ("ffn", _i), ("n_experts", _i), ("top_k", _i), ("group", _i),
                ("routed_scale", ctypes.c_float),
                ("w_router", _p), ("sel_bias", _p),
                ("gate_q", _p), ("up_q", _p), ("down_q", _p),
                ("gate_s", _p), ("up_s", _p), ("down_s", _p), ("top_p", ctypes.c_float),
                ("act_int8", ctypes.c_int), ("prefetch_next", _p)]


def lib():
    return _lib


def status_string(st):
    return _lib.coli_status_string(st).decode()


def last_error():
    return _lib.coli_last_error().decode()


def _check(st):
    if st != 0:
        raise ColiError(st)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


class Layer:
    """One MoE layer: device tensors in the library's layout (expert E = shared)."""

    def __init__(self, hidden, ffn, n_experts, top_k, routed_scale, w_router, sel_bias,
                 gate_q, gate_s, up_q, up_s, down_q, down_s, group=64, top_p=0.0, act_int8=False):
        self.tensors = dict(w_router=w_router, sel_bias=sel_bias, gate_q=gate_q, gate_s=gate_s,
                            up_q=up_q, up_s=up_s, down_q=down_q, down_s=down_s)
        self.hidden, self.ffn, self.n_experts, self.top_k = hidden, ffn, n_experts, top_k
        self.routed_scale = routed_scale
        self.struct = _LayerStruct(hidden, ffn, n_experts, top_k, group, routed_scale,
                                   *[_ptr(self.tensors[n]) for n in
                                     ("w_router", "sel_bias", "gate_q", "up_q", "down_q", "gate_s", "up_s",
                                      "down_s")], float(top_p), 1 if act_int8 else 0)

    @property
    def ref(self):
        return ctypes.byref(self.struct)

    def set_prefetch_next(self, other):
        """Name the layer the next call runs (None: none), for the router-lookahead
        prefetch of its router and shared expert; see include/coli.h."""
        self._next = other  # keeps the other layer's struct alive while it is named here
        self.struct.prefetch_next = None if other is None else ctypes.addressof(other.struct)


def router_topk(x, w_router, sel_bias, k, routed_scale, topk_idx, topk_w, stream=None):
    T, H = x.shape
    E = w_router.shape[0]
    _check(_lib.coli_router_topk(_ptr(x), _dtype_code(x), T, H, _ptr(w_router), _ptr(sel_bias), E, k,
                                 float(routed_scale), _ptr(topk_idx), _ptr(topk_w), _stream(stream)))


def expert_union(topk_idx, E, count, offset, active, n_active, perm, inv_perm, stream=None):
    T, k = topk_idx.shape
    _check(_lib.coli_expert_union(_ptr(topk_idx), T, k, E, _ptr(count), _ptr(offset), _ptr(active),
                                  _ptr(n_active), _ptr(perm), _ptr(inv_perm), _stream(stream)))


def moe_workspace_size(layer, T):
    return int(_lib.coli_moe_workspace_size(layer.ref, T))


def moe_path(layer, T):
    """Name of the kernel chain moe_forward runs for T tokens of this layer:
    "single" (one token, fused decode-layer kernel), "decode" (fused
    decode-layer kernel, up to 64 tokens), "prefill" (tensor cores), "wide"
    (CUDA-core expert phases, for batches neither takes) or "none" (empty or
    invalid call)."""
    return PATHS[int(_lib.coli_moe_path(layer.ref, T))]


def moe_status_word_offset(layer, T):
    """Byte offset of the device status word in the workspace of a call with T
    tokens, or None when such a call does not write it."""
    off = int(_lib.coli_moe_status_word_offset(layer.ref, T))
    return None if off == ctypes.c_size_t(-1).value else off


def moe_forward(layer, x, out, workspace, topk_idx_out=None, topk_w_out=None, stream=None, T=None):
    T = x.shape[0] if T is None else T
    _check(_lib.coli_moe_forward(layer.ref, _ptr(x), _dtype_code(x), T, _ptr(out), _dtype_code(out),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _ptr(topk_idx_out), _ptr(topk_w_out), _stream(stream)))


def moe_forward_host(layer, x_host, x_dev, out_host, out_dev, workspace, stream=None):
    """The layer from host memory: x_host (pinned CPU tensor) is copied into
    x_dev, the layer runs into out_dev, and out_dev is copied into out_host
    (pinned CPU tensor), all on the stream; see include/coli.h."""
    if x_host.dtype != x_dev.dtype or out_host.dtype != out_dev.dtype:
        raise ValueError("host and device buffers must have the same dtype")
    _check(_lib.coli_moe_forward_host(layer.ref, _ptr(x_host), _ptr(x_dev), _dtype_code(x_dev), x_host.shape[0],
                                      _ptr(out_host), _ptr(out_dev), _dtype_code(out_dev), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_forward_noalloc(layer, x, out, topk_idx_out=None, topk_w_out=None, stream=None):
    """moe_forward without a caller workspace: the library's static per-device
    scratch (COLI_NOALLOC_SCRATCH_BYTES) is used instead; see include/coli.h."""
    _check(_lib.coli_moe_forward_noalloc(layer.ref, _ptr(x), _dtype_code(x), x.shape[0], _ptr(out),
                                         _dtype_code(out), _ptr(topk_idx_out), _ptr(topk_w_out),
                                         _stream(stream)))


def moe_profile_next(events):
    """Arm stage timing for the next moe_forward on this thread: events is a list of
    2 * len(STAGES) torch.cuda.Event(enable_timing=True) objects (or None to disarm)."""
    global _prof_keep
    if events is None:
        _prof_keep = None
        _check(_lib.coli_moe_profile_next(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _prof_keep = arr
    _check(_lib.coli_moe_profile_next(ctypes.cast(arr, ctypes.c_void_p), len(events)))


_prof_keep = None


def debug_set_wait_ns(ns):
    """Test hook: limit (ns) of the kernels' bounded waits for the launches that
    follow; 0 restores the built-in limit.  See include/coli.h."""
    _lib.coli_debug_set_wait_ns(int(ns))


def debug_phase_stamps(buf):
    """Test hook: record the decode kernel's per-block phase times into buf (a
    torch int64 CUDA tensor of at least SMs x 16 elements), or stop (None)."""
    _lib.coli_debug_phase_stamps(None if buf is None else buf.data_ptr())
