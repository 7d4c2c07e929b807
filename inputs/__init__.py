"""Seeded synthetic inputs for the routed-expert MoE layer (tests and benchmark).

This module only draws inputs: activations, router weights and bias (numpy),
and int4-gs64 expert weights from the counter-based hash in gen_core.h (host C
or device CUDA, bit-identical).  It holds none of the layer's arithmetic and is
shared by the CUDA side and the oracle side alike.

Workloads (shapes of the colibri pages' GLM-5.2 MoE layer: hidden 6144, 256
routed experts of about 19 MB int4 each plus one shared expert, top-8):

  cfg 0  tiny      H 1024, F 512, E 64, T 4, fp32 x, Gaussian weights quantised
  cfg 1  decode-1  H 6144, F 2048, E 256, T 1, fp32 x, zero bias
  cfg 2  verify-4  T 4 bf16 x, tokens correlated (rho) so routing overlaps
  cfg 3  decode-64 T 64 bf16 x, Zipf-skewed selection bias (hot experts)
  cfg 4  prefill   T 4096 bf16 x, zero bias, bf16 output
"""
import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(HERE, "coli_inputs.cu")
_HDR = os.path.join(HERE, "gen_core.h")
LIB = os.path.join(HERE, "libcoli_inputs.so")

NVCC_ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def build(force=False):
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
            os.path.getmtime(_SRC), os.path.getmtime(_HDR)):
        return LIB
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    cmd = [nvcc, *NVCC_ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-o", LIB + ".tmp", _SRC]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.coli_inputs_gen_matrix_host.restype = ctypes.c_int
        L.coli_inputs_gen_matrix_host.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                                  ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64,
                                                  ctypes.c_void_p, ctypes.c_void_p]
        L.coli_inputs_gen_matrix_device.restype = ctypes.c_int
        L.coli_inputs_gen_matrix_device.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                                    ctypes.c_uint32, ctypes.c_uint32, ctypes.c_int64,
                                                    ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                                    ctypes.c_void_p]
        _lib = L
    return _lib


# ---------------------------------------------------------------------------
# workload definitions

@dataclass(frozen=True)
class Config:
    cfg: int
    name: str
    H: int
    F: int
    E: int
    k: int
    T: int
    x_dtype: str        # "f32" or "bf16"
    out_dtype: str      # "f32" or "bf16"
    layers: int
    routed_scale: float = 2.5
    group: int = 64

    @property
    def expert_bytes(self):
        """int4 nibbles + fp32 gs64 scales of one expert (gate, up, down)."""
        return 3 * self.H * self.F // 2 + 3 * self.H * self.F // self.group * 4


CONFIGS = {
    0: Config(0, "tiny", 1024, 512, 64, 8, 4, "f32", "f32", 1),
    1: Config(1, "decode-1", 6144, 2048, 256, 8, 1, "f32", "f32", 8),
    2: Config(2, "verify-4", 6144, 2048, 256, 8, 4, "bf16", "f32", 8),
    3: Config(3, "decode-64", 6144, 2048, 256, 8, 64, "bf16", "f32", 8),
    4: Config(4, "prefill-4096", 6144, 2048, 256, 8, 4096, "bf16", "bf16", 8),
}

# cfg 2: correlation of the three draft tokens with the verified token.  Chosen
# once (seeded search over the oracle router, tests/golden/search_rho.py) so that
# on average ~60 % of a draft's experts are also token 0's and the batch union
# holds 16-24 experts.
VERIFY_RHO = 0.81

# cfg 3: Zipf exponent and amplitude of the per-expert selection bias.
ZIPF_S = 1.1
ZIPF_BETA = 1.0


# ---------------------------------------------------------------------------
# bf16 encoding of activations (round to nearest even from fp32)

def to_bf16_bits(a32):
    a32 = np.ascontiguousarray(a32, dtype=np.float32)
    b = a32.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(b16):
    return (np.asarray(b16, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# router parameters and activations (numpy, seeded)

def _rng(*key):
    return np.random.default_rng([int(k) & 0xFFFFFFFF for k in key])


def router_params(c: Config, seed: int, layer: int):
    """(w_router fp32 [E,H], sel_bias fp32 [E]) for configs 1-4."""
    rng = _rng(seed, c.cfg, layer, 0x5A17)
    w = rng.standard_normal((c.E, c.H), dtype=np.float64) * 0.02
    if c.cfg == 3:
        r = _rng(seed, c.cfg, layer, 0x21FF).permutation(c.E) + 1  # ranks 1..E
        b = ZIPF_BETA * r.astype(np.float64) ** (-ZIPF_S)
    else:
        b = np.zeros(c.E)
    return w.astype(np.float32), b.astype(np.float32)


def activations(c: Config, seed: int, step: int, layer: int, subseeds=None):
    """Stored activations for one (step, layer) call: fp32 [T,H] or bf16 bits uint16 [T,H].

    subseeds: optional int array [T]; token t is drawn from sub-seed subseeds[t]
    (used to redraw single tokens whose routing scores nearly tie)."""
    T, H = c.T, c.H
    if subseeds is None:
        subseeds = np.zeros(T, np.int64)
    subseeds = np.asarray(subseeds)
    if c.cfg == 2:
        z0 = _rng(seed, c.cfg, step, layer, 0xC0, 0).standard_normal(H)
        x = np.empty((T, H))
        for t in range(T):
            zt = _rng(seed, c.cfg, step, layer, 0xC1 + t, subseeds[t]).standard_normal(H)
            if t == 0 and subseeds[0] != 0:
                z0 = zt
            x[t] = z0 if t == 0 else math.sqrt(VERIFY_RHO) * z0 + math.sqrt(1 - VERIFY_RHO) * zt
    elif np.all(subseeds == 0):
        x = _rng(seed, c.cfg, step, layer, 0xA0).standard_normal((T, H))
    else:
        x = _rng(seed, c.cfg, step, layer, 0xA0).standard_normal((T, H))
        for t in np.nonzero(subseeds)[0]:
            x[t] = _rng(seed, c.cfg, step, layer, 0xA1, t, subseeds[t]).standard_normal(H)
    x32 = x.astype(np.float32)
    return x32 if c.x_dtype == "f32" else to_bf16_bits(x32)


# ---------------------------------------------------------------------------
# expert weights

def gen_expert_host(c: Config, seed: int, layer: int, expert: int):
    """All six arrays of one expert (expert == E is the shared expert), on the host."""
    L = lib()
    out = {}
    for which, name, N, K in ((0, "gate", c.F, c.H), (1, "up", c.F, c.H), (2, "down", c.H, c.F)):
        q = np.empty(N * K // 2, np.uint8)
        s = np.empty(N * K // 64, np.float32)
        rc = L.coli_inputs_gen_matrix_host(seed, layer, expert, which, N, K,
                                           q.ctypes.data, s.ctypes.data)
        if rc != 0:
            raise RuntimeError("host weight generation failed")
        out[name + "_q"] = q.reshape(N, K // 2)
        out[name + "_s"] = s.reshape(N, K // 64)
    return out


def gen_layer_device(c: Config, seed: int, layer: int, bufs: dict, stream_ptr: int):
    """Fill device buffers gate_q/gate_s/up_q/up_s/down_q/down_s (E+1 experts each,
    expert-major) for one layer.  bufs maps names to device pointers."""
    L = lib()
    for which, name, N, K in ((0, "gate", c.F, c.H), (1, "up", c.F, c.H), (2, "down", c.H, c.F)):
        rc = L.coli_inputs_gen_matrix_device(seed, layer, 0, c.E + 1, which, N, K,
                                             bufs[name + "_q"], bufs[name + "_s"], stream_ptr)
        if rc != 0:
            raise RuntimeError("device weight generation failed")


# ---------------------------------------------------------------------------
# cfg 0: Gaussian weights quantised to int4-gs64 (numpy default_rng(0))

def quantise_gs64(w):
    """Symmetric per-64 quantisation of a f64 matrix [N,K] (data preparation only):
    s = absmax/7 (1 if the group is all zero), q = clamp(rint(w / s), -8, 7)."""
    N, K = w.shape
    g = w.reshape(N, K // 64, 64)
    amax = np.abs(g).max(axis=2)
    s = np.where(amax > 0, amax / 7.0, 1.0).astype(np.float32)
    q = np.clip(np.rint(g / s[:, :, None].astype(np.float64)), -8, 7).astype(np.int64)
    return pack_int4(q.reshape(N, K)), s


def pack_int4(q):
    """Pack integers in [-8,7] of shape [N,K] into bytes [N,K/2], low nibble = even k."""
    q = np.asarray(q, np.int64)
    if q.min() < -8 or q.max() > 7:
        raise ValueError("int4 value out of range")
    u = (q & 0xF).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def tiny_layer(seed=0):
    """cfg 0 in the fixed draw order W_r, b, (gate, up, down) per expert, shared last, x."""
    c = CONFIGS[0]
    rng = np.random.default_rng(seed)
    w_router = (rng.standard_normal((c.E, c.H)) * 0.02).astype(np.float32)
    sel_bias = (rng.standard_normal(c.E) * 0.02).astype(np.float32)
    experts = {}
    for e in range(c.E + 1):
        ex = {}
        for name, N, K in (("gate", c.F, c.H), ("up", c.F, c.H), ("down", c.H, c.F)):
            q, s = quantise_gs64(rng.standard_normal((N, K)) * 0.02)
            ex[name + "_q"] = q
            ex[name + "_s"] = s
        experts[e] = ex
    x = rng.standard_normal((c.T, c.H)).astype(np.float32)
    return dict(w_router=w_router, sel_bias=sel_bias, experts=experts, x=x)


def tiny_redraw(t, subseed, seed=0):
    """Replacement fp32 activation row for token t of cfg 0 (sub-seed >= 1)."""
    return _rng(seed, 0, 0xA2, t, subseed).standard_normal(CONFIGS[0].H).astype(np.float32)


def stack_experts(experts, E):
    """Stack a dict {e: six arrays} for e = 0..E into expert-major arrays."""
    return {n: np.stack([experts[e][n] for e in range(E + 1)]) for n in
            ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")}


def device_layer_tensors(torch, c: Config, seed: int, layer: int, device="cuda"):
    """Allocate and fill one layer's expert weights on the device (torch tensors,
    expert-major, shared expert last)."""
    E1 = c.E + 1
    bufs = dict(
        gate_q=torch.empty((E1, c.F, c.H // 2), dtype=torch.uint8, device=device),
        gate_s=torch.empty((E1, c.F, c.H // 64), dtype=torch.float32, device=device),
        up_q=torch.empty((E1, c.F, c.H // 2), dtype=torch.uint8, device=device),
        up_s=torch.empty((E1, c.F, c.H // 64), dtype=torch.float32, device=device),
        down_q=torch.empty((E1, c.H, c.F // 2), dtype=torch.uint8, device=device),
        down_s=torch.empty((E1, c.H, c.F // 64), dtype=torch.float32, device=device))
    gen_layer_device(c, seed, layer, {n: t.data_ptr() for n, t in bufs.items()},
                     torch.cuda.current_stream().cuda_stream)
    return bufs
