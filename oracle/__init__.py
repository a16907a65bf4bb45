"""CPU oracle for the DeepSeek-V3 MoE layer forward pass (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``fine_grained_moe_gemm_b200``) never does, and shares no code with it.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64 accumulation); this
module compiles it with gcc and exposes numpy-level wrappers.  Every function
names the page and box it follows in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile ``moe_oracle.c`` into ``oracle/liboracle.so`` (gcc, -ffp-contract=off)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-pthread", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class OrcLayer(ctypes.Structure):
    _fields_ = [
        ("d", ctypes.c_int), ("E", ctypes.c_int), ("H", ctypes.c_int), ("Hs", ctypes.c_int),
        ("k", ctypes.c_int), ("x_is_f32", ctypes.c_int), ("fp8", ctypes.c_int),
        ("routed_scale", ctypes.c_double),
        ("w_gate", ctypes.POINTER(ctypes.c_void_p)), ("w_up", ctypes.POINTER(ctypes.c_void_p)),
        ("w_down", ctypes.POINTER(ctypes.c_void_p)),
        ("s_gate", ctypes.POINTER(ctypes.c_void_p)), ("s_up", ctypes.POINTER(ctypes.c_void_p)),
        ("s_down", ctypes.POINTER(ctypes.c_void_p)),
        ("ws_gate", ctypes.c_void_p), ("ws_up", ctypes.c_void_p), ("ws_down", ctypes.c_void_p),
        ("ss_gate", ctypes.c_void_p), ("ss_up", ctypes.c_void_p), ("ss_down", ctypes.c_void_p),
    ]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            L.orc_sigmoid.restype = ctypes.c_float
            L.orc_sigmoid.argtypes = [ctypes.c_float]
            L.orc_sigmoid_array.argtypes = [P, P, ctypes.c_int64]
            L.orc_bf16_from_f64.restype = ctypes.c_uint16
            L.orc_bf16_from_f64.argtypes = [ctypes.c_double]
            L.orc_bf16_to_f64.restype = ctypes.c_double
            L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
            L.orc_e4m3_from_f32.restype = ctypes.c_uint8
            L.orc_e4m3_from_f32.argtypes = [ctypes.c_float]
            L.orc_e4m3_to_f64.restype = ctypes.c_double
            L.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
            L.orc_router_logits.argtypes = [P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
            L.orc_select.restype = ctypes.c_int
            L.orc_select.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
            L.orc_permute.restype = ctypes.c_int
            L.orc_permute.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P]
            L.orc_quant_act.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P]
            L.orc_update_bias.argtypes = [P, ctypes.c_int, P, ctypes.c_float]
            L.orc_rmsnorm.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_double, P]
            L.orc_expert_tokens.restype = ctypes.c_int
            L.orc_expert_tokens.argtypes = [ctypes.POINTER(OrcLayer), P, P, P, P, ctypes.c_int, ctypes.c_int, P]
            L.orc_expert_single.argtypes = [ctypes.POINTER(OrcLayer), ctypes.c_int, P, P]
            _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------- scalars

def sigmoid(l) -> np.ndarray:
    """sigmoid_spec on an fp32 array (router box: ``logits.sigmoid()``)."""
    a = np.ascontiguousarray(np.asarray(l, dtype=np.float32))
    out = np.empty_like(a)
    lib().orc_sigmoid_array(_ptr(a), _ptr(out), a.size)
    return out


def bf16_from_f64(v: float) -> int:
    return int(lib().orc_bf16_from_f64(float(v)))


def bf16_to_f64(h: int) -> float:
    return float(lib().orc_bf16_to_f64(int(h)))


def e4m3_from_f32(v: float) -> int:
    return int(lib().orc_e4m3_from_f32(float(np.float32(v))))


def e4m3_to_f64(c: int) -> float:
    return float(lib().orc_e4m3_to_f64(int(c)))


def bf16_bits_from_f64_array(v: np.ndarray) -> np.ndarray:
    f = lib().orc_bf16_from_f64
    flat = np.asarray(v, dtype=np.float64).ravel()
    return np.array([f(float(x)) for x in flat], dtype=np.uint16).reshape(np.shape(v))


def bf16_bits_to_f64_array(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp64 values (the top half of a binary32)."""
    u = (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16)
    return u.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- stages

def router_logits(x: np.ndarray, w_router_bf16: np.ndarray) -> np.ndarray:
    """S1: fp32 logits [T, E] with fp64 accumulation.  ``x`` is fp32 or bf16 bits (uint16)."""
    x = np.ascontiguousarray(x)
    w = np.ascontiguousarray(w_router_bf16, dtype=np.uint16)
    T, d = x.shape
    E = w.shape[0]
    assert w.shape[1] == d
    out = np.empty((T, E), dtype=np.float32)
    lib().orc_router_logits(_ptr(x), 1 if x.dtype == np.float32 else 0, _ptr(w), T, d, E, _ptr(out))
    return out


def select(logits: np.ndarray, bias: np.ndarray, n_groups: int, topk_groups: int, top_k: int):
    """S2: group-limited top-k.  Returns (idx int32 [T,k], w fp32 [T,k])."""
    l = np.ascontiguousarray(logits, dtype=np.float32)
    b = np.ascontiguousarray(bias, dtype=np.float32)
    T, E = l.shape
    idx = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float32)
    rc = lib().orc_select(_ptr(l), _ptr(b), T, E, n_groups, topk_groups, top_k, _ptr(idx), _ptr(w))
    if rc != 0:
        raise ValueError("oracle select: invalid sizes")
    return idx, w


def permute(idx: np.ndarray, n_experts: int):
    """S3: counting sort of (t, j) pairs by expert, ascending t inside each expert."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.empty(n_experts, dtype=np.int32)
    offsets = np.empty(n_experts + 1, dtype=np.int32)
    src = np.empty(T * k, dtype=np.int32)
    inv = np.empty(T * k, dtype=np.int32)
    rc = lib().orc_permute(_ptr(idx), T, k, n_experts, _ptr(counts), _ptr(offsets), _ptr(src), _ptr(inv))
    if rc != 0:
        raise ValueError("oracle permute: expert id out of range")
    return counts, offsets, src, inv


def update_bias(counts: np.ndarray, bias: np.ndarray, gamma: float = 1e-3) -> np.ndarray:
    """Bias controller ("MoE router" box, update_bias): a new fp32 bias, -gamma for
    experts above the mean count, +gamma for the others."""
    c = np.ascontiguousarray(counts, dtype=np.int32)
    b = np.ascontiguousarray(bias, dtype=np.float32).copy()
    lib().orc_update_bias(_ptr(c), c.size, _ptr(b), float(np.float32(gamma)))
    return b


RMS_EPS = float(np.float32(1e-6))  # the page's eps, as the fp32 value an fp32 tensor adds


def rmsnorm(h_bf16: np.ndarray, g_bf16: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """Pre-norm ("RMSNorm" box): bf16(bf16(h * r) * g), r = 1/sqrt(mean(h^2) + eps) in fp64.
    Inputs and output are bf16 bit patterns (uint16)."""
    h = np.ascontiguousarray(h_bf16, dtype=np.uint16)
    g = np.ascontiguousarray(g_bf16, dtype=np.uint16)
    T, d = h.shape
    assert g.shape == (d,)
    out = np.empty((T, d), dtype=np.uint16)
    lib().orc_rmsnorm(_ptr(h), _ptr(g), T, d, float(eps), _ptr(out))
    return out


def quant_act(x_bf16: np.ndarray):
    """S6: per-token, per-128-channel e4m3 quantisation.  Returns (codes uint8, scales fp32)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, d = x.shape
    assert d % 128 == 0
    q = np.empty((T, d), dtype=np.uint8)
    sx = np.empty((T, d // 128), dtype=np.float32)
    lib().orc_quant_act(_ptr(x), T, d, _ptr(q), _ptr(sx))
    return q, sx


class Layer:
    """Weights of one MoE layer as host arrays, in the layouts the oracle reads.

    Routed weights are given per expert (a list of E arrays, ``None`` for an
    expert the caller does not need), so that a full-size check can hand over
    only the experts its sampled tokens use.
    """

    def __init__(self, d, n_experts, hidden, shared_hidden, top_k, routed_scale,
                 w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                 s_gate=None, s_up=None, s_down=None, ss_gate=None, ss_up=None, ss_down=None,
                 x_is_f32=False):
        self.keep = []  # keeps every array alive while the struct points at it
        fp8 = s_gate is not None

        def arr(a, dt):
            a = np.ascontiguousarray(a, dtype=dt)
            self.keep.append(a)
            return a

        def plist(lst, dt):
            ptrs = (ctypes.c_void_p * n_experts)()
            for e in range(n_experts):
                a = lst[e] if lst is not None else None
                ptrs[e] = _ptr(arr(a, dt)).value if a is not None else None
            self.keep.append(ptrs)
            return ctypes.cast(ptrs, ctypes.POINTER(ctypes.c_void_p))

        wdt = np.uint8 if fp8 else np.uint16
        s = OrcLayer()
        s.d, s.E, s.H, s.Hs, s.k = d, n_experts, hidden, shared_hidden, top_k
        s.x_is_f32, s.fp8, s.routed_scale = int(x_is_f32), int(fp8), float(routed_scale)
        s.w_gate, s.w_up, s.w_down = plist(w_gate, wdt), plist(w_up, wdt), plist(w_down, wdt)
        if fp8:
            s.s_gate, s.s_up, s.s_down = (plist(s_gate, np.float32), plist(s_up, np.float32),
                                          plist(s_down, np.float32))
            s.ss_gate = _ptr(arr(ss_gate, np.float32)).value
            s.ss_up = _ptr(arr(ss_up, np.float32)).value
            s.ss_down = _ptr(arr(ss_down, np.float32)).value
        s.ws_gate = _ptr(arr(ws_gate, wdt)).value
        s.ws_up = _ptr(arr(ws_up, wdt)).value
        s.ws_down = _ptr(arr(ws_down, wdt)).value
        self.s = s
        self.d = d


def expert_tokens(layer: Layer, x: np.ndarray, idx: np.ndarray, w: np.ndarray, tokens, n_threads=None):
    """S4+S5: fp64 layer output (before any residual) for the listed tokens.

    ``x`` holds all T tokens (fp32 or bf16 bits), ``idx``/``w`` the routing of all
    T tokens.  Returns fp64 [len(tokens), d].
    """
    x = np.ascontiguousarray(x)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
    n = int(tok.size)
    y = np.empty((n, layer.d), dtype=np.float64)
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    n_threads = max(1, min(int(n_threads), n))
    if n == 0:
        return y
    rc = lib().orc_expert_tokens(ctypes.byref(layer.s), _ptr(x), _ptr(idx), _ptr(w), _ptr(tok), n,
                                 n_threads, _ptr(y))
    if rc != 0:
        raise ValueError("oracle expert_tokens: routed expert missing or out of range")
    return y


def dense_ffn(x: np.ndarray, w_gate, w_up, w_down, s_gate=None, s_up=None, s_down=None, tokens=None,
              x_is_f32=False, n_threads=None) -> np.ndarray:
    """Dense SwiGLU FFN ("SwiGLU MLP" box; the first layers of the model have a dense FFN
    of hidden 18432 instead of experts): fp64 y = W_down(SiLU(W_gate x) * (W_up x)) for the
    listed tokens, h stored in bf16 (e4m3 with 1x128 scales when the weights are e4m3 with
    128x128 block scales, and x quantised per 1x128 tile).  It is the layer's expert math
    with no routed expert and the dense weights in the always-on slot."""
    d = x.shape[1]
    Hd = np.asarray(w_gate).shape[0]
    fp8 = s_gate is not None
    kw = dict(s_gate=[], s_up=[], s_down=[], ss_gate=s_gate, ss_up=s_up, ss_down=s_down) if fp8 else {}
    L = Layer(d, 0, Hd, Hd, 0, 1.0, [], [], [], w_gate, w_up, w_down, x_is_f32=x_is_f32, **kw)
    T = x.shape[0]
    tokens = np.arange(T, dtype=np.int32) if tokens is None else tokens
    return expert_tokens(L, x, np.zeros((T, 0), np.int32), np.zeros((T, 0), np.float32), tokens, n_threads)


def expert_single(layer: Layer, e: int, xh: np.ndarray) -> np.ndarray:
    """One expert (e < 0: shared) on an fp64 input row, for closed-form pins."""
    xh = np.ascontiguousarray(xh, dtype=np.float64)
    o = np.empty(layer.d, dtype=np.float64)
    lib().orc_expert_single(ctypes.byref(layer.s), int(e), _ptr(xh), _ptr(o))
    return o
