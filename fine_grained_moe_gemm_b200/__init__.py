"""B200 (sm_100a) DeepSeek-V3 MoE layer forward pass: Python binding of the C ABI.

Argument marshalling only: every step of the layer runs in the CUDA kernels
of ``libmoe_b200.so`` (``include/moe.h``).  PyTorch supplies device memory and
streams.  There is no CPU fallback: without the built library every call
raises.

    cfg = MoeConfig(d=7168, n_experts=256, n_groups=8, topk_groups=4, top_k=8,
                    hidden=2048, n_shared=1, shared_hidden=2048, routed_scale=2.5)
    ws = torch.empty(workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    moe_forward(cfg, weights, x, bias, y, workspace=ws)
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "libmoe_b200_debug.so")
_DEFAULT_LIB_PATH = LIB_PATH
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_DEVICE, MOE_ERR_CUDA = range(6)
MOE_F32, MOE_BF16, MOE_E4M3 = 0, 1, 2
MOE_DEVERR_BAD_EXPERT, MOE_DEVERR_TIMEOUT, MOE_DEVERR_BAD_ROWS, MOE_DEVERR_NONFINITE, MOE_DEVERR_BOUNDS = 1, 2, 4, 8, 16
MOE_DEBUG_TABLE_ROW_TOK, MOE_DEBUG_TABLE_ROW_OFF = 0, 1

_lib = None
_lock = threading.Lock()


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class MoeConfig(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("n_experts", ctypes.c_int), ("n_groups", ctypes.c_int),
                ("topk_groups", ctypes.c_int), ("top_k", ctypes.c_int), ("hidden", ctypes.c_int),
                ("n_shared", ctypes.c_int), ("shared_hidden", ctypes.c_int), ("routed_scale", ctypes.c_float),
                ("act_dtype", ctypes.c_int), ("weight_dtype", ctypes.c_int)]

    def __init__(self, d, n_experts, n_groups, topk_groups, top_k, hidden, n_shared=1, shared_hidden=None,
                 routed_scale=2.5, act_dtype=MOE_BF16, weight_dtype=MOE_BF16):
        super().__init__(d, n_experts, n_groups, topk_groups, top_k, hidden, n_shared,
                         hidden if shared_hidden is None else shared_hidden, routed_scale, act_dtype, weight_dtype)


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_router", "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down",
        "ws_gate", "ws_up", "ws_down", "ss_gate", "ss_up", "ss_down")]


def _configure(L):
    """Result and argument types of every entry point of a loaded library."""
    P, I = ctypes.c_void_p, ctypes.c_int
    L.moe_workspace_size.restype = ctypes.c_size_t
    L.moe_workspace_size.argtypes = [ctypes.POINTER(MoeConfig), I]
    L.moe_route.restype = I
    L.moe_route.argtypes = [ctypes.POINTER(MoeConfig), P, P, P, P, I, P, P, P]
    L.moe_permute.restype = I
    L.moe_permute.argtypes = [ctypes.POINTER(MoeConfig), P, I, P, P, P, P, P]
    L.moe_forward.restype = I
    L.moe_forward.argtypes = [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), P, P, I, P, I, I, P,
                              ctypes.c_size_t, P]
    L.moe_forward_ex.restype = I
    L.moe_forward_ex.argtypes = [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), P, P, I, P, I, I, P,
                                 ctypes.c_size_t, P, P, P]
    L.moe_host_workspace_size.restype = ctypes.c_size_t
    L.moe_host_workspace_size.argtypes = [ctypes.POINTER(MoeConfig), I, I]
    L.moe_forward_host.restype = I
    L.moe_forward_host.argtypes = [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), P, P, I, P, I, I, P,
                                   ctypes.c_size_t, P]
    L.moe_ep_max_send_rows.restype = I
    L.moe_ep_max_send_rows.argtypes = [ctypes.POINTER(MoeConfig), I, I]
    L.moe_ep_dispatch.restype = I
    L.moe_ep_dispatch.argtypes = [ctypes.POINTER(MoeConfig), I, P, P, P, I, P, P, P, P, P, P, P]
    L.moe_experts_routed_workspace_size.restype = ctypes.c_size_t
    L.moe_experts_routed_workspace_size.argtypes = [ctypes.POINTER(MoeConfig), I, I]
    L.moe_experts_routed.restype = I
    L.moe_experts_routed.argtypes = [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), I, I, P, I, P, P,
                                     P, P, ctypes.c_size_t, P]
    L.moe_ep_combine.restype = I
    L.moe_ep_combine.argtypes = [I, I, I, P, P, P, P, P, P]
    L.moe_rmsnorm.restype = I
    L.moe_rmsnorm.argtypes = [P, P, ctypes.c_float, I, I, P, P, P, P]
    L.moe_block_workspace_size.restype = ctypes.c_size_t
    L.moe_block_workspace_size.argtypes = [ctypes.POINTER(MoeConfig), I]
    L.moe_forward_block.restype = I
    L.moe_forward_block.argtypes = [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), P, ctypes.c_float,
                                    P, P, I, P, P, ctypes.c_size_t, P, P, P]
    L.moe_dense_workspace_size.restype = ctypes.c_size_t
    L.moe_dense_workspace_size.argtypes = [I, I, I, I, I]
    L.moe_dense_ffn.restype = I
    L.moe_dense_ffn.argtypes = [I, I, I, I, P, P, P, P, P, P, P, I, P, I, I, P, ctypes.c_size_t, P, P]
    L.moe_forward_plan.restype = I
    L.moe_forward_plan.argtypes = [ctypes.POINTER(MoeConfig), I, I, ctypes.c_void_p]
    L.moe_selftest_wait_timeout.restype = I
    L.moe_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, P]
    L.moe_launch_count.restype = ctypes.c_ulonglong
    L.moe_launch_count.argtypes = []
    L.moe_update_bias.restype = I
    L.moe_update_bias.argtypes = [ctypes.POINTER(MoeConfig), P, P, ctypes.c_float, P]
    L.moe_quantize_act.restype = I
    L.moe_quantize_act.argtypes = [P, I, I, P, P, P]
    L.moe_device_error.restype = I
    L.moe_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), P]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [I]
    L.moe_abi_version.restype = I
    L.moe_ep_packed_row_bytes.restype = ctypes.c_size_t
    L.moe_ep_packed_row_bytes.argtypes = [ctypes.POINTER(MoeConfig)]
    L.moe_ep_dispatch_packed.restype = I
    L.moe_ep_dispatch_packed.argtypes = [ctypes.POINTER(MoeConfig), I, I, P, P, P, I, P, P, P, P]
    L.moe_ep_unpack.restype = I
    L.moe_ep_unpack.argtypes = [ctypes.POINTER(MoeConfig), I, P, P, P, P, P]
    L.moe_ep_dispatch_peer.restype = I
    L.moe_ep_dispatch_peer.argtypes = [ctypes.POINTER(MoeConfig), I, I, I, P, P, P, I, P, P, P, P]
    L.moe_ep_combine_peer.restype = I
    L.moe_ep_combine_peer.argtypes = [I, I, I, I, I, P, P, P, P, P, P]
    L.moe_forward_noalloc.restype = I
    L.moe_forward_noalloc.argtypes = [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), P, P, I, P, I, I, P]
    L.moe_debug_build.restype = I
    L.moe_debug_build.argtypes = []
    L.moe_debug_corrupt_next.restype = I
    L.moe_debug_corrupt_next.argtypes = [I, I, I]
    return L


def lib():
    """The loaded ``libmoe_b200.so``.  The in-tree library is (re)built first when it is
    missing or older than its sources and nvcc is at hand; without it the call raises
    (there is no CPU fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if os.path.abspath(LIB_PATH) == os.path.abspath(_DEFAULT_LIB_PATH):
                try:
                    from . import build as _build
                    _build.build()  # a no-op when the library is newer than every source
                except Exception as e:
                    if not os.path.exists(LIB_PATH):
                        raise RuntimeError(f"{LIB_PATH} is missing and could not be built: {e}") from e
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with fine_grained_moe_gemm_b200.build.build() "
                                   "(there is no CPU fallback)")
            _lib = _configure(ctypes.CDLL(LIB_PATH))
    return _lib


_debug_lib = None


def debug_lib():
    """The checking build ``libmoe_b200_debug.so`` (the same entry points; kernels
    check every table-dependent access against its buffer and flag
    MOE_DEVERR_BOUNDS instead of touching memory outside it).  Built with the
    regular library."""
    global _debug_lib
    lib()  # builds both libraries when they are stale
    with _lock:
        if _debug_lib is None:
            if not os.path.exists(DEBUG_LIB_PATH):
                raise RuntimeError(f"{DEBUG_LIB_PATH} is missing: build it with fine_grained_moe_gemm_b200.build.build()")
            _debug_lib = _configure(ctypes.CDLL(DEBUG_LIB_PATH))
    return _debug_lib


def declared_symbols() -> list[str]:
    """Entry points declared in include/moe.h."""
    text = open(HEADER_PATH).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MOE_F32
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return MOE_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t: torch.Tensor, name: str):
    if t is not None and (not t.is_cuda or not t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if t is not None and t.device.index != torch.cuda.current_device():
        # the library launches on the current device: a pointer into another GPU is not its memory
        raise ValueError(f"{name} is on {t.device}, the current device is cuda:{torch.cuda.current_device()}")


def _shape(t, name, shape, dtypes):
    """The C ABI takes raw pointers: check here what it cannot (shape and element type)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")


_ACT = {MOE_F32: (torch.float32,), MOE_BF16: (torch.bfloat16,)}
_OUT = (torch.float32, torch.bfloat16)


def workspace_size(cfg: MoeConfig, T: int) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(cfg), int(T)))


def moe_route(cfg: MoeConfig, x, w_router, logits, bias, topk_idx, topk_w, stream=None):
    """Router + selection.  ``x=None``: ``logits`` is an input (logits-in mode)."""
    for n, t in (("x", x), ("w_router", w_router), ("logits", logits), ("bias", bias), ("topk_idx", topk_idx),
                 ("topk_w", topk_w)):
        _dev(t, n)
    T = logits.shape[0]
    E, k = cfg.n_experts, cfg.top_k
    _shape(x, "x", (T, cfg.d), _ACT.get(cfg.act_dtype, ()))
    _shape(w_router, "w_router", (E, cfg.d), (torch.bfloat16,))
    _shape(logits, "logits", (T, E), (torch.float32,))
    _shape(bias, "bias", (E,), (torch.float32,))
    _shape(topk_idx, "topk_idx", (T, k), (torch.int32,))
    _shape(topk_w, "topk_w", (T, k), (torch.float32,))
    _check(lib().moe_route(ctypes.byref(cfg), _p(x), _p(w_router), _p(logits), _p(bias), T, _p(topk_idx),
                           _p(topk_w), _stream(stream)), "moe_route")


def moe_permute(cfg: MoeConfig, topk_idx, counts, offsets, src, inv, stream=None):
    for n, t in (("topk_idx", topk_idx), ("counts", counts), ("offsets", offsets), ("src", src), ("inv", inv)):
        _dev(t, n)
    T = topk_idx.shape[0]
    E, k = cfg.n_experts, cfg.top_k
    _shape(topk_idx, "topk_idx", (T, k), (torch.int32,))
    for n, t, shp in (("counts", counts, (E,)), ("offsets", offsets, (E + 1,))):
        _shape(t, n, shp, (torch.int32,))
    for n, t in (("src", src), ("inv", inv)):  # flat buffers of at least T * k entries
        if t.dtype != torch.int32 or t.dim() != 1 or t.numel() < T * k:
            raise ValueError(f"{n}: needs an int32 vector of at least {T * k} entries")
    _check(lib().moe_permute(ctypes.byref(cfg), _p(topk_idx), T, _p(counts), _p(offsets), _p(src), _p(inv),
                             _stream(stream)), "moe_permute")


def make_weights(w: dict) -> MoeWeights:
    """MoeWeights from a dict of CUDA tensors (keys as in ``MoeWeights``; missing keys are NULL)."""
    mw = MoeWeights()
    for name, _ in MoeWeights._fields_:
        t = w.get(name)
        if t is not None:
            _dev(t, name)
            setattr(mw, name, t.data_ptr())
    return mw


class MoeStageEvents(ctypes.Structure):
    _fields_ = [("ev", ctypes.c_void_p * 6)]


class MoeRoutingOut(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("logits", "topk_idx", "topk_w", "counts", "offsets", "src", "inv")]


class MoePlan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("token_tile", "cta_pair", "fp8", "router_splits", "permute_ctas",
                                            "launches")]


STAGES = ("route", "permute+gather", "gate_up", "down+combine", "cast")


def forward_plan(cfg: MoeConfig, T: int, y_dtype=torch.bfloat16) -> dict:
    """The kernels ``moe_forward`` runs for ``T`` tokens on the current device (see ``MoePlan``)."""
    plan = MoePlan()
    code = MOE_F32 if y_dtype == torch.float32 else MOE_BF16
    _check(lib().moe_forward_plan(ctypes.byref(cfg), int(T), code, ctypes.byref(plan)), "moe_forward_plan")
    return {n: getattr(plan, n) for n, _ in MoePlan._fields_}


def _events(stage_events):
    if stage_events is None:
        return None
    ev = MoeStageEvents()
    for i, e in enumerate(stage_events):
        if e is not None and e.cuda_event == 0:
            e.record()  # torch creates the underlying event lazily
        ev.ev[i] = e.cuda_event if e is not None else None
    return ev


def _routing(routing_out):
    if routing_out is None:
        return None
    ro = MoeRoutingOut()
    for name, _ in MoeRoutingOut._fields_:
        t = routing_out.get(name)
        if t is not None:
            _dev(t, name)
            setattr(ro, name, t.data_ptr())
    return ro


def moe_forward(cfg: MoeConfig, weights, x, bias, y, accumulate: bool = False, workspace=None, stream=None,
                stage_events=None, routing_out=None):
    """y (+)= MoE(x).  ``weights`` is a MoeWeights or a dict of tensors; ``workspace`` a uint8 CUDA tensor of at
    least ``workspace_size(cfg, T)`` bytes.  ``stage_events``: optional list of six torch.cuda.Event(
    enable_timing=True) recorded around the stages (see ``STAGES``).  ``routing_out``: optional dict with any of
    ``logits`` [T, E] f32, ``topk_idx`` [T, k] int32, ``topk_w`` [T, k] f32 CUDA tensors that receive the routing
    the layer used, and ``counts`` [E], ``offsets`` [E+1], ``src``/``inv`` [T*k] int32 for its permutation."""
    for n, t in (("x", x), ("bias", bias), ("y", y), ("workspace", workspace)):
        _dev(t, n)
    mw = weights if isinstance(weights, MoeWeights) else make_weights(weights)
    T = x.shape[0]
    _shape(x, "x", (T, cfg.d), _ACT.get(cfg.act_dtype, ()))
    _shape(bias, "bias", (cfg.n_experts,), (torch.float32,))
    _shape(y, "y", (T, cfg.d), _OUT)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    ev, ro = _events(stage_events), _routing(routing_out)
    _check(lib().moe_forward_ex(ctypes.byref(cfg), ctypes.byref(mw), _p(x), _p(bias), T, _p(y), _dtype_code(y),
                                1 if accumulate else 0, _p(workspace), ws_bytes, _stream(stream),
                                ctypes.byref(ev) if ev is not None else None,
                                ctypes.byref(ro) if ro is not None else None), "moe_forward")


def host_workspace_size(cfg: MoeConfig, T: int, y_dtype=torch.bfloat16) -> int:
    """Device workspace bytes of ``moe_forward_host`` for up to T tokens."""
    code = MOE_F32 if y_dtype == torch.float32 else MOE_BF16
    return int(lib().moe_host_workspace_size(ctypes.byref(cfg), int(T), code))


def _host(t: torch.Tensor, name: str):
    if t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host (CPU) tensor")


def moe_forward_host(cfg: MoeConfig, weights, x_host, bias, y_host, accumulate: bool = False, workspace=None,
                     stream=None):
    """y_host (+)= MoE(x_host) with the activations in host memory: the call enqueues the copy in, the layer and
    the copy out on ``stream`` and returns; ``y_host`` holds the result once the stream has passed that work.
    Pin both host tensors (``pin_memory()``) for the copies to be asynchronous.  ``workspace``: a uint8 CUDA
    tensor of at least ``host_workspace_size(cfg, T, y_host.dtype)`` bytes."""
    _host(x_host, "x_host")
    _host(y_host, "y_host")
    for n, t in (("bias", bias), ("workspace", workspace)):
        _dev(t, n)
    mw = weights if isinstance(weights, MoeWeights) else make_weights(weights)
    T = x_host.shape[0]
    _shape(x_host, "x_host", (T, cfg.d), _ACT.get(cfg.act_dtype, ()))
    _shape(bias, "bias", (cfg.n_experts,), (torch.float32,))
    _shape(y_host, "y_host", (T, cfg.d), _OUT)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().moe_forward_host(ctypes.byref(cfg), ctypes.byref(mw), _p(x_host), _p(bias), T, _p(y_host),
                                  _dtype_code(y_host), 1 if accumulate else 0, _p(workspace), ws_bytes,
                                  _stream(stream)), "moe_forward_host")


def ep_max_send_rows(cfg: MoeConfig, T: int, n_ranks: int) -> int:
    """Rows the dispatch of T tokens over n_ranks ranks can produce: T * min(k, n_ranks)."""
    return int(lib().moe_ep_max_send_rows(ctypes.byref(cfg), int(T), int(n_ranks)))


def moe_ep_dispatch(cfg: MoeConfig, n_ranks: int, topk_idx, topk_w, x, send_counts, send_offsets, send_tok, send_x,
                    send_idx, send_w, stream=None):
    """Expert-parallel dispatch: the rows this rank sends to each of ``n_ranks`` ranks (contiguous expert blocks),
    rank-major, each token once per rank.  Output arrays hold ``ep_max_send_rows(cfg, T, n_ranks)`` rows."""
    T = x.shape[0]
    rows = ep_max_send_rows(cfg, T, n_ranks)
    for n, t in (("topk_idx", topk_idx), ("topk_w", topk_w), ("x", x), ("send_counts", send_counts),
                 ("send_offsets", send_offsets), ("send_tok", send_tok), ("send_x", send_x),
                 ("send_idx", send_idx), ("send_w", send_w)):
        _dev(t, n)
    k = cfg.top_k
    _shape(topk_idx, "topk_idx", (T, k), (torch.int32,))
    _shape(topk_w, "topk_w", (T, k), (torch.float32,))
    _shape(x, "x", (T, cfg.d), _ACT.get(cfg.act_dtype, ()))
    _shape(send_counts, "send_counts", (n_ranks,), (torch.int32,))
    _shape(send_offsets, "send_offsets", (n_ranks + 1,), (torch.int32,))
    for n, t, shp, dt in (("send_tok", send_tok, (rows,), torch.int32), ("send_x", send_x, (rows, cfg.d), torch.bfloat16),
                          ("send_idx", send_idx, (rows, k), torch.int32), ("send_w", send_w, (rows, k), torch.float32)):
        if t.shape[0] < rows or tuple(t.shape[1:]) != shp[1:] or t.dtype != dt:
            raise ValueError(f"{n}: shape {tuple(t.shape)} {t.dtype}, expected at least {shp} {dt}")
    _check(lib().moe_ep_dispatch(ctypes.byref(cfg), int(n_ranks), _p(topk_idx), _p(topk_w), _p(x), T,
                                 _p(send_counts), _p(send_offsets), _p(send_tok), _p(send_x), _p(send_idx),
                                 _p(send_w), _stream(stream)), "moe_ep_dispatch")


def ep_packed_row_bytes(cfg: MoeConfig) -> int:
    """Bytes of one packed dispatch row: bf16 x | int32 ids | fp32 weights, padded to 16."""
    return int(lib().moe_ep_packed_row_bytes(ctypes.byref(cfg)))


def moe_ep_dispatch_packed(cfg: MoeConfig, n_ranks: int, capacity: int, topk_idx, topk_w, x, send_counts, send_tok,
                           packed, stream=None):
    """Fixed-capacity packed dispatch: rank q's rows at slots [q*capacity, q*capacity + send_counts[q]) of
    ``packed`` [n_ranks*capacity, ep_packed_row_bytes] uint8 and ``send_tok`` [n_ranks*capacity] int32; padding
    slots have token -1 and expert ids -1."""
    T = x.shape[0]
    for n, t in (("topk_idx", topk_idx), ("topk_w", topk_w), ("x", x), ("send_counts", send_counts),
                 ("send_tok", send_tok), ("packed", packed)):
        _dev(t, n)
    k, slots = cfg.top_k, n_ranks * capacity
    _shape(topk_idx, "topk_idx", (T, k), (torch.int32,))
    _shape(topk_w, "topk_w", (T, k), (torch.float32,))
    _shape(x, "x", (T, cfg.d), _ACT.get(cfg.act_dtype, ()))
    _shape(send_counts, "send_counts", (n_ranks,), (torch.int32,))
    _shape(send_tok, "send_tok", (slots,), (torch.int32,))
    _shape(packed, "packed", (slots, ep_packed_row_bytes(cfg)), (torch.uint8,))
    _check(lib().moe_ep_dispatch_packed(ctypes.byref(cfg), int(n_ranks), int(capacity), _p(topk_idx), _p(topk_w),
                                        _p(x), T, _p(send_counts), _p(send_tok), _p(packed), _stream(stream)),
           "moe_ep_dispatch_packed")


def _ptr_array(ptrs, n: int, name: str):
    """A device array of n device pointers: an int64 CUDA tensor of n entries, or the raw address of one."""
    if isinstance(ptrs, torch.Tensor):
        _dev(ptrs, name)
        if ptrs.dtype != torch.int64 or ptrs.numel() != n or not ptrs.is_contiguous():
            raise ValueError(f"{name}: expected {n} contiguous int64 device pointers, got {tuple(ptrs.shape)} "
                             f"{ptrs.dtype}")
        return _p(ptrs)
    return ctypes.c_void_p(int(ptrs))


def moe_ep_dispatch_peer(cfg: MoeConfig, n_ranks: int, capacity: int, my_rank: int, topk_idx, topk_w, x,
                         send_counts, send_tok, recv_bufs, stream=None):
    """Peer-memory packed dispatch: rank q's rows written straight into rank q's receive buffer (entry q of
    ``recv_bufs``, n_ranks device pointers) at slots [my_rank*capacity, ...), padding marked as in
    moe_ep_dispatch_packed; ``send_tok`` [n_ranks*capacity] as there."""
    T = x.shape[0]
    for n, t in (("topk_idx", topk_idx), ("topk_w", topk_w), ("x", x), ("send_counts", send_counts),
                 ("send_tok", send_tok)):
        _dev(t, n)
    k, slots = cfg.top_k, n_ranks * capacity
    _shape(topk_idx, "topk_idx", (T, k), (torch.int32,))
    _shape(topk_w, "topk_w", (T, k), (torch.float32,))
    _shape(x, "x", (T, cfg.d), _ACT.get(cfg.act_dtype, ()))
    _shape(send_counts, "send_counts", (n_ranks,), (torch.int32,))
    _shape(send_tok, "send_tok", (slots,), (torch.int32,))
    _check(lib().moe_ep_dispatch_peer(ctypes.byref(cfg), int(n_ranks), int(capacity), int(my_rank), _p(topk_idx),
                                      _p(topk_w), _p(x), T, _p(send_counts), _p(send_tok),
                                      _ptr_array(recv_bufs, n_ranks, "recv_bufs"), _stream(stream)),
           "moe_ep_dispatch_peer")


def moe_ep_combine_peer(n_ranks: int, capacity: int, my_rank: int, result_bufs, send_tok, y_acc, y=None,
                        residual=None, stream=None):
    """Peer-memory combine: this rank's slot i read from the result buffer of rank i // capacity (entry of
    ``result_bufs``, n_ranks device pointers to [n_ranks*capacity, d] fp32) at row my_rank*capacity +
    i % capacity and added into y_acc[send_tok[i]]; then y = bf16(y_acc + residual) when ``y`` is given."""
    for n, t in (("send_tok", send_tok), ("y_acc", y_acc), ("y", y), ("residual", residual)):
        _dev(t, n)
    T, d = y_acc.shape
    _shape(y_acc, "y_acc", (T, d), (torch.float32,))
    _shape(send_tok, "send_tok", (n_ranks * capacity,), (torch.int32,))
    _shape(y, "y", (T, d), (torch.bfloat16,))
    _shape(residual, "residual", (T, d), (torch.bfloat16,))
    _check(lib().moe_ep_combine_peer(T, d, int(n_ranks), int(capacity), int(my_rank),
                                     _ptr_array(result_bufs, n_ranks, "result_bufs"), _p(send_tok), _p(y_acc), _p(y),
                                     _p(residual), _stream(stream)), "moe_ep_combine_peer")


def moe_ep_unpack(cfg: MoeConfig, packed, x_rows, topk_idx, topk_w, stream=None):
    """Packed rows -> x_rows [n, d] bf16, topk_idx / topk_w [n, k] (padding rows: ids -1)."""
    for n, t in (("packed", packed), ("x_rows", x_rows), ("topk_idx", topk_idx), ("topk_w", topk_w)):
        _dev(t, n)
    n = packed.shape[0]
    _shape(packed, "packed", (n, ep_packed_row_bytes(cfg)), (torch.uint8,))
    _shape(x_rows, "x_rows", (n, cfg.d), (torch.bfloat16,))
    _shape(topk_idx, "topk_idx", (n, cfg.top_k), (torch.int32,))
    _shape(topk_w, "topk_w", (n, cfg.top_k), (torch.float32,))
    _check(lib().moe_ep_unpack(ctypes.byref(cfg), n, _p(packed), _p(x_rows), _p(topk_idx), _p(topk_w),
                               _stream(stream)), "moe_ep_unpack")


def experts_routed_workspace_size(cfg: MoeConfig, n_local: int, n_rows: int) -> int:
    return int(lib().moe_experts_routed_workspace_size(ctypes.byref(cfg), int(n_local), int(n_rows)))


def moe_experts_routed(cfg: MoeConfig, local_weights, expert_lo: int, n_local: int, x_rows, topk_idx, topk_w, y_rows,
                       workspace=None, stream=None):
    """y_rows = routed_scale * sum of the experts of block [expert_lo, expert_lo + n_local) over the given rows'
    slots (the receiving side of the dispatch).  ``local_weights``: dict with the block's w_gate / w_up [n_local,
    H, d] and w_down [n_local, d, H] (e4m3: plus s_gate / s_up / s_down)."""
    for n, t in (("x_rows", x_rows), ("topk_idx", topk_idx), ("topk_w", topk_w), ("y_rows", y_rows),
                 ("workspace", workspace)):
        _dev(t, n)
    mw = local_weights if isinstance(local_weights, MoeWeights) else make_weights(local_weights)
    n = x_rows.shape[0]
    _shape(x_rows, "x_rows", (n, cfg.d), (torch.bfloat16,))
    _shape(topk_idx, "topk_idx", (n, cfg.top_k), (torch.int32,))
    _shape(topk_w, "topk_w", (n, cfg.top_k), (torch.float32,))
    _shape(y_rows, "y_rows", (n, cfg.d), (torch.float32,))
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().moe_experts_routed(ctypes.byref(cfg), ctypes.byref(mw), int(expert_lo), int(n_local), _p(x_rows), n,
                                    _p(topk_idx), _p(topk_w), _p(y_rows), _p(workspace), ws_bytes,
                                    _stream(stream)), "moe_experts_routed")


def moe_ep_combine(back_rows, send_tok, y_acc, y=None, residual=None, stream=None):
    """y_acc[send_tok[i]] += back_rows[i] (the partial sums the ranks returned), then y = bf16(y_acc + residual)
    when ``y`` is given."""
    for n, t in (("back_rows", back_rows), ("send_tok", send_tok), ("y_acc", y_acc), ("y", y),
                 ("residual", residual)):
        _dev(t, n)
    T, d = y_acc.shape
    n = back_rows.shape[0]
    _shape(back_rows, "back_rows", (n, d), (torch.float32,))
    _shape(y_acc, "y_acc", (T, d), (torch.float32,))
    if send_tok.shape[0] < n or send_tok.dtype != torch.int32:
        raise ValueError(f"send_tok: {tuple(send_tok.shape)} {send_tok.dtype}, expected at least ({n},) int32")
    _shape(y, "y", (T, d), (torch.bfloat16,))
    _shape(residual, "residual", (T, d), (torch.bfloat16,))
    _check(lib().moe_ep_combine(T, d, n, _p(back_rows), _p(send_tok), _p(y_acc), _p(y), _p(residual),
                                _stream(stream)), "moe_ep_combine")


def selftest_wait_timeout(limit_ns: int = 1_000_000, stream=None):
    """Launches a kernel whose bounded wait runs out after limit_ns; the device error word then holds
    MOE_DEVERR_TIMEOUT."""
    _check(lib().moe_selftest_wait_timeout(int(limit_ns), _stream(stream)), "moe_selftest_wait_timeout")


def launch_count() -> int:
    """Kernels the library has launched in this process (all devices and streams)."""
    return int(lib().moe_launch_count())


def moe_update_bias(cfg: MoeConfig, counts, bias, gamma: float = 1e-3, stream=None):
    """Bias controller: bias[e] -= gamma where counts[e] is above the mean count, else += gamma (in place)."""
    for n, t in (("counts", counts), ("bias", bias)):
        _dev(t, n)
    _check(lib().moe_update_bias(ctypes.byref(cfg), _p(counts), _p(bias), float(gamma), _stream(stream)),
           "moe_update_bias")


RMS_EPS = 1e-6


def block_workspace_size(cfg: MoeConfig, T: int) -> int:
    return int(lib().moe_block_workspace_size(ctypes.byref(cfg), int(T)))


def moe_rmsnorm(h, g, out, q=None, sx=None, eps: float = RMS_EPS, stream=None):
    """out = bf16(bf16(h * r) * g), r = 1/sqrt(mean(h^2) + eps) per row of bf16 h [T, d]; with q (uint8 [T, d])
    and sx (fp32 [T, d/128]) also the e4m3 activation codes and scales of out."""
    for n, t in (("h", h), ("g", g), ("out", out), ("q", q), ("sx", sx)):
        _dev(t, n)
    T, d = h.shape
    _check(lib().moe_rmsnorm(_p(h), _p(g), float(eps), T, d, _p(out), _p(q), _p(sx), _stream(stream)),
           "moe_rmsnorm")


def moe_forward_block(cfg: MoeConfig, weights, norm_g, h, bias, y, eps: float = RMS_EPS, workspace=None,
                      stream=None, stage_events=None, routing_out=None):
    """y = bf16(h + MoE(RMSNorm(h))) for the bf16 residual stream h [T, d]; y may be h itself.  ``workspace``: at
    least ``block_workspace_size(cfg, T)`` bytes.  ``stage_events`` / ``routing_out`` as in ``moe_forward``."""
    for n, t in (("norm_g", norm_g), ("h", h), ("bias", bias), ("y", y), ("workspace", workspace)):
        _dev(t, n)
    mw = weights if isinstance(weights, MoeWeights) else make_weights(weights)
    T = h.shape[0]
    _shape(h, "h", (T, cfg.d), (torch.bfloat16,))
    _shape(norm_g, "norm_g", (cfg.d,), (torch.bfloat16,))
    _shape(bias, "bias", (cfg.n_experts,), (torch.float32,))
    _shape(y, "y", (T, cfg.d), (torch.bfloat16,))
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    ev, ro = _events(stage_events), _routing(routing_out)
    _check(lib().moe_forward_block(ctypes.byref(cfg), ctypes.byref(mw), _p(norm_g), float(eps), _p(h), _p(bias), T,
                                   _p(y), _p(workspace), ws_bytes, _stream(stream),
                                   ctypes.byref(ev) if ev is not None else None,
                                   ctypes.byref(ro) if ro is not None else None), "moe_forward_block")


def dense_workspace_size(d: int, hidden: int, act_dtype: int, weight_dtype: int, T: int) -> int:
    return int(lib().moe_dense_workspace_size(int(d), int(hidden), int(act_dtype), int(weight_dtype), int(T)))


def moe_dense_ffn(w_gate, w_up, w_down, x, y, s_gate=None, s_up=None, s_down=None, accumulate: bool = False,
                  workspace=None, stream=None, stage_events=None):
    """Dense SwiGLU FFN: y (+)= W_down(SiLU(W_gate x) * (W_up x)).  Weights bf16, or uint8 e4m3 codes with fp32
    128x128 block scales s_*; x [T, d] bf16 (or fp32 for bf16 weights); y fp32 or bf16."""
    for n, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down), ("x", x), ("y", y),
                 ("s_gate", s_gate), ("s_up", s_up), ("s_down", s_down), ("workspace", workspace)):
        _dev(t, n)
    hidden, d = w_gate.shape
    wdt = MOE_E4M3 if w_gate.dtype == torch.uint8 else MOE_BF16
    T = x.shape[0]
    wt = (torch.uint8,) if wdt == MOE_E4M3 else (torch.bfloat16,)
    _shape(w_up, "w_up", (hidden, d), wt)
    _shape(w_down, "w_down", (d, hidden), wt)
    _shape(x, "x", (T, d), (torch.bfloat16,) if wdt == MOE_E4M3 else (torch.bfloat16, torch.float32))
    _shape(y, "y", (T, d), _OUT)
    if wdt == MOE_E4M3:
        for n, t, shp in (("s_gate", s_gate, (hidden // 128, d // 128)), ("s_up", s_up, (hidden // 128, d // 128)),
                          ("s_down", s_down, (d // 128, hidden // 128))):
            if t is None:
                raise ValueError(f"{n}: e4m3 weights need their block scales")
            _shape(t, n, shp, (torch.float32,))
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    ev = _events(stage_events)
    _check(lib().moe_dense_ffn(d, hidden, _dtype_code(x), wdt, _p(w_gate), _p(w_up), _p(w_down), _p(s_gate),
                               _p(s_up), _p(s_down), _p(x), T, _p(y), _dtype_code(y), 1 if accumulate else 0,
                               _p(workspace), ws_bytes, _stream(stream),
                               ctypes.byref(ev) if ev is not None else None), "moe_dense_ffn")


def moe_quantize_act(x, q, sx, stream=None):
    """Per-token, per-128-channel e4m3 quantisation of bf16 x [T, d] into codes q (uint8 [T, d]) and scales sx
    (fp32 [T, d/128])."""
    for n, t in (("x", x), ("q", q), ("sx", sx)):
        _dev(t, n)
    T, d = x.shape
    _check(lib().moe_quantize_act(_p(x), T, d, _p(q), _p(sx), _stream(stream)), "moe_quantize_act")


def device_error(stream=None) -> int:
    """Reads and clears the device error word (synchronises the stream); returns the MOE_DEVERR_* bits."""
    flags = ctypes.c_uint(0)
    st = lib().moe_device_error(ctypes.byref(flags), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        raise MoeError(st, "moe_device_error")
    return int(flags.value)
