"""Seeded synthetic workloads for the MoE layer (shapes, distributions, seeds).

This module only draws random inputs; it holds none of the layer's arithmetic.
Both the CUDA path (tests, bench) and the CPU oracle consume what it produces.

Workloads (DeepSeek-V3 MoE layer; "Teardown: DeepSeek-V3", section 6 and the
"At a glance" table; "DeepSeek-V3" llm-vis, "MoE router" / "Routed experts"):

=========  =====  =====  ===  =====  ======  ===  =====  =======================
name       T      d      E    G      groups  k    H=Hs   inputs
=========  =====  =====  ===  =====  ======  ===  =====  =======================
tiny       64     256    16   4x4    2       4    128    x fp32 N(0,1); bias U[-.1,.1]
decode     128    7168   256  8x32   4       8    2048   x bf16 N(0,1); bias U[-.1,.1]
prefill    4096   7168   256  8x32   4       8    2048   bias 0 (near-uniform load)
skewed     16384  7168   256  8x32   4       8    2048   bias +2.0 on 16 Zipf(1.2) hot experts
fp8        8192   7168   256  8x32   4       8    2048   e4m3 weights, 128x128 fp32 scales; bias 0
=========  =====  =====  ===  =====  ======  ===  =====  =======================

All weights are N(0, 0.02) drawn in fp32 and rounded once to bf16 (the router
weight included).  The FP8 workload quantises those bf16 expert weights to
e4m3 with one fp32 scale per 128x128 block (scale = amax / 448), the form in
which FP8 expert weights are shipped; the router stays bf16.

Every tensor has its own torch.Generator seeded from (seed, workload id,
tensor id).  Values are reproducible per device type (the CPU and CUDA
generators are different algorithms); a test that needs the same values on
both sides generates once and copies.
"""
from __future__ import annotations

import dataclasses
import hashlib

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    wid: int
    T: int
    d: int
    n_experts: int
    n_groups: int
    topk_groups: int
    top_k: int
    hidden: int
    shared_hidden: int
    routed_scale: float = 2.5
    x_f32: bool = False          # activations fp32 (tiny) instead of bf16
    fp8: bool = False            # expert weights e4m3 + block scales, activations quantised
    bias: str = "uniform"        # "uniform" U[-0.1, 0.1] | "zero" | "hot"
    n_hot: int = 16
    hot_bias: float = 2.0
    zipf_s: float = 1.2

    def with_T(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=int(T))

    # parameter / byte accounting ("Teardown: DeepSeek-V3", section 6)
    @property
    def params_per_expert(self) -> int:
        return 3 * self.d * self.hidden

    @property
    def params_shared(self) -> int:
        return 3 * self.d * self.shared_hidden

    @property
    def flops_per_token(self) -> int:
        """2 x (router MACs + (k routed + shared) expert MACs)."""
        return 2 * (self.n_experts * self.d + self.top_k * self.params_per_expert + self.params_shared)


WORKLOADS = {
    "tiny": Workload("tiny", 0, 64, 256, 16, 4, 2, 4, 128, 128, x_f32=True, bias="uniform"),
    "decode": Workload("decode", 1, 128, 7168, 256, 8, 4, 8, 2048, 2048, bias="uniform"),
    "prefill": Workload("prefill", 2, 4096, 7168, 256, 8, 4, 8, 2048, 2048, bias="zero"),
    "skewed": Workload("skewed", 3, 16384, 7168, 256, 8, 4, 8, 2048, 2048, bias="hot"),
    "fp8": Workload("fp8", 4, 8192, 7168, 256, 8, 4, 8, 2048, 2048, fp8=True, bias="zero"),
    # Small cases of the same kernels for hardware-counter captures: full width
    # (d = 7168, H = 2048) but 32 experts (2.8 GB of bf16 weights, more than the
    # L2), with the decode, prefill and FP8 rows per expert (4, 128 and 256).
    "profile_decode": Workload("profile_decode", 5, 16, 7168, 32, 8, 4, 8, 2048, 2048, bias="uniform"),
    "profile_prefill": Workload("profile_prefill", 6, 512, 7168, 32, 8, 4, 8, 2048, 2048, bias="zero"),
    "profile_fp8": Workload("profile_fp8", 7, 1024, 7168, 32, 8, 4, 8, 2048, 2048, fp8=True, bias="zero"),
}

# tensor ids of the per-tensor generators
_TID = {"x": 1, "w_router": 2, "bias": 3, "w_gate": 4, "w_up": 5, "w_down": 6,
        "ws_gate": 7, "ws_up": 8, "ws_down": 9, "hot": 10, "residual": 11, "norm_g": 12}

WEIGHT_STD = 0.02
BIAS_RANGE = 0.1


def _seed(seed: int, wid: int, tensor: str, sub: int = 0) -> int:
    h = hashlib.sha256(f"{seed}/{wid}/{_TID[tensor]}/{sub}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_bf16(shape, std, device, seed, chunk_rows=None):
    """N(0, std) drawn in fp32, rounded once to bf16."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    g = _gen(device, seed)
    flat = out.view(shape[0], -1)
    step = chunk_rows or shape[0]
    for r0 in range(0, shape[0], step):
        r1 = min(shape[0], r0 + step)
        tmp = torch.randn((r1 - r0, flat.shape[1]), generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        flat[r0:r1].copy_(tmp)
    return out


def hot_experts(wl: Workload, seed: int = 0) -> np.ndarray:
    """16 distinct hot experts: ranks r in [1, E] drawn with P(r) ~ r^-s, duplicates redrawn; id = r - 1."""
    rng = np.random.default_rng(_seed(seed, wl.wid, "hot"))
    r = np.arange(1, wl.n_experts + 1, dtype=np.float64)
    p = r ** (-wl.zipf_s)
    p /= p.sum()
    hot: list[int] = []
    while len(hot) < wl.n_hot:
        e = int(rng.choice(wl.n_experts, p=p))
        if e not in hot:
            hot.append(e)
    return np.array(sorted(hot), dtype=np.int64)


def make_bias(wl: Workload, device="cpu", seed: int = 0) -> torch.Tensor:
    if wl.bias == "uniform":
        g = _gen(device, _seed(seed, wl.wid, "bias"))
        b = torch.rand(wl.n_experts, generator=g, device=device, dtype=torch.float32)
        return b.mul_(2 * BIAS_RANGE).sub_(BIAS_RANGE)
    b = torch.zeros(wl.n_experts, dtype=torch.float32, device=device)
    if wl.bias == "hot":
        b[torch.as_tensor(hot_experts(wl, seed), device=device)] = wl.hot_bias
    return b


def make_x(wl: Workload, device="cpu", seed: int = 0, T: int | None = None) -> torch.Tensor:
    T = wl.T if T is None else T
    g = _gen(device, _seed(seed, wl.wid, "x", T))
    x = torch.randn((T, wl.d), generator=g, device=device, dtype=torch.float32)
    return x if wl.x_f32 else x.to(torch.bfloat16)


def make_residual(wl: Workload, device="cpu", seed: int = 0, T: int | None = None,
                  dtype=torch.bfloat16) -> torch.Tensor:
    T = wl.T if T is None else T
    g = _gen(device, _seed(seed, wl.wid, "residual", T))
    return torch.randn((T, wl.d), generator=g, device=device, dtype=torch.float32).to(dtype)


def make_norm_gain(wl: Workload, device="cpu", seed: int = 0) -> torch.Tensor:
    """Per-feature gain of the pre-norm, bf16 U[0.5, 1.5] (a trained gain; the pages
    initialise it to ones)."""
    g = _gen(device, _seed(seed, wl.wid, "norm_g"))
    return (torch.rand(wl.d, generator=g, device=device, dtype=torch.float32) + 0.5).to(torch.bfloat16)


def make_stream(wl: Workload, device="cpu", seed: int = 0, T: int | None = None, scale: float = 4.0) -> torch.Tensor:
    """Residual stream h entering the MoE sublayer: bf16 N(0, scale^2) (larger than the
    normalised activations, as the stream grows with depth)."""
    return (make_residual(wl, device, seed, T, dtype=torch.float32) * scale).to(torch.bfloat16)


def _quantise_blocks_e4m3(w: torch.Tensor):
    """bf16 [R, C] -> (e4m3 codes as uint8 [R, C], fp32 scales [R/128, C/128]), scale = amax/448."""
    R, C = w.shape
    wf = w.float().view(R // 128, 128, C // 128, 128)
    amax = wf.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (wf / scale[:, None, :, None]).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.view(R, C).view(torch.uint8), scale.contiguous()


def make_weights(wl: Workload, device="cpu", seed: int = 0) -> dict:
    """All layer weights.  Routed: w_gate/w_up [E, H, d], w_down [E, d, H]
    (nn.Linear [out, in] per expert, stacked); shared: ws_gate/ws_up [Hs, d],
    ws_down [d, Hs]; router w_router [E, d]; all bf16.  For the FP8 workload
    the expert and shared weights are replaced by e4m3 codes (uint8) plus
    fp32 block scales s_* [E, rows/128, cols/128] and ss_* [rows/128, cols/128]."""
    E, d, H, Hs = wl.n_experts, wl.d, wl.hidden, wl.shared_hidden
    W = {"w_router": _normal_bf16((E, d), WEIGHT_STD, device, _seed(seed, wl.wid, "w_router"))}
    for name, shape in (("w_gate", (E, H, d)), ("w_up", (E, H, d)), ("w_down", (E, d, H))):
        W[name] = _normal_bf16(shape, WEIGHT_STD, device, _seed(seed, wl.wid, name), chunk_rows=1)
    for name, shape in (("ws_gate", (Hs, d)), ("ws_up", (Hs, d)), ("ws_down", (d, Hs))):
        W[name] = _normal_bf16(shape, WEIGHT_STD, device, _seed(seed, wl.wid, name))
    if wl.fp8:
        for name in ("w_gate", "w_up", "w_down"):
            src = W[name]
            q = torch.empty(src.shape, dtype=torch.uint8, device=device)
            s = torch.empty((src.shape[0], src.shape[1] // 128, src.shape[2] // 128),
                            dtype=torch.float32, device=device)
            for e in range(src.shape[0]):
                q[e], s[e] = _quantise_blocks_e4m3(src[e])
            W[name], W["s" + name[1:]] = q, s
            del src
        for name in ("ws_gate", "ws_up", "ws_down"):
            q, s = _quantise_blocks_e4m3(W[name])
            W[name], W["ss" + name[2:]] = q, s
    return W


DENSE_HIDDEN = 18432  # the dense FFN width of the model's first layers ("At a glance" table)
DENSE_WID = 20       # generator stream of the dense FFN weights


def make_dense_weights(d: int, hidden: int, fp8: bool, device="cpu", seed: int = 0) -> dict:
    """Dense SwiGLU FFN weights w_gate/w_up [hidden, d], w_down [d, hidden], bf16 N(0, 0.02);
    with fp8 the e4m3 codes (uint8) plus fp32 128x128 block scales s_gate/s_up/s_down."""
    W = {}
    for name, shape in (("w_gate", (hidden, d)), ("w_up", (hidden, d)), ("w_down", (d, hidden))):
        W[name] = _normal_bf16(shape, WEIGHT_STD, device, _seed(seed, DENSE_WID + d % 7, name, hidden))
    if fp8:
        for name in ("w_gate", "w_up", "w_down"):
            W[name], W["s" + name[1:]] = _quantise_blocks_e4m3(W[name])
    return W


def make_inputs(wl: Workload, device="cpu", seed: int = 0, T: int | None = None) -> dict:
    """Weights, x and bias of one workload on ``device``."""
    W = make_weights(wl, device, seed)
    W["x"] = make_x(wl, device, seed, T)
    W["bias"] = make_bias(wl, device, seed)
    return W
