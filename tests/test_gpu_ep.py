"""Expert parallelism on one GPU: the ranks' dispatch, block experts and combine run
one after another on this GPU with the all-to-all done by the test (copies of the
rows between the ranks' buffers), and the whole expert-parallel layer through
torch.distributed with a one-rank NCCL group.

Bars: the dispatch tables and rows are integer and byte work, compared bit for bit
with the dispatch's definition computed on the host.  The layer output is compared
with moe_forward's on the same tokens within 1e-3 x RMS: the routed experts see the
same rows in the same tiles, but the combine adds a token's partial sums in another
order and the shared expert runs on the dense-FFN kernels (another tile shape, a
split-K down GEMM), where an h value may round to the neighbouring bf16 now and
then; a lost or doubled expert contribution is O(RMS).  On sampled tokens it is
also compared with the oracle (max |err| <= 1e-2 x RMS(y_ref))."""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch

import fine_grained_moe_gemm_b200 as moe
from moe_testlib import assert_close_rms, cfg_of, weights_for_forward
from test_ep_cpu import dispatch_def
from test_gpu_forward import oracle_y, run_forward
from workloads import WORKLOADS, make_inputs, make_x

pytestmark = pytest.mark.gpu

DEV = "cuda"

_cache = {}


def inputs(name):
    if name not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        if name == "tiny_fp8":
            wl = dataclasses.replace(WORKLOADS["tiny"], name="tiny_fp8", x_f32=False, fp8=True)
            W = {k: v.to(DEV) for k, v in make_inputs(wl, "cpu").items()}
        else:
            wl = WORKLOADS[name]
            W = {k: v.to(DEV) for k, v in make_inputs(wl, "cpu" if wl.d <= 1024 else DEV).items()}
        _cache[name] = (wl, W)
    return _cache[name]


def close_to(a, b, rel=1e-3):
    """max |a - b| <= rel x RMS(b)."""
    a64, b64 = a.double(), b.double()
    rms = float(b64.pow(2).mean().sqrt())
    err = float((a64 - b64).abs().max())
    assert err <= rel * rms, f"max |err| {err:.3g} > {rel} x RMS {rms:.3g}"


def block_weights(wl, W, lo, n):
    keys = ["w_gate", "w_up", "w_down"] + (["s_gate", "s_up", "s_down"] if wl.fp8 else [])
    return {k: W[k][lo:lo + n].contiguous() for k in keys}


def shared_weights(wl, W):
    m = {"w_gate": "ws_gate", "w_up": "ws_up", "w_down": "ws_down"}
    if wl.fp8:
        m.update(s_gate="ss_gate", s_up="ss_up", s_down="ss_down")
    return {k: W[v] for k, v in m.items()}


def emulated_ep(wl, W, x, R):
    """The expert-parallel layer with R ranks emulated on this GPU (ranks own consecutive token slices).
    Returns (y fp32 [T, d], y bf16, per-rank dispatch outputs)."""
    cfg = cfg_of(wl)
    T, d, k, E = x.shape[0], wl.d, wl.top_k, wl.n_experts
    # the routing of the whole batch, sliced per rank (the router's split-K depends on T, so the ranks
    # take the rows of one routing call for a comparison with moe_forward on the whole batch)
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.moe_route(cfg, x, W["w_router"], logits, W["bias"], idx, w)
    bounds = np.linspace(0, T, R + 1).astype(int)
    disp = []
    for q in range(R):
        a, b = bounds[q], bounds[q + 1]
        xq, iq, wq = x[a:b].contiguous(), idx[a:b].contiguous(), w[a:b].contiguous()
        rows = max(moe.ep_max_send_rows(cfg, b - a, R), 1)
        o = {"counts": torch.empty(R, dtype=torch.int32, device=DEV),
             "offsets": torch.empty(R + 1, dtype=torch.int32, device=DEV),
             "tok": torch.full((rows,), -7, dtype=torch.int32, device=DEV),
             "x": torch.empty((rows, d), dtype=torch.bfloat16, device=DEV),
             "idx": torch.empty((rows, k), dtype=torch.int32, device=DEV),
             "w": torch.empty((rows, k), dtype=torch.float32, device=DEV)}
        moe.moe_ep_dispatch(cfg, R, iq, wq, xq, o["counts"], o["offsets"], o["tok"], o["x"], o["idx"], o["w"])
        o.update(xq=xq, iq=iq, wq=wq)
        disp.append(o)
    torch.cuda.synchronize()
    offs = [o["offsets"].cpu().tolist() for o in disp]
    # all-to-all (by the test): rank p receives, from q = 0 .. R-1, q's rows for p
    outs = []
    lo_n = [(p * (E // R), E // R) for p in range(R)]
    for p in range(R):
        recv = {key: torch.cat([disp[q][key][offs[q][p]:offs[q][p + 1]] for q in range(R)])
                for key in ("x", "idx", "w")}
        n = recv["x"].shape[0]
        y_rows = torch.empty((n, d), dtype=torch.float32, device=DEV)
        if n:
            lo, nl = lo_n[p]
            ws = torch.empty(moe.experts_routed_workspace_size(cfg, nl, n), dtype=torch.uint8, device=DEV)
            moe.moe_experts_routed(cfg, block_weights(wl, W, lo, nl), lo, nl, recv["x"], recv["idx"], recv["w"],
                                   y_rows, workspace=ws)
        outs.append((y_rows, [offs[q][p + 1] - offs[q][p] for q in range(R)]))
    # back: rank q receives from p the results of its rows for p, in p order = q's send order
    ys, yb = [], []
    sh = shared_weights(wl, W)
    for q in range(R):
        parts = []
        for p in range(R):
            y_rows, sizes = outs[p]
            start = sum(sizes[:q])
            parts.append(y_rows[start:start + sizes[q]])
        back = torch.cat(parts)
        xq = disp[q]["xq"]
        Tq = xq.shape[0]
        y_acc = torch.empty((Tq, d), dtype=torch.float32, device=DEV)
        wdt = moe.MOE_E4M3 if wl.fp8 else moe.MOE_BF16
        dws = torch.empty(moe.dense_workspace_size(d, wl.shared_hidden, cfg.act_dtype, wdt, Tq), dtype=torch.uint8,
                          device=DEV)
        moe.moe_dense_ffn(sh["w_gate"], sh["w_up"], sh["w_down"], xq, y_acc, sh.get("s_gate"), sh.get("s_up"),
                          sh.get("s_down"), workspace=dws)
        y_b = torch.empty((Tq, d), dtype=torch.bfloat16, device=DEV)
        moe.moe_ep_combine(back, disp[q]["tok"], y_acc, y_b)
        ys.append(y_acc)
        yb.append(y_b)
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    return torch.cat(ys), torch.cat(yb), disp


def check_dispatch(wl, disp, R):
    """Every rank's dispatch against its definition, bit for bit."""
    for o in disp:
        iq = o["iq"].cpu().numpy()
        counts, tok = dispatch_def(iq, wl.n_experts, R)
        n = int(counts.sum())
        assert np.array_equal(o["counts"].cpu().numpy(), counts)
        assert np.array_equal(o["offsets"].cpu().numpy(), np.concatenate([[0], np.cumsum(counts)]).astype(np.int32))
        assert np.array_equal(o["tok"][:n].cpu().numpy(), tok)
        t = torch.from_numpy(tok).long().to(DEV)
        xr = o["xq"][t].to(torch.bfloat16) if o["xq"].dtype == torch.float32 else o["xq"][t]
        assert torch.equal(o["x"][:n], xr)
        assert torch.equal(o["idx"][:n], o["iq"][t])
        assert torch.equal(o["w"][:n].view(torch.int32), o["wq"][t].view(torch.int32))


@pytest.mark.parametrize("name,R", [("decode", 8), ("decode", 2), ("tiny", 4), ("tiny_fp8", 4)])
def test_emulated_ranks_match_the_layer(name, R):
    wl, W = inputs(name)
    x = W["x"] if name != "tiny_fp8" else make_x(wl, "cpu").to(DEV)
    y, yb, disp = emulated_ep(wl, W, x, R)
    check_dispatch(wl, disp, R)
    ref = run_forward(wl, W, x, torch.float32)
    close_to(y, ref)
    # the bf16 output is y rounded once
    assert torch.equal(yb, y.to(torch.bfloat16))


def test_emulated_ranks_against_the_oracle():
    wl, W = inputs("decode")
    x = W["x"]
    y, _, _ = emulated_ep(wl, W, x, 8)
    toks = np.array([0, 5, 17, 64, 100, 127], np.int32)
    assert_close_rms(y.cpu().numpy()[toks], oracle_y(wl, W, x, toks), 1e-2)


def test_block_with_no_rows_and_foreign_slots_only():
    """Rows whose slots all belong to other blocks give zero rows and no device error."""
    wl, W = inputs("tiny")
    cfg = cfg_of(wl)
    n, k, d = 5, wl.top_k, wl.d
    x_rows = make_x(wl, "cpu", T=n).to(torch.bfloat16).to(DEV)
    idx = torch.tensor([[12, 13, 14, 15]] * n, dtype=torch.int32, device=DEV)   # block 3 of 4
    w = torch.full((n, k), 0.25, dtype=torch.float32, device=DEV)
    y = torch.full((n, d), 9.0, dtype=torch.float32, device=DEV)
    ws = torch.empty(moe.experts_routed_workspace_size(cfg, 4, n), dtype=torch.uint8, device=DEV)
    moe.moe_experts_routed(cfg, block_weights(wl, W, 0, 4), 0, 4, x_rows, idx, w, y, workspace=ws)
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    assert bool((y == 0).all())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_forward_ep_one_rank_nccl():
    """The expert-parallel layer through torch.distributed (NCCL, one rank: every expert local)."""
    import datetime

    import torch.distributed as dist
    from fine_grained_moe_gemm_b200 import ep

    wl, W = inputs("decode")
    cfg = cfg_of(wl)
    x = W["x"]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device(DEV, torch.cuda.current_device()))
    try:
        y = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device=DEV)
        ep.moe_forward_ep(cfg, W["w_router"], block_weights(wl, W, 0, wl.n_experts), shared_weights(wl, W),
                          W["bias"], x, y)
        torch.cuda.synchronize()
        assert moe.device_error() == 0
    finally:
        dist.destroy_process_group()
    ref = run_forward(wl, W, x, torch.float32)
    # one bf16 rounding (half an ulp of |ref|, up to 2^-8 |ref|) away from a value close to ref
    rms = float(ref.double().pow(2).mean().sqrt())
    assert bool(((y.double() - ref.double()).abs() <= 2.0 ** -8 * ref.double().abs() + 1e-3 * rms).all())


def test_combine_flags_a_token_outside_the_batch():
    """A returned row whose token is not in the batch is skipped and flagged (MOE_DEVERR_BAD_ROWS) by the
    kernel's bounds check; the other rows land."""
    T, d = 4, 256
    y_acc = torch.zeros((T, d), dtype=torch.float32, device=DEV)
    back = torch.arange(3 * d, dtype=torch.float32, device=DEV).reshape(3, d)
    tok = torch.tensor([0, 7, 2], dtype=torch.int32, device=DEV)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_ep_combine(back, tok, y_acc, y)
    torch.cuda.synchronize()
    assert moe.device_error() == moe.MOE_DEVERR_BAD_ROWS
    expect = torch.zeros((T, d), dtype=torch.float32, device=DEV)
    expect[0], expect[2] = back[0], back[2]
    assert torch.equal(y_acc, expect)
    assert torch.equal(y, expect.to(torch.bfloat16))


def test_dispatch_of_no_tokens_writes_zero_counts():
    wl, W = inputs("decode")
    cfg = cfg_of(wl)
    R = 8
    counts = torch.full((R,), -1, dtype=torch.int32, device=DEV)
    offsets = torch.full((R + 1,), -1, dtype=torch.int32, device=DEV)
    e = lambda *shape, dt=torch.int32: torch.empty(shape, dtype=dt, device=DEV)
    moe.moe_ep_dispatch(cfg, R, e(0, wl.top_k), e(0, wl.top_k, dt=torch.float32), e(0, wl.d, dt=torch.bfloat16),
                        counts, offsets, e(1), e(1, wl.d, dt=torch.bfloat16), e(1, wl.top_k),
                        e(1, wl.top_k, dt=torch.float32))
    torch.cuda.synchronize()
    assert counts.tolist() == [0] * R and offsets.tolist() == [0] * (R + 1)
