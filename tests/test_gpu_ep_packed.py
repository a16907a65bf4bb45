"""The fixed-capacity expert-parallel exchange (moe_ep_dispatch_packed, moe_ep_unpack,
ep.EpLayer) on one GPU.

Emulated ranks: the ranks' dispatches run one after another on this GPU and the test
does the all-to-all (block q of rank p's send buffer becomes block p of rank q's
receive buffer, as an equal-split all-to-all moves it).  The packed rows are integer
and byte work, compared bit for bit with the dispatch's definition (rank q's tokens
in slots [q*cap, q*cap + count), then padding with token -1 and ids -1).  The layer
output is compared with moe_forward's within 1e-3 x RMS (the combine adds a token's
partial sums in another order, and the shared expert runs on the dense-FFN tiles)
and, on sampled tokens, with the oracle.

EpLayer: through torch.distributed with a one-rank NCCL group, eagerly and as a
captured CUDA graph replayed on new inputs (no host round trip in the forward)."""
import datetime
import os

import numpy as np
import pytest
import torch

import fine_grained_moe_gemm_b200 as moe
from moe_testlib import assert_close_rms, cfg_of
from test_ep_cpu import dispatch_def
from test_gpu_ep import _free_port, block_weights, close_to, inputs, shared_weights
from test_gpu_forward import oracle_y, run_forward
from workloads import make_x

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _row_fields(cfg, packed):
    """(x bf16 [n, d], ids int32 [n, k], w fp32 [n, k]) views of packed rows."""
    d, k = cfg.d, cfg.top_k
    x = packed[:, :2 * d].contiguous().view(torch.bfloat16)
    ids = packed[:, 2 * d:2 * d + 4 * k].contiguous().view(torch.int32)
    w = packed[:, 2 * d + 4 * k:2 * d + 8 * k].contiguous().view(torch.float32)
    return x, ids, w


def emulated_packed(wl, W, x, R, cap):
    cfg = cfg_of(wl)
    T, d, k, E = x.shape[0], wl.d, wl.top_k, wl.n_experts
    rb = moe.ep_packed_row_bytes(cfg)
    assert rb == (2 * d + 8 * k + 15) // 16 * 16
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.moe_route(cfg, x, W["w_router"], logits, W["bias"], idx, w)
    bounds = np.linspace(0, T, R + 1).astype(int)
    ranks = []
    for q in range(R):
        a, b = bounds[q], bounds[q + 1]
        o = {"xq": x[a:b].contiguous(), "iq": idx[a:b].contiguous(), "wq": w[a:b].contiguous(),
             "counts": torch.full((R,), -3, dtype=torch.int32, device=DEV),
             "tok": torch.full((R * cap,), -9, dtype=torch.int32, device=DEV),
             "send": torch.full((R * cap, rb), 0xAB, dtype=torch.uint8, device=DEV)}
        moe.moe_ep_dispatch_packed(cfg, R, cap, o["iq"], o["wq"], o["xq"], o["counts"], o["tok"], o["send"])
        ranks.append(o)
    torch.cuda.synchronize()
    # the dispatch against its definition, bit for bit
    for o in ranks:
        iq = o["iq"].cpu().numpy()
        counts, tok = dispatch_def(iq, E, R)
        assert np.array_equal(o["counts"].cpu().numpy(), counts)
        px, pid, pw = _row_fields(cfg, o["send"])
        base = 0
        for p in range(R):
            n = int(counts[p])
            t = torch.from_numpy(tok[base:base + n]).long().to(DEV)
            sl = slice(p * cap, p * cap + n)
            assert np.array_equal(o["tok"][sl].cpu().numpy(), tok[base:base + n])
            xr = o["xq"][t].to(torch.bfloat16) if o["xq"].dtype == torch.float32 else o["xq"][t]
            assert torch.equal(px[sl], xr)
            assert torch.equal(pid[sl], o["iq"][t])
            assert torch.equal(pw[sl].view(torch.int32), o["wq"][t].view(torch.int32))
            pad = slice(p * cap + n, (p + 1) * cap)
            assert bool((o["tok"][pad] == -1).all()) and bool((pid[pad] == -1).all())
            base += n
    # rows out: block p of rank q -> block q of rank p
    ys, yb = [], []
    outs = []
    for p in range(R):
        recv = torch.cat([ranks[q]["send"][p * cap:(p + 1) * cap] for q in range(R)])
        rx = torch.empty((R * cap, d), dtype=torch.bfloat16, device=DEV)
        ri = torch.empty((R * cap, k), dtype=torch.int32, device=DEV)
        rw = torch.empty((R * cap, k), dtype=torch.float32, device=DEV)
        moe.moe_ep_unpack(cfg, recv, rx, ri, rw)
        px, pid, pw = _row_fields(cfg, recv)
        live = (pid >= 0).any(1)
        assert torch.equal(ri, pid) and torch.equal(rx[live], px[live])
        assert torch.equal(rw[live].view(torch.int32), pw[live].view(torch.int32)) and bool((rw[~live] == 0).all())
        lo, nl = p * (E // R), E // R
        ry = torch.full((R * cap, d), 5.0, dtype=torch.float32, device=DEV)
        ws = torch.empty(moe.experts_routed_workspace_size(cfg, nl, R * cap), dtype=torch.uint8, device=DEV)
        moe.moe_experts_routed(cfg, block_weights(wl, W, lo, nl), lo, nl, rx, ri, rw, ry, workspace=ws)
        assert bool((ry[~live] == 0).all())
        outs.append(ry)
    sh = shared_weights(wl, W)
    for q in range(R):
        back = torch.cat([outs[p][q * cap:(q + 1) * cap] for p in range(R)])
        xq = ranks[q]["xq"]
        Tq = xq.shape[0]
        y_acc = torch.empty((Tq, d), dtype=torch.float32, device=DEV)
        wdt = moe.MOE_E4M3 if wl.fp8 else moe.MOE_BF16
        dws = torch.empty(moe.dense_workspace_size(d, wl.shared_hidden, cfg.act_dtype, wdt, Tq), dtype=torch.uint8,
                          device=DEV)
        moe.moe_dense_ffn(sh["w_gate"], sh["w_up"], sh["w_down"], xq, y_acc, sh.get("s_gate"), sh.get("s_up"),
                          sh.get("s_down"), workspace=dws)
        y_b = torch.empty((Tq, d), dtype=torch.bfloat16, device=DEV)
        moe.moe_ep_combine(back, ranks[q]["tok"], y_acc, y_b)
        ys.append(y_acc)
        yb.append(y_b)
    torch.cuda.synchronize()
    assert moe.device_error() == 0          # padding slots are skipped silently
    return torch.cat(ys), torch.cat(yb)


@pytest.mark.parametrize("name,R,cap_extra", [("decode", 8, 0), ("decode", 2, 5), ("tiny", 4, 3), ("tiny_fp8", 4, 0)])
def test_packed_exchange_matches_the_layer(name, R, cap_extra):
    wl, W = inputs(name)
    x = W["x"] if name != "tiny_fp8" else make_x(wl, "cpu").to(DEV)
    cap = (x.shape[0] + R - 1) // R + cap_extra
    y, yb = emulated_packed(wl, W, x, R, cap)
    ref = run_forward(wl, W, x, torch.float32)
    close_to(y, ref)
    assert torch.equal(yb, y.to(torch.bfloat16))
    if name == "decode" and R == 8:
        toks = np.array([0, 9, 31, 64, 90, 127], np.int32)
        assert_close_rms(y.cpu().numpy()[toks], oracle_y(wl, W, x, toks), 1e-2)


def test_ep_layer_one_rank_nccl_eager_and_graph():
    import torch.distributed as dist
    from fine_grained_moe_gemm_b200 import ep

    wl, W = inputs("decode")
    cfg = cfg_of(wl)
    T = wl.T
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device(DEV, torch.cuda.current_device()))
    graph = None
    try:
        layer = ep.EpLayer(cfg, T, DEV)
        local, shared = block_weights(wl, W, 0, wl.n_experts), shared_weights(wl, W)
        x_in = W["x"].clone()
        y = torch.empty((T, wl.d), dtype=torch.bfloat16, device=DEV)
        layer.forward(W["w_router"], local, shared, W["bias"], x_in, y)
        torch.cuda.synchronize()
        assert moe.device_error() == 0
        y_eager = y.clone()
        # the same forward captured once and replayed on a new batch in the same input buffer
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            layer.forward(W["w_router"], local, shared, W["bias"], x_in, y)
        x2 = make_x(wl, DEV, seed=9)
        x_in.copy_(x2)
        graph.replay()
        torch.cuda.synchronize()
        assert moe.device_error() == 0
        y_graph = y.clone()
    finally:
        del graph
        dist.destroy_process_group()
    for got, xx in ((y_eager, W["x"]), (y_graph, x2)):
        ref = run_forward(wl, W, xx, torch.float32)
        rms = float(ref.double().pow(2).mean().sqrt())
        assert bool(((got.double() - ref.double()).abs() <= 2.0 ** -8 * ref.double().abs() + 1e-3 * rms).all())
