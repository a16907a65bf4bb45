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
captured CUDA graph replayed on new inputs (no host round trip in the forward), with
the all-to-all exchange and with the peer-memory one (symmetric memory).  The
peer-memory dispatch and combine are also run with emulated ranks whose "peer"
buffers all live on this GPU."""
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


@pytest.mark.parametrize("name,R,cap_extra", [("decode", 8, 0), ("tiny", 4, 3), ("tiny_fp8", 4, 0)])
def test_peer_exchange_matches_the_packed_layout(name, R, cap_extra):
    """The peer-memory dispatch and combine with the ranks emulated on one GPU: every rank's
    "peer" buffers are local, so after all ranks' dispatch calls each receive buffer must hold
    what the packed dispatch plus an equal-split all-to-all delivers (bit for bit on the live
    rows, ids -1 on the padding), and the combine reading the ranks' result buffers must give
    what the combine of the returned rows gives."""
    wl, W = inputs(name)
    x = W["x"] if name != "tiny_fp8" else make_x(wl, "cpu").to(DEV)
    cfg = cfg_of(wl)
    T, d, k, E = x.shape[0], wl.d, wl.top_k, wl.n_experts
    cap = (T + R - 1) // R + cap_extra
    rb = moe.ep_packed_row_bytes(cfg)
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.moe_route(cfg, x, W["w_router"], logits, W["bias"], idx, w)
    bounds = np.linspace(0, T, R + 1).astype(int)
    recv = [torch.full((R * cap, rb), 0x5A, dtype=torch.uint8, device=DEV) for _ in range(R)]
    recv_ptrs = torch.tensor([b.data_ptr() for b in recv], dtype=torch.int64, device=DEV)
    ranks = []
    for p in range(R):
        a, b = bounds[p], bounds[p + 1]
        o = {"xq": x[a:b].contiguous(), "iq": idx[a:b].contiguous(), "wq": w[a:b].contiguous()}
        o["counts"] = torch.full((R,), -3, dtype=torch.int32, device=DEV)
        o["tok"] = torch.full((R * cap,), -9, dtype=torch.int32, device=DEV)
        moe.moe_ep_dispatch_peer(cfg, R, cap, p, o["iq"], o["wq"], o["xq"], o["counts"], o["tok"], recv_ptrs)
        # the packed form of the same dispatch, for comparison
        o["counts2"] = torch.empty((R,), dtype=torch.int32, device=DEV)
        o["tok2"] = torch.empty((R * cap,), dtype=torch.int32, device=DEV)
        o["send"] = torch.empty((R * cap, rb), dtype=torch.uint8, device=DEV)
        moe.moe_ep_dispatch_packed(cfg, R, cap, o["iq"], o["wq"], o["xq"], o["counts2"], o["tok2"], o["send"])
        ranks.append(o)
    torch.cuda.synchronize()
    for o in ranks:
        assert torch.equal(o["counts"], o["counts2"]) and torch.equal(o["tok"], o["tok2"])
    for q in range(R):
        want = torch.cat([ranks[p]["send"][q * cap:(q + 1) * cap] for p in range(R)])
        gx, gid, gw = _row_fields(cfg, recv[q])
        wx, wid, ww = _row_fields(cfg, want)
        live = (wid >= 0).any(1)
        assert torch.equal(gid, wid)
        assert torch.equal(gx[live], wx[live]) and torch.equal(gw[live].view(torch.int32), ww[live].view(torch.int32))
    # each rank's block of experts on its received rows, into its result buffer
    res = []
    for q in range(R):
        rx = torch.empty((R * cap, d), dtype=torch.bfloat16, device=DEV)
        ri = torch.empty((R * cap, k), dtype=torch.int32, device=DEV)
        rw = torch.empty((R * cap, k), dtype=torch.float32, device=DEV)
        moe.moe_ep_unpack(cfg, recv[q], rx, ri, rw)
        lo, nl = q * (E // R), E // R
        ry = torch.empty((R * cap, d), dtype=torch.float32, device=DEV)
        ws = torch.empty(moe.experts_routed_workspace_size(cfg, nl, R * cap), dtype=torch.uint8, device=DEV)
        moe.moe_experts_routed(cfg, block_weights(wl, W, lo, nl), lo, nl, rx, ri, rw, ry, workspace=ws)
        res.append(ry)
    res_ptrs = torch.tensor([t.data_ptr() for t in res], dtype=torch.int64, device=DEV)
    for p in range(R):
        o = ranks[p]
        Tp = o["xq"].shape[0]
        base = torch.randn((Tp, d), generator=torch.Generator().manual_seed(p), dtype=torch.float32).to(DEV)
        acc_peer, acc_ref = base.clone(), base.clone()
        y_peer = torch.empty((Tp, d), dtype=torch.bfloat16, device=DEV)
        moe.moe_ep_combine_peer(R, cap, p, res_ptrs, o["tok"], acc_peer, y_peer)
        back = torch.cat([res[q][p * cap:(p + 1) * cap] for q in range(R)])
        moe.moe_ep_combine(back, o["tok"], acc_ref)
        torch.cuda.synchronize()
        rms = float(acc_ref.double().pow(2).mean().sqrt())
        # the same sums, the atomics in another order: up to eight fp32 additions an element
        assert float((acc_peer - acc_ref).abs().max()) <= 1e-5 * rms
        assert torch.equal(y_peer, acc_peer.to(torch.bfloat16))
    assert moe.device_error() == 0


def _ep_layer_one_rank(exchange):
    import torch.distributed as dist
    from fine_grained_moe_gemm_b200 import ep

    wl, W = inputs("decode")
    cfg = cfg_of(wl)
    T = wl.T
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device(DEV, torch.cuda.current_device()))
    graph = layer = None
    try:
        layer = ep.EpLayer(cfg, T, DEV, exchange=exchange)
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
        del graph, layer
        dist.destroy_process_group()
    for got, xx in ((y_eager, W["x"]), (y_graph, x2)):
        ref = run_forward(wl, W, xx, torch.float32)
        rms = float(ref.double().pow(2).mean().sqrt())
        assert bool(((got.double() - ref.double()).abs() <= 2.0 ** -8 * ref.double().abs() + 1e-3 * rms).all())


def test_ep_layer_peer_one_rank_symmetric_memory_eager_and_graph():
    """EpLayer(exchange="peer"): symmetric-memory buffers on a one-rank NCCL group, the dispatch and
    combine through the peer pointer tables, one-element all-reduces as fences; eager and replayed."""
    _ep_layer_one_rank("peer")


def test_ep_layer_one_rank_nccl_eager_and_graph():
    _ep_layer_one_rank("all_to_all")
