"""Expert parallelism on the CPU: the exchange protocol of moe_forward_ep with gloo
ranks (world size 2 and 4), and the EP entry points' argument checks (no device).

The exchange test runs the protocol moe_forward_ep runs (counts all-to-all, then
rows, routing and results) on rows built by the dispatch's definition: for each
destination rank the tokens with an expert in its block, ascending, rank-major.
Each rank stands in for the expert kernels with a known map of the rows it
received (row * (rank + 1) + slot count of its block), so a row that comes back
from the wrong rank, in the wrong order or to the wrong token fails."""
import ctypes
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import fine_grained_moe_gemm_b200 as moe
from moe_testlib import cfg_of
from workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def dispatch_def(idx: np.ndarray, E: int, R: int):
    """The dispatch by its definition: per destination rank the tokens with at least one expert in its block,
    ascending; returns (counts, send_tok) with send_tok rank-major."""
    epr = E // R
    rows = [[t for t in range(idx.shape[0]) if any(0 <= e < E and e // epr == q for e in idx[t])] for q in range(R)]
    return np.array([len(r) for r in rows], np.int32), np.array([t for r in rows for t in r], np.int32)


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from fine_grained_moe_gemm_b200 import ep

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    E, k, T, d = 16, 4, 11 + 3 * rank, 8
    rng = np.random.default_rng(100 + rank)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    x = torch.from_numpy(rng.standard_normal((T, d)).astype(np.float32))
    counts, send_tok = dispatch_def(idx, E, world)
    send_x = x[torch.from_numpy(send_tok).long()]
    send_idx = torch.from_numpy(idx[send_tok])
    recv_counts = ep.exchange_counts(torch.from_numpy(counts), None)
    sc, rc = counts.tolist(), recv_counts.tolist()
    recv_x = ep.exchange(send_x, sc, rc)
    recv_idx = ep.exchange(send_idx, sc, rc)
    # stand-in for this rank's experts: a map the origin rank can predict
    epr = E // world
    mine = ((recv_idx >= rank * epr) & (recv_idx < (rank + 1) * epr)).sum(1, keepdim=True).float()
    recv_y = recv_x * (rank + 1) + mine
    back = ep.exchange(recv_y, rc, sc)
    # the rows came back in send order: row i is token send_tok[i] after rank q's map
    ok = True
    base = 0
    for q in range(world):
        for i in range(base, base + sc[q]):
            t = send_tok[i]
            n_q = int(((idx[t] >= q * epr) & (idx[t] < (q + 1) * epr)).sum())
            ok &= n_q > 0 and torch.equal(back[i], x[t] * (q + 1) + n_q)
        base += sc[q]
    total = torch.tensor([int(recv_counts.sum())])
    dist.all_reduce(total)
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out, f"r{rank}"), "w") as f:
        f.write(f"{int(ok)} {int(counts.sum())} {int(total)}")


@pytest.mark.parametrize("world", [2, 4])
def test_exchange_protocol_gloo(tmp_path, world):
    port = _free_port()
    mp.spawn(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    res = [open(tmp_path / f"r{r}").read().split() for r in range(world)]
    assert all(r[0] == "1" for r in res)
    # every row sent was received: the sum of the ranks' send rows = the rows all ranks received
    assert sum(int(r[1]) for r in res) == int(res[0][2])


def test_dispatch_definition_bounds():
    """A token reaches at most min(k, ranks) ranks, and with ranks = groups at most topk_groups of them
    when its experts come from topk_groups groups."""
    E, G, k = 256, 8, 8
    rng = np.random.default_rng(0)
    groups = [rng.choice(G, 4, replace=False) for _ in range(64)]
    idx = np.stack([np.concatenate([rng.choice(32, 2, replace=False) + 32 * g for g in gs]) for gs in groups])
    counts, tok = dispatch_def(idx.astype(np.int32), E, G)
    per_token = np.bincount(tok, minlength=64)
    assert per_token.max() <= 4 and per_token.min() >= 1 and counts.sum() == per_token.sum()


@pytest.fixture(scope="module")
def L():
    return moe.lib()


def test_ep_entry_arguments(L):
    cfg = cfg_of(WORKLOADS["decode"])
    P = ctypes.c_void_p
    assert L.moe_ep_max_send_rows(ctypes.byref(cfg), 128, 8) == 128 * 8
    assert L.moe_ep_max_send_rows(ctypes.byref(cfg), 128, 4) == 128 * 4
    assert L.moe_ep_max_send_rows(ctypes.byref(cfg), 128, 0) == 0
    disp = lambda R, counts: L.moe_ep_dispatch(ctypes.byref(cfg), R, P(16), P(16), P(16), 4, counts, P(16), P(16),
                                               P(16), P(16), P(16), None)
    assert disp(0, P(16)) == moe.MOE_ERR_INVALID_ARG          # no ranks
    assert disp(33, P(16)) == moe.MOE_ERR_INVALID_ARG         # more than 32
    assert disp(3, P(16)) == moe.MOE_ERR_INVALID_ARG          # 256 experts do not split over 3
    assert disp(8, None) == moe.MOE_ERR_INVALID_ARG           # no counts
    assert L.moe_ep_dispatch(ctypes.byref(cfg), 8, P(16), P(16), P(18), 4, P(16), P(16), P(16), P(16), P(16), P(16),
                             None) == moe.MOE_ERR_INVALID_ARG  # misaligned x
    # the block computation: block inside [0, E), enough workspace
    assert L.moe_experts_routed_workspace_size(ctypes.byref(cfg), 32, 1024) > 0
    assert L.moe_experts_routed_workspace_size(ctypes.byref(cfg), 0, 1024) == 0
    w = moe.MoeWeights(w_gate=16, w_up=16, w_down=16)
    er = lambda lo, n, ws: L.moe_experts_routed(ctypes.byref(cfg), ctypes.byref(w), lo, n, P(16), 4, P(16), P(16),
                                                P(16), P(1 << 20), ws, None)
    assert er(240, 32, 1 << 30) == moe.MOE_ERR_INVALID_ARG   # past the last expert
    assert er(-1, 32, 1 << 30) == moe.MOE_ERR_INVALID_ARG
    assert er(0, 32, 1024) == moe.MOE_ERR_WORKSPACE
    assert L.moe_experts_routed(ctypes.byref(cfg), ctypes.byref(w), 0, 32, P(16), 0, None, None, None, None, 0,
                                None) == moe.MOE_OK           # no rows: a no-op
    # the combine
    assert L.moe_ep_combine(4, 7164, 2, P(16), P(16), P(16), None, None, None) == moe.MOE_ERR_INVALID_ARG  # d % 8
    assert L.moe_ep_combine(4, 7168, 2, P(16), P(16), None, None, None, None) == moe.MOE_ERR_INVALID_ARG  # no y_acc
    assert L.moe_ep_combine(0, 7168, 0, None, None, None, None, None, None) == moe.MOE_OK
    assert L.moe_ep_combine(0, 7168, 3, None, None, None, None, None, None) == moe.MOE_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- moe_forward_ep's control flow
# The real moe_forward_ep runs on gloo ranks with the library calls replaced by CPU stand-ins of known
# arithmetic (routing: the top-k of the first E features; expert e: x -> (e + 1) x; shared: x -> x / 2),
# so each token's output has a closed form: bf16(x/2 + 2.5 * sum_j w_j (idx_j + 1) x).  A row sent to
# the wrong rank, a slot counted twice or dropped, or a result combined into the wrong token fails.

def _stand_ins(ep_mod, E_total):
    def route(cfg, x, w_router, logits, bias, idx, w, stream=None):
        s = x.float()[:, :cfg.n_experts]
        top = torch.topk(s, cfg.top_k, dim=1)
        idx.copy_(top.indices.to(torch.int32))
        p = torch.sigmoid(top.values)
        w.copy_(p / p.sum(1, keepdim=True))

    def dispatch(cfg, R, idx, w, x, counts, offsets, send_tok, send_x, send_idx, send_w, stream=None):
        c, tok = dispatch_def(idx.numpy(), cfg.n_experts, R)
        counts.copy_(torch.from_numpy(c))
        offsets.copy_(torch.from_numpy(np.concatenate([[0], np.cumsum(c)]).astype(np.int32)))
        n = len(tok)
        t = torch.from_numpy(tok).long()
        send_tok[:n] = t.to(torch.int32)
        send_x[:n] = x[t].to(send_x.dtype)
        send_idx[:n] = idx[t]
        send_w[:n] = w[t]

    def experts(cfg, local_weights, lo, n, x_rows, idx, w, y_rows, workspace=None, stream=None):
        mine = (idx >= lo) & (idx < lo + n)
        coef = (w * (idx.float() + 1) * mine.float()).sum(1, keepdim=True)
        y_rows.copy_(cfg.routed_scale * coef * x_rows.float())

    def dense(wg, wu, wd, x, y, *a, **k):
        y.copy_(0.5 * x.float())

    def combine(back, send_tok, y_acc, y=None, residual=None, stream=None):
        y_acc.index_add_(0, send_tok[: back.shape[0]].long(), back)
        if y is not None:
            y.copy_((y_acc + (residual.float() if residual is not None else 0)).to(torch.bfloat16))

    ep_mod.moe_route, ep_mod.moe_ep_dispatch, ep_mod.moe_experts_routed = route, dispatch, experts
    ep_mod.moe_dense_ffn, ep_mod.moe_ep_combine = dense, combine
    ep_mod.ep_max_send_rows = lambda cfg, T, R: T * min(cfg.top_k, R)
    ep_mod.experts_routed_workspace_size = lambda cfg, n, rows: 1
    ep_mod.dense_workspace_size = lambda *a: 1


def _forward_rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import fine_grained_moe_gemm_b200 as moe_pkg
    from fine_grained_moe_gemm_b200 import ep

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    E, k, d = 16, 4, 32
    cfg = moe_pkg.MoeConfig(d * 4, E, 4, 2, k, 128, 1, 128, 2.5)  # d field unused by the stand-ins
    cfg.d = d
    _stand_ins(ep, E)
    T = 9 + 5 * rank
    g = torch.Generator().manual_seed(7 + rank)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    y = torch.empty((T, d), dtype=torch.bfloat16)
    shared = {n: torch.empty((128, d), dtype=torch.bfloat16) for n in ("w_gate", "w_up", "w_down")}
    ep.moe_forward_ep(cfg, None, {}, shared, torch.zeros(E), x, y)
    # the closed form per token
    xf = x.double()
    top = torch.topk(xf.float()[:, :E], k, dim=1)
    p = torch.sigmoid(top.values)
    wts = (p / p.sum(1, keepdim=True)).double()
    coef = (wts * (top.indices.double() + 1)).sum(1, keepdim=True)
    ref = 0.5 * xf + 2.5 * coef * xf
    ulp = 2.0 ** -7 * ref.abs() + 1e-6
    ok = bool(((y.double() - ref).abs() <= ulp).all())
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out, f"f{rank}"), "w") as f:
        f.write(str(int(ok)))


@pytest.mark.parametrize("world", [2, 4])
def test_forward_ep_control_flow_gloo(tmp_path, world):
    port = _free_port()
    mp.spawn(_forward_rank, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    assert all(open(tmp_path / f"f{r}").read() == "1" for r in range(world))


# ----------------------------------------------------------------------------- fixed-capacity exchange

def test_packed_entry_arguments(L):
    cfg = cfg_of(WORKLOADS["decode"])
    P = ctypes.c_void_p
    assert L.moe_ep_packed_row_bytes(ctypes.byref(cfg)) == 2 * 7168 + 8 * 8          # 14400, a multiple of 16
    tiny = cfg_of(WORKLOADS["tiny"])
    assert L.moe_ep_packed_row_bytes(ctypes.byref(tiny)) == (2 * 256 + 8 * 4 + 15) // 16 * 16
    dp = lambda R, cap, T, counts=P(16), packed=P(16): L.moe_ep_dispatch_packed(
        ctypes.byref(cfg), R, cap, P(16), P(16), P(16), T, counts, P(16), packed, None)
    assert dp(8, 3, 4) == moe.MOE_ERR_INVALID_ARG              # capacity below T
    assert dp(0, 4, 4) == moe.MOE_ERR_INVALID_ARG              # no ranks
    assert dp(3, 4, 4) == moe.MOE_ERR_INVALID_ARG              # 256 experts do not split over 3
    assert dp(8, 4, 4, counts=None) == moe.MOE_ERR_INVALID_ARG
    assert dp(8, 4, 4, packed=P(24)) == moe.MOE_ERR_INVALID_ARG  # misaligned rows
    assert L.moe_ep_unpack(ctypes.byref(cfg), -1, P(16), P(16), P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ep_unpack(ctypes.byref(cfg), 4, None, P(16), P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ep_unpack(ctypes.byref(cfg), 0, None, None, None, None, None) == moe.MOE_OK


def test_peer_entry_arguments(L):
    """The peer-memory dispatch and combine reject bad arguments on the host, before any device work."""
    cfg = cfg_of(WORKLOADS["decode"])
    P = ctypes.c_void_p
    dp = lambda R, cap, me, T, bufs=P(64), counts=P(16): L.moe_ep_dispatch_peer(
        ctypes.byref(cfg), R, cap, me, P(16), P(16), P(16), T, counts, P(16), bufs, None)
    assert dp(8, 3, 0, 4) == moe.MOE_ERR_INVALID_ARG            # capacity below T
    assert dp(8, 4, 8, 4) == moe.MOE_ERR_INVALID_ARG            # rank outside [0, n_ranks)
    assert dp(8, 4, -1, 4) == moe.MOE_ERR_INVALID_ARG
    assert dp(3, 4, 0, 4) == moe.MOE_ERR_INVALID_ARG            # 256 experts do not split over 3
    assert dp(8, 4, 0, 4, bufs=None) == moe.MOE_ERR_INVALID_ARG
    assert dp(8, 4, 0, 4, bufs=P(68)) == moe.MOE_ERR_INVALID_ARG  # the pointer array misaligned
    assert dp(8, 4, 0, 4, counts=None) == moe.MOE_ERR_INVALID_ARG
    cp = lambda T, d, R, cap, me, bufs=P(64), tok=P(16), acc=P(16): L.moe_ep_combine_peer(
        T, d, R, cap, me, bufs, tok, acc, None, None, None)
    assert cp(4, 7168, 8, 3, 0) == moe.MOE_ERR_INVALID_ARG       # capacity below T
    assert cp(4, 7168, 8, 4, 8) == moe.MOE_ERR_INVALID_ARG       # rank outside [0, n_ranks)
    assert cp(4, 7164, 8, 4, 0) == moe.MOE_ERR_INVALID_ARG       # d not a multiple of 8
    assert cp(4, 7168, 8, 4, 0, bufs=None) == moe.MOE_ERR_INVALID_ARG
    assert cp(4, 7168, 8, 4, 0, tok=None) == moe.MOE_ERR_INVALID_ARG
    assert cp(4, 7168, 8, 4, 0, acc=P(24)) == moe.MOE_ERR_INVALID_ARG  # y_acc misaligned
    assert cp(0, 7168, 8, 4, 0, bufs=None, tok=None, acc=None) == moe.MOE_OK  # nothing to do


def _packed_stand_ins(ep_mod):
    """CPU stand-ins of the packed dispatch / unpack that follow the header's layout
    (bf16 x | int32 ids | fp32 weights | padding; padding slots: token -1, ids -1)."""
    def row_bytes(cfg):
        return (2 * cfg.d + 8 * cfg.top_k + 15) // 16 * 16

    def dispatch_packed(cfg, R, cap, idx, w, x, counts, send_tok, packed, stream=None):
        d, k = cfg.d, cfg.top_k
        c, tok = dispatch_def(idx.numpy(), cfg.n_experts, R)
        counts.copy_(torch.from_numpy(c))
        send_tok.fill_(-1)
        packed.zero_()
        ids_view = packed[:, 2 * d:2 * d + 4 * k]
        ids_view.copy_(torch.full((packed.shape[0], k), -1, dtype=torch.int32).view(torch.uint8))
        base = 0
        for q in range(R):
            for j in range(int(c[q])):
                t = int(tok[base + j])
                s = q * cap + j
                send_tok[s] = t
                packed[s, :2 * d] = x[t].to(torch.bfloat16).view(torch.uint8)
                packed[s, 2 * d:2 * d + 4 * k] = idx[t].view(torch.uint8)
                packed[s, 2 * d + 4 * k:2 * d + 8 * k] = w[t].view(torch.uint8)
            base += int(c[q])

    def unpack(cfg, packed, x_rows, idx, w, stream=None):
        d, k = cfg.d, cfg.top_k
        x_rows.copy_(packed[:, :2 * d].contiguous().view(torch.bfloat16))
        idx.copy_(packed[:, 2 * d:2 * d + 4 * k].contiguous().view(torch.int32))
        w.copy_(packed[:, 2 * d + 4 * k:2 * d + 8 * k].contiguous().view(torch.float32))
        w[(idx < 0).all(1)] = 0.0

    def combine(back, send_tok, y_acc, y=None, residual=None, stream=None):
        keep = send_tok[: back.shape[0]] >= 0
        y_acc.index_add_(0, send_tok[: back.shape[0]][keep].long(), back[keep])
        if y is not None:
            y.copy_((y_acc + (residual.float() if residual is not None else 0)).to(torch.bfloat16))

    ep_mod.ep_packed_row_bytes = row_bytes
    ep_mod.moe_ep_dispatch_packed, ep_mod.moe_ep_unpack, ep_mod.moe_ep_combine = dispatch_packed, unpack, combine


def _ep_layer_rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import fine_grained_moe_gemm_b200 as moe_pkg
    from fine_grained_moe_gemm_b200 import ep

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    E, k, d = 16, 4, 32
    cfg = moe_pkg.MoeConfig(d * 4, E, 4, 2, k, 128, 1, 128, 2.5)
    cfg.d = d
    _stand_ins(ep, E)
    _packed_stand_ins(ep)
    T_max = 9 + 5 * (world - 1)                               # the largest batch, the same on every rank
    layer = ep.EpLayer(cfg, T_max, "cpu")
    shared = {n: torch.empty((128, d), dtype=torch.bfloat16) for n in ("w_gate", "w_up", "w_down")}
    ok = True
    for step, T in enumerate((9 + 5 * rank, 3 + rank, T_max)):   # ranks differ in T; the blocks stay T_max rows
        g = torch.Generator().manual_seed(7 + rank + 100 * step)
        x = torch.randn((T, d), generator=g).to(torch.bfloat16)
        y = torch.empty((T, d), dtype=torch.bfloat16)
        layer.forward(None, {}, shared, torch.zeros(E), x, y)
        xf = x.double()
        top = torch.topk(xf.float()[:, :E], k, dim=1)
        p = torch.sigmoid(top.values)
        wts = (p / p.sum(1, keepdim=True)).double()
        coef = (wts * (top.indices.double() + 1)).sum(1, keepdim=True)
        ref = 0.5 * xf + 2.5 * coef * xf
        ok &= bool(((y.double() - ref).abs() <= 2.0 ** -7 * ref.abs() + 1e-6).all())
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out, f"p{rank}"), "w") as f:
        f.write(str(int(ok)))


@pytest.mark.parametrize("world", [2, 4])
def test_ep_layer_control_flow_gloo(tmp_path, world):
    """EpLayer.forward end to end on gloo ranks (equal-split all-to-alls of packed rows and of the fp32
    results), three batches of different sizes through the same buffers, every token against its closed form."""
    port = _free_port()
    mp.spawn(_ep_layer_rank, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    assert all(open(tmp_path / f"p{r}").read() == "1" for r in range(world))
