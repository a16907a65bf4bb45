"""Expert parallelism: the MoE layer forward with the routed experts split over the
ranks of a process group (one process per GPU) in contiguous blocks of E / world
experts.  With world = n_groups each rank holds one group of 32 experts: the
groups are device-aligned ("DeepSeek-V3" llm-vis, "MoE router" box), so a token's
rows go to at most topk_groups ranks.

One forward on every rank, in the same order on all of them:

    moe_route         own tokens -> topk_idx, topk_w
    moe_ep_dispatch   rows for each rank (each token once per rank), rank-major
    exchange          counts, then rows, expert ids and weights (all-to-all)
    moe_experts_routed  this rank's block of experts on the rows it received
    exchange          the fp32 partial sums back to the ranks the rows came from
    moe_dense_ffn     the shared expert on own tokens, fp32 (y_acc)
    moe_ep_combine    y_acc[token] += partial sums; y = bf16(y_acc)

Every step but the exchange runs in the library's kernels; the exchange is
torch.distributed's all-to-all (NCCL between GPUs, gloo on CPU).  The result
equals moe_forward's on the same tokens up to the order of fp32 additions.

Two forms of the same layer:
  moe_forward_ep  variable-size exchange: the row counts go to the host, so only
                  the rows that exist cross the link (large batches); it syncs
                  the host once per forward and allocates per call.
  EpLayer         fixed-capacity exchange, for decode-sized batches: every
                  buffer is allocated once for up to T_max tokens per rank; rank
                  q's rows travel in a block of T_max packed rows (x, expert ids
                  and weights in one row; unused slots marked by ids -1), so both
                  all-to-alls have equal splits known in advance, nothing waits
                  on the host, and a forward can be captured in a CUDA graph.
                  The price is padding: each block is T_max rows whatever the
                  count.  With exchange="peer" the same layer moves its rows
                  without an all-to-all: the receive and result buffers are
                  symmetric memory (every rank maps the others' buffers), the
                  dispatch kernel stores each rank's packed rows straight into
                  that rank's receive buffer and the combine kernel reads the
                  partial sums straight from the result buffer of the rank that
                  computed them (peer stores and loads over NVLink between GPUs);
                  a one-element all-reduce on the stream after the dispatch and
                  after the experts orders those accesses across the ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (MOE_BF16, MOE_E4M3, MoeConfig, dense_workspace_size, ep_max_send_rows, ep_packed_row_bytes,
               experts_routed_workspace_size, moe_dense_ffn, moe_ep_combine, moe_ep_combine_peer, moe_ep_dispatch,
               moe_ep_dispatch_packed, moe_ep_dispatch_peer, moe_ep_unpack, moe_experts_routed, moe_route)


def exchange_counts(send_counts: torch.Tensor, group=None) -> torch.Tensor:
    """send_counts[q] = rows this rank sends to rank q; returns recv_counts[q] = rows rank q sends here."""
    recv = torch.empty_like(send_counts)
    dist.all_to_all_single(recv, send_counts, group=group)
    return recv


def exchange(send: torch.Tensor, send_counts: list[int], recv_counts: list[int], group=None) -> torch.Tensor:
    """Rows of ``send`` (rank-major: send_counts[q] rows for rank q) to their ranks; returns the rows this rank
    receives, rank-major (recv_counts[q] rows from rank q)."""
    recv = send.new_empty((sum(recv_counts),) + tuple(send.shape[1:]))
    dist.all_to_all_single(recv, send[: sum(send_counts)].contiguous(), recv_counts, send_counts, group=group)
    return recv


def expert_block(cfg: MoeConfig, rank: int, world: int) -> tuple[int, int]:
    """(first expert, number of experts) of ``rank``'s block."""
    if cfg.n_experts % world:
        raise ValueError(f"{cfg.n_experts} experts do not split over {world} ranks")
    n = cfg.n_experts // world
    return rank * n, n


def moe_forward_ep(cfg: MoeConfig, w_router, local_weights: dict, shared_weights: dict, bias, x, y, group=None,
                   residual=None):
    """y = MoE(x) (+ residual) for this rank's tokens x [T, d], with this rank's block of experts.

    ``local_weights``: the block's w_gate / w_up [n, H, d], w_down [n, d, H] (e4m3: plus s_gate / s_up / s_down),
    n = E / world.  ``shared_weights``: the shared expert's w_gate / w_up [Hs, d], w_down [d, Hs] (e4m3: plus
    their scales).  ``y`` [T, d] bf16 (may be ``residual``).  Every rank of ``group`` calls this together.  The
    kernels run on the current stream, which torch.distributed orders the collectives with."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    lo, n_local = expert_block(cfg, rank, world)
    if cfg.n_shared != 1:
        raise ValueError("the expert-parallel layer takes one shared expert")
    dev = x.device
    T, d, k = x.shape[0], cfg.d, cfg.top_k
    # (1) routing of this rank's tokens
    logits = torch.empty((T, cfg.n_experts), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    moe_route(cfg, x, w_router, logits, bias, idx, w)
    # (2) dispatch
    rows = ep_max_send_rows(cfg, T, world)
    counts = torch.empty(world, dtype=torch.int32, device=dev)
    offsets = torch.empty(world + 1, dtype=torch.int32, device=dev)
    send_tok = torch.empty(max(rows, 1), dtype=torch.int32, device=dev)
    send_x = torch.empty((max(rows, 1), d), dtype=torch.bfloat16, device=dev)
    send_idx = torch.empty((max(rows, 1), k), dtype=torch.int32, device=dev)
    send_w = torch.empty((max(rows, 1), k), dtype=torch.float32, device=dev)
    moe_ep_dispatch(cfg, world, idx, w, x, counts, offsets, send_tok, send_x, send_idx, send_w)
    # (3) exchange: the split sizes must be known on the host
    recv_counts = exchange_counts(counts, group)
    sc, rc = counts.tolist(), recv_counts.tolist()
    recv_x = exchange(send_x, sc, rc, group)
    recv_idx = exchange(send_idx, sc, rc, group)
    recv_w = exchange(send_w, sc, rc, group)
    # (4) this rank's experts on the rows it received
    n_recv = recv_x.shape[0]
    recv_y = torch.empty((n_recv, d), dtype=torch.float32, device=dev)
    if n_recv:
        ws = torch.empty(experts_routed_workspace_size(cfg, n_local, n_recv), dtype=torch.uint8, device=dev)
        moe_experts_routed(cfg, local_weights, lo, n_local, recv_x, recv_idx, recv_w, recv_y, workspace=ws)
    # (5) the partial sums back to where the rows came from
    back = exchange(recv_y, rc, sc, group)
    # (6) the shared expert on this rank's tokens, (7) combine
    y_acc = torch.empty((T, d), dtype=torch.float32, device=dev)
    if T:
        wdt = MOE_E4M3 if shared_weights["w_gate"].dtype == torch.uint8 else MOE_BF16
        hs = shared_weights["w_gate"].shape[0]
        dws = torch.empty(dense_workspace_size(d, hs, cfg.act_dtype, wdt, T), dtype=torch.uint8, device=dev)
        moe_dense_ffn(shared_weights["w_gate"], shared_weights["w_up"], shared_weights["w_down"], x, y_acc,
                      shared_weights.get("s_gate"), shared_weights.get("s_up"), shared_weights.get("s_down"),
                      workspace=dws)
        moe_ep_combine(back, send_tok, y_acc, y, residual)


class EpLayer:
    """The expert-parallel layer with a device-resident, fixed-capacity exchange (see the module docstring).

    Every rank of ``group`` builds one with the same ``T_max`` and calls :meth:`forward` together.  Buffers are
    allocated here, once; a forward allocates nothing, never reads a count on the host, and its two all-to-alls
    have equal splits (T_max packed rows per peer there, T_max fp32 rows back), so on NCCL it can be captured in a
    CUDA graph.  ``shared_hidden`` / ``shared_e4m3`` size the shared expert's workspace.

    ``exchange``: "all_to_all" (NCCL all-to-alls of the packed rows and of the partial sums) or "peer" (the
    receive and result buffers in symmetric memory; the dispatch stores into the peers' receive buffers and the
    combine loads from their result buffers, with an all-reduce of one element after each as the fence)."""

    def __init__(self, cfg: MoeConfig, T_max: int, device, group=None, shared_hidden: int | None = None,
                 shared_e4m3: bool = False, exchange: str = "all_to_all"):
        if cfg.n_shared != 1:
            raise ValueError("the expert-parallel layer takes one shared expert")
        if exchange not in ("all_to_all", "peer"):
            raise ValueError(f"exchange: {exchange!r}, expected 'all_to_all' or 'peer'")
        self.cfg, self.T_max, self.group, self.exchange = cfg, int(T_max), group, exchange
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.lo, self.n_local = expert_block(cfg, self.rank, self.world)
        d, k, E = cfg.d, cfg.top_k, cfg.n_experts
        slots = self.world * self.T_max
        rb = ep_packed_row_bytes(cfg)
        dev = torch.device(device)
        f32, i32 = torch.float32, torch.int32
        self.logits = torch.empty((self.T_max, E), dtype=f32, device=dev)
        self.idx = torch.empty((self.T_max, k), dtype=i32, device=dev)
        self.w = torch.empty((self.T_max, k), dtype=f32, device=dev)
        self.counts = torch.empty(self.world, dtype=i32, device=dev)
        self.send_tok = torch.empty(slots, dtype=i32, device=dev)
        self.send = torch.empty((slots, rb), dtype=torch.uint8, device=dev) if exchange == "all_to_all" else None
        self.recv = self._buffer((slots, rb), torch.uint8, dev)
        self.recv_x = torch.empty((slots, d), dtype=torch.bfloat16, device=dev)
        self.recv_idx = torch.empty((slots, k), dtype=i32, device=dev)
        self.recv_w = torch.empty((slots, k), dtype=f32, device=dev)
        self.recv_y = self._buffer((slots, d), f32, dev)
        self.back = torch.empty((slots, d), dtype=f32, device=dev) if exchange == "all_to_all" else None
        if exchange == "peer":
            self.recv_ptrs = self._peer_pointers(self.recv)
            self.result_ptrs = self._peer_pointers(self.recv_y)
            self.fence_buf = torch.zeros(1, dtype=torch.int32, device=dev)
        self.y_acc = torch.empty((self.T_max, d), dtype=f32, device=dev)
        self.ws = torch.empty(max(experts_routed_workspace_size(cfg, self.n_local, slots), 1), dtype=torch.uint8,
                              device=dev)
        hs = cfg.shared_hidden if shared_hidden is None else shared_hidden
        wdt = MOE_E4M3 if shared_e4m3 else MOE_BF16
        self.dws = torch.empty(max(dense_workspace_size(d, hs, cfg.act_dtype, wdt, self.T_max), 1),
                               dtype=torch.uint8, device=dev)

    def _buffer(self, shape, dtype, dev):
        if self.exchange == "all_to_all":
            return torch.empty(shape, dtype=dtype, device=dev)
        import torch.distributed._symmetric_memory as symm_mem
        return symm_mem.empty(*shape, dtype=dtype, device=dev)

    def _peer_pointers(self, buf: torch.Tensor) -> torch.Tensor:
        """Device array of every rank's address of ``buf`` (a symmetric-memory tensor), as this process maps
        them; entry ``rank`` is ``buf`` itself."""
        import torch.distributed._symmetric_memory as symm_mem
        handle = symm_mem.rendezvous(buf, self.group if self.group is not None else dist.group.WORLD)
        ptrs = [int(p) + int(handle.offset) for p in handle.buffer_ptrs]
        if ptrs[self.rank] != buf.data_ptr():
            raise RuntimeError("symmetric memory: this rank's mapped address is not the tensor's")
        self._handles = getattr(self, "_handles", []) + [handle]  # the mappings live as long as the layer
        return torch.tensor(ptrs, dtype=torch.int64, device=buf.device)

    def _fence(self):
        """Every rank's earlier kernels on this stream are done before any rank's later ones start."""
        dist.all_reduce(self.fence_buf, group=self.group)

    def forward(self, w_router, local_weights: dict, shared_weights: dict, bias, x, y, residual=None):
        """y = MoE(x) (+ residual) for this rank's tokens x [T, d], T <= T_max; arguments as moe_forward_ep."""
        cfg, T = self.cfg, x.shape[0]
        if T > self.T_max:
            raise ValueError(f"{T} tokens, the layer was built for at most {self.T_max}")
        # (1) routing of this rank's tokens, (2) dispatch into fixed-capacity packed rows
        moe_route(cfg, x, w_router, self.logits[:T], bias, self.idx[:T], self.w[:T])
        if self.exchange == "peer":
            # (2+3) the packed rows stored straight into each rank's receive buffer
            moe_ep_dispatch_peer(cfg, self.world, self.T_max, self.rank, self.idx[:T], self.w[:T], x, self.counts,
                                 self.send_tok, self.recv_ptrs)
            self._fence()
        else:
            moe_ep_dispatch_packed(cfg, self.world, self.T_max, self.idx[:T], self.w[:T], x, self.counts,
                                   self.send_tok, self.send)
            # (3) rows to their ranks: equal blocks of T_max rows, no counts needed
            dist.all_to_all_single(self.recv, self.send, group=self.group)
        # (4) this rank's experts on every received slot (padding slots carry no local expert)
        moe_ep_unpack(cfg, self.recv, self.recv_x, self.recv_idx, self.recv_w)
        moe_experts_routed(cfg, local_weights, self.lo, self.n_local, self.recv_x, self.recv_idx, self.recv_w,
                           self.recv_y, workspace=self.ws)
        # (5) partial sums back, block for block (peer: left in place, read by the combine)
        if self.exchange == "peer":
            self._fence()
        else:
            dist.all_to_all_single(self.back, self.recv_y, group=self.group)
        # (6) the shared expert on this rank's tokens, (7) combine (padding slots skipped)
        if T:
            moe_dense_ffn(shared_weights["w_gate"], shared_weights["w_up"], shared_weights["w_down"], x,
                          self.y_acc[:T], shared_weights.get("s_gate"), shared_weights.get("s_up"),
                          shared_weights.get("s_down"), workspace=self.dws)
            if self.exchange == "peer":
                moe_ep_combine_peer(self.world, self.T_max, self.rank, self.result_ptrs, self.send_tok,
                                    self.y_acc[:T], y, residual)
            else:
                moe_ep_combine(self.back, self.send_tok, self.y_acc[:T], y, residual)
