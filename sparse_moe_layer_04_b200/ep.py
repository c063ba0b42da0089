"""Expert parallelism for the MoE layer over several GPUs.

Layout (the pages' default multi-GPU layout is expert parallelism: "GLM-5.2",
PocketLLM, Implemented execution path): rank r owns a contiguous block of the
routed experts and holds only their weights; every rank holds the router, the
bias and the shared expert; tokens stay on their home rank.  One layer pass:

  1. route the home tokens over all E experts (router replicated);
  2. group the (token, slot) pairs by expert -- experts are blocked by owner,
     so the grouped rows are also ordered by destination rank -- and gather
     their hidden rows into a send buffer;
  3. exchange the per-expert row counts (all-gather of E ints per rank) and
     send each owner its rows (all-to-all with per-rank splits);
  4. the owner groups the received rows by its local experts (sources in rank
     order inside each expert) and runs the expert MLPs on them;
  5. the expert outputs travel back in the order they arrived (all-to-all);
  6. the home rank adds the shared expert and merges with the routing weights.

The result equals the single-GPU layer on the same tokens: the same rows meet
the same experts, and the merge runs in the same fixed order.

The collectives are torch.distributed all-gather / all_to_all_single (NCCL
over NVLink on GPUs).  The row counts must reach the host to size the splits,
so a pass synchronises the stream once after the grouping.  Device work goes
through the library's C ABI (`CudaOps`); another implementation of the same
`Ops` methods can be passed in (the CPU tests pass the oracle's).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist


# ---------------------------------------------------------------------------
# planning (host)
# ---------------------------------------------------------------------------
def owner_ranges(E: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous expert blocks [lo, hi) per rank; the first E % world ranks
    own one expert more."""
    if world < 1 or E < world:
        raise ValueError(f"need 1 <= world <= E (world={world}, E={E})")
    base, extra = divmod(E, world)
    out, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


@dataclass
class ExchangePlan:
    """Row counts and orders of one pass on one rank.

    send_counts[r]      rows this rank sends to rank r (its pairs routed to r's experts)
    recv_counts[s]      rows this rank receives from rank s
    recv_expert[s, e]   rows from rank s for local expert e
    local_offsets       [E_local + 1] grouped-row offsets of the local experts
    local_perm          [R] grouped row -> received row (sources in rank order
                        inside each local expert)
    local_inv           [R] received row -> grouped row
    """
    send_counts: List[int]
    recv_counts: List[int]
    recv_expert: np.ndarray
    local_offsets: np.ndarray
    local_perm: np.ndarray
    local_inv: np.ndarray


def plan_exchange(all_counts: np.ndarray, ranges: Sequence[Tuple[int, int]],
                  rank: int) -> ExchangePlan:
    """Plan from every rank's per-expert pair counts `all_counts` [world, E]."""
    all_counts = np.asarray(all_counts, dtype=np.int64)
    world = len(ranges)
    lo, hi = ranges[rank]
    send = [int(all_counts[rank, a:b].sum()) for a, b in ranges]
    recv_expert = all_counts[:, lo:hi]                       # [world, E_local]
    recv = [int(x) for x in recv_expert.sum(axis=1)]
    e_local = hi - lo
    per_expert = recv_expert.sum(axis=0)
    local_offsets = np.zeros(e_local + 1, dtype=np.int64)
    np.cumsum(per_expert, out=local_offsets[1:])
    R = int(local_offsets[-1])
    # received row of (source s, local expert e, i): source block start + the
    # source's rows for earlier local experts + i
    src_start = np.concatenate([[0], np.cumsum(recv)[:-1]]) if world else np.zeros(0, np.int64)
    src_exp_start = src_start[:, None] + np.concatenate(
        [np.zeros((world, 1), np.int64), np.cumsum(recv_expert, axis=1)[:, :-1]], axis=1)
    # grouped row of (e, s, i): expert start + rows of earlier sources + i
    grp_src_start = local_offsets[:-1][None, :] + np.concatenate(
        [np.zeros((1, e_local), np.int64), np.cumsum(recv_expert, axis=0)[:-1]], axis=0)
    local_perm = np.empty(R, dtype=np.int64)
    for s in range(world):
        for e in range(e_local):
            n = int(recv_expert[s, e])
            if n:
                g0, r0 = int(grp_src_start[s, e]), int(src_exp_start[s, e])
                local_perm[g0:g0 + n] = np.arange(r0, r0 + n)
    local_inv = np.empty(R, dtype=np.int64)
    local_inv[local_perm] = np.arange(R)
    return ExchangePlan(send, recv, recv_expert, local_offsets, local_perm, local_inv)


# ---------------------------------------------------------------------------
# device work through the C ABI
# ---------------------------------------------------------------------------
class CudaOps:
    """The device steps of an expert-parallel pass, each one call of the
    library's C ABI on the current stream."""

    y_dtype = torch.float32   # expert outputs and the merge input

    def __init__(self):
        import sparse_moe_layer_04_b200 as moe
        self.moe = moe
        self._ws = {}

    def _workspace(self, d):
        """One workspace per call shape apart from T, grown when a larger T
        needs more (the received row count changes from pass to pass)."""
        key = (d.D, d.E, d.F, d.k, d.S, d.Fs)
        need = self.moe.moe_workspace_size(d)
        ws = self._ws.get(key)
        if ws is None or ws.numel() < need:
            ws = self.moe.alloc_workspace(d)
            self._ws[key] = ws
        return ws

    def route(self, h, Wr, bias, d):
        ws = self._workspace(d)
        logits = torch.empty((d.T, d.E), dtype=torch.float32, device=h.device)
        idx = torch.empty((d.T, d.k), dtype=torch.int32, device=h.device)
        w = torch.empty((d.T, d.k), dtype=torch.float32, device=h.device)
        self.moe.moe_router_logits(h, Wr, d, logits, ws)
        self.moe.moe_route(logits, bias, d, idx, w, ws)
        return idx, w

    def permute(self, idx, d):
        ws = self._workspace(d)
        dev = idx.device
        counts = torch.empty(d.E, dtype=torch.int32, device=dev)
        offsets = torch.empty(d.E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(d.T * d.k, dtype=torch.int32, device=dev)
        inv = torch.empty((d.T, d.k), dtype=torch.int32, device=dev)
        self.moe.moe_permute(idx, d, counts, offsets, perm, inv, ws)
        return counts, offsets, perm, inv

    def gather_rows(self, src, idx, n_rows):
        dst = torch.empty((n_rows, src.shape[1]), dtype=src.dtype, device=src.device)
        if n_rows:
            self.moe.moe_gather_rows(src, idx, dst)
        return dst

    def expert_ffn(self, x, perm, offsets, W1, W3, W2, D, F):
        """Routed expert MLPs on received rows x [R, D] (grouped by `offsets`
        over the local experts, row order `perm`) -> [R, D] fp32, grouped order."""
        R = x.shape[0]
        y = torch.empty((R, D), dtype=torch.float32, device=x.device)
        if R == 0:
            return y
        e_local = W1.shape[0]
        d = self.moe.dims(T=R, D=D, E=e_local, F=F, k=1, S=0, Fs=16)
        ws = self._workspace(d)
        self.moe.moe_expert_ffn(x, perm, offsets, W1, W3, W2, None, None, None, d, y, ws)
        return y

    def shared_ffn(self, h, Ws1, Ws3, Ws2, y_full, routed_rows):
        """Shared experts on every home token, written to the shared part of
        the merge input: rows routed_rows.. of y_full [routed_rows + S*T, D]."""
        T, D = h.shape
        S, Fs = Ws1.shape[0], Ws1.shape[1]
        if T == 0 or S == 0:
            return
        # one routed expert with no rows (offsets all zero), so only the shared
        # tiles run; the library places shared rows after its T routed rows,
        # so its output view starts T rows before the shared part
        d = self.moe.dims(T=T, D=D, E=1, F=Fs, k=1, S=S, Fs=Fs)
        ws = self._workspace(d)
        perm = torch.zeros(T, dtype=torch.int32, device=h.device)
        offsets = torch.zeros(2, dtype=torch.int32, device=h.device)
        view = y_full[routed_rows - T:]
        self.moe.moe_expert_ffn(h, perm, offsets, Ws1, Ws3, Ws2, Ws1, Ws3, Ws2, d, view, ws)

    def combine(self, y_full, w, inv, d):
        out = torch.empty((d.T, d.D), dtype=torch.float32, device=y_full.device)
        self.moe.moe_combine(y_full, w, inv, d, out, self._workspace(d))
        return out


# ---------------------------------------------------------------------------
# one layer pass
# ---------------------------------------------------------------------------
def _all_gather_counts(counts: torch.Tensor, world: int, group) -> np.ndarray:
    c = counts.to(torch.int64).reshape(1, -1)
    out = [torch.empty_like(c) for _ in range(world)]
    dist.all_gather(out, c, group=group)
    return torch.cat(out).cpu().numpy()


def ep_forward(h: torch.Tensor, Wr: torch.Tensor, bias: torch.Tensor,
               W1_local: torch.Tensor, W3_local: torch.Tensor, W2_local: torch.Tensor,
               Ws1: Optional[torch.Tensor], Ws3: Optional[torch.Tensor],
               Ws2: Optional[torch.Tensor], dims, group=None, ops=None):
    """One expert-parallel layer pass on this rank's tokens h [T, D].

    W1_local/W3_local [E_r, F, D] and W2_local [E_r, D, F] are the weights of
    this rank's experts (owner_ranges(E, world)[rank]); Ws* the shared experts
    (or None when dims.S == 0).  Every rank of `group` must call this with the
    same E, D, F, k, S (T may differ).  Returns (out [T, D] fp32, idx [T, k],
    w [T, k]) with idx/w the routing of the home tokens.
    """
    ops = ops if ops is not None else CudaOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ranges = owner_ranges(dims.E, world)
    lo, hi = ranges[rank]
    if W1_local.shape[0] != hi - lo:
        raise ValueError(f"rank {rank} owns experts [{lo}, {hi}) but got {W1_local.shape[0]}")
    T, D, k, S = dims.T, dims.D, dims.k, dims.S
    dev = h.device

    # 1-2: route, group by expert (= by destination), gather the send rows
    if T > 0:
        idx, w = ops.route(h, Wr, bias, dims)
        counts, offsets, perm, inv = ops.permute(idx, dims)
    else:
        idx = torch.empty((0, k), dtype=torch.int32, device=dev)
        w = torch.empty((0, k), dtype=torch.float32, device=dev)
        counts = torch.zeros(dims.E, dtype=torch.int32, device=dev)
        inv = torch.empty((0, k), dtype=torch.int32, device=dev)
        perm = torch.empty(0, dtype=torch.int32, device=dev)
    xsend = ops.gather_rows(h, perm, T * k)

    # 3: counts to every rank, then the rows to their owners
    plan = plan_exchange(_all_gather_counts(counts, world, group), ranges, rank)
    R = int(plan.local_offsets[-1])
    xrecv = torch.empty((R, D), dtype=h.dtype, device=dev)
    dist.all_to_all_single(xrecv, xsend, plan.recv_counts, plan.send_counts, group=group)

    # 4: the local experts on the received rows (grouped order), then back to
    # arrival order
    perm_l = torch.as_tensor(plan.local_perm, dtype=torch.int32).to(dev)
    offs_l = torch.as_tensor(plan.local_offsets, dtype=torch.int32).to(dev)
    inv_l = torch.as_tensor(plan.local_inv, dtype=torch.int32).to(dev)
    y_grouped = ops.expert_ffn(xrecv, perm_l, offs_l, W1_local, W3_local, W2_local, D,
                               W1_local.shape[1])
    y_arrival = ops.gather_rows(y_grouped, inv_l, R)

    # 5: outputs back to the home ranks, landing in the home grouped order
    y_full = torch.empty((T * k + S * T, D), dtype=getattr(ops, "y_dtype", torch.float32),
                         device=dev)
    dist.all_to_all_single(y_full[:T * k], y_arrival, plan.send_counts, plan.recv_counts,
                           group=group)

    # 6: shared experts on the home tokens, then the fixed-order merge
    if T == 0:
        return torch.empty((0, D), dtype=torch.float32, device=dev), idx, w
    if S > 0:
        ops.shared_ffn(h, Ws1, Ws3, Ws2, y_full, T * k)
    out = ops.combine(y_full, w, inv, dims)
    return out, idx, w
