"""Sequence-parallel block-sparse attention over several ranks with run-time
head balancing (FVAttn review, §1 Key Terms "Ulysses" and "RLB", §3).

Every rank holds a sequence shard of Q, K and V, [B, H, N/W, d] for W ranks.
One call:
  1. Ulysses all-to-all: the shards become whole sequences of H/W heads per rank,
     [B, H/W, N, d]; a (batch, head) pair is a unit, rank r's unit i having the
     home index r * U + i (U = B * H/W units per rank);
  2. routing of the local units (the per-head top-p block masks) and an
     all-gather of their selected-block counts;
  3. RLB: `fvattn_rlb_plan` on the counts; a unit whose final owner is another
     rank sends its Q, K and V there point to point (one send per unit, however
     many moves the plan made of it);
  4. every rank computes the attention of the units it now holds;
  5. O and LSE of moved units go back to their home ranks, and the reverse
     all-to-all returns every rank's sequence shard of O and LSE.
The collectives are torch.distributed calls on the given process group (NCCL on
GPUs; gloo on the host in the tests).  Routing and attention run in the
library's kernels, or in a compute function the caller injects (the tests use
one built on the oracle).
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist

from . import FvattnPlan, fvattn_rlb_plan


@dataclasses.dataclass
class UlyssesStats:
    """Per-rank selected-block loads before and after balancing, and the moves."""
    loads_before: list
    loads_after: list
    moves: list          # (home unit index, source rank, destination rank), in plan order
    units_sent: int      # units this rank sent out (their final owner is another rank)
    units_received: int  # units this rank received

    @property
    def lif_before(self) -> float:
        m = sum(self.loads_before) / len(self.loads_before)
        return max(self.loads_before) / m if m > 0 else 1.0

    @property
    def lif_after(self) -> float:
        m = sum(self.loads_after) / len(self.loads_after)
        return max(self.loads_after) / m if m > 0 else 1.0


def seq_to_head(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, H, N/W, d] sequence shard -> [B, H/W, N, d] whole sequences of this rank's
    head group (heads r*H/W .. (r+1)*H/W - 1), by one all-to-all."""
    W = dist.get_world_size(group)
    B, H, Nl = x.shape[:3]
    rest = x.shape[3:]
    if H % W:
        raise ValueError(f"{H} heads do not split over {W} ranks")
    send = x.reshape(B, W, H // W, Nl, *rest).movedim(1, 0).contiguous()   # [W(dest), B, H/W, Nl, ...]
    recv = torch.empty_like(send)                                           # [W(source), B, H/W, Nl, ...]
    dist.all_to_all_single(recv, send, group=group)
    return recv.movedim(0, 2).reshape(B, H // W, W * Nl, *rest)


def head_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of :func:`seq_to_head`: [B, H/W, N, ...] -> [B, H, N/W, ...]."""
    W = dist.get_world_size(group)
    B, Hl, N = y.shape[:3]
    rest = y.shape[3:]
    if N % W:
        raise ValueError(f"{N} tokens do not split over {W} ranks")
    send = y.reshape(B, Hl, W, N // W, *rest).movedim(2, 0).contiguous()   # [W(dest), B, H/W, N/W, ...]
    recv = torch.empty_like(send)                                           # [W(source head group), ...]
    dist.all_to_all_single(recv, send, group=group)
    return recv.movedim(0, 1).reshape(B, W * Hl, N // W, *rest)


def _final_owners(moves, total_units: int, units: int) -> list:
    owner = [u // units for u in range(total_units)]
    for u, s, d in moves:
        if owner[u] != s:
            raise RuntimeError("inconsistent load-balancing plan")
        owner[u] = d
    return owner


def kernel_compute(p: float, block: int, causal: bool = False):
    """The default compute: the library's routing and sparse attention on a stack of
    units [1, U, N, d] (bf16, on a CUDA device); returns (O bf16, LSE fp32) and the
    per-unit selected-block counts."""
    plans = {}

    def routes(Q, K):
        key = tuple(Q.shape)
        if key not in plans:
            plans[key] = FvattnPlan(*Q.shape, block, device=Q.device)
        plan = plans[key]
        plan.run_route(Q, K, p)
        return plan

    def counts(Q, K):
        return routes(Q, K).route.head_counts.to(torch.int64)

    def attention(Q, K, V):
        plan = routes(Q, K)
        O, LSE, _ = plan.run_fwd(Q, K, V, causal)
        plan.check()
        return O.clone(), LSE.clone()

    return counts, attention


def ulysses_attention(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, counts_fn, attention_fn, group=None):
    """One sequence-parallel attention step (see the module docstring).

    Q, K, V: this rank's sequence shard [B, H, N/W, d].  counts_fn(Q, K) on a unit
    stack [1, U, N, d] returns its per-unit selected-block counts (int64 [U]);
    attention_fn(Q, K, V) on a unit stack returns (O [1, U, N, d], LSE [1, U, N]).
    Returns this rank's shard of O [B, H, N/W, d] and LSE [B, H, N/W], and the
    balancing statistics."""
    W = dist.get_world_size(group)
    me = dist.get_rank(group)
    Qh, Kh, Vh = (seq_to_head(x, group) for x in (Q, K, V))      # [B, H/W, N, d]
    B, Hl, N, d = Qh.shape
    U = B * Hl
    units = [x.reshape(1, U, N, d) for x in (Qh, Kh, Vh)]
    # per-unit work of every rank
    local = counts_fn(units[0], units[1]).to(torch.int64).reshape(U)
    gathered = [torch.empty_like(local) for _ in range(W)]
    dist.all_gather(gathered, local, group=group)
    work = torch.stack(gathered).cpu()                             # [W, U]
    moves = fvattn_rlb_plan(work.numpy()) if W > 1 else []
    owner = _final_owners(moves, W * U, U)
    loads_before = work.sum(1).tolist()
    loads_after = [0] * W
    for u in range(W * U):
        loads_after[owner[u]] += int(work.reshape(-1)[u])
    # the units this rank computes: its own that stay, then those it receives (home order)
    mine = [u for u in range(W * U) if owner[u] == me]
    send_units = [u for u in range(me * U, (me + 1) * U) if owner[u] != me]
    recv_units = [u for u in mine if u // U != me]
    stacks = [torch.empty((1, len(mine), N, d), dtype=x.dtype, device=x.device) for x in units]
    pos = {u: k for k, u in enumerate(mine)}
    for u in mine:
        if u // U == me:
            for s, x in zip(stacks, units):
                s[0, pos[u]] = x[0, u - me * U]
    ops = []
    for u in send_units:
        for x in units:
            ops.append(dist.P2POp(dist.isend, x[0, u - me * U].contiguous(), owner[u], group=group))
    for u in recv_units:
        for s in stacks:
            ops.append(dist.P2POp(dist.irecv, s[0, pos[u]], u // U, group=group))
    _run_p2p(ops, group)
    # attention of the units held here
    O_m, L_m = attention_fn(*stacks) if mine else (None, None)
    # results of received units back to their homes
    O_loc = torch.empty((1, U, N, d), dtype=O_m.dtype if O_m is not None else Q.dtype, device=Q.device)
    L_loc = torch.empty((1, U, N), dtype=L_m.dtype if L_m is not None else torch.float32, device=Q.device)
    for u in mine:
        if u // U == me:
            O_loc[0, u - me * U] = O_m[0, pos[u]]
            L_loc[0, u - me * U] = L_m[0, pos[u]]
    ops = []
    for u in recv_units:
        ops.append(dist.P2POp(dist.isend, O_m[0, pos[u]].contiguous(), u // U, group=group))
        ops.append(dist.P2POp(dist.isend, L_m[0, pos[u]].contiguous(), u // U, group=group))
    for u in send_units:
        ops.append(dist.P2POp(dist.irecv, O_loc[0, u - me * U], owner[u], group=group))
        ops.append(dist.P2POp(dist.irecv, L_loc[0, u - me * U], owner[u], group=group))
    _run_p2p(ops, group)
    O = head_to_seq(O_loc.reshape(B, Hl, N, d), group)
    LSE = head_to_seq(L_loc.reshape(B, Hl, N), group)
    stats = UlyssesStats(loads_before, loads_after, moves, len(send_units), len(recv_units))
    return O, LSE, stats


def _run_p2p(ops, group):
    """Batched point-to-point operations; every rank calls this at the same step,
    with or without operations of its own (an empty list still takes part)."""
    if ops:
        for r in dist.batch_isend_irecv(ops):
            r.wait()
    dist.barrier(group=group)
