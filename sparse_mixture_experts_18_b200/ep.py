"""Expert parallelism for the sparse-MoE block: the n experts are partitioned over the R ranks
of a process group, tokens are sent to the rank that holds their expert, and the expert
outputs come back to each token's original position ("Mixtral 8x7B: Model Bahasa Sparse
Mixture of Experts", id.news.hada.io, section "Implementasi dan Efisiensi Inferensi":
expert parallelism routes a token to the GPU of its expert and returns the expert's output
to the token's position; the load across GPUs has to be balanced).

Rank r holds experts [r*nl, (r+1)*nl), nl = n / R (n % R == 0); every rank has its own batch
of T tokens.  One forward on rank r:
  1. moe_route (library): router, TopK, softmax, and the token rows grouped by expert,
     unpadded, in x_grouped; so the rows bound for rank q are one contiguous slice.
  2. counts exchange: an all-to-all of the per-expert row counts (nl to each peer), after
     which each rank knows how many rows it receives from every source for each local expert.
  3. dispatch: an all-to-all of x_grouped's rows (send split q = rows of q's experts).
  4. moe_experts_forward (library) on the received rows with the local experts' weights;
     outputs in fp32, in received order, not gated.
  5. return: the reverse all-to-all of those fp32 rows.
  6. moe_combine (library): out[t] = sum_k G_k * y[token_rows[t, k]], rounded once.
Steps 2, 3 and 5 are torch.distributed all-to-alls (NCCL's grouped send/receive on GPUs; gloo
on CPU ranks in the tests); this module does no arithmetic on the data, only the host
bookkeeping of the splits.  Without a group (or with one rank) the exchanges are identities
and the result equals the single-GPU block within rounding.

Load balancing (the same page: the load across GPUs has to be balanced) by replicating hot
experts: an ExpertPlacement puts expert e on the ranks replicas[e]; every source splits its
rows of e into len(replicas[e]) contiguous near-equal parts, part j for replicas[e][j].  The
counts exchange becomes an all-gather of every rank's per-expert counts, the grouped rows are
put in destination order by the library's row gather (moe_gather_rows) before the dispatch,
and the returned rows back in grouped order after it; each rank's experts run on the parts
it receives, source-major, each source's parts in the rank's expert order.
"""
from __future__ import annotations

import dataclasses

import torch

from . import moe


@dataclasses.dataclass(frozen=True)
class ExpertPartition:
    """Experts [rank*nl, (rank+1)*nl) live on `rank`; nl = n / world."""
    n: int
    world: int
    rank: int

    def __post_init__(self):
        if self.world < 1 or not 0 <= self.rank < self.world or self.n % self.world:
            raise ValueError(f"{self.n} experts cannot be split evenly over {self.world} ranks")

    @property
    def n_local(self) -> int:
        return self.n // self.world

    def local_experts(self) -> range:
        return range(self.rank * self.n_local, (self.rank + 1) * self.n_local)

    def send_splits(self, counts) -> list[int]:
        """Rows this rank sends to each peer: the rows routed to that peer's experts."""
        c = [int(v) for v in counts]
        nl = self.n_local
        return [sum(c[q * nl:(q + 1) * nl]) for q in range(self.world)]

    @staticmethod
    def recv_splits(recv_counts) -> list[int]:
        """Rows received from each source, from the exchanged counts [world, nl]."""
        return [int(v) for v in recv_counts.reshape(recv_counts.shape[0], -1).sum(dim=1)]


@dataclasses.dataclass(frozen=True)
class ExpertPlacement:
    """Expert e lives on the ranks replicas[e] (ascending, at least one).  A source splits its
    c rows of e into r = len(replicas[e]) contiguous parts, the first c % r of them one row
    longer, part j going to replicas[e][j]."""
    n: int
    world: int
    replicas: tuple

    def __post_init__(self):
        if len(self.replicas) != self.n or self.world < 1:
            raise ValueError("one replica list per expert is needed")
        for reps in self.replicas:
            if not reps or list(reps) != sorted(set(reps)) or reps[0] < 0 or \
                    reps[-1] >= self.world:
                raise ValueError(f"bad replica list {reps}")

    @classmethod
    def contiguous(cls, n: int, world: int) -> "ExpertPlacement":
        """The unreplicated placement of ExpertPartition: expert e on rank e // (n / world)."""
        if n % world:
            raise ValueError(f"{n} experts cannot be split evenly over {world} ranks")
        nl = n // world
        return cls(n, world, tuple((e // nl,) for e in range(n)))

    @classmethod
    def balanced(cls, loads, world: int, slots: int) -> "ExpertPlacement":
        """Start from the contiguous placement and fill each rank up to `slots` experts: give
        the expert with the most rows per replica one more replica, on the least loaded rank
        (rows of its experts, each expert's rows shared evenly by its replicas) that has a free
        slot and does not hold it yet; ties to the lower expert and rank."""
        loads = [float(v) for v in loads]
        n = len(loads)
        base = cls.contiguous(n, world)
        if slots < n // world:
            raise ValueError("fewer slots than the contiguous placement needs")
        reps = [list(r) for r in base.replicas]
        held = [[e for e in range(n) if q in reps[e]] for q in range(world)]

        def rank_load(q):
            return sum(loads[e] / len(reps[e]) for e in held[q])

        while True:
            free = [q for q in range(world) if len(held[q]) < slots]
            best = None
            for e in sorted(range(n), key=lambda e: (-loads[e] / len(reps[e]), e)):
                cand = [q for q in free if q not in reps[e]]
                if cand:
                    best = (e, min(cand, key=lambda q: (rank_load(q), q)))
                    break
            if best is None or loads[best[0]] == 0:
                break
            e, q = best
            reps[e] = sorted(reps[e] + [q])
            held[q] = sorted(held[q] + [e])
        return cls(n, world, tuple(tuple(r) for r in reps))

    def local_experts(self, rank: int) -> list:
        return [e for e in range(self.n) if rank in self.replicas[e]]

    @staticmethod
    def split(count: int, r: int) -> list:
        base, extra = divmod(int(count), r)
        return [base + (1 if j < extra else 0) for j in range(r)]

    def send_order(self, counts):
        """For one source's per-expert counts: the row indices of its grouped rows in
        destination order (destination, then the destination's experts, then the rows of
        the part) and the rows sent to each destination."""
        c = [int(v) for v in counts]
        start = [0] * (self.n + 1)
        for e in range(self.n):
            start[e + 1] = start[e] + c[e]
        order, send = [], []
        for q in range(self.world):
            total = 0
            for e in self.local_experts(q):
                j = self.replicas[e].index(q)
                parts = self.split(c[e], len(self.replicas[e]))
                lo = start[e] + sum(parts[:j])
                order.extend(range(lo, lo + parts[j]))
                total += parts[j]
            send.append(total)
        return order, send

    def recv_counts(self, all_counts, rank: int):
        """Rows this rank receives from each source for each of its experts: [world][n_local]
        from every source's per-expert counts [world][n]."""
        local = self.local_experts(rank)
        out = []
        for s in range(self.world):
            row = []
            for e in local:
                j = self.replicas[e].index(rank)
                row.append(self.split(int(all_counts[s][e]), len(self.replicas[e]))[j])
            out.append(row)
        return out

    def load_per_rank(self, loads) -> list:
        """Rows each rank receives in all, from the global per-expert counts (the parts add
        over sources the way the global count splits, within one row per source)."""
        return [sum(float(loads[e]) / len(self.replicas[e]) for e in self.local_experts(q))
                for q in range(self.world)]


def _world(group):
    import torch.distributed as dist
    if group is None or not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def exchange_counts(counts: torch.Tensor, part: ExpertPartition, group=None) -> torch.Tensor:
    """All-to-all of the per-expert counts [n] (int32): returns [world, nl], row s = the rows
    source s routed to each local expert."""
    if part.world == 1:
        return counts.reshape(1, -1).clone()
    import torch.distributed as dist
    recv = torch.empty_like(counts)
    dist.all_to_all_single(recv, counts.contiguous(), group=group)
    return recv.reshape(part.world, part.n_local)


def dispatch(x_grouped: torch.Tensor, send: list[int], recv: list[int], group=None):
    """All-to-all of the grouped rows: send[q] rows to peer q, recv[s] rows from source s."""
    if len(send) == 1:
        return x_grouped
    import torch.distributed as dist
    out = torch.empty((sum(recv), x_grouped.shape[1]), dtype=x_grouped.dtype,
                      device=x_grouped.device)
    dist.all_to_all_single(out, x_grouped.contiguous(), output_split_sizes=recv,
                           input_split_sizes=send, group=group)
    return out


def return_rows(y_rows: torch.Tensor, send: list[int], recv: list[int], group=None):
    """The reverse of dispatch: each source gets back its rows, in the order it sent them."""
    if len(send) == 1:
        return y_rows
    import torch.distributed as dist
    out = torch.empty((sum(send), y_rows.shape[1]), dtype=y_rows.dtype, device=y_rows.device)
    dist.all_to_all_single(out, y_rows.contiguous(), output_split_sizes=send,
                           input_split_sizes=recv, group=group)
    return out


def exchange_all_counts(counts: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-gather of every rank's per-expert counts [n] (int32): returns [world, n]."""
    if world == 1:
        return counts.reshape(1, -1).clone()
    import torch.distributed as dist
    parts = [torch.empty_like(counts) for _ in range(world)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts)


def _forward_placed(x, W_g, W1_local, W3_local, W2_local, K, placement, group, out, stream):
    world, rank = _world(group)
    n = W_g.shape[1]
    if placement.n != n or placement.world != world:
        raise ValueError("the placement does not match the router or the group")
    local = placement.local_experts(rank)
    if W1_local.shape[0] != len(local):
        raise ValueError(f"rank {rank} holds experts {local}, got {W1_local.shape[0]} weights")
    T, d = x.shape
    if T > 0:
        xg, _, gate, counts, rows = moe.moe_route(x, W_g, K, stream=stream)
    else:
        xg = x.new_empty((0, d))
        gate = torch.empty((0, K), dtype=torch.float32, device=x.device)
        rows = torch.empty((0, K), dtype=torch.int32, device=x.device)
        counts = torch.zeros((n,), dtype=torch.int32, device=x.device)
    all_counts = exchange_all_counts(counts, world, group).cpu()
    order, send = placement.send_order(all_counts[rank])
    seg = placement.recv_counts(all_counts, rank)
    recv = [sum(r) for r in seg]
    inv_order = [0] * len(order)  # host bookkeeping: where each grouped row went
    for i, r in enumerate(order):
        inv_order[r] = i
    perm = torch.tensor(order, dtype=torch.int32).to(x.device)
    inv = torch.tensor(inv_order, dtype=torch.int32).to(x.device)
    x_send = moe.moe_gather_rows(xg, perm, stream=stream) if len(order) else xg
    x_recv = dispatch(x_send, send, recv, group)
    y_recv = moe.moe_experts_forward(
        x_recv, torch.tensor(seg, dtype=torch.int32, device=x.device).reshape(world, -1),
        W1_local, W3_local, W2_local, stream=stream)
    y_send_back = return_rows(y_recv, send, recv, group)
    y_back = moe.moe_gather_rows(y_send_back, inv, stream=stream) if len(order) else y_send_back
    return moe.moe_combine(y_back, rows, gate, out, stream=stream)


def moe_forward_ep(x, W_g, W1_local, W3_local, W2_local, K: int, group=None, out=None,
                   stream=None, placement=None):
    """The MoE block with expert parallelism over `group` (None: one rank).  x [T, d] is this
    rank's batch; W_g [d, n] the full router; W1_local/W3_local [nl, F, d] and W2_local
    [nl, d, F] the weights of this rank's experts (with a placement: of
    placement.local_experts(rank), in that order).  Returns out [T, d] (x's dtype)."""
    if out is None:
        out = torch.empty_like(x)
    if placement is not None:
        return _forward_placed(x, W_g, W1_local, W3_local, W2_local, K, placement, group, out,
                               stream)
    world, rank = _world(group)
    n = W_g.shape[1]
    part = ExpertPartition(n, world, rank)
    if W1_local.shape[0] != part.n_local:
        raise ValueError(f"rank {rank} holds {part.n_local} experts, got {W1_local.shape[0]}")
    if out is None:
        out = torch.empty_like(x)
    T, d = x.shape
    if T == 0 and world == 1:
        return out
    if T > 0:
        xg, _, gate, counts, rows = moe.moe_route(x, W_g, K, stream=stream)
    else:  # nothing to send, but the exchanges still take part
        xg = x.new_empty((0, d))
        gate = torch.empty((0, K), dtype=torch.float32, device=x.device)
        rows = torch.empty((0, K), dtype=torch.int32, device=x.device)
        counts = torch.zeros((n,), dtype=torch.int32, device=x.device)
    recv_counts = exchange_counts(counts, part, group)
    send = part.send_splits(counts.cpu())
    recv = part.recv_splits(recv_counts.cpu())
    x_recv = dispatch(xg, send, recv, group)
    y_recv = moe.moe_experts_forward(x_recv, recv_counts.to(torch.int32), W1_local, W3_local,
                                     W2_local, stream=stream)
    y_back = return_rows(y_recv, send, recv, group)
    return moe.moe_combine(y_back, rows, gate, out, stream=stream)


def load_per_rank(counts, world: int) -> list[int]:
    """Rows each rank's experts receive, from global per-expert counts (for load reports)."""
    nl = len(counts) // world
    return [int(sum(counts[q * nl:(q + 1) * nl])) for q in range(world)]
