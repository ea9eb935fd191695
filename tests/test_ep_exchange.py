"""Expert parallelism's exchange logic on CPU ranks (gloo): the counts exchange, the dispatch
of grouped rows to the rank that holds their expert, and the return of the expert outputs to
their sender, bit for bit.

Each rank routes its own batch with the oracle's router (test infrastructure; the product
path routes on the GPU), groups its (token, slot) rows by expert in the single-rank order
(stable: by expert, then token, then slot), and runs the module's exchange steps.  A
stand-in expert op (row * (1 + global expert id), fp32) is applied on the receiving rank, so
that a row that reached the wrong rank or came back to the wrong place shows up."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _group_rows(x, idx, n, K):
    """Single-rank grouping: x_grouped, token_rows [T, K], counts [n], expert of each row."""
    T = x.shape[0]
    flat = idx.reshape(-1)
    order = sorted(range(T * K), key=lambda i: (int(flat[i]), i))
    xg = x.repeat_interleave(K, dim=0)[order] if T else x.new_empty((0, x.shape[1]))
    rows = np.empty(T * K, np.int64)
    rows[order] = np.arange(T * K)
    counts = np.bincount(flat, minlength=n).astype(np.int32)
    return xg, rows.reshape(T, K), counts, flat[order]


def _stand_in_expert(rows, experts):
    return rows * (1.0 + torch.as_tensor(experts, dtype=torch.float32)).reshape(-1, 1)


def _worker(rank, world, port, Ts, n, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import moe_inputs
    import oracle
    from sparse_mixture_experts_18_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        K, d = 2, 64
        T = Ts[rank]
        w = moe_inputs.small(T=max(T, 1), d=d, F=64, n=n, K=K, dtype="f32", rms_x=False,
                             seed=100 + rank)
        x = moe_inputs.make_x(w)[:T]
        Wg = moe_inputs.make_layer(w.replace(seed=7))["Wg"]     # one router for all ranks
        idx = oracle.route(x, Wg, n, K)[1] if T else np.zeros((0, K), np.int32)
        xg, rows, counts, row_expert = _group_rows(x, idx, n, K)

        part = ep.ExpertPartition(n, world, rank)
        recv_counts = ep.exchange_counts(torch.from_numpy(counts), part)
        send, recv = part.send_splits(counts), part.recv_splits(recv_counts)
        x_recv = ep.dispatch(xg, send, recv)

        # what should have arrived: every source's rows of this rank's experts, source-major
        everyone = [None] * world
        dist.all_gather_object(everyone, (xg, counts, row_expert))
        lo, hi = part.local_experts().start, part.local_experts().stop
        want, want_e = [], []
        for sxg, sc, se in everyone:
            start = int(sc[:lo].sum())
            stop = int(sc[:hi].sum())
            want.append(sxg[start:stop])
            want_e.append(se[start:stop])
        want_e = np.concatenate(want_e) if want_e else np.zeros(0, np.int32)
        arrived_ok = torch.equal(x_recv, torch.cat(want))
        counts_ok = all(int(recv_counts[s_, e - lo]) == int(everyone[s_][1][e])
                        for s_ in range(world) for e in range(lo, hi))

        y_recv = _stand_in_expert(x_recv, want_e)
        y_back = ep.return_rows(y_recv, send, recv)
        back_ok = torch.equal(y_back, _stand_in_expert(xg, row_expert))
        # each (token, slot) finds its own expert's output at token_rows[t, k]
        pos_ok = all(torch.equal(y_back[rows[t, k]], x[t] * (1.0 + float(idx[t, k])))
                     for t in range(T) for k in range(K))
        q.put((rank, arrived_ok, counts_ok, back_ok, pos_ok, send, recv))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,Ts,n", [(2, (37, 5), 8), (2, (0, 9), 8), (4, (11, 3, 20, 1), 8),
                                        (2, (30, 30), 16)])
def test_dispatch_and_return_over_gloo(world, Ts, n):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, Ts, n, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, arrived_ok, counts_ok, back_ok, pos_ok, send, recv in res:
        assert counts_ok, rank
        assert arrived_ok, rank
        assert back_ok, rank
        assert pos_ok, rank
        assert sum(send) == Ts[rank] * 2
    # everything sent is received somewhere
    assert sum(sum(r[6]) for r in res) == sum(Ts) * 2


def test_partition_and_load_bookkeeping():
    from sparse_mixture_experts_18_b200 import ep
    part = ep.ExpertPartition(8, 4, 2)
    assert part.n_local == 2 and list(part.local_experts()) == [4, 5]
    assert part.send_splits([1, 2, 3, 4, 5, 6, 7, 8]) == [3, 7, 11, 15]
    assert ep.ExpertPartition.recv_splits(torch.tensor([[1, 2], [0, 0], [5, 1], [2, 2]])) == \
        [3, 0, 6, 4]
    with pytest.raises(ValueError):
        ep.ExpertPartition(8, 3, 0)
    with pytest.raises(ValueError):
        ep.ExpertPartition(8, 2, 2)
    # the skewed workload's measured expert loads (28081 ... 2318 rows of 65536) over 2 and 8
    # ranks: the busiest rank carries 81% and 43% of all rows
    loads = [28081, 12230, 7519, 5326, 4073, 3270, 2719, 2318]
    assert ep.load_per_rank(loads, 2) == [53156, 12380]
    assert max(ep.load_per_rank(loads, 8)) / sum(loads) == pytest.approx(0.4285, abs=1e-3)


# ------------------------------------------------------------------ replicated experts

SKEWED_LOADS = [28081, 12230, 7519, 5326, 4073, 3270, 2719, 2318]


def test_balanced_placement_invariants():
    from sparse_mixture_experts_18_b200 import ep
    for world, slots in [(2, 4), (2, 6), (4, 2), (4, 3), (8, 1), (8, 2), (8, 4)]:
        pl = ep.ExpertPlacement.balanced(SKEWED_LOADS, world, slots)
        held = [pl.local_experts(q) for q in range(world)]
        assert all(len(h) <= slots for h in held)
        assert all(len(r) >= 1 for r in pl.replicas)
        # the contiguous placement is kept: every expert stays on its home rank
        assert all(e // (8 // world) in pl.replicas[e] for e in range(8))
        load = pl.load_per_rank(SKEWED_LOADS)
        assert sum(load) == pytest.approx(sum(SKEWED_LOADS))
        if slots == 8 // world:
            assert pl == ep.ExpertPlacement.contiguous(8, world)
        else:  # more slots never make the busiest rank busier, and here they help
            base = max(ep.load_per_rank(SKEWED_LOADS, world))
            assert max(load) < base
    # 8 ranks with two slots each: the busiest rank drops from 42.8% of the rows to <= 21.5%
    pl = ep.ExpertPlacement.balanced(SKEWED_LOADS, 8, 2)
    assert max(pl.load_per_rank(SKEWED_LOADS)) / sum(SKEWED_LOADS) <= 0.215
    assert len(pl.replicas[0]) >= 4


def test_send_order_and_receive_counts():
    from sparse_mixture_experts_18_b200 import ep
    pl = ep.ExpertPlacement(8, 4, ((0, 2, 3), (0, 1), (0, 1), (1,), (2,), (2,), (3,), (3,)))
    counts = [5, 3, 2, 1, 0, 0, 1, 2]
    order, send = pl.send_order(counts)
    assert sorted(order) == list(range(sum(counts)))          # every grouped row once
    assert order == [0, 1, 5, 6, 8, 7, 9, 10, 2, 3, 4, 11, 12, 13] and send == [5, 3, 2, 4]
    assert ep.ExpertPlacement.split(5, 3) == [2, 2, 1] and ep.ExpertPlacement.split(0, 2) == [0, 0]
    all_counts = [counts, [0, 4, 1, 0, 0, 0, 0, 0], [7, 0, 0, 0, 3, 0, 0, 0], [1] * 8]
    for q in range(4):
        seg = pl.recv_counts(all_counts, q)
        # what q receives from s is what s sends to q
        assert [sum(r) for r in seg] == [pl.send_order(all_counts[s])[1][q] for s in range(4)]
    with pytest.raises(ValueError):
        ep.ExpertPlacement(8, 4, ((0,),) * 7)
    with pytest.raises(ValueError):
        ep.ExpertPlacement(8, 4, ((1, 0),) * 8)


def _placed_worker(rank, world, port, Ts, n, slots, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import moe_inputs
    import oracle
    from sparse_mixture_experts_18_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        K, d = 2, 64
        T = Ts[rank]
        w = moe_inputs.small(T=max(T, 1), d=d, F=64, n=n, K=K, dtype="f32", rms_x=False,
                             seed=300 + rank)
        x = moe_inputs.make_x(w)[:T]
        Wg = moe_inputs.make_layer(w.replace(seed=9))["Wg"]
        idx = oracle.route(x, Wg, n, K)[1] if T else np.zeros((0, K), np.int32)
        xg, rows, counts, row_expert = _group_rows(x, idx, n, K)
        all_counts = ep.exchange_all_counts(torch.from_numpy(counts), world).numpy()
        pl = ep.ExpertPlacement.balanced(all_counts.sum(axis=0), world, slots)
        order, send = pl.send_order(all_counts[rank])
        seg = pl.recv_counts(all_counts, rank)
        recv = [sum(r) for r in seg]
        x_send = xg[torch.tensor(order, dtype=torch.long)] if order else xg
        x_recv = ep.dispatch(x_send, send, recv)
        # the expert of every received row: source-major, the rank's experts in order
        local = pl.local_experts(rank)
        got_e = [e for s in range(world) for e, c in zip(local, seg[s]) for _ in range(c)]
        y_recv = _stand_in_expert(x_recv, got_e)
        y_send_back = ep.return_rows(y_recv, send, recv)
        y_back = torch.empty_like(y_send_back)
        if order:
            y_back[torch.tensor(order, dtype=torch.long)] = y_send_back
        back_ok = torch.equal(y_back, _stand_in_expert(xg, row_expert))
        pos_ok = all(torch.equal(y_back[rows[t, k]], x[t] * (1.0 + float(idx[t, k])))
                     for t in range(T) for k in range(K))
        q.put((rank, back_ok, pos_ok, sum(recv), max(pl.load_per_rank(all_counts.sum(axis=0)))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,Ts,n,slots", [(2, (37, 21), 8, 6), (4, (11, 3, 20, 9), 8, 3),
                                              (2, (0, 9), 8, 5)])
def test_replicated_dispatch_and_return_over_gloo(world, Ts, n, slots):
    """Rows of replicated experts reach every replica's rank in their parts and come back to
    their sender's grouped order bit for bit."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_placed_worker, args=(r, world, port, Ts, n, slots, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, back_ok, pos_ok, _, _ in res:
        assert back_ok, rank
        assert pos_ok, rank
    assert sum(r[3] for r in res) == sum(Ts) * 2
