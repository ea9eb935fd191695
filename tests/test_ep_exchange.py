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
