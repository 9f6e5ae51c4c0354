"""Expert parallelism over two ranks as two gloo processes on the CPU.

Each rank routes its own tokens with the oracle, publishes its per-expert slot
counts to every rank (all_gather), sends each kept slot's row to the owner of
its expert at the row the library's dispatch kernel computes (the owner's
earlier experts, then earlier ranks' rows of the same expert, then the slot's
place in the rank's own stable order), runs the owned experts with the oracle,
and sums the returned rows in slot order. The result must equal the oracle
layer on the concatenated batch bit for bit, since no arithmetic changes. The
peer-mapping exchange helper of the binding is driven through the same process
group with stand-in export/open functions."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(world, E, k, d, I, ns):
    rng = np.random.default_rng(7)
    x = [rng.standard_normal((n, d)).astype(np.float32) for n in ns]
    w_r = rng.standard_normal((E, d)).astype(np.float32)
    wg = (rng.standard_normal((E, I, d)) / np.sqrt(d)).astype(np.float32)
    wu = (rng.standard_normal((E, I, d)) / np.sqrt(d)).astype(np.float32)
    wd = (rng.standard_normal((E, d, I)) / np.sqrt(I)).astype(np.float32)
    return x, w_r, wg, wu, wd


def _gather(obj, world):
    out = [None] * world
    dist.all_gather_object(out, obj)
    return out


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from oracle import oracle as O

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        E, k, d, I, ns = 8, 2, 16, 8, [37, 23]
        Eq = E // world
        cfg = O.Cfg(d_model=d, n_routed=E, top_k=k, moe_intermediate_size=I, renormalize=1)
        x, w_r, wg, wu, wd = _inputs(world, E, k, d, I, ns)
        xs = x[rank]
        # 1. route locally, local stable permutation, counts to every rank
        idx, tw, _, _, _ = O.route(cfg, O.router_logits(xs, w_r))
        counts, off, perm, dest = O.dispatch(idx, E)
        T = np.array(_gather(counts, world))  # [world, E]
        col = T.sum(axis=0)

        def base(s, e):  # first row at e's owner of rank s's slots with expert e
            q0 = (e // Eq) * Eq
            return int(col[q0:e].sum() + T[:s, e].sum())

        # 2. rows to their owners (the exchange is an all_gather of (owner, row, data) triples)
        sent = []
        for r in range(len(perm)):
            e = int(np.searchsorted(off, r, side="right") - 1)
            sent.append((e // Eq, base(rank, e) + r - int(off[e]), xs[perm[r]]))
        recv = {}
        for triples in _gather(sent, world):
            for owner, row, data in triples:
                if owner == rank:
                    assert row not in recv
                    recv[row] = data
        # 3. owned experts over the received rows
        own = np.arange(rank * Eq, (rank + 1) * Eq)
        roff = np.concatenate([[0], np.cumsum(col[own])])
        assert sorted(recv) == list(range(int(roff[-1])))
        rx = np.array([recv[i] for i in range(len(recv))], np.float64).reshape(-1, d)
        out = np.zeros_like(rx)
        for i, e in enumerate(own):
            lo, hi = roff[i], roff[i + 1]
            if hi > lo:
                out[lo:hi] = O.swiglu(rx[lo:hi], wg[e], wu[e], wd[e])
        outs = _gather(out, world)
        # 4. combine from the owners' rows, slot order
        eo = np.zeros((len(perm), d))
        for r in range(len(perm)):
            e = int(np.searchsorted(off, r, side="right") - 1)
            eo[r] = outs[e // Eq][base(rank, e) + r - int(off[e])]
        y = O.combine(eo, dest, tw)
        # the binding's peer-mapping exchange, with stand-ins for the CUDA calls
        import top_routing_expert_router_b200 as moe

        peers = moe.ep_open_peers({"recv_x": "rx%d" % rank, "flags": "fl%d" % rank}, rank, world,
                                  lambda o: _gather(o, world), export=lambda t: ("rec", t),
                                  open_=lambda rec: "mapped:" + rec[1])
        q.put((rank, y, peers))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_expert_parallel_layer_equals_the_oracle_layer():
    from oracle import oracle as O

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r, (y, peers)) for r, y, peers in (q.get(timeout=180) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    E, k, d, I, ns = 8, 2, 16, 8, [37, 23]
    x, w_r, wg, wu, wd = _inputs(world, E, k, d, I, ns)
    cfg = O.Cfg(d_model=d, n_routed=E, top_k=k, moe_intermediate_size=I, renormalize=1)
    ref = O.layer(cfg, np.concatenate(x), w_r, wg, wu, wd)["y"]
    np.testing.assert_array_equal(np.concatenate([res[0][0], res[1][0]]), ref)
    assert res[0][1] == {"recv_x": ["rx0", "mapped:rx1"], "flags": ["fl0", "mapped:fl1"]}
    assert res[1][1] == {"recv_x": ["mapped:rx0", "rx1"], "flags": ["mapped:fl0", "fl1"]}
