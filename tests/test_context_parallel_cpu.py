"""Context-parallel prefill plumbing on CPU: zig-zag chunk ownership, and the one
exchange step (the all-gather of the key side) over two gloo ranks on 127.0.0.1.

The per-chunk work each rank is left with is checked against the oracle run on
the whole sequence: a query chunk at offset c*chunk over the gathered key prefix
gives the same rows as the whole problem (query rows only read keys 0..t)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from sparse_attention_19_b200 import context_parallel as cp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,rounds", [(1, 1), (2, 1), (2, 3), (4, 2), (8, 1)])
def test_zigzag_owns_every_chunk_once_with_equal_causal_work(world, rounds):
    n = 2 * world * rounds
    owned = [cp.zigzag_chunks(n, world, r) for r in range(world)]
    assert sorted(c for o in owned for c in o) == list(range(n))
    work = {cp.causal_pairs_of(o, 512) for o in owned}
    assert len(work) == 1                                   # exactly balanced
    assert work.pop() * world == cp.causal_pairs_of(range(n), 512)


def test_zigzag_rejects_uneven_splits():
    with pytest.raises(ValueError):
        cp.zigzag_chunks(6, 2, 0)
    with pytest.raises(ValueError):
        cp.zigzag_chunks(8, 2, 2)


def _key_side(L, seed=0):
    from dsa_inputs import WORKLOADS, make_key_side
    wl = WORKLOADS["tiny"].with_(Lq=L, Lk=L)
    return make_key_side(wl, "cpu", seed), wl


def _rank_main(rank, world, port, n_chunks, chunk, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from dsa_inputs import make_query_side
        full, wl = _key_side(n_chunks * chunk)
        mine = cp.zigzag_chunks(n_chunks, world, rank)
        local = cp.local_key_side(full, mine, chunk)
        keys = cp.gather_key_side(local, n_chunks, chunk, world, rank)
        same = all(torch.equal(keys[f], full[f]) for f in cp.KEY_FIELDS)
        # this rank's share of the work: its query chunks over the gathered key prefix
        qs = make_query_side(wl, "cpu", 0)
        got = {}
        for c in mine:
            rows = np.arange(c * chunk, (c + 1) * chunk)
            Lk = (c + 1) * chunk
            r = oracle.rows_from_inputs(qs, rows, wl.Lq, 0)
            kd = oracle.keys_from_inputs({f: keys[f][:, :Lk] for f in cp.KEY_FIELDS})
            res = oracle.dsa_forward(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], kd["k_I"],
                                     kd["k_scale"], r["q"], kd["kv"], wl.k, wl.scale, wl.Dv)
            got[c] = (res["indices"], res["out"])
        q.put((rank, same, got))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_the_key_side_and_split_the_work():
    world, n_chunks, chunk = 2, 4, 64
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, n_chunks, chunk, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=600) for _ in range(world)]
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert all(same for _, same, _ in res), "gathered key side differs from the whole sequence"
    per_chunk = {}
    for _, _, got in res:
        per_chunk.update(got)
    assert sorted(per_chunk) == list(range(n_chunks))
    # the whole sequence in one oracle call
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from dsa_inputs import make_query_side
    full, wl = _key_side(n_chunks * chunk)
    qs = make_query_side(wl, "cpu", 0)
    rows = np.arange(n_chunks * chunk)
    r = oracle.rows_from_inputs(qs, rows, wl.Lq, 0)
    kd = oracle.keys_from_inputs(full)
    whole = oracle.dsa_forward(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], kd["k_I"], kd["k_scale"],
                               r["q"], kd["kv"], wl.k, wl.scale, wl.Dv)
    for c in range(n_chunks):
        sl = slice(c * chunk, (c + 1) * chunk)
        assert np.array_equal(per_chunk[c][0], whole["indices"][sl])
        assert np.array_equal(per_chunk[c][1], whole["out"][sl])


def _gather_only(rank, world, port, n_chunks, chunk, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        full, _ = _key_side(n_chunks * chunk, seed=7)
        local = cp.local_key_side(full, cp.zigzag_chunks(n_chunks, world, rank), chunk)
        keys = cp.gather_key_side(local, n_chunks, chunk, world, rank)
        q.put((rank, all(torch.equal(keys[f], full[f]) for f in cp.KEY_FIELDS)))
    finally:
        dist.destroy_process_group()


def test_four_gloo_ranks_two_rounds_gather_the_whole_sequence():
    world, n_chunks, chunk = 4, 16, 16
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_only, args=(r, world, port, n_chunks, chunk, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert res == {r: True for r in range(world)}
