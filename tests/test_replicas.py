"""Replica plumbing of bench.py on CPU: two gloo ranks (no GPU, no collective on the data path)."""
import importlib.util
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    bench = _load_bench()
    from nvfp4_weight_only_route_b200 import synth
    r, w, local, pg = bench.dist_setup(world, backend="gloo")
    try:
        bench.barrier(pg, torch, cuda=False)
        # each rank "measures" a different time; everyone must see the slowest
        ms = bench.max_over_ranks(pg, torch, 10.0 + 5.0 * r, device="cpu")
        shape = synth.custom_shape(H=128, I=64, E=4, k=2)
        digest = synth.layer_digest(synth.make_layer(shape, bench.replica_seed(3, r)))
        q.put((r, w, ms, digest, bench.weak_value(w, 8, 100, ms)))
    finally:
        pg.destroy_process_group()


def test_two_gloo_replicas():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[2] == pytest.approx(15.0) for r in res)            # max over ranks
    assert res[0][3] != res[1][3]                                   # replicas hold different layers
    assert res[0][4] == pytest.approx(2 * 8 * 100 / 0.015)          # weak-scaling tokens/s


def test_single_process_needs_no_group():
    import torch
    bench = _load_bench()
    r, w, local, pg = bench.dist_setup(1)
    assert (r, w, pg) == (0, 1, None)
    assert bench.max_over_ranks(pg, torch, 3.5) == 3.5
    assert bench.replica_seed(5, 0) == 5
