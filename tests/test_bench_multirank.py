"""CPU (gloo, world size 2) test of bench.py's multi-rank host logic: every
rank contributes its own device time, all take the maximum in the same
collective order, and the whole-job value counts the units of every rank."""

import importlib.util
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        local_ms = [12.5, 20.0][rank]          # the second rank is the slow one
        ms = b.max_over_ranks(local_ms, world, torch.device("cpu"), dist)
        units = 1000
        out[rank] = (ms, b.weak_scaling_value(units, world, 4, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms, value = res[rank]
        assert ms == 20.0                      # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 1000 * 4 / 0.020)


def test_single_rank_is_unchanged():
    b = _bench()
    assert b.max_over_ranks(7.0, 1, None, None) == 7.0
    assert b.weak_scaling_value(10, 1, 2, 1000.0) == pytest.approx(20.0)


def test_ranks_draw_disjoint_inputs():
    """Weak scaling: every rank quantizes and decodes its own batch, drawn from
    seeds no other rank uses, so no two ranks repeat each other's work."""
    import numpy as np

    import workloads as W
    b = _bench()
    seeds = [b.rank_seeds(r) for r in range(8)]
    flat = [s[k] for s in seeds for k in ("k", "v", "q")]
    assert len(set(flat)) == len(flat)
    k0 = W.kv_host(1, 2, 16, 64, seed=seeds[0]["k"])
    k1 = W.kv_host(1, 2, 16, 64, seed=seeds[1]["k"])
    assert not np.any(np.all(k0 == k1, axis=1))
