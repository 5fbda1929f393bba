"""The benchmark's multi-rank path on CPU: world size 2 over gloo.  Each rank
runs an independent replica (the attention core is not sharded), so the job
time is the max over ranks of each rank's device time."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    local = [10.0 + rank, 5.0 - rank, 7.5 * (rank + 1)]
    q.put((rank, bench.reduce_max_over_ranks(local)))
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got[0] == got[1] == [11.0, 5.0, 15.0]


def test_reduce_max_without_process_group_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_over_ranks([1.5, 2.0]) == [1.5, 2.0]


class _OracleOps:
    """The attention of the chunk-parallel mode on the CPU: the oracle."""
    @staticmethod
    def attention_prefill(q, k, v, q_pos0, window):
        import oracle
        import torch
        o, _ = oracle.attention(q, k, v, q_pos0, window)
        return torch.from_numpy(o)


def _cp_rank(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    import oracle
    import workloads as wl
    from shared_kv_decoder_b200 import chunk_parallel as cp
    shape = dict(Tc=48, Hq=4, Hkv=2, D=64, W=20, self_layers=2, cross_layers=2)
    rep, (o_s, o_c) = bench.chunk_parallel_measure(cp.DistComm(), _OracleOps, torch.device("cpu"),
                                                   torch.float64, 1, 1, **shape)
    # this rank's rows of the last layers equal the unchunked oracle's
    Tc, Hq, Hkv, D, W = (shape[k] for k in ("Tc", "Hq", "Hkv", "D", "W"))
    T, s0, L = world * Tc, rank * Tc, shape["self_layers"] - 1
    full = lambda seeds, H: torch.cat([wl.normal((1, Tc, H, D), s + r, torch.float64)
                                       for r, s in zip(range(world), seeds)], dim=1)
    q_ = full([6000 + 100 * L] * world, Hq)
    k_ = full([6010 + 100 * L] * world, Hkv)
    v_ = full([6020 + 100 * L] * world, Hkv)
    o_ref, _ = oracle.attention(q_, k_, v_, 0, W)
    Lc = shape["cross_layers"] - 1
    qc = full([6050 + 100 * Lc] * world, Hq)
    kg, vg = full([6030] * world, Hkv), full([6040] * world, Hkv)
    oc_ref, _ = oracle.attention(qc, kg, vg, 0, 0)
    ok = (np.allclose(o_s.numpy(), o_ref[:, s0:s0 + Tc], atol=1e-12) and
          np.allclose(o_c.numpy(), oc_ref[:, s0:s0 + Tc], atol=1e-12))
    q.put((rank, rep, ok))
    dist.barrier()
    dist.destroy_process_group()


def test_chunk_parallel_bench_mode_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = dict((r, (rep, ok)) for r, rep, ok in (q.get(timeout=5) for _ in range(2)))
    for r in range(2):
        rep, ok = got[r]
        assert ok, f"rank {r}: outputs differ from the unchunked oracle"
        assert rep["rank"] == r and rep["ms_step"] > 0 and rep["ms_gather"] >= 0
    # rank 1's cross rows attend to twice the keys of rank 0's on average
    assert got[1][0]["flops_cross"] > 2.5 * got[0][0]["flops_cross"]
