"""Chunk-parallel prefill across ranks, on CPU: world sizes 2 and 3 over gloo.
Each rank holds one chunk of the prompt, exchanges the sliding-window halo
with its neighbour, gathers the global K/V once and runs its cross-decoder
rows; the attention calls are the oracle's (the GPU kernels' chunk semantics
are checked by tests/test_gpu_chunks.py).  Every rank's rows must equal the
oracle's unchunked run."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleOps:
    @staticmethod
    def attention_prefill(q, k, v, q_pos0, window):
        import oracle
        o, _ = oracle.attention(q, k, v, q_pos0, window)
        return torch.from_numpy(o)


def _rank(rank, world, port, q_out, B, Tc, Hq, Hkv, D, W):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import workloads as wl
    from shared_kv_decoder_b200 import chunk_parallel as cp
    T = world * Tc
    q = wl.normal((B, T, Hq, D), 3100, torch.float64)
    k = wl.normal((B, T, Hkv, D), 3101, torch.float64)
    v = wl.normal((B, T, Hkv, D), 3102, torch.float64)
    qc = wl.normal((B, T, Hq, D), 3103, torch.float64)
    s0 = rank * Tc
    comm = cp.DistComm()
    o_swa = cp.swa_chunk(q[:, s0:s0 + Tc], k[:, s0:s0 + Tc], v[:, s0:s0 + Tc], W, comm, OracleOps)
    kg, vg = cp.gather_global_kv(k[:, s0:s0 + Tc].contiguous(), v[:, s0:s0 + Tc].contiguous(), comm)
    o_cross = cp.cross_chunk(qc[:, s0:s0 + Tc], kg, vg, s0, OracleOps)
    q_out.put((rank, o_swa.numpy(), o_cross.numpy(), bool(torch.equal(kg, k)) and bool(torch.equal(vg, v))))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,B,Tc,W", [(2, 1, 40, 9), (3, 2, 24, 25), (2, 1, 16, 1), (3, 1, 20, 7)])
def test_chunked_prefill_equals_unchunked(world, B, Tc, W):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    import workloads as wl
    Hq, Hkv, D = 4, 2, 16
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q_out, B, Tc, Hq, Hkv, D, W)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, (a, b, c)) for r, a, b, c in (q_out.get(timeout=120) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    T = world * Tc
    q = wl.normal((B, T, Hq, D), 3100, torch.float64)
    k = wl.normal((B, T, Hkv, D), 3101, torch.float64)
    v = wl.normal((B, T, Hkv, D), 3102, torch.float64)
    qc = wl.normal((B, T, Hq, D), 3103, torch.float64)
    ref_swa, _ = oracle.attention(q, k, v, 0, W)
    ref_cross, _ = oracle.attention(qc, k, v, 0, 0)
    for r in range(world):
        o_swa, o_cross, gathered_ok = got[r]
        assert gathered_ok, f"rank {r}: gathered global K/V differs from the sequence's"
        np.testing.assert_allclose(o_swa, ref_swa[:, r * Tc:(r + 1) * Tc], rtol=0, atol=1e-12)
        np.testing.assert_allclose(o_cross, ref_cross[:, r * Tc:(r + 1) * Tc], rtol=0, atol=1e-12)


def test_window_past_previous_chunk_is_rejected():
    import sys
    sys.path.insert(0, ROOT)
    from shared_kv_decoder_b200 import chunk_parallel as cp
    z = torch.zeros((1, 8, 2, 16), dtype=torch.float64)
    with pytest.raises(ValueError):
        cp.swa_chunk(z, z, z, 10, comm=None, ops=OracleOps)
