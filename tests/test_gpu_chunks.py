"""The GPU side of chunk-parallel prefill: yoco_attention_prefill on one
rank's chunk -- the sliding-window chunk over [halo | chunk] keys, and the
cross-decoder chunk over the gathered global K/V -- equals the same rows of
the unchunked attention (oracle and GPU).  The rank exchanges themselves are
tested over gloo on the CPU (tests/test_chunk_parallel.py); here a stand-in
for them hands each chunk the halo and the gathered K/V of one process."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from shared_kv_decoder_b200 import chunk_parallel as cp
from tests.util import assert_close

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


class SliceComm:
    """The exchanges of virtual rank r, served from the whole sequence."""

    def __init__(self, rank, k_full, v_full, Tc):
        self.rank, self.k, self.v, self.Tc = rank, k_full, v_full, Tc

    def halo(self, k_tail, v_tail):
        if self.rank == 0:
            return None, None
        h = k_tail.shape[1]
        s = self.rank * self.Tc
        return self.k[:, s - h:s], self.v[:, s - h:s]


@pytest.mark.parametrize("B,world,Tc,Hq,Hkv,D,W", [(1, 4, 384, 8, 2, 128, 200), (2, 3, 256, 4, 4, 64, 129),
                                                    (1, 2, 500, 32, 8, 128, 1)])
def test_chunked_swa_and_cross_match_unchunked(cuda_lib, B, world, Tc, Hq, Hkv, D, W):
    T = world * Tc
    q = wl.normal((B, T, Hq, D), 3200, BF)
    k = wl.normal((B, T, Hkv, D), 3201, BF)
    v = wl.normal((B, T, Hkv, D), 3202, BF)
    qc = wl.normal((B, T, Hq, D), 3203, BF)
    ref_swa, _ = oracle.attention(q, k, v, 0, W)
    ref_cross, _ = oracle.attention(qc, k, v, 0, 0)
    kd, vd = k.cuda(), v.cuda()
    full_swa = cuda_lib.swa_prefill(q.cuda(), kd, vd, W)
    for r in range(world):
        s = slice(r * Tc, (r + 1) * Tc)
        comm = SliceComm(r, kd, vd, Tc)
        o = cp.swa_chunk(q[:, s].cuda(), kd[:, s], vd[:, s], W, comm)
        assert_close(o, ref_swa[:, s], BF, f"swa chunk {r}")
        assert_close(o, full_swa[:, s].float().cpu().numpy(), BF, f"swa chunk {r} vs unchunked GPU")
        oc = cp.cross_chunk(qc[:, s].cuda(), kd, vd, r * Tc)
        assert_close(oc, ref_cross[:, s], BF, f"cross chunk {r}")


def test_attention_prefill_window_with_offset(cuda_lib):
    # a window over a key buffer that starts before the queries, ragged sizes
    B, Tq, Tkv, Hq, Hkv, D, q0, W = 1, 333, 700, 8, 2, 128, 367, 150
    q = wl.normal((B, Tq, Hq, D), 3300, BF)
    k = wl.normal((B, Tkv, Hkv, D), 3301, BF)
    v = wl.normal((B, Tkv, Hkv, D), 3302, BF)
    o, lse = cuda_lib.attention_prefill(q.cuda(), k.cuda(), v.cuda(), q_pos0=q0, window=W, want_lse=True)
    ro, rlse = oracle.attention(q, k, v, q0, W)
    assert_close(o, ro, BF, "o")
    assert_close(lse, rlse.transpose(0, 2, 1), BF, "lse", max_abs=1e-3, rel_l2=1e-4)
