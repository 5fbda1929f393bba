"""GPU parity of the self-decoder decode step (yoco_swa_decode_step):
the new tokens' K/V projection with the YOCO++ blend, the window decode over
the ring and the ring write, against the oracle's projection -- rounded to
bf16, as the call stores it in the ring -- followed by the oracle's ring push
and window attention, step after step."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.util import assert_close, to_np

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


def _bf16_round(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(BF).double().numpy()


@pytest.mark.parametrize("B,Hq,Hkv,D,W,T,d,steps,ln,base", [
    (4, 32, 8, 128, 1024, 1500, 4096, 2, True, True),   # the benchmark's layer shape: two window chunks a CTA
    (1, 8, 2, 128, 300, 700, 1024, 2, True, False),     # one sequence, short last slice
    (3, 16, 2, 128, 129, 100, 2048, 2, True, True),     # ring not yet full; group 8
    (4, 8, 8, 128, 64, 200, 512, 2, False, True),       # group 1, no LayerNorm
    (2, 4, 2, 128, 16, 40, 1024, 3, True, True),        # window 16
    (2, 8, 2, 128, 2100, 2200, 1024, 2, True, True),    # five 128-slot chunks a CTA on two stages, the last one short
    (2, 8, 4, 64, 100, 150, 1024, 2, True, True),       # head_dim 64
    (5, 8, 2, 128, 100, 150, 1024, 2, True, True),      # five tokens: the other projection kernels, plain window copies
    (2, 8, 2, 128, 100, 150, 320, 2, True, True),       # d_model 320: the other projection kernels
])
def test_swa_decode_step_matches_oracle(cuda_lib, B, Hq, Hkv, D, W, T, d, steps, ln, base):
    seed = 900 + W + d + B
    k0 = wl.normal((B, T, Hkv, D), seed, BF)
    v0 = wl.normal((B, T, Hkv, D), seed + 1, BF)
    rings = [oracle.ring_from_prefill(k0[b], v0[b], W) for b in range(B)]
    rk = torch.stack([torch.from_numpy(r[0]) for r in rings]).to(BF).cuda()
    rv = torch.stack([torch.from_numpy(r[1]) for r in rings]).to(BF).cuda()
    sp = torch.stack([torch.from_numpy(r[2]) for r in rings]).to(torch.int32).cuda()
    w = wl.normal((2 * Hkv * D, d), seed + 2, BF, std=d ** -0.5)
    wg = w.cuda()
    written = [set() for _ in range(B)]
    for s in range(steps):
        p = T + s
        # row mean 3 with the LayerNorm (its fold subtracts the mean); unit rows
        # without it, so that K/V stay unit-scale (the bf16 bar's premise)
        x = (wl.normal((B, d), seed + 10 + s, BF).float() + (3.0 if ln else 0.0)).to(BF)
        q = wl.normal((B, Hq, D), seed + 20 + s, BF)
        kb = wl.normal((B, Hkv, D), seed + 30 + s, BF) if base else None
        vb = wl.normal((B, Hkv, D), seed + 40 + s, BF) if base else None
        ko = torch.empty((B, Hkv, D), dtype=BF, device="cuda")
        vo = torch.empty((B, Hkv, D), dtype=BF, device="cuda")
        pos = torch.full((B,), p, dtype=torch.int64, device="cuda")
        n0 = cuda_lib.launch_count()
        o = cuda_lib.swa_decode_step(x.cuda(), wg, q.cuda(), pos, rk, rv, sp, W,
                                     kb.cuda() if base else None, vb.cuda() if base else None, 0.3, 0.7,
                                     apply_ln=ln, k_out=ko, v_out=vo)
        assert cuda_lib.launch_count() - n0 == 2     # the projection, then the window decode
        rkn, rvn = oracle.kv_project_blend(x, w, Hkv, D, kb, vb, 0.3 if base else 0.0, 0.7 if base else 0.0,
                                           apply_ln=ln)
        assert_close(ko, rkn, BF, f"k_new@{p}")
        assert_close(vo, rvn, BF, f"v_new@{p}")
        kn16, vn16 = _bf16_round(rkn), _bf16_round(rvn)
        got_k, got_v, got_sp = to_np(rk), to_np(rv), sp.cpu().numpy()
        slot = p % W
        for b in range(B):
            oracle.ring_push(rings[b][0], rings[b][1], rings[b][2], p, kn16[b], vn16[b])
            ro, _ = oracle.swa_decode_ring(q[b], rings[b][0], rings[b][1], rings[b][2], p)
            assert_close(o[b], ro, BF, f"o@{p} b{b}")
            np.testing.assert_array_equal(got_sp[b], rings[b][2])
            # the stored K/V of the new token is the one the call reported
            np.testing.assert_array_equal(got_k[b, slot], to_np(ko[b]))
            np.testing.assert_array_equal(got_v[b, slot], to_np(vo[b]))
            # slots this test never wrote are untouched, bit for bit
            written[b].add(slot)
            keep = [j for j in range(W) if j not in written[b]]
            np.testing.assert_array_equal(got_k[b, keep], rings[b][0][keep])
            np.testing.assert_array_equal(got_v[b, keep], rings[b][1][keep])
            for j in written[b]:
                assert_close(got_k[b, j], rings[b][0][j], BF, f"ring k slot {j}")
                assert_close(got_v[b, j], rings[b][1][j], BF, f"ring v slot {j}")


def test_swa_decode_step_outputs_optional(cuda_lib):
    # without k_out / v_out the call still writes the ring and o; the same
    # inputs give the same o and ring as the call that reports them
    B, Hq, Hkv, D, W, T, d = 4, 32, 8, 128, 1024, 1100, 4096
    k0 = wl.normal((B, T, Hkv, D), 950, BF)
    v0 = wl.normal((B, T, Hkv, D), 951, BF)
    rings = [oracle.ring_from_prefill(k0[b], v0[b], W) for b in range(B)]
    mk = lambda i: torch.stack([torch.from_numpy(r[i]) for r in rings])
    rk1, rv1, sp1 = mk(0).to(BF).cuda(), mk(1).to(BF).cuda(), mk(2).to(torch.int32).cuda()
    rk2, rv2, sp2 = rk1.clone(), rv1.clone(), sp1.clone()
    x = wl.normal((B, d), 952, BF).cuda()
    w = wl.normal((2 * Hkv * D, d), 953, BF, std=d ** -0.5).cuda()
    q = wl.normal((B, Hq, D), 954, BF).cuda()
    pos = torch.full((B,), T, dtype=torch.int64, device="cuda")
    ko = torch.empty((B, Hkv, D), dtype=BF, device="cuda")
    vo = torch.empty((B, Hkv, D), dtype=BF, device="cuda")
    o1 = cuda_lib.swa_decode_step(x, w, q, pos, rk1, rv1, sp1, W, k_out=ko, v_out=vo)
    o2 = cuda_lib.swa_decode_step(x, w, q, pos, rk2, rv2, sp2, W)
    assert torch.equal(o1, o2)
    assert torch.equal(rk1, rk2) and torch.equal(rv1, rv2) and torch.equal(sp1, sp2)
    assert cuda_lib.device_status() == 0
