"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times, on sampled outputs the oracle computes row by row:

  cross prefill  T=32768, 32q/8kv heads, head_dim 128 (one shared K/V, two
                 layers with their own Q), plus a needle variant whose outputs
                 are of unit scale;
  cross decode   batch 16, ragged lengths in [65536, 131072], every sequence
                 and head;
  SWA            B=4, T=65536, window 1024: blended K/V projection (d=4096),
                 prefill rows around window and tile edges, the ring, and
                 decode steps past the prompt;
  long context   1M tokens: the last 32K-query chunk of the causal prefill and
                 a decode step over the full 1M cache.

Inputs are drawn on the device by the seeded generators (the same bits are
copied to the host for the oracle)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.util import assert_close, to_np

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _rows(T, extra, seed, n=24):
    return wl.sample_rows(T, n, seed, extra)


def _check_rows(o_gpu, q, k, v, rows, q_pos0=0, window=0, what=""):
    ro, _ = oracle.attention(q, k, v, q_pos0, window, rows=[(0, r) for r in rows])
    got = torch.stack([o_gpu[0, r] for r in rows])
    return assert_close(got, ro, BF, what)


def test_cross_prefill_32k_sampled(cuda_lib):
    T, Hq, Hkv, D = 32768, 32, 8, 128
    k = wl.normal((1, T, Hkv, D), 1300, BF, "cuda")
    v = wl.normal((1, T, Hkv, D), 1301, BF, "cuda")
    kh, vh = k.cpu(), v.cpu()
    for layer in range(2):
        q = wl.normal((1, T, Hq, D), 1200 + layer, BF, "cuda")
        o = cuda_lib.cross_prefill(q, k, v)
        rows = _rows(T, [127, 128, 1024, 16383, 16384], 50 + layer)
        _check_rows(o, q.cpu(), kh, vh, rows, what=f"layer {layer}")


def test_cross_prefill_32k_needle(cuda_lib):
    # plant, for a set of query rows, one earlier key aligned with the query so
    # the softmax is peaked and the output is a unit-scale value row
    T, Hq, Hkv, D = 32768, 32, 8, 128
    G = Hq // Hkv
    q = wl.normal((1, T, Hq, D), 1400, BF, "cuda")
    k = wl.normal((1, T, Hkv, D), 1401, BF, "cuda")
    v = wl.normal((1, T, Hkv, D), 1402, BF, "cuda")
    rows = _rows(T, [128, 4096, 32767], 60)
    for n, r in enumerate(rows):
        j = (r * 7 + n) % (r + 1)
        k[0, j] = (q[0, r].view(Hkv, G, D)[:, 0] * 1.5).to(BF)
    o = cuda_lib.cross_prefill(q, k, v)
    ro, _ = oracle.attention(q.cpu(), k.cpu(), v.cpu(), 0, 0, rows=[(0, r) for r in rows])
    got = torch.stack([o[0, r] for r in rows])
    assert float(np.abs(ro).max()) > 0.5      # outputs are unit scale, not ~1/sqrt(n)
    assert_close(got, ro, BF, "needle")


def test_cross_decode_128k_ragged(cuda_lib):
    B, Hq, Hkv, D = 16, 32, 8, 128
    lens = wl.ragged_lengths(B, 65536, 131072, 2000)
    starts = torch.cumsum(torch.cat([torch.zeros(1, dtype=torch.int64), lens[:-1]]), 0)
    rows = int(lens.sum())
    kc = wl.normal((rows, Hkv, D), 2001, BF, "cuda")
    vc = wl.normal((rows, Hkv, D), 2002, BF, "cuda")
    q = wl.normal((B, Hq, D), 2100, BF, "cuda")
    o, lse = cuda_lib.cross_decode(q, kc, vc, starts.cuda(), lens.to(torch.int32).cuda(),
                                   int(lens.max()), want_lse=True)
    ro, rlse = oracle.cross_decode(q.cpu(), kc.cpu(), vc.cpu(), starts.numpy(), lens.numpy())
    assert_close(o, ro, BF, "o")
    assert_close(lse, rlse, BF, "lse", max_abs=1e-3, rel_l2=1e-4)


def test_swa_64k_blend_prefill_ring_decode(cuda_lib):
    B, T, W, Hq, Hkv, D, d = 4, 65536, 1024, 32, 8, 128, 4096
    n = B * T
    x = wl.normal((n, d), 3001, BF, "cuda")
    w = wl.normal((2 * Hkv * D, d), 3002, BF, "cuda", std=d ** -0.5)
    k1 = wl.normal((n, Hkv, D), 3003, BF, "cuda")
    v1 = wl.normal((n, Hkv, D), 3004, BF, "cuda")
    wl_ = float(wl.uniform((1,), 3005)[0])
    k, v = cuda_lib.kv_project_blend(x, w, Hkv, D, k1, v1, wl_, wl_)
    # projection + blend on sampled token rows
    tok = sorted(set(wl.sample_rows(n, 24, 70, [T - 1, T, 2 * T])))
    rk, rv = oracle.kv_project_blend(x[tok].cpu(), w.cpu(), Hkv, D, k1[tok].cpu(), v1[tok].cpu(), wl_, wl_)
    assert_close(k[tok], rk, BF, "k blend")
    assert_close(v[tok], rv, BF, "v blend")
    # SWA prefill over the projected K/V (oracle reads the same K/V bits)
    q = wl.normal((B, T, Hq, D), 3006, BF, "cuda")
    k4, v4 = k.view(B, T, Hkv, D), v.view(B, T, Hkv, D)
    ring = (torch.empty((B, W, Hkv, D), dtype=BF, device="cuda"),
            torch.empty((B, W, Hkv, D), dtype=BF, device="cuda"),
            torch.empty((B, W), dtype=torch.int32, device="cuda"))
    o = cuda_lib.swa_prefill(q, k4, v4, W, ring=ring)
    rows = _rows(T, [W - 1, W, 2 * W, 127, 128, T - 128], 71, n=12)
    for b in (0, 3):
        ro, _ = oracle.attention(q[b:b + 1].cpu(), k4[b:b + 1].cpu(), v4[b:b + 1].cpu(), 0, W,
                                 rows=[(0, r) for r in rows])
        assert_close(torch.stack([o[b, r] for r in rows]), ro, BF, f"swa b{b}")
    sp_ref = oracle.ring_prefill_slots(T, W)
    for b in range(B):
        np.testing.assert_array_equal(ring[2][b].cpu().numpy(), sp_ref)
    # ring contents are the last W rows in slot order (bit-exact copies)
    slots = torch.from_numpy(sp_ref.astype(np.int64)).cuda()
    assert torch.equal(ring[0], k4[:, slots]) and torch.equal(ring[1], v4[:, slots])
    # decode steps past the prompt, each checked against window attention
    kh, vh = k4.cpu(), v4.cpu()
    for step in range(3):
        p = T + step
        qd = wl.normal((B, Hq, D), 3100 + step, BF, "cuda")
        kn = wl.normal((B, Hkv, D), 3200 + step, BF, "cuda")
        vn = wl.normal((B, Hkv, D), 3300 + step, BF, "cuda")
        pos = torch.full((B,), p, dtype=torch.int64, device="cuda")
        od = cuda_lib.swa_decode(qd, kn, vn, pos, ring[0], ring[1], ring[2], W)
        kh = torch.cat([kh, kn.cpu()[:, None]], 1)
        vh = torch.cat([vh, vn.cpu()[:, None]], 1)
        for b in (0, 2):
            lo = p - W + 1
            ro, _ = oracle.attention(qd[b].cpu()[None, None], kh[b:b + 1, lo:p + 1],
                                     vh[b:b + 1, lo:p + 1], W - 1, W)
            assert_close(od[b], ro[0, 0], BF, f"swa decode step {step} b{b}")


def test_long_context_1m(cuda_lib):
    T, C, Hq, Hkv, D = 1 << 20, 32768, 32, 8, 128
    k = wl.normal((1, T, Hkv, D), 5001, BF, "cuda")
    v = wl.normal((1, T, Hkv, D), 5002, BF, "cuda")
    q0 = T - C
    q = wl.normal((1, C, Hq, D), 5003, BF, "cuda")
    o = cuda_lib.cross_prefill(q, k, v, q_pos0=q0)
    rows = _rows(C, [0, 1, 127, 128, C - 1], 80, n=8)
    kh, vh = k.cpu(), v.cpu()
    _check_rows(o, q.cpu(), kh, vh, rows, q_pos0=q0, what="1M last chunk")
    # decode at full context over the 1M cache (+1 appended row)
    qd = wl.normal((1, Hq, D), 5004, BF, "cuda")
    ss = torch.zeros(1, dtype=torch.int64, device="cuda")
    sl = torch.tensor([T], dtype=torch.int32, device="cuda")
    od = cuda_lib.cross_decode(qd, k[0], v[0], ss, sl, T)
    ro, _ = oracle.cross_decode(qd.cpu(), kh[0], vh[0], [0], [T])
    assert_close(od, ro, BF, "1M decode")
