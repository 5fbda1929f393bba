"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times, on sampled outputs the oracle computes row by row:

  cross prefill  T=32768, 32q/8kv heads, head_dim 128 (one shared K/V, two
                 layers with their own Q), plus a needle variant whose outputs
                 are of unit scale;
  cross decode   batch 16, ragged lengths in [65536, 131072], every sequence
                 and head, with needles in six sequences (first row, middle,
                 last rows of a partial pipeline stage);
  SWA            B=4, T=65536, window 1024: blended K/V projection (d=4096),
                 prefill rows around window and tile edges, the ring, and
                 decode steps past the prompt; then window-edge sentinels for
                 the prefill and the ring decode (values of 1e4 at the first
                 position outside the window on each side, a needle at the
                 oldest position inside);
  long context   1M tokens: the last 32K-query chunk of the causal prefill and
                 a decode step over the full 1M cache, each with needles
                 (earliest keys, the chunk boundary, the last rows).

With random N(0,1) keys the softmax over 64K-1M keys is nearly flat and the
outputs are ~1/sqrt(n), so the max-abs bound alone would be vacuous there:
rel-L2 binds on those rows, and the needle rows (one planted key aligned with
the query, so one weight dominates) have unit-scale outputs on which both
bounds bind.  A sentinel of 1e4 leaked with weight ~1/window would move an
output by ~10.

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
    G = Hq // Hkv
    lens = wl.ragged_lengths(B, 65536, 131072, 2000)
    starts = torch.cumsum(torch.cat([torch.zeros(1, dtype=torch.int64), lens[:-1]]), 0)
    rows = int(lens.sum())
    kc = wl.normal((rows, Hkv, D), 2001, BF, "cuda")
    vc = wl.normal((rows, Hkv, D), 2002, BF, "cuda")
    q = wl.normal((B, Hq, D), 2100, BF, "cuda")
    # needles: in six sequences one key row aligned with the first query head
    # of every KV group -- the first row, a middle row, and the last rows of
    # sequences whose final 16-token pipeline stage is partial
    L = lens.tolist()
    partial = [b for b in range(B) if L[b] % 16 != 0]
    plant = {0: 0, 5: L[5] // 2, 9: 1}
    for b in partial[-3:]:
        plant[b] = L[b] - 1 - (b % 3)
    for b, off in plant.items():
        kc[int(starts[b]) + off] = (q[b].view(Hkv, G, D)[:, 0] * 1.5).to(BF)
    o, lse = cuda_lib.cross_decode(q, kc, vc, starts.cuda(), lens.to(torch.int32).cuda(),
                                   int(lens.max()), want_lse=True)
    ro, rlse = oracle.cross_decode(q.cpu(), kc.cpu(), vc.cpu(), starts.numpy(), lens.numpy())
    for b in range(B):
        assert_close(o[b], ro[b], BF, f"sequence {b}")
        if b in plant:
            assert float(np.abs(ro[b]).max()) > 0.5       # the needle dominates: unit-scale output
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


def test_swa_64k_window_edges(cuda_lib):
    # Prefill at the sliding-window workload's shape.  For sampled rows p
    # (2W+ apart, at several offsets inside their 128-row tile, so no row sees
    # another's plants): V at p - W (just below the window) and at p + 1 (the
    # next position) is 1e4, and K at p - W + 1 (the oldest key inside) is a
    # needle aligned with the first query head of every KV group.  The needle
    # heads' outputs are that V row (unit scale: a window one key too narrow
    # loses it); the other heads' softmax is flat over the window, so a
    # sentinel leaked with weight ~1/W would add ~10.
    B, T, W, Hq, Hkv, D = 4, 65536, 1024, 32, 8, 128
    G = Hq // Hkv
    q = wl.normal((B, T, Hq, D), 3500, BF, "cuda")
    k = wl.normal((B, T, Hkv, D), 3501, BF, "cuda")
    v = wl.normal((B, T, Hkv, D), 3502, BF, "cuda")
    rows = [W, 3 * W + 1, 5 * W + 63, 8 * W + 127, 11 * W + 64, 20 * W + 5, 30 * W + 100, 45 * W + 17,
            60 * W + 2, T - 1]
    for p in rows:
        for b in range(B):
            v[b, p - W] = 1e4
            if p + 1 < T:
                v[b, p + 1] = 1e4
            k[b, p - W + 1] = (q[b, p].view(Hkv, G, D)[:, 0] * 1.5).to(BF)
    o = cuda_lib.swa_prefill(q, k, v, W)
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    for b in range(B):
        ro, _ = oracle.attention(qh[b:b + 1], kh[b:b + 1], vh[b:b + 1], 0, W, rows=[(0, p) for p in rows])
        got = torch.stack([o[b, p] for p in rows])
        assert_close(got, ro, BF, f"window edges b{b}")
        assert float(np.abs(ro[:, 0::G]).max()) > 0.5         # needle heads: unit scale
        assert float(np.abs(ro).max()) < 50.0                  # no sentinel reached a checked row

    # Ring decode after the prefill: the ring holds positions T - W .. T - 1,
    # and the step at p = T writes slot T mod W.  Plant, in other slots, a
    # stored position p - W (just outside) and p + 1 (ahead of the query), both
    # with V = 1e4, and a needle in the slot of p - W + 1 (the oldest inside).
    ring = (torch.empty((B, W, Hkv, D), dtype=BF, device="cuda"),
            torch.empty((B, W, Hkv, D), dtype=BF, device="cuda"),
            torch.empty((B, W), dtype=torch.int32, device="cuda"))
    cuda_lib.swa_prefill(q, k, v, W, ring=ring)
    p = T
    qd = wl.normal((B, Hq, D), 3510, BF, "cuda")
    kn = wl.normal((B, Hkv, D), 3511, BF, "cuda")
    vn = wl.normal((B, Hkv, D), 3512, BF, "cuda")
    s_out, s_ahead, s_in = 5, 9, (p - W + 1) % W
    ring[2][:, s_out] = p - W
    ring[1][:, s_out] = 1e4
    ring[2][:, s_ahead] = p + 1
    ring[1][:, s_ahead] = 1e4
    for b in range(B):
        assert int(ring[2][b, s_in]) == p - W + 1
        ring[0][b, s_in] = (qd[b].view(Hkv, G, D)[:, 0] * 1.5).to(BF)
    host = [t.cpu() for t in ring]
    pos = torch.full((B,), p, dtype=torch.int64, device="cuda")
    od = cuda_lib.swa_decode(qd, kn, vn, pos, ring[0], ring[1], ring[2], W)
    for b in range(B):
        rk, rv = host[0][b].double().numpy().copy(), host[1][b].double().numpy().copy()
        sp = host[2][b].numpy().copy()
        oracle.ring_push(rk, rv, sp, p, kn[b].cpu(), vn[b].cpu())
        np.testing.assert_array_equal(ring[2][b].cpu().numpy(), sp)       # slot positions bit-exact
        ro, _ = oracle.swa_decode_ring(qd[b].cpu(), rk, rv, sp, p)
        assert_close(od[b], ro, BF, f"ring decode edges b{b}")
        assert float(np.abs(ro[0::G]).max()) > 0.5
        assert float(np.abs(ro).max()) < 50.0


def test_long_context_1m(cuda_lib):
    T, C, Hq, Hkv, D = 1 << 20, 32768, 32, 8, 128
    G = Hq // Hkv
    k = wl.normal((1, T, Hkv, D), 5001, BF, "cuda")
    v = wl.normal((1, T, Hkv, D), 5002, BF, "cuda")
    q0 = T - C
    q = wl.normal((1, C, Hq, D), 5003, BF, "cuda")
    rows = _rows(C, [0, 1, 127, 128, C - 1], 80, n=8)
    # needles for every other sampled row: the earliest keys, a key far back,
    # the last key before the chunk, and the row's own position
    needle_rows = rows[::2]
    for n, r in enumerate(needle_rows):
        j = [3, 70000, q0 - 1, q0 + r][n % 4]
        k[0, j] = (q[0, r].view(Hkv, G, D)[:, 0] * 1.5).to(BF)
    plain_rows = [r for r in rows if r not in needle_rows]
    o = cuda_lib.cross_prefill(q, k, v, q_pos0=q0)
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    _check_rows(o, qh, kh, vh, plain_rows, q_pos0=q0, what="1M last chunk")
    ro, _ = oracle.attention(qh, kh, vh, q0, 0, rows=[(0, r) for r in needle_rows])
    assert float(np.abs(ro[:, 0::G]).max()) > 0.5
    assert_close(torch.stack([o[0, r] for r in needle_rows]), ro, BF, "1M last chunk needles")
    # decode at full context over the 1M cache: every KV head gets its own
    # needle position, from the first row to the last stage
    qd = wl.normal((1, Hq, D), 5004, BF, "cuda")
    for g, j in enumerate([0, 1, 1000, T // 2, T - C, T - 40, T - 17, T - 1]):
        k[0, j, g] = (qd[0, g * G] * 1.5).to(BF)
    kh = k.cpu()
    ss = torch.zeros(1, dtype=torch.int64, device="cuda")
    sl = torch.tensor([T], dtype=torch.int32, device="cuda")
    od = cuda_lib.cross_decode(qd, k[0], v[0], ss, sl, T)
    ro, _ = oracle.cross_decode(qd.cpu(), kh[0], vh[0], [0], [T])
    needle_heads = list(range(0, Hq, G))
    other_heads = [h for h in range(Hq) if h % G]
    assert float(np.abs(ro[0, needle_heads]).max(axis=-1).min()) > 0.5   # every needle found
    assert_close(od[0, needle_heads], ro[0, needle_heads], BF, "1M decode, needle heads")
    assert_close(od[0, other_heads], ro[0, other_heads], BF, "1M decode, other heads")
