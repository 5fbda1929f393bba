"""GPU parity: every C-ABI call against the CPU fp64 oracle on the same
seeded inputs, element by element, at sizes that span several tiles and a
ragged tail; integer / index / ring outputs bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.util import assert_close, to_np

pytestmark = pytest.mark.gpu

BF, F32 = torch.bfloat16, torch.float32


def _qkv(B, Tq, Tkv, Hq, Hkv, D, dtype, seed):
    q = wl.normal((B, Tq, Hq, D), seed, dtype)
    k = wl.normal((B, Tkv, Hkv, D), seed + 1, dtype)
    v = wl.normal((B, Tkv, Hkv, D), seed + 2, dtype)
    return q, k, v


# ------------------------------------------------------------ cross prefill
@pytest.mark.parametrize("dtype", [BF, F32])
@pytest.mark.parametrize("B,Tq,Tkv,Hq,Hkv,D,q_pos0", [
    (1, 300, 300, 4, 2, 64, 0),
    (2, 257, 257, 8, 2, 128, 0),
    (1, 129, 400, 8, 1, 128, 271),   # chunk at the end of a longer KV
    (1, 64, 64, 8, 8, 128, 0),
    (1, 1, 1, 2, 1, 64, 0),          # single row: output = v_0
    (3, 130, 130, 16, 2, 128, 0),    # group 8
])
def test_cross_prefill_matches_oracle(cuda_lib, dtype, B, Tq, Tkv, Hq, Hkv, D, q_pos0):
    q, k, v = _qkv(B, Tq, Tkv, Hq, Hkv, D, dtype, 100 + Tq + D)
    o, lse = cuda_lib.cross_prefill(q.cuda(), k.cuda(), v.cuda(), q_pos0, want_lse=True)
    ro, rlse = oracle.attention(q, k, v, q_pos0, 0)
    assert_close(o, ro, dtype, "o")
    assert_close(lse, rlse.transpose(0, 2, 1), dtype, "lse", max_abs=1e-3, rel_l2=1e-4)


def test_cross_prefill_mask_leak(cuda_lib):
    # Future keys carry huge values: any leak across the causal mask explodes.
    B, T, Hq, Hkv, D = 1, 200, 4, 2, 128
    q, k, v = _qkv(B, T, T, Hq, Hkv, D, BF, 7)
    q0 = 120
    v2 = v.clone()
    v2[:, q0 + 80:] = 1e4
    o = cuda_lib.cross_prefill(q[:, :q0 + 80].contiguous().cuda(), k.cuda(), v2.cuda(), 0)
    ro, _ = oracle.attention(q[:, :q0 + 80], k, v2, 0, 0)
    assert_close(o, ro, BF, "o")


# -------------------------------------------------------------- swa prefill
@pytest.mark.parametrize("dtype", [BF, F32])
@pytest.mark.parametrize("B,T,Hq,Hkv,D,W", [
    (1, 256, 4, 2, 64, 32),
    (2, 333, 8, 2, 128, 100),
    (1, 200, 8, 8, 128, 1),     # window 1: each row sees only itself
    (1, 90, 4, 1, 64, 500),     # window > T: plain causal
])
def test_swa_prefill_and_ring_match_oracle(cuda_lib, dtype, B, T, Hq, Hkv, D, W):
    q, k, v = _qkv(B, T, T, Hq, Hkv, D, dtype, 200 + T + W)
    rk = torch.full((B, W, Hkv, D), 7.0, dtype=dtype, device="cuda")
    rv = torch.full((B, W, Hkv, D), 7.0, dtype=dtype, device="cuda")
    sp = torch.full((B, W), -7, dtype=torch.int32, device="cuda")
    o, lse = cuda_lib.swa_prefill(q.cuda(), k.cuda(), v.cuda(), W, ring=(rk, rv, sp), want_lse=True)
    ro, rlse = oracle.attention(q, k, v, 0, W)
    assert_close(o, ro, dtype, "o")
    assert_close(lse, rlse.transpose(0, 2, 1), dtype, "lse", max_abs=1e-3, rel_l2=1e-4)
    for b in range(B):
        ek, ev, esp = oracle.ring_from_prefill(k[b], v[b], W)
        np.testing.assert_array_equal(sp[b].cpu().numpy(), esp)
        np.testing.assert_array_equal(to_np(rk[b]), ek)   # copies: bit-exact
        np.testing.assert_array_equal(to_np(rv[b]), ev)


@pytest.mark.parametrize("D,W", [(128, 0), (64, 0), (128, 128), (64, 100)])
def test_prefill_output_16B_aligned(cuda_lib, D, W):
    # o 16 bytes past a 32-byte boundary: the paired kernel writes rows with
    # 16-byte stores there (32-byte stores otherwise)
    B, T, Hq, Hkv = 2, 300, 8, 2
    q, k, v = _qkv(B, T, T, Hq, Hkv, D, BF, 300 + D + W)
    flat = torch.zeros(q.numel() + 8, dtype=BF, device="cuda")
    o = flat[8:].view(q.shape)
    assert o.data_ptr() % 32 == 16
    if W:
        cuda_lib.swa_prefill(q.cuda(), k.cuda(), v.cuda(), W, o=o)
    else:
        cuda_lib.cross_prefill(q.cuda(), k.cuda(), v.cuda(), 0, o=o)
    ro, _ = oracle.attention(q, k, v, 0, W)
    assert_close(o, ro, BF, "o")
    assert float(flat[:8].float().abs().max()) == 0.0   # nothing written before o


# -------------------------------------------------------------- swa decode
@pytest.mark.parametrize("dtype", [BF, F32])
def test_swa_decode_steps_match_oracle(cuda_lib, dtype):
    B, T, n_dec, Hq, Hkv, D, W = 3, 40, 30, 8, 2, 128, 16
    N = T + n_dec
    q, k, v = _qkv(B, N, N, Hq, Hkv, D, dtype, 300)
    rk = torch.empty((B, W, Hkv, D), dtype=dtype, device="cuda")
    rv = torch.empty((B, W, Hkv, D), dtype=dtype, device="cuda")
    sp = torch.empty((B, W), dtype=torch.int32, device="cuda")
    cuda_lib.swa_prefill(q[:, :T].contiguous().cuda(), k[:, :T].contiguous().cuda(),
                         v[:, :T].contiguous().cuda(), W, ring=(rk, rv, sp))
    ro, _ = oracle.attention(q, k, v, 0, W)
    rings = [oracle.ring_from_prefill(k[b, :T], v[b, :T], W) for b in range(B)]
    for p in range(T, N):
        pos = torch.full((B,), p, dtype=torch.int64, device="cuda")
        o = cuda_lib.swa_decode(q[:, p].contiguous().cuda(), k[:, p].contiguous().cuda(),
                                v[:, p].contiguous().cuda(), pos, rk, rv, sp, W)
        assert_close(o, ro[:, p], dtype, f"o@{p}")
        for b in range(B):
            oracle.ring_push(rings[b][0], rings[b][1], rings[b][2], p, k[b, p], v[b, p])
            np.testing.assert_array_equal(sp[b].cpu().numpy(), rings[b][2])
            np.testing.assert_array_equal(to_np(rk[b]), rings[b][0])


@pytest.mark.parametrize("Hq,Hkv,D,W,T", [
    (8, 8, 128, 300, 700),      # group 1; three slices of 112 slots, the last one short
    (8, 4, 64, 1000, 1500),     # group 2; eight slices, the last one 104 slots
    (16, 2, 128, 2048, 2500),   # group 8; two 128-slot chunks per slice (two stages)
    (32, 8, 128, 5000, 5100),   # group 4; five chunks per slice
    (8, 2, 128, 129, 100),      # ring not yet full (empty slots), two slices
])
def test_swa_decode_window_shapes(cuda_lib, Hq, Hkv, D, W, T):
    # the bf16 window decode at group sizes, windows and slice shapes that the
    # 16-slot window above does not reach; ring and slot_pos bit-exact
    B, n_dec = 2, 3
    N = T + n_dec
    q, k, v = _qkv(B, N, N, Hq, Hkv, D, BF, 320 + W)
    rk = torch.empty((B, W, Hkv, D), dtype=BF, device="cuda")
    rv = torch.empty((B, W, Hkv, D), dtype=BF, device="cuda")
    sp = torch.empty((B, W), dtype=torch.int32, device="cuda")
    cuda_lib.swa_prefill(q[:, :T].contiguous().cuda(), k[:, :T].contiguous().cuda(),
                         v[:, :T].contiguous().cuda(), W, ring=(rk, rv, sp))
    rings = [oracle.ring_from_prefill(k[b, :T], v[b, :T], W) for b in range(B)]
    for p in range(T, N):
        pos = torch.full((B,), p, dtype=torch.int64, device="cuda")
        o = cuda_lib.swa_decode(q[:, p].contiguous().cuda(), k[:, p].contiguous().cuda(),
                                v[:, p].contiguous().cuda(), pos, rk, rv, sp, W)
        ro, _ = oracle.attention(q, k, v, 0, W, rows=[(b, p) for b in range(B)])
        assert_close(o, ro, BF, f"o@{p}")
        for b in range(B):
            oracle.ring_push(rings[b][0], rings[b][1], rings[b][2], p, k[b, p], v[b, p])
            np.testing.assert_array_equal(sp[b].cpu().numpy(), rings[b][2])
            np.testing.assert_array_equal(to_np(rk[b]), rings[b][0])
            np.testing.assert_array_equal(to_np(rv[b]), rings[b][1])


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 1, 128), (4, 2, 64)])
def test_swa_decode_window_one_is_the_new_value(cuda_lib, Hq, Hkv, D):
    # window 1: the only slot is the new token's, so every ring slot is left
    # out and o is the new token's value row, exactly (weight 2^0 / 2^0)
    B, W = 3, 1
    q = wl.normal((B, Hq, D), 330, BF).cuda()
    kn = wl.normal((B, Hkv, D), 331, BF).cuda()
    vn = wl.normal((B, Hkv, D), 332, BF).cuda()
    rk = wl.normal((B, W, Hkv, D), 333, BF).cuda()
    rv = (wl.normal((B, W, Hkv, D), 334, BF) * 1e4).to(BF).cuda()   # would dominate if read
    sp = torch.full((B, W), 5, dtype=torch.int32, device="cuda")
    pos = torch.tensor([6, 7, 100], dtype=torch.int64, device="cuda")
    o = cuda_lib.swa_decode(q, kn, vn, pos, rk, rv, sp, W)
    assert torch.equal(o, vn.repeat_interleave(Hq // Hkv, dim=1))
    assert torch.equal(rk[:, 0], kn) and torch.equal(rv[:, 0], vn)
    assert sp[:, 0].tolist() == [6, 7, 100]


@pytest.mark.parametrize("W,T", [(2, 5), (2, 1)])
def test_swa_decode_window_two(cuda_lib, W, T):
    # the smallest window with a ring read: one old slot plus the new token
    B, Hq, Hkv, D, n_dec = 2, 8, 1, 128, 3
    N = T + n_dec
    q, k, v = _qkv(B, N, N, Hq, Hkv, D, BF, 340 + T)
    rk = torch.empty((B, W, Hkv, D), dtype=BF, device="cuda")
    rv = torch.empty((B, W, Hkv, D), dtype=BF, device="cuda")
    sp = torch.empty((B, W), dtype=torch.int32, device="cuda")
    cuda_lib.swa_prefill(q[:, :T].contiguous().cuda(), k[:, :T].contiguous().cuda(),
                         v[:, :T].contiguous().cuda(), W, ring=(rk, rv, sp))
    ro, _ = oracle.attention(q, k, v, 0, W)
    for p in range(T, N):
        pos = torch.full((B,), p, dtype=torch.int64, device="cuda")
        o = cuda_lib.swa_decode(q[:, p].contiguous().cuda(), k[:, p].contiguous().cuda(),
                                v[:, p].contiguous().cuda(), pos, rk, rv, sp, W)
        assert_close(o, ro[:, p], BF, f"o@{p}")


def test_swa_decode_ragged_positions(cuda_lib):
    # sequences at different positions, some with a partly empty ring
    B, Hq, Hkv, D, W = 4, 4, 2, 64, 8
    pos_list = [0, 3, 8, 21]
    N = max(pos_list) + 1
    q, k, v = _qkv(B, N, N, Hq, Hkv, D, BF, 310)
    rk = torch.zeros((B, W, Hkv, D), dtype=BF, device="cuda")
    rv = torch.zeros((B, W, Hkv, D), dtype=BF, device="cuda")
    sp = torch.full((B, W), -1, dtype=torch.int32, device="cuda")
    rings = []
    for b, p in enumerate(pos_list):
        ek, ev, esp = oracle.ring_from_prefill(k[b, :p], v[b, :p], W)
        rings.append((ek, ev, esp))
        rk[b] = torch.from_numpy(ek).to(BF)
        rv[b] = torch.from_numpy(ev).to(BF)
        sp[b] = torch.from_numpy(esp)
    pos = torch.tensor(pos_list, dtype=torch.int64, device="cuda")
    qd = torch.stack([q[b, p] for b, p in enumerate(pos_list)]).contiguous()
    kd = torch.stack([k[b, p] for b, p in enumerate(pos_list)]).contiguous()
    vd = torch.stack([v[b, p] for b, p in enumerate(pos_list)]).contiguous()
    o = cuda_lib.swa_decode(qd.cuda(), kd.cuda(), vd.cuda(), pos, rk, rv, sp, W)
    ro, _ = oracle.attention(q, k, v, 0, W)
    assert_close(o, np.stack([ro[b, p] for b, p in enumerate(pos_list)]), BF, "o")


# ------------------------------------------------------------- cross decode
@pytest.mark.parametrize("dtype", [BF, F32])
@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (4, 2, 64), (8, 1, 128), (16, 2, 64), (8, 4, 128)])
def test_cross_decode_matches_oracle(cuda_lib, dtype, Hq, Hkv, D):
    lens = [1, 17, 300, 1000, 2051, 128]
    B = len(lens)
    starts = np.cumsum([0] + [l + 5 for l in lens[:-1]])   # gaps between sequences
    rows = int(starts[-1] + lens[-1] + 3)
    kc = wl.normal((rows, Hkv, D), 400, dtype)
    vc = wl.normal((rows, Hkv, D), 401, dtype)
    q = wl.normal((B, Hq, D), 402, dtype)
    ss = torch.tensor(starts, dtype=torch.int64)
    sl = torch.tensor(lens, dtype=torch.int32)
    o, lse = cuda_lib.cross_decode(q.cuda(), kc.cuda(), vc.cuda(), ss.cuda(), sl.cuda(), max(lens),
                                   want_lse=True)
    ro, rlse = oracle.cross_decode(q, kc, vc, starts, lens)
    assert_close(o, ro, dtype, "o")
    assert_close(lse, rlse, dtype, "lse", max_abs=1e-3, rel_l2=1e-4)


def test_cross_decode_equals_prefill_rows(cuda_lib):
    # decode at position p over cache rows 0..p equals prefill row p (GPU vs GPU
    # and both vs oracle)
    B, T, Hq, Hkv, D = 1, 700, 32, 8, 128
    q, k, v = _qkv(B, T, T, Hq, Hkv, D, BF, 500)
    op = cuda_lib.cross_prefill(q.cuda(), k.cuda(), v.cuda())
    ps = [0, 1, 127, 128, 699]
    ss = torch.zeros(len(ps), dtype=torch.int64, device="cuda")
    sl = torch.tensor([p + 1 for p in ps], dtype=torch.int32, device="cuda")
    qd = torch.stack([q[0, p] for p in ps]).contiguous().cuda()
    od = cuda_lib.cross_decode(qd, k[0].contiguous().cuda(), v[0].contiguous().cuda(), ss, sl, T)
    ro, _ = oracle.attention(q, k, v)
    for n, p in enumerate(ps):
        assert_close(od[n], ro[0, p], BF, f"decode@{p}")
        assert_close(op[0, p], ro[0, p], BF, f"prefill@{p}")


def test_cross_decode_large_values_needle(cuda_lib):
    # a planted high-score key dominates: output ~ its value row (unit scale)
    Hq, Hkv, D, n = 8, 2, 128, 5000
    kc = wl.normal((n, Hkv, D), 600, BF)
    vc = wl.normal((n, Hkv, D), 601, BF)
    q = wl.normal((1, Hq, D), 602, BF)
    kc[3333] = (q[0].view(Hkv, Hq // Hkv, D)[:, 0] * 2.0).to(BF)
    ss = torch.zeros(1, dtype=torch.int64)
    sl = torch.tensor([n], dtype=torch.int32)
    o = cuda_lib.cross_decode(q.cuda(), kc.cuda(), vc.cuda(), ss.cuda(), sl.cuda(), n)
    ro, _ = oracle.cross_decode(q, kc, vc, [0], [n])
    assert_close(o, ro, BF, "o")


# --------------------------------------------------------- projection + blend
@pytest.mark.parametrize("dtype", [BF, F32])
@pytest.mark.parametrize("n,d,Hkv,D", [(1, 256, 2, 64), (77, 512, 2, 128), (300, 256, 8, 64), (4, 1024, 8, 128),
                                       (16, 512, 8, 128), (17, 512, 2, 64)])
def test_kv_project_blend_matches_oracle(cuda_lib, dtype, n, d, Hkv, D):
    x = wl.normal((n, d), 700 + n, dtype)
    w = wl.normal((2 * Hkv * D, d), 701 + n, dtype, std=d ** -0.5)
    kb = wl.normal((n, Hkv, D), 702, dtype)
    vb = wl.normal((n, Hkv, D), 703, dtype)
    k, v = cuda_lib.kv_project_blend(x.cuda(), w.cuda(), Hkv, D, kb.cuda(), vb.cuda(), 0.5, 0.25)
    rk, rv = oracle.kv_project_blend(x, w, Hkv, D, kb, vb, 0.5, 0.25)
    assert_close(k, rk, dtype, "k")
    assert_close(v, rv, dtype, "v")
    # w = 0 and no base: the plain global-KV projection; identical to w=0 with a base
    k0, v0 = cuda_lib.kv_project_blend(x.cuda(), w.cuda(), Hkv, D)
    k0b, v0b = cuda_lib.kv_project_blend(x.cuda(), w.cuda(), Hkv, D, kb.cuda(), vb.cuda(), 0.0, 0.0)
    rk0, rv0 = oracle.kv_project_blend(x, w, Hkv, D)
    assert_close(k0, rk0, dtype, "k0")
    assert torch.equal(k0, k0b) and torch.equal(v0, v0b)


def test_kv_project_scatter_rows_exact(cuda_lib):
    # appending to the shared cache: only the addressed rows change
    n, d, Hkv, D, rows = 5, 256, 2, 64, 40
    x = wl.normal((n, d), 710, BF)
    w = wl.normal((2 * Hkv * D, d), 711, BF, std=d ** -0.5)
    dst = torch.tensor([3, 39, 0, 17, 18], dtype=torch.int64)
    kc = torch.full((rows, Hkv, D), 123.0, dtype=BF, device="cuda")
    vc = torch.full((rows, Hkv, D), -5.0, dtype=BF, device="cuda")
    cuda_lib.kv_project_blend(x.cuda(), w.cuda(), Hkv, D, dst_rows=dst.cuda(), k_out=kc, v_out=vc)
    rk, rv = oracle.kv_project_blend(x, w, Hkv, D)
    untouched = sorted(set(range(rows)) - set(dst.tolist()))
    assert torch.all(kc[untouched] == 123.0) and torch.all(vc[untouched] == -5.0)
    assert_close(kc[dst.cuda()], rk, BF, "k")
    assert_close(vc[dst.cuda()], rv, BF, "v")


@pytest.mark.parametrize("dtype", [BF, F32])
def test_linear_matches_oracle(cuda_lib, dtype):
    x = wl.normal((70, 256), 720, dtype)
    w = wl.normal((192, 256), 721, dtype, std=1 / 16)
    base = wl.normal((70, 192), 722, dtype)
    out = cuda_lib.linear(x.cuda(), w.cuda(), base.cuda(), 1.0, apply_ln=True)
    ref = oracle.project(x, w, True) + to_np(base)
    assert_close(out, ref, dtype, "out")


# ------------------------------------------- tensor-core projection (n >= 512)
@pytest.mark.parametrize("n,d,Hkv,D,mean,apply_ln", [
    (1000, 512, 8, 128, 0.0, True),     # 8 row tiles of 127 with a ragged tail
    (640, 1024, 2, 64, 0.0, True),      # one 256-wide output chunk holding K and V
    (2048, 4096, 8, 128, 3.0, True),    # large row mean: exercises the LayerNorm fold
    (777, 256, 4, 128, 0.0, False),
])
def test_kv_project_blend_tensor_core(cuda_lib, n, d, Hkv, D, mean, apply_ln):
    x = (wl.normal((n, d), 730 + n, torch.float32) + mean).to(BF)
    w = wl.normal((2 * Hkv * D, d), 731, BF, std=d ** -0.5)
    kb = wl.normal((n, Hkv, D), 732, BF)
    vb = wl.normal((n, Hkv, D), 733, BF)
    k, v = cuda_lib.kv_project_blend(x.cuda(), w.cuda(), Hkv, D, kb.cuda(), vb.cuda(), 0.3, 0.7,
                                     apply_ln=apply_ln)
    rk, rv = oracle.kv_project_blend(x, w, Hkv, D, kb, vb, 0.3, 0.7, apply_ln=apply_ln)
    assert_close(k, rk, BF, "k")
    assert_close(v, rv, BF, "v")


def test_kv_project_tensor_core_scatter(cuda_lib):
    n, d, Hkv, D = 600, 512, 8, 128
    rows = 1500
    x = wl.normal((n, d), 740, BF)
    w = wl.normal((2 * Hkv * D, d), 741, BF, std=d ** -0.5)
    dst = torch.randperm(rows, generator=wl.gen(742))[:n].to(torch.int64)
    kc = torch.full((rows, Hkv, D), 9.0, dtype=BF, device="cuda")
    vc = torch.full((rows, Hkv, D), -9.0, dtype=BF, device="cuda")
    cuda_lib.kv_project_blend(x.cuda(), w.cuda(), Hkv, D, dst_rows=dst.cuda(), k_out=kc, v_out=vc)
    rk, rv = oracle.kv_project_blend(x, w, Hkv, D)
    untouched = sorted(set(range(rows)) - set(dst.tolist()))
    assert torch.all(kc[untouched] == 9.0) and torch.all(vc[untouched] == -9.0)
    assert_close(kc[dst.cuda()], rk, BF, "k")
    assert_close(vc[dst.cuda()], rv, BF, "v")


@pytest.mark.parametrize("window", [0, 300])
def test_prefill_huge_score_growth(cuda_lib, window):
    # For some query rows, a key in a LATER KV tile scores far above everything
    # seen before (hundreds of log2 units): the kernel must move its running
    # reference max (redoing that tile) without overflow or loss.
    B, T, Hq, Hkv, D = 1, 700, 8, 2, 128
    G = Hq // Hkv
    q, k, v = _qkv(B, T, T, Hq, Hkv, D, BF, 760)
    for i, j in [(650, 600), (699, 520), (300, 290), (259, 257)]:
        k[0, j] = (q[0, i].view(Hkv, G, D)[:, 0] * 20.0).to(BF)
    o, lse = cuda_lib.cross_prefill(q.cuda(), k.cuda(), v.cuda(), want_lse=True) if window == 0 else \
        cuda_lib.swa_prefill(q.cuda(), k.cuda(), v.cuda(), window, want_lse=True)
    ro, rlse = oracle.attention(q, k, v, 0, window)
    assert_close(o, ro, BF, "o")
    assert_close(lse, rlse.transpose(0, 2, 1), BF, "lse", max_abs=2e-3, rel_l2=1e-4)
