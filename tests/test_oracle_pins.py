"""Pins for the CPU fp64 oracle: each check compares it with something other
than itself -- a library routine (torch fp64 scaled_dot_product_attention,
torch layer_norm, numpy matmul), a closed form, a worked value, or an
invariant the pages state.  The cases are chosen so that a plausible slip in
the oracle (a dropped scale, an off-by-one window, a wrong GQA index, a
transposed weight, a missing blend term, a sign error) fails at least one."""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads as wl

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _sdpa(q, k, v, q_pos0=0, window=0):
    """torch fp64 SDPA with an explicit visibility mask, GQA by enable_gqa."""
    q = torch.as_tensor(q, dtype=torch.float64).permute(0, 2, 1, 3)
    k = torch.as_tensor(k, dtype=torch.float64).permute(0, 2, 1, 3)
    v = torch.as_tensor(v, dtype=torch.float64).permute(0, 2, 1, 3)
    Tq, Tkv = q.shape[2], k.shape[2]
    p = torch.arange(Tq)[:, None] + q_pos0
    j = torch.arange(Tkv)[None, :]
    m = j <= p
    if window > 0:
        m = m & (j > p - window)
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=m, enable_gqa=True)
    return o.permute(0, 2, 1, 3).numpy()


def _rand(shape, seed):
    return wl.normal(shape, seed, torch.float32).double().numpy()


# ----------------------------------------------------------------- LayerNorm
def test_layernorm_worked_value():
    # mean 2.5, biased variance 1.25 -> (x - 2.5) / sqrt(1.25 + eps)
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    s = math.sqrt(1.25 + 1e-5)
    np.testing.assert_allclose(oracle.layernorm(x, 1e-5)[0],
                               [-1.5 / s, -0.5 / s, 0.5 / s, 1.5 / s], rtol=0, atol=1e-15)


def test_layernorm_vs_torch():
    x = _rand((37, 96), 1) * 3.0 + 0.7
    ref = F.layer_norm(torch.from_numpy(x), (96,), eps=1e-5).numpy()
    np.testing.assert_allclose(oracle.layernorm(x, 1e-5), ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- projection
@pytest.mark.parametrize("apply_ln", [True, False])
def test_project_vs_numpy(apply_ln):
    x = _rand((19, 64), 2) + 0.3
    w = _rand((48, 64), 3)  # [out, in]
    h = F.layer_norm(torch.from_numpy(x), (64,), eps=1e-5).numpy() if apply_ln else x
    np.testing.assert_allclose(oracle.project(x, w, apply_ln), h @ w.T, rtol=0, atol=1e-11)


def test_project_non_square_orientation():
    # W with a single nonzero entry at [out=2, in=5] picks x[:, 5] into column 2.
    x = _rand((4, 8), 4)
    w = np.zeros((3, 8)); w[2, 5] = 1.0
    out = oracle.project(x, w, apply_ln=False)
    np.testing.assert_array_equal(out[:, 2], x[:, 5])
    np.testing.assert_array_equal(out[:, :2], 0.0)


# --------------------------------------------------------------------- blend
def test_blend_closed_form_and_zero_weight():
    a = np.array([1.0, -2.0, 3.5]); base = np.array([4.0, 8.0, -2.0])
    np.testing.assert_array_equal(oracle.blend(a, base, 0.5), [3.0, 2.0, 2.5])
    np.testing.assert_array_equal(oracle.blend(a, base, 0.0), a)  # w = 0: YOCO


def test_kv_project_blend_linearity():
    x = _rand((10, 32), 5); w = _rand((2 * 2 * 8, 32), 6)
    kb = _rand((10, 2, 8), 7); vb = _rand((10, 2, 8), 8)
    k0, v0 = oracle.kv_project_blend(x, w, 2, 8)
    k1, v1 = oracle.kv_project_blend(x, w, 2, 8, kb, vb, 0.25, 0.75)
    np.testing.assert_allclose(k1, k0 + 0.25 * kb, atol=1e-13)
    np.testing.assert_allclose(v1, v0 + 0.75 * vb, atol=1e-13)
    # K columns come first, then V columns, in the [out, in] weight.
    h = F.layer_norm(torch.from_numpy(x), (32,), eps=1e-5).numpy()
    np.testing.assert_allclose(k0.reshape(10, 16), h @ w[:16].T, atol=1e-12)
    np.testing.assert_allclose(v0.reshape(10, 16), h @ w[16:].T, atol=1e-12)


# ----------------------------------------------------------------- attention
@pytest.mark.parametrize("B,Tq,Tkv,Hq,Hkv,D,q_pos0,window", [
    (1, 17, 17, 4, 2, 8, 0, 0),
    (2, 33, 33, 4, 1, 16, 0, 0),
    (2, 33, 33, 6, 3, 8, 0, 5),
    (1, 40, 40, 2, 2, 4, 0, 1),
    (1, 9, 30, 4, 2, 8, 21, 0),     # chunk: queries at positions 21..29
    (1, 9, 30, 4, 2, 8, 21, 7),
    (3, 12, 12, 8, 2, 16, 0, 64),   # window larger than T
])
def test_attention_vs_torch_sdpa(B, Tq, Tkv, Hq, Hkv, D, q_pos0, window):
    seed = B * 100 + Tq + window
    q = _rand((B, Tq, Hq, D), seed); k = _rand((B, Tkv, Hkv, D), seed + 1)
    v = _rand((B, Tkv, Hkv, D), seed + 2)
    o, lse = oracle.attention(q, k, v, q_pos0, window)
    np.testing.assert_allclose(o, _sdpa(q, k, v, q_pos0, window), rtol=0, atol=1e-12)
    # lse: recompute sum_j exp(s_j - lse) over the visible keys -> 1
    G = Hq // Hkv
    s = np.einsum("bihd,bjhd->bhij", q, np.repeat(k, G, axis=2)) / math.sqrt(D)
    p = np.arange(Tq)[:, None] + q_pos0; j = np.arange(Tkv)[None, :]
    vis = (j <= p) & ((j > p - window) if window > 0 else True)
    e = np.where(vis[None, None], np.exp(s - lse.transpose(0, 2, 1)[..., None]), 0.0)
    np.testing.assert_allclose(e.sum(-1), 1.0, atol=1e-12)


def test_attention_constant_values():
    # every visible value row equal to c => every output equals c exactly
    q = _rand((1, 20, 4, 8), 11); k = _rand((1, 20, 2, 8), 12)
    c = _rand((8,), 13)
    v = np.broadcast_to(c, (1, 20, 2, 8)).copy()
    for window in (0, 3):
        o, _ = oracle.attention(q, k, v, 0, window)
        np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), atol=1e-14)


@pytest.mark.parametrize("window", [0, 1, 4, 7])
def test_attention_equal_keys_is_window_mean(window):
    # zero keys => all scores 0 => o_i = mean of the visible v_j; with
    # v_j = j that mean is (lo + i) / 2, lo = first visible position; lse = log(count)
    T = 23
    q = _rand((1, T, 2, 4), 14); k = np.zeros((1, T, 1, 4))
    v = np.broadcast_to(np.arange(T, dtype=np.float64)[None, :, None, None], (1, T, 1, 4)).copy()
    o, lse = oracle.attention(q, k, v, 0, window)
    i = np.arange(T)
    lo = np.maximum(0, i - window + 1) if window > 0 else np.zeros(T)
    cnt = i - lo + 1
    np.testing.assert_allclose(o[0, :, :, 0], np.repeat(((lo + i) / 2.0)[:, None], 2, 1), atol=1e-12)
    np.testing.assert_allclose(lse[0], np.repeat(np.log(cnt)[:, None], 2, 1), atol=1e-12)


def test_attention_first_row_sees_only_itself():
    q = _rand((2, 6, 4, 8), 15); k = _rand((2, 6, 2, 8), 16); v = _rand((2, 6, 2, 8), 17)
    o, _ = oracle.attention(q, k, v)
    np.testing.assert_allclose(o[:, 0], np.repeat(v[:, 0], 2, axis=1), atol=1e-15)


def test_attention_two_keys_scale():
    # D = 4, scale 1/2: q.k0 = 2, q.k1 = 0 -> weights softmax([1, 0])
    q = np.zeros((1, 2, 1, 4)); q[0, 1, 0] = [1, 1, 0, 0]
    k = np.zeros((1, 2, 1, 4)); k[0, 0, 0] = [1, 1, 0, 0]
    v = np.zeros((1, 2, 1, 4)); v[0, 0, 0, 0] = 1.0; v[0, 1, 0, 1] = 1.0
    o, lse = oracle.attention(q, k, v)
    e = math.e
    np.testing.assert_allclose(o[0, 1, 0, :2], [e / (e + 1), 1 / (e + 1)], atol=1e-15)
    np.testing.assert_allclose(lse[0, 1, 0], math.log(e + 1), atol=1e-15)


def test_attention_gqa_grouping_is_contiguous():
    # KV head 0 carries +1 values, KV head 1 carries -1: with Hq=4, Hkv=2 query
    # heads 0,1 read head 0 and 2,3 read head 1 (h // G, not h % Hkv).
    q = _rand((1, 5, 4, 8), 18); k = _rand((1, 5, 2, 8), 19)
    v = np.zeros((1, 5, 2, 8)); v[:, :, 0] = 1.0; v[:, :, 1] = -1.0
    o, _ = oracle.attention(q, k, v)
    np.testing.assert_allclose(o[0, :, 0:2], 1.0, atol=1e-15)
    np.testing.assert_allclose(o[0, :, 2:4], -1.0, atol=1e-15)


def test_attention_needle():
    # one key aligned with the query (score s), the rest orthogonal (score 0)
    T, D = 16, 8
    q = np.zeros((1, T, 1, D)); q[0, T - 1, 0, 0] = 4.0
    k = np.zeros((1, T, 1, D)); k[0, 5, 0, 0] = 4.0
    v = _rand((1, T, 1, D), 20)
    o, _ = oracle.attention(q, k, v)
    s = 16.0 / math.sqrt(D)
    w_needle = math.exp(s) / (math.exp(s) + T - 1)
    expect = w_needle * v[0, 5, 0] + (1 - w_needle) / (T - 1) * (v[0, :, 0].sum(0) - v[0, 5, 0])
    np.testing.assert_allclose(o[0, T - 1, 0], expect, atol=1e-13)


def test_window_at_least_T_equals_causal():
    q = _rand((2, 30, 4, 8), 21); k = _rand((2, 30, 2, 8), 22); v = _rand((2, 30, 2, 8), 23)
    oc, lc = oracle.attention(q, k, v, 0, 0)
    for W in (30, 31, 1000):
        ow, lw = oracle.attention(q, k, v, 0, W)
        np.testing.assert_array_equal(ow, oc)
        np.testing.assert_array_equal(lw, lc)


def test_chunked_equals_unchunked_and_rows():
    # Chunk parallelism claim (Appendix A): splitting the queries into chunks
    # does not change the result; sampled rows equal the full tensor's rows.
    q = _rand((1, 48, 4, 8), 24); k = _rand((1, 48, 2, 8), 25); v = _rand((1, 48, 2, 8), 26)
    for window in (0, 10):
        full, lfull = oracle.attention(q, k, v, 0, window)
        for c0 in (0, 16, 32):
            oc, lc = oracle.attention(q[:, c0:c0 + 16], k[:, :c0 + 16], v[:, :c0 + 16], c0, window)
            np.testing.assert_array_equal(oc, full[:, c0:c0 + 16])
            np.testing.assert_array_equal(lc, lfull[:, c0:c0 + 16])
        rows = [(0, 0), (0, 17), (0, 47)]
        orow, lrow = oracle.attention(q, k, v, 0, window, rows=rows)
        for n, (_, i) in enumerate(rows):
            np.testing.assert_array_equal(orow[n], full[0, i])
            np.testing.assert_array_equal(lrow[n], lfull[0, i])


# -------------------------------------------------------------------- decode
def test_decode_step_equals_prefill_row():
    # Decode of position p over cache rows 0..p == prefill row p (shared-KV
    # cross-attention is ordinary causal attention with K_g, V_g).
    B, T, Hq, Hkv, D = 3, 20, 4, 2, 8
    k = _rand((B, T, Hkv, D), 27); v = _rand((B, T, Hkv, D), 28); q = _rand((B, T, Hq, D), 29)
    full, lfull = oracle.attention(q, k, v)
    lens = np.array([5, 20, 13])
    # pack the three sequences' prefixes into one cache with gaps
    starts = np.array([0, 7, 31])
    kc = np.zeros((50, Hkv, D)); vc = np.zeros((50, Hkv, D))
    for b in range(B):
        kc[starts[b]:starts[b] + lens[b]] = k[b, :lens[b]]
        vc[starts[b]:starts[b] + lens[b]] = v[b, :lens[b]]
    qd = np.stack([q[b, lens[b] - 1] for b in range(B)])
    o, lse = oracle.cross_decode(qd, kc, vc, starts, lens)
    for b in range(B):
        np.testing.assert_array_equal(o[b], full[b, lens[b] - 1])
        np.testing.assert_array_equal(lse[b], lfull[b, lens[b] - 1])


# ---------------------------------------------------------------- visibility
@pytest.mark.parametrize("Tq,Tkv,q_pos0,W", [(5, 5, 0, 0), (7, 12, 5, 0), (9, 9, 0, 3), (6, 20, 14, 4),
                                             (4, 10, 6, 100), (1, 1, 0, 1)])
def test_visibility_is_a_shifted_band(Tq, Tkv, q_pos0, W):
    # causal: numpy's lower triangle shifted by the chunk offset; window W:
    # that triangle minus the one W diagonals further down
    m = oracle.visibility(Tq, Tkv, q_pos0, W)
    expect = np.tril(np.ones((Tq, Tkv), dtype=bool), k=q_pos0)
    if W > 0:
        expect &= ~np.tril(np.ones((Tq, Tkv), dtype=bool), k=q_pos0 - W)
    np.testing.assert_array_equal(m, expect)
    # row counts: min(p + 1, W) keys for the query at absolute position p
    p = np.arange(Tq) + q_pos0
    cnt = np.minimum(p + 1, Tkv) if W <= 0 else np.minimum(np.minimum(p + 1, W), Tkv)
    np.testing.assert_array_equal(m.sum(1), cnt)


# ---------------------------------------------------------------------- ring
@pytest.mark.parametrize("T,W", [(0, 4), (3, 4), (4, 4), (5, 4), (17, 4), (1000, 32), (31, 32)])
def test_ring_slots_closed_form(T, W):
    s = np.arange(W)
    expect = np.where(s < T, s + W * ((T - 1 - s) // W), -1)
    np.testing.assert_array_equal(oracle.ring_prefill_slots(T, W), expect.astype(np.int32))


def test_ring_decode_equals_window_attention():
    # After a prefill of T tokens plus pushes of later tokens, a decode read
    # from the ring equals the window-attention row of the full sequence.
    T, n_dec, W, Hq, Hkv, D = 11, 9, 4, 4, 2, 8
    N = T + n_dec
    q = _rand((1, N, Hq, D), 30); k = _rand((1, N, Hkv, D), 31); v = _rand((1, N, Hkv, D), 32)
    full, lfull = oracle.attention(q, k, v, 0, W)
    rk, rv, sp = oracle.ring_from_prefill(k[0, :T], v[0, :T], W)
    np.testing.assert_array_equal(sp, oracle.ring_prefill_slots(T, W))
    for p in range(T, N):
        oracle.ring_push(rk, rv, sp, p, k[0, p], v[0, p])
        assert sorted(sp.tolist()) == list(range(p - W + 1, p + 1))
        o, lse = oracle.swa_decode_ring(q[0, p], rk, rv, sp, p)
        np.testing.assert_allclose(o, full[0, p], atol=1e-14)
        np.testing.assert_allclose(lse, lfull[0, p], atol=1e-13)


# ---------------------------------------------------------------- accounting
def _golden(name):
    path = os.path.join(os.path.dirname(__file__), "golden", name)
    out = {}
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            key, val = line.split()
            out[key] = int(val)
    return out


def test_cache_accounting_matches_pages():
    g = _golden("cache_accounting_3b.txt")
    L, Ls, H, D, e, W, N = (g[k] for k in
                            ("layers", "self_layers", "kv_heads", "head_dim", "elem_bytes",
                             "window", "N"))
    assert oracle.cache_bytes_transformer(L, 1, H, D, e) == g["transformer_bytes_per_token"]
    assert oracle.cache_bytes_yoco(0, W, 1, H, D, e) == g["yoco_global_bytes_per_token"]
    assert oracle.cache_bytes_transformer(L, N, H, D, e) == g["transformer_bytes"]
    assert oracle.cache_bytes_yoco(Ls, W, N, H, D, e) == g["yoco_bytes"]
    # "roughly L-times lower" as N grows
    r = oracle.cache_bytes_transformer(L, 1 << 40, H, D, e) / oracle.cache_bytes_yoco(Ls, W, 1 << 40, H, D, e)
    assert abs(r - L) < 1e-3


# ---------------------------------------------------------------- tiny stack
def _small_stack(T, w2):
    cfg = wl.TinyStack(T=T, n_decode=0, d=32, Hq=4, Hkv=2, D=8, window=5,
                       w_blend=[0.0, w2], seed=3)
    x, w = wl.tiny_stack_inputs(cfg)
    return cfg, x, w


def test_tiny_stack_is_causal():
    # Row t of every intermediate depends only on rows <= t, so the stack run
    # on a prefix reproduces the prefix of the longer run exactly (this is
    # what makes decode == prefill and early exit exact).
    cfg, x, w = _small_stack(24, 0.5)
    full = oracle.tiny_stack(x, w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.w_blend)
    pre = oracle.tiny_stack(x[:15], w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.w_blend)
    for key in ("x", "k_g", "v_g"):
        np.testing.assert_allclose(pre[key], full[key][:15], atol=1e-12)
    for key in ("self_o", "cross_o"):
        for a, b in zip(pre[key], full[key]):
            np.testing.assert_allclose(a, b[:15], atol=1e-12)


def test_tiny_stack_blend_weight_zero_is_yoco():
    # With w = 0 the YOCO++ stack is the YOCO stack; with w != 0 only the
    # blended layer's K/V change by w * (bottom layer's K/V).
    cfg, x, w = _small_stack(16, 0.0)
    a = oracle.tiny_stack(x, w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, [0.0, 0.0])
    b = oracle.tiny_stack(x, w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, [0.0, 0.7])
    np.testing.assert_array_equal(a["self_k"][0], b["self_k"][0])
    np.testing.assert_allclose(b["self_k"][1] - a["self_k"][1], 0.7 * a["self_k"][0], atol=1e-12)
    np.testing.assert_allclose(b["self_v"][1] - a["self_v"][1], 0.7 * a["self_v"][0], atol=1e-12)
    assert not np.allclose(a["x"], b["x"])


def test_tiny_stack_cross_layers_share_one_kv():
    # Every cross layer attends to the same K_g, V_g: recomputing each cross
    # layer's output with torch SDPA over (K_g, V_g) reproduces it.
    cfg, x, w = _small_stack(20, 0.5)
    out = oracle.tiny_stack(x, w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.w_blend)
    for c in range(2):
        q = out["cross_q"][c][None]
        ref = _sdpa(q, out["k_g"][None], out["v_g"][None])
        np.testing.assert_allclose(out["cross_o"][c], ref[0], atol=1e-12)


def test_tiny_stack_early_exit_is_exact():
    # The pages: prefill may exit before the cross-decoder for all but the last
    # prompt row without changing the output.  Row by row the oracle computes
    # the same sums, so the early-exit row equals the full run's last row.
    cfg = wl.TinyStack()
    x, w = wl.tiny_stack_inputs(cfg, torch.float32)
    T = cfg.T
    full = oracle.tiny_stack(x[:T], w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.w_blend)
    ee = oracle.tiny_stack_early_exit(x[:T], w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.w_blend)
    np.testing.assert_allclose(ee, full["x"][T - 1], rtol=0, atol=1e-12)
    # and it differs from the row before: the check is not vacuous
    assert np.abs(ee - full["x"][T - 2]).max() > 1e-3


# ----------------------------------------------------------- gated retention
def _gret_inputs(B, T, H, D, seed, gate_mean=2.0, tau=4.0):
    q = _rand((B, T, H, D), seed)
    k = _rand((B, T, H, D), seed + 1)
    v = _rand((B, T, H, D), seed + 2)
    g = _rand((B, T, H), seed + 3) * 2.0 + gate_mean
    return q, k, v, oracle.gret_log_decay(g, tau)


def test_gret_log_decay_is_a_tempered_sigmoid():
    g = np.array([-50.0, -3.0, -0.5, 0.0, 0.7, 4.0, 50.0])
    for tau in (1.0, 4.0, 16.0):
        got = oracle.gret_log_decay(g, tau)
        # gamma^tau is the sigmoid itself
        np.testing.assert_allclose(np.exp(got * tau), 1.0 / (1.0 + np.exp(-g)), rtol=1e-12, atol=0)
        assert np.all(got <= 0.0)
    assert oracle.gret_log_decay(np.array([0.0]), 1.0)[0] == pytest.approx(np.log(0.5), abs=1e-15)


@pytest.mark.parametrize("chunk", [1, 4, 16, 37, 64])
@pytest.mark.parametrize("with_state", [False, True])
def test_gret_three_forms_agree(chunk, with_state):
    # the pages: the parallel, recurrent and chunkwise forms give the same result
    B, T, H, D = 2, 37, 3, 8
    q, k, v, lg = _gret_inputs(B, T, H, D, 900)
    s0 = _rand((B, H, D, D), 950) if with_state else None
    o_r, s_r = oracle.gret_recurrent(q, k, v, lg, state=s0)
    o_p = oracle.gret_parallel(q, k, v, lg, state=s0)
    o_c, s_c = oracle.gret_chunkwise(q, k, v, lg, chunk, state=s0)
    np.testing.assert_allclose(o_p, o_r, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(o_c, o_r, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(s_c, s_r, rtol=1e-11, atol=1e-11)


def test_gret_without_decay_is_cumulative_linear_attention():
    # gamma = 1: o_t = scale * q_t (sum_{s<=t} k_s^T v_s), by numpy cumsum
    B, T, H, D = 1, 20, 2, 6
    q, k, v, _ = _gret_inputs(B, T, H, D, 910)
    lg = np.zeros((B, T, H))
    scale = 0.37
    states = np.cumsum(np.einsum("bthd,bthe->bthde", k, v), axis=1)
    expect = scale * np.einsum("bthd,bthde->bthe", q, states)
    o, s = oracle.gret_recurrent(q, k, v, lg, scale=scale)
    np.testing.assert_allclose(o, expect, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s, scale * states[:, -1], rtol=1e-12, atol=1e-12)


def test_gret_full_decay_keeps_only_the_current_token():
    # gamma -> 0: o_t = scale * (q_t . k_t) v_t
    B, T, H, D = 2, 9, 2, 5
    q, k, v, _ = _gret_inputs(B, T, H, D, 920)
    lg = np.full((B, T, H), -1e4)
    o = oracle.gret_parallel(q, k, v, lg, scale=0.5)
    expect = 0.5 * np.einsum("bthd,bthd->bth", q, k)[..., None] * v
    np.testing.assert_allclose(o, expect, rtol=1e-12, atol=1e-12)


def test_gret_constant_decay_is_geometric():
    # constant gamma: weight gamma^(t-s) on token s, written as an explicit loop
    B, T, H, D = 1, 12, 1, 4
    q, k, v, _ = _gret_inputs(B, T, H, D, 930)
    gam = 0.8
    lg = np.full((B, T, H), np.log(gam))
    expect = np.zeros_like(q)
    for t in range(T):
        for s in range(t + 1):
            expect[0, t, 0] += gam ** (t - s) * 0.25 * np.dot(q[0, t, 0], k[0, s, 0]) * v[0, s, 0]
    o, _ = oracle.gret_chunkwise(q, k, v, lg, 5, scale=0.25)
    np.testing.assert_allclose(o, expect, rtol=1e-12, atol=1e-12)


def test_gret_state_continues_across_calls():
    # prefill of T1 tokens, then T2 more from the carried state == one run of T1 + T2
    B, T, H, D = 2, 30, 2, 6
    q, k, v, lg = _gret_inputs(B, T, H, D, 940)
    o_all, s_all = oracle.gret_recurrent(q, k, v, lg)
    o1, s1 = oracle.gret_chunkwise(q[:, :17], k[:, :17], v[:, :17], lg[:, :17], 8)
    o2, s2 = oracle.gret_recurrent(q[:, 17:], k[:, 17:], v[:, 17:], lg[:, 17:], state=s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], 1), o_all, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(s2, s_all, rtol=1e-11, atol=1e-11)
    # and the decay applies to the state before the token's own k^T v is added
    o_first, _ = oracle.gret_recurrent(q[:, :1], k[:, :1], v[:, :1], lg[:, :1])
    np.testing.assert_allclose(o_first[:, 0], (1.0 / np.sqrt(D)) * np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0])[..., None]
                               * v[:, 0], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- 8-bit K/V
def test_quantize_i8_worked_example():
    # absmax 2.54 -> scale 0.02; 1.0 -> 50, -2.54 -> -127, 2.54 -> 127
    x = np.array([[[1.0, -2.54, 0.01, 0.03, 2.54, -0.05]]], dtype=np.float32)
    codes, scales = oracle.quantize_kv_i8(x)
    s = np.float32(np.float32(2.54) / np.float32(127.0))
    assert scales[0, 0] == s
    expect = np.rint((x[0, 0] / s).astype(np.float32)).astype(np.int8)
    np.testing.assert_array_equal(codes[0, 0], expect)
    assert codes[0, 0, 1] == -127 and codes[0, 0, 4] == 127 and codes[0, 0, 0] == 50


def test_quantize_i8_bounds_and_round_trip():
    x = _rand((50, 8, 128), 960).astype(np.float32) * 3.0
    x[3, 2] = 0.0                                    # an all-zero head row
    codes, scales = oracle.quantize_kv_i8(x)
    assert codes.dtype == np.int8 and codes.min() >= -127 and codes.max() <= 127
    assert scales[3, 2] == 0 and not codes[3, 2].any()
    # the largest magnitude of every head row maps to +-127
    amax_idx = np.argmax(np.abs(x), axis=-1)
    top = np.take_along_axis(codes, amax_idx[..., None], -1)[..., 0]
    nz = scales > 0
    assert np.all(np.abs(top[nz]) == 127)
    # round trip within half a step (plus fp32 rounding of the step)
    err = np.abs(oracle.dequantize_kv_i8(codes, scales) - x)
    assert np.all(err <= 0.5 * scales[..., None] * (1 + 1e-6) + 1e-12)
    # and the step really is absmax / 127
    np.testing.assert_allclose(scales, np.abs(x).max(-1) / 127.0, rtol=1e-6)
