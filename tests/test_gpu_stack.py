"""The small YOCO++ attention stack end to end on the GPU (fp32, B=1,
T=256 + 16 decode steps, d=256, 4 query / 2 KV heads, head_dim 64, two
sliding-window self layers with window 32 and a w=0.5 blend on layer 2, two
cross layers over one global KV), against the oracle's stack.

Prefill covers rows 0..255; each decode step t runs one token through every
layer (ring write + window read, global-KV append, cross decode over the
whole cache) and must reproduce row t of the oracle's 272-row run -- the
decode == prefill-row invariant of the method (rows depend only on earlier
rows), and the reason early exit is exact.

In bf16 the stack stores every intermediate in bf16; its outputs are checked
stage by stage against a float64 model that rounds at the same points
(tests/stack_model.py) at the bf16 bar, and end to end against the
unrounded oracle within bounds derived from that model."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests import stack_model as sm
from tests.util import BF16_MAX_ABS, BF16_REL_L2, assert_close, errors, to_np

pytestmark = pytest.mark.gpu


def gpu_stack(yoco, x, w, cfg):
    T, nd, Hq, Hkv, D, W = cfg.T, cfg.n_decode, cfg.Hq, cfg.Hkv, cfg.D, cfg.window
    dev = x.device
    out = {"self_k": [], "self_v": [], "self_o": [], "cross_o": []}
    xs = x[:T].contiguous()
    rings = []
    kb = vb = None
    for l in range(cfg.n_self):
        q = yoco.linear(xs, w["self_q"][l], apply_ln=True)
        if l == 0:
            k, v = yoco.kv_project_blend(xs, w["self_kv"][l], Hkv, D)
            kb, vb = k, v
        else:
            k, v = yoco.kv_project_blend(xs, w["self_kv"][l], Hkv, D, kb, vb,
                                         cfg.w_blend[l], cfg.w_blend[l])
        ring = (torch.empty((1, W, Hkv, D), dtype=x.dtype, device=dev),
                torch.empty((1, W, Hkv, D), dtype=x.dtype, device=dev),
                torch.empty((1, W), dtype=torch.int32, device=dev))
        rings.append(ring)
        o = yoco.swa_prefill(q.view(1, T, Hq, D), k.view(1, T, Hkv, D), v.view(1, T, Hkv, D), W,
                             ring=ring)
        xs = yoco.linear(o.view(T, Hq * D), w["self_o"][l], base=xs, base_w=1.0)
        out["self_k"].append(k); out["self_v"].append(v); out["self_o"].append(o[0])
    kg = torch.zeros((T + nd, Hkv, D), dtype=x.dtype, device=dev)
    vg = torch.zeros((T + nd, Hkv, D), dtype=x.dtype, device=dev)
    yoco.kv_project_blend(xs, w["g_kv"], Hkv, D, k_out=kg, v_out=vg)
    for c in range(cfg.n_cross):
        q = yoco.linear(xs, w["cross_q"][c], apply_ln=True)
        o = yoco.cross_prefill(q.view(1, T, Hq, D), kg[:T].view(1, T, Hkv, D),
                               vg[:T].view(1, T, Hkv, D))
        xs = yoco.linear(o.view(T, Hq * D), w["cross_o"][c], base=xs, base_w=1.0)
        out["cross_o"].append(o[0])
    out["x_prefill"] = xs
    x_dec = []
    seq_start = torch.zeros(1, dtype=torch.int64, device=dev)
    for t in range(T, T + nd):
        xt = x[t:t + 1].contiguous()
        pos = torch.tensor([t], dtype=torch.int64, device=dev)
        kb_t = vb_t = None
        for l in range(cfg.n_self):
            q = yoco.linear(xt, w["self_q"][l], apply_ln=True)
            if l == 0:
                kn, vn = yoco.kv_project_blend(xt, w["self_kv"][l], Hkv, D)
                kb_t, vb_t = kn, vn
            else:
                kn, vn = yoco.kv_project_blend(xt, w["self_kv"][l], Hkv, D, kb_t, vb_t,
                                               cfg.w_blend[l], cfg.w_blend[l])
            rk, rv, sp = rings[l]
            o = yoco.swa_decode(q.view(1, Hq, D), kn.view(1, Hkv, D), vn.view(1, Hkv, D), pos,
                                rk, rv, sp, W)
            xt = yoco.linear(o.view(1, Hq * D), w["self_o"][l], base=xt, base_w=1.0)
        yoco.kv_project_blend(xt, w["g_kv"], Hkv, D, dst_rows=pos, k_out=kg, v_out=vg)
        seq_len = torch.tensor([t + 1], dtype=torch.int32, device=dev)
        for c in range(cfg.n_cross):
            q = yoco.linear(xt, w["cross_q"][c], apply_ln=True)
            o = yoco.cross_decode(q.view(1, Hq, D), kg, vg, seq_start, seq_len, T + nd)
            xt = yoco.linear(o.view(1, Hq * D), w["cross_o"][c], base=xt, base_w=1.0)
        x_dec.append(xt[0])
    out["x_decode"] = torch.stack(x_dec)
    out["k_g"], out["v_g"] = kg, vg
    return out


def _close_to_bf16_steps(got, ref, what, steps=1):
    """The bf16 bar for a stored bf16 tensor whose values reach past 4 (the
    residual stream x, |x| up to ~6; K and V): where one bf16 step exceeds
    2e-2 a value may sit one step (2^-7 |value| at most) from the
    reference's for each bf16 rounding on its path that can land on the other
    side of a boundary, so max-abs allows 2e-2 plus `steps` steps; rel-L2
    stays 5e-3."""
    g, r = to_np(got), to_np(ref)
    assert np.all(np.isfinite(g)), what
    excess = float(np.max(np.abs(g - r) - steps * 2.0 ** -7 * np.abs(r)))
    _, rl = errors(g, r)
    assert excess <= BF16_MAX_ABS and rl <= BF16_REL_L2, f"{what}: excess {excess:.3e}, rel_l2 {rl:.3e}"


def _check_against_rounding_model(got, x, w, cfg):
    """Stage by stage against the float64 model that rounds to bf16 where the
    GPU stores bf16: only the kernels' own arithmetic differs, so every stored
    tensor meets the bf16 bar (2e-2, 5e-3), its max-abs part widened by one
    bf16 step where the values reach 4 and a step exceeds 2e-2 (K, V and x
    have such values; a value next to a rounding boundary lands one step
    apart)."""
    T = cfg.T
    m = sm.stack(x, w, cfg)
    for key in ("self_k", "self_v", "self_o", "cross_o"):
        for l in range(len(m[key])):
            _close_to_bf16_steps(got[key][l], m[key][l][:T], f"{key}{l} vs rounding model")
    _close_to_bf16_steps(got["k_g"], m["k_g"], "k_g vs rounding model")
    _close_to_bf16_steps(got["v_g"], m["v_g"], "v_g vs rounding model")
    # x after the stack went through one bf16 rounding per residual addition
    n_add = cfg.n_self + cfg.n_cross
    _close_to_bf16_steps(got["x_prefill"], m["x"][:T], "x prefill vs rounding model", n_add)
    _close_to_bf16_steps(got["x_decode"], m["x"][T:], "x decode vs rounding model", n_add)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_tiny_stack_prefill_and_decode(cuda_lib, dtype):
    cfg = wl.TinyStack()
    x, w = wl.tiny_stack_inputs(cfg, dtype)
    ref = oracle.tiny_stack(x, w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.w_blend)
    wc = {k: ([t.cuda() for t in v] if isinstance(v, list) else v.cuda()) for k, v in w.items()}
    got = gpu_stack(cuda_lib, x.cuda(), wc, cfg)
    T = cfg.T
    if dtype == torch.float32:
        tol = dict(max_abs=2e-3, rel_l2=2e-5)
    else:
        # against the unrounded oracle: the bf16 storage of every intermediate
        # costs up to half of these bounds by itself (tests/stack_model.py)
        tol = dict(max_abs=sm.BF16_STACK_MAX_ABS, rel_l2=sm.BF16_STACK_REL_L2)
        _check_against_rounding_model(got, x, w, cfg)
    for l in range(cfg.n_self):
        assert_close(got["self_k"][l], ref["self_k"][l][:T], dtype, f"self_k{l}", **tol)
        assert_close(got["self_v"][l], ref["self_v"][l][:T], dtype, f"self_v{l}", **tol)
        assert_close(got["self_o"][l], ref["self_o"][l][:T], dtype, f"self_o{l}", **tol)
    assert_close(got["k_g"], ref["k_g"], dtype, "k_g", **tol)
    assert_close(got["v_g"], ref["v_g"], dtype, "v_g", **tol)
    for c in range(cfg.n_cross):
        assert_close(got["cross_o"][c], ref["cross_o"][c][:T], dtype, f"cross_o{c}", **tol)
    assert_close(got["x_prefill"], ref["x"][:T], dtype, "x prefill", **tol)
    assert_close(got["x_decode"], ref["x"][T:], dtype, "x decode", **tol)


def gpu_early_exit(yoco, x, w, cfg):
    """Early-exit prefill on the GPU: the self-decoder and the global K/V over
    all T prompt rows, then only row T-1 through the cross layers, each a
    cross decode of that row over the whole global K/V."""
    T, Hq, Hkv, D, W = cfg.T, cfg.Hq, cfg.Hkv, cfg.D, cfg.window
    dev = x.device
    xs = x[:T].contiguous()
    kb = vb = None
    for l in range(cfg.n_self):
        q = yoco.linear(xs, w["self_q"][l], apply_ln=True)
        if l == 0:
            k, v = yoco.kv_project_blend(xs, w["self_kv"][l], Hkv, D)
            kb, vb = k, v
        else:
            k, v = yoco.kv_project_blend(xs, w["self_kv"][l], Hkv, D, kb, vb,
                                         cfg.w_blend[l], cfg.w_blend[l])
        o = yoco.swa_prefill(q.view(1, T, Hq, D), k.view(1, T, Hkv, D), v.view(1, T, Hkv, D), W)
        xs = yoco.linear(o.view(T, Hq * D), w["self_o"][l], base=xs, base_w=1.0)
    kg, vg = yoco.kv_project_blend(xs, w["g_kv"], Hkv, D)
    xt = xs[T - 1:T].contiguous()
    seq_start = torch.zeros(1, dtype=torch.int64, device=dev)
    seq_len = torch.tensor([T], dtype=torch.int32, device=dev)
    for c in range(cfg.n_cross):
        q = yoco.linear(xt, w["cross_q"][c], apply_ln=True)
        o = yoco.cross_decode(q.view(1, Hq, D), kg, vg, seq_start, seq_len, T)
        xt = yoco.linear(o.view(1, Hq * D), w["cross_o"][c], base=xt, base_w=1.0)
    return xt[0]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_tiny_stack_early_exit(cuda_lib, dtype):
    # the last prompt row through the cross layers alone equals the full
    # prefill's last row: against the oracle's early exit, and against the
    # GPU's own full prefill
    cfg = wl.TinyStack()
    x, w = wl.tiny_stack_inputs(cfg, dtype)
    T = cfg.T
    ref = oracle.tiny_stack_early_exit(x[:T], w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.w_blend)
    wc = {k: ([t.cuda() for t in v] if isinstance(v, list) else v.cuda()) for k, v in w.items()}
    got = gpu_early_exit(cuda_lib, x.cuda(), wc, cfg)
    full = gpu_stack(cuda_lib, x.cuda(), wc, cfg)["x_prefill"][T - 1]
    if dtype == torch.float32:
        tol = dict(max_abs=2e-3, rel_l2=2e-5)
        assert_close(got, full.float().cpu().numpy(), dtype, "early exit vs full prefill", **tol)
    else:
        tol = dict(max_abs=sm.BF16_STACK_MAX_ABS, rel_l2=sm.BF16_STACK_REL_L2)
        # the residual stream at the bf16 bar, scaled to x's magnitude
        n_add = cfg.n_self + cfg.n_cross
        _close_to_bf16_steps(got, sm.stack(x[:T], w, cfg, early_exit=True), "early exit vs rounding model", n_add)
        _close_to_bf16_steps(got, full.float().cpu().numpy(), "early exit vs full prefill", n_add)
    assert_close(got, ref, dtype, "early exit vs oracle", **tol)
