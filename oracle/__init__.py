"""CPU fp64 oracle for the YOCO / YOCO++ attention core.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product library never imports,
links or executes anything here, and this package imports nothing from it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over query rows
and heads).  This module marshals numpy arrays and composes the tiny
attention stack from those C functions.  Inputs are first rounded to the
storage dtype by the caller (they are generated as bf16 / fp32 tensors) and
then widened to fp64 here.

Sources: "You Only Cache Once: Decoder-Decoder Architectures for Language
Models" (paperlayer summary of arXiv 2405.05254v2), sections 1-3; the YOCO
podcast transcript, cues 12 and 26; "YOCO++: Enhancing YOCO with KV Residual
Connections for Efficient LLM Inference", Abstract.

Parity pins: every function here is pinned in tests/test_oracle_pins.py
against library routines (torch fp64 scaled_dot_product_attention, numpy
matmul), closed forms and invariants; none is "parity unpinned".
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_LIB = None
_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)
_I32 = ctypes.POINTER(ctypes.c_int32)


def load(path):
    """Load an oracle shared library from path and declare its signatures."""
    L = ctypes.CDLL(path)
    i64, dbl, i32 = ctypes.c_int64, ctypes.c_double, ctypes.c_int
    L.oracle_layernorm.argtypes = [_D, i64, i64, dbl, _D]
    L.oracle_project.argtypes = [_D, i64, i64, _D, i64, i32, dbl, _D]
    L.oracle_blend.argtypes = [_D, _D, i64, dbl, _D]
    L.oracle_attention.argtypes = [_D, _D, _D, i64, i64, i64, i64, i64, i64, i64, i64,
                                   dbl, _D, _D]
    L.oracle_attention_rows.argtypes = [_D, _D, _D, i64, i64, i64, i64, i64, i64, i64,
                                        i64, dbl, _I64, _I64, i64, _D, _D]
    L.oracle_cross_decode.argtypes = [_D, _D, _D, _I64, _I64, i64, i64, i64, i64, dbl,
                                      _D, _D]
    L.oracle_ring_prefill_slots.argtypes = [i64, i64, _I32]
    L.oracle_ring_push.argtypes = [_D, _D, _I32, i64, i64, i64, i64, _D, _D]
    L.oracle_swa_decode_ring.argtypes = [_D, _D, _D, _I32, i64, i64, i64, i64, i64, dbl,
                                         _D, _D]
    L.oracle_cache_bytes_yoco.argtypes = [i64, i64, i64, i64, i64, i64]
    L.oracle_cache_bytes_yoco.restype = dbl
    L.oracle_cache_bytes_transformer.argtypes = [i64, i64, i64, i64, i64]
    L.oracle_cache_bytes_transformer.restype = dbl
    L.oracle_visibility.argtypes = [i64, i64, i64, i64, ctypes.POINTER(ctypes.c_uint8)]
    L.oracle_gret_log_decay.argtypes = [_D, i64, dbl, _D]
    L.oracle_gret_recurrent.argtypes = [_D, _D, _D, _D, i64, i64, i64, i64, dbl, _D, _D]
    L.oracle_gret_parallel.argtypes = [_D, _D, _D, _D, i64, i64, i64, i64, dbl, _D, _D]
    L.oracle_gret_chunkwise.argtypes = [_D, _D, _D, _D, i64, i64, i64, i64, dbl, i64, _D, _D]
    L.oracle_num_threads.restype = i32
    L.oracle_set_num_threads.argtypes = [i32]
    return L


def lib():
    global _LIB
    if _LIB is None:
        _LIB = load(_build.build())
    return _LIB


def _f64(a):
    """Widen any array-like (numpy or torch CPU tensor) to contiguous fp64."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch
        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a, t=_D):
    return a.ctypes.data_as(t) if a is not None else None


def num_threads():
    return int(lib().oracle_num_threads())


def set_num_threads(n):
    lib().oracle_set_num_threads(int(n))


def default_scale(D):
    return 1.0 / math.sqrt(D)


def layernorm(x, eps=1e-5):
    x = _f64(x)
    n, d = x.shape
    out = np.empty_like(x)
    lib().oracle_layernorm(_p(x), n, d, eps, _p(out))
    return out


def project(x, w, apply_ln=True, eps=1e-5):
    """N(x) . W^T with W [m, d] (one output feature per row)."""
    x, w = _f64(x), _f64(w)
    n, d = x.shape
    m, d2 = w.shape
    assert d == d2
    out = np.empty((n, m), dtype=np.float64)
    lib().oracle_project(_p(x), n, d, _p(w), m, int(bool(apply_ln)), eps, _p(out))
    return out


def blend(a, base, w):
    """YOCO++ weighted residual: a + w * base."""
    a, base = _f64(a), _f64(base)
    assert a.shape == base.shape
    out = np.empty_like(a)
    lib().oracle_blend(_p(a), _p(base), a.size, float(w), _p(out))
    return out


def kv_project_blend(x, w_kv, Hkv, D, k_base=None, v_base=None, w_k=0.0, w_v=0.0,
                     apply_ln=True, eps=1e-5):
    """K/V producer of one self-decoder layer (or the global KV when no base):
    [K | V] = N(x) . W_kv^T, then K += w_k * K_base, V += w_v * V_base.
    Returns K, V as [n, Hkv, D]."""
    kv = project(x, w_kv, apply_ln, eps)
    n = kv.shape[0]
    k = kv[:, : Hkv * D].reshape(n, Hkv, D).copy()
    v = kv[:, Hkv * D:].reshape(n, Hkv, D).copy()
    if k_base is not None:
        k = blend(k, _f64(k_base).reshape(n, Hkv, D), w_k)
    if v_base is not None:
        v = blend(v, _f64(v_base).reshape(n, Hkv, D), w_v)
    return k, v


def visibility(Tq, Tkv, q_pos0=0, window=0):
    """Boolean [Tq, Tkv]: key j visible to query row i at absolute position
    q_pos0 + i (causal; within the window when window > 0)."""
    out = np.zeros((Tq, Tkv), dtype=np.uint8)
    lib().oracle_visibility(Tq, Tkv, q_pos0, window, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    return out.astype(bool)


def attention(q, k, v, q_pos0=0, window=0, scale=None, rows=None):
    """Causal (window <= 0) or sliding-window GQA attention.

    q [B, Tq, Hq, D]; k, v [B, Tkv, Hkv, D]; query row i sits at absolute
    position q_pos0 + i.  rows: optional list of (b, i) pairs; then returns
    o [n_rows, Hq, D], lse [n_rows, Hq], else o [B, Tq, Hq, D], lse [B, Tq, Hq].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Tq, Hq, D = q.shape
    B2, Tkv, Hkv, D2 = k.shape
    assert B == B2 and D == D2 and v.shape == k.shape and Hq % Hkv == 0
    if scale is None:
        scale = default_scale(D)
    if rows is None:
        o = np.empty_like(q)
        lse = np.empty((B, Tq, Hq), dtype=np.float64)
        lib().oracle_attention(_p(q), _p(k), _p(v), B, Tq, Tkv, Hq, Hkv, D, q_pos0, window,
                               scale, _p(o), _p(lse))
        return o, lse
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
    rb = np.ascontiguousarray(rows[:, 0])
    ri = np.ascontiguousarray(rows[:, 1])
    n = rows.shape[0]
    o = np.empty((n, Hq, D), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64)
    lib().oracle_attention_rows(_p(q), _p(k), _p(v), B, Tq, Tkv, Hq, Hkv, D, q_pos0, window,
                                scale, _p(rb, _I64), _p(ri, _I64), n, _p(o), _p(lse))
    return o, lse


def cross_decode(q, k_cache, v_cache, seq_start, seq_len, scale=None):
    """One decode step of a cross-decoder layer over a packed shared cache.
    q [B, Hq, D]; caches [rows, Hkv, D]; sequence b owns rows
    [seq_start[b], seq_start[b] + seq_len[b]).  Returns o [B, Hq, D], lse [B, Hq]."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Hq, D = q.shape
    rows, Hkv, D2 = kc.shape
    assert D == D2 and vc.shape == kc.shape
    ss = np.ascontiguousarray(np.asarray(seq_start, dtype=np.int64))
    sl = np.ascontiguousarray(np.asarray(seq_len, dtype=np.int64))
    assert np.all(sl >= 1) and np.all(ss + sl <= rows)
    if scale is None:
        scale = default_scale(D)
    o = np.empty_like(q)
    lse = np.empty((B, Hq), dtype=np.float64)
    lib().oracle_cross_decode(_p(q), _p(kc), _p(vc), _p(ss, _I64), _p(sl, _I64), B, Hq, Hkv,
                              D, scale, _p(o), _p(lse))
    return o, lse


def ring_prefill_slots(T, W):
    out = np.empty((W,), dtype=np.int32)
    lib().oracle_ring_prefill_slots(int(T), int(W), _p(out, _I32))
    return out


def ring_from_prefill(k, v, W):
    """Ring contents of one sequence after a prefill: k, v [T, Hkv, D] ->
    ring_k, ring_v [W, Hkv, D] (zeros in empty slots), slot_pos [W]."""
    k, v = _f64(k), _f64(v)
    T, Hkv, D = k.shape
    rk = np.zeros((W, Hkv, D))
    rv = np.zeros((W, Hkv, D))
    sp = np.full((W,), -1, dtype=np.int32)
    for p in range(T):
        lib().oracle_ring_push(_p(rk), _p(rv), _p(sp, _I32), W, Hkv, D, p,
                               _p(np.ascontiguousarray(k[p])), _p(np.ascontiguousarray(v[p])))
    return rk, rv, sp


def ring_push(ring_k, ring_v, slot_pos, pos, k_new, v_new):
    """In-place push of one token into one sequence's ring (fp64 arrays)."""
    W, Hkv, D = ring_k.shape
    kn, vn = _f64(k_new), _f64(v_new)
    lib().oracle_ring_push(_p(ring_k), _p(ring_v), _p(slot_pos, _I32), W, Hkv, D, int(pos),
                           _p(kn), _p(vn))


def swa_decode_ring(q, ring_k, ring_v, slot_pos, pos, scale=None):
    """q [Hq, D] at absolute position pos over one sequence's ring."""
    q = _f64(q)
    Hq, D = q.shape
    W, Hkv, _ = ring_k.shape
    if scale is None:
        scale = default_scale(D)
    o = np.empty_like(q)
    lse = np.empty((Hq,))
    sp = np.ascontiguousarray(slot_pos, dtype=np.int32)
    lib().oracle_swa_decode_ring(_p(q), _p(np.ascontiguousarray(ring_k)),
                                 _p(np.ascontiguousarray(ring_v)), _p(sp, _I32), W, Hq, Hkv, D,
                                 int(pos), scale, _p(o), _p(lse))
    return o, lse


def cache_bytes_yoco(L_self, window, N, Hkv, D, elem_bytes):
    return lib().oracle_cache_bytes_yoco(L_self, window, N, Hkv, D, elem_bytes)


def cache_bytes_transformer(L, N, Hkv, D, elem_bytes):
    return lib().oracle_cache_bytes_transformer(L, N, Hkv, D, elem_bytes)


# ------------------------------------------------------------- 8-bit K/V
def quantize_kv_i8(x):
    """Symmetric 8-bit quantisation of a K or V cache, one scale per (token,
    KV head) (the pages' "8-bit cache quantization", podcast cue 1; the scheme
    is not stated -- reading: absmax over the head's D values, scale =
    absmax / 127, code = round-half-even(x / scale) in [-127, 127]).

    x [rows, Hkv, D] (bf16 / fp32 tensor or array).  Every decision that
    yields an integer is taken in fp32 (IEEE division, round-half-even), the
    precision the kernel uses, so the codes are reproducible bit for bit.
    Returns (codes int8 [rows, Hkv, D], scales float32 [rows, Hkv])."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu", torch.float32).numpy()
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = np.rint((x / safe[..., None]).astype(np.float32))
    q = np.where(scale[..., None] > 0, q, 0.0)
    return np.clip(q, -127, 127).astype(np.int8), scale


def dequantize_kv_i8(codes, scales):
    """codes [rows, Hkv, D] int8, scales [rows, Hkv] -> fp64 values code * scale."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[..., None]


# ------------------------------------------------------------ gated retention
def gret_log_decay(g, tau):
    """log gamma = log(sigmoid(g)) / tau, elementwise (any shape)."""
    g = _f64(g)
    out = np.empty_like(g)
    lib().oracle_gret_log_decay(_p(g), g.size, float(tau), _p(out))
    return out


def _gret_args(q, k, v, log_gamma, scale, state):
    q, k, v, lg = _f64(q), _f64(k), _f64(v), _f64(log_gamma)
    B, T, H, D = q.shape
    assert k.shape == q.shape and v.shape == q.shape and lg.shape == (B, T, H)
    if scale is None:
        scale = default_scale(D)
    st = None if state is None else _f64(state).reshape(B, H, D, D).copy()
    return q, k, v, lg, B, T, H, D, scale, st


def gret_recurrent(q, k, v, log_gamma, scale=None, state=None):
    """Recurrent gated retention.  q, k, v [B, T, H, D]; log_gamma [B, T, H];
    state [B, H, D, D] initial state (None: zero).  Returns (o, final state)."""
    q, k, v, lg, B, T, H, D, scale, st = _gret_args(q, k, v, log_gamma, scale, state)
    if st is None:
        st = np.zeros((B, H, D, D))
    o = np.empty_like(q)
    lib().oracle_gret_recurrent(_p(q), _p(k), _p(v), _p(lg), B, T, H, D, scale, _p(st), _p(o))
    return o, st


def gret_parallel(q, k, v, log_gamma, scale=None, state=None):
    """Parallel gated retention (the same function as gret_recurrent's o)."""
    q, k, v, lg, B, T, H, D, scale, st = _gret_args(q, k, v, log_gamma, scale, state)
    o = np.empty_like(q)
    lib().oracle_gret_parallel(_p(q), _p(k), _p(v), _p(lg), B, T, H, D, scale, _p(st), _p(o))
    return o


def gret_chunkwise(q, k, v, log_gamma, chunk, scale=None, state=None):
    """Chunkwise gated retention with chunks of `chunk` tokens.  Returns
    (o, final state)."""
    q, k, v, lg, B, T, H, D, scale, st = _gret_args(q, k, v, log_gamma, scale, state)
    if st is None:
        st = np.zeros((B, H, D, D))
    o = np.empty_like(q)
    lib().oracle_gret_chunkwise(_p(q), _p(k), _p(v), _p(lg), B, T, H, D, scale, int(chunk), _p(st), _p(o))
    return o, st


def _self_decoder(x, weights, Hq, Hkv, D, window, w_blend, eps, out):
    """Self-decoder layers over every row of x, then the global K/V (see
    tiny_stack); fills out and returns (x, k_g, v_g)."""
    T = x.shape[0]
    k_bottom = v_bottom = None
    for l in range(len(weights["self_q"])):
        q = project(x, weights["self_q"][l], True, eps).reshape(1, T, Hq, D)
        if l == 0:
            k, v = kv_project_blend(x, weights["self_kv"][l], Hkv, D, eps=eps)
            k_bottom, v_bottom = k, v
        else:
            k, v = kv_project_blend(x, weights["self_kv"][l], Hkv, D, k_bottom, v_bottom,
                                    w_blend[l], w_blend[l], eps=eps)
        o, _ = attention(q, k.reshape(1, T, Hkv, D), v.reshape(1, T, Hkv, D), 0, window)
        x = x + project(o.reshape(T, Hq * D), weights["self_o"][l], False)
        out["self_q"].append(q.reshape(T, Hq, D))
        out["self_k"].append(k)
        out["self_v"].append(v)
        out["self_o"].append(o.reshape(T, Hq, D))
        out["x_self"].append(x.copy())
    kg, vg = kv_project_blend(x, weights["g_kv"], Hkv, D, eps=eps)
    out["k_g"], out["v_g"] = kg, vg
    return x, kg, vg


def tiny_stack(x, weights, Hq, Hkv, D, window, w_blend, eps=1e-5):
    """The small YOCO++ attention stack, end to end, for every row of x.

    x [T, d]; weights: dict with per-layer lists
      'self_q', 'self_kv', 'self_o'  (one entry per self-decoder layer),
      'g_kv'                          (global KV producer),
      'cross_q', 'cross_o'            (one entry per cross-decoder layer);
    projection weights are [out_features, in_features].
    w_blend[l] is the YOCO++ residual weight of self layer l (layer 0 is the
    bottom layer and is never blended).  Returns a dict of every intermediate.

    Self-decoder layer: h = LN(x); q, k, v from h; k, v blended with the
    bottom layer's k, v; x += SWA(q, k, v) W_o (podcast cue 12; the feed-
    forward sub-layer is outside the attention core and omitted).
    Global KV: K_g, V_g = LN(x) W_kv^g, produced once.
    Cross-decoder layer: q = LN(x) W_q; x += CausalAttn(q, K_g, V_g) W_o.
    """
    x = _f64(x).copy()
    T, d = x.shape
    out = {"self_q": [], "self_k": [], "self_v": [], "self_o": [], "x_self": [],
           "cross_q": [], "cross_o": [], "x_cross": []}
    x, kg, vg = _self_decoder(x, weights, Hq, Hkv, D, window, w_blend, eps, out)
    for c in range(len(weights["cross_q"])):
        q = project(x, weights["cross_q"][c], True, eps).reshape(1, T, Hq, D)
        o, _ = attention(q, kg.reshape(1, T, Hkv, D), vg.reshape(1, T, Hkv, D), 0, 0)
        x = x + project(o.reshape(T, Hq * D), weights["cross_o"][c], False)
        out["cross_q"].append(q.reshape(T, Hq, D))
        out["cross_o"].append(o.reshape(T, Hq, D))
        out["x_cross"].append(x.copy())
    out["x"] = x
    return out


def tiny_stack_early_exit(x, weights, Hq, Hkv, D, window, w_blend, eps=1e-5):
    """Early-exit prefill of the same stack ("You Only Cache Once", paperlayer
    summary, section 2, and podcast transcript, the Figure 3 discussion): the
    self-decoder runs over every prompt row and writes the global K/V, and only
    the LAST row goes through the cross-decoder, each cross layer attending
    from that row to the whole global K/V.  Returns the last row's final x [d]."""
    x = _f64(x).copy()
    T, d = x.shape
    out = {"self_q": [], "self_k": [], "self_v": [], "self_o": [], "x_self": []}
    x, kg, vg = _self_decoder(x, weights, Hq, Hkv, D, window, w_blend, eps, out)
    xt = x[T - 1:T].copy()
    for c in range(len(weights["cross_q"])):
        q = project(xt, weights["cross_q"][c], True, eps).reshape(1, Hq, D)
        o, _ = cross_decode(q, kg, vg, [0], [T])
        xt = xt + project(o.reshape(1, Hq * D), weights["cross_o"][c], False)
    return xt[0]
