"""Python binding of libyoco.so, the B200 (sm_100a) attention core of the
YOCO / YOCO++ decoder-decoder architecture.

Argument marshalling only: every function passes torch CUDA tensors as raw
device pointers, plus the current CUDA stream, to the C ABI declared in
include/yoco.h, and raises YocoError on a non-OK status.  Every computation
runs in the library's CUDA kernels; there is no CPU or PyTorch fallback, and
importing a function fails loudly when libyoco.so is missing.

Entry points (same names as the C ABI, without the ``yoco_`` prefix):
kv_project_blend, swa_prefill, swa_decode, cross_prefill, cross_decode,
attention_prefill,
gret_prefill, gret_decode, kv_quantize_i8, cross_decode_i8,
plus linear, workspace sizes, cache_bytes, device_status and the test-only
debug_tile_schedule.
"""
import ctypes
import os

import torch

__all__ = ["YocoError", "load", "lib_path", "kv_project_blend", "linear", "swa_prefill",
           "swa_decode", "swa_decode_step", "swa_decode_step_workspace_size", "cross_prefill",
           "cross_decode", "cross_decode_workspace_size",
           "swa_decode_workspace_size", "cache_bytes", "device_status", "launch_count", "AttnCfg",
           "debug_tile_schedule", "SCHEDULE_PREFILL", "SCHEDULE_DECODE", "gret_prefill", "gret_decode",
           "kv_i8_row_bytes", "kv_quantize_i8", "cross_decode_i8",
           "attention_prefill", "debug_exp2_poly", "gret_prefill_workspace_size"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE, ERR_TIMEOUT = range(6)
BF16, FP32 = 0, 1
SCHEDULE_PREFILL, SCHEDULE_DECODE = 0, 1
_DT = {torch.bfloat16: BF16, torch.float32: FP32}


class YocoError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = _LIB.yoco_status_string(status).decode() if _LIB is not None else str(status)
        super().__init__(f"{where}: {msg} (status {status})")


class AttnCfg(ctypes.Structure):
    _fields_ = [("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int32)]


def lib_path():
    return os.path.join(_HERE, "libyoco.so")


def load():
    """Load libyoco.so (built in-tree by shared_kv_decoder_b200.build)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"libyoco.so not found at {path}; build it with "
                           "`python -m shared_kv_decoder_b200.build`")
    L = ctypes.CDLL(path)
    vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
    cfgp = ctypes.POINTER(AttnCfg)
    st = ctypes.c_int
    sigs = {
        "yoco_kv_project_blend": (st, [vp, i64, i32, vp, i32, f32, vp, vp, f32, f32, vp, vp, vp,
                                       cfgp, vp]),
        "yoco_linear": (st, [vp, i64, i32, vp, i32, i32, f32, vp, f32, vp, i32, vp]),
        "yoco_swa_prefill": (st, [vp, vp, vp, i32, i64, i32, vp, vp, vp, vp, vp, cfgp, vp]),
        "yoco_swa_decode": (st, [vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, vp, sz, cfgp, vp]),
        "yoco_swa_decode_step": (st, [vp, i32, vp, i32, f32, vp, vp, f32, f32, vp, vp, i32, i32, vp, vp, vp,
                                      vp, vp, vp, vp, sz, cfgp, vp]),
        "yoco_swa_decode_step_workspace_size": (sz, [i32, i32, cfgp]),
        "yoco_cross_prefill": (st, [vp, vp, vp, i32, i64, i64, i64, vp, vp, cfgp, vp]),
        "yoco_attention_prefill": (st, [vp, vp, vp, i32, i64, i64, i64, i32, vp, vp, cfgp, vp]),
        "yoco_cross_decode": (st, [vp, vp, vp, i64, vp, vp, i32, i64, vp, vp, vp, sz, cfgp, vp]),
        "yoco_cross_decode_static": (st, [vp, vp, vp, i64, vp, vp, i32, i64, vp, vp, cfgp, vp]),
        "yoco_cross_decode_workspace_size": (sz, [i32, i64, cfgp]),
        "yoco_swa_decode_workspace_size": (sz, [i32, i32, cfgp]),
        "yoco_cache_bytes": (ctypes.c_double, [i32, i32, i64, cfgp]),
        "yoco_gret_prefill": (st, [vp, vp, vp, vp, i32, i64, f32, vp, vp, vp, sz, cfgp, vp]),
        "yoco_gret_prefill_workspace_size": (sz, [i32, i64, cfgp]),
        "yoco_kv_i8_row_bytes": (i64, [cfgp]),
        "yoco_kv_quantize_i8": (st, [vp, vp, i64, vp, vp, vp, cfgp, vp]),
        "yoco_cross_decode_i8": (st, [vp, vp, vp, i64, vp, vp, i32, i64, vp, vp, vp, sz, cfgp, vp]),
        "yoco_gret_decode": (st, [vp, vp, vp, vp, i32, f32, vp, vp, cfgp, vp]),
        "yoco_debug_tile_schedule": (st, [i32, cfgp, i32, i64, i64, i64, i32, vp, vp, i64, i32, vp,
                                          i64, ctypes.POINTER(ctypes.c_int64)]),
        "yoco_get_device_status": (st, [vp]),
        "yoco_debug_wait_timeout_probe": (st, [vp]),
        "yoco_debug_exp2_poly": (st, [vp, vp, i64, vp]),
        "yoco_status_string": (ctypes.c_char_p, [st]),
        "yoco_version": (ctypes.c_char_p, []),
        "yoco_launch_count": (ctypes.c_uint64, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = L
    return L


def _check(status, where):
    if status != OK:
        raise YocoError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("libyoco takes CUDA tensors only")
            if not t.is_contiguous():
                raise ValueError("libyoco takes contiguous tensors only")


def _cfg(Hq, Hkv, D, dtype, scale=0.0):
    return AttnCfg(int(Hq), int(Hkv), int(D), float(scale), _DT[dtype])


def kv_project_blend(x, w_kv, Hkv, D, k_base=None, v_base=None, w_k=0.0, w_v=0.0,
                     dst_rows=None, k_out=None, v_out=None, apply_ln=True, eps=1e-5):
    """[K | V] = LN(x) W_kv^T (+ w_k K_base, + w_v V_base), fused epilogue.
    x [n, d]; w_kv [2*Hkv*D, d]; bases [n, Hkv, D]; returns (k_out, v_out)."""
    L = load()
    n, d = x.shape
    if k_out is None:
        k_out = torch.empty((n, Hkv, D), dtype=x.dtype, device=x.device)
    if v_out is None:
        v_out = torch.empty((n, Hkv, D), dtype=x.dtype, device=x.device)
    _dev(x, w_kv, k_base, v_base, dst_rows, k_out, v_out)
    cfg = _cfg(Hkv, Hkv, D, x.dtype)
    _check(L.yoco_kv_project_blend(_ptr(x), n, d, _ptr(w_kv), int(bool(apply_ln)), eps,
                                   _ptr(k_base), _ptr(v_base), float(w_k), float(w_v),
                                   _ptr(dst_rows), _ptr(k_out), _ptr(v_out), ctypes.byref(cfg),
                                   _stream()), "yoco_kv_project_blend")
    return k_out, v_out


def linear(x, w, base=None, base_w=1.0, apply_ln=False, eps=1e-5, out=None):
    """out = N(x) W^T + base_w * base.  x [n, d_in]; w [d_out, d_in]."""
    L = load()
    n, d_in = x.shape
    d_out = w.shape[0]
    if out is None:
        out = torch.empty((n, d_out), dtype=x.dtype, device=x.device)
    _dev(x, w, base, out)
    _check(L.yoco_linear(_ptr(x), n, d_in, _ptr(w), d_out, int(bool(apply_ln)), eps, _ptr(base),
                         float(base_w), _ptr(out), _DT[x.dtype], _stream()), "yoco_linear")
    return out


def swa_prefill(q, k, v, window, ring=None, want_lse=False, scale=0.0, o=None):
    """Sliding-window prefill.  q [B, T, Hq, D]; k, v [B, T, Hkv, D].
    ring: None, or a tuple (ring_k, ring_v, slot_pos) to fill.
    Returns o (and lse [B, Hq, T] when want_lse)."""
    L = load()
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    if o is None:
        o = torch.empty_like(q)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device) if want_lse else None
    rk, rv, sp = ring if ring is not None else (None, None, None)
    _dev(q, k, v, o, lse, rk, rv, sp)
    cfg = _cfg(Hq, Hkv, D, q.dtype, scale)
    _check(L.yoco_swa_prefill(_ptr(q), _ptr(k), _ptr(v), B, T, int(window), _ptr(o), _ptr(lse),
                              _ptr(rk), _ptr(rv), _ptr(sp), ctypes.byref(cfg), _stream()),
           "yoco_swa_prefill")
    return (o, lse) if want_lse else o


def swa_decode_workspace_size(B, window, Hq, Hkv, D, dtype):
    cfg = _cfg(Hq, Hkv, D, dtype)
    return int(load().yoco_swa_decode_workspace_size(B, window, ctypes.byref(cfg)))


def swa_decode(q, k_new, v_new, pos, ring_k, ring_v, slot_pos, window, workspace=None,
               scale=0.0, o=None):
    """One sliding-window decode step.  q [B, Hq, D]; k_new, v_new [B, Hkv, D];
    pos int64 [B]; ring_k, ring_v [B, window, Hkv, D]; slot_pos int32 [B, window]."""
    L = load()
    B, Hq, D = q.shape
    Hkv = k_new.shape[1]
    if workspace is None:
        workspace = torch.empty(swa_decode_workspace_size(B, window, Hq, Hkv, D, q.dtype),
                                dtype=torch.uint8, device=q.device)
    if o is None:
        o = torch.empty_like(q)
    _dev(q, k_new, v_new, pos, ring_k, ring_v, slot_pos, o, workspace)
    cfg = _cfg(Hq, Hkv, D, q.dtype, scale)
    _check(L.yoco_swa_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(pos), B, int(window),
                             _ptr(ring_k), _ptr(ring_v), _ptr(slot_pos), _ptr(o), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), ctypes.byref(cfg),
                             _stream()), "yoco_swa_decode")
    return o


def swa_decode_step_workspace_size(B, window, Hq, Hkv, D, dtype):
    cfg = _cfg(Hq, Hkv, D, dtype)
    return int(load().yoco_swa_decode_step_workspace_size(B, window, ctypes.byref(cfg)))


def swa_decode_step(x, w_kv, q, pos, ring_k, ring_v, slot_pos, window, k_base=None, v_base=None,
                    w_k=0.0, w_v=0.0, apply_ln=True, eps=1e-5, o=None, k_out=None, v_out=None,
                    workspace=None, scale=0.0):
    """One self-decoder decode step: kv_project_blend of the B new tokens, then
    swa_decode with that K/V.  x [B, d]; w_kv [2*Hkv*D, d]; q [B, Hq, D];
    pos int64 [B]; ring_k, ring_v [B, window, Hkv, D]; slot_pos int32 [B, window];
    k_out / v_out [B, Hkv, D] (optional) receive the blended new K / V."""
    L = load()
    B, Hq, D = q.shape
    Hkv = ring_k.shape[2]
    d = x.shape[1]
    if workspace is None:
        workspace = torch.empty(swa_decode_step_workspace_size(B, window, Hq, Hkv, D, q.dtype),
                                dtype=torch.uint8, device=q.device)
    if o is None:
        o = torch.empty_like(q)
    _dev(x, w_kv, q, pos, ring_k, ring_v, slot_pos, k_base, v_base, o, k_out, v_out, workspace)
    cfg = _cfg(Hq, Hkv, D, q.dtype, scale)
    _check(L.yoco_swa_decode_step(_ptr(x), d, _ptr(w_kv), int(bool(apply_ln)), eps, _ptr(k_base),
                                  _ptr(v_base), float(w_k), float(w_v), _ptr(q), _ptr(pos), B, int(window),
                                  _ptr(ring_k), _ptr(ring_v), _ptr(slot_pos), _ptr(o), _ptr(k_out),
                                  _ptr(v_out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  ctypes.byref(cfg), _stream()), "yoco_swa_decode_step")
    return o


def cross_prefill(q, k, v, q_pos0=0, want_lse=False, scale=0.0, o=None):
    """Causal cross-attention over the shared KV.  q [B, Tq, Hq, D];
    k, v [B, Tkv, Hkv, D]; query row i at absolute position q_pos0 + i."""
    L = load()
    B, Tq, Hq, D = q.shape
    Tkv, Hkv = k.shape[1], k.shape[2]
    if o is None:
        o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device) if want_lse else None
    _dev(q, k, v, o, lse)
    cfg = _cfg(Hq, Hkv, D, q.dtype, scale)
    _check(L.yoco_cross_prefill(_ptr(q), _ptr(k), _ptr(v), B, Tq, Tkv, int(q_pos0), _ptr(o),
                                _ptr(lse), ctypes.byref(cfg), _stream()), "yoco_cross_prefill")
    return (o, lse) if want_lse else o


def cross_decode_workspace_size(B, max_len, Hq, Hkv, D, dtype):
    cfg = _cfg(Hq, Hkv, D, dtype)
    return int(load().yoco_cross_decode_workspace_size(B, max_len, ctypes.byref(cfg)))


def cross_decode(q, k_cache, v_cache, seq_start, seq_len, max_len, workspace=None,
                 want_lse=False, scale=0.0, o=None):
    """One cross-decoder decode step over the packed shared cache.
    q [B, Hq, D]; caches [rows, Hkv, D]; seq_start int64 [B]; seq_len int32 [B]."""
    L = load()
    B, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must have the same shape")
    if workspace is None:
        workspace = torch.empty(cross_decode_workspace_size(B, max_len, Hq, Hkv, D, q.dtype),
                                dtype=torch.uint8, device=q.device)
    if o is None:
        o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if want_lse else None
    _dev(q, k_cache, v_cache, seq_start, seq_len, o, lse, workspace)
    cfg = _cfg(Hq, Hkv, D, q.dtype, scale)
    _check(L.yoco_cross_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), k_cache.shape[0], _ptr(seq_start),
                               _ptr(seq_len), B, int(max_len), _ptr(o), _ptr(lse),
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               ctypes.byref(cfg), _stream()), "yoco_cross_decode")
    return (o, lse) if want_lse else o


def cache_bytes(L_self, window, N, Hkv, D, dtype=torch.bfloat16):
    cfg = _cfg(Hkv, Hkv, D, dtype)
    return float(load().yoco_cache_bytes(L_self, window, N, ctypes.byref(cfg)))


def launch_count():
    """Kernels launched by the library so far in this process."""
    return int(load().yoco_launch_count())


def device_status():
    """Synchronise the current stream and return the device status code."""
    return int(load().yoco_get_device_status(_stream()))


def debug_tile_schedule(kind, Hq, Hkv, D, dtype=torch.bfloat16, B=1, Tq=0, Tkv=0, q_pos0=0, window=0,
                        seq_start=None, seq_len=None, max_len=1, n_cta=0):
    """The kernels' work plan, computed on the host (test-only; see
    yoco_debug_tile_schedule).  Returns an int64 numpy array [n, 6]:
    prefill {cta, b, head, query tile, KV tile, masked};
    decode {cta, b, split, first row, tokens, stages}.  seq_start / seq_len
    are host sequences (decode only)."""
    import numpy as np
    L = load()
    cfg = _cfg(Hq, Hkv, D, dtype)
    ss = sl = None
    if kind == SCHEDULE_DECODE:
        ss = np.ascontiguousarray(np.asarray(seq_start, dtype=np.int64))
        sl = np.ascontiguousarray(np.asarray(seq_len, dtype=np.int32))
    n = ctypes.c_int64(0)
    args = lambda rec, cap: (int(kind), ctypes.byref(cfg), int(B), int(Tq), int(Tkv), int(q_pos0),
                             int(window), None if ss is None else ss.ctypes.data_as(ctypes.c_void_p),
                             None if sl is None else sl.ctypes.data_as(ctypes.c_void_p), int(max_len),
                             int(n_cta), rec, cap, ctypes.byref(n))
    _check(L.yoco_debug_tile_schedule(*args(None, 0)), "yoco_debug_tile_schedule")
    out = np.zeros((n.value, 6), dtype=np.int64)
    _check(L.yoco_debug_tile_schedule(*args(out.ctypes.data_as(ctypes.c_void_p), n.value)),
           "yoco_debug_tile_schedule")
    return out


def gret_prefill_workspace_size(B, T, H, D, dtype=torch.bfloat16):
    cfg = _cfg(H, H, D, dtype)
    return int(load().yoco_gret_prefill_workspace_size(B, int(T), ctypes.byref(cfg)))


def gret_prefill(q, k, v, g, tau, state=None, scale=0.0, o=None, workspace="auto"):
    """Chunkwise gated retention over a prompt.  q, k, v [B, T, H, D] bf16;
    g [B, T, H] fp32 gate logits; state [B, H, D, D] fp32 initial state,
    overwritten with the final state (None: start from zero).
    workspace: a uint8 CUDA tensor for the split over superchunks, "auto" to
    allocate one of the size the library asks for, or None (no split).
    Returns o."""
    L = load()
    B, T, H, D = q.shape
    if o is None:
        o = torch.empty_like(q)
    if isinstance(workspace, str):
        n = gret_prefill_workspace_size(B, T, H, D, q.dtype)
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device) if n > 0 else None
    _dev(q, k, v, g, state, o, workspace)
    cfg = _cfg(H, H, D, q.dtype, scale)
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(L.yoco_gret_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, T, float(tau), _ptr(state), _ptr(o),
                               _ptr(workspace), ws_bytes, ctypes.byref(cfg), _stream()), "yoco_gret_prefill")
    return o


def gret_decode(q, k, v, g, tau, state, scale=0.0, o=None):
    """One recurrent gated-retention step.  q, k, v [B, H, D]; g [B, H] fp32;
    state [B, H, D, D] fp32, updated in place.  Returns o [B, H, D]."""
    L = load()
    B, H, D = q.shape
    if o is None:
        o = torch.empty_like(q)
    _dev(q, k, v, g, state, o)
    cfg = _cfg(H, H, D, q.dtype, scale)
    _check(L.yoco_gret_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, float(tau), _ptr(state), _ptr(o),
                              ctypes.byref(cfg), _stream()), "yoco_gret_decode")
    return o


def kv_i8_row_bytes(Hkv, D):
    """Bytes of one row of an 8-bit K or V cache (codes, then padded scales)."""
    return int(load().yoco_kv_i8_row_bytes(ctypes.byref(_cfg(Hkv, Hkv, D, torch.bfloat16))))


def kv_quantize_i8(k, v, k_i8=None, v_i8=None, dst_rows=None):
    """8-bit quantisation of K, V [n, Hkv, D] into cache rows (uint8 tensors
    [rows, row_bytes]); dst_rows (int64, device) places row i at dst_rows[i].
    Returns (k_i8, v_i8)."""
    L = load()
    n, Hkv, D = k.shape
    rb = kv_i8_row_bytes(Hkv, D)
    if k_i8 is None:
        k_i8 = torch.empty((n, rb), dtype=torch.uint8, device=k.device)
    if v_i8 is None:
        v_i8 = torch.empty((n, rb), dtype=torch.uint8, device=k.device)
    _dev(k, v, dst_rows, k_i8, v_i8)
    cfg = _cfg(Hkv, Hkv, D, k.dtype)
    _check(L.yoco_kv_quantize_i8(_ptr(k), _ptr(v), n, _ptr(dst_rows), _ptr(k_i8), _ptr(v_i8), ctypes.byref(cfg),
                                 _stream()), "yoco_kv_quantize_i8")
    return k_i8, v_i8


def cross_decode_i8(q, k_i8, v_i8, Hkv, seq_start, seq_len, max_len, workspace=None, o=None, want_lse=False,
                    scale=0.0):
    """cross_decode over 8-bit caches (uint8 rows from kv_quantize_i8)."""
    L = load()
    B, Hq, D = q.shape
    if o is None:
        o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if want_lse else None
    cfg = _cfg(Hq, Hkv, D, q.dtype, scale)
    if workspace is None:
        n = L.yoco_cross_decode_workspace_size(B, int(max_len), ctypes.byref(cfg))
        workspace = torch.empty(max(int(n), 16), dtype=torch.uint8, device=q.device)
    _dev(q, k_i8, v_i8, seq_start, seq_len, o, lse, workspace)
    if v_i8.shape != k_i8.shape:
        raise ValueError("k_i8 and v_i8 must have the same shape")
    _check(L.yoco_cross_decode_i8(_ptr(q), _ptr(k_i8), _ptr(v_i8), k_i8.shape[0], _ptr(seq_start), _ptr(seq_len), B,
                                  int(max_len), _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(),
                                  ctypes.byref(cfg), _stream()), "yoco_cross_decode_i8")
    return (o, lse) if want_lse else o


def attention_prefill(q, k, v, q_pos0=0, window=0, o=None, want_lse=False, scale=0.0):
    """Causal (window 0) or windowed attention of q [B, Tq, Hq, D] over keys
    k, v [B, Tkv, Hkv, D], query row i at key position q_pos0 + i."""
    L = load()
    B, Tq, Hq, D = q.shape
    Tkv, Hkv = k.shape[1], k.shape[2]
    if o is None:
        o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device) if want_lse else None
    _dev(q, k, v, o, lse)
    cfg = _cfg(Hq, Hkv, D, q.dtype, scale)
    _check(L.yoco_attention_prefill(_ptr(q), _ptr(k), _ptr(v), B, Tq, Tkv, int(q_pos0), int(window), _ptr(o),
                                    _ptr(lse), ctypes.byref(cfg), _stream()), "yoco_attention_prefill")
    return (o, lse) if want_lse else o


def debug_exp2_poly(x, y=None):
    """Test-only: the prefill softmax's polynomial 2^x (the FMA-pipe half of its
    exponentials) applied elementwise to an fp32 CUDA tensor."""
    L = load()
    if y is None:
        y = torch.empty_like(x)
    _dev(x, y)
    if x.dtype != torch.float32 or y.dtype != torch.float32 or y.numel() != x.numel():
        raise ValueError("debug_exp2_poly takes fp32 tensors of one size")
    _check(L.yoco_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream()), "yoco_debug_exp2_poly")
    return y
