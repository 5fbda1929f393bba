"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, validates arguments before launching anything, and its host
helpers (workspace sizing, cache accounting) are right."""
import ctypes
import os
import re

import pytest
import torch

import oracle
import shared_kv_decoder_b200 as yoco

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(yoco_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    L = yoco.load()
    names = _declared()
    assert len(names) >= 12
    for n in sorted(names):
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert L.yoco_version().startswith(b"yoco-b200")


def test_status_strings():
    L = yoco.load()
    for s in range(6):
        assert L.yoco_status_string(s)
    assert L.yoco_status_string(99) == b"unknown status"


def _cfg(Hq=32, Hkv=8, D=128, dtype=0, scale=0.0):
    return yoco.AttnCfg(Hq, Hkv, D, scale, dtype)


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


@pytest.mark.parametrize("cfg,expect", [
    (_cfg(Hq=30, Hkv=8), yoco.ERR_INVALID),          # Hq % Hkv
    (_cfg(D=96), yoco.ERR_UNSUPPORTED),               # head dim not built
    (_cfg(Hq=48, Hkv=3), yoco.ERR_UNSUPPORTED),       # group 16
    (_cfg(dtype=7), yoco.ERR_INVALID),
    (_cfg(scale=-1.0), yoco.ERR_INVALID),
])
def test_bad_cfg_rejected_before_launch(cfg, expect):
    L = yoco.load()
    st = L.yoco_cross_prefill(FAKE, FAKE, FAKE, 1, 128, 128, 0, FAKE, None, ctypes.byref(cfg), None)
    assert st == expect


def test_bad_arguments_rejected_before_launch():
    L = yoco.load()
    c = _cfg()
    b = ctypes.byref(c)
    # q_pos0 + Tq > Tkv
    assert L.yoco_cross_prefill(FAKE, FAKE, FAKE, 1, 128, 100, 0, FAKE, None, b, None) == yoco.ERR_INVALID
    # null and misaligned pointers
    assert L.yoco_cross_prefill(None, FAKE, FAKE, 1, 128, 128, 0, FAKE, None, b, None) == yoco.ERR_INVALID
    assert L.yoco_cross_prefill(MISALIGNED, FAKE, FAKE, 1, 128, 128, 0, FAKE, None, b, None) == yoco.ERR_INVALID
    # window < 1, partial ring arguments
    assert L.yoco_swa_prefill(FAKE, FAKE, FAKE, 1, 64, 0, FAKE, None, None, None, None, b, None) == yoco.ERR_INVALID
    assert L.yoco_swa_prefill(FAKE, FAKE, FAKE, 1, 64, 8, FAKE, None, FAKE, None, None, b, None) == yoco.ERR_INVALID
    # decode: max_len < 1, cache_rows out of [1, 2^31 - 1], workspace missing / too small
    R = 4096
    assert L.yoco_cross_decode(FAKE, FAKE, FAKE, R, FAKE, FAKE, 2, 0, FAKE, None, FAKE, 1 << 30, b, None) == yoco.ERR_INVALID
    assert L.yoco_cross_decode(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 2, 1000, FAKE, None, FAKE, 1 << 30, b, None) == yoco.ERR_INVALID
    assert L.yoco_cross_decode(FAKE, FAKE, FAKE, 1 << 31, FAKE, FAKE, 2, 1000, FAKE, None, FAKE, 1 << 30, b,
                               None) == yoco.ERR_INVALID
    assert L.yoco_cross_decode(FAKE, FAKE, FAKE, R, FAKE, FAKE, 2, 1000, FAKE, None, None, 0, b, None) == yoco.ERR_WORKSPACE
    assert L.yoco_cross_decode(FAKE, FAKE, FAKE, R, FAKE, FAKE, 2, 1000, FAKE, None, FAKE, 16, b, None) == yoco.ERR_WORKSPACE
    assert L.yoco_cross_decode_static(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 2, 1000, FAKE, None, b, None) == yoco.ERR_INVALID
    # test-only exp2 probe: negative size, null pointers
    assert L.yoco_debug_exp2_poly(FAKE, FAKE, -1, None) == yoco.ERR_INVALID
    assert L.yoco_debug_exp2_poly(None, FAKE, 8, None) == yoco.ERR_INVALID
    assert L.yoco_debug_exp2_poly(FAKE, FAKE, 0, None) == yoco.OK
    # projection: bad eps
    assert L.yoco_kv_project_blend(FAKE, 4, 64, FAKE, 1, 0.0, None, None, 0.0, 0.0, None, FAKE, FAKE, b, None) == yoco.ERR_INVALID
    # empty inputs are a successful no-op (nothing launched)
    assert L.yoco_cross_prefill(FAKE, FAKE, FAKE, 0, 128, 128, 0, FAKE, None, b, None) == yoco.OK
    assert L.yoco_cross_prefill(FAKE, FAKE, FAKE, 1, 0, 128, 0, FAKE, None, b, None) == yoco.OK
    assert L.yoco_kv_project_blend(FAKE, 0, 64, FAKE, 1, 1e-5, None, None, 0.0, 0.0, None, FAKE, FAKE, b, None) == yoco.OK


def test_gret_arguments_rejected_before_launch():
    L = yoco.load()
    same = ctypes.byref(_cfg(Hq=8, Hkv=8))
    grouped = ctypes.byref(_cfg(Hq=8, Hkv=2))
    fp32 = ctypes.byref(_cfg(Hq=8, Hkv=8, dtype=1))
    # heads must match, tau > 0, pointers valid
    assert L.yoco_gret_prefill(FAKE, FAKE, FAKE, FAKE, 1, 64, 4.0, None, FAKE, None, 0, grouped, None) == yoco.ERR_INVALID
    assert L.yoco_gret_prefill(FAKE, FAKE, FAKE, FAKE, 1, 64, 0.0, None, FAKE, None, 0, same, None) == yoco.ERR_INVALID
    assert L.yoco_gret_prefill(FAKE, FAKE, FAKE, None, 1, 64, 4.0, None, FAKE, None, 0, same, None) == yoco.ERR_INVALID
    assert L.yoco_gret_prefill(FAKE, FAKE, FAKE, FAKE, 1, 64, 4.0, MISALIGNED, FAKE, None, 0, same,
                               None) == yoco.ERR_INVALID
    # the chunkwise prefill is built for bf16 only
    assert L.yoco_gret_prefill(FAKE, FAKE, FAKE, FAKE, 1, 64, 4.0, None, FAKE, None, 0, fp32, None) == yoco.ERR_UNSUPPORTED
    # the split's workspace: too small is refused before launch; none is needed
    # once B x H sequences fill the GPU, nor for D = 64
    d128 = ctypes.byref(_cfg(Hq=32, Hkv=32))
    need = L.yoco_gret_prefill_workspace_size(1, 65536, d128)
    assert need == 32 * 8 * (128 * 128 + 1) * 4
    assert L.yoco_gret_prefill(FAKE, FAKE, FAKE, FAKE, 1, 65536, 4.0, None, FAKE, FAKE, need - 16, d128,
                               None) == yoco.ERR_WORKSPACE
    assert L.yoco_gret_prefill_workspace_size(8, 65536, d128) == 0
    assert L.yoco_gret_prefill_workspace_size(1, 65536, ctypes.byref(_cfg(Hq=8, Hkv=8, D=64))) == 0
    # decode needs its state
    assert L.yoco_gret_decode(FAKE, FAKE, FAKE, FAKE, 1, 4.0, None, FAKE, same, None) == yoco.ERR_INVALID
    assert L.yoco_gret_decode(FAKE, FAKE, FAKE, FAKE, 1, -1.0, FAKE, FAKE, same, None) == yoco.ERR_INVALID
    # empty inputs: successful no-op
    assert L.yoco_gret_prefill(FAKE, FAKE, FAKE, FAKE, 0, 64, 4.0, None, FAKE, None, 0, same, None) == yoco.OK
    assert L.yoco_gret_decode(FAKE, FAKE, FAKE, FAKE, 0, 4.0, FAKE, FAKE, same, None) == yoco.OK


def test_i8_cache_arguments_rejected_before_launch():
    L = yoco.load()
    c = _cfg()
    b = ctypes.byref(c)
    assert L.yoco_kv_i8_row_bytes(b) == 8 * 128 + 32
    assert L.yoco_kv_i8_row_bytes(ctypes.byref(_cfg(Hq=8, Hkv=1))) == 128 + 16
    # the 8-bit decode is built for D = 128 and bf16
    R = 4096
    assert L.yoco_cross_decode_i8(FAKE, FAKE, FAKE, R, FAKE, FAKE, 2, 100, FAKE, None, FAKE, 1 << 30,
                                  ctypes.byref(_cfg(D=64)), None) == yoco.ERR_UNSUPPORTED
    assert L.yoco_cross_decode_i8(FAKE, FAKE, FAKE, R, FAKE, FAKE, 2, 100, FAKE, None, None, 0, b, None) == yoco.ERR_WORKSPACE
    assert L.yoco_cross_decode_i8(FAKE, MISALIGNED, FAKE, R, FAKE, FAKE, 2, 100, FAKE, None, FAKE, 1 << 30, b,
                                  None) == yoco.ERR_INVALID
    assert L.yoco_cross_decode_i8(FAKE, FAKE, FAKE, -1, FAKE, FAKE, 2, 100, FAKE, None, FAKE, 1 << 30, b,
                                  None) == yoco.ERR_INVALID
    assert L.yoco_kv_quantize_i8(FAKE, FAKE, -1, None, FAKE, FAKE, b, None) == yoco.ERR_INVALID
    assert L.yoco_kv_quantize_i8(FAKE, FAKE, 0, None, FAKE, FAKE, b, None) == yoco.OK


def test_swa_decode_step_arguments_rejected_before_launch():
    L = yoco.load()
    c = _cfg()
    b = ctypes.byref(c)
    B, W, d = 4, 1024, 4096
    need = L.yoco_swa_decode_step_workspace_size(B, W, b)
    # the decode workspace plus the new K/V scratch of the fallback path
    assert need == L.yoco_swa_decode_workspace_size(B, W, b) + 2 * B * 8 * 128 * 2
    assert L.yoco_swa_decode_step_workspace_size(B, 0, b) == 0
    assert L.yoco_swa_decode_step_workspace_size(-1, W, b) == 0

    def call(x=FAKE, dm=d, w=FAKE, eps=1e-5, wk=0.5, q=FAKE, pos=FAKE, nb=B, win=W, o=FAKE, ko=None, ws=FAKE,
             wsb=None):
        return L.yoco_swa_decode_step(x, dm, w, 1, eps, FAKE, FAKE, wk, 0.5, q, pos, nb, win, FAKE, FAKE, FAKE,
                                      o, ko, None, ws, need if wsb is None else wsb, b, None)
    assert call(nb=-1) == yoco.ERR_INVALID
    assert call(win=0) == yoco.ERR_INVALID
    assert call(dm=0) == yoco.ERR_INVALID
    assert call(dm=100) == yoco.ERR_INVALID              # x rows not a multiple of 16 bytes
    assert call(eps=0.0) == yoco.ERR_INVALID
    assert call(wk=float("nan")) == yoco.ERR_INVALID
    assert call(x=None) == yoco.ERR_INVALID
    assert call(pos=None) == yoco.ERR_INVALID
    assert call(o=MISALIGNED) == yoco.ERR_INVALID
    assert call(ko=MISALIGNED) == yoco.ERR_INVALID        # optional outputs must still be aligned
    assert call(ws=None) == yoco.ERR_WORKSPACE
    assert call(wsb=need - 16) == yoco.ERR_WORKSPACE
    assert call(ws=MISALIGNED) == yoco.ERR_WORKSPACE
    assert L.yoco_swa_decode_step(FAKE, d, FAKE, 1, 1e-5, None, None, 0.0, 0.0, FAKE, FAKE, B, W, FAKE, FAKE,
                                  FAKE, FAKE, None, None, FAKE, need, ctypes.byref(_cfg(D=96)),
                                  None) == yoco.ERR_UNSUPPORTED
    # an empty batch is a successful no-op (nothing launched)
    assert call(nb=0) == yoco.OK


def test_workspace_size_monotone_and_positive():
    sizes = [yoco.cross_decode_workspace_size(B, L, 32, 8, 128, torch.bfloat16)
             for B, L in [(1, 1), (1, 4096), (16, 131072), (16, 262144)]]
    assert all(s > 0 for s in sizes)
    assert sizes == sorted(sizes)
    assert yoco.cross_decode_workspace_size(1, 0, 32, 8, 128, torch.bfloat16) == 0
    # group size 16 has no decode build
    assert yoco.cross_decode_workspace_size(1, 100, 32, 2, 128, torch.bfloat16) == 0


@pytest.mark.parametrize("L_self,window,N", [(13, 1024, 1 << 20), (2, 32, 16), (0, 8, 100), (3, 64, 0)])
def test_cache_bytes_matches_oracle(L_self, window, N):
    got = yoco.cache_bytes(L_self, window, N, 8, 128, torch.bfloat16)
    assert got == oracle.cache_bytes_yoco(L_self, window, N, 8, 128, 2)
