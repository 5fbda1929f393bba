"""yoco_cross_decode_static: the decode step for callers that cannot allocate
device memory (a host or plugin given only its input and output buffers, or
a process whose framework holds nearly all device memory), whose split-KV
scratch is a fixed array inside the library.

Checks, through the C ABI, that two calls in a row (the second finding the
first call's partials still in the shared array) match both the CPU oracle
and the workspace entry point within the parity tolerance, and that a decode
too large for the array is refused with YOCO_ERR_WORKSPACE.  This file is
collected last."""
import ctypes

import pytest
import torch

import oracle
import workloads as wl
from tests.util import assert_close

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _static_entry(yoco):
    fn = yoco.load().yoco_cross_decode_static
    vp = ctypes.c_void_p
    fn.restype = ctypes.c_int
    fn.argtypes = [vp, vp, vp, ctypes.c_int64, vp, vp, ctypes.c_int32, ctypes.c_int64, vp, vp,
                   ctypes.POINTER(yoco.AttnCfg), vp]
    return fn


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def test_static_scratch_decode_matches_workspace_decode(cuda_lib):
    fn = _static_entry(cuda_lib)
    Hq, Hkv, D = 32, 8, 128
    cfg = cuda_lib.AttnCfg(Hq, Hkv, D, 0.0, cuda_lib.BF16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # call 1 uses many splits; call 2 fewer and shorter sequences, so stale
    # partials of call 1 remain in the array around call 2's
    cases = [([70000, 131072, 1, 4097, 65536, 99999], 10), ([300, 2048, 17], 20)]
    for lens, seed in cases:
        B = len(lens)
        starts = torch.cumsum(torch.tensor([0] + [l + 3 for l in lens[:-1]]), 0)
        rows = int(starts[-1]) + lens[-1]
        kc = wl.normal((rows, Hkv, D), seed, BF, "cuda")
        vc = wl.normal((rows, Hkv, D), seed + 1, BF, "cuda")
        q = wl.normal((B, Hq, D), seed + 2, BF, "cuda")
        ss = starts.to(torch.int64).cuda()
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        ref, ref_lse = cuda_lib.cross_decode(q, kc, vc, ss, sl, max(lens), want_lse=True)
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        st = fn(_ptr(q), _ptr(kc), _ptr(vc), rows, _ptr(ss), _ptr(sl), B, max(lens), _ptr(o), _ptr(lse),
                ctypes.byref(cfg), stream)
        assert st == cuda_lib.OK, f"status {st}"
        torch.cuda.synchronize()
        ro, rlse = oracle.cross_decode(q.cpu(), kc.cpu(), vc.cpu(), starts.numpy(), lens)
        for b in range(B):     # per sequence: the random-key outputs are far below unit scale
            assert_close(o[b], ro[b], BF, f"o vs oracle, sequence {b}")
        assert_close(lse, rlse, BF, "lse vs oracle", max_abs=1e-3, rel_l2=1e-4)
        assert_close(o, ref, BF, "o vs workspace entry point")
        assert_close(lse, ref_lse, BF, "lse vs workspace entry point", max_abs=1e-3, rel_l2=1e-4)
    assert cuda_lib.device_status() == cuda_lib.OK


def test_static_scratch_rejects_oversized_decode(cuda_lib):
    fn = _static_entry(cuda_lib)
    cfg = cuda_lib.AttnCfg(64, 8, 128, 0.0, cuda_lib.BF16)
    B, max_len = 4096, 1 << 20
    need = cuda_lib.cross_decode_workspace_size(B, max_len, 64, 8, 128, BF)
    assert need > (32 << 20)
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = _ptr(dummy)
    st = fn(p, p, p, 1 << 20, p, p, B, max_len, p, None, ctypes.byref(cfg), None)
    assert st == cuda_lib.ERR_WORKSPACE
