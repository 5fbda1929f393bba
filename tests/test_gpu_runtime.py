"""Runtime properties of the library on the GPU: the bounded waits report a
timeout as a status instead of hanging (a kernel waits on an mbarrier phase
that nothing completes), the context survives it, and the hot calls can be
captured into a CUDA graph (no host synchronisation or allocation inside)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.util import assert_close

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _decode_case(seed=4100):
    Hq, Hkv, D = 8, 2, 128
    lens = [300, 1000, 17]
    starts = np.cumsum([0] + lens[:-1])
    rows = int(sum(lens))
    kc = wl.normal((rows, Hkv, D), seed, BF)
    vc = wl.normal((rows, Hkv, D), seed + 1, BF)
    q = wl.normal((len(lens), Hq, D), seed + 2, BF)
    return q, kc, vc, starts, lens


def test_bounded_wait_reports_timeout_and_context_survives(cuda_lib):
    L = cuda_lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    assert cuda_lib.device_status() == cuda_lib.OK
    assert L.yoco_debug_wait_timeout_probe(stream) == cuda_lib.OK
    assert cuda_lib.device_status() == cuda_lib.ERR_TIMEOUT     # recorded, not hung
    assert cuda_lib.device_status() == cuda_lib.OK              # and cleared by the read
    # the context still works
    q, kc, vc, starts, lens = _decode_case()
    ss = torch.tensor(starts, dtype=torch.int64, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o = cuda_lib.cross_decode(q.cuda(), kc.cuda(), vc.cuda(), ss, sl, max(lens))
    ro, _ = oracle.cross_decode(q, kc, vc, starts, lens)
    assert_close(o, ro, BF, "decode after a timeout")
    assert cuda_lib.device_status() == cuda_lib.OK


def test_hot_calls_capture_into_a_cuda_graph(cuda_lib):
    q, kc, vc, starts, lens = _decode_case(4200)
    qd, kd, vd = q.cuda(), kc.cuda(), vc.cuda()
    ss = torch.tensor(starts, dtype=torch.int64, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(cuda_lib.cross_decode_workspace_size(3, max(lens), 8, 2, 128, BF), dtype=torch.uint8,
                     device="cuda")
    qp = wl.normal((1, 512, 8, 128), 4210, BF).cuda()
    kp = wl.normal((1, 512, 2, 128), 4211, BF).cuda()
    vp = wl.normal((1, 512, 2, 128), 4212, BF).cuda()
    od, op = torch.empty_like(qd), torch.empty_like(qp)
    # eager results first (this also sets each kernel's attributes once)
    ref_d = cuda_lib.cross_decode(qd, kd, vd, ss, sl, max(lens), workspace=ws).clone()
    ref_p = cuda_lib.cross_prefill(qp, kp, vp).clone()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cuda_lib.cross_decode(qd, kd, vd, ss, sl, max(lens), workspace=ws, o=od)
        cuda_lib.cross_prefill(qp, kp, vp, o=op)
    od.zero_()
    op.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(od, ref_d) and torch.equal(op, ref_p)
    g.reset()


def test_out_of_range_sequences_read_nothing_and_are_reported(cuda_lib):
    # A packed cache of R rows and five sequences: one in range, and four whose
    # arguments are not (length above max_len, rows past the cache's end, a
    # negative start, length 0).  The kernels' range check gives the four no
    # work: each output is 0 with lse -inf, the in-range sequence is exact, and
    # the status word reports the bad arguments once, without a fault.
    Hq, Hkv, D, R, max_len = 8, 2, 128, 5000, 3000
    kc = wl.normal((R, Hkv, D), 4300, BF, "cuda")
    vc = wl.normal((R, Hkv, D), 4301, BF, "cuda")
    starts = [100, 0, 4000, -8, 50]
    lens = [2900, 3001, 1001, 64, 0]
    B = len(lens)
    q = wl.normal((B, Hq, D), 4302, BF, "cuda")
    ss = torch.tensor(starts, dtype=torch.int64, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    assert cuda_lib.device_status() == cuda_lib.OK
    o, lse = cuda_lib.cross_decode(q, kc, vc, ss, sl, max_len, want_lse=True)
    assert cuda_lib.device_status() == cuda_lib.ERR_INVALID
    assert cuda_lib.device_status() == cuda_lib.OK               # cleared by the read
    ro, rlse = oracle.cross_decode(q[:1].cpu(), kc.cpu(), vc.cpu(), starts[:1], lens[:1])
    assert_close(o[:1], ro, BF, "in-range sequence")
    assert_close(lse[:1], rlse, BF, "in-range lse", max_abs=1e-3, rel_l2=1e-4)
    assert torch.all(o[1:] == 0)
    assert torch.all(torch.isneginf(lse[1:]))
    # the same plan over the 8-bit cache
    kq, vq = cuda_lib.kv_quantize_i8(kc, vc)
    o8 = cuda_lib.cross_decode_i8(q, kq, vq, Hkv, ss, sl, max_len)
    assert cuda_lib.device_status() == cuda_lib.ERR_INVALID
    assert torch.all(o8[1:] == 0)
    # a call after the report runs normally
    o2 = cuda_lib.cross_decode(q[:1].contiguous(), kc, vc, ss[:1].contiguous(), sl[:1].contiguous(), max_len)
    assert cuda_lib.device_status() == cuda_lib.OK
    assert_close(o2, ro, BF, "decode after the report")


def test_polynomial_exp2_within_its_bound(cuda_lib):
    # The prefill kernels take a quarter of their softmax exponentials from a
    # degree-3 polynomial (Cody-Waite reduction + minimax fit).  Over its
    # input range the relative error against 2^x stays within 7.5e-5; inputs
    # below -125 (and -inf, a masked score) give 2^-125 instead of 0, which is
    # ~1e-38 of the row's largest weight, below any fp32 sum's resolution.
    x = np.concatenate([np.linspace(-125.0, 9.0, 2_000_001),
                        np.array([0.0, -0.5, 0.5, -1.0, 1.0, 8.0, -124.5, -125.0])])
    xt = torch.tensor(x, dtype=torch.float32, device="cuda")
    y = cuda_lib.debug_exp2_poly(xt).cpu().double().numpy()
    ref = np.exp2(xt.cpu().double().numpy())
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 7.5e-5, f"max relative error {rel.max():.3e}"
    low = torch.tensor([-125.5, -130.0, -1e4, -np.inf], dtype=torch.float32, device="cuda")
    yl = cuda_lib.debug_exp2_poly(low).cpu().double().numpy()
    assert np.all(yl > 0) and np.all(yl <= 2.0 ** -124)
    assert cuda_lib.device_status() == cuda_lib.OK
