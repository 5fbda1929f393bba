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
