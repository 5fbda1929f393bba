"""Gated retention on the GPU against the oracle: the chunkwise prefill
(outputs and final state, ragged last chunk, carried initial state, weak and
strong decay) and the recurrent decode step, alone and continuing a
prefill.  The oracle's three forms are pinned to each other on the CPU; here
the GPU is compared with its recurrent form.

Tolerance: bf16 storage of q, k, v, and of the decayed scores, the decayed
keys and the state's two-part split inside the kernel, give relative errors
of a few 2^-9; outputs scale with the state (up to ~sqrt(T) for decay near
1), so max-abs is bounded relative to the output's own scale."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.util import errors

pytestmark = pytest.mark.gpu
BF, F32 = torch.bfloat16, torch.float32


def _inputs(B, T, H, D, seed, gate_mean, dtype=BF):
    q = wl.normal((B, T, H, D), seed, dtype)
    k = wl.normal((B, T, H, D), seed + 1, dtype)
    v = wl.normal((B, T, H, D), seed + 2, dtype)
    g = wl.normal((B, T, H), seed + 3, F32) + gate_mean
    return q, k, v, g


def _check(got, ref, what, rel_l2=5e-3, max_rel=2e-2):
    g = got.float().cpu().numpy() if hasattr(got, "cpu") else np.asarray(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    scale = max(1.0, float(np.abs(ref).max()))
    ma, rl = errors(got, ref)
    assert ma <= max_rel * scale and rl <= rel_l2, f"{what}: max_abs {ma:.3e} (<= {max_rel * scale:.3e}), rel_l2 {rl:.3e}"


@pytest.mark.parametrize("B,T,H,D,gate_mean,tau", [
    (1, 100, 2, 64, 3.0, 4.0),     # decay near 1, ragged last chunk
    (2, 257, 4, 128, 3.0, 16.0),   # several chunks plus one token
    (1, 64, 1, 128, -2.0, 1.0),    # one full chunk, strong decay
    (1, 1, 2, 128, 0.0, 1.0),      # a single token
    (3, 200, 2, 64, 0.5, 2.0),
])
@pytest.mark.parametrize("with_state", [False, True])
def test_gret_prefill_matches_oracle(cuda_lib, B, T, H, D, gate_mean, tau, with_state):
    q, k, v, g = _inputs(B, T, H, D, 1000 + T + D, gate_mean)
    s0 = wl.normal((B, H, D, D), 1090, F32) * 0.5 if with_state else None
    lg = oracle.gret_log_decay(g.numpy(), tau)
    ro, rs = oracle.gret_recurrent(q, k, v, lg, state=s0)
    st = s0.clone().cuda() if with_state else None
    o = cuda_lib.gret_prefill(q.cuda(), k.cuda(), v.cuda(), g.cuda(), tau, state=st)
    _check(o, ro, "o")
    if with_state:
        _check(st, rs, "final state")


def test_gret_prefill_final_state_and_decode_continue(cuda_lib):
    # GPU prefill of T tokens, then GPU decode steps from its final state,
    # equal the oracle's recurrence over T + n tokens
    B, T, H, D, n, tau = 2, 300, 4, 128, 6, 8.0
    q, k, v, g = _inputs(B, T + n, H, D, 1200, 2.0)
    lg = oracle.gret_log_decay(g.numpy(), tau)
    ro, rs = oracle.gret_recurrent(q, k, v, lg)
    st = torch.zeros((B, H, D, D), dtype=F32, device="cuda")
    o = cuda_lib.gret_prefill(q[:, :T].contiguous().cuda(), k[:, :T].contiguous().cuda(),
                              v[:, :T].contiguous().cuda(), g[:, :T].contiguous().cuda(), tau, state=st)
    _check(o, ro[:, :T], "prefill o")
    for t in range(T, T + n):
        od = cuda_lib.gret_decode(q[:, t].contiguous().cuda(), k[:, t].contiguous().cuda(),
                                  v[:, t].contiguous().cuda(), g[:, t].contiguous().cuda(), tau, st)
        _check(od, ro[:, t], f"decode o@{t}")
    _check(st, rs, "state after decode")


@pytest.mark.parametrize("dtype,D", [(F32, 64), (BF, 128), (F32, 128)])
def test_gret_decode_steps_match_oracle(cuda_lib, dtype, D):
    B, H, n, tau = 3, 2, 5, 4.0
    q, k, v, g = _inputs(B, n, H, D, 1300 + D, 1.0, dtype)
    s0 = wl.normal((B, H, D, D), 1350, F32)
    lg = oracle.gret_log_decay(g.numpy(), tau)
    ro, rs = oracle.gret_recurrent(q, k, v, lg, state=s0)
    st = s0.clone().cuda()
    for t in range(n):
        od = cuda_lib.gret_decode(q[:, t].contiguous().cuda(), k[:, t].contiguous().cuda(),
                                  v[:, t].contiguous().cuda(), g[:, t].contiguous().cuda(), tau, st)
        if dtype == F32:
            _check(od, ro[:, t], f"o@{t}", rel_l2=2e-5, max_rel=2e-4)
        else:
            _check(od, ro[:, t], f"o@{t}")
    _check(st, rs, "state", rel_l2=2e-5 if dtype == F32 else 5e-3, max_rel=2e-4 if dtype == F32 else 2e-2)


def test_gret_prefill_long_sequence(cuda_lib):
    # 8K tokens (128 chunks) with decay close to 1: the carried state must not drift
    B, T, H, D, tau = 1, 8192, 2, 128, 16.0
    q, k, v, g = _inputs(B, T, H, D, 1400, 4.0)
    lg = oracle.gret_log_decay(g.numpy(), tau)
    ro, rs = oracle.gret_recurrent(q, k, v, lg)
    st = torch.zeros((B, H, D, D), dtype=F32, device="cuda")
    o = cuda_lib.gret_prefill(q.cuda(), k.cuda(), v.cuda(), g.cuda(), tau, state=st)
    _check(o, ro, "o")
    _check(st, rs, "final state")


def test_gret_prefill_mixed_decay_chunks(cuda_lib):
    # Chunks of 128 tokens whose gates alternate between strong decay (a
    # chunk's total decay far below 2^-60), weak decay (far above) and levels
    # either side of 2^-60, with a carried state and a ragged last chunk: the
    # kernel's two score paths and every switch between them in one launch.
    B, H, D, tau, C = 2, 3, 128, 1.0, 128
    levels = [8.0, -3.0, 8.0, 0.93, 0.98, -3.0, -3.0, 8.0, 0.5]   # gate logit per chunk
    T = C * (len(levels) - 1) + 37
    q, k, v, _ = _inputs(B, T, H, D, 1500, 0.0)
    base = torch.tensor([levels[t // C] for t in range(T)], dtype=F32)
    g = base[None, :, None] + 0.05 * wl.normal((B, T, H), 1505, F32)
    s0 = wl.normal((B, H, D, D), 1510, F32) * 0.5
    lg = oracle.gret_log_decay(g.numpy(), tau)
    # the levels do straddle the threshold: some chunk totals above 2^-60, some below
    totals = [lg[0, i * C:(i + 1) * C, 0].sum() / np.log(2) for i in range(len(levels) - 1)]
    assert min(totals) < -60 < max(totals)
    ro, rs = oracle.gret_recurrent(q, k, v, lg, state=s0)
    st = s0.clone().cuda()
    o = cuda_lib.gret_prefill(q.cuda(), k.cuda(), v.cuda(), g.cuda(), tau, state=st)
    _check(o, ro, "o")
    _check(st, rs, "final state")


@pytest.mark.parametrize("B,T,H,gate_mean,tau,with_state", [
    (1, 8192 + 37, 4, 4.0, 16.0, True),    # 65 chunks -> 8 superchunks of 9, ragged last chunk
    (1, 4096, 2, 0.5, 2.0, False),         # strong decay: early superchunks' states fade out
    (2, 3000, 3, 2.0, 8.0, True),          # 24 chunks -> 3 superchunks of 8
])
def test_gret_prefill_split_over_superchunks(cuda_lib, B, T, H, gate_mean, tau, with_state):
    # With a workspace and few sequences, each sequence runs as superchunks on
    # separate CTAs: outputs and the final state must still follow the
    # recurrence, and agree with the one-CTA-per-sequence launch.
    D = 128
    assert cuda_lib.gret_prefill_workspace_size(B, T, H, D) > 0
    q, k, v, g = _inputs(B, T, H, D, 1600 + T, gate_mean)
    s0 = wl.normal((B, H, D, D), 1690, F32) * 0.5 if with_state else None
    lg = oracle.gret_log_decay(g.numpy(), tau)
    ro, rs = oracle.gret_recurrent(q, k, v, lg, state=s0)
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), g.cuda()
    st = s0.clone().cuda() if with_state else None
    o = cuda_lib.gret_prefill(qd, kd, vd, gd, tau, state=st)                  # split (workspace "auto")
    _check(o, ro, "o, split")
    if with_state:
        _check(st, rs, "final state, split")
    st1 = s0.clone().cuda() if with_state else None
    o1 = cuda_lib.gret_prefill(qd, kd, vd, gd, tau, state=st1, workspace=None)  # one CTA per sequence
    _check(o, o1.float().cpu().numpy(), "split vs one CTA per sequence")
    if with_state:
        _check(st, st1.cpu().numpy(), "final state, split vs one CTA")
    assert cuda_lib.device_status() == cuda_lib.OK
