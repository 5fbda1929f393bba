"""The tolerance of the gated-retention prefill, derived from its arithmetic.

A float64 model of the tcgen05 kernel's chunk loop (128-token chunks) that
rounds to bf16 exactly where the kernel does:
  * the decayed keys K_w = scale 2^{c_last - c_u} k_u (the update's operand);
  * the scores' P before P V;
  * the copy of S_prev for the cross term;
  * the output.
Chunks whose total decay is at least 2^-60 take their scores from Q K_w^T.
The others take scale 2^{c_r - c_u} (Q K^T).  The state itself stays
unrounded, as it stays fp32 in tensor memory.

Compared with the oracle's exact recurrence, the model must stay inside the
GPU tests' bound (rel-L2 5e-3) at decays from near 1 to strong, and near the
roundings' own size (a few 2^-9).  This is a model of the arithmetic, not of
the kernel's code: the GPU parity tests check the kernel itself."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

C = 128


def _bf16(x):
    """Round to bf16 (nearest, ties to even) and widen back to float64."""
    x32 = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x32.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def _model(q, k, v, lg, rnd=_bf16):
    """q, k, v [T, D] (bf16 values), lg [T] natural-log decays -> o [T, D];
    rnd is the rounding applied where the kernel rounds to bf16."""
    T, D = q.shape
    scale = D ** -0.5
    S = np.zeros((D, D))
    out = np.zeros((T, D))
    for t0 in range(0, T, C):
        Q, K, V = q[t0:t0 + C], k[t0:t0 + C], v[t0:t0 + C]
        c = np.cumsum(lg[t0:t0 + C]) / np.log(2.0)
        n = len(c)
        Kw = rnd(K * (scale * 2.0 ** (c[-1] - c))[:, None])
        causal = np.arange(n)[None, :] <= np.arange(n)[:, None]
        if c[-1] >= -60.0:
            P = np.where(causal, (Q @ Kw.T) * 2.0 ** (c[:, None] - c[-1]), 0.0)
        else:
            P = np.where(causal, (Q @ K.T) * scale * 2.0 ** (c[:, None] - c[None, :]), 0.0)
        O = rnd(P) @ V
        X = Q @ rnd(S)
        out[t0:t0 + n] = rnd(O + 2.0 ** c[:, None] * X)
        S = 2.0 ** c[-1] * S + Kw.T @ V
    return out


@pytest.mark.parametrize("gate_mean,tau", [(3.0, 16.0), (3.0, 4.0), (0.5, 2.0), (-2.0, 1.0)])
def test_kernel_rounding_model_within_bound(gate_mean, tau):
    T, D = 1024, 128
    bf = torch.bfloat16
    q = wl.normal((1, T, 1, D), 5, bf).double().numpy()[0, :, 0]
    k = wl.normal((1, T, 1, D), 6, bf).double().numpy()[0, :, 0]
    v = wl.normal((1, T, 1, D), 7, bf).double().numpy()[0, :, 0]
    g = wl.normal((1, T, 1), 8, torch.float32).numpy() + gate_mean
    lg = oracle.gret_log_decay(g, tau)[0, :, 0].astype(np.float64)
    ro, _ = oracle.gret_recurrent(torch.from_numpy(q[None, :, None]), torch.from_numpy(k[None, :, None]),
                                  torch.from_numpy(v[None, :, None]), lg[None, :, None])
    ro = np.asarray(ro)[0, :, 0]
    o = _model(q, k, v, lg)
    rel = np.linalg.norm(o - ro) / np.linalg.norm(ro)
    # inside the GPU bound, and of the order of the bf16 roundings themselves
    assert rel <= 5e-3, rel
    assert 5e-4 <= rel, rel


def test_model_without_rounding_is_the_recurrence():
    # the same chunk loop with every rounding removed must equal the oracle's
    # recurrence to float64 precision: the model's algebra is the method's
    T, D = 300, 128
    bf = torch.bfloat16
    q = wl.normal((1, T, 1, D), 15, bf).double().numpy()[0, :, 0]
    k = wl.normal((1, T, 1, D), 16, bf).double().numpy()[0, :, 0]
    v = wl.normal((1, T, 1, D), 17, bf).double().numpy()[0, :, 0]
    g = wl.normal((1, T, 1), 18, torch.float32).numpy() + 1.0
    lg = oracle.gret_log_decay(g, 2.0)[0, :, 0].astype(np.float64)
    ro, _ = oracle.gret_recurrent(torch.from_numpy(q[None, :, None]), torch.from_numpy(k[None, :, None]),
                                  torch.from_numpy(v[None, :, None]), lg[None, :, None])
    o = _model(q, k, v, lg, rnd=lambda x: np.asarray(x, dtype=np.float64))
    np.testing.assert_allclose(o, np.asarray(ro)[0, :, 0], rtol=1e-9, atol=1e-9)
