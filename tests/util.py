"""Comparison helpers for the parity tests."""
import numpy as np
import torch

# Tolerances for bf16 inputs with fp32 softmax/accumulate, on unit-scale outputs.
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
# fp32 path: the kernels round nothing below fp32, so errors are fp32
# accumulation order over at most a few thousand terms.
FP32_MAX_ABS = 2e-4
FP32_REL_L2 = 2e-5


def to_np(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def errors(got, ref):
    g, r = to_np(got), to_np(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    d = g - r
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    den = float(np.linalg.norm(r.ravel()))
    rel = float(np.linalg.norm(d.ravel()) / den) if den > 0 else float(np.linalg.norm(d.ravel()))
    return max_abs, rel


def assert_close(got, ref, dtype, what="", max_abs=None, rel_l2=None):
    if max_abs is None:
        max_abs = BF16_MAX_ABS if dtype == torch.bfloat16 else FP32_MAX_ABS
    if rel_l2 is None:
        rel_l2 = BF16_REL_L2 if dtype == torch.bfloat16 else FP32_REL_L2
    g = to_np(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    ma, rl = errors(got, ref)
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max_abs {ma:.3e} (<= {max_abs}), rel_l2 {rl:.3e} (<= {rel_l2})"
    return ma, rl
