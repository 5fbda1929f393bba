"""The bf16 tiny stack's tolerance, derived: a float64 model that rounds to
bf16 exactly where the GPU path stores bf16 (tests/stack_model.py) against
the unrounded fp64 oracle.  The model must (1) reduce to oracle.tiny_stack
bit for bit when its rounding is the identity, so it is the oracle's stack and
nothing else, and (2) stay within half of the end-to-end bounds that the GPU
stack test uses, so that those bounds are the storage roundings' own cost
with an equal margin for the kernels' arithmetic."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests import stack_model as sm
from tests.util import errors


@pytest.fixture(scope="module")
def case():
    cfg = wl.TinyStack()
    x, w = wl.tiny_stack_inputs(cfg, torch.bfloat16)
    ref = oracle.tiny_stack(x, w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window, cfg.w_blend)
    return cfg, x, w, ref


def _pairs(a, b):
    for key in ("self_k", "self_v", "self_o", "cross_o"):
        for l in range(len(b[key])):
            yield f"{key}{l}", a[key][l], b[key][l]
    for key in ("k_g", "v_g", "x"):
        yield key, a[key], b[key]


def test_model_without_rounding_is_the_oracle_stack(case):
    cfg, x, w, ref = case
    m = sm.unrounded(x, w, cfg)
    for name, got, want in _pairs(m, ref):
        np.testing.assert_array_equal(got, want, err_msg=name)
    ee = sm.unrounded(x[:cfg.T], w, cfg, early_exit=True)
    np.testing.assert_allclose(ee, oracle.tiny_stack_early_exit(x[:cfg.T], w, cfg.Hq, cfg.Hkv, cfg.D, cfg.window,
                                                                cfg.w_blend), rtol=0, atol=1e-12)


def test_bf16_rounding_cost_within_half_the_stack_bound(case):
    cfg, x, w, ref = case
    m = sm.stack(x, w, cfg)
    worst_abs = worst_rel = 0.0
    for name, got, want in _pairs(m, ref):
        ma, rl = errors(got, want)
        worst_abs, worst_rel = max(worst_abs, ma), max(worst_rel, rl)
    assert worst_abs <= sm.BF16_STACK_MAX_ABS / 2, worst_abs
    assert worst_rel <= sm.BF16_STACK_REL_L2 / 2, worst_rel
    # and the bound is not loose by more than the stated factor of two margins
    assert worst_abs > sm.BF16_STACK_MAX_ABS / 4 and worst_rel > sm.BF16_STACK_REL_L2 / 4


def test_rounding_model_rounds_where_the_gpu_stores(case):
    # every stored intermediate of the model is a bf16 value
    cfg, x, w, _ = case
    m = sm.stack(x, w, cfg)
    for name, got, _ in _pairs(m, m):
        np.testing.assert_array_equal(sm.bf16_round(got), got, err_msg=name)
