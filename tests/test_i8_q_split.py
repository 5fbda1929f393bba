"""The 8-bit decode's split of q into two int8 operands, checked on the CPU.

The kernel holds each query head as 15-bit fixed point: x = rint(q * 16256 /
amax) clamped to +-16256, then x = 128 hi + lo with hi = rint(x / 128), so
that S = 128 (K hi) + (K lo) is exact in int32 against the int8 K codes.
This test repeats those float32 steps with numpy (IEEE single, like the
kernel's operators) and pins what the kernel relies on:
  * hi and lo fit int8 (hi in [-127, 127], lo in [-64, 64]);
  * 128 hi + lo reproduces x exactly;
  * s_q x is within half a step of q (step s_q = amax / 16256);
  * the score against int8 codes is within that bound of the exact score,
    far below the error of bf16-rounding q itself."""
import numpy as np
import pytest

import workloads as wl
import torch

Q_MAX = 16256.0


def _split(q):
    """q [G, D] float32 (bf16 values) -> (hi, lo, x, s_q) as the kernel forms them."""
    q = q.astype(np.float32)
    amax = np.abs(q).max(axis=1, keepdims=True).astype(np.float32)
    inv = np.where(amax > 0, np.float32(Q_MAX) / np.where(amax > 0, amax, np.float32(1)), np.float32(0))
    x = np.clip(np.rint(q * inv.astype(np.float32)), -Q_MAX, Q_MAX).astype(np.float32)
    hi = np.rint(x * np.float32(1.0 / 128.0)).astype(np.float32)
    lo = (x - np.float32(128.0) * hi).astype(np.float32)
    s_q = (amax * np.float32(1.0 / Q_MAX)).astype(np.float32)
    return hi, lo, x, s_q


@pytest.mark.parametrize("scale", [1.0, 1e-3, 50.0])
def test_split_fits_int8_and_reconstructs(scale):
    q = (wl.normal((64, 128), 7000, torch.bfloat16).float().numpy() * scale).astype(np.float32)
    q[3] = 0.0                      # an all-zero head
    q[5, 17] = -np.abs(q[5]).max()   # a tie for the largest magnitude
    hi, lo, x, s_q = _split(q)
    assert hi.min() >= -127 and hi.max() <= 127
    assert lo.min() >= -64 and lo.max() <= 64
    assert np.array_equal(128.0 * hi.astype(np.float64) + lo.astype(np.float64), x.astype(np.float64))
    assert np.all(x[3] == 0)
    # within half a step, up to float32 rounding: s_q and 1 / inv are rounded
    # separately, and their relative mismatch (~1e-7) times |x| <= 16256 is
    # ~2e-3 of a step
    err = np.abs(q.astype(np.float64) - s_q.astype(np.float64) * x.astype(np.float64))
    assert np.all(err <= 0.5 * s_q.astype(np.float64) * (1 + 1e-2) + 1e-30)


def test_integer_scores_are_close_to_exact():
    q = wl.normal((8, 128), 7001, torch.bfloat16).float().numpy().astype(np.float32)
    codes = np.random.default_rng(7002).integers(-127, 128, size=(4096, 128)).astype(np.int64)
    hi, lo, x, s_q = _split(q)
    acc = 128 * (codes @ hi.astype(np.int64).T) + codes @ lo.astype(np.int64).T   # int32 in the kernel
    assert np.abs(acc).max() < 2 ** 31
    got = acc.astype(np.float64) * s_q.astype(np.float64).T
    exact = codes.astype(np.float64) @ q.astype(np.float64).T
    # the fixed-point error per score is at most half a step times sum |code|
    bound = 0.5 * s_q.astype(np.float64).T * np.abs(codes).sum(axis=1, keepdims=True)
    assert np.all(np.abs(got - exact) <= bound * (1 + 1e-2))
    # and in practice far below bf16's own rounding of q (relative 2^-9 per element)
    rel = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    assert rel < 2e-4, rel
