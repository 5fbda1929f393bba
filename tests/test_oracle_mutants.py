"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake into a temporary copy of oracle.c
(the source under oracle/ is never modified), builds it, swaps it in for the
real oracle and runs the pin checks of test_oracle_pins.py.  Every mutant
must fail at least one pin: a mutant that survives means the pins have a
blind spot."""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "causal_off_by_one": ("if (j > p) return 0;", "if (j >= p) return 0;"),
    "window_off_by_one": ("j <= p - window) return 0;", "j < p - window) return 0;"),
    "scale_dropped": ("s *= scale;", ";"),
    "gqa_interleaved": ("int64_t g = h / G;\n                const double *qv",
                        "int64_t g = h % Hkv;\n                const double *qv"),
    "ln_unbiased_var": ("var /= (double)d;", "var /= (double)(d - 1);"),
    "ln_mean_dropped": ("mean /= (double)d;", "mean = 0.0;"),
    "blend_sign": ("out[i] = a[i] + w * base[i];", "out[i] = a[i] - w * base[i];"),
    "weight_transposed": ("w[c * d + i]", "w[i * m + c]"),
    "lse_max_dropped": ("*lse_out = mx + log(den);", "*lse_out = log(den);"),
    "no_normalisation": ("for (int64_t c = 0; c < D; ++c) o[c] /= den;", "(void)den;"),
    "ring_slot_shift": ("slot_pos[p % W] = (int32_t)p;", "slot_pos[(p + 1) % W] = (int32_t)p;"),
    "ring_push_slot": ("int64_t s = pos % W;", "int64_t s = (pos + 1) % W;"),
    "decode_drops_newest": ("int64_t n = seq_len[b];", "int64_t n = seq_len[b] - 1;"),
    "accounting_no_window": ("(double)L_self * (double)c", "(double)L_self"),
    "gret_decay_after_add": ("S[d * D + e] = gam * S[d * D + e] + scale * kt[d] * vt[e];",
                             "S[d * D + e] = gam * (S[d * D + e] + scale * kt[d] * vt[e]);"),
    "gret_scale_dropped": ("const double w = exp(c[t] - c[s]) * scale * dot;",
                           "const double w = exp(c[t] - c[s]) * dot;"),
    "gret_state_transposed": ("for (int64_t d = 0; d < D; ++d) acc += qt[d] * S[d * D + e];\n                    o[row * D + e] = acc;",
                              "for (int64_t d = 0; d < D; ++d) acc += qt[d] * S[e * D + d];\n                    o[row * D + e] = acc;"),
    "gret_chunk_cross_undecayed": ("const double f = exp(a[r]);", "const double f = 1.0;"),
    "gret_chunk_state_off_by_one": ("const double w = exp(a[len - 1] - a[u]) * scale;",
                                    "const double w = exp(a[len - 1] - a[u] + log_gamma[(b * T + j0 + u) * H + h]) * scale;"),
    "gret_gate_no_temperature": ("out[i] = ls / tau;", "out[i] = ls;"),
}


def _checks():
    """Every pin, as (name, zero-arg callable)."""
    out = []
    for name in dir(pins):
        fn = getattr(pins, name)
        if not name.startswith("test_") or not callable(fn):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            out.append((name, fn))
            continue
        argnames, values = params[0].args[0], params[0].args[1]
        argnames = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else argnames
        for val in values:
            val = val if isinstance(val, tuple) else (val,)
            out.append((f"{name}{val}", (lambda f, kw: (lambda: f(**kw)))(fn, dict(zip(argnames, val)))))
    return out


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutant_is_caught(mutant, tmp_path):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {mutant} not found"
    path_c = tmp_path / "mutant.c"
    path_so = tmp_path / "libmutant.so"
    path_c.write_text(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o",
                           str(path_so), str(path_c), "-lm"])
    real = oracle.lib()
    oracle._LIB = oracle.load(str(path_so))
    failed = []
    try:
        for name, check in _checks():
            try:
                check()
            except AssertionError:
                failed.append(name)
            except Exception:
                failed.append(name)
    finally:
        oracle._LIB = real
    assert failed, f"mutant {mutant} survived every pin"
