"""The oracle's pins must reject plausible mistakes.

Each case copies la_oracle.c, plants one mistake in the copy (on the CPU, in a temporary
directory), compiles it with the oracle's own flags and checks that the pins of test_oracle.py
(hand-derived cases and the O(N^2) brute force) fail for it.  The real oracle is untouched.
"""
import json
import os

import numpy as np
import pytest

import oracle
from long_context_attention_la_b200 import synth
from tests.test_oracle import GOLDEN, _f32, _rand, brute_force

SRC = os.path.join(os.path.dirname(oracle.__file__), "la_oracle.c")

MUTANTS = {
    "no_decay": ("Si[j] = lambda * Si[j] + ki * vt[j];", "Si[j] = Si[j] + ki * vt[j];"),
    "decay_sign": ("exp(-(double)slopes[h])", "exp((double)slopes[h])"),
    "wrong_head_slope": ("const double lambda = exp(-(double)slopes[h]);\n    double* S",
                         "const double lambda = exp(-(double)slopes[(h + 1) % H]);\n    double* S"),
    "transposed_readout": ("ot[j] += qi * Si[j];", "ot[j] += qi * S[j * d + i];"),
    "readout_before_update": ("          Si[j] = lambda * Si[j] + ki * vt[j];\n          ot[j] += qi * Si[j];",
                              "          ot[j] += qi * Si[j];\n          Si[j] = lambda * Si[j] + ki * vt[j];"),
    "head_major_layout": ("const int64_t row = ((b * N + t) * H + h) * d;",
                          "const int64_t row = ((b * H + h) * N + t) * d;"),
    "k_v_swapped": ("Si[j] = lambda * Si[j] + ki * vt[j];", "Si[j] = lambda * Si[j] + vt[i] * kt[j];"),
}


def _pins_pass(lib) -> bool:
    for case in json.load(open(GOLDEN))["cases"]:
        B, N, H, d = case["B"], case["N"], case["H"], case["d"]
        q, k, v = (_f32(case[x]).reshape(B, N, H, d) for x in "qkv")
        o, st = oracle.prefill(q, k, v, _f32(case["slopes"]), lib=lib)
        o = o.reshape(B, H, N, d).transpose(0, 2, 1, 3)
        if not (np.allclose(o.ravel(), case["o"], rtol=max(case["rtol"], 1e-12), atol=1e-12)
                and np.allclose(st.ravel(), case["state"], rtol=max(case["rtol"], 1e-12),
                                atol=1e-12)):
            return False
    B, N, H, d = 2, 40, 3, 4
    q, k, v = _rand(B, N, H, d, 21)
    sl = synth.slopes(H).numpy()
    o, st = oracle.prefill(q, k, v, sl, lib=lib)
    o = o.reshape(B, H, N, d).transpose(0, 2, 1, 3)
    ob, sb = brute_force(q, k, v, sl)
    return bool(np.allclose(o, ob, rtol=1e-10, atol=1e-10) and
                np.allclose(st.reshape(B, H, d, d), sb, rtol=1e-10, atol=1e-10))


def test_unmutated_copy_passes(tmp_path):
    src = tmp_path / "copy.c"
    src.write_text(open(SRC).read())
    lib = oracle.open_library(oracle.compile_source(str(src), str(tmp_path / "libcopy.so")))
    assert _pins_pass(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    src = tmp_path / f"{name}.c"
    src.write_text(text.replace(old, new, 1))  # first site: the prefill loop
    lib = oracle.open_library(oracle.compile_source(str(src), str(tmp_path / f"lib{name}.so")))
    assert not _pins_pass(lib), f"the pins did not catch the planted mistake {name}"
