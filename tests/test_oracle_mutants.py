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


# The fold of part states (oracle.fold_states): each mutant is planted in a copy of the function's
# source, executed on the CPU, and must fail the context-parallel invariant of test_oracle.py.
FOLD_MUTANTS = {
    "fold_decays_h_too": ("S = lam_l * S + parts[j]", "S = lam_l * (S + parts[j])"),
    "fold_no_decay": ("S = lam_l * S + parts[j]", "S = S + parts[j]"),
    "fold_next_part_length": ("np.exp(-sl * lengths[j])",
                              "np.exp(-sl * lengths[min(j + 1, n - 1)])"),
    "fold_reversed_order": ("for j in range(n):", "for j in reversed(range(n)):"),
    "fold_head_axis_wrong": ("[None, :, None, None]", "[None, None, :, None]"),
}


def _fold_from_source(src: str):
    ns = {"np": np}
    exec(compile(src, "<fold mutant>", "exec"), ns)  # noqa: S102 - test-only source mutation
    return ns["fold_states"]


def _fold_pins_pass(fold) -> bool:
    from tests.test_oracle import _part_states
    B, N, H, d = 2, 40, 3, 5
    q, k, v = _rand(B, N, H, d, 31)
    sl = np.array([0.05, 0.7, 2.5], dtype=np.float32)
    s0 = np.random.default_rng(32).normal(size=(B, H, d, d))
    _, st0 = oracle.prefill(q, k, v, sl, state_in=s0.reshape(B * H, d, d))
    for cuts in ([0, 13, 40], [0, 7, 7, 25, 40], [0, 1, 2, 3, 40]):
        S = fold(_part_states(q, k, v, sl, cuts), np.diff(cuts), sl, state_in=s0)
        if S.shape != (B, H, d, d) or not np.allclose(S, st0.reshape(B, H, d, d), rtol=1e-12,
                                                      atol=1e-12):
            return False
    return True


def test_unmutated_fold_copy_passes():
    import inspect
    assert _fold_pins_pass(_fold_from_source(inspect.getsource(oracle.fold_states)))


@pytest.mark.parametrize("name", sorted(FOLD_MUTANTS))
def test_fold_mutant_is_caught(name):
    import inspect
    old, new = FOLD_MUTANTS[name]
    text = inspect.getsource(oracle.fold_states)
    assert text.count(old) == 1, f"mutation site for {name} not found"
    try:
        ok = _fold_pins_pass(_fold_from_source(text.replace(old, new)))
    except (ValueError, IndexError):
        ok = False  # a shape error is a failed pin too
    assert not ok, f"the pins did not catch the planted mistake {name}"
