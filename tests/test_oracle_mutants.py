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


# The FP8 E4M3 encoder (oracle.e4m3_encode): each mutant must fail the format's hand codes or the
# comparison with torch's conversion in test_oracle.py.
E4M3_MUTANTS = {
    "e4m3_bias_8": ("((e_n + 7) << 3)", "((e_n + 8) << 3)"),
    "e4m3_round_half_up": ("np.rint((2.0 * frac - 1.0) * 8.0)", "np.floor((2.0 * frac - 1.0) * 8.0 + 0.5)"),
    "e4m3_truncate": ("np.rint((2.0 * frac - 1.0) * 8.0)", "np.floor((2.0 * frac - 1.0) * 8.0)"),
    "e4m3_no_carry": ("e_n = e + (mant_n == 8)", "e_n = e"),
    "e4m3_subnormal_step": ("np.rint(a / 2.0 ** -9)", "np.rint(a / 2.0 ** -10)"),
    "e4m3_no_saturation": ("np.minimum(np.abs(x), E4M3_MAX)", "np.abs(x)"),
    "e4m3_sign_lost": ("return code | sign", "return code"),
}


def _e4m3_pins_pass(encode) -> bool:
    import tests.test_oracle as t
    saved = oracle.e4m3_encode
    oracle.e4m3_encode = encode
    try:
        for pin in (t.test_e4m3_hand_codes, t.test_e4m3_matches_torch_conversion):
            try:
                pin()
            except (AssertionError, ValueError, OverflowError):
                return False
        return True
    finally:
        oracle.e4m3_encode = saved


def _encode_from_source(src: str):
    ns = {"np": np, "E4M3_MAX": oracle.E4M3_MAX}
    with np.errstate(all="ignore"):
        exec(compile(src, "<e4m3 mutant>", "exec"), ns)  # noqa: S102 - test-only source mutation
    return ns["e4m3_encode"]


def test_unmutated_e4m3_copy_passes():
    import inspect
    assert _e4m3_pins_pass(_encode_from_source(inspect.getsource(oracle.e4m3_encode)))


@pytest.mark.parametrize("name", sorted(E4M3_MUTANTS))
def test_e4m3_mutant_is_caught(name):
    import inspect
    old, new = E4M3_MUTANTS[name]
    text = inspect.getsource(oracle.e4m3_encode)
    assert text.count(old) == 1, f"mutation site for {name} not found"
    with np.errstate(all="ignore"):
        ok = _e4m3_pins_pass(_encode_from_source(text.replace(old, new)))
    assert not ok, f"the pins did not catch the planted mistake {name}"
