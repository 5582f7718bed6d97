"""Pins of the fp64 oracle against things other than itself (CPU only).

The report (Ling and Ring 2.6 Technical Report, Chinese translation, garden.houmin.site) prints
no numeric example for the kernel, so the oracle is pinned by:
  * hand-derived worked examples (tests/golden/hand_cases.json);
  * the textbook O(N^2) form  o_t = sum_{s<=t} lambda^(t-s) (q_t . k_s) v_s  (numpy, fp64, with
    lambda^(t-s) from exp, not from repeated multiplication), and the state
    S = sum_s lambda^(N-1-s) k_s^T v_s;
  * closed forms: lambda = 1 is a causal cumulative sum of outer products; lambda = 0 keeps only
    the diagonal; N = 1 is (q.k) v;
  * invariants: linearity in v and q, prefix causality, decode-after-prefill, resume from a state.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_la_b200 import synth
from tests.helpers import oracle_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _rand(B, N, H, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return tuple(_f32(rng.standard_normal((B, N, H, d)) * scale) for _ in range(3))


def brute_force(q, k, v, slopes):
    """O(N^2) decayed masked attention in fp64 (independent of the recurrence)."""
    q = q.astype(np.float64)
    k = k.astype(np.float64)
    v = v.astype(np.float64)
    B, N, H, d = q.shape
    o = np.zeros((B, N, H, d))
    st = np.zeros((B, H, d, d))
    t = np.arange(N)
    for b in range(B):
        for h in range(H):
            s = float(np.float32(slopes[h]))
            diff = t[:, None] - t[None, :]
            decay = np.where(diff >= 0, np.exp(-np.maximum(diff, 0) * s), 0.0)
            A = (q[b, :, h, :] @ k[b, :, h, :].T) * decay
            o[b, :, h, :] = A @ v[b, :, h, :]
            w = np.exp(-(N - 1 - t) * s)
            st[b, h] = (k[b, :, h, :] * w[:, None]).T @ v[b, :, h, :]
    return o, st


def run_oracle(q, k, v, slopes, **kw):
    B, N, H, d = q.shape
    o, st = oracle.prefill(q, k, v, _f32(slopes), **kw)
    return o.reshape(B, H, -1, d).transpose(0, 2, 1, 3), st.reshape(B, H, d, d)


def test_oracle_builds():
    assert os.path.exists(oracle.build())
    assert oracle.num_threads(3) == 3


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_cases(case):
    B, N, H, d = case["B"], case["N"], case["H"], case["d"]
    q = _f32(case["q"]).reshape(B, N, H, d)
    k = _f32(case["k"]).reshape(B, N, H, d)
    v = _f32(case["v"]).reshape(B, N, H, d)
    o, st = run_oracle(q, k, v, case["slopes"])
    exp_o = np.asarray(case["o"], dtype=np.float64).reshape(B, N, H, d)
    exp_s = np.asarray(case["state"], dtype=np.float64).reshape(B, H, d, d)
    np.testing.assert_allclose(o, exp_o, rtol=case["rtol"], atol=0)
    np.testing.assert_allclose(st, exp_s, rtol=case["rtol"], atol=0)


@pytest.mark.parametrize("B,N,H,d,seed", [(1, 1, 1, 4, 0), (2, 37, 3, 4, 1), (1, 300, 2, 64, 2),
                                          (1, 512, 1, 4, 3), (2, 129, 4, 8, 4)])
def test_brute_force(B, N, H, d, seed):
    q, k, v = _rand(B, N, H, d, seed)
    sl = synth.slopes(H).numpy()
    o, st = run_oracle(q, k, v, sl)
    ob, sb = brute_force(q, k, v, sl)
    scale_o = np.max(np.abs(ob))
    scale_s = np.max(np.abs(sb))
    assert np.max(np.abs(o - ob)) <= 1e-12 * max(scale_o, 1.0) * np.sqrt(N)
    assert np.max(np.abs(st - sb)) <= 1e-12 * max(scale_s, 1.0) * np.sqrt(N)


def test_brute_force_wide_slopes():
    # Slopes spanning no decay to fast decay in one call, with per-head checks.
    B, N, H, d = 1, 200, 4, 16
    q, k, v = _rand(B, N, H, d, 11)
    sl = np.array([0.0, 1e-3, 0.3, 2.0], dtype=np.float32)
    o, st = run_oracle(q, k, v, sl)
    ob, sb = brute_force(q, k, v, sl)
    for h in range(H):
        np.testing.assert_allclose(o[:, :, h], ob[:, :, h], rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(st[:, h], sb[:, h], rtol=1e-11, atol=1e-11)


def test_lambda_one_is_causal_cumsum():
    B, N, H, d = 1, 64, 2, 8
    q, k, v = _rand(B, N, H, d, 5)
    sl = np.zeros(H, dtype=np.float32)
    o, st = run_oracle(q, k, v, sl)
    qd, kd, vd = (x.astype(np.float64) for x in (q, k, v))
    outer = np.einsum("bnhi,bnhj->bnhij", kd, vd)
    C = np.cumsum(outer, axis=1)
    expect = np.einsum("bnhi,bnhij->bnhj", qd, C)
    np.testing.assert_allclose(o, expect, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st, C[:, -1], rtol=1e-12, atol=1e-12)


def test_lambda_zero_keeps_diagonal():
    B, N, H, d = 2, 17, 2, 8
    q, k, v = _rand(B, N, H, d, 6)
    sl = np.full(H, 1e4, dtype=np.float32)  # exp(-1e4) underflows to exactly 0 in double
    o, st = run_oracle(q, k, v, sl)
    qd, kd, vd = (x.astype(np.float64) for x in (q, k, v))
    diag = np.einsum("bnhi,bnhi->bnh", qd, kd)[..., None] * vd
    np.testing.assert_allclose(o, diag, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(st, np.einsum("bhi,bhj->bhij", kd[:, -1], vd[:, -1]), rtol=0, atol=0)


def test_single_token():
    q, k, v = _rand(3, 1, 2, 16, 7)
    o, st = run_oracle(q, k, v, synth.slopes(2).numpy())
    qd, kd, vd = (x.astype(np.float64) for x in (q, k, v))
    np.testing.assert_allclose(o[:, 0], np.einsum("bhi,bhi->bh", qd[:, 0], kd[:, 0])[..., None]
                               * vd[:, 0], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(st, np.einsum("bhi,bhj->bhij", kd[:, 0], vd[:, 0]), rtol=0, atol=0)


def test_linearity():
    q, k, v = _rand(1, 50, 2, 8, 8)
    sl = synth.slopes(2).numpy()
    o, st = run_oracle(q, k, v, sl)
    o2, st2 = run_oracle(q, k, _f32(2 * v), sl)          # scaling by 2 is exact
    np.testing.assert_array_equal(o2, 2 * o)
    np.testing.assert_array_equal(st2, 2 * st)
    o3, _ = run_oracle(_f32(2 * q), k, v, sl)
    np.testing.assert_array_equal(o3, 2 * o)
    # additivity in v (catches a dropped term that scaling alone would not); values on a 2^-10
    # grid so that v + w is exact in float32
    _, _, w = _rand(1, 50, 2, 8, 9)
    vg = _f32(np.round(v * 1024) / 1024)
    wg = _f32(np.round(w * 1024) / 1024)
    assert np.array_equal(_f32(vg + wg).astype(np.float64), vg.astype(np.float64) + wg)
    og, _ = run_oracle(q, k, vg, sl)
    oa, _ = run_oracle(q, k, wg, sl)
    ob, _ = run_oracle(q, k, _f32(vg + wg), sl)
    np.testing.assert_allclose(ob, og + oa, rtol=1e-12, atol=1e-12)


def test_prefix_causality():
    q, k, v = _rand(2, 90, 2, 8, 10)
    sl = synth.slopes(2).numpy()
    o, _ = run_oracle(q, k, v, sl)
    o_short, _ = run_oracle(*(np.ascontiguousarray(x[:, :33]) for x in (q, k, v)), sl)
    np.testing.assert_array_equal(o[:, :33], o_short)


def test_bf16_bits_upcast_exactly():
    t = torch.randn(1, 20, 2, 8, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    bits = oracle_bits(t)
    as_f32 = t.float().numpy()
    sl = synth.slopes(2).numpy()
    o1, s1 = run_oracle(bits, bits, bits, sl)
    o2, s2 = run_oracle(as_f32, as_f32, as_f32, sl)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_decode_equals_prefill():
    B, N, H, d = 2, 12, 3, 8
    q, k, v = _rand(B, N, H, d, 12)
    sl = synth.slopes(H).numpy()
    o, st = run_oracle(q, k, v, sl)
    S = np.zeros((B, H, d, d))
    for t in range(N):
        ot = oracle.decode(q[:, t], k[:, t], v[:, t], sl, S)
        np.testing.assert_array_equal(ot, o[:, t])
    np.testing.assert_array_equal(S, st)


def test_resume_from_state():
    B, N, H, d = 1, 40, 2, 8
    q, k, v = _rand(B, N, H, d, 13)
    sl = synth.slopes(H).numpy()
    o, st = run_oracle(q, k, v, sl)
    n1 = 15
    _, s1 = oracle.prefill(*(np.ascontiguousarray(x[:, :n1]) for x in (q, k, v)), sl)
    o2, s2 = oracle.prefill(*(np.ascontiguousarray(x[:, n1:]) for x in (q, k, v)), sl, state_in=s1)
    np.testing.assert_array_equal(o2.reshape(B, H, -1, d).transpose(0, 2, 1, 3), o[:, n1:])
    np.testing.assert_array_equal(s2.reshape(B, H, d, d), st)


def test_head_and_token_selection():
    B, N, H, d = 2, 30, 3, 4
    q, k, v = _rand(B, N, H, d, 14)
    sl = synth.slopes(H).numpy()
    o_all, st_all = oracle.prefill(q, k, v, sl)
    heads = [5, 1, 3]
    tsel = [0, 7, 29]
    o_sel, st_sel = oracle.prefill(q, k, v, sl, heads=heads, t_sel=tsel, nthreads=2)
    np.testing.assert_array_equal(o_sel, o_all[heads][:, tsel])
    np.testing.assert_array_equal(st_sel, st_all[heads])


def test_thread_count_invariance():
    q, k, v = _rand(1, 64, 8, 8, 15)
    sl = synth.slopes(8).numpy()
    a = oracle.prefill(q, k, v, sl, nthreads=1)
    b = oracle.prefill(q, k, v, sl, nthreads=4)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_rejects_bad_arguments():
    q, k, v = _rand(1, 4, 2, 4, 16)
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v, np.zeros(3, np.float32))
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v, np.zeros(2, np.float32), t_sel=[3, 1])
    with pytest.raises(TypeError):
        oracle.prefill(q.astype(np.float64), k, v, np.zeros(2, np.float32))


def test_slope_schedule_values():
    # Decays quoted for the schedule s_h = 2^(-8(h+1)/H): H=64 -> 0.39972 .. 0.99610,
    # H=2 -> 0.93941, 0.99610.
    lam64 = np.exp(-synth.slopes(64).double().numpy())
    lam2 = np.exp(-synth.slopes(2).double().numpy())
    assert abs(lam64[0] - 0.39972) < 1e-5 and abs(lam64[63] - 0.99610) < 1e-5
    assert abs(lam2[0] - 0.93941) < 1e-5 and abs(lam2[1] - 0.99610) < 1e-5


# ---------------------------------------------------------------------------------------------
# gated_rmsnorm: the grouped RMSNorm + sigmoid gate after the kernel
# ---------------------------------------------------------------------------------------------
def test_gated_rmsnorm_hand_case():
    # one head of d = 4: o = [1, 2, 3, 4] has mean square 30/4 = 7.5; gamma = [1, 1, 2, 2];
    # g = 0 gives sigmoid 1/2, so y = [1, 2, 6, 8] / (2 sqrt(7.5))
    o = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    gamma = np.array([[1.0, 1.0, 2.0, 2.0]], dtype=np.float32)
    y = oracle.gated_rmsnorm(o, np.zeros((1, 1, 4), np.float32), gamma, 0.0)
    want = np.array([1.0, 2.0, 6.0, 8.0]) / (2.0 * np.sqrt(7.5))
    assert np.allclose(y[0, 0], want, rtol=1e-15, atol=0)
    # epsilon enters under the root: mean square 7.5 + 0.5 = 8
    y = oracle.gated_rmsnorm(o, np.zeros((1, 1, 4), np.float32), gamma, 0.5)
    assert np.allclose(y[0, 0], np.array([1.0, 2.0, 6.0, 8.0]) / (2.0 * np.sqrt(8.0)), rtol=1e-15)


def test_gated_rmsnorm_groups_are_heads_and_gate_is_elementwise():
    rng = np.random.default_rng(5)
    o = rng.standard_normal((3, 2, 8))                 # [tokens, H, d]
    g = rng.standard_normal((3, 2, 8)).astype(np.float32)
    gamma = rng.standard_normal((2, 8)).astype(np.float32)
    y = oracle.gated_rmsnorm(o, g, gamma, 0.0)
    # scale invariance per head (eps = 0): scaling one head's vector leaves y unchanged
    o2 = o.copy()
    o2[1, 0] *= 37.0
    assert np.allclose(oracle.gated_rmsnorm(o2, g, gamma, 0.0), y, rtol=1e-13, atol=0)
    # each head normalised on its own: with gamma = 1 and a saturated gate, mean(y^2) = 1 per head
    big = np.full(o.shape, 60.0, np.float32)
    y1 = oracle.gated_rmsnorm(o, big, np.ones((2, 8), np.float32), 0.0)
    assert np.allclose(np.mean(y1 * y1, axis=-1), 1.0, rtol=1e-13)
    # sigmoid(g) + sigmoid(-g) = 1
    y_neg = oracle.gated_rmsnorm(o, -g, gamma, 0.0)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True))
    assert np.allclose(y + y_neg, gamma.astype(np.float64) * o / rms, rtol=1e-12, atol=1e-14)


def test_gated_rmsnorm_reads_bf16_bits_exactly():
    g = np.array([0x3F80, 0xC000, 0x0000, 0x3F00], dtype=np.uint16).reshape(1, 1, 4)  # 1,-2,0,0.5
    o = np.ones((1, 1, 4))
    y = oracle.gated_rmsnorm(o, g, np.ones((1, 4), np.float32), 0.0)
    sig = 1.0 / (1.0 + np.exp(-np.array([1.0, -2.0, 0.0, 0.5])))
    assert np.array_equal(y[0, 0], sig)


# ---------------------------------------------------------------------------------------------
# FP8 E4M3 quantize of the fused post-kernel operator
# ---------------------------------------------------------------------------------------------
def test_e4m3_hand_codes():
    # from the format: code = sign << 7 | (exponent + 7) << 3 | mantissa; exponent field 0 holds
    # m * 2^-9; ties round to the even mantissa; magnitudes above 448 saturate to 0x7E
    cases = [(1.0, 0x38), (-2.0, 0xC0), (448.0, 0x7E), (0.5, 0x30), (1.75, 0x3E), (2.0 ** -6, 0x08),
             (2.0 ** -9, 0x01), (7 * 2.0 ** -9, 0x07), (0.0, 0x00), (-0.0, 0x80),
             (1.0625, 0x38),            # halfway 1 .. 1.125: even mantissa 0
             (1.1875, 0x3A),            # halfway 1.125 .. 1.25: even mantissa 2
             (2.0 ** -10, 0x00),        # halfway 0 .. 2^-9: even 0
             (3 * 2.0 ** -10, 0x02),    # halfway 2^-9 .. 2^-8: even 2
             (15 * 2.0 ** -10, 0x08),   # halfway 7 * 2^-9 .. 2^-6: carries into the normals
             (1.96875, 0x40),           # halfway 1.875 .. 2: carries into the next exponent
             (464.0, 0x7E), (1.0e6, 0x7E), (-600.0, 0xFE)]
    x = np.array([c[0] for c in cases])
    assert oracle.e4m3_encode(x).tolist() == [c[1] for c in cases]


def test_e4m3_round_trip_and_order():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254 and np.isnan(vals[[0x7F, 0xFF]]).all()
    assert np.array_equal(oracle.e4m3_encode(vals[finite]), codes[finite])
    pos = vals[:0x7F]
    assert np.all(np.diff(pos) > 0) and pos[-1] == 448.0 and pos[1] == 2.0 ** -9


def test_e4m3_matches_torch_conversion():
    # torch's float8_e4m3fn conversion (a library routine, CPU) rounds to nearest even; it does not
    # saturate past 464, so the sweep stays within +-464
    reps = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = 0.5 * (reps[1:] + reps[:-1])
    rng = np.random.default_rng(9)
    x = np.concatenate([reps, mids, -mids, rng.uniform(-464, 464, 20000),
                        rng.standard_normal(20000) * 2.0 ** -7, [464.0, -464.0]]).astype(np.float32)
    ours = oracle.e4m3_encode(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_gated_rmsnorm_fp8_blocks():
    rng = np.random.default_rng(6)
    o = rng.standard_normal((5, 3, 16)) * rng.uniform(0.01, 100, (5, 3, 1))
    g = rng.standard_normal((5, 3, 16)).astype(np.float32)
    gamma = rng.standard_normal((3, 16)).astype(np.float32)
    o[2, 1] = 0.0  # an all-zero block (eps > 0 keeps y finite: y = 0)
    codes, scale = oracle.gated_rmsnorm_fp8(o, g, gamma, 1e-6)
    y = oracle.gated_rmsnorm(o, g, gamma, 1e-6)
    assert codes.shape == o.shape and codes.dtype == np.uint8 and scale.shape == (5, 3)
    amax = np.max(np.abs(y), axis=-1)
    assert np.allclose(scale, amax / 448.0, rtol=1e-15, atol=0)
    assert scale[2, 1] == 0.0 and not (codes[2, 1] & 0x7F).any()  # signed zeros
    # the block's largest magnitude maps to the largest code, with y's sign
    j = np.argmax(np.abs(y), axis=-1)
    top = np.take_along_axis(codes, j[..., None], axis=-1)[..., 0]
    sgn = np.take_along_axis(y, j[..., None], axis=-1)[..., 0] < 0
    live = amax > 0
    assert np.array_equal(top[live] & 0x7F, np.full(live.sum(), 0x7E))
    assert np.array_equal((top[live] >> 7).astype(bool), sgn[live])
    # dequantized values are within half an E4M3 step of y (3 mantissa bits: relative 2^-4 for
    # normals, absolute 2^-10 * scale for the subnormals)
    deq = oracle.e4m3_decode(codes) * scale[..., None]
    bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10 * scale[..., None]) * (1 + 1e-12)
    assert np.all(np.abs(deq - y) <= bound)


def test_fp8_bar_accepts_reference_and_rejects_corruptions():
    """The GPU tests' FP8 bar (tests.helpers.check_fp8) passes the reference quantization of y
    itself and fails codes two steps off, a wrong scale, and codes of the wrong sign."""
    from tests.helpers import check_fp8
    rng = np.random.default_rng(12)
    y = rng.standard_normal((40, 3, 128)) * rng.uniform(0.1, 10, (40, 3, 1))
    y32 = y.astype(np.float32)
    amax = np.max(np.abs(y32), axis=-1)
    codes = oracle.e4m3_encode((y32 * (np.float32(448) / amax)[..., None]).astype(np.float64))
    scales = (amax / 448.0).astype(np.float32).T.copy()
    check_fp8(codes, scales, y, io_dtype=torch.float32)
    bad = codes.copy()
    mid = np.argwhere((np.abs(oracle.e4m3_decode(codes)) >= 64) &
                      (np.abs(oracle.e4m3_decode(codes)) < 256))[0]
    bad[tuple(mid)] = bad[tuple(mid)] + 2  # two steps up in magnitude, below saturation
    with pytest.raises(AssertionError):
        check_fp8(bad, scales, y, io_dtype=torch.float32)
    s_bad = scales.copy()
    s_bad[2, 9] *= 1.05
    with pytest.raises(AssertionError):
        check_fp8(codes, s_bad, y, io_dtype=torch.float32)
    with pytest.raises(AssertionError):
        check_fp8(codes ^ 0x80, scales, y, io_dtype=torch.float32)


# ---------------------------------------------------------------------------------------------
# qk_norm_rope: QK RMSNorm + partial rotary embedding before the kernel
# ---------------------------------------------------------------------------------------------
def test_qk_norm_rope_hand_case():
    # d = 4, r = 2, theta irrelevant for i = 0 (w_0 = 1): x = [1, 0, 1, 1] has mean square 3/4;
    # at position 1 the pair (y_0, y_1) turns by 1 radian, dims 2, 3 are only normalised
    x = np.array([[[1.0, 0.0, 1.0, 1.0]]], dtype=np.float32)
    y = oracle.qk_norm_rope(x, np.ones(4, np.float32), [1], 2, 10000.0, 0.0)
    s = 1.0 / np.sqrt(0.75)
    want = np.array([s * np.cos(1.0), s * np.sin(1.0), s, s])
    assert np.allclose(y[0, 0], want, rtol=1e-15, atol=1e-15)
    # the second frequency of r = 4: w_1 = theta^(-1/2); pair (y_1, y_3) turns by pos * w_1
    x = np.array([[[0.0, 1.0, 0.0, 0.0]]], dtype=np.float32)
    y = oracle.qk_norm_rope(x, np.ones(4, np.float32), [3], 4, 100.0, 0.0)
    a = 3.0 / 10.0
    assert np.allclose(y[0, 0], [0.0, 2.0 * np.cos(a), 0.0, 2.0 * np.sin(a)], atol=1e-15)


def test_qk_norm_rope_invariants():
    rng = np.random.default_rng(9)
    T, H, d, r = 6, 3, 16, 8
    x = rng.standard_normal((T, H, d)).astype(np.float32)
    gamma = rng.standard_normal(d).astype(np.float32)
    pos = rng.integers(0, 100000, T)
    y = oracle.qk_norm_rope(x, gamma, pos, r, 6.0e6, 1e-6)
    y0 = oracle.qk_norm_rope(x, gamma, np.zeros(T, np.int64), r, 6.0e6, 1e-6)
    # position 0 is the plain RMSNorm
    xd = x.astype(np.float64)
    plain = gamma.astype(np.float64) * xd / np.sqrt(np.mean(xd * xd, -1, keepdims=True) + 1e-6)
    assert np.allclose(y0, plain, rtol=1e-14, atol=1e-15)
    # rotation keeps each pair's length; dims >= r are untouched by it
    h = r // 2
    assert np.allclose(y[..., :h] ** 2 + y[..., h:r] ** 2, plain[..., :h] ** 2 + plain[..., h:r] ** 2,
                       rtol=1e-12)
    assert np.array_equal(y[..., r:], plain[..., r:])
    # relative positions: <rope(q, m), rope(k, n)> depends on m - n only
    q = oracle.qk_norm_rope(x[:1], gamma, [1000], r, 6.0e6, 1e-6)
    k = oracle.qk_norm_rope(x[1:2], gamma, [400], r, 6.0e6, 1e-6)
    q2 = oracle.qk_norm_rope(x[:1], gamma, [1000 + 77777], r, 6.0e6, 1e-6)
    k2 = oracle.qk_norm_rope(x[1:2], gamma, [400 + 77777], r, 6.0e6, 1e-6)
    assert np.allclose(np.sum(q * k, -1), np.sum(q2 * k2, -1), rtol=1e-9)


def _part_states(q, k, v, sl, cuts):
    """Local states (each from zero) of the parts [cuts[j], cuts[j+1]) of the token axis."""
    B, N, H, d = q.shape
    hs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        if b == a:
            hs.append(np.zeros((B, H, d, d)))
            continue
        _, st = oracle.prefill(q[:, a:b].copy(), k[:, a:b].copy(), v[:, a:b].copy(), sl)
        hs.append(st.reshape(B, H, d, d))
    return np.stack(hs)


@pytest.mark.parametrize("cuts", [[0, 13, 40], [0, 7, 7, 25, 40], [0, 1, 2, 3, 40], [0, 40]])
def test_fold_of_part_states_equals_sequential_state(cuts):
    """The context-parallel invariant of §4.1.1 (local recurrence, then global correction):
    folding the parts' local states gives the state of one sequential pass, for any cut."""
    B, N, H, d = 2, 40, 3, 5
    q, k, v = _rand(B, N, H, d, 31)
    sl = np.array([0.05, 0.7, 2.5], dtype=np.float32)
    _, st = oracle.prefill(q, k, v, sl)
    S = oracle.fold_states(_part_states(q, k, v, sl, cuts), np.diff(cuts), sl)
    np.testing.assert_allclose(S, st.reshape(B, H, d, d), rtol=1e-12, atol=1e-12)
    # with an initial state (a cached prefix)
    s0 = np.random.default_rng(32).normal(size=(B, H, d, d))
    _, st0 = oracle.prefill(q, k, v, sl, state_in=s0.reshape(B * H, d, d))
    S0 = oracle.fold_states(_part_states(q, k, v, sl, cuts), np.diff(cuts), sl, state_in=s0)
    np.testing.assert_allclose(S0, st0.reshape(B, H, d, d), rtol=1e-12, atol=1e-12)
    # the incoming state of part r continues the sequence exactly where part r starts
    r = len(cuts) - 2
    hs = _part_states(q, k, v, sl, cuts)
    Sr = oracle.fold_states(hs[:r], np.diff(cuts)[:r], sl, state_in=s0)
    a = cuts[r]
    o_tail, _ = oracle.prefill(q[:, a:].copy(), k[:, a:].copy(), v[:, a:].copy(), sl,
                               state_in=Sr.reshape(B * H, d, d))
    o_all, _ = oracle.prefill(q, k, v, sl, state_in=s0.reshape(B * H, d, d))
    np.testing.assert_allclose(o_tail, o_all[:, a:], rtol=1e-12, atol=1e-12)


def test_fold_closed_forms():
    """lambda = 1: the fold is state_in plus the plain sum of the parts; lambda^L = 0 (a long
    part with a large slope): the state before that part is forgotten; no parts: state_in."""
    rng = np.random.default_rng(33)
    n, B, H, d = 3, 2, 2, 4
    parts = rng.normal(size=(n, B, H, d, d))
    s0 = rng.normal(size=(B, H, d, d))
    np.testing.assert_allclose(oracle.fold_states(parts, [5, 9, 2], np.zeros(H, np.float32),
                                                  state_in=s0),
                               s0 + parts.sum(axis=0), rtol=1e-13, atol=1e-13)
    big = np.full(H, 50.0, dtype=np.float32)  # exp(-50 * 40) underflows to exactly 0
    np.testing.assert_array_equal(oracle.fold_states(parts, [40, 40, 40], big, state_in=s0),
                                  parts[2])
    np.testing.assert_array_equal(oracle.fold_states(parts[:0], [], big, state_in=s0), s0)
    # one part: lambda^L S_in + h, per head with its own lambda
    sl = np.array([0.1, 0.9], dtype=np.float32)
    lam = np.exp(-sl.astype(np.float64) * 7)
    want = lam[None, :, None, None] * s0 + parts[0]
    np.testing.assert_allclose(oracle.fold_states(parts[:1], [7], sl, state_in=s0), want,
                               rtol=1e-14, atol=1e-14)

