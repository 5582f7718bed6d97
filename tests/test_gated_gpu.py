"""The fused grouped RMSNorm + sigmoid gate epilogue of la_prefill_varlen against the fp64 oracle,
on a GPU, through the C ABI.

Reference: oracle.prefill gives o in fp64; oracle.gated_rmsnorm applies, per token and head,
y = gamma * o / sqrt(mean(o^2) + eps) * sigmoid(g) in fp64 on the same gate bits.  Bar: bf16
relL2 <= 1e-2 and maxabs <= 2e-2 * max|ref| on y (the epilogue rounds O to bf16 once before the
norm, as the unfused layer's norm reads a bf16 o, and once after the gate).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_attention_la_b200 import la, synth
from tests.helpers import check_close, check_fp8, oracle_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"
EPS = 1e-6


def draw_packed(lengths, H, d, seed, dist="scaled_normal"):
    T = sum(lengths)
    q, k, v = synth.draw_qkv(1, max(T, 1), H, d, dist=dist, seed=seed, device=DEV)
    return q[0, :T].contiguous(), k[0, :T].contiguous(), v[0, :T].contiguous()


def draw_gate(T, H, d, seed, scale=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    x = torch.randn((T, H, d), generator=g, device=DEV) * scale
    gamma = 1.0 + 0.5 * torch.randn((H, d), generator=g, device=DEV)
    return x.to(torch.bfloat16), gamma.float().contiguous()


def reference(q, k, v, sl, cu, gate, gamma, eps, state_in=None, heads=None):
    """fp64 y [tokens, n_heads, d] for every sequence, concatenated along tokens."""
    ys = []
    H = q.shape[1]
    hs = list(range(H)) if heads is None else list(heads)
    gam = gamma.cpu().numpy()[hs]
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b == a:
            continue
        sin = None if state_in is None else state_in[s].double().cpu().numpy()[hs]
        o, _ = oracle.prefill(oracle_bits(q[a:b].unsqueeze(0)), oracle_bits(k[a:b].unsqueeze(0)),
                              oracle_bits(v[a:b].unsqueeze(0)), sl.cpu().numpy(),
                              heads=None if heads is None else hs, state_in=sin)
        o = np.transpose(o, (1, 0, 2))  # [len, n_heads, d]
        gb = oracle_bits(gate[a:b][:, hs].contiguous())
        ys.append(oracle.gated_rmsnorm(o, gb, gam, eps))
    return np.concatenate(ys, axis=0)


@pytest.mark.parametrize("chunk", [64, 128, 256])
@pytest.mark.parametrize("segments", [0, 3])
def test_gated_epilogue_edge_lengths(segments, chunk):
    H, d = 4, 128
    lengths = [1, 127, 128, 129, 0, 300, 1000, 2049, 5]
    cu = synth.cu_from_lengths(lengths)
    q, k, v = draw_packed(lengths, H, d, seed=101)
    sl = synth.slopes(H, DEV)
    gate, gamma = draw_gate(sum(lengths), H, d, seed=102)
    sin = synth.draw_states(len(lengths), H, d, seed=103, scale=0.3, device=DEV)
    y, st = la.prefill_varlen(q, k, v, sl, cu, state_in=sin, gate=gate, gamma=gamma, eps=EPS,
                              segments=segments, chunk=chunk)
    torch.cuda.synchronize()
    ref = reference(q, k, v, sl, cu, gate, gamma, EPS, state_in=sin)
    check_close(y.float().cpu().numpy(), ref, torch.bfloat16, "y")


def test_gated_epilogue_saturated_gate_and_large_eps():
    """Gate pre-activations of scale 6 drive the sigmoid into both tails, and eps = 0.5 is
    comparable to the mean square of o, so the epsilon term is exercised."""
    H, d = 8, 128
    lengths = [700, 333]
    cu = synth.cu_from_lengths(lengths)
    q, k, v = draw_packed(lengths, H, d, seed=111, dist="silu_qk")
    sl = synth.slopes(H, DEV)
    gate, gamma = draw_gate(sum(lengths), H, d, seed=112, scale=6.0)
    for eps in (0.0, 0.5):
        y, _ = la.prefill_varlen(q, k, v, sl, cu, gate=gate, gamma=gamma, eps=eps)
        torch.cuda.synchronize()
        check_close(y.float().cpu().numpy(), reference(q, k, v, sl, cu, gate, gamma, eps),
                    torch.bfloat16, f"y eps={eps}")


def test_gated_epilogue_matches_norm_applied_to_plain_output():
    """The fused epilogue equals the norm + gate applied to the plain bf16 output of the same
    call (GPU against GPU, within the bf16 bar)."""
    H, d = 4, 128
    lengths = [1500, 40]
    cu = synth.cu_from_lengths(lengths)
    q, k, v = draw_packed(lengths, H, d, seed=121)
    sl = synth.slopes(H, DEV)
    gate, gamma = draw_gate(sum(lengths), H, d, seed=122)
    o, s0 = la.prefill_varlen(q, k, v, sl, cu)
    y, s1 = la.prefill_varlen(q, k, v, sl, cu, gate=gate, gamma=gamma, eps=EPS)
    torch.cuda.synchronize()
    assert torch.equal(s0, s1)  # the epilogue does not touch the state
    y_from_o = oracle.gated_rmsnorm(o.double().cpu().numpy(), oracle_bits(gate),
                                    gamma.cpu().numpy(), EPS)
    check_close(y.float().cpu().numpy(), y_from_o, torch.bfloat16, "fused vs unfused")


def test_gated_epilogue_zero_output_rows():
    """v = 0 makes o = 0: with eps > 0 the normalised output is exactly 0."""
    H, d, T = 2, 128, 260
    q, k, v = draw_packed([T], H, d, seed=131)
    v.zero_()
    sl = synth.slopes(H, DEV)
    gate, gamma = draw_gate(T, H, d, seed=132)
    y, _ = la.prefill_varlen(q, k, v, sl, [0, T], gate=gate, gamma=gamma, eps=1e-6)
    torch.cuda.synchronize()
    assert bool((y == 0).all())


def test_gated_epilogue_layer_width_sampled_heads():
    """The layer's width (H = 64) on two 16,384-token sequences; six seeded heads checked in
    full against the oracle."""
    H, d, N = 64, 128, 16384
    cu = [0, N, 2 * N]
    q, k, v = draw_packed([N, N], H, d, seed=141)
    sl = synth.slopes(H, DEV)
    gate, gamma = draw_gate(2 * N, H, d, seed=142)
    y, _ = la.prefill_varlen(q, k, v, sl, cu, gate=gate, gamma=gamma, eps=EPS)
    torch.cuda.synchronize()
    heads = sorted(np.random.default_rng(143).choice(H, 6, replace=False).tolist())
    ref = reference(q, k, v, sl, cu, gate, gamma, EPS, heads=heads)
    check_close(y[:, heads].float().cpu().numpy(), ref, torch.bfloat16, "y")


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 128),
                                     (torch.bfloat16, 64)])
def test_standalone_gate_norm_matches_oracle(dtype, d):
    """la_gate_norm_apply (the post-kernel operator on its own) on random o."""
    T, H = 333, 8
    g = torch.Generator(device=DEV)
    g.manual_seed(151)
    o = (torch.randn((T, H, d), generator=g, device=DEV) * 0.7).to(dtype)
    gate = (torch.randn((T, H, d), generator=g, device=DEV) * 3).to(dtype)
    gamma = (1.0 + 0.5 * torch.randn((H, d), generator=g, device=DEV)).float()
    y = la.gate_norm(o, gate, gamma, eps=1e-6)
    torch.cuda.synchronize()
    ref = oracle.gated_rmsnorm(o.double().cpu().numpy(), oracle_bits(gate), gamma.cpu().numpy(),
                               1e-6)
    check_close(y.float().cpu().numpy(), ref, dtype, "y")
    # in place gives the same bits
    o2 = o.clone()
    la.gate_norm(o2, gate, gamma, eps=1e-6, out=o2)
    torch.cuda.synchronize()
    assert torch.equal(o2, y)


def test_standalone_gate_norm_equals_fused_epilogue_path():
    """prefill then la_gate_norm_apply agrees with the fused epilogue within the bf16 bar."""
    H, d = 4, 128
    lengths = [900, 300]
    cu = synth.cu_from_lengths(lengths)
    q, k, v = draw_packed(lengths, H, d, seed=161)
    sl = synth.slopes(H, DEV)
    gate, gamma = draw_gate(sum(lengths), H, d, seed=162)
    o, _ = la.prefill_varlen(q, k, v, sl, cu)
    y_sep = la.gate_norm(o, gate, gamma, eps=EPS)
    y_fused, _ = la.prefill_varlen(q, k, v, sl, cu, gate=gate, gamma=gamma, eps=EPS)
    torch.cuda.synchronize()
    check_close(y_sep.float().cpu().numpy(), y_fused.double().cpu().numpy(), torch.bfloat16, "y")


# ---------------------------------------------------------------------------------------------
# FP8 E4M3 output of the fused operator ("group norm + sigmoid gate + quantize")
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 128),
                                     (torch.bfloat16, 64)])
def test_standalone_gate_norm_fp8_matches_oracle(dtype, d):
    """la_gate_norm_apply with FP8 output on random o (ragged head count: rows past H in the
    last sweep)."""
    T, H = 333, 7
    g = torch.Generator(device=DEV)
    g.manual_seed(171)
    o = (torch.randn((T, H, d), generator=g, device=DEV) * 0.7).to(dtype)
    gate = (torch.randn((T, H, d), generator=g, device=DEV) * 3).to(dtype)
    gamma = (1.0 + 0.5 * torch.randn((H, d), generator=g, device=DEV)).float()
    codes, scales = la.gate_norm(o, gate, gamma, eps=1e-6, fp8=True)
    torch.cuda.synchronize()
    ref = oracle.gated_rmsnorm(o.double().cpu().numpy(), oracle_bits(gate), gamma.cpu().numpy(),
                               1e-6)
    check_fp8(codes.cpu().numpy(), scales.cpu().numpy(), ref, "standalone fp8", io_dtype=dtype)


def test_standalone_gate_norm_fp8_zero_blocks_and_saturated_gate():
    """All-zero o gives scale 0 and zero codes; a gate of scale 6 pushes the sigmoid into both
    tails, so blocks mix large and tiny values; and the prefill's own output quantizes within
    the bar (prefill, then the stand-alone operator with FP8 output)."""
    H, d, T = 3, 128, 260
    o = torch.zeros((T, H, d), dtype=torch.bfloat16, device=DEV)
    gate, gamma = draw_gate(T, H, d, seed=191)
    codes, scales = la.gate_norm(o, gate, gamma, eps=1e-6, fp8=True)
    torch.cuda.synchronize()
    assert bool((scales == 0).all()) and bool(((codes & 0x7F) == 0).all())
    lengths = [700, 333]
    cu = synth.cu_from_lengths(lengths)
    q, k, v = draw_packed(lengths, 8, d, seed=111, dist="silu_qk")
    sl = synth.slopes(8, DEV)
    gate, gamma = draw_gate(sum(lengths), 8, d, seed=112, scale=6.0)
    o, _ = la.prefill_varlen(q, k, v, sl, cu)
    codes, scales = la.gate_norm(o, gate, gamma, eps=0.5, fp8=True)
    torch.cuda.synchronize()
    check_fp8(codes.cpu().numpy(), scales.cpu().numpy(),
              reference(q, k, v, sl, cu, gate, gamma, 0.5), "prefill then fp8 operator")
