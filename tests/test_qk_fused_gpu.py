"""la_prefill_varlen_qk (QK RMSNorm + partial RoPE applied inside the prefill kernel) on a GPU,
through the C ABI.

Two bars:
- exact: the fused call equals la_qk_norm_rope followed by la_prefill_varlen with the same
  segments, o and the final states, value for value (torch.equal: +0 and -0 agree);
- oracle: against the fp64 chain oracle.qk_norm_rope -> oracle.prefill on the same input bits,
  the bf16 bar of test_parity_gpu (relL2 <= 1e-2, maxabs <= 2e-2 * max|ref|).
q and k must come back unchanged (the transform happens in shared memory only).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_attention_la_b200 import la, synth
from tests.helpers import check_close, oracle_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"
THETA, EPS = 6.0e6, 1e-6

# ragged lengths around the 128-token tile, an empty sequence, multi-tile sequences
EDGE_LENGTHS = [1, 127, 128, 129, 0, 300, 1000, 2049, 5]


def draw(lengths, H, seed, prefix=None):
    """Packed raw q, k, v [T, H, 128] bf16, norm weights, and each token's position in its
    sequence (plus prefix[s] for a sequence that continues a cached prefix)."""
    d = 128
    T = sum(lengths)
    q, k, v = synth.draw_qkv(1, max(T, 1), H, d, dist="scaled_normal", seed=seed,
                             dtype=torch.bfloat16, device=DEV)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed + 1)
    gq = (1.0 + 0.3 * torch.randn(d, generator=g, device=DEV)).float()
    gk = (1.0 + 0.3 * torch.randn(d, generator=g, device=DEV)).float()
    prefix = prefix or [0] * len(lengths)
    pos = torch.cat([torch.arange(n, dtype=torch.int64) + p for n, p in zip(lengths, prefix)])
    return (q[0, :T].contiguous(), k[0, :T].contiguous(), v[0, :T].contiguous(), gq, gk,
            pos.to(DEV))


def two_step(q, k, v, sl, cu, gq, gk, pos, r, sin, segments):
    qh, kh = la.qk_norm_rope(q, k, gq, gk, pos, rotary_dim=r, theta=THETA, eps=EPS)
    return la.prefill_varlen(qh, kh, v, sl, cu, state_in=sin, segments=segments, chunk=128)


def oracle_chain(q, k, v, sl, cu, gq, gk, pos, r, sin, heads=None, t_sel=None):
    """fp64: qk_norm_rope, then the recurrence per sequence (q_hat, k_hat passed as float32, v
    as its exact float32 values)."""
    res = []
    H, d = q.shape[1], q.shape[2]
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        st_in = None if sin is None else sin[s].double().cpu().numpy()
        if b == a:
            res.append((np.zeros((H, 0, d)), np.zeros((H, d, d)) if st_in is None else st_in))
            continue
        p = pos[a:b].cpu().numpy()
        qh = oracle.qk_norm_rope(oracle_bits(q[a:b]), gq.cpu().numpy(), p, r, THETA, EPS)
        kh = oracle.qk_norm_rope(oracle_bits(k[a:b]), gk.cpu().numpy(), p, r, THETA, EPS)
        o, st = oracle.prefill(qh.astype(np.float32)[None], kh.astype(np.float32)[None],
                               oracle_bits(v[a:b].float().unsqueeze(0)), sl.cpu().numpy(),
                               heads=heads, t_sel=t_sel, state_in=st_in)
        res.append((o, st))
    return res


@pytest.mark.parametrize("r", [64, 16, 128])
@pytest.mark.parametrize("segments", [0, 1, 3])
@pytest.mark.parametrize("with_state", [False, True])
def test_fused_equals_two_step(r, segments, with_state):
    H = 4
    cu = synth.cu_from_lengths(EDGE_LENGTHS)
    prefix = [0, 0, 0, 0, 0, 262000, 0, 17, 0]  # one sequence continues a 262,000-token prefix
    q, k, v, gq, gk, pos = draw(EDGE_LENGTHS, H, seed=301, prefix=prefix)
    sl = synth.slopes(H, DEV)
    sin = None
    if with_state:
        g = torch.Generator(device=DEV)
        g.manual_seed(302)
        sin = torch.randn((len(EDGE_LENGTHS), H, 128, 128), generator=g, device=DEV) * 0.5
    q0, k0 = q.clone(), k.clone()
    out, st = la.prefill_varlen_qk(q, k, v, sl, cu, gq, gk, pos, rotary_dim=r, theta=THETA,
                                   eps=EPS, state_in=sin, segments=segments)
    out2, st2 = two_step(q, k, v, sl, cu, gq, gk, pos, r, sin, segments)
    torch.cuda.synchronize()
    assert torch.equal(q, q0) and torch.equal(k, k0), "q or k was modified"
    assert torch.equal(out, out2), (out.float() - out2.float()).abs().max().item()
    assert torch.equal(st, st2), (st - st2).abs().max().item()


@pytest.mark.parametrize("segments", [0, 3])
def test_fused_matches_oracle(segments):
    H = 4
    cu = synth.cu_from_lengths(EDGE_LENGTHS)
    q, k, v, gq, gk, pos = draw(EDGE_LENGTHS, H, seed=311, prefix=[5, 0, 0, 0, 0, 0, 0, 99991, 0])
    sl = synth.slopes(H, DEV)
    out, st = la.prefill_varlen_qk(q, k, v, sl, cu, gq, gk, pos, rotary_dim=64, theta=THETA,
                                   eps=EPS, segments=segments)
    torch.cuda.synchronize()
    ref = oracle_chain(q, k, v, sl, cu, gq, gk, pos, 64, None)
    o_gpu = np.concatenate([out[cu[s]:cu[s + 1]].permute(1, 0, 2).float().cpu().numpy()
                            for s in range(len(cu) - 1)], axis=1)
    check_close(o_gpu, np.concatenate([r_[0] for r_ in ref], axis=1), torch.bfloat16, "o")
    check_close(st.cpu().numpy(), np.stack([r_[1] for r_ in ref]), torch.bfloat16, "state")


def test_fused_full_size_equals_two_step_and_samples_match_oracle():
    """The bench's workload (2 sequences of 32,768 tokens, 64 heads, packed) in the launch
    configuration the bench times: exact against the two-step path, and sampled tokens of two
    heads against the oracle chain."""
    H, N = 64, 32768
    lengths = [N, N]
    cu = synth.cu_from_lengths(lengths)
    q, k, v, gq, gk, pos = draw(lengths, H, seed=321)
    sl = synth.slopes(H, DEV)
    out, st = la.prefill_varlen_qk(q, k, v, sl, cu, gq, gk, pos)
    out2, st2 = two_step(q, k, v, sl, cu, gq, gk, pos, 64, None, 0)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
    assert torch.equal(st, st2)
    # sampled outputs of heads 0 and 63 of the second sequence against the fp64 chain
    heads = [0, 63]
    t_sel = np.array([0, 1, 127, 128, 4095, 20000, N - 1], dtype=np.int64)
    a, b = cu[1], cu[2]
    p = pos[a:b].cpu().numpy()
    for h in heads:
        gqn, gkn = gq.cpu().numpy(), gk.cpu().numpy()
        qh = oracle.qk_norm_rope(oracle_bits(q[a:b, h:h + 1]), gqn, p, 64, THETA, EPS)
        kh = oracle.qk_norm_rope(oracle_bits(k[a:b, h:h + 1]), gkn, p, 64, THETA, EPS)
        o, s_ = oracle.prefill(qh.astype(np.float32)[None], kh.astype(np.float32)[None],
                               oracle_bits(v[a:b, h:h + 1].float().unsqueeze(0)),
                               sl[h:h + 1].cpu().numpy(), t_sel=t_sel)
        got = out[a + torch.as_tensor(t_sel, device=DEV), h].float().cpu().numpy()
        check_close(got, o[0], torch.bfloat16, f"o head {h}")
        check_close(st[1, h].cpu().numpy(), s_[0], torch.bfloat16, f"state head {h}")
