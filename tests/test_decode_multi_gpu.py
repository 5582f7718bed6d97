"""la_decode_multi (n tokens per sequence in one pass over the state, optional fused norm + gate)
against the fp64 oracle's decode step applied n times, on a GPU.

Bar: bf16 relL2 <= 1e-2 and maxabs <= 2e-2 * max|ref| on o and the state; fp32 relL2 <= 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_attention_la_b200 import la, synth
from tests.helpers import check_close, oracle_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"


def draw(B, n, H, d, seed, dtype):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    x = [(torch.randn((B, n, H, d), generator=g, device=DEV) / d ** 0.5).to(dtype)
         for _ in range(3)]
    state = torch.randn((B, H, d, d), generator=g, device=DEV) * 0.05
    return x[0], x[1], x[2], state


def oracle_steps(q, k, v, sl, state):
    """o [B, n, H, d] and the final state, fp64, by n oracle decode steps."""
    S = state.double().cpu().numpy().copy()
    outs = []
    for j in range(q.shape[1]):
        outs.append(oracle.decode(oracle_bits(q[:, j].contiguous()), oracle_bits(k[:, j].contiguous()),
                                  oracle_bits(v[:, j].contiguous()), sl.cpu().numpy(), S))
    return np.stack(outs, axis=1), S


@pytest.mark.parametrize("n", [1, 3, 8])
@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.bfloat16),
                                     (128, torch.float32), (64, torch.float32)])
def test_decode_multi_matches_oracle(n, d, dtype):
    B, H = 3, 4
    q, k, v, state = draw(B, n, H, d, seed=301 + n, dtype=dtype)
    sl = synth.slopes(H, DEV)
    st = state.clone()
    o = la.decode_multi(q, k, v, sl, st)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_steps(q, k, v, sl, state)
    check_close(o.float().cpu().numpy(), o_ref, dtype, "o")
    check_close(st.cpu().numpy(), s_ref, dtype, "state")


def test_one_token_is_the_decode_step_bit_for_bit():
    B, H, d = 5, 8, 128
    q, k, v, state = draw(B, 1, H, d, seed=311, dtype=torch.bfloat16)
    sl = synth.slopes(H, DEV)
    s1, s2 = state.clone(), state.clone()
    o1 = la.decode_multi(q, k, v, sl, s1)
    o2 = la.decode_step(q[:, 0].contiguous(), k[:, 0].contiguous(), v[:, 0].contiguous(), sl, s2)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, 0], o2) and torch.equal(s1, s2)


def test_decode_multi_continues_a_prefill():
    """prefill(N) then decode_multi(n) equals the last n outputs of one prefill over N + n."""
    N, n, H, d = 700, 6, 4, 128
    q, k, v = synth.draw_qkv(1, N + n, H, d, seed=321, device=DEV)
    sl = synth.slopes(H, DEV)
    o_all, s_all = la.prefill(q, k, v, sl)
    _, st = la.prefill(q[:, :N].contiguous(), k[:, :N].contiguous(), v[:, :N].contiguous(), sl)
    o = la.decode_multi(q[:, N:].contiguous(), k[:, N:].contiguous(), v[:, N:].contiguous(), sl, st)
    torch.cuda.synchronize()
    check_close(o.float().cpu().numpy(), o_all[:, N:].float().cpu().numpy(), torch.bfloat16, "o")
    check_close(st.cpu().numpy(), s_all.cpu().numpy(), torch.bfloat16, "state")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_multi_gated(dtype):
    B, n, H, d = 4, 4, 8, 128
    q, k, v, state = draw(B, n, H, d, seed=331, dtype=dtype)
    sl = synth.slopes(H, DEV)
    g = torch.Generator(device=DEV)
    g.manual_seed(332)
    gate = (torch.randn((B, n, H, d), generator=g, device=DEV) * 2).to(dtype)
    gamma = (1.0 + 0.5 * torch.randn((H, d), generator=g, device=DEV)).float()
    st = state.clone()
    y = la.decode_multi(q, k, v, sl, st, gate=gate, gamma=gamma, eps=1e-6)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_steps(q, k, v, sl, state)
    y_ref = oracle.gated_rmsnorm(o_ref, oracle_bits(gate), gamma.cpu().numpy(), 1e-6)
    check_close(y.float().cpu().numpy(), y_ref, dtype, "y")
    check_close(st.cpu().numpy(), s_ref, dtype, "state")


def test_decode_multi_serving_width_sampled():
    """256 sequences x 64 heads x d = 128 (a 1 GiB state), 4 tokens; 16 seeded sequences checked."""
    B, n, H, d = 256, 4, 64, 128
    q, k, v, state = draw(B, n, H, d, seed=341, dtype=torch.bfloat16)
    sl = synth.slopes(H, DEV)
    rng = np.random.default_rng(342)
    pick = torch.as_tensor(np.sort(rng.choice(B, 16, replace=False)), device=DEV)
    before = state[pick].clone()
    o = la.decode_multi(q, k, v, sl, state)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_steps(q[pick], k[pick], v[pick], sl, before)
    check_close(o[pick].float().cpu().numpy(), o_ref, torch.bfloat16, "o")
    check_close(state[pick].cpu().numpy(), s_ref, torch.bfloat16, "state")
