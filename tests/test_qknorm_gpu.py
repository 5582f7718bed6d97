"""la_qk_norm_rope (QK RMSNorm + partial rotate-half RoPE) against the fp64 oracle on a GPU.

Bar: bf16 relL2 <= 1e-2 and maxabs <= 2e-2 * max|ref| on q_hat and k_hat.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_attention_la_b200 import la
from tests.helpers import check_close, oracle_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"


def draw(T, H, d, seed, scale=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = (torch.randn((T, H, d), generator=g, device=DEV) * scale).to(torch.bfloat16)
    k = (torch.randn((T, H, d), generator=g, device=DEV) * scale).to(torch.bfloat16)
    gq = (1.0 + 0.3 * torch.randn(d, generator=g, device=DEV)).float()
    gk = (1.0 + 0.3 * torch.randn(d, generator=g, device=DEV)).float()
    return q, k, gq, gk


def ref(x, gamma, pos, r, theta, eps):
    return oracle.qk_norm_rope(oracle_bits(x.contiguous()), gamma.cpu().numpy(),
                               pos.cpu().numpy(), r, theta, eps)


@pytest.mark.parametrize("d,r", [(128, 64), (128, 128), (128, 16), (64, 32), (64, 64)])
def test_qk_norm_rope_matches_oracle(d, r):
    T, H = 300, 4
    q, k, gq, gk = draw(T, H, d, seed=201)
    # positions of two packed sequences, the second continuing a 262,000-token prefix
    pos = torch.cat([torch.arange(100), 262000 + torch.arange(200)]).to(DEV)
    qh, kh = la.qk_norm_rope(q, k, gq, gk, pos, rotary_dim=r, theta=6.0e6, eps=1e-6)
    torch.cuda.synchronize()
    check_close(qh.float().cpu().numpy(), ref(q, gq, pos, r, 6.0e6, 1e-6), torch.bfloat16, "q")
    check_close(kh.float().cpu().numpy(), ref(k, gk, pos, r, 6.0e6, 1e-6), torch.bfloat16, "k")


def test_qk_norm_rope_views_into_a_fused_projection_and_in_place():
    """q and k as strided views of one [T, 4*H*d] projection output (q, k, v, gate), and the
    in-place form on contiguous copies."""
    T, H, d = 257, 8, 128
    g = torch.Generator(device=DEV)
    g.manual_seed(211)
    qkvg = torch.randn((T, 4 * H * d), generator=g, device=DEV).to(torch.bfloat16)
    q = qkvg[:, :H * d].view(T, H, d)
    k = qkvg[:, H * d:2 * H * d].view(T, H, d)
    gq = torch.ones(d, device=DEV)
    gk = torch.full((d,), 0.5, device=DEV)
    pos = torch.arange(T, device=DEV) * 997
    qh, kh = la.qk_norm_rope(q, k, gq, gk, pos, theta=1.0e4, eps=1e-5)
    torch.cuda.synchronize()
    check_close(qh.float().cpu().numpy(), ref(q, gq, pos, 64, 1.0e4, 1e-5), torch.bfloat16, "q")
    check_close(kh.float().cpu().numpy(), ref(k, gk, pos, 64, 1.0e4, 1e-5), torch.bfloat16, "k")
    qc, kc = q.contiguous(), k.contiguous()
    la.qk_norm_rope(qc, kc, gq, gk, pos, theta=1.0e4, eps=1e-5, q_out=qc, k_out=kc)
    torch.cuda.synchronize()
    assert torch.equal(qc, qh) and torch.equal(kc, kh)


def test_qk_norm_rope_position_zero_is_plain_rmsnorm():
    T, H, d = 64, 2, 128
    q, k, gq, gk = draw(T, H, d, seed=221, scale=3.0)
    pos = torch.zeros(T, dtype=torch.int64, device=DEV)
    qh, _ = la.qk_norm_rope(q, k, gq, gk, pos)
    torch.cuda.synchronize()
    x = q.double().cpu().numpy()
    plain = gq.double().cpu().numpy() * x / np.sqrt(np.mean(x * x, -1, keepdims=True) + 1e-6)
    check_close(qh.float().cpu().numpy(), plain, torch.bfloat16, "q")


def test_qk_norm_rope_layer_width_sampled():
    """65,536 tokens at the layer's width (H = 64); 512 seeded (token, head) rows checked."""
    T, H, d = 65536, 64, 128
    q, k, gq, gk = draw(T, H, d, seed=231)
    pos = torch.arange(T, device=DEV) % 40000 + 1000
    qh, kh = la.qk_norm_rope(q, k, gq, gk, pos)
    torch.cuda.synchronize()
    rng = np.random.default_rng(232)
    toks = torch.as_tensor(np.sort(rng.choice(T, 512, replace=False)), device=DEV)
    check_close(qh[toks].float().cpu().numpy(), ref(q[toks], gq, pos[toks], 64, 6.0e6, 1e-6),
                torch.bfloat16, "q")
    check_close(kh[toks].float().cpu().numpy(), ref(k[toks], gk, pos[toks], 64, 6.0e6, 1e-6),
                torch.bfloat16, "k")
