"""The context-parallel steps on a GPU, through the C ABI, against the fp64 oracle.

- la_prefill_state (the state of a prefill without outputs) against oracle.prefill's final state;
- la_state_fold against oracle.fold_states;
- the whole context-parallel forward with its ranks run one after another on this GPU (the
  exchange replaced by stacking the parts' states, which is what all_gather returns), against
  one sequential oracle pass: outputs of every part and the final state;
- prefill_cp itself on a one-rank NCCL group.
Bar: bf16 relL2 <= 1e-2 and maxabs <= 2e-2 * max|ref|; fp32 relL2 <= 1e-5.
"""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from long_context_attention_la_b200 import cp, la, synth
from tests.helpers import check_close, oracle_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"


def oracle_state(k, v, sl, state_in=None, heads=None):
    """fp64 [n_heads, d, d]: oracle.prefill's final state (q does not enter it)."""
    kb = oracle_bits(k)
    sin = None
    if state_in is not None:
        s = state_in.double().cpu().numpy()
        s = s.reshape(-1, *s.shape[-2:])
        sin = s if heads is None else s[heads]
    _, st = oracle.prefill(np.zeros_like(kb), kb, oracle_bits(v), sl.cpu().numpy(), heads=heads,
                           state_in=sin)
    return st


@pytest.mark.parametrize("B,N,H", [(1, 1000, 4), (1, 4096, 64), (2, 129, 8), (4, 300, 64),
                                   (1, 5, 2), (3, 128, 3)])
def test_prefill_state_matches_oracle(B, N, H):
    """Covers every work split: heads cut over many CTAs (combined in range order), heads whole
    in one CTA, both in one launch, and ragged last chunks."""
    d = 128
    _, k, v = synth.draw_qkv(B, N, H, d, dist="silu_qk", seed=201 + N, device=DEV)
    sl = synth.slopes(H, DEV)
    st = la.prefill_state(k, v, sl)
    torch.cuda.synchronize()
    heads = None if B * H <= 16 else sorted(np.random.default_rng(N).choice(B * H, 12, replace=False).tolist())
    ref = oracle_state(k, v, sl, heads=heads)
    got = st.reshape(B * H, d, d).cpu().numpy()
    check_close(got if heads is None else got[heads], ref, torch.bfloat16, "state")


@pytest.mark.parametrize("B,N,H", [(2, 700, 4), (1, 4096, 64)])
def test_prefill_state_from_initial_state_and_in_place(B, N, H):
    d = 128
    _, k, v = synth.draw_qkv(B, N, H, d, seed=211, device=DEV)
    sl = synth.slopes(H, DEV)
    s0 = synth.draw_states(B, H, d, seed=212, scale=0.5, device=DEV)
    st = la.prefill_state(k, v, sl, state_in=s0)
    torch.cuda.synchronize()
    heads = None if B * H <= 16 else [0, 7, 31, 63]
    ref = oracle_state(k, v, sl, state_in=s0, heads=heads)
    got = st.reshape(B * H, d, d).cpu().numpy()
    check_close(got if heads is None else got[heads], ref, torch.bfloat16, "state")
    s1 = s0.clone()
    la.prefill_state(k, v, sl, state_in=s1, state_out=s1)  # in place
    torch.cuda.synchronize()
    assert torch.equal(s1, st)


def test_prefill_state_equals_prefill_state_out():
    """The state-only pass and the full prefill agree (GPU against GPU, within the bf16 bar)."""
    B, N, H, d = 2, 2000, 8, 128
    q, k, v = synth.draw_qkv(B, N, H, d, seed=221, device=DEV)
    sl = synth.slopes(H, DEV)
    _, st_full = la.prefill(q, k, v, sl)
    st = la.prefill_state(k, v, sl)
    torch.cuda.synchronize()
    check_close(st.cpu().numpy(), st_full.double().cpu().numpy(), torch.bfloat16, "state")


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.float32, 128), (torch.bfloat16, 64)])
def test_prefill_state_recurrent_path(dtype, d):
    """fp32 and d = 64 take the token recurrence with no q and no read-out."""
    B, N, H = 2, 300, 3
    _, k, v = synth.draw_qkv(B, N, H, d, seed=231, device=DEV)
    k, v = k.to(dtype), v.to(dtype)
    sl = synth.slopes(H, DEV)
    s0 = synth.draw_states(B, H, d, seed=232, scale=0.5, device=DEV)
    st = la.prefill_state(k, v, sl, state_in=s0)
    torch.cuda.synchronize()
    check_close(st.reshape(B * H, d, d).cpu().numpy(), oracle_state(k, v, sl, state_in=s0), dtype,
                "state")


@pytest.mark.parametrize("n,d,with_in", [(0, 128, True), (0, 128, False), (1, 128, True),
                                         (3, 128, False), (5, 64, True)])
def test_state_fold_matches_oracle(n, d, with_in):
    B, H = 2, 64
    g = torch.Generator(device=DEV)
    g.manual_seed(240 + n)
    parts = torch.randn((n, B, H, d, d), generator=g, device=DEV)
    lengths = [37, 4096, 1, 0, 300][:n]
    sl = synth.slopes(H, DEV)
    s0 = torch.randn((B, H, d, d), generator=g, device=DEV) if with_in else None
    S = la.state_fold(parts, lengths, sl, state_in=s0)
    torch.cuda.synchronize()
    ref = oracle.fold_states(parts.cpu().numpy(), lengths, sl.cpu().numpy(),
                             None if s0 is None else s0.cpu().numpy())
    check_close(S.cpu().numpy(), ref, torch.float32, "fold")
    if with_in:
        s1 = s0.clone()
        la.state_fold(parts, lengths, sl, state_in=s1, out=s1)  # in place
        torch.cuda.synchronize()
        assert torch.equal(s1, S)


def _cp_emulated(q, k, v, sl, cuts, state_in=None):
    """The context-parallel forward with its ranks one after another: outputs of every part
    (concatenated) and every rank's outgoing state."""
    parts = [(a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    ops = cp.DeviceOps()
    hs = torch.stack([ops.local_state(k[:, a:b].contiguous(), v[:, a:b].contiguous(), sl)
                      for a, b in parts])  # what all_gather returns, in rank order
    lengths = np.diff(cuts).tolist()
    outs, states = [], []
    for r, (a, b) in enumerate(parts):
        s_r = ops.fold(hs[:r].contiguous(), lengths[:r], sl, state_in)
        o, st = ops.prefill_from(q[:, a:b].contiguous(), k[:, a:b].contiguous(),
                                 v[:, a:b].contiguous(), sl, s_r)
        outs.append(o)
        states.append(st)
    return torch.cat(outs, dim=1), states


@pytest.mark.parametrize("cuts", [[0, 1500, 3000], [0, 700, 700, 2100, 2177, 3000],
                                  [0, 128, 256, 384, 3000]])
def test_context_parallel_emulated_matches_sequential_oracle(cuts):
    B, N, H, d = 1, cuts[-1], 8, 128
    q, k, v = synth.draw_qkv(B, N, H, d, dist="silu_qk", seed=251, device=DEV)
    sl = synth.slopes(H, DEV)
    s0 = synth.draw_states(B, H, d, seed=252, scale=0.3, device=DEV)
    o, states = _cp_emulated(q, k, v, sl, cuts, state_in=s0)
    torch.cuda.synchronize()
    o_ref, st_ref = oracle.prefill(oracle_bits(q), oracle_bits(k), oracle_bits(v),
                                   sl.cpu().numpy(), state_in=s0.double().cpu().numpy()[0])
    o_ref = o_ref.reshape(B, H, N, d).transpose(0, 2, 1, 3)
    check_close(o.float().cpu().numpy(), o_ref, torch.bfloat16, "o")
    check_close(states[-1].cpu().numpy(), st_ref.reshape(B, H, d, d), torch.bfloat16, "state")


def test_context_parallel_layer_width_sampled_heads():
    """H = 64 over 4 parts of a 16,384-token sequence; six heads checked in full."""
    B, N, H, d = 1, 16384, 64, 128
    cuts = [0, 4096, 8192, 12288, 16384]
    q, k, v = synth.draw_qkv(B, N, H, d, dist="silu_qk", seed=261, device=DEV)
    sl = synth.slopes(H, DEV)
    o, states = _cp_emulated(q, k, v, sl, cuts)
    torch.cuda.synchronize()
    heads = sorted(np.random.default_rng(262).choice(H, 6, replace=False).tolist())
    o_ref, st_ref = oracle.prefill(oracle_bits(q), oracle_bits(k), oracle_bits(v),
                                   sl.cpu().numpy(), heads=heads)
    o_ref = o_ref.transpose(1, 0, 2)  # [N, heads, d]
    check_close(o[0][:, heads].float().cpu().numpy(), o_ref, torch.bfloat16, "o")
    check_close(states[-1][0, heads].cpu().numpy(), st_ref, torch.bfloat16, "state")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_prefill_cp_one_rank_nccl_group():
    """prefill_cp through a real NCCL process group of one rank: the single part is the whole
    sequence, so the result equals a plain prefill from the initial state."""
    B, N, H, d = 2, 1000, 4, 128
    q, k, v = synth.draw_qkv(B, N, H, d, seed=271, device=DEV)
    sl = synth.slopes(H, DEV)
    s0 = synth.draw_states(B, H, d, seed=272, scale=0.3, device=DEV)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True,
                          timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        o, st = cp.prefill_cp(q, k, v, sl, state_in=s0)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    cu = [0, N, 2 * N]
    o_ref, st_ref = la.prefill_varlen(q.view(B * N, H, d), k.view(B * N, H, d),
                                      v.view(B * N, H, d), sl, cu, state_in=s0)
    torch.cuda.synchronize()
    assert torch.equal(o.view(B * N, H, d), o_ref)
    assert torch.equal(st, st_ref)
