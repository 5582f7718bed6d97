"""Parity of la_prefill_varlen (packed variable-length sequences, optional initial state) against
the fp64 oracle, on a GPU, through the C ABI.

Each sequence s of the packed [T, H, d] tensors is an independent recurrence over its tokens
[cu[s], cu[s+1]) that starts from state_in[s] (zero when absent); the oracle runs it sequence by
sequence on the same bits.  Bar as in test_parity_gpu: bf16 relL2 <= 1e-2 and maxabs <=
2e-2 * max|ref| for o and the final states; fp32 relL2 <= 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_attention_la_b200 import la, synth
from tests.helpers import check_close, oracle_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"

# ragged lengths around the chunk size (128), an empty sequence, and some multi-chunk ones
EDGE_LENGTHS = [1, 127, 128, 129, 0, 300, 1000, 2049, 5]


def draw_packed(lengths, H, d, seed, dtype=torch.bfloat16, dist="scaled_normal"):
    T = sum(lengths)
    q, k, v = synth.draw_qkv(1, max(T, 1), H, d, dist=dist, seed=seed, dtype=dtype, device=DEV)
    return q[0, :T].contiguous(), k[0, :T].contiguous(), v[0, :T].contiguous()


def draw_states(n, H, d, seed, scale=0.5):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn((n, H, d, d), generator=g, device=DEV, dtype=torch.float32) * scale)


def oracle_varlen(q, k, v, slopes, cu, state_in=None):
    """Per-sequence oracle: list of (o [len, H, d] as [H, len, d], state [H, d, d]) in fp64."""
    res = []
    H, d = q.shape[1], q.shape[2]
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        sin = None if state_in is None else state_in[s].double().cpu().numpy()
        if b == a:
            st = np.zeros((H, d, d)) if sin is None else sin
            res.append((np.zeros((H, 0, d)), st))
            continue
        o, st = oracle.prefill(oracle_bits(q[a:b].unsqueeze(0)), oracle_bits(k[a:b].unsqueeze(0)),
                               oracle_bits(v[a:b].unsqueeze(0)), slopes.cpu().numpy(),
                               state_in=sin)
        res.append((o, st))
    return res


def gpu_seq(out, cu, s):
    a, b = cu[s], cu[s + 1]
    return out[a:b].permute(1, 0, 2).float().cpu().numpy()  # [H, len, d]


def check_all(out, st, ref, cu, dtype):
    o_gpu = np.concatenate([gpu_seq(out, cu, s) for s in range(len(cu) - 1)], axis=1)
    o_ref = np.concatenate([r[0] for r in ref], axis=1)
    check_close(o_gpu, o_ref, dtype, "o")
    check_close(st.cpu().numpy(), np.stack([r[1] for r in ref]), dtype, "state")


@pytest.mark.parametrize("chunk", [64, 128, 256])
@pytest.mark.parametrize("segments", [0, 1, 3])
@pytest.mark.parametrize("with_state", [False, True])
def test_varlen_tensor_edge_lengths(segments, with_state, chunk):
    H, d = 4, 128
    cu = synth.cu_from_lengths(EDGE_LENGTHS)
    q, k, v = draw_packed(EDGE_LENGTHS, H, d, seed=21)
    sl = synth.slopes(H, DEV)
    sin = draw_states(len(EDGE_LENGTHS), H, d, seed=22) if with_state else None
    out, st = la.prefill_varlen(q, k, v, sl, cu, state_in=sin, segments=segments, chunk=chunk)
    torch.cuda.synchronize()
    ref = oracle_varlen(q, k, v, sl, cu, sin)
    check_all(out, st, ref, cu, torch.bfloat16)
    # the empty sequence passes its initial state through exactly
    e = EDGE_LENGTHS.index(0)
    want = sin[e] if with_state else torch.zeros_like(st[e])
    assert torch.equal(st[e], want)


@pytest.mark.parametrize("d,dtype", [(64, torch.float32), (128, torch.float32),
                                     (64, torch.bfloat16)])
def test_varlen_recurrent(d, dtype):
    H = 3
    lengths = [5, 0, 130, 1, 64]
    cu = synth.cu_from_lengths(lengths)
    q, k, v = draw_packed(lengths, H, d, seed=31, dtype=dtype)
    sl = synth.slopes(H, DEV)
    sin = draw_states(len(lengths), H, d, seed=32)
    out, st = la.prefill_varlen(q, k, v, sl, cu, state_in=sin)
    torch.cuda.synchronize()
    check_all(out, st, oracle_varlen(q, k, v, sl, cu, sin), cu, dtype)


@pytest.mark.parametrize("segments", [1, 2, 3])
def test_varlen_equal_lengths_match_fixed_batch(segments):
    """B sequences of N tokens packed back to back are the [B, N, H, d] problem: with the same
    explicit segment count both forms plan the same segments, so the bits agree; the automatic
    plans (balanced ranges for the fixed form) agree within the parity bar."""
    B, N, H, d = 3, 1000, 4, 128
    q, k, v = synth.draw_qkv(B, N, H, d, seed=41, device=DEV)
    sl = synth.slopes(H, DEV)
    o_fixed, s_fixed = la.prefill(q, k, v, sl, segments=segments)
    cu = [0, N, 2 * N, 3 * N]
    o_var, s_var = la.prefill_varlen(q.view(B * N, H, d), k.view(B * N, H, d),
                                     v.view(B * N, H, d), sl, cu, segments=segments)
    o_auto, s_auto = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    assert torch.equal(o_var.view(B, N, H, d), o_fixed)
    assert torch.equal(s_var, s_fixed)
    check_close(o_auto.float().cpu().numpy(), o_var.view(B, N, H, d).float().cpu().numpy(),
                torch.bfloat16, "o automatic plan")
    check_close(s_auto.cpu().numpy(), s_var.cpu().numpy(), torch.bfloat16, "state automatic plan")


@pytest.mark.parametrize("split", [128, 700, 1])
def test_state_in_continues_a_prefill(split):
    """prefill(first part) -> state; prefill_varlen(rest, state_in=state) gives the outputs and
    final state of one prefill over the whole sequence (P-decode's prefix form)."""
    N, H, d = 1600, 8, 128
    q, k, v = synth.draw_qkv(1, N, H, d, seed=51, device=DEV)
    sl = synth.slopes(H, DEV)
    o_all, s_all = la.prefill(q, k, v, sl)
    _, s1 = la.prefill(q[:, :split].contiguous(), k[:, :split].contiguous(),
                       v[:, :split].contiguous(), sl)
    rest = N - split
    o2, s2 = la.prefill_varlen(q[0, split:].contiguous(), k[0, split:].contiguous(),
                               v[0, split:].contiguous(), sl, [0, rest], state_in=s1)
    torch.cuda.synchronize()
    # against the oracle over the whole sequence
    o_ref, s_ref = oracle.prefill(oracle_bits(q), oracle_bits(k), oracle_bits(v),
                                  sl.cpu().numpy(), t_sel=np.arange(split, N))
    check_close(o2.permute(1, 0, 2).float().cpu().numpy(), o_ref[:, :, :], torch.bfloat16, "o")
    check_close(s2[0].cpu().numpy(), s_ref, torch.bfloat16, "state")
    # and against the one-shot GPU prefill
    check_close(o2.float().cpu().numpy(), o_all[0, split:].float().cpu().numpy(), torch.bfloat16,
                "o vs one-shot")


def test_state_in_in_place_equals_out_of_place():
    lengths = [700, 300, 1500]
    H, d = 4, 128
    cu = synth.cu_from_lengths(lengths)
    q, k, v = draw_packed(lengths, H, d, seed=61)
    sl = synth.slopes(H, DEV)
    sin = draw_states(3, H, d, seed=62)
    o1, s1 = la.prefill_varlen(q, k, v, sl, cu, state_in=sin, segments=2)
    st = sin.clone()
    o2, s2 = la.prefill_varlen(q, k, v, sl, cu, state_in=st, state_out=st, segments=2)
    torch.cuda.synchronize()
    assert s2.data_ptr() == st.data_ptr()
    assert torch.equal(o1, o2)
    assert torch.equal(s1, st)


def test_state_in_through_the_segment_scan_near_unit_decay():
    """With lambda within ~1e-6 of 1 the initial state reaches every token: a long sequence cut
    into 7 segments must still carry state_in through the decayed prefix scan."""
    N, H, d = 7 * 512 + 37, 2, 128
    q, k, v = synth.draw_qkv(1, N, H, d, seed=71, device=DEV)
    sl = synth.slopes(H, DEV) * 1e-5
    sin = draw_states(1, H, d, seed=72, scale=1.0)
    out, st = la.prefill_varlen(q[0], k[0], v[0], sl, [0, N], state_in=sin, segments=7)
    torch.cuda.synchronize()
    ref = oracle_varlen(q[0], k[0], v[0], sl, [0, N], sin)
    check_all(out, st, ref, [0, N], torch.bfloat16)


def test_varlen_fragmented_mix_sampled():
    """A fragmented packed batch at the layer's width (H = 64): 48 sequences, most of them short,
    65,536 tokens in all; a seeded sample of sequences is checked in full (all heads)."""
    H, d, T, n = 64, 128, 65536, 48
    lengths = synth.draw_seqlens(T, n, seed=81)
    cu = synth.cu_from_lengths(lengths)
    q, k, v = draw_packed(lengths, H, d, seed=82, dist="silu_qk")
    sl = synth.slopes(H, DEV)
    sin = draw_states(n, H, d, seed=83, scale=0.1)
    out, st = la.prefill_varlen(q, k, v, sl, cu, state_in=sin)
    torch.cuda.synchronize()
    rng = np.random.default_rng(84)
    order = np.argsort(lengths)
    pick = sorted(set([int(order[0]), int(order[-1])] + rng.choice(n, 4, replace=False).tolist()))
    for s in pick:
        a, b = cu[s], cu[s + 1]
        sub = oracle_varlen(q[a:b], k[a:b], v[a:b], sl, [0, b - a], sin[s:s + 1])
        check_all(out[a:b], st[s:s + 1], sub, [0, b - a], torch.bfloat16)


@pytest.mark.parametrize("path", [la.LA_PATH_AUTO, la.LA_PATH_RECURRENT])
def test_invalid_cu_seqlens_is_reported_by_the_device(path):
    """cu_seqlens lives on the device, so a decreasing run is caught by the planning kernel:
    the call is enqueued, the workspace status reads LA_ERR_SHAPE, and no output is written."""
    H, d, T = 2, 128, 300
    q, k, v = draw_packed([T], H, d, seed=91)
    sl = synth.slopes(H, DEV)
    cu = torch.tensor([0, 350, T], dtype=torch.int64, device=DEV)
    out = torch.full_like(q, 7.0)
    st = torch.full((2, H, d, d), 7.0, device=DEV)
    desc = la.la_varlen_desc(T, 2, H, d, la.LA_BF16, 0, 0, path)
    ws = torch.empty(la.la_prefill_varlen_workspace_bytes(desc), dtype=torch.uint8, device=DEV)
    s = torch.cuda.current_stream().cuda_stream
    rc = la.la_prefill_varlen(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                              cu.data_ptr(), 0, out.data_ptr(), st.data_ptr(), ws.data_ptr(),
                              ws.numel(), s)
    assert rc == la.LA_OK
    assert la.la_workspace_status(ws.data_ptr(), s) == la.LA_ERR_SHAPE
    assert bool((out == 7.0).all()) and bool((st == 7.0).all())


@pytest.mark.parametrize("path", [la.LA_PATH_AUTO, la.LA_PATH_RECURRENT])
def test_all_sequences_empty(path):
    """T = 0: nothing to read or write but the states, which pass through (or start at zero)."""
    H, d, n = 2, 128, 3
    buf = torch.zeros((1, H, d), dtype=torch.bfloat16, device=DEV)  # addresses only; unused
    sl = synth.slopes(H, DEV)
    cu = torch.zeros(n + 1, dtype=torch.int64, device=DEV)
    desc = la.la_varlen_desc(0, n, H, d, la.LA_BF16, 0, 0, path)
    ws = torch.empty(la.la_prefill_varlen_workspace_bytes(desc), dtype=torch.uint8, device=DEV)
    s = torch.cuda.current_stream().cuda_stream
    sin = draw_states(n, H, d, seed=92)
    for state_in, want in [(sin, sin), (None, torch.zeros_like(sin))]:
        st = torch.full_like(sin, 3.0)
        rc = la.la_prefill_varlen(desc, buf.data_ptr(), buf.data_ptr(), buf.data_ptr(),
                                  sl.data_ptr(), cu.data_ptr(),
                                  0 if state_in is None else state_in.data_ptr(), buf.data_ptr(),
                                  st.data_ptr(), ws.data_ptr(), ws.numel(), s)
        assert rc == la.LA_OK
        assert la.la_workspace_status(ws.data_ptr(), s) == la.LA_OK
        assert torch.equal(st, want)
