"""Parity of the CUDA path (through the C ABI) against the fp64 oracle, on a GPU.

Bar: bf16 I/O relL2 <= 1e-2 and maxabs <= 2e-2 * max|ref| for o and the final state; fp32 I/O
relL2 <= 1e-5.  Inputs are seeded synthetic draws (long_context_attention_la_b200.synth); the
oracle receives the exact bits the GPU read.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_attention_la_b200 import la, synth
from tests.helpers import check_close, oracle_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _heads_of(t, heads):
    """[B, N, H, d] tensor -> list of [N, d] per flat head b*H+h (on the same device)."""
    B, N, H, d = t.shape
    return [t[f // H, :, f % H, :] for f in heads]


def oracle_on(q, k, v, slopes, heads=None, t_sel=None, state_in=None):
    """Runs the oracle on the selected flat heads of GPU/CPU tensors q, k, v [B, N, H, d]."""
    B, N, H, d = q.shape
    if heads is None:
        return oracle.prefill(oracle_bits(q), oracle_bits(k), oracle_bits(v),
                              slopes.cpu().numpy(), t_sel=t_sel, state_in=state_in)
    # gather the selected heads into a [1, N, n_sel, d] problem with per-head slopes
    sel = list(heads)
    qs = torch.stack(_heads_of(q, sel), dim=1).unsqueeze(0)
    ks = torch.stack(_heads_of(k, sel), dim=1).unsqueeze(0)
    vs = torch.stack(_heads_of(v, sel), dim=1).unsqueeze(0)
    sl = slopes.cpu()[[f % H for f in sel]]
    return oracle.prefill(oracle_bits(qs), oracle_bits(ks), oracle_bits(vs), sl.numpy(),
                          t_sel=t_sel, state_in=state_in)


def gpu_heads(out, heads, t_sel=None):
    B, N, H, d = out.shape
    x = out.permute(0, 2, 1, 3).reshape(B * H, N, d)
    x = x[list(heads)] if heads is not None else x
    if t_sel is not None:
        x = x[:, torch.as_tensor(t_sel, device=x.device)]
    return x.float().cpu().numpy()


def state_heads(state, heads):
    B, H, d, _ = state.shape
    x = state.reshape(B * H, d, d)
    x = x[list(heads)] if heads is not None else x
    return x.cpu().numpy()


def draw(B, N, H, d, seed, dtype=torch.bfloat16, dist="scaled_normal"):
    return synth.draw_qkv(B, N, H, d, dist=dist, seed=seed, dtype=dtype, device=DEV)


# ------------------------------------------------------------------------------------------
# fp32 path (tiny fp32 workload) and the recurrent kernel
# ------------------------------------------------------------------------------------------
def test_tiny_fp32_full():
    w = synth.WORKLOADS["tiny_fp32"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    out, st = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_on(q, k, v, sl)
    check_close(gpu_heads(out, None), o_ref, torch.float32, "o")
    check_close(state_heads(st, None), s_ref, torch.float32, "state")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_recurrent_path(d, dtype):
    q, k, v = draw(2, 77, 3, d, 11, dtype)
    sl = synth.slopes(3, DEV)
    out, st = la.prefill(q, k, v, sl, path=la.LA_PATH_RECURRENT)
    o_ref, s_ref = oracle_on(q, k, v, sl)
    check_close(gpu_heads(out, None), o_ref, dtype, "o")
    check_close(state_heads(st, None), s_ref, dtype, "state")


# ------------------------------------------------------------------------------------------
# tensor-core chunked path
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 255, 256, 257, 1000, 2100])
@pytest.mark.parametrize("segments", [0, 1, 2, 3, 7])
def test_tensor_small(N, segments):
    B, H = 2, 3
    q, k, v = draw(B, N, H, 128, 100 + N)
    sl = synth.slopes(H, DEV)
    out, st = la.prefill(q, k, v, sl, segments=segments, path=la.LA_PATH_TENSOR)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_on(q, k, v, sl)
    check_close(gpu_heads(out, None), o_ref, torch.bfloat16, f"o N={N} seg={segments}")
    check_close(state_heads(st, None), s_ref, torch.bfloat16, f"state N={N} seg={segments}")


def test_tensor_prefill_4k_full():
    w = synth.WORKLOADS["prefill_4k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    out, st = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_on(q, k, v, sl)
    check_close(gpu_heads(out, None), o_ref, torch.bfloat16, "o")
    check_close(state_heads(st, None), s_ref, torch.bfloat16, "state")


def test_tensor_prefill_32k_sampled_heads():
    """Full-size mid-context launch (B=2, N=32768, H=64); the oracle checks 8 heads fully."""
    w = synth.WORKLOADS["prefill_32k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    out, st = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(st).all()
    heads = [0, 63, 64 + 31, 64 + 1, 17, 64 + 48, 40, 127]
    o_ref, s_ref = oracle_on(q, k, v, sl, heads=heads)
    check_close(gpu_heads(out, heads), o_ref, torch.bfloat16, "o")
    check_close(state_heads(st, heads), s_ref, torch.bfloat16, "state")


def test_tensor_prefill_256k_windows():
    """Long context (N=262144): o on 8 seeded 4096-token windows and the final state, for four
    heads from the fastest to the slowest decay."""
    w = synth.WORKLOADS["prefill_256k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    out, st = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    starts = synth.window_starts(w.N, 8, 4096, 1002)
    t_sel = sorted(set(t for s0 in starts for t in range(s0, s0 + 4096)))
    heads = [0, 21, 42, 63]
    o_ref, s_ref = oracle_on(q, k, v, sl, heads=heads, t_sel=t_sel)
    check_close(gpu_heads(out, heads, t_sel), o_ref, torch.bfloat16, "o windows")
    check_close(state_heads(st, heads), s_ref, torch.bfloat16, "state")
    del q, k, v, out


@pytest.mark.parametrize("slope", [0.0, 1e-6])
def test_scan_long_no_forgetting(slope):
    """With lambda = 1 (or within 1e-6 of it) nothing is forgotten, so a segment scan that lost
    cross-segment state would fail here even though decaying heads would hide it."""
    B, N, H = 1, 65536, 2
    q, k, v = draw(B, N, H, 128, 7)
    sl = torch.full((H,), slope, dtype=torch.float32, device=DEV)
    out, st = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    t_sel = list(range(0, N, 97)) + [N - 1]
    t_sel = sorted(set(t_sel))
    o_ref, s_ref = oracle_on(q, k, v, sl, t_sel=t_sel)
    check_close(gpu_heads(out, None, t_sel), o_ref, torch.bfloat16, "o")
    check_close(state_heads(st, None), s_ref, torch.bfloat16, "state")


def test_segment_count_invariance():
    B, N, H = 1, 8192, 4
    q, k, v = draw(B, N, H, 128, 8)
    sl = synth.slopes(H, DEV)
    o_ref, s_ref = oracle_on(q, k, v, sl)
    outs = []
    for seg in [1, 2, 3, 7, 64]:
        out, st = la.prefill(q, k, v, sl, segments=seg, path=la.LA_PATH_TENSOR)
        torch.cuda.synchronize()
        check_close(gpu_heads(out, None), o_ref, torch.bfloat16, f"o seg={seg}")
        check_close(state_heads(st, None), s_ref, torch.bfloat16, f"state seg={seg}")
        outs.append(out.float())
    for o in outs[1:]:
        check_close(o.cpu().numpy(), outs[0].cpu().numpy(), torch.bfloat16, "segment agreement")


def test_chunked_matches_recurrent():
    """Chunk length 128 (tensor cores) and chunk length 1 (token recurrence) agree."""
    q, k, v = draw(1, 3000, 4, 128, 9)
    sl = synth.slopes(4, DEV)
    o1, s1 = la.prefill(q, k, v, sl, path=la.LA_PATH_TENSOR)
    o2, s2 = la.prefill(q, k, v, sl, path=la.LA_PATH_RECURRENT)
    torch.cuda.synchronize()
    check_close(o1.float().cpu().numpy(), o2.float().cpu().numpy(), torch.bfloat16, "o")
    check_close(s1.cpu().numpy(), s2.cpu().numpy(), torch.bfloat16, "state")


def test_no_memory_limit():
    """lambda -> 0 (slope 1e4): o_t = (q_t . k_t) v_t; exercises the general decay-mask path."""
    q, k, v = draw(1, 300, 2, 128, 10)
    sl = torch.full((2,), 1e4, dtype=torch.float32, device=DEV)
    out, st = la.prefill(q, k, v, sl, path=la.LA_PATH_TENSOR)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_on(q, k, v, sl)
    check_close(gpu_heads(out, None), o_ref, torch.bfloat16, "o")
    check_close(state_heads(st, None), s_ref, torch.bfloat16, "state")


def test_silu_inputs_wide_slopes():
    q, k, v = draw(1, 1500, 4, 128, 12, dist="silu_qk")
    sl = torch.tensor([0.0, 0.05, 0.9, 2.5], dtype=torch.float32, device=DEV)
    out, st = la.prefill(q, k, v, sl, path=la.LA_PATH_TENSOR)
    o_ref, s_ref = oracle_on(q, k, v, sl)
    check_close(gpu_heads(out, None), o_ref, torch.bfloat16, "o")
    check_close(state_heads(st, None), s_ref, torch.bfloat16, "state")


def test_prefix_causality():
    q, k, v = draw(1, 2000, 2, 128, 13)
    sl = synth.slopes(2, DEV)
    o_long, _ = la.prefill(q, k, v, sl)
    o_short, _ = la.prefill(q[:, :700].contiguous(), k[:, :700].contiguous(),
                            v[:, :700].contiguous(), sl)
    torch.cuda.synchronize()
    check_close(o_long[:, :700].float().cpu().numpy(), o_short.float().cpu().numpy(),
                torch.bfloat16, "prefix")


def test_linear_in_v():
    q, k, v = draw(1, 1000, 2, 128, 14)
    sl = synth.slopes(2, DEV)
    o1, s1 = la.prefill(q, k, v, sl)
    o2, s2 = la.prefill(q, k, (2 * v.float()).to(torch.bfloat16), sl)  # exact doubling
    torch.cuda.synchronize()
    assert torch.equal(o2.float(), 2 * o1.float())
    assert torch.equal(s2, 2 * s1)


def test_deterministic():
    w = synth.WORKLOADS["prefill_4k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    o1, s1 = la.prefill(q, k, v, sl)
    o2, s2 = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert torch.equal(s1, s2)


def test_workspace_status_and_size_errors():
    q, k, v = draw(1, 4096, 2, 128, 15)
    sl = synth.slopes(2, DEV)
    desc = la.make_desc(1, 4096, 2, 128, torch.bfloat16)
    need = la.la_prefill_workspace_bytes(desc)
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q)
    st = torch.empty(1, 2, 128, 128, dtype=torch.float32, device=DEV)
    s = torch.cuda.current_stream().cuda_stream
    rc = la.la_prefill(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                       out.data_ptr(), st.data_ptr(), ws.data_ptr(), need, s)
    assert rc == la.LA_OK
    assert la.la_workspace_status(ws.data_ptr(), s) == la.LA_OK
    rc = la.la_prefill(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                       out.data_ptr(), st.data_ptr(), ws.data_ptr(), need - 1, s)
    assert rc == la.LA_ERR_WORKSPACE
    rc = la.la_prefill(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                       out.data_ptr(), st.data_ptr(), ws.data_ptr() + 16, need - 16, s)
    assert rc in (la.LA_ERR_ALIGN, la.LA_ERR_WORKSPACE)
    # library-allocated workspace (NULL)
    rc = la.la_prefill(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                       out.data_ptr(), st.data_ptr(), 0, 0, s)
    assert rc == la.LA_OK
    torch.cuda.synchronize()


# ------------------------------------------------------------------------------------------
# decode
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_steps_match_oracle(d, dtype):
    B, H, steps = 3, 5, 6
    g = torch.Generator(device=DEV).manual_seed(21)
    state = torch.randn(B, H, d, d, generator=g, device=DEV) * 0.1
    sl = synth.slopes(H, DEV)
    ref = state.double().cpu().numpy().copy()
    for t in range(steps):
        q, k, v = synth.draw_decode_token(g, B, H, d, dtype=dtype, device=DEV)
        o = la.decode_step(q, k, v, sl, state)
        o_ref = oracle.decode(oracle_bits(q), oracle_bits(k), oracle_bits(v), sl.cpu().numpy(),
                              ref)
        check_close(o.float().cpu().numpy(), o_ref, dtype, f"o step {t}")
    check_close(state.cpu().numpy(), ref, dtype, "state")


def test_decode_continues_prefill():
    """prefill(N1) then n decode steps == prefill(N1 + n) on the tail, and the same state."""
    B, N1, n, H = 2, 600, 9, 3
    q, k, v = draw(B, N1 + n, H, 128, 22)
    sl = synth.slopes(H, DEV)
    o_full, s_full = la.prefill(q, k, v, sl)
    _, state = la.prefill(q[:, :N1].contiguous(), k[:, :N1].contiguous(),
                          v[:, :N1].contiguous(), sl)
    for t in range(N1, N1 + n):
        o = la.decode_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), sl,
                           state)
        check_close(o.float().cpu().numpy(), o_full[:, t].float().cpu().numpy(), torch.bfloat16,
                    f"token {t}")
    check_close(state.cpu().numpy(), s_full.cpu().numpy(), torch.bfloat16, "state")


def test_decode_workload_sampled():
    """256 sequences x 64 heads: 2048-token prefill, then 512 decode steps; every step's o and
    the final state are checked on two sequences (all heads)."""
    w = synth.WORKLOADS["decode_256x2k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    _, state = la.prefill(q, k, v, sl)
    seqs = [0, 201]
    heads = [b * w.H + h for b in seqs for h in range(w.H)]
    _, s_ref = oracle_on(q, k, v, sl, heads=heads)
    s_ref = s_ref.reshape(len(seqs), w.H, w.d, w.d).copy()
    del q, k, v
    g = synth.decode_token_generator(w.decode_seed, DEV)
    worst = 0.0
    for t in range(w.decode_steps):
        qt, kt, vt = synth.draw_decode_token(g, w.B, w.H, w.d, device=DEV)
        o = la.decode_step(qt, kt, vt, sl, state)
        o_ref = oracle.decode(oracle_bits(qt[seqs]), oracle_bits(kt[seqs]),
                              oracle_bits(vt[seqs]), sl.cpu().numpy(), s_ref)
        r, _ = check_close(o[seqs].float().cpu().numpy(), o_ref, torch.bfloat16, f"step {t}")
        worst = max(worst, r)
    check_close(state[seqs].cpu().numpy(), s_ref, torch.bfloat16, "final state")
