"""Parity of the CUDA path (through the C ABI) against the fp64 oracle, on a GPU.

Bar: bf16 I/O relL2 <= 1e-2 and maxabs <= 2e-2 * max|ref| for o and the final state; fp32 I/O
relL2 <= 1e-5.  Inputs are seeded synthetic draws (long_context_attention_la_b200.synth); the
oracle receives the exact bits the GPU read.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_la_b200 import la, synth
from tests.helpers import ParityAccumulator, check_close, oracle_bits

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


@pytest.mark.parametrize("chunk", [64, 256])
@pytest.mark.parametrize("N", [1, 5, 63, 64, 65, 127, 128, 129, 255, 256, 257, 383, 1000, 2100])
@pytest.mark.parametrize("segments", [0, 1, 2, 3])
def test_tensor_small_chunks(chunk, N, segments):
    """Chunk lengths 64 (two chunks per 128-token tile) and 256 (two tiles per chunk): ragged
    lengths around both chunk sizes, with and without segments."""
    B, H = 2, 3
    q, k, v = draw(B, N, H, 128, 400 + N)
    sl = synth.slopes(H, DEV)
    out, st = la.prefill(q, k, v, sl, chunk=chunk, segments=segments, path=la.LA_PATH_TENSOR)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_on(q, k, v, sl)
    what = f"C={chunk} N={N} seg={segments}"
    check_close(gpu_heads(out, None), o_ref, torch.bfloat16, f"o {what}")
    check_close(state_heads(st, None), s_ref, torch.bfloat16, f"state {what}")


def test_tensor_prefill_4k_full():
    w = synth.WORKLOADS["prefill_4k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    out, st = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_on(q, k, v, sl)
    check_close(gpu_heads(out, None), o_ref, torch.bfloat16, "o")
    check_close(state_heads(st, None), s_ref, torch.bfloat16, "state")


def gather_heads(t, heads, t_sel=None):
    """[B, N, H, d] tensor -> float64-ready numpy [len(heads), n_t, d] of the flat heads b*H+h
    (gathered head by head on the device, so no copy of the whole tensor is made)."""
    B, N, H, d = t.shape
    idx = None if t_sel is None else torch.as_tensor(t_sel, device=t.device)
    parts = []
    for f in heads:
        x = t[f // H, :, f % H, :]
        parts.append(x if idx is None else x.index_select(0, idx))
    return torch.stack(parts).float().cpu().numpy()


def test_tensor_prefill_32k_full():
    """Full-size mid-context launch (B=2, N=32768, H=64): every output and the whole final state
    against the oracle, 16 flat heads per oracle call."""
    w = synth.WORKLOADS["prefill_32k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    out, st = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    acc_o = ParityAccumulator(torch.bfloat16, "prefill_32k o")
    acc_s = ParityAccumulator(torch.bfloat16, "prefill_32k state")
    t0 = time.perf_counter()
    for f0 in range(0, w.B * w.H, 16):
        heads = list(range(f0, f0 + 16))
        o_ref, s_ref = oracle_on(q, k, v, sl, heads=heads)
        acc_o.add(gather_heads(out, heads), o_ref, tag=f"heads {f0}..{f0 + 15}")
        acc_s.add(state_heads(st, heads), s_ref, tag=f"heads {f0}..{f0 + 15}")
    print(f"prefill_32k: oracle + compare {time.perf_counter() - t0:.1f} s")
    acc_o.check()
    acc_s.check()


def test_chunk_sweep_prefill_32k_full():
    """P-chunk: the mid-context workload (B=2, N=32768, H=64) with chunk lengths 64, 128 and 256
    on the tensor cores; each is compared with the oracle over every output and the whole final
    state, and with the others.  The results differ only in where bf16 roundings fall."""
    w = synth.WORKLOADS["prefill_32k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    chunks = [64, 128, 256]
    res = {}
    for c in chunks:
        res[c] = la.prefill(q, k, v, sl, chunk=c)
    torch.cuda.synchronize()
    acc_o = {c: ParityAccumulator(torch.bfloat16, f"prefill_32k C={c} o") for c in chunks}
    acc_s = {c: ParityAccumulator(torch.bfloat16, f"prefill_32k C={c} state") for c in chunks}
    for f0 in range(0, w.B * w.H, 16):
        heads = list(range(f0, f0 + 16))
        o_ref, s_ref = oracle_on(q, k, v, sl, heads=heads)
        for c in chunks:
            out, st = res[c]
            acc_o[c].add(gather_heads(out, heads), o_ref, tag=f"heads {f0}..{f0 + 15}")
            acc_s[c].add(state_heads(st, heads), s_ref, tag=f"heads {f0}..{f0 + 15}")
    for c in chunks:
        acc_o[c].check()
        acc_s[c].check()
    # the chunk lengths against one another (C = 128 as the reference)
    for c in (64, 256):
        check_close(res[c][0].float().cpu().numpy(), res[128][0].float().cpu().numpy(),
                    torch.bfloat16, f"o C={c} vs C=128")
        check_close(res[c][1].cpu().numpy(), res[128][1].cpu().numpy(), torch.bfloat16,
                    f"state C={c} vs C=128")


def test_tensor_prefill_256k_windows_full():
    """Long context (N=262144, H=64): o of every head on 8 seeded 4096-token windows, and the
    whole final state, against the oracle (which runs the full recurrence of every head)."""
    w = synth.WORKLOADS["prefill_256k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    out, st = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    starts = synth.window_starts(w.N, 8, 4096, 1002)
    t_sel = sorted(set(t for s0 in starts for t in range(s0, s0 + 4096)))
    acc_o = ParityAccumulator(torch.bfloat16, "prefill_256k o windows")
    acc_s = ParityAccumulator(torch.bfloat16, "prefill_256k state")
    t0 = time.perf_counter()
    for h0 in range(0, w.H, 16):
        heads = list(range(h0, h0 + 16))
        o_ref, s_ref = oracle_on(q, k, v, sl, heads=heads, t_sel=t_sel)
        acc_o.add(gather_heads(out, heads, t_sel), o_ref, tag=f"heads {h0}..{h0 + 15}")
        acc_s.add(state_heads(st, heads), s_ref, tag=f"heads {h0}..{h0 + 15}")
    print(f"prefill_256k: oracle + compare {time.perf_counter() - t0:.1f} s")
    del q, k, v, out
    acc_o.check()
    acc_s.check()


@pytest.mark.parametrize("segments", [0, la.LA_SEGMENTS_BALANCED])
@pytest.mark.parametrize("chunk", [64, 128, 256])
@pytest.mark.parametrize("slope", [0.0, 1e-6])
def test_scan_long_no_forgetting(slope, chunk, segments):
    """With lambda = 1 (or within 1e-6 of it) nothing is forgotten, so a segment scan that lost
    cross-segment state would fail here even though decaying heads would hide it.  The balanced
    plan passes each sequence's state along a chain of about 74 ranges."""
    B, N, H = 1, 65536, 2
    q, k, v = draw(B, N, H, 128, 7)
    sl = torch.full((H,), slope, dtype=torch.float32, device=DEV)
    out, st = la.prefill(q, k, v, sl, chunk=chunk, segments=segments)
    torch.cuda.synchronize()
    t_sel = list(range(0, N, 97)) + [N - 1]
    t_sel = sorted(set(t_sel))
    o_ref, s_ref = oracle_on(q, k, v, sl, t_sel=t_sel)
    check_close(gpu_heads(out, None, t_sel), o_ref, torch.bfloat16, "o")
    check_close(state_heads(st, None), s_ref, torch.bfloat16, "state")


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_segment_count_invariance(chunk):
    B, N, H = 1, 8192, 4
    q, k, v = draw(B, N, H, 128, 8)
    sl = synth.slopes(H, DEV)
    o_ref, s_ref = oracle_on(q, k, v, sl)
    outs = []
    # LA_SEGMENTS_BALANCED: one range of about 1.7 tiles per SM, so nearly every range is cut
    # inside a sequence and hands its state to the next through the look-back ring
    for seg in [1, 2, 3, 7, 64, la.LA_SEGMENTS_BALANCED]:
        out, st = la.prefill(q, k, v, sl, chunk=chunk, segments=seg, path=la.LA_PATH_TENSOR)
        torch.cuda.synchronize()
        check_close(gpu_heads(out, None), o_ref, torch.bfloat16, f"o seg={seg}")
        check_close(state_heads(st, None), s_ref, torch.bfloat16, f"state seg={seg}")
        outs.append(out.float())
    for o in outs[1:]:
        check_close(o.cpu().numpy(), outs[0].cpu().numpy(), torch.bfloat16, "segment agreement")


@pytest.mark.parametrize("segments", [0, la.LA_SEGMENTS_BALANCED])
@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_chunked_matches_recurrent(chunk, segments):
    """Chunk lengths 64, 128, 256 (tensor cores) and chunk length 1 (token recurrence) agree, on
    sequences with a ragged last tile (also under the balanced plan)."""
    q, k, v = draw(1, 3000, 4, 128, 9)
    sl = synth.slopes(4, DEV)
    o1, s1 = la.prefill(q, k, v, sl, chunk=chunk, segments=segments, path=la.LA_PATH_TENSOR)
    o2, s2 = la.prefill(q, k, v, sl, path=la.LA_PATH_RECURRENT)
    torch.cuda.synchronize()
    check_close(o1.float().cpu().numpy(), o2.float().cpu().numpy(), torch.bfloat16, "o")
    check_close(s1.cpu().numpy(), s2.cpu().numpy(), torch.bfloat16, "state")


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_no_memory_limit(chunk):
    """lambda -> 0 (slope 1e4): o_t = (q_t . k_t) v_t; exercises the general decay-mask path."""
    q, k, v = draw(1, 300, 2, 128, 10)
    sl = torch.full((2,), 1e4, dtype=torch.float32, device=DEV)
    out, st = la.prefill(q, k, v, sl, chunk=chunk, path=la.LA_PATH_TENSOR)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_on(q, k, v, sl)
    check_close(gpu_heads(out, None), o_ref, torch.bfloat16, "o")
    check_close(state_heads(st, None), s_ref, torch.bfloat16, "state")


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_silu_inputs_wide_slopes(chunk):
    q, k, v = draw(1, 1500, 4, 128, 12, dist="silu_qk")
    sl = torch.tensor([0.0, 0.05, 0.9, 2.5], dtype=torch.float32, device=DEV)
    out, st = la.prefill(q, k, v, sl, chunk=chunk, path=la.LA_PATH_TENSOR)
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


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_deterministic(chunk):
    w = synth.WORKLOADS["prefill_4k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    o1, s1 = la.prefill(q, k, v, sl, chunk=chunk)
    o2, s2 = la.prefill(q, k, v, sl, chunk=chunk)
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


def test_decode_workload_full():
    """256 sequences x 64 heads: a 2048-token prefill, then 512 decode steps.  Every step's o of
    16 seeded sequences (all heads) is checked against the oracle's decode step; the states of all
    256 sequences are checked after the prefill and after the last step (the oracle continues the
    recurrence of every sequence from its own prefill state over the same 512 tokens)."""
    w = synth.WORKLOADS["decode_256x2k"]
    q, k, v = synth.draw_workload(w, device=DEV)
    sl = synth.slopes(w.H, DEV)
    _, state = la.prefill(q, k, v, sl)
    torch.cuda.synchronize()
    gsel = torch.Generator(device="cpu")
    gsel.manual_seed(1005)
    seqs = sorted(torch.randperm(w.B, generator=gsel)[:16].tolist())
    t0 = time.perf_counter()
    # the oracle's state after the prefill, every sequence (16 sequences per call)
    s_init = np.empty((w.B * w.H, w.d, w.d), dtype=np.float64)
    acc_p = ParityAccumulator(torch.bfloat16, "decode_256x2k state after the prefill")
    for b0 in range(0, w.B, 16):
        heads = list(range(b0 * w.H, (b0 + 16) * w.H))
        _, s_ref = oracle_on(q, k, v, sl, heads=heads, t_sel=[])
        s_init[b0 * w.H:(b0 + 16) * w.H] = s_ref
        acc_p.add(state[b0:b0 + 16].reshape(-1, w.d, w.d).cpu().numpy(), s_ref,
                  tag=f"sequences {b0}..{b0 + 15}")
    t_init = time.perf_counter() - t0
    del q, k, v
    acc_p.check()
    s_ref16 = s_init.reshape(w.B, w.H, w.d, w.d)[seqs].copy()
    g = synth.decode_token_generator(w.decode_seed, DEV)
    toks = []
    acc_o = ParityAccumulator(torch.bfloat16, "decode_256x2k o (16 sequences, every step)")
    for t in range(w.decode_steps):
        qt, kt, vt = synth.draw_decode_token(g, w.B, w.H, w.d, device=DEV)
        toks.append((qt, kt, vt))
        o = la.decode_step(qt, kt, vt, sl, state)
        o_ref = oracle.decode(oracle_bits(qt[seqs]), oracle_bits(kt[seqs]),
                              oracle_bits(vt[seqs]), sl.cpu().numpy(), s_ref16)
        acc_o.add(o[seqs].float().cpu().numpy(), o_ref, tag=f"step {t}")
    acc_o.check()
    # final states of all 256 sequences: the oracle's recurrence over the 512 decode tokens from
    # its own prefill state
    acc_s = ParityAccumulator(torch.bfloat16, "decode_256x2k final state (all sequences)")
    t1 = time.perf_counter()
    for b0 in range(0, w.B, 32):
        qs, ks, vs = (torch.stack([tk[i][b0:b0 + 32] for tk in toks], dim=1) for i in range(3))
        _, s_ref = oracle.prefill(oracle_bits(qs), oracle_bits(ks), oracle_bits(vs),
                                  sl.cpu().numpy(), t_sel=[],
                                  state_in=s_init[b0 * w.H:(b0 + 32) * w.H])
        acc_s.add(state[b0:b0 + 32].reshape(-1, w.d, w.d).cpu().numpy(), s_ref,
                  tag=f"sequences {b0}..{b0 + 31}")
    print(f"decode_256x2k: oracle prefill states {t_init:.1f} s, final states "
          f"{time.perf_counter() - t1:.1f} s")
    acc_s.check()
