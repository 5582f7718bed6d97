"""GPU test of la_prefill_noalloc, the entry point for callers that cannot allocate device
memory.

Some callers of this library cannot call cudaMalloc while they run.  One kind is a serving
process that handed all device memory to its own pool at start-up, where a stray allocation
would fail or stall the device.  Another is a host framework that gives a kernel library its
inputs and outputs but no allocator.  la_prefill_noalloc serves them from a fixed scratch array
built into the library.  This test calls it through the C ABI twice in a row, with different
problems, so the second call meets the first call's leftover scratch contents.  It checks each
result against la_prefill with a workspace the test allocates.  Both entry points run the same
kernel with the same plan, and that kernel is deterministic, so the results must be equal bit
for bit: any effect of stale scratch contents shows, however small.  It also checks that a
problem larger than the array is refused.

The file name sorts last, so a run that stops at the first failure has run every other test.
"""
import pytest
import torch

from long_context_attention_la_b200 import la, synth

pytestmark = pytest.mark.gpu


def _reference(q, k, v, sl):
    """Output and final state from the existing entry point with an allocated workspace."""
    return la.prefill(q, k, v, sl)


def _noalloc(q, k, v, sl):
    B, N, H, d = q.shape
    desc = la.make_desc(B, N, H, d, q.dtype)
    out = torch.empty_like(q)
    st = torch.empty(B, H, d, d, dtype=torch.float32, device=q.device)
    rc = la.la_prefill_noalloc(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                               out.data_ptr(), st.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert rc == la.LA_OK, la.la_status_string(rc)
    return out, st


def test_noalloc_matches_allocating_entry_point_twice():
    # call 1: one 64-head sequence long enough for a multi-segment scan (largest scratch use)
    q1, k1, v1 = synth.draw_qkv(1, 8192, 64, 128, seed=31, device="cuda")
    sl1 = synth.slopes(64, "cuda")
    # call 2: a different shape, so stale flags or ring contents from call 1 would show
    q2, k2, v2 = synth.draw_qkv(2, 3000, 16, 128, seed=32, device="cuda")
    sl2 = synth.slopes(16, "cuda")

    o1, s1 = _noalloc(q1, k1, v1, sl1)
    o2, s2 = _noalloc(q2, k2, v2, sl2)
    torch.cuda.synchronize()
    r1, rs1 = _reference(q1, k1, v1, sl1)
    r2, rs2 = _reference(q2, k2, v2, sl2)
    torch.cuda.synchronize()
    assert torch.equal(o1, r1), "call 1 o"
    assert torch.equal(s1, rs1), "call 1 state"
    assert torch.equal(o2, r2), "call 2 o"
    assert torch.equal(s2, rs2), "call 2 state"


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 4 x 64 sequences cut into 2 segments each need a 32 MiB ring: more than the array holds
    B, N, H, d = 4, 4096, 64, 128
    desc = la.make_desc(B, N, H, d, torch.bfloat16, segments=2)
    assert la.la_prefill_workspace_bytes(desc) > la.LA_NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, N, H, d, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    sl = synth.slopes(H, "cuda")
    rc = la.la_prefill_noalloc(desc, q.data_ptr(), q.data_ptr(), q.data_ptr(), sl.data_ptr(),
                               out.data_ptr(), 0, torch.cuda.current_stream().cuda_stream)
    assert rc == la.LA_ERR_WORKSPACE
