"""Failure detection on the GPU without a GPU fault.

Every device wait of the chunked prefill is bounded.  A host-side switch withholds the scan flag
of segment 0, so segment 1 of every sequence waits for a flag that nothing sets.  The kernel must
give up after the (shortened) limit, unwind, free its tensor memory and report LA_ERR_TIMEOUT in
the workspace status word, and the same CUDA context must then run a normal prefill correctly.
"""
import os

import pytest
import torch

from long_context_attention_la_b200 import la, synth
from tests.helpers import check_close

pytestmark = pytest.mark.gpu


def _run(q, k, v, sl, segments):
    B, N, H, d = q.shape
    desc = la.make_desc(B, N, H, d, q.dtype, segments=segments)
    need = la.la_prefill_workspace_bytes(desc)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    st = torch.empty(B, H, d, d, dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    rc = la.la_prefill(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                       out.data_ptr(), st.data_ptr(), ws.data_ptr(), need, s)
    assert rc == la.LA_OK
    return la.la_workspace_status(ws.data_ptr(), s), out, st


def test_withheld_scan_flag_times_out_and_context_survives(monkeypatch):
    q, k, v = synth.draw_qkv(1, 2048, 4, 128, seed=41, device="cuda")
    sl = synth.slopes(4, "cuda")
    monkeypatch.setenv("LA_DEBUG_WITHHOLD_SEGMENT", "0")
    monkeypatch.setenv("LA_DEBUG_WAIT_LIMIT_MS", "300")
    status, _, _ = _run(q, k, v, sl, segments=2)
    assert status == la.LA_ERR_TIMEOUT, la.la_status_string(status)
    monkeypatch.delenv("LA_DEBUG_WITHHOLD_SEGMENT")
    monkeypatch.delenv("LA_DEBUG_WAIT_LIMIT_MS")
    # the context is intact: a normal call succeeds and matches the recurrent kernel
    status, out, st = _run(q, k, v, sl, segments=2)
    assert status == la.LA_OK
    ref_o, ref_s = la.prefill(q, k, v, sl, path=la.LA_PATH_RECURRENT)
    torch.cuda.synchronize()
    check_close(out.float().cpu().numpy(), ref_o.float().cpu().numpy(), torch.bfloat16, "o")
    check_close(st.cpu().numpy(), ref_s.cpu().numpy(), torch.bfloat16, "state")
