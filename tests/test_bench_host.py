"""Host-side logic of bench.py (CPU only): the committed counter record, the algorithmic bytes
behind the roofline fraction, and the executed-flops table behind the tensor-pipe field."""
import hashlib
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILE = os.path.join(ROOT, "profiles", "chunked_prefill_kernel_counters.md")


def _record():
    text = open(PROFILE).read()
    start = text.index("```json\n") + len("```json\n")
    return text, json.loads(text[start:text.index("\n```", start)])


def test_counter_record_is_well_formed():
    _, rec = _record()
    for key in ("sources", "source_sha256", "dram_bytes_read", "dram_bytes_write",
                "sm__pipe_tensor_cycles_active_pct_active",
                "sm__pipe_tensor_cycles_active_pct_elapsed"):
        assert key in rec
    assert all(os.path.exists(os.path.join(ROOT, p)) for p in rec["sources"])
    # the DRAM traffic of one prefill_32k launch is close to its algorithmic bytes
    algorithmic = 2 * 32768 * 64 * bench.prefill_bytes_per_token_head(128) + 2 * 64 * 128 * 128 * 4
    traffic = rec["dram_bytes_read"] + rec["dram_bytes_write"]
    assert 0.95 * algorithmic <= traffic <= 1.05 * algorithmic
    assert 0.0 < rec["sm__pipe_tensor_cycles_active_pct_active"] <= 100.0


def test_counter_record_follows_the_sources(tmp_path):
    text, rec = _record()
    h = hashlib.sha256()
    for src in rec["sources"]:
        h.update(open(os.path.join(ROOT, src), "rb").read())
    current = bench.measured_counters(PROFILE)
    assert (current is not None) == (h.hexdigest() == rec["source_sha256"])
    # a record taken on other sources is not reported
    stale = tmp_path / "stale.md"
    stale.write_text(text.replace(rec["source_sha256"], "0" * 64))
    assert bench.measured_counters(str(stale)) is None
    assert bench.measured_counters(str(tmp_path / "missing.md")) is None


@pytest.mark.parametrize("kw,want", [
    (dict(), 1024),                                   # q, k, v read, o written
    (dict(gate=True), 1280),                          # + the gate read
    (dict(gate_separate=True), 1792),                 # + o and the gate read again, y written
    (dict(gate_separate=True, fp8=True), 1024 + 512 + 128 + 4),
])
def test_prefill_bytes_per_token_head(kw, want):
    assert bench.prefill_bytes_per_token_head(128, **kw) == want


def test_executed_flops_table():
    d = 128
    # four 128 x 128 x 128 products per 128-token tile at C = 128: 4 d^2 + 4 C d per token-head
    assert bench.EXECUTED_FLOPS_PER_TOKEN_HEAD[128] == 4 * d * d + 4 * 128 * d
    # C = 64 and C = 256: five such products per tile (per two tiles: ten)
    assert bench.EXECUTED_FLOPS_PER_TOKEN_HEAD[64] == 5 * 2 * 128 ** 3 // 128
    assert bench.EXECUTED_FLOPS_PER_TOKEN_HEAD[256] == 5 * 2 * 128 ** 3 // 128
