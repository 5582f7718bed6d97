"""The C ABI library builds, loads, and exports every function include/la.h declares; host-side
argument checks return their status codes before any CUDA work (CPU only)."""
import ctypes
import os
import re

import pytest

from long_context_attention_la_b200 import build as labuild
from long_context_attention_la_b200 import la

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "la.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(la_[a-z0-9_]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    path = labuild.build()
    return la.library(path)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["la_prefill", "la_decode_step", "la_prefill_workspace_bytes",
              "la_workspace_status", "la_status_string", "la_version"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in la.h but not exported"


def test_version_and_status_strings(lib):
    assert la.la_version() == 1000
    for code in range(-10, 1):
        assert la.la_status_string(code) not in ("", "unknown status")
    assert la.la_status_string(-99) == "unknown status"


def _desc(**kw):
    base = dict(B=1, N=16, H=2, d=128, dtype=la.LA_BF16, chunk=0, segments=0, path=0)
    base.update(kw)
    return la.la_desc(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), la.LA_ERR_SHAPE), (dict(N=0), la.LA_ERR_SHAPE), (dict(H=0), la.LA_ERR_SHAPE),
    (dict(d=96), la.LA_ERR_SHAPE), (dict(dtype=7), la.LA_ERR_DTYPE),
    (dict(path=9), la.LA_ERR_UNSUPPORTED), (dict(chunk=64), la.LA_ERR_UNSUPPORTED),
    (dict(dtype=la.LA_F32, path=la.LA_PATH_TENSOR), la.LA_ERR_UNSUPPORTED),
    (dict(B=1 << 40, N=1 << 40), la.LA_ERR_OVERFLOW), (dict(segments=-1), la.LA_ERR_SHAPE),
])
def test_prefill_rejects_bad_descriptors(lib, kw, status):
    d = _desc(**kw)
    assert la.la_prefill(d, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0, 0, 0, 0) == status


def test_prefill_null_and_alignment(lib):
    d = _desc()
    assert la.la_prefill(d, 0, 0x2000, 0x3000, 0x4000, 0x5000, 0, 0, 0, 0) == la.LA_ERR_NULL
    assert la.la_prefill(d, 0x1008, 0x2000, 0x3000, 0x4000, 0x5000, 0, 0, 0, 0) == la.LA_ERR_ALIGN
    assert lib.la_prefill(None, None, None, None, None, None, None, None, 0, None) == la.LA_ERR_NULL


def test_prefill_rejects_aliasing(lib):
    d = _desc(N=16, H=2, d=128)
    nbytes = 16 * 2 * 128 * 2
    base = 0x100000
    assert la.la_prefill(d, base, base + nbytes, base + 2 * nbytes, 0x4000, base + 64, 0, 0, 0,
                         0) == la.LA_ERR_ALIAS


def test_decode_rejects_bad_arguments(lib):
    ok = (0x1000, 0x2000, 0x3000, 0x4000, 0x50000, 0x9000, 0)
    assert la.la_decode_step(0, 2, 128, la.LA_BF16, *ok) == la.LA_ERR_SHAPE
    assert la.la_decode_step(1, 2, 32, la.LA_BF16, *ok) == la.LA_ERR_SHAPE
    assert la.la_decode_step(1, 2, 128, 5, *ok) == la.LA_ERR_DTYPE
    assert la.la_decode_step(1, 2, 128, la.LA_BF16, 0, *ok[1:]) == la.LA_ERR_NULL
    assert la.la_decode_step(1, 2, 128, la.LA_BF16, 0x1004, *ok[1:]) == la.LA_ERR_ALIGN
    # out overlapping the state
    assert la.la_decode_step(1, 2, 128, la.LA_BF16, 0x1000, 0x2000, 0x3000, 0x4000, 0x50000,
                             0x50000 + 256, 0) == la.LA_ERR_ALIAS


def test_workspace_status_null(lib):
    assert la.la_workspace_status(0, 0) == la.LA_ERR_NULL


def test_recurrent_path_needs_no_workspace(lib):
    assert la.la_prefill_workspace_bytes(_desc(dtype=la.LA_F32, d=64)) == 0
    assert la.la_prefill_workspace_bytes(_desc(path=la.LA_PATH_RECURRENT)) == 0
    assert la.la_prefill_workspace_bytes(_desc(dtype=7)) == 0


def test_tensor_path_workspace_covers_the_scan(lib):
    # one sequence of 64 chunks -> several segments, so the ring of two d x d fp32 states per
    # sequence and the flags must fit
    w = la.la_prefill_workspace_bytes(_desc(B=1, H=1, N=64 * 128))
    assert w >= 256 + 2 * 4 + 2 * 128 * 128 * 4
    # single segment per sequence: only the header
    w1 = la.la_prefill_workspace_bytes(_desc(B=1, H=1, N=64 * 128, segments=1))
    assert w1 == 256 or w1 == 512
