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


# The argument checks below hand the library made-up device addresses and expect an error code
# before any launch.  On a machine with a GPU a missed check would launch a kernel on them, so
# this module runs only where no GPU is present.
try:
    import torch as _torch
    _HAS_GPU = _torch.cuda.is_available()
except Exception:  # pragma: no cover
    _HAS_GPU = False
pytestmark = pytest.mark.skipif(_HAS_GPU, reason="fake device addresses; CPU-only host checks")


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
    assert la.la_version() == 1004
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
    (dict(path=9), la.LA_ERR_UNSUPPORTED), (dict(chunk=32), la.LA_ERR_UNSUPPORTED),
    (dict(chunk=96), la.LA_ERR_UNSUPPORTED), (dict(chunk=512), la.LA_ERR_UNSUPPORTED),
    (dict(chunk=64, path=la.LA_PATH_RECURRENT), la.LA_ERR_UNSUPPORTED),
    (dict(dtype=la.LA_F32, path=la.LA_PATH_TENSOR), la.LA_ERR_UNSUPPORTED),
    (dict(B=1 << 40, N=1 << 40), la.LA_ERR_OVERFLOW), (dict(segments=-2), la.LA_ERR_SHAPE),
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


def test_plan_cache_returns_the_same_plan(lib):
    # the library keeps the last few plans: sizes asked for again, after the cache has turned
    # over, must come out the same as the first time
    shapes = [dict(B=b, H=h, N=n, segments=sg) for b, h, n in
              [(1, 64, 1 << 18), (2, 64, 1 << 15), (1, 64, 4096), (1, 2, 1 << 16), (4, 16, 1 << 16),
               (1, 1, 64 * 128), (3, 5, 3000)] for sg in (0, la.LA_SEGMENTS_BALANCED)]
    first = [la.la_prefill_workspace_bytes(_desc(**kw)) for kw in shapes]
    again = [la.la_prefill_workspace_bytes(_desc(**kw)) for kw in reversed(shapes)][::-1]
    assert first == again
    assert all(w >= 256 for w in first)


def test_balanced_plan_workspace(lib):
    # LA_SEGMENTS_BALANCED: one range per SM (at most one per tile), each with a flag and one
    # d x d fp32 state: 64 tiles -> 64 ranges on any GPU of 64 SMs or more
    w = la.la_prefill_workspace_bytes(_desc(B=1, H=1, N=64 * 128,
                                            segments=la.LA_SEGMENTS_BALANCED))
    assert w == 256 + 256 + 64 * 128 * 128 * 4
    # many tiles: at most one range per SM (256 at most), within the no-allocation scratch
    wl = la.la_prefill_workspace_bytes(_desc(B=4, H=64, N=1 << 18,
                                             segments=la.LA_SEGMENTS_BALANCED))
    assert 256 + 148 * 128 * 128 * 4 <= wl <= la.LA_NOALLOC_SCRATCH_BYTES


# ---------------------------------------------------------------------------------------------
# la_prefill_varlen: host-side argument checks (CPU only; these return before any CUDA call).
# cu_seqlens is a device array; its contents are checked on the device (GPU tests).
# ---------------------------------------------------------------------------------------------
def _vdesc(**kw):
    base = dict(T=300, n_seqs=3, H=2, d=128, dtype=la.LA_BF16, chunk=0, segments=0, path=0)
    base.update(kw)
    return la.la_varlen_desc(**base)


_P = (0x1000, 0x2000, 0x3000, 0x4000)  # q, k, v, slopes
_CU = 0x6000


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=9), la.LA_ERR_DTYPE), (dict(d=32), la.LA_ERR_SHAPE), (dict(H=0), la.LA_ERR_SHAPE),
    (dict(T=-1), la.LA_ERR_SHAPE), (dict(n_seqs=0), la.LA_ERR_SHAPE),
    (dict(chunk=32), la.LA_ERR_UNSUPPORTED), (dict(path=5), la.LA_ERR_UNSUPPORTED),
    (dict(dtype=la.LA_F32, path=la.LA_PATH_TENSOR), la.LA_ERR_UNSUPPORTED),
    (dict(segments=-2), la.LA_ERR_SHAPE), (dict(T=1 << 40, H=1 << 20), la.LA_ERR_OVERFLOW),
])
def test_varlen_rejects_bad_descriptors(lib, kw, status):
    d = _vdesc(**kw)
    assert la.la_prefill_varlen(d, *_P, _CU, 0, 0x50000, 0, 0, 0, 0) == status
    assert la.la_prefill_varlen_workspace_bytes(d) == 0


def test_varlen_null_alignment_aliasing(lib):
    d = _vdesc()
    assert lib.la_prefill_varlen(None, *_P, _CU, None, None, 0x50000, None, None, 0,
                                 None) == la.LA_ERR_NULL
    assert la.la_prefill_varlen(d, *_P, 0, 0, 0x50000, 0, 0, 0, 0) == la.LA_ERR_NULL
    assert la.la_prefill_varlen(d, 0, *_P[1:], _CU, 0, 0x50000, 0, 0, 0, 0) == la.LA_ERR_NULL
    assert la.la_prefill_varlen(d, *_P, _CU, 0x7008, 0x50000, 0, 0, 0, 0) == la.LA_ERR_ALIGN
    assert la.la_prefill_varlen(d, *_P, _CU, 0, 0x50000, 0x9004, 0, 0, 0) == la.LA_ERR_ALIGN
    nbytes = 300 * 2 * 128 * 2
    # out overlapping k
    assert la.la_prefill_varlen(d, 0x100000, 0x100000 + nbytes, 0x100000 + 2 * nbytes, 0x4000,
                                _CU, 0, 0x100000 + nbytes + 512, 0, 0, 0, 0) == la.LA_ERR_ALIAS
    # state_out overlapping state_in without being the same array
    sbytes = 3 * 2 * 128 * 128 * 4
    assert la.la_prefill_varlen(d, *_P, _CU, 0x10000000, 0x50000000, 0x10000000 + sbytes // 2, 0,
                                0, 0) == la.LA_ERR_ALIAS


def test_varlen_workspace_capacity(lib):
    # tensor path: header + one 48-byte work unit per head for every sequence and every chunk
    T, n, H = 3000, 3, 2
    w = la.la_prefill_varlen_workspace_bytes(_vdesc(T=T, n_seqs=n, H=H, segments=1))
    assert w >= 256 + H * (n + -(-T // 128)) * 48
    # forcing several segments adds the scan flags and state ring of every (sequence, head)
    w2 = la.la_prefill_varlen_workspace_bytes(_vdesc(T=T, n_seqs=n, H=H, segments=3))
    assert w2 >= w + n * H * 2 * 128 * 128 * 4
    # recurrent path: the header only (it reads cu_seqlens in place)
    w3 = la.la_prefill_varlen_workspace_bytes(_vdesc(dtype=la.LA_F32, d=64))
    assert 256 <= w3 < 4096
    # T = 0 (every sequence empty) is a valid problem
    assert la.la_prefill_varlen_workspace_bytes(_vdesc(T=0)) >= 256


def test_varlen_epilogue_checks(lib):
    d = _vdesc()
    ok = la.la_gate_norm(0x800000, 0x900000, 1e-6)

    def call(desc, epi, out=0x50000):
        return la.la_prefill_varlen(desc, *_P, _CU, 0, out, 0, 0, 0, 0, epilogue=epi)

    # the fused norm + gate is a tensor-core epilogue
    assert call(_vdesc(dtype=la.LA_F32, d=64), ok) == la.LA_ERR_UNSUPPORTED
    assert call(_vdesc(path=la.LA_PATH_RECURRENT), ok) == la.LA_ERR_UNSUPPORTED
    assert call(d, la.la_gate_norm(0, 0x900000, 1e-6)) == la.LA_ERR_NULL
    assert call(d, la.la_gate_norm(0x800000, 0, 1e-6)) == la.LA_ERR_NULL
    assert call(d, la.la_gate_norm(0x800008, 0x900000, 1e-6)) == la.LA_ERR_ALIGN
    assert call(d, la.la_gate_norm(0x800000, 0x900004, 1e-6)) == la.LA_ERR_ALIGN
    assert call(d, la.la_gate_norm(0x800000, 0x900000, float("nan"))) == la.LA_ERR_SHAPE
    assert call(d, la.la_gate_norm(0x800000, 0x900000, -1.0)) == la.LA_ERR_SHAPE
    # gate overlapping out
    assert call(d, la.la_gate_norm(0x800000, 0x900000, 1e-6), out=0x800000 + 64) == la.LA_ERR_ALIAS
    # FP8 output is the stand-alone operator's, not this epilogue's
    assert call(d, la.la_gate_norm(0x800000, 0x900000, 1e-6, 0xA00000)) == la.LA_ERR_UNSUPPORTED


def test_varlen_qk_prologue_checks(lib):
    """la_prefill_varlen_qk: the in-tile QK norm + RoPE has one kernel instance (bf16, d = 128,
    tensor path, 128-token chunks); its parameters are checked like la_qk_norm_rope's."""
    ok = dict(gamma_q=0x800000, gamma_k=0x900000, positions=0xA00000, rotary_dim=64, theta=6e6,
              eps=1e-6, pad=0)

    def call(desc=None, out=0x50000, **kw):
        qk = la.la_qk_prologue(**{**ok, **kw})
        return la.la_prefill_varlen_qk(desc or _vdesc(), qk, *_P, _CU, 0, out, 0, 0, 0, 0)

    assert la.la_prefill_varlen_qk(_vdesc(), None, *_P, _CU, 0, 0x50000, 0, 0, 0,
                                   0) == la.LA_ERR_NULL
    # descriptor errors first, as for la_prefill_varlen
    assert call(_vdesc(d=32)) == la.LA_ERR_SHAPE
    assert call(_vdesc(dtype=9)) == la.LA_ERR_DTYPE
    # only the bf16, d = 128, C = 128 tensor-core instance carries it
    assert call(_vdesc(dtype=la.LA_F32)) == la.LA_ERR_UNSUPPORTED
    assert call(_vdesc(d=64)) == la.LA_ERR_UNSUPPORTED
    assert call(_vdesc(path=la.LA_PATH_RECURRENT)) == la.LA_ERR_UNSUPPORTED
    for chunk in (64, 256):
        assert call(_vdesc(chunk=chunk)) == la.LA_ERR_UNSUPPORTED
    assert call(gamma_q=0) == la.LA_ERR_NULL
    assert call(gamma_k=0) == la.LA_ERR_NULL
    assert call(positions=0) == la.LA_ERR_NULL
    assert call(gamma_q=0x800004) == la.LA_ERR_ALIGN
    assert call(gamma_k=0x900008) == la.LA_ERR_ALIGN
    assert call(positions=0xA00004) == la.LA_ERR_ALIGN
    for r in (0, 8, 24, 144):
        assert call(rotary_dim=r) == la.LA_ERR_SHAPE
    for theta in (0.0, -1.0, float("nan"), float("inf")):
        assert call(theta=theta) == la.LA_ERR_SHAPE
    for eps in (-1e-6, float("nan")):
        assert call(eps=eps) == la.LA_ERR_SHAPE
    # q, k, v are only read: out must still not overlap them
    assert call(out=0x1000 + 64) == la.LA_ERR_ALIAS


# ---------------------------------------------------------------------------------------------
# la_qk_norm_rope: host-side argument checks
# ---------------------------------------------------------------------------------------------
def _qdesc(**kw):
    base = dict(T=10, H=2, d=128, q_stride=256, k_stride=256, rotary_dim=64, theta=6e6, eps=1e-6,
                pad=0)
    base.update(kw)
    return la.la_qk_norm_rope_desc(**base)


_Q = (0x100000, 0x200000, 0x300000, 0x300400, 0x400000, 0x500000, 0x600000, 0)


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), la.LA_ERR_SHAPE), (dict(H=0), la.LA_ERR_SHAPE), (dict(T=-1), la.LA_ERR_SHAPE),
    (dict(rotary_dim=8), la.LA_ERR_SHAPE), (dict(rotary_dim=40), la.LA_ERR_SHAPE),
    (dict(rotary_dim=144), la.LA_ERR_SHAPE), (dict(theta=0.0), la.LA_ERR_SHAPE),
    (dict(theta=float("nan")), la.LA_ERR_SHAPE), (dict(eps=-1.0), la.LA_ERR_SHAPE),
    (dict(q_stride=128), la.LA_ERR_SHAPE), (dict(k_stride=260), la.LA_ERR_SHAPE),
])
def test_qk_norm_rope_rejects_bad_descriptors(lib, kw, status):
    assert la.la_qk_norm_rope(_qdesc(**kw), *_Q) == status


def test_qk_norm_rope_null_alignment_alias(lib):
    d = _qdesc()
    assert la.la_qk_norm_rope(d, 0, *_Q[1:]) == la.LA_ERR_NULL
    assert la.la_qk_norm_rope(d, *_Q[:4], 0, *_Q[5:]) == la.LA_ERR_NULL
    assert la.la_qk_norm_rope(d, 0x100008, *_Q[1:]) == la.LA_ERR_ALIGN
    assert la.la_qk_norm_rope(d, *_Q[:2], 0x300004, *_Q[3:]) == la.LA_ERR_ALIGN
    # q_out overlapping k; k_out onto a strided k (not in place)
    assert la.la_qk_norm_rope(d, *_Q[:5], 0x200000 + 64, *_Q[6:]) == la.LA_ERR_ALIAS
    ds = _qdesc(k_stride=512)
    assert la.la_qk_norm_rope(ds, *_Q[:6], 0x200000, 0) == la.LA_ERR_ALIAS


def test_decode_multi_rejects_bad_arguments(lib):
    ok = (0x1000, 0x2000, 0x3000, 0x4000, 0x50000)  # q, k, v, slopes, state
    out = 0x9000
    assert la.la_decode_multi(1, 2, 128, 0, la.LA_BF16, *ok, out, 0) == la.LA_ERR_SHAPE
    assert la.la_decode_multi(1, 2, 96, 2, la.LA_BF16, *ok, out, 0) == la.LA_ERR_SHAPE
    assert la.la_decode_multi(1, 2, 128, 2, 7, *ok, out, 0) == la.LA_ERR_DTYPE
    assert la.la_decode_multi(1, 2, 128, 2, la.LA_BF16, 0, *ok[1:], out, 0) == la.LA_ERR_NULL
    assert la.la_decode_multi(1, 2, 128, 2, la.LA_BF16, 0x1004, *ok[1:], out, 0) == la.LA_ERR_ALIGN
    # out overlapping the state
    assert la.la_decode_multi(1, 2, 128, 2, la.LA_BF16, *ok, 0x50000 + 512, 0) == la.LA_ERR_ALIAS
    bad = la.la_gate_norm(0x800008, 0x900000, 1e-6)
    assert la.la_decode_multi(1, 2, 128, 2, la.LA_BF16, *ok, out, 0,
                              epilogue=bad) == la.LA_ERR_ALIGN
    nan = la.la_gate_norm(0x800000, 0x900000, float("nan"))
    assert la.la_decode_multi(1, 2, 128, 2, la.LA_BF16, *ok, out, 0,
                              epilogue=nan) == la.LA_ERR_SHAPE
    # no FP8 output on the decode path
    fp8 = la.la_gate_norm(0x800000, 0x900000, 1e-6, 0xA00000)
    assert la.la_decode_multi(1, 2, 128, 2, la.LA_BF16, *ok, out, 0,
                              epilogue=fp8) == la.LA_ERR_UNSUPPORTED


def test_gate_norm_apply_rejects_bad_arguments(lib):
    gn = la.la_gate_norm(0x800000, 0x900000, 1e-6)
    o, y = 0x100000, 0x200000
    assert la.la_gate_norm_apply(4, 2, 128, 9, o, gn, y, 0) == la.LA_ERR_DTYPE
    assert la.la_gate_norm_apply(4, 2, 96, la.LA_BF16, o, gn, y, 0) == la.LA_ERR_SHAPE
    assert la.la_gate_norm_apply(-1, 2, 128, la.LA_BF16, o, gn, y, 0) == la.LA_ERR_SHAPE
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, 0, gn, y, 0) == la.LA_ERR_NULL
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, o, None, y, 0) == la.LA_ERR_NULL
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, o + 8, gn, y, 0) == la.LA_ERR_ALIGN
    nan = la.la_gate_norm(0x800000, 0x900000, float("nan"))
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, o, nan, y, 0) == la.LA_ERR_SHAPE
    # y overlapping o without being o, or overlapping the gate
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, o, gn, o + 64, 0) == la.LA_ERR_ALIAS
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, o, gn, 0x800000, 0) == la.LA_ERR_ALIAS
    # FP8 output: not in place, scales aligned and apart from o, y and the gate
    fp8 = la.la_gate_norm(0x800000, 0x900000, 1e-6, 0xA00000)
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, o, fp8, o, 0) == la.LA_ERR_ALIAS
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, o, la.la_gate_norm(
        0x800000, 0x900000, 1e-6, 0xA00008), y, 0) == la.LA_ERR_ALIGN
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, o, la.la_gate_norm(
        0x800000, 0x900000, 1e-6, y + 16), y, 0) == la.LA_ERR_ALIAS
    assert la.la_gate_norm_apply(4, 2, 128, la.LA_BF16, o, la.la_gate_norm(
        0x800000, 0x900000, 1e-6, 0x800000 + 16), y, 0) == la.LA_ERR_ALIAS


def test_prefill_state_rejects_bad_arguments(lib):
    d = _desc(N=1000, H=4)
    ps = la.la_prefill_state
    assert ps(_desc(N=0), 0x1000, 0x2000, 0x3000, 0, 0x40000, 0, 0, 0) == la.LA_ERR_SHAPE
    assert ps(_desc(dtype=5), 0x1000, 0x2000, 0x3000, 0, 0x40000, 0, 0, 0) == la.LA_ERR_DTYPE
    assert ps(d, 0, 0x2000, 0x3000, 0, 0x40000, 0, 0, 0) == la.LA_ERR_NULL
    assert ps(d, 0x1000, 0x2000, 0x3000, 0, 0, 0, 0, 0) == la.LA_ERR_NULL
    assert ps(d, 0x1000, 0x2000, 0, 0, 0x40000, 0, 0, 0) == la.LA_ERR_NULL
    assert ps(d, 0x1008, 0x2000, 0x3000, 0, 0x40000, 0, 0, 0) == la.LA_ERR_ALIGN
    assert ps(d, 0x1000, 0x2000, 0x3000, 0x5008, 0x40000, 0, 0, 0) == la.LA_ERR_ALIGN
    # k spans 1000 * 4 * 128 * 2 bytes from 0x100000: a state_out inside it overlaps
    assert ps(d, 0x100000, 0x900000, 0x3000, 0, 0x100100, 0, 0, 0) == la.LA_ERR_ALIAS
    # state_in and state_out partly overlapping (identical is the in-place form, allowed)
    assert ps(d, 0x100000, 0x900000, 0x3000, 0x2000000, 0x2000100, 0, 0, 0) == la.LA_ERR_ALIAS


def test_prefill_state_workspace(lib):
    # tensor path: a header and two fp32 d x d partial slots per CTA; recurrent path: none
    need = la.la_prefill_state_workspace_bytes(_desc(N=4096, H=64))
    assert need >= 256 + 2 * 128 * 128 * 4 and (need - 256) % (2 * 128 * 128 * 4) == 0
    assert la.la_prefill_state_workspace_bytes(_desc(dtype=la.LA_F32)) == 0
    assert la.la_prefill_state_workspace_bytes(_desc(d=64)) == 0
    assert la.la_prefill_state_workspace_bytes(_desc(N=0)) == 0


def test_state_fold_rejects_bad_arguments(lib):
    f = la.la_state_fold
    ok = dict(parts=0x100000, lengths=[3, 4], slopes=0x3000, state_in=0, state_out=0x40000000)

    def call(n=2, BH=8, H=4, d=128, **kw):
        a = dict(ok)
        a.update(kw)
        return f(n, BH, H, d, a["parts"], a["lengths"], a["slopes"], a["state_in"],
                 a["state_out"], 0)

    assert call(n=-1) == la.LA_ERR_SHAPE
    assert call(n=257, lengths=[1] * 257) == la.LA_ERR_SHAPE
    assert call(BH=6) == la.LA_ERR_SHAPE  # not a multiple of H
    assert call(d=96) == la.LA_ERR_SHAPE
    assert call(parts=0) == la.LA_ERR_NULL
    assert call(lengths=None) == la.LA_ERR_NULL
    assert call(slopes=0) == la.LA_ERR_NULL
    assert call(state_out=0) == la.LA_ERR_NULL
    assert call(lengths=[3, -1]) == la.LA_ERR_SHAPE
    assert call(parts=0x100008) == la.LA_ERR_ALIGN
    assert call(state_in=0x5004) == la.LA_ERR_ALIGN
    # parts span 2 * 8 * 128 * 128 * 4 bytes: a state_out inside them overlaps
    assert call(state_out=0x100000 + 4096) == la.LA_ERR_ALIAS
    assert call(state_in=0x40000000 + 256) == la.LA_ERR_ALIAS


@pytest.mark.parametrize("B,N,H", [(1, 262144, 64), (2, 32768, 64), (1, 4096, 64), (4, 300, 64),
                                   (1, 5, 2), (3, 128, 3)])
def test_prefill_state_workspace_follows_the_range_split(lib, B, N, H):
    """The state pass cuts the B*H*ceil(N/128) chunk-loads into one contiguous range per CTA (at
    most one CTA per SM, 148 when no device is visible) and keeps two partial-state slots per CTA
    behind a 256-byte header."""
    total = B * H * ((N + 127) // 128)
    grid0 = max(1, min(148, total))
    width = -(-total // grid0)
    grid = -(-total // width)
    need = la.la_prefill_state_workspace_bytes(_desc(B=B, N=N, H=H))
    assert need == 256 + 2 * grid * 128 * 128 * 4
    assert grid <= 148 and (grid - 1) * width < total <= grid * width


def test_prefill_rejects_state_overlapping_an_activation(lib):
    d = _desc(N=16, H=2, d=128)
    nbytes = 16 * 2 * 128 * 2
    q, k, v, out = 0x100000, 0x200000, 0x300000, 0x400000
    for st in (q + 256, k, v + nbytes - 16, out + 512):
        assert la.la_prefill(d, q, k, v, 0x4000, out, st, 0, 0, 0) == la.LA_ERR_ALIAS
        assert la.la_prefill_noalloc(d, q, k, v, 0x4000, out, st, 0) == la.LA_ERR_ALIAS


def test_decode_rejects_state_overlapping_a_token_row(lib):
    q, k, v, out = 0x1000000, 0x2000000, 0x3000000, 0x4000000
    sb = 2 * 128 * 128 * 4
    for st in (q - 1024, k, v - sb + 16):
        assert la.la_decode_step(1, 2, 128, la.LA_BF16, q, k, v, 0x4000, st, out,
                                 0) == la.LA_ERR_ALIAS
        assert la.la_decode_multi(1, 2, 128, 2, la.LA_BF16, q, k, v, 0x4000, st, out,
                                  0) == la.LA_ERR_ALIAS


def test_noalloc_refuses_the_failure_injection_it_cannot_report(lib, monkeypatch):
    monkeypatch.setenv("LA_DEBUG_WITHHOLD_SEGMENT", "0")
    d = _desc()
    assert la.la_prefill_noalloc(d, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0,
                                 0) == la.LA_ERR_UNSUPPORTED


@pytest.mark.parametrize("chunk", [0, 64, 128, 256])
def test_every_supported_chunk_passes_the_host_checks(lib, chunk):
    # the descriptor is valid, so the call gets as far as the pointer checks
    d = _desc(chunk=chunk)
    assert la.la_prefill(d, 0, 0x2000, 0x3000, 0x4000, 0x5000, 0, 0, 0, 0) == la.LA_ERR_NULL
    assert la.la_prefill_workspace_bytes(d) > 0


def test_256_token_chunks_keep_segments_whole(lib):
    # 7 tiles of 128 tokens forced into 3 segments: 3 tiles each with 128-token chunks, but
    # segments of whole 256-token chunks need 4 tiles, so only 2 segments (same ring size, since
    # the ring holds two states per sequence whatever the count)
    w128 = la.la_prefill_workspace_bytes(_desc(B=1, H=1, N=7 * 128, segments=3, chunk=128))
    w256 = la.la_prefill_workspace_bytes(_desc(B=1, H=1, N=7 * 128, segments=3, chunk=256))
    assert w128 == w256 > 256
