"""ctypes binding of the C ABI in include/la.h.

The functions named like the C entry points (``la_prefill``, ``la_decode_step``, ...) take raw
device pointers (ints) and return the status code, exactly like the C calls.  ``prefill`` and
``decode_step`` are the tensor-level conveniences: they only check and marshal torch CUDA tensors
into those calls; every step of the computation runs in the library's CUDA kernels.

There is no fallback: if libla_b200.so has not been built, or the tensors are not on a CUDA
device, these functions raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libla_b200.so")

LA_OK = 0
LA_ERR_NULL = -1
LA_ERR_SHAPE = -2
LA_ERR_DTYPE = -3
LA_ERR_ALIGN = -4
LA_ERR_OVERFLOW = -5
LA_ERR_WORKSPACE = -6
LA_ERR_CUDA = -7
LA_ERR_TIMEOUT = -8
LA_ERR_UNSUPPORTED = -9
LA_ERR_ALIAS = -10

LA_BF16 = 0
LA_F32 = 1

LA_PATH_AUTO = 0
LA_PATH_TENSOR = 1
LA_PATH_RECURRENT = 2
LA_SEGMENTS_BALANCED = -1  # la_desc.segments: the balanced range plan


class la_desc(ctypes.Structure):  # noqa: N801 - mirrors the C type name
    _fields_ = [("B", ctypes.c_int64), ("N", ctypes.c_int64), ("H", ctypes.c_int64),
                ("d", ctypes.c_int64), ("dtype", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("segments", ctypes.c_int32), ("path", ctypes.c_int32)]


class la_varlen_desc(ctypes.Structure):  # noqa: N801 - mirrors the C type name
    _fields_ = [("T", ctypes.c_int64), ("n_seqs", ctypes.c_int64), ("H", ctypes.c_int64),
                ("d", ctypes.c_int64), ("dtype", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("segments", ctypes.c_int32), ("path", ctypes.c_int32)]


class la_gate_norm(ctypes.Structure):  # noqa: N801 - mirrors the C type name
    _fields_ = [("gate", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("eps", ctypes.c_float),
                ("fp8_scales", ctypes.c_void_p)]


class la_qk_norm_rope_desc(ctypes.Structure):  # noqa: N801 - mirrors the C type name
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int64), ("d", ctypes.c_int64),
                ("q_stride", ctypes.c_int64), ("k_stride", ctypes.c_int64),
                ("rotary_dim", ctypes.c_int32), ("theta", ctypes.c_float), ("eps", ctypes.c_float),
                ("pad", ctypes.c_int32)]


class la_qk_prologue(ctypes.Structure):  # noqa: N801 - mirrors the C type name
    _fields_ = [("gamma_q", ctypes.c_void_p), ("gamma_k", ctypes.c_void_p),
                ("positions", ctypes.c_void_p), ("rotary_dim", ctypes.c_int32),
                ("theta", ctypes.c_float), ("eps", ctypes.c_float), ("pad", ctypes.c_int32)]


class LaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {la_status_string(status)} ({status})")


_lock = threading.Lock()
_lib = None

# When True, the tensor conveniences below synchronise the stream after each call and raise on a
# device-side error recorded in the workspace status word (a scan timeout, or a cu_seqlens the
# planning kernel rejected).  Off by default: it costs a stream synchronisation per call.
CHECK_STATUS = False


def _check_device_status(ws_ptr: int, stream_ptr: int, what: str, check) -> None:
    if ws_ptr and (CHECK_STATUS if check is None else check):
        st = la_workspace_status(ws_ptr, stream_ptr)
        if st != LA_OK:
            raise LaError(st, f"{what} (device status)")


def library(path: str | None = None):
    """The loaded libla_b200.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with "
                               "`python -m long_context_attention_la_b200.build`")
        lib = ctypes.CDLL(p)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        lib.la_prefill_workspace_bytes.argtypes = [ctypes.POINTER(la_desc)]
        lib.la_prefill_workspace_bytes.restype = sz
        lib.la_prefill.argtypes = [ctypes.POINTER(la_desc), vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.la_prefill.restype = ctypes.c_int
        lib.la_prefill_noalloc.argtypes = [ctypes.POINTER(la_desc), vp, vp, vp, vp, vp, vp, vp]
        lib.la_prefill_noalloc.restype = ctypes.c_int
        lib.la_prefill_varlen_workspace_bytes.argtypes = [ctypes.POINTER(la_varlen_desc)]
        lib.la_prefill_varlen_workspace_bytes.restype = sz
        lib.la_prefill_varlen.argtypes = [ctypes.POINTER(la_varlen_desc), vp, vp, vp, vp, vp, vp,
                                          ctypes.POINTER(la_gate_norm), vp, vp, vp, sz, vp]
        lib.la_prefill_varlen.restype = ctypes.c_int
        lib.la_prefill_varlen_qk.argtypes = [ctypes.POINTER(la_varlen_desc),
                                             ctypes.POINTER(la_qk_prologue), vp, vp, vp, vp, vp,
                                             vp, vp, vp, vp, sz, vp]
        lib.la_prefill_varlen_qk.restype = ctypes.c_int
        lib.la_qk_norm_rope.argtypes = [ctypes.POINTER(la_qk_norm_rope_desc), vp, vp, vp, vp, vp,
                                        vp, vp, vp]
        lib.la_qk_norm_rope.restype = ctypes.c_int
        lib.la_decode_multi.argtypes = [i64, i64, i64, i64, i32, vp, vp, vp, vp, vp,
                                        ctypes.POINTER(la_gate_norm), vp, vp]
        lib.la_decode_multi.restype = ctypes.c_int
        lib.la_gate_norm_apply.argtypes = [i64, i64, i64, i32, vp, ctypes.POINTER(la_gate_norm),
                                           vp, vp]
        lib.la_gate_norm_apply.restype = ctypes.c_int
        lib.la_prefill_state_workspace_bytes.argtypes = [ctypes.POINTER(la_desc)]
        lib.la_prefill_state_workspace_bytes.restype = sz
        lib.la_prefill_state.argtypes = [ctypes.POINTER(la_desc), vp, vp, vp, vp, vp, vp, sz, vp]
        lib.la_prefill_state.restype = ctypes.c_int
        lib.la_state_fold.argtypes = [i64, i64, i64, i64, vp, ctypes.POINTER(ctypes.c_int64), vp,
                                      vp, vp, vp]
        lib.la_state_fold.restype = ctypes.c_int
        lib.la_decode_step.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp]
        lib.la_decode_step.restype = ctypes.c_int
        lib.la_workspace_status.argtypes = [vp, vp]
        lib.la_workspace_status.restype = ctypes.c_int
        lib.la_status_string.argtypes = [ctypes.c_int]
        lib.la_status_string.restype = ctypes.c_char_p
        lib.la_version.argtypes = []
        lib.la_version.restype = ctypes.c_int
        if path is None:
            _lib = lib
        return lib


# ------------------------------------------------------------------------------------------
# the C entry points, one to one
# ------------------------------------------------------------------------------------------
def la_prefill_workspace_bytes(desc: la_desc) -> int:
    return int(library().la_prefill_workspace_bytes(ctypes.byref(desc)))


def la_prefill(desc: la_desc, q: int, k: int, v: int, slopes: int, out: int, state_out: int,
               workspace: int, workspace_bytes: int, stream: int) -> int:
    return int(library().la_prefill(ctypes.byref(desc), q, k, v, slopes, out, state_out or None,
                                    workspace or None, workspace_bytes, stream or None))


def la_prefill_noalloc(desc: la_desc, q: int, k: int, v: int, slopes: int, out: int,
                       state_out: int, stream: int) -> int:
    """la_prefill on the library's built-in scratch array (no device allocation); see la.h."""
    return int(library().la_prefill_noalloc(ctypes.byref(desc), q, k, v, slopes, out,
                                            state_out or None, stream or None))


LA_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024 + 4096


def la_prefill_varlen_workspace_bytes(desc: la_varlen_desc) -> int:
    return int(library().la_prefill_varlen_workspace_bytes(ctypes.byref(desc)))


def la_prefill_varlen(desc: la_varlen_desc, q: int, k: int, v: int, slopes: int, cu_seqlens: int,
                      state_in: int, out: int, state_out: int, workspace: int,
                      workspace_bytes: int, stream: int,
                      epilogue: la_gate_norm | None = None) -> int:
    """All pointers are device addresses; cu_seqlens is a device int64[n_seqs + 1]; epilogue is
    the optional fused norm + gate (la_gate_norm)."""
    return int(library().la_prefill_varlen(ctypes.byref(desc), q, k, v, slopes, cu_seqlens or None,
                                           state_in or None,
                                           None if epilogue is None else ctypes.byref(epilogue),
                                           out, state_out or None, workspace or None,
                                           workspace_bytes, stream or None))


def la_prefill_varlen_qk(desc: la_varlen_desc, qk: la_qk_prologue | None, q: int, k: int, v: int,
                         slopes: int, cu_seqlens: int, state_in: int, out: int, state_out: int,
                         workspace: int, workspace_bytes: int, stream: int) -> int:
    """la_prefill_varlen with the QK norm + RoPE applied inside the kernel (qk: la_qk_prologue)."""
    return int(library().la_prefill_varlen_qk(ctypes.byref(desc),
                                              None if qk is None else ctypes.byref(qk),
                                              q or None, k or None, v or None, slopes or None,
                                              cu_seqlens or None, state_in or None, out or None,
                                              state_out or None, workspace or None,
                                              workspace_bytes, stream or None))


def la_qk_norm_rope(desc: la_qk_norm_rope_desc, q: int, k: int, gamma_q: int, gamma_k: int,
                    positions: int, q_out: int, k_out: int, stream: int) -> int:
    return int(library().la_qk_norm_rope(ctypes.byref(desc), q or None, k or None,
                                         gamma_q or None, gamma_k or None, positions or None,
                                         q_out or None, k_out or None, stream or None))


def la_decode_step(B: int, H: int, d: int, dtype: int, q: int, k: int, v: int, slopes: int,
                   state_inout: int, out: int, stream: int) -> int:
    return int(library().la_decode_step(B, H, d, dtype, q, k, v, slopes, state_inout, out,
                                        stream or None))


def la_decode_multi(B: int, H: int, d: int, n_tok: int, dtype: int, q: int, k: int, v: int,
                    slopes: int, state_inout: int, out: int, stream: int,
                    epilogue: la_gate_norm | None = None) -> int:
    return int(library().la_decode_multi(B, H, d, n_tok, dtype, q or None, k or None, v or None,
                                         slopes or None, state_inout or None,
                                         None if epilogue is None else ctypes.byref(epilogue),
                                         out or None, stream or None))


def la_gate_norm_apply(T: int, H: int, d: int, dtype: int, o: int, gn: la_gate_norm | None,
                       y: int, stream: int) -> int:
    return int(library().la_gate_norm_apply(T, H, d, dtype, o or None,
                                            None if gn is None else ctypes.byref(gn), y or None,
                                            stream or None))


def la_prefill_state_workspace_bytes(desc: la_desc) -> int:
    return int(library().la_prefill_state_workspace_bytes(ctypes.byref(desc)))


def la_prefill_state(desc: la_desc, k: int, v: int, slopes: int, state_in: int, state_out: int,
                     workspace: int, workspace_bytes: int, stream: int) -> int:
    return int(library().la_prefill_state(ctypes.byref(desc), k or None, v or None,
                                          slopes or None, state_in or None, state_out or None,
                                          workspace or None, workspace_bytes, stream or None))


def la_state_fold(n_parts: int, BH: int, H: int, d: int, parts: int, lengths, slopes: int,
                  state_in: int, state_out: int, stream: int) -> int:
    """lengths: a sequence of n_parts host integers (or None)."""
    arr = None
    if lengths is not None:
        arr = (ctypes.c_int64 * max(1, len(lengths)))(*[int(x) for x in lengths])
    return int(library().la_state_fold(n_parts, BH, H, d, parts or None, arr, slopes or None,
                                       state_in or None, state_out or None, stream or None))


def la_workspace_status(workspace: int, stream: int) -> int:
    return int(library().la_workspace_status(workspace, stream or None))


def la_status_string(status: int) -> str:
    return library().la_status_string(int(status)).decode()


def la_version() -> int:
    return int(library().la_version())


# ------------------------------------------------------------------------------------------
# tensor conveniences (argument marshalling only)
# ------------------------------------------------------------------------------------------
_DT = {torch.bfloat16: LA_BF16, torch.float32: LA_F32}


def _cuda_ptr(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def make_desc(B, N, H, d, dtype, chunk=0, segments=0, path=LA_PATH_AUTO) -> la_desc:
    return la_desc(B, N, H, d, _DT[dtype] if isinstance(dtype, torch.dtype) else int(dtype),
                   chunk, segments, path)


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor, *,
            out: torch.Tensor | None = None, state_out: torch.Tensor | None = None,
            want_state: bool = True, chunk: int = 0, segments: int = 0,
            path: int = LA_PATH_AUTO, workspace: torch.Tensor | None = None,
            stream: torch.cuda.Stream | None = None, check: bool | None = None):
    """o, state = prefill(q, k, v, slopes): q, k, v [B, N, H, d] (bf16 or fp32, CUDA,
    contiguous), slopes float32[H].  Returns out [B, N, H, d] and the final fp32 state
    [B, H, d, d] (None if want_state is False and no state_out is given)."""
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, N, H, d] shape")
    if q.dtype not in _DT or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must all be bfloat16 or all float32")
    B, N, H, d = q.shape
    if slopes.dtype != torch.float32 or slopes.shape != (H,):
        raise ValueError("slopes must be float32[H]")
    if out is None:
        out = torch.empty_like(q)
    if state_out is None and want_state:
        state_out = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    desc = make_desc(B, N, H, d, q.dtype, chunk, segments, path)
    need = la_prefill_workspace_bytes(desc)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = 0 if workspace is None else _cuda_ptr(workspace, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = la_prefill(desc, _cuda_ptr(q, "q"), _cuda_ptr(k, "k"), _cuda_ptr(v, "v"),
                    _cuda_ptr(slopes, "slopes"), _cuda_ptr(out, "out"),
                    0 if state_out is None else _cuda_ptr(state_out, "state_out"), ws_ptr,
                    ws_bytes, s.cuda_stream)
    if st != LA_OK:
        raise LaError(st, "la_prefill")
    _check_device_status(ws_ptr, s.cuda_stream, "la_prefill", check)
    return out, state_out


def _varlen_operands(q, k, v, slopes, cu_seqlens, state_in, out, state_out, want_state):
    """Checks of the packed operands; returns cu_seqlens on the device, out and state_out."""
    if q.dim() != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [T, H, d] shape")
    if q.dtype not in _DT or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must all be bfloat16 or all float32")
    if not (isinstance(cu_seqlens, torch.Tensor) and cu_seqlens.is_cuda):
        cu_seqlens = torch.as_tensor(cu_seqlens, dtype=torch.int64).to(q.device)
    if cu_seqlens.dtype != torch.int64 or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be int64 [n_seqs + 1]")
    T, H, d = q.shape
    n = cu_seqlens.numel() - 1
    if n < 1:
        raise ValueError("cu_seqlens needs at least two entries")
    if slopes.dtype != torch.float32 or slopes.shape != (H,):
        raise ValueError("slopes must be float32[H]")
    if state_in is not None and (state_in.dtype != torch.float32 or
                                 tuple(state_in.shape) != (n, H, d, d)):
        raise ValueError("state_in must be float32 [n_seqs, H, d, d]")
    if out is None:
        out = torch.empty_like(q)
    if state_out is None and want_state:
        state_out = torch.empty((n, H, d, d), dtype=torch.float32, device=q.device)
    return cu_seqlens, out, state_out


def prefill_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor,
                   cu_seqlens, *, state_in: torch.Tensor | None = None,
                   gate: torch.Tensor | None = None, gamma: torch.Tensor | None = None,
                   eps: float = 1e-6,
                   out: torch.Tensor | None = None, state_out: torch.Tensor | None = None,
                   want_state: bool = True, chunk: int = 0, segments: int = 0,
                   path: int = LA_PATH_AUTO, workspace: torch.Tensor | None = None,
                   stream: torch.cuda.Stream | None = None, check: bool | None = None):
    """o, state = prefill_varlen(q, k, v, slopes, cu_seqlens): q, k, v [T, H, d] hold n_seqs
    sequences back to back, sequence s at tokens [cu_seqlens[s], cu_seqlens[s+1]).  cu_seqlens is
    a CUDA int64 tensor of n_seqs + 1 entries (a host list or array is copied to the device
    first).  state_in: optional fp32 [n_seqs, H, d, d] initial states (state_out may be the same
    tensor).  gate [T, H, d] bf16 and gamma fp32 [H, d] switch on the fused grouped RMSNorm +
    sigmoid gate, so out holds gamma * o / rms(o) * sigmoid(gate) per head (FP8 output is
    gate_norm's, the stand-alone operator).
    Returns out [T, H, d] and the final fp32 states [n_seqs, H, d, d].  An invalid
    cu_seqlens is reported by the device: check la_workspace_status(workspace) when it is not
    known to be valid."""
    cu_seqlens, out, state_out = _varlen_operands(q, k, v, slopes, cu_seqlens, state_in, out,
                                                  state_out, want_state)
    T, H, d = q.shape
    n = cu_seqlens.numel() - 1
    epi = None
    if gate is not None or gamma is not None:
        if gate is None or gamma is None:
            raise ValueError("the fused norm + gate needs both gate and gamma")
        if gate.shape != q.shape or gate.dtype != q.dtype:
            raise ValueError("gate must match q's [T, H, d] shape and dtype")
        if gamma.dtype != torch.float32 or tuple(gamma.shape) != (H, d):
            raise ValueError("gamma must be float32 [H, d]")
        epi = la_gate_norm(_cuda_ptr(gate, "gate"), _cuda_ptr(gamma, "gamma"), float(eps))
    desc = la_varlen_desc(T, n, H, d, _DT[q.dtype], chunk, segments, path)
    need = la_prefill_varlen_workspace_bytes(desc)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = 0 if workspace is None else _cuda_ptr(workspace, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = la_prefill_varlen(desc, _cuda_ptr(q, "q"), _cuda_ptr(k, "k"), _cuda_ptr(v, "v"),
                           _cuda_ptr(slopes, "slopes"), _cuda_ptr(cu_seqlens, "cu_seqlens"),
                           0 if state_in is None else _cuda_ptr(state_in, "state_in"),
                           _cuda_ptr(out, "out"),
                           0 if state_out is None else _cuda_ptr(state_out, "state_out"),
                           ws_ptr, ws_bytes, s.cuda_stream, epi)
    if st != LA_OK:
        raise LaError(st, "la_prefill_varlen")
    _check_device_status(ws_ptr, s.cuda_stream, "la_prefill_varlen", check)
    return out, state_out


def prefill_varlen_qk(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor,
                      cu_seqlens, gamma_q: torch.Tensor, gamma_k: torch.Tensor,
                      positions: torch.Tensor, *, rotary_dim: int = 64, theta: float = 6.0e6,
                      eps: float = 1e-6, state_in: torch.Tensor | None = None,
                      out: torch.Tensor | None = None, state_out: torch.Tensor | None = None,
                      want_state: bool = True, segments: int = 0,
                      workspace: torch.Tensor | None = None,
                      stream: torch.cuda.Stream | None = None, check: bool | None = None):
    """o, state = prefill_varlen_qk(q, k, v, slopes, cu_seqlens, gamma_q, gamma_k, positions):
    prefill_varlen of the raw q and k projections, with qk_norm_rope (gamma_* fp32 [d],
    positions int64 [T], rotary_dim, theta, eps) applied inside the kernel to each tile before
    use.  bf16, d = 128, tensor-core path, 128-token chunks.  Equals qk_norm_rope followed by
    prefill_varlen exactly."""
    cu_seqlens, out, state_out = _varlen_operands(q, k, v, slopes, cu_seqlens, state_in, out,
                                                  state_out, want_state)
    T, H, d = q.shape
    n = cu_seqlens.numel() - 1
    if positions.dtype != torch.int64 or tuple(positions.shape) != (T,):
        raise ValueError("positions must be int64 [T]")
    for name, g in (("gamma_q", gamma_q), ("gamma_k", gamma_k)):
        if g.dtype != torch.float32 or tuple(g.shape) != (d,):
            raise ValueError(f"{name} must be float32 [d]")
    qk = la_qk_prologue(_cuda_ptr(gamma_q, "gamma_q"), _cuda_ptr(gamma_k, "gamma_k"),
                        _cuda_ptr(positions, "positions"), rotary_dim, theta, eps, 0)
    desc = la_varlen_desc(T, n, H, d, _DT[q.dtype], 0, segments, LA_PATH_AUTO)
    need = la_prefill_varlen_workspace_bytes(desc)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = 0 if workspace is None else _cuda_ptr(workspace, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = la_prefill_varlen_qk(desc, qk, _cuda_ptr(q, "q"), _cuda_ptr(k, "k"), _cuda_ptr(v, "v"),
                              _cuda_ptr(slopes, "slopes"), _cuda_ptr(cu_seqlens, "cu_seqlens"),
                              0 if state_in is None else _cuda_ptr(state_in, "state_in"),
                              _cuda_ptr(out, "out"),
                              0 if state_out is None else _cuda_ptr(state_out, "state_out"),
                              ws_ptr, ws_bytes, s.cuda_stream)
    if st != LA_OK:
        raise LaError(st, "la_prefill_varlen_qk")
    _check_device_status(ws_ptr, s.cuda_stream, "la_prefill_varlen_qk", check)
    return out, state_out


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor,
                state: torch.Tensor, *, out: torch.Tensor | None = None,
                stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """o = decode_step(q, k, v, slopes, state): q, k, v [B, H, d]; state fp32 [B, H, d, d] is
    updated in place (decay, add k^T v, read out)."""
    if q.dim() != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, H, d] shape")
    if q.dtype not in _DT or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must all be bfloat16 or all float32")
    B, H, d = q.shape
    if state.dtype != torch.float32 or tuple(state.shape) != (B, H, d, d):
        raise ValueError("state must be float32 [B, H, d, d]")
    if out is None:
        out = torch.empty_like(q)
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = la_decode_step(B, H, d, _DT[q.dtype], _cuda_ptr(q, "q"), _cuda_ptr(k, "k"),
                        _cuda_ptr(v, "v"), _cuda_ptr(slopes, "slopes"),
                        _cuda_ptr(state, "state"), _cuda_ptr(out, "out"), s.cuda_stream)
    if st != LA_OK:
        raise LaError(st, "la_decode_step")
    return out


def qk_norm_rope(q: torch.Tensor, k: torch.Tensor, gamma_q: torch.Tensor, gamma_k: torch.Tensor,
                 positions: torch.Tensor, *, rotary_dim: int = 64, theta: float = 6.0e6,
                 eps: float = 1e-6, q_out: torch.Tensor | None = None,
                 k_out: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None):
    """q_hat, k_hat = qk_norm_rope(q, k, gamma_q, gamma_k, positions): q, k [T, H, d] bf16 CUDA
    views whose head and channel dims are contiguous (the token stride may be larger, e.g. views
    into one fused projection output); gamma_* fp32 [d]; positions int64 [T].  Returns new
    contiguous [T, H, d] tensors (or writes q_out / k_out)."""
    if q.dim() != 3 or q.shape != k.shape or q.dtype != torch.bfloat16 or k.dtype != q.dtype:
        raise ValueError("q, k must be bf16 [T, H, d] of one shape")
    T, H, d = q.shape
    for name, t in (("q", q), ("k", k)):
        if not t.is_cuda or t.stride(2) != 1 or t.stride(1) != d:
            raise ValueError(f"{name} must be a CUDA view with contiguous [H, d] rows")
    if positions.dtype != torch.int64 or tuple(positions.shape) != (T,):
        raise ValueError("positions must be int64 [T]")
    for name, g in (("gamma_q", gamma_q), ("gamma_k", gamma_k)):
        if g.dtype != torch.float32 or tuple(g.shape) != (d,):
            raise ValueError(f"{name} must be float32 [d]")
    if q_out is None:
        q_out = torch.empty((T, H, d), dtype=q.dtype, device=q.device)
    if k_out is None:
        k_out = torch.empty((T, H, d), dtype=q.dtype, device=q.device)
    desc = la_qk_norm_rope_desc(T, H, d, q.stride(0), k.stride(0), rotary_dim, theta, eps, 0)
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = la_qk_norm_rope(desc, q.data_ptr(), k.data_ptr(), _cuda_ptr(gamma_q, "gamma_q"),
                         _cuda_ptr(gamma_k, "gamma_k"), _cuda_ptr(positions, "positions"),
                         _cuda_ptr(q_out, "q_out"), _cuda_ptr(k_out, "k_out"), s.cuda_stream)
    if st != LA_OK:
        raise LaError(st, "la_qk_norm_rope")
    return q_out, k_out


def decode_multi(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor,
                 state: torch.Tensor, *, gate: torch.Tensor | None = None,
                 gamma: torch.Tensor | None = None, eps: float = 1e-6,
                 out: torch.Tensor | None = None,
                 stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """o = decode_multi(q, k, v, slopes, state): q, k, v [B, n, H, d]; state fp32 [B, H, d, d]
    takes all n tokens in order, in place.  gate [B, n, H, d] and gamma fp32 [H, d] switch on
    the fused grouped RMSNorm + sigmoid gate of each output row."""
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, n, H, d] shape")
    if q.dtype not in _DT or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must all be bfloat16 or all float32")
    B, n, H, d = q.shape
    if state.dtype != torch.float32 or tuple(state.shape) != (B, H, d, d):
        raise ValueError("state must be float32 [B, H, d, d]")
    epi = None
    if gate is not None or gamma is not None:
        if gate is None or gamma is None or gate.shape != q.shape or gate.dtype != q.dtype:
            raise ValueError("the fused norm + gate needs gate (like q) and gamma")
        if gamma.dtype != torch.float32 or tuple(gamma.shape) != (H, d):
            raise ValueError("gamma must be float32 [H, d]")
        epi = la_gate_norm(_cuda_ptr(gate, "gate"), _cuda_ptr(gamma, "gamma"), float(eps))
    if out is None:
        out = torch.empty_like(q)
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = la_decode_multi(B, H, d, n, _DT[q.dtype], _cuda_ptr(q, "q"), _cuda_ptr(k, "k"),
                         _cuda_ptr(v, "v"), _cuda_ptr(slopes, "slopes"), _cuda_ptr(state, "state"),
                         _cuda_ptr(out, "out"), s.cuda_stream, epi)
    if st != LA_OK:
        raise LaError(st, "la_decode_multi")
    return out


def gate_norm(o: torch.Tensor, gate: torch.Tensor, gamma: torch.Tensor, *, eps: float = 1e-6,
              fp8: bool = False, out: torch.Tensor | None = None,
              stream: torch.cuda.Stream | None = None):
    """y = gate_norm(o, gate, gamma): o, gate [T, H, d] (bf16 or fp32, CUDA, contiguous), gamma
    fp32 [H, d]; y = gamma * o / rms(o) * sigmoid(gate) per token and head (out may be o).
    fp8=True returns (codes, scales): y as FP8 E4M3 codes (uint8 [T, H, d]) and one fp32 scale
    per (head, token) block, [H, T]."""
    if o.dim() != 3 or gate.shape != o.shape or gate.dtype != o.dtype or o.dtype not in _DT:
        raise ValueError("o and gate must share one [T, H, d] shape and dtype")
    T, H, d = o.shape
    if gamma.dtype != torch.float32 or tuple(gamma.shape) != (H, d):
        raise ValueError("gamma must be float32 [H, d]")
    if out is None:
        out = torch.empty(o.shape, dtype=torch.uint8, device=o.device) if fp8 else \
            torch.empty_like(o)
    scales = torch.empty((H, T), dtype=torch.float32, device=o.device) if fp8 else None
    s = stream if stream is not None else torch.cuda.current_stream(o.device)
    gn = la_gate_norm(_cuda_ptr(gate, "gate"), _cuda_ptr(gamma, "gamma"), float(eps),
                      _cuda_ptr(scales, "scales") if fp8 else None)
    st = la_gate_norm_apply(T, H, d, _DT[o.dtype], _cuda_ptr(o, "o"), gn, _cuda_ptr(out, "out"),
                            s.cuda_stream)
    if st != LA_OK:
        raise LaError(st, "la_gate_norm_apply")
    return (out, scales) if fp8 else out


def prefill_state(k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor, *,
                  state_in: torch.Tensor | None = None, state_out: torch.Tensor | None = None,
                  path: int = LA_PATH_AUTO, workspace: torch.Tensor | None = None,
                  stream: torch.cuda.Stream | None = None,
                  check: bool | None = None) -> torch.Tensor:
    """state = prefill_state(k, v, slopes): the final fp32 state [B, H, d, d] of a prefill of
    k, v [B, N, H, d] (bf16 or fp32, CUDA, contiguous) from state_in (or zero), without outputs:
    lambda^N state_in + sum_t lambda^(N-1-t) k_t^T v_t.  state_out may be state_in."""
    if k.dim() != 4 or k.shape != v.shape or k.dtype != v.dtype or k.dtype not in _DT:
        raise ValueError("k, v must share one [B, N, H, d] shape and dtype")
    B, N, H, d = k.shape
    if slopes.dtype != torch.float32 or slopes.shape != (H,):
        raise ValueError("slopes must be float32[H]")
    if state_in is not None and (state_in.dtype != torch.float32 or
                                 tuple(state_in.shape) != (B, H, d, d)):
        raise ValueError("state_in must be float32 [B, H, d, d]")
    if state_out is None:
        state_out = torch.empty((B, H, d, d), dtype=torch.float32, device=k.device)
    desc = make_desc(B, N, H, d, k.dtype, 0, 0, path)
    need = la_prefill_state_workspace_bytes(desc)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
    ws_ptr = 0 if workspace is None else _cuda_ptr(workspace, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    s = stream if stream is not None else torch.cuda.current_stream(k.device)
    st = la_prefill_state(desc, _cuda_ptr(k, "k"), _cuda_ptr(v, "v"), _cuda_ptr(slopes, "slopes"),
                          0 if state_in is None else _cuda_ptr(state_in, "state_in"),
                          _cuda_ptr(state_out, "state_out"), ws_ptr, ws_bytes, s.cuda_stream)
    if st != LA_OK:
        raise LaError(st, "la_prefill_state")
    _check_device_status(ws_ptr, s.cuda_stream, "la_prefill_state", check)
    return state_out


def state_fold(parts: torch.Tensor, lengths, slopes: torch.Tensor, *,
               state_in: torch.Tensor | None = None, out: torch.Tensor | None = None,
               stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """S = state_fold(parts, lengths, slopes): parts fp32 [n, B, H, d, d] (the local states of n
    consecutive parts of lengths[j] tokens); returns the state after all n parts, starting from
    state_in (fp32 [B, H, d, d], or zero): S <- lambda^lengths[j] S + parts[j] in order."""
    if parts.dim() != 5 or parts.dtype != torch.float32:
        raise ValueError("parts must be float32 [n_parts, B, H, d, d]")
    n, B, H, d, _ = parts.shape
    lengths = [int(x) for x in lengths]
    if len(lengths) != n:
        raise ValueError("lengths must have one entry per part")
    if slopes.dtype != torch.float32 or slopes.shape != (H,):
        raise ValueError("slopes must be float32[H]")
    if state_in is not None and (state_in.dtype != torch.float32 or
                                 tuple(state_in.shape) != (B, H, d, d)):
        raise ValueError("state_in must be float32 [B, H, d, d]")
    if out is None:
        out = torch.empty((B, H, d, d), dtype=torch.float32, device=parts.device)
    s = stream if stream is not None else torch.cuda.current_stream(parts.device)
    st = la_state_fold(n, B * H, H, d, _cuda_ptr(parts, "parts") if n > 0 else 0, lengths,
                       _cuda_ptr(slopes, "slopes"),
                       0 if state_in is None else _cuda_ptr(state_in, "state_in"),
                       _cuda_ptr(out, "out"), s.cuda_stream)
    if st != LA_OK:
        raise LaError(st, "la_state_fold")
    return out
