"""fp64 CPU oracle of the Lightning Attention layer kernel — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
package.  The product path (``long_context_attention_la_b200``) never imports it, and this package
imports nothing from the product: the two share no code.

The arithmetic lives in ``la_oracle.c`` (plain C, fp64, OpenMP over heads).  This module only
compiles it (``build()``) and marshals numpy arrays through ``ctypes``.

Source of the method: "Ling and Ring 2.6 Technical Report" (Chinese translation,
garden.houmin.site), §4.1.1 (linear attention as an RNN-style recurrence with a [B,H,D,D] state)
and §2.1 Fig. 2 (kernel placement, no normaliser inside); the decayed recurrence
``S_t = lambda S_{t-1} + k_t^T v_t, o_t = q_t S_t`` is Lightning Attention's (the report's
reference 7), which the pages name without printing it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libla_oracle.so")
_lock = threading.Lock()
_lib = None

BF16 = 0
F32 = 1


def build(force: bool = False) -> str:
    """Compile la_oracle.c into oracle/_build/libla_oracle.so (gcc, -O2, no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    return compile_source(_SRC, _LIB_PATH)


def open_library(path: str):
    """ctypes handle of a compiled oracle library with its signatures declared."""
    lib = ctypes.CDLL(path)
    i64, p, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.la_oracle_prefill.argtypes = [i64, i64, i64, i64, i32, p, p, p, p, p, i64, p, i64,
                                      p, p, p, i32]
    lib.la_oracle_prefill.restype = i32
    lib.la_oracle_decode.argtypes = [i64, i64, i64, i32, p, p, p, p, p, p, i32]
    lib.la_oracle_decode.restype = i32
    lib.orc_num_threads.argtypes = [i32]
    lib.orc_num_threads.restype = i32
    return lib


def compile_source(src: str, out_path: str) -> str:
    """Compile an oracle C source with the oracle's own flags (used by build() and by the tests
    that check the pins reject deliberately broken copies of the source)."""
    tmp = out_path + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
           "-std=c11", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out_path)
    return out_path


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = open_library(build())
    return _lib


def num_threads(requested: int = 0) -> int:
    """OpenMP threads the oracle uses for a call with ``nthreads=requested``."""
    return int(_load().orc_num_threads(int(requested)))


def _dtype_code(a: np.ndarray) -> int:
    # bf16 tensors are passed as their raw uint16 bit patterns.
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle inputs must be uint16 (bf16 bits) or float32, got {a.dtype}")


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def prefill(q, k, v, slopes, heads=None, t_sel=None, state_in=None, nthreads: int = 0, lib=None):
    """Run the fp64 recurrence.

    q, k, v: [B, N, H, d] arrays, uint16 (bf16 bits) or float32, C-contiguous.
    slopes: float32[H] (decay lambda_h = exp(-slope_h)).
    heads: optional int64 list of flat head indices b*H+h to evaluate (default: all, in order).
    t_sel: optional sorted int64 list of token indices whose outputs to record (default: all).
    state_in: optional float64 [n_heads, d, d] initial state (default zero).
    lib: optional handle from open_library() (default: the built oracle).
    Returns (o, state): o float64 [n_heads, n_t, d], state float64 [n_heads, d, d].
    """
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    if not (q.shape == k.shape == v.shape) or q.ndim != 4:
        raise ValueError("q, k, v must share one [B, N, H, d] shape")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    B, N, H, d = q.shape
    slopes = np.ascontiguousarray(slopes, dtype=np.float32)
    if slopes.shape != (H,):
        raise ValueError("slopes must be float32[H]")
    heads_a = None if heads is None else np.ascontiguousarray(heads, dtype=np.int64)
    n_sel = B * H if heads_a is None else int(heads_a.size)
    t_a = None if t_sel is None else np.ascontiguousarray(t_sel, dtype=np.int64)
    if t_a is not None and (np.any(np.diff(t_a) <= 0) or (t_a.size and (t_a[0] < 0 or t_a[-1] >= N))):
        raise ValueError("t_sel must be strictly increasing token indices in [0, N)")
    n_t = N if t_a is None else int(t_a.size)
    o = np.zeros((n_sel, n_t, d), dtype=np.float64)
    state = np.zeros((n_sel, d, d), dtype=np.float64)
    sin = None
    if state_in is not None:
        sin = np.ascontiguousarray(state_in, dtype=np.float64)
        if sin.shape != (n_sel, d, d):
            raise ValueError("state_in must be float64 [n_heads, d, d]")
    rc = (lib or _load()).la_oracle_prefill(B, N, H, d, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(slopes), _ptr(heads_a), 0 if heads_a is None else n_sel,
                                   _ptr(t_a), n_t, _ptr(o), _ptr(state), _ptr(sin), int(nthreads))
    if rc != 0:
        raise RuntimeError("la_oracle_prefill rejected its arguments")
    return o, state


def decode(q, k, v, slopes, state, nthreads: int = 0):
    """One decode step.  q, k, v: [B, H, d] (uint16 bf16 bits or float32); state: float64
    [B, H, d, d], updated IN PLACE.  Returns o float64 [B, H, d]."""
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    if not (q.shape == k.shape == v.shape) or q.ndim != 3:
        raise ValueError("q, k, v must share one [B, H, d] shape")
    B, H, d = q.shape
    if state.dtype != np.float64 or state.shape != (B, H, d, d) or not state.flags.c_contiguous:
        raise ValueError("state must be a C-contiguous float64 [B, H, d, d] array")
    slopes = np.ascontiguousarray(slopes, dtype=np.float32)
    o = np.zeros((B, H, d), dtype=np.float64)
    rc = _load().la_oracle_decode(B, H, d, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(slopes), _ptr(state), _ptr(o), int(nthreads))
    if rc != 0:
        raise RuntimeError("la_oracle_decode rejected its arguments")
    return o


def _upcast(x) -> np.ndarray:
    """Exact fp64 values of bf16 bit patterns (uint16) or float32 arrays."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def gated_rmsnorm(o, gate, gamma, eps: float):
    """The layer's step after the kernel, in fp64: a grouped RMSNorm of each head's output vector
    followed by the sigmoid gate ("Ling and Ring 2.6 Technical Report", §2.1 Fig. 2: Linear
    Attention Kernel -> Grouped RMSNorm, multiplied by sigmoid(Gate Projection); §4.3: the group
    norm and sigmoid gate run as one fused operator).  Each head is one group:

        y[..., j] = gamma[h, j] * o[..., j] / sqrt(mean_j(o[..., j]^2) + eps) * sigmoid(g[..., j])

    o: fp64 [..., H, d] attention outputs (token-major, heads on the second-to-last axis);
    gate: the gate pre-activation g = x W_gate with o's shape (uint16 bf16 bits or float32);
    gamma: float32 [H, d]; eps: the RMSNorm epsilon.  Returns fp64 y with o's shape.
    """
    o = np.asarray(o, dtype=np.float64)
    g = _upcast(gate)
    gam = np.asarray(gamma, dtype=np.float32).astype(np.float64)
    if g.shape != o.shape or gam.shape != o.shape[-2:]:
        raise ValueError("gate must match o, gamma must be [H, d]")
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return gam * (o / np.sqrt(ms + float(eps))) * (1.0 / (1.0 + np.exp(-g)))


E4M3_MAX = 448.0  # largest finite FP8 E4M3 value: 2^8 x 1.75


def e4m3_encode(x) -> np.ndarray:
    """FP8 E4M3 codes of real values, rounded to nearest with ties to even and saturated to the
    largest finite value (the 8-bit format of the report's FP8 inference path, "Ling and Ring
    2.6 Technical Report" §4.3 and Table 7: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
    bits; exponent field 0 holds the subnormals m * 2^-9; no infinities; 0x7F / 0xFF are NaN, so
    the largest finite magnitude is 0x7E = 448).  x: any real array; returns uint8 codes."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.uint8) << 7
    a = np.minimum(np.abs(x), E4M3_MAX)  # saturate: nothing rounds past 448
    frac, ex = np.frexp(a)  # a = frac * 2^ex, frac in [0.5, 1)
    e = ex.astype(np.int64) - 1  # a = s * 2^e with s in [1, 2)
    normal = a >= 2.0 ** -6
    # normal: 3 mantissa bits of s - 1, a carry into the exponent when they round up to 8
    mant_n = np.rint((2.0 * frac - 1.0) * 8.0).astype(np.int64)
    e_n = e + (mant_n == 8)
    mant_n = np.where(mant_n == 8, 0, mant_n)
    code_n = ((e_n + 7) << 3) | mant_n
    # subnormal: m * 2^-9; m = 8 is the smallest normal 2^-6, whose code is 8 as well
    code_s = np.rint(a / 2.0 ** -9).astype(np.int64)
    code = np.where(normal, code_n, code_s).astype(np.uint8)
    return code | sign


def e4m3_decode(code) -> np.ndarray:
    """Real values (fp64) of FP8 E4M3 codes (NaN for 0x7F / 0xFF); the inverse of e4m3_encode on
    the representable values."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    sgn = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(ef == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(ef - 7.0))
    mag = np.where((ef == 15) & (m == 7), np.nan, mag)
    return sgn * mag


def gated_rmsnorm_fp8(o, gate, gamma, eps: float):
    """The fused post-kernel operator with its quantize step, in fp64 ("Ling and Ring 2.6
    Technical Report" §4.3: "group norm + sigmoid gate + quantize" fused before out_proj; the FP8
    path quantizes the projection inputs blockwise, §4.3 and Table 7).  y is gated_rmsnorm's;
    each head's d channels of one token are one block with one scale:

        amax = max_j |y_j|,  scale = amax / 448,  code_j = E4M3(y_j * 448 / amax)

    (code 0 and scale 0 for an all-zero block), so code_j * scale reproduces y_j to within half an
    E4M3 step.  This is the exact-arithmetic definition; the kernels quantize y after rounding it
    to the I/O dtype, and their tests take the reference codes in that same precision.  Returns
    (uint8 codes with o's shape, fp64 scales [..., H])."""
    y = gated_rmsnorm(o, gate, gamma, eps)
    amax = np.max(np.abs(y), axis=-1)
    inv = np.where(amax > 0, E4M3_MAX / np.where(amax > 0, amax, 1.0), 0.0)
    codes = e4m3_encode(y * inv[..., None])
    return codes, amax / E4M3_MAX


def qk_norm_rope(x, gamma, positions, rotary_dim: int, theta: float, eps: float):
    """The layer's step before the kernel, in fp64 ("Ling and Ring 2.6 Technical Report", §2.1
    Fig. 2: QKV Projection -> QK Norm -> RoPE -> Linear Attention Kernel; §2.1.1: RMSNorm with
    eps = 1e-6, partial RoPE over 64 of the 128 head dims with theta = 6,000,000; §4.3: split + QK
    norm + RoPE run as one fused operator).  Per token t and head h:

        y = gamma * x / sqrt(mean(x^2) + eps)                        (RMSNorm over d)
        for i < r/2, w_i = theta^(-2i/r), a = positions[t] * w_i:   (rotate-half pairs)
            (y_i, y_{i+r/2}) <- (y_i cos a - y_{i+r/2} sin a, y_{i+r/2} cos a + y_i sin a)

    dims >= r pass through normalised only.  x: [T, H, d] (uint16 bf16 bits or float32);
    gamma: float32 [d] (shared by the heads); positions: int [T]; returns fp64 [T, H, d].
    """
    x = _upcast(x)
    T, H, d = x.shape
    r = int(rotary_dim)
    if r % 2 or r > d or r <= 0:
        raise ValueError("rotary_dim must be even and in (0, d]")
    gam = np.asarray(gamma, dtype=np.float32).astype(np.float64)
    pos = np.asarray(positions, dtype=np.int64).astype(np.float64)
    if gam.shape != (d,) or pos.shape != (T,):
        raise ValueError("gamma must be [d] and positions [T]")
    y = gam * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + float(eps))
    half = r // 2
    w = float(theta) ** (-2.0 * np.arange(half, dtype=np.float64) / r)
    ang = pos[:, None] * w[None, :]                      # [T, r/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a = y[..., :half].copy()
    b = y[..., half:r].copy()
    y[..., :half] = a * c - b * s
    y[..., half:r] = b * c + a * s
    return y


def fold_states(parts, lengths, slopes, state_in=None):
    """The report's "fused update h" in fp64 ("Ling and Ring 2.6 Technical Report", §4.1.1
    Context Parallel for Lightning Attention, Fig. 10: local h of every part -> AllGather ->
    update h): the state after consecutive parts j = 0 .. n-1 of a sequence, part j holding
    lengths[j] tokens and having local state h_j (its state when started from zero):

        S = state_in (or 0);   for j in order:  S <- lambda^lengths[j] * S + h_j

    with lambda_h = exp(-slope_h) per head.  parts: [n, B, H, d, d] (any real dtype); lengths:
    n non-negative integers; slopes: float32[H]; state_in: [B, H, d, d] or None.  Returns fp64
    [B, H, d, d].
    """
    parts = np.asarray(parts, dtype=np.float64)
    if parts.ndim != 5:
        raise ValueError("parts must be [n, B, H, d, d]")
    n, B, H, d, _ = parts.shape
    lengths = [int(x) for x in lengths]
    if len(lengths) != n or any(x < 0 for x in lengths):
        raise ValueError("lengths must be n non-negative integers")
    sl = np.asarray(slopes, dtype=np.float32).astype(np.float64)
    if sl.shape != (H,):
        raise ValueError("slopes must be float32[H]")
    S = np.zeros((B, H, d, d)) if state_in is None else np.array(state_in, dtype=np.float64)
    for j in range(n):
        lam_l = np.exp(-sl * lengths[j])[None, :, None, None]
        S = lam_l * S + parts[j]
    return S
