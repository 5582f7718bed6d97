"""Test helpers: tensor <-> oracle marshalling and the error metrics of the parity bar."""
import numpy as np
import torch


def oracle_bits(t: torch.Tensor) -> np.ndarray:
    """Exact stored bits of a bf16 / fp32 tensor as the numpy array the oracle takes
    (uint16 bit patterns for bf16, float32 for fp32)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    if den == 0.0:
        return float(num)
    return float(num / den)


def max_abs(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


# Parity bar: bf16 I/O with fp32 accumulation: relL2 <= 1e-2 and maxabs <= 2e-2 * max|ref|;
# fp32 I/O: relL2 <= 1e-5.  Applied to o and to the final state.
BF16_REL_L2 = 1e-2
BF16_MAX_ABS_FRAC = 2e-2
F32_REL_L2 = 1e-5


def check_close(x, ref, dtype, what=""):
    r = rel_l2(x, ref)
    if dtype == torch.float32:
        assert r <= F32_REL_L2, f"{what}: relL2 {r:.3e} > {F32_REL_L2}"
        return r, max_abs(x, ref)
    m = max_abs(x, ref)
    scale = float(np.max(np.abs(np.asarray(ref, dtype=np.float64)))) if np.size(ref) else 0.0
    assert r <= BF16_REL_L2, f"{what}: relL2 {r:.3e} > {BF16_REL_L2}"
    assert m <= BF16_MAX_ABS_FRAC * scale + 1e-30, f"{what}: maxabs {m:.3e} > 2e-2*{scale:.3e}"
    return r, m


class ParityAccumulator:
    """The same bar as check_close, for a tensor compared in pieces (for example a few heads at a
    time against the oracle): relL2 is accumulated as sums of squares over the whole tensor,
    maxabs and max|ref| as maxima.  ``worst`` keeps the largest per-piece relL2 as a diagnostic.
    """

    def __init__(self, dtype, what=""):
        self.dtype = dtype
        self.what = what
        self.num = 0.0
        self.den = 0.0
        self.maxabs = 0.0
        self.scale = 0.0
        self.worst = (0.0, None)
        self.pieces = 0

    def add(self, x, ref, tag=None):
        x = np.asarray(x, dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        if x.shape != ref.shape:
            raise ValueError(f"{self.what}: shape {x.shape} != {ref.shape}")
        diff = x - ref
        n = float(np.sum(diff * diff))
        d = float(np.sum(ref * ref))
        self.num += n
        self.den += d
        if x.size:
            self.maxabs = max(self.maxabs, float(np.max(np.abs(diff))))
            self.scale = max(self.scale, float(np.max(np.abs(ref))))
        r = (n / d) ** 0.5 if d > 0 else n ** 0.5
        if r >= self.worst[0]:
            self.worst = (r, tag)
        self.pieces += 1

    def rel_l2(self) -> float:
        return (self.num / self.den) ** 0.5 if self.den > 0 else self.num ** 0.5

    def check(self):
        r = self.rel_l2()
        if self.dtype == torch.float32:
            assert r <= F32_REL_L2, f"{self.what}: relL2 {r:.3e} > {F32_REL_L2}"
        else:
            assert r <= BF16_REL_L2, f"{self.what}: relL2 {r:.3e} > {BF16_REL_L2}"
            assert self.maxabs <= BF16_MAX_ABS_FRAC * self.scale + 1e-30, \
                f"{self.what}: maxabs {self.maxabs:.3e} > 2e-2*{self.scale:.3e}"
        print(f"{self.what}: relL2 {r:.3e}, maxabs {self.maxabs:.3e} (max|ref| {self.scale:.3e}), "
              f"worst piece {self.worst[0]:.3e} at {self.worst[1]}, {self.pieces} pieces")
        return r, self.maxabs


def _e4m3_ordinal(codes: np.ndarray) -> np.ndarray:
    """Monotone integer position of E4M3 codes on the real line (+-0 both at 0)."""
    c = np.asarray(codes, dtype=np.int64)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def check_fp8(codes, scales_ht, y_ref, what="", io_dtype=torch.bfloat16):
    """The bar for FP8 E4M3 output (codes uint8 [T, H, d], scales fp32 [H, T]) against the fp64 y
    of the oracle.  The quantize step is a rounding decision, so the reference codes are taken
    in the kernel's precision: y rounded to fp32 and then to the I/O dtype (the value the
    kernels quantize), amax of those values, the fp32 product y * (448 / amax) rounded to E4M3
    (oracle.e4m3_encode).  Codes may still differ where the
    kernel's y sits on the other side of a rounding boundary than the oracle's, by at most one
    E4M3 step, so:
      * every block scale within 1e-2 plus one ulp of the I/O dtype of the reference scale
        (relative; amax is one of the rounded values, and a small difference in y can move it to
        the neighbouring one), zero blocks exact;
      * every code within one step of the reference code where the reference value has
        magnitude >= 32 (in units of amax / 448), and no more than 15 % of those codes off by
        that step.  At the bf16 bar the kernel's y differs from the oracle's by about 3e-3 of
        its RMS, which is ~0.5 such units (a few units at the extremes of 10^6 values); from 32
        up an E4M3 step is 4 units or more, so the difference can cross at most one rounding
        boundary.  Below 32 the steps are finer than that difference, and the next check covers
        those values;
      * dequantized values (code value * scale) as close to y as the reference codes are, in
        relL2, to within the bf16 bar 1e-2."""
    import oracle
    y_ref = np.asarray(y_ref, dtype=np.float64)
    codes = np.asarray(codes, dtype=np.uint8)
    s = np.asarray(scales_ht, dtype=np.float64).T  # [T, H]
    y32 = torch.from_numpy(y_ref.astype(np.float32)).to(io_dtype).float().numpy()
    amax = np.max(np.abs(y32), axis=-1)
    inv = np.where(amax > 0, np.float32(448.0) / np.where(amax > 0, amax, np.float32(1.0)),
                   np.float32(0.0)).astype(np.float32)
    v32 = (y32 * inv[..., None]).astype(np.float32)
    ref = oracle.e4m3_encode(v32.astype(np.float64))
    s_ref = amax.astype(np.float64) / 448.0
    assert s.shape == s_ref.shape, f"{what}: scales {s.shape} vs {s_ref.shape}"
    live = s_ref > 0
    assert np.all(s[~live] == 0.0), f"{what}: non-zero scale of a zero block"
    ulp = 2.0 ** -7 if io_dtype == torch.bfloat16 else 2.0 ** -23
    rel = np.abs(s[live] / s_ref[live] - 1.0)
    assert rel.size == 0 or rel.max() <= 1e-2 + ulp, f"{what}: scale off by {rel.max():.3e}"
    big = np.abs(v32) >= 32.0
    dord = np.abs(_e4m3_ordinal(codes) - _e4m3_ordinal(ref))[big]
    assert dord.size == 0 or dord.max() <= 1, f"{what}: a code {dord.max()} steps off"
    frac = float(np.mean(dord > 0)) if dord.size else 0.0
    assert frac <= 0.15, f"{what}: {frac:.3f} of the codes one step off"
    deq = oracle.e4m3_decode(codes) * s[..., None]
    deq_ref = oracle.e4m3_decode(ref) * s_ref[..., None]
    r, r_ref = rel_l2(deq, y_ref), rel_l2(deq_ref, y_ref)
    assert r <= r_ref + BF16_REL_L2, f"{what}: relL2 {r:.3e} vs the reference codes' {r_ref:.3e}"
    return r, r_ref, frac
