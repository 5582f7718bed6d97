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
