"""Seeded synthetic inputs for the Lightning Attention layer kernel.

This module only draws numbers: it holds none of the attention arithmetic, and both the CUDA
path's tests and the CPU oracle receive the exact bits it produces.

Shapes follow "Ling and Ring 2.6 Technical Report" (Chinese translation, garden.houmin.site),
§2.1.1 and Table 1: 64 attention heads of dimension 128 for Ling-2.6-1T (hidden 8,192), context up
to 262,144 tokens.  The report trains and serves on its own data; no dataset is used here, every
input is drawn from a seeded normal distribution.

Decay schedule.  The pages give none.  The slope of head h (0-based) of H heads is read as
``s_h = 2 ** (-8 (h + 1) / H)`` and the decay is ``lambda_h = exp(-s_h)`` (Lightning Attention's
ALiBi-style geometric schedule); for H = 64 the decays run from 0.39972 (head 0) to 0.99610
(head 63).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


def slopes(H: int, device="cpu") -> torch.Tensor:
    """float32[H]: s_h = 2^(-8 (h+1) / H), computed in double and rounded once to float32."""
    vals = [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]
    return torch.tensor(vals, dtype=torch.float64).to(torch.float32).to(device)


@dataclass(frozen=True)
class Workload:
    """One synthetic workload.  ``dist``: 'scaled_normal' draws q, k, v ~ N(0,1)/sqrt(d);
    'silu_qk' draws q, k = SiLU(N(0,1)) and v ~ N(0,1)."""
    name: str
    B: int
    N: int
    H: int
    d: int
    dtype: torch.dtype
    dist: str
    seed: int
    decode_steps: int = 0
    decode_seed: int = 0
    notes: str = field(default="", compare=False)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 256, 2, 64, torch.float32, "scaled_normal", 0,
                          notes="fp32 I/O, full o and state compared, relL2 <= 1e-5"),
    "prefill_4k": Workload("prefill_4k", 1, 4096, 64, 128, torch.bfloat16, "silu_qk", 5,
                           notes="Ling-2.6-1T layer shape (H=64, d=128), N=4096"),
    "prefill_32k": Workload("prefill_32k", 2, 32768, 64, 128, torch.bfloat16, "scaled_normal", 1,
                            notes="mid-context prefill, B=2, N=32768"),
    "prefill_256k": Workload("prefill_256k", 1, 262144, 64, 128, torch.bfloat16, "scaled_normal",
                             2, notes="long-context prefill, N=262144, segment scan"),
    "decode_256x2k": Workload("decode_256x2k", 256, 2048, 64, 128, torch.bfloat16,
                              "scaled_normal", 3, decode_steps=512, decode_seed=4,
                              notes="2048-token prefill of 256 sequences, then 512 decode steps"),
}


def _transform(x: torch.Tensor, kind: str, d: int) -> torch.Tensor:
    if kind == "scaled":
        return x * (1.0 / math.sqrt(d))
    if kind == "silu":
        return torch.nn.functional.silu(x)
    if kind == "plain":
        return x
    raise ValueError(kind)


def draw_qkv(B: int, N: int, H: int, d: int, *, dist: str = "scaled_normal", seed: int = 0,
             dtype: torch.dtype = torch.bfloat16, device="cpu", generator=None):
    """q, k, v as [B, N, H, d] tensors of ``dtype`` on ``device``.

    One torch.Generator on ``device`` seeded with ``seed`` draws q, then k, then v as float32
    N(0,1); each is transformed (scale or SiLU) in float32 and rounded once to ``dtype``.  The
    stream differs between CPU and CUDA generators; parity never depends on it because the oracle
    receives the very bits drawn here.
    """
    g = generator
    if g is None:
        g = torch.Generator(device=device)
        g.manual_seed(seed)
    if dist == "scaled_normal":
        kinds = ("scaled", "scaled", "scaled")
    elif dist == "silu_qk":
        kinds = ("silu", "silu", "plain")
    else:
        raise ValueError(f"unknown dist {dist!r}")
    out = []
    for kind in kinds:
        x = torch.randn((B, N, H, d), generator=g, dtype=torch.float32, device=device)
        x = _transform(x, kind, d).to(dtype)
        out.append(x)
    return tuple(out)


def draw_workload(w: Workload, device="cpu", N=None, B=None):
    """q, k, v for a named workload (optionally with a smaller N or B for quick cases)."""
    return draw_qkv(B if B is not None else w.B, N if N is not None else w.N, w.H, w.d,
                    dist=w.dist, seed=w.seed, dtype=w.dtype, device=device)


def decode_token_generator(seed: int, device="cpu") -> torch.Generator:
    """The generator that draws every decode step's q, k, v (in that order, per step)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def draw_decode_token(g: torch.Generator, B: int, H: int, d: int, *, dtype=torch.bfloat16,
                      device="cpu"):
    """One decode step's q, k, v: [B, H, d], N(0,1)/sqrt(d) rounded to ``dtype``."""
    out = []
    for _ in range(3):
        x = torch.randn((B, H, d), generator=g, dtype=torch.float32, device=device)
        out.append((x * (1.0 / math.sqrt(d))).to(dtype))
    return tuple(out)


def window_starts(N: int, count: int = 8, length: int = 4096, seed: int = 1002):
    """Sorted start tokens of ``count`` windows of ``length`` tokens, drawn uniformly from
    [0, N - length] by a CPU generator seeded ``seed`` (windows may overlap)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    hi = max(N - length, 0)
    starts = torch.randint(0, hi + 1, (count,), generator=g).tolist()
    return sorted(int(s) for s in starts)


def draw_seqlens(total: int, n_seqs: int, seed: int = 7, short_frac: float = 0.75) -> list[int]:
    """Lengths of ``n_seqs`` packed sequences summing to ``total`` tokens, in a fragmented mix:
    about ``short_frac`` of the sequences are short (1..256 tokens, log-uniform) and the rest
    share the remaining tokens in random proportions.  Seeded CPU generator; returns a list."""
    g = torch.Generator()
    g.manual_seed(seed)
    n_short = min(n_seqs - 1, int(round(short_frac * n_seqs))) if n_seqs > 1 else 0
    short = torch.exp(torch.rand(n_short, generator=g, dtype=torch.float64) * math.log(256.0))
    short = [max(1, int(x)) for x in short.tolist()]
    while sum(short) > total // 2 and short:
        short.pop()
    rest = total - sum(short)
    n_long = n_seqs - len(short)
    w = torch.rand(n_long, generator=g, dtype=torch.float64) + 0.05
    cuts = [int(x) for x in (w / w.sum() * rest).tolist()]
    cuts[-1] += rest - sum(cuts)
    lens = short + cuts
    perm = torch.randperm(len(lens), generator=g).tolist()
    return [lens[i] for i in perm]


def cu_from_lengths(lengths) -> list[int]:
    """Exclusive prefix sums [0, l0, l0 + l1, ...] (n + 1 entries)."""
    cu = [0]
    for x in lengths:
        cu.append(cu[-1] + int(x))
    return cu


@dataclass(frozen=True)
class VarlenWorkload:
    """A packed batch of ``n_seqs`` sequences (lengths from ``draw_seqlens(T, n_seqs, len_seed)``)
    with initial states N(0,1) * ``state_scale`` (seed ``state_seed``); q, k, v drawn as
    ``draw_qkv(1, T, H, d, dist, seed)``."""
    name: str
    T: int
    n_seqs: int
    H: int
    d: int
    dtype: torch.dtype
    dist: str
    seed: int
    len_seed: int
    state_seed: int
    state_scale: float = 0.1


VARLEN_WORKLOADS = {
    "varlen_64k": VarlenWorkload("varlen_64k", 65536, 48, 64, 128, torch.bfloat16, "silu_qk", 82,
                                 81, 83),
}


def draw_states(n: int, H: int, d: int, *, seed: int, scale: float, device="cpu") -> torch.Tensor:
    """fp32 [n, H, d, d] initial states: N(0,1) * scale from one generator on ``device``."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn((n, H, d, d), generator=g, device=device, dtype=torch.float32) * scale
