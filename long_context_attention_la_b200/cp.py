"""Context-parallel prefill of Lightning Attention across the ranks of a torch.distributed group.

"Ling and Ring 2.6 Technical Report", §4.1.1 Context Parallel for Lightning Attention, Fig. 10
(chunk QKV -> local h -> AllGather h -> fused update h -> fused update O).  A long sequence is cut
into consecutive parts, part r on rank r (ranks in group order).  Every rank:

  1. computes its part's local state  h_r = sum_t lambda^(L_r-1-t) k_t^T v_t   (la_prefill_state)
  2. gathers every rank's h and part length                                    (all_gather)
  3. folds the states of the parts before it into its incoming state
         S_r = lambda^(L_{r-1}) ( ... (lambda^(L_0) S_in + h_0) ... ) + h_{r-1}  (la_state_fold)
  4. computes its outputs and outgoing state starting from S_r                 (la_prefill_varlen)

The last rank's outgoing state is the state after the whole sequence.  The only exchange is one
all_gather of B*H*d*d fp32 per rank (4 MiB for B = 1, H = 64, d = 128).

This orders the work differently from the report, which computes the local outputs first and
then corrects them with O += diag(lambda^(i+1)) Q S_r.  Here the outputs are computed once, from
the folded state, so a rank reads K and V twice and Q once and writes O once: 1,536 bytes per
token-head in bf16, against 2,304 for local outputs plus a correction pass that re-reads Q and O
and writes O again.

The kernels are reached through an ``ops`` object (``DeviceOps``, the default, calls the C ABI on
CUDA tensors); any object with the same three methods can stand in for them, which is how the
host-side exchange is tested on CPU ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import la


class DeviceOps:
    """The three device steps, through the C ABI (CUDA tensors)."""

    def local_state(self, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor) -> torch.Tensor:
        """fp32 [B, H, d, d]: the part's state from zero (step 1; zero for an empty part)."""
        B, L, H, d = k.shape
        if L == 0:
            return torch.zeros((B, H, d, d), dtype=torch.float32, device=k.device)
        return la.prefill_state(k, v, slopes)

    def fold(self, parts: torch.Tensor, lengths, slopes: torch.Tensor,
             state_in: torch.Tensor | None) -> torch.Tensor:
        """fp32 [B, H, d, d]: the incoming state after parts[0..n-1] (step 3)."""
        return la.state_fold(parts, lengths, slopes, state_in=state_in)

    def prefill_from(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                     slopes: torch.Tensor, state_in: torch.Tensor):
        """(out [B, N, H, d], state_out [B, H, d, d]) of the part from state_in (step 4)."""
        B, N, H, d = q.shape
        if N == 0:
            return torch.empty_like(q), state_in.clone()
        cu = torch.arange(B + 1, dtype=torch.int64, device=q.device) * N
        out, st = la.prefill_varlen(q.view(B * N, H, d), k.view(B * N, H, d),
                                    v.view(B * N, H, d), slopes, cu, state_in=state_in)
        return out.view(B, N, H, d), st


def _gather(x: torch.Tensor, group, world: int) -> torch.Tensor:
    """[world, *x.shape]: every rank's x, in rank order."""
    out = torch.empty((world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, x.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), x.contiguous(), group=group)
    return out


def prefill_cp(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor, *,
               group=None, state_in: torch.Tensor | None = None, part_lengths=None,
               ops=None):
    """out, state = prefill_cp(q, k, v, slopes): this rank's part of a context-parallel prefill.

    q, k, v: [B, L_r, H, d], this rank's consecutive tokens of every sequence (rank r of `group`
    holds part r; L_r may differ between ranks and may be 0).  slopes: fp32[H].  state_in:
    optional fp32 [B, H, d, d] initial state of the sequences, the same on every rank.
    part_lengths: every rank's L_r.  Pass it on the hot path: without it the lengths are
    exchanged with a collective and read back to the host, which synchronises the device on
    every call.  Returns this rank's outputs [B, L_r, H, d] and
    the state after its part (on the last rank: after the whole sequence).  Collective: every
    rank of the group must call it with the same B, H, d.
    """
    ops = ops if ops is not None else DeviceOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, L, H, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, L, H, d] shape")
    if part_lengths is None:
        n = torch.tensor([L], dtype=torch.int64, device=q.device)
        part_lengths = _gather(n, group, world).view(-1).tolist()
    part_lengths = [int(x) for x in part_lengths]
    if len(part_lengths) != world or part_lengths[rank] != L:
        raise ValueError("part_lengths must list every rank's token count, this rank's = L")

    # 1. local state of this part
    h = ops.local_state(k, v, slopes)
    # 2. every part's local state, in rank order
    hs = _gather(h, group, world)
    # 3. incoming state: the parts before this one folded onto the initial state
    s_r = ops.fold(hs[:rank], part_lengths[:rank], slopes, state_in)
    # 4. this part's outputs and outgoing state
    return ops.prefill_from(q, k, v, slopes, s_r)
