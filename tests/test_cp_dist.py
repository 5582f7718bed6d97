"""The context-parallel exchange on CPU ranks (gloo, world sizes 2 and 3).

prefill_cp's host logic (length exchange, all_gather of the parts' states in rank order, the
choice of the parts each rank folds, empty parts) runs in separate processes with the fp64 oracle
standing in for the three device steps.  The concatenated outputs and every rank's outgoing state
must equal one sequential oracle pass over the whole sequence.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from long_context_attention_la_b200 import cp

B, H, d = 2, 3, 8
SLOPES = np.array([0.02, 0.4, 1.5], dtype=np.float32)


class OracleOps:
    """The three device steps of prefill_cp, computed by the oracle on CPU tensors (fp64)."""

    def local_state(self, k, v, slopes):
        b, L, h, dd = k.shape
        if L == 0:
            return torch.zeros((b, h, dd, dd), dtype=torch.float64)
        kk = k.numpy()
        _, st = oracle.prefill(np.zeros_like(kk), kk, v.numpy(), slopes.numpy())
        return torch.from_numpy(st.reshape(b, h, dd, dd))

    def fold(self, parts, lengths, slopes, state_in):
        return torch.from_numpy(oracle.fold_states(
            parts.numpy(), lengths, slopes.numpy(),
            None if state_in is None else state_in.double().numpy()))

    def prefill_from(self, q, k, v, slopes, state_in):
        b, L, h, dd = q.shape
        if L == 0:
            return torch.empty((b, 0, h, dd), dtype=torch.float64), state_in.clone()
        o, st = oracle.prefill(q.numpy(), k.numpy(), v.numpy(), slopes.numpy(),
                               state_in=state_in.numpy().reshape(b * h, dd, dd))
        o = o.reshape(b, h, L, dd).transpose(0, 2, 1, 3).copy()
        return torch.from_numpy(o), torch.from_numpy(st.reshape(b, h, dd, dd))


def _inputs(N):
    rng = np.random.default_rng(300 + N)
    q, k, v = ((rng.normal(size=(B, N, H, d)) / np.sqrt(d)).astype(np.float32) for _ in range(3))
    s0 = rng.normal(size=(B, H, d, d)) * 0.3
    return q, k, v, s0


def _worker(rank, world, port, cuts, with_state_in, give_lengths, outdir):
    store = dist.TCPStore("127.0.0.1", port, world, rank == 0,
                          timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("gloo", store=store, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, s0 = _inputs(cuts[-1])
        a, b = cuts[rank], cuts[rank + 1]
        part = [torch.from_numpy(x[:, a:b].copy()) for x in (q, k, v)]
        out, st = cp.prefill_cp(*part, torch.from_numpy(SLOPES),
                                state_in=torch.from_numpy(s0) if with_state_in else None,
                                part_lengths=np.diff(cuts).tolist() if give_lengths else None,
                                ops=OracleOps())
        torch.save({"out": out, "st": st}, os.path.join(outdir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("cuts,with_state_in,give_lengths", [
    ([0, 17, 40], False, False),
    ([0, 29, 29, 40], True, False),   # an empty middle part
    ([0, 1, 39, 40], True, True),     # lengths known up front: no length exchange
])
def test_prefill_cp_gloo_ranks_match_sequential_oracle(tmp_path, cuts, with_state_in,
                                                       give_lengths):
    world = len(cuts) - 1
    mp.start_processes(_worker, args=(world, _free_port(), cuts, with_state_in, give_lengths,
                                      str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    q, k, v, s0 = _inputs(cuts[-1])
    sin = s0.reshape(B * H, d, d) if with_state_in else None
    o_ref, st_ref = oracle.prefill(q, k, v, SLOPES, state_in=sin)
    o_ref = o_ref.reshape(B, H, -1, d).transpose(0, 2, 1, 3)
    res = [torch.load(os.path.join(tmp_path, f"r{r}.pt")) for r in range(world)]
    o = np.concatenate([r["out"].numpy() for r in res], axis=1)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    # every rank's outgoing state is the sequence's state at the end of its part
    for r in range(world):
        end = cuts[r + 1]
        if end == 0:
            continue
        _, st_end = oracle.prefill(q[:, :end].copy(), k[:, :end].copy(), v[:, :end].copy(),
                                   SLOPES, state_in=sin)
        np.testing.assert_allclose(res[r]["st"].numpy(), st_end.reshape(B, H, d, d),
                                   rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res[-1]["st"].numpy(), st_ref.reshape(B, H, d, d), rtol=1e-10,
                               atol=1e-12)


def _one_rank_group():
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True,
                          timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("gloo", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=30))


def test_prefill_cp_rejects_inconsistent_arguments():
    """Shape and part-length errors are raised before any exchange on the rank that sees them."""
    _one_rank_group()
    try:
        x = torch.zeros((B, 5, H, d))
        sl = torch.from_numpy(SLOPES)
        with pytest.raises(ValueError):
            cp.prefill_cp(x, x, x, sl, part_lengths=[4], ops=OracleOps())   # this rank holds 5
        with pytest.raises(ValueError):
            cp.prefill_cp(x, x, x, sl, part_lengths=[5, 5], ops=OracleOps())  # one rank only
        with pytest.raises(ValueError):
            cp.prefill_cp(x, torch.zeros((B, 4, H, d)), x, sl, ops=OracleOps())
        # a one-rank group is a plain prefill from the initial state
        rng = np.random.default_rng(5)
        q, k, v = (torch.from_numpy(rng.normal(size=(B, 5, H, d)).astype(np.float32))
                   for _ in range(3))
        out, st = cp.prefill_cp(q, k, v, sl, ops=OracleOps())
        o_ref, st_ref = oracle.prefill(q.numpy(), k.numpy(), v.numpy(), SLOPES)
        np.testing.assert_allclose(out.numpy(), o_ref.reshape(B, H, 5, d).transpose(0, 2, 1, 3),
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(st.numpy(), st_ref.reshape(B, H, d, d), rtol=1e-12, atol=1e-12)
    finally:
        dist.destroy_process_group()


def test_product_modules_do_not_import_the_oracle():
    """The oracle is test infrastructure: no module of the package imports it."""
    import ast
    import pathlib
    pkg = pathlib.Path(cp.__file__).parent
    for path in pkg.glob("*.py"):
        tree = ast.parse(path.read_text())
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                assert all(not a.name.split(".")[0] == "oracle" for a in node.names), path
            if isinstance(node, ast.ImportFrom):
                assert (node.module or "").split(".")[0] != "oracle", path
