"""Benchmark of the Lightning Attention layer kernel (prefill + decode step) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill_32k|prefill_4k|prefill_256k|varlen_64k]

One step = one whole pass of the hot path over one batch of synthetic input:
  * la_prefill of the prefill workload (default: B=2, N=32768, H=64, d=128, bf16, seed 1), which
    writes o for every token and the final fp32 state;
  * one la_decode_step of 256 sequences x 64 heads x d=128 on a resident fp32 state (2 GiB).
``--workload varlen_64k`` runs la_prefill_varlen instead: 65,536 tokens of 48 packed sequences of a
fragmented length mix, each continuing from an fp32 initial state.
The JSON line's ``value`` is prefill tokens/s (tokens = B*N positions, all 64 heads) summed over
ranks; the decode step is reported under ``decode`` as state GB/s.  Under torchrun each rank runs
an independent replica (weak scaling, no collective on the data path).

Timing: W untimed warm-up steps, then K steps between a barrier + device synchronize on both
sides, CUDA events on the launching stream, max over ranks.  Inputs are larger than L2 (4 GiB of
prefill activations, 2 GiB of decode state), so no flush is needed between steps.

``--impl reference`` times the fp64 CPU oracle (test infrastructure) on the host cores instead:
a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from long_context_attention_la_b200 import synth  # noqa: E402

METRIC = "lightning-attn prefill tok/s & TFLOP/s (H=64,d=128); decode state GB/s vs peak"
DECODE = dict(B=256, H=64, d=128)


def measured_counters(path=None):
    """Counters of one prefill launch of the default workload from the committed ncu capture
    (the fenced json record in profiles/chunked_prefill_kernel_counters.md), or None when the
    kernel sources changed since that capture: DRAM bytes and the tensor-pipe activity."""
    import hashlib
    path = path or os.path.join(ROOT, "profiles", "chunked_prefill_kernel_counters.md")
    try:
        with open(path) as f:
            text = f.read()
        start = text.index("```json\n") + len("```json\n")
        rec = json.loads(text[start:text.index("\n```", start)])
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return rec
    except Exception:
        return None


def prefill_bytes_per_token_head(d, gate=False, gate_separate=False, fp8=False):
    """Algorithmic bytes of one token-head of the timed prefill step (bf16 rows of d values):
    read q, k, v and write o; the fused norm + gate also reads the gate; the separate pass reads
    o and the gate and writes y; an FP8 y is d bytes plus a 4-byte block scale."""
    row = 2 * d
    y_row = d + 4 if fp8 else row
    if gate:
        return 3 * row + row + row
    if gate_separate:
        return 4 * row + 2 * row + y_row
    return 4 * row


# Tensor-core flops the prefill kernel executes per token and head at d = 128, by chunk length:
# four 128 x 128 x 128 products per 128-token tile at C = 128 (S, the inter product, the state
# update, P V); five at C = 64 (a second inter product) and at C = 256 (per two tiles: three
# score blocks, two inter products, two state updates, three P V blocks).
EXECUTED_FLOPS_PER_TOKEN_HEAD = {64: 163840.0, 128: 131072.0, 256: 163840.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------------------------
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        cmd = ["nvidia-smi", f"--id={self.index}",
               "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", "100"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 4:
                continue
            try:
                s, m = float(parts[0]), float(parts[1])
                bits = int(parts[3], 16)
            except ValueError:
                continue
            sm.append(s)
            mx = m
            for b, name in REASON_BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------------------------
# distributed plumbing (replicas only)
# --------------------------------------------------------------------------------------------
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on the host cores, bounded sample
# --------------------------------------------------------------------------------------------
def host_cpu():
    """(cores this process may run on, CPU model string) of the host."""
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:  # pragma: no cover
        n = os.cpu_count()
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except Exception:  # pragma: no cover
        pass
    return n, model


def oracle_sample(w, seconds_target=15.0):
    """Times the oracle on n_threads heads x n_tok tokens of the workload's distribution.
    Returns (tok/s scaled to the workload's all-heads token, cores, description)."""
    import numpy as np

    import oracle
    cores = oracle.num_threads()
    n_heads = cores
    # ~2 * 2 * d^2 fp64 flops per token-head; aim at about seconds_target of CPU time
    n_tok = min(w.N, 8192)
    q, k, v = synth.draw_qkv(1, n_tok, n_heads, w.d, dist=w.dist, seed=w.seed, dtype=w.dtype)
    bits = [x.view(torch.int16).numpy().view(np.uint16) for x in (q, k, v)]
    sl = synth.slopes(w.H).numpy()[:n_heads] if n_heads <= w.H else np.resize(
        synth.slopes(w.H).numpy(), n_heads)
    t0 = time.perf_counter()
    oracle.prefill(*bits, sl.astype(np.float32), nthreads=cores)
    dt = time.perf_counter() - t0
    reps = max(1, int(seconds_target / max(dt, 1e-3)))
    reps = min(reps, 64)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.prefill(*bits, sl.astype(np.float32), nthreads=cores)
    dt = (time.perf_counter() - t0) / reps
    token_heads_per_s = n_heads * n_tok / dt
    desc = (f"fp64 oracle, {n_heads} heads x {n_tok} tokens of the {w.name} distribution "
            f"({reps} reps, {dt:.2f} s each); tok/s = token-heads/s / H={w.H}")
    return token_heads_per_s / w.H, cores, desc


# --------------------------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------------------------
def cp_launches(B, N, H):
    """Kernels of one context-parallel state step: the state pass, its combine kernel when a
    range boundary falls inside a head (the split of la_state.cu for this GPU's SM count), and
    the fold."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    nc = (N + 127) // 128
    total = B * H * nc
    g0 = max(1, min(sms, total))
    width = (total + g0 - 1) // g0
    grid = (total + width - 1) // width
    return 2 + (1 if grid > 1 and width % nc else 0)


def run_ours(args):
    from long_context_attention_la_b200 import build as labuild
    from long_context_attention_la_b200 import la

    labuild.build()
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    vw = synth.VARLEN_WORKLOADS.get(args.workload)
    w = synth.WORKLOADS[args.workload] if vw is None else synth.Workload(
        vw.name, 1, vw.T, vw.H, vw.d, vw.dtype, vw.dist, vw.seed)
    B, N, H, d = w.B, w.N, w.H, w.d
    if args.cp:
        # context parallel: rank r holds tokens [r N/world, (r+1) N/world) of every sequence
        if vw is not None or args.gate or args.gate_separate or N % world:
            raise SystemExit("--cp takes a fixed-length workload whose N divides by the ranks")
        N = N // world
    q, k, v = synth.draw_qkv(B, N, H, d, dist=w.dist, seed=w.seed + 1000 * rank, dtype=w.dtype,
                             device=dev)
    sl = synth.slopes(H, dev)
    if args.qk_fused and (args.gate or args.cp or args.qk_rope or args.chunk not in (0, 128)):
        raise SystemExit("--qk-fused is the plain-output, 128-token-chunk prefill of raw q, k")
    if args.fp8 and not args.gate_separate:
        raise SystemExit("--fp8 is an output format of --gate-separate (the stand-alone "
                         "norm + gate + quantize operator)")
    # with --fp8 the norm + gate stores FP8 E4M3 codes (one byte per value) and one fp32 scale
    # per (head, token) block of d values
    fp8_scales = (torch.empty((H, B * N), dtype=torch.float32, device=dev) if args.fp8
                  else None)
    out = torch.empty_like(q)
    y8 = torch.empty(q.shape, dtype=torch.uint8, device=dev) if args.fp8 and \
        args.gate_separate else None
    extra_in = []  # further inputs copied from the host in the e2e leg
    epi = None
    sep = None
    if args.gate_separate:
        gg = torch.Generator(device=dev)
        gg.manual_seed(77 + 1000 * rank)
        gate = (torch.randn((B * N, H, d), generator=gg, device=dev)).to(w.dtype)
        gamma = (1.0 + 0.1 * torch.randn((H, d), generator=gg, device=dev)).float()
        extra_in += [gate]
        sep = la.la_gate_norm(gate.data_ptr(), gamma.data_ptr(), 1e-6,
                              fp8_scales.data_ptr() if args.fp8 else None)
    if args.gate:
        # fused grouped RMSNorm + sigmoid gate on the prefill output: a gate pre-activation the
        # size of q and a norm weight per head and channel (synthetic, seeded)
        gg = torch.Generator(device=dev)
        gg.manual_seed(77 + 1000 * rank)
        gate = (torch.randn((B * N, H, d), generator=gg, device=dev)).to(w.dtype)
        gamma = (1.0 + 0.1 * torch.randn((H, d), generator=gg, device=dev)).float()
        extra_in += [gate]
        epi = la.la_gate_norm(gate.data_ptr(), gamma.data_ptr(), 1e-6)
    if vw is None and (args.gate or args.cp or args.qk_fused):
        # the fused epilogue, the in-kernel QK norm and the initial state are options of the
        # packed entry points: B sequences of N tokens
        n_states = B
        cu = torch.arange(0, B * N + 1, N, dtype=torch.int64, device=dev)
        sin = None
        if args.cp:
            # the incoming state of this rank's part, folded from the gathered part states
            sin = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
            h_loc = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
            h_all = (torch.empty(world, B, H, d, d, dtype=torch.float32, device=dev)
                     if world > 1 else h_loc.unsqueeze(0))
            sdesc = la.make_desc(B, N, H, d, w.dtype)
            s_ws_bytes = la.la_prefill_state_workspace_bytes(sdesc)
            s_ws = torch.empty(max(s_ws_bytes, 256), dtype=torch.uint8, device=dev)
            part_lengths = [N] * world
        st = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
        desc = la.la_varlen_desc(B * N, B, H, d, la.LA_BF16, args.chunk, args.segments,
                                 la.LA_PATH_AUTO)
        ws_bytes = la.la_prefill_varlen_workspace_bytes(desc)
    elif vw is None:
        n_states = B
        st = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
        desc = la.make_desc(B, N, H, d, w.dtype, chunk=args.chunk, segments=args.segments)
        ws_bytes = la.la_prefill_workspace_bytes(desc)
    else:
        lengths = synth.draw_seqlens(vw.T, vw.n_seqs, seed=vw.len_seed)
        cu = torch.tensor(synth.cu_from_lengths(lengths), dtype=torch.int64, device=dev)
        n_states = vw.n_seqs
        sin = synth.draw_states(vw.n_seqs, H, d, seed=vw.state_seed, scale=vw.state_scale,
                                device=dev)
        st = torch.empty_like(sin)
        extra_in += [sin, cu]
        desc = la.la_varlen_desc(vw.T, vw.n_seqs, H, d, la.LA_BF16, args.chunk, args.segments,
                                 la.LA_PATH_AUTO)
        ws_bytes = la.la_prefill_varlen_workspace_bytes(desc)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    qk = None
    if args.qk_rope:
        # QK RMSNorm + partial RoPE (rotary dim 64, theta 6e6) turns raw projections into the
        # prefill's q and k every step
        gq_ = torch.Generator(device=dev)
        gq_.manual_seed(78 + 1000 * rank)
        q_raw = torch.randn(q.shape, generator=gq_, device=dev).to(w.dtype)
        k_raw = torch.randn(q.shape, generator=gq_, device=dev).to(w.dtype)
        gam_q = (1.0 + 0.1 * torch.randn(d, generator=gq_, device=dev)).float()
        gam_k = (1.0 + 0.1 * torch.randn(d, generator=gq_, device=dev)).float()
        positions = (torch.arange(B * N, device=dev) % N).to(torch.int64)
        qk = la.la_qk_norm_rope_desc(B * N, H, d, H * d, H * d, 64, 6.0e6, 1e-6, 0)
        extra_in += [q_raw, k_raw]
    qkp = None
    if args.qk_fused:
        # the same operator inside the prefill kernel: q and k (as drawn) are the raw
        # projections, normalised and rotated tile by tile in shared memory
        gq_ = torch.Generator(device=dev)
        gq_.manual_seed(78 + 1000 * rank)
        gam_q = (1.0 + 0.1 * torch.randn(d, generator=gq_, device=dev)).float()
        gam_k = (1.0 + 0.1 * torch.randn(d, generator=gq_, device=dev)).float()
        positions = (torch.arange(B * N, device=dev) % N).to(torch.int64)
        qkp = la.la_qk_prologue(gam_q.data_ptr(), gam_k.data_ptr(), positions.data_ptr(), 64,
                                6.0e6, 1e-6, 0)

    Bd, Hd, dd = DECODE["B"], DECODE["H"], DECODE["d"]
    if args.no_decode:
        Bd = 1  # placeholder tensors only; the decode call is skipped
    dstate = torch.randn(Bd, Hd, dd, dd, dtype=torch.float32, device=dev) * 0.05
    gdec = synth.decode_token_generator(4 + 1000 * rank, dev)
    n_mtp = max(1, args.mtp)
    if n_mtp == 1:
        dq, dk, dv = synth.draw_decode_token(gdec, Bd, Hd, dd, device=dev)
    else:
        # n_mtp tokens per sequence in one multi-token step, [B, n, H, d]
        toks = [synth.draw_decode_token(gdec, Bd, Hd, dd, device=dev) for _ in range(n_mtp)]
        dq, dk, dv = (torch.stack([t[i] for t in toks], dim=1).contiguous() for i in range(3))
    dout = torch.empty_like(dq)
    dsl = synth.slopes(Hd, dev)

    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    packed = vw is not None or args.gate or args.cp or args.qk_fused

    def cp_state_call():
        # local state of this rank's part, all ranks' states, the fold of those before it
        rc = la.la_prefill_state(sdesc, k.data_ptr(), v.data_ptr(), sl.data_ptr(), 0,
                                 h_loc.data_ptr(), s_ws.data_ptr(), s_ws_bytes, sp)
        if rc != la.LA_OK:
            raise la.LaError(rc, "la_prefill_state")
        if world > 1:
            torch.distributed.all_gather_into_tensor(h_all, h_loc)
        rc = la.la_state_fold(rank, B * H, H, d, h_all.data_ptr() if rank > 0 else 0,
                              part_lengths[:rank], sl.data_ptr(), 0, sin.data_ptr(), sp)
        if rc != la.LA_OK:
            raise la.LaError(rc, "la_state_fold")

    def prefill_call():
        if not packed:
            rc = la.la_prefill(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                               out.data_ptr(), st.data_ptr(), ws.data_ptr(), ws_bytes, sp)
        elif qkp is not None:
            rc = la.la_prefill_varlen_qk(desc, qkp, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         sl.data_ptr(), cu.data_ptr(),
                                         0 if sin is None else sin.data_ptr(), out.data_ptr(),
                                         st.data_ptr(), ws.data_ptr(), ws_bytes, sp)
        else:
            rc = la.la_prefill_varlen(desc, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                      sl.data_ptr(), cu.data_ptr(),
                                      0 if sin is None else sin.data_ptr(), out.data_ptr(),
                                      st.data_ptr(), ws.data_ptr(), ws_bytes, sp, epilogue=epi)
        if rc != la.LA_OK:
            raise la.LaError(rc, "la_prefill")

    def sep_call():
        # the post-kernel operator on its own, in place on the prefill's output (FP8: into its
        # own byte buffer)
        rc = la.la_gate_norm_apply(B * N, H, d, la.LA_BF16, out.data_ptr(), sep,
                                   (y8 if y8 is not None else out).data_ptr(), sp)
        if rc != la.LA_OK:
            raise la.LaError(rc, "la_gate_norm_apply")

    def qk_call():
        rc = la.la_qk_norm_rope(qk, q_raw.data_ptr(), k_raw.data_ptr(), gam_q.data_ptr(),
                                gam_k.data_ptr(), positions.data_ptr(), q.data_ptr(),
                                k.data_ptr(), sp)
        if rc != la.LA_OK:
            raise la.LaError(rc, "la_qk_norm_rope")

    def decode_call():
        if args.no_decode:
            return
        if n_mtp == 1:
            rc = la.la_decode_step(Bd, Hd, dd, la.LA_BF16, dq.data_ptr(), dk.data_ptr(),
                                   dv.data_ptr(), dsl.data_ptr(), dstate.data_ptr(),
                                   dout.data_ptr(), sp)
        else:
            rc = la.la_decode_multi(Bd, Hd, dd, n_mtp, la.LA_BF16, dq.data_ptr(), dk.data_ptr(),
                                    dv.data_ptr(), dsl.data_ptr(), dstate.data_ptr(),
                                    dout.data_ptr(), sp)
        if rc != la.LA_OK:
            raise la.LaError(rc, "la_decode_step")

    for _ in range(args.warmup):
        if qk is not None:
            qk_call()
        if args.cp:
            cp_state_call()
        prefill_call()
        if sep is not None:
            sep_call()
        decode_call()
    torch.cuda.synchronize(dev)
    st_rc = la.la_workspace_status(ws.data_ptr(), sp)
    if st_rc != la.LA_OK:
        raise la.LaError(st_rc, "device status after warm-up")

    K = args.steps
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(5)) for _ in range(K)]
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        t_all0.record(stream)
        for i in range(K):
            ev[i][3].record(stream)
            if qk is not None:
                qk_call()
            ev[i][0].record(stream)
            if args.cp:
                cp_state_call()
            ev[i][4].record(stream)
            prefill_call()
            if sep is not None:
                sep_call()
            ev[i][1].record(stream)
            decode_call()
            ev[i][2].record(stream)
        t_all1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    total_ms = t_all0.elapsed_time(t_all1)
    pre_ms = sum(e[4].elapsed_time(e[1]) for e in ev) / K
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / K
    qk_ms = sum(e[3].elapsed_time(e[0]) for e in ev) / K
    cp_ms = sum(e[0].elapsed_time(e[4]) for e in ev) / K
    st_rc = la.la_workspace_status(ws.data_ptr(), sp)
    if st_rc != la.LA_OK:
        raise la.LaError(st_rc, "device status after the timed steps")

    total_ms = max_over_ranks(total_ms, world)
    pre_ms_max = max_over_ranks(pre_ms, world)
    dec_ms_max = max_over_ranks(dec_ms, world)
    qk_ms_max = max_over_ranks(qk_ms, world)
    cp_ms_max = max_over_ranks(cp_ms, world)
    step_ms_max = max_over_ranks(cp_ms + pre_ms, world)  # the whole prefill of a part

    # ---- e2e: host buffers through the C ABI, copies inside the timed region ----
    e2e = None
    if not args.no_e2e:
        hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        hk = torch.empty_like(hq).pin_memory()
        hv = torch.empty_like(hq).pin_memory()
        hq.copy_(q.cpu())
        hk.copy_(k.cpu())
        hv.copy_(v.cpu())
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hy8 = torch.empty(y8.shape, dtype=y8.dtype, pin_memory=True) if y8 is not None else None
        hsc = (torch.empty(fp8_scales.shape, dtype=fp8_scales.dtype, pin_memory=True)
               if fp8_scales is not None else None)
        hst = torch.empty(st.shape, dtype=st.dtype, pin_memory=True)
        hdq = torch.empty(dq.shape, dtype=dq.dtype, pin_memory=True)
        hdk = torch.empty_like(hdq).pin_memory()
        hdv = torch.empty_like(hdq).pin_memory()
        hdq.copy_(dq.cpu())
        hdk.copy_(dk.cpu())
        hdv.copy_(dv.cpu())
        hdout = torch.empty_like(hdq).pin_memory()
        hextra = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in extra_in]
        for hx, x in zip(hextra, extra_in):
            hx.copy_(x.cpu())
        n_e2e = max(1, min(K, 10))
        # The inputs copied every step are double-buffered on the device, so that the copy of
        # step i + 1's inputs (on a copy stream) overlaps step i's kernels and the read-back of
        # its result (on the compute stream): the link carries both directions at once.  Inputs
        # whose address a call captured at set-up (the gate, initial states, cu_seqlens) keep
        # one buffer, and their copy waits for the previous step's kernels.
        copy_stream = torch.cuda.Stream(dev)
        per_step = [(q, hq), (k, hk), (v, hv)]
        if not args.no_decode:
            per_step += [(dq, hdq), (dk, hdk), (dv, hdv)]
        sets = [[x for x, _ in per_step], [torch.empty_like(x) for x, _ in per_step]]
        landed = [torch.cuda.Event() for _ in range(n_e2e)]
        done = [torch.cuda.Event() for _ in range(n_e2e)]
        barrier(world)
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        copy_stream.wait_event(e0)
        for i in range(n_e2e):
            bset = sets[i % 2]
            with torch.cuda.stream(copy_stream):
                if i >= 2:
                    copy_stream.wait_event(done[i - 2])  # step i - 2 has read this buffer set
                for x, (_, hx) in zip(bset, per_step):
                    x.copy_(hx, non_blocking=True)
                if hextra:
                    if i >= 1:
                        copy_stream.wait_event(done[i - 1])
                    for x, hx in zip(extra_in, hextra):
                        x.copy_(hx, non_blocking=True)
                landed[i].record(copy_stream)
            stream.wait_event(landed[i])
            q, k, v = bset[0], bset[1], bset[2]
            if not args.no_decode:
                dq, dk, dv = bset[3], bset[4], bset[5]
            if qk is not None:
                qk_call()
            if args.cp:
                cp_state_call()
            prefill_call()
            if sep is not None:
                sep_call()
            decode_call()
            done[i].record(stream)
            hout.copy_(out, non_blocking=True)
            if hy8 is not None:
                hy8.copy_(y8, non_blocking=True)
            if hsc is not None:
                hsc.copy_(fp8_scales, non_blocking=True)
            hst.copy_(st, non_blocking=True)
            if not args.no_decode:
                hdout.copy_(dout, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        q, k, v = sets[0][0], sets[0][1], sets[0][2]
        if not args.no_decode:
            dq, dk, dv = sets[0][3], sets[0][4], sets[0][5]
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
        dec_io = 0 if args.no_decode else 1
        bi = 3 * q.numel() * q.element_size() + dec_io * 3 * dq.numel() * dq.element_size() + sum(
            x.numel() * x.element_size() for x in extra_in)
        bo = out.numel() * out.element_size() + st.numel() * 4 + \
            dec_io * dout.numel() * dout.element_size() + \
            (y8.numel() if y8 is not None else 0) + \
            (fp8_scales.numel() * 4 if fp8_scales is not None else 0)
        e2e = {"value": world * B * N / (e2e_ms * 1e-3), "unit": "tok/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": e2e_ms,
               "steps": n_e2e}

    if rank == 0:
        hbm_peak, tc_peak, peak_kind = load_peaks()
        # committed counters describe the default launch only (prefill_32k, plain output, the
        # default chunk and plan)
        counters = (measured_counters() if args.workload == "prefill_32k" and not (
            args.gate or args.gate_separate or args.cp or args.chunk or args.segments or
            args.qk_fused) else None)
        tokens = B * N
        tok_s = world * tokens / ((step_ms_max if args.cp else pre_ms_max) * 1e-3)
        # algorithmic bytes of one prefill launch: read q, k, v and write o (bf16), write the
        # final states (and read the initial states of the packed workload)
        per_th = prefill_bytes_per_token_head(d, args.gate, args.gate_separate, args.fp8)
        pre_bytes = per_th * B * N * H + \
            n_states * H * d * d * 4 * (1 if vw is None and not args.cp else 2) + \
            (8 * B * N if args.qk_fused else 0)  # the in-kernel RoPE reads one position a token
        achieved = pre_bytes / (pre_ms_max * 1e-3) / 1e9
        canon = 4.0 * d * d * B * N * H  # recurrent-form flops
        chunk = args.chunk if args.chunk else 128
        executed = EXECUTED_FLOPS_PER_TOKEN_HEAD[chunk] * B * N * H
        dec_bytes = 2 * Bd * Hd * dd * dd * 4 + 4 * Bd * Hd * dd * 2 * n_mtp
        dec_gbs = dec_bytes / max(dec_ms_max * 1e-3, 1e-12) / 1e9
        cpu = None
        if world == 1 and not args.no_cpu:
            try:
                v_cpu, cores, sample = oracle_sample(w)
                n_aff, model = host_cpu()
                cpu = {"value": v_cpu, "unit": "tok/s", "cores": cores, "kind": "oracle",
                       "sample": sample, "affinity_cores": n_aff, "cpu_model": model}
            except Exception as exc:  # pragma: no cover - reported, not fatal
                cpu = {"value": None, "unit": "tok/s", "cores": None, "kind": "oracle",
                       "sample": f"failed: {exc}"}
        line = {
            "metric": METRIC, "value": tok_s, "unit": "tok/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": (f"{w.name}: B={B} N={N} H={H} d={d} bf16" if vw is None else
                                    f"{vw.name}: T={vw.T} tokens in {vw.n_seqs} packed sequences "
                                    f"(fragmented lengths), H={H} d={d} bf16, fp32 initial "
                                    f"states") + (", fused grouped RMSNorm + sigmoid gate epilogue"
                                                  if args.gate else "") +
                                   (", QK RMSNorm + RoPE (rotary dim 64) inside the prefill "
                                    "kernel on raw q, k" if args.qk_fused else "") +
                                   (", QK RMSNorm + RoPE pass (rotary dim 64) before the prefill"
                                    if args.qk_rope else "") +
                                   (", then the grouped RMSNorm + sigmoid gate pass"
                                    if args.gate_separate else "") +
                                   (" with FP8 E4M3 output (one fp32 scale per token-head)"
                                    if args.fp8 else "") +
                                   (f", context parallel over {world} rank(s): {N} tokens per "
                                    f"rank, state pass + all_gather + fold + prefill from the "
                                    f"folded state" if args.cp else "") +
                                   ("" if args.no_decode else
                                    f" + decode step B={Bd} H={Hd} d={dd} (fp32 state)") +
                                   (f", chunk C={args.chunk}" if args.chunk else "") +
                                   (f", {args.segments} segments per sequence"
                                    if args.segments else ""),
                       "global_batch": world * B if not args.cp else B,
                       "seq_len": N if not args.cp else N * world,
                       "parallelism": f"replicas{world}" if not args.cp else f"cp{world}",
                       "l2": "inputs larger than L2 (no flush)"},
            "prefill": {"ms": pre_ms_max, "tok_s": world * tokens / (pre_ms_max * 1e-3),
                        "tflops_canonical": world * canon / (pre_ms_max * 1e-3) / 1e12,
                        "tflops_executed": world * executed / (pre_ms_max * 1e-3) / 1e12,
                        "chunk": chunk,
                        "hbm_gbs": achieved},
            "decode": None if args.no_decode else {
                "ms": dec_ms_max, "state_gbs": dec_gbs, "frac_of_measured": dec_gbs / hbm_peak,
                "frac_of_8tbs": dec_gbs / 8000.0, "tokens_per_step": n_mtp,
                "tok_s": world * Bd * n_mtp / (dec_ms_max * 1e-3)},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak,
                         "traffic": (counters["dram_bytes_read"] + counters["dram_bytes_write"]
                                     if counters else None),
                         "algorithmic_bytes": pre_bytes,
                         "kernel": "chunked_prefill_kernel", "peak_kind": peak_kind,
                         # the tensor pipe of the same kernel: executed MMA flops per second
                         # against the measured bf16 burst peak, and ncu's pipe activity
                         "tensor_pipe": {
                             "executed_tflops": world * executed / (pre_ms_max * 1e-3) / 1e12,
                             "peak_tflops": tc_peak,
                             "frac": world * executed / (pre_ms_max * 1e-3) / 1e12 / tc_peak,
                             "chunk": chunk,
                             "ncu_pipe_tensor_active_pct": (
                                 counters["sm__pipe_tensor_cycles_active_pct_active"]
                                 if counters else None),
                             "ncu_pipe_tensor_elapsed_pct": (
                                 counters["sm__pipe_tensor_cycles_active_pct_elapsed"]
                                 if counters else None)}},
            "cp": None if not args.cp else {
                "state_fold_gather_ms": cp_ms_max, "step_ms": step_ms_max,
                # the state pass reads k and v of the part and writes the d x d states; the
                # time also holds the gather and the fold
                "state_step_hbm_gbs": (2 * B * N * H * d * 2 + B * H * d * d * 4) /
                (cp_ms_max * 1e-3) / 1e9},
            "qk_norm_rope": ({"in_prefill_kernel": True} if args.qk_fused else
                             None if qk is None else {
                "ms": qk_ms_max,
                # read q, k (raw) and write q_hat, k_hat: 4 * d * 2 bytes per token-head
                "hbm_gbs": 8 * B * N * H * d / (qk_ms_max * 1e-3) / 1e9}),
            "cpu_baseline": cpu,
            "clocks": clk.summary(),
            "e2e": e2e,
            # per step: the prefill kernel (after the planning kernel for packed input) and the
            # decode kernel
            # (context parallel: the state pass, its combine kernel when a head is split over
            # CTAs, and the fold)
            "gpu_launches": ((2 if packed else 1) + (0 if args.no_decode else 1) +
                             (1 if qk is not None else 0) +
                             (1 if sep is not None else 0) +
                             (cp_launches(B, N, H) if args.cp else 0)) * K,
        }
        print(json.dumps(line), flush=True)
    dist_teardown(world)


# --------------------------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# --------------------------------------------------------------------------------------------
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np

    import oracle
    vw = synth.VARLEN_WORKLOADS.get(args.workload)
    w = synth.WORKLOADS[args.workload] if vw is None else synth.Workload(
        vw.name, 1, vw.T, vw.H, vw.d, vw.dtype, vw.dist, vw.seed)
    cores = oracle.num_threads()
    n_heads = cores
    n_tok = min(w.N, 4096)
    q, k, v = synth.draw_qkv(1, n_tok, n_heads, w.d, dist=w.dist, seed=w.seed, dtype=w.dtype)
    bits = [x.view(torch.int16).numpy().view(np.uint16) for x in (q, k, v)]
    sl = np.resize(synth.slopes(w.H).numpy(), n_heads).astype(np.float32)
    for _ in range(args.warmup):
        oracle.prefill(*bits, sl, nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.prefill(*bits, sl, nthreads=cores)
    dt = (time.perf_counter() - t0) / args.steps
    tok_s = n_heads * n_tok / dt / w.H
    sample = (f"fp64 oracle, {n_heads} heads x {n_tok} tokens of the {w.name} distribution per "
              f"step; tok/s = token-heads/s / H={w.H}")
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tok/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w.name}: B={w.B} N={w.N} H={w.H} d={w.d} (sampled)",
                       "global_batch": w.B, "seq_len": w.N, "parallelism": "host cores"},
            "cpu_baseline": {"value": tok_s, "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": sample, "affinity_cores": host_cpu()[0],
                             "cpu_model": host_cpu()[1]},
            "e2e": {"value": tok_s, "unit": "tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill_32k", "prefill_4k", "prefill_256k",
                                           "varlen_64k"],
                    default="prefill_32k")
    ap.add_argument("--mtp", type=int, default=1,
                    help="decode this many tokens per sequence per step (multi-token step)")
    ap.add_argument("--qk-rope", action="store_true",
                    help="run the QK RMSNorm + partial RoPE operator before each prefill")
    ap.add_argument("--qk-fused", action="store_true",
                    help="apply the QK RMSNorm + partial RoPE inside the prefill kernel "
                         "(la_prefill_varlen_qk on raw q, k)")
    ap.add_argument("--gate-separate", action="store_true",
                    help="run the grouped RMSNorm + sigmoid gate as its own pass after the prefill")
    ap.add_argument("--gate", action="store_true",
                    help="fuse the grouped RMSNorm + sigmoid gate into the prefill's output")
    ap.add_argument("--fp8", action="store_true",
                    help="with --gate-separate: store y as FP8 E4M3 with blockwise scales (the "
                         "quantize step before out_proj)")
    ap.add_argument("--cp", action="store_true",
                    help="context parallel: split each sequence over the ranks (state pass, "
                         "all_gather of the part states, fold, prefill from the folded state)")
    ap.add_argument("--chunk", type=int, default=0,
                    help="chunk length C of the tensor-core prefill (0: the library's default)")
    ap.add_argument("--segments", type=int, default=0,
                    help="segments per sequence (0: the library's automatic plan)")
    ap.add_argument("--no-decode", action="store_true",
                    help="time the prefill alone (no decode state on the device)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer e2e leg")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline leg")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
