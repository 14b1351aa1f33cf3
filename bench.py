#!/usr/bin/env python
"""Benchmark of one MLA decode layer-step through libmla's C ABI on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl mla|reference]

A step is one pass of the whole hot path over one batch: append the new token's latent row,
absorb the query, latent attention over every cached token, output projection (for the
12-layer running-model workload: all 12 layers). A workload whose sequences each bring a chunk
of several new tokens (``chunk`` > 1, e.g. production_b8_n4096_chunk128_bf16) runs the same
step for all of them with causal mla_prefill_attention in place of mla_decode_attention. Inputs (weights, caches, new hidden states)
are seeded synthetic data resident in HBM before timing. With N > 1 (torchrun, one process per
GPU) every rank runs its own replica of the workload: sequences are independent, so there is no
data-path collective; ``value`` aggregates the ranks and the time is the max over ranks.

One JSON line on rank 0. ``value`` is µs per layer-step of the whole job (step time divided by
layers and by N). ``e2e`` is the same metric with host buffers: the step's inputs copied from
pinned host memory and its output copied back inside the timed region. ``roofline`` reports
the dominant call, the attention call, against max(bytes / HBM, flops / tensor peak) with the
measured peaks. ``cpu_baseline`` times the fp64 oracle on a bounded sample (rank 0, N = 1).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA absorbed decode µs/layer, TFLOP/s & latent-cache GB/s vs B200 roofline"
UNIT = "us/layer-step"
DEFAULT_WORKLOAD = "production_b64_n4096_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dims_desc(d):
    return (f"d={d.d_model}, n_h={d.n_heads}, d_h={d.d_head}, d_c={d.d_c}, d_c'={d.d_cq}, d_R={d.d_rope}, "
            f"page={d.page_size}")


# ----------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            rows.append((ts, parts))
        inside = [r for r in rows if t0 <= r[0] <= t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "samples_under_load": 0,
                    "note": "no nvidia-smi sample fell inside the timed region"}
        sm = [float(p[0]) for _, p in inside if p[0].replace(".", "").isdigit()]
        mx = [float(p[1]) for _, p in inside if p[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, p in inside for i in range(4) if p[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside), "samples_under_load": len(inside)}


# ----------------------------------------------------------------------------------- CPU oracle
class OracleSample:
    """A bounded sample of the workload for the fp64 oracle, one layer: the first ``n`` sequences
    of a decode step, or the first ``n`` new tokens of sequence 0 of a multi-token step. ``frac``
    is the sample's share of the step's attended tokens (the oracle's cost is linear in them)."""

    def __init__(self, w, n, layer=0):
        import oracle as O
        from mla_latent_kv_42_b200 import synth
        self.O, self.w = O, w
        self.cached = synth.cached_lengths(w)
        self.W64 = {k: O.as64(v) for k, v in synth.weights(w, layer).items()}
        c = w.chunk
        total = float(np.sum(c * (self.cached + 1) + c * (c - 1) // 2))
        if c == 1:
            self.picks = list(range(min(n, w.batch)))
            self.k = len(self.picks)
            sub = self.cached[self.picks]
            self.attended = int(np.sum(sub + 1))
            self.h = O.as64(synth.hidden(w))[self.picks]
            self.what = f"{self.k} of {w.batch} sequences"
        else:
            self.picks = [0]
            self.k = min(n, c)
            sub = self.cached[:1]
            self.attended = int(sum(int(sub[0]) + i + 1 for i in range(self.k)))
            self.h = O.as64(synth.hidden(w, batch=w.batch * c))[:self.k]
            self.what = f"the first {self.k} of {c} new tokens of sequence 0 of {w.batch}"
        rows = synth.prefix_rows(w, sub, layer=layer, device="cpu")
        offs = np.concatenate([[0], np.cumsum(sub)])
        self.prefix = [O.as64(rows[offs[i]:offs[i + 1]]) for i in range(len(sub))]
        self.frac = self.attended / total

    def run(self):
        """Seconds for the naive oracle over the sample."""
        t = time.perf_counter()
        if self.w.chunk == 1:
            self.O.layer_step_naive(self.W64, self.h, self.prefix, self.w.dims)
        else:
            self.O.chunk_step_naive(self.W64, self.h, self.prefix, [self.k], self.w.dims)
        return time.perf_counter() - t


def cpu_baseline(w, target_s=12.0):
    """Time the naive oracle on a bounded sample (whole sequences, or the first new tokens of
    one sequence for a multi-token step); extrapolate to the step by attended tokens."""
    probe = OracleSample(w, 1)
    t1 = probe.run()
    n = max(1, min(w.batch if w.chunk == 1 else w.chunk, int(target_s / max(t1, 1e-3))))
    smp = OracleSample(w, n)
    t = smp.run()
    cores = len(os.sched_getaffinity(0))
    return {"value": t / smp.frac * 1e6, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": (f"naive fp64 oracle, one layer, {smp.what} (all heads, {smp.attended} attended tokens), "
                       f"extrapolated by attended tokens x{1 / smp.frac:.1f}; {t:.1f} s of CPU time")}


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands, on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from mla_latent_kv_42_b200 import synth
    w = synth.workload(args.workload)
    smp = OracleSample(w, 1)
    per = []
    for i in range(args.warmup + args.steps):
        t = smp.run()
        if i >= args.warmup:
            per.append(t / smp.frac)
    us = float(np.mean(per)) * 1e6
    cores = len(os.sched_getaffinity(0))
    sample = (f"naive fp64 oracle on {smp.what} each step (all heads, {smp.attended} attended tokens), "
              f"extrapolated by attended tokens to the whole step")
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": us * w.layers / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "layers": w.layers, "dims": dims_desc(w.dims)},
        "cpu_baseline": {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------- multi-rank helpers
def rank_workload(w, rank: int):
    """Each rank owns its own sequences: the same workload shape with a rank-specific seed."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 1000 * rank) if rank else w


def measured_decode_traffic(workload: str):
    """DRAM bytes (read + write) of one attention-kernel launch on this workload, from the table of
    ncu captures in profiles/decode_tc_traffic.txt (lines ``workload sha256-prefix bytes``), if the
    capture was taken with the kernel source as it is now; otherwise None."""
    import hashlib
    table = os.path.join(ROOT, "profiles", "decode_tc_traffic.txt")
    src = os.path.join(ROOT, "mla_latent_kv_42_b200", "csrc", "decode_tc.cuh")
    if not os.path.exists(table):
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    for line in open(table):
        parts = line.split()
        if len(parts) == 3 and not line.startswith("#") and parts[0] == workload and digest.startswith(parts[1]):
            return int(parts[2])
    return None


def max_over_ranks(values, device, world: int):
    """Element-wise MAX over ranks of per-rank device times (a plain list when world == 1)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_us_per_layer_step(ms_total: float, steps: int, layers: int, world: int) -> float:
    """µs per layer-step of the whole job: every rank advances its own batch one layer per layer-step."""
    return ms_total / steps * 1e3 / layers / world


# ----------------------------------------------------------------------------------- GPU arm
def run_mla(args):
    import torch
    import torch.distributed as dist

    import mla_latent_kv_42_b200 as M
    from mla_latent_kv_42_b200 import build, harness, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0 or not os.path.exists(M.library_path()):
        build.build()
    if world > 1:
        dist.barrier()
    M.load_library()

    w = rank_workload(synth.workload(args.workload), rank)
    d = w.dims
    cached = synth.cached_lengths(w)
    chunk = w.chunk                  # new tokens per sequence per step; > 1 runs mla_prefill_attention
    ix = harness.step_index(cached, device=dev, chunk=chunk)
    layers = [harness.make_layer(w, cached, layer=l, device=dev, spare_tokens=chunk) for l in range(w.layers)]
    B = w.batch
    T = B * chunk                    # new tokens per step
    h0 = synth.hidden(w, batch=T).to(dev)
    h = h0.clone()
    fp8 = w.cache == "fp8"           # FP8 latent cache: mla_append_kv_fp8 and mla_decode_attention_fp8
    if fp8 and chunk > 1:
        raise SystemExit(f"workload {w.name}: the FP8 cache serves decode steps")
    attn_call = (M.CALL_PREFILL_ATTENTION if chunk > 1 else M.CALL_DECODE_ATTENTION_FP8 if fp8
                 else M.CALL_DECODE_ATTENTION)
    append_call = M.CALL_APPEND_KV_FP8 if fp8 else M.CALL_APPEND_KV
    calls = (append_call, M.CALL_ABSORB_QUERY, attn_call, M.CALL_OUT_PROJ)
    fused = args.fused
    if fused and (chunk > 1 or fp8 or not M.layer_step_small_supported(d)):
        raise SystemExit(f"--fused: workload {w.name} is not a decode step with small-head dims")
    if fused:
        calls = (M.CALL_LAYER_STEP_SMALL,)
    ws = torch.empty(max(M.workspace_size(d, c, T, ix.max_seq_len) for c in calls), dtype=torch.uint8, device=dev)
    # per-step index input besides the positions: the attended lengths (decode) or each new
    # token's sequence (prefill)
    aux0 = ix.seq_idx if chunk > 1 else ix.seq_lens
    e = synth.storage_dtype(d)
    outs = [{"q": torch.empty((T, d.n_heads, d.D), dtype=e, device=dev),
             "o_lat": torch.empty((T, d.n_heads, d.d_c), dtype=e, device=dev),
             "lse": torch.empty((T, d.n_heads), dtype=torch.float32, device=dev),
             "u": torch.empty((T, d.d_model), dtype=e, device=dev)} for _ in layers]
    stream = torch.cuda.current_stream(dev)
    EV = lambda: torch.cuda.Event(enable_timing=True)
    call_ms = np.zeros(4)
    launches = [0]
    kernel_events = []

    def one_step(record=False, inp=None, outs_=None):
        x, pos, aux = inp if inp is not None else (h, ix.pos, aux0)
        seq_idx = aux if chunk > 1 else ix.seq_idx
        if fused:  # the whole layer step in one launch (mla_layer_step_small)
            for L, o in zip(layers, outs if outs_ is None else outs_):
                if record:
                    ev = [EV() for _ in range(5)]
                    ev[0].record(stream)
                M.layer_step_small(L.state, x, aux, ix.max_seq_len, ws=ws, out=o, stream=stream)
                if record:
                    for k in range(1, 5):
                        ev[k].record(stream)
                    pending.append(ev)
                launches[0] += M.last_launch_count(M.CALL_LAYER_STEP_SMALL)
                if len(layers) > 1:
                    x = x + o["u"]
            return o["u"]
        for L, o in zip(layers, outs if outs_ is None else outs_):
            st, w_ = L.state, L.state.w
            if record:
                ev = [EV() for _ in range(5)]
                ev[0].record(stream)
            (M.append_kv_fp8 if fp8 else M.append_kv)(d, x, w_["w_dkv_kr"], seq_idx, pos, st.block_table, st.pool,
                                                      ws=ws, stream=stream)
            n = M.last_launch_count(append_call)
            if record:
                ev[1].record(stream)
            M.absorb_query(d, x, w_["w_dq"], w_["w_uq_qr"], w_["w_uk"], pos, q_out=o["q"], ws=ws, stream=stream)
            n += M.last_launch_count(1)
            if record:
                ev[2].record(stream)
            if record:  # the attention kernel alone, apart from its planner and merge
                kev = [EV(), EV()]
                for x_ in kev:
                    x_.record(stream)
                M.set_decode_timing_events(kev[0], kev[1])
            if chunk > 1:
                M.prefill_attention(d, o["q"], st.pool, st.block_table, seq_idx, pos, ix.max_seq_len,
                                    o_lat=o["o_lat"], lse=o["lse"], ws=ws, stream=stream)
            else:
                (M.decode_attention_fp8 if fp8 else M.decode_attention)(
                    d, o["q"], st.pool, st.block_table, aux, ix.max_seq_len, o_lat=o["o_lat"], lse=o["lse"], ws=ws,
                    stream=stream)
            if record:
                M.set_decode_timing_events(None, None)
                kernel_events.append(kev)
            n += M.last_launch_count(attn_call)
            if record:
                ev[3].record(stream)
            M.out_proj(d, o["o_lat"], w_["w_uv"], w_["w_o"], u=o["u"], ws=ws, stream=stream)
            n += M.last_launch_count(3)
            if record:
                ev[4].record(stream)
                pending.append(ev)
            launches[0] += n
            if len(layers) > 1:
                x = x + o["u"]          # residual between layers (harness glue, torch)
        return o["u"]

    pending = []
    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize(dev)
    assert M.read_device_status(stream) == 0

    gpu_uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", local))
    if gpu_uuid and not gpu_uuid.startswith("GPU-") and len(gpu_uuid) == 36:
        gpu_uuid = "GPU-" + gpu_uuid
    sampler = ClockSampler(gpu_uuid if gpu_uuid else str(local))
    sampler.start()
    time.sleep(0.3)

    # ---- timed region: K steps, device time, barrier + synchronize on both sides. The K-step
    # region is repeated (at least 3 times, until about a second has been timed, so that the
    # clock sampler sees it) and the median repetition is reported; every rank runs the same number
    # of repetitions (the count is agreed from rank 0's first one).
    # With --flush-l2 every step runs cold: a 256 MiB write (twice L2) precedes it, outside its
    # own pair of events, and the region's time is the sum of the steps' times.
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if args.flush_l2 else None

    def timed_block():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        if flush_buf is not None:
            total = 0.0
            evs = []
            for _ in range(args.steps):
                flush_buf.fill_(1)
                a, b = EV(), EV()
                a.record(stream)
                one_step()
                b.record(stream)
                evs.append((a, b))
            torch.cuda.synchronize(dev)
            total = sum(a.elapsed_time(b) for a, b in evs)
        else:
            start, end = EV(), EV()
            start.record(stream)
            for _ in range(args.steps):
                one_step()
            end.record(stream)
            torch.cuda.synchronize(dev)
            total = start.elapsed_time(end)
        if world > 1:
            dist.barrier()
        return total

    pending.clear()
    t_wall0 = time.time()
    launches[0] = 0
    rep_ms = [timed_block()]
    n_timed_launches = launches[0]
    reps = int(min(args.max_reps, max(3, -(-args.min_timed_s * 1e3 // max(rep_ms[0], 1e-3)))))
    if world > 1:
        r_t = torch.tensor([reps], dtype=torch.int64, device=dev)
        dist.broadcast(r_t, 0)
        reps = int(r_t.item())
    while len(rep_ms) < reps:
        rep_ms.append(timed_block())
    t_wall1 = time.time()
    ms_total = float(np.median(rep_ms))

    # ---- per-call breakdown, a separate pass: events between the calls stop each call's first
    # kernel from launching early into the previous call's tail, so this pass runs a little
    # slower than the timed one; the decode call's time (for the roofline) comes from here
    launches[0] = 0
    for _ in range(args.steps):
        one_step(record=True)
    torch.cuda.synchronize(dev)
    launches[0] = n_timed_launches
    for ev in pending:
        for c in range(4):
            call_ms[c] += ev[c].elapsed_time(ev[c + 1])
    gpu_launches = launches[0]
    n_layer_steps = args.steps * len(layers)
    call_ms /= n_layer_steps
    kernel_ms = sum(k0.elapsed_time(k1) for k0, k1 in kernel_events) / n_layer_steps
    if fused:  # one launch per layer: the call is the kernel
        kernel_ms = call_ms[0]
        call_ms[2] = call_ms[0]

    # ---- e2e: host buffers through the public API (pinned h in, u out, inside the timed region)
    h_host = h0.cpu().pin_memory()
    pos_host = ix.pos.cpu().pin_memory()
    aux_host = aux0.cpu().pin_memory()
    u_host = torch.empty((T, d.d_model), dtype=e).pin_memory()
    if world > 1:
        dist.barrier()
    # Pipelined as a serving loop would run it: step k+1's inputs go up on a copy stream and
    # step k-1's result comes back while step k computes. Inputs are double-buffered (a buffer
    # is refilled once the step two earlier has finished with it) and so are the per-layer
    # outputs (a set is rewritten once its read-back has finished). Every step's copies lie
    # inside the timed region, which spans both streams.
    copy_stream = torch.cuda.Stream(dev)
    ins = [(torch.empty_like(h), torch.empty_like(ix.pos), torch.empty_like(aux0)) for _ in range(2)]
    outs_pp = [outs, [{k: torch.empty_like(v) for k, v in o.items()} for o in outs]]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    torch.cuda.synchronize(dev)
    s2, e2 = EV(), EV()
    s2.record(stream)
    copy_stream.wait_event(s2)

    def upload(k):
        with torch.cuda.stream(copy_stream):
            if k >= 2:
                copy_stream.wait_event(ev_done[k % 2])  # step k-2 no longer reads these buffers
            hb, pb, lb = ins[k % 2]
            hb.copy_(h_host, non_blocking=True)
            pb.copy_(pos_host, non_blocking=True)
            lb.copy_(aux_host, non_blocking=True)
            ev_in[k % 2].record(copy_stream)

    upload(0)
    for k in range(args.steps):
        if k + 1 < args.steps:
            upload(k + 1)
        stream.wait_event(ev_in[k % 2])
        if k >= 2:
            stream.wait_event(ev_out[k % 2])  # step k-2's result has been read back from this set
        u = one_step(inp=ins[k % 2], outs_=outs_pp[k % 2])
        ev_done[k % 2].record(stream)
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(ev_done[k % 2])
            u_host.copy_(u, non_blocking=True)
            ev_out[k % 2].record(copy_stream)
    for ev in ev_out:
        stream.wait_event(ev)
    e2.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms_e2e = s2.elapsed_time(e2)
    sampler.stop()
    assert M.read_device_status(stream) == 0

    # max over ranks
    ms_total, ms_e2e, decode_ms, kernel_ms = max_over_ranks([ms_total, ms_e2e, call_ms[2], kernel_ms], dev, world)

    if rank == 0:
        peaks, peak_src = load_peaks()
        ms_step = ms_total / args.steps
        us_layer_job = job_us_per_layer_step(ms_total, args.steps, len(layers), world)
        us_e2e_job = job_us_per_layer_step(ms_e2e, args.steps, len(layers), world)
        dbytes, dflops = harness.attention_work(d, cached, chunk, w.cache)
        sbytes, sflops = harness.layer_work(d, cached, chunk, w.cache)
        if fused:  # the fused kernel does the whole layer: its roofline is the layer's
            dbytes, dflops = sbytes, sflops
        dec_s = decode_ms * 1e-3    # the whole call: planner + attention kernel + merge
        ker_s = kernel_ms * 1e-3    # the attention kernel alone (events around its launch)
        t_mem = dbytes / (peaks["hbm_gbs"] * 1e9)
        t_flop = dflops / (peaks["bf16_tflops"] * 1e12)
        if t_mem >= t_flop:
            roof = {"bound": "hbm", "achieved": dbytes / ker_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
            call_frac = dbytes / dec_s / 1e9 / peaks["hbm_gbs"]
        else:
            roof = {"bound": "tensor", "achieved": dflops / ker_s / 1e12, "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s"}
            call_frac = dflops / dec_s / 1e12 / peaks["bf16_tflops"]
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["frac_whole_call"] = call_frac  # counting the planner and merge launches too
        roof["traffic"] = measured_decode_traffic(w.name)
        roof["kernel"] = ("k_layer_small (mla_layer_step_small: the whole layer step in one launch)" if fused
                          else "attention kernel of mla_decode_attention_fp8 (k_decode_tc with the FP8 converting "
                               "warps)" if fp8
                          else "attention kernel of mla_prefill_attention (k_decode_tc, one item per new token)"
                          if chunk > 1 else "attention kernel of mla_decode_attention (k_decode_tc; warp-MMA "
                                            "k_decode_mma at small n_h)")
        roof["kernel_us"] = kernel_ms * 1e3
        roof["peak_source"] = peak_src + " (burst; MEASURED_PEAKS.json)" if peak_src == "measured" else peak_src
        roof["roofline_us"] = max(t_mem, t_flop) * 1e6
        roof["algorithmic_bytes"] = dbytes
        roof["algorithmic_flops"] = dflops
        step_s = ms_step * 1e-3 / len(layers)
        line = {
            "metric": METRIC, "value": us_layer_job, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if d.dtype == "bf16" else "fp16", "data": "synthetic",
            "config": {"workload": w.name, "batch": B, "cached_tokens": (int(cached[0]) if not w.ragged else
                                                                         f"U[{w.cached[0]},{w.cached[1]}], sum "
                                                                         f"{int(cached.sum())}"),
                       "layers": len(layers), "dims": dims_desc(d), "paging": w.paging,
                       **({"cache": "fp8 e4m3 rows + (s_c, s_r) float32 per token, 584 B"} if fp8 else {}),
                       **({"chunk": chunk, "new_tokens": T} if chunk > 1 else {}),
                       "path": ("one launch per layer (mla_layer_step_small)" if fused else
                                "four C-ABI calls per layer"),
                       "l2": ("flushed before every step (256 MiB write, outside the step's events)" if args.flush_l2
                              else "inputs larger than L2" if sbytes > 126e6 else "L2 not flushed (inputs below L2)"),
                       "parallelism": f"replicas x{world} (sequence-independent, no collective)",
                       "timed_reps": len(rep_ms),
                       "timing": (f"median of {len(rep_ms)} repetitions of the {args.steps}-step timed region "
                                  f"(min {min(rep_ms) / args.steps * 1e3 / len(layers):.1f}, max "
                                  f"{max(rep_ms) / args.steps * 1e3 / len(layers):.1f} us per layer-step)")},
            "tflops": sflops / step_s / 1e12,
            "cache_gbs": dbytes / dec_s / 1e9,
            "decode_us": decode_ms * 1e3,
            "decode_kernel_us": kernel_ms * 1e3,
            "per_call_us": ({"layer_step_small": call_ms[0] * 1e3} if fused else
                            {"append_kv": call_ms[0] * 1e3, "absorb_query": call_ms[1] * 1e3,
                             ("prefill_attention" if chunk > 1 else "decode_attention"): call_ms[2] * 1e3,
                             "out_proj": call_ms[3] * 1e3}),
            "layer_step_roofline_us": max(sbytes / (peaks["hbm_gbs"] * 1e9), sflops / (peaks["bf16_tflops"] * 1e12))
            * 1e6,
            "roofline": roof,
            "e2e": {"value": us_e2e_job, "unit": UNIT,
                    "h2d_bytes_per_step": int(h0.numel() * 2 + ix.pos.numel() * 4 + aux0.numel() * 4),
                    "d2h_bytes_per_step": int(T * d.d_model * 2)},
            "gpu_launches": int(gpu_launches),
            "clocks": sampler.summary(t_wall0 - 0.1, t_wall1 + 0.1),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["mla", "reference"], default="mla")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--min-timed-s", type=float, default=1.0,
                    help="repeat the K-step timed region until this many seconds are timed (at least 3 times)")
    ap.add_argument("--max-reps", type=int, default=1000)
    ap.add_argument("--flush-l2", action="store_true", help="write 256 MiB before every timed step (cold L2)")
    ap.add_argument("--fused", action="store_true",
                    help="small-head decode workloads: the whole layer step in one launch (mla_layer_step_small)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)     # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_mla(args)


if __name__ == "__main__":
    sys.exit(main())
