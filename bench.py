#!/usr/bin/env python
"""Decode throughput over a DepthWeave-KV compressed KV cache on B200.

Workload (default ``llama8b_64k``): Llama-3-8B attention shapes -- 32 layers in 16
two-layer groups, 32 query heads / 8 kv heads, head_dim 128, batch 1, 64K context;
bases r_max = 64 per (group, kv-head, K/V); tiers {16, 32, 64} with probabilities
0.6 / 0.3 / 0.1; residual s = 16 int4 channels with an fp16 scale.  The cache holds
65535 compressed tokens (synthetic, seeded, imported before timing).  One step = for
each of the 32 layers one launch of dwkv_append_decode_attention: encode + append the
step's new token of every sequence, then fused decode attention over each whole context.
Metric: decode tokens/s (batch / step time) and the compressed-KV bytes/s of the decode
kernel against the measured HBM copy bandwidth.  Attention only (no projections / MLP: no
weights exist).  ``--workload llama8b_ragged_b8`` (8 sequences of 16K-32K tokens, int8) and
``--workload llama8b_131k_deep`` (131072 tokens, 4-layer groups, r_max 128) run the same
step on the other decode workloads.

Timing: W warm-up steps, then K steps captured in one CUDA graph and replayed once,
bracketed by a barrier + synchronize, timed with CUDA events; max over ranks.  Each
step streams GBs of pages (> 126 MB L2), so no L2 flush is needed.  Every launch in the
timed region is the fused decode kernel, so its average launch duration is the region's
time over its launches (the roofline); a second replay with an external event around every
launch is reported beside it.  Decode launches overlap their predecessor (programmatic
dependent launch) unless ``--no-overlap``.  The probe (dwkv_probe, one launch per layer) is
timed over the same cache after the steps.  ``e2e`` repeats the step with host (pinned)
inputs copied in (one block a step) and the outputs copied out inside the timed region.
``step_distribution`` gives the median / p90 of up to 50 steps timed one by one (an event
node between steps) and the eager (no graph) time of a step.  Clocks: nvidia-smi every 20 ms
and NVML every ~1 ms during the timed region.

The default single-GPU run also measures, in fewer steps, the ragged batch-8 and 131K
workloads and the bulk encode (below), each with its own roofline, e2e and CPU baseline,
under ``workloads`` in the same JSON line (``--headline-only`` skips them).

``--workload llama8b_encode_16k`` measures bulk encode instead: 4 sequences x 16384 new
dense tokens per layer through dwkv_append (32 layers a step, the sequences reset between
steps), then one decode step and one probe pass over the encoded cache.

``cpu_baseline`` / ``--impl reference``: the CPU oracle (plain fp64 C) on every host core,
OpenMP over (layer, kv-head) problems of sequence 0 at its full context (at least one problem
per core), scaled to the whole step.

Multi-GPU (torchrun): every rank runs an independent replica (the path shards by
sequence with no exchange); value = total tokens of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode tok/s at 64K (8B shapes); compressed-KV HBM GB/s, % of peak"
UNIT = "tok/s"


def dense_kv_bytes(layers: int, kv_heads: int, head_dim: int, tokens: int, elem_bytes: int = 2) -> int:
    """Bytes of an uncompressed KV cache: 2 (K and V) x layers x heads x dim x tokens x bytes."""
    return 2 * layers * kv_heads * head_dim * tokens * elem_bytes


def token_bytes(rank: int, s: int, bits: int, coeff_bits: int = 16) -> int:
    """Stored bytes of one token of one (layer, kv-head), keys + values: the coefficients (bf16,
    or 8-bit codes with an fp16 scale per block of 16), s indices, s codes, one fp16 scale."""
    cb = rank + rank // 8 if coeff_bits == 8 else 2 * rank
    return 2 * (cb + s + s * bits // 8 + 2)


def tier_counts_of(wl) -> list:
    """Residual channels a token of each tier keeps."""
    return list(wl.tier_resid) if wl.tier_resid else [wl.resid_channels] * len(wl.tiers)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("dwkv_decode.cuh", "dwkv_common.cuh", "dwkv_encode.cuh"):
        h.update(open(os.path.join(ROOT, "decode_attention_depthweave_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken on the
    current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", f"decode_{workload}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_source_sha") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 20 ms; summary() keeps the
    samples that fall inside the marked region (wall clock)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, uuid: str | None = None):
        self.gpu = gpu_index
        self.uuid = uuid
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None
        self.nvml = []                  # (t, sm_mhz, max_mhz, reasons bitmask) every ~1 ms
        self._stop = None
        self._thread = None

    def _nvml_loop(self):
        """SM clock and clock-event reasons read through NVML about every millisecond, so that
        a timed region of a few tens of ms still holds many samples."""
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                hd = pynvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid else None
            except pynvml.NVMLError:
                hd = None
            if hd is None:
                hd = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(hd, pynvml.NVML_CLOCK_SM)
            reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            while not self._stop.is_set():
                self.nvml.append((time.time(), pynvml.nvmlDeviceGetClockInfo(hd, pynvml.NVML_CLOCK_SM), mx,
                                  int(reasons(hd)) if reasons else 0))
                time.sleep(0.001)
        except Exception:              # no NVML: the nvidia-smi samples stand alone
            pass

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # nvidia-smi's first query can take a while on a fresh box: start timing only once
        # it is sampling, so its start-up never overlaps the timed region
        t_end = time.time() + 10.0
        while self.proc is not None and time.time() < t_end:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)
        import threading
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._nvml_loop, daemon=True)
        self._thread.start()
        time.sleep(0.2)
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        import datetime
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
            os.unlink(self.path)

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        def ts(x):
            try:
                return datetime.datetime.strptime(x, "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                return None

        inside = [r for r in rows if self.t0 and ts(r[0]) is not None and self.t0 - 0.01 <= ts(r[0]) <= self.t1 + 0.01]
        use = inside if inside else rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        # NVML reason bits of the same four events (nvmlClocksEventReason*)
        bits = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}
        nv_in = [x for x in self.nvml if self.t0 and self.t0 <= x[0] <= self.t1]
        if not use and not nv_in:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [num(r[2]) for r in use if num(r[2]) is not None]
        mx = [num(r[3]) for r in use if num(r[3]) is not None]
        reasons = {names[i] for r in use for i in range(4) if r[6 + i].lower().startswith("active")}
        if nv_in:
            sm = [float(x[1]) for x in nv_in]
            mx = mx + [float(x[2]) for x in nv_in]
            reasons |= {n for n in names for x in nv_in if x[3] & bits[n]}
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(use) + len(nv_in),
                "samples_in_region": len(inside) + len(nv_in),
                "sources": {"nvidia_smi_20ms_in_region": len(inside), "nvml_1ms_in_region": len(nv_in)}}


# ----------------------------------------------------------------------------- dist
def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:                                        # host-side runs of the same plumbing
            dist.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value: float) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (ms * 1e-3)


# ----------------------------------------------------------------------------- oracle sample
def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_oracle_sample(wl, probs_in, threads):
    """Time the CPU oracle on the given (layer, kv-head) problems on ``threads`` host threads.
    ``probs_in`` is a list of (bases, tier_idx, comp, q, layer, head).  Returns wall seconds."""
    import oracle
    items = [oracle.head_problem(wl, b, t, c, q, layer, h) for (b, t, c, q, layer, h) in probs_in]
    t0 = time.perf_counter()
    oracle.decode_many(items, nthreads=threads)
    return time.perf_counter() - t0


def oracle_layers_for(wl, cores: int) -> int:
    """Layers whose kv-heads give every host core at least one (layer, kv-head) problem."""
    return max(1, min(wl.num_layers, -(-cores // wl.num_kv_heads)))


# ----------------------------------------------------------------------------- main path
def run_dwkv(args, world, rank, local, workload=None, steps=None, warmup=None, e2e_steps=None, light=False):
    """One decode workload: import the synthetic compressed cache of every sequence, then time
    K steps of (per layer) one fused append + decode launch over all sequences.  ``light``
    skips the per-step distribution and the event-bracketed replay (extra workloads of the
    default run)."""
    import torch

    import decode_attention_depthweave_b200 as dw
    import synth

    name = workload or args.workload
    steps = args.steps if steps is None else steps
    warmup = args.warmup if warmup is None else warmup
    e2e_steps = args.e2e_steps if e2e_steps is None else e2e_steps
    wl = synth.workload(name)
    if args.layers:
        wl = wl.scaled(num_layers=args.layers)
    dev = torch.device("cuda", local)
    B = wl.batch
    lengths = [args.context] * B if args.context else synth.make_context_lengths(wl)
    seqs = list(range(B))
    sid = [rank * B + b for b in seqs]                 # seed index of each sequence (replicas differ)
    n_steps = warmup + steps + e2e_steps
    n_dist = 0 if light else min(steps, 50)           # steps timed one by one (median / p90)
    n_eager = 0 if light else 5                        # steps launched without a graph
    prof_steps = 0 if light else args.profile_steps
    extra = prof_steps + n_dist + n_eager + 64
    bases = synth.make_bases(wl)
    cfg = dw.config_from(num_layers=wl.num_layers, layers_per_group=wl.layers_per_group,
                         num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim,
                         r_max=wl.r_max, tiers=wl.tiers, resid_channels=wl.resid_channels,
                         resid_bits=wl.resid_bits, max_batch=B, max_context=max(lengths) + n_steps + extra,
                         tier_resid=wl.tier_resid or None, coeff_bits=wl.coeff_bits)
    stream = torch.cuda.Stream(device=dev)
    cache = dw.Cache(cfg, bases[0], bases[1], device=dev, ws_seqs=B, stream=stream)
    if args.tuning:
        c, w_, s_ = (int(x) for x in args.tuning.split(","))
        cache.set_decode_tuning(c, w_, s_)
    cache.set_decode_overlap(not args.no_overlap)
    h = cache.h
    lpg = wl.layers_per_group

    # ---- import the T_b - 1 cached tokens of every sequence (seeded synthetic compressed form)
    do_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    cores = os.cpu_count() or 1
    keep_layers = set(range(oracle_layers_for(wl, cores))) if do_cpu else set()
    comp_cpu, tiers_cpu = {}, {}
    tier_counts = torch.zeros(len(wl.tiers), dtype=torch.int64)
    with torch.cuda.stream(stream):
        for b in seqs:
            tiers_dev = {}
            for layer in range(wl.num_layers):
                g = layer // lpg
                if g not in tiers_dev:
                    tiers_dev[g] = synth.make_tiers(wl, sid[b], g, lengths[b] - 1, device=dev)
                    tier_counts += torch.bincount(tiers_dev[g].reshape(-1).long(), minlength=len(wl.tiers)).cpu()
                comp = synth.make_compressed(wl, sid[b], layer, tiers_dev[g], device=dev)
                coeff = (comp["ccodes"], comp["cscales"]) if "ccodes" in comp else comp["coeff"]
                cache.append_compressed(layer, [b], [lengths[b] - 1], tiers_dev[g], coeff, comp["idx"],
                                        comp["codes"], comp["scales"], stream=stream)
                if b == 0 and layer in keep_layers:
                    comp_cpu[layer] = {k: v.cpu() for k, v in comp.items()}
                    tiers_cpu[layer] = tiers_dev[g].cpu()
                del comp
            del tiers_dev
    cache.sync(stream)

    # ---- per-step inputs of every sequence, resident in HBM: [steps][B][...]
    Kn, Vn, Qs, Tn = [], [], [], {}
    for layer in range(wl.num_layers):
        kv = [synth.make_dense_vectors(wl, sid[b], layer, n_steps, bases, device=dev, start=lengths[b] - 1)
              for b in seqs]
        Kn.append(torch.stack([x[0] for x in kv], 1).contiguous())
        Vn.append(torch.stack([x[1] for x in kv], 1).contiguous())
        del kv
        Qs.append(synth.make_queries(wl, layer, batch=n_steps * B, device=dev, step=rank)
                  .view(n_steps, B, wl.num_q_heads, wl.head_dim))
        g = layer // lpg
        if g not in Tn:
            Tn[g] = torch.stack([synth.make_tiers(wl, sid[b], g, n_steps, device=dev, start=lengths[b] - 1)
                                 for b in seqs], 1).contiguous()
            tier_counts += torch.bincount(Tn[g][: warmup + steps].reshape(-1).long(), minlength=len(wl.tiers)).cpu()
    out = torch.empty(wl.num_layers, B, wl.num_q_heads, wl.head_dim, dtype=torch.float32, device=dev)
    ws = cache.workspace

    def step(s, ev=None):
        # per layer, one launch: append the step's token of every sequence and attend over
        # each sequence's whole context
        for layer in range(wl.num_layers):
            g = layer // lpg
            if ev is not None:
                ev[layer][0].record(stream)
            dw.dwkv_append_decode_attention(h, layer, seqs, Kn[layer][s], Vn[layer][s],
                                            Tn[g][s] if layer % lpg == 0 else None, Qs[layer][s], out[layer], ws,
                                            stream)
            if ev is not None:
                ev[layer][1].record(stream)

    launches_per_step = wl.num_layers                          # one fused append + decode per layer

    # ---- warm-up (graph of W steps, replayed once)
    torch.cuda.synchronize(dev)
    g_warm = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, stream=stream):
        for s in range(warmup):
            step(s)
    with torch.cuda.stream(stream):
        g_warm.replay()
    torch.cuda.synchronize(dev)
    cache.sync(stream)

    # ---- timed: K steps in one graph, replayed once
    g_main = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_main, stream=stream):
        for s in range(warmup, warmup + steps):
            step(s)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local, gpu_uuid(local)) as clk:
        clk.mark_start()
        with torch.cuda.stream(stream):
            e0.record(stream)
            g_main.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
    barrier(world)
    ms_total = e0.elapsed_time(e1)
    cache.sync(stream)
    ms_total = max_over_ranks(world, ms_total)
    ms_per_step = ms_total / steps
    clocks = clk.summary()
    del g_warm

    # ---- per-launch durations bracketed by CUDA events, for reference (re-running the timed
    #      steps appends more tokens, which changes the work by < 0.1 %).  The event nodes
    #      between launches add their own gaps, so the roofline below uses the timed region.
    dec_ms_mean = None
    if prof_steps:
        evs = [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
                for _ in range(wl.num_layers)] for _ in range(prof_steps)]
        g_prof = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_prof, stream=stream):
            for i in range(prof_steps):
                step(warmup + i, evs[i])
        with torch.cuda.stream(stream):
            g_prof.replay()
        torch.cuda.synchronize(dev)
        dec_ms = [evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(prof_steps) for l in range(wl.num_layers)]
        dec_ms_mean = statistics.mean(dec_ms)

    # ---- probe (with / without residual, one launch per layer) over the same cache
    err = torch.empty(wl.num_layers, B, wl.num_kv_heads, dtype=torch.float32, device=dev)
    g_probe = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_probe, stream=stream):
        for layer in range(wl.num_layers):
            dw.dwkv_probe(h, layer, seqs, Qs[layer][warmup], err[layer], None, ws, stream)
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    probe_reps = max(prof_steps, 1)
    with torch.cuda.stream(stream):
        g_probe.replay()
        p0.record(stream)
        for _ in range(probe_reps):
            g_probe.replay()
        p1.record(stream)
    torch.cuda.synchronize(dev)
    cache.sync(stream)
    assert torch.isfinite(err).all()
    probe_launch_ms = p0.elapsed_time(p1) / (probe_reps * wl.num_layers)
    held_probe = sum(lengths) - B + B * (warmup + steps + prof_steps)

    # ---- algorithmic bytes: every stored byte of the attended tokens (per-token bytes of
    #      its tier), plus the two bases, the queries and the outputs of each launch
    held = sum(lengths) - B + B * (warmup + steps)            # tokens per head after the timed steps
    tok_bytes = torch.tensor([token_bytes(r, n, wl.resid_bits, wl.coeff_bits) for r, n in zip(wl.tiers, tier_counts_of(wl))],
                             dtype=torch.float64)
    bytes_per_tok_head = float((tier_counts.double() * tok_bytes).sum()) / (wl.num_groups * wl.num_kv_heads * held)
    basis_bytes = 2 * wl.num_kv_heads * wl.head_dim * wl.r_max * 2
    io_bytes = B * wl.num_q_heads * wl.head_dim * (2 + 4)

    def layer_bytes(ctx):
        return bytes_per_tok_head * wl.num_kv_heads * ctx + basis_bytes + io_bytes

    ctx_timed = sum(lengths) - B + B * (warmup + (steps + 1) / 2.0)   # attended tokens of all sequences, mean over the timed steps
    comp_bytes_layer = bytes_per_tok_head * wl.num_kv_heads * ctx_timed
    peaks = measured_peaks()
    # the timed region holds nothing but the fused decode kernel (one launch per layer): its
    # average launch duration, inter-launch gaps included, is the region's time over its launches
    launch_ms = ms_per_step / launches_per_step
    alg_bytes = layer_bytes(ctx_timed)
    achieved = alg_bytes / (launch_ms * 1e-3) / 1e9
    traffic = profiled_traffic(name)
    probe_bytes = layer_bytes(held_probe) - B * wl.num_q_heads * wl.head_dim * 4 + B * wl.num_kv_heads * 4

    # ---- e2e: host inputs in, host outputs out, one step per graph replay
    e2e = None
    if e2e_steps > 0:
        s0 = warmup + steps
        sK = torch.stack([Kn[l][s0:] for l in range(wl.num_layers)], 1)
        sV = torch.stack([Vn[l][s0:] for l in range(wl.num_layers)], 1)
        sQ = torch.stack([Qs[l][s0:] for l in range(wl.num_layers)], 1)
        sT = torch.stack([Tn[g][s0:] for g in range(wl.num_groups)], 1)
        # one pinned host block per step (K | V | Q | tiers, each 16-byte aligned), one copy in
        host_in, offs, sizes = pack_step_inputs((sK, sV, sQ, sT))
        del sK, sV, sQ, sT
        host_in = host_in.pin_memory()
        # two staging / output buffer pairs, one graph each: step i's inputs go in (copy stream
        # h2d) while step i - 1 computes, and its outputs come out (copy stream d2h) while step
        # i + 1 computes; every step's copies stay inside the timed region
        shp = lambda *t: (wl.num_layers,) + t                                       # noqa: E731
        outs = [out, torch.empty_like(out)]
        stages, graphs = [], []
        for b in range(2):
            stage = torch.empty(host_in.shape[1], dtype=torch.uint8, device=dev)
            dK = stage[offs[0]:offs[0] + sizes[0]].view(torch.bfloat16).view(shp(B, wl.num_kv_heads, wl.head_dim))
            dV = stage[offs[1]:offs[1] + sizes[1]].view(torch.bfloat16).view(shp(B, wl.num_kv_heads, wl.head_dim))
            dQ = stage[offs[2]:offs[2] + sizes[2]].view(torch.bfloat16).view(shp(B, wl.num_q_heads, wl.head_dim))
            dT = stage[offs[3]:offs[3] + sizes[3]].view(wl.num_groups, B, wl.num_kv_heads)
            g_e2e = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_e2e, stream=stream):
                for layer in range(wl.num_layers):
                    g = layer // lpg
                    dw.dwkv_append_decode_attention(h, layer, seqs, dK[layer], dV[layer],
                                                    dT[g] if layer % lpg == 0 else None, dQ[layer], outs[b][layer],
                                                    ws, stream)
            stages.append(stage)
            graphs.append(g_e2e)
        host_out = torch.empty((e2e_steps,) + tuple(out.shape), dtype=torch.float32).pin_memory()
        h2d_stream = torch.cuda.Stream(device=dev)
        d2h_stream = torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        torch.cuda.synchronize(dev)
        barrier(world)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        go = torch.cuda.Event()
        a0.record(stream)
        go.record(stream)
        h2d_stream.wait_event(go)
        d2h_stream.wait_event(go)

        def copy_in(i):
            b = i % 2
            if i >= 2:
                h2d_stream.wait_event(ev_done[b])          # graph i - 2 has read stage b
            with torch.cuda.stream(h2d_stream):
                stages[b].copy_(host_in[i], non_blocking=True)
            ev_in[b].record(h2d_stream)

        copy_in(0)
        with torch.cuda.stream(stream):                     # graphs replay on the current stream
            for i in range(e2e_steps):
                b = i % 2
                if i + 1 < e2e_steps:
                    copy_in(i + 1)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])            # outputs of step i - 2 are out
                graphs[b].replay()
                ev_done[b].record(stream)
                d2h_stream.wait_event(ev_done[b])
                with torch.cuda.stream(d2h_stream):
                    host_out[i].copy_(outs[b], non_blocking=True)
                ev_out[b].record(d2h_stream)
            stream.wait_stream(d2h_stream)
            stream.wait_stream(h2d_stream)
            a1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        e2e_ms = max_over_ranks(world, a0.elapsed_time(a1)) / e2e_steps
        h2d = host_in.shape[1]
        d2h = out.numel() * 4
        assert torch.isfinite(host_out).all()
        e2e = {"value": round(aggregate_rate(world, B, e2e_ms), 2), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e2e_ms, 4),
               "timing": "pinned host inputs in and fp32 outputs out every step on two copy streams, "
                         "double-buffered so step i's copies overlap steps i - 1 / i + 1; CUDA events "
                         "around all steps"}
        del graphs
    cache.sync(stream)

    # ---- per-step distribution (one graph of n_dist steps, an event between steps) and the
    #      eager time (the same launches without a graph); inputs of the timed steps reused
    dist = None
    if n_dist > 0:
        sev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_dist + 1)]
        g_dist = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_dist, stream=stream):
            for i in range(n_dist):
                sev[i].record(stream)
                step(warmup + i % steps)
            sev[n_dist].record(stream)
        with torch.cuda.stream(stream):
            g_dist.replay()
        torch.cuda.synchronize(dev)
        per = sorted(sev[i].elapsed_time(sev[i + 1]) for i in range(n_dist))
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for i in range(n_eager):
                step(warmup + i % steps)
            ev1.record(stream)
        torch.cuda.synchronize(dev)
        cache.sync(stream)
        dist = {"steps": n_dist, "ms_p50": round(statistics.median(per), 5),
                "ms_p90": round(per[min(n_dist - 1, int(math.ceil(0.9 * n_dist)) - 1)], 5),
                "ms_min": round(per[0], 5), "ms_max": round(per[-1], 5),
                "eager_ms_per_step": round(ev0.elapsed_time(ev1) / n_eager, 5),
                "timing": f"graph of the steps with an event node between steps; eager: {wl.num_layers} launches a "
                          "step from Python, no graph"}

    # ---- CPU oracle baseline (rank 0, N = 1 only): every kv-head of the first layers of
    #      sequence 0 at its full context, one problem per host core, scaled to the step
    cpu = None
    if do_cpu and comp_cpu:
        probs_in = [(bases, tiers_cpu[l], comp_cpu[l], Qs[l][warmup][0].cpu(), l, hh)
                    for l in sorted(comp_cpu) for hh in range(wl.num_kv_heads)]
        dt = cpu_oracle_sample(wl, probs_in, cores)
        scale = (wl.num_layers * wl.num_kv_heads / len(probs_in)) * (sum(lengths) - B) / (lengths[0] - 1)
        step_s = dt * scale
        dt1 = cpu_oracle_sample(wl, probs_in[:1], 1)
        step1_s = dt1 * wl.num_layers * wl.num_kv_heads * (sum(lengths) - B) / (lengths[0] - 1)
        cpu = {"value": round(B / step_s, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"sequence 0, layers 0-{len(comp_cpu) - 1} x {wl.num_kv_heads} kv-heads = {len(probs_in)} "
                         f"problems of {lengths[0] - 1} cached tokens (fp64 C oracle, OpenMP over the problems, "
                         f"{dt:.1f} s wall on {cores} threads), scaled x{scale:.2f} to one step of all "
                         f"{B} sequence(s) and {wl.num_layers} layers",
               "single_thread_value": round(B / step1_s, 6),
               "single_thread_sample": f"one problem (layer 0, kv-head 0, {lengths[0] - 1} tokens) on 1 thread "
                                       f"({dt1:.1f} s), scaled to the step",
               "nproc": cores, "cpu_model": cpu_model()}

    value = aggregate_rate(world, B, ms_per_step)
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 storage, fp32 math",
        "data": "synthetic (seeded compressed cache; no model weights)",
        "config": {"workload": name, "layers": wl.num_layers, "groups": wl.num_groups,
                   "q_heads": wl.num_q_heads, "kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                   "batch_per_gpu": B, "context": lengths[0] if B == 1 else lengths, "r_max": wl.r_max,
                   "tiers": list(wl.tiers), "tier_probs": list(wl.tier_probs), "resid_channels": wl.resid_channels,
                   **({"tier_resid": list(wl.tier_resid)} if wl.tier_resid else {}),
                   **({"coeff_bits": wl.coeff_bits} if wl.coeff_bits != 16 else {}),
                   "resid_bits": wl.resid_bits, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2 (~{comp_bytes_layer * wl.num_layers / 1e9:.1f} GB of pages per step); "
                         "no flush",
                   "graph": "CUDA graph of K steps, replayed once",
                   "launch_overlap": not args.no_overlap},
        "gpu_launches": launches_per_step * steps,
        "compressed_gb_per_step": round(comp_bytes_layer * wl.num_layers / 1e9, 4),
        "compressed_tb_s": round(comp_bytes_layer * wl.num_layers / (ms_per_step * 1e-3) / 1e12, 4),
        "dense_bf16_gb_per_step": round(dense_kv_bytes(wl.num_layers, wl.num_kv_heads, wl.head_dim, int(ctx_timed)) / 1e9, 4),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": traffic, "kernel": f"dwkv::decode_kernel<{wl.resid_bits},false>",
                     "alg_bytes_per_launch": int(alg_bytes), "launch_ms": round(launch_ms, 5),
                     "launch_ms_source": "timed region / launches (CUDA events on the launching stream)",
                     "launch_ms_bracketed": None if dec_ms_mean is None else round(dec_ms_mean, 5),
                     "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, copy)",
                     "frac_of_8tbs_spec": round(achieved / 8000.0, 4)},
        "probe": {"kernel": f"dwkv::decode_kernel<{wl.resid_bits},true>", "launch_ms": round(probe_launch_ms, 5),
                  "context": held_probe,
                  "achieved_gbs": round(probe_bytes / (probe_launch_ms * 1e-3) / 1e9, 1),
                  "frac": round(probe_bytes / (probe_launch_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                  "timing": f"graph of {wl.num_layers} probe launches, {probe_reps} replay(s) after one warm-up"},
        "step_distribution": dist,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    cache.close()
    del cache, Kn, Vn, Qs, Tn, out, err, g_main, g_probe
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return res


def gpu_uuid(local: int):
    """NVML-style UUID of cuda:local (for the clock sampler), or None."""
    try:
        import torch
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


def pack_step_inputs(tensors):
    """Per-step inputs packed for one host -> device copy a step: ``tensors`` are [steps, ...]
    arrays of any dtype; returns (uint8 [steps, bytes] block, offsets, sizes), every part at a
    16-byte-aligned offset (the library's alignment rule for k_new / v_new)."""
    import torch
    parts = [x.reshape(x.shape[0], -1).contiguous().view(torch.uint8) for x in tensors]
    sizes = [x.shape[1] for x in parts]
    offs = [0]
    for n_ in sizes[:-1]:
        offs.append(offs[-1] + (n_ + 15) // 16 * 16)
    block = torch.zeros(parts[0].shape[0], offs[-1] + sizes[-1], dtype=torch.uint8)
    for x, o, n_ in zip(parts, offs, sizes):
        block[:, o:o + n_] = x.cpu()
    return block, offs, sizes


def fp32_alu_peak_tflops(sm_mhz: float, sms: int = 148) -> float:
    """FP32 FMA peak: 128 fp32 lanes per SM, one FMA (2 flops) per lane per clock."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def run_encode(args, world, rank, local):
    """Bulk encode (a7) at the encode workload's sizes: per step, every layer compresses
    ``batch`` sequences x ``new_tokens`` dense K/V tokens through dwkv_append (placement +
    encode kernels); the sequences are reset before each step, outside the timed events.
    Then one fused decode step and one probe pass over the encoded cache."""
    import torch

    import decode_attention_depthweave_b200 as dw
    import synth

    wl = synth.workload(args.workload)
    if args.layers:
        wl = wl.scaled(num_layers=args.layers)
    dev = torch.device("cuda", local)
    B, N = wl.batch, wl.new_tokens
    lpg = wl.layers_per_group
    bases = synth.make_bases(wl)
    cfg = dw.config_from(num_layers=wl.num_layers, layers_per_group=lpg, num_q_heads=wl.num_q_heads,
                         num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim, r_max=wl.r_max, tiers=wl.tiers,
                         resid_channels=wl.resid_channels, resid_bits=wl.resid_bits, max_batch=B,
                         max_context=N + 64, tier_resid=wl.tier_resid or None, coeff_bits=wl.coeff_bits)
    stream = torch.cuda.Stream(device=dev)
    cache = dw.Cache(cfg, bases[0], bases[1], device=dev, ws_seqs=B, stream=stream)
    h = cache.h
    seqs = list(range(B))
    K, V, Tg = [], [], {}
    tier_counts = torch.zeros(len(wl.tiers), dtype=torch.int64)
    with torch.cuda.stream(stream):
        for layer in range(wl.num_layers):
            g = layer // lpg
            if g not in Tg:
                Tg[g] = torch.cat([synth.make_tiers(wl, rank * B + b, g, N, device=dev) for b in seqs])
                for k in range(len(wl.tiers)):
                    tier_counts[k] += int((Tg[g] == k).sum())
            kv = [synth.make_dense_vectors(wl, rank * B + b, layer, N, bases, device=dev) for b in seqs]
            K.append(torch.cat([x[0] for x in kv]))
            V.append(torch.cat([x[1] for x in kv]))
            del kv
    torch.cuda.synchronize(dev)

    def encode_step():
        for layer in range(wl.num_layers):
            dw.dwkv_append(h, layer, seqs, [N] * B, K[layer], V[layer], Tg[layer // lpg], stream=stream)

    def reset():
        for b in seqs:
            dw.dwkv_reset_sequence(h, b, stream)

    for _ in range(args.warmup):
        reset()
        encode_step()
    torch.cuda.synchronize(dev)
    cache.sync(stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local, gpu_uuid(local)) as clk:
        clk.mark_start()
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                reset()
                ev[i][0].record(stream)
                encode_step()
                ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
    barrier(world)
    cache.sync(stream)
    ms_steps = [a.elapsed_time(b) for a, b in ev]
    ms_per_step = max_over_ranks(world, statistics.mean(ms_steps))
    clocks = clk.summary()

    # ---- algorithmic work per step: every vector reads its dense bf16 row and writes its
    #      stored bytes; 2 d r_t fp32 FMAs (projection onto the first r_t basis columns, and
    #      the residual against the stored coefficients)
    vecs_tier = tier_counts.double() * 2 * lpg       # (seq, head, token) entries x K and V x layers of a group
    n_vec = float(vecs_tier.sum())
    stored = sum(float(tier_counts[k]) * lpg * token_bytes(r, n, wl.resid_bits, wl.coeff_bits)   # K + V bytes
                 for k, (r, n) in enumerate(zip(wl.tiers, tier_counts_of(wl))))
    dense = n_vec * wl.head_dim * 2
    flops = sum(float(vecs_tier[k]) * 4 * wl.head_dim * r for k, r in enumerate(wl.tiers))
    step_s = ms_per_step * 1e-3
    peaks = measured_peaks()
    sm_mhz = float(clocks.get("sm_max_mhz") or 1965.0) if isinstance(clocks, dict) else 1965.0
    alu_peak = fp32_alu_peak_tflops(sm_mhz)

    # ---- one decode step (append 1 token per sequence + attend, every layer) and one probe pass
    kn = [synth.make_dense_vectors(wl, rank * B + b, 0, 1, bases, device=dev, start=N) for b in seqs]
    k1 = torch.cat([x[0] for x in kn])
    v1 = torch.cat([x[1] for x in kn])
    t1 = torch.cat([synth.make_tiers(wl, rank * B + b, 0, 1, device=dev, start=N) for b in seqs])
    q = [synth.make_queries(wl, layer, batch=B, device=dev) for layer in range(wl.num_layers)]
    out = torch.empty(wl.num_layers, B, wl.num_q_heads, wl.head_dim, dtype=torch.float32, device=dev)
    err = torch.empty(wl.num_layers, B, wl.num_kv_heads, dtype=torch.float32, device=dev)
    ws = cache.workspace
    d0, d1, p0, p1 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
    with torch.cuda.stream(stream):
        d0.record(stream)
        for layer in range(wl.num_layers):
            dw.dwkv_append_decode_attention(h, layer, seqs, k1, v1, t1 if layer % lpg == 0 else None, q[layer],
                                            out[layer], ws, stream)
        d1.record(stream)
        for layer in range(wl.num_layers):                                    # warm
            dw.dwkv_probe(h, layer, seqs, q[layer], err[layer], None, ws, stream)
        p0.record(stream)
        for layer in range(wl.num_layers):
            dw.dwkv_probe(h, layer, seqs, q[layer], err[layer], None, ws, stream)
        p1.record(stream)
    torch.cuda.synchronize(dev)
    cache.sync(stream)
    assert torch.isfinite(out).all() and torch.isfinite(err).all()
    held = N + 1
    dec_bytes = (float(tier_counts.double() @ torch.tensor([token_bytes(r, n, wl.resid_bits, wl.coeff_bits)
                                                             for r, n in zip(wl.tiers, tier_counts_of(wl))],
                                                            dtype=torch.float64))
                 * lpg)                                                         # every layer; K + V bytes
    dec_ms = d0.elapsed_time(d1)
    probe_ms = p0.elapsed_time(p1)

    # ---- re-tiering (f1): one dwkv_retier call on a cache of window 0's layers alone (the
    #      workload's compressed tokens imported, an arena with room for any moves): every 8th
    #      token of each sequence moves to the next tier on every kv-head; CUDA events on the
    #      launching stream around the call
    rcfg = dw.config_from(num_layers=lpg, layers_per_group=lpg, num_q_heads=wl.num_q_heads,
                          num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim, r_max=wl.r_max, tiers=wl.tiers,
                          resid_channels=wl.resid_channels, resid_bits=wl.resid_bits, max_batch=B,
                          max_context=N + 64, tier_resid=wl.tier_resid or None, coeff_bits=wl.coeff_bits)
    rcache = dw.Cache(rcfg, bases[0][:1].contiguous(), bases[1][:1].contiguous(), device=dev, ws_seqs=B,
                      stream=stream, arena_bytes=dw.dwkv_arena_bytes_all_tiers(rcfg))
    n_mv = N // 8
    r0_, r1_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for layer in range(lpg):
            for b in seqs:
                tb = Tg[0][b * N:(b + 1) * N].contiguous()
                comp = synth.make_compressed(wl, rank * B + b, layer, tb, device=dev)
                coeff = (comp["ccodes"], comp["cscales"]) if "ccodes" in comp else comp["coeff"]
                rcache.append_compressed(layer, [b], [N], tb, coeff, comp["idx"], comp["codes"], comp["scales"],
                                         stream=stream)
        pos_mv = torch.arange(0, 8 * n_mv, 8, dtype=torch.int32, device=dev)
        nt_mv = torch.cat([((Tg[0][b * N:(b + 1) * N][pos_mv.long()].int() + 1) % len(wl.tiers)).to(torch.uint8)
                           for b in seqs]).contiguous()
        pos_all = pos_mv.repeat(B).contiguous()
        r0_.record(stream)
        dw.dwkv_retier(rcache.h, 0, seqs, [n_mv] * B, pos_all, nt_mv, stream)
        r1_.record(stream)
    torch.cuda.synchronize(dev)
    rcache.sync(stream)
    rt_ms = r0_.elapsed_time(r1_)
    rt_vec = n_mv * B * wl.num_kv_heads * lpg * 2
    retier = {"ms": round(rt_ms, 4), "moved_tokens": n_mv * B, "kv_heads": wl.num_kv_heads, "layers": lpg,
              "moved_vectors": rt_vec, "vectors_per_s": round(rt_vec / (rt_ms * 1e-3), 1),
              "timing": "one dwkv_retier call: every 8th token of each sequence to the next tier on every kv-head "
                        "(window 0, imported tokens), CUDA events"}
    del rcache

    # ---- CPU oracle baseline (rank 0, N = 1 only): the oracle's encode of sequence 0's keys
    #      and values of layer 0, kv-head 0 (2 N vectors), OpenMP over the vectors on all cores
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import numpy as np

        import oracle
        cores = os.cpu_count() or 1
        ranks0 = np.asarray(wl.tiers, np.int32)[Tg[0][:N, 0].long().cpu().numpy()]
        t0 = time.perf_counter()
        for z, X in enumerate((K[0], V[0])):
            oracle.encode_many(bases[z][0, 0], X[:N, 0].cpu(), ranks0, wl.resid_channels, wl.resid_bits,
                               nthreads=cores)
        dt = time.perf_counter() - t0
        gbs = 2 * N * wl.head_dim * 2 / dt / 1e9
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"sequence 0, layer 0, kv-head 0: {2 * N} key and value vectors encoded by the fp32 C "
                         f"oracle (OpenMP over the vectors, {dt:.2f} s wall on {cores} threads); GB/s of dense "
                         "bf16 input, the rate the step's vectors would see",
               "nproc": cores, "cpu_model": cpu_model()}

    # ---- online bases of window 0 (f2): the moving-average update with the re-projection of
    #      every stored token of the window (valid: the tokens were encoded on the current
    #      bases), then a sketch from the window's prefill rows (it replaces the bases; the cache
    #      is not used after it)
    online = None
    if wl.r_max <= 64:
        L = wl.num_layers
        n_upd = 1024
        u0, u1, s0, s1 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
        with torch.cuda.stream(stream):                  # the inputs are made on the launching stream
            k_upd = torch.stack([K[l][:n_upd] for l in range(L)]).contiguous()
            v_upd = torch.stack([V[l][:n_upd] for l in range(L)]).contiguous()
            omega = synth.make_test_matrix(wl, device=dev)
            u0.record(stream)
            dw.dwkv_basis_update(h, dw.DWKV_ALL_GROUPS, n_upd, k_upd, v_upd, 0.9, seqs, None, stream)
            u1.record(stream)
        torch.cuda.synchronize(dev)
        del k_upd, v_upd
        with torch.cuda.stream(stream):
            k_sk = torch.stack(K).contiguous()
            v_sk = torch.stack(V).contiguous()
            s0.record(stream)
            dw.dwkv_basis_sketch(h, dw.DWKV_ALL_GROUPS, k_sk.shape[1], k_sk, v_sk, omega, 2, None, stream)
            s1.record(stream)
        torch.cuda.synchronize(dev)
        cache.sync(stream)
        del k_sk, v_sk
        upd_ms, sk_ms = u0.elapsed_time(u1), s0.elapsed_time(s1)
        rows = L * B * N                                     # rows a kv-head, all windows
        moment_flops = 2.0 * rows * wl.head_dim * wl.head_dim * wl.num_kv_heads * 2
        n_rep = B * held * wl.num_kv_heads * L * 2
        online = {"sketch_ms": round(sk_ms, 4), "windows": wl.num_groups, "sketch_rows_per_head": rows,
                  "power_steps": 2, "moment_tflops_lower_bound": round(moment_flops / (sk_ms * 1e-3) / 1e12, 2),
                  "update_ms": round(upd_ms, 4), "update_rows_per_head": L * n_upd,
                  "reprojected_vectors": n_rep, "reprojected_vectors_per_s": round(n_rep / (upd_ms * 1e-3), 1),
                  "timing": "every window in one call each (update first, on the encoded cache), CUDA events"}

    value = aggregate_rate(world, dense / 1e9, ms_per_step)
    res = {
        "metric": "bulk encode: dense bf16 K/V GB/s compressed (a7)", "value": round(value, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp32 math",
        "data": "synthetic (seeded dense K/V: basis span + outliers + noise; no model weights)",
        "config": {"workload": args.workload, "layers": wl.num_layers, "kv_heads": wl.num_kv_heads,
                   "head_dim": wl.head_dim, "batch_per_gpu": B, "new_tokens": N, "r_max": wl.r_max,
                   "tiers": list(wl.tiers), "tier_probs": list(wl.tier_probs), "resid_channels": wl.resid_channels,
                   **({"tier_resid": list(wl.tier_resid)} if wl.tier_resid else {}),
                   **({"coeff_bits": wl.coeff_bits} if wl.coeff_bits != 16 else {}),
                   "resid_bits": wl.resid_bits, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (8.6 GB of dense K/V a step); no flush",
                   "timing": "eager launches, CUDA events around each step's appends (resets outside)"},
        "gpu_launches": 2 * wl.num_layers * args.steps,
        "vectors_per_s": round(aggregate_rate(world, n_vec, ms_per_step), 1),
        "roofline": {"bound": "alu", "achieved": round(flops / step_s / 1e12, 3), "unit": "TFLOP/s",
                     "peak": round(alu_peak, 2), "frac": round(flops / step_s / 1e12 / alu_peak, 4),
                     "traffic": None, "kernel": f"dwkv::encode_kernel<{wl.resid_bits}>",
                     "peak_source": f"148 SMs x 128 fp32 lanes x 2 flops x {sm_mhz:.0f} MHz (sampled max SM clock)",
                     "flops_per_step": flops},
        "hbm": {"bytes_per_step": dense + stored, "achieved_gbs": round((dense + stored) / step_s / 1e9, 1),
                "frac": round((dense + stored) / step_s / 1e9 / peaks["hbm_gbs"], 4)},
        "decode_step": {"context": held, "batch": B, "ms": round(dec_ms, 4),
                        "tok_s": round(B / (dec_ms * 1e-3), 1),
                        "compressed_gbs": round(dec_bytes / (dec_ms * 1e-3) / 1e9, 1),
                        "timing": "one eager step (32 fused append + decode launches)"},
        "probe": {"ms_all_layers": round(probe_ms, 4),
                  "achieved_gbs": round(dec_bytes / (probe_ms * 1e-3) / 1e9, 1),
                  "frac": round(dec_bytes / (probe_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
        "retier": retier,
        "online_basis": online,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    cache.close()
    del cache, K, V
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return res


def run_reference(args, world, rank, local):
    """The CPU oracle, as it stands, timed on the host cores over a bounded sample of the same
    workload.  One bench step here is one sample: every kv-head of the first layers of
    sequence 0 (one (layer, kv-head) problem per core at least) at the sequence's full
    context, fp64, OpenMP over the problems on all cores.  ``value`` scales the sample's
    time to a whole decode step of the workload (all sequences, all layers); ``ms_per_step``
    is the sample's own measured time."""
    import synth
    wl = synth.workload(args.workload)
    B = wl.batch
    lengths = [args.context] * B if args.context else synth.make_context_lengths(wl)
    cores = os.cpu_count() or 1
    nl = oracle_layers_for(wl, cores)
    bases = synth.make_bases(wl)
    probs_in = []
    tiers_g = {}
    for layer in range(nl):
        g = layer // wl.layers_per_group
        if g not in tiers_g:
            tiers_g[g] = synth.make_tiers(wl, 0, g, lengths[0] - 1)
        comp = synth.make_compressed(wl, 0, layer, tiers_g[g])
        q = synth.make_queries(wl, layer, batch=1)[0]
        probs_in += [(bases, tiers_g[g], comp, q, layer, hh) for hh in range(wl.num_kv_heads)]
    scale = (wl.num_layers * wl.num_kv_heads / len(probs_in)) * (sum(lengths) - B) / (lengths[0] - 1)
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, probs_in, cores)
    times = [cpu_oracle_sample(wl, probs_in, cores) for _ in range(args.steps)]
    sample_s = statistics.mean(times)
    value = B / (sample_s * scale)
    sample = (f"per step: sequence 0, layers 0-{nl - 1} x {wl.num_kv_heads} kv-heads = {len(probs_in)} problems of "
              f"{lengths[0] - 1} cached tokens (fp64 C oracle, OpenMP over the problems on {cores} threads); value "
              f"scales the step's time x{scale:.2f} to a whole decode step ({B} sequence(s), {wl.num_layers} layers)")
    return {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(sample_s * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded compressed cache)",
        "config": {"workload": args.workload, "layers": wl.num_layers, "kv_heads": wl.num_kv_heads,
                   "context": lengths[0] if B == 1 else lengths, "batch_per_gpu": B},
        "impl": "reference",
        "ms_per_full_step_scaled": round(sample_s * scale * 1e3, 1),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                         "nproc": cores, "cpu_model": cpu_model()},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


EXTRA_WORKLOADS = ("llama8b_64k_c8", "llama8b_ragged_b8", "llama8b_131k_deep", "llama8b_routed_64k", "llama8b_encode_16k")


def summary_of(res: dict) -> dict:
    """The keys of a workload's line that the default run repeats for the extra workloads."""
    keep = ("metric", "value", "unit", "ms_per_step", "steps", "warmup", "config", "gpu_launches", "roofline",
            "compressed_gb_per_step", "compressed_tb_s", "probe", "e2e", "cpu_baseline", "clocks", "hbm",
            "decode_step", "vectors_per_s", "online_basis")
    return {k: res[k] for k in keep if k in res}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dwkv", choices=["dwkv", "reference"])
    ap.add_argument("--workload", default="llama8b_64k")
    ap.add_argument("--context", type=int, default=0, help="override the context length")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs)")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--profile-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tuning", default="", help="ctas_per_sm,waves,stages")
    ap.add_argument("--headline-only", action="store_true", help="skip the other workloads of the default run")
    ap.add_argument("--no-overlap", action="store_true", help="serialise the decode launches (measurement)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 1)
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            if rank != 0:
                return
            res = run_reference(args, world, rank, local)
        elif args.workload == "llama8b_encode_16k":
            res = run_encode(args, world, rank, local)
        else:
            res = run_dwkv(args, world, rank, local)
            # the default single-GPU run also measures the other workloads, each with its own
            # roofline, e2e and CPU baseline, in fewer steps (the headline stays the 64K line)
            if world == 1 and args.workload == "llama8b_64k" and not args.headline_only and not args.layers:
                extra = {}
                for wname in EXTRA_WORKLOADS:
                    if wname == "llama8b_encode_16k":
                        sub = argparse.Namespace(**vars(args))
                        sub.workload, sub.steps, sub.warmup = wname, 2, 1
                        extra[wname] = summary_of(run_encode(sub, world, rank, local))
                    else:
                        extra[wname] = summary_of(run_dwkv(args, world, rank, local, workload=wname,
                                                           steps=min(args.steps, 10), warmup=3, e2e_steps=2,
                                                           light=True))
                res["workloads"] = extra
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
