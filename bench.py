"""Decode-step benchmark: KV-cache GB/s and us per step on the skewed batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole decode path for a batch without a prologue: the
dynamic tile plan, attention and the split merge (hpa_decode_step: the plan
made inside the decode kernel, two launches; hpa_decode_plan +
hpa_decode_run above 512 sequences) over the skewed workload: 1 x 131072 +
31 x 4096 KV tokens, 64 query heads, 8 KV heads, head_dim 128, bf16 cache,
64-token pages shuffled over HBM (xiaodao.ai "HPC-Ops TPOT -48.8%",
Attention section, the 1 x 128K + 31 x 4K case).  Inputs are synthetic
(seeded N(0,1)) and resident in HBM; 1.06 GB of live KV per step is far
above the 126 MB L2, so no flush is needed between steps.

Printed (rank 0, one JSON line): value = live KV bytes per step / step time
(whole job over N GPUs: each rank runs its own batch, weak scaling), the run
kernel's roofline against the measured HBM copy bandwidth, an end-to-end
figure through the public API with host buffers, the fp64 oracle timed on
the host cores, SM clocks sampled during the timed region, and comparisons
timed as interleaved A/B runs: the static split-KV plans and the
length-aware plan fed to the same kernel, the three-launch form, and the
batch split by page range over 2 and 8 shares (run one after another on
this GPU, then merged).

--impl reference times the oracle (the plain fp64 CPU implementation) on the
host cores on a bounded sample of the same workload and prints the same line
with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV-cache GB/s (% of HBM peak), µs/decode step, skewed 1x128K+31x4K"
L2_BYTES = 126 * 1000 * 1000  # B200 L2 capacity
WORKLOAD = "skewed"
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_run_skewed_ncu.md")
KERNEL_SOURCES = [os.path.join(ROOT, "mixed_length_paged_b200", "csrc", f)
                  for f in ("decode.cu", "hpa_common.cuh", "plan_geom.cuh", "prologue_math.cuh")]


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--num-ctas", type=int, default=0,
                    help="persistent CTAs of the dynamic plan (0: the library default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="time eager launches instead of CUDA-graph replays of the step")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the comparisons (static, length-aware and three-launch plans, "
                         "page-sharded shares, separate prologue) and the e2e leg")
    return ap.parse_args()


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


WORKLOAD_DESC = {
    "skewed": "skewed decode: 1 x 131072 + 31 x 4096 KV tokens, 64 q heads, 8 kv heads, "
              "head_dim 128, bf16 KV, 64-token pages shuffled; dynamic plan",
    "skewed_quarter": "skewed decode at a quarter of the lengths: 1 x 32768 + 31 x 1024",
    "uniform": "uniform decode: 64 x 512 KV tokens, 64 q heads, 8 kv heads, head_dim 128, bf16",
    "tiny": "tiny decode: 2 sequences {37, 200}, 8 q heads, 2 kv heads, head_dim 64, bf16",
    "mix_prologue": "continuous-batching mix: 128 sequences, lengths log-uniform in [256, 65536], "
                    "32 q heads, 8 kv heads, head_dim 128, bf16; fused RMSNorm+RoPE+KV-write "
                    "prologue in every step",
    "fp8": "FP8 KV: 256 sequences, lengths geometric (mean 2048, cap 16384), 64 q heads, "
           "8 kv heads, head_dim 128, e4m3 K/V with fp32 per-(page, kv head) scales",
    "fp8_quarter": "the first 64 sequences of the FP8 batch (profiler captures)",
    "skewed_mtp2": "multi-token decode on the skewed batch: 2 query tokens per sequence "
                   "(causal among themselves), 64 q heads, 8 kv heads, head_dim 128, bf16",
}


def _quantize_e4m3(values, live):
    """Input preparation for the FP8 workload (not part of the timed step):
    e4m3 codes + fp32 per-(page, kv head) scales = amax of the live tokens /
    448, via torch's float8 cast.  Dead slots get the NaN code."""
    import torch
    P, Hkv, S, D = values.shape
    slot = torch.arange(S, device=values.device).view(1, 1, S, 1)
    alive = slot < live.view(P, 1, 1, 1).to(values.device)
    amax = (values.abs() * alive).amax(dim=(2, 3))
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).float()
    codes = (values / scale.view(P, Hkv, 1, 1)).clamp(-448, 448).to(torch.float8_e4m3fn)
    codes = codes.view(torch.uint8).masked_fill(~alive, 0x7F)
    return codes.contiguous(), scale.contiguous()


def _code_only(text: str) -> str:
    """Source text without comments and blank lines (what the compiler sees;
    the kernel sources hold no string literal with a comment marker)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def _kernel_hash() -> str:
    """Fingerprint of the run kernel's code (comments do not count)."""
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def _profiled_traffic():
    """DRAM bytes per launch of the run kernel from the committed ncu summary,
    if it was taken on the current kernel source; else None."""
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    kv = {}
    for line in text.splitlines():
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            kv[k.strip()] = v.strip().strip("`")
    if kv.get("kernel_source_sha256_16") != _kernel_hash():
        return None
    try:
        return int(kv["dram_bytes_per_launch_full_workload"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of every rank's x (device-timed durations are combined this
    way: the job takes as long as its slowest rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank: int, world: int, seconds: float) -> float:
    """Whole-job GB/s under weak scaling: every rank streams its own batch of
    bytes_per_rank in `seconds` (the max over ranks)."""
    return world * bytes_per_rank / seconds / 1e9


def _smi_index(local_rank: int) -> str:
    """nvidia-smi id of this rank's GPU (honours CUDA_VISIBLE_DEVICES)."""
    vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    return vis[local_rank] if local_rank < len(vis) else str(local_rank)


def _cpu_baseline_sample(batch_host, rows):
    """Time the oracle (as it stands) on sequences `rows` of the workload."""
    import numpy as np

    import oracle
    D = batch_host["D"]
    t0 = time.perf_counter()
    oracle.paged_decode(batch_host["q"], batch_host["k"], batch_host["v"], batch_host["pt"],
                        batch_host["sl"], batch_host["Hkv"], 1.0 / math.sqrt(D),
                        rows=np.array(rows, dtype=np.int32))
    dt = time.perf_counter() - t0
    toks = int(sum(int(batch_host["sl"][b]) for b in rows))
    nbytes = toks * 2 * batch_host["Hkv"] * D * 2
    return nbytes / dt / 1e9, dt, toks


def _host_sample(batch, rows):
    """Host (numpy) copy of the sampled sequences only, pages renumbered."""
    import numpy as np
    import torch
    pt = batch.page_table.cpu().numpy()
    sl = batch.seq_lens.cpu().numpy()
    used = []
    new_pt = np.full((len(rows), pt.shape[1]), -1, dtype=np.int32)
    for i, b in enumerate(rows):
        n = (int(sl[b]) + 63) // 64
        new_pt[i, :n] = np.arange(len(used), len(used) + n)
        used.extend(pt[b, :n].tolist())
    idx = torch.tensor(used, dtype=torch.long, device=batch.k_cache.device)

    def bits(t):
        return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    return {"q": bits(batch.q[rows]), "k": bits(batch.k_cache.index_select(0, idx)),
            "v": bits(batch.v_cache.index_select(0, idx)), "pt": new_pt,
            "sl": sl[rows].astype(np.int32), "Hkv": batch.shape.num_kv_heads,
            "D": batch.shape.head_dim}


# the reference arm's sample: the 31 short sequences of the skewed batch
CPU_SAMPLE_ROWS = list(range(1, 32))
CPU_BASELINE_SECONDS = 10.0   # the CPU baseline repeats the whole step for at least this long
REF_BUDGET_SECONDS = 150.0    # the whole --impl reference run (all of its steps)


def _oracle_for(host, rows, min_seconds: float):
    """The oracle on sequences `rows`, repeated until at least `min_seconds`
    have passed: (GB/s over all repetitions, seconds, repetitions)."""
    reps, secs, nbytes = 0, 0.0, 0
    while reps == 0 or secs < min_seconds:
        _, dt, toks = _cpu_baseline_sample(host, rows)
        secs += dt
        nbytes += toks * 2 * host["Hkv"] * host["D"] * 2
        reps += 1
    return nbytes / secs / 1e9, secs, reps


def _reference_rows(t_one: float, calls: int, available: int) -> int:
    """Sequences per reference step so that `calls` steps of the oracle fit
    the run's time budget (one sequence takes `t_one` seconds)."""
    per_call = REF_BUDGET_SECONDS / max(1, calls)
    return max(1, min(available, int(per_call / max(t_one, 1e-6))))


def run_reference(args, rank: int):
    """--impl reference: the oracle on the host cores, bounded sample per step."""
    if rank != 0:
        return
    import torch

    import oracle
    from mixed_length_paged_b200 import workloads as W
    batch = W.build(args.workload, device="cpu")
    host = _host_sample(batch, CPU_SAMPLE_ROWS)
    cores = oracle.num_threads()
    # size each step so that all of them fit the run's budget: one sequence
    # timed after a warm-up call, then as many sequences per step as fit
    _cpu_baseline_sample(host, [0])
    _, t_one, _ = _cpu_baseline_sample(host, [0])
    calls = args.steps + min(args.warmup, 1)
    rows = list(range(_reference_rows(t_one, calls, len(CPU_SAMPLE_ROWS))))
    for _ in range(min(args.warmup, 1)):
        _cpu_baseline_sample(host, rows)
    times, gbs = [], []
    for _ in range(args.steps):
        g, dt, toks = _cpu_baseline_sample(host, rows)
        times.append(dt)
        gbs.append(g)
    value = statistics.median(gbs)
    sample = (f"oracle (fp64, OpenMP over (sequence, head)) per step on {len(rows)} of the "
              f"skewed batch's 4096-token sequences ({toks:,} KV tokens), sized so that all "
              f"{args.steps} steps fit about {REF_BUDGET_SECONDS:.0f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "skewed 1x131072+31x4096 sample", "sample": sample},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    del torch
    print(json.dumps(line), flush=True)


def run_ours(args, rank: int, world: int, local_rank: int):
    import numpy as np
    import torch
    import torch.distributed as dist

    import mixed_length_paged_b200 as hpa
    from mixed_length_paged_b200 import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hpa.lib()
    batch = W.build(args.workload, device=dev, seed=0)
    shape = batch.shape
    B, Hq, Hkv, D = batch.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim
    fp8 = shape.kv_dtype == "fp8_e4m3"
    k_scale = v_scale = None
    if fp8:
        batch.k_cache, k_scale = _quantize_e4m3(batch.k_cache, batch.live)
        batch.v_cache, v_scale = _quantize_e4m3(batch.v_cache, batch.live)
    lens = batch.seq_lens.cpu().numpy()
    elt = 1 if fp8 else 2
    kv_bytes = W.live_kv_bytes(lens, Hkv, D, elt)
    tiles = int(((lens + 63) // 64).sum())
    # algorithmic bytes of one run launch: live KV + q + out + page-table entries
    # read (+ the two fp32 scales of every (page, kv head) tile for FP8)
    T = shape.q_tokens
    run_bytes = kv_bytes + 2 * B * T * Hq * D * 2 + tiles * 4 + (tiles * Hkv * 8 if fp8 else 0)
    if shape.prologue:
        # the fused prologue also reads the new token's raw K and V rows and
        # writes them (normalised, rotated) into their cache slots
        run_bytes += 4 * B * Hkv * D * 2
    scale = 1.0 / math.sqrt(D)
    num_ctas = args.num_ctas or hpa.decode_num_ctas(Hq, Hkv, shape.q_tokens, local_rank)
    stream = torch.cuda.current_stream()
    dec = hpa.PagedDecoder(B, Hq, Hkv, D, batch.pt_stride, num_ctas=num_ctas, q_tokens=T,
                           device=dev)
    out = torch.empty(batch.q.shape if T > 1 else (B, Hq, D), dtype=torch.bfloat16, device=dev)
    seq_lens = batch.seq_lens
    if shape.prologue:
        # The step starts from the new token's raw projections: plan, then the
        # run with the prologue (RMSNorm + RoPE of q and the new K row, the K/V
        # slot write) fused into the decode kernel, attending over L + 1.
        batch.q = torch.empty_like(batch.q_raw)

    def prologue():  # the separate prologue kernel (comparator only)
        hpa.kv_prologue(batch.q_raw, batch.k_raw, batch.v_raw, batch.q_gamma, batch.k_gamma,
                        batch.positions, batch.page_table, batch.k_cache, batch.v_cache,
                        batch.q, eps=1e-6, rope_theta=10000.0)

    def run():
        if shape.prologue:
            dec.run_prologue(batch.q_raw, batch.k_raw, batch.v_raw, batch.q_gamma, batch.k_gamma,
                             batch.k_cache, batch.v_cache, batch.page_table, out, scale,
                             eps=1e-6, rope_theta=10000.0)
        else:
            dec.run(batch.q, batch.k_cache, batch.v_cache, batch.page_table, out, scale,
                    k_scale=k_scale, v_scale=v_scale)

    # The dynamic plan is made inside the decode kernel (hpa_decode_step /
    # hpa_decode_step_prologue) where the batch fits its shared memory.
    use_step = B <= hpa.MAX_STEP_BATCH

    def step():
        if use_step and shape.prologue:
            dec.step_prologue(batch.q_raw, batch.k_raw, batch.v_raw, batch.q_gamma,
                              batch.k_gamma, batch.k_cache, batch.v_cache, batch.page_table,
                              seq_lens, out, scale, eps=1e-6, rope_theta=10000.0)
        elif use_step:
            dec.step(batch.q, batch.k_cache, batch.v_cache, batch.page_table, seq_lens, out,
                     scale, k_scale=k_scale, v_scale=v_scale)
        else:
            dec.plan(seq_lens)
            run()

    def plan_then_run():  # the three-launch form (comparator)
        dec.plan(seq_lens)
        run()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        step()
    barrier()

    def graphed(fn):
        """One step captured as a CUDA graph (plan -> run -> merge keep their
        programmatic-dependent-launch edges); replaying it costs one launch
        call on the host.  A decode loop in a serving engine replays its step
        this way; eagerly, ~35 us steps are bound by the host's launch rate."""
        if args.eager:
            return fn
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        graphs.append(g)
        return g.replay

    graphs = []
    timed_step = graphed(step)
    barrier()
    K = args.steps
    sampler = ClockSampler(_smi_index(local_rank))
    sampler.start()
    # Timed region 1 (the reported value): K back-to-back steps, events only
    # at the ends, so plan -> run -> merge chain through programmatic
    # dependent launch exactly as a caller's stream would.
    barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(K):
        timed_step()
    end.record(stream)
    barrier()
    # Timed region 2 (per-kernel durations for the roofline): the same K
    # steps with events around the plan and around the run call (one call,
    # decode + merge, when the plan is made in the kernel).
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3 * K)]
    for i in range(K):
        ev[3 * i].record(stream)
        if not use_step:
            dec.plan(seq_lens)
        ev[3 * i + 1].record(stream)
        if use_step:
            step()
        else:
            run()
        ev[3 * i + 2].record(stream)
    barrier()
    clocks = sampler.stop()
    total_ms = start.elapsed_time(end)
    run_ms = [ev[3 * i + 1].elapsed_time(ev[3 * i + 2]) for i in range(K)]
    plan_ms = [ev[3 * i].elapsed_time(ev[3 * i + 1]) for i in range(K)]
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / K
    status = dec.status()

    # static split-KV comparators: the same run kernel fed the static plans
    extras = {}
    if not args.no_extras and use_step:
        # the same step as plan kernel + run (three launches), interleaved A/B
        sep = graphed(plan_then_run)
        blocks, per = 10, max(5, min(40, K // 10))
        ab = {"step": 0.0, "plan_run": 0.0}
        for _ in range(blocks):
            for name, fn in (("step", timed_step), ("plan_run", sep)):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(per):
                    fn()
                b.record(stream)
                torch.cuda.synchronize()
                ab[name] += a.elapsed_time(b)
        n = blocks * per
        extras["plan_kernel_then_run"] = {
            "us_per_step": 1e3 * ab["plan_run"] / n,
            "in_kernel_plan_us_per_step_same_blocks": 1e3 * ab["step"] / n,
            "in_kernel_plan_speedup": ab["plan_run"] / ab["step"],
            "method": f"interleaved A/B, {blocks} x {per} steps each"}
    if not args.no_extras and shape.prologue:
        # The same step with the prologue as its own kernel before plan + run,
        # timed as an interleaved A/B against the fused step (blocks of 20
        # steps each, alternating) so that clock and power drift over the run
        # falls on both alike.
        def separate():
            prologue()
            dec.plan(seq_lens)
            dec.run(batch.q, batch.k_cache, batch.v_cache, batch.page_table, out, scale)

        for _ in range(3):
            separate()
        torch.cuda.synchronize()
        separate_step = graphed(separate)
        blocks, per = 10, 20
        ab = {"fused": 0.0, "separate": 0.0}
        for _ in range(blocks):
            for name, fn in (("fused", timed_step), ("separate", separate_step)):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(per):
                    fn()
                b.record(stream)
                torch.cuda.synchronize()
                ab[name] += a.elapsed_time(b)
        n = blocks * per
        extras["separate_prologue_kernel"] = {
            "us_per_step": 1e3 * ab["separate"] / n,
            "fused_us_per_step_same_blocks": 1e3 * ab["fused"] / n,
            "fused_speedup": ab["separate"] / ab["fused"],
            "method": f"interleaved A/B, {blocks} x {per} steps each"}

    plain = not fp8 and not shape.prologue and T == 1
    if not args.no_extras and plain:
        # each static plan against the dynamic one as an interleaved A/B
        # (alternating blocks of steps), so drift falls on both alike
        blocks, per = 10, max(5, min(40, K // 10))
        for name, kind in (("static_nsplit", hpa.PLAN_STATIC_NSPLIT),
                           ("static_chunk", hpa.PLAN_STATIC_CHUNK)):
            sd = hpa.PagedDecoder(B, Hq, Hkv, D, batch.pt_stride, kind=kind, num_ctas=num_ctas,
                                  max_seq_len=int(lens.max()), device=dev)

            def static_step():
                sd(batch.q, batch.k_cache, batch.v_cache, batch.page_table, seq_lens, out, scale)

            for _ in range(3):
                static_step()
            torch.cuda.synchronize()
            static_timed = graphed(static_step)
            ab = {"dynamic": 0.0, "static": 0.0}
            for _ in range(blocks):
                for which, fn in (("dynamic", timed_step), ("static", static_timed)):
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    for _ in range(per):
                        fn()
                    b.record(stream)
                    torch.cuda.synchronize()
                    ab[which] += a.elapsed_time(b)
            ms = ab["static"] / (blocks * per)
            extras[name] = {"us_per_step": 1e3 * ms, "GB_s": kv_bytes / (ms * 1e-3) / 1e9,
                            "grid": sd.grid,
                            "dynamic_us_per_step_same_blocks": 1e3 * ab["dynamic"] / (blocks * per),
                            "dynamic_speedup": ab["static"] / ab["dynamic"],
                            "method": f"interleaved A/B, {blocks} x {per} steps each"}
        extras["dynamic_speedup_vs_best_static"] = min(
            extras[k]["dynamic_speedup"] for k in ("static_nsplit", "static_chunk"))

    if not args.no_extras and not shape.prologue:
        # The length-aware plan (cut points moved off segment ends, smallest
        # end piece m tiles) against the dynamic plan, both as plan kernel +
        # run, interleaved A/B.
        blocks, per = 10, max(5, min(40, K // 10))
        kw = dict(k_scale=k_scale, v_scale=v_scale)
        dd = hpa.PagedDecoder(B, Hq, Hkv, D, batch.pt_stride, num_ctas=num_ctas, q_tokens=T,
                              device=dev)

        def dyn_pr():
            dd(batch.q, batch.k_cache, batch.v_cache, batch.page_table, seq_lens, out, scale, **kw)

        for _ in range(3):
            dyn_pr()
        dyn_timed = graphed(dyn_pr)
        extras["length_aware"] = {}
        for m in (2, 4, 8):
            ld = hpa.PagedDecoder(B, Hq, Hkv, D, batch.pt_stride, kind=hpa.PLAN_LENGTH_AWARE,
                                  param=m, num_ctas=num_ctas, q_tokens=T, device=dev)

            def la_step(ld=ld):
                ld(batch.q, batch.k_cache, batch.v_cache, batch.page_table, seq_lens, out, scale,
                   **kw)

            for _ in range(3):
                la_step()
            torch.cuda.synchronize()
            la_timed = graphed(la_step)
            ab = {"dynamic": 0.0, "length_aware": 0.0}
            for _ in range(blocks):
                for which, fn in (("dynamic", dyn_timed), ("length_aware", la_timed)):
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    for _ in range(per):
                        fn()
                    b.record(stream)
                    torch.cuda.synchronize()
                    ab[which] += a.elapsed_time(b)
            n = blocks * per
            extras["length_aware"][f"m{m}"] = {
                "us_per_step": 1e3 * ab["length_aware"] / n,
                "dynamic_plan_run_us_same_blocks": 1e3 * ab["dynamic"] / n,
                "speedup_vs_dynamic": ab["dynamic"] / ab["length_aware"],
                "method": f"plan kernel + run each, interleaved A/B, {blocks} x {per} steps"}

    if not args.no_extras and plain and use_step:
        # The batch spread by page range over R ranks (sharding.page_shard),
        # the R shares run one after another on this GPU, each a decode step
        # with log-sum-exps, then the merge of the R states.  The slowest
        # share is what one of R GPUs would spend on its decode; the all-gather
        # between the two is not measured (one GPU).  A sleep kernel first
        # lets the host queue a whole round, so the events time the GPU only;
        # consecutive shares read different pages, so L2 carries nothing over.
        from mixed_length_paged_b200 import sharding as SH
        extras["page_sharded"] = {}
        for R in (2, 8):
            parts = []
            for r in range(R):
                lr, ptr = SH.page_shard(batch.seq_lens, batch.page_table, R, r)
                parts.append((hpa.PagedDecoder(B, Hq, Hkv, D, batch.pt_stride, num_ctas=num_ctas,
                                               device=dev),
                              lr.to(dev), ptr.to(dev),
                              torch.empty(B, Hq, D, dtype=torch.float32, device=dev),
                              torch.empty(B, Hq, dtype=torch.float32, device=dev)))
            o_parts, l_parts = [p[3] for p in parts], [p[4] for p in parts]
            reps = 20
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(R + 2)]
                   for _ in range(reps)]
            for rep in range(reps + 3):
                torch.cuda._sleep(5_000_000)
                e = evs[rep - 3] if rep >= 3 else None
                for r, (sd, lr, ptr, o, l) in enumerate(parts):
                    if e:
                        e[r].record(stream)
                    sd.step(batch.q, batch.k_cache, batch.v_cache, ptr, lr, o, scale, lse=l)
                if e:
                    e[R].record(stream)
                hpa.merge_states(o_parts, l_parts, out)
                if e:
                    e[R + 1].record(stream)
                torch.cuda.synchronize()
            share = np.array([[e[r].elapsed_time(e[r + 1]) for r in range(R)] for e in evs])
            merge = np.array([e[R].elapsed_time(e[R + 1]) for e in evs])
            extras["page_sharded"][str(R)] = {
                "max_share_step_us": 1e3 * float(np.median(share, axis=0).max()),
                "mean_share_step_us": 1e3 * float(np.median(share, axis=0).mean()),
                "merge_states_us": 1e3 * float(np.median(merge)),
                "all_shares_and_merge_on_one_gpu_us": 1e3 * float(np.median(share.sum(1) + merge)),
                "method": f"median of {reps} rounds, events between launches"}

    # End to end through the public API (eager calls): every step copies its
    # inputs (q, seq_lens, page table) from pinned host memory to the device
    # and its output back, inside the timed region.  As a serving loop would,
    # the steps are pipelined over three streams -- copies in, compute, copy
    # out -- with double-buffered device inputs and outputs, so step i's
    # copies overlap the compute of its neighbours.
    e2e = None
    if not args.no_extras and plain:
        q_h = batch.q.cpu().pin_memory()
        sl_h = batch.seq_lens.cpu().pin_memory()
        pt_h = batch.page_table.cpu().pin_memory()
        out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        q_d = [torch.empty_like(batch.q) for _ in range(2)]
        sl_d = [torch.empty_like(seq_lens) for _ in range(2)]
        pt_d = [torch.empty_like(batch.page_table) for _ in range(2)]
        out_d = [torch.empty_like(out) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        s_comp = stream
        ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "done", "out")}
        started = [False, False]

        def e2e_step(i):
            k = i % 2
            with torch.cuda.stream(s_in):
                if started[k]:
                    s_in.wait_event(ev["done"][k])   # step i-2 has read its inputs
                q_d[k].copy_(q_h, non_blocking=True)
                sl_d[k].copy_(sl_h, non_blocking=True)
                pt_d[k].copy_(pt_h, non_blocking=True)
                ev["in"][k].record(s_in)
            s_comp.wait_event(ev["in"][k])
            if started[k]:
                s_comp.wait_event(ev["out"][k])      # step i-2's output is on the host
            dec.step(q_d[k], batch.k_cache, batch.v_cache, pt_d[k], sl_d[k], out_d[k], scale,
                     stream=s_comp)
            ev["done"][k].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["done"][k])
                out_h[k].copy_(out_d[k], non_blocking=True)
                ev["out"][k].record(s_out)
            started[k] = True

        for i in range(4):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        n = max(10, min(500, K))
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        for i in range(n):
            e2e_step(i)
        s_in.wait_stream(s_out)                     # the last output is on the host
        s_in.wait_stream(s_comp)
        b.record(s_in)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(a.elapsed_time(b) / n, world, dev)
        h2d = q_h.numel() * 2 + sl_h.numel() * 4 + pt_h.numel() * 4
        e2e = {"value": job_throughput(kv_bytes, world, e_ms * 1e-3), "unit": "GB/s",
               "us_per_step": 1e3 * e_ms, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(out_h[0].numel() * 2),
               "method": "eager public-API calls; copies in / compute / copy out on three "
                         "streams, double-buffered, each step's copies inside the timed region"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == WORKLOAD:
        import oracle
        # the whole step (every sequence of the batch), repeated for at least
        # CPU_BASELINE_SECONDS
        rows = list(range(B))
        host = _host_sample(batch, rows)
        _cpu_baseline_sample(host, [1])  # warm-up
        g, dt, reps = _oracle_for(host, rows, CPU_BASELINE_SECONDS)
        cpu = {"value": g, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
               "sample": (f"oracle (fp64, OpenMP over (sequence, head)) on the whole skewed "
                          f"step (1 x 131072 + 31 x 4096 tokens), {reps} times in {dt:.1f} s"),
               "seconds": dt}

    if rank != 0:
        return
    peak, peak_kind = _peaks()
    run_avg_ms = statistics.mean(run_ms)
    achieved = run_bytes / (run_avg_ms * 1e-3) / 1e9
    traffic = _profiled_traffic()
    value = job_throughput(kv_bytes, world, ms_per_step * 1e-3)
    metric = METRIC if args.workload == WORKLOAD else \
        f"KV-cache GB/s (% of HBM peak), µs/decode step, {args.workload}"
    line = {
        "metric": metric, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 KV / bf16" if fp8 else "bf16",
        "data": "synthetic", "us_per_step": 1e3 * ms_per_step,
        "pct_of_hbm_peak": 100.0 * (kv_bytes / (ms_per_step * 1e-3) / 1e9) / peak,
        "config": {
            "workload": WORKLOAD_DESC.get(args.workload, args.workload),
            "batch": B, "kv_bytes_per_step_per_gpu": kv_bytes, "num_ctas": num_ctas,
            "l2": (f"no flush: {kv_bytes / 1e9:.3g} GB of KV per step is larger than the "
                   "126 MB L2" if kv_bytes > L2_BYTES else
                   f"L2-resident: {kv_bytes / 1e6:.3g} MB of KV per step fits the 126 MB L2 "
                   "(a latency figure, not an HBM one)"),
            "launch": "eager calls" if args.eager else
                      "CUDA-graph replay of one captured step",
            "plan": "in the decode kernel (hpa_decode_step)" if use_step else
                    "plan kernel (hpa_decode_plan) before the run",
            "parallelism": f"data-parallel replicas x{world} (independent batches, no collective)",
        },
        "breakdown_us": {"plan": 1e3 * statistics.mean(plan_ms), "run": 1e3 * run_avg_ms,
                         "note": "events between the calls (timed region 2); the step time "
                                 "comes from timed region 1 without them"},
        "roofline": {"bound": "hbm",
                     "kernel": ("hpa_decode_step_prologue (decode_kernel with the prologue and "
                                "the plan inside + merge_kernel)" if shape.prologue and use_step
                                else "hpa_decode_run_prologue (decode_kernel + merge_kernel)"
                                if shape.prologue else
                                "hpa_decode_step (decode_kernel with the plan inside + "
                                "merge_kernel)" if use_step else
                                "hpa_decode_run (decode_kernel + merge_kernel)"),
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "traffic": traffic, "algorithmic_bytes_per_launch": run_bytes},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": (2 if use_step else 3) * K,  # (plan,) decode, merge
        "clocks": clocks,
        "plan_kernel_then_run": extras.get("plan_kernel_then_run"),
        "static_splitkv": {k: v for k, v in extras.items()
                           if k.startswith(("static", "dynamic"))} or None,
        "separate_prologue": extras.get("separate_prologue_kernel"),
        "page_sharded": extras.get("page_sharded"),
        "length_aware": extras.get("length_aware"),
        "device_status": status,
    }
    print(json.dumps(line), flush=True)


def main():
    args = _args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
