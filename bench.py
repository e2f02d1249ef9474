"""Decode-step benchmark: KV-cache GB/s and us per step, five configurations.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole decode path: the dynamic tile plan, attention and the
split merge (hpa_decode_step: the plan made inside the decode kernel, two
launches; with the fused RMSNorm + RoPE + KV-write prologue for the mix;
plan kernel + run above 512 sequences).  Inputs are synthetic (seeded
N(0,1)), shaped like the pages' workloads, and resident in HBM (xiaodao.ai
"HPC-Ops TPOT -48.8%", Attention section: uniform 64 x 0.5K and skewed
1 x 128K + 31 x 4K; bitbyai.com "vLLM x HPC-Ops", Attention Backend:
mixed-length batches with the fused prologue; aipuzi.cn "HPC-Ops", section
2.3: FP8 KV).

The headline (`value`) is the skewed batch -- 1 x 131072 + 31 x 4096 KV
tokens, 64 query heads, 8 KV heads, head_dim 128, bf16 cache, 64-token pages
shuffled over HBM -- over K back-to-back steps: live KV bytes per step / step
time, the whole job over N GPUs (each rank runs its own batch, weak
scaling).  `workloads` holds one record per configuration (tiny, uniform,
skewed, mix_prologue, fp8): median and p90 step time over 50 timed steps
after 10 untimed ones (the L2 flushed before each where the batch is not
well above the L2), the roofline against the measured HBM copy bandwidth,
the per-CTA tail idle of one step, the static split-KV plans fed to the same
kernel as interleaved A/B runs, an end-to-end figure through the public API
with host buffers, and the fp64 oracle timed on the host cores.  SM clocks
are sampled during every timed region.  The headline also gets the
three-launch form, the length-aware plan and the batch split by page range
over 2 and 8 shares (run one after another on this GPU, then merged).

--impl reference times the oracle (the plain fp64 CPU implementation) on the
host cores on a bounded sample of the skewed workload and prints the same
line with "impl": "reference".
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
    ap.add_argument("--no-workloads", action="store_true",
                    help="measure the headline workload only (no per-configuration records)")
    ap.add_argument("--ncu", action="store_true",
                    help="profiler mode: run --warmup then --steps eager steps of --workload and "
                         "exit (no timing, no JSON line), so a capture sees only decode steps")
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
    "skewed_mtp4": "multi-token decode on the skewed batch: 4 query tokens per sequence "
                   "(32 query rows per kv head), 64 q heads, 8 kv heads, head_dim 128, bf16",
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

    def stop_rows(self) -> list | None:
        """Stops sampling; the raw samples (None if nvidia-smi is missing)."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        return rows

    def stop(self) -> dict:
        return self.summarize(self.stop_rows())

    @staticmethod
    def summarize(rows) -> dict:
        """Median SM clock, max clock and the throttle reasons seen in the samples
        (of one or several timed regions)."""
        if rows is None or any(r is None for r in rows):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
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


def _add_rows(acc, rows):
    """Adds one timed region's clock samples (None: nvidia-smi missing)."""
    if rows is None:
        acc.append(None)
    else:
        acc.extend(rows)


# The benchmark configurations, each measured in every default run; the
# headline (`value`) is the skewed one.
CONFIGS = ["tiny", "uniform", "skewed", "mix_prologue", "fp8"]
ITER_WARMUP, ITERS = 10, 50        # per-config timing: 10 untimed + 50 timed steps
CPU_CONFIG_SECONDS = 3.0           # CPU baseline of each config but the headline
AB_BLOCKS, AB_PER = 5, 10          # interleaved A/B: blocks x steps on each side
CHAIN, CHAIN_REPLAYS = 8, 10       # steps per graph and replays of the chained measurement


class Case:
    """One workload's inputs, resident on the device, and its decode step
    through the public API (hpa_decode_step / hpa_decode_step_prologue; plan +
    run above 512 sequences)."""

    def __init__(self, name, dev, num_ctas, local_rank):
        import torch

        import mixed_length_paged_b200 as hpa
        from mixed_length_paged_b200 import workloads as W
        self.name, self.dev = name, dev
        b = W.build(name, device=dev, seed=0)
        s = b.shape
        self.B, self.Hq, self.Hkv, self.D, self.T = (b.batch, s.num_q_heads, s.num_kv_heads,
                                                     s.head_dim, s.q_tokens)
        self.fp8, self.prologue = s.kv_dtype == "fp8_e4m3", s.prologue
        self.k_scale = self.v_scale = None
        if self.fp8:
            b.k_cache, self.k_scale = _quantize_e4m3(b.k_cache, b.live)
            b.v_cache, self.v_scale = _quantize_e4m3(b.v_cache, b.live)
        self.batch = b
        self.lens = b.seq_lens.cpu().numpy()
        elt = 1 if self.fp8 else 2
        self.kv_bytes = W.live_kv_bytes(self.lens, self.Hkv, self.D, elt)
        tiles = int(((self.lens + 63) // 64).sum())
        # algorithmic bytes of one step: live KV + q + out + page-table entries
        # read (+ the two fp32 scales of every (page, kv head) tile for FP8;
        # + the new token's raw K/V rows read and written for the prologue)
        self.run_bytes = (self.kv_bytes + 2 * self.B * self.T * self.Hq * self.D * 2 + tiles * 4
                          + (tiles * self.Hkv * 8 if self.fp8 else 0)
                          + (4 * self.B * self.Hkv * self.D * 2 if self.prologue else 0))
        self.scale = 1.0 / math.sqrt(self.D)
        self.num_ctas = num_ctas or hpa.decode_num_ctas(self.Hq, self.Hkv, self.T, local_rank)
        self.dec = self.decoder(hpa.PLAN_DYNAMIC)
        shape = b.q_raw.shape if self.prologue else b.q.shape
        self.out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        self.use_step = self.B <= hpa.MAX_STEP_BATCH

    def decoder(self, kind, param=0):
        import mixed_length_paged_b200 as hpa
        return hpa.PagedDecoder(self.B, self.Hq, self.Hkv, self.D, self.batch.pt_stride,
                                kind=kind, param=param, num_ctas=self.num_ctas,
                                max_seq_len=int(self.lens.max()), q_tokens=self.T,
                                device=self.dev)

    def inputs(self):
        """The tensors a caller brings to every step (the KV cache, scales and
        norm weights are resident state)."""
        b = self.batch
        names = (["q_raw", "k_raw", "v_raw"] if self.prologue else ["q"]) + \
            ["seq_lens", "page_table"]
        return {n: getattr(b, n) for n in names}

    def step(self, dec=None, out=None, stream=None, inputs=None):
        b, i = self.batch, inputs or self.inputs()
        dec = dec or self.dec
        out = self.out if out is None else out
        if self.prologue:
            dec.step_prologue(i["q_raw"], i["k_raw"], i["v_raw"], b.q_gamma, b.k_gamma,
                              b.k_cache, b.v_cache, i["page_table"], i["seq_lens"], out,
                              self.scale, stream=stream, eps=1e-6, rope_theta=10000.0)
        else:
            dec.step(i["q"], b.k_cache, b.v_cache, i["page_table"], i["seq_lens"], out,
                     self.scale, k_scale=self.k_scale, v_scale=self.v_scale, stream=stream)

    def launches_per_step(self):
        return 2 if self.use_step else 3  # (plan,) decode, merge

    def kernel_name(self):
        if self.prologue:
            return ("hpa_decode_step_prologue (decode_kernel with the prologue and the plan "
                    "inside + merge_kernel)")
        return ("hpa_decode_step (decode_kernel with the plan inside + merge_kernel)"
                if self.use_step else "hpa_decode_plan + hpa_decode_run (plan_kernel, "
                "decode_kernel, merge_kernel)")


def _graphed(fn, dev, eager=False):
    """fn captured once as a CUDA graph (the PDL edges between the step's
    kernels stay programmatic edges); replaying it costs one launch call on the
    host, as a serving loop's replay of its decode step does."""
    import torch
    if eager:
        return fn, None
    stream = torch.cuda.current_stream(dev)
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
    return g.replay, g


class L2Flush:
    """Evicts the step's data from L2 before a timed iteration: writes one
    buffer of 2 x L2, then reads another of the same size, so that the L2 holds
    clean lines of unrelated data (no write-back of the flush is left to be
    charged to the step)."""

    def __init__(self, dev):
        import torch
        l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", L2_BYTES)
        n = 2 * max(int(l2), L2_BYTES) // 4
        self.a = torch.empty(n, dtype=torch.float32, device=dev)
        self.b = torch.zeros(n, dtype=torch.float32, device=dev)
        self.bytes = 2 * max(int(l2), L2_BYTES)

    def __call__(self):
        self.a.fill_(1.0)
        self.b.sum()


def _time_iters(fn, n, stream, flush=None):
    """Per-iteration CUDA-event times (ms) of n calls of fn on `stream`, each
    preceded (outside its events) by an L2 flush if given.  A sleep kernel
    first lets the host queue every iteration before the GPU reaches them."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    torch.cuda._sleep(20_000_000)
    for a, b in evs:
        if flush is not None:
            flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


class ABTotals(dict):
    """Total ms per side of an interleaved A/B, with each block's mean step
    time (us) per side in `.blocks` for the spread."""

    def spread(self, k):
        xs = sorted(self.blocks[k])
        return {"block_median_us": statistics.median(xs), "block_p90_us": _pct(xs, 0.9),
                "block_min_us": xs[0], "block_max_us": xs[-1]}


def _interleaved_ab(fns, stream, blocks=AB_BLOCKS, per=AB_PER):
    """Total ms of each function over `blocks` alternating blocks of `per`
    calls, so that clock and power drift over the run falls on all alike."""
    import torch
    tot = ABTotals({k: 0.0 for k in fns})
    tot.blocks = {k: [] for k in fns}
    for _ in range(blocks):
        for k, fn in fns.items():
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(per):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b)
            tot[k] += ms
            tot.blocks[k].append(1e3 * ms / per)
    return tot


def _pct(xs, q):
    ys = sorted(xs)
    return ys[min(len(ys) - 1, int(math.ceil(q * len(ys))) - 1)]


def _e2e(case, n, world, dev, stream):
    """The case's metric end to end through the public API (eager calls): every
    step copies its inputs from pinned host memory to the device and its
    output back, inside the timed region.  As a serving loop would, steps are
    pipelined over three streams -- copies in, compute, copy out -- with
    double-buffered device inputs and outputs, so one step's copies overlap its
    neighbours' compute."""
    import torch
    host = {k: v.cpu().pin_memory() for k, v in case.inputs().items()}
    dbuf = [{k: torch.empty_like(v) for k, v in case.inputs().items()} for _ in range(2)]
    out_h = [torch.empty(case.out.shape, dtype=case.out.dtype).pin_memory() for _ in range(2)]
    out_d = [torch.empty_like(case.out) for _ in range(2)]
    s_in, s_out, s_comp = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev), stream
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "done", "out")}
    started = [False, False]

    def one(i):
        k = i % 2
        with torch.cuda.stream(s_in):
            if started[k]:
                s_in.wait_event(ev["done"][k])   # step i-2 has read its inputs
            for name, t in host.items():
                dbuf[k][name].copy_(t, non_blocking=True)
            ev["in"][k].record(s_in)
        s_comp.wait_event(ev["in"][k])
        if started[k]:
            s_comp.wait_event(ev["out"][k])      # step i-2's output is on the host
        case.step(out=out_d[k], stream=s_comp, inputs=dbuf[k])
        ev["done"][k].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["done"][k])
            out_h[k].copy_(out_d[k], non_blocking=True)
            ev["out"][k].record(s_out)
        started[k] = True

    for i in range(4):
        one(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(n):
        one(i)
    s_in.wait_stream(s_out)                       # the last output is on the host
    s_in.wait_stream(s_comp)
    b.record(s_in)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(a.elapsed_time(b) / n, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    return {"value": job_throughput(case.kv_bytes, world, e_ms * 1e-3), "unit": "GB/s",
            "us_per_step": 1e3 * e_ms, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(out_h[0].numel() * out_h[0].element_size()),
            "steps": n,
            "method": "eager public-API calls; copies in / compute / copy out on three "
                      "streams, double-buffered, each step's copies inside the timed region"}


def _host_case(case, rows):
    """Host (numpy) copy of the sequences `rows` of a case, pages renumbered,
    for the oracle: bf16 bits, or e4m3 codes + scales, and the prologue's raw
    rows and weights."""
    import numpy as np
    import torch
    b = case.batch
    pt = b.page_table.cpu().numpy()
    sl = b.seq_lens.cpu().numpy()
    used = []
    new_pt = np.full((len(rows), pt.shape[1]), -1, dtype=np.int32)
    for i, r in enumerate(rows):
        n = (int(sl[r]) + 63) // 64
        new_pt[i, :n] = np.arange(len(used), len(used) + n)
        used.extend(pt[r, :n].tolist())
    idx = torch.tensor(used, dtype=torch.long, device=b.k_cache.device)

    def bits(t):
        return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    def rows_of(t):
        return t[rows]

    h = {"pt": new_pt, "sl": sl[rows].astype(np.int32), "Hkv": case.Hkv, "D": case.D,
         "fp8": case.fp8, "prologue": case.prologue}
    if case.fp8:
        h["k"] = b.k_cache.index_select(0, idx).cpu().numpy()
        h["v"] = b.v_cache.index_select(0, idx).cpu().numpy()
        h["ks"] = case.k_scale.index_select(0, idx).cpu().numpy()
        h["vs"] = case.v_scale.index_select(0, idx).cpu().numpy()
    else:
        h["k"] = bits(b.k_cache.index_select(0, idx))
        h["v"] = bits(b.v_cache.index_select(0, idx))
    if case.prologue:
        for n in ("q_raw", "k_raw", "v_raw"):
            h[n] = bits(rows_of(getattr(b, n)))
        h["q_gamma"] = b.q_gamma.cpu().numpy()
        h["k_gamma"] = b.k_gamma.cpu().numpy()
        h["pos"] = b.positions.cpu().numpy()[rows].astype(np.int32)
    else:
        h["q"] = bits(rows_of(b.q))
    return h


def _oracle_step(h):
    """The oracle (as it stands) on a host case: the prologue then attention,
    or attention alone; returns (seconds, live KV bytes)."""
    import oracle
    scale = 1.0 / math.sqrt(h["D"])
    if h["prologue"]:
        kc, vc = h["k"].copy(), h["v"].copy()  # the prologue writes its slots
    t0 = time.perf_counter()
    if h["prologue"]:
        q = oracle.prologue(h["q_raw"], h["k_raw"], h["v_raw"], h["q_gamma"], h["k_gamma"], 1e-6,
                            1e4, h["pos"], h["pt"], kc, vc)
        oracle.paged_decode(q, kc, vc, h["pt"], h["sl"], h["Hkv"], scale)
    elif h["fp8"]:
        oracle.paged_decode(h["q"], h["k"], h["v"], h["pt"], h["sl"], h["Hkv"], scale,
                            kv_fp8=True, k_scale=h["ks"], v_scale=h["vs"])
    else:
        oracle.paged_decode(h["q"], h["k"], h["v"], h["pt"], h["sl"], h["Hkv"], scale)
    dt = time.perf_counter() - t0
    elt = 1 if h["fp8"] else 2
    return dt, int(h["sl"].astype("int64").sum()) * 2 * h["Hkv"] * h["D"] * elt


def _cpu_leg(case, rows, min_seconds, what):
    """The oracle on the sequences `rows` of the case, repeated for at least
    min_seconds (one warm-up call first)."""
    import oracle
    h = _host_case(case, rows)
    _oracle_step(h)
    reps, secs, nbytes = 0, 0.0, 0
    while reps == 0 or secs < min_seconds:
        dt, nb = _oracle_step(h)
        secs += dt
        nbytes += nb
        reps += 1
    return {"value": nbytes / secs / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": secs,
            "sample": f"oracle (fp64, OpenMP over (sequence, kv head)) on {what}, "
                      f"{reps} times in {secs:.1f} s"}


def measure_case(case, args, world, dev, stream, peak, sampler_rows, headline):
    """One config's record: median / p90 step time over ITERS timed steps (L2
    flushed before each where the batch fits the L2), roofline, tail idle,
    static split-KV A/B, e2e."""
    import torch

    import mixed_length_paged_b200 as hpa
    for _ in range(max(3, args.warmup)):
        case.step()
    torch.cuda.synchronize()
    step, graph = _graphed(case.step, dev, args.eager)
    flush = L2Flush(dev) if case.kv_bytes <= 2 * L2_BYTES else None
    for _ in range(ITER_WARMUP):
        if flush is not None:
            flush()
        step()
    sampler = ClockSampler(_smi_index(dev.index or 0))
    sampler.start()
    ms = _time_iters(step, ITERS, stream, flush)
    _add_rows(sampler_rows, sampler.stop_rows())
    med, p90, mean = statistics.median(ms), _pct(ms, 0.9), statistics.mean(ms)
    med_max = max_over_ranks(med, world, dev)
    rec = {
        "workload": WORKLOAD_DESC.get(case.name, case.name),
        "batch": case.B, "kv_bytes_per_step": case.kv_bytes,
        "us_per_step": {"median": 1e3 * med_max, "p90": 1e3 * p90, "mean": 1e3 * mean,
                        "min": 1e3 * min(ms), "iters": ITERS, "warmup": ITER_WARMUP},
        "GB_s": job_throughput(case.kv_bytes, world, med_max * 1e-3),
        "pct_of_hbm_peak": 100.0 * case.kv_bytes / (med * 1e-3) / 1e9 / peak,
        "l2": (f"flushed before every timed step (write {flush.bytes / 1e6:.0f} MB, read "
               f"{flush.bytes / 1e6:.0f} MB; outside the step's events)" if flush is not None
               else f"no flush: {case.kv_bytes / 1e9:.3g} GB of KV per step is more than twice "
                    "the 126 MB L2"),
        "launch": "eager calls" if args.eager else "CUDA-graph replay of one captured step",
        "num_ctas": case.num_ctas,
        "roofline": {"bound": "hbm", "kernel": case.kernel_name(),
                     "achieved": case.run_bytes / (mean * 1e-3) / 1e9, "peak": peak,
                     "unit": "GB/s", "frac": case.run_bytes / (mean * 1e-3) / 1e9 / peak,
                     "basis": f"CUDA events around each of {ITERS} timed steps (all of the "
                              "step's launches), mean",
                     "algorithmic_bytes_per_launch": case.run_bytes},
    }
    # The same steps as a model's graph would hold them: CHAIN consecutive
    # steps captured in one graph, each step's decode kernel chained to the
    # merge before it by programmatic dependent launch, so its CTAs are
    # resident before that merge ends (one graph launch per CHAIN steps).
    # Only where the batch is well above the L2: consecutive steps of a
    # smaller batch would find it in the L2.
    rec["chained_us_per_step"] = None
    if flush is None:
        chain, cgraph = _graphed(lambda: [case.step() for _ in range(CHAIN)], dev, args.eager)
        for _ in range(2):
            chain()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(CHAIN_REPLAYS):
            chain()
        b.record(stream)
        torch.cuda.synchronize()
        rec["chained_us_per_step"] = 1e3 * a.elapsed_time(b) / (CHAIN * CHAIN_REPLAYS)
        rec["chained_method"] = (f"{CHAIN} steps captured in one CUDA graph (each decode kernel "
                                 f"PDL-chained to the merge before it), {CHAIN_REPLAYS} replays")
        del cgraph
    # load balance of one step, from the run kernel's per-CTA timeline
    case.step()
    torch.cuda.synchronize()
    rec["device_status"] = case.dec.status()
    rec["tail_idle"] = hpa.tail_idle(case.dec.cta_times())
    if not args.no_extras:
        # static split-KV: the same run kernel fed the two static plans,
        # interleaved A/B against the dynamic step
        rec["static_splitkv"] = {}
        for sname, kind in (("fixed_split_count", hpa.PLAN_STATIC_NSPLIT),
                            ("fixed_split_size", hpa.PLAN_STATIC_CHUNK)):
            sd = case.decoder(kind)
            for _ in range(3):
                case.step(dec=sd)
            torch.cuda.synchronize()
            s_fn, s_graph = _graphed(lambda sd=sd: case.step(dec=sd), dev, args.eager)
            tot = _interleaved_ab({"dynamic": step, "static": s_fn}, stream)
            n = AB_BLOCKS * AB_PER
            rec["static_splitkv"][sname] = {
                "us_per_step": 1e3 * tot["static"] / n, "grid": sd.grid,
                "dynamic_us_per_step_same_blocks": 1e3 * tot["dynamic"] / n,
                "dynamic_speedup": tot["static"] / tot["dynamic"],
                "static_blocks": tot.spread("static"), "dynamic_blocks": tot.spread("dynamic"),
                "method": f"interleaved A/B, {AB_BLOCKS} x {AB_PER} graph replays each, no flush"}
            del s_graph
        rec["static_splitkv"]["dynamic_speedup_vs_best_static"] = min(
            v["dynamic_speedup"] for v in rec["static_splitkv"].values())
        rec["e2e"] = _e2e(case, max(ITERS, min(500, args.steps)) if headline else ITERS,
                          world, dev, stream)
    del graph
    return rec, step


def _cpu_rows(name, B):
    """Sequences of a config the CPU baseline runs, and how they are named."""
    if name == "mix_prologue":
        return list(range(0, B, 8)), f"{len(range(0, B, 8))} of the 128 sequences (every 8th), prologue + attention"
    if name == "fp8":
        return list(range(0, B, 4)), f"{len(range(0, B, 4))} of the 256 sequences (every 4th), e4m3 KV"
    return list(range(B)), f"the whole {name} step ({B} sequences)"


def _headline_extras(case, args, world, dev, stream, step):
    """Comparisons on the headline workload only: the three-launch form, the
    length-aware plan, the batch spread by page range, the separate prologue."""
    import numpy as np
    import torch

    import mixed_length_paged_b200 as hpa
    extras = {}
    b = case.batch
    n = AB_BLOCKS * AB_PER * 2
    blocks, per = 2 * AB_BLOCKS, AB_PER
    if case.use_step and not case.prologue:
        # the same step as plan kernel + run (three launches), interleaved A/B
        pr = case.decoder(hpa.PLAN_DYNAMIC)

        def plan_then_run():
            pr(b.q, b.k_cache, b.v_cache, b.page_table, b.seq_lens, case.out, case.scale,
               k_scale=case.k_scale, v_scale=case.v_scale)

        for _ in range(3):
            plan_then_run()
        sep, g = _graphed(plan_then_run, dev, args.eager)
        ab = _interleaved_ab({"step": step, "plan_run": sep}, stream, blocks, per)
        extras["plan_kernel_then_run"] = {
            "us_per_step": 1e3 * ab["plan_run"] / n,
            "in_kernel_plan_us_per_step_same_blocks": 1e3 * ab["step"] / n,
            "in_kernel_plan_speedup": ab["plan_run"] / ab["step"],
            "plan_run_blocks": ab.spread("plan_run"), "step_blocks": ab.spread("step"),
            "method": f"interleaved A/B, {blocks} x {per} steps each"}
        # the length-aware plan (cut points moved off segment ends, smallest
        # end piece m tiles) against the dynamic plan, both as plan kernel + run
        extras["length_aware"] = {}
        for m in (2, 4, 8):
            ld = case.decoder(hpa.PLAN_LENGTH_AWARE, param=m)

            def la_step(ld=ld):
                ld(b.q, b.k_cache, b.v_cache, b.page_table, b.seq_lens, case.out, case.scale,
                   k_scale=case.k_scale, v_scale=case.v_scale)

            for _ in range(3):
                la_step()
            la, g2 = _graphed(la_step, dev, args.eager)
            ab = _interleaved_ab({"dynamic": sep, "length_aware": la}, stream, blocks, per)
            extras["length_aware"][f"m{m}"] = {
                "us_per_step": 1e3 * ab["length_aware"] / n,
                "dynamic_plan_run_us_same_blocks": 1e3 * ab["dynamic"] / n,
                "speedup_vs_dynamic": ab["dynamic"] / ab["length_aware"],
                "length_aware_blocks": ab.spread("length_aware"),
                "method": f"plan kernel + run each, interleaved A/B, {blocks} x {per} steps"}
    if case.prologue:
        # the prologue as its own kernel before plan + run, against the fused step
        q_out = torch.empty_like(b.q_raw)
        pr = case.decoder(hpa.PLAN_DYNAMIC)

        def separate():
            hpa.kv_prologue(b.q_raw, b.k_raw, b.v_raw, b.q_gamma, b.k_gamma, b.positions,
                            b.page_table, b.k_cache, b.v_cache, q_out, eps=1e-6,
                            rope_theta=10000.0)
            pr(q_out, b.k_cache, b.v_cache, b.page_table, b.seq_lens, case.out, case.scale)

        for _ in range(3):
            separate()
        sep, g = _graphed(separate, dev, args.eager)
        ab = _interleaved_ab({"fused": step, "separate": sep}, stream, blocks, per)
        extras["separate_prologue_kernel"] = {
            "us_per_step": 1e3 * ab["separate"] / n,
            "fused_us_per_step_same_blocks": 1e3 * ab["fused"] / n,
            "fused_speedup": ab["separate"] / ab["fused"],
            "separate_blocks": ab.spread("separate"), "fused_blocks": ab.spread("fused"),
            "method": f"interleaved A/B, {blocks} x {per} steps each"}
    if case.use_step and not case.prologue and not case.fp8 and case.T == 1:
        # The batch spread by page range over R ranks (sharding.page_shard),
        # the R shares run one after another on this GPU, each a decode step
        # with log-sum-exps, then the merge of the R states.  The slowest
        # share is what one of R GPUs would spend on its decode; the
        # all-gather between the two is not measured (one GPU).
        from mixed_length_paged_b200 import sharding as SH
        extras["page_sharded"] = {}
        for R in (2, 8):
            parts = []
            for r in range(R):
                lr, ptr = SH.page_shard(b.seq_lens, b.page_table, R, r)
                parts.append((case.decoder(hpa.PLAN_DYNAMIC), lr.to(dev), ptr.to(dev),
                              torch.empty(case.B, case.Hq, case.D, dtype=torch.float32, device=dev),
                              torch.empty(case.B, case.Hq, dtype=torch.float32, device=dev)))
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
                    sd.step(b.q, b.k_cache, b.v_cache, ptr, lr, o, case.scale, lse=l)
                if e:
                    e[R].record(stream)
                hpa.merge_states(o_parts, l_parts, case.out)
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
    return extras


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import mixed_length_paged_b200 as hpa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hpa.lib()
    stream = torch.cuda.current_stream()
    peak, peak_kind = _peaks()
    clock_rows = []

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # 1. the headline workload: its record, then K back-to-back steps (the value)
    case = Case(args.workload, dev, args.num_ctas, local_rank)
    if args.ncu:
        for _ in range(args.warmup + args.steps):
            case.step()
        torch.cuda.synchronize()
        print(f"ncu mode: {args.warmup + args.steps} steps of {case.name}, device status "
              f"{case.dec.status()}", flush=True)
        return
    rec, step = measure_case(case, args, world, dev, stream, peak, clock_rows, headline=True)
    K = args.steps
    barrier()
    sampler = ClockSampler(_smi_index(local_rank))
    sampler.start()
    barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(K):
        step()
    end.record(stream)
    barrier()
    _add_rows(clock_rows, sampler.stop_rows())
    ms_per_step = max_over_ranks(start.elapsed_time(end), world, dev) / K
    extras = {} if args.no_extras else _headline_extras(case, args, world, dev, stream, step)
    cpu_legs = rank == 0 and world == 1 and not args.no_cpu_baseline
    if cpu_legs:
        rows, what = _cpu_rows(case.name, case.B)
        secs = CPU_BASELINE_SECONDS if case.name == WORKLOAD else CPU_CONFIG_SECONDS
        rec["cpu_baseline"] = _cpu_leg(case, rows, secs, what)
    head = dict(name=case.name, kv_bytes=case.kv_bytes, B=case.B, num_ctas=case.num_ctas,
                launches=case.launches_per_step(), fp8=case.fp8)
    del case, step
    torch.cuda.empty_cache()

    # 2. every other benchmark configuration, one at a time
    records = {head["name"]: rec}
    if args.workload == WORKLOAD and not args.no_workloads:
        for name in CONFIGS:
            if name in records:
                continue
            c = Case(name, dev, args.num_ctas, local_rank)
            r, _ = measure_case(c, args, world, dev, stream, peak, clock_rows, headline=False)
            if cpu_legs:
                rows, what = _cpu_rows(name, c.B)
                r["cpu_baseline"] = _cpu_leg(c, rows, CPU_CONFIG_SECONDS, what)
            records[name] = r
            del c, _
            torch.cuda.empty_cache()
        records = {n: records[n] for n in CONFIGS}
    clocks = ClockSampler.summarize(clock_rows)

    if rank != 0:
        return
    roof = dict(rec["roofline"])
    if head["name"] == WORKLOAD:
        roof["traffic"] = _profiled_traffic()
    roof["peak_kind"] = f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
    value = job_throughput(head["kv_bytes"], world, ms_per_step * 1e-3)
    metric = METRIC if head["name"] == WORKLOAD else \
        f"KV-cache GB/s (% of HBM peak), µs/decode step, {head['name']}"
    line = {
        "metric": metric, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 KV / bf16" if head["fp8"] else "bf16", "data": "synthetic",
        "us_per_step": 1e3 * ms_per_step,
        "us_per_step_median": rec["us_per_step"]["median"],
        "us_per_step_p90": rec["us_per_step"]["p90"],
        "us_per_step_chained_in_graph": rec.get("chained_us_per_step"),
        "pct_of_hbm_peak": 100.0 * (head["kv_bytes"] / (ms_per_step * 1e-3) / 1e9) / peak,
        "config": {
            "workload": WORKLOAD_DESC.get(head["name"], head["name"]),
            "batch": head["B"], "kv_bytes_per_step_per_gpu": head["kv_bytes"],
            "num_ctas": head["num_ctas"],
            "l2": rec["l2"],
            "launch": rec["launch"],
            "timing": f"value: {K} back-to-back steps between two CUDA events; median/p90: "
                      f"{ITERS} steps with events around each",
            "parallelism": f"data-parallel replicas x{world} (independent batches, no collective)",
        },
        "roofline": roof,
        "cpu_baseline": rec.get("cpu_baseline"),
        "e2e": rec.get("e2e"),
        "gpu_launches": head["launches"] * K,
        "clocks": clocks,
        "tail_idle": rec["tail_idle"],
        "static_splitkv": rec.get("static_splitkv"),
        "plan_kernel_then_run": extras.get("plan_kernel_then_run"),
        "separate_prologue": extras.get("separate_prologue_kernel"),
        "page_sharded": extras.get("page_sharded"),
        "length_aware": extras.get("length_aware"),
        "device_status": rec["device_status"],
        "workloads": records if len(records) > 1 else None,
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
