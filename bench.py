#!/usr/bin/env python
"""Benchmark of one chunk-step of block-causal sink + window TwinCache attention.

A step is one chunk of the stream at steady state (window full, eviction on):
every denoising step's attention (sa_stage_keys + sa_attend_staged; the last
step reads the clean tier) followed by the append of the chunk's noisy and
clean K/V (sa_append_chunk x2). Inputs are seeded synthetic bf16 tensors of the
workload's shape, resident in HBM before the timed region.

Prints ONE JSON line (rank 0). ``value`` is attention TFLOP/s over all ranks
(FLOPs = 4 * B * H * L * Lkv * D per attention); ``ms_per_step`` the time of a
chunk-step. With torchrun each rank runs its own independent stream (weak
scaling, no data-path collective); the barrier and the max over ranks of the
device time use NCCL.

``--impl reference`` times the float64 CPU oracle on the host cores on a
bounded sample of the same workload instead.
"""

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms per chunk-step and attention TFLOP/s (% of B200 bf16 peak) at 720p shape"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2 ** 20
SUSTAINED_REGION_S = 2.0  # timed regions at least this long compare with the sustained peak


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="refiner_720p")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--sparsity", type=float, default=0.0,
                    help="block-sparse mode: share of 128x128 blocks skipped (seeded random mask)")
    ap.add_argument("--ulysses", action="store_true",
                    help="head-sharded attention over the ranks (Ulysses, fp8 exchange)")
    ap.add_argument("--transport", choices=["nccl", "p2p"], default="nccl",
                    help="Ulysses exchange: NCCL all-to-all, or quantise straight into peer memory")
    ap.add_argument("--editing", action="store_true",
                    help="frame-aligned editing attention (source frames of the chunk as extra keys)")
    ap.add_argument("--ref-frames", type=int, default=0,
                    help="frames of a reference image every chunk also attends (0: none)")
    ap.add_argument("--launch-gaps", type=int, default=0, metavar="STEPS",
                    help="after the timed region, trace STEPS more chunk-steps with the CUDA "
                         "activity profiler and report the idle gaps between kernels")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    args = ap.parse_args()
    if not 0.0 <= args.sparsity < 1.0:
        ap.error("--sparsity must be in [0, 1)")
    if sum((args.ulysses, args.editing, args.sparsity > 0)) > 1:
        ap.error("--ulysses, --editing and --sparsity select different workloads; give one")
    if args.sparsity > 0 and args.ref_frames > 0:
        ap.error("block-sparse attention takes no reference image (--ref-frames 0)")
    return args


def attend_flops(w):
    return 4.0 * w.batch * w.heads * w.chunk_len * w.kv_len * w.head_dim


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_code_hash(path):
    """First 16 hex digits of the SHA-256 of a CUDA source with its // comments
    and blank lines removed and each line stripped, so that an edit to comments
    alone keeps the hash (and a profile taken on that code stays valid)."""
    lines = []
    for line in open(path, encoding="utf-8").read().splitlines():
        code = re.sub(r"//.*$", "", line).strip()
        if code:
            lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def kernel_traffic(kernel_file, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the kernel code as it is now (comments aside); else None."""
    src = os.path.join(ROOT, "block_causal_streaming_sa_b200", "csrc", "kernels", kernel_file)
    summ = os.path.join(ROOT, "profiles", f"attend_tc_{workload}.txt")
    try:
        sha = kernel_code_hash(src)
        text = open(summ).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*(\d+)\s*;\s*source_sha256_16:\s*([0-9a-f]+)", text)
    if m and m.group(2) == sha:
        return int(m.group(1))
    return None


class ClockSampler:
    """SM clock, power and clock-event reasons sampled through NVML every ~2 ms
    on a thread while the timed region runs (so a region of tens of ms still
    gets tens of samples); ``stop`` keeps the samples taken between
    ``mark_start`` and ``mark_stop`` (host times that bracket the device's
    timed region). Falls back to ``nvidia-smi -lms`` when NVML is missing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    # NVML clock-event reason bits of the four names above
    BITS = (0x8, 0x40, 0x20, 0x4)
    PERIOD_S = 0.002

    def __init__(self, bus_id):
        import threading

        self.samples = []  # (host time, sm MHz, max sm MHz, power W, reason bits)
        self.t0 = self.t1 = None
        self.proc = None
        self.nvml = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.dev = pynvml.nvmlDeviceGetHandleByPciBusId(bus_id)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.dev, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.halt = threading.Event()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", bus_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def _loop(self):
        n = self.nvml
        reasons_fn = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            n.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.halt.is_set():
            try:
                t = time.perf_counter()
                sm = n.nvmlDeviceGetClockInfo(self.dev, n.NVML_CLOCK_SM)
                power = n.nvmlDeviceGetPowerUsage(self.dev) / 1000.0
                bits = reasons_fn(self.dev)
                self.samples.append((t, float(sm), float(self.max_mhz), power, int(bits),
                                     time.perf_counter()))
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_stop(self):
        self.t1 = time.perf_counter()

    def stop(self):
        if self.nvml is not None:
            self.halt.set()
            self.thread.join(timeout=5)
            # a sample counts when its queries overlap the region
            rows = [s for s in self.samples
                    if (self.t0 is None or s[5] >= self.t0) and (self.t1 is None or s[0] <= self.t1)]
            sm = [r[1] for r in rows]
            smax = [r[2] for r in rows]
            power = [r[3] for r in rows]
            reasons = {name for r in rows for name, bit in zip(self.NAMES, self.BITS)
                       if r[4] & bit}
            source = "nvml"
        elif self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            sm, smax, power, reasons = [], [], [], set()
            for line in out.strip().splitlines():
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for name, val in zip(self.NAMES, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
            source = "nvidia-smi"
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"],
                    "source": source}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "sm_mhz_min": min(sm), "power_w_median": statistics.median(power),
                "samples": len(sm), "source": source, "reasons": sorted(reasons)}


def bus_id_of(dev):
    import torch

    p = torch.cuda.get_device_properties(dev)
    return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


# ------------------------------------------------------------------ oracle (CPU) legs


class OracleSample:
    """The float64 oracle on a bounded sample of the workload: the generating
    chunk at steady state, one (batch, head) pair and a few query rows per call,
    in the mode the bench line names (reference image, frame-aligned editing or
    a block-sparse mask), with the same seeded inputs and mask as the GPU arm."""

    def __init__(self, w, ref_frames=0, editing=False, sparsity=0.0):
        import numpy as np
        import torch

        from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle
        from sa_inputs import normal_bf16, seed_of

        self.np = np
        self.w = w
        self.editing = editing
        cfg = OracleConfig(w.batch, w.heads, w.head_dim, w.frames, w.tok_h, w.tok_w, w.sink,
                           w.window, ref_frames=ref_frames)
        self.orc = StreamOracle(cfg)
        f64 = lambda t: t.to(torch.float64).numpy()  # noqa: E731
        hw = w.tok_h * w.tok_w
        if ref_frames > 0:
            shape = (w.batch, ref_frames * hw, w.heads, w.head_dim)
            self.orc.set_reference(*(f64(normal_bf16(seed_of(w.name, "reference", n), shape))
                                     for n in ("K", "V")))
        pool = [{n: f64(w.tensor(n, c)) for n in ("Kn", "Vn", "Kcl", "Vcl")} for c in range(2)]
        for c in range(w.sink + w.window - 1):
            s = pool[c % 2]
            self.orc.append(NOISY, s["Kn"], s["Vn"])
            self.orc.append(CLEAN, s["Kcl"], s["Vcl"])
        names = ("Q", "Kc", "Vc") + (("Ks", "Vs") if editing else ())
        self.cur = {n: f64(w.tensor(n, 9)) for n in names}
        # keys each query row sees (sparse: per query tile, from the mask)
        self.row_keys = w.kv_len + ref_frames * hw + (hw if editing else 0)
        self.mask = None
        if sparsity > 0:
            nq = -(-w.chunk_len // 128)
            gen = torch.Generator().manual_seed(1234)
            mask = torch.rand((w.batch, w.heads, nq, (w.sink + w.window) * nq), generator=gen)
            self.mask = (mask >= sparsity).numpy()
            tile_keys = np.full(nq, 128)
            tile_keys[-1] = w.chunk_len - 128 * (nq - 1)
            self.tile_row_keys = (self.mask * np.tile(tile_keys, w.sink + w.window)).sum(-1)
        self.rng = np.random.default_rng(3)
        self.calls = 0
        self.mode = ("block-sparse" if sparsity > 0 else "frame-aligned editing" if editing
                     else "dense") + (f", {ref_frames}-frame reference" if ref_frames else "")

    def run(self, rows):
        """One sample: `rows` query rows of one (b, h); returns its FLOPs."""
        from oracle.editing import frame_aligned_attend
        from oracle.sparse import block_sparse_attend

        w = self.w
        bh = self.calls % (w.batch * w.heads)
        self.calls += 1
        b, h = divmod(bh, w.heads)
        sel = self.rng.choice(w.chunk_len, size=rows, replace=False)
        cur = self.cur
        if self.mask is not None:
            block_sparse_attend(self.orc, cur["Q"], cur["Kc"], cur["Vc"], True, self.mask,
                                rows=sel, heads=[h], batches=[b])
            return 4.0 * w.head_dim * float(self.tile_row_keys[b, h, sel // 128].sum())
        if self.editing:
            frame_aligned_attend(self.orc, cur["Q"], cur["Kc"], cur["Vc"], cur["Ks"], cur["Vs"],
                                 True, rows=sel, heads=[h], batches=[b])
        else:
            self.orc.attend(cur["Q"], cur["Kc"], cur["Vc"], True, rows=sel, heads=[h],
                            batches=[b])
        return 4.0 * rows * self.row_keys * w.head_dim

    def calibrate(self, seconds):
        """Rows per call such that one call takes about `seconds`."""
        t = time.perf_counter()
        self.run(16)
        t16 = time.perf_counter() - t
        t = time.perf_counter()
        self.run(128)
        t128 = time.perf_counter() - t
        per_row = max((t128 - t16) / 112, 1e-6)
        fixed = max(t16 - 16 * per_row, 0.0)
        return int(min(self.w.chunk_len, max(16, (seconds - fixed) / per_row)))


def oracle_sample(w, args):
    o = OracleSample(w, ref_frames=args.ref_frames, editing=args.editing,
                     sparsity=args.sparsity)
    if args.ulysses:
        o.mode += " (Ulysses layer: all heads, exchanges not sampled)"
    return o


def cpu_baseline(w, args):
    o = oracle_sample(w, args)
    seconds = args.cpu_seconds
    rows = o.calibrate(min(seconds / 3, 5.0))
    flops, t0 = 0.0, time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        flops += o.run(rows)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{o.calls - 2} calls x {rows} query rows of one (b,h) each, "
                      f"{o.mode} attention over the chunk's keys, final (clean-tier) step "
                      f"at steady state, {dt:.1f} s of float64 numpy on the host"}


def workload_config(w, args, world):
    """The `config` object of a bench line (both arms describe the same workload)."""
    cache_bytes_read = 2 * (w.kv_len - w.chunk_len) * w.batch * w.heads * w.head_dim * 2
    return {
        "workload": w.name, "batch": w.batch, "heads": w.heads, "head_dim": w.head_dim,
        "chunk_tokens": w.chunk_len, "kv_tokens": w.kv_len, "sink_chunks": w.sink,
        "window_chunks": w.window, "denoise_steps_per_chunk": w.steps, "layers": w.layers,
        "step": "all denoising attentions of one chunk (every layer) + noisy and clean appends",
        "l2": f"inputs larger than L2: {cache_bytes_read / 2**20:.0f} MiB of cached K/V "
              f"read per attention vs {L2_BYTES / 2**20:.0f} MiB L2",
        "parallelism": (f"ulysses{world}-{args.transport}" if args.ulysses else
                        f"replicas{world}" if world > 1 else "single"),
        "block_sparsity": args.sparsity,
        "ref_frames": args.ref_frames,
        "ref_tokens": args.ref_frames * w.tok_h * w.tok_w,
        "frame_aligned_editing": args.editing,
    }


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    o = oracle_sample(w, args)
    rows = o.calibrate(0.15)
    for _ in range(args.warmup):
        o.run(rows)
    flops, t0 = 0.0, time.perf_counter()
    for _ in range(args.steps):
        flops += o.run(rows)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = (f"each step: {rows} query rows of one (b,h), {o.mode} attention over the "
              f"chunk's keys (float64 numpy oracle, host cores)")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": dict(workload_config(w, args, args.gpus), sample=sample),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def launch_gap_trace(run_steps, n_steps):
    """Kernel timeline of n_steps chunk-steps from the CUDA activity profiler
    (CUPTI through torch.profiler; outside every timed region): busy time,
    idle gaps between consecutive kernels, and time per kernel name."""
    import tempfile

    import torch
    from torch.profiler import ProfilerActivity, profile

    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        run_steps(n_steps)
        torch.cuda.synchronize()
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "trace.json")
        prof.export_chrome_trace(path)
        with open(path) as f:
            events = json.load(f).get("traceEvents", [])
    ks = sorted((float(e["ts"]), float(e["dur"]), e["name"]) for e in events
                if e.get("cat") == "kernel")
    if not ks:
        return {"kernels": 0, "note": "the profiler recorded no kernel"}
    gaps = [max(0.0, ks[i + 1][0] - (ks[i][0] + ks[i][1])) for i in range(len(ks) - 1)]
    span = ks[-1][0] + ks[-1][1] - ks[0][0]
    busy = sum(k[1] for k in ks)
    per_name = {}
    for _, dur, name in ks:
        short = re.sub(r"\(.*", "", name)
        c, t = per_name.get(short, (0, 0.0))
        per_name[short] = (c + 1, t + dur)
    q = statistics.quantiles(gaps, n=10) if len(gaps) >= 2 else [0.0] * 9
    return {
        "steps": n_steps, "kernels": len(ks), "span_ms": span / 1e3, "busy_ms": busy / 1e3,
        "idle_ms": (span - busy) / 1e3, "idle_share": (span - busy) / span,
        "gap_us": {"median": statistics.median(gaps) if gaps else 0.0, "p90": q[8],
                   "max": max(gaps) if gaps else 0.0, "sum": sum(gaps)},
        "by_kernel": {k: {"launches": c, "ms": t / 1e3} for k, (c, t) in per_name.items()},
    }


# ------------------------------------------------------------------ ranks


class Ranks:
    """Rank plumbing of a torchrun launch (also runs on CPU with gloo in tests).

    Every rank takes the same collective steps in the same order: a barrier
    around the timed region and one max-reduction per reported time.
    """

    def __init__(self, backend="nccl", device=None, timeout_s=120):
        import torch.distributed as dist

        self.dist = dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        if self.world > 1:
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max(self, x):
        """Max of a float over ranks (the slowest rank's time)."""
        import torch

        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        if self.world > 1:
            self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def append_line(append_ms, append_gbs, launch_ms, launch_bytes, hbm):
    """The `append` object: one append launch on its own (K and V of one tier, each
    read once and written once: launch_bytes) against the HBM peak, and the whole
    chunk's appends (every layer, both tiers, kernel boundaries included)."""
    out = {"chunk_ms": statistics.fmean(append_ms), "chunk_GB_per_s": append_gbs,
           "chunk_frac_of_hbm": append_gbs / hbm, "bytes_per_launch": launch_bytes}
    if launch_ms:
        t = statistics.fmean(launch_ms)
        out.update({"ms": t, "GB_per_s": launch_bytes / (t * 1e-3) / 1e9,
                    "frac_of_hbm": launch_bytes / (t * 1e-3) / 1e9 / hbm})
    return out


def whole_job_tflops(flops_per_rank, ms_max, world):
    """Aggregate throughput: the work of all ranks over the slowest rank's time."""
    return flops_per_rank * world / (ms_max * 1e-3) / 1e12


# ------------------------------------------------------------------ GPU leg


def run_ours(args, w):
    import torch

    import block_causal_streaming_sa_b200 as sa
    from sa_inputs import normal_bf16, seed_of

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    barrier, max_over_ranks = ranks.barrier, ranks.max

    stream = torch.cuda.Stream(device=dev)
    names = ("Q", "Kc", "Vc", "Kn", "Vn", "Kcl", "Vcl") + (("Ks", "Vs") if args.editing else ())
    shard = slice(None)
    if args.ulysses:
        # Ulysses: every rank holds 1/N of each chunk's tokens with all heads
        if w.chunk_len % world or w.heads % world:
            raise SystemExit("--ulysses needs tokens and heads divisible by the rank count")
        t = w.chunk_len // world
        shard = slice(rank * t, (rank + 1) * t)
    pool_host = [{n: w.tensor(n, 100 + c, layer=0 if args.ulysses else rank)[:, shard]
                  .contiguous().pin_memory() for n in names} for c in range(2)]
    pool = [{n: t.to(dev) for n, t in s.items()} for s in pool_host]
    out_shape = tuple(pool[0]["Q"].shape)
    out = torch.empty(out_shape, dtype=torch.bfloat16, device=dev)
    out_host = torch.empty(out_shape, dtype=torch.bfloat16).pin_memory()

    # One handle (its own two-tier cache) per attention layer of the workload.
    cfg = dict(w.config_dict(), ref_frames=args.ref_frames)
    if args.ulysses:
        from block_causal_streaming_sa_b200.ulysses import UlyssesAttention

        layers = [UlyssesAttention(cfg, device=dev, transport=args.transport)
                  for _ in range(w.layers)]
    else:
        layers = [sa.StreamingAttention(cfg, device=dev) for _ in range(w.layers)]
    attn = layers[0]
    sp = stream.cuda_stream
    flops = attend_flops(w)
    ref_len = args.ref_frames * w.tok_h * w.tok_w
    if args.ref_frames > 0:
        # A reference image of ref_frames frames, set once (its keys are rotated
        # on the way in); every attention also reads its ref_len keys.
        ref_shape = (w.batch, ref_len, w.heads, w.head_dim)
        ref_shard = slice(None)
        if args.ulysses:
            t = ref_len // world
            ref_shard = slice(rank * t, (rank + 1) * t)
        Kref, Vref = (normal_bf16(seed_of(w.name, "reference", n), ref_shape)[:, ref_shard]
                      .contiguous().to(dev) for n in ("K", "V"))
        for layer in layers:
            layer.set_reference(Kref, Vref)
        torch.cuda.synchronize(dev)
        flops += 4.0 * w.batch * w.heads * w.chunk_len * ref_len * w.head_dim
    if args.editing:
        # every query row also sees the tok_h * tok_w source tokens of its own frame
        flops += 4.0 * w.batch * w.heads * w.chunk_len * (w.tok_h * w.tok_w) * w.head_dim
    steps_per_chunk = w.steps
    attends_per_chunk = steps_per_chunk * w.layers
    appends_per_chunk = 2 * w.layers

    def append_all(s, launch_ev=None):
        """The chunk's appends; launch_ev = three events around the first layer's two
        append launches (each launch timed on its own)."""
        if args.ulysses:
            for layer in layers:
                layer.append(sa.SA_TIER_NOISY, s["Kn"], s["Vn"])
                layer.append(sa.SA_TIER_CLEAN, s["Kcl"], s["Vcl"])
            return
        for li, layer in enumerate(layers):
            h = layer.handle
            timed = launch_ev is not None and li == 0
            if timed:
                launch_ev[0].record(stream)
            sa.sa_append_chunk(h, sa.SA_TIER_NOISY, s["Kn"].data_ptr(), s["Vn"].data_ptr(), sp)
            if timed:
                launch_ev[1].record(stream)
            sa.sa_append_chunk(h, sa.SA_TIER_CLEAN, s["Kcl"].data_ptr(), s["Vcl"].data_ptr(), sp)
            if timed:
                launch_ev[2].record(stream)

    block_mask = None
    if args.sparsity > 0:
        # Steady-state chunk: S + W attended chunks; a seeded mask with the given share
        # of 128x128 blocks skipped. FLOPs count only the flagged blocks.
        nq = -(-w.chunk_len // 128)
        nk = (w.sink + w.window) * nq
        gen = torch.Generator().manual_seed(1234)
        block_mask = (torch.rand((w.batch, w.heads, nq, nk), generator=gen) >= args.sparsity)
        rows = torch.full((nq,), 128.0)
        rows[-1] = w.chunk_len - 128 * (nq - 1)
        keys = rows.repeat(w.sink + w.window)
        flops = float(4.0 * w.head_dim * (block_mask.double() * rows[:, None].double()
                                          * keys[None, :].double()).sum())
        block_mask = block_mask.to(torch.uint8).to(dev)

    res = [out]  # the last attention output (the Ulysses layer returns its own tensor)

    def chunk_step(s, ev=None):
        """One chunk: every denoising step's attention in every layer, then the appends."""
        a = 0
        for k in range(steps_per_chunk):
            final = k == steps_per_chunk - 1
            for layer in layers:
                if args.ulysses:
                    # the whole layer call: exchanges in, attention, exchange out
                    if ev is not None:
                        ev[0][a].record(stream)
                    res[0] = layer.attend(s["Q"], s["Kc"], s["Vc"], final)
                    if ev is not None:
                        ev[1][a].record(stream)
                    a += 1
                    continue
                h = layer.handle
                if args.editing:
                    # editing: the staging of Kc and Ks is inside the timed call
                    if ev is not None:
                        ev[0][a].record(stream)
                    sa.sa_attend_aligned(h, s["Q"].data_ptr(), s["Kc"].data_ptr(),
                                         s["Vc"].data_ptr(), s["Ks"].data_ptr(),
                                         s["Vs"].data_ptr(), w.frames, final, out.data_ptr(), 0,
                                         sp)
                elif block_mask is not None:
                    # sparse: the staging kernel is inside the timed attention call
                    if ev is not None:
                        ev[0][a].record(stream)
                    sa.sa_attend_sparse(h, s["Q"].data_ptr(), s["Kc"].data_ptr(),
                                        s["Vc"].data_ptr(), final, block_mask.data_ptr(),
                                        out.data_ptr(), 0, sp)
                else:
                    sa.sa_stage_keys(h, s["Kc"].data_ptr(), sp)
                    if ev is not None:
                        ev[0][a].record(stream)
                    sa.sa_attend_staged(h, s["Q"].data_ptr(), s["Vc"].data_ptr(), final,
                                        out.data_ptr(), 0, sp)
                if ev is not None:
                    ev[1][a].record(stream)
                a += 1
        if ev is not None:
            ev[2].record(stream)
        append_all(s, ev[4] if ev is not None else None)
        if ev is not None:
            ev[3].record(stream)

    with torch.cuda.stream(stream):
        # Fill the window so every timed chunk attends to S + W chunks.
        # the clock sampler runs from before the warm-up, so that it is in its
        # steady state when a short timed region starts
        clocks = ClockSampler(bus_id_of(dev)) if rank == 0 else None
        for c in range(w.sink + w.window - 1):
            append_all(pool[c % 2])
        for i in range(args.warmup):
            chunk_step(pool[i % 2])
        stream.synchronize()

        mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        evs = [([mk() for _ in range(attends_per_chunk)], [mk() for _ in range(attends_per_chunk)],
                mk(), mk(), [mk(), mk(), mk()]) for _ in range(args.steps)]
        start, stop = mk(), mk()
        barrier()
        torch.cuda.synchronize(dev)
        if clocks is not None:
            clocks.mark_start()
        start.record(stream)
        for i in range(args.steps):
            chunk_step(pool[i % 2], evs[i])
        stop.record(stream)
        stream.synchronize()
        if clocks is not None:
            clocks.mark_stop()
        torch.cuda.synchronize(dev)
        clock_info = clocks.stop() if clocks is not None else None
        # the SM clock the last timed attention kernel ran at, from its own
        # per-CTA cycle-counter and global-timer stamps
        try:
            kernel_clock = sa.sa_debug_kernel_clock()
        except sa.SaError:
            kernel_clock = None
        barrier()
        ms_local = start.elapsed_time(stop)
        attend_ms = [e[0][k].elapsed_time(e[1][k]) for e in evs for k in range(attends_per_chunk)]
        append_ms = [e[2].elapsed_time(e[3]) for e in evs]
        # each append launch alone (first layer's noisy and clean appends)
        launch_ms = ([e[4][0].elapsed_time(e[4][1]) for e in evs] +
                     [e[4][1].elapsed_time(e[4][2]) for e in evs]) if not args.ulysses else []
        assert attn.status(stream) == sa.SA_OK, "device status word reports a timeout"

        # End to end through the public API with host buffers: every step copies
        # its seven input tensors host -> device and its output device -> host,
        # all inside the timed region. As a streaming caller would, the copies are
        # pipelined: inputs of step i+1 go up (one copy stream) and the output of
        # step i comes down (another) while step i computes; two input buffer sets
        # and two output staging buffers, ordered by events.
        e2e_steps = max(1, args.e2e_steps)
        h2d = sum(t.numel() * t.element_size() for t in pool_host[0].values())
        d2h = out_host.numel() * out_host.element_size()
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        dev_bufs = [{n: torch.empty_like(t) for n, t in pool[0].items()} for _ in range(2)]
        out_dev = [torch.empty_like(out) for _ in range(2)]
        out_hosts = [out_host, torch.empty_like(out_host).pin_memory()]

        def e2e_run(n_steps, start_ev=None):
            copied = [mk() for _ in range(n_steps)]
            computed = [mk() for _ in range(n_steps)]
            fetched = [mk() for _ in range(n_steps)]
            for i in range(n_steps):
                k = i % 2
                with torch.cuda.stream(up):
                    if i == 0 and start_ev is not None:
                        up.wait_event(start_ev)
                    if i >= 2:
                        up.wait_event(computed[i - 2])  # buffer set k is free again
                    for n, t in pool_host[i % 2].items():
                        dev_bufs[k][n].copy_(t, non_blocking=True)
                    copied[i].record(up)
                stream.wait_event(copied[i])
                chunk_step(dev_bufs[k])
                if i >= 2:
                    stream.wait_event(fetched[i - 2])  # staging buffer k was read
                out_dev[k].copy_(res[0], non_blocking=True)
                computed[i].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(computed[i])
                    out_hosts[k].copy_(out_dev[k], non_blocking=True)
                    fetched[i].record(down)
            stream.wait_event(fetched[n_steps - 1])

        with torch.cuda.stream(stream):
            e2e_run(2)
        stream.synchronize()
        barrier()
        e0, e1 = mk(), mk()
        e0.record(stream)
        e2e_run(e2e_steps, e0)
        e1.record(stream)
        stream.synchronize()
        e2e_ms_local = e0.elapsed_time(e1)
        barrier()

    ms_max = max_over_ranks(ms_local)
    e2e_ms_max = max_over_ranks(e2e_ms_local)
    # Ulysses splits one layer's attention over the ranks (strong scaling): each
    # rank does 1/world of it; replicas each do a whole one (weak scaling).
    flops_rank = flops / world if args.ulysses else flops
    value = whole_job_tflops(flops_rank * attends_per_chunk * args.steps, ms_max, world)
    e2e_value = whole_job_tflops(flops_rank * attends_per_chunk * e2e_steps, e2e_ms_max, world)

    gaps = None
    if args.launch_gaps > 0 and world == 1:
        def run_steps(n):
            with torch.cuda.stream(stream):
                for i in range(n):
                    chunk_step(pool[i % 2])
        gaps = launch_gap_trace(run_steps, args.launch_gaps)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args)

    ranks.close()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    attend_avg = statistics.fmean(attend_ms)
    achieved = flops_rank / (attend_avg * 1e-3) / 1e12
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    # The burst peak is cuBLAS timed alone; the sustained one a seconds-long loop
    # under the power cap. A timed region shorter than that compares with burst.
    region_s = ms_max * 1e-3
    long_region = region_s >= SUSTAINED_REGION_S
    peak = sustained if long_region else burst
    peak_kind = (f"bf16 {'sustained' if long_region else 'burst'} ({peak_src}); timed region "
                 f"{region_s:.3f} s")
    per_clock = None
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    if kernel_clock is not None or (clock_info and clock_info.get("sm_mhz")):
        per_clock = {"sms": sms, "dense_mma_flop_per_sm_clock": 8192}
        if kernel_clock is not None:
            # The last timed attention launch by its own per-CTA stamps: the SM
            # clock it ran at (cycle counter / global timer) and first start to
            # last end. NVML can read the maximum clock while the SMs run slower.
            mhz, span_us = kernel_clock
            per_clock["kernel_last_launch"] = {
                "sm_mhz": mhz, "span_ms": span_us * 1e-3,
                "flop_per_sm_clock": flops_rank / (span_us * 1e-6 * mhz * 1e6 * sms)}
        if clock_info and clock_info.get("sm_mhz"):
            nv = clock_info["sm_mhz"]
            per_clock["nvml_sm_mhz_median"] = nv
            per_clock["ms_x_nvml_mhz"] = attend_avg * nv
            per_clock["flop_per_sm_clock_at_nvml_mhz"] = flops_rank / (attend_avg * 1e-3 * nv * 1e6
                                                                       * sms)
    append_bytes = appends_per_chunk * 2 * 2 * (w.batch * w.chunk_len * w.heads * w.head_dim * 2)
    # (per append of one tier: K and V, each read once and written once)
    append_gbs = append_bytes / (statistics.fmean(append_ms) * 1e-3) / 1e9
    launch_bytes = 2 * 2 * (w.batch * w.chunk_len * w.heads * w.head_dim * 2)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "strong" if args.ulysses else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(w, args, world),
        "roofline": {
            "bound": "tensor",
            "kernel": "attend_tc_kernel<128>" + (
                " (Ulysses layer call: fp8 pack, all-to-all, staging, attention, unpack)"
                if args.ulysses else
                " (sparse, timed with its staging kernel)" if block_mask is not None else
                " (frame-aligned, timed with its staging kernel)" if args.editing else ""),
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_kind": peak_kind, "frac_of_burst_peak": achieved / burst,
            "frac_of_sustained_peak": achieved / sustained,
            "per_clock": per_clock,
            "traffic": kernel_traffic("attend_tc.cuh", w.name),
            "flops_per_launch": flops, "avg_launch_ms": attend_avg,
        },
        "append": append_line(append_ms, append_gbs, launch_ms, launch_bytes, hbm),
        "ms_per_attention": attend_avg,
        "attention_tflops_kernel": achieved,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms_max / e2e_steps,
                "pipelining": "inputs of step i+1 up and output of step i down on two copy "
                              "streams while step i computes"},
        # per attention: stage + attend (+ the mask packing when block-sparse; + 4
        # pack/unpack pairs with Ulysses); per append: one kernel (+ 2 pack/unpack
        # pairs with Ulysses)
        "gpu_launches": args.steps * ((10 if args.ulysses else 3 if args.sparsity > 0 else 2)
                                      * attends_per_chunk
                                      + (5 if args.ulysses else 1) * appends_per_chunk),
        "clocks": clock_info,
        "cpu_baseline": cpu,
    }
    if gaps is not None:
        line["launch_gaps"] = gaps
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    from sa_inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
