"""Benchmark of the PLE n-gram embedding layer on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ple|reference]

Default workload: full-scale prefill, a packed batch of 16,384 tokens
(sequences of 1,000 / 3,384 / 4,000 / 8,000 tokens, Zipf(1.1) tokens over a
248,320 vocabulary), hidden size 2560, a 51,200,245,760-byte FP8 table resident
in HBM. A step is one ple_forward call: n-gram IDs, gate, row gather and
dequantisation, projection, conv and residual for the whole batch. Inputs
rotate over several sets whose combined size is well above the 126 MB L2, so
each step starts with its own inputs out of L2.

Prints one JSON line (rank 0). With torchrun, every rank runs an independent
replica (the layer shards by batch with no exchange), time is the max over ranks
and the value sums all ranks' tokens.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "PLE layer tokens/s (prefill & decode) and gathered-row HBM GB/s vs peak, 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_SOURCES = ["gram_embedding_lookup_b200/csrc/ple_gemm.cu", "gram_embedding_lookup_b200/csrc/ple_device.cuh"]
GATHER_SOURCES = ["gram_embedding_lookup_b200/csrc/ple_kernels.cu", "gram_embedding_lookup_b200/csrc/ple_device.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ple", "reference"], default="ple")
    ap.add_argument("--table-rows", type=int, default=0,
                    help="rows per sub-table (default: the full 10,000,048); smaller only for profiling captures")
    ap.add_argument("--sets", type=int, default=3, help="rotating input sets")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the e2e, decode and clocks measurements")
    ap.add_argument("--extras", default="e2e,decode,mtp,long,nvfp4,heads,prepared,pipelined,gather_fused",
                    help="comma-separated extra lines to measure (for profiling one of them alone)")
    ap.add_argument("--ref-tokens", type=int, default=512, help="tokens per reference-arm step")
    ap.add_argument("--path", type=int, default=0,
                    help="forward path of the timed prefill steps (ple_set_forward_path; 0 = automatic, "
                         "4 = gather fused into the projection)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel: str, workload: str, src_hash: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload:
                return float(parts[3]) if parts[2] == src_hash else None
    return None


_SAMPLER = r"""
import sys, time
try:
    import pynvml
    pynvml.nvmlInit()
    bus, idx, period = sys.argv[1], int(sys.argv[2]), float(sys.argv[3])
    dev = None
    if bus != "-":
        try:
            dev = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            dev = None
    if dev is None:
        dev = pynvml.nvmlDeviceGetHandleByIndex(idx)
    print("max", pynvml.nvmlDeviceGetMaxClockInfo(dev, pynvml.NVML_CLOCK_SM), flush=True)
except Exception as exc:
    print("error", type(exc).__name__, str(exc).replace(chr(10), " ")[:200], flush=True)
    sys.exit(0)
while True:
    try:
        print(pynvml.nvmlDeviceGetClockInfo(dev, pynvml.NVML_CLOCK_SM),
              pynvml.nvmlDeviceGetCurrentClocksEventReasons(dev), flush=True)
    except Exception as exc:
        print("error", type(exc).__name__, str(exc).replace(chr(10), " ")[:200], flush=True)
    time.sleep(period)
"""

_SMI_QUERY = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """SM clock and throttle reasons, sampled while running by a separate process that
    only reads: NVML every few milliseconds, or, if NVML cannot be used there,
    `nvidia-smi --query-gpu ... -lms 200`. When neither produces a sample, stop() says
    why instead of returning nothing."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}
    SMI_REASONS = ("hw_slowdown", "sw_thermal_slowdown", "hw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index: int, period_s: float = 0.005, pci_bus_id: str | None = None):
        self.index = index
        self.period = period_s
        self.pci_bus_id = pci_bus_id
        self.proc = None
        self.kind = None
        self.errors = []
        self.max_mhz = float("nan")

    def start(self):
        """Starts the sampler and returns once it is producing samples (or has failed)."""
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER, self.pci_bus_id or "-", str(self.index),
                                          str(self.period)], stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                         text=True)
            first = self.proc.stdout.readline().split()
            if len(first) == 2 and first[0] == "max":
                self.max_mhz = float(first[1])
                self.kind = "nvml"
                self.proc.stdout.readline()         # one sample taken: the sampler is live
                return
            self.errors.append("NVML sampler: " + (" ".join(first) or f"exited with {self.proc.wait()}"))
            self.proc.wait()
        except Exception as exc:  # pragma: no cover - no NVML on this host
            self.errors.append(f"NVML sampler: {type(exc).__name__}: {exc}")
        self.proc = None
        target = self.pci_bus_id or str(self.index)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", target, f"--query-gpu={_SMI_QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
            self.kind = "nvidia-smi"
            time.sleep(0.3)
        except Exception as exc:
            self.errors.append(f"nvidia-smi: {type(exc).__name__}: {exc}")
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"unavailable": "; ".join(self.errors) or "no sampler started"}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        mhz, reasons, other = [], set(), []
        for line in out.splitlines():
            if self.kind == "nvml":
                parts = line.split()
                try:
                    m, r = float(parts[0]), int(parts[1])
                except (ValueError, IndexError):
                    other.append(line.strip())
                    continue
                mhz.append(m)
                reasons |= {n for n, bit in self.REASONS.items() if r & bit}
            else:
                parts = [p.strip() for p in line.split(",")]
                try:
                    m, mx = float(parts[0]), float(parts[1])
                except (ValueError, IndexError):
                    other.append(line.strip())
                    continue
                mhz.append(m)
                self.max_mhz = mx
                reasons |= {n for n, v in zip(self.SMI_REASONS, parts[2:]) if v.lower() == "active"}
        if not mhz:
            why = "; ".join(self.errors + [f"{self.kind}: " + (" | ".join(o for o in other if o)[:300]
                                                                or "no output in the timed region")])
            return {"unavailable": why}
        res = {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": self.max_mhz, "sm_min_mhz": float(min(mhz)),
               "reasons": sorted(reasons), "samples": len(mhz),
               "source": f"{self.kind} in a separate process, sampled inside the timed region"}
        if self.errors:
            res["note"] = "; ".join(self.errors)
        return res


def tensor_peak(peaks, region_s: float):
    """The tensor-core peak a kernel is compared with: the burst figure for a timed region
    shorter than a second (the GPU has not yet settled at its power cap), the sustained
    figure for a seconds-long loop. Returns (TFLOP/s, the MEASURED_PEAKS key used)."""
    if region_s >= 1.0 and "bf16_tflops_sustained" in peaks:
        return peaks["bf16_tflops_sustained"], "bf16_tflops_sustained"
    return peaks["bf16_tflops"], "bf16_tflops"


def host_cpu(threads_used: int) -> dict:
    """The host the CPU baseline ran on: its logical core count and CPU model, and how
    the oracle used it (numpy's BLAS threads for the matmuls, one thread elsewhere)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu": model,
            "threads": f"{threads_used} BLAS thread(s) for the projection and gate matmuls; the sequence map, "
                       f"hash, row gather and conv run as Python loops on one thread"}


# ----------------------------------------------------------------------------- CPU oracle legs
def oracle_prefill_sample(w, tokens, offsets, hidden, n_tok):
    """The first n_tok tokens of the batch as a packed batch of its own."""
    offs = [int(o) for o in offsets if o < n_tok] + [n_tok]
    return tokens[:n_tok], np.array(offs, dtype=np.int64), hidden[:n_tok]


def time_oracle(w, tokens, offsets, hidden, weights):
    """Runs the CPU oracle once on the given (small) batch; returns (seconds, threads)."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        threads = 1
    # the synthetic rows are input generation: materialise them before the clock starts
    ids = O.ngram_ids(tokens, offsets, w.rows_per_order)
    table = w.table()
    cache = {n: dict(zip(ids[:, n].tolist(), zip(table.codes(n, ids[:, n]), table.scales(n, ids[:, n]))))
             for n in range(2)}

    class Cached:
        def codes(self, n, rows):
            return np.stack([cache[n][int(r)][0] for r in rows])

        def scales(self, n, rows):
            return np.array([cache[n][int(r)][1] for r in rows], dtype=np.float32)

    t0 = time.perf_counter()
    O.ple_forward(tokens, offsets, hidden, weights.w_proj, weights.w_gate, weights.conv_w, Cached(),
                  w.rows_per_order)
    return time.perf_counter() - t0, threads


def run_reference(args, rank):
    """The reference arm: the CPU oracle as it stands, on bounded samples of the workload."""
    import ple_inputs as pi
    if rank != 0:
        return
    w = pi.workload("prefill")
    weights = w.weights()
    tokens, offsets, hidden = pi.prefill_batch(w)
    tk, of, hd = oracle_prefill_sample(w, tokens, offsets, hidden, args.ref_tokens)
    for _ in range(args.warmup):
        time_oracle(w, tk, of, hd, weights)
    total, threads = 0.0, 1
    for _ in range(args.steps):
        s, threads = time_oracle(w, tk, of, hd, weights)
        total += s
    value = args.ref_tokens * args.steps / total
    sample = f"first {args.ref_tokens} tokens of the prefill batch per step, offsets {of.tolist()}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": prefill_config(args, w, 1),
        "timed_tokens_per_step": args.ref_tokens,
        "timed_sample": f"each step times the first {args.ref_tokens} of the config's {16384} tokens, as a packed "
                        f"batch of their own; value is those tokens per second",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample,
                         **host_cpu(threads)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def prefill_config(args, w, world):
    return {"workload": "full-scale prefill: 16,384 packed tokens (sequences 1000/3384/4000/8000), "
                        "Zipf(1.1) tokens over 248,320, hidden 2560, 2 x 10,000,048 x 2560 FP8 table in HBM",
            "model": "PLE n-gram embedding layer", "global_batch": 16384 * world, "seq_len": 16384,
            "table_rows_per_order": w.rows_per_order, "parallelism": f"replicas x{world}",
            "l2": f"{args.sets} rotating input sets (>2x L2 per step)", "out_dtype": "bf16",
            "forward_path": args.path}


# ----------------------------------------------------------------------------- ranks
class Comm:
    """Coordination of the replicas (one process per GPU, no data-path collective):
    a barrier around the timed region and the maximum of a time over the ranks.
    NCCL on the GPUs; the CPU tests run the same code over gloo."""

    def __init__(self, world: int, dist=None, device: str = "cuda"):
        self.world = world
        self.dist = dist
        self.device = device

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max(self, x: float) -> float:
        if self.world == 1:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())


def replica_value(tokens_per_step: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processes tokens_per_step per step (weak
    scaling); the time is the slowest rank's."""
    return tokens_per_step * world * steps / (ms_max / 1e3)


def replica_variant(v: int, rank: int) -> int:
    """Input-set index of rank ``rank``: each replica draws its own batches."""
    return v + 100 * rank


# ----------------------------------------------------------------------------- GPU arm
def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist
    import gram_embedding_lookup_b200 as ple
    import ple_inputs as pi
    from ple_inputs.device import DeviceLayer, bf16_tensor

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))

    comm = Comm(world, dist, "cuda")
    barrier, max_over_ranks = comm.barrier, comm.max

    ctx = dict(torch=torch, ple=ple, pi=pi, bf16_tensor=bf16_tensor, barrier=barrier,
               max_over_ranks=max_over_ranks, world=world, args=args)
    stream = torch.cuda.current_stream()
    w0 = pi.workload("prefill")
    w = w0 if args.table_rows <= 0 else pi.Workload("prefill", w0.vocab, args.table_rows, w0.row_dim, w0.hidden,
                                                      w0.table_seed, w0.seed, w0.extra)
    layer = DeviceLayer(w, max_tokens=16384, max_seqs=64, prepare_slots=2)
    h = layer.handle
    H, D = w.hidden, w.row_dim

    sets = []
    for v in range(args.sets):
        tokens, offsets, hidden = pi.prefill_batch(w, variant=replica_variant(v, rank))
        sets.append(dict(tokens=torch.from_numpy(tokens).cuda(), offsets=torch.from_numpy(offsets).cuda(),
                         hidden=bf16_tensor(hidden), out=torch.empty(len(tokens), H, dtype=torch.bfloat16,
                                                                      device="cuda"),
                         T=len(tokens), S=len(offsets) - 1, host=(tokens, offsets, hidden)))

    def step(i):
        s = sets[i % len(sets)]
        ple.ple_forward(h, s["tokens"], s["T"], s["offsets"], s["S"], s["hidden"], s["out"], ple.PLE_OUT_BF16,
                        None, stream)

    ple.ple_set_forward_path(h, args.path)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if ple.ple_get_error(h) != 0:
        raise SystemExit("device status error during warm-up")

    # ------------------------------------------------------------------ timed region
    # The workload alone: library stage events between the two kernels of a step
    # would keep the projection from starting before the embed kernel ends
    # (programmatic dependent launch), so they are recorded in a second pass.
    props = torch.cuda.get_device_properties(local)
    bus = None
    if hasattr(props, "pci_bus_id"):
        bus = f"{getattr(props, 'pci_domain_id', 0):08x}:{props.pci_bus_id:02x}:{getattr(props, 'pci_device_id', 0):02x}.0"
    clocks = ClockSampler(local, pci_bus_id=bus)
    clocks.start()
    launches0 = ple.ple_launch_count(h)
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()     # stops at the end of the timed region (it started just before it)
    barrier()
    launches = ple.ple_launch_count(h) - launches0
    # per-kernel durations: the same steps again, with the library's stage events
    prof_steps = min(args.steps, 300)
    ple.ple_set_profiling(h, True)
    ple.ple_get_stage_times(h)
    for i in range(prof_steps):
        step(i)
    torch.cuda.synchronize()
    stage = ple.ple_get_stage_times(h)
    ple.ple_set_profiling(h, False)
    ple.ple_set_forward_path(h, 0)
    status = ple.ple_get_error(h)
    ms = max_over_ranks(ev0.elapsed_time(ev1))
    T = sets[0]["T"]
    ms_per_step = ms / args.steps
    value = replica_value(T, world, args.steps, ms)

    peaks, peak_kind = load_peaks()
    gemm_ms, gemm_n = stage["gemm"]
    gemm_s = gemm_ms / 1e3 / max(gemm_n, 1)
    flops = 2.0 * D * H * T
    achieved_tf = flops / gemm_s / 1e12
    peak_tf, peak_name = tensor_peak(peaks, ms / 1e3)
    roofline = {"kernel": "gemm_kernel (tcgen05 projection + fused gate/conv/residual)", "bound": "tensor",
                "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved_tf / peak_tf,
                "peak_source": f"{peak_kind} {peak_name}: the timed region lasted {ms / 1e3:.3f} s "
                               f"({'under' if peak_name == 'bf16_tflops' else 'over'} 1 s); fp16 nominal ratio 1.0",
                "frac_of_burst_peak": achieved_tf / peaks["bf16_tflops"],
                "frac_of_sustained_peak": achieved_tf / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                "traffic": load_traffic("gemm", "prefill", source_hash(GEMM_SOURCES)),
                "algorithmic_flops_per_launch": flops, "launch_ms": gemm_s * 1e3}
    roofline["library_same_shape"] = library_gemm_same_shape(torch, T, D, H)
    e_ms, e_n = stage["prepare"]
    e_s = e_ms / 1e3 / max(e_n, 1)
    if args.path == 4:      # the first kernel computes only IDs and gate: h and tokens in; ids, meta out
        embed_bytes, embed_name = T * (2 * H + 8 + 16 + 4), "embed_kernel without rows (ids + gate)"
    else:                   # h, rows, scales in; e, ids, meta out; tokens
        embed_bytes, embed_name = T * (2 * H + 2 * D + 8 + 2 * D + 8 + 16 + 4), (
            "ids_meta_kernel + embed_bulk_kernel (row IDs; bulk-copied rows dequantised; gate)")
    embed = {"kernel": embed_name, "bound": "hbm",
             "achieved": embed_bytes / e_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": embed_bytes / e_s / 1e9 / peaks["hbm_gbs"], "launch_ms": e_s * 1e3,
             "algorithmic_bytes_per_launch": embed_bytes,
             "gathered_row_gbs": (0 if args.path == 4 else T * 2 * D) / e_s / 1e9,
             "traffic": load_traffic("embed", "prefill", source_hash(GATHER_SOURCES))}
    if args.path != 4:
        embed["library_same_bytes"] = library_stream_same_bytes(torch, T, D, peaks["hbm_gbs"])

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic", "config": prefill_config(args, w, world),
        "roofline": roofline, "embed_roofline": embed,
        "stage_ms_per_launch": {k: (v[0] / max(v[1], 1)) for k, v in stage.items() if v[1]},
        "gpu_launches": int(launches) * world, "device_status": int(status),
        "gathered_row_gbs_end_to_end": T * 2 * D * args.steps / (ms / 1e3) / 1e9,
        "timing_note": "device time of the K-step loop (CUDA events on the launching stream, no events in "
                       "between); per-kernel durations from a following pass of min(K, 300) steps with the "
                       "library's stage events",
    }
    line["clocks"] = clk
    line["gather_roofline"] = gather_bench(ctx, layer, sets, stream, peaks)
    # the HBM-bound stages beside the projection, in the line's top-level roofline
    for key, src in (("embed", embed), ("gather", line["gather_roofline"])):
        roofline[key] = {k: src[k] for k in ("kernel", "bound", "achieved", "peak", "unit", "frac",
                                             "gathered_row_gbs", "launch_ms", "algorithmic_bytes_per_launch",
                                             "traffic") if k in src}
        roofline[key]["gathered_row_frac"] = src["gathered_row_gbs"] / peaks["hbm_gbs"]

    if not args.no_extras:
        want = set(args.extras.split(","))
        if "e2e" in want:
            line["e2e"] = e2e_prefill(args, ple, h, sets, stream, world, max_over_ranks, barrier)
        if "decode" in want:
            line["decode"] = decode_bench(ctx, layer, stream)
        if "mtp" in want:
            line["mtp"] = mtp_bench(ctx, layer, stream)
        if "long" in want:
            line["long_context"] = long_bench(ctx, layer, stream)
        if "nvfp4" in want:
            # the two layouts of the same NVFP4 contents, the array layout first
            arrays = nvfp4_bench(ctx, w, sets, stream, peaks, ple.PLE_TABLE_NVFP4)
            line["nvfp4"] = nvfp4_bench(ctx, w, sets, stream, peaks, ple.PLE_TABLE_NVFP4_ROWS)
            line["nvfp4"]["arrays_layout"] = arrays
        if "heads" in want:
            line["heads"] = heads_bench(ctx, sets, stream, peaks, args.table_rows)
        if "prepared" in want:
            line["prepared"] = prepared_bench(ctx, layer, sets, stream)
        if "pipelined" in want:
            line["pipelined"] = pipelined_bench(ctx, layer, sets, stream)
        if "gather_fused" in want:
            line["gather_fused"] = gather_fused_bench(ctx, layer, sets, stream, peaks)

    if rank == 0 and not args.no_cpu_baseline and world == 1:
        tokens, offsets, hidden = sets[0]["host"]
        n_tok = 256
        tk, of, hd = oracle_prefill_sample(w, tokens, offsets, hidden, n_tok)
        secs, threads = time_oracle(w, tk, of, hd, w.weights())
        reps = max(1, int(10.0 / max(secs, 1e-3)))
        total = secs
        for _ in range(min(reps, 20) - 1):
            s2, threads = time_oracle(w, tk, of, hd, w.weights())
            total += s2
        n_runs = min(reps, 20)
        line["cpu_baseline"] = {"value": n_tok * n_runs / total, "unit": "tokens/s", "cores": threads,
                                "kind": "oracle", **host_cpu(threads),
                                "sample": f"first {n_tok} tokens of the prefill batch, {n_runs} run(s), "
                                          f"rows materialised before timing"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    layer.close()
    if world > 1:
        dist.destroy_process_group()


def library_gemm_same_shape(torch, T, D, H, n=300):
    """Context for the projection's roofline: cuBLAS (torch.matmul) on a plain fp16
    GEMM of the same shape, [T x D] @ [D x H] with fp32 accumulation, timed back
    to back like the layer's loop. The library kernel has no gate, conv or
    residual epilogue; it is a measurement beside the layer, not part of it."""
    prev = torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    try:
        a = torch.randn(T, D, device="cuda").to(torch.float16)
        b = torch.randn(D, H, device="cuda").to(torch.float16)
        c = torch.empty(T, H, device="cuda", dtype=torch.float16)
        for _ in range(10):
            torch.matmul(a, b, out=c)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            torch.matmul(a, b, out=c)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / n
    finally:
        torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = prev
    return {"kernel": "cuBLAS fp16 GEMM via torch.matmul (no epilogue)", "ms": ms,
            "tflops": 2.0 * T * D * H / (ms / 1e3) / 1e12, "launches": n}


def library_stream_same_bytes(torch, T, D, peak_gbs, n=300, sets=4):
    """Context for the embed kernel's roofline: a plain elementwise torch.add of
    two fp16 [T x D] tensors into a third moves the embed launch's main bytes in
    the same mix (2 x T*D*2 read, T*D*2 written) with no gather, hash or gate.
    It runs back to back over `sets` distinct buffer triples (more than L2
    holds), like the layer's loop; a launch this short does not reach the
    seconds-long copy rate that the peak was measured with."""
    bufs = [[torch.empty(T, D, device="cuda", dtype=torch.float16) for _ in range(3)] for _ in range(sets)]
    for b in bufs:
        for x in b:
            x.fill_(1.0)
    for i in range(10):
        a, b, c = bufs[i % sets]
        torch.add(a, b, out=c)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        a, b, c = bufs[i % sets]
        torch.add(a, b, out=c)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    nbytes = 3 * T * D * 2
    gbs = nbytes / (ms / 1e3) / 1e9
    del bufs
    torch.cuda.empty_cache()
    return {"kernel": "torch.add, fp16 [T x D] + [T x D] -> [T x D] (same read/write mix, no gather)", "ms": ms,
            "bytes": nbytes, "gbs": gbs, "frac_of_peak": gbs / peak_gbs, "launches": n}


def timed(ctx, stream, fn, n):
    """Device time (ms) of n calls of fn on `stream`, max over ranks."""
    torch = ctx["torch"]
    ctx["barrier"]()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ctx["barrier"]()
    return ctx["max_over_ranks"](e0.elapsed_time(e1))


def gather_bench(ctx, layer, sets, stream, peaks):
    """The gather stage alone (ple_gather_rows) over the prefill batches' row IDs:
    algorithmic bytes per launch = T x (2 rows x D codes + 2 scales + 2 ids + D fp16 written)."""
    torch, ple = ctx["torch"], ctx["ple"]
    h = layer.handle
    D = layer.w.row_dim
    ids, es = [], []
    for s in sets:
        t = torch.empty(s["T"], 2, dtype=torch.int32, device="cuda")
        ple.ple_ngram_ids(h, s["tokens"], s["T"], s["offsets"], s["S"], None, t, stream)
        ids.append(t)
        es.append(torch.empty(s["T"], D, dtype=torch.float16, device="cuda"))
    T = sets[0]["T"]

    def fn(i):
        k = i % len(sets)
        ple.ple_gather_rows(h, ids[k], T, es[k], stream)

    for i in range(5):
        fn(i)
    n = 200
    ms = timed(ctx, stream, fn, n)
    per = ms / 1e3 / n
    nbytes = T * (2 * D + 8 + 8 + 2 * D)
    return {"kernel": "gather_kernel (ple_gather_rows, standalone)", "bound": "hbm",
            "achieved": nbytes / per / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": nbytes / per / 1e9 / peaks["hbm_gbs"], "gathered_row_gbs": T * 2 * D / per / 1e9,
            "launch_ms": per * 1e3, "launches": n, "algorithmic_bytes_per_launch": nbytes,
            "traffic": load_traffic("gather", "prefill", source_hash(GATHER_SOURCES))}


def e2e_prefill(args, ple, h, sets, stream, world, max_over_ranks, barrier):
    """Same metric through the C ABI with host buffers: every step's inputs go up from
    pinned host memory and its output comes back down, all inside the timed region.

    As a serving loop would run it, the copies overlap the layer. Step i+1's inputs
    go up on one copy stream and step i-1's output comes down on another while step i
    runs on the compute stream. The input sets form a ring of device buffers, and
    events order each buffer's upload, layer call and download. The same steps run
    in series on one stream are reported beside it."""
    import torch
    hosts = []
    for s in sets:
        tokens, offsets, hidden = s["host"]
        hosts.append(dict(tokens=torch.from_numpy(tokens).pin_memory(), offsets=torch.from_numpy(offsets).pin_memory(),
                          hidden=torch.from_numpy(hidden.view(np.int16)).view(torch.bfloat16).pin_memory(),
                          out=torch.empty_like(s["out"], device="cpu").pin_memory()))
    nb = len(sets)
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    up_done = [torch.cuda.Event() for _ in range(nb)]
    comp_done = [torch.cuda.Event() for _ in range(nb)]
    down_done = [torch.cuda.Event() for _ in range(nb)]

    def step_overlapped(i):
        b = i % nb
        s, hs = sets[b], hosts[b]
        s_up.wait_event(comp_done[b])           # the layer is done with this buffer's inputs
        with torch.cuda.stream(s_up):
            s["tokens"].copy_(hs["tokens"], non_blocking=True)
            s["offsets"].copy_(hs["offsets"], non_blocking=True)
            s["hidden"].copy_(hs["hidden"], non_blocking=True)
        up_done[b].record(s_up)
        stream.wait_event(up_done[b])
        stream.wait_event(down_done[b])         # this buffer's previous output is down
        ple.ple_forward(h, s["tokens"], s["T"], s["offsets"], s["S"], s["hidden"], s["out"], ple.PLE_OUT_BF16,
                        None, stream)
        comp_done[b].record(stream)
        s_down.wait_event(comp_done[b])
        with torch.cuda.stream(s_down):
            hs["out"].copy_(s["out"], non_blocking=True)
        down_done[b].record(s_down)

    def step_serial(i):
        s, hs = sets[i % nb], hosts[i % nb]
        s["tokens"].copy_(hs["tokens"], non_blocking=True)
        s["offsets"].copy_(hs["offsets"], non_blocking=True)
        s["hidden"].copy_(hs["hidden"], non_blocking=True)
        ple.ple_forward(h, s["tokens"], s["T"], s["offsets"], s["S"], s["hidden"], s["out"], ple.PLE_OUT_BF16,
                        None, stream)
        hs["out"].copy_(s["out"], non_blocking=True)

    steps = 20

    def timed_steps(step, first, last):
        for i in range(max(args.warmup, 3)):
            step(i)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(first)
        for i in range(steps):
            step(i)
        last.wait_stream(stream)
        e1.record(last)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1))

    ms = timed_steps(step_overlapped, s_up, s_down)
    ms_serial = timed_steps(step_serial, stream, stream)
    s0 = sets[0]
    h2d = s0["tokens"].numel() * 4 + s0["offsets"].numel() * 4 + s0["hidden"].numel() * 2
    d2h = s0["out"].numel() * 2
    return {"value": s0["T"] * world * steps / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps, "ms_per_step": ms / steps,
            "copies": "overlapped with the layer (copy streams, ring of 3 buffer sets)",
            "serial": {"value": s0["T"] * world * steps / (ms_serial / 1e3), "ms_per_step": ms_serial / steps}}


def gather_fused_bench(ctx, layer, sets, stream, peaks, steps=300):
    """Forward path 4 on the headline batches: the rows are gathered and
    dequantised inside the projection kernel (the fp16 rows never reach HBM),
    after a kernel that computes only the row IDs and the gate. Step time with
    no events in between, then per-kernel times from a pass with stage events."""
    torch, ple = ctx["torch"], ctx["ple"]
    h = layer.handle
    D, H = layer.w.row_dim, layer.w.hidden

    def step(i):
        s = sets[i % len(sets)]
        ple.ple_forward(h, s["tokens"], s["T"], s["offsets"], s["S"], s["hidden"], s["out"], ple.PLE_OUT_BF16,
                        None, stream)

    ple.ple_set_forward_path(h, 4)
    try:
        for i in range(5):
            step(i)
        ms = timed(ctx, stream, step, steps) / steps
        ple.ple_set_profiling(h, True)
        ple.ple_get_stage_times(h)
        for i in range(min(steps, 100)):
            step(i)
        torch.cuda.synchronize()
        st = ple.ple_get_stage_times(h)
        ple.ple_set_profiling(h, False)
    finally:
        ple.ple_set_forward_path(h, 0)
    status = ple.ple_get_error(h)
    T = sets[0]["T"]
    gemm_ms = st["gemm"][0] / max(st["gemm"][1], 1)
    tf = 2.0 * D * H * T / (gemm_ms / 1e3) / 1e12
    peak, peak_name = tensor_peak(peaks, ms * steps / 1e3)
    return {"workload": "full-scale prefill batches, forward path 4 (gather fused into the projection)",
            "value": T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "stage_ms_per_launch": {k: v[0] / max(v[1], 1) for k, v in st.items() if v[1]},
            "gemm_tflops": tf, "gemm_frac_of_peak": tf / peak, "peak": peak_name, "device_status": int(status)}


def prepared_bench(ctx, layer, sets, stream, steps=200):
    """The layer split in two (ple_prepare, ple_forward_prepared) on the headline
    batches: the time of each call, and of ple_forward, with CUDA events on the
    launching stream. ple_prepare depends only on the tokens, so a model can issue
    it while earlier layers run; ple_forward_prepared is what is left once the
    hidden states exist."""
    torch, ple = ctx["torch"], ctx["ple"]
    h = layer.handle

    def prep(i):
        s = sets[i % len(sets)]
        ple.ple_prepare(h, s["tokens"], s["T"], s["offsets"], s["S"], None, stream)

    def rest(i):
        s = sets[i % len(sets)]
        ple.ple_forward_prepared(h, s["hidden"], s["out"], ple.PLE_OUT_BF16, None, stream)

    def whole(i):
        s = sets[i % len(sets)]
        ple.ple_forward(h, s["tokens"], s["T"], s["offsets"], s["S"], s["hidden"], s["out"], ple.PLE_OUT_BF16,
                        None, stream)

    for i in range(5):
        prep(i)
        rest(i)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        ev[i][0].record(stream)
        prep(i)
        ev[i][1].record(stream)
        rest(i)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    t_prep = sum(a.elapsed_time(b) for a, b, _ in ev) / steps
    t_rest = sum(b.elapsed_time(c) for _, b, c in ev) / steps
    t_whole = timed(ctx, stream, whole, steps) / steps
    status = ple.ple_get_error(h)
    return {"workload": "full-scale prefill batches, the layer in two calls",
            "prepare_ms": t_prep, "forward_prepared_ms": t_rest, "forward_ms": t_whole,
            "after_hidden_ready_ms_saved": t_whole - t_rest, "device_status": int(status),
            "note": "ple_prepare needs only the tokens; ple_forward_prepared (gate, projection, conv, residual) "
                    "is the part that waits for the hidden states"}


def pipelined_bench(ctx, layer, sets, stream, steps=300):
    """The headline batches as a stream with two in flight (ple_prepare_slot /
    ple_forward_prepared_slot): batch i + 1's IDs and rows are prepared into the
    other slot on a side stream while batch i's gate, projection and epilogue run
    on the main stream. Each batch is fresh sequences, so a prepare waits only
    for its slot to be free. Device time from the main stream's events around the
    whole stream of batches, max over ranks."""
    torch, ple = ctx["torch"], ctx["ple"]
    h = layer.handle
    side = torch.cuda.Stream()

    def run(n):
        prepared = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event() for _ in range(n)]
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        side.wait_event(start)
        for i in range(n):
            s = sets[i % len(sets)]
            slot = i % 2
            if i >= 2:
                side.wait_event(done[i - 2])
            ple.ple_prepare_slot(h, slot, s["tokens"], s["T"], s["offsets"], s["S"], None, side)
            prepared[i].record(side)
            stream.wait_event(prepared[i])
            ple.ple_forward_prepared_slot(h, slot, s["hidden"], s["out"], ple.PLE_OUT_BF16, None, stream)
            done[i].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    run(6)
    ctx["barrier"]()
    ms = ctx["max_over_ranks"](run(steps))
    ctx["barrier"]()
    status = ple.ple_get_error(h)
    T = sets[0]["T"]
    world = ctx["world"]
    return {"workload": "full-scale prefill batches, two in flight (prepare of the next batch on a side stream)",
            "value": T * world * steps / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms / steps,
            "device_status": int(status)}


def heads_bench(ctx, sets, stream, peaks, table_rows=0, steps=300):
    """The multi-head row layout (PLE_TABLE_E4M3_HEADS: 16 lookups of 160-byte rows
    per token, 16 sub-tables of 20,000,096 rows, the same 51.2 GB): the headline
    prefill batches and the 8 x 1 decode workload (a split-K step on this layout).
    With table_rows > 0 (--table-rows) each head sub-table has 2 * table_rows rows,
    the same bytes as a two-order table of table_rows rows per order."""
    torch, ple, pi = ctx["torch"], ctx["ple"], ctx["pi"]
    from ple_inputs.device import DeviceLayer
    w = pi.workload("heads_full")
    if table_rows > 0:
        w = pi.Workload(w.name, w.vocab, 2 * table_rows, w.row_dim, w.hidden, w.table_seed, w.seed, w.extra)
    R, D, H = w.rows_per_order, w.row_dim, w.hidden
    need = R * D + 16 * R * 4
    free, _ = torch.cuda.mem_get_info()
    if free < need + (4 << 30):
        return {"skipped": f"needs {need / 1e9:.1f} GB free for the multi-head table, {free / 1e9:.1f} GB free"}
    layer = DeviceLayer(w, max_tokens=16384, max_seqs=64, table_format=ple.PLE_TABLE_E4M3_HEADS)
    h = layer.handle
    tokens, hidden, hist, conv = pi.decode_batch(pi.workload("decode"))
    B, q = tokens.shape
    tk = torch.from_numpy(tokens).cuda()
    hd = ctx["bf16_tensor"](hidden)
    hs = torch.from_numpy(hist.astype(np.int32)).cuda()
    cs = torch.from_numpy(conv).cuda()
    out = torch.empty(B * q, H, dtype=torch.bfloat16, device="cuda")

    def dstep(i):
        ple.ple_decode_step(h, tk, B, q, hd, out, ple.PLE_OUT_BF16, hs, cs, None, stream)

    for i in range(5):
        dstep(i)
    n_dec = 500
    d_ms = timed(ctx, stream, dstep, n_dec)

    def step(i):
        s = sets[i % len(sets)]
        ple.ple_forward(h, s["tokens"], s["T"], s["offsets"], s["S"], s["hidden"], s["out"], ple.PLE_OUT_BF16,
                        None, stream)

    for i in range(5):
        step(i)
    # each measurement starts from an idle GPU, as the headline's steps do: a
    # second's pause lets the clock come back from the power cap that the
    # previous lines' steps drove it into
    idle_pause(ctx)
    ms = timed(ctx, stream, step, steps)            # no events between the kernels
    idle_pause(ctx)
    ple.ple_set_profiling(h, True)                  # then per-kernel durations
    ple.ple_get_stage_times(h)
    for i in range(min(steps, 100)):
        step(i)
    torch.cuda.synchronize()
    stage = ple.ple_get_stage_times(h)
    ple.ple_set_profiling(h, False)
    T = sets[0]["T"]
    e_ms, e_n = stage["prepare"]
    e_s = e_ms / 1e3 / max(e_n, 1)
    row_bytes = D + 16 * 4                        # 16 rows of D / 16 codes and their scales
    embed_bytes = T * (2 * H + row_bytes + 2 * D + 16 * 4 + 16 + 4)   # h, rows in; e, ids, meta out; tokens
    g_ms, g_n = stage["gemm"]
    status = ple.ple_get_error(h)
    layer.close()
    del layer                                       # the table back to the device for the next line
    torch.cuda.empty_cache()
    world = ctx["world"]
    return {"workload": "full-scale prefill (the headline batches) and 8 x 1 decode on the multi-head table "
                        f"(16 x {R:,} rows x 160 codes)",
            "table_bytes": int(need), "value": T * world * steps / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms / steps, "stage_ms_per_launch": {"embed": e_s * 1e3, "gemm": g_ms / max(g_n, 1)},
            "embed_roofline": {"bound": "hbm", "achieved": embed_bytes / e_s / 1e9, "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": embed_bytes / e_s / 1e9 / peaks["hbm_gbs"],
                               "algorithmic_bytes_per_launch": embed_bytes},
            "gathered_row_gbs": T * row_bytes / e_s / 1e9,
            "measured": "value over 300 steps, then stage_ms_per_launch over 100 steps (CUDA events around "
                        "each kernel), each from an idle GPU after a 1 s pause",
            "decode_us_per_step": d_ms / n_dec * 1e3, "device_status": int(status)}


def nvfp4_bench(ctx, w, sets, stream, peaks, fmt, steps=300):
    """The NVFP4 table variant: the same prefill batches and the decode workload on
    a table of packed E2M1 codes with E4M3 block scales per 16 elements (28.8 GB at
    full scale instead of 51.2 GB), in layout `fmt`: PLE_TABLE_NVFP4 (codes and
    block scales in two arrays) or PLE_TABLE_NVFP4_ROWS (each row's block scales
    after its codes)."""
    torch, ple, pi = ctx["torch"], ctx["ple"], ctx["pi"]
    from ple_inputs.device import DeviceLayer
    R, D, H = w.rows_per_order, w.row_dim, w.hidden
    need = 2 * R * (D // 2 + D // 16) + 2 * R * 4
    free, _ = torch.cuda.mem_get_info()
    if free < need + (4 << 30):
        return {"skipped": f"needs {need / 1e9:.1f} GB free for the NVFP4 table, {free / 1e9:.1f} GB free"}
    layer = DeviceLayer(w, max_tokens=16384, max_seqs=64, table_format=fmt)
    h = layer.handle
    rows = fmt == ple.PLE_TABLE_NVFP4_ROWS

    # the decode step first, before the prefill loop heats the GPU into its power cap
    # (the headline decode line also runs on a GPU that has been mostly idle)
    wd = pi.workload("decode")
    tokens, hidden, hist, conv = pi.decode_batch(wd)
    B, q = tokens.shape
    tk = torch.from_numpy(tokens).cuda()
    hd = ctx["bf16_tensor"](hidden)
    hs = torch.from_numpy(hist.astype(np.int32)).cuda()
    cs = torch.from_numpy(conv).cuda()
    out = torch.empty(B * q, H, dtype=torch.bfloat16, device="cuda")

    def dstep(i):
        ple.ple_decode_step(h, tk, B, q, hd, out, ple.PLE_OUT_BF16, hs, cs, None, stream)

    for i in range(5):
        dstep(i)
    n_dec = 500
    d_ms = timed(ctx, stream, dstep, n_dec)

    def step(i):
        s = sets[i % len(sets)]
        ple.ple_forward(h, s["tokens"], s["T"], s["offsets"], s["S"], s["hidden"], s["out"], ple.PLE_OUT_BF16,
                        None, stream)

    for i in range(5):
        step(i)
    # each measurement starts from an idle GPU, as the headline's steps do: a
    # second's pause lets the clock come back from the power cap that the
    # previous lines' steps drove it into
    idle_pause(ctx)
    ms = timed(ctx, stream, step, steps)            # no events between the kernels
    idle_pause(ctx)
    ple.ple_set_profiling(h, True)                  # then per-kernel durations
    ple.ple_get_stage_times(h)
    for i in range(min(steps, 100)):
        step(i)
    torch.cuda.synchronize()
    stage = ple.ple_get_stage_times(h)
    ple.ple_set_profiling(h, False)
    T = sets[0]["T"]
    e_ms, e_n = stage["prepare"]
    e_s = e_ms / 1e3 / max(e_n, 1)
    row_bytes = 2 * (D // 2 + D // 16) + 8                  # both rows' codes and block scales, row scales
    embed_bytes = T * (2 * H + row_bytes + 2 * D + 8 + 16 + 4)
    g_ms, g_n = stage["gemm"]

    status = ple.ple_get_error(h)
    layer.close()
    del layer                                       # the table back to the device for the next line
    torch.cuda.empty_cache()
    world = ctx["world"]
    layout = ("rows: each row's 1,280 code bytes, then its 160 block-scale bytes" if rows
              else "arrays: codes [2][R][1280], block scales [2][R][160]")
    return {"workload": "full-scale prefill (the headline batches) and 8 x 1 decode on the NVFP4 table",
            "layout": layout, "table_bytes": int(need), "value": T * world * steps / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms / steps, "stage_ms_per_launch": {"embed": e_s * 1e3, "gemm": g_ms / max(g_n, 1)},
            "embed_roofline": {"bound": "hbm", "achieved": embed_bytes / e_s / 1e9, "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": embed_bytes / e_s / 1e9 / peaks["hbm_gbs"],
                               "algorithmic_bytes_per_launch": embed_bytes},
            "gathered_row_gbs": T * row_bytes / e_s / 1e9,
            "measured": "value over 300 steps, then stage_ms_per_launch over 100 steps (CUDA events around "
                        "each kernel), each from an idle GPU after a 1 s pause",
            "decode_us_per_step": 1e3 * d_ms / n_dec, "device_status": int(status)}


def idle_pause(ctx, seconds=1.0):
    """All ranks idle for `seconds` with no work queued (the GPU's clock recovers
    from the power cap between two measurements)."""
    ctx["torch"].cuda.synchronize()
    time.sleep(seconds)
    ctx["barrier"]()


def timed_each(ctx, stream, fn, n, flush=None):
    """Mean device time (ms) of fn(i) over n calls, each bracketed by its own CUDA
    events on `stream`. With `flush`, a write of a buffer larger than L2 runs
    before every call, outside the events, so each call starts with cold L2 (the
    state a layer sees after the rest of a model has run)."""
    torch = ctx["torch"]
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    ctx["barrier"]()
    torch.cuda.synchronize()
    for i in range(n):
        if flush is not None:
            flush.add_(1)
        ev[i][0].record(stream)
        fn(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    ctx["barrier"]()
    return ctx["max_over_ranks"](sum(a.elapsed_time(b) for a, b in ev) / n)


def graph_time(ctx, stream, fns, reps=20, n=5):
    """Device time (ms) of one pass of fns (each fn(st) enqueues its work on stream
    st), from a CUDA graph of reps passes back to back, replayed n times between two
    events on `stream`; max over ranks."""
    torch = ctx["torch"]
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for f in fns:
            f(side)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        cur = torch.cuda.current_stream()
        for _ in range(reps):
            for f in fns:
                f(cur)
    g.replay()
    ctx["barrier"]()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ctx["barrier"]()
    del g
    return ctx["max_over_ranks"](e0.elapsed_time(e1) / (n * reps))


def graph_delta(ctx, stream, base, extra, reps=20):
    """Device time (ms) that the calls `extra` add to a pass of `base` (for example
    an L2 flush, so that they start from a cold L2), as the difference of two
    graph timings: no host launch latency and no events between the kernels."""
    return graph_time(ctx, stream, base + extra, reps) - graph_time(ctx, stream, base, reps)


def l2_flush_buffer(torch):
    """256 MB, twice the B200's 126 MB L2."""
    return torch.zeros(64 << 20, dtype=torch.int32, device="cuda")


def decode_bench(ctx, layer, stream):
    """Full-scale decode: 8 sequences x 1 new token per step with carried history and
    conv state. Warm (steps back to back on one batch, W_proj and rows in L2),
    replayed from CUDA graphs of one and of ten steps, and cold (L2 flushed before
    every step); the two-call form split into its tokens-only and hidden-dependent
    halves."""
    torch, ple, pi, bf16_tensor = ctx["torch"], ctx["ple"], ctx["pi"], ctx["bf16_tensor"]
    wd = pi.workload("decode")
    tokens, hidden, hist, conv = pi.decode_batch(wd)
    B, q = tokens.shape
    tk = torch.from_numpy(tokens).cuda()
    hd = bf16_tensor(hidden)
    hs = torch.from_numpy(hist.astype(np.int32)).cuda()
    cs = torch.from_numpy(conv).cuda()
    out = torch.empty(B * q, wd.hidden, dtype=torch.bfloat16, device="cuda")
    h = layer.handle

    def eager(i, st=stream):
        ple.ple_decode_step(h, tk, B, q, hd, out, ple.PLE_OUT_BF16, hs, cs, None, st)

    for i in range(5):
        eager(i)
    n = 500
    ms_eager = timed(ctx, stream, eager, n)
    ple.ple_set_profiling(h, True)
    ple.ple_get_stage_times(h)
    for i in range(50):
        eager(i)
    torch.cuda.synchronize()
    stage = ple.ple_get_stage_times(h)
    ple.ple_set_profiling(h, False)

    graphs = {}
    for per_graph in (1, 10):
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(3):
                eager(i, side)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            for i in range(per_graph):
                eager(i, torch.cuda.current_stream())
        graphs[per_graph] = timed(ctx, stream, lambda i: graph.replay(), n // per_graph) / (n // per_graph * per_graph)
        del graph

    flush = l2_flush_buffer(torch)
    n_cold = 200
    fl = lambda st: flush.add_(1)  # noqa: E731
    ms_cold = graph_delta(ctx, stream, [fl], [lambda st: eager(0, st)])
    # the same after the flush as one eager call between two events: adds the host's
    # submission and the events' own cost, which the same two events around a
    # one-element torch kernel show
    ms_cold_eager = timed_each(ctx, stream, eager, n_cold, flush)
    tiny = torch.zeros(1, device="cuda")
    ms_tiny_eager = timed_each(ctx, stream, lambda i: tiny.add_(1), n_cold, flush)

    def prep(i):
        ple.ple_decode_prepare(h, tk, B, q, hs, stream)

    def rest(i):
        ple.ple_decode_step_prepared(h, hd, out, ple.PLE_OUT_BF16, hs, cs, None, stream)

    pr = lambda st: ple.ple_decode_prepare(h, tk, B, q, hs, st)  # noqa: E731
    rs = lambda st: ple.ple_decode_step_prepared(h, hd, out, ple.PLE_OUT_BF16, hs, cs, None, st)  # noqa: E731
    # each half from a cold L2: flush, prepare, flush, step (the step's rows evicted too)
    prep_cold = graph_delta(ctx, stream, [fl], [pr])
    rest_cold = graph_delta(ctx, stream, [fl, pr, fl], [rs])
    # the hidden-dependent half right after its prepare, from a cold L2: flush, prepare, step
    # (the prepare also pulls W_proj into L2, as it would ahead of the hidden states)
    rest_after_prep = graph_delta(ctx, stream, [fl, pr], [rs])
    prep_warm = graph_time(ctx, stream, [pr])
    rest_warm = graph_delta(ctx, stream, [pr], [rs])
    del flush
    torch.cuda.empty_cache()
    status = ple.ple_get_error(h)

    peaks, _ = load_peaks()
    D, H = wd.row_dim, wd.hidden
    # algorithmic bytes of a step: W_proj fp16, both rows and scales per token, hidden in and
    # out, conv state in and out, tokens and history
    step_bytes = D * H * 2 + B * q * (2 * D + 8 + 2 * H + 2 * H + 8) + B * (2 * 3 * H * 4 + 16)
    world = ctx["world"]
    us = lambda ms: 1e3 * ms  # noqa: E731
    return {"workload": "full-scale decode: 8 sequences x 1 token, 2-token history + 3x2560 conv state",
            "value": B * q * world * n / (ms_eager / 1e3), "unit": "tokens/s", "us_per_step": us(ms_eager) / n,
            "graph_us_per_step": us(graphs[1]), "graph10_us_per_step": us(graphs[10]),
            "cold_us_per_step": us(ms_cold),
            "cold_eager_us_per_step": us(ms_cold_eager), "cold_eager_tiny_torch_kernel_us": us(ms_tiny_eager),
            "cold_roofline": {"bound": "hbm", "algorithmic_bytes_per_step": step_bytes,
                              "achieved_gbs": step_bytes / (ms_cold / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                              "frac": step_bytes / (ms_cold / 1e3) / 1e9 / peaks["hbm_gbs"]},
            "prepared": {"prepare_us_cold": us(prep_cold), "step_prepared_us_cold": us(rest_cold),
                         "step_prepared_us_after_cold_prepare": us(rest_after_prep),
                         "prepare_us_warm": us(prep_warm), "step_prepared_us_warm": us(rest_warm),
                         "note": "ple_decode_prepare needs only the tokens and history; ple_decode_step_prepared "
                                 "(gate, projection, conv, residual, state) is the part that waits for hidden"},
            "stage_us_per_launch": {k: 1e3 * v[0] / max(v[1], 1) for k, v in stage.items() if v[1]},
            "device_status": int(status),
            "note": "warm: one batch reused, steps back to back (W_proj and rows stay in L2, each step's W_proj "
                    "copies overlap the previous step under programmatic dependent launch); graph: one or ten "
                    "captured steps per replay (no overlap across replays); cold: 256 MB written before every "
                    "step, the step's time the difference between graphs of 20 x (write, step) and 20 x (write) "
                    "(the same for the prepared halves, warm ones as graphs of 20 x (prepare, step) minus 20 x "
                    "(prepare)); cold_eager: one eager call after the write between two events, with the host's "
                    "submission inside, beside the same around a one-element torch kernel"}


def mtp_bench(ctx, layer, stream):
    """MTP-style decode: 64 sequences x 3 tokens per step (1 accepted + 2 drafts) for 100
    steps after a 512-token prompt per sequence (19 sequences share prompt and continuation);
    the state advances by each step's n_commit."""
    torch, ple, pi, bf16_tensor = ctx["torch"], ctx["ple"], ctx["pi"], ctx["bf16_tensor"]
    w = pi.workload("mtp")
    sess = pi.mtp_session(w)
    B, P = sess["prompts"].shape
    q = w.extra["q"]
    h = layer.handle
    hist = torch.full((B, 2), -1, dtype=torch.int32, device="cuda")
    conv = torch.zeros(B, 3, w.hidden, dtype=torch.float32, device="cuda")
    half = B // 2
    for b0 in (0, half):                       # prompts in two packed batches of 16,384 tokens
        toks = torch.from_numpy(np.ascontiguousarray(sess["prompts"][b0:b0 + half].reshape(-1))).cuda()
        offs = torch.from_numpy((np.arange(half + 1) * P).astype(np.int32)).cuda()
        hid = bf16_tensor(sess["prompt_hidden"][b0 * P:(b0 + half) * P])
        out = torch.empty_like(hid)
        ple.ple_forward(h, toks, half * P, offs, half, hid, out, ple.PLE_OUT_BF16,
                        (hist[b0:b0 + half], conv[b0:b0 + half]), stream)
    steps = [(torch.from_numpy(t).cuda(), bf16_tensor(hd), torch.from_numpy(nc).cuda())
             for t, hd, nc in sess["steps"]]
    out = torch.empty(B * q, w.hidden, dtype=torch.bfloat16, device="cuda")

    def step(i):
        tk, hd, nc = steps[i % len(steps)]
        ple.ple_decode_step(h, tk, B, q, hd, out, ple.PLE_OUT_BF16, hist, conv, nc, stream)

    hist0, conv0 = hist.clone(), conv.clone()
    for i in range(3):
        step(i)
    n = len(steps)
    hist.copy_(hist0)
    conv.copy_(conv0)
    ms = timed(ctx, stream, step, n)
    # the first 20 steps captured in one CUDA graph, replayed (no host in the loop;
    # consecutive steps overlap under programmatic dependent launch)
    hist.copy_(hist0)
    conv.copy_(conv0)
    ms_graph = graph_time(ctx, stream, [lambda st, i=i: ple.ple_decode_step(
        h, steps[i][0], B, q, steps[i][1], out, ple.PLE_OUT_BF16, hist, conv, steps[i][2], st) for i in range(20)], reps=1)
    ms_graph /= 20
    # the same 100 steps again from the same state, each after an L2 flush
    hist.copy_(hist0)
    conv.copy_(conv0)
    flush = l2_flush_buffer(torch)
    ms_cold_eager = timed_each(ctx, stream, step, n, flush)
    ms_cold = graph_delta(ctx, stream, [lambda st: flush.add_(1)],
                          [lambda st: ple.ple_decode_step(h, steps[0][0], B, q, steps[0][1], out, ple.PLE_OUT_BF16,
                                                          hist, conv, steps[0][2], st)])
    del flush
    torch.cuda.empty_cache()
    status = ple.ple_get_error(h)
    committed = int(sum(int(nc.sum()) for _, _, nc in sess["steps"]))
    world = ctx["world"]
    return {"workload": "MTP decode: 64 sequences x 3 tokens/step, 100 steps, 30% shared prefix",
            "value": B * q * world * n / (ms / 1e3), "unit": "tokens/s (processed)",
            "committed_tokens_per_s": committed * world / (ms / 1e3), "us_per_step": 1e3 * ms / n,
            "graph20_us_per_step": 1e3 * ms_graph,
            "cold_us_per_step": 1e3 * ms_cold, "cold_eager_us_per_step": 1e3 * ms_cold_eager,
            "device_status": int(status),
            "note": "us_per_step: 100 eager steps back to back; graph20: 20 consecutive steps in one CUDA graph, "
                    "replayed; cold: 256 MB written before every step, the step's time the difference between "
                    "graphs of 20 x (write, step) and 20 x (write); cold_eager: the 100 steps each after the write, "
                    "one eager call between two events"}


def long_bench(ctx, layer, stream):
    """Long-context chunked prefill: one 262,144-token sequence of uniform tokens in 16
    chunks of 16,384, conv state and the last two tokens carried across chunks."""
    torch, ple, pi, bf16_tensor = ctx["torch"], ctx["ple"], ctx["pi"], ctx["bf16_tensor"]
    w = pi.workload("long")
    chunk = w.extra["chunk"]
    n_chunks = w.extra["total"] // chunk
    rng = np.random.default_rng([w.seed, 13])
    toks = [torch.from_numpy(pi.tokens_uniform(rng, chunk, w.vocab)).cuda() for _ in range(n_chunks)]
    hids = [bf16_tensor(pi.hidden_bf16(rng, chunk, w.hidden)) for _ in range(4)]   # hidden values reused
    offs = torch.tensor([0, chunk], dtype=torch.int32, device="cuda")
    out = torch.empty(chunk, w.hidden, dtype=torch.bfloat16, device="cuda")
    hist = torch.full((1, 2), -1, dtype=torch.int32, device="cuda")
    conv = torch.zeros(1, 3, w.hidden, dtype=torch.float32, device="cuda")
    h = layer.handle

    def fn(i):
        ple.ple_forward(h, toks[i % n_chunks], chunk, offs, 1, hids[i % 4], out, ple.PLE_OUT_BF16, (hist, conv),
                        stream)

    fn(0)
    hist.fill_(-1)
    conv.zero_()
    ms = timed(ctx, stream, fn, n_chunks)
    world = ctx["world"]
    return {"workload": "long context: 262,144 uniform tokens, 16 chunks of 16,384 with carried state",
            "value": chunk * n_chunks * world / (ms / 1e3), "unit": "tokens/s", "ms_total": ms}


if __name__ == "__main__":
    main()
