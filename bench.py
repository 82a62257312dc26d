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
GATHER_SOURCES = ["gram_embedding_lookup_b200/csrc/ple_kernels.cu"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ple", "reference"], default="ple")
    ap.add_argument("--table-rows", type=int, default=0,
                    help="rows per sub-table (default: the full 10,000,048); smaller only for profiling captures")
    ap.add_argument("--sets", type=int, default=3, help="rotating input sets")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the e2e, decode and clocks measurements")
    ap.add_argument("--ref-tokens", type=int, default=512, help="tokens per reference-arm step")
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


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.environ.get("PLE_CLOCKS_CSV") or os.path.join(
            tempfile.gettempdir(), f"ple_clocks_{os.getpid()}_{index}.csv")

    def start(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                c = [x.strip() for x in line.split(",")]
                if len(c) < 9:
                    continue
                try:
                    sms.append(float(c[1]))
                    maxs.append(float(c[2]))
                except ValueError:
                    continue
                for n, v in zip(names, c[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        if not sms:
            return None
        return {"sm_mhz": float(np.median(sms)), "sm_max_mhz": float(max(maxs)), "reasons": sorted(reasons),
                "samples": len(sms)}


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
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def prefill_config(args, w, world):
    return {"workload": "full-scale prefill: 16,384 packed tokens (sequences 1000/3384/4000/8000), "
                        "Zipf(1.1) tokens over 248,320, hidden 2560, 2 x 10,000,048 x 2560 FP8 table in HBM",
            "model": "PLE n-gram embedding layer", "global_batch": 16384 * world, "seq_len": 16384,
            "table_rows_per_order": w.rows_per_order, "parallelism": f"replicas x{world}",
            "l2": f"{args.sets} rotating input sets (>2x L2 per step)", "out_dtype": "bf16"}


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

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    stream = torch.cuda.current_stream()
    w0 = pi.workload("prefill")
    w = w0 if args.table_rows <= 0 else pi.Workload("prefill", w0.vocab, args.table_rows, w0.row_dim, w0.hidden,
                                                      w0.table_seed, w0.seed, w0.extra)
    layer = DeviceLayer(w, max_tokens=16384, max_seqs=64)
    h = layer.handle
    H = w.hidden

    sets = []
    for v in range(args.sets):
        tokens, offsets, hidden = pi.prefill_batch(w, variant=v + 100 * rank)
        sets.append(dict(tokens=torch.from_numpy(tokens).cuda(), offsets=torch.from_numpy(offsets).cuda(),
                         hidden=bf16_tensor(hidden), out=torch.empty(len(tokens), H, dtype=torch.bfloat16,
                                                                      device="cuda"),
                         T=len(tokens), S=len(offsets) - 1, host=(tokens, offsets, hidden)))

    def step(i):
        s = sets[i % len(sets)]
        ple.ple_forward(h, s["tokens"], s["T"], s["offsets"], s["S"], s["hidden"], s["out"], ple.PLE_OUT_BF16,
                        None, stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if ple.ple_get_error(h) != 0:
        raise SystemExit("device status error during warm-up")

    ple.ple_set_profiling(h, True)
    ple.ple_get_stage_times(h)
    clocks = ClockSampler(local) if not args.no_extras else None
    if clocks:
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
    barrier()
    launches = ple.ple_launch_count(h) - launches0
    clk = clocks.stop() if clocks else None
    stage = ple.ple_get_stage_times(h)
    ple.ple_set_profiling(h, False)
    status = ple.ple_get_error(h)
    ms = max_over_ranks(ev0.elapsed_time(ev1))
    T = sets[0]["T"]
    ms_per_step = ms / args.steps
    value = T * world * args.steps / (ms / 1e3)

    peaks, peak_kind = load_peaks()
    D = w.row_dim
    gemm_ms, gemm_n = stage["gemm"]
    gemm_s = gemm_ms / 1e3 / max(gemm_n, 1)
    flops = 2.0 * D * H * T
    achieved_tf = flops / gemm_s / 1e12
    peak_tf = peaks["bf16_tflops"]   # fp16 and bf16 share the nominal dense rate (ratio 1)
    gemm_traffic = load_traffic("gemm", "prefill", source_hash(GEMM_SOURCES))
    roofline = {"kernel": "ple gemm (tcgen05 projection + fused gate/conv/residual)", "bound": "tensor",
                "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved_tf / peak_tf,
                "peak_source": f"{peak_kind} bf16_tflops (burst); fp16 nominal ratio 1.0",
                "traffic": gemm_traffic, "algorithmic_flops_per_launch": flops, "launch_ms": gemm_s * 1e3}

    g_ms, g_n = stage["gather"]
    g_s = g_ms / 1e3 / max(g_n, 1)
    gather_bytes = T * (2 * D + 8 + 8 + 2 * D)   # rows + scales + ids in, fp16 e out
    gather = {"bound": "hbm", "achieved": gather_bytes / g_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
              "frac": gather_bytes / g_s / 1e9 / peaks["hbm_gbs"],
              "gathered_row_gbs": T * 2 * D / g_s / 1e9, "launch_ms": g_s * 1e3,
              "traffic": load_traffic("gather", "prefill", source_hash(GATHER_SOURCES)),
              "algorithmic_bytes_per_launch": gather_bytes}
    stages_ms = {k: (v[0] / max(v[1], 1)) for k, v in stage.items()}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic", "config": prefill_config(args, w, world),
        "roofline": roofline, "gather_roofline": gather, "stage_ms_per_launch": stages_ms,
        "gpu_launches": int(launches) * world, "device_status": int(status),
        "gathered_row_gbs_end_to_end": T * 2 * D * args.steps / (ms / 1e3) / 1e9,
    }
    if clk:
        line["clocks"] = clk

    if not args.no_extras:
        line["e2e"] = e2e_prefill(args, ple, h, sets, stream, world, max_over_ranks, barrier)
        line["decode"] = decode_bench(args, ple, pi, layer, stream, max_over_ranks, barrier, world)

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
                                "kind": "oracle",
                                "sample": f"first {n_tok} tokens of the prefill batch, {n_runs} run(s), "
                                          f"rows materialised before timing"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    layer.close()
    if world > 1:
        dist.destroy_process_group()


def e2e_prefill(args, ple, h, sets, stream, world, max_over_ranks, barrier):
    """Same metric through the C ABI with host buffers: H2D of the step's inputs from
    pinned memory, the layer, D2H of the output, all inside the timed region."""
    import torch
    hosts = []
    for s in sets:
        tokens, offsets, hidden = s["host"]
        hosts.append(dict(tokens=torch.from_numpy(tokens).pin_memory(), offsets=torch.from_numpy(offsets).pin_memory(),
                          hidden=torch.from_numpy(hidden.view(np.int16)).view(torch.bfloat16).pin_memory(),
                          out=torch.empty_like(s["out"], device="cpu").pin_memory()))

    def step(i):
        s, hs = sets[i % len(sets)], hosts[i % len(sets)]
        s["tokens"].copy_(hs["tokens"], non_blocking=True)
        s["offsets"].copy_(hs["offsets"], non_blocking=True)
        s["hidden"].copy_(hs["hidden"], non_blocking=True)
        ple.ple_forward(h, s["tokens"], s["T"], s["offsets"], s["S"], s["hidden"], s["out"], ple.PLE_OUT_BF16,
                        None, stream)
        hs["out"].copy_(s["out"], non_blocking=True)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    steps = max(3, min(args.steps, 20))
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1))
    s0 = sets[0]
    h2d = s0["tokens"].numel() * 4 + s0["offsets"].numel() * 4 + s0["hidden"].numel() * 2
    d2h = s0["out"].numel() * 2
    return {"value": s0["T"] * world * steps / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps, "ms_per_step": ms / steps}


def decode_bench(args, ple, pi, layer, stream, max_over_ranks, barrier, world):
    """Full-scale decode: 8 sequences x 1 new token per step, carried history and conv state."""
    import torch
    from ple_inputs.device import bf16_tensor
    wd = pi.workload("decode")
    tokens, hidden, hist, conv = pi.decode_batch(wd)
    B, q = tokens.shape
    tk = torch.from_numpy(tokens).cuda()
    hd = bf16_tensor(hidden)
    hs = torch.from_numpy(hist.astype(np.int32)).cuda()
    cs = torch.from_numpy(conv).cuda()
    out = torch.empty(B * q, wd.hidden, dtype=torch.bfloat16, device="cuda")
    h = layer.handle

    def step():
        ple.ple_decode_step(h, tk, B, q, hd, out, ple.PLE_OUT_BF16, hs, cs, None, stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    barrier()
    n = 200
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ple.ple_set_profiling(h, True)
    ple.ple_get_stage_times(h)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    stage = ple.ple_get_stage_times(h)
    ple.ple_set_profiling(h, False)
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1))
    return {"workload": "full-scale decode: 8 sequences x 1 token, 2-token history + 3x2560 conv state",
            "value": B * q * world * n / (ms / 1e3), "unit": "tokens/s", "us_per_step": 1e3 * ms / n,
            "stage_us_per_launch": {k: 1e3 * v[0] / max(v[1], 1) for k, v in stage.items()},
            "note": "consecutive steps reuse one batch; W_proj (13 MB) stays L2-resident, as in a real decode loop"}


if __name__ == "__main__":
    main()
