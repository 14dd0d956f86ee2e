"""Benchmark of the HSA operator on B200.

One step = one HSA prefill forward of the 32K workload (B2 T32768 H8 D128, chunk 64, topk 16,
chunk-mean landmarks): retrieval scoring + top-K + fusion weights, chunk-major dispatch, per-chunk
attention with the fused blend, bf16 output. The headline metric is prefill tokens/s (B*T tokens per
step). The same run also times every other workload of the benchmark set, each against its roofline
and next to the CPU oracle timed on a bounded sample on the host cores (a reported baseline): the 4K
forward (B1 T4096 H4 D64 topk 8), the 1M-token decode (B16, H8, D128, topk 16), the 16M-token decode
(B1, H8, D128, topk 32; microseconds per token) and the 64K forward+backward.

Peaks: the timed loops last tens of milliseconds, so tensor-core fractions are taken against the
measured burst bf16 figure (bf16_tflops), HBM fractions against the measured copy bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--skip-decode] [--skip-backward]
                  [--skip-prefill] [--skip-cpu] [--decode-cache-len N]

Multi-GPU (torchrun, one process per GPU): HSA's (batch, head) problems are independent, so every
rank runs its own copy of the workload with no data-path collective (weak scaling); the only
collectives are the timing barrier and a max-reduction of the elapsed time.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS_PER_FORWARD = 6     # score_topk (with the chunk counts), scan, tile list, scatter, chunk_attn, finalize
KERNELS_PER_DECODE = 2      # decode_scan, decode_attend
KERNELS_PER_BACKWARD = 6    # delta, count, scan, tile list, scatter, chunk_bwd


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed regions run."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"hsa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                clk, mx = float(parts[1]), float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            sm.append(clk)
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        loaded = [c for c, p in zip(sm, power) if p > 300.0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "samples_under_load": len(loaded)}


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world, cuda=True):
    """All ranks meet (when there are several), then this rank's device work is drained."""
    import torch

    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def max_over_ranks(x, world):
    """The largest x over all ranks (the slowest rank's time); the reduction runs where the process
    group's backend keeps its tensors (the GPU for NCCL, the CPU for gloo)."""
    import torch

    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms_per_step):
    """Throughput of the whole job: every rank processes units_per_rank per step, and a step lasts as
    long as the slowest rank's (ms_per_step, already the max over ranks)."""
    return world * units_per_rank / (ms_per_step / 1e3)


def timed(fn, steps, warmup, world):
    """Device time of `steps` calls of fn (CUDA events on the current stream), max over ranks, ms."""
    import torch

    for _ in range(warmup):
        fn()
    barrier(world)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        fn()
    e1.record(s)
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1), world)


def timed_after(prep, fn, steps, warmup, world):
    """Device time of fn alone, per step, with prep (an L2 flush) run before each step outside the timed
    interval: a pair of CUDA events brackets each fn call on the current stream (max over ranks, ms)."""
    import torch

    for _ in range(warmup):
        prep()
        fn()
    barrier(world)
    s = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        prep()
        e0.record(s)
        fn()
        e1.record(s)
    barrier(world)
    return max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps, world)


def clean(*workspaces):
    """Raise if a bounded device wait of the last call on any of these workspaces ran out (a timed number
    from such a run would be meaningless)."""
    from ultra_long_context_b200 import hsa

    for ws in workspaces:
        hsa.hsa_workspace_status(ws)


def kernel_profile(fn, steps):
    """Per-launch-site device time over `steps` calls, from the library's event hooks."""
    import torch

    from ultra_long_context_b200 import hsa

    torch.cuda.synchronize()
    hsa.hsa_profile_enable(True)
    for _ in range(steps):
        fn()
    torch.cuda.synchronize()
    prof = hsa.hsa_profile_summary()
    hsa.hsa_profile_enable(False)
    return prof


# ------------------------------------------------------------------------------------------------
# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu capture of the
# current kernels on these workloads; set back to None whenever the kernel changes.
TRAFFIC_BYTES = {
    ("fwd_t32k_h8_d128_k16", "chunk_attn"): 737_926_144 + 235_332_096,
    ("fwd_t32k_h8_d128_k16", "score_topk"): 136_467_456 + 279_436_032,
    ("decode_16m_b1_h8_d128_k32", "decode_scan"): 536_948_992 + 3_297_792,
    ("fwdbwd_t64k_h8_d128_k16", "chunk_bwd"): 2_288_028_416 + 1_252_866_048,
}
SCORE_LIMITER = ("ALU pipe (per-row selection: group maxima, candidate keys, sorting networks); "
                 "the tensor pipe is busy about 14% of the time")
# fp32 reductions into L2-resident rows, 4 rows x 128 B per red.global.add.v4.f32, 16-24 warps per SM:
# the ceiling measured on this GPU type for the combine of the chunk attention (GB/s)
COMBINE_PEAK_GBS = 6252.1


# ------------------------------------------------------------------------------------------------
# algorithmic work


def pairs_closed_form(w, topk=None):
    """Selected (token, chunk) pairs of a forward workload: every row keeps min(topk, n_t) chunks."""
    import numpy as np

    k = topk or w.topk
    n_t = np.minimum((np.arange(w.T) + 1) // w.chunk, w.T // w.chunk)
    return int(w.B * w.H * np.minimum(n_t, k).sum())


def forward_config(w, world):
    """The `config` of a forward workload's line (shared by both arms, so that they name the same job)."""
    return {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "D": w.D, "chunk": w.chunk, "topk": w.topk,
            "landmarks": "chunk mean + N(0, 0.1^2)" if w.landmarks == "chunk_mean" else "iid N(0, 1)",
            "pairs": pairs_closed_form(w), "l2": "inputs larger than L2 (Q, K, V = 402 MB)",
            "parallelism": f"dp{world}"}


def forward_work(w, sel_idx):
    """Causal scoring flops, chunk-attention flops (selected pairs only) and pair count."""
    B, H, T, D, C = w.B, w.H, w.T, w.D, w.chunk
    t = __import__("numpy").arange(T)
    n_t = (t + 1) // C
    score_flops = 2.0 * D * B * H * float(n_t.sum())
    pairs = int((sel_idx >= 0).sum().item())
    attn_flops = 4.0 * C * D * pairs
    return score_flops, attn_flops, pairs


def roofline_entry(name, prof, algo, unit, peak, bound, peak_kind, traffic=None):
    cnt, ms = prof[name]
    avg_s = ms / cnt / 1e3
    achieved = algo / avg_s / (1e12 if unit == "TFLOP/s" else 1e9)
    return {"kernel": name, "bound": bound, "achieved": round(achieved, 3), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic, "avg_launch_us": round(avg_s * 1e6, 3),
            "peak_source": peak_kind}


# ------------------------------------------------------------------------------------------------
# CPU oracle baseline


def oracle_forward_sample(w, Qh, Kh, Vh, Lh, target_s=10.0, rng_seed=0):
    """Time the oracle on a growing sample of token rows until ~target_s of wall time."""
    import numpy as np

    import oracle

    rng = np.random.default_rng(rng_seed)
    BH, T = w.B * w.H, w.T
    n, spent, rows_done = 256, 0.0, 0
    while spent < target_s and n <= (1 << 20):
        rows = rng.integers(0, BH * T, n)
        t0 = time.perf_counter()
        oracle.forward(Qh, Kh, Vh, Lh, chunk=w.chunk, topk=w.topk, rows=rows)
        dt = time.perf_counter() - t0
        spent += dt
        rows_done += n
        n *= 2
    # a token is H rows (one per head); sampled rows are uniform over (b, h, t)
    tokens_per_s = rows_done / w.H / spent
    return tokens_per_s, rows_done, spent


def oracle_decode_sample(q, Kc, Vc, Lc, lens, topk, rows):
    """Time the oracle's decode (Step 2 over every landmark, then Steps 3-4 on the gathered chunks) for the
    listed (b, h) rows; the host copies and the gather of the selected chunks are not timed. Returns the
    seconds spent."""
    import numpy as np

    import oracle

    spent = 0.0
    D = q.shape[-1]
    for b, h in rows:
        qh = q[b:b + 1, h:h + 1].float().cpu().numpy()
        Lh = Lc[b:b + 1, h:h + 1].float().cpu().numpy()
        ln = lens[b:b + 1].cpu().numpy()
        t0 = time.perf_counter()
        sel = oracle.decode_select(qh, Lh, ln, chunk=64, topk=topk)
        spent += time.perf_counter() - t0
        idx = sel["sel_idx"].reshape(-1)
        k = int((idx >= 0).sum())
        Kg = np.zeros((1, topk, 64, D), np.float32)
        Vg = np.zeros_like(Kg)
        Lg = np.zeros((1, topk, D), np.float32)
        for j in range(k):
            c = int(idx[j])
            Kg[0, j] = Kc[b, h, 64 * c:64 * (c + 1)].float().cpu().numpy()
            Vg[0, j] = Vc[b, h, 64 * c:64 * (c + 1)].float().cpu().numpy()
            Lg[0, j] = Lh[0, 0, c]
        t0 = time.perf_counter()
        oracle.attend_gathered(qh.reshape(1, D), Lg, Kg, Vg, np.array([k], np.int32))
        spent += time.perf_counter() - t0
    return spent


def decode_entry(hsa, inputs, wd, dev, steps, warmup, world, peaks, peak_kind, cpu=False):
    """Time one decode workload (device time per step and per token) against the HBM roofline; with cpu,
    also the oracle on a bounded sample of its (b, h) rows."""
    import torch

    q, Kc, Vc, Lc, lens, _ = inputs.workload_inputs(wd, device=dev)
    dout_ = torch.empty_like(q)
    didx = torch.empty((wd.B, wd.H, wd.topk), dtype=torch.int32, device=dev)
    dw = torch.empty((wd.B, wd.H, wd.topk), dtype=torch.float32, device=dev)
    dws = torch.empty(hsa.hsa_decode_workspace_size(wd.B, wd.H, wd.cache_len, wd.D, 64, wd.topk) + 256,
                      dtype=torch.uint8, device=dev)

    def dec():
        hsa.hsa_decode(q, Kc, Vc, Lc, lens, wd.topk, out=dout_, sel_idx=didx, sel_w=dw, workspace=dws)

    dms = timed(dec, steps, warmup, world) / steps
    clean(dws)
    prof = kernel_profile(dec, steps)
    n = wd.cache_len // 64
    scan_bytes = wd.B * wd.H * (n * wd.D * 2 + wd.D * 2)
    gather_bytes = wd.B * wd.H * wd.topk * 2 * 64 * wd.D * 2
    hbm = peaks["hbm_gbs"]
    step_gbs = (scan_bytes + gather_bytes) / (dms / 1e3) / 1e9
    entry = {
        "workload": wd.name,
        "config": {"workload": wd.name, "B": wd.B, "H": wd.H, "D": wd.D, "cache_len": wd.cache_len, "chunk": 64,
                   "topk": wd.topk, "l2": "inputs larger than L2 (landmarks alone are 512 MiB)",
                   "parallelism": f"dp{world}"},
        "us_per_step": round(dms * 1e3, 3), "us_per_token": round(dms * 1e3 / wd.B, 3), "ms_per_step": round(dms, 5),
        "steps": steps,
        "roofline": roofline_entry("decode_scan", prof, scan_bytes, "GB/s", hbm, "hbm", f"{peak_kind} hbm_gbs",
                                   TRAFFIC_BYTES.get((wd.name, "decode_scan"))),
        "step_vs_hbm": {"algorithmic_bytes": scan_bytes + gather_bytes, "achieved_GBs": round(step_gbs, 1),
                        "frac": round(step_gbs / hbm, 4),
                        "target": f"70% of measured HBM: <= {(scan_bytes + gather_bytes) / (0.7 * hbm * 1e3):.1f} "
                                  "us per step"},
        "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof.items()},
    }
    if cpu:
        rows = [(0, 0), (wd.B - 1, wd.H - 1)]
        spent = oracle_decode_sample(q, Kc, Vc, Lc, lens, wd.topk, rows)
        per_row = spent / len(rows)
        entry["cpu_baseline"] = {"value": round(per_row * wd.H * 1e6, 1), "unit": "us/token", "cores": host_cores(),
                                 "kind": "oracle",
                                 "sample": f"{len(rows)} (b, h) rows of the workload (fp64 oracle: every landmark "
                                           f"scored, then the selected chunks attended), {spent:.2f} s; a token is "
                                           f"{wd.H} rows"}
    del q, Kc, Vc, Lc, dws
    return entry


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ------------------------------------------------------------------------------------------------


def run_reference(args):
    """Reference arm: the CPU oracle, as it stands, on the host cores (rank 0 only).

    Each step is a bounded sample of the headline workload: a fixed number of token-head rows drawn
    uniformly from it, run through the fp64 oracle. ms_per_step is the wall time of one such sample
    step as measured, and value the token rate over all timed steps (a token is H rows)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np

    import oracle
    from ultra_long_context_b200 import inputs

    w = inputs.WORKLOADS["fwd_t32k_h8_d128_k16"]
    Q, K, V, L = inputs.forward_inputs(w.B, w.H, w.T, w.D, w.seed, landmarks=w.landmarks, device="cpu")
    Qh, Kh, Vh, Lh = (x.float().numpy() for x in (Q, K, V, L))
    BH = w.B * w.H
    # rows per step: about 20 s of oracle work over all timed steps (measured on a probe sample)
    probe = np.random.default_rng(99).integers(0, BH * w.T, 2048)
    t0 = time.perf_counter()
    oracle.forward(Qh, Kh, Vh, Lh, chunk=w.chunk, topk=w.topk, rows=probe)
    rate = len(probe) / max(1e-6, time.perf_counter() - t0)
    rows_per_step = int(max(256, min(1 << 20, rate * 20.0 / max(1, args.steps))))

    def step(i):
        rows = np.random.default_rng(i).integers(0, BH * w.T, rows_per_step)
        t = time.perf_counter()
        oracle.forward(Qh, Kh, Vh, Lh, chunk=w.chunk, topk=w.topk, rows=rows)
        return time.perf_counter() - t

    for i in range(args.warmup):
        step(1000 + i)
    spent = [step(i) for i in range(args.steps)]
    total = sum(spent)
    value = args.steps * rows_per_step / w.H / total
    sample = (f"each step: {rows_per_step} token-head rows drawn uniformly from the 32K workload (B2 H8 T32768 "
              f"D128 topk16), fp64 oracle with OpenMP; {args.steps} steps, {total:.1f} s")
    line = {"impl": "reference", "metric": "HSA prefill tokens/s (B2 T32768 H8 D128 chunk64 topk16)",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "step": f"a sample of {rows_per_step} token-head rows (not the full {BH * w.T}-row workload)",
            "config": forward_config(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--skip-prefill", action="store_true", help="time only the decode / backward parts")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-decode-1m", action="store_true", help="of the decode, time only the 16M-token cache")
    ap.add_argument("--skip-backward", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-options", action="store_true",
                    help="skip the timings of the optional paths (query-key norm, separate retrieval query)")
    ap.add_argument("--grouped-decode-only", action="store_true",
                    help="of the decode, time only the 16:1 grouped-head case (small footprint, for profiling)")
    ap.add_argument("--decode-cache-len", type=int, default=None,
                    help="override the decode cache length (small cases for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return

    import numpy as np
    import torch

    from ultra_long_context_b200 import hsa, inputs

    world, rank, local = dist_setup(args)
    peaks, peak_kind = load_peaks()
    clocks = ClockSampler(local)
    dev = torch.device("cuda", local)

    clocks.start()
    # ---------------- prefill forward (headline) ----------------
    value = ms_per_step = None
    roof = roof_score = roof_combine = breakdown = e2e = None
    pairs = 0
    # the timed loops last tens of milliseconds: the burst figure is the denominator (the sustained one
    # is for kernels timed inside a seconds-long loop under the power cap)
    tensor_peak = peaks["bf16_tflops"]
    tensor_kind = f"{peak_kind} bf16_tflops (burst: timed loops of tens of ms)"
    w = inputs.WORKLOADS["fwd_t32k_h8_d128_k16"]
    if not args.skip_prefill:
        w = inputs.WORKLOADS["fwd_t32k_h8_d128_k16"]
        Q, K, V, L = inputs.forward_inputs(w.B, w.H, w.T, w.D, w.seed + rank, landmarks=w.landmarks, device=dev)
        out = torch.empty_like(Q)
        sel_idx = torch.empty((w.B, w.H, w.T, w.topk), dtype=torch.int32, device=dev)
        sel_w = torch.empty((w.B, w.H, w.T, w.topk), dtype=torch.float32, device=dev)
        ws = torch.empty(hsa.hsa_forward_workspace_size(w.B, w.H, w.T, w.D, w.chunk, w.topk) + 256, dtype=torch.uint8,
                         device=dev)

        def fwd():
            hsa.hsa_forward(Q, K, V, L, w.topk, out=out, sel_idx=sel_idx, sel_w=sel_w, workspace=ws)

        ms = timed(fwd, args.steps, args.warmup, world)
        clean(ws)
        ms_per_step = ms / args.steps
        tokens = w.B * w.T
        value = whole_job_rate(tokens, world, ms_per_step)
        prof_fwd = kernel_profile(fwd, args.steps)
        score_flops, attn_flops, pairs = forward_work(w, sel_idx)
        assert pairs == pairs_closed_form(w), (pairs, pairs_closed_form(w))
        dominant = max((k for k in prof_fwd if k != "memset"), key=lambda k: prof_fwd[k][1])
        algo = {"chunk_attn": attn_flops, "score_topk": score_flops}
        roof = roofline_entry(dominant, prof_fwd, algo.get(dominant, attn_flops), "TFLOP/s", tensor_peak, "tensor",
                              tensor_kind, TRAFFIC_BYTES.get((w.name, dominant)))
        roof_score = roofline_entry("score_topk", prof_fwd, score_flops, "TFLOP/s", tensor_peak, "tensor",
                                    tensor_kind, TRAFFIC_BYTES.get((w.name, "score_topk")))
        roof_score["limiter"] = SCORE_LIMITER
        # the combine of the chunk attention: pairs x D fp32 reductions into the tokens' accumulator rows
        roof_combine = roofline_entry("chunk_attn", prof_fwd, pairs * w.D * 4, "GB/s", COMBINE_PEAK_GBS, "l2-red",
                                      "measured red.global.add.v4.f32 ceiling, L2-resident rows")
        breakdown = {k: {"launches": c, "avg_us": round(t / c * 1e3, 2), "share": round(t / sum(x[1] for x in
                                                                                               prof_fwd.values()), 4)}
                     for k, (c, t) in prof_fwd.items()}

        # ---------------- e2e: host buffers through the public API ----------------
        # Every step copies its inputs from pinned host memory and reads its output back, as an input
        # pipeline does: step i + 1's inputs go up on one stream while step i computes on the current
        # stream, and step i's output comes back on a third (inputs and outputs double-buffered on the
        # device). All the copies of the timed steps are inside the timed region.
        hQ, hK, hV, hL = (x.cpu().pin_memory() for x in (Q, K, V, L))
        hout = [tuple(torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in (out, sel_idx, sel_w))
                for _ in range(2)]
        dev_in = [tuple(torch.empty_like(x) for x in (Q, K, V, L)) for _ in range(2)]
        dev_out = [tuple(torch.empty_like(x) for x in (out, sel_idx, sel_w)) for _ in range(2)]
        s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
        comp = torch.cuda.current_stream()
        ev_in, ev_used, ev_out, ev_read = ([torch.cuda.Event() for _ in range(2)] for _ in range(4))

        def upload(i):
            b = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_used[b])  # step i - 2 is done reading this buffer
                for d, h in zip(dev_in[b], (hQ, hK, hV, hL)):
                    d.copy_(h, non_blocking=True)
                ev_in[b].record(s_up)

        def e2e_run(n):
            upload(0)
            for i in range(n):
                b = i % 2
                if i + 1 < n:
                    upload(i + 1)
                comp.wait_event(ev_in[b])
                if i >= 2:
                    comp.wait_event(ev_read[b])  # step i - 2's output has been read back
                dq, dk, dv, dl = dev_in[b]
                do, di, dw = dev_out[b]
                hsa.hsa_forward(dq, dk, dv, dl, w.topk, out=do, sel_idx=di, sel_w=dw, workspace=ws)
                ev_used[b].record(comp)
                ev_out[b].record(comp)
                with torch.cuda.stream(s_down):
                    s_down.wait_event(ev_out[b])
                    for h_, d_ in zip(hout[b], dev_out[b]):
                        h_.copy_(d_, non_blocking=True)
                    ev_read[b].record(s_down)
            comp.wait_stream(s_up)
            comp.wait_stream(s_down)

        e2e_run(args.warmup)
        barrier(world)
        t0_ev, t1_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0_ev.record(comp)
        e2e_run(args.steps)
        t1_ev.record(comp)
        barrier(world)
        e2e_ms = max_over_ranks(t0_ev.elapsed_time(t1_ev), world) / args.steps
        h2d = sum(x.numel() * x.element_size() for x in (hQ, hK, hV, hL))
        d2h = sum(x.numel() * x.element_size() for x in hout[0])
        e2e = {"value": whole_job_rate(tokens, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
               "returned": "out, sel_idx and sel_w",
               "pipeline": "inputs of step i+1 uploaded and step i's results read back while step i computes"}
        del hQ, hK, hV, hL, hout, dev_in, dev_out

    extra = {}
    # ---------------- optional paths on the same 32K workload ----------------
    if not args.skip_prefill and not args.skip_options:
        osteps = max(3, args.steps // 2)
        opts = {}
        ws_n = torch.empty(hsa.hsa_forward_ex_workspace_size(w.B, w.H, w.H, w.T, w.D, w.chunk, w.topk,
                                                             hsa.HSA_QK_NORM) + 256, dtype=torch.uint8, device=dev)

        def fwd_norm():
            hsa.hsa_forward(Q, K, V, L, w.topk, out=out, sel_idx=sel_idx, sel_w=sel_w, workspace=ws_n, qk_norm=True)

        n_ms = timed(fwd_norm, osteps, args.warmup, world) / osteps
        clean(ws_n)
        prof_n = kernel_profile(fwd_norm, osteps)
        norm_bytes = 2 * (2 * w.B * w.H * w.T * w.D * 2)  # read Q and K, write their normalised copies
        opts["qk_norm"] = {
            "ms_per_step": round(n_ms, 4), "tokens_per_s": round(whole_job_rate(w.B * w.T, world, n_ms), 1),
            "vs_plain": round(n_ms / ms_per_step, 4),
            "roofline": roofline_entry("qk_norm", prof_n, norm_bytes, "GB/s", peaks["hbm_gbs"], "hbm",
                                       f"{peak_kind} hbm_gbs"),
        }
        Qs_ = inputs.forward_inputs(w.B, w.H, w.T, w.D, w.seed + 7 + rank, landmarks=w.landmarks, device=dev)[0]

        def fwd_qs():
            hsa.hsa_forward(Q, K, V, L, w.topk, out=out, sel_idx=sel_idx, sel_w=sel_w, workspace=ws, Qs=Qs_)

        s_ms = timed(fwd_qs, osteps, args.warmup, world) / osteps
        clean(ws)
        opts["separate_retrieval_query"] = {
            "ms_per_step": round(s_ms, 4), "tokens_per_s": round(whole_job_rate(w.B * w.T, world, s_ms), 1),
            "vs_plain": round(s_ms / ms_per_step, 4)}
        del ws_n, Qs_
        # topk 64 (the per-token procedure's default) on the same workload
        k64 = 64
        ws_64 = torch.empty(hsa.hsa_forward_workspace_size(w.B, w.H, w.T, w.D, w.chunk, k64) + 256, dtype=torch.uint8,
                            device=dev)
        idx_64 = torch.empty((w.B, w.H, w.T, k64), dtype=torch.int32, device=dev)
        w_64 = torch.empty((w.B, w.H, w.T, k64), dtype=torch.float32, device=dev)

        def fwd_k64():
            hsa.hsa_forward(Q, K, V, L, k64, out=out, sel_idx=idx_64, sel_w=w_64, workspace=ws_64)

        k_ms = timed(fwd_k64, osteps, args.warmup, world) / osteps
        clean(ws_64)
        prof_k = kernel_profile(fwd_k64, osteps)
        pairs_64 = pairs_closed_form(w, k64)
        opts["topk_64"] = {
            "shape": f"B{w.B} H{w.H} T{w.T} D{w.D} topk{k64}", "ms_per_step": round(k_ms, 4),
            "tokens_per_s": round(whole_job_rate(w.B * w.T, world, k_ms), 1), "pairs": pairs_64,
            "roofline": roofline_entry("chunk_attn", prof_k, 4.0 * w.chunk * w.D * pairs_64, "TFLOP/s", tensor_peak,
                                       "tensor", tensor_kind),
            "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof_k.items()}}
        del ws_64, idx_64, w_64
        torch.cuda.empty_cache()
        # 16 query heads per key/value head (the pages' ratio): B1 H16 Hkv1, the same query rows and pairs
        # as the headline workload, one K/V/L head
        Hg, Hkv_g, Bg = 16, 1, 1
        gQ = inputs.forward_inputs(Bg, Hg, w.T, w.D, w.seed + 11 + rank, landmarks=w.landmarks, device=dev)[0]
        _, gK, gV, gL = inputs.forward_inputs(Bg, Hkv_g, w.T, w.D, w.seed + 12 + rank, landmarks=w.landmarks,
                                              device=dev)
        gout = torch.empty_like(gQ)
        gidx = torch.empty((Bg, Hg, w.T, w.topk), dtype=torch.int32, device=dev)
        gw = torch.empty((Bg, Hg, w.T, w.topk), dtype=torch.float32, device=dev)
        gws = torch.empty(hsa.hsa_forward_ex_workspace_size(Bg, Hg, Hkv_g, w.T, w.D, w.chunk, w.topk, 0) + 256,
                          dtype=torch.uint8, device=dev)

        def fwd_gqa():
            hsa.hsa_forward(gQ, gK, gV, gL, w.topk, out=gout, sel_idx=gidx, sel_w=gw, workspace=gws)

        g_ms = timed(fwd_gqa, osteps, args.warmup, world) / osteps
        clean(gws)
        prof_g = kernel_profile(fwd_gqa, osteps)
        opts["grouped_heads_16to1"] = {
            "shape": f"B{Bg} H{Hg} Hkv{Hkv_g} T{w.T} D{w.D} topk{w.topk}", "ms_per_step": round(g_ms, 4),
            "tokens_per_s": round(whole_job_rate(Bg * w.T, world, g_ms), 1),
            "token_heads_per_s": round(whole_job_rate(Bg * w.T * Hg, world, g_ms), 1),
            "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof_g.items()}}
        del gQ, gK, gV, gL, gout, gidx, gw, gws
        torch.cuda.empty_cache()
        # variable-length batches in the packed token-major layout: the headline batch itself (2 x 32768,
        # the cost of the layout moves), and 65536 tokens in 7 sequences of 1K to 32K
        tm = lambda x: x.transpose(1, 2).reshape(-1, x.shape[1], x.shape[3]).contiguous()
        for name, lens in (("varlen_equal_2x32k", [w.T, w.T]),
                           ("varlen_mixed_7seq", [32768, 16384, 8192, 4096, 2048, 1024, 1024])):
            vQ = torch.cat([tm(inputs.forward_inputs(1, w.H, T, w.D, w.seed + 20 + i, landmarks=w.landmarks,
                                                     device=dev)[0]) for i, T in enumerate(lens)])
            vK, vV = torch.empty_like(vQ).normal_(), torch.empty_like(vQ).normal_()
            vL = torch.randn((sum(T // 64 for T in lens), w.H, w.D), device=dev).to(torch.bfloat16)
            cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device=dev)
            vout = torch.empty_like(vQ)
            vidx = torch.empty((vQ.shape[0], w.H, w.topk), dtype=torch.int32, device=dev)
            vw = torch.empty((vQ.shape[0], w.H, w.topk), dtype=torch.float32, device=dev)
            vws = torch.empty(hsa.lib().hsa_forward_varlen_workspace_size(len(lens), w.H, w.H, max(lens), w.D, 64,
                                                                          w.topk, 0) + 256, dtype=torch.uint8,
                              device=dev)

            def fwd_var():
                hsa.hsa_forward_varlen(vQ, vK, vV, vL, cu, max(lens), w.topk, out=vout, sel_idx=vidx, sel_w=vw,
                                       workspace=vws)

            v_ms = timed(fwd_var, osteps, args.warmup, world) / osteps
            clean(vws)
            prof_v = kernel_profile(fwd_var, osteps)
            opts[name] = {"lengths": lens, "ms_per_step": round(v_ms, 4),
                          "tokens_per_s": round(whole_job_rate(sum(lens), world, v_ms), 1),
                          "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)}
                                      for k, (c, t) in prof_v.items()}}
            del vQ, vK, vV, vL, vout, vidx, vw, vws
            torch.cuda.empty_cache()
        extra["fwd_options"] = dict(workload=w.name, steps=osteps, **opts)

    # ---------------- small forward, 4K tokens (B1 T4096 H4 D64 topk 8) ----------------
    if not args.skip_prefill:
        w1 = inputs.WORKLOADS["fwd_t4k_h4_d64_k8"]
        Q1, K1, V1, L1 = inputs.forward_inputs(w1.B, w1.H, w1.T, w1.D, w1.seed + rank, landmarks=w1.landmarks,
                                               device=dev)
        out1 = torch.empty_like(Q1)
        idx1 = torch.empty((w1.B, w1.H, w1.T, w1.topk), dtype=torch.int32, device=dev)
        sw1 = torch.empty((w1.B, w1.H, w1.T, w1.topk), dtype=torch.float32, device=dev)
        ws1 = torch.empty(hsa.hsa_forward_workspace_size(w1.B, w1.H, w1.T, w1.D, w1.chunk, w1.topk) + 256,
                          dtype=torch.uint8, device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # larger than L2

        def fwd1():
            hsa.hsa_forward(Q1, K1, V1, L1, w1.topk, out=out1, sel_idx=idx1, sel_w=sw1, workspace=ws1)

        def fwd1_cold():  # the workload fits in L2: flush it between steps, outside the forward's kernels
            flush.zero_()
            fwd1()

        steps1 = max(args.steps, 50)
        ms1_fwd = timed_after(flush.zero_, fwd1, steps1, args.warmup, world)
        clean(ws1)
        prof1 = kernel_profile(fwd1_cold, steps1)
        sf1, af1, pairs1 = forward_work(w1, idx1)
        entry1 = {
            "workload": w1.name, "config": forward_config(w1, world) | {"l2": "L2 flushed before each step (256 MB "
                                                                               "write, outside the per-step events)"},
            "tokens_per_s": round(whole_job_rate(w1.B * w1.T, world, ms1_fwd), 1), "ms_per_step": round(ms1_fwd, 5),
            "steps": steps1,
            "roofline": roofline_entry("chunk_attn", prof1, af1, "TFLOP/s", tensor_peak, "tensor", tensor_kind),
            "roofline_score_topk": roofline_entry("score_topk", prof1, sf1, "TFLOP/s", tensor_peak, "tensor",
                                                  tensor_kind),
            "bound": "launch latency: 2.1 GFLOP over 6 kernels is a few microseconds of tensor work",
            "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof1.items()},
        }
        if rank == 0 and world == 1 and not args.skip_cpu:
            Q1h, K1h, V1h, L1h = (x.float().cpu().numpy() for x in (Q1, K1, V1, L1))
            v1, rows1, spent1 = oracle_forward_sample(w1, Q1h, K1h, V1h, L1h, target_s=3.0)
            entry1["cpu_baseline"] = {"value": round(v1, 2), "unit": "tokens/s", "cores": host_cores(),
                                      "kind": "oracle",
                                      "sample": f"{rows1} token-head rows drawn uniformly from the 4K workload, "
                                                f"fp64 oracle with OpenMP, {spent1:.1f} s wall"}
        # forward + backward at head dim 64 on the same shape (the tcgen05 backward's head-dim-64 form)
        dO1 = inputs.upstream_grad(w1.B, w1.H, w1.T, w1.D, w1.seed + rank, device=dev)
        bws1 = torch.empty(hsa.hsa_backward_workspace_size(w1.B, w1.H, w1.T, w1.D, 64, w1.topk) + 256,
                           dtype=torch.uint8, device=dev)
        g1 = tuple(torch.empty(x.shape, dtype=torch.float32, device=dev) for x in (Q1, K1, V1, L1))

        def fwdbwd1():
            fwd1()
            hsa.hsa_backward(Q1, K1, V1, L1, out1, dO1, idx1, sw1, grads=g1, workspace=bws1)

        fb_ms = timed_after(flush.zero_, fwdbwd1, steps1, args.warmup, world)
        clean(ws1, bws1)
        prof_fb1 = kernel_profile(lambda: (flush.zero_(), fwdbwd1()), steps1)
        entry1["fwdbwd_d64"] = {
            "ms_per_step": round(fb_ms, 5), "tokens_per_s": round(whole_job_rate(w1.B * w1.T, world, fb_ms), 1),
            "roofline": roofline_entry("chunk_bwd", prof_fb1, 10.0 * 64 * w1.D * pairs1, "TFLOP/s", tensor_peak,
                                       "tensor", tensor_kind),
            "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof_fb1.items()}}
        extra["fwd_4k"] = entry1
        del Q1, K1, V1, L1, out1, idx1, sw1, ws1, flush, dO1, bws1, g1
        torch.cuda.empty_cache()

    # ---------------- decode, 1M-token caches, batch 16 ----------------
    if not args.skip_decode and not args.grouped_decode_only and not args.skip_decode_1m:
        wm = inputs.WORKLOADS["decode_1m_b16_h8_d128_k16"]
        extra["decode_1m"] = decode_entry(hsa, inputs, wm, dev, max(args.steps, 50), args.warmup, world, peaks,
                                          peak_kind, cpu=rank == 0 and world == 1 and not args.skip_cpu)
        torch.cuda.empty_cache()

    # ---------------- decode, 16M-token cache ----------------
    if not args.skip_decode:
        wd = inputs.WORKLOADS["decode_16m_b1_h8_d128_k32"]
        if args.decode_cache_len:
            import dataclasses

            wd = dataclasses.replace(wd, name=f"decode_{args.decode_cache_len}_b1_h8_d128_k32",
                                     cache_len=args.decode_cache_len)
        dsteps = max(args.steps, 50)
        n = wd.cache_len // 64
        if not args.grouped_decode_only:
            q, Kc, Vc, Lc, lens, _ = inputs.workload_inputs(wd, device=dev)
            dout_ = torch.empty_like(q)
            didx = torch.empty((wd.B, wd.H, wd.topk), dtype=torch.int32, device=dev)
            dw = torch.empty((wd.B, wd.H, wd.topk), dtype=torch.float32, device=dev)
            dws = torch.empty(hsa.hsa_decode_workspace_size(wd.B, wd.H, wd.cache_len, wd.D, 64, wd.topk) + 256,
                              dtype=torch.uint8, device=dev)

            def dec():
                hsa.hsa_decode(q, Kc, Vc, Lc, lens, wd.topk, out=dout_, sel_idx=didx, sel_w=dw, workspace=dws)

            dms = timed(dec, dsteps, args.warmup, world) / dsteps
            clean(dws)
            prof_dec = kernel_profile(dec, dsteps)
            scan_bytes = wd.B * wd.H * (n * wd.D * 2 + wd.D * 2)
            gather_bytes = wd.B * wd.H * wd.topk * 2 * 64 * wd.D * 2
            hbm_peak = peaks["hbm_gbs"]
            extra["decode_16m"] = {
                "workload": wd.name, "us_per_token": round(dms * 1e3 / wd.B, 3), "ms_per_step": round(dms, 5),
                "steps": dsteps,
                "roofline": roofline_entry("decode_scan", prof_dec, scan_bytes, "GB/s", hbm_peak, "hbm",
                                           f"{peak_kind} hbm_gbs", TRAFFIC_BYTES.get((wd.name, "decode_scan"))),
                "step_vs_hbm": {"algorithmic_bytes": scan_bytes + gather_bytes,
                                "achieved_GBs": round((scan_bytes + gather_bytes) / (dms / 1e3) / 1e9, 1),
                                "frac": round((scan_bytes + gather_bytes) / (dms / 1e3) / 1e9 / hbm_peak, 4),
                                "target": f"70% of measured HBM: <= "
                                          f"{(scan_bytes + gather_bytes) / (0.7 * hbm_peak * 1e3):.1f} us per step"},
                "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof_dec.items()},
            }
            if rank == 0 and world == 1 and not args.skip_cpu:
                spent = oracle_decode_sample(q, Kc, Vc, Lc, lens, wd.topk, [(0, 0)])
                extra["decode_16m"]["cpu_baseline"] = {
                    "value": round(spent * wd.H * 1e6, 1), "unit": "us/token", "cores": host_cores(), "kind": "oracle",
                    "sample": f"one (b, h) row of the workload (fp64 oracle: all {n} landmarks scored, then the "
                              f"selected chunks attended), {spent:.2f} s, times {wd.H} heads per token"}
            if not args.skip_options:  # 4 query tokens per sequence in one step (e.g. verifying 4 drafted tokens)
                Tq = 4
                mq = inputs.forward_inputs(wd.B, wd.H, Tq, wd.D, wd.seed + 5, device=dev)[0]
                mout = torch.empty_like(mq)
                midx = torch.empty((wd.B, wd.H, Tq, wd.topk), dtype=torch.int32, device=dev)
                mw = torch.empty((wd.B, wd.H, Tq, wd.topk), dtype=torch.float32, device=dev)
                mbytes = hsa.hsa_decode_ex_workspace_size(wd.B, wd.H, wd.H, wd.cache_len, wd.D, 64, wd.topk, 0, Tq)
                mws = torch.empty(mbytes + 256, dtype=torch.uint8, device=dev)

                def dec_multi():
                    hsa.hsa_decode(mq, Kc, Vc, Lc, lens, wd.topk, out=mout, sel_idx=midx, sel_w=mw, workspace=mws)

                mms = timed(dec_multi, dsteps, args.warmup, world) / dsteps
                clean(mws)
                prof_m = kernel_profile(dec_multi, dsteps)
                extra["decode_16m"]["multi_token_4"] = {
                    "shape": f"B{wd.B} H{wd.H} Tq{Tq} cache {wd.cache_len} D{wd.D} topk{wd.topk}",
                    "us_per_step": round(mms * 1e3, 3), "us_per_token": round(mms * 1e3 / (wd.B * Tq), 3),
                    "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof_m.items()}}
                del mq, mout, mws
            del q, Kc, Vc, Lc, dws
            torch.cuda.empty_cache()
        if not args.skip_options or args.grouped_decode_only:  # 16 query heads on one key/value head
            Hg = 16
            gq = inputs.decode_inputs(wd.B, Hg, 0, wd.D, seed=wd.seed + 3, Tmax=64, device=dev)[0]
            _, gKc, gVc, gLc, glens, _ = inputs.decode_inputs(wd.B, 1, wd.cache_len, wd.D, seed=wd.seed + 4,
                                                              device=dev)
            gout_ = torch.empty_like(gq)
            gidx_ = torch.empty((wd.B, Hg, wd.topk), dtype=torch.int32, device=dev)
            gw_ = torch.empty((wd.B, Hg, wd.topk), dtype=torch.float32, device=dev)
            gdws = torch.empty(hsa.hsa_decode_ex_workspace_size(wd.B, Hg, 1, wd.cache_len, wd.D, 64, wd.topk, 0) + 256,
                               dtype=torch.uint8, device=dev)

            def dec_gqa():
                hsa.hsa_decode(gq, gKc, gVc, gLc, glens, wd.topk, out=gout_, sel_idx=gidx_, sel_w=gw_, workspace=gdws)

            gms = timed(dec_gqa, dsteps, args.warmup, world) / dsteps
            clean(gdws)
            prof_gd = kernel_profile(dec_gqa, dsteps)
            lm_bytes = wd.B * (n * wd.D * 2)  # one landmark head, read once from HBM at best
            extra.setdefault("decode_16m", {})["grouped_heads_16to1"] = {
                "shape": f"B{wd.B} H{Hg} Hkv1 cache {wd.cache_len} D{wd.D} topk{wd.topk}",
                "us_per_token": round(gms * 1e3 / wd.B, 3),
                "landmark_bytes": lm_bytes,
                "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof_gd.items()}}
            del gq, gKc, gVc, gLc, gdws
            torch.cuda.empty_cache()

    # ---------------- forward + backward, 64K ----------------
    if not args.skip_backward:
        wb = inputs.WORKLOADS["fwdbwd_t64k_h8_d128_k16"]
        bQ, bK, bV, bL, bdO = inputs.workload_inputs(wb, device=dev)
        bout = torch.empty_like(bQ)
        bidx = torch.empty((wb.B, wb.H, wb.T, wb.topk), dtype=torch.int32, device=dev)
        bw = torch.empty((wb.B, wb.H, wb.T, wb.topk), dtype=torch.float32, device=dev)
        fws = torch.empty(hsa.hsa_forward_workspace_size(wb.B, wb.H, wb.T, wb.D, 64, wb.topk) + 256,
                          dtype=torch.uint8, device=dev)
        bws = torch.empty(hsa.hsa_backward_workspace_size(wb.B, wb.H, wb.T, wb.D, 64, wb.topk) + 256,
                          dtype=torch.uint8, device=dev)
        grads = (torch.empty(bQ.shape, dtype=torch.float32, device=dev),
                 torch.empty(bQ.shape, dtype=torch.float32, device=dev),
                 torch.empty(bQ.shape, dtype=torch.float32, device=dev),
                 torch.empty(bL.shape, dtype=torch.float32, device=dev))

        def fwdbwd():
            hsa.hsa_forward(bQ, bK, bV, bL, wb.topk, out=bout, sel_idx=bidx, sel_w=bw, workspace=fws)
            hsa.hsa_backward(bQ, bK, bV, bL, bout, bdO, bidx, bw, grads=grads, workspace=bws)

        bsteps = max(3, args.steps // 2)
        bms = timed(fwdbwd, bsteps, args.warmup, world) / bsteps
        clean(fws, bws)
        prof_b = kernel_profile(fwdbwd, bsteps)
        sf, af, bpairs = forward_work(wb, bidx)
        bwd_flops = 10.0 * 64 * wb.D * bpairs
        extra["fwdbwd_64k"] = {
            "workload": wb.name, "tokens_per_s": round(wb.B * wb.T / (bms / 1e3), 1), "ms_per_step": round(bms, 4),
            "steps": bsteps,
            "roofline": roofline_entry("chunk_bwd", prof_b, bwd_flops, "TFLOP/s", tensor_peak, "tensor",
                                       tensor_kind, TRAFFIC_BYTES.get((wb.name, "chunk_bwd"))),
            "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof_b.items()},
        }
        if not args.skip_options:  # the same step with query-key normalisation
            fws_n = torch.empty(hsa.hsa_forward_ex_workspace_size(wb.B, wb.H, wb.H, wb.T, wb.D, 64, wb.topk,
                                                                  hsa.HSA_QK_NORM) + 256, dtype=torch.uint8,
                                device=dev)
            bws_n = torch.empty(hsa.hsa_backward_ex_workspace_size(wb.B, wb.H, wb.H, wb.T, wb.D, 64, wb.topk,
                                                                   hsa.HSA_QK_NORM) + 256, dtype=torch.uint8,
                                device=dev)

            def fwdbwd_norm():
                hsa.hsa_forward(bQ, bK, bV, bL, wb.topk, out=bout, sel_idx=bidx, sel_w=bw, workspace=fws_n,
                                qk_norm=True)
                hsa.hsa_backward(bQ, bK, bV, bL, bout, bdO, bidx, bw, grads=grads, workspace=bws_n, qk_norm=True)

            nms = timed(fwdbwd_norm, bsteps, args.warmup, world) / bsteps
            clean(fws_n, bws_n)
            prof_bn = kernel_profile(fwdbwd_norm, bsteps)
            extra["fwdbwd_64k"]["qk_norm"] = {
                "ms_per_step": round(nms, 4), "vs_plain": round(nms / bms, 4),
                "kernels": {k: {"launches": c, "avg_us": round(t / c * 1e3, 2)} for k, (c, t) in prof_bn.items()}}
            del fws_n, bws_n
        del bQ, bK, bV, bL, bdO, fws, bws, grads
        torch.cuda.empty_cache()
    clk = clocks.stop()

    # ---------------- CPU oracle baseline (rank 0, one GPU) ----------------
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu and not args.skip_prefill:
        Qh, Kh, Vh, Lh = (x.float().cpu().numpy() for x in (Q, K, V, L))
        v, rows_done, spent = oracle_forward_sample(w, Qh, Kh, Vh, Lh, target_s=10.0)
        cpu = {"value": round(v, 2), "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
               "sample": f"{rows_done} token-head rows drawn uniformly from the same 32K workload, fp64 oracle "
                         f"with OpenMP, {spent:.1f} s wall"}

    launches = 0 if args.skip_prefill else args.steps * KERNELS_PER_FORWARD
    if rank == 0:
        line = {
            "metric": "HSA prefill tokens/s (B2 T32768 H8 D128 chunk64 topk16)",
            "value": round(value, 1) if value else None, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4) if ms_per_step else None,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": forward_config(w, world),
            "roofline": roof,
            "roofline_score_topk": roof_score,
            "roofline_combine": roof_combine,
            "kernels": breakdown,
            "gpu_launches": launches,
            "e2e": e2e,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        line.update(extra)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    del np


if __name__ == "__main__":
    main()
