"""Benchmark of the block-FP8 linear hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input
on the headline layer (M=512 tokens, K=5120, N=25600, the largest linear of a
32B-class decoder):
  quantize_weight (BF16 W -> E4M3 codes + scales), dequantize (-> BF16),
  linear_w8a16 (x BF16 . dequant(W)^T) and linear_w8a8 (x quantized per
  1x128 K-group, then the FP8 GEMM).
`value` = FLOPs of the step's two linears (2 * 2MNK) / device time of the
whole step, summed over ranks / max over ranks; the step's time includes the
converter and the dequantizer, so `value` is no single call's throughput --
the per-call times, TFLOP/s, weight GB/s and roofline fractions in `calls`
carry that. `targets` times the two linears alone on the large-token and the
small-token (weight-streaming) shapes, each call with a clean L2, and gives
their fractions of the measured and of the datasheet peaks with the clocks
seen meanwhile. L2 is flushed between
steps outside the step's CUDA events: a 512 MiB memset, then a 256 MiB read,
so the step starts with no input in L2 and no dirty flush lines to write back.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU (torchrun): replicas only -- each rank runs its own copy of the
layer; there is no data-path collective (NCCL is used only for the barrier
and the max-over-ranks timing reduction).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "block-FP8 linear TFLOP/s and weight-stream GB/s (M=512,K=5120,N=25600)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0   # nominal dense FP8 / BF16 tensor ratio (4.5 / 2.25 PFLOP/s)
# B200 datasheet figures (dense): HBM3e bandwidth, BF16 and FP8 tensor throughput
DATASHEET = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0, "fp8_tflops": 4500.0}
ROTATE_BYTES = 2 * 126 * 10**6   # back-to-back timings rotate weights over twice the L2
FLUSH_BYTES = 512 << 20
FLUSH_READ_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="fp8blk", choices=["fp8blk", "reference"])
    ap.add_argument("--workload", default="linear_m512_k5120_n25600")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--stack", type=int, default=0,
                    help="instead of the step: stream the FP8 weights of this many 32B-shaped "
                         "layers from pinned host memory (one GPU)")
    ap.add_argument("--decode", type=int, default=0,
                    help="instead of the step: one 32B-shaped layer's four linears at this many "
                         "tokens, as separate calls, as one sequence, and as a CUDA graph of it")
    ap.add_argument("--stack-mode", type=int, default=0, choices=[0, 1], help="0 W8A16, 1 W8A8")
    ap.add_argument("--stack-m", type=int, default=512)
    ap.add_argument("--stack-slots", type=int, default=2)
    ap.add_argument("--call", default="", choices=["", "w8a16", "w8a8", "quantize_weight",
                                                   "dequantize"],
                    help="instead of the step: time one call on --shape (used for profiling)")
    ap.add_argument("--shape", default="512,5120,25600", help="M,K,N for --call")
    ap.add_argument("--reps", type=int, default=10, help="timed calls for --call")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip the per-call timings of the large- and small-token linears")
    ap.add_argument("--no-ab", action="store_true",
                    help="skip the A/B timings of the library BF16 route and shared act quantization")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        loaded = [r for r in rows if r[2] > 250.0] or rows
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(1, 5) if r[3][i] == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(loaded),
                "sm_mhz_all_samples": statistics.median(r[0] for r in rows),
                "samples_all": len(rows), "power_w_max": max(r[2] for r in rows)}


# --------------------------------------------------------------- oracle arm
def oracle_sample_step(wl, wb, xb, n_rows):
    """The step on the first n_rows output rows (n_rows % 128 == 0): every
    stage's work is proportional to N, so this is the step scaled by n_rows/N."""
    import oracle
    w_s = wb[:n_rows]
    q, s = oracle.quantize_weight(w_s)
    oracle.dequantize(q, s)
    oracle.linear_w8a16(xb, q, s, n_rows, wl.K)
    qx, sx = oracle.act_quant(xb)
    oracle.linear_w8a8(qx, sx, q, s, n_rows, wl.K)
    return 4.0 * wl.M * n_rows * wl.K


def calibrate_oracle_rows(wl, wb, xb, seconds: float) -> int:
    """Rows (a multiple of 128) for a sample step of about `seconds`: the
    fixed cost (threads, the activation stage) and the cost per row are
    fitted from two trials, 128 and 512 rows."""
    nb = -(-wl.N // 128)
    times = []
    for rows in (128, min(512, 128 * nb)):
        t = time.perf_counter()
        oracle_sample_step(wl, wb, xb, rows)
        times.append((rows, time.perf_counter() - t))
    (r1, t1), (r2, t2) = times
    per_row = (t2 - t1) / (r2 - r1) if r2 > r1 and t2 > t1 else t2 / r2
    fixed = max(0.0, t1 - per_row * r1)
    blocks = int((seconds - fixed) / max(per_row * 128, 1e-9))
    return 128 * max(1, min(nb, blocks))


def run_oracle(wl, wb, xb, seconds: float):
    import oracle
    rows = calibrate_oracle_rows(wl, wb, xb, seconds)
    t = time.perf_counter()
    flops = oracle_sample_step(wl, wb, xb, rows)
    dt = time.perf_counter() - t
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": f"the step on {rows} of {wl.N} output rows (all M={wl.M} tokens, "
                      f"K={wl.K}): {dt:.1f} s of CPU work"}


def reference_arm(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from block_scaled_fp8_fp8blk_b200 import synth
    wb = synth.bf16_bits(wl.weight_bf16())
    xb = synth.bf16_bits(wl.x_bf16())
    per_step = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    rows = calibrate_oracle_rows(wl, wb, xb, per_step)
    for _ in range(args.warmup):
        oracle_sample_step(wl, wb, xb, rows)
    times = []
    flops = 0.0
    for _ in range(args.steps):
        t = time.perf_counter()
        flops = oracle_sample_step(wl, wb, xb, rows)
        times.append(time.perf_counter() - t)
    total = sum(times)
    value = flops * args.steps / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "M": wl.M, "K": wl.K, "N": wl.N,
                   "sample_rows": rows, "parallelism": "single process, CPU threads"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.threads(),
                         "kind": "oracle",
                         "sample": f"each step: the step on {rows} of {wl.N} output rows"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------- replicas (N > 1 host logic)
def replica_workload(wl, rank: int):
    """The layer rank `rank` runs: its own seeded copy (replicas, no exchange)."""
    from dataclasses import replace
    return replace(wl, seed=wl.seed + rank)


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest `value` over all ranks (every rank calls this, in the same
    order); the job's time is the slowest rank's."""
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ GPU arm
def traffic_for(kernel_file: str, key: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    source is unchanged since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(key)
        src = os.path.join(ROOT, "block_scaled_fp8_fp8blk_b200", "csrc", kernel_file)
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()[:16]
        if rec and rec.get("source_sha256_16") == digest:
            return rec.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


def measure_targets(fb, dev, peaks, flush_l2, clock_sampler):
    """Per-call device times of the two linears on the large-token shapes
    (M = 4096, 16384; K = 5120, N = 25600: tensor-bound) and on the
    weight-streaming sweep (M = 1, 16, 64 on the decoder's QKV, o_proj,
    gate_up and down shapes: HBM-bound), each call alone with L2 flushed
    before it (median over repetitions, CUDA events on the launching stream).
    Fractions are given against the measured peaks (copy bandwidth, cuBLAS
    BF16; FP8 = 2 x BF16) and against the datasheet figures."""
    import torch
    g = torch.Generator(device=dev).manual_seed(123)

    def weights(N, K):
        ldw = -(-K // 8) * 8
        w = (torch.randn(N, ldw, device=dev, generator=g) * 0.02).to(torch.bfloat16)[:, :K]
        q, s = fb.quantize_weight(w)
        del w
        return q, s

    def activations(M, K):
        x = torch.randn(M, K, device=dev, generator=g)
        ch = torch.randperm(K, device=dev, generator=g)[:max(1, K // 100)]
        x[:, ch] *= 20.0
        return x.to(torch.bfloat16)

    def timed(fn, reps):
        fn()
        ts = []
        for _ in range(reps):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(); fn(); b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        return 1e3 * statistics.median(a.elapsed_time(b) for a, b in ts)

    def back_to_back(call, copies, rounds=4):
        """Per-call time of calls run back to back from a CUDA graph, each on
        the next weight copy in turn (a pass over the copies is twice the L2,
        so every call streams its weight from HBM): the decode-time regime,
        where one linear follows another and launch latency overlaps the
        kernel before."""
        cs = torch.cuda.Stream()
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs):
            for qq, ss in copies:
                call(qq, ss)
        torch.cuda.current_stream().wait_stream(cs)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cs):
            for _ in range(rounds):
                for qq, ss in copies:
                    call(qq, ss)
        graph.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(3):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(); graph.replay(); b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        del graph
        return 1e3 * statistics.median(a.elapsed_time(b) for a, b in ts) / (rounds * len(copies))

    out = {"large_m": [], "small_m": []}
    # The weight-streaming sweep runs first, after a short idle: the
    # tensor-bound calls below draw enough power to lower the clocks for a
    # while, which short latency-bound calls would feel.
    torch.cuda.synchronize()
    time.sleep(1.0)
    clock_sampler.start()
    time.sleep(0.15)
    shapes = [("qkv", 5120, 10240), ("o_proj", 8192, 5120), ("gate_up", 5120, 51200),
              ("down", 25600, 5120)]
    for name, K, N in shapes:
        # enough copies of the weight that one pass over them is twice the L2
        copies = [weights(N, K)]
        wbytes = N * K + 4 * copies[0][1].numel()
        while len(copies) < max(2, -(-ROTATE_BYTES // wbytes)):
            copies.append(weights(N, K))
        q, s = copies[0]
        for M in (1, 16, 64):
            x = activations(M, K)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws16 = torch.empty(max(1, fb.workspace_size(0, M, N, K)), dtype=torch.uint8, device=dev)
            ws8 = torch.empty(max(1, fb.workspace_size(1, M, N, K)), dtype=torch.uint8, device=dev)
            for mode in ("w8a16", "w8a8"):
                f = fb.linear_w8a16 if mode == "w8a16" else fb.linear_w8a8
                ws = ws16 if mode == "w8a16" else ws8
                us = timed(lambda: f(x, q, s, out=y, workspace=ws), 20)
                us_b2b = back_to_back(lambda qq, ss: f(x, qq, ss, out=y, workspace=ws), copies)
                gbs, gbs_b2b = wbytes / (us * 1e-6) / 1e9, wbytes / (us_b2b * 1e-6) / 1e9
                out["small_m"].append({"mode": mode, "layer": name, "M": M, "K": K, "N": N,
                                       "us": us, "weight_gbs": gbs,
                                       "frac_measured": gbs / peaks["hbm_gbs"],
                                       "frac_datasheet": gbs / DATASHEET["hbm_gbs"],
                                       "us_back_to_back": us_b2b, "weight_gbs_back_to_back": gbs_b2b,
                                       "frac_measured_back_to_back": gbs_b2b / peaks["hbm_gbs"],
                                       "frac_datasheet_back_to_back": gbs_b2b / DATASHEET["hbm_gbs"],
                                       "weight_copies": len(copies)})
            del x, y, ws16, ws8
        del q, s, copies
    out["clocks_small_m"] = clock_sampler.stop()
    clock_sampler.start()
    time.sleep(0.15)
    K, N = 5120, 25600
    q, s = weights(N, K)
    for M in (4096, 16384):
        x = activations(M, K)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws8 = torch.empty(max(1, fb.workspace_size(1, M, N, K)), dtype=torch.uint8, device=dev)
        reps = 10 if M <= 4096 else 5
        fl = 2.0 * M * N * K
        for mode in ("w8a8", "w8a16"):
            if mode == "w8a8":
                us = timed(lambda: fb.linear_w8a8(x, q, s, out=y, workspace=ws8), reps)
                pk, ds = FP8_OVER_BF16 * peaks["bf16_tflops"], DATASHEET["fp8_tflops"]
            else:
                us = timed(lambda: fb.linear_w8a16(x, q, s, out=y), reps)
                pk, ds = peaks["bf16_tflops"], DATASHEET["bf16_tflops"]
            tf = fl / (us * 1e-6) / 1e12
            out["large_m"].append({"mode": mode, "M": M, "K": K, "N": N, "us": us, "tflops": tf,
                                   "frac_measured": tf / pk, "frac_datasheet": tf / ds,
                                   "peak_measured": pk, "peak_datasheet": ds})
        del x, y, ws8
    # A library FP8 GEMM on the same shapes and on 8192^3 (torch._scaled_mm:
    # E4M3 operands, one FP32 scale per tensor, BF16 out, timed like the
    # calls above): this box's measured FP8 tensor rate for a GEMM without
    # block scales, next to the W8A8 linears.
    out["library_fp8"] = []
    try:
        one = torch.ones((), device=dev, dtype=torch.float32)
        for M, Kl, Nl in ((4096, K, N), (16384, K, N), (8192, 8192, 8192)):
            a8 = torch.randn(M, Kl, device=dev, generator=g).to(torch.float8_e4m3fn)
            b8 = torch.randn(Nl, Kl, device=dev, generator=g).to(torch.float8_e4m3fn)
            us = timed(lambda: torch._scaled_mm(a8, b8.t(), scale_a=one, scale_b=one,
                                                out_dtype=torch.bfloat16), 5 if M > 8192 else 10)
            tf = 2.0 * M * Nl * Kl / (us * 1e-6) / 1e12
            rec = {"M": M, "K": Kl, "N": Nl, "us": us, "tflops": tf,
                   "frac_of_2x_bf16_burst": tf / (FP8_OVER_BF16 * peaks["bf16_tflops"])}
            ours = [r for r in out["large_m"] if r["mode"] == "w8a8" and r["M"] == M
                    and (Kl, Nl) == (K, N)]
            if ours:
                rec["w8a8_linear_over_library"] = ours[0]["tflops"] / tf
            out["library_fp8"].append(rec)
            del a8, b8
    except (RuntimeError, TypeError) as e:
        out["library_fp8"] = {"unavailable": str(e).splitlines()[0][:200]}
    out["clocks_large_m"] = clock_sampler.stop()
    # Sustained: W8A8 back to back for about a second per shape (the regime
    # in which the sustained BF16 peak was measured: a seconds-long loop under
    # the power cap), with its own clock record.
    out["w8a8_sustained"] = []
    for M in (4096, 16384):
        x = activations(M, K)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws8 = torch.empty(max(1, fb.workspace_size(1, M, N, K)), dtype=torch.uint8, device=dev)
        run = lambda: fb.linear_w8a8(x, q, s, out=y, workspace=ws8)
        run()
        torch.cuda.synchronize()
        calls = max(20, int(1.0 / (out["large_m"][0 if M == 4096 else 2]["us"] * 1e-6)))
        clock_sampler.start()
        time.sleep(0.15)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(calls):
            run()
        b.record()
        torch.cuda.synchronize()
        clk = clock_sampler.stop()
        us = 1e3 * a.elapsed_time(b) / calls
        tf = 2.0 * M * N * K / (us * 1e-6) / 1e12
        pk = FP8_OVER_BF16 * peaks["bf16_tflops_sustained"]
        out["w8a8_sustained"].append({"M": M, "calls": calls, "us_per_call": us, "tflops": tf,
                                      "peak_sustained": pk, "frac_sustained": tf / pk,
                                      "frac_burst": tf / (FP8_OVER_BF16 * peaks["bf16_tflops"]),
                                      "clocks": clk})
        del x, y, ws8
    del q, s
    torch.cuda.synchronize()
    assert fb.read_device_error() == 0
    w8a8_large = [r for r in out["large_m"] if r["mode"] == "w8a8"]
    w8a16_small = [r for r in out["small_m"] if r["mode"] == "w8a16"]
    out["north_star"] = {
        "w8a16_m_le_64_min_frac_measured_back_to_back": min(r["frac_measured_back_to_back"]
                                                            for r in w8a16_small),
        "w8a8_m_ge_4096_min_frac_measured": min(r["frac_measured"] for r in w8a8_large),
        "w8a8_m_ge_4096_min_frac_datasheet": min(r["frac_datasheet"] for r in w8a8_large),
        "w8a8_m_ge_4096_min_frac_sustained_back_to_back": min(r["frac_sustained"]
                                                              for r in out["w8a8_sustained"]),
        "w8a8_target": 0.60,
        "w8a16_m_le_64_min_frac_measured": min(r["frac_measured"] for r in w8a16_small),
        "w8a16_m_le_64_min_frac_datasheet": min(r["frac_datasheet"] for r in w8a16_small),
        "w8a16_target": 0.70,
    }
    out["timing"] = ("per call: median of 10 (M=4096), 5 (M=16384) or 20 (small M) calls, "
                     "each alone with L2 flushed before it; back to back (small M): a CUDA "
                     "graph of 4 rounds over weight copies totalling twice the L2, per call; "
                     "synthetic seeded weights (N(0, 0.02^2) BF16, converted by the library) "
                     "and activations (N(0,1), 1% of channels x20)")
    return out


# Linears of one decoder layer of the 32B class the pages' encoder belongs to
# (hidden 5120, 64 query heads x 128, 8 KV heads, MLP 25600): (K, N).
STACK_LAYER = [("qkv", 5120, 10240), ("o_proj", 8192, 5120), ("gate_up", 5120, 51200),
               ("down", 25600, 5120)]


def stack_arm(args):
    """Layerwise FP8 weight streaming: every layer's codes and scales in their
    own pinned host buffers, run through a ring of device slots
    (fp8blk_streamed_linears), against the same linears on resident weights
    and against the copies alone. One GPU; synthetic codes (no NaN)."""
    import torch
    import block_scaled_fp8_fp8blk_b200 as fb
    L, M, mode, nslots = args.stack, args.stack_m, args.stack_mode, args.stack_slots
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev).manual_seed(5)
    host, dev_w, xs, ys = [], [], {}, {}
    slot_bytes, ws_need, layer_bytes = 0, 0, 0
    for name, K, N in STACK_LAYER:
        ldq = -(-K // 16) * 16
        slot_bytes = max(slot_bytes, fb.stream_slot_bytes(N, K, ldq))
        ws_need = max(ws_need, fb.workspace_size(mode, M, N, K))
        layer_bytes += N * ldq + 4 * (-(-N // 128)) * (-(-K // 128))
        xs[name] = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        ys[name] = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    slot_bytes = -(-slot_bytes // 256) * 256
    for layer in range(L):
        for name, K, N in STACK_LAYER:
            ldq = -(-K // 16) * 16
            # codes 0x00..0x7E with a random sign: every finite E4M3 value
            q = (torch.randint(0, 0x7F, (N, ldq), device=dev, generator=g, dtype=torch.uint8)
                 | (torch.randint(0, 2, (N, ldq), device=dev, generator=g, dtype=torch.uint8) << 7))
            s = torch.rand(-(-N // 128), -(-K // 128), device=dev, generator=g) * 1e-3 + 1e-4
            qh = torch.empty((N, ldq), dtype=torch.uint8, pin_memory=True)
            qh.copy_(q)
            sh = torch.empty(s.shape, dtype=torch.float32, pin_memory=True)
            sh.copy_(s)
            host.append((name, qh[:, :K], sh))
            dev_w.append((q[:, :K], s))
    torch.cuda.synchronize()
    jobs = [(mode, qh, sh, xs[name], ys[name]) for name, qh, sh in host]
    slots = torch.empty(nslots * slot_bytes, dtype=torch.uint8, device=dev)
    ws = torch.empty(max(1, ws_need), dtype=torch.uint8, device=dev)
    compute, copy = torch.cuda.Stream(), torch.cuda.Stream()
    events = [torch.cuda.Event() for _ in range(2 * nslots)]
    f = fb.linear_w8a16 if mode == 0 else fb.linear_w8a8

    def timed(run, reps):
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(compute)
            copy.wait_event(a)
            run()
            compute.wait_stream(copy)
            b.record(compute)
            ts.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ts)

    def streamed():
        fb.streamed_linears(jobs, slots, slot_bytes, nslots, ws, compute, copy, events)

    def resident():
        with torch.cuda.stream(compute):
            for (name, qh, sh), (q, s) in zip(host, dev_w):
                f(xs[name], q, s, out=ys[name], workspace=ws)

    def copies_only():
        with torch.cuda.stream(copy):
            for i, (name, qh, sh) in enumerate(host):
                k = i % nslots
                slots[k * slot_bytes:k * slot_bytes + qh.shape[0] * qh.stride(0)].copy_(
                    qh.as_strided((qh.shape[0] * qh.stride(0),), (1,)), non_blocking=True)

    reps = max(3, min(args.steps, 10))
    for run in (streamed, resident, copies_only):
        timed(run, 1)
    t_stream = timed(streamed, reps) / L
    t_res = timed(resident, reps) / L
    t_copy = timed(copies_only, reps) / L
    assert fb.read_device_error() == 0
    h2d = layer_bytes / (t_stream * 1e-3) / 1e9
    line = {
        "metric": "streamed FP8 linear stack: ms per layer, weights from pinned host memory",
        "value": t_stream, "unit": "ms/layer", "higher_is_better": False, "n_gpus": 1,
        "steps": reps, "data": "synthetic (random finite E4M3 codes and scales)",
        "dtype": "e4m3 weights, bf16 activations" if mode == 0 else "e4m3 weights and activations",
        "config": {"workload": f"stack32b_m{M}_L{L}", "layers": L, "linears_per_layer": 4,
                   "shapes_KN": [[k, n] for _, k, n in STACK_LAYER], "M": M,
                   "mode": "w8a16" if mode == 0 else "w8a8", "slots": nslots},
        "fp8_bytes_per_layer": layer_bytes,
        "h2d_gbs_streamed": h2d,
        "copy_only_ms_per_layer": t_copy,
        "h2d_gbs_copy_only": layer_bytes / (t_copy * 1e-3) / 1e9,
        "resident_ms_per_layer": t_res,
        "overlap_efficiency": max(t_copy, t_res) / t_stream,
        "device_weight_bytes_streamed": nslots * slot_bytes,
        "device_weight_bytes_resident_fp8": L * layer_bytes,
        "device_weight_bytes_resident_bf16": L * sum(2 * k * n for _, k, n in STACK_LAYER),
        "bf16_stream_ms_per_layer_at_same_h2d": sum(2 * k * n for _, k, n in STACK_LAYER) / (h2d * 1e9) * 1e3,
    }
    print(json.dumps(line), flush=True)


def decode_arm(args):
    """One decoder layer of the 32B class at a small token count: the weight
    stream (487.7 MB of FP8 codes per layer) is the whole cost. Timed as four
    separate linear calls, as one fp8blk_linear_sequence (each GEMM streams
    its weights while the kernel before it ends), and as a CUDA graph of that
    sequence; L2 flushed (memset + read) before each timed layer."""
    import torch
    import block_scaled_fp8_fp8blk_b200 as fb
    M, mode = args.decode, args.stack_mode
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev).manual_seed(7)
    jobs, wbytes, ws_need = [], 0, 0
    for name, K, N in STACK_LAYER:
        ldq = -(-K // 16) * 16
        q = (torch.randint(0, 0x7F, (N, ldq), device=dev, generator=g, dtype=torch.uint8)
             | (torch.randint(0, 2, (N, ldq), device=dev, generator=g, dtype=torch.uint8) << 7))[:, :K]
        s = torch.rand(-(-N // 128), -(-K // 128), device=dev, generator=g) * 1e-3 + 1e-4
        x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        jobs.append((mode, x, q, s, y))
        wbytes += N * K + 4 * s.numel()
        ws_need = max(ws_need, fb.workspace_size(mode, M, N, K))
    ws = torch.empty(max(1, ws_need), dtype=torch.uint8, device=dev)
    f = fb.linear_w8a16 if mode == 0 else fb.linear_w8a8
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(FLUSH_READ_BYTES // 4, dtype=torch.float32, device=dev)

    def separate():
        for m_, x, q, s, y in jobs:
            f(x, q, s, out=y, workspace=ws)

    def sequence():
        fb.linear_sequence(jobs, workspace=ws)

    for run in (separate, sequence):
        run()
    torch.cuda.synchronize()
    cs = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cs):
        sequence()
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=cs):
            sequence()
    torch.cuda.synchronize()
    reps = max(5, min(args.steps, 50))

    def timed(run):
        ts = []
        for _ in range(reps):
            flush.zero_()
            flush_rd.sum()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(); run(); b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        return 1e3 * statistics.median(a.elapsed_time(b) for a, b in ts)

    res = {"separate_calls": timed(separate), "sequence": timed(sequence),
           "sequence_cuda_graph": timed(graph.replay)}
    assert fb.read_device_error() == 0
    peaks, peak_kind = load_peaks()
    line = {
        "metric": "decode layer: weight-stream GB/s (4 linears of a 32B-class layer, FP8 weights)",
        "value": wbytes / (res["sequence"] * 1e-6) / 1e9, "unit": "GB/s", "higher_is_better": True,
        "n_gpus": 1, "steps": reps, "data": "synthetic (random finite E4M3 codes and scales)",
        "dtype": "e4m3 weights, bf16 activations" if mode == 0 else "e4m3 weights and activations",
        "config": {"workload": f"decode_layer32b_m{M}", "M": M,
                   "shapes_KN": [[k, n] for _, k, n in STACK_LAYER],
                   "mode": "w8a16" if mode == 0 else "w8a8",
                   "l2": "flushed (memset + read) before each timed layer"},
        "weight_bytes_per_layer": wbytes,
        "us_per_layer": res,
        "weight_stream_gbs": {k: wbytes / (v * 1e-6) / 1e9 for k, v in res.items()},
        "hbm_frac": {k: wbytes / (v * 1e-6) / 1e9 / peaks["hbm_gbs"] for k, v in res.items()},
        "peak_gbs": peaks["hbm_gbs"], "peak_kind": peak_kind,
    }
    print(json.dumps(line), flush=True)


def call_arm(args):
    """One call on one shape, repeated: `--reps` timed calls after one
    untimed one, L2 flushed before each, CUDA events on the launching stream.
    Prints the median time and the call's throughput."""
    import torch
    import block_scaled_fp8_fp8blk_b200 as fb
    M, K, N = (int(v) for v in args.shape.split(","))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev).manual_seed(7)
    ldw = -(-K // 8) * 8
    w = (torch.randn(N, ldw, device=dev, generator=g) * 0.02).to(torch.bfloat16)[:, :K]
    q, s = fb.quantize_weight(w)
    x = torch.randn(M, ldw, device=dev, generator=g).to(torch.bfloat16)[:, :K]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    wd = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    mode = 0 if args.call == "w8a16" else 1
    ws = torch.empty(max(1, fb.workspace_size(mode, M, N, K)), dtype=torch.uint8, device=dev)
    run = {"w8a16": lambda: fb.linear_w8a16(x, q, s, out=y, workspace=ws),
           "w8a8": lambda: fb.linear_w8a8(x, q, s, out=y, workspace=ws),
           "quantize_weight": lambda: fb.quantize_weight(w, q=q, scale_inv=s),
           "dequantize": lambda: fb.dequantize(q, s, out=wd)}[args.call]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(FLUSH_READ_BYTES // 4, dtype=torch.float32, device=dev)
    run()
    ts = []
    for _ in range(args.reps):
        flush.zero_()
        flush_rd.sum()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(); run(); b.record()
        ts.append((a, b))
    torch.cuda.synchronize()
    assert fb.read_device_error() == 0
    us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in ts)
    NB, KB = -(-N // 128), -(-K // 128)
    line = {"call": args.call, "M": M, "K": K, "N": N, "reps": args.reps, "us": us,
            "weight_gbs": (N * K + 4 * NB * KB) / (us * 1e-6) / 1e9}
    if args.call in ("w8a16", "w8a8"):
        line["tflops"] = 2.0 * M * N * K / (us * 1e-6) / 1e12
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    from block_scaled_fp8_fp8blk_b200 import workloads
    wl = workloads.ALL[args.workload]
    if args.stack > 0:
        if int(os.environ.get("RANK", "0")) == 0:
            stack_arm(args)
        return
    if args.decode > 0:
        if int(os.environ.get("RANK", "0")) == 0:
            decode_arm(args)
        return
    if args.call:
        if int(os.environ.get("RANK", "0")) == 0:
            call_arm(args)
        return
    if args.impl == "reference":
        return reference_arm(args, wl)

    import torch
    import torch.distributed as dist

    import block_scaled_fp8_fp8blk_b200 as fb
    from block_scaled_fp8_fp8blk_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    M, K, N = wl.M, wl.K, wl.N
    # replicas: each rank its own seeded copy of the layer
    wl_r = replica_workload(wl, rank)
    w_h = wl_r.weight_bf16()
    x_h = wl_r.x_bf16()
    w = w_h.to(dev)
    x = x_h.to(dev)
    ldq = -(-K // 16) * 16
    q = torch.empty((N, ldq), dtype=torch.uint8, device=dev)[:, :K]
    s = torch.empty((-(-N // 128), -(-K // 128)), dtype=torch.float32, device=dev)
    wd = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    y16 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    y8 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws16 = torch.empty(max(1, fb.workspace_size(0, M, N, K)), dtype=torch.uint8, device=dev)
    ws8 = torch.empty(max(1, fb.workspace_size(1, M, N, K)), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(FLUSH_READ_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # Write more than L2 holds, then read another buffer twice its size:
        # the step starts with an L2 that holds none of its inputs and no
        # dirty lines of the flush to write back.
        flush.zero_()
        flush_rd.sum()

    def step(ev=None, w=w, x=x, y16=y16, y8=y8):
        if ev: ev[0].record()
        fb.quantize_weight(w, q=q, scale_inv=s)
        if ev: ev[1].record()
        fb.dequantize(q, s, out=wd)
        if ev: ev[2].record()
        fb.linear_w8a16(x, q, s, out=y16, workspace=ws16)
        if ev: ev[3].record()
        fb.linear_w8a8(x, q, s, out=y8, workspace=ws8)
        if ev: ev[4].record()

    for _ in range(max(3, args.warmup)):
        flush_l2()
        step()
    torch.cuda.synchronize()
    assert fb.read_device_error() == 0

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(visible.split(",")[local] if visible else str(local))
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.15)
    for i in range(args.steps):
        flush_l2()
        step(events[i])
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()

    calls = ["quantize_weight", "dequantize", "linear_w8a16", "linear_w8a8"]
    per_call = {c: [ev[j].elapsed_time(ev[j + 1]) for ev in events] for j, c in enumerate(calls)}
    step_ms_total = sum(ev[0].elapsed_time(ev[4]) for ev in events)
    step_ms_max = max_over_ranks(step_ms_total, world, dev) / args.steps

    flops_step = 2.0 * (2.0 * M * N * K)
    value = world * flops_step / (step_ms_max * 1e-3) / 1e12

    peaks, peak_kind = load_peaks()
    NB, KB = -(-N // 128), -(-K // 128)
    wbytes = N * K + 4 * NB * KB
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    call_stats = {}
    for c in calls:
        ms = statistics.mean(per_call[c])
        if c == "quantize_weight":
            alg = 2 * N * K + N * K + 4 * NB * KB
            ach = alg / (ms * 1e-3) / 1e9
            call_stats[c] = {"us": 1e3 * ms, "bound": "hbm", "achieved": ach, "unit": "GB/s",
                             "peak": peaks["hbm_gbs"], "frac": ach / peaks["hbm_gbs"],
                             "alg_bytes": alg}
        elif c == "dequantize":
            alg = N * K + 4 * NB * KB + 2 * N * K
            ach = alg / (ms * 1e-3) / 1e9
            call_stats[c] = {"us": 1e3 * ms, "bound": "hbm", "achieved": ach, "unit": "GB/s",
                             "peak": peaks["hbm_gbs"], "frac": ach / peaks["hbm_gbs"],
                             "alg_bytes": alg}
        else:
            fl = 2.0 * M * N * K
            tf = fl / (ms * 1e-3) / 1e12
            peak = peaks["bf16_tflops"] if c == "linear_w8a16" else fp8_peak
            hbm_bytes = wbytes + 2 * M * K + 2 * M * N
            call_stats[c] = {"us": 1e3 * ms, "bound": "tensor", "achieved": tf, "unit": "TFLOP/s",
                             "peak": peak, "frac": tf / peak, "alg_flops": fl,
                             "weight_stream_gbs": wbytes / (ms * 1e-3) / 1e9,
                             "hbm_frac": hbm_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    dominant = max(calls, key=lambda c: call_stats[c]["us"])
    d = call_stats[dominant]
    kernel_file = {"quantize_weight": "quant.cu", "dequantize": "quant.cu",
                   "linear_w8a16": "gemm_w8a16.cu", "linear_w8a8": "gemm_w8a8.cu"}[dominant]
    roofline = {"kernel": dominant, "bound": d["bound"], "achieved": d["achieved"],
                "peak": d["peak"], "unit": d["unit"], "frac": d["frac"],
                "peak_kind": f"{peak_kind} burst" + (" x2 (fp8 nominal ratio)" if dominant == "linear_w8a8" else ""),
                "traffic": traffic_for(kernel_file, f"{dominant}:{wl.name}")}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3/bf16 operands, f32 accumulate", "data": "synthetic",
        "config": {"workload": wl.name, "M": M, "K": K, "N": N,
                   "step": "quantize_weight + dequantize + linear_w8a16 + linear_w8a8",
                   "l2": "flushed between steps outside the step events (512 MiB memset, then a 256 MiB read so no dirty flush lines remain)",
                   "parallelism": f"replicas x{world}"},
        "weight_stream_gbs": {c: call_stats[c]["weight_stream_gbs"]
                              for c in ("linear_w8a16", "linear_w8a8")},
        "calls": call_stats, "roofline": roofline,
        "gpu_launches": 5 * args.steps,
        "clocks": clk,
    }

    # e2e: the same step through the public API with inputs from pinned host
    # memory and the two linear outputs read back, every step. Steps are
    # pipelined over three streams with two sets of device inputs and
    # outputs: step i + 1's inputs are uploaded while step i computes and
    # step i - 1's outputs come back (each step still copies its own W and x
    # in and its own y16 and y8 out inside the timed region).
    if not args.no_e2e:
        w_pin = w_h.pin_memory()
        x_pin = x_h.pin_memory()
        y16_pin = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        y8_pin = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        e_steps = max(3, min(args.steps, 20))
        bufs = [(w, x, y16, y8), (torch.empty_like(w), torch.empty_like(x), torch.empty_like(y16),
                                  torch.empty_like(y8))]
        h2d, comp, d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for e in ev_comp + ev_out:
            e.record(comp)

        def e2e_steps(n):
            for i in range(n):
                b = i & 1
                wb, xb, y16b, y8b = bufs[b]
                h2d.wait_event(ev_comp[b])        # step i - 2 has read these inputs
                with torch.cuda.stream(h2d):
                    wb.copy_(w_pin, non_blocking=True)
                    xb.copy_(x_pin, non_blocking=True)
                ev_in[b].record(h2d)
                comp.wait_event(ev_in[b])
                comp.wait_event(ev_out[b])        # step i - 2's outputs are back
                with torch.cuda.stream(comp):
                    step(w=wb, x=xb, y16=y16b, y8=y8b)
                ev_comp[b].record(comp)
                d2h.wait_event(ev_comp[b])
                with torch.cuda.stream(d2h):
                    y16_pin.copy_(y16b, non_blocking=True)
                    y8_pin.copy_(y8b, non_blocking=True)
                ev_out[b].record(d2h)

        torch.cuda.synchronize()
        e2e_steps(2)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        h2d.wait_event(e0)
        e2e_steps(e_steps)
        comp.wait_stream(d2h)
        comp.wait_stream(h2d)
        e1.record(comp)
        torch.cuda.synchronize()
        te = max_over_ranks(e0.elapsed_time(e1) / e_steps, world, dev)
        line["e2e"] = {"value": world * flops_step / (te * 1e-3) / 1e12,
                       "unit": "TFLOP/s", "ms_per_step": te, "steps": e_steps,
                       "h2d_bytes_per_step": 2 * N * K + 2 * M * K,
                       "d2h_bytes_per_step": 2 * 2 * M * N,
                       "pipelined": "steps overlap: upload of step i+1, compute of step i, "
                                    "download of step i-1 (three streams, two buffer sets)"}
        del bufs
    else:
        line["e2e"] = None

    if not args.no_targets and world == 1:
        line["targets"] = measure_targets(fb, dev, peaks, flush_l2, ClockSampler(
            visible.split(",")[local] if visible else str(local)))

    # A/B, outside the step: (1) the route of FP8-less tensor cores, our
    # dequantize then a library BF16 GEMM on the expanded weight, against the
    # fused W8A16 call; (2) one activation quantization shared by sibling
    # linears (fp8blk_quantize_act + fp8blk_linear_w8a8_quantized) against
    # the all-in-one W8A8 call, which re-quantizes x each time.
    if not args.no_ab:
        def timed(fn, iters=20):
            ts = []
            for _ in range(iters):
                flush_l2()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(); fn(); b.record()
                ts.append((a, b))
            torch.cuda.synchronize()
            return 1e3 * statistics.mean(a.elapsed_time(b) for a, b in ts)

        # the route's matmul accumulates in FP32 throughout (no reduced-precision
        # split reduction), as the parity test of this route checks it
        torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = False
        y_lib = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        qx, sx = fb.quantize_act(x)
        for _ in range(3):
            fb.dequantize(q, s, out=wd); torch.matmul(x, wd.t(), out=y_lib)
            fb.linear_w8a8_quantized(qx, sx, q, s, out=y8)
        torch.cuda.synchronize()
        us_deq = timed(lambda: fb.dequantize(q, s, out=wd))
        us_mm = timed(lambda: torch.matmul(x, wd.t(), out=y_lib))
        us_route = timed(lambda: (fb.dequantize(q, s, out=wd), torch.matmul(x, wd.t(), out=y_lib)))
        us_w16 = timed(lambda: fb.linear_w8a16(x, q, s, out=y16, workspace=ws16))
        us_act = timed(lambda: fb.quantize_act(x, qx, sx))
        us_w8q = timed(lambda: fb.linear_w8a8_quantized(qx, sx, q, s, out=y8))
        us_w8 = timed(lambda: fb.linear_w8a8(x, q, s, out=y8, workspace=ws8))
        fl = 2.0 * M * N * K
        line["ab"] = {
            "library_bf16_route": {
                "dequantize_us": us_deq, "cublas_bf16_matmul_us": us_mm,
                "route_us": us_route, "route_tflops": fl / (us_route * 1e-6) / 1e12,
                "linear_w8a16_us": us_w16, "linear_w8a16_tflops": fl / (us_w16 * 1e-6) / 1e12,
                "speedup_w8a16_over_route": us_route / us_w16},
            "shared_act_quantization": {
                "quantize_act_us": us_act, "linear_w8a8_quantized_us": us_w8q,
                "linear_w8a8_us": us_w8,
                "saved_per_sibling_us": us_w8 - us_w8q},
            "iters": 20, "l2": "flushed (memset + read) before each timed call"}
        del y_lib, qx, sx

    assert fb.read_device_error() == 0
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = run_oracle(wl, synth.bf16_bits(w_h), synth.bf16_bits(x_h), 12.0)
    elif rank == 0:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
