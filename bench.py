"""Benchmark of the SVDQuant NVFP4 W4A4 + low-rank linear (libsvdq) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload qkv]
    python bench.py --suite [names] [--steps K]     (one line per workload; rank-overhead sweep)

One step = one forward pass of the layer over one batch of synthetic tokens: K1
(svdq_quant_act_lora_down: smoothing, NVFP4 activation quantization, low-rank down-projection)
then K2 (svdq_gemm_w4a4_lora_up: block-scaled FP4 GEMM + low-rank up-projection + bias).
Default workload: the FLUX-like fused QKV projection, M = 4608 tokens, K = 3072, N = 9216,
rank 32. Inputs are resident in HBM when the timed region starts; successive steps rotate
over three buffer sets (inputs, activations, outputs and layer copies, >3x the 126 MB L2) so
that no step finds its operands in L2.

The timed region replays one CUDA graph captured from the library calls: the K steps back to
back (K1 then K2 per step, buffer sets rotating), so it measures the device rather than
per-call host work, and each kernel's prologue overlaps its predecessor (the library launches
with programmatic dependent launch). Per-kernel durations, for the roofline, come from two more
graphs of K back-to-back launches of K1 alone and of K2 alone, timed with CUDA events on the
same stream. The e2e number goes through the host-buffer entry point call by call.

Metric: layer TFLOPS = (2MNK + 2MNr + 2MKr) / step time, summed over ranks (weak scaling:
every rank runs its own replica on its own batch, no collective on the data path).
Rank 0 prints one JSON line. ``--impl reference`` times the fp64 CPU oracle instead (the
only reference implementation of this method available here): W untimed warm-up steps, then K
timed steps, each step one bounded slice of the workload's tokens.

``--suite`` also covers the fused QKV layer with the Q/K normalization + rotary output stage
(``qkv_qknorm_rope``: against the plain K2 and against plain K2 + the separate step) and the
awq_w4a16 GEMV on FLUX's double-block modulation shape (``awq_mod``, ``awq_mod_m2``: 1 and 2
tokens, against the HBM roof).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import CONFIGS, make_inputs  # noqa: E402

METRIC = "W4A4+LoRA linear TFLOPS & fraction of B200 FP4 peak; quant-pass HBM GB/s"
FP4_OVER_BF16 = 9.0 / 2.25  # nominal dense NVFP4 / BF16 tensor throughput ratio on B200
# Measured on this GPU model with a kind::mxf4nvf4 MMA-only microbenchmark (no operand loads, all
# SMs): 128 cycles per one-CTA M128 N256 K64 MMA, i.e. 148 x 2 x 128 x 256 x 64 / 128 flops per
# cycle at 1965 MHz.
MMA_ONLY_FP4_TFLOPS = 148 * 2 * 128 * 256 * 64 / 128 * 1965e6 / 1e12
L2_BYTES = 126 * 1024 * 1024


def layer_flops(M, K, N, r):
    return 2.0 * M * N * K + 2.0 * M * N * r + 2.0 * M * K * r


def k1_bytes(M, K, r):
    """Algorithmic HBM bytes of K1: read X, inv_lambda, L1; write codes, scales, lora_act."""
    return 2.0 * M * K + 4.0 * K + 2.0 * K * r + M * K / 2 + M * K / 16 + 2.0 * M * r


def aggregate(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOPS: every rank runs `steps` steps of its own replica; the job takes the
    slowest rank's time (max over ranks)."""
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12


def max_over_ranks(value_ms: float, dist, device) -> float:
    """Max of a per-rank elapsed time over all ranks (identity without a process group)."""
    if dist is None:
        return value_ms
    import torch

    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def k2_flops(M, K, N, r):
    return 2.0 * M * N * K + 2.0 * M * N * r


def k2_bytes(M, K, N, r):
    """Algorithmic HBM bytes of K2: codes and scales of X and of R, the hi/lo down-projection,
    L2, bias, the bf16 output."""
    return M * K / 2 + M * K / 16 + N * K / 2 + N * K / 16 + 4.0 * M * r + 2.0 * r * N + 4.0 * N + 2.0 * M * N


def kernel_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` ("k1" or "k2") from the committed ncu capture of
    consecutive launches (profiles/<kernel>_traffic.json), if it was taken on the current sources
    of that kernel (the file records the sha1 of kernel_sources_sha1) and this workload; otherwise
    None."""
    tr_path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.json")
    if not os.path.exists(tr_path):
        return None
    with open(tr_path) as f:
        tr = json.load(f)
    if tr.get("workload") == workload and tr.get("source_sha1") == kernel_sources_sha1(kernel):
        return tr.get("bytes_per_launch")
    return None


def kernel_sources_sha1(kernel: str) -> str:
    """sha1 over the kernel's source file and the device headers it includes, in that order."""
    import hashlib

    csrc = os.path.join(ROOT, "bit_rank_compensated_b200", "csrc")
    h = hashlib.sha1()
    for name in ({"k1": "quant_act.cu", "k2": "gemm.cu"}[kernel], "common.cuh", "nvfp4.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def host_link_times(Xh, Xd, Yh, Yd, dev, reps=5):
    """Median ms of one step's host-to-device copy of X, device-to-host copy of Y, and both
    together on two streams (pinned host buffers)."""
    import torch

    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def timed(fn):
        out = []
        for _ in range(reps):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            fn()
            torch.cuda.synchronize()
            out.append((time.perf_counter() - t0) * 1e3)
        return statistics.median(out)

    def h2d():
        with torch.cuda.stream(s_in):
            Xd.copy_(Xh, non_blocking=True)

    def d2h():
        with torch.cuda.stream(s_out):
            Yh.copy_(Yd, non_blocking=True)

    h2d_ms = timed(h2d)
    d2h_ms = timed(d2h)
    both_ms = timed(lambda: (h2d(), d2h()))
    return {"h2d_ms": h2d_ms, "d2h_ms": d2h_ms, "both_ms": both_ms,
            "h2d_gbs": Xh.numel() * 2 / (h2d_ms * 1e-3) / 1e9, "d2h_gbs": Yh.numel() * 2 / (d2h_ms * 1e-3) / 1e9}


def read_sustained_bf16():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            v = json.load(f).get("bf16_tflops_sustained")
        return float(v) if v else None
    return None


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling (every 100 ms) around the timed work. mark_start() /
    mark_end() bracket the loaded period; the summary covers the samples taken inside it."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except FileNotFoundError:
            self.proc = None
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]

    @staticmethod
    def _epoch(ts: str):
        try:
            return datetime.datetime.strptime(ts.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def summary(self):
        sm, mx, reasons, n_all = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 10:
                continue
            n_all += 1
            t = self._epoch(f[0])
            if self.t0 is not None and (t is None or t < self.t0 or t > self.t1):
                continue
            try:
                sm.append(float(f[2]))
                mx = float(f[3])
            except ValueError:
                continue
            for n, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
               "samples": len(sm), "samples_total": n_all}
        if self.t0 is not None:
            out["window_s"] = round(self.t1 - self.t0, 3)
        return out


def clock_snapshot(gpu_index: int = 0):
    """One nvidia-smi reading of the SM clock and the active throttle reasons, taken right after a
    workload's timed region (the clock state it ran in); None where nvidia-smi is missing."""
    try:
        out = subprocess.run(["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={ClockSampler.Q}",
                              "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10).stdout
    except (FileNotFoundError, subprocess.TimeoutExpired):
        return None
    f = [x.strip() for x in out.strip().split(",")]
    if len(f) < 10:
        return None
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    try:
        return {"sm_mhz": float(f[2]), "sm_max_mhz": float(f[3]),
                "reasons": [n for n, v in zip(names, f[6:10]) if v.lower() == "active"]}
    except ValueError:
        return None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_oracle_sample(shape, rows: int, seed: int = 0, budget_s: float = 20.0, threads: int | None = None,
                      layer=None, X=None, steps: int | None = None, warmup: int = 0):
    """Times the fp64 oracle's forward pass (quantize + down-projection + dequantized GEMM +
    up-projection) on `rows`-token slices of the workload: for about budget_s seconds, or, with
    `steps`, for exactly that many slices after `warmup` untimed ones; the SVD prepare is timed
    apart. threads: BLAS thread limit (None: numpy's default pool)."""
    from oracle import svdq_oracle as O
    from synth import bf16_bits_to_f32

    t_prep = 0.0
    if layer is None:
        Xb, W, b, _ = make_inputs(shape, seed=seed)
        X = bf16_bits_to_f32(Xb).astype(np.float64)
        t0 = time.perf_counter()
        layer = O.prepare(W, b, O.calibration_absmax(X), shape.rank)
        t_prep = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
    except Exception:  # pragma: no cover - threadpoolctl is in the image
        threadpool_info = threadpool_limits = None
    import contextlib

    ctx = threadpool_limits(threads) if (threads and threadpool_limits) else contextlib.nullcontext()
    with ctx:
        for w in range(warmup):
            O.layer_forward(X[(w * rows) % shape.M:(w * rows) % shape.M + rows], layer)
        done, t_fwd, reps = 0, 0.0, 0
        while (reps < steps) if steps is not None else (t_fwd < budget_s and reps < 64):
            sl = X[(reps * rows) % shape.M:(reps * rows) % shape.M + rows]
            t0 = time.perf_counter()
            O.layer_forward(sl, layer)
            t_fwd += time.perf_counter() - t0
            done += sl.shape[0]
            reps += 1
        if threadpool_info is not None:
            used = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        else:
            used = os.cpu_count()
    flops = layer_flops(done, shape.K, shape.N, shape.rank)
    return {"value": flops / t_fwd / 1e12, "seconds": t_fwd, "tokens": done, "cores": used,
            "prepare_s": t_prep, "reps": reps, "layer": layer, "X": X}


# Tokens per step of the reference arm. A step of the oracle costs about the same for any slice
# up to a few hundred tokens (each call first dequantizes the whole weight), so smaller slices
# would not shorten the run, only lower the measured rate.
REFERENCE_ROWS = 256


def run_reference(args, shape, rank, world):
    if rank != 0:
        return 0
    rows = min(REFERENCE_ROWS, shape.M)
    res = cpu_oracle_sample(shape, rows, steps=args.steps, warmup=args.warmup)
    ms = res["seconds"] / res["reps"] * 1e3
    res1 = cpu_oracle_sample(shape, 64, budget_s=8.0, threads=1, layer=res["layer"], X=res["X"])
    line = {
        "impl": "reference", "metric": METRIC, "value": res["value"], "unit": "TFLOPS", "n_gpus": args.gpus,
        "steps": res["reps"], "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(shape), "M": shape.M, "K": shape.K, "N": shape.N, "rank": shape.rank},
        "cpu_baseline": {"value": res["value"], "unit": "TFLOPS", "cores": res["cores"], "kind": "oracle",
                         "sample": f"{res['reps']} timed steps of {rows} tokens ({res['tokens']} tokens) of the "
                                   f"workload after {args.warmup} untimed ones; fp64 numpy oracle forward pass, "
                                   f"prepare (SVD) excluded ({res['prepare_s']:.1f} s)",
                         "cpu_model": cpu_model(), "nproc": os.cpu_count(),
                         "single_thread": {"value": res1["value"], "unit": "TFLOPS",
                                           "sample": f"{res1['reps']} slices of 64 tokens, 1 BLAS thread"}},
        "e2e": {"value": res["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_name(shape):
    return f"{shape.name}: SVDQuant NVFP4 W4A4+LoRA linear M={shape.M} K={shape.K} N={shape.N} rank={shape.rank}"


def capture_sequence(n, fns_of):
    """One CUDA graph holding steps 0 .. n-1: the callables fns_of(i) (None entries skipped),
    each launching one kernel on the stream it is given, back to back. Replaying it submits
    the n steps without the per-call host work (argument checks, tensor-map encoding)."""
    import torch

    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        st = torch.cuda.current_stream()
        for i in range(n):
            for fn in fns_of(i):
                if fn is not None:
                    fn(st)
    torch.cuda.synchronize()
    return g


def time_graphs(stream, graphs):
    """Replays the graphs one after the other, each between two CUDA events on `stream`;
    returns the device time (ms) of each."""
    import torch

    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(graphs) + 1)]
    evs[0].record(stream)
    for g, e in zip(graphs, evs[1:]):
        g.replay()
        e.record(stream)
    torch.cuda.synchronize()
    return [evs[k].elapsed_time(evs[k + 1]) for k in range(len(graphs))]


def time_graphs_rep(stream, graphs, reps):
    """time_graphs repeated `reps` times (the graphs interleaved); per graph the list of times."""
    out = [[] for _ in graphs]
    for _ in range(reps):
        for lst, t in zip(out, time_graphs(stream, graphs)):
            lst.append(t)
    return out


def med_best(ms_list, per):
    """(median, best) of a list of graph times divided by `per` launches each."""
    v = sorted(x / per for x in ms_list)
    return statistics.median(v), v[0]


def clone_layer(src, dev):
    """A second copy of a prepared layer's device buffers (so rotating steps do not share weights
    that would then stay in L2)."""
    from bit_rank_compensated_b200 import svdq

    L = svdq.Layer(src.N, src.K, src.rank, device=dev, with_bias=src.bias is not None)
    for name in ("wq", "ws", "inv_lambda", "lam", "L1t", "L2t", "bias"):
        t = getattr(src, name)
        if t is not None:
            getattr(L, name).copy_(t)
    L.s.w_tensor_scale, L.s.x_tensor_scale = src.s.w_tensor_scale, src.s.x_tensor_scale
    return L


AWQ_WORKLOADS = {"awq_mod": (1, 3072, 18432), "awq_mod_m2": (2, 3072, 18432)}


def awq_bytes(M, K, N):
    """Algorithmic HBM bytes of the 4-bit-weight GEMV: int4 codes, fp16 scales and zero points
    (3 bytes per group of 64; the packed layout carries 4, counted as 3), bf16 X and Y, fp32 bias."""
    return N * K / 2.0 + N * (K / 64) * 3.0 + 2.0 * M * K + 2.0 * M * N + 4.0 * N


def time_awq(M, K, N, steps, warmup, dev, stream, nb=5):
    """Mean device time (ms) of svdq_awq_gemv_w4a16 over K back-to-back launches (one graph),
    rotating over `nb` weight sets (more bytes than the L2 holds)."""
    import torch
    from bit_rank_compensated_b200 import svdq
    from synth import make_modulation_inputs

    Xb, W, b = make_modulation_inputs(M, K, N)
    X = torch.from_numpy(Xb.view(np.int16)).to(dev).view(torch.bfloat16)
    bias = torch.from_numpy(b).to(dev)
    sets = [svdq.AwqLinear.from_float(torch.from_numpy(W).to(dev), bias) for _ in range(nb)]
    Ys = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(nb)]

    def launch(i):
        return [lambda st: svdq.awq_gemv_w4a16(X, sets[i % nb], Ys[i % nb], st)]

    for i in range(warmup):
        launch(i)[0](stream)
    torch.cuda.synchronize()
    g = capture_sequence(steps, launch)
    g.replay()
    torch.cuda.synchronize()
    (tot,) = time_graphs_rep(stream, [g], REPS)
    assert svdq.last_device_error() == 0
    return med_best(tot, steps)[0]


REPS = 7  # timed replays of each graph; medians are reported


def time_mlp_pair(steps, warmup, dev, stream, nb=3):
    """The FLUX feed-forward pair (M 4608, 3072 -> 12288 -> 3072, rank 32) fused and unfused.
    Fused: K1 (up), the up layer's GEMM with the GELU + down-quantization output stage, the partial
    sums' reduction, K2 (down). Unfused: K1 (up), K2 (up) writing bf16 GELU(Y1), K1 (down) reading it
    back, K2 (down). Returns (fused_ms, unfused_ms, middle_ms) per step (medians over REPS timings of
    K back-to-back steps, buffer sets rotating)."""
    import torch
    from bit_rank_compensated_b200 import svdq

    up_s, down_s = CONFIGS["mlp_up"], CONFIGS["mlp_down"]
    M = up_s.M
    Xb, Wu, bu, _ = make_inputs(up_s, seed=0)
    _, Wd, bd, _ = make_inputs(down_s, seed=0)
    X0 = torch.from_numpy(Xb.view(np.int16)).to(dev).view(torch.bfloat16)
    up = svdq.prepare_weights(torch.from_numpy(Wu).to(dev), torch.from_numpy(bu).to(dev), svdq.act_absmax(X0),
                              up_s.rank)
    # the down layer is calibrated on the intermediate the up layer produces
    xq, xs, la = svdq.quant_act_lora_down(X0, up)
    H = svdq.gemm_w4a4_lora_up_gelu(xq, xs, la, M, up)
    down = svdq.prepare_weights(torch.from_numpy(Wd).to(dev), torch.from_numpy(bd).to(dev), svdq.act_absmax(H),
                                down_s.rank)
    ups = [up] + [clone_layer(up, dev) for _ in range(nb - 1)]
    downs = [down] + [clone_layer(down, dev) for _ in range(nb - 1)]
    Xs = [X0] + [X0.clone() for _ in range(nb - 1)]
    b_up = [svdq.alloc_activations(M, up, dev) for _ in range(nb)]
    b_dn = [svdq.alloc_activations(M, down, dev) for _ in range(nb)]
    ws = [svdq.alloc_mlp_workspace(M, up, down, dev) for _ in range(nb)]
    Hs = [torch.empty(M, up.N, dtype=torch.bfloat16, device=dev) for _ in range(nb)]
    Zs = [torch.empty(M, down.N, dtype=torch.bfloat16, device=dev) for _ in range(nb)]

    def fused(j):
        q, s_, l = b_up[j]
        return [lambda st: svdq.quant_act_lora_down(Xs[j], ups[j], q, s_, l, st),
                lambda st: svdq.gemm_w4a4_lora_up_gelu_quant(q, s_, l, M, ups[j], downs[j], b_dn[j], ws[j], st),
                lambda st: svdq.gemm_w4a4_lora_up(*b_dn[j], M, downs[j], Zs[j], st)]

    def unfused(j):
        q, s_, l = b_up[j]
        qd, sd, ld = b_dn[j]
        return [lambda st: svdq.quant_act_lora_down(Xs[j], ups[j], q, s_, l, st),
                lambda st: svdq.gemm_w4a4_lora_up_gelu(q, s_, l, M, ups[j], Hs[j], st),
                lambda st: svdq.quant_act_lora_down(Hs[j], downs[j], qd, sd, ld, st),
                lambda st: svdq.gemm_w4a4_lora_up(qd, sd, ld, M, downs[j], Zs[j], st)]

    for i in range(warmup):
        for fn in fused(i % nb) + unfused(i % nb):
            fn(stream)
    torch.cuda.synchronize()
    g_f = capture_sequence(steps, lambda i: fused(i % nb))
    g_u = capture_sequence(steps, lambda i: unfused(i % nb))
    g_mid = capture_sequence(steps, lambda i: fused(i % nb)[1:2])
    for g in (g_f, g_u, g_mid):
        g.replay()
    torch.cuda.synchronize()
    tf, tu, tm = time_graphs_rep(stream, [g_f, g_u, g_mid], REPS)
    assert svdq.last_device_error() == 0
    return med_best(tf, steps)[0], med_best(tu, steps)[0], med_best(tm, steps)[0]

SUITE = ["qkv", "qkv_qknorm_rope", "mlp_pair", "awq_mod", "awq_mod_m2", "mlp_up", "mlp_down", "sweep_m256", "sweep_m1024", "sweep_m4096", "sweep_m16384",
         "sweep_r0", "sweep_r16", "sweep_r32", "sweep_r64", "sweep_r128"]
HEAD_DIM = 128


def qk_stage_bytes(M, N):
    """Algorithmic HBM bytes of the unfused Q/K normalization + rotary step: read and rewrite the
    bf16 Q and K sections (2/3 of Y), read the (cos, sin) table (M x 64 x 2 fp32)."""
    return 2.0 * (2.0 * M * (2 * N // 3)) + M * (HEAD_DIM // 2) * 8.0


def time_layer(shape, steps, warmup, dev, stream, unfused=False, nb=3, stage="plain"):
    """Mean device time (ms) per step of the layer on one GPU over `nb` rotating buffer sets:
    fused K1 + K2, or the unfused four-kernel path. stage = "qknr": K2 with the fused QKV output
    stage (Q/K normalization and rotary embedding); "qknr_unfused": plain K2 followed by the
    separate normalization + rotary step. Returns (step_ms, k1_ms, k2_ms); for "qknr_unfused"
    k2_ms covers K2 and the separate step."""
    import torch
    from bit_rank_compensated_b200 import svdq
    from synth import qk_norm_weights, rope_table

    M, K, N, r = shape.M, shape.K, shape.N, shape.rank
    Xb, W, b, _ = make_inputs(shape, seed=0)
    X0 = torch.from_numpy(Xb.view(np.int16)).to(dev).view(torch.bfloat16)
    ax = svdq.act_absmax(X0)
    L0 = svdq.prepare_weights(torch.from_numpy(W).to(dev), torch.from_numpy(b).to(dev), ax, r)
    Ls = [L0] + [clone_layer(L0, dev) for _ in range(nb - 1)]
    Xs = [X0] + [X0.clone() for _ in range(nb - 1)]
    bufs = [svdq.alloc_activations(M, L0, dev) for _ in range(nb)]
    Ys = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(nb)]
    heads = N // (3 * HEAD_DIM)
    if stage != "plain":
        wq, wk = (torch.from_numpy(w).to(dev) for w in qk_norm_weights(HEAD_DIM))
        ropes = [torch.from_numpy(rope_table(M, HEAD_DIM)).to(dev) for _ in range(nb)]

    def k2_part(j):
        xq, xs, la = bufs[j]
        L = Ls[j]
        if stage == "qknr":
            return lambda st: svdq.gemm_w4a4_lora_up_qk_norm_rope(xq, xs, la, M, L, heads, wq, wk, ropes[j], 1e-6,
                                                                  Ys[j], st)
        if stage == "qknr_unfused":
            def both(st):
                svdq.gemm_w4a4_lora_up(xq, xs, la, M, L, Ys[j], st)
                svdq.qk_norm_rope(Ys[j], heads, wq, wk, ropes[j], 1e-6, st)
            return both
        return lambda st: svdq.gemm_w4a4_lora_up(xq, xs, la, M, L, Ys[j], st)

    def step_on(j):
        # part 0: K1 (or the whole unfused path), part 1: K2 (None when unfused)
        xq, xs, la = bufs[j]
        L = Ls[j]
        if unfused:
            return (lambda st: svdq.unfused_forward(Xs[j], L, bufs[j], Ys[j], st)), None
        return (lambda st: svdq.quant_act_lora_down(Xs[j], L, xq, xs, la, st)), k2_part(j)

    def step(i):
        a, b = step_on(i % nb)
        a(stream)
        if b is not None:
            b(stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    g_steps = capture_sequence(steps, lambda i: step_on(i % nb))
    if unfused:
        g_steps.replay()
        (tot,) = time_graphs_rep(stream, [g_steps], REPS)
        assert svdq.last_device_error() == 0
        return med_best(tot, steps)[0], None, None
    g_k1 = capture_sequence(steps, lambda i: step_on(i % nb)[:1])
    g_k2 = capture_sequence(steps, lambda i: step_on(i % nb)[1:])
    for g in (g_steps, g_k1, g_k2):  # warm replay
        g.replay()
    torch.cuda.synchronize()
    tot, k1, k2 = time_graphs_rep(stream, [g_steps, g_k1, g_k2], REPS)
    assert svdq.last_device_error() == 0
    return med_best(tot, steps)[0], med_best(k1, steps)[0], med_best(k2, steps)[0]


def run_suite(args):
    """One JSON line per named workload (device time, fused path; the rank sweep also times
    rank 0 and the unfused four-kernel path at the same rank). Not part of the default run."""
    import torch
    from bit_rank_compensated_b200 import build, svdq

    if not os.path.exists(svdq.LIB_PATH):
        build.build()
    svdq.load()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    hbm_gbs, bf16_tf, peak_kind = read_peaks()
    fp4_peak = bf16_tf * FP4_OVER_BF16
    r0_ms = None
    plain_k2 = {}
    for name in args.suite.split(","):
        if name == "mlp_pair":
            f_ms, u_ms, mid_ms = time_mlp_pair(args.steps, args.warmup, dev, stream)
            us, ds = CONFIGS["mlp_up"], CONFIGS["mlp_down"]
            fl = layer_flops(us.M, us.K, us.N, us.rank) + layer_flops(ds.M, ds.K, ds.N, ds.rank)
            print(json.dumps({
                "metric": METRIC, "value": fl / (f_ms * 1e-3) / 1e12, "unit": "TFLOPS", "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": f_ms, "higher_is_better": True,
                "dtype": "nvfp4", "data": "synthetic",
                "config": {"workload": f"mlp_pair: FLUX feed-forward M={us.M} {us.K} -> {us.N} -> {ds.N}, GELU "
                                       f"(tanh), rank {us.rank}/{ds.rank}, fused (no 16-bit intermediate)"},
                "mlp_pair": {"fused_us": f_ms * 1e3, "unfused_us": u_ms * 1e3, "unfused_over_fused": u_ms / f_ms,
                             "fused_middle_us": mid_ms * 1e3,
                             "intermediate_bytes_saved": 2 * 2 * us.M * us.N},
                "clocks_after": clock_snapshot(), "peaks": peak_kind}), flush=True)
            torch.cuda.empty_cache()
            continue
        if name in AWQ_WORKLOADS:
            M, K, N = AWQ_WORKLOADS[name]
            ms = time_awq(M, K, N, args.steps, args.warmup, dev, stream)
            gbs = awq_bytes(M, K, N) / (ms * 1e-3) / 1e9
            print(json.dumps({
                "metric": "awq_w4a16 modulation GEMV HBM GB/s", "value": gbs, "unit": "GB/s", "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "dtype": "int4 x bf16 -> fp32", "data": "synthetic",
                "config": {"workload": f"{name}: awq_w4a16 GEMV M={M} K={K} N={N} (FLUX double-block modulation)",
                           "M": M, "K": K, "N": N},
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
                             "bytes_per_launch": awq_bytes(M, K, N)},
                "clocks_after": clock_snapshot(), "peaks": peak_kind}), flush=True)
            torch.cuda.empty_cache()
            continue
        qknr = name.endswith("_qknorm_rope")
        shape = CONFIGS[name[:-len("_qknorm_rope")] if qknr else name]
        M, K, N, r = shape.M, shape.K, shape.N, shape.rank
        step_ms, k1_ms, k2_ms = time_layer(shape, args.steps, args.warmup, dev, stream,
                                           stage="qknr" if qknr else "plain")
        line = {"metric": METRIC, "value": layer_flops(M, K, N, r) / (step_ms * 1e-3) / 1e12, "unit": "TFLOPS",
                "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
                "higher_is_better": True, "dtype": "nvfp4", "data": "synthetic",
                "config": {"workload": workload_name(shape) + (", fused Q/K RMS norm + rotary output stage"
                                                               if qknr else ""), "M": M, "K": K, "N": N, "rank": r},
                "k1": {"us": k1_ms * 1e3, "gbs": k1_bytes(M, K, r) / (k1_ms * 1e-3) / 1e9,
                       "frac_hbm": k1_bytes(M, K, r) / (k1_ms * 1e-3) / 1e9 / hbm_gbs},
                "k2": {"us": k2_ms * 1e3, "tflops": k2_flops(M, K, N, r) / (k2_ms * 1e-3) / 1e12,
                       "frac_fp4": k2_flops(M, K, N, r) / (k2_ms * 1e-3) / 1e12 / fp4_peak,
                       "gbs": k2_bytes(M, K, N, r) / (k2_ms * 1e-3) / 1e9,
                       "frac_hbm": k2_bytes(M, K, N, r) / (k2_ms * 1e-3) / 1e9 / hbm_gbs,
                       # the binding roof: the larger of the tensor time and the HBM time of the algorithmic work
                       "binding": "tensor" if k2_flops(M, K, N, r) / (fp4_peak * 1e12) >= k2_bytes(M, K, N, r) / (hbm_gbs * 1e9)
                       else "hbm",
                       "frac_binding": max(k2_flops(M, K, N, r) / (fp4_peak * 1e12),
                                           k2_bytes(M, K, N, r) / (hbm_gbs * 1e9)) / (k2_ms * 1e-3)},
                "tokens_per_s": M / (step_ms * 1e-3), "clocks_after": clock_snapshot(), "peaks": peak_kind}
        if not qknr:
            plain_k2[shape.name] = k2_ms
        else:
            if shape.name not in plain_k2:
                plain_k2[shape.name] = time_layer(shape, args.steps, args.warmup, dev, stream)[2]
            unf_ms, _, unf_k2 = time_layer(shape, args.steps, args.warmup, dev, stream, stage="qknr_unfused")
            # the separate step alone: the unfused K2 + step minus the plain K2
            sep_ms = unf_k2 - plain_k2[shape.name]
            line["qknorm_rope"] = {
                "fused_stage_overhead_vs_plain_k2": k2_ms / plain_k2[shape.name] - 1.0,
                "unfused_step_ms": unf_ms, "unfused_over_fused": unf_ms / step_ms,
                "separate_step_us": sep_ms * 1e3,
                "separate_step_gbs": qk_stage_bytes(M, N) / (sep_ms * 1e-3) / 1e9 if sep_ms > 0 else None,
                "separate_step_frac_hbm": qk_stage_bytes(M, N) / (sep_ms * 1e-3) / 1e9 / hbm_gbs if sep_ms > 0 else None}
        if name.startswith("sweep_r"):
            if r == 0:
                r0_ms = step_ms
            else:
                unf_ms, _, _ = time_layer(shape, args.steps, args.warmup, dev, stream, unfused=True)
                line["unfused_ms"] = unf_ms
                line["unfused_over_fused"] = unf_ms / step_ms
                if r0_ms is not None:
                    line["lowrank_overhead_vs_r0"] = step_ms / r0_ms - 1.0
        print(json.dumps(line), flush=True)
        torch.cuda.empty_cache()
    return 0


def run_ncu_target(args, shape):
    """Launch list for ncu: prepare the workload, then `steps` back-to-back plain launches of one
    kernel (k1, or k2 after one K1; mlp: the fused MLP pair's middle kernel on the FLUX feed-forward
    shapes; awq: the awq_w4a16 GEMV on the double-block modulation shape), without graphs, so that
    a capture of consecutive launches (e.g. -k regex:k2_gemm -c 3 --cache-control none) counts the
    output each launch leaves in L2 against the next one. Prints one line; no timing."""
    import torch
    from bit_rank_compensated_b200 import svdq

    svdq.load()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    if args.ncu_kernel == "awq":
        from synth import make_modulation_inputs

        M, K, N = AWQ_WORKLOADS["awq_mod"]
        Xb, W, b = make_modulation_inputs(M, K, N)
        lin = svdq.AwqLinear.from_float(torch.from_numpy(W).to(dev), torch.from_numpy(b).to(dev))
        X = torch.from_numpy(Xb.view(np.int16)).to(dev).view(torch.bfloat16)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        for _ in range(args.steps):
            svdq.awq_gemv_w4a16(X, lin, Y, stream)
        torch.cuda.synchronize()
        assert svdq.last_device_error() == 0
        print(json.dumps({"ncu_target": "awq", "launches": args.steps}), flush=True)
        return 0
    if args.ncu_kernel == "mlp":
        up_s, down_s = CONFIGS["mlp_up"], CONFIGS["mlp_down"]
        M = up_s.M
        Xb, Wu, bu, _ = make_inputs(up_s, seed=0)
        _, Wd, bd, _ = make_inputs(down_s, seed=0)
        X = torch.from_numpy(Xb.view(np.int16)).to(dev).view(torch.bfloat16)
        up = svdq.prepare_weights(torch.from_numpy(Wu).to(dev), torch.from_numpy(bu).to(dev), svdq.act_absmax(X),
                                  up_s.rank)
        xq, xs, la = svdq.quant_act_lora_down(X, up)
        H = svdq.gemm_w4a4_lora_up_gelu(xq, xs, la, M, up)
        down = svdq.prepare_weights(torch.from_numpy(Wd).to(dev), torch.from_numpy(bd).to(dev), svdq.act_absmax(H),
                                    down_s.rank)
        del H
        bufs = svdq.alloc_activations(M, down, dev)
        ws = svdq.alloc_mlp_workspace(M, up, down, dev)
        for _ in range(args.steps):
            svdq.gemm_w4a4_lora_up_gelu_quant(xq, xs, la, M, up, down, bufs, ws, stream)
        torch.cuda.synchronize()
        assert svdq.last_device_error() == 0
        print(json.dumps({"ncu_target": "mlp", "launches": args.steps}), flush=True)
        return 0
    M, K, N, r = shape.M, shape.K, shape.N, shape.rank
    Xb, W, b, _ = make_inputs(shape, seed=0)
    X = torch.from_numpy(Xb.view(np.int16)).to(dev).view(torch.bfloat16)
    L = svdq.prepare_weights(torch.from_numpy(W).to(dev), torch.from_numpy(b).to(dev), svdq.act_absmax(X), r)
    xq, xs, la = svdq.alloc_activations(M, L, dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    if args.ncu_kernel == "k2":
        svdq.quant_act_lora_down(X, L, xq, xs, la, stream)
    for _ in range(args.steps):
        if args.ncu_kernel == "k1":
            svdq.quant_act_lora_down(X, L, xq, xs, la, stream)
        else:
            svdq.gemm_w4a4_lora_up(xq, xs, la, M, L, Y, stream)
    torch.cuda.synchronize()
    assert svdq.last_device_error() == 0
    print(json.dumps({"ncu_target": args.ncu_kernel, "workload": shape.name, "launches": args.steps}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qkv", choices=sorted(CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--soak-s", type=float, default=1.0,
                    help="seconds of untimed step replays inside the clock-sampling window before the timed region")
    ap.add_argument("--suite", nargs="?", const=",".join(SUITE), default=None,
                    help="time a comma-separated list of workloads (default: all) and print one line each")
    ap.add_argument("--ncu-kernel", choices=["k1", "k2", "mlp", "awq"], default=None,
                    help="only launch one kernel `--steps` times back to back (for an ncu capture)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    if args.suite:
        return run_suite(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    shape = CONFIGS[args.workload]

    if args.impl == "reference":
        return run_reference(args, shape, rank, world)
    if args.ncu_kernel:
        return run_ncu_target(args, shape)

    import torch

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    from bit_rank_compensated_b200 import build, svdq

    if not os.path.exists(svdq.LIB_PATH):
        build.build()
    svdq.load()

    M, K, N, r = shape.M, shape.K, shape.N, shape.rank
    Xb, W, b, _ = make_inputs(shape, seed=0)
    dev = torch.device("cuda", local)
    NB = 3  # rotating buffer sets
    Xd0 = torch.from_numpy(Xb.view(np.int16)).to(dev).view(torch.bfloat16)
    Wd = torch.from_numpy(W).to(dev)
    bd = torch.from_numpy(b).to(dev)
    ax = svdq.act_absmax(Xd0)
    layers = [svdq.prepare_weights(Wd, bd, ax, r)]
    layers += [clone_layer(layers[0], dev) for _ in range(NB - 1)]
    del Wd
    Xs = [Xd0] + [Xd0.clone() for _ in range(NB - 1)]
    bufs = [svdq.alloc_activations(M, layers[0], dev) for _ in range(NB)]
    Ys = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(NB)]
    set_bytes = (Xs[0].numel() * 2 + sum(t.numel() * t.element_size() for t in bufs[0] if t is not None)
                 + Ys[0].numel() * 2 + layers[0].wq.numel() + layers[0].ws.numel())
    stream = torch.cuda.current_stream()

    def parts(j):
        xq, xs, la = bufs[j]
        return ((lambda st: svdq.quant_act_lora_down(Xs[j], layers[j], xq, xs, la, st)),
                (lambda st: svdq.gemm_w4a4_lora_up(xq, xs, la, M, layers[j], Ys[j], st)))

    for i in range(args.warmup):
        for fn in parts(i % NB):
            fn(stream)
    torch.cuda.synchronize()
    assert svdq.last_device_error() == 0

    g_steps = capture_sequence(args.steps, lambda i: parts(i % NB))
    g_k1 = capture_sequence(args.steps, lambda i: parts(i % NB)[:1])
    g_k2 = capture_sequence(args.steps, lambda i: parts(i % NB)[1:])
    # K1 over one buffer set only: X (and L1s) stay in L2 between launches (the unflushed figure)
    g_k1_warm = capture_sequence(args.steps, lambda i: parts(0)[:1])
    for g in (g_steps, g_k1, g_k2, g_k1_warm):  # warm replay
        g.replay()
    torch.cuda.synchronize()

    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    # burst: per-kernel durations right after the warm-up, before the GPU has run long under load
    with ClockSampler(gpu_index) as clk_b:
        clk_b.mark_start()
        k1b_runs, k2b_runs, k1wb_runs = time_graphs_rep(stream, [g_k1, g_k2, g_k1_warm], REPS)
        clk_b.mark_end()
    with ClockSampler(gpu_index) as clk:
        clk.mark_start()
        # untimed replays first, so that the clock samples of the window see the GPU under this load
        t_soak = time.time()
        n_soak = 0
        while time.time() - t_soak < args.soak_s:
            g_steps.replay()
            torch.cuda.synchronize()
            n_soak += 1
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        g_steps.replay()
        t_end.record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        # per-kernel durations: K back-to-back launches of each kernel alone, same stream, REPS times
        k1_runs, k2_runs, k1w_runs = time_graphs_rep(stream, [g_k1, g_k2, g_k1_warm], REPS)
        clk.mark_end()
    total_ms = t_start.elapsed_time(t_end)
    k1_avg, k1_best = med_best(k1b_runs, args.steps)
    k2_avg, k2_best = med_best(k2b_runs, args.steps)
    k1w_avg, k1w_best = med_best(k1wb_runs, args.steps)
    k1s_avg, k1s_best = med_best(k1_runs, args.steps)
    k2s_avg, k2s_best = med_best(k2_runs, args.steps)
    err = svdq.last_device_error()

    total_ms = max_over_ranks(total_ms, dist, dev)

    # ---------------- end to end through the host-buffer entry point
    Xh = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, args.e2e_steps)
    for i in range(2):
        svdq.linear_forward_host(Xh, layers[0], Xs[0], bufs[0], Ys[0], Yh, stream)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        svdq.linear_forward_host(Xh, layers[i % NB], Xs[i % NB], bufs[i % NB], Ys[i % NB], Yh, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    # the host link alone: one step's copy in and copy out (pinned), each direction timed alone and
    # both at once on two streams; with the copies overlapped the step cannot beat the slower one
    link = host_link_times(Xh, Xs[0], Yh, Ys[0], dev)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    flops = layer_flops(M, K, N, r)
    value = aggregate(flops, args.steps, world, total_ms)
    e2e_value = aggregate(flops, e2e_steps, world, e2e_ms)
    hbm_gbs, bf16_tf, peak_kind = read_peaks()
    bf16_tf_sus = read_sustained_bf16() or bf16_tf
    fp4_peak = bf16_tf * FP4_OVER_BF16
    fp4_peak_sus = bf16_tf_sus * FP4_OVER_BF16
    k2_tf = k2_flops(M, K, N, r) / (k2_avg * 1e-3) / 1e12
    k2s_tf = k2_flops(M, K, N, r) / (k2s_avg * 1e-3) / 1e12
    k1_gbs = k1_bytes(M, K, r) / (k1_avg * 1e-3) / 1e9
    k1s_gbs = k1_bytes(M, K, r) / (k1s_avg * 1e-3) / 1e9
    k1w_gbs = k1_bytes(M, K, r) / (k1w_avg * 1e-3) / 1e9
    tr2 = kernel_traffic("k2", shape.name)
    tr1 = kernel_traffic("k1", shape.name)
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        res = cpu_oracle_sample(shape, 256, budget_s=15.0)
        res1 = cpu_oracle_sample(shape, 64, budget_s=8.0, threads=1, layer=res["layer"], X=res["X"])
        cpu = {"value": res["value"], "unit": "TFLOPS", "cores": res["cores"], "kind": "oracle",
               "sample": f"{res['reps']} slices of 256 tokens ({res['tokens']} tokens) of the workload; fp64 numpy "
                         f"oracle forward pass, prepare (SVD) excluded ({res['prepare_s']:.1f} s)",
               "cpu_model": cpu_model(), "nproc": os.cpu_count(),
               "single_thread": {"value": res1["value"], "unit": "TFLOPS",
                                 "sample": f"{res1['reps']} slices of 64 tokens ({res1['tokens']} tokens), 1 BLAS thread"}}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": workload_name(shape), "M": M, "K": K, "N": N, "rank": r,
                   "l2": f"{NB} rotating buffer sets of {set_bytes / 1e6:.0f} MB (> 126 MB L2 in total)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "svdq_gemm_w4a4_lora_up (K2)", "bound": "tensor", "achieved": k2_tf,
                     "peak": fp4_peak, "unit": "TFLOP/s", "frac": k2_tf / fp4_peak, "traffic": tr2,
                     "traffic_over_algorithmic": (tr2 / k2_bytes(M, K, N, r)) if tr2 else None,
                     "algorithmic_bytes": k2_bytes(M, K, N, r),
                     "peak_source": f"{peak_kind} bf16 {bf16_tf:.0f} TF/s x {FP4_OVER_BF16:.0f} (nvfp4/bf16 nominal)",
                     "frac_vs_mma_only": k2_tf / MMA_ONLY_FP4_TFLOPS,
                     "mma_only_peak": MMA_ONLY_FP4_TFLOPS,
                     "achieved_basis": f"2MNK + 2MNr per launch / median over {REPS} timings of K back-to-back "
                                       f"launches (CUDA events) / K, timed right after the warm-up (burst)",
                     "sustained": {"us": k2s_avg * 1e3, "achieved": k2s_tf, "peak": fp4_peak_sus,
                                   "frac": k2s_tf / fp4_peak_sus,
                                   "peak_source": f"{peak_kind} sustained bf16 {bf16_tf_sus:.1f} TF/s x "
                                                  f"{FP4_OVER_BF16:.0f}",
                                   "basis": f"same timing after {args.soak_s:.1f} s of back-to-back steps (clocks "
                                            f"below)"}},
        "quant_pass": {"kernel": "svdq_quant_act_lora_down (K1)", "bound": "hbm", "achieved": k1_gbs,
                       "peak": hbm_gbs, "unit": "GB/s", "frac": k1_gbs / hbm_gbs, "us": k1_avg * 1e3,
                       "us_best": k1_best * 1e3, "frac_of_8TBs_datasheet": k1_gbs / 8000.0,
                       "traffic": tr1, "traffic_over_algorithmic": (tr1 / k1_bytes(M, K, r)) if tr1 else None,
                       "l2_warm": {"us": k1w_avg * 1e3, "gbs": k1w_gbs, "frac": k1w_gbs / hbm_gbs,
                                   "note": "K launches over one buffer set (X stays in L2)"},
                       "sustained": {"us": k1s_avg * 1e3, "achieved": k1s_gbs, "frac": k1s_gbs / hbm_gbs}},
        "k2": {"us": k2_avg * 1e3, "us_best": k2_best * 1e3, "tflops": k2_tf},
        "timing": {"reps": REPS, "k1_us": [round(t / args.steps * 1e3, 3) for t in k1b_runs],
                   "k2_us": [round(t / args.steps * 1e3, 3) for t in k2b_runs],
                   "k1_us_sustained": [round(t / args.steps * 1e3, 3) for t in k1_runs],
                   "k2_us_sustained": [round(t / args.steps * 1e3, 3) for t in k2_runs], "soak_replays": n_soak,
                   "value_basis": f"the K-step graph replayed once after {args.soak_s:.1f} s of replays (sustained)"},
        "tokens_per_s": world * M * args.steps / (total_ms * 1e-3),
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": int(M * K * 2),
                "d2h_bytes_per_step": int(M * N * 2), "api": "svdq_linear_forward_host",
                "ms_per_step": e2e_ms / e2e_steps,
                # the copies alone (host clock, synchronised): the step's floor is both directions at once
                "link": {k: round(v, 4) for k, v in link.items()},
                "frac_of_link_floor": link["both_ms"] / (e2e_ms / e2e_steps)},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
        "clocks_burst": clk_b.summary(),
        "device_error": err,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
