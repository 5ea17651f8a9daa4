#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 linear layer on B200.

One step = one forward pass of the layer's hot path over one batch:
svdq_quantize_act (smoothing, NVFP4 quantisation, low-rank down-projection)
then svdq_linear (block-scaled FP4 GEMM + low-rank up-projection + bias).
The residual packer runs once per weight; it is timed separately and
reported beside the step (pack_residual_us).

Default workload: the FLUX.1-shaped MLP up-projection, M = 4608 tokens
(4096 image + 512 text), K = 3072, N = 12288, rank 32, synthetic data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU runs are independent replicas (the layer is one GPU's work; there
is no exchange step), launched one process per GPU by torchrun; the value is
all ranks' work divided by the slowest rank's device time.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SVDQuant W4A4 linear effective TFLOPS & µs/layer; % of B200 FP4/HBM roofline"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 512 << 20  # > 4x the 126 MB L2


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="flux_mlp_up")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--once", choices=["quantize_act", "quantize_act_gelu", "linear", "pack_residual"],
                    help="no timing: three launches of one kernel on the workload (for profilers)")
    ap.add_argument("--rows", type=int, default=None,
                    help="with --once: M rows instead of the workload's (same distributions)")
    ap.add_argument("--sweep", action="store_true",
                    help="the K = N = 3072 sweep over M and rank: one JSON line per point")
    ap.add_argument("--stack", action="store_true",
                    help="the synthetic 12B DiT stack (152 linears, rank 32 + LoRA 32): ms per pass, "
                         "with the oracle's extrapolated time beside it")
    ap.add_argument("--no-stack", action="store_true",
                    help="leave the DiT stack pass out of the default single-GPU line")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch the layer kernels plainly (svdq_set_launch_overlap(0)), for comparison")
    return ap.parse_args()


# DRAM bytes (read + write) of one linear_kernel launch from an ncu capture of
# `bench.py --once linear --workload <name>` (L2-warm), per workload.  A figure
# is reported only while the kernel sources hash to the captured ones.
LINEAR_TRAFFIC_CAPTURES = {
    "flux_mlp_up": {"bytes": 30394112 + 58369792, "sources_sha256": "9e65a425524d6420"},
}


def kernel_sources_sha():
    """Hash of the linear kernel's sources: its header and the helpers it is
    built from."""
    import hashlib
    csrc = os.path.join(ROOT, "bit_w4a4_quantized_smooth_b200", "csrc")
    h = hashlib.sha256()
    for name in ("linear.cuh", "common.cuh", "ptx.cuh"):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def linear_traffic(workload):
    cap = LINEAR_TRAFFIC_CAPTURES.get(workload)
    if cap is None or kernel_sources_sha() != cap["sources_sha256"]:
        return None
    return cap["bytes"]


# ----------------------------------------------------------------- peaks ---

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# FP4 dense / bf16 dense on B200: 9 / 2.25 PFLOP/s (spec sheet, dense)
FP4_OVER_BF16 = 4.0


# ------------------------------------------------ library FP4 reference ---

LIBRARY_FP4_PEAK_SHAPE = (8192, 8192, 8192)


def library_fp4_times(device, flush_l2, shapes, reps=20):
    """Median µs of cuBLASLt's NVFP4 GEMM (torch's block-scaled scaled_mm:
    E2M1 codes, E4M3 scales per 16 along K in the 128 x 4 tile layout,
    bf16 output) for each (M, N, K) of `shapes`, on random codes with unit
    scales and L2 flushed before every rep.  A library-achieved FP4 rate to
    read the linear kernel against; nothing of the layer's path uses it.
    -> ({shape: us}, api) or (None, reason) when torch does not expose it."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    try:
        from torch.nn.functional import ScalingType, SwizzleType, scaled_mm
    except ImportError as e:
        return None, f"torch.nn.functional.scaled_mm unavailable ({e})"
    out = {}
    for (M, N, K) in shapes:
        g = torch.Generator(device=device)
        g.manual_seed(0)
        a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=device, generator=g)
        b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=device, generator=g)
        sa = torch.full((svdq.packed_sizes(M, K)[1],), 0x38, dtype=torch.uint8, device=device)  # E4M3 1.0
        sb = torch.full((svdq.packed_sizes(N, K)[1],), 0x38, dtype=torch.uint8, device=device)
        A, B = a.view(torch.float4_e2m1fn_x2), b.view(torch.float4_e2m1fn_x2).t()
        SA, SB = sa.view(torch.float8_e4m3fn), sb.view(torch.float8_e4m3fn)

        def fn():
            return scaled_mm(A, B, SA, ScalingType.BlockWise1x16, SB, ScalingType.BlockWise1x16,
                             swizzle_a=SwizzleType.SWIZZLE_32_4_4, swizzle_b=SwizzleType.SWIZZLE_32_4_4,
                             output_dtype=torch.bfloat16)
        try:
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
        except Exception as e:  # an unsupported build or device
            return None, f"scaled_mm NVFP4 failed: {type(e).__name__}: {str(e)[:120]}"
        ev = []
        for _ in range(reps):
            flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            ev.append((e0, e1))
        torch.cuda.synchronize()
        out[(M, N, K)] = statistics.median(1e3 * e0.elapsed_time(e1) for e0, e1 in ev)
    return out, "torch.nn.functional.scaled_mm, BlockWise1x16 E4M3 scales (cuBLASLt)"


# ---------------------------------------------------------------- clocks ---

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), max=float(parts[2]), util=float(parts[4]),
                                     hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r["util"] > 0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(load)}


# ------------------------------------------------------------- workload ---

def workload_desc(name, M, K, N, r):
    return {"workload": f"{name}: M={M} K={K} N={N} rank={r}, NVFP4 group 16",
            "M": M, "K": K, "N": N, "rank": r, "l2": "flushed before every step (512 MB write, then 256 MB read: cold, clean L2)"}


def setup_layer(name: str, device, M=None):
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import prep
    from svdq_inputs import make_layer_inputs

    li = make_layer_inputs(name, M=M)

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)

    X = bf16(li.X)
    W = bf16(li.W)
    bias = None if li.bias is None else bf16(li.bias)
    lam, inv = prep.smoothing(X, W)
    L1, L2, R = prep.lowrank(W, lam, li.r)
    rc, rs = svdq.pack_residual(R)
    torch.cuda.synchronize()
    return dict(li=li, X=X, W=W, inv=inv, L1=L1, L2=L2, R=R, bias=bias, rc=rc, rs=rs,
                M=li.M, K=li.K, N=li.N, r=li.r)


def layer_flops(M, K, N, r):
    return 2.0 * M * N * K + 2.0 * M * (K + N) * r


def linear_bytes(M, K, N, r):
    """Algorithmic bytes of the layer: X bf16, packed R, L1, L2, Y, bias."""
    return 2 * M * K + N * K // 2 + N * K // 16 + 2 * K * r + 2 * r * N + 2 * M * N + 2 * N


# ------------------------------------------------------ across ranks ---

def max_over_ranks(x, device=None):
    """The largest value of `x` over all ranks (x itself without a process
    group): every multi-GPU number is the slowest rank's device time."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def step_stats(ms):
    """Median, p10 and p90 of per-step times in µs (the single value when
    only one step ran)."""
    us = sorted(1e3 * float(x) for x in ms)
    if not us:
        return None
    if len(us) == 1:
        return {"median_us": round(us[0], 2), "p10_us": round(us[0], 2), "p90_us": round(us[0], 2)}
    dec = statistics.quantiles(us, n=10, method="inclusive")
    return {"median_us": round(statistics.median(us), 2), "p10_us": round(dec[0], 2),
            "p90_us": round(dec[-1], 2)}


def whole_job_tflops(flops_per_step, steps_per_rank, world, max_ms):
    """Every rank's work over the slowest rank's time (weak scaling)."""
    return world * flops_per_step * steps_per_rank / (max_ms * 1e-3) / 1e12


# -------------------------------------------------------- oracle (CPU) ---

def oracle_sample(X_bits, inv, L1_bits, L2_bits, R, bias_bits, M, K, N, r, target_s):
    """Time the oracle's forward (activation step + linear) on a bounded row
    sample; returns (TFLOP/s, rows, seconds, threads)."""
    import oracle
    rc, rs = oracle.pack_residual(R)  # per-weight preparation, not timed

    out = {}

    def run(rows):
        t0 = time.perf_counter()
        xc, xs, T = oracle.quantize_act(X_bits[:rows], inv, L1_bits, r)
        out["Y"] = oracle.linear_rows(xc, xs, T, rc, rs, L2_bits, bias_bits, rows, K, N, r, np.arange(rows))
        return time.perf_counter() - t0

    # grow the sample until it takes about target_s (small samples leave most
    # OpenMP threads idle, so one probe underestimates the rate)
    rows = min(M, 2 * oracle.num_threads())
    t = run(rows)
    for _ in range(4):
        if t >= 0.6 * target_s or rows >= M:
            break
        rows = int(max(rows + 1, min(M, rows * 0.9 * target_s / max(t, 1e-3))))
        t = run(rows)
    return layer_flops(rows, K, N, r) / t / 1e12, rows, t, oracle.num_threads(), out["Y"]


def rel_err(Y, ref) -> float:
    """Relative Frobenius error of Y against ref (fp64 host arrays or device tensors)."""
    import torch
    if isinstance(Y, torch.Tensor):
        Y = Y.double()
        ref = ref.double()
        return float(torch.linalg.norm(Y - ref) / torch.linalg.norm(ref))
    return float(np.linalg.norm(Y - ref) / np.linalg.norm(ref))


def quality_stats(L, Y):
    """The layer's quantisation error against the unquantised product X W +
    bias (fp32 device matmul of the bf16 operands, a statistic only), for the
    output `Y` of the timed path and for the same layer with per-tensor
    global scales (NVFP4 two-level scaling)."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import prep
    X, W, bias = L["X"], L["W"], L["bias"]
    ref = X.float() @ W.float()
    if bias is not None:
        ref += bias.float()[None, :]
    out = {"reference": "unquantised X W + bias, fp32 device matmul of the bf16 operands",
           "rel_err_gpu": round(rel_err(Y, ref), 5)}
    gx = prep.activation_global_scale(X.abs().amax(dim=0).float(), L["inv"])
    gw = prep.global_scale(float(L["R"].abs().max()))
    inv_s, L2_s, R_s, alpha = prep.apply_global_scales(L["inv"], L["L2"], L["R"], gx, gw)
    rc, rs = svdq.pack_residual(R_s)
    xc, xs, T = svdq.quantize_act(X, inv_s, L["L1"])
    Yg = svdq.linear(xc, xs, T, rc, rs, L2_s, bias, L["M"], L["K"], L["N"], alpha=alpha)
    out["rel_err_gpu_global_scale"] = round(rel_err(Yg, ref), 5)
    out["global_scales"] = {"g_x": gx, "g_w": gw}
    return out, ref


# ------------------------------------------------------------- our arm ---

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import bit_w4a4_quantized_smooth_b200 as svdq

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    L = setup_layer(args.workload, device)
    M, K, N, r = L["M"], L["K"], L["N"], L["r"]
    X, inv, L1, L2, bias, rc, rs = L["X"], L["inv"], L["L1"], L["L2"], L["bias"], L["rc"], L["rs"]
    cb, sb = svdq.packed_sizes(M, K)
    xc = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
    xs = torch.empty(sb, dtype=torch.uint8, device=device)
    T = torch.empty((M, r), dtype=torch.bfloat16, device=device) if r else None
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    flush_rd = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def flush_l2():
        # write a buffer larger than L2, then read another one: every line the
        # timed step finds in L2 is clean and none of its inputs, so the step
        # pays neither hits nor the write-back of the flush's dirty lines
        flush.zero_()
        flush_rd.sum()

    def step():
        svdq.quantize_act(X, inv, L1, x_codes=xc, x_scales=xs, T=T, stream=stream)
        svdq.linear(xc, xs, T, rc, rs, L2, bias, M, K, N, Y=Y, stream=stream)

    for _ in range(max(3, args.warmup)):
        flush_l2()
        step()
    torch.cuda.synchronize()
    st, where = svdq.sync_status()
    if st != 0:
        raise RuntimeError(f"kernel wait expired during warm-up (id {where})")

    # the timed steps: the layer's two launches back to back on one stream,
    # as a caller runs them, an event on either side of each step
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush_l2()
        e0, e2 = ev[i]
        e0.record(stream)
        svdq.quantize_act(X, inv, L1, x_codes=xc, x_scales=xs, T=T, stream=stream)
        svdq.linear(xc, xs, T, rc, rs, L2, bias, M, K, N, Y=Y, stream=stream)
        e2.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), device)
    st, where = svdq.sync_status()
    if st != 0:
        raise RuntimeError(f"kernel wait expired in the timed region (id {where})")

    flops = layer_flops(M, K, N, r)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(flops, args.steps, world, total_ms)

    # ---- per-kernel figures (this rank): the same steps with an event
    # between the two launches ----
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush_l2()
        e0, e1, e2 = evk[i]
        e0.record(stream)
        svdq.quantize_act(X, inv, L1, x_codes=xc, x_scales=xs, T=T, stream=stream)
        e1.record(stream)
        svdq.linear(xc, xs, T, rc, rs, L2, bias, M, K, N, Y=Y, stream=stream)
        e2.record(stream)
    torch.cuda.synchronize()
    qa_us = 1e3 * statistics.mean(e[0].elapsed_time(e[1]) for e in evk)
    lin_us = 1e3 * statistics.mean(e[1].elapsed_time(e[2]) for e in evk)

    # host cost of one step through the Python binding (argument checks, the
    # cached tensor maps, the two launches), on the CPU clock while the GPU
    # runs behind; no flush, nothing synchronised inside the loop
    host_steps = 50
    t_host = time.perf_counter()
    for _ in range(host_steps):
        step()
    host_us = (time.perf_counter() - t_host) * 1e6 / host_steps
    torch.cuda.synchronize()

    # plain FP4 GEMM (rank 0 branch switched off) on the same operands, for
    # the low-rank overhead
    def time_linear(rr, reps=20):
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for a, b in es:
            flush_l2()
            a.record(stream)
            svdq.linear(xc, xs, T if rr else None, rc, rs, L2 if rr else None, bias, M, K, N, Y=Y,
                        stream=stream)
            b.record(stream)
        torch.cuda.synchronize()
        return 1e3 * statistics.mean(a.elapsed_time(b) for a, b in es)

    lin_r0_us = time_linear(0) if r else lin_us

    # the activation step with GELU fused (svdq_quantize_act_gelu) on the same X
    def time_qa_gelu(reps=20):
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in es:
            flush_l2()
            a.record(stream)
            svdq.quantize_act(X, inv, L1, x_codes=xc, x_scales=xs, T=T, stream=stream, gelu=True)
            b.record(stream)
        torch.cuda.synchronize()
        return 1e3 * statistics.mean(a.elapsed_time(b) for a, b in es)

    qa_gelu_us = time_qa_gelu()

    # residual packer, once per weight
    pk = []
    for _ in range(10):
        flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        svdq.pack_residual(L["R"], r_codes=rc, r_scales=rs, stream=stream)
        b.record(stream)
        pk.append((a, b))
    torch.cuda.synchronize()
    pack_us = 1e3 * statistics.mean(a.elapsed_time(b) for a, b in pk)

    # ---- end to end through the public API with host buffers ----
    # A serving loop's schedule: three streams (host->device copy of X, the
    # layer, device->host copy of Y) with double-buffered X and Y on the
    # device, so that step i's copies overlap steps i-1 and i+1.  Every step
    # still copies its own X in from pinned memory and its own Y out.  No L2
    # flush inside this region: each step streams its fresh X and Y through
    # L2, while the packed weights (a few tens of MB) may stay L2-resident
    # from one step to the next, as they would in a serving loop.
    X_host = torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True)
    X_host.copy_(X)
    Y_host = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    X_dev = [torch.empty_like(X) for _ in range(2)]
    Y_dev = [torch.empty_like(Y) for _ in range(2)]
    s_in = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # X_dev[b] holds this step's X
    ev_used = [torch.cuda.Event() for _ in range(2)]  # the layer is done with X_dev[b], Y_dev[b] written
    ev_out = [torch.cuda.Event() for _ in range(2)]   # Y_dev[b] copied to the host

    def run_e2e(nsteps):
        for i in range(nsteps):
            b = i & 1
            if i >= 2:
                s_in.wait_event(ev_used[b])
            with torch.cuda.stream(s_in):
                X_dev[b].copy_(X_host, non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])
            svdq.quantize_act(X_dev[b], inv, L1, x_codes=xc, x_scales=xs, T=T, stream=stream)
            svdq.linear(xc, xs, T, rc, rs, L2, bias, M, K, N, Y=Y_dev[b], stream=stream)
            ev_used[b].record(stream)
            s_out.wait_event(ev_used[b])
            with torch.cuda.stream(s_out):
                Y_host[b].copy_(Y_dev[b], non_blocking=True)
            ev_out[b].record(s_out)

    run_e2e(max(3, args.warmup))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_last_out = torch.cuda.Event()
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    s_in.wait_event(t_start)
    run_e2e(args.steps)
    t_last_out.record(s_out)
    stream.wait_event(t_last_out)
    t_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t_start.elapsed_time(t_end), device)
    e2e_value = whole_job_tflops(flops, args.steps, world, e2e_ms)

    peaks = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    # the linear kernel's own work: the FP4 product and the rank-r up-projection
    lin_flops = 2.0 * M * N * K + 2.0 * M * N * r
    achieved = lin_flops / (lin_us * 1e-6) / 1e12
    qa_bytes = 2 * M * K + M * K // 2 + M * K // 16 + 2 * M * r + 2 * K * r + 4 * K
    layer_roof_us = max(flops / (fp4_peak * 1e12), linear_bytes(M, K, N, r) / (peaks["hbm_gbs"] * 1e9)) * 1e6

    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4",
        "data": "synthetic",
        "config": dict(workload_desc(args.workload, M, K, N, r), parallelism=f"replicas{world}"),
        "us_per_layer": round(1e3 * ms_per_step, 2),
        "step_us": step_stats(step_ms),
        "quantize_act_us": round(qa_us, 2),
        "quantize_act_gelu_us": round(qa_gelu_us, 2),
        "linear_us": round(lin_us, 2),
        "linear_r0_us": round(lin_r0_us, 2),
        "lowrank_overhead": round(lin_us / lin_r0_us - 1.0, 4),
        "pack_residual_us": round(pack_us, 2),
        "pack_residual_gbs": round((K * N * 4 + N * K // 2 + N * K // 16) / (pack_us * 1e-6) / 1e9, 1),
        "quantize_act_gbs": round(qa_bytes / (qa_us * 1e-6) / 1e9, 1),
        "host_us_per_step": round(host_us, 2),
        "layer_roofline_us": round(layer_roof_us, 2),
        "layer_roofline_frac": round(layer_roof_us / (1e3 * ms_per_step), 4),
        "roofline": {
            "kernel": "linear_kernel",
            "bound": "tensor",
            "achieved": round(achieved, 1),
            "peak": round(fp4_peak, 1),
            "unit": "TFLOP/s",
            "frac": round(achieved / fp4_peak, 4),
            "traffic": linear_traffic(args.workload),
            "traffic_note": "DRAM bytes of one launch from an ncu capture with L2 warm "
                            "(bench.py --once linear); null when the kernel changed since",
            "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s x 4 (FP4/bf16 dense ratio)",
        },
        "spec_sheet": {"fp4_tflops": SPEC_FP4_TFLOPS, "hbm_gbs": SPEC_HBM_GBS,
                       "linear_frac": round(achieved / SPEC_FP4_TFLOPS, 4),
                       "layer_roofline_frac": round(max(flops / (SPEC_FP4_TFLOPS * 1e12),
                                                        linear_bytes(M, K, N, r) / (SPEC_HBM_GBS * 1e9))
                                                    * 1e6 / (1e3 * ms_per_step), 4)},
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT,
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
                "ms_per_step": round(e2e_ms / args.steps, 4),
                "schedule": "copy-in, layer and copy-out streams, double-buffered X and Y"},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
    }
    # library-achieved FP4 rate (outside every timed region): cuBLASLt's
    # NVFP4 GEMM at 8192^3 and on this layer's FP4 product
    lib, api = library_fp4_times(device, flush_l2, [LIBRARY_FP4_PEAK_SHAPE, (M, N, K)])
    if lib is None:
        out["fp4_library"] = {"unavailable": api}
    else:
        pm, pn, pk = LIBRARY_FP4_PEAK_SHAPE
        lib_peak = 2.0 * pm * pn * pk / (lib[LIBRARY_FP4_PEAK_SHAPE] * 1e-6) / 1e12
        out["fp4_library"] = {
            "api": api, "peak_shape": f"{pm}x{pn}x{pk}", "peak_tflops": round(lib_peak, 1),
            "linear_frac": round(achieved / lib_peak, 4),
            "same_shape_us": round(lib[(M, N, K)], 2),
            "note": "library-achieved FP4 rate (random codes, unit scales, L2 flushed); the FP4 product "
                    "only (no low-rank branch, no bias); not on the layer's path"}
    # quality statistic, outside every timed region: the timed path's Y
    # (recomputed: the r = 0 loop above overwrote the buffer) against the
    # unquantised product
    step()
    torch.cuda.synchronize()
    out["quality"], L["quality_ref"] = quality_stats(L, Y)
    return out, L


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    if args.no_overlap:
        import bit_w4a4_quantized_smooth_b200 as svdq
        svdq.set_launch_overlap(False)
    if args.once:
        return run_once(args)
    if args.sweep:
        return run_sweep(args)
    if args.stack:
        return run_stack(args)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        out, L = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            li = L["li"]
            to_np = lambda t: None if t is None else t.detach().cpu().contiguous()
            bits = lambda t: None if t is None else to_np(t).view(torch.int16).numpy().view(np.uint16)
            v, rows, secs, thr, Yo = oracle_sample(li.X, to_np(L["inv"]).numpy(), bits(L["L1"]),
                                                   bits(L["L2"]), to_np(L["R"]).numpy(), li.bias,
                                                   L["M"], L["K"], L["N"], L["r"], args.cpu_seconds)
            out["cpu_baseline"] = {"value": round(v, 6), "unit": UNIT, "cores": thr, "kind": "oracle",
                                   "sample": f"{rows} of {L['M']} rows (activation step + linear), "
                                             f"{secs:.1f} s, fp64 OpenMP"}
            if "quality" in out:
                ref = L["quality_ref"][:rows].double().cpu().numpy()
                out["quality"]["rel_err_oracle"] = round(rel_err(Yo, ref), 5)
                out["quality"]["oracle_rows"] = rows
        if world == 1 and not args.no_stack:
            # the whole synthetic DiT stack, one CUDA graph per pass (3 s of
            # preparation on the device, well under a second of timing)
            del L
            torch.cuda.empty_cache()
            t0 = time.perf_counter()
            layers = prepare_stack(torch.device("cuda", local_rank))
            prep_s = time.perf_counter() - t0
            g_ms, e_ms, launches = time_stack(layers, torch.device("cuda", local_rank))
            out["stack"] = stack_summary(layers, g_ms, e_ms, launches, prep_s, load_peaks())
            del layers
        out["launch_overlap"] = not args.no_overlap
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


def run_once(args):
    """Three launches of one kernel on the workload, no timing, no L2 flush:
    the command that profiler captures of a single kernel run."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    L = setup_layer(args.workload, device, M=args.rows)
    M, K, N, r = L["M"], L["K"], L["N"], L["r"]
    xc, xs, T = svdq.quantize_act(L["X"], L["inv"], L["L1"])
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    for _ in range(3):
        if args.once in ("quantize_act", "quantize_act_gelu"):
            svdq.quantize_act(L["X"], L["inv"], L["L1"], x_codes=xc, x_scales=xs, T=T,
                              gelu=args.once == "quantize_act_gelu")
        elif args.once == "linear":
            svdq.linear(xc, xs, T, L["rc"], L["rs"], L["L2"], L["bias"], M, K, N, Y=Y)
        else:
            svdq.pack_residual(L["R"], r_codes=L["rc"], r_scales=L["rs"])
    torch.cuda.synchronize()
    st, where = svdq.sync_status()
    if st != 0:
        raise RuntimeError(f"kernel wait expired (id {where})")
    print(json.dumps({"once": args.once, "workload": args.workload, "M": M, "K": K, "N": N, "r": r}))
    return 0


SPEC_FP4_TFLOPS = 9000.0   # B200 dense FP4 (the spec sheet's 18 PF is 2:4 sparse)
SPEC_HBM_GBS = 8000.0


def run_sweep(args):
    """The memory-bound sweep at K = N = 3072: every M in SWEEP_M and rank in
    SWEEP_R, one W and one smoothing calibration (4608 rows) for all points,
    the SVD taken once per rank, X the leading M rows of one draw.  Each point
    times the layer (quantize_act + linear) with L2 flushed before every rep
    and reports TFLOP/s and the layer's algorithmic bytes per second."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import prep
    from svdq_inputs import make_layer_inputs
    from svdq_inputs.workloads import SWEEP_M, SWEEP_R
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    li = make_layer_inputs("sweep_3072", M=max(SWEEP_M), r=max(SWEEP_R), cal_rows=4608)

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)

    X, W, Xcal = bf16(li.X), bf16(li.W), bf16(li.Xcal)
    bias = None if li.bias is None else bf16(li.bias)
    lam, inv = prep.smoothing(Xcal, W)
    K, N = li.K, li.N
    peaks = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    flush_rd = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.float32, device=device)
    reps = max(5, min(args.steps, 20))
    for r in SWEEP_R:
        L1, L2, R = prep.lowrank(W, lam, r)
        rc, rs = svdq.pack_residual(R)
        del R
        for M in SWEEP_M:
            Xm = X[:M]
            xc, xs, T = svdq.quantize_act(Xm, inv, L1)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            for _ in range(3):
                svdq.quantize_act(Xm, inv, L1, x_codes=xc, x_scales=xs, T=T)
                svdq.linear(xc, xs, T, rc, rs, L2, bias, M, K, N, Y=Y)
            # the step (both launches back to back), then the per-kernel times
            # from the same steps with an event between the launches
            steps, ev = [], []
            for _ in range(reps):
                flush.zero_()
                flush_rd.sum()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record()
                svdq.quantize_act(Xm, inv, L1, x_codes=xc, x_scales=xs, T=T)
                svdq.linear(xc, xs, T, rc, rs, L2, bias, M, K, N, Y=Y)
                e[1].record()
                steps.append(e)
            for _ in range(reps):
                flush.zero_()
                flush_rd.sum()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                e[0].record()
                svdq.quantize_act(Xm, inv, L1, x_codes=xc, x_scales=xs, T=T)
                e[1].record()
                svdq.linear(xc, xs, T, rc, rs, L2, bias, M, K, N, Y=Y)
                e[2].record()
                ev.append(e)
            torch.cuda.synchronize()
            st, where = svdq.sync_status()
            if st != 0:
                raise RuntimeError(f"kernel wait expired (id {where})")
            qa_us = 1e3 * statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
            lin_us = 1e3 * statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
            us = 1e3 * statistics.mean(e[0].elapsed_time(e[1]) for e in steps)
            flops = layer_flops(M, K, N, r)
            nbytes = linear_bytes(M, K, N, r)
            roof_us = max(flops / (fp4_peak * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9)) * 1e6
            print(json.dumps({
                "sweep": "K=N=3072", "M": M, "rank": r, "us_per_layer": round(us, 2),
                "quantize_act_us": round(qa_us, 2), "linear_us": round(lin_us, 2),
                "tflops": round(flops / (us * 1e-6) / 1e12, 2),
                "algorithmic_gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
                "bound": "tensor" if flops / (fp4_peak * 1e12) > nbytes / (peaks["hbm_gbs"] * 1e9) else "hbm",
                "roofline_frac": round(roof_us / us, 4), "reps": reps,
                "l2": "flushed before every rep", "launch_overlap": not args.no_overlap}), flush=True)
    return 0


STACK_M = 4608


def stack_shape_counts():
    """{(K, N): number of stack layers of that shape}."""
    from svdq_inputs import stack_layer_shapes
    counts = {}
    for K, N, _ in stack_layer_shapes():
        counts[(K, N)] = counts.get((K, N), 0) + 1
    return counts


def is_mlp_down(i: int) -> bool:
    """Stack layer i is a double-stream block's MLP down-projection."""
    return i < 76 and i % 4 == 3


def prepare_stack(device, M=STACK_M, layer_ids=None):
    """Draw and prepare the layers of the synthetic DiT stack (all 152 by
    default) on the device, untimed: smoothing, rank-32 randomized SVD, the
    rank-32 LoRA adapter joined to the low-rank branch (effective rank 64, R
    not re-quantised), R packed to NVFP4.  A double-stream block's MLP
    down-projection that directly follows its up-projection is chained: its
    input is GELU of the up-projection's output, applied inside its
    activation step (svdq_quantize_act_gelu), and its smoothing statistics
    come from that output; every other layer reads its own synthetic
    activations."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import prep
    from svdq_inputs import stack_layer_shapes, torch_gen
    layers = []
    for i in (range(len(stack_layer_shapes())) if layer_ids is None else layer_ids):
        chain = is_mlp_down(i) and bool(layers) and layers[-1]["id"] == i - 1
        d = torch_gen.make_stack_layer(i, M, device, with_x=not chain)
        if chain:
            up = layers[-1]
            xc, xs, T = svdq.quantize_act(up["X"], up["inv"], up["L1"], gelu=up["gelu"])
            Yup = svdq.linear(xc, xs, T, up["rc"], up["rs"], up["L2"], None, M, up["K"], up["N"])
            amax = torch.nn.functional.gelu(Yup.float()).abs().amax(dim=0)  # calibration statistic only
            lam, inv = prep.smoothing_from_stats(amax, d["W"])
            del xc, xs, T, Yup
        else:
            lam, inv = prep.smoothing(d["X"], d["W"])
        L1, L2, R = prep.lowrank_randomized(d["W"], lam, 32, seed=i)
        del d["W"]
        L1, L2 = svdq.attach_lora(L1, L2, lam, d["A"], d["B"])
        rc, rs = svdq.pack_residual(R)
        del R
        layers.append(dict(id=i, X=d["X"], gelu=chain, inv=inv, L1=L1, L2=L2, rc=rc, rs=rs, K=d["K"], N=d["N"]))
    torch.cuda.synchronize()
    return layers


def stack_pass_fn(layers, device, M=STACK_M, Y_out=None):
    """One pass over the stack in layer order on the current stream, into
    buffers shared by all layers (sized for the widest): the activation
    codes, scales and T of layer i are consumed by its linear before layer
    i + 1 overwrites them.  Y goes to one shared buffer too, or to the
    per-layer tensors of `Y_out`.  Allocates nothing when called."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import binding
    Kmax = max(L["K"] for L in layers)
    Nmax = max(L["N"] for L in layers)
    rmax = max(L["L1"].shape[1] for L in layers)
    xc = torch.empty(M * Kmax // 2, dtype=torch.uint8, device=device)
    xs = torch.empty(svdq.packed_sizes(M, Kmax)[1], dtype=torch.uint8, device=device)
    T = torch.empty(M * rmax, dtype=torch.bfloat16, device=device)
    Y = torch.empty(M * Nmax, dtype=torch.bfloat16, device=device)
    ws_bytes = max(binding.quantize_act_workspace_bytes(M, L["K"], L["L1"].shape[1]) for L in layers)
    ws = torch.zeros(max(ws_bytes, 1 << 20), dtype=torch.uint8, device=device)
    views = []
    for L in layers:
        K, N, r = L["K"], L["N"], L["L1"].shape[1]
        views.append((xc[: M * K // 2].view(M, K // 2), xs[: svdq.packed_sizes(M, K)[1]],
                      T[: M * r].view(M, r), Y[: M * N].view(M, N) if Y_out is None else Y_out[len(views)]))
    # a chained layer reads the previous layer's output (in stream order: the
    # previous linear has written it, and this layer's activation step reads
    # it before its own linear overwrites the shared buffer)
    inputs = [views[j - 1][3] if L["gelu"] else L["X"] for j, L in enumerate(layers)]

    def run():
        for L, Xk, (xck, xsk, Tk, Yk) in zip(layers, inputs, views):
            svdq.quantize_act(Xk, L["inv"], L["L1"], x_codes=xck, x_scales=xsk, T=Tk, workspace_buf=ws,
                              gelu=L["gelu"])
            svdq.linear(xck, xsk, Tk, L["rc"], L["rs"], L["L2"], None, M, L["K"], L["N"], Y=Yk)
    return run


def stack_roofline_ms(layers, peaks, M=STACK_M):
    """Sum over the layers of each layer's roofline time (the slower of its
    FP4 FLOPs at the measured FP4 peak and its bytes at the measured HBM
    rate)."""
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    tot = 0.0
    for L in layers:
        K, N, r = L["K"], L["N"], L["L1"].shape[1]
        tot += max(layer_flops(M, K, N, r) / (fp4_peak * 1e12), linear_bytes(M, K, N, r) / (peaks["hbm_gbs"] * 1e9))
    return tot * 1e3


def time_stack(layers, device, passes=10, warmup=3):
    """-> (ms per pass replayed from a CUDA graph, ms per pass launched
    eagerly, launches per pass).  Inputs (10 GB of activations, 3.6 GB of
    packed weights) are far larger than L2, so no flush is needed."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    run = stack_pass_fn(layers, device)
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()

    def timed(fn, n):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, b in ev:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    eager_ms = timed(run, max(3, passes // 2))
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()  # the capture stream's own warm-up
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        run()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    graph_ms = timed(g.replay, passes)
    st, where = svdq.sync_status()
    if st != 0:
        raise RuntimeError(f"kernel wait expired in the stack (id {where})")
    del g
    return graph_ms, eager_ms, 2 * len(layers)


def stack_summary(layers, graph_ms, eager_ms, launches, prep_s, peaks, M=STACK_M):
    flops = sum(layer_flops(M, L["K"], L["N"], L["L1"].shape[1]) for L in layers)
    roof = stack_roofline_ms(layers, peaks, M)
    wbytes = sum(L["rc"].numel() + L["rs"].numel() + 2 * (L["L1"].numel() + L["L2"].numel()) for L in layers)
    return {
        "workload": "synthetic 12B DiT stack: 19 double-stream blocks (QKV 3072->9216, out 3072->3072, "
                    "MLP 3072->12288->3072) + 38 single-stream blocks (fused 3072->21504, 15360->3072), "
                    f"M={M}, rank 32 + LoRA 32 (effective 64), no bias; each MLP down-projection reads "
                    "GELU of its up-projection's output (GELU fused into its activation step)",
        "chained_layers": sum(1 for L in layers if L["gelu"]),
        "layers": len(layers), "ms_per_pass": round(graph_ms, 3), "ms_per_pass_eager": round(eager_ms, 3),
        "tflops": round(flops / (graph_ms * 1e-3) / 1e12, 1),
        "roofline_ms": round(roof, 3), "roofline_frac": round(roof / graph_ms, 4),
        "gpu_launches_per_pass": launches, "packed_weight_gb": round(wbytes / 1e9, 3),
        "schedule": "one CUDA graph of the 304 launches (quantize_act + linear per layer), one stream",
        "prep_s": round(prep_s, 1),
    }


def stack_cpu_baseline(rows=8):
    """The oracle (activation step + linear, rank 64) timed on `rows` rows of
    every distinct stack shape, extrapolated by rows and layer counts to the
    whole pass.  The operands are stand-ins of the right sizes (R = W, zero
    low-rank factors, unit smoothing): the oracle's cost does not depend on
    the values.  -> (seconds per pass, threads, sample description)."""
    import oracle
    from svdq_inputs import make_stack_layer_inputs, stack_layer_shapes
    first = {}
    for i, (K, N, _) in enumerate(stack_layer_shapes()):
        first.setdefault((K, N), i)
    r = 64
    total_s = 0.0
    for (K, N), n_layers in stack_shape_counts().items():
        li = make_stack_layer_inputs(first[(K, N)], M=rows)
        R = (np.asarray(li.W, dtype=np.uint32) << 16).view(np.float32)
        rc, rs = oracle.pack_residual(R)
        inv = np.ones(K, dtype=np.float32)
        L1 = np.zeros((K, r), dtype=np.uint16)
        L2 = np.zeros((r, N), dtype=np.uint16)
        t0 = time.perf_counter()
        if K == 12288:  # the MLP down-projections: GELU inside the activation step
            xc, xs, T = oracle.quantize_act_gelu(li.X[:rows], inv, L1, r)
        else:
            xc, xs, T = oracle.quantize_act(li.X[:rows], inv, L1, r)
        oracle.linear_rows(xc, xs, T, rc, rs, L2, None, rows, K, N, r, np.arange(rows))
        total_s += (time.perf_counter() - t0) * (STACK_M / rows) * n_layers
    return total_s, oracle.num_threads(), (f"{rows} rows of each of the {len(first)} distinct layer shapes, "
                                           f"extrapolated to {STACK_M} rows x 152 layers; stand-in operands")


def run_stack(args):
    import torch
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    t0 = time.perf_counter()
    layers = prepare_stack(device)
    prep_s = time.perf_counter() - t0
    graph_ms, eager_ms, launches = time_stack(layers, device, passes=max(5, min(args.steps, 20)),
                                              warmup=max(3, args.warmup))
    out = {"stack": stack_summary(layers, graph_ms, eager_ms, launches, prep_s, load_peaks())}
    if not args.no_cpu_baseline:
        secs, thr, sample = stack_cpu_baseline()
        out["stack"]["cpu_baseline"] = {"ms_per_pass": round(secs * 1e3, 1), "cores": thr, "kind": "oracle",
                                        "sample": sample}
    out["launch_overlap"] = not args.no_overlap
    print(json.dumps(out), flush=True)
    return 0


def run_reference(args):
    """The oracle (plain CPU implementation) on the same workload and metric."""
    import oracle
    from svdq_inputs import make_layer_inputs
    li = make_layer_inputs(args.workload)
    lam, inv = oracle.smooth(li.Xcal, li.W)
    L1, L2, R, _ = oracle.lowrank(li.W, lam, li.r)
    rc, rs = oracle.pack_residual(R)
    M, K, N, r = li.M, li.K, li.N, li.r
    per_step_s = max(0.5, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    # rows per step sized from one probe
    t0 = time.perf_counter()
    xc, xs, T = oracle.quantize_act(li.X[:4], inv, L1 if r else None, r)
    oracle.linear_rows(xc, xs, T, rc, rs, L2 if r else None, li.bias, 4, K, N, r, np.arange(4))
    probe = time.perf_counter() - t0
    rows = int(max(1, min(M, 4 * per_step_s / max(probe, 1e-3))))
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        xc, xs, T = oracle.quantize_act(li.X[:rows], inv, L1 if r else None, r)
        oracle.linear_rows(xc, xs, T, rc, rs, L2 if r else None, li.bias, rows, K, N, r, np.arange(rows))
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = layer_flops(rows, K, N, r) * len(times) / total / 1e12
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": UNIT,
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / len(times), 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        # the same workload description as our arm's line; where it ran is in cpu_baseline
        "config": dict(workload_desc(args.workload, M, K, N, r), parallelism=f"replicas{args.gpus}"),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle", "device": "host cores (rank 0)",
                         "sample": f"{rows} of {M} rows per step"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


if __name__ == "__main__":
    sys.exit(main())
