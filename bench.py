"""Benchmark: one NVFP4 MLP block step (fwd + bwd) of a 12B hybrid
Mamba-Transformer layer shape on B200, through the C ABI.

A step = up-projection Fprop, squared ReLU, down-projection Fprop, then both
layers' Dgrad and Wgrad (RHT + SR on the Wgrad operands): 12 NVFP4 operands
from two-pass quantisations (each weight's two operands from one read), 6
block-scaled NVFP4 GEMMs, 2 elementwise kernels.  With N > 1
GPUs (torchrun) every rank runs the step on its own token shard and the weight
gradients are summed over NCCL (weak scaling).

Prints one JSON line.  `value` = GEMM FLOPs of all ranks / device step time
(max over ranks).  `e2e` = the same through the public calls with pinned host
inputs copied in and the block output copied back every step (on copy streams,
double-buffered, overlapping the neighbouring steps' compute).  `--impl
reference` times the CPU oracle on a bounded sample of the same step instead.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_bit_precision_quantize_b200 import dp  # noqa: E402
from nvfp4_bit_precision_quantize_b200 import workloads as W  # noqa: E402

METRIC = "NVFP4 GEMM TFLOPS and quantize GB/s on 1 B200, % of FP4/HBM peak"
M_TOK, HID, FFN = W.TOKENS, W.HIDDEN, W.FFN
GEMM_FLOPS = 6 * 2 * M_TOK * HID * FFN            # 1.031e13 per step per GPU
SEED = 1234
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
FP4_PER_BF16 = 4.0                                 # nominal dense ratio 9 / 2.25 PFLOP/s
WORKLOAD = ("mlp_fwd_bwd: tokens 8192, hidden 5120, ffn 20480, up -> relu^2 -> down; "
            "6 NVFP4 GEMMs + 12 NVFP4 operands (8 single quantisations, 2 dual-orientation ones for the "
            "weights; RHT+SR on Wgrad operands) + 2 relu^2 kernels that also return max|out| and max|RHT(out)| "
            "for the two quantisations of their output")
QUANT_BYTES_SINGLE = 4.5625   # bf16, two passes: read 2 + 2, write 0.5 + 1/16 bytes per element
QUANT_BYTES_DUAL = 5.125      # bf16, two passes, two outputs: read 2 + 2, write 2 x (0.5 + 1/16)
QUANT_BYTES_AMAX_IN = 2.5625  # bf16, amax supplied by the producer: read 2, write 0.5 + 1/16
MX_BYTES = 2.53125            # bf16 MXFP4: read 2, write 0.5 + 1/32


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK, "fallback"


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# -------------------------------------------------------------- the GPU step
class MlpStep:
    """Device buffers and the C-ABI call sequence of one MLP block step."""

    def __init__(self, B, device, data_seed=None):
        self.B = B
        w = W.mlp(seed=5, data_seed=data_seed)
        pin = lambda a: W.bits_to_torch_bf16(a).pin_memory()  # noqa: E731
        self.host = {k: pin(v) for k, v in w.items()}
        self.d = {k: v.to(device, non_blocking=True) for k, v in self.host.items()}
        bf = dict(dtype=torch.bfloat16, device=device)
        self.Y1 = torch.empty((M_TOK, FFN), **bf)
        self.h = torch.empty_like(self.Y1)
        self.Y2 = torch.empty((M_TOK, HID), **bf)
        self.dh = torch.empty_like(self.Y1)
        self.dY1 = torch.empty_like(self.Y1)
        self.dX = torch.empty((M_TOK, HID), **bf)
        self.dW1 = torch.empty((FFN, HID), dtype=torch.float32, device=device)
        self.dW2 = torch.empty((HID, FFN), dtype=torch.float32, device=device)
        self.ws = B.workspace(max(B.nvfp4_linear_workspace_size(M_TOK, FFN, HID),
                                  B.nvfp4_linear_workspace_size(M_TOK, HID, FFN)), device)
        self.qws = B.workspace(B.nvfp4_quantize_dual_workspace_size(), device)
        self.amax_h = torch.zeros(4, dtype=torch.float32, device=device)    # max|h|, from relu^2
        self.amax_dy1 = torch.zeros(4, dtype=torch.float32, device=device)  # max|dY1|, from relu^2 bwd
        self.amax_h_rht = torch.zeros(4, dtype=torch.float32, device=device)     # max|RHT(h)|
        self.amax_dy1_rht = torch.zeros(4, dtype=torch.float32, device=device)   # max|RHT(dY1)|
        mk = B.empty_nvfp4
        # NVFP4 operands of the explicit call sequence (same work as linear_fwd/bwd)
        self.q = {
            "X_r": mk(M_TOK, HID, device), "W1_r": mk(FFN, HID, device), "h_r": mk(M_TOK, FFN, device),
            "W2_r": mk(HID, FFN, device),
            "dY2_r": mk(M_TOK, HID, device), "W2_c": mk(FFN, HID, device), "dY2_c": mk(HID, M_TOK, device),
            "h_c": mk(FFN, M_TOK, device),
            "dY1_r": mk(M_TOK, FFN, device), "W1_c": mk(HID, FFN, device), "dY1_c": mk(FFN, M_TOK, device),
            "X_c": mk(HID, M_TOK, device),
        }
        self.launches = 0
        torch.cuda.synchronize()

    def _quant(self, x, key, colwise=False, sr=False, rht=False, amax_in=None, ev=None):
        B = self.B
        B.nvfp4_quantize(x, orientation=B.NVFP4_COLWISE if colwise else B.NVFP4_ROWWISE,
                         rounding=B.NVFP4_SR if sr else B.NVFP4_RTN, rht=rht, seed=SEED, amax_in=amax_in,
                         out=self.q[key], ws=self.qws)
        self.launches += B.nvfp4_last_launch_count()
        if ev is not None:
            per_elem = QUANT_BYTES_AMAX_IN if amax_in is not None else QUANT_BYTES_SINGLE
            ev.append(("quant", x.numel() * per_elem, torch.cuda.Event(enable_timing=True)))
            ev[-1][2].record()

    def _dual(self, x, key_r, key_c, sr=False, rht=False, ev=None):
        """Rowwise RTN and colwise operands of one tensor from one read."""
        B = self.B
        B.nvfp4_quantize_dual(x, col_rounding=B.NVFP4_SR if sr else B.NVFP4_RTN, col_rht=rht, seed=SEED,
                              out_row=self.q[key_r], out_col=self.q[key_c], ws=self.qws)
        self.launches += B.nvfp4_last_launch_count()
        if ev is not None:
            ev.append(("quant", x.numel() * QUANT_BYTES_DUAL, torch.cuda.Event(enable_timing=True)))
            ev[-1][2].record()

    def _gemm(self, a, b, out, ev=None):
        B = self.B
        B.nvfp4_gemm(self.q[a], self.q[b], out=out, ws=self.ws)
        self.launches += B.nvfp4_last_launch_count()
        if ev is not None:
            ev.append(("gemm", 2 * self.q[a].rows * self.q[b].rows * self.q[a].k,
                        torch.cuda.Event(enable_timing=True)))
            ev[-1][2].record()

    def device_step(self, ev=None):
        """Explicit C-ABI sequence; events (if given) mark the end of every call."""
        B, d = self.B, self.d
        if ev is not None:
            ev.append(("start", 0, torch.cuda.Event(enable_timing=True)))
            ev[-1][2].record()
        # forward.  A weight's two operands (rowwise, colwise without RHT) come from one
        # dual-orientation call; where the colwise operand carries the Hadamard transform
        # (and SR) that pass is ALU-bound and the two single calls are faster.
        self._quant(d["X"], "X_r", ev=ev)
        self._dual(d["W1"], "W1_r", "W1_c", ev=ev)
        self._gemm("X_r", "W1_r", self.Y1, ev)
        # relu^2 also returns max|h| and max|RHT(h)|, so both quantisations of h skip their amax pass
        B.nvfp4_relu2_fwd_amax_rht(self.Y1, seed=SEED, out=self.h, amax_out=self.amax_h,
                                   amax_rht_out=self.amax_h_rht, ws=self.qws)
        self.launches += B.nvfp4_last_launch_count()
        if ev is not None:
            ev.append(("relu2", self.Y1.numel(), torch.cuda.Event(enable_timing=True)))
            ev[-1][2].record()
        self._quant(self.h, "h_r", amax_in=self.amax_h, ev=ev)
        self._dual(d["W2"], "W2_r", "W2_c", ev=ev)
        self._gemm("h_r", "W2_r", self.Y2, ev)
        # down-projection backward: dh = dY2 . W2, dW2 = dY2^T h
        self._quant(d["dY2"], "dY2_r", ev=ev)
        self._gemm("dY2_r", "W2_c", self.dh, ev)
        self._quant(d["dY2"], "dY2_c", colwise=True, sr=True, rht=True, ev=ev)
        self._quant(self.h, "h_c", colwise=True, rht=True, amax_in=self.amax_h_rht, ev=ev)
        self._gemm("dY2_c", "h_c", self.dW2, ev)
        B.nvfp4_relu2_bwd_amax_rht(self.dh, self.Y1, seed=SEED, out=self.dY1, amax_out=self.amax_dy1,
                                   amax_rht_out=self.amax_dy1_rht, ws=self.qws)
        self.launches += B.nvfp4_last_launch_count()
        if ev is not None:
            ev.append(("relu2", self.Y1.numel(), torch.cuda.Event(enable_timing=True)))
            ev[-1][2].record()
        # up-projection backward: dX = dY1 . W1, dW1 = dY1^T X
        self._quant(self.dY1, "dY1_r", amax_in=self.amax_dy1, ev=ev)
        self._gemm("dY1_r", "W1_c", self.dX, ev)
        self._quant(self.dY1, "dY1_c", colwise=True, sr=True, rht=True, amax_in=self.amax_dy1_rht, ev=ev)
        self._quant(d["X"], "X_c", colwise=True, rht=True, ev=ev)
        self._gemm("dY1_c", "X_c", self.dW1, ev)
        dp.allreduce_grads([self.dW1, self.dW2])

    def public_step(self, X=None, dY2=None, Y2=None):
        """The same step through the composite public calls (linear_fwd/bwd, relu2)."""
        B, d = self.B, self.d
        X = d["X"] if X is None else X
        dY2 = d["dY2"] if dY2 is None else dY2
        Y2 = self.Y2 if Y2 is None else Y2
        B.nvfp4_linear_fwd(X, d["W1"], out=self.Y1, ws=self.ws)
        self.launches += B.nvfp4_last_launch_count()
        B.nvfp4_relu2_fwd(self.Y1, out=self.h)
        self.launches += B.nvfp4_last_launch_count()
        B.nvfp4_linear_fwd(self.h, d["W2"], out=Y2, ws=self.ws)
        self.launches += B.nvfp4_last_launch_count()
        B.nvfp4_linear_bwd(dY2, self.h, d["W2"], seed=SEED, dX=self.dh, dW=self.dW2, ws=self.ws)
        self.launches += B.nvfp4_last_launch_count()
        B.nvfp4_relu2_bwd(self.dh, self.Y1, out=self.dY1)
        self.launches += B.nvfp4_last_launch_count()
        B.nvfp4_linear_bwd(self.dY1, X, d["W1"], seed=SEED, dX=self.dX, dW=self.dW1, ws=self.ws)
        self.launches += B.nvfp4_last_launch_count()
        dp.allreduce_grads([self.dW1, self.dW2])


class E2EPipeline:
    """Steps through the public calls with every step's host->device input copy and
    device->host output copy on their own streams, double-buffered, so that step i+1's
    inputs arrive and step i-1's output leaves while step i computes (a training loop's
    prefetch).  Every step still moves its own bytes inside the timed region."""

    def __init__(self, step):
        self.step = step
        self.xs = [step.d["X"], torch.empty_like(step.d["X"])]
        self.dys = [step.d["dY2"], torch.empty_like(step.d["dY2"])]
        self.y2s = [step.Y2, torch.empty_like(step.Y2)]
        self.y2_host = [torch.empty(step.Y2.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run(self, n):
        st, comp = self.step, torch.cuda.current_stream()
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def load(b):
            with torch.cuda.stream(self.s_in):
                self.xs[b].copy_(st.host["X"], non_blocking=True)
                self.dys[b].copy_(st.host["dY2"], non_blocking=True)
                in_ready[b].record(self.s_in)

        self.s_in.wait_stream(comp)
        self.s_out.wait_stream(comp)
        load(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                if i >= 1:
                    self.s_in.wait_event(done[1 - b])  # step i-1 no longer reads buffer 1-b
                load(1 - b)
            comp.wait_event(in_ready[b])
            if i >= 2:
                comp.wait_event(out_done[b])           # step i-2's output has left buffer b
            st.public_step(self.xs[b], self.dys[b], self.y2s[b])
            done[b].record(comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(done[b])
                self.y2_host[b].copy_(self.y2s[b], non_blocking=True)
                out_done[b].record(self.s_out)
        comp.wait_stream(self.s_out)
        comp.wait_stream(self.s_in)


def kernel_stats(events_per_step):
    """Average device time and algorithmic work per call kind over the timed steps."""
    acc = {}
    for ev in events_per_step:
        for (kind, work, e), (_, _, prev) in zip(ev[1:], ev[:-1]):
            ms = prev.elapsed_time(e)
            a = acc.setdefault(kind, [0.0, 0.0, 0])
            a[0] += ms
            a[1] += work
            a[2] += 1
    return acc


def traffic_record(kernel):
    """DRAM traffic per launch from the committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, "nvfp4_bit_precision_quantize_b200", "csrc", rec["source"])
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != rec["sha256_16"]:
            return None
    return rec


# ------------------------------------------------------------ CPU oracle arm
def oracle_sample(budget_s=12.0):
    """Time the oracle as it stands on a bounded sample of the MLP step and
    extrapolate the full step's CPU time.  Returns (est_step_s, description)."""
    import oracle
    rng = np.random.default_rng(0)
    t_all = time.perf_counter()
    # quantiser: per-element cost of each mode on a 2048 x 5120 bf16 slice (amax + quantise)
    x = W.bf16_bits(W.normal(rng, (2048, 5120)))
    per_elem = {}
    for mode in [(False, False, False), (True, False, False), (True, True, True), (True, False, True)]:
        t0 = time.perf_counter()
        oracle.quantize(x, colwise=mode[0], sr=mode[1], rht=mode[2], seed=SEED)
        per_elem[mode] = (time.perf_counter() - t0) / x.size
    n_x, n_w, n_h = M_TOK * HID, FFN * HID, M_TOK * FFN
    quant_s = (per_elem[(False, False, False)] * (n_x + n_w + n_h + n_w + n_x + n_h)
               + per_elem[(True, False, False)] * (n_w + n_w)
               + per_elem[(True, True, True)] * (n_x + n_h)
               + per_elem[(True, False, True)] * (n_h + n_x))
    # GEMM: FP64 dot products of sampled outputs at each reduction length
    gemm_s = 0.0
    macs_done = 0
    for K, reps in ((HID, 2), (FFN, 2), (M_TOK, 2)):
        a = (rng.integers(0, 256, (64, K // 2), dtype=np.uint8), rng.integers(0x20, 0x50, (64, K // 16),
                                                                             dtype=np.uint8), 1.0)
        b = (rng.integers(0, 256, (64, K // 2), dtype=np.uint8), rng.integers(0x20, 0x50, (64, K // 16),
                                                                             dtype=np.uint8), 1.0)
        n = 2560
        ms, ns = rng.integers(0, 64, n), rng.integers(0, 64, n)
        t0 = time.perf_counter()
        oracle.gemm_sampled(a, b, ms, ns)
        dt = time.perf_counter() - t0
        macs_done += n * K
        gemm_s += dt / (n * K) * (reps * M_TOK * HID * FFN)
    # relu^2 pair
    y = W.bf16_bits(W.normal(rng, (1 << 23,)))
    t0 = time.perf_counter()
    oracle.relu2_fwd(y)
    oracle.relu2_bwd(y, y)
    relu_s = (time.perf_counter() - t0) / y.size * n_h
    est = quant_s + gemm_s + relu_s
    desc = ("oracle (plain C, 1 thread) on a bounded sample: 4 quantise modes on a 2048x5120 bf16 slice, "
            "%d FP64 sampled GEMM outputs (K = 5120/20480/8192), relu^2 on 2^23 elements; extrapolated "
            "to the full step (%.1f s measured)" % (3 * 2560, time.perf_counter() - t_all))
    return est, desc


def run_reference(args):
    ws, rank, _ = dp.world()
    if rank != 0:
        return
    t_start = time.perf_counter()
    for _ in range(args.warmup):
        oracle_sample()
    ests = [oracle_sample()[0] for _ in range(args.steps)]
    est, desc = oracle_sample()
    step_s = statistics.median(ests)
    value = GEMM_FLOPS / step_s / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantise / f64 GEMM (CPU oracle)",
            "data": "synthetic", "config": {"workload": WORKLOAD, "parallelism": "cpu"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": time.perf_counter() - t_start}
    print(json.dumps(line))


# ------------------------------------------------------------------- our arm
def run_ours(args):
    nproc, rank, local = dp.init("nccl")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    from nvfp4_bit_precision_quantize_b200 import binding as B
    from nvfp4_bit_precision_quantize_b200 import build as lib_build
    lib_build.build()
    B.load()
    step = MlpStep(B, device, dp.shard_data_seed(5, rank))

    # warm-up
    for _ in range(args.warmup):
        step.device_step()
    B.nvfp4_check(step.ws)
    dp.barrier()
    torch.cuda.synchronize()

    # timed region: exactly K device steps
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(vis.split(",")[local].strip() if vis else str(local))
    clocks.start()
    step.launches = 0
    events = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    dp.barrier()
    torch.cuda.synchronize()
    t0.record()
    for _ in range(args.steps):
        ev = []
        step.device_step(ev)
        events.append(ev)
    t1.record()
    torch.cuda.synchronize()
    dp.barrier()
    clk = clocks.stop()
    launches = step.launches
    ms = t0.elapsed_time(t1) / args.steps
    ms_max = dp.max_over_ranks(ms, device)
    B.nvfp4_check(step.ws)
    stats = kernel_stats(events)

    # end to end through the public calls: pinned host inputs in, block output out, every step
    h2d = step.host["X"].numel() * 2 + step.host["dY2"].numel() * 2
    d2h = step.Y2.numel() * 2
    pipe = E2EPipeline(step)
    pipe.run(3)
    dp.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    pipe.run(args.steps)
    e1.record()
    torch.cuda.synchronize()
    dp.barrier()
    e2e_ms = dp.max_over_ranks(e0.elapsed_time(e1) / args.steps, device)
    B.nvfp4_check(step.ws)

    # MXFP4 (the pages' comparison format) rowwise quantisation of the step's h, timed apart
    # from the step: one pass, 2 B read + 0.5 + 1/32 B written per element
    mx_out = B.nvfp4_quantize_mx(step.h)
    for _ in range(3):
        B.nvfp4_quantize_mx(step.h, out=mx_out)
    torch.cuda.synchronize()
    m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    m0.record()
    for _ in range(20):
        B.nvfp4_quantize_mx(step.h, out=mx_out)
    m1.record()
    torch.cuda.synchronize()
    mx_us = m0.elapsed_time(m1) / 20 * 1e3

    pk, src = peaks()
    if rank == 0:
        g = stats["gemm"]
        q = stats["quant"]
        gemm_ms = g[0] / g[2]
        gemm_flops = g[1] / g[2]
        gemm_tflops = gemm_flops / (gemm_ms / 1e3) / 1e12
        fp4_peak = pk["bf16_tflops_sustained"] * FP4_PER_BF16
        # algorithmic bytes of the quantise calls (two-pass, dual-orientation: 5.125 B per element)
        q_gbs = q[1] / (q[0] / 1e3) / 1e9
        tr = traffic_record("gemm_nvfp4_kernel")
        line = {
            "metric": METRIC, "value": nproc * GEMM_FLOPS / (ms_max / 1e3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": nproc, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4 (e2m1 x e4m3 block16 x fp32 tensor scale), fp32 accumulate",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens_per_gpu": M_TOK, "hidden": HID, "ffn": FFN,
                       "global_tokens": nproc * M_TOK, "parallelism": "dp%d" % nproc,
                       "l2": "no flush: every step touches ~2.5 GB, far beyond the 126 MB L2",
                       "seed": SEED},
            "roofline": {"bound": "tensor", "kernel": "gemm_nvfp4_kernel", "achieved": gemm_tflops,
                         "peak": fp4_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                         "traffic": tr["bytes_per_launch"] if tr else None,
                         "peak_source": "%s bf16_tflops_sustained x %.0f (nominal dense fp4/bf16)" % (src,
                                                                                            FP4_PER_BF16),
                         "launch_ms": gemm_ms, "flop_per_launch": gemm_flops},
            "roofline_quantize": {"bound": "hbm", "kernels": "amax*, quantize_rowwise, quantize_colwise (+dual)",
                                  "achieved": q_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                  "frac": q_gbs / pk["hbm_gbs"],
                                  "bytes_per_elem": {"single": QUANT_BYTES_SINGLE, "dual": QUANT_BYTES_DUAL,
                                                     "amax_supplied": QUANT_BYTES_AMAX_IN},
                                  "calls_per_step": q[2] // args.steps, "peak_source": src + " hbm_gbs",
                                  "call_ms": q[0] / q[2]},
            "mxfp4_quantize": {"tensor": "h %dx%d bf16, rowwise" % tuple(step.h.shape), "us_per_call": mx_us,
                               "achieved": step.h.numel() * MX_BYTES / (mx_us * 1e-6) / 1e9, "unit": "GB/s",
                               "peak": pk["hbm_gbs"],
                               "frac": step.h.numel() * MX_BYTES / (mx_us * 1e-6) / 1e9 / pk["hbm_gbs"],
                               "bytes_per_elem": MX_BYTES},
            "breakdown_ms_per_step": {k: v[0] / args.steps for k, v in stats.items()},
            "e2e": {"value": nproc * GEMM_FLOPS / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": clk,
        }
        if nproc == 1 and not args.no_cpu_baseline:
            est, desc = oracle_sample()
            line["cpu_baseline"] = {"value": GEMM_FLOPS / est / 1e12, "unit": "TFLOP/s", "cores": 1,
                                    "kind": "oracle", "sample": desc}
        print(json.dumps(line))
    dp.finish()


def run_profile_case(case):
    """A few calls of one kernel at a full workload size, for ncu captures (untimed)."""
    from nvfp4_bit_precision_quantize_b200 import binding as B
    from nvfp4_bit_precision_quantize_b200 import build as lib_build
    lib_build.build()
    B.load()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    rng = np.random.default_rng(7)
    if case == "gemm":  # Fprop shape, random NVFP4 operands, bf16 out
        def operand(rows, k):
            return B.NVFP4Tensor(
                codes=torch.randint(0, 256, (rows, k // 2), dtype=torch.uint8, device=dev, generator=g),
                scales=torch.randint(0x20, 0x50, (B.nvfp4_scales_bytes(rows, k),), dtype=torch.uint8, device=dev,
                                     generator=g),
                tensor_scale=torch.ones(1, device=dev), rows=rows, k=k)
        a, b = operand(M_TOK, HID), operand(FFN, HID)
        out = torch.empty((M_TOK, FFN), dtype=torch.bfloat16, device=dev)
        ws = B.workspace(256, dev)
        for _ in range(3):
            B.nvfp4_gemm(a, b, out=out, ws=ws)
        B.nvfp4_check(ws)
    elif case in ("quant_x", "quant_dy"):
        if case == "quant_x":  # Fprop activation, rowwise RTN
            x = W.bits_to_torch_bf16(W.bf16_bits(W.normal(rng, (M_TOK, HID)))).to(dev)
            kw = dict(orientation=B.NVFP4_ROWWISE)
        else:  # Wgrad gradient operand: colwise, RHT + SR
            x = W.bits_to_torch_bf16(W.bf16_bits(W.heavy_rows(rng, (2 * M_TOK, FFN), 1e-3, 2))).to(dev)
            kw = dict(orientation=B.NVFP4_COLWISE, rounding=B.NVFP4_SR, rht=True)
        ws = B.workspace(B.nvfp4_quantize_workspace_size(), dev)
        q = None
        for _ in range(3):
            q = B.nvfp4_quantize(x, out=q, ws=ws, seed=SEED, **kw)
    elif case == "quant_mx":  # MXFP4 rowwise of an h-shaped tensor
        x = W.bits_to_torch_bf16(W.bf16_bits(W.normal(rng, (M_TOK, FFN)))).to(dev)
        q = None
        for _ in range(3):
            q = B.nvfp4_quantize_mx(x, out=q)
    elif case == "quant_dual":  # the step's dY1: rowwise RTN + colwise RHT + SR from one read
        x = W.bits_to_torch_bf16(W.bf16_bits(W.normal(rng, (M_TOK, FFN), 1e-3))).to(dev)
        ws = B.workspace(B.nvfp4_quantize_dual_workspace_size(), dev)
        r = c = None
        for _ in range(3):
            r, c = B.nvfp4_quantize_dual(x, col_rounding=B.NVFP4_SR, col_rht=True, seed=SEED, out_row=r, out_col=c,
                                         ws=ws)
    else:
        raise SystemExit("unknown profile case " + case)
    torch.cuda.synchronize()
    print("profile case %s ok" % case)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=["gemm", "quant_x", "quant_dy", "quant_dual", "quant_mx"],
                    help="run one kernel a few times for an ncu capture instead of the benchmark")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
