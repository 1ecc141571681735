"""Benchmark: causal prefill attention TFLOP/s on B200 (FP8 e4m3 / BF16).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--S S]
                    [--dtype leanp|exact|bf16] [--hadamard] [--descale tensor|kv]
                    [--T T] [--impl reference] [--no-extra] [--no-e2e] [--no-cpu]
                    [--no-energy] [--cpu-seconds SEC]
    python bench.py --gemm-peaks
    python bench.py --trace [--workload NAME] [--S S] [--dtype ...]

A step is one pass of the whole hot path over one batch of synthetic input:
for FP8, the quantisation of Q, K and V (fp32 -> e4m3: one multi-tensor
quantiser call with one scale per tensor, or with --descale kv three grouped
calls with one scale per (batch, kv head)) followed
by the attention kernel; for BF16 the attention kernel alone.  The headline
workload is the Gaussian peak-sweep point at S = 32768 (B=1, Hq=Hkv=32,
d=128), FP8 with Lean P and per-64-key block scaling -- the configuration the
pages quote their best FP8 number on.  One JSON line is printed (rank 0).

value      causal TFLOP/s = 2*B*Hq*S^2*(d_qk+d_v)/2 / step time (inputs resident
           in HBM), summed over ranks (weak scaling: every rank runs its own
           batch of the same size).
e2e        same metric through the C ABI from pinned host buffers: H2D copy of
           fp32 Q/K/V, the step, D2H of the bf16 output, all inside the timed
           region.
roofline   attention kernel only: algorithmic FLOPs per launch / CUDA-event
           launch time (mean of back-to-back launches; min and max of single
           launches beside it), against the burst BF16 GEMM peak (x2 for FP8,
           the nominal ratio) and against the datasheet dense peak.
quant_share_of_attention  FP8: time of the three quantiser calls / attention.
deterministic  two further launches equal the timed one bit for bit.
also       (N=1) the other workloads of the metric, one compact entry each:
           BF16 32K/16K, FP8 exact 32K, Lean P 16K, MLA 16K, GQA 4K and long
           16K (TFLOP/J), long 16K with the Hadamard rotation, headroom T = 0.
cpu_baseline  the fp64 oracle (FP8 emulation of the same mode) on host cores
           over a bounded row sample, in the same unit; also its
           single-thread rate, the CPU model, and the GPU output's rel-RMSE
           on a seeded row sample against the oracle on the kernel inputs and
           against the exact reference on the unquantised inputs.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
DATASHEET_DENSE_TFLOPS = {"bf16": 2250.0, "fp8": 4500.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gauss")
    ap.add_argument("--S", type=int, default=None)
    ap.add_argument("--dtype", default="leanp", choices=["leanp", "exact", "bf16"])
    ap.add_argument("--hadamard", action="store_true")
    ap.add_argument("--descale", default="tensor", choices=["tensor", "kv"],
                    help="FP8 scales: one per tensor, or one per (batch, kv head)")
    ap.add_argument("--T", type=int, default=8, help="FP8 headroom T (block maximum lands in (2^(T-1), 2^T])")
    ap.add_argument("--no-energy", action="store_true", help="skip the attention-only power measurement")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads measured after the headline (N=1)")
    ap.add_argument("--trace", action="store_true",
                    help="only run the debug kernel on one long unit and print its per-role pipeline timing")
    ap.add_argument("--gemm-peaks", action="store_true",
                    help="only measure library FP8 / BF16 GEMM throughput on this GPU and print it")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers
def dist_setup(n):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def _reduce_over_ranks(x: float, world: int, op_name: str) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    # NCCL reduces device tensors; gloo (the CPU tests of this path) host ones
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=getattr(dist.ReduceOp, op_name))
    return float(t.item())


def max_over_ranks(x: float, world: int) -> float:
    return _reduce_over_ranks(x, world, "MAX")


def sum_over_ranks(x: float, world: int) -> float:
    return _reduce_over_ranks(x, world, "SUM")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        loaded = [s for s, p in zip(sm, power) if p > 300] or sm
        loaded_p = [p for p in power if p > 300] or power
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None,
                "power_w_mean": statistics.mean(loaded_p) if loaded_p else None}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def tensor_peak(kind: str):
    """Dense tensor peak for the attention kernel, TFLOP/s.  The kernel is
    timed alone (a few hundred ms of back-to-back launches), so the burst
    cuBLAS BF16 figure is the reference; FP8 takes it times the nominal
    FP8:BF16 ratio 2."""
    pk, src = measured_peaks()
    base = pk.get("bf16_tflops")
    if kind == "fp8":
        return base * 2.0, "%s bf16 burst x2 (nominal fp8:bf16 ratio)" % src
    return base, "%s bf16 burst" % src


def sustained_peak(kind: str):
    pk, src = measured_peaks()
    base = pk.get("bf16_tflops_sustained")
    if base is None:
        return None
    return base * (2.0 if kind == "fp8" else 1.0)


def gemm_peaks():
    """Library GEMM throughput measured on one B200 by `bench.py --gemm-peaks`
    (committed under profiles/), or None."""
    path = os.path.join(ROOT, "profiles", "gemm_peaks.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        return json.load(f)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def kernel_sources_digest(read=None) -> str:
    """sha256 over the attention kernels' sources: attn_fwd.cu, attn_pp.cu
    and every header beside them, by name in sorted order.  `read(name)`
    returns a file's bytes (default: the files in csrc)."""
    import hashlib

    csrc = os.path.join(ROOT, "bf16_causal_prefill_02_b200", "csrc")
    if read is None:
        names = sorted(n for n in os.listdir(csrc) if n in ("attn_fwd.cu", "attn_pp.cu") or n.endswith((".h", ".cuh")))

        def read(n):
            with open(os.path.join(csrc, n), "rb") as f:
                return f.read()
    else:
        names = sorted(read(None))
    h = hashlib.sha256()
    for n in names:
        h.update(n.encode() + b"\0" + read(n) + b"\0")
    return h.hexdigest()


def load_traffic(key: str):
    """DRAM bytes per attention launch from profiles/traffic.json, or None.
    The counters hold only for the kernel they were taken on: when the
    kernel's sources no longer hash to the digest recorded with them, the
    figure is returned as stale (second value) and the first is None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        d = json.load(f)
    val = d.get(key)
    if val is None:
        return None, None
    if d.get("_kernel_sources_sha256") != kernel_sources_digest():
        return None, val
    return val, None


# --------------------------------------------------------------- our arm
class Step:
    """The hot path for one workload on one GPU; inputs resident in HBM."""

    def __init__(self, w: workloads.Workload, dtype: str, hadamard: bool, seed_offset: int = 0, T: int = 8,
                 per_kv: bool = False, host_inputs=None):
        import bf16_causal_prefill_02_b200 as zq

        self.zq, self.w, self.dtype, self.hadamard = zq, w, dtype, hadamard
        self.per_kv = per_kv and dtype != "bf16"
        if host_inputs is None:
            q, k, v = workloads.make_inputs(w, seed=w.seed + seed_offset)
            host_inputs = [t.pin_memory() for t in (q, k, v)]
        self.host = host_inputs
        dev = torch.device("cuda")
        self.q32, self.k32, self.v32 = (t.to(dev) for t in self.host)
        B, S, Hq, Hkv, dqk, dv = w.B, w.S, w.Hq, w.Hkv, w.dqk, w.dv
        self.out = torch.empty((B, S, Hq, dv), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
        self.out_host = torch.empty_like(self.out, device="cpu").pin_memory()
        if dtype == "bf16":
            self.qb, self.kb, self.vb = (t.to(torch.bfloat16) for t in (self.q32, self.k32, self.v32))
        else:
            f8 = torch.float8_e4m3fn
            self.qc = torch.empty(self.q32.shape, dtype=f8, device=dev)
            self.kc = torch.empty(self.k32.shape, dtype=f8, device=dev)
            self.vc = torch.empty(self.v32.shape, dtype=f8, device=dev)
            if self.per_kv:
                # one scale per (batch, kv head); the query heads of a kv
                # head share its scale
                g = Hq // Hkv
                self.dsq = torch.zeros((B, Hkv), dtype=torch.float32, device=dev)
                self.dsk = torch.zeros((B, Hkv), dtype=torch.float32, device=dev)
                self.dsv = torch.zeros((B, Hkv), dtype=torch.float32, device=dev)
                nb = max(zq.zq_quantize_grouped_workspace_bytes(B, Hq, g),
                         zq.zq_quantize_grouped_workspace_bytes(B, Hkv, 1))
                self.ws = torch.empty(3, nb, dtype=torch.uint8, device=dev)
                self.group_q = g
            else:
                self.ds = torch.zeros(3, dtype=torch.float32, device=dev)
                self.dsq, self.dsk, self.dsv = self.ds[0:1], self.ds[1:2], self.ds[2:3]
                self.ws = torch.empty(zq.zq_quantize_multi_workspace_bytes(), dtype=torch.uint8, device=dev)
        self.mode = zq.ZQ_SOFTMAX_EXACT if dtype == "exact" else zq.ZQ_SOFTMAX_LEANP
        self.T = T

    def launches_per_step(self) -> int:
        if self.dtype == "bf16":
            return 1
        # per-tensor scales: one amax and one write kernel for Q, K and V
        # together; per-(batch, kv head) scales: both kernels per tensor
        return 7 if self.per_kv else 3

    def attention(self, out=None):
        zq = self.zq
        out = self.out if out is None else out
        if self.dtype == "bf16":
            zq.attn_fwd(self.qb, self.kb, self.vb, out=out, lse=self.lse)
        else:
            zq.attn_fwd(self.qc, self.kc, self.vc, out=out, lse=self.lse,
                        q_descale=self.dsq, k_descale=self.dsk, v_descale=self.dsv,
                        softmax_mode=self.mode, block_scale=True, headroom_T=self.T)

    def quantize(self):
        zq = self.zq
        if self.per_kv:
            zq.quantize_fp8_grouped(self.q32, self.group_q, hadamard=self.hadamard, out=self.qc,
                                    descale=self.dsq, workspace=self.ws[0])
            zq.quantize_fp8_grouped(self.k32, 1, hadamard=self.hadamard, out=self.kc, descale=self.dsk,
                                    workspace=self.ws[1])
            zq.quantize_fp8_grouped(self.v32, 1, hadamard=False, out=self.vc, descale=self.dsv,
                                    workspace=self.ws[2])
            return
        zq.quantize_fp8_multi([self.q32, self.k32, self.v32], hadamard=[self.hadamard, self.hadamard, False],
                              outs=[self.qc, self.kc, self.vc], descales=[self.dsq, self.dsk, self.dsv],
                              workspace=self.ws)

    def step(self):
        if self.dtype != "bf16":
            self.quantize()
        self.attention()

    def e2e_step(self):
        """Host buffers in, host buffer out, through the same C-ABI calls."""
        self.q32.copy_(self.host[0], non_blocking=True)
        self.k32.copy_(self.host[1], non_blocking=True)
        self.v32.copy_(self.host[2], non_blocking=True)
        if self.dtype == "bf16":
            self.qb.copy_(self.q32)
            self.kb.copy_(self.k32)
            self.vb.copy_(self.v32)
        self.step()
        self.out_host.copy_(self.out, non_blocking=True)

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.host)

    def d2h_bytes(self):
        return self.out.numel() * self.out.element_size()


def time_steps(fn, steps, warmup, world):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1)
    return max_over_ranks(ms, world)


def time_back_to_back(fn, n):
    """Average time of `n` launches of fn between two events on the current
    stream, behind one launch already queued (no host time between launches
    enters), plus min / max of `n` individually bracketed launches."""
    st = torch.cuda.current_stream()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fn()
    a0.record(st)
    for _ in range(n):
        fn()
    a1.record(st)
    torch.cuda.synchronize()
    mean = a0.elapsed_time(a1) / n
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    fn()
    for b0, b1 in evs:
        b0.record(st)
        fn()
        b1.record(st)
    torch.cuda.synchronize()
    each = [b0.elapsed_time(b1) for b0, b1 in evs]
    return mean, min(each), max(each)


def measure_energy(step, flops, seconds=1.0):
    """Attention launches back to back for about `seconds` while nvidia-smi
    samples the board power every 100 ms."""
    st = torch.cuda.current_stream()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step.attention()
    a0.record(st)
    step.attention()
    a1.record(st)
    torch.cuda.synchronize()
    n = max(1, int(seconds * 1000.0 / max(a0.elapsed_time(a1), 1e-3)))
    es = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    es.start()
    time.sleep(0.3)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step.attention()
    b0.record(st)
    for _ in range(n):
        step.attention()
    b1.record(st)
    torch.cuda.synchronize()
    ec = es.stop()
    e_ms = b0.elapsed_time(b1) / n
    pw = ec.get("power_w_mean")
    if not pw:
        return None
    tf = flops / (e_ms * 1e-3) / 1e12
    return {"tflop_per_joule": round(tf / pw, 3), "attn_tflops": round(tf, 1),
            "power_w_mean": round(pw, 1), "sm_mhz": ec.get("sm_mhz"),
            "reasons": ec.get("reasons"), "samples": ec.get("samples"),
            "basis": "%d back-to-back attention launches; board power.draw from nvidia-smi "
                     "every 100 ms, mean over the loaded samples" % n}


def measure(step, steps, warmup, world, energy=True):
    """Step time (whole hot path), attention-only time (mean, min, max),
    quantiser time per step (FP8), clocks during the timed regions, and
    optionally energy.  Returns a dict of plain numbers."""
    w = step.w
    flops = w.causal_flops()
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    for _ in range(max(warmup, 3)):
        step.step()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.25)
    ms_total = time_steps(step.step, steps, warmup, world)
    attn_ms, attn_min, attn_max = time_back_to_back(step.attention, steps)
    quant_ms = None
    if step.dtype != "bf16":
        quant_ms, _, _ = time_back_to_back(step.quantize, steps)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    r = {"flops": flops, "ms_step": ms_total / steps, "attn_ms": max_over_ranks(attn_ms, world),
         "attn_ms_min": attn_min, "attn_ms_max": attn_max, "quant_ms": quant_ms, "clocks": clocks}
    r["energy"] = measure_energy(step, flops) if energy else None
    return r


def _oracle_inputs(w, dtype, hadamard, per_kv=False, original=None):
    """The kernel's inputs for `w` as fp64 arrays (FP8: quantised and decoded,
    as the kernel sees them)."""
    import oracle

    q, k, v = (t.numpy() for t in (original or workloads.make_inputs(w)))
    if dtype == "bf16":
        return tuple(torch.from_numpy(t).to(torch.bfloat16).double().numpy() for t in (q, k, v))
    deq = []
    if per_kv:
        for t, g, rot in ((q, w.Hq // w.Hkv, hadamard), (k, 1, hadamard), (v, 1, False)):
            c, d = oracle.quantize_fp8_grouped(t, heads_per_scale=g, hadamard=rot)
            deq.append(oracle.dequant_grouped(c, d))
        return tuple(deq)
    for t, rot in ((q, hadamard), (k, hadamard), (v, False)):
        c, d = oracle.quantize_fp8(t, hadamard=rot)
        deq.append(oracle.dequant_e4m3(c, float(d)))
    return tuple(deq)


def _oracle_rows(w, dtype, qd, kd, vd, rows):
    """Run the oracle (R1 for bf16, R2 of the mode for FP8) on `rows`;
    returns the causal FLOPs those rows stand for."""
    import oracle

    if dtype == "bf16":
        oracle.attn_ref(qd, kd, vd, rows=rows)
    else:
        oracle.attn_fp8_emul(qd, kd, vd, rows=rows,
                             mode=oracle.MODE_EXACT if dtype == "exact" else oracle.MODE_LEANP)
    i = rows % w.S
    return float(np.sum(2.0 * (w.dqk + w.dv) * (i + 1)))


def _time_oracle(w, dtype, qd, kd, vd, seconds, seed):
    rng = np.random.default_rng(seed)
    done_rows, flops, elapsed = 0, 0.0, 0.0
    batch = 64
    while elapsed < seconds:
        rows = rng.integers(0, w.B * w.Hq * w.S, size=batch)
        t0 = time.perf_counter()
        flops += _oracle_rows(w, dtype, qd, kd, vd, rows)
        elapsed += time.perf_counter() - t0
        done_rows += batch
        batch = min(batch * 2, 4096)
    return flops / elapsed / 1e12, done_rows, elapsed


def cpu_baseline_leg(w, dtype, seconds, hadamard=False, per_kv=False, step=None, acc_rows=256):
    """The oracle as it stands on the host cores: its rate on a bounded
    sample of uniformly drawn query rows (all cores, then one thread), and
    the GPU output's error on a seeded row sample against the oracle on the
    kernel inputs and against the exact reference on the unquantised inputs.
    Returns the cpu_baseline dict."""
    import oracle

    original = workloads.make_inputs(w)
    qd, kd, vd = _oracle_inputs(w, dtype, hadamard, per_kv, original=original)
    tf, done_rows, elapsed = _time_oracle(w, dtype, qd, kd, vd, seconds, 0)
    cores = oracle.num_threads()
    prev = cores
    oracle.set_num_threads(1)
    tf1, rows1, el1 = _time_oracle(w, dtype, qd, kd, vd, max(2.0, seconds / 4), 1)
    oracle.set_num_threads(prev)
    desc = ("%d uniformly drawn query rows of %s (fp64 %s on kernel inputs; inputs quantised "
            "beforehand, untimed), %.1f s" % (done_rows, w.name,
                                               "R1 exact" if dtype == "bf16" else "R2 " + dtype, elapsed))
    res = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
           "cpu_model": cpu_model(),
           "single_thread": {"value": tf1, "unit": "TFLOP/s", "rows": rows1, "seconds": round(el1, 1)}}
    if step is not None:
        res["accuracy"] = accuracy_on_rows(w, dtype, hadamard, step, qd, kd, vd, original, acc_rows)
    return res


def accuracy_on_rows(w, dtype, hadamard, step, qd, kd, vd, original, n_rows):
    """rel-RMSE of the GPU output (bf16) on `n_rows` seeded query rows:
    against the oracle on the kernel's own inputs (R1 exact reference, and
    R2 of the same mode for FP8) and against R1 on the unquantised fp32
    inputs (the end-to-end error, where the rotation matters)."""
    import oracle

    step.attention()
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    rows = np.sort(rng.integers(0, w.B * w.Hq * w.S, size=n_rows))
    b, rem = rows // (w.Hq * w.S), rows % (w.Hq * w.S)
    h, i = rem // w.S, rem % w.S
    o = step.out.float().cpu().numpy().astype(np.float64)[b, i, h]
    r1, _ = oracle.attn_ref(qd, kd, vd, rows=rows)
    acc = {"rows": int(n_rows), "hadamard": bool(hadamard), "vs_kernel_inputs_r1": oracle.rel_rmse(o, r1)}
    if dtype != "bf16":
        r2, _ = oracle.attn_fp8_emul(qd, kd, vd, rows=rows,
                                     mode=oracle.MODE_EXACT if dtype == "exact" else oracle.MODE_LEANP)
        acc["vs_kernel_inputs_r2"] = oracle.rel_rmse(o, r2)
    q, k, v = (t.numpy().astype(np.float64) for t in original)
    r0, _ = oracle.attn_ref(q, k, v, rows=rows)
    acc["vs_original"] = oracle.rel_rmse(o, r0)
    return acc


def oracle_steps(w, dtype, steps, warmup, rows_per_step, hadamard=False, per_kv=False):
    """The reference arm: `warmup` untimed and `steps` timed oracle steps,
    each over `rows_per_step` query rows drawn uniformly (seeded) from the
    workload.  Returns (TFLOP/s, ms per step, cores, sample description)."""
    import oracle

    qd, kd, vd = _oracle_inputs(w, dtype, hadamard, per_kv)
    rng = np.random.default_rng(1)
    for _ in range(warmup):
        _oracle_rows(w, dtype, qd, kd, vd, rng.integers(0, w.B * w.Hq * w.S, size=rows_per_step))
    flops, elapsed = 0.0, 0.0
    for _ in range(steps):
        rows = rng.integers(0, w.B * w.Hq * w.S, size=rows_per_step)
        t0 = time.perf_counter()
        flops += _oracle_rows(w, dtype, qd, kd, vd, rows)
        elapsed += time.perf_counter() - t0
    desc = ("%d timed steps of %d uniformly drawn query rows of %s each (fp64 %s on kernel inputs; "
            "inputs quantised beforehand, untimed), %.1f s" %
            (steps, rows_per_step, w.name, "R1 exact" if dtype == "bf16" else "R2 " + dtype, elapsed))
    return flops / elapsed / 1e12, elapsed / max(steps, 1) * 1e3, oracle.num_threads(), desc


def _variant_suffix(args) -> str:
    suf = "_hadamard" if args.hadamard else ""
    if args.dtype != "bf16" and getattr(args, "descale", "tensor") == "kv":
        suf += "_kvscale"
    return suf


def config_dict(w, args, world):
    """The workload description shared by both arms of the benchmark."""
    kind = "bf16" if args.dtype == "bf16" else "fp8"
    per_kv = kind == "fp8" and args.descale == "kv"
    return {"workload": "%s_%s%s" % (w.name, args.dtype, _variant_suffix(args)),
            "B": w.B, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv, "d_qk": w.dqk, "d_v": w.dv,
            "causal": True, "softmax": args.dtype,
            "block_scale": kind == "fp8", "headroom_T": args.T if kind == "fp8" else None,
            "step": (("quantise Q,K,V (fp32->e4m3, %s scales%s) + attention" %
                      ("per-(batch, kv head)" if per_kv else "per-tensor",
                       ", Hadamard on Q,K" if args.hadamard else ""))
                     if kind == "fp8" else "attention"),
            "l2": "inputs larger than L2 (%.0f MB fp32 Q/K/V), no flush" %
                  ((w.B * w.S * (w.Hq * w.dqk + w.Hkv * (w.dqk + w.dv))) * 4 / 1e6),
            "parallelism": "dp%d (independent batches, no collective)" % world}


def attention_kernel_name(kind, dqk, sq):
    """The kernel launch_attention runs: the paired one (two query tiles per
    CTA) for BF16 at d = 128 with more than 64 query tiles of 128 rows, else
    the single-tile one."""
    return "attn_pp_kernel" if kind == "bf16" and dqk == 128 and (sq + 127) // 128 > 64 else "attn_fwd_kernel"


def roofline_dict(kind, flops, m, tkey, dqk, sq):
    peak, peak_src = tensor_peak(kind)
    achieved = flops / (m["attn_ms"] * 1e-3) / 1e12
    traffic, traffic_stale = load_traffic(tkey)
    r = {"bound": "tensor", "kernel": attention_kernel_name(kind, dqk, sq), "achieved": round(achieved, 1),
         "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
         "peak_source": peak_src,
         "frac_of_datasheet_dense": round(achieved / DATASHEET_DENSE_TFLOPS[kind], 4),
         "datasheet_dense_tflops": DATASHEET_DENSE_TFLOPS[kind],
         "traffic": traffic, "traffic_stale": traffic_stale,
         "kernel_sources_sha256": kernel_sources_digest(),
         "attn_ms": round(m["attn_ms"], 4), "attn_ms_min": round(m["attn_ms_min"], 4),
         "attn_ms_max": round(m["attn_ms_max"], 4)}
    sp = sustained_peak(kind)
    if sp:
        r["frac_of_sustained"] = round(achieved / sp, 4)
    gp = gemm_peaks()
    if gp and gp.get("%s_tflops" % ("fp8_e4m3" if kind == "fp8" else "bf16")):
        g = gp["%s_tflops" % ("fp8_e4m3" if kind == "fp8" else "bf16")]
        r["frac_of_measured_gemm"] = round(achieved / g, 4)
        r["measured_gemm_tflops"] = g
    return r


def run_ours(args, rank, world, w):
    import bf16_causal_prefill_02_b200 as zq  # noqa: F401  (fails loudly without the .so)

    step = Step(w, args.dtype, args.hadamard, seed_offset=rank, T=args.T, per_kv=args.descale == "kv")
    flops = w.causal_flops()
    m = measure(step, args.steps, args.warmup, world, energy=not args.no_energy)
    ms_step = m["ms_step"]
    total_flops = sum_over_ranks(flops, world)
    value = total_flops / (ms_step * 1e-3) / 1e12
    # determinism: two more launches into fresh buffers, compared bit for bit
    o1, o2 = torch.empty_like(step.out), torch.empty_like(step.out)
    step.attention(out=o1)
    step.attention(out=o2)
    torch.cuda.synchronize()
    deterministic = bool(torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and
                         torch.equal(o1.view(torch.int16), step.out.view(torch.int16)))
    del o1, o2
    e2e = None
    if not args.no_e2e:
        e2e_steps = max(3, min(args.steps, 10))
        ms_e2e = time_steps(step.e2e_step, e2e_steps, 2, world) / e2e_steps
        e2e = {"value": round(total_flops / (ms_e2e * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "ms_per_step": round(ms_e2e, 3),
               "h2d_bytes_per_step": step.h2d_bytes(), "d2h_bytes_per_step": step.d2h_bytes()}
    kind = "bf16" if args.dtype == "bf16" else "fp8"
    tkey = "%s_%s_S%d%s" % (w.name.split("_S")[0], args.dtype, w.S, _variant_suffix(args))
    res = {
        "metric": METRIC,
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3" if kind == "fp8" else "bf16", "data": "synthetic",
        "config": config_dict(w, args, world),
        "roofline": roofline_dict(kind, flops, m, tkey, w.dqk, w.S),
        "clocks": m["clocks"],
        "energy": m["energy"],
        "e2e": e2e,
        "gpu_launches": step.launches_per_step() * args.steps,
        "deterministic": deterministic,
    }
    if kind == "fp8":
        res["quant_ms"] = round(m["quant_ms"], 4)
        res["quant_share_of_attention"] = round(m["quant_ms"] / m["attn_ms"], 4)
    return res, step


# Other workloads of the pages' metric, measured after the headline at N=1
# (attention alone and the whole step, with clocks): BF16 at 32K and 16K, FP8
# exact at 32K, MLA 16K, GQA 4K and long 16K (energy: the pages' TFLOP/J
# figures are on those two layer shapes), long 16K with the Hadamard rotation,
# and the headline with headroom T = 0 (clock study).
EXTRAS = [
    # name, S, dtype, hadamard, T, energy
    ("gauss", 32768, "bf16", False, 8, False),
    ("gauss", 16384, "bf16", False, 8, False),
    ("gauss", 32768, "exact", False, 8, False),
    ("gauss", 16384, "leanp", False, 8, False),
    ("mla", None, "leanp", False, 8, False),
    ("mla", None, "bf16", False, 8, False),
    ("gqa", None, "leanp", False, 8, True),
    ("gqa", None, "bf16", False, 8, True),
    ("long", None, "leanp", False, 8, True),
    ("long", None, "leanp", True, 8, True),
    ("long", None, "exact", True, 8, False),
    ("gauss", 32768, "leanp", False, 0, True),
]


def run_extras(args, world, steps):
    out = []
    cache = {}
    for name, S, dt, had, T, energy in EXTRAS:
        w = workloads.get(name, S)
        if w.name not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            cache[w.name] = [t.pin_memory() for t in workloads.make_inputs(w)]
        step = Step(w, dt, had, T=T, host_inputs=cache[w.name])
        m = measure(step, steps, 3, world, energy=energy)
        kind = "bf16" if dt == "bf16" else "fp8"
        attn = m["flops"] / (m["attn_ms"] * 1e-3) / 1e12
        peak, _ = tensor_peak(kind)
        e = {"w": "%s_%s%s%s" % (w.name, dt, "_hadamard" if had else "", "_T%d" % T if T != 8 else ""),
             "attn_tflops": round(attn, 1), "step_tflops": round(m["flops"] / (m["ms_step"] * 1e-3) / 1e12, 1),
             "frac": round(attn / peak, 3), "frac_dense": round(attn / DATASHEET_DENSE_TFLOPS[kind], 3),
             "attn_ms": [round(m["attn_ms"], 3), round(m["attn_ms_min"], 3), round(m["attn_ms_max"], 3)],
             "sm_mhz": m["clocks"].get("sm_mhz"), "reasons": m["clocks"].get("reasons")}
        if m["quant_ms"] is not None:
            e["quant_share"] = round(m["quant_ms"] / m["attn_ms"], 4)
        if m["energy"]:
            e["tflop_per_j"] = m["energy"]["tflop_per_joule"]
            e["energy_mhz"] = m["energy"]["sm_mhz"]
        out.append(e)
        del step
    cache.clear()
    torch.cuda.empty_cache()
    return out


METRIC = "causal prefill attention TFLOP/s (FP8, BF16) at S=16K/32K; % of B200 tensor peak"


def gemm_peak_run():
    """Library GEMM throughput on this GPU (cuBLASLt through torch), M=N=K=8192,
    local tensors: FP8 e4m3 (torch._scaled_mm, fp32 scales, bf16 out) and
    BF16 (torch.mm).  Burst figure: 20 launches after warm-up, CUDA events."""
    dev = torch.device("cuda")
    n = 8192
    a = torch.randn((n, n), device=dev)
    b = torch.randn((n, n), device=dev)
    res = {}
    st = torch.cuda.current_stream()
    one = torch.ones((), device=dev)
    a8 = a.to(torch.float8_e4m3fn)
    b8 = b.to(torch.float8_e4m3fn).t().contiguous().t()  # column-major second operand
    ab, bb = a.bfloat16(), b.bfloat16()
    cases = {"fp8_e4m3": lambda: torch._scaled_mm(a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16),
             "bf16": lambda: torch.mm(ab, bb)}
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    time.sleep(0.25)
    for name, fn in cases.items():
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(20):
            fn()
        e1.record(st)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 20
        res["%s_tflops" % name] = round(2.0 * n ** 3 / (ms * 1e-3) / 1e12, 1)
    res["clocks"] = sampler.stop()
    res["shape"] = "M=N=K=%d, 20 launches after 5 warm-up, CUDA events" % n
    res["device"] = torch.cuda.get_device_name(0)
    return res


def _pair_trace(dbg, off, w, args, t, bh):
    """The paired kernel's trace (one team: the traced 128-row tile t):
    per 64-key tile j, team slots [0] S_j seen, [1] loaded, [2] P_j
    computed, [3] released (warp 0 of the team); its issuer: [4] QK_j issue
    starts, [5] QK_j committed, [6] P_j seen, [7] PV_j committed."""
    tr = dbg[off:].cpu().numpy().view(np.uint64)[: 512 * 16].reshape(512, 2, 8)[:, t & 1].astype(np.int64)
    n = min((128 * t + 127) // 64 + 1, 512)
    lo, hi = 20, n - 2
    if hi - lo < 8:
        lo, hi = 1, n - 2
    r, nxt = tr[lo:hi], tr[lo + 1:hi + 1]
    med = lambda x: float(np.median(x))
    out = {
        "trace": "%s tile %d of flat head %d (team %d of its pair, %d key tiles of 64), SM cycles, medians over "
                 "tiles %d..%d" % (w.name + "_" + args.dtype, t, bh, t & 1, n, lo, hi - 1),
        "period_cycles": med(np.diff(tr[lo:hi + 1, 3])),
        "softmax": {"S_ready_after_QK_commit_issue": med(r[:, 0] - r[:, 5]), "S_load": med(r[:, 1] - r[:, 0]),
                    "P_compute": med(r[:, 2] - r[:, 1]), "P_store_and_release": med(r[:, 3] - r[:, 2]),
                    "next_S_seen_after_release": med(nxt[:, 0] - r[:, 3])},
        "issuer": {"P_seen_after_release": med(r[:, 6] - r[:, 3]), "PV_issue": med(r[:, 7] - r[:, 6]),
                   "next_QK_start_after_S_load": med(nxt[:, 4] - r[:, 1]), "QK_issue": med(r[:, 5] - r[:, 4])},
    }
    return out


def pipeline_trace(args, w):
    """Per-role timing of one unit from the debug instantiation's clock64
    trace (SM cycles), medians over the unit's key tiles 20 .. n-2.  The
    debug kernel carries the trace stores, so absolute times run a little
    long; the shares between roles are the point.  Slots: softmax warp 0
    saw S_j [0], loaded it [1], computed P_j [2], released it [3]; warps 3,
    1, 5 released P_j [4], [11], [12] (warps 1 and 5 share their SM
    sub-partition with the MMA issuer); MMA issuer: K_j landed and QK_j
    issue starts [5], QK_j issued and committed [6], P_j seen [7], scales
    copied [8], PV_j issued [9] and committed [10]."""
    import bf16_causal_prefill_02_b200 as zq

    step = Step(w, args.dtype, args.hadamard, T=args.T)
    step.step()
    torch.cuda.synchronize()
    n_tiles = (w.S + 127) // 128
    t = min(n_tiles - 1, 200)
    bh = min(5, w.B * w.Hq - 1)
    dbg = torch.zeros(zq.ZQ_DEBUG_BYTES // 4, dtype=torch.int32, device="cuda")
    kw = dict(out=step.out, lse=step.lse, debug=dbg, debug_at=(bh, t))
    if args.dtype == "bf16":
        zq.attn_fwd(step.qb, step.kb, step.vb, **kw)
    else:
        zq.attn_fwd(step.qc, step.kc, step.vc, q_descale=step.dsq, k_descale=step.dsk, v_descale=step.dsv,
                    softmax_mode=step.mode, block_scale=True, headroom_T=step.T, **kw)
    torch.cuda.synchronize()
    off = 128 * 128 + 128 * 64 + 256
    if attention_kernel_name("bf16" if args.dtype == "bf16" else "fp8", w.dqk, w.S) == "attn_pp_kernel":
        return _pair_trace(dbg, off, w, args, t, bh)
    tr = dbg[off:].cpu().numpy().view(np.uint64)[: 512 * 16].reshape(512, 16).astype(np.int64)
    n = t + 1 if w.S > 0 else 0
    lo, hi = 20, n - 2
    if hi - lo < 8:
        lo, hi = 1, n - 2
    r = tr[lo:hi]
    nxt = tr[lo + 2:hi + 2]
    med = lambda x: float(np.median(x))
    rel = np.stack([r[:, 3], r[:, 4], r[:, 11], r[:, 12]], axis=1)
    last = rel.max(axis=1)
    out = {
        "trace": "%s tile %d of flat head %d (%d key tiles), SM cycles, medians over tiles %d..%d"
                 % (w.name + "_" + args.dtype, t, bh, n, lo, hi - 1),
        "period_cycles": med(np.diff(tr[lo:hi + 1, 3])),
        "softmax": {"S_ready_after_QK_commit_issue": med(r[:, 0] - r[:, 6]),
                    "S_load": med(r[:, 1] - r[:, 0]), "P_compute": med(r[:, 2] - r[:, 1]),
                    "P_store_and_release_warp0": med(r[:, 3] - r[:, 2]),
                    "release_after_warp0": {"warp3": med(r[:, 4] - r[:, 3]), "warp1": med(r[:, 11] - r[:, 3]),
                                            "warp5": med(r[:, 12] - r[:, 3])}},
        "mma": {"P_seen_after_last_release": med(r[:, 7] - last), "scales_copied": med(r[:, 8] - r[:, 7]),
                "PV_issued": med(r[:, 9] - r[:, 8]), "PV_committed": med(r[:, 10] - r[:, 9]),
                "next_QK_start_after_PV_commit": med(nxt[:, 5] - r[:, 10]),
                "QK_issue": med(r[:, 6] - r[:, 5])},
    }
    out["share_of_period"] = {
        "softmax_warp0_busy": round((out["softmax"]["S_load"] + out["softmax"]["P_compute"] +
                                     out["softmax"]["P_store_and_release_warp0"]) / out["period_cycles"], 3),
        "last_release_lag": round(med(last - r[:, 3]) / out["period_cycles"], 3),
        "mma_issue_PV_and_QK": round((med(r[:, 9] - r[:, 7]) + out["mma"]["QK_issue"]) / out["period_cycles"], 3)}
    return out


def main():
    args = parse()
    w = workloads.get(args.workload, args.S)
    if args.trace:
        torch.cuda.set_device(0)
        print(json.dumps(pipeline_trace(args, w)), flush=True)
        return
    if args.gemm_peaks:
        torch.cuda.set_device(0)
        print(json.dumps(gemm_peak_run()), flush=True)
        return
    if args.impl == "reference":
        # host-only: rank 0 times the oracle, the other ranks exit without
        # work (no process group, no GPU)
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank == 0:
            # each step a bounded sample: about 0.1-0.3 s of oracle work at 32K
            rows = max(32, min(1024, int(256 * 32768 / max(w.S, 1))))
            tf, ms, cores, desc = oracle_steps(w, args.dtype, args.steps, args.warmup, rows, args.hadamard,
                                                args.descale == "kv")
            line = {"impl": "reference", "metric": METRIC, "value": tf, "unit": "TFLOP/s",
                    "n_gpus": world, "steps": args.steps,
                    "warmup": args.warmup, "ms_per_step": round(ms, 3),
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                    "dtype": "f64", "data": "synthetic",
                    "config": config_dict(w, args, world),
                    "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                     "sample": desc, "cpu_model": cpu_model()},
                    "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                            "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    res, step = run_ours(args, rank, world, w)
    if world == 1 and not args.no_extra:
        res["also"] = run_extras(args, world, min(args.steps, 10))
    if rank == 0 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline_leg(w, args.dtype, args.cpu_seconds, args.hadamard,
                                               args.descale == "kv", step=step)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
