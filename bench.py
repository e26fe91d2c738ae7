"""Benchmark of the fused attention forward pass on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl reference]

One step = one pass of the hot path over one batch of synthetic input: attn_fwd (plus, for the
K-mean workload, k_smooth_mean_sub -- the K mean and K - mean in one launch -- before it; for the
FP8 workload, the K-smoothing
gate, fp8_quantize of Q, K (smoothed) and V, then attn_fwd_fp8). Inputs are seeded N(0,1) bf16 tensors
of the workload's shape, resident in HBM before timing starts. Each step is timed with CUDA
events on the launching stream; the L2 cache is flushed (a 256 MiB write) before every step,
outside the events. Under torchrun every rank runs its own independent batch (weak scaling, no
data-path collective); the reported time is the max over ranks.

Prints ONE JSON line on rank 0. The metric is attention-forward TFLOP/s with
FLOPs = 2*b*hq*sq*sk*(dqk+dv), halved for causal, also given as a fraction of B200 dense BF16
peak (2250 TFLOP/s datasheet) and of the measured cuBLAS bf16 figure.

--impl reference times the CPU oracle (oracle/, plain fp64 C) on the host cores instead, on a
bounded sample of the same workload's rows per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILED_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
GATE_THRESHOLD = 0.25  # K-smoothing gate threshold of the FP8 recipe and the gate timing
FP8_OVER_BF16 = 2.0    # nominal dense E4M3 / BF16 tensor throughput on B200 (4.5 / 2.25 PFLOP/s)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK), "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    # default: the largest single-GPU workload (b1 h5 65536^2 d128 causal)
    ap.add_argument("--config", type=int, default=5, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with this many query heads (kv heads scaled by the "
                         "same factor): a smaller case of the same kernel, for profiler captures")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU work budget of the oracle baseline sample")
    return ap.parse_args()


# ---------------------------------------------------------------------------------------------
# oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------------------------
def _row_flops(c, rows):
    """Algorithmic FLOPs of the given output rows: 2 * |allowed keys| * (dqk + dv) each."""
    total = 0
    for (_, _, i) in rows:
        d = int(i) + c["sk"] - c["sq"]
        hi = min(c["sk"] - 1, d) if c["causal"] else c["sk"] - 1
        lo = max(0, d - c["window"]) if c.get("window") is not None else 0
        total += 2 * max(hi - lo + 1, 0) * (c["dqk"] + c["dv"])
    return float(total)


class OracleSampler:
    """Times the CPU oracle on seeded row samples of workload c (inputs drawn once)."""

    def __init__(self, c, inputs=None):
        import oracle
        self.oracle = oracle
        self.c = c
        q, k, v = inputs if inputs is not None else workloads.config_inputs(c)
        self.fp8 = bool(c.get("fp8"))
        if self.fp8:
            # the FP8 recipe's inputs, made by the oracle once (gate, smoothing, quantisation)
            # and decoded once; the timed part is the attention on them
            from oracle import fp8 as ofp8
            self.ofp8 = ofp8
            b, hq, hk, sq, sk, d = c["b"], c["hq"], c["hk"], c["sq"], c["sk"], c["dqk"]
            _, m32, _, _ = oracle.k_gate(workloads.bf16_bits(k), b, hk, sk, d, GATE_THRESHOLD)
            q8, dq = ofp8.quantize(workloads.bf16_bits(q), b, sq, hq, d)
            k8, dk = ofp8.quantize(workloads.bf16_bits(k), b, sk, hk, d, mean32=m32)
            v8, dv = ofp8.quantize(workloads.bf16_bits(v), b, sk, hk, c["dv"])
            self.qf = ofp8.dequantize(q8, dq, b, sq, hq, d)
            self.kf = ofp8.dequantize(k8, dk, b, sk, hk, d)
            self.vf = ofp8.dequantize(v8, dv, b, sk, hk, c["dv"])
        if c["kmean"]:
            _, m32 = oracle.k_mean(workloads.bf16_bits(k), c["b"], c["hk"], c["sk"], c["dqk"])
            self.kb = oracle.k_sub(workloads.bf16_bits(k), m32, c["b"], c["hk"], c["sk"], c["dqk"])
        else:
            self.kb = workloads.bf16_bits(k)
        self.qb, self.vb = workloads.bf16_bits(q), workloads.bf16_bits(v)
        self.threads = oracle.default_threads()
        import numpy as np
        self.np = np
        all_rows = workloads.sample_rows(c, n_pos=min(c["sq"], 4096)).numpy()
        rng = np.random.default_rng(3000 + c["id"])
        self.rows = all_rows[rng.permutation(len(all_rows))]
        self.cursor = 0

    def run(self, n_rows):
        np = self.np
        idx = np.arange(self.cursor, self.cursor + n_rows) % len(self.rows)
        self.cursor += n_rows
        rows = self.rows[idx]
        c = self.c
        t0 = time.perf_counter()
        if self.fp8:
            self.ofp8.attn_rows_decoded(self.qf, self.kf, self.vf, c["b"], c["hq"], c["hk"],
                                        c["sq"], c["sk"], c["dqk"], c["dv"], c["causal"],
                                        c["scale"], rows, nthreads=self.threads)
            return time.perf_counter() - t0, _row_flops(c, rows), len(rows)
        sk_logits = workloads.sinks(c)
        self.oracle.attn_rows(self.qb, self.kb, self.vb, c["b"], c["hq"], c["hk"], c["sq"],
                              c["sk"], c["dqk"], c["dv"], c["causal"], c["scale"], rows,
                              nthreads=self.threads,
                              window=c["window"] if c.get("window") is not None else -1,
                              sinks=sk_logits.double().numpy() if sk_logits is not None else None)
        return time.perf_counter() - t0, _row_flops(c, rows), len(rows)

    def rows_for(self, seconds):
        """Rows that take about `seconds` of oracle time (calibrated on a small sample)."""
        n = max(self.threads, 8)
        dt, _, _ = self.run(n)
        while dt < 0.5 and n < len(self.rows) * 64:
            n *= 4
            dt, _, _ = self.run(n)
        return max(1, int(n * seconds / max(dt, 1e-6)))


def varlen_first_sequence(c, inputs):
    """A packed-sequence workload's first sequence as a dense b = 1 config and its inputs."""
    q, k, v, cu_q, cu_k = inputs
    n_q, n_k = int(cu_q[1]), int(cu_k[1])
    c0 = dict(c, b=1, sq=n_q, sk=n_k, varlen=False,
              workload=f"{c['workload']} (sequence 0: {n_q} queries)")
    return c0, (q[:n_q].unsqueeze(0), k[:n_k].unsqueeze(0), v[:n_k].unsqueeze(0))


def cpu_baseline(c, inputs, seconds):
    s = OracleSampler(c, inputs)
    n = s.rows_for(seconds)
    dt, fl, nr = s.run(n)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": s.threads, "kind": "oracle",
            "sample": f"{nr} seeded output rows (all heads/batches, {c['workload']}), "
                      f"{fl / 1e9:.2f} GFLOP in {dt:.1f} s, fp64 plain C oracle"
                      + (" on the oracle's decoded E4M3 recipe inputs" if s.fp8 else "")}


# ---------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event (throttle) reasons during the timed region.

    Polls NVML every few milliseconds from a thread (the timed regions are short); reports None
    when NVML is not available."""

    REASONS = {  # NVML clocks-event reason bits
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, gpu_index, period_s=0.004):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._thread = None
        self._stop = False

    def _poll(self, nvml, h):
        while not self._stop:
            try:
                self.samples.append(nvml.nvmlDeviceGetClockInfo(h, nvml.NVML_CLOCK_SM))
                bits = nvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, bit in self.REASONS.items():
                    if bits & bit:
                        self.reasons.add(name)
            except Exception:  # pragma: no cover
                pass
            time.sleep(self.period)

    def start(self):
        try:
            import pynvml as nvml
            import threading
            nvml.nvmlInit()
            h = nvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = nvml.nvmlDeviceGetMaxClockInfo(h, nvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._poll, args=(nvml, h), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None

    def stop(self):
        if self._thread is None:
            return None
        self._stop = True
        self._thread.join(timeout=5)
        if not self.samples:
            return None
        load = [x for x in self.samples if x > 0.5 * max(self.samples)] or self.samples
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "NVML, polled every 4 ms during the timed region"}


def attn_source_hash():
    """Hash of the attention kernel's sources with comments and blank space removed (profiled
    traffic is valid only for this code; editing a comment does not change it)."""
    import hashlib
    import re
    h = hashlib.sha256()
    d = os.path.join(ROOT, "head_attention_forward_flash_b200", "csrc")
    for f in ("attn_fwd_kernel.cuh", "sm100_ptx.cuh", "attn_api.cu"):
        with open(os.path.join(d, f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)   # block comments
        src = re.sub(r"//[^\n]*", " ", src)                # line comments
        src = re.sub(r"\s+", " ", src)
        h.update(src.encode())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------------------------
# multi-rank plumbing (replicas: every rank runs its own batch; ranks meet only for the barrier
# and the max-over-ranks time)
# ---------------------------------------------------------------------------------------------
def rank_seed(seed: int, rank: int) -> int:
    """Every rank draws its own independent batch."""
    return seed + 7919 * rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of the ranks' x (the slowest rank sets the job's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, flops_per_step: float, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time."""
    return world * flops_per_step / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------------
def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()


    import head_attention_forward_flash_b200 as b2

    c = workloads.with_heads(workloads.config(args.config), args.heads)
    c_rank = dict(c)
    c_rank["seed"] = rank_seed(c["seed"], rank)
    varlen = bool(c.get("varlen"))
    if varlen:  # packed sequences: [total, h, d] tensors and int32 offsets
        q_h, k_h, v_h, cuq_h, cuk_h = workloads.config_varlen_inputs(c_rank)
        cu_q, cu_k = cuq_h.to(dev), cuk_h.to(dev)
        o = torch.empty((q_h.shape[0], c["hq"], c["dv"]), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((c["hq"], q_h.shape[0]), dtype=torch.float32, device=dev)
    else:
        q_h, k_h, v_h = workloads.config_inputs(c_rank)
        o = torch.empty((c["b"], c["sq"], c["hq"], c["dv"]), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((c["b"], c["hq"], c["sq"]), dtype=torch.float32, device=dev)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    mean = torch.empty((c["b"], c["hk"], c["dqk"]), dtype=torch.float32, device=dev)
    k_s = torch.empty_like(k) if c["kmean"] else None
    windowed = c.get("window") is not None or bool(c.get("sinks"))
    fp8 = bool(c.get("fp8"))
    if fp8:  # the recipe's E4M3 buffers and per-(batch, head) descales
        q8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
        k8 = torch.empty(k.shape, dtype=torch.uint8, device=dev)
        v8 = torch.empty(v.shape, dtype=torch.uint8, device=dev)
        dq = torch.empty((c["b"], c["hq"]), dtype=torch.float32, device=dev)
        dk = torch.empty((c["b"], c["hk"]), dtype=torch.float32, device=dev)
        dv = torch.empty((c["b"], c["hk"]), dtype=torch.float32, device=dev)
        gate = torch.empty((c["b"], c["hk"]), dtype=torch.int32, device=dev)
    sk_h = workloads.sinks(c)
    sinks_d = sk_h.to(dev) if sk_h is not None else None
    window = c["window"] if c.get("window") is not None else -1
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # K-mean workload: k_smooth_mean_sub + attention; FP8: the gate, one launch per quantised
    # tensor, attention
    launches_per_step = 2 if c["kmean"] else (5 if fp8 else 1)

    def step():
        kk = k
        if fp8:
            b2.k_smooth_gate(k, GATE_THRESHOLD, mean=mean, gate=gate, return_ratio=False)
            b2.fp8_quantize(q, out=q8, descale=dq)
            b2.fp8_quantize(k, mean=mean, out=k8, descale=dk)
            b2.fp8_quantize(v, out=v8, descale=dv)
            ev_a0.record(stream)
            b2.attn_fwd_fp8(q8, k8, v8, dq, dk, dv, causal=c["causal"], scale=c["scale"], out=o,
                            lse=lse)
            ev_a1.record(stream)
            return
        if c["kmean"]:
            b2.k_smooth_mean_sub(k, mean, k_s)
            kk = k_s
        ev_a0.record(stream)
        if varlen:
            b2.attn_fwd_varlen(q, kk, v, cu_q, cu_k, c["sq"], causal=c["causal"],
                               scale=c["scale"], out=o, lse=lse)
        elif windowed:
            b2.attn_fwd_window_sink(q, kk, v, causal=c["causal"], window_left=window,
                                    sinks=sinks_d, scale=c["scale"], out=o, lse=lse)
        else:
            b2.attn_fwd(q, kk, v, causal=c["causal"], scale=c["scale"], out=o, lse=lse)
        ev_a1.record(stream)

    ev_a0 = torch.cuda.Event(enable_timing=True)
    ev_a1 = torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if b2.attn_debug_status() != 0:
        raise RuntimeError("a kernel reported a bounded-wait timeout during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    a_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    a_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.05)
    for s in range(args.steps):
        flush.zero_()
        starts[s].record(stream)
        ev_a0, ev_a1 = a_starts[s], a_ends[s]
        step()
        ends[s].record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if clocks else None
    if clk is not None and "reasons" in clk and clk["sm_max_mhz"] is None:
        clk["sm_max_mhz"] = clk["sm_mhz"]
    step_ms = [starts[s].elapsed_time(ends[s]) for s in range(args.steps)]
    attn_ms = [a_starts[s].elapsed_time(a_ends[s]) for s in range(args.steps)]
    # the pre-pass (K mean + K subtract, or gate + quantisation): step start -> attention start
    pre_ms = [starts[s].elapsed_time(a_starts[s]) for s in range(args.steps)]
    status = b2.attn_debug_status()
    if status != 0:
        raise RuntimeError(f"a kernel reported status {status} in the timed region")

    ms_local = sum(step_ms) / len(step_ms)
    ms = max_over_ranks(ms_local, world, dev)
    fl = workloads.flops(c)
    value = job_value(world, fl, ms)
    attn_avg_ms = sum(attn_ms) / len(attn_ms)
    achieved = fl / (attn_avg_ms * 1e-3) / 1e12
    peaks, peak_src = measured_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
    peak_note = f"{peak_src} cuBLAS bf16 burst (kernel timed alone)"
    if fp8:  # a contraction takes its own dtype's peak
        peak *= FP8_OVER_BF16
        peak_note = (f"{peak_src} cuBLAS bf16 burst x {FP8_OVER_BF16:g} (nominal E4M3 / BF16 "
                     f"dense ratio; kernel timed alone)")
    traffic = None
    try:
        with open(PROFILED_TRAFFIC_FILE) as f:
            prof = json.load(f)
        if prof.get("attn_source_hash") == attn_source_hash():
            traffic = prof.get(c["workload"])
    except (OSError, ValueError):
        traffic = None
    srt = sorted(attn_ms)
    lo, hi = int(0.1 * len(srt)), max(int(0.9 * len(srt)), int(0.1 * len(srt)) + 1)

    # the K-smoothing gate on the same K (K-mean workload): its own event-timed calls
    kgate = None
    if c["kmean"] or fp8:
        ge0 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
        ge1 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
        for _ in range(3):
            b2.k_smooth_gate(k, GATE_THRESHOLD)
        for s_ in range(10):
            flush.zero_()
            ge0[s_].record(stream)
            b2.k_smooth_gate(k, GATE_THRESHOLD)
            ge1[s_].record(stream)
        torch.cuda.synchronize()
        g_us = 1e3 * statistics.median(ge0[s_].elapsed_time(ge1[s_]) for s_ in range(10))
        stride = (c["sk"] + 2047) // 2048
        n_samp = (c["sk"] + stride - 1) // stride
        g_bytes = c["b"] * n_samp * c["hk"] * c["dqk"] * 2
        kgate = {"us_median": g_us, "sampled_bytes": g_bytes,
                 "gbs": g_bytes / (g_us * 1e-6) / 1e9, "threshold": GATE_THRESHOLD,
                 "launches": 2, "note": "k_smooth_gate alone, L2 flushed before each call"}

    # Workloads whose step has no pre-pass: the K-smoothing pre-pass kernels timed beside the
    # step (not inside it) on this workload's own K, so that every bench line carries their
    # HBM rate. Each call alone, event-timed, L2 flushed before it.
    prepass_beside = None
    if not (c["kmean"] or fp8 or varlen) and c["dqk"] in (64, 128, 256):
        hbm = measured_peaks()[0].get("hbm_gbs", FALLBACK["hbm_gbs"])
        n_kb = k.numel() * 2
        k_tmp = torch.empty_like(k)
        m_tmp = torch.empty_like(mean)
        calls = {
            "k_smooth_mean": (lambda: b2.k_smooth_mean(k, m_tmp), n_kb,
                              "read K once"),
            "k_smooth_mean_sub": (lambda: b2.k_smooth_mean_sub(k, m_tmp, k_tmp), 3 * n_kb,
                                  "read K, read it again, write K - mean"),
            "k_smooth_gate": (lambda: b2.k_smooth_gate(k, GATE_THRESHOLD, mean=m_tmp,
                                                       return_ratio=False),
                              c["b"] * ((c["sk"] + (c["sk"] + 2047) // 2048 - 1)
                                        // ((c["sk"] + 2047) // 2048)) * c["hk"] * c["dqk"] * 2,
                              "read the strided key sample"),
        }
        prepass_beside = {"note": "not part of the step: each kernel alone on this workload's K, "
                                  "L2 flushed before each call, median of 10",
                          "measured_hbm_gbs": hbm}
        for name, (fn, nbytes, what) in calls.items():
            e0 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
            e1 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
            for _ in range(3):
                fn()
            for s_ in range(10):
                flush.zero_()
                e0[s_].record(stream)
                fn()
                e1[s_].record(stream)
            torch.cuda.synchronize()
            us = 1e3 * statistics.median(e0[s_].elapsed_time(e1[s_]) for s_ in range(10))
            gbs = nbytes / (us * 1e-6) / 1e9
            prepass_beside[name] = {"us_median": us, "bytes": nbytes, "bytes_are": what,
                                    "gbs": gbs, "frac_of_measured_hbm": gbs / hbm,
                                    "frac_of_datasheet_8tbs": gbs / 8000.0}
        del k_tmp, m_tmp
        if b2.attn_debug_status() != 0:
            raise RuntimeError("a pre-pass kernel reported a bounded-wait timeout")

    # end to end through the public API with host buffers (pinned), copies inside the timing.
    # Every step copies its own inputs in and its own result out. Two timings:
    #   serial     one stream, step after step (copy in, compute, copy out);
    #   pipelined  three streams and two sets of device buffers: while step s computes, step
    #              s+1's inputs come in and step s-1's result goes out (PCIe is full duplex),
    #              as a serving loop would run it. The reported value.
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        op = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        lp = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        e_steps = max(3, min(args.steps, 10))
        cqp = ckp = None
        if varlen:
            cqp, ckp = cuq_h.pin_memory(), cuk_h.pin_memory()
        skp = sk_h.pin_memory() if sk_h is not None else None

        def device_set():
            """One set of device buffers for a step's inputs, intermediates and outputs."""
            d = {"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
                 "o": torch.empty_like(o), "l": torch.empty_like(lse),
                 "mean": torch.empty_like(mean)}
            if c["kmean"]:
                d["ks"] = torch.empty_like(k)
            if varlen:
                d["cq"], d["ck"] = torch.empty_like(cu_q), torch.empty_like(cu_k)
            if skp is not None:
                d["sk"] = torch.empty_like(sinks_d)
            if fp8:
                d.update(q8=torch.empty_like(q8), k8=torch.empty_like(k8),
                         v8=torch.empty_like(v8), dq=torch.empty_like(dq),
                         dk=torch.empty_like(dk), dv=torch.empty_like(dv),
                         gate=torch.empty_like(gate))
            return d

        def copy_in(d):
            d["q"].copy_(qp, non_blocking=True)
            d["k"].copy_(kp, non_blocking=True)
            d["v"].copy_(vp, non_blocking=True)
            if varlen:
                d["cq"].copy_(cqp, non_blocking=True)
                d["ck"].copy_(ckp, non_blocking=True)
            if skp is not None:
                d["sk"].copy_(skp, non_blocking=True)

        def compute(d):  # the public API, on the current stream, into the set's buffers
            qd, kd, vd = d["q"], d["k"], d["v"]
            if fp8:
                b2.k_smooth_gate(kd, GATE_THRESHOLD, mean=d["mean"], gate=d["gate"],
                                 return_ratio=False)
                b2.fp8_quantize(qd, out=d["q8"], descale=d["dq"])
                b2.fp8_quantize(kd, mean=d["mean"], out=d["k8"], descale=d["dk"])
                b2.fp8_quantize(vd, out=d["v8"], descale=d["dv"])
                b2.attn_fwd_fp8(d["q8"], d["k8"], d["v8"], d["dq"], d["dk"], d["dv"],
                                causal=c["causal"], scale=c["scale"], out=d["o"], lse=d["l"])
                return
            if c["kmean"]:
                b2.k_smooth_mean_sub(kd, d["mean"], d["ks"])
                kd = d["ks"]
            if varlen:
                b2.attn_fwd_varlen(qd, kd, vd, d["cq"], d["ck"], c["sq"], causal=c["causal"],
                                   scale=c["scale"], out=d["o"], lse=d["l"])
            elif windowed:
                b2.attn_fwd_window_sink(qd, kd, vd, causal=c["causal"], window_left=window,
                                        sinks=d.get("sk"), scale=c["scale"], out=d["o"],
                                        lse=d["l"])
            else:
                b2.attn_fwd(qd, kd, vd, causal=c["causal"], scale=c["scale"], out=d["o"],
                            lse=d["l"])

        def copy_out(d):
            op.copy_(d["o"], non_blocking=True)
            lp.copy_(d["l"], non_blocking=True)

        sets = [device_set(), device_set()]
        # serial: one stream, an L2 flush between steps (outside the events)
        ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(e_steps + 1)]
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(e_steps + 1)]
        for st_i in range(e_steps + 1):  # the first one is a warm-up
            flush.zero_()
            ev0[st_i].record(stream)
            copy_in(sets[0])
            compute(sets[0])
            copy_out(sets[0])
            ev1[st_i].record(stream)
        torch.cuda.synchronize()
        serial_ms = max_over_ranks(sum(ev0[i].elapsed_time(ev1[i]) for i in range(1, e_steps + 1))
                                   / e_steps, world, dev)

        # pipelined: inputs of 134 MB and more per step pass through L2 on their way in, so
        # each step meets a cold L2 without a flush
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def run_pipeline(n):
            ready = [torch.cuda.Event() for _ in range(n)]
            done = [torch.cuda.Event() for _ in range(n)]
            out_done = [torch.cuda.Event() for _ in range(n)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(s_in)
            s_out.wait_event(t0)
            for i in range(n):
                d = sets[i % 2]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(done[i - 2])  # set i % 2's inputs consumed
                    copy_in(d)
                    ready[i].record(s_in)
                with torch.cuda.stream(stream):
                    stream.wait_event(ready[i])
                    if i >= 2:
                        stream.wait_event(out_done[i - 2])  # set i % 2's result copied out
                    compute(d)
                    done[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done[i])
                    copy_out(d)
                    out_done[i].record(s_out)
            t1.record(s_out)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1) / n

        run_pipeline(2)  # warm-up
        e_ms = max_over_ranks(run_pipeline(e_steps), world, dev)
        h2d = (q_h.numel() + k_h.numel() + v_h.numel()) * 2
        if varlen:
            h2d += (cuq_h.numel() + cuk_h.numel()) * 4
        if sk_h is not None:
            h2d += sk_h.numel() * 4
        d2h = o.numel() * 2 + lse.numel() * 4
        e2e = {"value": job_value(world, fl, e_ms), "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelined": "3 streams (copy in / compute / copy out), 2 buffer sets",
               "serial_value": job_value(world, fl, serial_ms), "serial_ms_per_step": serial_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if varlen:  # the oracle on rows of the first sequence, as a dense b = 1 problem
            c0, inputs0 = varlen_first_sequence(c, (q_h, k_h, v_h, cuq_h, cuk_h))
            cpu = cpu_baseline(c0, inputs0, args.cpu_seconds)
        else:
            cpu = cpu_baseline(c, (q_h, k_h, v_h), args.cpu_seconds)

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": "attention fwd TFLOP/s (causal-halved) and % of B200 dense BF16 peak",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 (fp32 accumulate)" if fp8 else "bf16",
        "data": "synthetic (seeded N(0,1) bf16)" + (", quantised on the GPU each step" if fp8 else ""),
        "pct_of_dense_bf16_peak": {"value": 100.0 * value / world / DATASHEET_BF16_TFLOPS,
                                   "peak_tflops": DATASHEET_BF16_TFLOPS,
                                   "peak_source": "B200 datasheet dense BF16"},
        "pct_of_measured_bf16": {"burst": 100.0 * value / world / peak,
                                 "sustained": 100.0 * value / world /
                                 peaks.get("bf16_tflops_sustained", FALLBACK[
                                     "bf16_tflops_sustained"]),
                                 "source": peak_src},
        "config": dict({"workload": c["workload"], "b": c["b"], "hq": c["hq"], "hk": c["hk"],
                        "sq": c["sq"], "sk": c["sk"], "dqk": c["dqk"], "dv": c["dv"],
                        "causal": c["causal"], "kmean_prepass": c["kmean"], "scale": c["scale"],
                        "l2": "flushed before every step (256 MiB write, outside the events)",
                        "parallelism": f"replicas x{world} (independent batches, no "
                                       f"collective)"},
                       **({"packed_sequence_lengths": workloads.varlen_lengths(c)}
                          if varlen else {}),
                       **({"window_left": window, "sinks": bool(c.get("sinks")),
                           "flops": "2*b*hq*(dqk+dv)*allowed (query, key) pairs"}
                          if windowed else {}),
                       **({"recipe": "k_smooth_gate (threshold "
                                     f"{GATE_THRESHOLD:g}) + fp8_quantize Q, K - mean, V + "
                                     "attn_fwd_fp8, all inside the step",
                           "scales": "one fp32 descale per (batch, head) per tensor"}
                          if fp8 else {})),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": f"attn_fwd_kernel d{c['dqk']}x{c['dv']}" + (" e4m3" if fp8 else ""),
                     "peak_source": peak_note},
        "dispatch_us": {"median": 1e3 * statistics.median(attn_ms),
                        "trimmed_mean_80": 1e3 * sum(srt[lo:hi]) / max(1, hi - lo),
                        "max": 1e3 * max(attn_ms), "min": 1e3 * min(attn_ms)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if fp8:  # the E4M3 path against its own datasheet figure (4.5 PFLOP/s dense)
        line["pct_of_dense_e4m3_peak"] = {
            "value": 100.0 * value / world / (DATASHEET_BF16_TFLOPS * FP8_OVER_BF16),
            "peak_tflops": DATASHEET_BF16_TFLOPS * FP8_OVER_BF16,
            "peak_source": "B200 datasheet dense E4M3"}
    if kgate is not None:
        line["k_smooth_gate"] = kgate
    if prepass_beside is not None:
        line["prepass_beside_step"] = prepass_beside
    if c["kmean"] or fp8:
        # bytes the pre-pass kernels move by design. K mean: read K; subtract: read K, write K'.
        # FP8: the gate's sampled rows, then per tensor two reads (amax, convert) of bf16 and
        # one write of E4M3 codes.
        n_q = c["b"] * c["sq"] * c["hq"] * c["dqk"]
        n_k = c["b"] * c["sk"] * c["hk"] * c["dqk"]
        n_v = c["b"] * c["sk"] * c["hk"] * c["dv"]
        if fp8:
            stride = (c["sk"] + 2047) // 2048
            sampled = c["b"] * ((c["sk"] + stride - 1) // stride) * c["hk"] * c["dqk"] * 2
            pre_bytes = sampled + 5 * (n_q + n_k + n_v)
            kernels = "k_gate_onepass, 3 x fp8_quant_onepass"
        else:
            pre_bytes = 3 * n_k * 2
            kernels = "k_mean_cols (K mean and K - mean in one launch)"
        pre_us = 1e3 * statistics.median(pre_ms)
        gbs = pre_bytes / (pre_us * 1e-6) / 1e9
        hbm = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
        line["prepass"] = {"us_median": pre_us, "bytes": pre_bytes, "gbs": gbs,
                           "frac_of_measured_hbm": gbs / hbm, "measured_hbm_gbs": hbm,
                           "frac_of_datasheet_8tbs": gbs / 8000.0, "kernels": kernels,
                           "note": "event-timed inside each step, L2 flushed before the step"}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# reference arm: the CPU oracle, as it stands, on the host cores
# ---------------------------------------------------------------------------------------------
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return  # the oracle arm runs on rank 0 only
    c = workloads.with_heads(workloads.config(args.config), args.heads)
    if c.get("varlen"):  # the oracle on rows of the first sequence (a dense b = 1 problem)
        c, inputs0 = varlen_first_sequence(c, workloads.config_varlen_inputs(c))
        s = OracleSampler(c, inputs0)
    else:
        s = OracleSampler(c)
    per_step = max(0.5, min(8.0, 90.0 / max(1, args.steps + args.warmup)))
    n = s.rows_for(per_step)
    for _ in range(args.warmup):
        s.run(n)
    times, fls = [], []
    for _ in range(args.steps):
        dt, fl, _ = s.run(n)
        times.append(dt)
        fls.append(fl)
    value = sum(fls) / sum(times) / 1e12
    ms = 1e3 * sum(times) / len(times)
    sample = (f"{n} seeded output rows per step of {c['workload']} (all heads/batches), "
              f"fp64 plain C oracle"
              + (" on the oracle's decoded E4M3 recipe inputs" if s.fp8 else ""))
    line = {
        "impl": "reference",
        "metric": "attention fwd TFLOP/s (causal-halved) and % of B200 dense BF16 peak",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) bf16)",
        "config": {"workload": c["workload"], "b": c["b"], "hq": c["hq"], "hk": c["hk"],
                   "sq": c["sq"], "sk": c["sk"], "dqk": c["dqk"], "dv": c["dv"],
                   "causal": c["causal"], "kmean_prepass": c["kmean"],
                   "sample": "bounded row sample per step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": s.threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
