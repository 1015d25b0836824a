"""Benchmark: exact attention forward (and backward) TFLOP/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one forward pass (all steps of the forward path in one kernel
launch) over the 4x16x4096x128 non-causal workload, inputs resident in HBM.
The JSON line also reports the 16384-token causal forward and the
forward+backward workload (backward timed alone) as extra sub-objects, a
roofline entry for the forward kernel, SM clocks sampled during the timed
region, an end-to-end number through the C ABI with host buffers (pinned
host -> device copies and the device -> host read of O and LSE inside the
timed region) and the fp64 oracle timed on a bounded sample on the host.

FLOP convention: forward 4*B*H*N^2*d, halved when causal; backward 2.5x that.
Multi-GPU (torchrun): every rank runs its own copy of the workload (heads are
independent -- no collective on the data path); value = all ranks' FLOPs /
the slowest rank's time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused attention fwd/bwd TFLOP/s and % of B200 dense-BF16 tensor-core peak"
UNIT = "TFLOP/s"
HEADLINE = "b4_h16_n4096_d128"
DROPOUT_P = 0.1  # attention-dropout rate of the dropout extras (the pages' attn_dropout = 0.1)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's B200 dense (no 2:4 sparsity) BF16 tensor figure, for context only;
# the roofline uses the measured peak.
NOMINAL_DENSE_BF16_TFLOPS = 2250.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha1()
    for name in ("fa_fwd.cuh", "sm100.cuh", "philox.cuh"):
        with open(os.path.join(ROOT, "io_aware_exact_31_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def recorded_traffic():
    """DRAM bytes per forward launch from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "fwd_traffic.txt")
    d = {}
    try:
        with open(path) as f:
            for line in f:
                if "=" in line and not line.lstrip().startswith("#"):
                    k, v = line.strip().split("=", 1)
                    d[k] = v
    except OSError:
        return None
    if d.get("kernel_source_sha1_12") != kernel_source_hash():
        return None
    try:
        return int(d["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every
    `period` seconds by a background thread while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period: float = 0.0):
        self.dev, self.period = device_index, period
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = None
        self._thr = None
        self.error = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self._nvml_index(pynvml))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception as e:  # noqa: BLE001 - report, don't fail the bench
            self.error = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for name, bit in self.REASONS.items():
                        if r & bit:
                            self.reasons.add(name)
                except Exception as e:  # noqa: BLE001
                    self.error = str(e)
                    return
                if self.period > 0:
                    self._stop.wait(self.period)

        self._thr = threading.Thread(target=loop, daemon=True)
        self._thr.start()
        return self

    def _nvml_index(self, pynvml):
        # NVML numbers devices by PCI order; map the CUDA device through its bus id.
        try:
            import torch
            bus = torch.cuda.get_device_properties(self.dev).pci_bus_id
            for i in range(pynvml.nvmlDeviceGetCount()):
                hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                if pynvml.nvmlDeviceGetPciInfo(hh).busId.decode().lower().endswith(bus.lower()[-12:]):
                    return i
        except Exception:  # noqa: BLE001
            pass
        return self.dev

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thr.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "samples": 0, "note": self.error}
        return {"sm_mhz": statistics.median(self.samples), "sm_min_mhz": min(self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples),
                "source": "NVML, back-to-back queries" if self.period <= 0
                else f"NVML, {self.period * 1e3:g} ms period"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    """Maximum of x over all ranks (identity for one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_tflops(flops_per_rank: float, world: int, ms_per_step_slowest: float) -> float:
    """Whole-job throughput: every rank's FLOPs over the slowest rank's time."""
    return flops_per_rank * world / (ms_per_step_slowest * 1e-3) / 1e12


def time_region(fn, steps, stream, sync):
    """CUDA-event time of `steps` calls on `stream`, bracketed by sync().  The
    host waits for the end event by polling with short sleeps, so that the
    clock-sampling thread gets the interpreter while the GPU works."""
    import torch
    sync()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    while not end.query():
        time.sleep(20e-6)
    end.synchronize()
    sync()
    return start.elapsed_time(end)  # ms


def run_gpu(args):
    import torch
    import torch.distributed as dist

    from io_aware_exact_31_b200 import binding
    from io_aware_exact_31_b200.workloads import WORKLOADS, workload_inputs

    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_ranks(x: float) -> float:
        return max_over_ranks(x, world, "cuda")

    peaks, peak_src = load_peaks()
    lib = binding.load_library()
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    w = WORKLOADS[HEADLINE]
    if args.only == "fwd" and args.workload:
        w = WORKLOADS[args.workload]

    fp8_cache = {}

    def fp8_args(a):
        """fa_forward_fp8 arguments for the bf16 buffers of `a`, quantised once."""
        if id(a) not in fp8_cache:
            ts, ds = [], []
            for ptr_t in fwd_tensors[id(a)][:3]:
                s_ = float(ptr_t.float().abs().max()) / 448.0
                ts.append((ptr_t.float() / s_).to(torch.float8_e4m3fn))
                ds.append(s_)
            fp8_cache[id(a)] = (ts, ds)
        (q8_, k8_, v8_), ds = fp8_cache[id(a)]
        return (q8_.data_ptr(), k8_.data_ptr(), v8_.data_ptr(), a[3], a[4], *ds, w.B, w.H, w.H,
                w.N, w.d, w.scale, int(w.causal), binding.ctypes.c_void_p(a[-1]))

    fwd_tensors = {}

    def fwd_setup(w):
        x = workload_inputs(w, seed=rank)
        q, k, v = (x[n].cuda() for n in ("Q", "K", "V"))
        o = torch.empty_like(q)
        lse = torch.empty(w.B, w.H, w.N, device="cuda", dtype=torch.float32)
        args_ = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B,
                 w.H, w.N, w.d, w.scale, int(w.causal), sh)
        fwd_tensors[id(args_)] = (q, k, v)
        return x, (q, k, v, o, lse), args_

    def launch_fwd(a):
        st = lib.fa_forward(*a[:-1], binding.ctypes.c_void_p(a[-1]))
        if st != 0:
            raise binding.FaError(st, "fa_forward")

    if args.only == "fwd" and args.fp8:
        # profiler runs of the E4M3 forward: the workload quantised per tensor
        def launch_fwd(a):  # noqa: F811
            st = lib.fa_forward_fp8(*fp8_args(a))
            if st != 0:
                raise binding.FaError(st, "fa_forward_fp8")

    if args.only == "fwd" and args.dropout > 0:
        # profiler runs of the dropout forward: same workload, fa_forward_dropout
        def launch_fwd(a):  # noqa: F811
            st = lib.fa_forward_dropout(*a[:5], None, w.B, w.H, w.H, w.N, w.d, w.scale,
                                        int(w.causal), args.dropout, 1234, 0,
                                        binding.ctypes.c_void_p(a[-1]))
            if st != 0:
                raise binding.FaError(st, "fa_forward_dropout")

    if args.only == "bwd":
        return run_bwd_only(args, torch, binding, WORKLOADS, workload_inputs, rank), rank

    # ---------------- headline: forward on the 4x16x4096x128 workload

    x, bufs, fargs = fwd_setup(w)
    for _ in range(args.warmup):
        launch_fwd(fargs)
    with ClockSampler(local) as clk:
        ms = time_region(lambda: launch_fwd(fargs), args.steps, stream, barrier)
    st, site = binding.check_device_error()
    if st != 0:
        raise RuntimeError(f"device error {site:#x}")
    ms = max_ranks(ms)
    ms_step = ms / args.steps
    tflops = weak_scaling_tflops(w.fwd_flops, world, ms_step)
    per_gpu = w.fwd_flops / (ms_step * 1e-3) / 1e12
    clocks = clk.summary()

    # ---------------- the same forward held for ~1.5 s: power-capped regime,
    # reported against the sustained peak
    sustained = None
    if args.sustained_seconds > 0:
        n_sus = max(args.steps, int(args.sustained_seconds * 1e3 / ms_step))
        with ClockSampler(local) as clk_s:
            ms_s = max_ranks(time_region(lambda: launch_fwd(fargs), n_sus, stream, barrier))
        ms_s /= n_sus
        tf_s = w.fwd_flops / (ms_s * 1e-3) / 1e12
        sustained = {"steps": n_sus, "ms_per_step": round(ms_s, 4),
                     "tflops_per_gpu": round(tf_s, 1),
                     "frac_of_bf16_peak_sustained": round(tf_s / peaks["bf16_tflops_sustained"], 4),
                     "clocks": clk_s.summary()}

    if args.only == "fwd":
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return {"metric": METRIC, "value": round(tflops, 1), "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
                "config": {"workload": f"{w.name} fwd", "dropout_p": args.dropout}, "clocks": clocks,
                "gpu_launches": args.steps}, rank

    # ---------------- e2e through the C ABI with host buffers.  Every step
    # uploads its own Q, K, V from pinned host memory, runs the forward and
    # reads O and LSE back; consecutive steps are pipelined over three
    # streams (upload of step i+1, kernel of step i, download of step i-1) on
    # two device buffer sets, as a caller streaming batches would run them.
    qh, kh, vh = (x[n].pin_memory() for n in ("Q", "K", "V"))
    s_up, s_comp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    dev_sets = []
    for i in range(2):
        q_, k_, v_, o_, lse_ = bufs if i == 0 else tuple(torch.empty_like(t) for t in bufs)
        a_ = (q_.data_ptr(), k_.data_ptr(), v_.data_ptr(), o_.data_ptr(), lse_.data_ptr(), w.B,
              w.H, w.N, w.d, w.scale, int(w.causal), s_comp.cuda_stream)
        dev_sets.append((q_, k_, v_, o_, lse_, a_))
    oh = [torch.empty(bufs[3].shape, dtype=bufs[3].dtype, pin_memory=True) for _ in range(2)]
    lh = [torch.empty(bufs[4].shape, dtype=bufs[4].dtype, pin_memory=True) for _ in range(2)]
    ev_up, ev_comp, ev_down = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_run(n):
        for i in range(n):
            b = i % 2
            q_, k_, v_, o_, lse_, a_ = dev_sets[b]
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_comp[b])  # kernel i-2 has read this input set
                q_.copy_(qh, non_blocking=True)
                k_.copy_(kh, non_blocking=True)
                v_.copy_(vh, non_blocking=True)
                ev_up[b].record(s_up)
            s_comp.wait_event(ev_up[b])
            if i >= 2:
                s_comp.wait_event(ev_down[b])  # outputs of step i-2 have been read back
            launch_fwd(a_)
            ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_comp[b])
                oh[b].copy_(o_, non_blocking=True)
                lh[b].copy_(lse_, non_blocking=True)
                ev_down[b].record(s_down)

    e2e_run(2)
    e2e_steps = max(4, args.steps // 4)
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_up)
    e2e_run(e2e_steps)
    t1.record(s_down)
    t1.synchronize()
    barrier()
    e2e_ms = max_ranks(t0.elapsed_time(t1)) / e2e_steps
    st, site = binding.check_device_error()
    if st != 0:
        raise RuntimeError(f"device error {site:#x}")
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh[0].numel() * oh[0].element_size() + lh[0].numel() * lh[0].element_size()
    del x, bufs, fargs, qh, kh, vh, oh, lh, dev_sets
    torch.cuda.empty_cache()

    # ---------------- extra: 16k causal forward
    extra = {}
    w4 = WORKLOADS["h16_n16384_d128_causal_x2"]
    _, b4, a4 = fwd_setup(w4)
    for _ in range(args.warmup):
        launch_fwd(a4)
    ms4 = max_ranks(time_region(lambda: launch_fwd(a4), args.steps, stream, barrier))
    ms4 /= args.steps
    extra[w4.name] = {"pass": "fwd", "ms": round(ms4, 4),
                      "tflops": round(w4.fwd_flops / (ms4 * 1e-3) / 1e12, 1),
                      "frac_of_bf16_peak": round(w4.fwd_flops / (ms4 * 1e-3) / 1e12 /
                                                 peaks["bf16_tflops"], 4)}
    del b4, a4
    torch.cuda.empty_cache()

    # ---------------- extra: the headline shape with E4M3 operands
    # (quantised once, outside the timed region; per-tensor descales)
    xq, bq, _ = fwd_setup(w)
    q8, k8, v8 = [], [], []
    descales = []
    for t, lst in zip(bq[:3], (q8, k8, v8)):
        s_ = float(t.float().abs().max()) / 448.0
        lst.append((t.float() / s_).to(torch.float8_e4m3fn))
        descales.append(s_)
    q8, k8, v8 = q8[0], k8[0], v8[0]
    o8, l8 = bq[3], bq[4]
    del xq

    def fp8_step():
        binding.forward_fp8(q8, k8, v8, *descales, causal=w.causal, scale=w.scale, out=o8,
                            lse=l8, stream=stream)

    for _ in range(args.warmup):
        fp8_step()
    ms8 = max_ranks(time_region(fp8_step, args.steps, stream, barrier)) / args.steps
    st, site = binding.check_device_error()
    if st != 0:
        raise RuntimeError(f"device error {site:#x}")
    tf8 = w.fwd_flops / (ms8 * 1e-3) / 1e12
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    extra[w.name + "_e4m3"] = {"pass": "fwd", "dtype": "e4m3 (P e4m3, fp32 accumulate)",
                               "ms": round(ms8, 4), "tflops": round(tf8, 1),
                               "frac_of_fp8_peak": round(tf8 / fp8_peak, 4),
                               "fp8_peak": fp8_peak,
                               "fp8_peak_source": "measured bf16_tflops x 2 (nominal 4.5/2.25)"}
    del bq, q8, k8, v8, o8, l8
    torch.cuda.empty_cache()

    # ---------------- extra: the headline forward with attention dropout p = 0.1
    _, bd, _ = fwd_setup(w)
    qd, kd, vd, od, ld = bd

    def drop_fwd_step():
        binding.forward(qd, kd, vd, causal=w.causal, scale=w.scale, out=od, lse=ld,
                        dropout_p=DROPOUT_P, seed=1234, offset=0, stream=stream)

    for _ in range(args.warmup):
        drop_fwd_step()
    msd = max_ranks(time_region(drop_fwd_step, args.steps, stream, barrier)) / args.steps
    st, site = binding.check_device_error()
    if st != 0:
        raise RuntimeError(f"device error {site:#x}")
    extra[w.name + "_dropout"] = {"pass": "fwd", "dropout_p": DROPOUT_P, "ms": round(msd, 4),
                                  "tflops": round(w.fwd_flops / (msd * 1e-3) / 1e12, 1),
                                  "frac_of_bf16_peak": round(w.fwd_flops / (msd * 1e-3) / 1e12 /
                                                             peaks["bf16_tflops"], 4)}
    del bd, qd, kd, vd, od, ld
    torch.cuda.empty_cache()

    # ---------------- extra: forward + backward workload
    w5 = WORKLOADS["b4_h16_n2048_d64_causal_bwd"]
    x5 = workload_inputs(w5, seed=rank)
    q5, k5, v5, do5 = (x5[n].cuda() for n in ("Q", "K", "V", "dO"))
    o5, l5 = binding.forward(q5, k5, v5, causal=True, scale=w5.scale)
    ws = torch.empty(binding.backward_workspace_bytes(w5.B, w5.H, w5.N, w5.d), device="cuda",
                     dtype=torch.uint8)
    dq5, dk5, dv5 = torch.empty_like(q5), torch.empty_like(k5), torch.empty_like(v5)

    def bwd_step():
        binding.backward(q5, k5, v5, o5, do5, l5, causal=True, scale=w5.scale, dq=dq5, dk=dk5,
                         dv=dv5, workspace=ws)

    def fwd5_step():
        binding.forward(q5, k5, v5, causal=True, scale=w5.scale, out=o5, lse=l5)

    def bwd5_drop_step():
        binding.backward(q5, k5, v5, o5, do5, l5, causal=True, scale=w5.scale, dq=dq5, dk=dk5,
                         dv=dv5, workspace=ws, dropout_p=DROPOUT_P, seed=99, offset=0)

    def fwd5_drop_step():
        binding.forward(q5, k5, v5, causal=True, scale=w5.scale, out=o5, lse=l5,
                        dropout_p=DROPOUT_P, seed=99, offset=0)

    def bwd_det_step():
        binding.backward(q5, k5, v5, o5, do5, l5, causal=True, scale=w5.scale, dq=dq5, dk=dk5,
                         dv=dv5, workspace=ws, deterministic=True)

    for _ in range(args.warmup):
        bwd_step()
        fwd5_step()
        bwd_det_step()
    msb = max_ranks(time_region(bwd_step, args.steps, stream, barrier)) / args.steps
    msf = max_ranks(time_region(fwd5_step, args.steps, stream, barrier)) / args.steps
    msbdet = max_ranks(time_region(bwd_det_step, args.steps, stream, barrier)) / args.steps
    for _ in range(args.warmup):
        fwd5_drop_step()
        bwd5_drop_step()
    msfd = max_ranks(time_region(fwd5_drop_step, args.steps, stream, barrier)) / args.steps
    msbd = max_ranks(time_region(bwd5_drop_step, args.steps, stream, barrier)) / args.steps
    st, site = binding.check_device_error()
    if st != 0:
        raise RuntimeError(f"device error {site:#x}")
    extra[w5.name] = {"pass": "fwd+bwd", "fwd_ms": round(msf, 4), "bwd_ms": round(msb, 4),
                      "fwd_tflops": round(w5.fwd_flops / (msf * 1e-3) / 1e12, 1),
                      "bwd_tflops": round(w5.bwd_flops / (msb * 1e-3) / 1e12, 1),
                      "bwd_launches_per_step": 3,
                      "deterministic_bwd": {
                          "ms": round(msbdet, 4),
                          "tflops": round(w5.bwd_flops / (msbdet * 1e-3) / 1e12, 1),
                          "cost_vs_default": round(msbdet / msb - 1.0, 4),
                          "how": "dQ blocks added in ascending key-block order"},
                      "dropout": {"p": DROPOUT_P, "fwd_ms": round(msfd, 4),
                                  "bwd_ms": round(msbd, 4),
                                  "fwd_tflops": round(w5.fwd_flops / (msfd * 1e-3) / 1e12, 1),
                                  "bwd_tflops": round(w5.bwd_flops / (msbd * 1e-3) / 1e12, 1)}}

    # ---------------- extra: grouped-query attention and padded batches on the
    # headline shape (forward) and on the 4x16x2048x64 causal shape (forward +
    # backward).  FLOPs count each query head against its keys (grouped-query)
    # and the real tokens of each batch only (padding).
    def gen(shape, seed_):
        g_ = torch.Generator(device="cpu").manual_seed(seed_)
        return torch.randn(*shape, generator=g_).to(torch.bfloat16).cuda()

    def padded_flops(lens, H_, d_, causal_):
        return sum(4.0 * H_ * n_ * n_ * d_ * (0.5 if causal_ else 1.0) for n_ in lens)

    def time_steps(fn):
        for _ in range(args.warmup):
            fn()
        return max_ranks(time_region(fn, args.steps, stream, barrier)) / args.steps

    hkv = 2
    qg = gen((w.B, w.H, w.N, w.d), 10 + rank)
    kg, vg = gen((w.B, hkv, w.N, w.d), 11 + rank), gen((w.B, hkv, w.N, w.d), 12 + rank)
    og = torch.empty_like(qg)
    lg = torch.empty(w.B, w.H, w.N, device="cuda", dtype=torch.float32)
    msg = time_steps(lambda: binding.forward(qg, kg, vg, causal=w.causal, scale=w.scale, out=og,
                                             lse=lg, stream=stream))
    extra[w.name + "_gqa"] = {"pass": "fwd", "H_kv": hkv, "ms": round(msg, 4),
                              "tflops": round(w.fwd_flops / (msg * 1e-3) / 1e12, 1),
                              "frac_of_bf16_peak": round(w.fwd_flops / (msg * 1e-3) / 1e12 /
                                                         peaks["bf16_tflops"], 4)}
    del kg, vg
    lens = [w.N, 3 * w.N // 4, w.N // 2, w.N // 4][:w.B]
    kp, vp = gen((w.B, w.H, w.N, w.d), 13 + rank), gen((w.B, w.H, w.N, w.d), 14 + rank)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    msp = time_steps(lambda: binding.forward(qg, kp, vp, causal=w.causal, scale=w.scale, out=og,
                                             lse=lg, stream=stream, seqlens=sl))
    fp = padded_flops(lens, w.H, w.d, w.causal)
    extra[w.name + "_padded"] = {"pass": "fwd", "seqlens": lens, "ms": round(msp, 4),
                                 "tflops_real_tokens": round(fp / (msp * 1e-3) / 1e12, 1),
                                 "frac_of_bf16_peak": round(fp / (msp * 1e-3) / 1e12 /
                                                            peaks["bf16_tflops"], 4)}
    del qg, kp, vp, og, lg, sl

    hkv5 = 4
    q5g, do5g = gen((w5.B, w5.H, w5.N, w5.d), 20 + rank), gen((w5.B, w5.H, w5.N, w5.d), 21 + rank)
    k5g, v5g = gen((w5.B, hkv5, w5.N, w5.d), 22 + rank), gen((w5.B, hkv5, w5.N, w5.d), 23 + rank)
    o5g, l5g = binding.forward(q5g, k5g, v5g, causal=True, scale=w5.scale)
    dq5g, dk5g, dv5g = torch.empty_like(q5g), torch.empty_like(k5g), torch.empty_like(v5g)
    msfg = time_steps(lambda: binding.forward(q5g, k5g, v5g, causal=True, scale=w5.scale,
                                              out=o5g, lse=l5g, stream=stream))
    msbg = time_steps(lambda: binding.backward(q5g, k5g, v5g, o5g, do5g, l5g, causal=True,
                                               scale=w5.scale, dq=dq5g, dk=dk5g, dv=dv5g,
                                               workspace=ws, stream=stream))
    k5p, v5p = gen((w5.B, w5.H, w5.N, w5.d), 24 + rank), gen((w5.B, w5.H, w5.N, w5.d), 25 + rank)
    lens5 = [w5.N, 3 * w5.N // 4, w5.N // 2, w5.N // 4][:w5.B]
    sl5 = torch.tensor(lens5, dtype=torch.int32, device="cuda")
    o5p, l5p = binding.forward(q5g, k5p, v5p, causal=True, scale=w5.scale, seqlens=sl5)
    dk5p, dv5p = torch.empty_like(k5p), torch.empty_like(v5p)
    msfp = time_steps(lambda: binding.forward(q5g, k5p, v5p, causal=True, scale=w5.scale,
                                              out=o5p, lse=l5p, stream=stream, seqlens=sl5))
    msbp = time_steps(lambda: binding.backward(q5g, k5p, v5p, o5p, do5g, l5p, causal=True,
                                               scale=w5.scale, dq=dq5g, dk=dk5p, dv=dv5p,
                                               workspace=ws, stream=stream, seqlens=sl5))
    st, site = binding.check_device_error()
    if st != 0:
        raise RuntimeError(f"device error {site:#x}")
    fp5 = padded_flops(lens5, w5.H, w5.d, True)
    extra[w5.name]["gqa"] = {"H_kv": hkv5, "fwd_ms": round(msfg, 4), "bwd_ms": round(msbg, 4),
                             "fwd_tflops": round(w5.fwd_flops / (msfg * 1e-3) / 1e12, 1),
                             "bwd_tflops": round(w5.bwd_flops / (msbg * 1e-3) / 1e12, 1)}
    extra[w5.name]["padded"] = {"seqlens": lens5, "fwd_ms": round(msfp, 4),
                                "bwd_ms": round(msbp, 4),
                                "fwd_tflops_real_tokens": round(fp5 / (msfp * 1e-3) / 1e12, 1),
                                "bwd_tflops_real_tokens": round(2.5 * fp5 / (msbp * 1e-3) / 1e12,
                                                                1)}
    del q5g, do5g, k5g, v5g, o5g, l5g, dq5g, dk5g, dv5g, k5p, v5p, o5p, l5p, dk5p, dv5p, sl5
    torch.cuda.empty_cache()

    # ---------------- extra: the two small workloads, each launch timed alone
    # after a 256 MB write that evicts L2 (their inputs would otherwise stay
    # resident); median over the launches
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def flushed_ms(fn, n):
        evs = []
        for _ in range(n):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        ts = sorted(a.elapsed_time(b) for a, b in evs)
        return ts[len(ts) // 2]

    def host_latency_us(a, n=200):
        """Host-side cost of one call through the C ABI: the enqueue alone
        (fa_forward returning) and the call plus a stream synchronise (the
        latency a caller that waits for the result sees); medians."""
        enq, full = [], []
        for _ in range(n):
            t0 = time.perf_counter()
            launch_fwd(a)
            t1 = time.perf_counter()
            stream.synchronize()
            t2 = time.perf_counter()
            enq.append(t1 - t0)
            full.append(t2 - t0)
        enq.sort()
        full.sort()
        return {"enqueue_us": round(enq[n // 2] * 1e6, 2),
                "call_and_sync_us": round(full[n // 2] * 1e6, 2), "calls": n,
                "note": "host wall clock around the ctypes call (Python overhead included); "
                        "tensor maps come from the library's cache after the first call"}

    for name in ("tiny_n256_d64", "transformer_h8_n1024_d64_causal"):
        ws_ = WORKLOADS[name]
        _, bs_, as_ = fwd_setup(ws_)
        for _ in range(args.warmup):
            launch_fwd(as_)
        msf_ = max_ranks(flushed_ms(lambda: launch_fwd(as_), max(args.steps, 20)))
        extra[name] = {"pass": "fwd", "ms": round(msf_, 4), "l2": "flushed before each launch",
                       "tflops": round(ws_.fwd_flops / (msf_ * 1e-3) / 1e12, 2),
                       "statistic": "median of single launches",
                       "latency_us": host_latency_us(as_)}
        del bs_, as_
    del flush
    torch.cuda.empty_cache()

    # ---------------- extra: the ex2 rate of the headline forward (one exp2 per
    # score) against the nominal 16 per clock per SM at the sampled SM clock
    n_exp = float(w.B * w.H) * w.N * w.N * (0.5 if w.causal else 1.0)
    sm_count = torch.cuda.get_device_properties(local).multi_processor_count
    ex2_peak = 16.0 * sm_count * clocks.get("sm_mhz", 1965.0) * 1e6
    extra["ex2_rate"] = {"workload": HEADLINE, "ex2_per_s": n_exp / (ms_step * 1e-3),
                         "nominal_peak_per_s": ex2_peak,
                         "frac": round(n_exp / (ms_step * 1e-3) / ex2_peak, 4),
                         "peak_basis": f"16 ex2/clk/SM x {sm_count} SMs x sampled sm_mhz"}

    # ---------------- context only: torch's own SDPA kernels on the same box
    try:
        extra["context_torch_sdpa"] = torch_sdpa_context(torch, w, w5, stream, args, max_ranks)
    except ImportError as e:  # a torch without torch.nn.attention
        extra["context_torch_sdpa"] = {"unavailable": f"{type(e).__name__}: {e}"}

    traffic = recorded_traffic()
    achieved = per_gpu
    roofline = {"bound": "tensor", "kernel": "fa_fwd_kernel<128>", "achieved": round(achieved, 1),
                "peak": peaks["bf16_tflops"], "peak_source": f"{peak_src} bf16_tflops (burst)",
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": traffic, "algorithmic_bytes": w.fwd_bytes,
                "algorithmic_flops": w.fwd_flops}

    # The backward of the 4x16x2048x64 causal workload: three launches (pre,
    # main, dQ finalise) timed together by CUDA events; the main kernel's share
    # of that time comes from the committed ncu launch list.
    roofline_bwd = {"bound": "tensor", "kernel": "fa_bwd_pre + fa_bwd_main_kernel<64> + "
                    "fa_bwd_dq (one backward)", "workload": w5.name,
                    "achieved": round(w5.bwd_flops / (msb * 1e-3) / 1e12, 1),
                    "peak": peaks["bf16_tflops"], "peak_source": f"{peak_src} bf16_tflops (burst)",
                    "unit": "TFLOP/s",
                    "frac": round(w5.bwd_flops / (msb * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                    "traffic": None, "algorithmic_bytes": w5.bwd_bytes,
                    "algorithmic_flops": w5.bwd_flops}

    result = {
        "metric": METRIC, "value": round(tflops, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded i.i.d. N(0,1) bf16, per rank)",
        "config": {"workload": f"{HEADLINE} fwd", "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "scale": "1/sqrt(d)", "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (3 x 67 MB)"},
        "frac_of_bf16_peak": round(per_gpu / peaks["bf16_tflops"], 4),
        "frac_of_bf16_peak_sustained": round(per_gpu / peaks["bf16_tflops_sustained"], 4),
        "frac_of_nominal_dense_bf16": round(per_gpu / NOMINAL_DENSE_BF16_TFLOPS, 4),
        "roofline": roofline,
        "roofline_bwd": roofline_bwd,
        "clocks": clocks,
        "sustained": sustained,
        "e2e": {"value": round(w.fwd_flops * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "pipelining": "upload i+1 | kernel i | download i-1 on three streams"},
        "gpu_launches": args.steps,
        "extra": extra,
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result, rank


def torch_sdpa_context(torch, w, w5, stream, args, max_ranks):
    """torch.nn.functional.scaled_dot_product_attention on the headline shape
    (forward) and on the 4x16x2048x64 causal shape (forward + backward), per
    available backend.  Context only: these are library kernels, not this
    library's path, and nothing here feeds a reported value."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    import torch.nn.functional as F

    out = {"note": "library kernels timed for context; not part of this library"}
    g = torch.Generator(device="cpu").manual_seed(0)

    def mk(wl, grad):
        ts = [torch.randn(wl.B, wl.H, wl.N, wl.d, generator=g).to(torch.bfloat16).cuda()
              for _ in range(3)]
        if grad:
            for t in ts:
                t.requires_grad_(True)
        return ts

    def timed(fn, n):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return max_ranks(e0.elapsed_time(e1) / n)

    n = max(10, min(args.steps, 30))
    for be in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION,
               SDPBackend.EFFICIENT_ATTENTION):
        rec = {}
        try:
            with sdpa_kernel([be]):
                q, k, v = mk(w, False)
                ms = timed(lambda: F.scaled_dot_product_attention(q, k, v, is_causal=w.causal), n)
                rec[f"{w.name} fwd"] = {"ms": round(ms, 4),
                                        "tflops": round(w.fwd_flops / (ms * 1e-3) / 1e12, 1)}
                del q, k, v
                q, k, v = mk(w5, True)
                do = torch.randn_like(q)

                def fb():
                    o = F.scaled_dot_product_attention(q, k, v, is_causal=True)
                    o.backward(do)

                msfb = timed(fb, n)
                msf = timed(lambda: F.scaled_dot_product_attention(q, k, v, is_causal=True), n)
                rec[f"{w5.name} fwd"] = {"ms": round(msf, 4),
                                         "tflops": round(w5.fwd_flops / (msf * 1e-3) / 1e12, 1)}
                rec[f"{w5.name} bwd (fwd+bwd minus fwd)"] = {
                    "ms": round(msfb - msf, 4),
                    "tflops": round(w5.bwd_flops / (max(msfb - msf, 1e-6) * 1e-3) / 1e12, 1)}
                del q, k, v, do
        except Exception as e:  # backend not available for this shape or device
            rec["unavailable"] = f"{type(e).__name__}: {str(e).splitlines()[0][:160]}"
        out[be.name] = rec
        torch.cuda.empty_cache()
    return out


def run_bwd_only(args, torch, binding, WORKLOADS, workload_inputs, rank):
    """Backward of the 4x16x2048x64 causal workload alone (for profiler runs);
    --bwd-d 128 takes the same shape at head dimension 128."""
    import dataclasses
    w5 = WORKLOADS["b4_h16_n2048_d64_causal_bwd"]
    if args.bwd_d != w5.d:
        w5 = dataclasses.replace(w5, name=f"b4_h16_n2048_d{args.bwd_d}_causal_bwd", d=args.bwd_d)
    x5 = workload_inputs(w5, seed=rank)
    q, k, v, do = (x5[n].cuda() for n in ("Q", "K", "V", "dO"))
    o, lse = binding.forward(q, k, v, causal=True, scale=w5.scale)
    ws = torch.empty(binding.backward_workspace_bytes(w5.B, w5.H, w5.N, w5.d), device="cuda",
                     dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    p = args.dropout
    if p > 0:
        o, lse = binding.forward(q, k, v, causal=True, scale=w5.scale, dropout_p=p, seed=99)

    def step():
        binding.backward(q, k, v, o, do, lse, causal=True, scale=w5.scale, dq=dq, dk=dk, dv=dv,
                         workspace=ws, dropout_p=p, seed=99, deterministic=args.deterministic)

    for _ in range(args.warmup):
        step()
    stream = torch.cuda.current_stream()
    ms = time_region(step, args.steps, stream, torch.cuda.synchronize) / args.steps
    return {"metric": METRIC, "value": round(w5.bwd_flops / (ms * 1e-3) / 1e12, 1),
            "unit": UNIT, "ms_per_step": round(ms, 4), "steps": args.steps,
            "config": {"workload": f"{w5.name} bwd", "dropout_p": p,
                       "deterministic": args.deterministic},
            "gpu_launches": 3 * args.steps}


def oracle_sample(target_s: float, step_rows: int | None = None):
    """Time the fp64 oracle on a bounded row sample of the headline workload.
    Returns (tflops, seconds, rows, threads)."""
    import numpy as np

    import oracle
    from io_aware_exact_31_b200.workloads import WORKLOADS, bf16_bits, workload_inputs

    w = WORKLOADS[HEADLINE]
    x = workload_inputs(w)
    Q, K, V = (bf16_bits(x[n]) for n in ("Q", "K", "V"))
    rng = np.random.default_rng(1)
    flops_per_row = 4.0 * w.N * w.d  # non-causal
    threads = oracle.num_threads()
    # calibrate on a few rows, then size the sample to about target_s
    probe = rng.choice(w.B * w.H * w.N, size=max(threads, 8), replace=False)
    t0 = time.perf_counter()
    oracle.attention_forward_rows(Q, K, V, w.scale, w.causal, probe)
    dt = time.perf_counter() - t0
    rows = step_rows or int(max(threads, min(200000, target_s / max(dt / probe.size, 1e-6))))
    sample = rng.choice(w.B * w.H * w.N, size=rows, replace=False)
    t0 = time.perf_counter()
    oracle.attention_forward_rows(Q, K, V, w.scale, w.causal, sample)
    dt = time.perf_counter() - t0
    return flops_per_row * rows / dt / 1e12, dt, rows, threads


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo where it exists)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine() or "unknown"


def oracle_baseline(c3_seconds: float):
    """The fp64 oracle timed on this host's cores, workload by workload:
    the 256-token and 8-head 1024-token forwards in full (all threads and one
    thread), the headline forward on a random row sample (about c3_seconds),
    the 16k causal forward on a stated row sample with its full time
    extrapolated, and the 4x16x2048x64 causal forward and backward in full.
    Returns the cpu_baseline object; its value is the headline's sample."""
    import numpy as np

    import oracle
    from io_aware_exact_31_b200.workloads import WORKLOADS, bf16_bits, workload_inputs

    threads = oracle.num_threads()
    per = {}

    def bits(w):
        return {n: bf16_bits(t) for n, t in workload_inputs(w).items()}

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    for name in ("tiny_n256_d64", "transformer_h8_n1024_d64_causal"):
        w = WORKLOADS[name]
        b = bits(w)

        def run(w=w, b=b):
            oracle.attention_forward(b["Q"], b["K"], b["V"], w.scale, w.causal)

        run()  # first touch of the inputs and the thread pool
        t_all = timed(run)
        oracle.set_num_threads(1)
        try:
            t_one = timed(run)
        finally:
            oracle.set_num_threads(threads)
        per[name + " fwd"] = {"run": "full", "seconds": round(t_all, 4),
                              "tflops": w.fwd_flops / t_all / 1e12,
                              "seconds_1_thread": round(t_one, 4),
                              "tflops_1_thread": w.fwd_flops / t_one / 1e12}

    tf3, dt3, rows3, _ = oracle_sample(c3_seconds)
    w3 = WORKLOADS[HEADLINE]
    per[HEADLINE + " fwd"] = {
        "run": f"row sample: {rows3} random query rows of {w3.B * w3.H * w3.N}, seed 1",
        "seconds": round(dt3, 3), "tflops": tf3,
        "full_seconds_extrapolated": round(w3.fwd_flops / (tf3 * 1e12), 1)}

    # 16k causal: every head's rows 0 and N-1 and 254 random rows (seed 1).
    # A causal row i costs (i + 1) key visits, so the full time is the
    # sample's time scaled by all rows' key visits over the sample's.
    w4 = WORKLOADS["h16_n16384_d128_causal_x2"]
    b4 = bits(w4)
    rng = np.random.default_rng(1)
    rows4 = []
    for bh in range(w4.B * w4.H):
        rnd = rng.choice(np.arange(1, w4.N - 1), size=254, replace=False)
        rows4.extend(bh * w4.N + i for i in sorted({0, w4.N - 1, *(int(v) for v in rnd)}))
    rows4 = np.array(rows4, np.int64)
    dt4 = timed(lambda: oracle.attention_forward_rows(b4["Q"], b4["K"], b4["V"], w4.scale,
                                                      w4.causal, rows4))
    visits_sample = float(np.sum(rows4 % w4.N + 1))
    visits_all = float(w4.B * w4.H) * w4.N * (w4.N + 1) / 2
    t4_full = dt4 * visits_all / visits_sample
    per[w4.name + " fwd"] = {
        "run": f"row sample, extrapolated: rows 0, N-1 and 254 random rows (seed 1) of each "
               f"of the {w4.B * w4.H} heads ({rows4.size} rows); full time = sample time x "
               f"(all rows' key visits / the sample's)",
        "seconds": round(dt4, 3), "full_seconds_extrapolated": round(t4_full, 1),
        "tflops": w4.fwd_flops / t4_full / 1e12}
    del b4

    w5 = WORKLOADS["b4_h16_n2048_d64_causal_bwd"]
    b5 = bits(w5)
    dt5f = timed(lambda: oracle.attention_forward(b5["Q"], b5["K"], b5["V"], w5.scale, True))
    dt5b = timed(lambda: oracle.attention_backward(b5["Q"], b5["K"], b5["V"], b5["dO"],
                                                   w5.scale, True))
    per[w5.name + " fwd"] = {"run": "full", "seconds": round(dt5f, 3),
                             "tflops": w5.fwd_flops / dt5f / 1e12}
    per[w5.name + " bwd"] = {"run": "full", "seconds": round(dt5b, 3),
                             "tflops": w5.bwd_flops / dt5b / 1e12}
    return {"value": tf3, "unit": UNIT, "cores": threads, "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"{rows3} random query rows of {HEADLINE} (forward, fp64, {dt3:.1f} s on "
                      f"{threads} threads)",
            "per_workload": per}


def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return None, rank
    # Each step times the oracle on a bounded sample (~2 s), so the whole run
    # stays within a few minutes.
    _, _, rows, threads = oracle_sample(args.ref_step_seconds)
    for _ in range(args.warmup):
        oracle_sample(0, step_rows=max(threads, rows // 8))
    times, flops = [], 0.0
    for _ in range(args.steps):
        tf, dt, r, threads = oracle_sample(0, step_rows=rows)
        times.append(dt)
        flops += 4.0 * 4096 * 128 * r
    total = sum(times)
    value = flops / total / 1e12
    sample = (f"{rows} random query rows of {HEADLINE} per step (forward, fp64 oracle, "
              f"full K/V of each row's head)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{HEADLINE} fwd", "B": 4, "H": 16, "N": 4096, "d": 128,
                   "causal": False},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }, rank


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--sustained-seconds", type=float, default=1.5,
                    help="length of the extra power-capped forward loop (0 to skip)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-step-seconds", type=float, default=2.0,
                    help="host time of one oracle step in --impl reference")
    ap.add_argument("--only", default=None, choices=[None, "fwd", "bwd"],
                    help="time only the headline forward / the backward (profiler runs)")
    ap.add_argument("--workload", default=None,
                    help="workload name of the --only fwd run (default: the headline)")
    ap.add_argument("--fp8", action="store_true",
                    help="--only fwd: time the E4M3 forward of the workload (d = 128)")
    ap.add_argument("--bwd-d", type=int, default=64, choices=[64, 128],
                    help="--only bwd: head dimension of the 4x16x2048 causal backward")
    ap.add_argument("--deterministic", action="store_true",
                    help="--only bwd: the deterministic backward")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="attention-dropout rate of the --only fwd / --only bwd runs")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="target host time of the oracle's headline row sample (0: no CPU "
                         "baseline)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        res, rank = run_reference(args)
        if rank == 0 and res is not None:
            print(json.dumps(res))
        return
    # The oracle sample runs before any CUDA work (the oracle uses OpenMP
    # threads; nothing is forked after CUDA initialisation).
    world, rank, _ = dist_setup(args)
    cpu = None
    if world == 1 and rank == 0 and args.cpu_seconds > 0:
        cpu = oracle_baseline(args.cpu_seconds)
    res, rank = run_gpu(args)
    if rank == 0:
        res["cpu_baseline"] = cpu
        print(json.dumps(res))


if __name__ == "__main__":
    main()
