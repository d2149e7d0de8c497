#!/usr/bin/env python
"""Benchmark: MoE layer forward+backward tokens/s on B200 (one replica per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload e128_bf16]
                    [--impl ours|reference] [--router] [--no-cpu-baseline]

One step is one pass of the whole hot path over one batch already resident in HBM:
routing, dispatch, grouped GEMM forward (FC1 + SwiGLU, FC2), combine, combine
backward, grouped GEMM backward (two dgrads, two wgrads), unpermute-reduce.  The
default workload is T=16384 tokens, d=2048, E=128 experts, top-4, d_ff=1024, bf16,
iid N(0,1) routing logits.  Under torchrun every rank runs its own replica on its own
GPU (tokens are independent; there is no exchange on the data path): weak scaling.

Prints one JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle on a
bounded token sample of the same workload instead.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "MoE layer fwd+bwd tokens/s at E=128 top-4; grouped-GEMM % of tensor peak"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="e128_bf16")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--router", action="store_true", help="compute logits = x.Wr on the device")
    ap.add_argument("--recompute", action="store_true",
                    help="activation recompute: the backward redoes dispatch, FC1 and FC2")
    ap.add_argument("--capacity", default=None,
                    help="capacity-padded layout (the comparator of the device-scheduled grouped "
                         "GEMM): 'auto' = the largest expert count of this routing, or a number")
    ap.add_argument("--shared-expert", action="store_true",
                    help="one shared expert (dense SwiGLU FFN on every token); the step is then "
                         "timed through the whole-layer calls")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flushed-reps", type=int, default=10,
                    help="L2-flushed timings of the HBM-bound stages (0 skips them)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--e2e-steps", type=int, default=30, help="0 skips the end-to-end leg")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (a smaller case of the workload, for profiling)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (a smaller case of the workload, for profiling)")
    ap.add_argument("--dtype", default=None, choices=["fp32", "bf16", "mxfp8"],
                    help="override the workload's GEMM precision (e.g. the MXFP8 shape in bf16)")
    return ap.parse_args()


# ------------------------------------------------------------------------------ helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    sm_max_mhz=d.get("sm_max_mhz"), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback",
                sm_max_mhz=1965.0)


# Nominal B200 figures (context beside the measured denominators): dense bf16 tensor
# throughput and the HGX HBM3e bandwidth.  Other precisions scale by the nominal ratios.
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 7700.0
DTYPE_RATIO = {"bf16": 1.0, "tf32": 1.1 / 2.25, "fp8": 4.5 / 2.25}


def tensor_peak(pk: dict, kind: str, clk: dict, timed_s: float) -> dict:
    """Tensor-core denominators of a GEMM of dtype `kind` timed in this run.

    The measured burst figure (a matmul timed alone, at full clock) applies when the
    run held the SM clock near its maximum through a short timed region; otherwise the
    sustained figure (the same matmul looped for seconds under the power cap).  Both
    fractions are reported, with the nominal dense peak for context."""
    r = DTYPE_RATIO[kind]
    burst, sustained = pk["bf16"] * r, pk["bf16_sustained"] * r
    sm, smax = clk.get("sm_mhz"), clk.get("sm_max_mhz") or pk.get("sm_max_mhz")
    at_max = bool(sm and smax and sm >= 0.95 * smax)
    use_burst = at_max and timed_s < 5.0
    how = {"bf16": "", "tf32": " x 1.1/2.25 (nominal tf32/bf16)",
           "fp8": " x 4.5/2.25 (nominal fp8/bf16)"}[kind]
    why = (f"burst: median SM clock {sm} MHz within 5% of {smax} MHz over a {timed_s:.2f} s "
           f"timed region" if use_burst else
           f"sustained: median SM clock {sm} MHz (max {smax} MHz) over a {timed_s:.2f} s "
           f"timed region")
    return {"peak": burst if use_burst else sustained, "burst": burst, "sustained": sustained,
            "nominal": NOMINAL_BF16_TFLOPS * r, "which": "burst" if use_burst else "sustained",
            "why": why, "kind": f"dense bf16{how}"}


def workload_desc(w):
    return (f"{w.name}: T={w.T}, d_model={w.d}, E={w.E}, top-{w.k}, SwiGLU d_ff={w.d_ff}, "
            f"{w.dtype}, " + ("logits = x.Wr on device" if w.router else
                              ("Zipf-skewed " if w.skew else "") + "iid N(0,1) routing logits"))


def stage_launches(w, keep_codes: bool) -> dict:
    """This library's kernel launches per call of each bench stage (the line's
    `gpu_launches` claim), following the library's own dispatch: routing is top-k + slots
    (+ a scan launch above 256 experts); the fp32 GEMM calls first round both weights to
    TF32 copies; MXFP8 adds the scale-prefix and quantiser launches (the backward's two
    weight passes are skipped when the forward kept the weight codes); the wgrad calls
    build their per-expert tensor maps with one launch."""
    mx, f32 = w.dtype == "mxfp8", w.dtype == "fp32"
    route = 3 if w.E > 256 else 2
    if mx:    # prefix, x rowwise, W13, FC1 (+ a's codes), W2, FC2
        fwd, bwd = 6, (10 if keep_codes else 12)
    else:     # (2 TF32 weight copies) FC1, FC2 | (2 copies) maps, FC2 dgrad, FC2 wgrad, FC1 dgrad, FC1 wgrad
        fwd, bwd = (4, 7) if f32 else (2, 5)
    # router: one GEMM; its backward: fp32 two CUDA-core GEMMs; bf16 a bf16 copy of
    # d_logits, two tensor-core GEMMs and their maps, and the add into dx (E % 64 == 0),
    # else two CUDA-core GEMMs and the add
    router_bwd = 2 if f32 else (5 if w.E % 64 == 0 else 3)
    n = {"router": 1, "route": route, "dispatch": 1, "gemm_fwd": fwd, "combine": 1,
         "combine_bwd": 1, "gemm_bwd": bwd, "dispatch_bwd": 1, "router_bwd": router_bwd}
    n["re_dispatch"], n["re_gemm_fwd"] = n["dispatch"], n["gemm_fwd"]
    # whole-layer calls (the shared-expert runs): routing, dispatch, 2 GEMMs, 2 shared-expert
    # GEMMs, combine (+ router); combine backward, the backward GEMMs, 5 shared-expert
    # launches, unpermute (+ router: bf16 copy, maps, 2 GEMMs)
    n["layer_fwd"] = route + 1 + fwd + 2 + 1 + (1 if w.router else 0)
    n["layer_bwd"] = 1 + bwd + 5 + 1 + (4 if w.router else 0)
    return n


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        with open(self.tmp.name) as fh:
            rows = [r.strip().split(", ") for r in fh if r.strip()]
        os.unlink(self.tmp.name)
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                power.append(float(r[3]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


class NvmlSampler:
    """SM clock and board power read in-process every ~2 ms while the timed steps run.

    nvidia-smi samples every 100 ms at best, so a timed region of a few tens of ms holds
    one sample or none, and the idle clock before it dominates the record.  NVML is read
    here from a thread, started right before the first timed launch and stopped right
    after the synchronize that ends the region (the GPU runs the queued steps meanwhile).
    The device is matched by PCI bus id (falls back to the index)."""

    def __init__(self, dev_index: int):
        self.h, self.samples, self.thread, self.stop_flag = None, [], None, False
        try:
            import pynvml
            self.nv = pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(dev_index)
            try:
                bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id,
                                            props.pci_device_id)
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:  # noqa: BLE001
                self.h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
        except Exception:  # noqa: BLE001
            self.h = None

    def _run(self):
        nv = self.nv
        while not self.stop_flag:
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0))
            except Exception:  # noqa: BLE001
                return
            time.sleep(0.002)

    def start(self):
        if self.h is None:
            return
        import threading
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self) -> dict:
        if self.thread is None:
            return {}
        self.stop_flag = True
        self.thread.join(timeout=5)
        if not self.samples:
            return {}
        sm = [c for c, _ in self.samples]
        pw = [w for _, w in self.samples]
        return {"sm_mhz": statistics.median(sm), "sm_mhz_min": min(sm), "samples": len(sm),
                "power_w_median": round(statistics.median(pw), 1), "power_w_max": round(max(pw), 1)}


def dist_setup():
    """One process per GPU under torchrun (NCCL); gloo when no GPU is visible (CPU runs of
    the multi-rank bookkeeping and of the reference arm)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's value (timing is reported as the max over ranks)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank: int, steps: int, ms_max: float) -> float:
    """Units all ranks processed per second, over the slowest rank's time."""
    return world * units_per_rank * steps / (ms_max / 1e3)


# ------------------------------------------------------------------------------ oracle timing
def oracle_sample_run(w, inp_cpu: dict, T_s: int):
    """One oracle fwd+bwd over the first T_s tokens of the workload; returns seconds."""
    import oracle
    x = inp_cpu["x"][:T_s].double().numpy()
    dy = inp_cpu["dy"][:T_s].double().numpy()
    W13, W2 = inp_cpu["W13np"], inp_cpu["W2np"]
    Wr = None if inp_cpu["Wr"] is None else inp_cpu["Wr"].double().numpy()
    L = None if inp_cpu["logits"] is None else inp_cpu["logits"][:T_s].double().numpy()
    t0 = time.perf_counter()
    fwd = oracle.layer_fwd(x, W13, W2, logits=L, Wr=Wr if L is None else None, k=w.k,
                           mx=w.dtype == "mxfp8")
    oracle.layer_bwd(fwd, dy, x, W13, W2, Wr=Wr, mx=w.dtype == "mxfp8")
    return time.perf_counter() - t0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:  # noqa: BLE001
        pass
    return len(os.sched_getaffinity(0))


def host_inputs(w, dev_inp: dict) -> dict:
    """The bench's own inputs on the host (weights as float32 numpy for the oracle)."""
    out = {k: (None if v is None else v.cpu()) for k, v in dev_inp.items()}
    out["W13np"] = dev_inp["W13"].float().cpu().numpy()
    out["W2np"] = dev_inp["W2"].float().cpu().numpy()
    return out


def cpu_baseline(w, inp_cpu, target_s: float) -> dict:
    """Oracle tokens/s on a bounded token sample: grown (at most 5 calls, each at most 4x
    the last) until one call takes about target_s seconds."""
    # MXFP8: the oracle quantises the weights of every expert a sample touches (several
    # seconds per expert at d=4096), so the sample is one token (its k experts) and stays so
    mx = w.dtype == "mxfp8"
    T_s = min(1 if mx else 64, w.T)
    t = oracle_sample_run(w, inp_cpu, T_s)
    for _ in range(0 if mx else 4):
        if t >= 0.6 * target_s or T_s >= w.T:
            break
        T_s = int(min(w.T, max(T_s + 1, T_s * min(4.0, target_s / max(t, 1e-3)))))
        t = oracle_sample_run(w, inp_cpu, T_s)
    return {"value": T_s / t, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 NumPy oracle fwd+bwd on the first {T_s} of {w.T} tokens of the same "
                      f"workload (the experts those tokens select), one call, {t:.1f} s"}


# ------------------------------------------------------------------------------ reference arm
def run_reference(args, w, world, rank):
    if rank != 0:
        return
    from routing_grouped_gemm_route_b200.inputs import make_inputs
    inp = make_inputs(w, device="cuda" if torch.cuda.is_available() else "cpu")
    inp_cpu = host_inputs(w, inp)
    del inp
    T_s = min(1 if w.dtype == "mxfp8" else 128, w.T)
    for _ in range(args.warmup):
        oracle_sample_run(w, inp_cpu, T_s)
    times = [oracle_sample_run(w, inp_cpu, T_s) for _ in range(args.steps)]
    tot = sum(times)
    value = T_s * args.steps / tot
    sample = (f"fp64 NumPy oracle fwd+bwd on the first {T_s} of {w.T} tokens of the workload per "
              f"step (the experts those tokens select)")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_desc(w), "tokens_per_step": T_s},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def flushed_stage_ms(run_stage, names, dev, reps: int) -> dict:
    """Median CUDA-event time of each named stage run alone after writing a 256 MB
    buffer (twice the 126 MB L2), so none of its inputs starts in L2."""
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    out = {}
    for s in names:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for e0, e1 in ev:
            flush.fill_(1)
            e0.record()
            run_stage(s)
            e1.record()
        torch.cuda.synchronize()
        out[s] = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
    return out


def run_e2e(args, w, desc, act, dev, world, x, dy, logits, W13, W2, Wr, y, dx, d_logits, dW13,
            dW2, dWr):
    """Same metric through the public whole-layer calls, with every step's inputs copied
    from pinned host memory and its results (y, dx) copied back, all inside the timed
    region.  The copies run on two copy streams, double-buffered: step i+1's inputs move
    to the device and step i-1's results to the host while step i computes, as a
    training loop would feed the layer."""
    from routing_grouped_gemm_route_b200 import lib
    T, d, E = w.T, w.d, w.E
    es = 4 if act == torch.float32 else 2
    E2E = max(3, args.e2e_steps)

    def z(*shape, dt=act):
        return torch.empty(*shape, dtype=dt, device=dev)

    def pinned(src, dt=act):
        h = torch.empty(*src.shape, dtype=dt, pin_memory=True)
        h.copy_(src.cpu())
        return h
    hx, hdy = pinned(x), pinned(dy)
    hl = None if w.router else pinned(logits, torch.float32)
    hy = [torch.empty(T, d, dtype=act, pin_memory=True) for _ in range(2)]
    hdx = [torch.empty(T, d, dtype=act, pin_memory=True) for _ in range(2)]
    layer = lib.Layer(desc, device=dev)
    x_in = [z(T, d) for _ in range(2)]
    dy_in = [z(T, d) for _ in range(2)]
    dl_in = [None if w.router else z(T, E, dt=torch.float32) for _ in range(2)]
    y_out = [y, z(T, d)]
    dx_out = [dx, z(T, d)]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_done = [ev(), ev()]        # inputs of buffer b on the device
    used = [ev(), ev()]           # step on buffer b finished reading its inputs / writing
    out_done = [ev(), ev()]       # results of buffer b on the host

    def copy_in(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(used[b])       # step i-2 no longer reads these buffers
            x_in[b].copy_(hx, non_blocking=True)
            if dl_in[b] is not None:
                dl_in[b].copy_(hl, non_blocking=True)
            dy_in[b].copy_(hdy, non_blocking=True)
            in_done[b].record(s_in)

    def compute(i):
        b = i % 2
        comp.wait_event(in_done[b])
        if i >= 2:
            comp.wait_event(out_done[b])       # step i-2's results have left y/dx[b]
        outs = dict(dx=dx_out[b], d_logits=d_logits, dW13=dW13, dW2=dW2, dWr=dWr)
        layer.fwd(x_in[b], W13, W2, logits=dl_in[b], Wr=Wr, y=y_out[b])
        layer.bwd(dy_in[b], W13, W2, x=x_in[b], Wr=Wr, out=outs)
        used[b].record(comp)

    def copy_out(i):
        b = i % 2
        with torch.cuda.stream(s_out):
            s_out.wait_event(used[b])
            hy[b].copy_(y_out[b], non_blocking=True)
            hdx[b].copy_(dx_out[b], non_blocking=True)
            out_done[b].record(s_out)

    def run(n):
        copy_in(0)
        for i in range(n):
            if i + 1 < n:
                copy_in(i + 1)
            compute(i)
            copy_out(i)

    run(2)                                     # warm-up
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)                            # before the first input copy
    run(E2E)
    comp.wait_stream(s_out)
    e1.record(comp)                            # after the last result copy
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = T * d * es * 2 + (0 if w.router else T * E * 4)
    d2h = T * d * es * 2
    e2e = {"value": world * T * E2E / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": E2E,
           "api": "moe_layer_fwd + moe_layer_bwd; pinned-host x, logits, dy in and y, dx out "
                  "every step on two copy streams, double-buffered against the compute"}
    if lib.moe_read_device_status(layer.ws) != 0:
        raise RuntimeError("device status set during the end-to-end run")
    return e2e


# ------------------------------------------------------------------------------ our arm
def main():
    args = parse()
    from routing_grouped_gemm_route_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS[args.workload]
    if args.router:
        w = w.replace(router=True)
    if args.tokens is not None:
        w = w.replace(T=args.tokens, name=w.name + f"[T={args.tokens}]")
    if args.experts is not None:
        w = w.replace(E=args.experts, name=w.name + f"[E={args.experts}]")
    if args.dtype is not None and args.dtype != w.dtype:
        w = w.replace(dtype=args.dtype, name=w.name + f"[{args.dtype}]")
    if args.shared_expert:
        w = w.replace(shared=True, name=w.name + "[shared expert]")
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, w, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    from routing_grouped_gemm_route_b200 import lib
    lib.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = make_inputs(w, device=dev, seed=w.seed + rank)
    # MXFP8: the backward of a training step reuses the weight codes its forward made
    # (the weights change only in the optimizer step after it)
    flags = (lib.MOE_FLAG_ROUTER if w.router else 0) | \
        (lib.MOE_FLAG_RECOMPUTE if args.recompute else 0) | \
        (lib.MOE_FLAG_SHARED_EXPERT if w.shared else 0) | \
        (lib.MOE_FLAG_MX_KEEP_WEIGHT_CODES if w.dtype == "mxfp8" else 0)
    desc = lib.make_desc(w.T, w.d, w.d_ff, w.E, w.k, w.dtype, flags)
    capacity = 0
    if args.capacity is not None:
        if args.capacity == "auto":
            # the largest count of this routing (read once on the host, before any timing;
            # the injected logits do not change between steps)
            probe = lib.make_desc(w.T, w.d, w.d_ff, w.E, w.k, w.dtype)
            lg = inp["logits"]
            if w.router:
                lg = torch.empty(w.T, w.E, dtype=torch.float32, device=dev)
                lib.moe_router_logits(probe, inp["x"], inp["Wr"], lg)
            pws = lib.alloc_workspace(probe)
            z32 = lambda *sh, dt=torch.int32: torch.empty(*sh, dtype=dt, device=dev)
            pc = z32(w.E)
            lib.moe_route(probe, lg, z32(w.T, w.k), z32(w.T, w.k, dt=torch.float32), pc,
                          z32(w.E + 1), z32(w.T, w.k), z32(w.T * w.k),
                          z32(w.T * w.k, dt=torch.float32), pws)
            capacity = int(pc.max().item())
            del pws
        else:
            capacity = int(args.capacity)
        desc.capacity = capacity
    act = lib.act_dtype(desc)
    T, d, f, E, k = w.T, w.d, w.d_ff, w.E, w.k
    R = lib.rows_of(desc)
    es = 4 if act == torch.float32 else 2
    ws = lib.alloc_workspace(desc)

    def z(*shape, dt=act):
        return torch.empty(*shape, dtype=dt, device=dev)
    x, W13, W2, dy = inp["x"], inp["W13"], inp["W2"], inp["dy"]
    Wr = inp["Wr"]
    logits = inp["logits"] if not w.router else z(T, E, dt=torch.float32)
    idx, gates = z(T, k, dt=torch.int32), z(T, k, dt=torch.float32)
    counts, offsets = z(E, dt=torch.int32), z(E + 1, dt=torch.int32)
    slot, row_token, row_gate = z(T, k, dt=torch.int32), z(R, dt=torch.int32), z(R, dt=torch.float32)
    x_perm, H13, a, y_perm, y = z(R, d), z(R, 2 * f), z(R, f), z(R, d), z(T, d)
    dy_perm, dH13, dx_perm, dx = z(R, d), z(R, 2 * f), z(R, d), z(T, d)
    d_logits = z(T, E, dt=torch.float32)
    nw = E + (1 if w.shared else 0)                 # weight slices (shared expert last)
    dW13, dW2 = z(nw, 2 * f, d), z(nw, d, f)
    dWr = z(d, E) if w.router else None

    stages = ["route", "dispatch", "gemm_fwd", "combine", "combine_bwd", "gemm_bwd",
              "dispatch_bwd"]
    if args.recompute:
        # the backward first recomputes the forward's activations (same buffers here)
        stages = stages[:4] + ["re_dispatch", "re_gemm_fwd"] + stages[4:]
    layer = None
    if w.shared:
        # the shared expert lives in the whole-layer calls: time those
        layer = lib.Layer(desc, device=dev)
        stages = ["layer_fwd", "layer_bwd"]
        layer_out = dict(dx=dx, d_logits=d_logits, dW13=dW13, dW2=dW2, dWr=dWr)
    if w.router:
        stages = ["router"] + stages + ["router_bwd"]
    mx = w.dtype == "mxfp8"
    launches = stage_launches(w, bool(flags & lib.MOE_FLAG_MX_KEEP_WEIGHT_CODES))

    def run_stage(name):
        if name == "router":
            lib.moe_router_logits(desc, x, Wr, logits)
        elif name == "route":
            lib.moe_route(desc, logits, idx, gates, counts, offsets, slot, row_token, row_gate, ws)
        elif name in ("dispatch", "re_dispatch"):
            lib.moe_dispatch(desc, x, slot, x_perm, ws)
        elif name in ("gemm_fwd", "re_gemm_fwd"):
            lib.moe_grouped_gemm_fwd(desc, x_perm, W13, W2, offsets, H13, a, y_perm, ws)
        elif name == "combine":
            lib.moe_combine(desc, y_perm, gates, slot, y, ws)
        elif name == "combine_bwd":
            lib.moe_combine_bwd(desc, dy, y_perm, gates, idx, slot, dy_perm, d_logits, ws)
        elif name == "gemm_bwd":
            lib.moe_grouped_gemm_bwd(desc, dy_perm, x_perm, H13, a, W13, W2, offsets, dH13,
                                     dx_perm, dW13, dW2, ws)
        elif name == "dispatch_bwd":
            lib.moe_dispatch_bwd(desc, dx_perm, slot, dx, ws)
        elif name == "router_bwd":
            lib.moe_router_bwd(desc, x, Wr, d_logits, dx, dWr, ws)
        elif name == "layer_fwd":
            layer.fwd(x, W13, W2, logits=None if w.router else logits, Wr=Wr, y=y)
        elif name == "layer_bwd":
            layer.bwd(dy, W13, W2, x=x, Wr=Wr, out=layer_out)

    K, W = args.steps, args.warmup
    for _ in range(W):
        for s in stages:
            run_stage(s)
    torch.cuda.synchronize()
    if lib.moe_read_device_status(layer.ws if layer else ws) != 0:
        raise RuntimeError("device status set during warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(K)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    nvml = NvmlSampler(local)
    nvml.start()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(K):
        e = ev[i]
        e[0].record()
        for j, s in enumerate(stages):
            run_stage(s)
            e[j + 1].record()
    stop.record()
    torch.cuda.synchronize()
    barrier(world)
    in_region = nvml.stop()
    clk = clocks.stop()
    if in_region.get("samples", 0) >= 3:
        # the in-region NVML record decides the clock; nvidia-smi gives the throttle reasons
        clk = dict(clk, smi_sm_mhz=clk.get("sm_mhz"), smi_samples=clk.get("samples"),
                   sm_mhz=in_region["sm_mhz"], sm_mhz_min=in_region["sm_mhz_min"],
                   samples=in_region["samples"], power_w_median=in_region["power_w_median"],
                   power_w_max=in_region["power_w_max"],
                   source="NVML every ~2 ms during the timed region (reasons: nvidia-smi)")
    ms_local = start.elapsed_time(stop)
    ms_total = max_over_ranks(ms_local, world)
    if lib.moe_read_device_status(layer.ws if layer else ws) != 0:
        raise RuntimeError("device status set during the timed region")
    if layer is not None:
        counts = layer.views()["counts"]
    # expert load of this routing (device statistics kernel, outside the timed region)
    st_buf = torch.zeros(64, dtype=torch.uint8, device=dev)
    lib.moe_load_stats(counts, st_buf)
    load = lib.decode_load_stats(st_buf)
    load = {"max_over_mean": round(load["max_over_mean"], 3), "cv": round(load["cv"], 4),
            "empty_experts": load["num_empty"], "max_rows": load["max_count"],
            "min_rows": load["min_count"]}

    stage_ms = {s: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)) / K
                for j, s in enumerate(stages)}
    value = whole_job_rate(world, T, K, ms_total)
    pk = peaks()

    # algorithmic work per stage
    # algorithmic work counts routed rows only (the padded layout's extra rows are waste)
    Ra = T * k
    gemm_flops = {"gemm_fwd": 6.0 * Ra * d * f, "gemm_bwd": 12.0 * Ra * d * f,
                  "re_gemm_fwd": 6.0 * Ra * d * f}
    hbm_bytes = {
        # logits in; idx, gates, slot, row_token, row_gate out; the histogram (per 64
        # tokens) and slot-CTA bases (per 256) written and read once each
        "route": T * E * 4 + T * k * 12 + Ra * 8 + 2 * 4 * E * ((T + 63) // 64 + (T + 255) // 256),
        "dispatch": T * d * es + T * k * 4 + Ra * d * es,
        "combine": Ra * d * es + T * k * 8 + T * d * es,
        "combine_bwd": T * d * es + 2 * Ra * d * es + T * k * 12 + T * E * 4,
        "dispatch_bwd": Ra * d * es + T * k * 4 + T * d * es,
    }
    hbm_bytes["re_dispatch"] = hbm_bytes["dispatch"]
    kind = "tf32" if act == torch.float32 else ("fp8" if mx else "bf16")
    tp = tensor_peak(pk, kind, clk, ms_local / 1e3)
    stage_rep = {}
    for s, ms in stage_ms.items():
        r = {"ms": round(ms, 4)}
        if s in gemm_flops:
            tf = gemm_flops[s] / (ms * 1e-3) / 1e12
            r.update({"TFLOP/s": round(tf, 1), "frac_of_peak": round(tf / tp["peak"], 3),
                      "frac_of_nominal": round(tf / tp["nominal"], 3)})
        elif s in hbm_bytes:
            gbs = hbm_bytes[s] / (ms * 1e-3) / 1e9
            r.update({"GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm"], 3),
                      "frac_of_nominal_hbm": round(gbs / NOMINAL_HBM_GBS, 3)})
        stage_rep[s] = r
    if args.flushed_reps > 0:
        # the HBM-bound stages again, one at a time, each after a 256 MB write that
        # evicts the 126 MB L2 (the main loop runs them back to back, where a stage can
        # find part of its input still in L2: combine reads the y_perm FC2 just wrote)
        flushed = flushed_stage_ms(run_stage, [s for s in stages if s in hbm_bytes], dev,
                                   args.flushed_reps)
        for s, ms in flushed.items():
            gbs = hbm_bytes[s] / (ms * 1e-3) / 1e9
            stage_rep[s].update({"l2_flushed_ms": round(ms, 4), "l2_flushed_GB/s": round(gbs, 1),
                                 "l2_flushed_frac_of_hbm": round(gbs / pk["hbm"], 3)})

    if layer is None:
        gemm_ms = stage_ms["gemm_fwd"] + stage_ms["gemm_bwd"]
        gemm_work = gemm_flops["gemm_fwd"] + gemm_flops["gemm_bwd"]
    else:
        # whole-layer timing: all GEMM flops (routed + shared expert) over the whole step,
        # a lower bound of the GEMM kernels' rate
        gemm_ms = stage_ms["layer_fwd"] + stage_ms["layer_bwd"]
        gemm_work = 18.0 * (Ra + T) * d * f
    gemm_tflops = gemm_work / (gemm_ms * 1e-3) / 1e12
    peak_tf = tp["peak"]
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "gemm_dram_traffic.json")
    if os.path.exists(tfile):
        import hashlib
        with open(tfile) as fh:
            tr = json.load(fh)
        src = open(os.path.join(ROOT, "routing_grouped_gemm_route_b200", "csrc",
                                "gemm_sm100.cu"), "rb").read()
        if tr.get("source_sha256") == hashlib.sha256(src).hexdigest() and \
                tr.get("workload") == w.name:
            traffic = tr.get("bytes_per_step")
    roofline = {"bound": "tensor", "achieved": round(gemm_tflops, 1), "peak": round(peak_tf, 1),
                "unit": "TFLOP/s", "frac": round(gemm_tflops / peak_tf, 4), "traffic": traffic,
                "frac_burst": round(gemm_tflops / tp["burst"], 4),
                "frac_sustained": round(gemm_tflops / tp["sustained"], 4),
                "frac_nominal": round(gemm_tflops / tp["nominal"], 4),
                "frac_is": tp["which"],
                "kernel": "grouped GEMM, 6 launches per step (FC1+SwiGLU, FC2, FC2 dgrad+SwiGLU "
                          "bwd, FC2 wgrad, FC1 dgrad, FC1 wgrad), algorithmic 18*T*k*d*d_ff flops",
                "peak_source": (f"{pk['source']} {tp['which']} {tp['kind']} (MEASURED_PEAKS.json; "
                                f"{tp['why']}); nominal {tp['nominal']:.0f} TFLOP/s"
                                if pk["source"] == "measured" else
                                f"fallback {tp['which']} {tp['kind']} ({tp['why']})")}
    if mx:
        roofline["kernel"] += "; the GEMM stages include the MXFP8 quantisers of their operands"
    if layer is not None:
        roofline["kernel"] = ("grouped GEMM incl. the shared expert (18*(T*k + T)*d*d_ff flops) "
                              "over the whole moe_layer_fwd + moe_layer_bwd time (lower bound)")

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if args.e2e_steps > 0:
        e2e = run_e2e(args, w, desc, act, dev, world, x, dy, logits, W13, W2, Wr, y, dx, d_logits,
                      dW13, dW2, dWr)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp_cpu = host_inputs(w, inp)
        cpu = cpu_baseline(w, inp_cpu, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_total / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": ("mxfp8-e4m3" if mx else "bf16") if act == torch.bfloat16 else "f32",
            "data": "synthetic (seeded N(0,1) activations/logits, N(0,0.02) weights)",
            "config": {"workload": workload_desc(w), "T": T, "d_model": d, "E": E, "top_k": k,
                       "d_ff": f, "router_on_device": w.router, "recompute": args.recompute, "shared_expert": w.shared,
                       "layout": (f"capacity-padded: every expert {capacity} rows, "
                                  f"{E * capacity} rows in all vs {T * k} routed"
                                  if capacity else "ragged (device-scheduled grouped GEMM)"),
                       "expert_load": load,
                       "parallelism": f"replicas x{world} (data parallel, no data-path collective)",
                       "l2": "no flush: each step's working set (~5 GB of weights, activations "
                             "and grads) exceeds the 126 MB L2"},
            "roofline": roofline,
            "gemm_frac_of_peak": round(gemm_tflops / peak_tf, 4),
            "stages": stage_rep,
            "gpu_launches": K * sum(launches[s] for s in stages),
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
