"""Benchmark of the COAT FP8-state AdamW step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one fused AdamW step (dequantise FP8 m/v, AdamW on the FP32 master,
bf16 copy, recompute k, requantise) over the whole parameter list, launched as a
single multi-tensor kernel.  Default workload: the Llama-2-7B-shaped parameter
list (291 tensors, 6,738,415,616 parameters, E4M3 m + E5M2 v, group 128), all
inputs resident in HBM (68 GB per step, far larger than the 126 MB L2, so no L2
flush is needed between steps).  Synthetic data from the seeded generator.

Multi-GPU (torchrun): every rank updates its own full parameter list (the
parameter groups are independent; there is no exchange step), so per-GPU work
is fixed ("weak" scaling); time = max over ranks of device time.

--impl reference times the CPU oracle (plain double-precision C) on every host
core, over a bounded sample of the workload's token embedding and first layer
per step.
"""
from __future__ import annotations

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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Gparams/s of FP8-state AdamW step; HBM GB/s as % of B200 roofline"
UNIT = "Gparams/s"
HBM_FALLBACK_GBS = 6650.0
KERNEL_SOURCES = ["fp8_optimizer_state_b200/csrc/adamw_fp8.cu",
                  "fp8_optimizer_state_b200/csrc/coat_device.cuh"]
# DRAM bytes (read + write) per parameter of the step kernel from an ncu
# capture on a 268,435,456-parameter tensor (profiles/), scaled to a launch by
# its parameter count; valid only for the kernel sources with this hash.
TRAFFIC = {"sources_sha256": "37c3d5b442fb280a", "bytes_per_param": 16.053}


def kernel_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def queue_ahead(steps):
    """Occupy the stream with a device-side delay while the host enqueues the
    timed launches, so that the GPU runs them back to back and host launch
    time (Python, ctypes) never falls between a launch's two events.  About
    50 ms plus 5 ms per step at 1.9 GHz, far more than enqueuing takes."""
    import torch
    torch.cuda._sleep(int(1e8 + 1e7 * steps))


QUEUE_NOTE = "timed launches queued behind a device-side delay: host launch time is not in the events"


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return None


def algorithmic_bytes(sizes, with_weight=True):
    """Per step: master read+write 8 B, grad 2 B, bf16 copy 2 B, m and v codes
    read+write 4 B per stored code (whole groups), 4 metadata floats read+write
    per group (32 B)."""
    tot = 0
    for n in sizes:
        ng = -(-n // 128)
        tot += 8 * n + 2 * n + (2 * n if with_weight else 0) + 4 * ng * 128 + 32 * ng
    return tot


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
def pci_bus_id(dev):
    """The device's PCI bus id as nvidia-smi prints it (for the clock sampler)."""
    import torch
    props = torch.cuda.get_device_properties(dev)
    return "%08x:%02x:%02x.0" % (int(getattr(props, "pci_domain_id", 0)),
                                 int(getattr(props, "pci_bus_id", 0)),
                                 int(getattr(props, "pci_device_id", 0)))


class ClockSampler:
    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = (bus_id or "").lower()
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            bus = parts[1].lower()
            if self.bus_id and not (bus.endswith(self.bus_id[-12:]) or self.bus_id.endswith(bus[-12:])):
                continue
            rows.append((ts, parts))
        inside = [p for ts, p in rows if t0 - 0.05 <= ts <= t1 + 0.05] or [p for _, p in rows]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[2]) for p in inside if num(p[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in inside:
            for name, val in zip(names, p[6:10]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(inside[0][3]), "reasons": sorted(reasons),
                "power_w_max": max((num(p[4]) or 0.0) for p in inside), "samples": len(inside)}


# ----------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline key)
# ----------------------------------------------------------------------------
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# The oracle is timed on a bounded sample of the Llama-2-7B list's token
# embedding and first layer (10 tensors; the step's cost per element does not
# depend on the tensor), extrapolated to the whole list.
SLICE_TENSORS = 10
SLICE_NAME = "token embedding + layer 0 of the Llama-2-7B list"
LLAMA2_7B_PARAMS = 6738415616


def oracle_slice_inputs(per_tensor, fmt_m, fmt_v, use_device):
    """Inputs of the first `per_tensor` elements (whole groups) of each tensor
    of the slice, concatenated: master, gradient bits and a stored state (codes,
    root scale, k) drawn by the seeded generator -- the same recipe as the
    parity tests' identical-input states.  On the device when one is in use
    (bit-identical and much faster than the NumPy generator), else NumPy on
    host threads."""
    import synth
    from synth.params import llama2_7b
    shapes = llama2_7b()[:SLICE_TENSORS]
    counts = [(min(n, per_tensor) if per_tensor > 0 else n) // 128 * 128 for _, n in shapes]

    def one(i):
        c = counts[i]
        ng = c // 128
        if use_device:
            import torch
            m = torch.empty(c, dtype=torch.float32, device="cuda")
            g = torch.empty(c, dtype=torch.int16, device="cuda")
            q = torch.empty(c, dtype=torch.uint8, device="cuda")
            synth.device_master(m, 0, i)
            synth.device_grad(g, 0, i, 1)
            master, grad = m.cpu().numpy(), g.cpu().numpy().view(np.uint16)
            synth.device_state_codes(q, 0, i, 1, fmt_m, True)
            mq = q.cpu().numpy()
            synth.device_state_codes(q, 0, i, 1, fmt_v, False)
            vq = q.cpu().numpy()
        else:
            master = synth.master(0, i, 0, c)
            grad = synth.grad_bits(0, i, 1, 0, c)
            mq = synth.state_codes(0, i, 1, 0, c, fmt_m, True)
            vq = synth.state_codes(0, i, 1, 0, c, fmt_v, False)
        km, sm, kv, sv = synth.state_groups(0, i, 1, 0, ng)
        return master, grad, mq, vq, sm, km, sv, kv

    if use_device:
        parts = [one(i) for i in range(len(shapes))]
    else:
        import concurrent.futures as cf
        with cf.ThreadPoolExecutor(min(len(shapes), host_cores())) as ex:
            parts = list(ex.map(one, range(len(shapes))))
    cat = [np.ascontiguousarray(np.concatenate([p[j] for p in parts])) for j in range(8)]
    return cat, counts


def time_oracle(cfg, per_tensor, steps, threads, use_device, inputs=None):
    """Per-step seconds of the oracle's step over the slice sample on `threads`
    host threads (group-aligned slices, one C call each; bit for bit the
    single-call result)."""
    import oracle as orc
    from synth.params import HYPER as H
    if inputs is None:
        inputs, _ = oracle_slice_inputs(per_tensor, cfg["fmt_m"], cfg["fmt_v"], use_device)
    master, grad, mq, vq, sm, km, sv, kv = (a.copy() for a in inputs)
    weight = np.zeros(master.size, np.uint16)
    times = []
    for t in range(1, steps + 1):
        t0 = time.perf_counter()
        orc.adamw_step_threads(master, weight, grad, mq, sm, km, vq, sv, kv, threads=threads,
                               lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"], eps=H["eps"],
                               wd=H["wd"], step=t, fmt_m=cfg["fmt_m"], fmt_v=cfg["fmt_v"])
        times.append(time.perf_counter() - t0)
    return times


def cpu_baseline(cfg, per_tensor, use_device):
    """The oracle on every host core over the slice (whole tensors when
    per_tensor is 0: one step; else the first per_tensor elements of each:
    median of three steps), next to one core on its first 2^21 elements, and
    the whole 7B list's step time extrapolated from the all-cores rate."""
    cores = host_cores()
    inputs, counts = oracle_slice_inputs(per_tensor, cfg["fmt_m"], cfg["fmt_v"], use_device)
    total = int(sum(counts))
    steps = 1 if per_tensor <= 0 else 3
    t_all = statistics.median(time_oracle(cfg, per_tensor, steps, cores, use_device, inputs))
    one = min(total, 1 << 21)
    t_one = time_oracle(cfg, per_tensor, 1, 1, use_device, [a[:one] if a.size == total else
                                                           a[:one // 128] for a in inputs])[0]
    rate = total / t_all
    what = ("the whole %d tensors of the %s" % (len(counts), SLICE_NAME) if per_tensor <= 0 else
            "first %d elements of each of the %d tensors of the %s" % (per_tensor, len(counts),
                                                                       SLICE_NAME))
    return {"value": round(rate / 1e9, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "%s (%d elements, stored states from the seeded generator), on %d host "
                      "threads, %s (%.2f s)" % (what, total, cores,
                                               "one step" if steps == 1 else
                                               "median of 3 steps, each", t_all),
            "one_core": {"value": round(one / t_one / 1e9, 6), "unit": UNIT, "cores": 1,
                         "sample": "first %d elements of the same sample, one step (%.2f s)"
                                   % (one, t_one)},
            "llama2_7b_step_s_extrapolated": round(LLAMA2_7B_PARAMS / rate, 1),
            "nproc": cores}


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x, ws, device):
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput_gparams(ws, n_params, steps, elapsed_ms):
    """Whole-job throughput: every rank steps its own n_params parameters
    (replicas, weak scaling), timed as the slowest rank."""
    return ws * n_params * steps / (elapsed_ms * 1e-3) / 1e9


def barrier(ws, device):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index] if device is not None and device.type == "cuda" else None)


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def make_workload(shapes, cfg, seed, coat):
    """Device-resident parameter set with warm-started states (each moment's FP32
    warm-start values quantised by the library's codec) and its multi-tensor plan."""
    import torch
    from synth.workload import DeviceParamSet
    ps = DeviceParamSet(shapes, seed=seed)
    ps.fill_master()
    ps.fill_grad(1)
    tmp = None
    for i in range(len(ps)):
        v = ps.views(i)
        if v["n"] == 0:
            continue
        tmp = ps.warm_values(i, "m", tmp)
        coat.coat_group_quantize(tmp.view(1, -1), 1, 128, True, cfg["fmt_m"], v["mq"].view(1, -1),
                                 v["ms"].view(1, -1), v["mk"].view(1, -1))
        tmp = ps.warm_values(i, "v", tmp)
        coat.coat_group_quantize(tmp.view(1, -1), 1, 128, True, cfg["fmt_v"], v["vq"].view(1, -1),
                                 v["vs"].view(1, -1), v["vk"].view(1, -1))
    del tmp
    descs = []
    for i in range(len(ps)):
        v = ps.views(i)
        descs.append(coat.make_desc(v["master"], v["weight"], v["grad"], v["mq"], v["ms"], v["mk"],
                                    v["vq"], v["vs"], v["vk"]))
    plan = coat.coat_multi_plan_create(descs, cfg["fmt_m"], cfg["fmt_v"])
    torch.cuda.synchronize()
    return ps, plan


def time_plan(plan, steps, warmup, H, coat, first_step=1):
    """Mean device time (ms) per step of `steps` steps after `warmup` untimed ones."""
    import torch
    for t in range(warmup):
        coat.coat_adamw_step_multi(plan, step=first_step + t, **H)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    queue_ahead(steps)
    a.record()
    for t in range(steps):
        coat.coat_adamw_step_multi(plan, step=first_step + warmup + t, **H)
    b.record()
    torch.cuda.synchronize()
    coat.coat_check_device_error()
    return a.elapsed_time(b) / steps


def run_ours(args, cfg, ws, rank, local):
    import torch
    import fp8_optimizer_state_b200 as coat
    from synth.params import HYPER as H

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    coat.lib()
    if args.exact_group_params:
        coat.coat_set_exact_group_params(True)

    ps, plan = make_workload(cfg["shapes"](), cfg, rank, coat)

    stream = torch.cuda.current_stream()
    step_no = [0]
    clip_buf = coat.new_grad_clip(dev) if args.clip is not None else None

    def one_step(mid=None):
        # with --clip: the gradient-norm pass, then the step on coef * g
        step_no[0] += 1
        if clip_buf is not None:
            plan.grad_norm(args.clip, clip_buf)
            if mid is not None:
                mid.record(stream)
            coat.coat_adamw_step_multi_clipped(plan, clip_buf, lr=H["lr"], beta1=H["beta1"],
                                               beta2=H["beta2"], eps=H["eps"], wd=H["wd"],
                                               step=step_no[0])
        else:
            coat.coat_adamw_step_multi(plan, lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"],
                                       eps=H["eps"], wd=H["wd"], step=step_no[0])

    nvtx = torch.cuda.nvtx
    nvtx.range_push("warm-up: %d steps" % args.warmup)
    for _ in range(args.warmup):
        one_step()
    nvtx.range_pop()
    torch.cuda.synchronize()
    coat.coat_check_device_error()

    sampler = ClockSampler(pci_bus_id(dev))
    sampler.start()
    time.sleep(0.3)
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
          for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(ws, dev)
    torch.cuda.synchronize()
    wall0 = time.time()
    nvtx.range_push("timed region: %d steps" % args.steps)
    t_start.record(stream)
    for i in range(args.steps):
        nvtx.range_push("step %d" % i)
        ev[i][0].record(stream)
        one_step(ev[i][2])
        ev[i][1].record(stream)
        nvtx.range_pop()
    t_end.record(stream)
    nvtx.range_pop()
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(ws, dev)
    time.sleep(0.2)
    sampler.stop()
    coat.coat_check_device_error()

    elapsed_ms = t_start.elapsed_time(t_end)
    if clip_buf is not None:
        # the step kernel alone: from the event after the norm pass
        launch_ms = [m.elapsed_time(b) for a, b, m in ev]
        norm_ms = max_over_ranks(statistics.mean([a.elapsed_time(m) for a, b, m in ev]), ws, dev)
    else:
        launch_ms = [a.elapsed_time(b) for a, b, m in ev]
    elapsed_ms = max_over_ranks(elapsed_ms, ws, dev)
    kernel_ms = max_over_ranks(statistics.mean(launch_ms), ws, dev)
    n_params = ps.total_elements
    n_tensors = len(ps)
    value = throughput_gparams(ws, n_params, args.steps, elapsed_ms)

    # roofline of the step kernel
    peaks = measured_peaks()
    peak = peaks["hbm_gbs"] if peaks and peaks.get("hbm_gbs") else HBM_FALLBACK_GBS
    alg = algorithmic_bytes(ps.sizes, with_weight=True)
    achieved = alg / (kernel_ms * 1e-3) / 1e9
    traffic = None
    if (TRAFFIC["sources_sha256"] == kernel_hash() and TRAFFIC["bytes_per_param"]
            and not args.exact_group_params):   # the capture is of the fast-mode kernel
        traffic = TRAFFIC["bytes_per_param"] * n_params
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_source": "measured" if peaks else "fallback",
                "algorithmic_bytes_per_launch": alg,
                "bytes_per_param": round(alg / n_params, 4), "kernel_ms": round(kernel_ms, 4),
                "frac_of_nominal_8TBs": round(achieved / 8000.0, 4)}
    clocks = sampler.summary(wall0, wall1)
    clip = None
    if clip_buf is not None:
        rec = coat.read_grad_clip(clip_buf)
        norm_bytes = 2 * n_params
        norm_gbs = norm_bytes / (norm_ms * 1e-3) / 1e9
        clip = {"max_norm": args.clip, "norm": float(rec.norm), "coef": float(rec.coef),
                "found_inf": int(rec.found_inf), "norm_kernel_ms": round(norm_ms, 4),
                "norm_algorithmic_bytes": norm_bytes, "norm_achieved_GBs": round(norm_gbs, 1),
                "norm_frac": round(norm_gbs / peak, 4),
                "how": "per step: gradient-norm pass (reads every bf16 gradient once) then the "
                       "step on coef * g; roofline above is the step kernel alone"}

    # end to end through the public API with host buffers: per step, H2D of the
    # bf16 gradients from pinned memory, the step (per tensor, overlapped with the
    # copies on separate streams), D2H of the bf16 weight copy
    e2e = None
    if not args.no_e2e and clip_buf is None:
        e2e = run_e2e(args, cfg, ps, ws, dev, H, coat)

    plan.destroy()
    n_total = ps.total_elements
    del ps
    torch.cuda.empty_cache()
    # many-tensor launch overhead: the same parameter count as one flat tensor
    vs_flat = None
    if n_tensors > 1 and args.compare_flat:
        fps, fplan = make_workload([("flat", n_total)], cfg, rank, coat)
        flat_ms = max_over_ranks(time_plan(fplan, args.steps, args.warmup, H, coat), ws, dev)
        fplan.destroy()
        del fps
        torch.cuda.empty_cache()
        flat_value = ws * n_total / (flat_ms * 1e-3) / 1e9
        vs_flat = {"flat_value": round(flat_value, 3), "unit": UNIT,
                   "flat_ms_per_step": round(flat_ms, 4), "ratio": round(value / flat_value, 4),
                   "how": "the same parameter count as one flat tensor, same formats and "
                          "hyperparameters, device events around the same number of steps"}
    extras = None
    if ws == 1 and args.extras and args.config == "llama2-7b" and clip_buf is None:
        extras = run_extras(args, coat, H, local)
    result = None
    if rank == 0:
        cpu = None
        if ws == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(cfg, args.cpu_sample, use_device=True)
        result = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": cfg["workload"], "params_per_gpu": n_params,
                       "tensors": n_tensors, "group": 128,
                       "fmt_m": FMT_NAMES[cfg["fmt_m"]],
                       "fmt_v": FMT_NAMES[cfg["fmt_v"]],
                       "hyper": H, "l2": "no flush: %.1f GB of inputs per step >> 126 MB L2"
                                         % (alg / 1e9),
                       "group_params": "exact" if args.exact_group_params else "fast",
                       "parallelism": "replicas%d (independent parameter groups, no collective)" % ws
                       if ws > 1 else "single GPU"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * (2 if clip_buf is not None else 1), "clocks": clocks,
        }
        if clip is not None:
            result["clip"] = clip
        if extras is not None:
            result["other_workloads"] = extras
        if vs_flat is not None:
            result["vs_flat_tensor"] = vs_flat
    if ws > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return result


def run_extras(args, coat, H, local):
    """Figures of the other workloads in the same run (one GPU), so that they are
    recorded next to the headline: the ragged 10,000-tensor list against one flat
    tensor of the same size (multi-tensor overhead), that flat tensor with exact
    group parameters, the Llama-2-13B list, the tiny one-tensor case (L2-resident)
    and the mixed-granularity codec workload.  Each list: device events around
    `steps` launches after 3 warm-up launches, inputs far larger than L2."""
    import torch
    from synth.params import CONFIGS
    peaks = measured_peaks()
    peak = peaks["hbm_gbs"] if peaks and peaks.get("hbm_gbs") else HBM_FALLBACK_GBS
    steps = max(3, min(args.steps, 10))
    out = {"how": "per workload: %d timed launches after 3 warm-up launches, CUDA events on the "
                  "launching stream; frac = algorithmic bytes / kernel time / peak (%s %.1f GB/s); "
                  "%s" % (steps, "measured" if peaks else "fallback", peak, QUEUE_NOTE)}

    def one_list(name, shapes):
        cfg = dict(CONFIGS[name]) if name in CONFIGS else None
        ps, plan = make_workload(shapes, cfg, 0, coat)
        ms = time_plan(plan, steps, 3, H, coat)
        n, sizes = ps.total_elements, list(ps.sizes)
        plan.destroy()
        del ps
        torch.cuda.empty_cache()
        alg = algorithmic_bytes(sizes, with_weight=True)
        gbs = alg / (ms * 1e-3) / 1e9
        return {"value": round(n / (ms * 1e-3) / 1e9, 3), "unit": UNIT, "ms_per_step": round(ms, 4),
                "params": n, "tensors": len(sizes), "achieved_GBs": round(gbs, 1),
                "frac": round(gbs / peak, 4)}, n

    from synth.params import ragged, llama2_13b
    r, n_r = one_list("ragged", ragged())
    flat_cfg = dict(CONFIGS["ragged"])
    fps, fplan = make_workload([("flat", n_r)], flat_cfg, 0, coat)
    fms = time_plan(fplan, steps, 3, H, coat)
    # the same flat tensor with exact group parameters (k and the root scales
    # recomputed in double from the codes)
    with coat.exact_group_params(True):
        ems = time_plan(fplan, steps, 3, H, coat)
    fplan.destroy()
    del fps
    torch.cuda.empty_cache()
    r["workload"] = CONFIGS["ragged"]["workload"]
    r["flat_value"] = round(n_r / (fms * 1e-3) / 1e9, 3)
    r["ratio_to_flat"] = round(r["value"] / r["flat_value"], 4)
    out["ragged"] = r
    egbs = algorithmic_bytes([n_r], with_weight=True) / (ems * 1e-3) / 1e9
    out["exact_group_params"] = {
        "value": round(n_r / (ems * 1e-3) / 1e9, 3), "unit": UNIT, "ms_per_step": round(ems, 4),
        "achieved_GBs": round(egbs, 1), "frac": round(egbs / peak, 4),
        "ratio_to_default": round(fms / ems, 4),
        "workload": "one flat tensor of %d params (E4M3 m + E5M2 v), exact group parameters "
                    "(coat_set_exact_group_params(1))" % n_r}
    b, _ = one_list("llama2-13b", llama2_13b())
    b["workload"] = CONFIGS["llama2-13b"]["workload"]
    out["llama2_13b"] = b
    from synth.params import tiny
    t, _ = one_list("tiny", tiny())
    t["workload"] = CONFIGS["tiny"]["workload"]
    t["l2"] = ("17 MB of inputs: L2-resident across launches, so not a roofline point "
               "(the fraction can exceed the HBM peak)")
    out["tiny"] = t
    cargs = argparse.Namespace(steps=steps, warmup=3, no_e2e=True, no_cpu_baseline=True,
                               e2e_steps=1)
    c = run_codec(cargs, 1, 0, local)
    out["act_codec"] = {"value": c["value"], "unit": c["unit"], "ms_per_step": c["ms_per_step"],
                        "workload": c["config"]["workload"],
                        "launches": [{k: x[k] for k in ("launch", "ms", "GB/s", "frac")}
                                     for x in c["launches"]]}
    coat.coat_check_device_error()
    return out


def run_e2e(args, cfg, ps, ws, dev, H, coat):
    import torch
    n_pad = ps.master.numel()
    host_grad = torch.empty(n_pad, dtype=torch.int16, pin_memory=True)
    host_w = torch.empty(n_pad, dtype=torch.int16, pin_memory=True)
    host_grad.copy_(ps.grad)
    torch.cuda.synchronize()
    comp = torch.cuda.current_stream()
    h2d = torch.cuda.Stream()
    d2h = torch.cuda.Stream()
    views = [ps.views(i) for i in range(len(ps))]
    offs = ps.off
    ev_in = [torch.cuda.Event() for _ in views]
    ev_done = [torch.cuda.Event() for _ in views]
    steps = max(1, min(args.steps, args.e2e_steps))
    base_step = 1000

    def step(t):
        for i, v in enumerate(views):
            a, n = int(offs[i]), v["n"]
            if n == 0:
                continue
            with torch.cuda.stream(h2d):
                v["grad"].copy_(host_grad[a:a + n], non_blocking=True)
                ev_in[i].record(h2d)
            comp.wait_event(ev_in[i])
            coat.coat_adamw_step(v["master"], v["weight"], v["grad"], v["mq"], v["ms"], v["mk"],
                                 v["vq"], v["vs"], v["vk"], lr=H["lr"], beta1=H["beta1"],
                                 beta2=H["beta2"], eps=H["eps"], wd=H["wd"], step=t,
                                 fmt_m=cfg["fmt_m"], fmt_v=cfg["fmt_v"], stream=comp)
            ev_done[i].record(comp)
            d2h.wait_event(ev_done[i])
            with torch.cuda.stream(d2h):
                host_w[a:a + n].copy_(v["weight"], non_blocking=True)
        d2h.synchronize()
        comp.synchronize()

    step(base_step)   # warm-up
    barrier(ws, dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for s in range(steps):
        step(base_step + 1 + s)
    torch.cuda.synchronize()
    el = time.perf_counter() - t0
    el = max_over_ranks(el, ws, dev)
    coat.coat_check_device_error()
    value = ws * ps.total_elements * steps / el / 1e9
    nbytes = 2 * ps.total_elements
    return {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": nbytes,
            "d2h_bytes_per_step": nbytes, "steps": steps,
            "how": "per step: H2D bf16 grads from pinned host memory, one coat_adamw_step per "
                   "tensor, D2H bf16 weight copy to pinned host memory; copies on two side "
                   "streams overlapped with the steps; host wall clock, max over ranks",
            "gpu_launches_per_step": sum(1 for v in views if v["n"] > 0)}


# ----------------------------------------------------------------------------
# the mixed-granularity codec workload: activations bf16 [8192 x 4096] with 1x128
# per-token groups and weights bf16 [4096 x 11008] with 128x128 blocks, to E4M3,
# expansion off and on, then the dequantisation round trip to bf16
# ----------------------------------------------------------------------------
FMT_NAMES = {0: "E4M3", 1: "E5M2", 2: "E5M2 (expanded to its own span)"}
CODEC_METRIC = "GB/s of the FP8 group codec (quantize + dequantize); HBM GB/s as % of B200 roofline"
CODEC_ACT = (8192, 4096)
CODEC_COPIES = 3
CODEC_W = (4096, 11008)


def codec_bytes(rows, cols, gr, gc):
    """Algorithmic bytes of one quantize (bf16 in, codes + scale + k out) or one
    dequantize (codes + scale + k in, bf16 out): 3 B per element + 8 B per group."""
    groups = -(-rows // gr) * -(-cols // gc)
    return 3 * rows * cols + 8 * groups


def run_codec(args, ws, rank, local):
    import torch
    import fp8_optimizer_state_b200 as coat
    import synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    coat.lib()
    E4M3 = 0
    shapes = {"act": (CODEC_ACT, 1, 128), "w": (CODEC_W, 128, 128)}
    # CODEC_COPIES copies of every buffer; launch n uses copy n % CODEC_COPIES, so
    # each launch touches data last used CODEC_COPIES launches earlier, with more
    # than the 126 MB L2 moved in between
    bufs = {}
    for name, ((r, c), gr, gc) in shapes.items():
        bufs[name] = []
        for cp in range(CODEC_COPIES):
            x = torch.empty(r, c, dtype=torch.bfloat16, device=dev)
            (synth.device_activations if name == "act" else synth.device_weight)(
                x.view(torch.int16).view(-1), rank, cp)
            nbr, nbc = -(-r // gr), -(-c // gc)
            bufs[name].append(dict(x=x, q=torch.empty(r, c, dtype=torch.uint8, device=dev),
                                   s=torch.empty(nbr, nbc, dtype=torch.float32, device=dev),
                                   k=torch.empty(nbr, nbc, dtype=torch.float32, device=dev),
                                   out=torch.empty(r, c, dtype=torch.bfloat16, device=dev),
                                   gr=gr, gc=gc))

    # the launches of one step, in order: (label, bytes, callable(copy))
    def launches():
        out = []
        for expand in (False, True):
            for name in ("act", "w"):
                b0 = bufs[name][0]
                out.append(("quantize %s %dx%d expand=%s" % (name, b0["gr"], b0["gc"], expand),
                            codec_bytes(*b0["x"].shape, b0["gr"], b0["gc"]),
                            (lambda cp, name=name, e=expand: coat.coat_group_quantize(
                                bufs[name][cp]["x"], bufs[name][cp]["gr"], bufs[name][cp]["gc"],
                                e, E4M3, bufs[name][cp]["q"], bufs[name][cp]["s"],
                                bufs[name][cp]["k"]))))
        for name in ("act", "w"):
            b0 = bufs[name][0]
            out.append(("dequantize %s %dx%d" % (name, b0["gr"], b0["gc"]),
                        codec_bytes(*b0["x"].shape, b0["gr"], b0["gc"]),
                        (lambda cp, name=name: coat.coat_group_dequantize(
                            bufs[name][cp]["q"], bufs[name][cp]["s"], bufs[name][cp]["k"],
                            bufs[name][cp]["gr"], bufs[name][cp]["gc"], E4M3,
                            bufs[name][cp]["out"]))))
        return out

    L = launches()
    stream = torch.cuda.current_stream()
    n_launch = 0
    for cp in range(CODEC_COPIES):   # every copy gets valid codes before any dequantize
        for name in ("act", "w"):
            b = bufs[name][cp]
            coat.coat_group_quantize(b["x"], b["gr"], b["gc"], True, E4M3, b["q"], b["s"], b["k"])
    for _ in range(args.warmup):
        for _, _, f in L:
            f(n_launch % CODEC_COPIES)
            n_launch += 1
    torch.cuda.synchronize()
    coat.coat_check_device_error()
    sampler = ClockSampler(pci_bus_id(dev))
    sampler.start()
    time.sleep(0.3)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in L] for _ in range(args.steps)]
    barrier(ws, dev)
    torch.cuda.synchronize()
    wall0 = time.time()
    queue_ahead(args.steps)
    for i in range(args.steps):
        for j, (_, _, f) in enumerate(L):
            ev[i][j][0].record(stream)
            f(n_launch % CODEC_COPIES)
            ev[i][j][1].record(stream)
            n_launch += 1
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(ws, dev)
    time.sleep(0.2)
    sampler.stop()
    coat.coat_check_device_error()
    per = [statistics.mean(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(args.steps))
           for j in range(len(L))]
    per = [max_over_ranks(x, ws, dev) for x in per]
    step_ms = sum(per)
    step_bytes = sum(b for _, b, _ in L)
    value = ws * step_bytes / (step_ms * 1e-3) / 1e9
    peaks = measured_peaks()
    peak = peaks["hbm_gbs"] if peaks and peaks.get("hbm_gbs") else HBM_FALLBACK_GBS
    kern = [{"launch": lab, "ms": round(t, 4), "algorithmic_bytes": b,
             "GB/s": round(b / (t * 1e-3) / 1e9, 1), "frac": round(b / (t * 1e-3) / 1e9 / peak, 4)}
            for (lab, b, _), t in zip(L, per)]
    top = max(range(len(L)), key=lambda j: per[j])
    roofline = {"bound": "hbm", "achieved": kern[top]["GB/s"], "peak": peak, "unit": "GB/s",
                "frac": kern[top]["frac"], "traffic": None, "kernel": kern[top]["launch"],
                "peak_source": "measured" if peaks else "fallback"}
    clocks = sampler.summary(wall0, wall1)

    e2e = None
    if not args.no_e2e:
        # public API with host buffers: H2D of the bf16 activations from pinned
        # memory, quantize (1x128, expansion on), D2H of codes, scales and k
        b = bufs["act"][0]
        hx = torch.empty(b["x"].shape, dtype=torch.bfloat16, pin_memory=True)
        hq = torch.empty(b["q"].shape, dtype=torch.uint8, pin_memory=True)
        hs = torch.empty(b["s"].shape, dtype=torch.float32, pin_memory=True)
        hk = torch.empty(b["k"].shape, dtype=torch.float32, pin_memory=True)
        hx.copy_(b["x"])
        torch.cuda.synchronize()
        steps = max(1, min(args.steps, args.e2e_steps))
        barrier(ws, dev)
        t0 = time.perf_counter()
        for _ in range(steps):
            b["x"].copy_(hx, non_blocking=True)
            coat.coat_group_quantize(b["x"], 1, 128, True, E4M3, b["q"], b["s"], b["k"])
            hq.copy_(b["q"], non_blocking=True)
            hs.copy_(b["s"], non_blocking=True)
            hk.copy_(b["k"], non_blocking=True)
        torch.cuda.synchronize()
        el = max_over_ranks(time.perf_counter() - t0, ws, dev)
        nb = codec_bytes(*b["x"].shape, 1, 128)
        e2e = {"value": round(ws * nb * steps / el / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": hx.numel() * 2,
               "d2h_bytes_per_step": hq.numel() + 4 * (hs.numel() + hk.numel()), "steps": steps,
               "how": "activations only: H2D bf16 from pinned memory, coat_group_quantize 1x128 "
                      "with expansion, D2H codes + scale + k; host wall clock"}
    result = None
    if rank == 0:
        cpu = None
        if ws == 1 and not args.no_cpu_baseline:
            import oracle as orc
            rows = 4096
            x = synth.bf16_bits_to_f32(synth.activations_bits(rank, 0, 0, rows * CODEC_ACT[1]))
            x = x.reshape(rows, CODEC_ACT[1]).astype(np.float64)
            t0 = time.perf_counter()
            orc.group_quantize(x, 1, 128, True, E4M3)
            el = time.perf_counter() - t0
            cpu = {"value": round(codec_bytes(rows, CODEC_ACT[1], 1, 128) / el / 1e9, 6),
                   "unit": "GB/s", "cores": 1, "kind": "oracle",
                   "sample": "first %d token rows of the activations, 1x128 groups with "
                             "expansion, one host thread (%.2f s)" % (rows, el)}
        result = {
            "metric": CODEC_METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "mixed-granularity codec: activations bf16 8192x4096 (N(0,1), "
                                   "0.1% x100 outliers) in 1x128 groups and weights bf16 "
                                   "4096x11008 in 128x128 blocks, to E4M3, expansion off and on, "
                                   "dequantize round trip to bf16",
                       "launch_queue": QUEUE_NOTE,
                       "l2": "inputs larger than L2: launch n uses copy n %% %d of its buffers "
                             "(%d copies of 238 MB)" % (CODEC_COPIES, CODEC_COPIES),
                       "parallelism": "single GPU" if ws == 1 else "replicas%d" % ws},
            "launches": kern, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": len(L) * args.steps, "clocks": clocks}
    if ws > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return result


SWIGLU_METRIC = ("GB/s of the FP8 SwiGLU layer (forward + backward, FP8 1x128 in/out); "
                 "HBM GB/s as % of B200 roofline")
SWIGLU_SHAPE = (8192, 11008)   # tokens x Llama-2-7B MLP width


def swiglu_bytes(rows, cols):
    """Algorithmic bytes: forward = two codes in, one out (3 B per element) + 24 B
    of scale / k per group; backward = dh in, two codes in, two bf16 out
    (8 B per element) + 16 B per group."""
    groups = rows * -(-cols // 128)
    return 3 * rows * cols + 24 * groups, 8 * rows * cols + 16 * groups


def run_swiglu(args, ws, rank, local):
    import torch
    import fp8_optimizer_state_b200 as coat
    import synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    coat.lib()
    E4M3 = 0
    T, F = SWIGLU_SHAPE
    ng = F // 128
    # the fused up/gate projection output [T, 2F] as bf16 activations, quantised
    # to E4M3 1x128 (no expansion) by the library's codec: gate = [:, :F], up = [:, F:]
    x = torch.empty(T, 2 * F, dtype=torch.bfloat16, device=dev)
    synth.device_activations(x.view(torch.int16).view(-1), rank, 0)
    xq = torch.empty(T, 2 * F, dtype=torch.uint8, device=dev)
    xs = torch.empty(T, 2 * ng, dtype=torch.float32, device=dev)
    xk = torch.empty(T, 2 * ng, dtype=torch.float32, device=dev)
    coat.coat_group_quantize(x, 1, 128, False, E4M3, xq, xs, xk)
    del x
    gate = (xq[:, :F], xs[:, :ng], xk[:, :ng])
    up = (xq[:, F:], xs[:, ng:], xk[:, ng:])
    out = (torch.empty(T, F, dtype=torch.uint8, device=dev),
           torch.empty(T, ng, dtype=torch.float32, device=dev),
           torch.empty(T, ng, dtype=torch.float32, device=dev))
    dh = torch.empty(T, F, dtype=torch.int16, device=dev)
    synth.device_grad(dh.view(-1), rank, 9, 1)
    grads = torch.empty(T, 2 * F, dtype=torch.int16, device=dev)
    fwd = lambda: coat.coat_swiglu_fp8_forward(gate, up, E4M3, False, out)
    bwd = lambda: coat.coat_swiglu_fp8_backward(dh, gate, up, E4M3, grads[:, :F], grads[:, F:])
    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(pci_bus_id(dev))
    sampler.start()
    time.sleep(0.3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(ws, dev)
    torch.cuda.synchronize()
    wall0 = time.time()
    queue_ahead(args.steps)
    for i in range(args.steps):
        ev[i][0].record(stream)
        fwd()
        ev[i][1].record(stream)
        bwd()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(ws, dev)
    time.sleep(0.2)
    sampler.stop()
    f_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in ev), ws, dev)
    b_ms = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in ev), ws, dev)
    fb, bb = swiglu_bytes(T, F)
    step_ms = f_ms + b_ms
    value = ws * (fb + bb) / (step_ms * 1e-3) / 1e9
    peaks = measured_peaks()
    peak = peaks["hbm_gbs"] if peaks and peaks.get("hbm_gbs") else HBM_FALLBACK_GBS
    kern = [{"launch": lab, "ms": round(t, 4), "algorithmic_bytes": b,
             "GB/s": round(b / (t * 1e-3) / 1e9, 1), "frac": round(b / (t * 1e-3) / 1e9 / peak, 4)}
            for lab, t, b in (("forward", f_ms, fb), ("backward", b_ms, bb))]
    top = 0 if f_ms >= b_ms else 1
    roofline = {"bound": "hbm", "achieved": kern[top]["GB/s"], "peak": peak, "unit": "GB/s",
                "frac": kern[top]["frac"], "traffic": None, "kernel": kern[top]["launch"],
                "peak_source": "measured" if peaks else "fallback"}
    clocks = sampler.summary(wall0, wall1)

    e2e = None
    if not args.no_e2e:
        # public API with host buffers: H2D of the FP8 gate/up (codes, scale, k)
        # and of dh from pinned memory, forward + backward, D2H of the FP8
        # output and of both bf16 input gradients
        hin = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (xq, xs, xk, dh)]
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (*out, grads)]
        for h, t in zip(hin, (xq, xs, xk, dh)):
            h.copy_(t)
        torch.cuda.synchronize()
        steps = max(1, min(args.steps, args.e2e_steps))
        barrier(ws, dev)
        t0 = time.perf_counter()
        for _ in range(steps):
            for h, t in zip(hin, (xq, xs, xk, dh)):
                t.copy_(h, non_blocking=True)
            fwd()
            bwd()
            for h, t in zip(hout, (*out, grads)):
                h.copy_(t, non_blocking=True)
        torch.cuda.synchronize()
        el = max_over_ranks(time.perf_counter() - t0, ws, dev)
        e2e = {"value": round(ws * (fb + bb) * steps / el / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": sum(h.numel() * h.element_size() for h in hin),
               "d2h_bytes_per_step": sum(h.numel() * h.element_size() for h in hout),
               "steps": steps,
               "how": "H2D of the FP8 inputs and dh from pinned memory, forward + backward, D2H "
                      "of the FP8 output and both bf16 gradients; host wall clock"}
    coat.coat_check_device_error()
    result = None
    if rank == 0:
        cpu = None
        if ws == 1 and not args.no_cpu_baseline:
            import oracle as orc
            rows = 16
            hq, hs, hk = xq[:rows].cpu().numpy(), xs[:rows].cpu().numpy(), xk[:rows].cpu().numpy()
            g_ = (hq[:, :F].copy(), hs[:, :ng].copy(), hk[:, :ng].copy())
            u_ = (hq[:, F:].copy(), hs[:, ng:].copy(), hk[:, ng:].copy())
            d_ = dh[:rows].cpu().numpy().view(np.uint16)
            t0 = time.perf_counter()
            orc.swiglu_fp8_forward(g_, u_, E4M3, False)
            orc.swiglu_fp8_backward(d_, g_, u_, E4M3)
            el = time.perf_counter() - t0
            sb = sum(swiglu_bytes(rows, F))
            cpu = {"value": round(sb / el / 1e9, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
                   "sample": "first %d token rows, forward + backward, one host thread (%.2f s)"
                             % (rows, el)}
        result = {
            "metric": SWIGLU_METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "FP8 SwiGLU layer, %d tokens x %d (Llama-2-7B MLP width): gate "
                                   "and up as the halves of one E4M3 1x128 [T, 2F] tensor "
                                   "(N(0,1) activations with 0.1%% x100 outliers), E4M3 1x128 "
                                   "output without expansion, bf16 gradients" % (T, F),
                       "launch_queue": QUEUE_NOTE,
                       "l2": "no flush: %.0f MB forward + %.0f MB backward per step >> 126 MB L2"
                             % (fb / 1e6, bb / 1e6),
                       "parallelism": "single GPU" if ws == 1 else "replicas%d" % ws},
            "launches": kern, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": 2 * args.steps, "clocks": clocks}
    if ws > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return result


RMSNORM_METRIC = ("GB/s of the FP8 RMSNorm layer (forward + backward, FP8 1x128 in/out); "
                  "HBM GB/s as % of B200 roofline")
RMSNORM_SHAPE = (8192, 4096)   # tokens x Llama-2-7B hidden size
RMSNORM_EPS = 1e-6


def rmsnorm_bytes(rows, d):
    """Algorithmic bytes: forward = codes in and out (2 B per element) + 16 B of
    scale / k per group + the bf16 weight; backward = dy in, codes in, dx out
    (5 B per element) + 8 B per group + the weight and the FP32 dw."""
    groups = rows * -(-d // 128)
    return 2 * rows * d + 16 * groups + 2 * d, 5 * rows * d + 8 * groups + 6 * d


def run_rmsnorm(args, ws, rank, local):
    import torch
    import fp8_optimizer_state_b200 as coat
    import synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    coat.lib()
    E4M3 = 0
    T, d = RMSNORM_SHAPE
    ng = d // 128
    w = torch.empty(d, dtype=torch.bfloat16, device=dev)
    synth.device_weight(w.view(torch.int16), rank, 1)
    w = (w.float() * 5.0 + 1.0).to(torch.bfloat16)      # a norm weight near 1
    dw = torch.empty(d, dtype=torch.float32, device=dev)
    wsp = torch.empty(coat.coat_rmsnorm_fp8_workspace_size(d), dtype=torch.uint8, device=dev)
    # CODEC_COPIES copies of the per-token tensors; step s runs the forward on
    # copy s and the backward on copy s + 1, so that neither finds its input in L2
    cps = []
    for cp in range(CODEC_COPIES):
        x = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
        synth.device_activations(x.view(torch.int16).view(-1), rank, cp)
        xa = (torch.empty(T, d, dtype=torch.uint8, device=dev),
              torch.empty(T, ng, dtype=torch.float32, device=dev),
              torch.empty(T, ng, dtype=torch.float32, device=dev))
        coat.coat_group_quantize(x, 1, 128, False, E4M3, *xa)
        del x
        dy = torch.empty(T, d, dtype=torch.int16, device=dev)
        synth.device_grad(dy.view(-1), rank, 9 + cp, 1)
        cps.append(dict(xa=xa, dy=dy, dx=torch.empty(T, d, dtype=torch.int16, device=dev),
                        out=(torch.empty(T, d, dtype=torch.uint8, device=dev),
                             torch.empty(T, ng, dtype=torch.float32, device=dev),
                             torch.empty(T, ng, dtype=torch.float32, device=dev))))
    xa, dy, dx, out = cps[0]["xa"], cps[0]["dy"], cps[0]["dx"], cps[0]["out"]
    fwd = lambda c=cps[0]: coat.coat_rmsnorm_fp8_forward(c["xa"], w, RMSNORM_EPS, E4M3, False,
                                                         c["out"])
    bwd = lambda c=cps[0]: coat.coat_rmsnorm_fp8_backward(c["dy"], c["xa"], w, RMSNORM_EPS,
                                                          E4M3, c["dx"], dw, wsp)
    nc = len(cps)
    for i in range(args.warmup):
        fwd(cps[i % nc])
        bwd(cps[(i + 1) % nc])
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(pci_bus_id(dev))
    sampler.start()
    time.sleep(0.3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(ws, dev)
    torch.cuda.synchronize()
    wall0 = time.time()
    queue_ahead(args.steps)
    for i in range(args.steps):
        ev[i][0].record(stream)
        fwd(cps[i % nc])
        ev[i][1].record(stream)
        bwd(cps[(i + 1) % nc])
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(ws, dev)
    time.sleep(0.2)
    sampler.stop()
    f_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in ev), ws, dev)
    b_ms = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in ev), ws, dev)
    fb, bb = rmsnorm_bytes(T, d)
    step_ms = f_ms + b_ms
    value = ws * (fb + bb) / (step_ms * 1e-3) / 1e9
    peaks = measured_peaks()
    peak = peaks["hbm_gbs"] if peaks and peaks.get("hbm_gbs") else HBM_FALLBACK_GBS
    kern = [{"launch": lab, "ms": round(t, 4), "algorithmic_bytes": b,
             "GB/s": round(b / (t * 1e-3) / 1e9, 1), "frac": round(b / (t * 1e-3) / 1e9 / peak, 4)}
            for lab, t, b in (("forward", f_ms, fb), ("backward (+ dw reduction)", b_ms, bb))]
    top = 0 if f_ms >= b_ms else 1
    roofline = {"bound": "hbm", "achieved": kern[top]["GB/s"], "peak": peak, "unit": "GB/s",
                "frac": kern[top]["frac"], "traffic": None, "kernel": kern[top]["launch"],
                "peak_source": "measured" if peaks else "fallback"}
    clocks = sampler.summary(wall0, wall1)

    e2e = None
    if not args.no_e2e:
        # H2D of the FP8 x (codes, scale, k) and dy from pinned memory, forward +
        # backward, D2H of the FP8 output, dx and dw
        ins = (*xa, dy)
        outs = (*out, dx, dw)
        hin = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ins]
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
        for h, t in zip(hin, ins):
            h.copy_(t)
        torch.cuda.synchronize()
        steps = max(1, min(args.steps, args.e2e_steps))
        barrier(ws, dev)
        t0 = time.perf_counter()
        for _ in range(steps):
            for h, t in zip(hin, ins):
                t.copy_(h, non_blocking=True)
            fwd()
            bwd()
            for h, t in zip(hout, outs):
                h.copy_(t, non_blocking=True)
        torch.cuda.synchronize()
        el = max_over_ranks(time.perf_counter() - t0, ws, dev)
        e2e = {"value": round(ws * (fb + bb) * steps / el / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": sum(h.numel() * h.element_size() for h in hin),
               "d2h_bytes_per_step": sum(h.numel() * h.element_size() for h in hout),
               "steps": steps,
               "how": "H2D of the FP8 x and dy from pinned memory, forward + backward, D2H of "
                      "the FP8 output, dx and dw; host wall clock"}
    coat.coat_check_device_error()
    result = None
    if rank == 0:
        cpu = None
        if ws == 1 and not args.no_cpu_baseline:
            import oracle as orc
            rows = 32
            h = tuple(t[:rows].cpu().numpy() for t in xa)
            wb = w.view(torch.int16).cpu().numpy().view(np.uint16)
            dyb = dy[:rows].cpu().numpy().view(np.uint16)
            t0 = time.perf_counter()
            orc.rmsnorm_fp8_forward(h, wb, RMSNORM_EPS, E4M3, False)
            orc.rmsnorm_fp8_backward(dyb, h, wb, RMSNORM_EPS, E4M3)
            el = time.perf_counter() - t0
            sb = sum(rmsnorm_bytes(rows, d))
            cpu = {"value": round(sb / el / 1e9, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
                   "sample": "first %d token rows, forward + backward, one host thread (%.2f s)"
                             % (rows, el)}
        result = {
            "metric": RMSNORM_METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "FP8 RMSNorm layer, %d tokens x %d (Llama-2-7B hidden size): "
                                   "x E4M3 1x128 (N(0,1) activations with 0.1%% x100 outliers), "
                                   "bf16 weight near 1, E4M3 1x128 output without expansion, "
                                   "bf16 dy / dx, FP32 dw" % (T, d),
                       "launch_queue": QUEUE_NOTE,
                       "l2": "inputs not in L2: %d copies of the per-token tensors, the forward "
                             "of step s on copy s, the backward on copy s+1 (%.0f MB forward + "
                             "%.0f MB backward per step)" % (CODEC_COPIES, fb / 1e6, bb / 1e6),
                       "parallelism": "single GPU" if ws == 1 else "replicas%d" % ws},
            "launches": kern, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": 3 * args.steps, "clocks": clocks}
    if ws > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return result


ZERO1_METRIC = ("Gparams/s of the ZeRO-1 sharded FP8-state AdamW step (reduce-scatter + step + "
                "all-gather); HBM GB/s as % of B200 roofline")


def run_zero1(args, cfg, ws, rank, local):
    """ZeRO-1 over the Llama-2-7B list on N ranks: per step an NCCL reduce-scatter
    (sum) of the flat bf16 gradients, the FP8 step on the rank's 1/N of the
    groups, an NCCL all-gather of the bf16 weights.  The list is fixed, so the
    per-rank work shrinks with N ("strong" scaling).  Device events around each
    phase on the launching stream; every figure is the max over ranks.  The
    gradient buffer is not refilled between steps (the reduce-scatter sums in
    place, so the shard's values grow by about N g per step, which changes no
    timing)."""
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    import fp8_optimizer_state_b200 as coat
    import synth
    from fp8_optimizer_state_b200.zero1 import Zero1AdamW
    from synth.params import HYPER as H

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws == 1 and "MASTER_PORT" not in os.environ:
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(sk.getsockname()[1]))
    dist.init_process_group("nccl", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=120), device_id=dev)
    coat.lib()
    shapes = cfg["shapes"]()
    sizes = [n for _, n in shapes]
    z = Zero1AdamW(sizes, device=dev, fmt_m=cfg["fmt_m"], fmt_v=cfg["fmt_v"])
    for i, n in enumerate(sizes):
        synth.device_grad(z.grad(i), rank, i, 1)
    tmp = None
    for piece in z.pieces:
        t, b, n, _ = piece
        v = z.piece_views(piece)
        synth.device_master(v["master"], 0, t, start=b)
        for which, q, sc, kk, fmt in (("m", "m_q", "m_scale", "m_k", cfg["fmt_m"]),
                                      ("v", "v_q", "v_scale", "v_k", cfg["fmt_v"])):
            if tmp is None or tmp.numel() < n:
                tmp = torch.empty(n, dtype=torch.float32, device=dev)
            (synth.device_m_warm if which == "m" else synth.device_v_warm)(tmp[:n], 0, t, start=b)
            coat.coat_group_quantize(tmp[:n].view(1, n), 1, 128, True, fmt, v[q].view(1, -1),
                                     v[sc].view(1, -1), v[kk].view(1, -1))
    del tmp
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    hp = dict(lr=H["lr"], beta1=H["beta1"], beta2=H["beta2"], eps=H["eps"], wd=H["wd"])
    step_no = [0]

    def one_step(ev=None):
        step_no[0] += 1
        if ev is not None:
            ev[0].record(stream)
        z.reduce_scatter_grads()
        if ev is not None:
            ev[1].record(stream)
        z.local_step(step=step_no[0], **hp)
        if ev is not None:
            ev[2].record(stream)
        z.all_gather_weights()
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    coat.coat_check_device_error()
    sampler = ClockSampler(pci_bus_id(dev))
    sampler.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    wall0 = time.time()
    t0.record(stream)
    for i in range(args.steps):
        one_step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    dist.barrier(device_ids=[local])
    time.sleep(0.2)
    sampler.stop()
    coat.coat_check_device_error()
    elapsed = max_over_ranks(t0.elapsed_time(t1), ws, dev)
    phase = [max_over_ranks(statistics.mean(e[k].elapsed_time(e[k + 1]) for e in evs), ws, dev)
             for k in range(3)]
    n_params = sum(sizes)
    shard_sizes = [n for _, _, n, _ in z.pieces]
    alg = algorithmic_bytes(shard_sizes, with_weight=True)
    alg_max = max_over_ranks(float(alg), ws, dev)
    peaks = measured_peaks()
    peak = peaks["hbm_gbs"] if peaks and peaks.get("hbm_gbs") else HBM_FALLBACK_GBS
    step_gbs = alg_max / (phase[1] * 1e-3) / 1e9 if phase[1] > 0 else 0.0
    mem = sum(x.numel() * x.element_size() for x in
              (z.flat_grad, z.flat_weight, z.master, z.m_q, z.v_q, z.m_scale, z.m_k, z.v_scale, z.v_k))
    clocks = sampler.summary(wall0, wall1)
    z.close()
    result = None
    if rank == 0:
        result = {
            "metric": ZERO1_METRIC, "value": round(n_params * args.steps / (elapsed * 1e-3) / 1e9, 3),
            "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(elapsed / args.steps, 4), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": cfg["workload"] + ", ZeRO-1 over %d ranks" % ws,
                       "params_total": n_params, "shard_elems": z.shard_elems,
                       "parallelism": "zero1-dp%d (NCCL reduce-scatter + all-gather)" % ws,
                       "l2": "no flush: every array is far larger than L2"},
            "phases_ms": {"reduce_scatter": round(phase[0], 4), "step": round(phase[1], 4),
                          "all_gather": round(phase[2], 4)},
            "roofline": {"bound": "hbm", "achieved": round(step_gbs, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(step_gbs / peak, 4), "traffic": None,
                         "kernel": "the step on the rank's shard",
                         "peak_source": "measured" if peaks else "fallback"},
            "bytes_per_rank": mem, "gpu_launches": args.steps, "clocks": clocks,
            "cpu_baseline": None, "e2e": None}
    dist.barrier(device_ids=[local])
    dist.destroy_process_group()
    return result


def run_reference(args, cfg, ws, rank):
    """The CPU oracle, every host core, on the bounded slice sample per step."""
    if rank != 0:
        return None
    cores = host_cores()
    inputs, counts = oracle_slice_inputs(args.ref_sample, cfg["fmt_m"], cfg["fmt_v"], False)
    total = int(sum(counts))
    times = time_oracle(cfg, args.ref_sample, args.warmup + args.steps, cores, False, inputs)
    timed = times[args.warmup:]
    el = sum(timed)
    value = total * len(timed) / el / 1e9
    sample = ("first %d elements of each of the %d tensors of the %s per step (%d elements; "
              "stored states from the seeded generator), oracle adamw_step on %d host threads "
              "(group-aligned slices)" % (args.ref_sample, len(counts), SLICE_NAME, total, cores))
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * el / len(timed), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg["workload"], "sample_elements": total},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    from synth.params import CONFIGS
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="llama2-7b",
                    choices=sorted(CONFIGS) + ["act-codec", "swiglu-fp8", "rmsnorm-fp8"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fmt-v", type=int, choices=[0, 1, 2], default=None,
                    help="override the workload's v format (2: E5M2 expanded to its own span)")
    ap.add_argument("--compare-flat", action="store_true",
                    help="also time one flat tensor of the same parameter count")
    ap.add_argument("--clip", type=float, default=None, metavar="MAX_NORM",
                    help="time the clipped step: gradient-norm pass + step on coef * g")
    ap.add_argument("--zero1", action="store_true",
                    help="time the ZeRO-1 sharded step (reduce-scatter, step, all-gather) over "
                         "the ranks instead of one replica per rank")
    ap.add_argument("--exact-group-params", action="store_true",
                    help="run the step with exact group parameters (coat_set_exact_group_params)")
    ap.add_argument("--no-extras", dest="extras", action="store_false",
                    help="skip the ragged, 13B and codec figures of the default run")
    ap.add_argument("--cpu-sample", type=int, default=0,
                    help="oracle baseline: elements per tensor of the 7B slice (0: whole "
                         "tensors, the slice's 333,455,360 parameters)")
    ap.add_argument("--ref-sample", type=int, default=1 << 21,
                    help="reference arm: elements per tensor of the 7B slice per step")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws, rank, local = dist_env()
    if args.config in ("act-codec", "swiglu-fp8", "rmsnorm-fp8"):
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "this workload has no "
                              "reference arm; the oracle CPU baseline is in the ours line"}))
            return
        run = {"act-codec": run_codec, "swiglu-fp8": run_swiglu,
               "rmsnorm-fp8": run_rmsnorm}[args.config]
        res = run(args, ws, rank, local)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    cfg = dict(CONFIGS[args.config])
    if args.fmt_v is not None and args.fmt_v != cfg["fmt_v"]:
        cfg["fmt_v"] = args.fmt_v
        cfg["workload"] = cfg["workload"].split(", E4M3")[0] + ", E4M3 m + %s v" % FMT_NAMES[args.fmt_v]
    if args.impl == "reference":
        res = run_reference(args, cfg, ws, rank)
    elif args.zero1:
        res = run_zero1(args, cfg, ws, rank, local)
    else:
        res = run_ours(args, cfg, ws, rank, local)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
