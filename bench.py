"""Benchmark: causal attention forward + backward through libcattn's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cattn,reference}]
                    [--workload INDEX]

One step = one pass of the whole hot path over one batch: attn_fwd (O, LSE)
then attn_bwd (Delta preprocess, main backward, dQ convert) on the GPT-2
124M attention layer (B=16, H=12, T=1024, D=64, bf16) unless --workload
picks another of the five workloads.  These are the plain calls (standard
bf16 mixed precision, which meets the stated tolerance on this workload);
--precise times attn_fwd_ex / attn_bwd_ex with the O residual instead (the
path that meets it on every workload).  Prints one JSON line on rank 0.

Throughput uses the causal FLOP convention: forward = 2*B*H*T^2*D (half of
the dense 4*B*H*T^2*D), backward = 2.5 x forward, step = 3.5 x forward.

L2 (126 MB): every step's working set (about 280 MB at the headline
workload) exceeds L2, and steps rotate over 3 input sets, so each step's
inputs were last touched two steps (>500 MB of traffic) earlier.

N > 1 (torchrun): the path does not shard inside one problem and needs no
collective, so every rank runs its own full replica of the workload
(weak scaling); NCCL is used only for the barrier and the max-over-ranks
timing.

--impl reference: the fp64 CPU oracle (the correctness reference; there is
no other implementation to compare with) timed on the host cores over a
bounded sample of heads of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import WORKLOADS, HEADLINE, seed_for, workload_inputs  # noqa: E402

METRIC = "causal attn fwd+bwd TFLOP/s at GPT-2 124M shape; % of B200 BF16 peak"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "causal_self_attention_flash_b200", "csrc")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's published dense bf16 tensor peak of one B200 (no sparsity), TFLOP/s
PUBLISHED_BF16_TFLOPS = 2250.0
N_SETS = 3


def fwd_flops(w) -> float:
    return 2.0 * w.B * w.H * w.T * w.T * w.D


def step_flops(w) -> float:
    return 3.5 * fwd_flops(w)


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "fwd_kernel": ("fwd.cuh", "philox.cuh", "sched.cuh", "sm100.cuh"),
    "bwd_kernel": ("bwd.cuh", "philox.cuh", "sm100.cuh"),
    "bwd_pre_kernel": ("bwd.cuh", "philox.cuh", "sm100.cuh"),
    "dq_convert_kernel": ("bwd.cuh", "philox.cuh", "sm100.cuh"),
}


def code_only(src: str) -> str:
    """C++ source without its comments and blank lines (so that a comment
    edit does not count as a change of the kernel)."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    lines = []
    for line in src.splitlines():
        cut = line.find("//")
        if cut >= 0 and line.count('"', 0, cut) % 2 == 0:
            line = line[:cut]
        if line.strip():
            lines.append(line.rstrip())
    return "\n".join(lines)


def source_hash(kernel: str) -> str:
    """Hash of the device code a kernel is compiled from, comments aside
    (its ncu traffic figure is reported only while this matches the one
    stored with it)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            h.update(f.encode())
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def kernel_algorithmic(w, name):
    """(amount per launch, unit, bound) for a kernel of the step."""
    bhtd = w.B * w.H * w.T * w.D
    bht = w.B * w.H * w.T
    tpad = (w.T + 127) // 128 * 128
    if name == "fwd_kernel":
        return fwd_flops(w), "flop", "tensor"
    if name == "bwd_kernel":
        return 2.5 * fwd_flops(w), "flop", "tensor"
    if name == "bwd_pre_kernel":
        # read O, dO (bf16), LSE; write Delta, LSE*log2e (padded); zero dQ acc
        return 2 * bhtd * 2 + bht * 4 + 2 * w.B * w.H * tpad * 4 + bhtd * 4, "byte", "hbm"
    if name == "dq_convert_kernel":
        return bhtd * 4 + bhtd * 2, "byte", "hbm"
    raise KeyError(name)


class ClockSampler:
    """NVML sampler of SM clock and throttle reasons during a region."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.ok = False
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001  (no NVML: clocks reported as unknown)
            self.ok = False

    def sample(self):
        if not self.ok:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, bit in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(self.period)

    def __enter__(self):
        self.sample()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self.t.join()
        self.sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = sorted(self.reasons - {"gpu_idle"})
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, x: float, device: str = "cuda") -> float:
    """The maximum of x over all ranks (every rank gets it); device is where
    the reduction tensor lives ("cuda" for NCCL, "cpu" for gloo)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def cpu_oracle_rate(w, index, budget_s=15.0, max_heads=None):
    """Time the fp64 oracle (fwd + bwd) on whole heads of the workload until
    about budget_s of CPU work; returns (TFLOP/s, heads, seconds)."""
    import oracle
    from workloads import as_f64, bf16_inputs, sample_heads
    heads = sample_heads(w.BH, max_heads or w.BH, seed=seed_for(index) + 77)
    per_head = step_flops(w) / w.BH
    done, t_total = 0, 0.0
    for f in heads:
        b, h = divmod(f, w.H)
        # draw this head's inputs on their own (the oracle sees the same
        # distribution as the workload; values need not match the GPU's)
        q, k, v, do = (as_f64(t) for t in bf16_inputs(1, 1, w.T, w.D, seed_for(index) * 1000 + f,
                                                       w.qk_std))
        t0 = time.perf_counter()
        oracle.attention_forward(q, k, v, w.scale)
        oracle.attention_backward(q, k, v, do, w.scale)
        t_total += time.perf_counter() - t0
        done += 1
        if t_total >= budget_s:
            break
    return per_head * done / t_total / 1e12, done, t_total


def run_reference(args, w, index, world, rank):
    if rank != 0:
        return
    # one step = one bounded sample of heads; K steps after W warm-ups
    per_step = max(1, min(w.BH, int(os.environ.get("CATTN_REF_HEADS", "4"))))
    import oracle
    from workloads import as_f64, bf16_inputs
    heads = [bf16_inputs(1, 1, w.T, w.D, seed_for(index) * 1000 + i, w.qk_std)
             for i in range(per_step)]
    heads = [[as_f64(t) for t in hd] for hd in heads]

    def step():
        for q, k, v, do in heads:
            oracle.attention_forward(q, k, v, w.scale)
            oracle.attention_backward(q, k, v, do, w.scale)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    flops = step_flops(w) / w.BH * per_step * args.steps
    value = flops / dt / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "D": w.D,
                   "parallelism": "replicas", "reference": "fp64 CPU oracle"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} of {w.BH} heads per step, fwd+bwd, fp64"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def compulsory_bytes(w):
    """HBM bytes a fwd+bwd step must move: the forward reads Q, K, V and
    writes O, LSE; the preprocess reads O, dO and writes Delta; the backward
    reads Q, K, V, dO, LSE, Delta and writes dQ, dK, dV (no L2-served
    re-reads, no fp32 dQ accumulator traffic)."""
    t = w.B * w.H * w.T * w.D * 2
    v = w.B * w.H * w.T * 4
    return (4 * t + v) + (2 * t + v) + (7 * t + 2 * v)


def measure_detail(args, w, sets, olos, step, stream, cattn):
    n = max(args.steps, 20)

    def timed(fn, count):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(count + 1)]
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(count):
            fn(i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        return [ev[i].elapsed_time(ev[i + 1]) for i in range(count)]

    def pct(xs, q):
        ys = sorted(xs)
        return ys[min(len(ys) - 1, int(q * (len(ys) - 1) + 0.5))]

    per_step = timed(step, n)
    tf = lambda flops, ms: flops / (ms / 1e3) / 1e12  # noqa: E731

    def fwd_only(i):
        qd, kd, vd, dod, o, lse, dq, dk, dv, ws = sets[i % N_SETS]
        if olos[i % N_SETS] is not None:
            cattn.attn_fwd_ex(qd, kd, vd, w.scale, o=o, lse=lse, o_lo=olos[i % N_SETS],
                              stream=stream)
        else:
            cattn.attn_fwd(qd, kd, vd, w.scale, o=o, lse=lse, stream=stream)

    def bwd_only(i):
        qd, kd, vd, dod, o, lse, dq, dk, dv, ws = sets[i % N_SETS]
        cattn.attn_bwd(qd, kd, vd, o, lse, dod, w.scale, dq=dq, dk=dk, dv=dv, workspace=ws,
                       stream=stream, o_lo=olos[i % N_SETS])

    for i in range(N_SETS):
        fwd_only(i)
    fwd_ms = timed(fwd_only, n)
    bwd_ms = timed(bwd_only, n)
    one_set = timed(lambda i: step(0), n)
    med = pct(per_step, 0.5)
    detail = {
        "step_ms": {"median": med, "p10": pct(per_step, 0.1), "p90": pct(per_step, 0.9),
                    "samples": n},
        "fwd_alone": {"tflops": tf(fwd_flops(w), pct(fwd_ms, 0.5)), "ms_median": pct(fwd_ms, 0.5)},
        "bwd_alone": {"tflops": tf(2.5 * fwd_flops(w), pct(bwd_ms, 0.5)),
                      "ms_median": pct(bwd_ms, 0.5),
                      "includes": "preprocess + main + dQ convert"},
        "single_input_set": {"tflops": tf(step_flops(w), pct(one_set, 0.5)),
                             "note": "no rotation: whatever of the step fits stays in L2"},
        "hbm_compulsory": {"bytes_per_step": compulsory_bytes(w),
                           "gbs_at_median_step": compulsory_bytes(w) / (med / 1e3) / 1e9},
    }
    # context: torch.nn.functional.scaled_dot_product_attention (a library
    # kernel; run and timed only) on the same inputs and shapes
    try:
        qd, kd, vd, dod = (t.detach() for t in sets[0][:4])
        q_, k_, v_ = (t.clone().requires_grad_(True) for t in (qd, kd, vd))

        def sdpa(i):
            out = torch.nn.functional.scaled_dot_product_attention(q_, k_, v_, is_causal=True,
                                                                   scale=w.scale)
            out.backward(dod)

        for i in range(3):
            sdpa(i)
        sd = timed(sdpa, n)
        detail["context_torch_sdpa"] = {"tflops_fwd_bwd": tf(step_flops(w), pct(sd, 0.5)),
                                        "ms_median": pct(sd, 0.5)}
    except Exception as e:  # noqa: BLE001  (context only)
        detail["context_torch_sdpa"] = {"unavailable": str(e)[:120]}
    try:
        detail["decode"] = measure_decode(w, sets, stream, cattn, n)
    except Exception as e:  # noqa: BLE001  (a side measurement; the step stands)
        detail["decode"] = {"unavailable": str(e)[:120]}
    try:
        detail["dropout"] = measure_dropout(w, sets, stream, cattn, timed, pct,
                                            pct(fwd_ms, 0.5), pct(bwd_ms, 0.5))
    except Exception as e:  # noqa: BLE001  (a side measurement; the step stands)
        detail["dropout"] = {"unavailable": str(e)[:120]}
    return detail


DROPOUT_P = 0.2  # the pages' Shakespeare model (nanoGPT page, section 3)


def measure_dropout(w, sets, stream, cattn, timed, pct, fwd_plain_ms, bwd_plain_ms):
    """The workload's forward and backward calls with attention dropout
    p = 0.2 (the _strided calls with a Dropout), keep bits drawn in both
    calls or kept by the forward for the backward (the keep-bit cache);
    median ms per call over the rotating input sets, and the ratio to the
    plain calls."""
    n = 20
    B, H, T = w.B, w.H, w.T
    masks = [cattn.attn_dropout_mask(B, H, T, sets[0][0].device) for _ in range(N_SETS)]
    out = {"p": DROPOUT_P, "calls": n}
    for kind in ("drawn", "cached"):
        def params(i):
            return cattn.dropout_params(DROPOUT_P, seed=1234, offset=i % N_SETS,
                                        mask=masks[i % N_SETS] if kind == "cached" else None)

        def fwd(i):
            qd, kd, vd, dod, o, lse, dq, dk, dv, ws = sets[i % N_SETS]
            cattn.attn_fwd_strided(qd, kd, vd, w.scale, o=o, lse=lse, stream=stream,
                                   dropout=params(i))

        def bwd(i):
            qd, kd, vd, dod, o, lse, dq, dk, dv, ws = sets[i % N_SETS]
            cattn.attn_bwd_strided(qd, kd, vd, o, lse, dod, w.scale, dq=dq, dk=dk, dv=dv,
                                   workspace=ws, stream=stream, dropout=params(i))

        for i in range(N_SETS):
            fwd(i)
        f = pct(timed(fwd, n), 0.5)
        # input set s's backward then holds its forward's mask (offset s)
        for i in range(N_SETS):
            fwd(i)
        b = pct(timed(bwd, n), 0.5)
        out[kind] = {"fwd_ms": f, "bwd_ms": b, "fwd_vs_plain": f / fwd_plain_ms,
                     "bwd_vs_plain": b / bwd_plain_ms}
    return out


def decode_bytes(B, H, L, D, Tq=1) -> int:
    """Compulsory HBM bytes of one decode call: the L cached K and V rows of
    every head (bf16), the Tq query rows and outputs (bf16), LSE (fp32)."""
    return 2 * B * H * L * D * 2 + 2 * B * H * Tq * D * 2 + B * H * Tq * 4


def measure_decode(w, sets, stream, cattn, n):
    """attn_decode of the Tq newest positions (Tq = 1, 4, 8) against the
    whole sequence's K and V as the cache, rotating over the input sets
    (their K, V together exceed L2).  The calls are captured in a CUDA graph
    and replayed, so the time is the GPU's (one kernel per call, no host
    launch gaps), as a serving loop would run it."""
    B, H, T, D = w.B, w.H, w.T, w.D
    peaks, src = load_peaks()
    out = {"peak_source": src, "kernels": "decode_kernel (one launch per call)",
           "timing": "CUDA graph of %d calls, replayed; device time per call" % n}
    for tq in (1, 4, 8):
        if tq > T:
            continue
        ws = torch.empty(max(cattn.attn_decode_workspace_bytes(B, H, tq, T, D), 1),
                         dtype=torch.uint8, device=sets[0][0].device)
        outs = [(torch.empty((B, H, tq, D), dtype=torch.bfloat16, device=ws.device),
                 torch.empty((B, H, tq), dtype=torch.float32, device=ws.device))
                for _ in range(N_SETS)]

        def call(i):
            qd, kd, vd = sets[i % N_SETS][:3]
            o, lse = outs[i % N_SETS]
            cattn.attn_decode(qd[:, :, T - tq:], kd, vd, T, w.scale, o=o, lse=lse,
                              workspace=ws)

        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for i in range(N_SETS):
                call(i)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(n):
                call(i)
        graph.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / n)
        per_ms = statistics.median(times)
        byts = decode_bytes(B, H, T, D, tq)
        gbs = byts / (per_ms / 1e3) / 1e9
        out[f"tq{tq}"] = {"shape": f"B={B} H={H} L={T} D={D} Tq={tq}",
                          "us_per_call": per_ms * 1e3, "bytes_per_call": byts, "gbs": gbs,
                          "frac_of_hbm": gbs / peaks["hbm_gbs"]}
        del graph
    return out


def run_cattn(args, w, index, world, rank, local):
    import causal_self_attention_flash_b200 as cattn
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    q0, k0, v0, do0 = workload_inputs(index)
    sets = []
    for s in range(N_SETS):
        # distinct buffers per set (same values: the work is identical)
        qd, kd, vd, dod = (t.to(dev) for t in (q0, k0, v0, do0))
        o = torch.empty_like(qd)
        lse = torch.empty(w.B, w.H, w.T, dtype=torch.float32, device=dev)
        dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
        ws = torch.empty(cattn.attn_bwd_workspace_bytes(w.B, w.H, w.T, w.D), dtype=torch.uint8,
                         device=dev)
        sets.append((qd, kd, vd, dod, o, lse, dq, dk, dv, ws))

    olos = [torch.empty_like(st[0]) for st in sets] if args.precise else [None] * N_SETS

    def step(i):
        qd, kd, vd, dod, o, lse, dq, dk, dv, ws = sets[i % N_SETS]
        if args.precise:
            olo = olos[i % N_SETS]
            cattn.attn_fwd_ex(qd, kd, vd, w.scale, o=o, lse=lse, o_lo=olo, stream=stream)
            cattn.attn_bwd(qd, kd, vd, o, lse, dod, w.scale, dq=dq, dk=dk, dv=dv, workspace=ws,
                           stream=stream, o_lo=olo)
        else:
            cattn.attn_fwd(qd, kd, vd, w.scale, o=o, lse=lse, stream=stream)
            cattn.attn_bwd(qd, kd, vd, o, lse, dod, w.scale, dq=dq, dk=dk, dv=dv, workspace=ws,
                           stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert cattn.cattn_get_device_status() == cattn.OK

    # ---- timed region: exactly K steps
    sampler = ClockSampler(local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(world, ms)
    status = cattn.cattn_get_device_status()
    total_flops = step_flops(w) * args.steps * world
    value = total_flops / (ms_max / 1e3) / 1e12

    # ---- per-kernel device time (same K steps again, events per launch)
    cattn.cattn_timing_enable(True)
    cattn.cattn_timing_read()
    for i in range(args.steps):
        step(i)
    torch.cuda.synchronize()
    ktimes = cattn.cattn_timing_read()
    cattn.cattn_timing_enable(False)
    total_k = sum(t for t, _ in ktimes.values()) or 1.0
    dom = max(ktimes, key=lambda n: ktimes[n][0])
    amount, unit, bound = kernel_algorithmic(w, dom)
    per_launch_ms = ktimes[dom][0] / max(ktimes[dom][1], 1)
    peaks, peak_src = load_peaks()
    if bound == "tensor":
        achieved = amount / (per_launch_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        r_unit = "TFLOP/s"
    else:
        achieved = amount / (per_launch_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        r_unit = "GB/s"
    traffic = None
    try:
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f)
        ent = tr.get(dom, {})
        if ent.get("source_hash") == source_hash(dom) and ent.get("workload") == w.name:
            traffic = ent.get("bytes_per_launch")
    except (OSError, ValueError):
        pass

    # ---- detail (rank 0): step-time spread, forward and backward alone, a
    # single (unrotated) input set, HBM rate on the compulsory bytes, and
    # torch's own fused attention on the same inputs as a context row
    detail = None
    if rank == 0:
        detail = measure_detail(args, w, sets, olos, step, stream, cattn)

    # ---- end to end: pinned host buffers -> device -> fwd+bwd -> host.
    # Three streams, as a training loop runs them: step i's inputs are
    # copied in (one copy engine) while step i-1 computes and step i-2's
    # results are copied out (the other engine).  Events keep each of the
    # N_SETS device buffer sets in order: its inputs are overwritten only
    # after the step three back has read them, its outputs only after they
    # were copied out.
    host_in = [t.pin_memory() for t in (q0, k0, v0, do0)]
    host_out = [torch.empty(w.B, w.H, w.T, w.D, dtype=torch.bfloat16).pin_memory()
                for _ in range(4)] + [torch.empty(w.B, w.H, w.T, dtype=torch.float32).pin_memory()]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    loaded = [torch.cuda.Event() for _ in range(N_SETS)]
    computed = [torch.cuda.Event() for _ in range(N_SETS)]
    drained = [torch.cuda.Event() for _ in range(N_SETS)]
    used = [False] * N_SETS

    def e2e_step(i):
        s = i % N_SETS
        qd, kd, vd, dod, o, lse, dq, dk, dv, ws = sets[s]
        if used[s]:
            cin.wait_event(computed[s])
        with torch.cuda.stream(cin):
            for dst, src in zip((qd, kd, vd, dod), host_in):
                dst.copy_(src, non_blocking=True)
        loaded[s].record(cin)
        stream.wait_event(loaded[s])
        if used[s]:
            stream.wait_event(drained[s])
        step(i)
        computed[s].record(stream)
        cout.wait_event(computed[s])
        with torch.cuda.stream(cout):
            for dst, src in zip(host_out, (o, dq, dk, dv, lse)):
                dst.copy_(src, non_blocking=True)
        drained[s].record(cout)
        used[s] = True

    for i in range(min(args.warmup, 3)):
        e2e_step(i)
    barrier(world)
    torch.cuda.synchronize()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    cin.wait_event(e2)
    cout.wait_event(e2)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_stream(cin)
    stream.wait_stream(cout)
    e3.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(world, e2.elapsed_time(e3))
    e2e_value = total_flops / (e2e_ms / 1e3) / 1e12

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, nheads, secs = cpu_oracle_rate(w, index, budget_s=args.cpu_budget)
        cpu = {"value": rate, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{nheads} of {w.BH} heads, fwd+bwd in fp64 ({secs:.1f} s)"}

    if rank == 0:
        clocks = sampler.summary()
        pct = value / world / peaks["bf16_tflops"] * 100.0
        fk_ms, fk_n = ktimes["fwd_kernel"]
        fwd_tf = fwd_flops(w) / (fk_ms / fk_n / 1e3) / 1e12 if fk_n else None
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "D": w.D,
                       "global_batch": w.B * world, "seq_len": w.T,
                       "parallelism": f"replicas x{world}",
                       "path": ("attn_fwd_ex + attn_bwd_ex with O residual" if args.precise
                                else "attn_fwd + attn_bwd"),
                       "l2": f"{N_SETS} rotating input sets, step working set > L2"},
            "pct_of_peak": pct,
            "peak_source": f"{peak_src} bf16 {peaks['bf16_tflops']} TFLOP/s (burst)",
            "pct_of_published_peak": value / world / PUBLISHED_BF16_TFLOPS * 100.0,
            "fwd_tflops": fwd_tf,
            "fwd_pct_of_peak": fwd_tf / peaks["bf16_tflops"] * 100.0 if fwd_tf else None,
            "fwd_pct_of_published_peak": fwd_tf / PUBLISHED_BF16_TFLOPS * 100.0 if fwd_tf else None,
            "kernels": {n: {"ms_per_launch": t / c if c else None, "launches": c,
                            "share": t / total_k} for n, (t, c) in ktimes.items()},
            "roofline": {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak,
                         "unit": r_unit, "frac": achieved / peak, "traffic": traffic,
                         "peak_source": peak_src,
                         "algorithmic_per_launch": amount, "algorithmic_unit": unit},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "pipeline": "copy-in, fwd+bwd and copy-out of consecutive steps on three streams"},
            "gpu_launches": sum(c for _, c in ktimes.values()),
            "clocks": clocks,
            "device_status": status,
            "detail": detail,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="cattn", choices=["cattn", "reference"])
    ap.add_argument("--workload", type=int, default=HEADLINE)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--precise", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, args.workload, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_cattn(args, w, args.workload, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
