"""Throughput of causal GQA attention forward+backward on B200.

One step = nea_attn_fwd_save + nea_attn_bwd_saved, the save-for-backward pair
(four kernels: the forward operand prologue, which keeps its planes for the
backward; the forward; the backward prologue, which converts dO and writes the
row terms; and the gradient kernel with its dK/dV and dQ units) over one batch
of synthetic inputs already resident in HBM.
Default workload: B=4, T=1024, Hq=12, Hkv=4, D=64, float32 storage, causal,
RoPE base 10000, Q,K ~ N(0, 9), V, dO ~ N(0, 1) -- the longer-context
configuration of the NanoEuler GPU model shape.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long]
    python bench.py --impl reference ...   # the fp64 CPU oracle, timed on host cores

Prints one JSON line (rank 0).  value = algorithmic TFLOP/s of the whole job
(7 * B * Hq * T^2 * D per causal step and layer, summed over ranks, divided by
the slowest rank's device time of the K timed steps).  L2 is flushed before
every timed step, outside the step's events: a 256 MiB write, then a 256 MiB
read of another buffer, which evicts the written lines so that their
write-back is not charged to the first kernel of the step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal GQA attention fwd+bwd TFLOP/s (% of tensor-core peak) and tokens/s"
KERNELS = ("attn_fwd_prologue", "attn_fwd", "attn_bwd_prologue", "attn_bwd")
# Algorithmic work per kernel in units of B*Hq*T^2*D (causal): the forward's
# two products; the gradient kernel's five (S, dP, dV, dK, dQ: its dQ units
# recompute S and dP, which are not credited again).
UNITS = {"attn_fwd": 2.0, "attn_bwd": 5.0}
L2_FLUSH_BYTES = 256 << 20


def prologue_bytes(w, kernel):
    """Algorithmic HBM bytes of one operand-prologue launch: every input
    element read once and every output element written once.  The forward's
    prologue converts Q, K, V (bf16 storage: rotates Q, K); the backward's, fed
    the saved planes, writes the row terms and (fp32 storage) dO's planes."""
    nq, nk = w.B * w.T * w.Hq * w.D, w.B * w.T * w.Hkv * w.D
    rope = w.rope_base > 0
    e = 4 if w.dtype == "f32" else 2
    if kernel == "attn_fwd_prologue":
        if w.dtype == "f32":  # fp32 in, bf16 hi + lo out
            return (nq + 2 * nk) * (4 + 4)
        return (nq + nk) * (2 + 2) if rope else 0  # rotated bf16 copies of Q, K
    # backward: row terms read O, dO (once) and LSE and write ws[B*Hq][2][Tp];
    # for fp32 storage the same pass writes dO's bf16 hi + lo planes
    tp = -(-w.T // 128) * 128
    b = 2 * nq * e + 4 * w.B * w.Hq * w.T + 8 * w.B * w.Hq * tp
    if w.dtype == "f32":
        b += nq * 4
    return b


def load_workloads():
    """The workload table and input generator, loaded by file path: importing
    it through the package would run the package's ``__init__``, which loads
    the CUDA library, and the reference arm must not load it."""
    import importlib.util

    name = "_nea_workloads"
    if name in sys.modules:
        return sys.modules[name]
    spec = importlib.util.spec_from_file_location(
        name, os.path.join(ROOT, "causal_gqa_attention_sm_b200", "workloads.py"))
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    spec.loader.exec_module(mod)
    return mod


L2_NOTE = "flushed before every timed step (256 MiB write, then 256 MiB read of another buffer)"
L2_BYTES = 126 << 20


def decode_copies(w):
    """Cache copies a decode benchmark cycles through: each step reads its own
    copy, and the copies together exceed twice the L2, so a copy is evicted
    before it is read again."""
    return max(2, -(-2 * L2_BYTES // w.cache_bytes()) + 1)


def decode_l2_note(w):
    n = decode_copies(w)
    return (f"each step reads its own copy of the cache: {n} copies of {w.cache_bytes() / 1e6:.1f} MB "
            f"({n * w.cache_bytes() / 1e6:.0f} MB, over twice the 126 MB L2), cycled")


def config_of(w, world):
    """The `config` object of a bench line; both arms print the same one."""
    storage = {"f32": "float32", "bf16": "bfloat16"}[w.dtype]
    if w.decode:
        return {"workload": w.name, "B": w.B, "Tc": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "storage": storage,
                "rope_base": w.rope_base, "lens": "all Tc", "l2": decode_l2_note(w),
                "parallelism": f"dp{world} (independent sequences per GPU)"}
    if w.block and w.ffn:
        return {"workload": w.name, "B": w.B, "T": w.T, "C": w.Hq * w.D, "F": w.ffn, "storage": storage,
                "rmsnorm_eps": 1e-5, "l2": L2_NOTE, "parallelism": f"dp{world} (independent batches per GPU)"}
    if w.block:
        return {"workload": w.name, "B": w.B, "T": w.T, "C": w.Hq * w.D, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                "storage": storage, "rmsnorm_eps": 1e-5, "l2": L2_NOTE,
                "parallelism": f"dp{world} (independent batches per GPU)"}
    return {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "storage": storage,
            "causal": w.causal, "rope_base": w.rope_base, "layers": w.layers, "qk_std": w.qk_std, "l2": L2_NOTE,
            "parallelism": f"dp{world} (independent batches per GPU)"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long")
    ap.add_argument("--impl", default="nea", choices=["nea", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--clocks-csv", default=None, help="keep the raw nvidia-smi clock samples in this file")
    ap.add_argument("--profile", action="store_true",
                    help="for runs under ncu: only warm-up, timed and per-kernel steps (no CPU baseline, no e2e, "
                         "no TF32 peak, no clock window); its numbers are not bench values")
    a = ap.parse_args()
    if a.profile:
        a.no_cpu_baseline = a.no_e2e = True
    a.warmup = max(a.warmup, 3)
    return a


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- distributed plumbing
def dist_init(n):
    if n <= 1 and "WORLD_SIZE" not in os.environ:
        return 0, 1, 0
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def batch_shard(B, world, rank):
    """Rows [lo, hi) of a batch of B that `rank` owns: contiguous, sizes differ
    by at most one.  Batches are independent, so shards exchange nothing."""
    base, extra = divmod(B, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(x, world, device="cuda"):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, path=None):
        self.idx = gpu_index
        self.proc = None
        # the raw samples: a file of the caller's choosing, else a temporary one
        self.path = path or os.path.join(tempfile.gettempdir(), f"nea_clocks_{os.getpid()}_{gpu_index}.csv")

    def __enter__(self):
        self.f = None
        try:
            os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
            if self.f is not None:
                self.f.close()
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            self.proc.wait(timeout=10)
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        num = lambda v: v.replace(".", "", 1).isdigit()  # noqa: E731  ("[N/A]" and the like are skipped)
        sm = [float(r[1]) for r in rows if num(r[1])]
        mx = max((float(r[2]) for r in rows if num(r[2])), default=None)
        load = ([s for s in sm if s > 0.5 * mx] if mx else []) or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows if num(r[3])), default=None)}


def clock_window(step, flush_l2, stream, dev, seconds):
    """Runs identical steps (each after an L2 flush, when `flush_l2` is given;
    else `step(i)` is called with the step's index) for at least `seconds` and
    returns their count and mean device time per step."""
    import torch

    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n, t0 = 0, time.perf_counter()
    s0.record(stream)
    while True:
        for _ in range(20):
            if flush_l2 is None:
                step(n)
            else:
                flush_l2(n)
                step()
            n += 1
        torch.cuda.synchronize(dev)
        if time.perf_counter() - t0 >= seconds:
            break
    s1.record(stream)
    torch.cuda.synchronize(dev)
    return {"steps": n, "seconds": time.perf_counter() - t0,
            "ms_per_step_incl_flush" if flush_l2 is not None else "ms_per_step": s0.elapsed_time(s1) / n,
            "note": "steps run under the clock sampler before the timed ones; not part of `value`"}


def measure_tf32_peak(dev, sustain_s=4.0):
    """Dense TF32 tensor-core throughput of this GPU, measured the way the
    bf16 peak is: a float32 8192^3 torch.matmul with TF32 allowed (a cuBLAS
    call, used only as a yardstick), as a burst of 10 and as a loop of about
    `sustain_s` seconds."""
    import torch

    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        n = 8192
        g = torch.Generator(device=dev).manual_seed(0)
        a = torch.randn((n, n), device=dev, generator=g)
        b = torch.randn((n, n), device=dev, generator=g)
        c = torch.empty((n, n), device=dev)
        for _ in range(3):
            torch.matmul(a, b, out=c)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record()
        for _ in range(10):
            torch.matmul(a, b, out=c)
        e1.record()
        torch.cuda.synchronize(dev)
        burst = 2.0 * n ** 3 * 10 / (e0.elapsed_time(e1) * 1e-3) / 1e12
        reps = max(10, int(sustain_s * burst * 1e12 / (2.0 * n ** 3)))
        e0.record()
        for _ in range(reps):
            torch.matmul(a, b, out=c)
        e1.record()
        torch.cuda.synchronize(dev)
        sustained = 2.0 * n ** 3 * reps / (e0.elapsed_time(e1) * 1e-3) / 1e12
        del a, b, c
        return {"tf32_tflops": burst, "tf32_tflops_sustained": sustained,
                "how": "torch.matmul float32 8192^3 with TF32 allowed (cuBLAS), burst of 10 and a ~4 s loop"}
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


# ---------------------------------------------------------------- ncu traffic records
# The sources that make up each kernel: its own header plus the shared device
# helpers, tile geometry and the host code that sets up its launch.
KERNEL_SOURCES = {"attn_fwd_prologue": ("nea_prep.cuh",), "attn_bwd_prologue": ("nea_prep.cuh",),
                  "attn_fwd": ("nea_fwd.cuh",), "attn_bwd": ("nea_bwd.cuh", "nea_bwd_f32.cuh"),
                  "attn_decode": ("nea_decode.cuh",)}
SHARED_SOURCES = ("nea_attn.cu", "nea_device.cuh", "nea_tiles.cuh")


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "causal_gqa_attention_sm_b200", "csrc")
    for name in sorted(SHARED_SOURCES + KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, or None when absent
    or when the kernel's sources changed since it was captured."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- CPU baseline (oracle)
def run_oracle_sample(w, max_units=None, min_seconds=0.0):
    """Times the fp64 oracle on (batch, kv-group) slices of the workload (each
    slice: one batch element, the G query heads of one kv head), all slices in
    one call so OpenMP spreads them over the host cores, repeated until at
    least `min_seconds` have passed.  Returns (seconds, flops, threads,
    description)."""
    import numpy as np

    import oracle

    make_inputs = load_workloads().make_inputs
    cores = len(os.sched_getaffinity(0))
    units = w.B * w.Hkv
    n = min(units, max_units or units)
    inp = make_inputs(w)
    G = w.G
    pairs = [(i // w.Hkv, i % w.Hkv) for i in range(n)]
    arr = {k: v.float().double().numpy() for k, v in inp.items()}
    qs = np.concatenate([arr["q"][b:b + 1, :, g * G:(g + 1) * G] for b, g in pairs])
    dos = np.concatenate([arr["do"][b:b + 1, :, g * G:(g + 1) * G] for b, g in pairs])
    ks = np.concatenate([arr["k"][b:b + 1, :, g:g + 1] for b, g in pairs])
    vs = np.concatenate([arr["v"][b:b + 1, :, g:g + 1] for b, g in pairs])
    threads = min(cores, n)
    oracle.set_threads(threads)
    reps, dt = 0, 0.0
    while reps == 0 or dt < min_seconds:
        t0 = time.perf_counter()
        oracle.attn_fwd(qs, ks, vs, w.rope_base, w.causal)
        oracle.attn_bwd(qs, ks, vs, dos, w.rope_base, w.causal)
        dt += time.perf_counter() - t0
        reps += 1
    flops = w.flops() / w.layers * n / units * reps
    desc = (f"{n} of {units} (batch, kv-group) slices of one layer, fwd+bwd, fp64, {threads} threads"
            + (f", {reps} repetitions" if reps > 1 else ""))
    return dt, flops, threads, desc


def reference_arm(a, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    per_step_units = max(1, min(w.B * w.Hkv, len(os.sched_getaffinity(0))))
    for _ in range(a.warmup):  # untimed steps of the same sample (page in, spin up the thread pool)
        run_oracle_sample(w, per_step_units)
    secs, flops = 0.0, 0.0
    threads = desc = None
    for _ in range(a.steps):
        dt, fl, threads, desc = run_oracle_sample(w, per_step_units)
        secs += dt
        flops += fl
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": secs / a.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, a.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- decode workloads
DECODE_METRIC = "GQA decode attention over a key/value cache: cache GB/s (HBM) and tokens/s"


def run_oracle_decode(w, min_seconds=0.0):
    """Times the fp64 oracle's decode on the whole workload, repeated until at
    least `min_seconds` have passed.  Returns (seconds, cache bytes, threads,
    description)."""
    import oracle

    inp = load_workloads().make_decode_inputs(w)
    arr = {k: v.float().double().numpy() if k != "lens" else v.numpy() for k, v in inp.items()}
    threads = min(len(os.sched_getaffinity(0)), w.B * w.Hq)
    oracle.set_threads(threads)
    reps, dt = 0, 0.0
    while reps == 0 or dt < min_seconds:
        t0 = time.perf_counter()
        oracle.attn_decode(arr["q"], arr["kc"], arr["vc"], arr["lens"], w.rope_base)
        dt += time.perf_counter() - t0
        reps += 1
    desc = f"whole decode step ({w.B} sequences x {w.T} cached positions), fp64, {threads} threads, {reps} repetitions"
    return dt, w.cache_bytes() * reps, threads, desc


def decode_main(a, w, rank, world, local):
    import torch

    import causal_gqa_attention_sm_b200 as nea
    from causal_gqa_attention_sm_b200.workloads import make_decode_inputs

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    inp = {n: t.to(dev) for n, t in make_decode_inputs(w).items()}
    # step i reads copy i % n of the cache; n copies exceed twice the L2
    copies = [(inp["kc"], inp["vc"])] + [(inp["kc"].clone(), inp["vc"].clone()) for _ in range(decode_copies(w) - 1)]
    o = torch.empty_like(inp["q"])
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)

    def step(i=0):
        kc, vc = copies[i % len(copies)]
        nea.nea_attn_decode(inp["q"], kc, vc, inp["lens"], w.rope_base, o=o, lse=lse)

    for i in range(max(a.warmup, len(copies))):
        step(i)
    torch.cuda.synchronize(dev)
    if nea.nea_device_status() != nea.NEA_OK:
        raise SystemExit("device status after warm-up")
    K = a.steps
    # the K steps are captured once in a CUDA graph and replayed, so that the
    # device time is the kernels' (a decode step is shorter than the host's
    # per-call argument checks and launch)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(K):
            step(i)
    graph.replay()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local, a.clocks_csv)
    barrier(world)
    torch.cuda.synchronize(dev)
    with clocks:
        window = None if a.profile else clock_window(lambda i=0: graph.replay(), None, stream, dev, 1.2)
        if window:
            window["ms_per_step"] /= K  # each clock-window step replays the K-step graph
        ev0.record(stream)
        graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    if nea.nea_device_status() != nea.NEA_OK:
        raise SystemExit("device status after timing")
    total_ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    byts = w.cache_bytes()
    value = byts * K * world / (total_ms * 1e-3) / 1e9
    pk = peaks()
    roof = {"bound": "hbm", "achieved": value / world, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": value / world / pk["hbm_gbs"], "traffic": ncu_traffic("attn_decode", w.name),
            "kernel": "attn_decode"}
    e2e = None
    if not a.no_e2e:
        host = {n: t.cpu().pin_memory() for n, t in inp.items()}
        ho, hl = torch.empty(o.shape, dtype=o.dtype, pin_memory=True), torch.empty(lse.shape, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()

        def e2e_step():
            for n in inp:
                inp[n].copy_(host[n], non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        for _ in range(a.warmup):
            e2e_step()
        torch.cuda.synchronize(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(K):
            e2e_step()
        s1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(s0.elapsed_time(s1), world)
        e2e = {"value": byts * K * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "tokens_per_s": w.B * K * world / (e2e_ms * 1e-3)}
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        dt, cb, threads, desc = run_oracle_decode(w, min_seconds=10.0)
        cpu = {"value": cb / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": dt}
    if rank == 0:
        line = {
            "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": a.warmup, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": config_of(w, world),
            "tokens_per_s": w.B * K * world / (total_ms * 1e-3),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks.summary(),
            "clock_window": window, "gpu_launches": 2 * K,  # stream kernel and merge kernel per step
        }
        print(json.dumps(line), flush=True)
    return 0


def reference_decode(a, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    secs, byts, threads, desc = 0.0, 0, None, None
    for _ in range(a.steps):
        dt, cb, threads, desc = run_oracle_decode(w)
        secs += dt
        byts += cb
    value = byts / secs / 1e9
    line = {
        "impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": secs / a.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, a.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- block workload
BLOCK_METRIC = ("decoder-block steps beside the attention (RMSNorm + q/k/v projections, output projection + "
                "residual), fwd+bwd TFLOP/s (% of tensor-core peak)")
BLOCK_STEPS = ("qkv_fwd", "out_fwd", "out_bwd", "qkv_bwd")
FFN_METRIC = "pre-norm SwiGLU feed-forward with residual, fwd+bwd TFLOP/s (% of tensor-core peak)"
FFN_STEPS = ("ffn_fwd", "ffn_bwd")


def block_metric(w):
    return FFN_METRIC if w.ffn else BLOCK_METRIC


def block_steps(w):
    return FFN_STEPS if w.ffn else BLOCK_STEPS


def block_step_flops(w):
    M, C, Nqkv, Nq = w.B * w.T, w.Hq * w.D, (w.Hq + 2 * w.Hkv) * w.D, w.Hq * w.D
    if w.ffn:
        return {"ffn_fwd": 6.0 * M * C * w.ffn, "ffn_bwd": 12.0 * M * C * w.ffn}
    return {"qkv_fwd": 2.0 * M * C * Nqkv, "out_fwd": 2.0 * M * Nq * C, "out_bwd": 4.0 * M * Nq * C,
            "qkv_bwd": 4.0 * M * C * Nqkv}


def run_oracle_block(w, rows=None, min_seconds=0.0):
    """Times the fp64 oracle (numpy) on the block steps for the first `rows`
    tokens (all by default), repeated until `min_seconds` have passed.
    Returns (seconds, FLOPs, threads, description)."""
    from oracle import block_ref

    inp = load_workloads().make_block_inputs(w)
    a = {n: t.float().double().numpy() for n, t in inp.items()}
    B = w.B if rows is None else max(1, rows // w.T)
    for n in ("x", "o", "dh", "dq", "dk", "dv"):
        if n in a:
            a[n] = a[n][:B]
    sub = load_workloads().replace(w, B=B)
    reps, dt = 0, 0.0
    while reps == 0 or dt < min_seconds:
        t0 = time.perf_counter()
        if w.ffn:
            _, sv = block_ref.ffn_fwd(a["x"], a["g"], a["Wg"], a["Wu"], a["Wd"])
            block_ref.ffn_bwd(a["x"], a["g"], a["Wg"], a["Wu"], a["Wd"], sv, a["dh"])
        else:
            q, k, v, y, rstd = block_ref.qkv_fwd(a["x"], a["g"], a["Wq"], a["Wk"], a["Wv"], w.Hq, w.Hkv, w.D)
            block_ref.out_fwd(a["x"], a["o"], a["Wo"])
            block_ref.out_bwd(a["o"], a["Wo"], a["dh"])
            block_ref.qkv_bwd(a["x"], a["g"], a["Wq"], a["Wk"], a["Wv"], y, rstd, a["dq"], a["dk"], a["dv"])
        dt += time.perf_counter() - t0
        reps += 1
    threads = len(os.sched_getaffinity(0))
    what = "feed-forward" if w.ffn else "block steps"
    desc = f"{what} on {B} x {w.T} tokens (of {w.B} x {w.T}), fp64 numpy, {reps} repetitions"
    return dt, sub.block_flops() * reps, threads, desc


def reference_block(a, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    run_oracle_block(w, rows=w.T)  # untimed warm-up of the same sample
    secs, flops, threads, desc = 0.0, 0.0, None, None
    for _ in range(a.steps):
        dt, fl, threads, desc = run_oracle_block(w, rows=w.T)
        secs += dt
        flops += fl
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": block_metric(w), "value": value, "unit": "TFLOP/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": secs / a.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, a.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def block_launches(w):
    """Library kernels per step (as the ncu launch lists count them).  Block:
    norm rows, q|k|v GEMM; out GEMM; do GEMM, dWo GEMM + split-K reduce; norm
    rows, dWq|dWk|dWv GEMM + reduce, dy GEMM, norm backward, dg sum (12).
    Feed-forward: norm rows, gate|up and down GEMMs; norm rows, dact, dWd,
    dWg|dWu and dy GEMMs, norm backward, dg sum (10).  Float32 storage adds
    one operand-plane launch per call (4 and 2) and, for the feed-forward,
    the split-K reduces of the down and dy products (2)."""
    if w.ffn:
        return 14 if w.dtype == "f32" else 10
    return 16 if w.dtype == "f32" else 12


def block_main(a, w, rank, world, local):
    import torch

    import causal_gqa_attention_sm_b200 as nea

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    d = {n: t.to(dev) for n, t in load_workloads().make_block_inputs(w).items()}
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    drain = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    drain_sum = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2(i):
        flush.fill_(float(i))
        torch.sum(drain, dim=0, out=drain_sum)

    steps = block_steps(w)
    saved = {}

    def call(name, inp):
        if name == "ffn_fwd":
            h, saved["a"], saved["b"] = nea.nea_block_ffn_fwd(inp["x"], inp["g"], inp["Wg"], inp["Wu"], inp["Wd"])
            return (h,)
        if name == "ffn_bwd":
            return nea.nea_block_ffn_bwd(inp["x"], inp["g"], inp["Wg"], inp["Wu"], inp["Wd"], saved["a"],
                                         saved["b"], inp["dh"])
        if name == "qkv_fwd":
            return nea.nea_block_qkv_fwd(inp["x"], inp["g"], inp["Wq"], inp["Wk"], inp["Wv"], w.Hq, w.Hkv, w.D)
        if name == "out_fwd":
            return (nea.nea_block_out_fwd(inp["x"], inp["o"], inp["Wo"]),)
        if name == "out_bwd":
            return nea.nea_block_out_bwd(inp["o"], inp["Wo"], inp["dh"])
        return nea.nea_block_qkv_bwd(inp["x"], inp["g"], inp["Wq"], inp["Wk"], inp["Wv"], inp["dq"], inp["dk"],
                                     inp["dv"], dres=inp["dh"])

    def step(inp=d, evs=None):
        outs = []
        for i, n in enumerate(steps):
            if evs:
                evs[i].record(stream)
            outs.extend(call(n, inp))
        if evs:
            evs[-1].record(stream)
        return outs

    for i in range(a.warmup):
        flush_l2(i)
        step()
    torch.cuda.synchronize(dev)
    if nea.nea_device_status() != nea.NEA_OK:
        raise SystemExit("device status after warm-up")
    K = a.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(local, a.clocks_csv)
    barrier(world)
    torch.cuda.synchronize(dev)
    with clocks:
        window = None if a.profile else clock_window(step, flush_l2, stream, dev, 1.2)
        for i in range(K):
            flush_l2(i)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    # per-step durations: the same steps again with events between the calls
    ev_k = [[torch.cuda.Event(enable_timing=True) for _ in range(len(steps) + 1)] for _ in range(K)]
    for i in range(K):
        flush_l2(i)
        step(evs=ev_k[i])
    torch.cuda.synchronize(dev)
    if nea.nea_device_status() != nea.NEA_OK:
        raise SystemExit("device status after timing")
    total_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in ev), world)
    flops = w.block_flops()
    value = flops * K * world / (total_ms * 1e-3) / 1e12
    sf = block_step_flops(w)
    kern_ms = {n: sum(e[j].elapsed_time(e[j + 1]) for e in ev_k) / K for j, n in enumerate(steps)}
    kernels = {n: {"ms_per_call": kern_ms[n], "tflops": sf[n] / (kern_ms[n] * 1e-3) / 1e12,
                   "share": kern_ms[n] / sum(kern_ms.values())} for n in steps}
    dominant = max(kern_ms, key=kern_ms.get)
    pk = peaks()
    tf32 = measure_tf32_peak(dev) if (w.dtype == "f32" and not a.profile) else None
    achieved = sf[dominant] / (kern_ms[dominant] * 1e-3) / 1e12
    if tf32:
        roof = {"bound": "tensor", "achieved": achieved, "peak": tf32["tf32_tflops"], "unit": "TFLOP/s",
                "frac": achieved / tf32["tf32_tflops"], "traffic": None,
                "kernel": dominant + " (its GEMMs with the norm and operand-plane kernels)",
                "peak_kind": "tf32 dense burst (measured in this run: " + tf32["how"] + ")",
                "frac_of_bf16_peak": achieved / pk["bf16_tflops"], "bf16_peak_kind": f"bf16 dense burst ({pk['source']})"}
    else:
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops"], "traffic": None,
                "kernel": dominant + " (its GEMMs with the norm and operand-plane kernels)",
                "peak_kind": f"bf16 dense burst ({pk['source']})"}
    e2e = None
    if not a.no_e2e:
        act = ("x", "dh") if w.ffn else ("x", "o", "dh", "dq", "dk", "dv")
        host = {n: d[n].cpu().pin_memory() for n in act}
        dev_in = {n: torch.empty_like(d[n]) for n in act}
        inp = dict(d)
        inp.update(dev_in)
        outs = step(inp)
        host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out)

        def e2e_step():
            for n in act:
                dev_in[n].copy_(host[n], non_blocking=True)
            for t, ho in zip(step(inp), host_out):
                ho.copy_(t, non_blocking=True)

        for _ in range(a.warmup):
            e2e_step()
        torch.cuda.synchronize(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(K):
            e2e_step()
        s1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(s0.elapsed_time(s1), world)
        e2e = {"value": flops * K * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        dt, fl, threads, desc = run_oracle_block(w, rows=w.T, min_seconds=10.0)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": dt}
    if rank == 0:
        line = {
            "metric": block_metric(w), "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": a.warmup, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16x3" if w.dtype == "f32" else "bf16", "data": "synthetic",
            "config": config_of(w, world), "tokens_per_s": w.B * w.T * K * world / (total_ms * 1e-3),
            "kernels": kernels, "roofline": roof, "tf32_peak": tf32, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clocks.summary(), "clock_window": window,
            "gpu_launches": K * block_launches(w),
        }
        print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm
def main():
    a = parse()
    w = load_workloads().WORKLOADS[a.workload]
    if a.impl == "reference":
        if w.block:
            return reference_block(a, w)
        return reference_decode(a, w) if w.decode else reference_arm(a, w)

    import torch

    import causal_gqa_attention_sm_b200 as nea
    from causal_gqa_attention_sm_b200.workloads import make_inputs

    rank, world, local = dist_init(a.gpus)
    torch.cuda.set_device(local)
    if w.decode or w.block:
        rc = (decode_main if w.decode else block_main)(a, w, rank, world, local)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return rc
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    # per-rank independent data: each rank processes its own batch (weak scaling)
    layers = []
    for layer in range(w.layers):
        inp = make_inputs(w, layer + 1000 * rank)
        layers.append({n: t.to(dev) for n, t in inp.items()})
    outs = []
    for L in layers:
        o = torch.empty_like(L["q"])
        lse = torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, device=dev)
        saved = torch.empty(nea.nea_attn_saved_bytes(w.B, w.T, w.Hq, w.Hkv, w.D, w.torch_dtype, w.rope_base),
                            dtype=torch.uint8, device=dev)
        outs.append({"o": o, "lse": lse, "dq": torch.empty_like(L["q"]), "dk": torch.empty_like(L["k"]),
                     "dv": torch.empty_like(L["v"]), "saved": saved})
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    drain = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    drain_sum = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2(i):
        flush.fill_(float(i))
        torch.sum(drain, dim=0, out=drain_sum)

    def layer_step(L, O, s=None):
        nea.nea_attn_fwd_save(L["q"], L["k"], L["v"], w.rope_base, w.causal, o=O["o"], lse=O["lse"],
                              saved=O["saved"], stream=s)
        nea.nea_attn_bwd_saved(L["q"], L["k"], L["v"], O["o"], O["lse"], L["do"], O["saved"], w.rope_base,
                               w.causal, dq=O["dq"], dk=O["dk"], dv=O["dv"], stream=s)

    def step():
        for L, O in zip(layers, outs):
            layer_step(L, O)

    for _ in range(a.warmup):
        flush_l2(1)
        step()
    torch.cuda.synchronize(dev)
    status = nea.nea_device_status()
    if status != nea.NEA_OK:
        raise SystemExit(f"device status after warm-up: {nea.nea_status_string(status)}")

    K = a.steps
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    # per-layer kernel-boundary events (7 per layer) of the profiling steps that
    # follow the timed ones: an event between two kernels would stop the next
    # kernel from starting while the previous one drains, so the timed steps
    # carry none
    ev_k = [[[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(w.layers)] for _ in range(K)]
    for evs in ev_k:
        for row in evs:
            for e in row:
                e.record(stream)  # materialise the CUDA events
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local, a.clocks_csv)
    barrier(world)
    torch.cuda.synchronize(dev)
    with clocks:
        # the sampler polls every 200 ms, far longer than the timed steps: a
        # block of identical steps of at least 1.2 s runs under it first, so
        # that the clock record spans kernel execution (reported apart as
        # `clock_window`; the value comes from the K steps after it only)
        window = None if a.profile else clock_window(step, flush_l2, stream, dev, 1.2)
        wall0 = time.perf_counter()
        for i in range(K):
            flush_l2(i)
            ev_step[i][0].record(stream)
            step()
            ev_step[i][1].record(stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
    barrier(world)
    # per-kernel durations: the same steps again with events between the kernels
    for i in range(K):
        flush_l2(i)
        for li, (L, O) in enumerate(zip(layers, outs)):
            nea.nea_set_profile_events(ev_k[i][li])
            layer_step(L, O)
        nea.nea_set_profile_events(None)
    torch.cuda.synchronize(dev)
    status = nea.nea_device_status()
    if status != nea.NEA_OK:
        raise SystemExit(f"device status after timing: {nea.nea_status_string(status)}")

    step_ms = [s.elapsed_time(e) for s, e in ev_step]
    total_ms = max_over_ranks(sum(step_ms), world)
    kern_ms = {k: 0.0 for k in KERNELS}
    for i in range(K):
        for li in range(w.layers):
            ev = ev_k[i][li]
            kern_ms["attn_fwd_prologue"] += ev[0].elapsed_time(ev[6])
            kern_ms["attn_fwd"] += ev[6].elapsed_time(ev[1])
            kern_ms["attn_bwd_prologue"] += ev[2].elapsed_time(ev[3])
            kern_ms["attn_bwd"] += ev[3].elapsed_time(ev[4])
    launches_per_kernel = K * w.layers

    flops_step = w.flops()
    value = flops_step * K * world / (total_ms * 1e-3) / 1e12
    tokens_s = w.tokens() * K * world / (total_ms * 1e-3)

    # roofline of the dominant kernel
    pk = peaks()
    dominant = max(kern_ms, key=kern_ms.get)
    per_launch_ms = kern_ms[dominant] / launches_per_kernel
    unit_flops = w.B * w.Hq * w.T * w.T * w.D * (1.0 if w.causal else 2.0)
    tf32 = measure_tf32_peak(dev) if (w.dtype == "f32" and not a.profile) else None
    if dominant in UNITS:
        achieved = UNITS[dominant] * unit_flops / (per_launch_ms * 1e-3) / 1e12
        if tf32:
            # float32 storage: the workload's precision class is TF32, so its
            # roofline is the TF32 peak measured in this run; the products are
            # executed as three bf16 products each, so the bf16 fraction is
            # given beside it
            roof = {"bound": "tensor", "achieved": achieved, "peak": tf32["tf32_tflops"], "unit": "TFLOP/s",
                    "frac": achieved / tf32["tf32_tflops"], "traffic": ncu_traffic(dominant, w.name),
                    "kernel": dominant,
                    "peak_kind": "tf32 dense burst (measured in this run: " + tf32["how"] + ")",
                    "frac_of_bf16_peak": achieved / pk["bf16_tflops"],
                    "bf16_peak_kind": f"bf16 dense burst ({pk['source']})"}
        else:
            roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": achieved / pk["bf16_tflops"], "traffic": ncu_traffic(dominant, w.name),
                    "kernel": dominant, "peak_kind": f"bf16 dense burst ({pk['source']})"}
    else:
        byts = prologue_bytes(w, dominant)
        achieved = byts / (per_launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": ncu_traffic(dominant, w.name), "kernel": dominant}
    kernels = {k: {"ms_per_launch": kern_ms[k] / launches_per_kernel,
                   "share": kern_ms[k] / max(sum(kern_ms.values()), 1e-12)} for k in KERNELS}
    for k, u in UNITS.items():
        kernels[k]["tflops"] = u * unit_flops / (kernels[k]["ms_per_launch"] * 1e-3) / 1e12

    # end to end through the public API with pinned host buffers
    e2e = None
    if not a.no_e2e:
        # End to end through the public API: every step copies its inputs from
        # pinned host memory and reads every output back.  Two buffer sets and
        # three streams overlap step i's compute with the copies of steps i+1
        # (in) and i-1 (out), as a pipelined caller would; the library calls
        # themselves stay on one stream (they share the device workspace).
        NB = 2
        host_in = [{n: t.cpu().pin_memory() for n, t in L.items()} for L in layers]
        dev_in = [[{n: torch.empty_like(t) for n, t in L.items()} for L in layers] for _ in range(NB)]
        dev_out = [[{"o": torch.empty_like(L["q"]), "lse": torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, device=dev),
                     "dq": torch.empty_like(L["q"]), "dk": torch.empty_like(L["k"]), "dv": torch.empty_like(L["v"]),
                     "saved": O["saved"]}
                    for L, O in zip(layers, outs)] for _ in range(NB)]
        host_out = [[{n: torch.empty(O[n].shape, dtype=O[n].dtype, pin_memory=True) for n in ("o", "dq", "dk", "dv")}
                     for O in dev_out[0]] for _ in range(NB)]
        h2d = sum(t.numel() * t.element_size() for H in host_in for t in H.values())
        d2h = sum(t.numel() * t.element_size() for H in host_out[0] for t in H.values())
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(NB)]
        ev_comp = [torch.cuda.Event() for _ in range(NB)]
        ev_out = [torch.cuda.Event() for _ in range(NB)]

        def e2e_step(i):
            bi = i % NB
            s_in.wait_event(ev_comp[bi])  # the compute that last read these inputs
            with torch.cuda.stream(s_in):
                for H, Dv in zip(host_in, dev_in[bi]):
                    for n in Dv:
                        Dv[n].copy_(H[n], non_blocking=True)
            ev_in[bi].record(s_in)
            stream.wait_event(ev_in[bi])
            stream.wait_event(ev_out[bi])  # the read-back that last used these outputs
            for Dv, O in zip(dev_in[bi], dev_out[bi]):
                layer_step(Dv, O, stream)
            ev_comp[bi].record(stream)
            s_out.wait_event(ev_comp[bi])
            with torch.cuda.stream(s_out):
                for O, HO in zip(dev_out[bi], host_out[bi]):
                    for n in HO:
                        HO[n].copy_(O[n], non_blocking=True)
            ev_out[bi].record(s_out)

        for i in range(a.warmup):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier(world)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(s_in)
        for i in range(K):
            e2e_step(i)
        s1.record(s_out)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(s0.elapsed_time(s1), world)
        e2e = {"value": flops_step * K * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "tokens_per_s": w.tokens() * K * world / (e2e_ms * 1e-3),
               "overlap": "copies of neighbouring steps overlap the compute (2 buffer sets, 3 streams)"}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        dt, fl, threads, desc = run_oracle_sample(w, min_seconds=10.0)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": dt}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": a.warmup,
            "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            # float32 storage: every product from bf16 high/low parts (hi*hi +
            # hi*lo + lo*hi, fp32 accumulation), finer than TF32
            "dtype": "bf16x3" if w.dtype == "f32" else "bf16", "data": "synthetic",
            "config": config_of(w, world),
            "tokens_per_s": tokens_s,
            "frac_of_bf16_peak": value / pk["bf16_tflops"],
            "tf32_peak": tf32,
            "frac_of_tf32_peak": (value / world / tf32["tf32_tflops"]) if tf32 else None,
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clocks.summary(), "clock_window": window, "gpu_launches": 4 * K * w.layers,
            "wall_s_timed": wall,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
