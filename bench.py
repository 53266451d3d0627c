#!/usr/bin/env python
"""Benchmark of the rdFFT hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one 256 x 4096 tensor of N(0,1) reals viewed as rows of p = 512 and of
p = 4096, bf16, in-place forward rdFFT then rdIFFT). One STEP transforms a pool of
POOL distinct such tensors in each view (forward then inverse, in place), issued
round-robin on STREAMS CUDA streams and replayed as one CUDA graph; the pool holds
256 MiB, twice the L2, so every launch reads HBM. The metric is whole-job GB/s:
algorithmic bytes (one read and one write of every element per transform) over the
device time of K steps, max over ranks. Rank r of N transforms its own pool (weak
scaling, no collective on the data path).

The same JSON line carries: a per-kernel breakdown, the roofline of the dominant
kernel, an end-to-end figure through the public API with pinned host buffers, the
block-circulant layer's tokens/s at D = 4096 (bf16), SM clocks sampled during the
timed region, and the float64 CPU oracle timed on a bounded sample (rank 0, N = 1).

--impl reference times the float64 CPU oracle on the host cores instead (rank 0
only), on a bounded slice of the same workload per step.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "rdFFT fwd/inv GB/s (% HBM peak); circulant layer tokens/s, D=4096 bf16"
PS = (512, 4096)
ELEMS = 256 * 4096          # reals per tensor
POOL = 64                   # tensors per view; 2 MiB each in bf16
STREAMS = 8
FALLBACK_HBM_GBS = 6650.0

ROWS_KERNEL_SOURCES = ("bulk_copy.cuh", "gen_twiddles.py", "packed_fft.cuh", "rdfft_kernels.cu", "rdfft_steps.cuh")

# ncu dram bytes per launch of the dominant kernel, with the hash of the kernel
# sources they were captured from (see profiles/); stale counters are reported null.
TRAFFIC_CAPTURE = {"sources_sha1": "7566fd1d3b92d0eeebfe681a79c3fb7205f22638",
                   "bytes_per_launch": {"bf16_p4096_inv": 3444835, "bf16_p4096_fwd": 3405674}}


def kernel_sources_sha1() -> str:
    """Hash of the sources of the rows kernel (the bench step's only kernel)."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "block_circulant_layers_b200", "csrc")
    for name in ROWS_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        sm, mx, reasons = [], [], set()
        for ts, line in self.lines:
            if not (t0 <= ts <= t1 + 0.15):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------- helpers
def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Seed of a rank's pool: every rank transforms its own distinct data."""
    return 1000 + rank


def graph_of(fn, torch):
    """Capture fn() (which issues work on the current stream) into a CUDA graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                               # warm-up outside capture (sets smem attributes)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(g, reps, torch):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record()
    for _ in range(reps):
        g.replay()
    end.record()
    torch.cuda.synchronize()
    return start.elapsed_time(end) / 1e3 / reps     # seconds per replay


def fanout(fn_per_item, items, nstreams, torch):
    """Issue fn_per_item(x) for every item round-robin on nstreams side streams."""
    cur = torch.cuda.current_stream()
    sts = [torch.cuda.Stream() for _ in range(nstreams)]
    for st in sts:
        st.wait_stream(cur)
    for i, it in enumerate(items):
        with torch.cuda.stream(sts[i % nstreams]):
            fn_per_item(it)
    for st in sts:
        cur.wait_stream(st)


# ---------------------------------------------------------------- oracle (CPU)
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_slice(rows512: int, rows4096: int, seed: int = 2):
    """Oracle forward + inverse on a slice of the workload; returns (bytes, seconds).

    Bytes count like the GPU metric: bf16 storage, one read and one write of every
    element per transform."""
    import oracle
    from synthetic import sample
    nbytes = 0
    t = 0.0
    for p, rows in ((512, rows512), (4096, rows4096)):
        if rows <= 0:
            continue
        s = sample(seed, (rows, p), "bf16")
        t0 = time.perf_counter()
        y = oracle.dft_packed(s.exact)
        oracle.idft_packed(y)
        t += time.perf_counter() - t0
        nbytes += 2 * 2 * rows * p * 2
    return nbytes, t


# --------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # one step: 1/8 of the 256 x 4096 tensor in each view (256 rows of p = 512 and
    # 32 rows of p = 4096, equal bytes), forward and inverse
    r512, r4096 = 256, 32
    for _ in range(max(args.warmup, 0)):
        oracle_slice(r512, r4096, seed=3)
        break                                       # the oracle has no warm-up state
    budget = 180.0
    total_b, total_t, steps = 0, 0.0, 0
    while steps < args.steps:
        b, t = oracle_slice(r512, r4096, seed=3)
        total_b += b
        total_t += t
        steps += 1
        if total_t > budget:
            break
    gbs = total_b / total_t / 1e9
    cores = cpu_threads()
    sample_desc = (f"float64 oracle (O(p^2) DFT by BLAS matmul) on {steps} step(s) of 256 rows at p=512 + "
                   f"32 rows at p=4096, forward and inverse, bf16 values; "
                   f"{'all' if steps >= args.steps else 'stopped after'} {steps} of {args.steps} requested steps "
                   f"(time budget {budget:.0f} s)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 6), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total_t / steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "rdFFT fwd+inv of a 256x4096 N(0,1) tensor as rows of p=512 and p=4096 (bf16 values)",
                   "slice_per_step": "256 rows p=512 + 32 rows p=4096"},
        "cpu_baseline": {"value": round(gbs, 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample_desc},
        "e2e": {"value": round(gbs, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    import block_circulant_layers_b200 as rd

    hbm_peak, peak_kind = measured_peaks()
    props = torch.cuda.get_device_properties(dev)
    uuid = None
    try:
        uuid = "GPU-" + str(props.uuid)
    except Exception:
        pass

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks_(x: float) -> float:
        return max_over_ranks(x, world, dev)

    gen = torch.Generator(device=dev)
    gen.manual_seed(rank_seed(rank))
    dt = torch.bfloat16
    pools = {p: [torch.randn(ELEMS // p, p, device=dev, generator=gen).to(dt) for _ in range(POOL)] for p in PS}
    bytes_per_transform = 2 * ELEMS * 2             # read + write, bf16

    def step():
        for p in PS:
            fanout(lambda t, p=p: (rd.rdfft_fwd(t, p), rd.rdfft_inv(t, p)), pools[p], STREAMS, torch)

    launches_per_step = len(PS) * POOL * 2
    bytes_per_step = launches_per_step * bytes_per_transform
    g = graph_of(step, torch)
    for _ in range(max(args.warmup, 3)):
        g.replay()
    torch.cuda.synchronize()

    # ---- timed region: K steps, barrier + synchronize on both sides
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(uuid) as clk:
        barrier()
        torch.cuda.synchronize()
        t_wall0 = time.time()
        start.record()
        for _ in range(args.steps):
            g.replay()
        end.record()
        torch.cuda.synchronize()
        barrier()
        t_wall1 = time.time()
    elapsed = max_over_ranks_(start.elapsed_time(end) / 1e3)
    clocks = clk.summary(t_wall0, t_wall1)
    value_gbs = world * bytes_per_step * args.steps / elapsed / 1e9

    # ---- breakdown: each (p, direction) alone over its pool, same streams
    def refill(p):
        for t in pools[p]:
            t.copy_(torch.randn(t.shape, device=dev, generator=gen).to(dt))

    breakdown = {}
    for p in PS:
        for name, fn in (("fwd", rd.rdfft_fwd), ("inv", rd.rdfft_inv)):
            refill(p)
            g1 = graph_of(lambda fn=fn, p=p: fanout(lambda t: fn(t, p), pools[p], STREAMS, torch), torch)
            t1 = time_graph(g1, 5, torch)       # few replays: a lone direction rescales the data
            breakdown[f"bf16_p{p}_{name}"] = {
                "GB_s": round(POOL * bytes_per_transform / t1 / 1e9, 1),
                "us_per_launch_amortized": round(1e6 * t1 / POOL, 3),
                "pct_hbm": round(100 * POOL * bytes_per_transform / t1 / 1e9 / hbm_peak, 1),
            }
            del g1
        refill(p)

    # single-launch latency with a cold L2 (context for the pages' per-call ms figures);
    # forward and inverse alternate so the data keep their scale
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    lat = {}
    for p in PS:
        t = pools[p][0]
        samples = {"fwd": [], "inv": []}
        for _ in range(10):
            for name, fn in (("fwd", rd.rdfft_fwd), ("inv", rd.rdfft_inv)):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record()
                fn(t, p)
                b.record()
                torch.cuda.synchronize()
                samples[name].append(a.elapsed_time(b))
        for name in samples:
            lat[f"bf16_p{p}_{name}_ms"] = round(statistics.median(samples[name]), 4)
    del flush

    # ---- roofline of the dominant kernel (largest share of the step)
    dom_key = max(breakdown, key=lambda k: breakdown[k]["us_per_launch_amortized"])
    dom = breakdown[dom_key]
    achieved = bytes_per_transform / (dom["us_per_launch_amortized"] * 1e-6) / 1e9
    srcs = kernel_sources_sha1()
    traffic = None
    if TRAFFIC_CAPTURE["sources_sha1"] == srcs:
        traffic = TRAFFIC_CAPTURE["bytes_per_launch"].get(dom_key)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "traffic": traffic, "kernel": dom_key,
                "peak_kind": peak_kind,
                "note": "achieved = bytes per launch (2 x 256 x 4096 x 2 B) / amortized launch time of "
                        f"{POOL} launches on {STREAMS} streams"}

    # ---- end to end through the public API with pinned host buffers
    e2e_pool = 8
    hosts = {p: [pools[p][i].cpu().pin_memory() for i in range(e2e_pool)] for p in PS}
    outs = {p: [torch.empty_like(h, device="cpu").pin_memory() for h in hosts[p]] for p in PS}

    def e2e_one(item):
        p, i = item
        d = pools[p][i]
        d.copy_(hosts[p][i], non_blocking=True)
        rd.rdfft_fwd(d, p)
        rd.rdfft_inv(d, p)
        outs[p][i].copy_(d, non_blocking=True)

    e2e_items = [(p, i) for i in range(e2e_pool) for p in PS]
    e2e_streams = 4

    def e2e_step():
        # tensor k on stream k % 4: one tensor's host-to-device copy, another's
        # transforms and a third's device-to-host copy run at the same time
        fanout(e2e_one, e2e_items, e2e_streams, torch)

    e2e_step()
    torch.cuda.synchronize()
    e2e_reps = max(3, min(args.steps, 50))
    barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(e2e_reps):
        e2e_step()
    b.record()
    torch.cuda.synchronize()
    barrier()
    e2e_t = max_over_ranks_(a.elapsed_time(b) / 1e3 / e2e_reps)
    e2e_bytes = len(PS) * e2e_pool * 2 * bytes_per_transform
    h2d = len(PS) * e2e_pool * ELEMS * 2
    e2e = {"value": round(world * e2e_bytes / e2e_t / 1e9, 3), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h2d,
           "note": f"{e2e_pool} tensors per view per step, each: pinned H2D copy, rdfft_fwd, rdfft_inv, D2H copy; "
                   f"tensors round-robin on {e2e_streams} streams so copies in both directions overlap the transforms"}

    # ---- block-circulant layer tokens/s at D = 4096 (bf16)
    layer = {}

    def layer_rate(B, D, p, reps):
        q = D // p
        c = torch.randn(q, q, p, device=dev, generator=gen) / D ** 0.5
        c_hat = torch.empty_like(c)
        x = torch.randn(B, D, device=dev, generator=gen).to(dt)
        gup = torch.randn(B, D, device=dev, generator=gen).to(dt)
        y = torch.empty_like(x)
        gx = torch.empty_like(x)
        gc = torch.empty_like(c)

        def body():
            rd.circ_prepare(c, out=c_hat)
            rd.circ_fwd(x, c_hat, p, y=y)
            rd.circ_bwd(gup, x, c_hat, p, grad_x=gx, grad_c=gc)

        gl = graph_of(body, torch)
        tt = time_graph(gl, reps, torch)
        return B / tt

    layer["d4096_p128_B256_fwd_bwd_tokens_s"] = round(layer_rate(256, 4096, 128, 50), 1)
    # B = 1 (one token): latency of prepare + forward + backward
    layer["d4096_p128_B1_fwd_bwd_us"] = round(1e6 / layer_rate(1, 4096, 128, 200), 2)
    layer["d4096_p512_B4096_fwd_bwd_tokens_s_per_adapter"] = round(layer_rate(4096, 4096, 512, 20), 1)
    # block-size extremes, B = 256: one whole-row transform per block (q = 1) and q = 4
    layer["d4096_p1024_B256_fwd_bwd_tokens_s"] = round(layer_rate(256, 4096, 1024, 50), 1)
    layer["d4096_p4096_B256_fwd_bwd_tokens_s"] = round(layer_rate(256, 4096, 4096, 50), 1)
    layer["d1024_p1024_B256_fwd_bwd_tokens_s"] = round(layer_rate(256, 1024, 1024, 50), 1)

    # LLaMA2-7B-shaped adapter stack: 32 layers x (q, v) adapters, 4096 tokens per step
    nl, B, D, p = 32, 4096, 4096, 512
    q = D // p
    from block_circulant_layers_b200.dp import GradCBucket
    xs = [torch.randn(B, D, device=dev, generator=gen).to(dt) for _ in range(nl)]
    gs = [torch.randn(B, D, device=dev, generator=gen).to(dt) for _ in range(2 * nl)]
    cs = [torch.randn(q, q, p, device=dev, generator=gen) / D ** 0.5 for _ in range(2 * nl)]
    chs = [torch.empty_like(c) for c in cs]
    # the 64 grad_c live in one flat bucket: with N ranks (4096 tokens each) the step
    # ends with one all-reduce of it, the layer's only exchange
    bucket = GradCBucket([c.shape for c in cs], device=dev)
    gcs = bucket.views
    ys = [torch.empty_like(xs[0]) for _ in range(2)]
    gxs = [torch.empty_like(xs[0]) for _ in range(2)]

    def stack_step():
        for a_ in range(2 * nl):
            rd.circ_prepare(cs[a_], out=chs[a_])
            rd.circ_fwd(xs[a_ // 2], chs[a_], p, y=ys[a_ % 2])
        for a_ in reversed(range(2 * nl)):
            rd.circ_bwd(gs[a_], xs[a_ // 2], chs[a_], p, grad_x=gxs[a_ % 2], grad_c=gcs[a_])

    gst = graph_of(stack_step, torch)
    reps = 5
    for _ in range(2):
        gst.replay()
        bucket.allreduce(world_size=world)
    torch.cuda.synchronize()
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        gst.replay()
        bucket.allreduce(world_size=world)
    b.record()
    torch.cuda.synchronize()
    barrier()
    st_t = max_over_ranks_(a.elapsed_time(b) / 1e3 / reps)
    layer["llama2_7b_shape_64_adapters_4096_tokens_per_step_tokens_s"] = round(world * B / st_t, 1)
    layer["llama2_7b_shape_ms_per_step"] = round(1e3 * st_t, 3)
    layer["llama2_7b_shape_tokens_per_rank"] = B
    layer["llama2_7b_shape_grad_c_allreduce_bytes"] = int(bucket.flat.numel() * 4) if world > 1 else 0
    del gst

    # single-layer training-step peak memory at D = 4096 through the autograd module
    # (in-place spectrum): parameter, its gradient, activations and their gradients
    del xs, gs, cs, chs, gcs, ys, gxs
    memory = {}
    for Bm in (1, 256):
        for pm in (128, 512, 1024, 4096):
            torch.cuda.synchronize()
            base = torch.cuda.memory_allocated(dev)
            torch.cuda.reset_peak_memory_stats(dev)
            lay = rd.BlockCirculantLinear(4096, pm, device=dev, generator=gen)
            xm = torch.randn(Bm, 4096, device=dev, generator=gen).to(dt).requires_grad_(True)
            ym = lay(xm)
            ym.backward(torch.ones_like(ym))
            torch.cuda.synchronize()
            memory[f"B{Bm}_p{pm}_MB"] = round((torch.cuda.max_memory_allocated(dev) - base) / 1e6, 3)
            del lay, xm, ym
    layer["single_layer_train_step_peak_memory_d4096_bf16"] = memory

    # ---- 2-D rdFFT and the explicit-spectrum cast (beside the step, not in it)
    spectral = {}
    for (n2, R2, C2, dt2, name2) in ((8, 4096, 4096, torch.bfloat16, "bf16_8x4096x4096"),
                                     (64, 1024, 1024, torch.float32, "f32_64x1024x1024")):
        imgs = torch.randn(n2, R2, C2, device=dev, generator=gen).to(dt2)
        nbytes = imgs.numel() * imgs.element_size()
        g2 = graph_of(lambda: (rd.rdfft2_fwd(imgs), rd.rdfft2_inv(imgs)), torch)
        t2 = time_graph(g2, 10, torch)
        gf = graph_of(lambda: rd.rdfft2_fwd(imgs), torch)
        tf = time_graph(gf, 1, torch)                   # one forward (rescales the data once)
        spectral[f"rdfft2_{name2}"] = {
            "fwd_inv_ms": round(1e3 * t2, 3), "fwd_ms": round(1e3 * tf, 3),
            "effective_GBs": round(2 * 2 * nbytes / t2 / 1e9, 1),     # read + write once per transform
            "moved_GBs": round(2 * 4 * nbytes / t2 / 1e9, 1),         # row half + column half, each r + w
            "note": "effective = minimum in-place traffic (read + write once) / time; the row and "
                    "column kernels each read and write the data once"}
        del imgs, g2, gf
    rows_c = ELEMS // 512 * 64                      # 128 MiB packed + 128 MiB complex: above L2
    packed = torch.randn(rows_c, 512, device=dev, generator=gen).to(dt)
    cplx = torch.empty(rows_c, 257, 2, device=dev, dtype=dt)
    gc2 = graph_of(lambda: rd.rdfft_to_complex(packed, 512, out=cplx), torch)
    tc = time_graph(gc2, 20, torch)
    spectral["to_complex_bf16_p512_GBs"] = round((packed.numel() + cplx.numel()) * 2 / tc / 1e9, 1)
    gc3 = graph_of(lambda: rd.rdfft_from_complex(cplx, out=packed), torch)
    tc3 = time_graph(gc3, 20, torch)
    spectral["from_complex_bf16_p512_GBs"] = round((packed.numel() + cplx.numel()) * 2 / tc3 / 1e9, 1)
    del packed, cplx, gc2, gc3

    # ---- CPU oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if world == 1 and rank == 0:
        b_, t_, n_ = 0, 0.0, 0
        while t_ < 10.0 and n_ < 64:                      # about 10 s of CPU work
            bb, tt = oracle_slice(2048, 256, seed=2 + n_)  # one whole 256 x 4096 tensor in each view
            b_, t_, n_ = b_ + bb, t_ + tt, n_ + 1
        cpu = {"value": round(b_ / t_ / 1e9, 6), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"float64 oracle forward + inverse of {n_} distinct 256x4096 tensors in each view "
                         f"(2048 rows p=512, 256 rows p=4096 per tensor), {t_:.1f} s"}

    line = {
        "metric": METRIC, "value": round(value_gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": round(1e3 * elapsed / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "rdFFT fwd+inv in place, 256x4096 N(0,1) bf16 tensor as rows of p=512 and p=4096",
                   "p": list(PS), "rows": [ELEMS // p for p in PS], "pool_tensors_per_view": POOL,
                   "streams": STREAMS, "l2": "inputs larger than L2 (256 MiB pool per rank)",
                   "parallelism": f"dp{world} (independent rows per rank)"},
        "pct_hbm": round(100 * value_gbs / world / hbm_peak, 1),
        "roofline": roofline,
        "breakdown": breakdown,
        "single_launch_cold_ms": lat,
        "layer": layer,
        "spectral": spectral,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        dist.destroy_process_group()
    return 0


PROFILE_CASES = {
    # name: (kind, args) -- one kernel on a buffer larger than L2, for ncu captures
    "rdfft_bf16_512_fwd": ("rows", (512, "bf16", "fwd")),
    "rdfft_bf16_512_inv": ("rows", (512, "bf16", "inv")),
    "rdfft_bf16_1024_fwd": ("rows", (1024, "bf16", "fwd")),
    "rdfft_bf16_2048_fwd": ("rows", (2048, "bf16", "fwd")),
    "rdfft_bf16_4096_fwd": ("rows", (4096, "bf16", "fwd")),
    "rdfft_bf16_4096_inv": ("rows", (4096, "bf16", "inv")),
    "rdfft_f32_4096_fwd": ("rows", (4096, "f32", "fwd")),
    "rdfft_bf16_4096_inv_config": ("rows_small", (4096, "bf16", "inv")),
    "rdfft2_bf16_4096_fwd": ("image", (4096, 4096, "bf16", "fwd")),
    "rdfft2_bf16_4096_inv": ("image", (4096, 4096, "bf16", "inv")),
    "circ_fwd_d4096_p512_b4096": ("circ", (4096, 4096, 512, "fwd")),
    "circ_bwdx_d4096_p512_b4096": ("circ", (4096, 4096, 512, "bwdx")),
    "circ_bwdc_d4096_p512_b4096": ("circ", (4096, 4096, 512, "bwdc")),
    "circ_fwd_d4096_p128_b256": ("circ", (256, 4096, 128, "fwd")),
    "circ_bwdc_d4096_p128_b256": ("circ", (256, 4096, 128, "bwdc")),
    "circ_step_d4096_p128_b1": ("circ_step", (1, 4096, 128)),
}


def run_profile_case(name: str) -> int:
    """Runs 4 launches of one kernel (the last ones are the ones to capture with ncu -s/-c).

    rows: a 160 MiB buffer (more than L2) of rows of p; rows_small: one 256 x 4096 tensor
    (the bench's per-launch size); circ: the layer kernel at (B, D, p); circ_step: the
    layer's prepare + forward + backward at (B, D, p), every kernel of it."""
    import torch
    import block_circulant_layers_b200 as rd
    kind, a = PROFILE_CASES[name]
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    if kind == "image":
        R, C, dts, d = a
        dt = torch.bfloat16 if dts == "bf16" else torch.float32
        x = torch.randn(160 * 1024 * 1024 // (R * C * 2), R, C, device=dev, generator=gen).to(dt)
        fn, undo = (rd.rdfft2_fwd, rd.rdfft2_inv) if d == "fwd" else (rd.rdfft2_inv, rd.rdfft2_fwd)
        for _ in range(4):
            fn(x)
            undo(x)
    elif kind in ("rows", "rows_small"):
        p, dts, d = a
        dt = torch.bfloat16 if dts == "bf16" else torch.float32
        esz = 2 if dts == "bf16" else 4
        rows = (160 * 1024 * 1024) // (p * esz) if kind == "rows" else ELEMS // p
        x = torch.randn(rows, p, device=dev, generator=gen).to(dt)
        fn, undo = (rd.rdfft_fwd, rd.rdfft_inv) if d == "fwd" else (rd.rdfft_inv, rd.rdfft_fwd)
        for _ in range(4):
            fn(x, p)
            undo(x, p)
    elif kind == "circ_step":
        B, D, p = a
        q = D // p
        c = torch.randn(q, q, p, device=dev, generator=gen) / D ** 0.5
        ch = torch.empty_like(c)
        x = torch.randn(B, D, device=dev, generator=gen).to(torch.bfloat16)
        g = torch.randn(B, D, device=dev, generator=gen).to(torch.bfloat16)
        y = torch.empty_like(x)
        gx = torch.empty_like(x)
        gc = torch.empty_like(c)
        for _ in range(4):
            rd.circ_prepare(c, out=ch)
            rd.circ_fwd(x, ch, p, y=y)
            rd.circ_bwd(g, x, ch, p, grad_x=gx, grad_c=gc)
    else:
        B, D, p, d = a
        q = D // p
        c = torch.randn(q, q, p, device=dev, generator=gen) / D ** 0.5
        ch = rd.circ_prepare(c)
        x = torch.randn(B, D, device=dev, generator=gen).to(torch.bfloat16)
        g = torch.randn(B, D, device=dev, generator=gen).to(torch.bfloat16)
        y = torch.empty_like(x)
        gc = torch.empty_like(c)
        for _ in range(4):
            if d == "fwd":
                rd.circ_fwd(x, ch, p, y=y)
            elif d == "bwdx":
                rd.circ_bwd(g, x, ch, p, grad_x=y, need_grad_c=False)
            else:
                rd.circ_bwd(g, x, ch, p, grad_c=gc, need_grad_x=False)
    torch.cuda.synchronize()
    print(f"profile case {name}: ok")
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--profile", choices=sorted(PROFILE_CASES), default=None,
                    help="run one kernel case for an ncu capture instead of the benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    args = ap.parse_args(argv)
    if args.profile:
        return run_profile_case(args.profile)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
