#!/usr/bin/env python
"""Benchmark of the rdFFT hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: one 256 x 4096 tensor of N(0,1) reals viewed as rows of p = 512 and of
p = 4096, bf16, transformed in place by rdFFT and then rdIFFT. The bench keeps a
pool of POOL distinct such tensors per view (256 MiB per view, twice the L2). One
ROUND is four sweeps over the pools: the forward of every p = 512 tensor, the
forward of every p = 4096 tensor, then the two inverses. Every tensor is therefore
last touched 768 MiB of traffic before its next transform, so every launch reads
HBM, and each tensor returns to its original values once a round. A sweep issues
its POOL launches round-robin on STREAMS CUDA streams and is replayed as one CUDA
graph. One STEP is R rounds, R fixed after warm-up so that a step takes about
STEP_TARGET_S seconds (so the clock sampler sees the timed region). The metric is
whole-job GB/s: algorithmic bytes (one read and one write of every element per
transform) over the device time of K steps, max over ranks. Rank r of N transforms
its own pools (weak scaling, no collective on the data path).

The timed region records a CUDA event before every sweep, so the per-kernel
breakdown and the roofline of the dominant kernel come from the same timed launches
as the headline. The JSON line also carries one large launch per kernel (the
asymptotic GB/s), an end-to-end figure through the public API with pinned host
buffers, the block-circulant layer at the D = 4096 workloads (tokens/s forward,
backward and both, GB/s, %HBM and %FP32 per kernel, and the float64 oracle timed on
the host beside it), SM clocks sampled during the timed region, and the float64 CPU
oracle timed on the rdFFT workload (rank 0, N = 1).

--impl reference times the float64 CPU oracle on the host cores instead (rank 0
only): each step is one whole 256 x 4096 tensor in each view, forward and inverse,
the same sample the cpu_baseline of our arm uses.
"""
from __future__ import annotations

import argparse
import contextlib
import hashlib
import json
import math
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
POOL = 128                  # tensors per view; 2 MiB each in bf16, 256 MiB per view
STREAMS = 8
SWEEPS = (("fwd", 512), ("fwd", 4096), ("inv", 512), ("inv", 4096))
STEP_TARGET_S = 0.06
FALLBACK_HBM_GBS = 6650.0
FP32_LANES_PER_SM = 128     # FP32 FMA lanes per B200 SM (4 sub-partitions x 32)
NOMINAL_SM_MHZ = 1965.0

ROWS_KERNEL_SOURCES = ("bulk_copy.cuh", "gen_twiddles.py", "packed_fft.cuh", "pdl.cuh", "rdfft_kernels.cu",
                       "rdfft_steps.cuh")

# ncu dram bytes per launch of the dominant kernel, with the hash of the kernel
# sources they were captured from (see profiles/); stale counters are reported null.
TRAFFIC_CAPTURE = {"sources_sha1": "8ce32fb741266a0465c22efae86bbb5aacc8ce3b",
                   "bytes_per_launch": {"bf16_p4096_inv": 3445299, "bf16_p4096_fwd": 3407856}}


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


@contextlib.contextmanager
def nvtx(name: str):
    """NVTX range around a phase of the bench (visible in nsys / ncu range filters)."""
    import torch
    torch.cuda.nvtx.range_push(name)
    try:
        yield
    finally:
        torch.cuda.nvtx.range_pop()


# ----------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def wait_first(self, timeout: float = 5.0):
        """Blocks until the first sample has arrived (nvidia-smi takes a moment to start)."""
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.01)

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
            if not (t0 <= ts <= t1 + 0.05):
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


def rounds_per_step(t_round: float, target: float = STEP_TARGET_S) -> int:
    """Rounds in one step so that a step takes about `target` seconds (at least 1)."""
    if not (t_round > 0):
        return 1
    return max(1, int(math.ceil(target / t_round)))


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


def fp32_peak_tflops(sm_mhz: float | None, n_sm: int) -> float:
    """Nominal FP32 CUDA-core peak: SMs x FP32 lanes x 2 flop (one FMA) x SM clock."""
    mhz = sm_mhz if sm_mhz else NOMINAL_SM_MHZ
    return n_sm * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12


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


@contextlib.contextmanager
def one_core():
    """Limits the oracle's BLAS to one thread inside the block."""
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        yield False
        return
    with threadpool_limits(limits=1, user_api="blas"):
        yield True


def oracle_tensor(seed: int):
    """Oracle forward + inverse of one whole 256 x 4096 tensor in each view (2048 rows
    of p = 512, 256 rows of p = 4096); returns (bytes, seconds).

    Bytes count like the GPU metric: bf16 storage, one read and one write of every
    element per transform."""
    import oracle
    from synthetic import sample
    nbytes = 0
    t = 0.0
    for p in PS:
        s = sample(seed, (ELEMS // p, p), "bf16")
        t0 = time.perf_counter()
        y = oracle.dft_packed(s.exact)
        oracle.idft_packed(y)
        t += time.perf_counter() - t0
        nbytes += 2 * 2 * ELEMS * 2
    return nbytes, t


def oracle_rdfft_rate(min_seconds: float, max_tensors: int, seed0: int = 2, single_core: bool = False):
    """GB/s of the oracle over distinct whole tensors until min_seconds of work."""
    b_, t_, n_ = 0, 0.0, 0
    ctx = one_core() if single_core else contextlib.nullcontext()
    with ctx:
        while (t_ < min_seconds or n_ == 0) and n_ < max_tensors:
            bb, tt = oracle_tensor(seed0 + n_)
            b_, t_, n_ = b_ + bb, t_ + tt, n_ + 1
    return b_ / t_ / 1e9, n_, t_


def oracle_layer_rate(B: int, D: int, p: int, seed: int, single_core: bool = False):
    """Tokens/s of the float64 oracle's forward + backward (dense circulant matrix) at
    (B, D, p) on bf16-valued inputs; returns (tokens/s, seconds)."""
    import oracle
    from synthetic import sample
    q = D // p
    c = sample(seed, (q, q, p), "f32", sigma=1.0 / math.sqrt(D)).exact
    x = sample(seed + 10, (B, D), "bf16").exact
    g = sample(seed + 20, (B, D), "bf16").exact
    ctx = one_core() if single_core else contextlib.nullcontext()
    with ctx:
        t0 = time.perf_counter()
        oracle.circ_forward(x, c)
        oracle.circ_backward(g, x, c)
        t = time.perf_counter() - t0
    return B / t, t


# --------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # the oracle keeps no state between calls, so warm-up steps only touch the code
    for w in range(min(max(args.warmup, 0), 1)):
        oracle_tensor(seed=2 + w)
    budget = 180.0
    total_b, total_t, steps = 0, 0.0, 0
    while steps < args.steps:
        b, t = oracle_tensor(seed=2 + steps)
        total_b += b
        total_t += t
        steps += 1
        if total_t > budget:
            break
    gbs = total_b / total_t / 1e9
    one, n1, t1 = oracle_rdfft_rate(0.0, 1, seed0=2, single_core=True)
    cores = cpu_threads()
    sample_desc = (f"float64 oracle (O(p^2) DFT by BLAS matmul), forward + inverse of one whole 256x4096 "
                   f"tensor in each view per step (2048 rows p=512 + 256 rows p=4096, bf16 values, "
                   f"distinct seeds); {'all' if steps >= args.steps else 'stopped after'} {steps} of "
                   f"{args.steps} requested steps (time budget {budget:.0f} s); 1 core: {one:.6f} GB/s "
                   f"on {n1} tensor(s)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 6), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total_t / steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "rdFFT fwd+inv of a 256x4096 N(0,1) tensor as rows of p=512 and p=4096 (bf16 values)",
                   "sample_per_step": "one whole tensor in each view"},
        "cpu_baseline": {"value": round(gbs, 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample_desc, "value_1core": round(one, 6)},
        "e2e": {"value": round(gbs, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- layer workloads
# (name, B, D, p, seed of c): the single layer at D = 4096, p = 128 (B = 256 and 1),
# the block-size extremes at B = 256, and one adapter of the LLaMA2-7B-shaped stack.
LAYER_CONFIGS = (
    ("d4096_p128_B256", 256, 4096, 128, 4),
    ("d4096_p128_B1", 1, 4096, 128, 4),
    ("d4096_p1024_B256", 256, 4096, 1024, 7),
    ("d4096_p4096_B256", 256, 4096, 4096, 8),
    ("d1024_p1024_B256", 256, 1024, 1024, 9),
    ("d4096_p512_B4096_adapter", 4096, 4096, 512, 300),
)


def fft_flops(p: int) -> float:
    """Nominal flops of one length-p real FFT (the usual 2.5 p log2 p)."""
    return 2.5 * p * math.log2(p)


def layer_work(B: int, D: int, p: int, s: int):
    """Algorithmic flops and bytes of the layer's kernels at (B, D, p), s bytes per
    activation element. The contraction of one token is q^2 packed products of p/2 - 1
    complex bins (8 flops) and two real bins (2 flops each)."""
    q = D // p
    contr = q * q * (8 * (p // 2 - 1) + 4)
    cb = 4 * q * q * p
    x_kernel = {"flops": B * (2 * q * fft_flops(p) + contr), "bytes": 2 * B * D * s + cb}
    gc_kernel = {"flops": B * (2 * q * fft_flops(p) + contr) + q * q * fft_flops(p), "bytes": 2 * B * D * s + cb}
    return {
        "fwd": x_kernel,
        "grad_x": x_kernel,
        "grad_c": gc_kernel,
        # backward as the method needs it: FFT(g), FFT(x), two contractions, IFFT(grad_x),
        # the q^2 IFFTs of grad_c; bytes g, x, c_hat, grad_x, grad_c
        "bwd": {"flops": B * (3 * q * fft_flops(p) + 2 * contr) + q * q * fft_flops(p),
                "bytes": 3 * B * D * s + 2 * cb},
    }


def run_layer_bench(rd, torch, dev, gen, hbm_peak, fp32_peak, n_sets_bytes=256 << 20):
    """Times the layer's calls on each workload. Activations rotate over enough sets
    that their total exceeds 2x the L2 (B = 1 excepted: a latency case), so each call
    reads its activations from HBM; c_hat is shared, as in training."""
    out = {}
    dt = torch.bfloat16
    s = 2
    dominant = None
    for name, B, D, p, seed in LAYER_CONFIGS:
        q = D // p
        per_set = 4 * B * D * s
        nsets = 1 if B == 1 else max(2, min(64, n_sets_bytes // per_set))
        c = torch.randn(q, q, p, device=dev, generator=gen) / D ** 0.5
        c_hat = torch.empty_like(c)
        gc = torch.empty_like(c)
        sets = []
        for _ in range(nsets):
            sets.append({"x": torch.randn(B, D, device=dev, generator=gen).to(dt),
                         "g": torch.randn(B, D, device=dev, generator=gen).to(dt),
                         "y": torch.empty(B, D, device=dev, dtype=dt),
                         "gx": torch.empty(B, D, device=dev, dtype=dt)})

        # the deterministic backward's workspace, allocated once outside the timed graphs
        ws = torch.empty(max(16, rd.circ_bwd_workspace_size(B, D, p, dt)), dtype=torch.uint8, device=dev)
        calls = {
            "prepare": lambda st: rd.circ_prepare(c, out=c_hat),
            "fwd": lambda st: rd.circ_fwd(st["x"], c_hat, p, y=st["y"]),
            "bwd": lambda st: rd.circ_bwd(st["g"], st["x"], c_hat, p, grad_x=st["gx"], grad_c=gc),
            "grad_x": lambda st: rd.circ_bwd(st["g"], st["x"], c_hat, p, grad_x=st["gx"], need_grad_c=False),
            "grad_c": lambda st: rd.circ_bwd(st["g"], st["x"], c_hat, p, grad_c=gc, need_grad_x=False),
            "bwd_deterministic": lambda st: rd.circ_bwd(st["g"], st["x"], c_hat, p, grad_x=st["gx"], grad_c=gc,
                                                        deterministic=True, workspace=ws),
        }

        def step_body(st):
            rd.circ_prepare(c, out=c_hat)
            rd.circ_fwd(st["x"], c_hat, p, y=st["y"])
            rd.circ_bwd(st["g"], st["x"], c_hat, p, grad_x=st["gx"], grad_c=gc)

        calls["fwd_bwd"] = step_body
        times = {}
        reps = 50 if B <= 256 else 10
        for key, fn in calls.items():
            g_ = graph_of(lambda fn=fn: [fn(st) for st in sets], torch)
            times[key] = time_graph(g_, max(3, reps // nsets), torch) / nsets
            del g_
        work = layer_work(B, D, p, s)
        res = {"B": B, "D": D, "p": p, "q": q,
               "activation_sets": nsets,
               "l2": ("activations rotate over %d sets (%.0f MiB), more than 2x L2" % (nsets, nsets * per_set / 2**20))
                     if nsets > 1 else "one set (latency case, activations L2-resident)",
               "fwd_tokens_s": round(B / times["fwd"], 1),
               "bwd_tokens_s": round(B / times["bwd"], 1),
               "fwd_bwd_tokens_s": round(B / times["fwd_bwd"], 1),
               "fwd_bwd_us": round(1e6 * times["fwd_bwd"], 2),
               "prepare_us": round(1e6 * times["prepare"], 2),
               # circ_bwd_deterministic: grad_c's token slices summed in order via a workspace
               "bwd_deterministic": {"us": round(1e6 * times["bwd_deterministic"], 2),
                                     "workspace_MiB": round(ws.numel() / 2**20, 2),
                                     "vs_bwd": round(times["bwd"] / times["bwd_deterministic"], 3)}}
        for key in ("fwd", "bwd", "grad_x", "grad_c"):
            t = times[key]
            w = work[key]
            res[key] = {"us": round(1e6 * t, 2),
                        "GB_s": round(w["bytes"] / t / 1e9, 1),
                        "pct_hbm": round(100 * w["bytes"] / t / 1e9 / hbm_peak, 1),
                        "TFLOP_s": round(w["flops"] / t / 1e12, 2),
                        "pct_fp32": round(100 * w["flops"] / t / 1e12 / fp32_peak, 1)}
        if B * D > 0 and p == 128 and D == 4096:
            # the same forward and grad_x with the contraction on the tensor cores
            tc = {}
            for key, fn in (("fwd", lambda st: rd.circ_fwd_tc(st["x"], c_hat, p, y=st["y"])),
                            ("grad_x", lambda st: rd.circ_bwd_x_tc(st["g"], c_hat, p, grad_x=st["gx"]))):
                g_ = graph_of(lambda fn=fn: [fn(st) for st in sets], torch)
                t = time_graph(g_, max(3, reps // nsets), torch) / nsets
                del g_
                tc[key] = {"us": round(1e6 * t, 2), "TFLOP_s": round(work[key]["flops"] / t / 1e12, 2),
                           "vs_cuda_core": round(times[key] / t, 3)}
            res["tensor_core_tcgen05"] = tc
        out[name] = res
        if name == "d4096_p128_B256":
            # the dominant layer call of the training step (forward, backward with both
            # gradients) at the D = 4096, p = 128, B = 256 workload
            kern = max(("fwd", "bwd"), key=lambda k: times[k])
            w = work[kern]
            dominant = {"bound": "alu", "achieved": round(w["flops"] / times[kern] / 1e12, 2),
                        "peak": round(fp32_peak, 1), "unit": "TFLOP/s",
                        "frac": round(w["flops"] / times[kern] / 1e12 / fp32_peak, 4), "traffic": None,
                        "kernel": {"fwd": "k_circ_x (forward)",
                                   "bwd": "k_circ_bwd_fused (grad_x and grad_c) + grad_c rdIFFT"}[kern],
                        "workload": "D=4096 p=128 B=256 bf16",
                        "peak_kind": "nominal FP32: SMs x 128 lanes x 2 flop x sampled SM clock",
                        "note": "achieved = algorithmic flops of the call (FFTs 2.5 p log2 p per row, packed "
                                "contraction 8 flops per complex bin) / its time, averaged over a CUDA graph "
                                "of calls on rotating activations"}
        del sets, c, c_hat, gc
    return out, dominant


def torch_fft_circulant(torch, x, c):
    """y = W x of the block-circulant layer the usual way (a measured reference, not the
    product): rfft of each block, per-bin complex contraction with rfft(c), irfft; fp32
    compute, the output cast back to the input's dtype."""
    B, D = x.shape
    q, _, p = c.shape
    xf = torch.fft.rfft(x.float().view(B, q, p), dim=-1)
    cf = torch.fft.rfft(c, dim=-1)
    yf = torch.einsum("ijk,bjk->bik", cf, xf)
    return torch.fft.irfft(yf, n=p, dim=-1).reshape(B, D).to(x.dtype)


def time_torch_fft_reference(torch, dev, gen, dt, B=256, D=4096, p=128, iters=50):
    """Forward + backward time of torch_fft_circulant at one workload, for context beside
    the layer's own numbers (eager launches, CUDA events, after warm-up)."""
    q = D // p
    c = (torch.randn(q, q, p, device=dev, generator=gen) / 64.0).requires_grad_(True)
    x = torch.randn(B, D, device=dev, generator=gen).to(dt).requires_grad_(True)
    g = torch.randn(B, D, device=dev, generator=gen).to(dt)

    def step():
        y = torch_fft_circulant(torch, x, c)
        y.backward(g)

    for _ in range(5):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        step()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / iters
    return {"fwd_bwd_us": round(us, 2), "tokens_s": round(B / (us * 1e-6), 1), "B": B, "D": D, "p": p,
            "note": "torch.fft rfft/irfft + complex einsum, fp32 compute, bf16 activations, autograd backward; "
                    "eager launches, context only"}


def run_adapter_stack(rd, torch, dev, gen, world, max_over_ranks_, barrier):
    """LLaMA2-7B-shaped stack: 32 layers x (q, v) adapters of D = 4096, p = 512, 4096
    tokens per rank per step; every adapter's forward then every backward, grad_c of all
    64 in one bucket all-reduced once per step (the layer's only exchange)."""
    nl, B, D, p = 32, 4096, 4096, 512
    q = D // p
    dt = torch.bfloat16
    from block_circulant_layers_b200.dp import GradCBucket
    xs = [torch.randn(B, D, device=dev, generator=gen).to(dt) for _ in range(nl)]
    gs = [torch.randn(B, D, device=dev, generator=gen).to(dt) for _ in range(2 * nl)]
    cs = [torch.randn(q, q, p, device=dev, generator=gen) / D ** 0.5 for _ in range(2 * nl)]
    chs = [torch.empty_like(c) for c in cs]
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
    res = {"tokens_s": round(world * B / st_t, 1), "ms_per_step": round(1e3 * st_t, 3),
           "tokens_per_rank": B, "adapters": 2 * nl,
           "grad_c_allreduce_bytes": int(bucket.flat.numel() * 4) if world > 1 else 0}
    del gst, xs, gs, cs, chs, gcs, ys, gxs, bucket
    return res


def layer_oracle_rates():
    """The float64 oracle's forward + backward on the layer workloads, all cores and
    one core: configs at B = 256 and B = 1 in full, the adapter on 64 tokens
    (extrapolated per token)."""
    res = {}
    cases = (("d4096_p128_B256", 256, 4096, 128, 4, "full"),
             ("d4096_p128_B1", 1, 4096, 128, 4, "full"),
             ("d4096_p1024_B256", 256, 4096, 1024, 7, "full"),
             ("d4096_p4096_B256", 256, 4096, 4096, 8, "full"),
             ("d1024_p1024_B256", 256, 1024, 1024, 9, "full"),
             ("d4096_p512_B4096_adapter", 64, 4096, 512, 300, "64 tokens of one adapter, extrapolated per token"))
    for name, B, D, p, seed, how in cases:
        r_all, t_all = oracle_layer_rate(B, D, p, seed)
        r_one, t_one = oracle_layer_rate(B, D, p, seed, single_core=True)
        res[name] = {"fwd_bwd_tokens_s": round(r_all, 2), "seconds": round(t_all, 3),
                     "fwd_bwd_tokens_s_1core": round(r_one, 2), "seconds_1core": round(t_one, 3),
                     "cores": cpu_threads(), "sample": how}
    # the 64-adapter stack from the per-token rate of one adapter (2 adapters x 64
    # tokens measure the same per-token cost)
    ad = res["d4096_p512_B4096_adapter"]
    res["llama2_7b_shape_64_adapters_tokens_s_extrapolated"] = round(ad["fwd_bwd_tokens_s"] / 64, 3)
    # config 1: the 64 x 16 fp32 round trip
    import oracle
    from synthetic import sample
    s = sample(1, (64, 16), "f32")
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < 0.2:
        oracle.idft_packed(oracle.dft_packed(s.exact))
        n += 1
    res["p16_64rows_roundtrip_rows_s"] = round(64 * n / (time.perf_counter() - t0), 1)
    return res


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
    # each view's pool is one contiguous buffer cut into POOL tensors of 256 x 4096
    flat = {p: torch.randn(POOL * ELEMS, device=dev, generator=gen).to(dt) for p in PS}
    pools = {p: [flat[p][i * ELEMS:(i + 1) * ELEMS].view(ELEMS // p, p) for i in range(POOL)] for p in PS}
    bytes_per_transform = 2 * ELEMS * 2             # read + write, bf16
    fns = {"fwd": rd.rdfft_fwd, "inv": rd.rdfft_inv}

    graphs = {}
    with nvtx("capture"):
        for d, p in SWEEPS:
            graphs[(d, p)] = graph_of(
                lambda d=d, p=p: fanout(lambda t: fns[d](t, p), pools[p], STREAMS, torch), torch)

    def run_round(evs=None):
        for d, p in SWEEPS:
            if evs is not None:
                ev = torch.cuda.Event(enable_timing=True)
                ev.record()
                evs.append(((d, p), ev))
            graphs[(d, p)].replay()

    with nvtx("warmup"):
        for _ in range(max(args.warmup, 3)):
            run_round()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(4):
            run_round()
        b.record()
        torch.cuda.synchronize()
    t_round = a.elapsed_time(b) / 1e3 / 4
    nrep = int(max_over_ranks_(float(rounds_per_step(t_round))))

    # ---- timed region: K steps of nrep rounds, barrier + synchronize on both sides
    evs = []
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(uuid) as clk:
        clk.wait_first()
        barrier()
        torch.cuda.synchronize()
        t_wall0 = time.time()
        with nvtx("timed"):
            start.record()
            for _ in range(args.steps):
                for _ in range(nrep):
                    run_round(evs)
            end.record()
            torch.cuda.synchronize()
        barrier()
        t_wall1 = time.time()
    elapsed = max_over_ranks_(start.elapsed_time(end) / 1e3)
    clocks = clk.summary(t_wall0, t_wall1)
    launches_per_round = len(SWEEPS) * POOL
    bytes_per_step = nrep * launches_per_round * bytes_per_transform
    value_gbs = world * bytes_per_step * args.steps / elapsed / 1e9

    # per-sweep device time inside the timed region (event before each sweep)
    sweep_t = {k: 0.0 for k in SWEEPS}
    marks = evs + [(None, end)]
    for (k, e0), (_, e1) in zip(marks[:-1], marks[1:]):
        sweep_t[k] += e0.elapsed_time(e1) / 1e3
    nsweeps = args.steps * nrep
    breakdown = {}
    for d, p in SWEEPS:
        t_launch = max_over_ranks_(sweep_t[(d, p)] / nsweeps / POOL)
        breakdown[f"bf16_p{p}_{d}"] = {
            "GB_s": round(bytes_per_transform / t_launch / 1e9, 1),
            "us_per_launch_amortized": round(1e6 * t_launch, 3),
            "pct_hbm": round(100 * bytes_per_transform / t_launch / 1e9 / hbm_peak, 1),
            "share": round(sweep_t[(d, p)] / sum(sweep_t.values()), 4),
        }
    del evs, marks

    # ---- roofline of the dominant kernel (largest share of the timed region)
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
                "note": "achieved = bytes per launch (2 x 256 x 4096 x 2 B) / its amortized launch time in the "
                        f"timed region (CUDA events around each sweep of {POOL} launches on {STREAMS} streams)"}

    # ---- one large launch per kernel: the whole 256 MiB pool of a view at once
    asym = {}
    with nvtx("large_launch"):
        for p in PS:
            ts = {"fwd": [], "inv": []}
            for _ in range(5):
                for d in ("fwd", "inv"):
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record()
                    fns[d](flat[p], p)
                    b.record()
                    torch.cuda.synchronize()
                    ts[d].append(a.elapsed_time(b) / 1e3)
            for d in ts:
                t = statistics.median(ts[d])
                asym[f"bf16_p{p}_{d}_256MiB"] = {
                    "GB_s": round(2 * flat[p].numel() * 2 / t / 1e9, 1),
                    "pct_hbm": round(100 * 2 * flat[p].numel() * 2 / t / 1e9 / hbm_peak, 1),
                    "us": round(1e6 * t, 1)}

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
    with nvtx("e2e"):
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
    del hosts, outs

    # ---- block-circulant layer at D = 4096 (bf16)
    fp32_peak = fp32_peak_tflops(clocks.get("sm_mhz"), props.multi_processor_count)
    with nvtx("layer"):
        layer, layer_roofline = run_layer_bench(rd, torch, dev, gen, hbm_peak, fp32_peak)
        layer["fp32_peak_tflops"] = round(fp32_peak, 1)
        layer["llama2_7b_shape_64_adapters_4096_tokens"] = run_adapter_stack(rd, torch, dev, gen, world,
                                                                             max_over_ranks_, barrier)

    # single-layer training-step peak memory at D = 4096 through the autograd module:
    # parameter, its gradient, activations and their gradients; with the in-place
    # spectrum (c_hat in c's own buffer) and with a temporary c_hat (the default)
    memory = {}
    for inplace in (True, False):
        for Bm in (1, 256):
            for pm in (128, 512, 1024, 4096):
                torch.cuda.synchronize()
                base = torch.cuda.memory_allocated(dev)
                torch.cuda.reset_peak_memory_stats(dev)
                lay = rd.BlockCirculantLinear(4096, pm, inplace_spectrum=inplace, device=dev, generator=gen)
                xm = torch.randn(Bm, 4096, device=dev, generator=gen).to(dt).requires_grad_(True)
                ym = lay(xm)
                ym.backward(torch.ones_like(ym))
                torch.cuda.synchronize()
                key = f"B{Bm}_p{pm}_MB" + ("_inplace_spectrum" if inplace else "")
                memory[key] = round((torch.cuda.max_memory_allocated(dev) - base) / 1e6, 3)
                del lay, xm, ym
    # the same training step for the usual FFT formulation, as a measured reference: torch
    # (cuFFT) rfft / irfft of each block, the per-bin contraction as a complex einsum, fp32
    # compute (cuFFT takes no bf16) with bf16 activations at the boundary; autograd keeps
    # what it needs for the backward
    for Bm in (1, 256):
        for pm in (128, 512, 1024, 4096):
            qm = 4096 // pm
            torch.cuda.synchronize()
            base = torch.cuda.memory_allocated(dev)
            torch.cuda.reset_peak_memory_stats(dev)
            cm = (torch.randn(qm, qm, pm, device=dev, generator=gen) / 64.0).requires_grad_(True)
            xm = torch.randn(Bm, 4096, device=dev, generator=gen).to(dt).requires_grad_(True)
            ym = torch_fft_circulant(torch, xm, cm)
            ym.backward(torch.ones_like(ym))
            torch.cuda.synchronize()
            memory[f"torch_fft_B{Bm}_p{pm}_MB"] = round((torch.cuda.max_memory_allocated(dev) - base) / 1e6, 3)
            del cm, xm, ym
    layer["single_layer_train_step_peak_memory_d4096_bf16"] = memory
    layer["torch_fft_reference_d4096_p128_B256"] = time_torch_fft_reference(torch, dev, gen, dt)

    # ---- 2-D rdFFT and the explicit-spectrum cast (beside the step, not in it)
    spectral = {}
    with nvtx("spectral"):
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

    # ---- CPU oracle (rank 0, N = 1 only): the rdFFT workload and the layer workloads
    cpu = None
    if world == 1 and rank == 0:
        gbs, n_, t_ = oracle_rdfft_rate(10.0, 64, seed0=2)
        one, n1, t1 = oracle_rdfft_rate(0.0, 1, seed0=2, single_core=True)
        cpu = {"value": round(gbs, 6), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"float64 oracle forward + inverse of {n_} distinct whole 256x4096 tensors in each view "
                         f"(2048 rows p=512, 256 rows p=4096 per tensor), {t_:.1f} s; the reference arm times the "
                         f"same per-tensor sample; 1 core: {one:.6f} GB/s on {n1} tensor",
               "value_1core": round(one, 6)}
        layer["oracle"] = layer_oracle_rates()

    line = {
        "metric": METRIC, "value": round(value_gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": round(1e3 * elapsed / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "rdFFT fwd+inv in place, 256x4096 N(0,1) bf16 tensor as rows of p=512 and p=4096",
                   "p": list(PS), "rows": [ELEMS // p for p in PS], "pool_tensors_per_view": POOL,
                   "streams": STREAMS, "rounds_per_step": nrep,
                   "step": "rounds of 4 sweeps (fwd p=512, fwd p=4096, inv p=512, inv p=4096) over the pools",
                   "l2": "inputs larger than L2: 256 MiB pool per view; a tensor's transforms are 768 MiB "
                         "of traffic apart",
                   "parallelism": f"dp{world} (independent rows per rank)"},
        "pct_hbm": round(100 * value_gbs / world / hbm_peak, 1),
        "roofline": roofline,
        "breakdown": breakdown,
        "large_launch": asym,
        "single_launch_cold_ms": lat,
        "layer": layer,
        "layer_roofline": layer_roofline,
        "spectral": spectral,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clocks,
        "gpu_launches": launches_per_round * nrep * args.steps,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs
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
    "circ_fwd_tc_d4096_p128_b256": ("circ", (256, 4096, 128, "fwd_tc")),
    "circ_bwd_d4096_p512_b4096": ("circ", (4096, 4096, 512, "bwd")),
    "circ_bwd_d4096_p128_b256": ("circ", (256, 4096, 128, "bwd")),
    "circ_step_d4096_p128_b1": ("circ_step", (1, 4096, 128)),
    "circ_step_d4096_p128_b256": ("circ_step", (256, 4096, 128)),
    "circ_step_d1024_p1024_b256": ("circ_step", (256, 1024, 1024)),
    "circ_bwd_det_d4096_p128_b256": ("circ", (256, 4096, 128, "bwd_det")),
    "circ_bwd_det_d4096_p512_b4096": ("circ", (4096, 4096, 512, "bwd_det")),
    "step_round": ("step_round", ()),
}


def run_profile_case(name: str) -> int:
    """Runs 4 launches of one kernel (the last ones are the ones to capture with ncu -s/-c).

    rows: a 160 MiB buffer (more than L2) of rows of p; rows_small: one 256 x 4096 tensor
    (the bench's per-launch size); circ: the layer kernel at (B, D, p); circ_step: the
    layer's prepare + forward + backward at (B, D, p), every kernel of it; step_round: the
    bench's pools, one warm-up round and one round of the timed step (4 x POOL launches
    each, issued eagerly on the same streams), for a launch list."""
    import torch
    import block_circulant_layers_b200 as rd
    kind, a = PROFILE_CASES[name]
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    if kind == "step_round":
        pools = {p: [torch.randn(ELEMS // p, p, device=dev, generator=gen).to(torch.bfloat16) for _ in range(POOL)]
                 for p in PS}
        fns = {"fwd": rd.rdfft_fwd, "inv": rd.rdfft_inv}
        for _ in range(2):
            for d, p in SWEEPS:
                fanout(lambda t, d=d, p=p: fns[d](t, p), pools[p], STREAMS, torch)
        torch.cuda.synchronize()
        print(f"profile case {name}: ok")
        return 0
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
        ws = torch.empty(max(16, rd.circ_bwd_workspace_size(B, D, p, torch.bfloat16)), dtype=torch.uint8, device=dev)
        for _ in range(4):
            if d == "fwd":
                rd.circ_fwd(x, ch, p, y=y)
            elif d == "fwd_tc":
                rd.circ_fwd_tc(x, ch, p, y=y)
            elif d == "bwd":
                rd.circ_bwd(g, x, ch, p, grad_x=y, grad_c=gc)
            elif d == "bwd_det":
                rd.circ_bwd(g, x, ch, p, grad_x=y, grad_c=gc, deterministic=True, workspace=ws)
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
