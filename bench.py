"""Benchmark of the PowerSGD compression step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 3] [--impl ours|reference]

One step = the whole hot path over one batch of synthetic gradients held in
HBM: psgd_step (error-feedback add, P = MQ, worker mean, orthogonalisation,
Q = M^T P_hat, worker mean, residual), plus, where the workload has them,
the uncompressed mean of the 1-D tensors and the post-compression momentum
update, all through the C ABI.  The default workload is the transformer-block
set (24 x (4096x12288, 4096x4096, 16384x4096, 4096x16384), bf16 gradients,
fp32 error memory, rank 4, 4 workers: 19.3 G worker elements per step), the
largest that fits one GPU.  Metric: gradient elements compressed per second
(W * sum(m*n) per step), whole job.  On one GPU the W workers are replica
buffers and the worker means are on-device sums.  With N GPUs (torchrun,
NCCL) every rank holds W workers and runs the distributed step: the P and Q
partial sums (and the 1-D gradients) are all-reduced between the library's
three calls, so the job has N * W workers (weak scaling) and value = N *
elements / max over ranks of the device time.

Rank 0 prints one JSON line: the roofline of the dominant kernel (HBM; plus
the products' compute side at ranks 16 and 32), the end-to-end figure
through host buffers (psgd_step_host_flat), the clocks seen from the
warm-up to the end of the timed region, the compression ratio and payload,
on one GPU the float64 oracle timed on the host cores, and "workloads": the
other workloads' eager steps (the LSTM set, the 8192^2 and 256 x 1024^2
rank sweeps with the subspace error of the latter, the ResNet-18 set), each
timed the same way.  --impl reference times the oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from synth import GradientSource, get as get_workload, pack_offsets  # noqa: E402

METRIC = "gradient elements compressed/sec"
UNIT = "elements/s"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def compute_roofline(elements: int, rank: int, pass_a_ms: float, pass_b_ms: float, sm_mhz: float,
                     bf16_tflops: float, sum_first: bool = False, workers: int = 1) -> dict:
    """Compute side of the first two passes (the two products): their
    algorithmic flops (2 r per worker element each; 2 r per matrix element
    for the first pass with sum-first) per second of the two passes, against
    the fp32 CUDA-core ceiling (148 SMs x 128 FMA lanes x 2 flop x SM clock)
    and the tf32 tensor-core ceiling (the measured bf16 GEMM peak x the
    nominal tf32 / bf16 ratio 1.1 / 2.25).  The tensor-core passes run three
    split products per term, which this does not count."""
    flops = 2 * rank * elements * (1.0 / workers if sum_first else 1.0) + 2 * rank * elements
    sec = (pass_a_ms + pass_b_ms) * 1e-3
    achieved = flops / sec / 1e12 if sec > 0 else 0.0
    fp32_peak = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12
    tf32_peak = bf16_tflops * 1.1 / 2.25
    return {"unit": "TFLOP/s", "achieved": round(achieved, 2),
            "fp32_cuda_core_peak": round(fp32_peak, 1), "fp32_frac": round(achieved / fp32_peak, 4),
            "tf32_tensor_peak": round(tf32_peak, 1), "tf32_frac": round(achieved / tf32_peak, 4),
            "note": "products of passes A and B only; ranks 16 and 32 run them on the tf32 tensor cores "
                    "with three split products per term (pass A mma.sync; pass B tcgen05 with A in tensor "
                    "memory on 16-byte rows), ranks <= 8 on the CUDA cores"}


def _code_tokens(text: str) -> str:
    """C++/CUDA source without comments and with whitespace collapsed: what
    the compiler sees, so that editing a comment keeps the hash."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":                       # string or character literal
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def _kernel_source_hash(csrc: str = None) -> str:
    """Hash of the CUDA sources' code (comments and layout ignored)."""
    h = hashlib.sha256()
    csrc = csrc or os.path.join(ROOT, "rank_gradient_compression_02_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_code_tokens(f.read()).encode())
    return h.hexdigest()[:16]


def _traffic_record(workload: str, mode: str):
    """DRAM bytes per launch of the first pass from a committed ncu summary,
    valid only for the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    key = f"{workload}/{mode}"
    r = rec.get(key)
    if not r or r.get("kernel_hash") != _kernel_source_hash():
        return None
    return r.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self, interval_ms: int = 50, wait_first_s: float = 5.0):
        """Start sampling; waits (up to wait_first_s) for the first sample so
        that a short timed region is still covered."""
        try:
            import tempfile
            self.path = os.path.join(tempfile.gettempdir(), f"clocks_bench_{os.getpid()}.csv")
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(interval_ms)], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < wait_first_s and self.proc.poll() is None:
            try:
                if os.path.getsize(self.path) > 0:
                    break
            except OSError:
                pass
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() in ("active", "1", "yes"):
                        reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def max_over_ranks(ms: float, world: int, device) -> float:
    """Max of a per-rank time over all ranks (the job's time)."""
    if world <= 1:
        return ms
    import torch.distributed as dist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(elements_per_replica: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank runs one replica of the workload."""
    return elements_per_replica * world / (ms_per_step * 1e-3)


# --------------------------------------------------------------------------
# workload buffers

class Buffers:
    def __init__(self, wl, rank, device, seed=1234):
        self.wl = wl
        self.rank = rank
        W, L = wl.workers, len(wl.layers)
        gdt = torch.bfloat16 if wl.grad_dtype == "bf16" else torch.float32
        align = 64  # elements: 256 B for fp32, 128 B for bf16
        self.offs = pack_offsets(wl.layers, align)
        total = self.offs[-1]
        self.G_flat = [torch.empty(total, dtype=gdt, device=device) for _ in range(W)]
        self.E_flat = [torch.zeros(total, dtype=torch.float32, device=device) for _ in range(W)]
        self.G = [[self.G_flat[w][self.offs[l]:self.offs[l] + m * n].view(m, n) for l, (m, n) in enumerate(wl.layers)]
                  for w in range(W)]
        self.E = [[self.E_flat[w][self.offs[l]:self.offs[l] + m * n].view(m, n) for l, (m, n) in enumerate(wl.layers)]
                  for w in range(W)]
        src = GradientSource(wl, seed)
        self.src = src
        self.device = device
        src.fill(0, self.G)
        self.set_rank(rank)
        self.params = self.mom = None
        if wl.momentum:
            self.params = [torch.zeros(m, n, device=device) for (m, n) in wl.layers]
            self.mom = [torch.zeros(m, n, device=device) for (m, n) in wl.layers]
        self.vecs = self.vout = self.vx = self.vmom = None
        if wl.vectors:
            self.vecs = [[t.to(device) for t in src.vector_grads(0, w)] for w in range(W)]
            self.vout = [torch.empty(k, device=device) for k in wl.vectors]
            self.vx = [torch.zeros(k, device=device) for k in wl.vectors]
            self.vmom = [torch.zeros(k, device=device) for k in wl.vectors]

    def set_rank(self, rank):
        """Initial Q and P_hat buffers for rank r; the error memory starts
        from zero again (a fresh run of the same gradients at another rank)."""
        self.rank = rank
        L = len(self.wl.layers)
        self.Q = [self.src.initial_q(l, rank).to(self.device) for l in range(L)]
        self.P = [torch.empty(m, rank, device=self.device) for (m, _) in self.wl.layers]
        for e in self.E_flat:
            e.zero_()

    def release(self):
        """Drop every device buffer (the caller then empties torch's cache)."""
        for name in ("G_flat", "E_flat", "G", "E", "Q", "P", "params", "mom", "vecs", "vout", "vx", "vmom"):
            setattr(self, name, None)


def device_bytes_needed(wl, rank):
    W = wl.workers
    gsz = 2 if wl.grad_dtype == "bf16" else 4
    e = wl.elements_per_worker
    b = W * e * (gsz + 4)
    if wl.momentum:
        b += 2 * e * 4
    return b


def run_step(lib, B, wl):
    lib.step(B.G, B.E, B.Q, B.P, None)
    if B.vecs is not None:
        beta, lr = wl.momentum if wl.momentum else (0.0, 0.0)
        lib.vec_mean(B.vecs, B.vout, B.vx, B.vmom, lr=lr, beta=beta)
    if B.params is not None:
        beta, lr = wl.momentum
        lib.momentum_step(B.params, B.mom, lr, beta)


class DistBuffers:
    """Send/receive buffers of the distributed step: the float64 P and Q
    partials (all-reduced in place) and a flat copy of every local worker's
    1-D gradients (all-reduced, then averaged over the global workers)."""

    def __init__(self, lib, B, wl, device):
        pe, qe = lib.dist_sizes()
        self.p = torch.empty(pe, dtype=torch.float64, device=device)
        self.q = torch.empty(qe, dtype=torch.float64, device=device)
        self.vflat = self.vsum = self.vviews = None
        if B.vecs is not None:
            # every vector in a 16-byte aligned slot (the library's rule)
            W = len(B.vecs)
            self.slots = []
            off = 0
            for w in range(W):
                for k in wl.vectors:
                    self.slots.append((off, k))
                    off += (k + 3) // 4 * 4
            self.vflat = torch.zeros(max(off, 4), dtype=B.vecs[0][0].dtype, device=device)
            self.pack(B.vecs)
            self.vsum = torch.empty_like(self.vflat)
            it = iter(self.slots)
            self.vviews = [[self.vsum[o:o + k] for (o, k) in [next(it) for _ in wl.vectors]] for _ in range(W)]

    def pack(self, vecs):
        it = iter(self.slots)
        for row in vecs:
            for t in row:
                o, k = next(it)
                self.vflat[o:o + k].copy_(t)


def dist_step(lib, B, wl, db, all_reduce):
    """One data-parallel step across ranks: the library's three distributed
    calls with the two all-reduces (SUM) of the P and Q partials between
    them, then the 1-D means over all workers and the momentum update."""
    lib.dist_p(B.G, B.E, B.Q, db.p, B.P, None)
    all_reduce(db.p)
    lib.dist_q(db.p, db.q)
    all_reduce(db.q)
    lib.dist_finish(db.q)
    if db.vflat is not None:
        db.vsum.copy_(db.vflat)
        all_reduce(db.vsum)
        beta, lr = wl.momentum if wl.momentum else (0.0, 0.0)
        lib.vec_mean(db.vviews, B.vout, B.vx, B.vmom, lr=lr, beta=beta)
    if B.params is not None:
        beta, lr = wl.momentum
        lib.momentum_step(B.params, B.mom, lr, beta)


def launches_per_step(lib, B, dist: bool = False):
    n = lib.step_launches + (2 if dist else 0)   # distributed: + orthogonalisation + Q_bar kernels
    if B.vecs is not None:
        n += 1
    if B.params is not None:
        n += 1
    return n


def roofline_block(wl, r: int, mode: str, kern_ms, kern_steps: int, ms_per_step: float, clk,
                   lazy: bool = False, sum_first: bool = False, iters: int = 1) -> dict:
    """The JSON line's roofline object: the dominant pass's algorithmic
    bytes per launch over its average event-timed launch (pass A reads G
    and E, or M, and writes M; pass B reads M; pass C reads M and writes
    E'), against the measured copy bandwidth; the step's minimum and design
    bytes over the step time; at r >= 16 the products' compute side."""
    peak, peak_kind = _peaks()
    gsz = 2 if wl.grad_dtype == "bf16" else 4
    per_launch_ms = [k / max(1, kern_steps) for k in kern_ms]
    alg = [wl.elements * (gsz + 8), wl.elements * 4, 0 if lazy else wl.elements * 8]
    names = ["pass_a", "pass_b", "pass_c"]
    dom = max(range(3), key=lambda i: per_launch_ms[i])
    achieved = alg[dom] / (per_launch_ms[dom] * 1e-3) / 1e9 if per_launch_ms[dom] > 0 else 0.0
    traffic = _traffic_record(wl.name, mode) if dom == 0 else None
    step_min_bytes = wl.elements * (gsz + 8)
    roofline = {"bound": "hbm", "kernel": names[dom], "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_kind": f"{peak_kind} hbm_gbs",
                "per_kernel_ms": {n: round(t, 4) for n, t in zip(names, per_launch_ms)},
                "step_algorithmic_frac": round(step_min_bytes / (ms_per_step * 1e-3) / 1e9 / peak, 4)}
    if iters == 1:
        # achieved DRAM bandwidth of the whole step: the bytes the three
        # passes move (ncu puts each pass's traffic at its design bytes)
        roofline["step_dram_frac"] = round(sum(alg) / (ms_per_step * 1e-3) / 1e9 / peak, 4)
    if r >= 16:
        # at ranks 16 and 32 the first two passes are bound by instruction
        # issue, not HBM: report their compute side too
        pk = {}
        pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
        if os.path.exists(pp):
            with open(pp) as f:
                pk = json.load(f)
        sm_mhz = (clk or {}).get("sm_mhz") or pk.get("sm_max_mhz", 1965.0)
        roofline["compute"] = compute_roofline(wl.elements, r, per_launch_ms[0], per_launch_ms[1], sm_mhz,
                                               pk.get("bf16_tflops", 1590.0), sum_first, wl.workers)
    return roofline


# --------------------------------------------------------------------------
# CPU oracle timing (bounded sample)

def oracle_sample(wl, rank, budget_s=15.0, seed=1234, max_layers=None, carry_bytes=4 << 30):
    """Time the float64 oracle on a bounded sample of the workload: whole
    layers (all workers) in list order, step after step with each layer's
    error memory and Q carried over, until the oracle time passes budget_s.
    Steps after the first are taken only when the carried float64 state
    (W * sum(m n) * 8 bytes) stays under carry_bytes.  Returns (elements/s,
    elements, seconds, threads, text)."""
    import oracle.powersgd64 as ora
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    src = GradientSource(wl, seed)
    done_el, spent, layers_done, steps_begun = 0, 0.0, 0, 0
    nl = len(wl.layers) if max_layers is None else min(max_layers, len(wl.layers))
    carry = wl.workers * sum(m * n for (m, n) in wl.layers[:nl]) * 8 <= carry_bytes
    state = {}
    shapes = []
    step = 0
    while spent < budget_s and nl > 0 and (step == 0 or carry):
        steps_begun += 1
        for l in range(nl):
            m, n = wl.layers[l]
            G = [src.layer_grad(step, w, l).to(torch.float64).numpy() for w in range(wl.workers)]
            if l in state:
                E, Q = state[l]
            else:
                E = [np.zeros((m, n)) for _ in range(wl.workers)]
                Q = src.initial_q(l, rank).to(torch.float64).numpy()
            t0 = time.perf_counter()
            res = ora.step(G, E, Q)
            spent += time.perf_counter() - t0
            done_el += wl.workers * m * n
            layers_done += 1
            if (m, n) not in shapes:
                shapes.append((m, n))
            if carry:
                state[l] = (res["E_new"], res["Q_bar"])
            del G, E, res
            if spent >= budget_s:
                break
        step += 1
    distinct = len(set(wl.layers[:nl]))
    text = (f"{layers_done} layer-steps over {steps_begun} step(s) of {len(wl.layers)} layers (all {wl.workers} "
            f"workers, error memory and Q carried, float64 NumPy; BLAS threads {threads}, elementwise ops "
            f"single-threaded); shapes sampled {len(shapes)} of {distinct}: "
            + ", ".join(f"{m}x{n}" for m, n in shapes))
    return done_el / spent, done_el, spent, threads, text


# --------------------------------------------------------------------------
# reports that need no timing

def compression_report(wl, r: int) -> dict:
    """What one worker sends per step with and without compression: the
    factors P (m x r) and Q (n x r) in float32, against the gradient itself
    (the "PowerSGD" glossary page: O(r(m + n)) instead of O(mn)); also the
    float64 P and Q partial sums the library's distributed step all-reduces
    (rank padded to a power of two)."""
    smn = sum(m * n for m, n in wl.layers)
    smpn = sum(m + n for m, n in wl.layers)
    R = 1
    while R < r:
        R *= 2
    gsz = 2 if wl.grad_dtype == "bf16" else 4
    return {"ratio": round(smn / (r * smpn), 2), "factor_bytes_per_worker": 4 * r * smpn,
            "gradient_bytes_per_worker": gsz * smn, "dist_partial_bytes_per_rank": 8 * R * smpn}


def sin_theta_max(U_ref: np.ndarray, P: np.ndarray) -> float:
    """Largest principal-angle sine between span(U_ref) and span(P) (both
    with orthonormal columns): the spectral norm of (I - U_ref U_ref^T) P."""
    Rm = P - U_ref @ (U_ref.T @ P)
    return float(np.linalg.norm(Rm, 2))


# --------------------------------------------------------------------------
# timing helpers

def timed_steps(step_fn, steps: int, warmup: int, lib, stream, barrier=lambda: None, before_timed=None):
    """warmup untimed steps, then exactly `steps` steps between two CUDA
    events on `stream`, with the library's per-pass events on.  Returns
    (ms per step, summed per-pass ms, profiled steps)."""
    for _ in range(warmup):
        step_fn()
    lib.status()
    barrier()
    torch.cuda.synchronize()
    if before_timed is not None:
        before_timed()
    lib.profile(True)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step_fn()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1)
    kern_ms, kern_steps = lib.profile_read()
    lib.profile(False)
    lib.status()
    return ms / max(1, steps), kern_ms, kern_steps


def _host_ram_available() -> float:
    try:
        with open("/proc/meminfo") as f:
            for line in f:
                if line.startswith("MemAvailable"):
                    return int(line.split()[1]) * 1024.0
    except Exception:
        pass
    return 0.0


def _pinned_empty(numel: int, dtype):
    return torch.empty(numel, dtype=dtype, pin_memory=True)


def _free_device_cache():
    import gc
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# --------------------------------------------------------------------------
# the other workloads (one GPU): eager step per workload and rank

def workload_line(wl, r: int, steps: int, warmup: int, stream, B=None, lazy_variant=False) -> dict:
    """Time the eager step of one workload at rank r (buffers B reused when
    given) and return its figures: ms per step, elements/s, the step's
    design-byte (DRAM) and minimum-byte fractions of the measured peak, and
    the per-pass times."""
    from rank_gradient_compression_02_b200 import PowerSGD
    lib = PowerSGD(wl.layers, r, wl.workers, grad_dtype=wl.grad_dtype)
    try:
        ms, kern_ms, ks = timed_steps(lambda: run_step(lib, B, wl), steps, warmup, lib, stream)
    finally:
        lib.close()
    rl = roofline_block(wl, r, "eager", kern_ms, ks, ms, None)
    out = {"rank": r, "ms_per_step": round(ms, 4), "value": job_value(wl.elements, 1, ms),
           "step_dram_frac": rl.get("step_dram_frac"), "step_algorithmic_frac": rl["step_algorithmic_frac"],
           "dominant": rl["kernel"], "dominant_frac": rl["frac"], "per_kernel_ms": rl["per_kernel_ms"],
           "pass_a_frac": round(wl.elements * ((2 if wl.grad_dtype == "bf16" else 4) + 8)
                                / (rl["per_kernel_ms"]["pass_a"] * 1e-3) / 1e9 / rl["peak"], 4)
           if rl["per_kernel_ms"]["pass_a"] > 0 else None,
           "steps": steps}
    if "compute" in rl:
        out["compute"] = {k: rl["compute"][k] for k in ("achieved", "unit", "fp32_frac", "tf32_frac")}
    if lazy_variant:
        B.set_rank(r)
        lib = PowerSGD(wl.layers, r, wl.workers, grad_dtype=wl.grad_dtype, lazy_errors=True)
        try:
            lms, _, _ = timed_steps(lambda: run_step(lib, B, wl), steps, warmup, lib, stream)
        finally:
            lib.close()
        peak = rl["peak"]
        gsz = 2 if wl.grad_dtype == "bf16" else 4
        out["lazy_errors"] = {"ms_per_step": round(lms, 4), "value": job_value(wl.elements, 1, lms),
                              "step_dram_frac": round(wl.elements * (gsz + 12) / (lms * 1e-3) / 1e9 / peak, 4),
                              "step_algorithmic_frac": round(wl.elements * (gsz + 8) / (lms * 1e-3) / 1e9 / peak,
                                                             4)}
    return out


def subspace_error_report(wl, ranks, device, steps: int, seed: int = 1234) -> dict:
    """Per rank: run `steps` warm-started steps of the workload's first
    matrix (its own seeded, slowly rotating gradients, all workers, error
    feedback) through the library and report sin of the largest principal
    angle between the last step's P_hat and the top-r left singular
    subspace of that step's worker mean M_bar = mean_w(G_w + E_w), from a
    float64 LAPACK SVD on the host."""
    from dataclasses import replace
    from rank_gradient_compression_02_b200 import PowerSGD
    one = replace(wl, layers=wl.layers[:1])
    m, n = one.layers[0]
    W = one.workers
    out = {}
    for r in ranks:
        src = GradientSource(one.with_rank(r), seed)
        gdt = torch.bfloat16 if one.grad_dtype == "bf16" else torch.float32
        G = [[torch.empty(m, n, dtype=gdt, device=device)] for _ in range(W)]
        E = [[torch.zeros(m, n, device=device)] for _ in range(W)]
        Q = [src.initial_q(0, r).to(device)]
        P = [torch.empty(m, r, device=device)]
        lib = PowerSGD(one.layers, r, W, grad_dtype=one.grad_dtype)
        try:
            for t in range(steps):
                src.fill(t, G)
                if t == steps - 1:
                    Mbar = sum(G[w][0].double() + E[w][0].double() for w in range(W)) / W
                lib.step(G, E, Q, P, None)
            torch.cuda.synchronize()
            lib.status()
        finally:
            lib.close()
        U = np.linalg.svd(Mbar.cpu().numpy(), full_matrices=False)[0][:, :r]
        Ph = P[0].double().cpu().numpy()
        checked = r <= one.spectrum_terms
        out[str(r)] = {"sin_theta_max": sin_theta_max(U, Ph), "steps": steps,
                       "status": "checked against the oracle's figure in the GPU tests" if checked else
                                 f"reported (directions beyond the {one.spectrum_terms}-term spectrum are noise)"}
        del G, E, Q, P, Mbar
    return {"matrix": f"{m}x{n}", "workers": W,
            "reference": "float64 LAPACK SVD of the last step's worker mean (numpy.linalg.svd)", "by_rank": out}


def run_workloads(keys, steps: int, warmup: int, device, stream, subspace_steps=None) -> dict:
    """The other workloads' eager steps on this GPU, one after another (each
    allocated, timed and released), with the rank sweeps of the sweep
    workloads, their compression figures and, for the 1024 x 1024 sweep,
    the subspace error."""
    res = {}
    for key in keys:
        wl = get_workload(key)
        ranks = list(wl.ranks) if wl.ranks else [wl.rank]
        if device_bytes_needed(wl, ranks[-1]) > torch.cuda.mem_get_info()[0] * 0.9:
            res[wl.name] = {"skipped": "not enough free device memory"}
            continue
        B = Buffers(wl, ranks[0], device)
        entry = {"elements_per_step": wl.elements, "workers": wl.workers, "grad_dtype": wl.grad_dtype,
                 "l2": "inputs larger than L2 (no flush needed)" if wl.elements * 4 > 4 * 126e6 else "inputs fit L2"}
        if wl.ranks:
            entry["by_rank"] = {}
            for r in ranks:
                B.set_rank(r)
                line = workload_line(wl.with_rank(r), r, steps, warmup, stream, B)
                line["compression"] = compression_report(wl, r)
                entry["by_rank"][str(r)] = line
        else:
            entry.update(workload_line(wl, wl.rank, steps, warmup, stream, B, lazy_variant=True))
            entry["compression"] = compression_report(wl, wl.rank)
        B.release()
        del B
        _free_device_cache()
        if wl.rotate and len(wl.layers) > 1:
            entry["subspace_error"] = subspace_error_report(wl, ranks, device,
                                                            subspace_steps or wl.steps)
        res[wl.name] = entry
    return res


# --------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="3", help="workload: 0, 1, 2, 3, 4a, 4b or a name (default 3, the "
                                                  "transformer set: the largest that fits one GPU)")
    ap.add_argument("--rank", type=int, default=None, help="rank r (default: the workload's)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--lazy", action="store_true", help="lazy error representation")
    ap.add_argument("--sum-first", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--oracle-budget", type=float, default=20.0)
    ap.add_argument("--layers", default=None, help="comma-separated layer indices (a subset, for small captures)")
    ap.add_argument("--workers", type=int, default=None, help="override the worker count (small captures)")
    ap.add_argument("--iters", type=int, default=1, help="power iterations per step")
    ap.add_argument("--no-variants", action="store_true", help="skip timing the lazy-error variant")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads' sub-lines (LSTM, ResNet-18, the two sweeps)")
    ap.add_argument("--workloads", default="2,4a,4b,1", help="workloads of the sub-lines")
    ap.add_argument("--workload-steps", type=int, default=10)
    ap.add_argument("--subspace-steps", type=int, default=None,
                    help="steps of the subspace-error runs (default: the workload's own)")
    ap.add_argument("--dist", action="store_true",
                    help="use the distributed step with NCCL all-reduces even on one GPU")
    args = ap.parse_args()

    from dataclasses import replace
    wl = get_workload(args.config)
    r = args.rank if args.rank is not None else wl.rank
    wl = wl.with_rank(r)
    if args.layers:
        idx = [int(x) for x in args.layers.split(",")]
        wl = replace(wl, name=f"{wl.name}[layers {args.layers}]", layers=tuple(wl.layers[i] for i in idx),
                     vectors=())
    if args.workers:
        wl = replace(wl, name=f"{wl.name}[W={args.workers}]", workers=args.workers)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank_id = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    mode = ("lazy" if args.lazy else "eager") + ("+sumfirst" if args.sum_first else "") + \
        (f"+iters{args.iters}" if args.iters != 1 else "")
    config = {"workload": wl.name, "layers": len(wl.layers), "elements_per_worker": wl.elements_per_worker,
              "workers": wl.workers, "rank": r, "grad_dtype": wl.grad_dtype, "mode": mode,
              "l2": "inputs larger than L2 (no flush needed)" if wl.elements * 4 > 4 * 126e6 else "inputs fit L2",
              "parallelism": (f"dp{world} (P and Q all-reduced over NCCL; {wl.workers} simulated workers per GPU)"
                              if (world > 1 or args.dist) else "1 GPU")}

    if args.impl == "reference":
        if rank_id != 0:
            return
        run_reference(args, wl, r, config, world)
        return

    import torch.distributed as dist
    if world > 1 or args.dist:
        torch.cuda.set_device(local)
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29533")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)

    from rank_gradient_compression_02_b200 import PowerSGD
    if world == 1:
        # one process: build libpsgd.so if it is missing or stale (a no-op
        # otherwise); several ranks never race on the build, they load it
        from rank_gradient_compression_02_b200 import build
        build.build()
    free, _ = torch.cuda.mem_get_info()
    need = device_bytes_needed(wl, r)
    if need > free * 0.95:
        raise SystemExit(f"workload needs {need/1e9:.1f} GB, {free/1e9:.1f} GB free")
    B = Buffers(wl, r, device)
    lib = PowerSGD(wl.layers, r, wl.workers, grad_dtype=wl.grad_dtype, lazy_errors=args.lazy,
                   sum_first=args.sum_first, power_iters=args.iters)
    dist_mode = world > 1 or args.dist
    if dist_mode:
        # every rank holds W local workers; P and Q are all-reduced over NCCL
        lib.set_global_workers(wl.workers * world)
        DB = DistBuffers(lib, B, wl, device)

        def _all_reduce(t):
            dist.all_reduce(t, op=dist.ReduceOp.SUM)

        def step_fn():
            dist_step(lib, B, wl, DB, _all_reduce)
    else:
        def step_fn():
            run_step(lib, B, wl)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    # clocks sampled from before the warm-up to the end of the timed region
    clocks = ClockSampler(local if world > 1 else 0)
    clocks.start()
    stream = torch.cuda.current_stream()
    ms_per_step, kern_ms, kern_steps = timed_steps(step_fn, args.steps, args.warmup, lib, stream, barrier)
    clk = clocks.stop()
    ms_per_step = max_over_ranks(ms_per_step * args.steps, world, device) / args.steps
    value = job_value(wl.elements, world, ms_per_step)

    roofline = roofline_block(wl, r, mode, kern_ms, kern_steps, ms_per_step, clk, lazy=args.lazy,
                              sum_first=args.sum_first, iters=args.iters)
    peak = roofline["peak"]
    gsz = 2 if wl.grad_dtype == "bf16" else 4
    step_min_bytes = wl.elements * (gsz + 8)

    # the lazy-error representation of the same step (E' rebuilt inside the
    # next step's first pass; bit-identical results), timed the same way
    variants = {}
    if not args.lazy and not args.no_variants and not dist_mode:
        lazy_lib = PowerSGD(wl.layers, r, wl.workers, grad_dtype=wl.grad_dtype, lazy_errors=True,
                            sum_first=args.sum_first, power_iters=args.iters)
        for _ in range(args.warmup):
            run_step(lazy_lib, B, wl)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            run_step(lazy_lib, B, wl)
        lazy_lib.materialize_errors(B.E)    # the last step's E' written out, inside the timed region
        e1.record(stream)
        torch.cuda.synchronize()
        lazy_lib.status()
        lms = max_over_ranks(e0.elapsed_time(e1), world, device) / args.steps
        variants["lazy_errors"] = {"ms_per_step": lms, "value": job_value(wl.elements, world, lms),
                                   "step_algorithmic_frac": round(step_min_bytes / (lms * 1e-3) / 1e9 / peak, 4),
                                   "step_dram_frac": (round(wl.elements * (gsz + 12) / (lms * 1e-3) / 1e9 / peak, 4)
                                                      if args.iters == 1 else None),
                                   "note": "error buffers hold M between steps; E' materialised once at the end "
                                           "of the timed region"}
        lazy_lib.close()

    cpu = None
    if rank_id == 0 and world == 1 and not args.no_cpu_baseline:
        v, el, sec, threads, text = oracle_sample(wl, r, budget_s=args.oracle_budget)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": text,
               "seconds": round(sec, 2)}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(lib, B, wl, r, args, world, device, DB if dist_mode else None)

    launches = args.steps * launches_per_step(lib, B, dist_mode)
    lib.close()
    B.release()
    del B
    if dist_mode:
        del DB
    _free_device_cache()

    workloads = None
    if world == 1 and not dist_mode and not args.no_workloads and not args.layers and not args.workers:
        keys = [k for k in args.workloads.split(",") if k and get_workload(k).name != wl.name]
        workloads = run_workloads(keys, args.workload_steps, 3, device, stream, args.subspace_steps)

    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f32" if wl.grad_dtype == "f32" else "bf16-in/f32",
           "data": "synthetic (seeded low-rank + noise gradients, resident in HBM)",
           "config": config, "gpu_launches": launches,
           "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk, "variants": variants,
           "hbm_gbs_step": round(step_min_bytes / (ms_per_step * 1e-3) / 1e9, 1),
           "compression": compression_report(wl, r), "workloads": workloads}
    if rank_id == 0:
        print(json.dumps(out), flush=True)
    if world > 1 or args.dist:
        dist.destroy_process_group()


def run_e2e(lib, B, wl, r, args, world, device, DB=None):
    """The same metric through the public API with host buffers: pinned
    host gradients, one flat buffer per worker, copied in every step
    (psgd_step_host_flat on one GPU, which uploads layer groups on a stream
    of its own and starts each group's passes once its copies have landed;
    one copy per worker into the device buffers before the distributed step
    on several), P_hat and Q_bar (and the 1-D means) read back.  When the library's device staging of the
    host gradients would not fit beside the resident buffers (the
    transformer set: 38.7 GB of bf16 gradients beside 77 GB of error
    memory), the device gradient buffers are released first: the staging
    takes their place."""
    gsz = 2 if wl.grad_dtype == "bf16" else 4
    import torch.distributed as dist
    W, L = wl.workers, len(wl.layers)
    span = max(B.offs[l] + m * n for l, (m, n) in enumerate(wl.layers))
    host_bytes = W * B.offs[-1] * gsz
    if host_bytes * 1.25 + 8e9 > _host_ram_available():
        return {"value": None, "unit": UNIT,
                "skipped": f"host RAM too small for {host_bytes / 1e9:.1f} GB of pinned gradients"}
    # one pinned host buffer per worker holding every layer (a flat gradient
    # bucket); the library uploads it in layer groups
    Gh = [_pinned_empty(B.offs[-1], B.G_flat[0].dtype) for _ in range(W)]
    for w in range(W):
        Gh[w].copy_(B.G_flat[w])
    stage_bytes = W * ((span * gsz + 255) // 256 * 256)
    released = False
    if DB is None and stage_bytes > torch.cuda.mem_get_info()[0] * 0.9:
        B.G_flat = None
        B.G = None
        _free_device_cache()
        released = True
    layer_offs = [B.offs[l] for l in range(L)]
    Ph = [torch.empty(m, r).pin_memory() for (m, _) in wl.layers]
    Qh = [torch.empty(n, r).pin_memory() for (_, n) in wl.layers]
    vbytes = 0
    if B.vecs is not None:
        # the 1-D gradients of all workers in one pinned buffer, 16-byte
        # aligned slots, one upload; the means come back in one download
        slots, off = [], 0
        for w in range(W):
            for k in wl.vectors:
                slots.append((off, k))
                off += (k + 3) // 4 * 4
        vflat_h = torch.zeros(max(off, 4)).pin_memory()
        it = iter(slots)
        for w in range(W):
            for t in B.vecs[w]:
                o, k = next(it)
                vflat_h[o:o + k].copy_(t.cpu())
        vflat_d = DB.vflat if DB is not None else torch.empty_like(vflat_h, device=device)
        it = iter(slots)
        vviews = [[vflat_d[o:o + k] for (o, k) in [next(it) for _ in wl.vectors]] for _ in range(W)]
        oslots, ooff = [], 0
        for k in wl.vectors:
            oslots.append((ooff, k))
            ooff += (k + 3) // 4 * 4
        vout_d = torch.empty(max(ooff, 4), device=device)
        vout_h = torch.empty(max(ooff, 4)).pin_memory()
        vout_views = [vout_d[o:o + k] for (o, k) in oslots]
        vbytes = vflat_h.numel() * 4
    stream = torch.cuda.current_stream()

    def one_dist():
        import torch.distributed as dist
        for w in range(W):
            B.G_flat[w].copy_(Gh[w], non_blocking=True)
        if B.vecs is not None:
            vflat_d.copy_(vflat_h, non_blocking=True)
        dist_step(lib, B, wl, DB, lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM))
        for l in range(L):
            Ph[l].copy_(B.P[l], non_blocking=True)
            Qh[l].copy_(B.Q[l], non_blocking=True)
        if B.vecs is not None:
            for (o, k), v in zip(oslots, B.vout):
                vout_d[o:o + k].copy_(v)
            vout_h.copy_(vout_d, non_blocking=True)

    def one():
        if DB is not None:
            return one_dist()
        lib.step_host_flat(Gh, layer_offs, B.E, B.Q, Ph, Qh)
        if B.vecs is not None:
            vflat_d.copy_(vflat_h, non_blocking=True)
            beta, lr = wl.momentum if wl.momentum else (0.0, 0.0)
            lib.vec_mean(vviews, vout_views, B.vx, B.vmom, lr=lr, beta=beta)
            vout_h.copy_(vout_d, non_blocking=True)
        if B.params is not None:
            beta, lr = wl.momentum
            lib.momentum_step(B.params, B.mom, lr, beta)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    per = ms / args.e2e_steps
    h2d = W * span * gsz + vbytes
    d2h = sum((m + n) * r * 4 for (m, n) in wl.layers) + (vout_h.numel() * 4 if B.vecs is not None else 0)
    out = {"value": wl.elements * world / (per * 1e-3), "unit": UNIT, "ms_per_step": per,
           "steps": args.e2e_steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if released:
        out["note"] = "device gradient buffers released first; the library's staging holds the uploads"
    del Gh
    return out


def run_reference(args, wl, r, config, world, full_max_elements=2e8, budget_s=180.0):
    """The float64 oracle on the host cores as the reference arm, same
    metric and unit.  A step is the whole workload step (every layer, all
    workers, error memory and Q carried, the gradients fixed as in the timed
    GPU loop) when the workload has at most full_max_elements worker
    elements and warm-up plus timed steps fit in about budget_s; otherwise
    each step is one layer (all workers), the layers taken in list order,
    cycling."""
    import oracle.powersgd64 as ora
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    src = GradientSource(wl, 1234)
    L = len(wl.layers)
    cache = {}

    def grads(l):
        if l not in cache:
            if len(cache) >= L or (not full and cache):
                cache.clear()
            cache[l] = [src.layer_grad(0, w, l).to(torch.float64).numpy() for w in range(wl.workers)]
        return cache[l]

    state = {}

    def layer_step(l):
        m, n = wl.layers[l]
        G = grads(l)
        E, Q = state.get(l) or ([np.zeros((m, n)) for _ in range(wl.workers)],
                                src.initial_q(l, r).double().numpy())
        t0 = time.perf_counter()
        o = ora.step(G, E, Q)
        dt = time.perf_counter() - t0
        state[l] = (o["E_new"], o["Q_bar"]) if full else None
        if not full:
            state.pop(l)
        return dt, wl.workers * m * n

    cursor = [0]

    def one():
        if full:
            res = [layer_step(l) for l in range(L)]
            return sum(x[0] for x in res), sum(x[1] for x in res)
        l = cursor[0] % L
        cursor[0] += 1
        return layer_step(l)

    full = wl.elements <= full_max_elements
    total = args.warmup + args.steps
    done = 0
    if full and total > 0:
        # the first warm-up step decides whether whole steps fit the bound
        t0 = time.perf_counter()
        one()
        done = 1
        if (time.perf_counter() - t0) * total > budget_s:
            full = False
            cache.clear()
            state.clear()
    for _ in range(done, args.warmup):
        one()
    spent, el = 0.0, 0
    for _ in range(args.steps):
        s_, e_ = one()
        spent += s_
        el += e_
    value = el / spent
    sample = (f"each step: the whole workload step ({L} layers, all {wl.workers} workers, error memory and Q "
              f"carried, gradients fixed), float64 NumPy oracle" if full else
              f"each step: one layer of the workload (all {wl.workers} workers), layers in list order, cycling, "
              f"float64 NumPy oracle")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": spent / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded low-rank + noise gradients)", "config": config,
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
