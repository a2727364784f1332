"""Benchmark of the FP8 block-scaled GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--scales fp32|ue8m0]

One step is one pass of the per-call hot path over one batch of synthetic
input: the activation quantizer (per token, per 128 channels) followed by the
GEMM (dense, contiguous-grouped or masked-grouped, per the workload). Weights
are quantized once before timing, as inference stores them (pass
--with-weight-quant to quantize them inside every step as well).

The default workload is contiguous_8x4096x7168 (MoE grouped GEMM in the
contiguous layout: 8 experts with the top-8-of-256 Zipf routing of 4096
tokens, N=4096, K=7168), the largest single-GPU configuration, with fp32
scales amax/448 (the promoted GEMM). Inputs are resident in HBM when the
timed region starts. By default
the step's operands (activations, quantized weights, scales, output) exist in
several copies whose total is three times the 126 MB L2, used in turn, so that
no step finds its inputs in L2; the K timed steps run back to back between one
pair of CUDA events (launch overheads overlap as they do in a serving loop, and
programmatic dependent launch lets each kernel's prologue overlap its
predecessor). `--l2 flush` instead flushes L2 before every step (a 256 MiB
write, then a 256 MiB read so that no dirty flush lines are written back during
the step) and times each step alone between its own events. `value` is FLOPs
(2*M_valid*N*K) per step time; `roofline` covers the GEMM kernel, timed alone
the same way as a burst of at most 20 launches (the denominators are burst
figures, and longer GEMM-only loops run into the power limit that the steps,
with the quantizer between GEMMs, do not reach), against the measured HBM
bandwidth or FP8 tensor peak; `e2e`
repeats the step through the public API from pinned host buffers with the
host<->device copies inside the timed region (uploads, compute and downloads
of consecutive steps pipelined on three streams, as a serving loop would);
`cpu_baseline` times the CPU oracle on a bounded sample of the same workload.
`--scales ue8m0` quantizes with power-of-two scales and runs the block-scaled
GEMM entry points (the oracle then uses the same power-of-two quantizers).

The default run (the contiguous workload) also times the other named GEMM
configurations (decode, both prefill shapes, the masked layout) the same way,
device-timed only, and lists them under `other_configs` in the same JSON line;
`--no-other-configs` skips them.

`--workload peak_fp8_mma_16384` measures the FP8 tensor-core rate itself: one
CTA per SM issues the GEMMs' MMA instruction back to back from operands that
stay in shared memory (no loads, no promotion), and the accumulators are
checked exactly; it is the in-library ceiling of the tensor-bound lines.

`--workload ep_32x512x8_4096x7168` times the expert-parallel layer
(quantize, dispatch into the masked layout, masked GEMM, combine) per call,
with NCCL's all-to-all over the ranks of the run, and its masked GEMM alone
for the roofline.

Multi-GPU (torchrun, one process per GPU): the GEMM path does not shard
across GPUs within one call, so every rank runs an independent replica (weak
scaling); the timed region is bracketed by a barrier and the reported time is
the max over ranks. The expert-parallel workload exchanges tokens between the
ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

DEFAULT_WORKLOAD = "contiguous_8x4096x7168"
# the other GEMM configurations the method's measurements name (decode, the two
# prefill shapes, the masked layout), timed in the default run as well
OTHER_CONFIGS = ("decode_64x4096x7168", "prefill_4096x7168x2048", "prefill_4096x2112x7168",
                 "masked_32x256x4096x7168")


METRIC = "FP8 block-scaled GEMM TFLOPS (device-timed) and % of B200 FP8/HBM roofline"
KERNEL_BURST = 20  # GEMM-only launches timed for the roofline (at most)
L2_FLUSH_BYTES = 256 << 20
SENTINEL_BF16 = 0x7FC1  # a bf16 NaN pattern the kernels never produce
ROTATE_MIN_BYTES = 3 * (126 << 20)  # operand sets in turn: three times the 126 MB L2
FP8_OVER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor throughput ratio
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 rated figures (vendor datasheet, dense): the second denominator of
# every roofline fraction, beside the measured one
RATED_FP8_TFLOPS = 4500.0
RATED_HBM_GBS = 8000.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--with-weight-quant", action="store_true")
    ap.add_argument("--scales", default="fp32", choices=["fp32", "ue8m0"],
                    help="fp32: scale = amax / 448 (the promoted GEMM); ue8m0: power-of-two "
                         "scales (the _ue8m0 quantizers and the block-scaled GEMM)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps from Python instead of replaying a CUDA graph")
    ap.add_argument("--l2", default="rotate", choices=["rotate", "flush"],
                    help="keep timed steps out of L2 by rotating operand sets larger than L2 "
                         "(steps back to back) or by flushing L2 before every step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="the default run also times the other named GEMM configurations "
                         "(device-timed, no CPU baseline or e2e) and lists them under "
                         "other_configs; this skips them")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample (a sample takes at "
                         "least 0.85 of it)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(files: dict) -> str:
    """Hash of {file name: source bytes} with C/C++ comments and whitespace
    removed, so that comment-only edits keep the hash."""
    h = hashlib.sha256()
    for name in sorted(files):
        text = re.sub(rb"/\*.*?\*/", b" ", files[name], flags=re.S)
        text = re.sub(rb"//[^\n]*", b" ", text)
        text = b" ".join(text.split())
        h.update(name.encode() + b"\0" + text)
    return h.hexdigest()[:16]


def kernel_source_hash() -> str:
    """source_hash of the kernel sources (moe_grouped_gemm_04_b200/csrc)."""
    csrc = os.path.join(ROOT, "moe_grouped_gemm_04_b200", "csrc")
    files = {}
    for name in os.listdir(csrc):
        with open(os.path.join(csrc, name), "rb") as f:
            files[name] = f.read()
    return source_hash(files)


def traffic_for(workload: str, ue8m0: bool = False):
    """DRAM bytes per GEMM launch from a committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload + ("@ue8m0" if ue8m0 else ""))
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------- CPU legs

# a CPU sample stops growing once it takes this fraction of the target time
SAMPLE_STOP = 0.85


def repeat_for(fn, target_s: float):
    """Calls fn() until at least target_s seconds have passed; returns
    (calls, seconds)."""
    t0 = time.perf_counter()
    calls = 0
    while True:
        fn()
        calls += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            return calls, dt


def cpu_sample(inp, kind: str, target_s: float, threads: int, cache: dict, ue8m0: bool = False):
    """Oracle on a bounded sample of the workload: quantize the sampled A rows
    and compute their outputs against all N columns (weights are quantized
    outside the timed part, as on the GPU side). Returns
    (flops_per_second, description, seconds)."""
    import oracle

    if kind == "ffn":
        return ffn_cpu_sample(inp, target_s, threads, cache)
    if kind == "kgrouped":
        return kgrouped_cpu_sample(inp, target_s, threads, cache)
    K, N = inp.K, inp.N
    if kind == "dense":
        a_rows, experts = inp.a, np.zeros(inp.M, np.int64)
    elif kind == "contiguous":
        valid = np.nonzero(inp.m_indices >= 0)[0]
        a_rows, experts = inp.a[valid], inp.m_indices[valid].astype(np.int64)
    else:
        sel = [(e, m) for e in range(inp.G) for m in range(int(inp.masked_m[e]))]
        a_rows = np.stack([inp.a[e, m] for e, m in sel]) if sel else inp.a[0, :0]
        experts = np.array([e for e, _ in sel], np.int64)

    def weights(e):
        if e not in cache:
            b = inp.b if kind == "dense" else inp.b[e]
            cache[e] = oracle.per_block_cast(b, threads=threads, ue8m0=ue8m0)
        return cache[e]

    order = np.random.default_rng(0).permutation(len(a_rows))
    rows = cache.get("rows", 1)
    while True:
        take = order[:min(rows, len(order))]
        for e in np.unique(experts[take]):
            weights(int(e))
        t0 = time.perf_counter()
        qa, sa = oracle.per_token_cast(a_rows[take], threads=threads, ue8m0=ue8m0)
        for e in np.unique(experts[take]):
            sub = np.nonzero(experts[take] == e)[0]
            qb, sb = weights(int(e))
            oracle.gemm_nt(qa[sub], sa[sub], qb, sb, threads=threads)
        dt = time.perf_counter() - t0
        if dt >= SAMPLE_STOP * target_s or len(take) >= len(order):
            break
        rows = max(rows * 2, int(rows * target_s / max(dt, 1e-3) * 1.05))
    cache["rows"] = rows
    done = len(take)
    passes = 1
    if done >= len(order) and dt < SAMPLE_STOP * target_s:
        # the whole workload is smaller than the target: repeat it until the
        # target time has passed
        def one_pass():
            qa, sa = oracle.per_token_cast(a_rows, threads=threads, ue8m0=ue8m0)
            for e in np.unique(experts):
                sub = np.nonzero(experts == e)[0]
                qb, sb = weights(int(e))
                oracle.gemm_nt(qa[sub], sa[sub], qb, sb, threads=threads)
        passes, dt = repeat_for(one_pass, target_s)
    flops = 2.0 * done * N * K * passes
    desc = "%d of %d valid A rows x all %d columns, K=%d (activation quantization + GEMM)" % (
        done, len(order), N, K)
    if passes > 1:
        desc += ", %d passes" % passes
    return flops / dt, desc, dt


def ffn_cpu_sample(inp, target_s: float, threads: int, cache: dict):
    """The oracle's expert-FFN chain (UE8M0 quantization of the sampled rows,
    first GEMM, bf16, SwiGLU, requantization, second GEMM) on a bounded sample
    of valid rows; expert weights are quantized outside the timed part."""
    import oracle

    H, I = inp.H, inp.I
    valid = np.nonzero(inp.m_indices >= 0)[0]
    experts = inp.m_indices[valid].astype(np.int64)

    def weights(e):
        if ("w", e) not in cache:
            cache[("w", e)] = (oracle.per_block_cast(inp.w1[e], threads=threads, ue8m0=True),
                               oracle.per_block_cast(inp.w2[e], threads=threads, ue8m0=True))
        return cache[("w", e)]

    order = np.random.default_rng(0).permutation(len(valid))
    rows = cache.get("rows", 1)
    while True:
        take = order[:min(rows, len(order))]
        for e in np.unique(experts[take]):
            weights(int(e))
        t0 = time.perf_counter()
        qa, sa = oracle.per_token_cast(inp.a[valid[take]], threads=threads, ue8m0=True)
        for e in np.unique(experts[take]):
            sub = np.nonzero(experts[take] == e)[0]
            (w1q, sw1), (w2q, sw2) = weights(int(e))
            gu = oracle.f64_to_bf16(oracle.gemm_nt(qa[sub], sa[sub], w1q, sw1, threads=threads))
            h = oracle.swiglu(gu[:, :I], gu[:, I:])
            hq, sh = oracle.per_token_cast(h, threads=threads, ue8m0=True)
            oracle.gemm_nt(hq, sh, w2q, sw2, threads=threads)
        dt = time.perf_counter() - t0
        if dt >= SAMPLE_STOP * target_s or len(take) >= len(order):
            break
        rows = max(rows * 2, int(rows * target_s / max(dt, 1e-3) * 1.05))
    cache["rows"] = rows
    flops = 6.0 * len(take) * H * I
    desc = ("%d of %d valid rows through the whole expert FFN (quantization, first GEMM, "
            "SwiGLU, requantization, second GEMM), H=%d, I=%d" % (len(take), len(order), H, I))
    return flops / dt, desc, dt


def kgrouped_cpu_sample(inp, target_s: float, threads: int, cache: dict):
    """The oracle's K-grouped GEMM for a bounded sample of A rows (quantized per
    row per 128 tokens) against all of B (quantized outside the timed part)."""
    import oracle

    if "qb" not in cache:
        cache["qb"] = oracle.per_token_cast(inp.b, threads=threads, ue8m0=True)
    qb, sb = cache["qb"]
    tv = int(inp.counts.sum())
    order = np.random.default_rng(0).permutation(inp.M)
    rows = cache.get("rows", 1)
    while True:
        take = np.sort(order[:min(rows, inp.M)])
        t0 = time.perf_counter()
        qa, sa = oracle.per_token_cast(inp.a[take], threads=threads, ue8m0=True)
        oracle.k_grouped(qa, sa, qb, sb, inp.ks, threads=threads)
        dt = time.perf_counter() - t0
        if dt >= SAMPLE_STOP * target_s or len(take) >= inp.M:
            break
        rows = max(rows * 2, int(rows * target_s / max(dt, 1e-3) * 1.05))
    cache["rows"] = rows
    flops = 2.0 * len(take) * inp.N * tv
    desc = ("%d of %d A rows x all %d B rows over all %d experts' tokens (T=%d, quantization "
            "of the sampled rows + K-grouped GEMM)" % (len(take), inp.M, inp.N, inp.G, inp.T))
    return flops / dt, desc, dt


# ---------------------------------------------------------------------- ranks

def max_over_ranks(dist, values, device):
    """Element-wise maximum of `values` (floats) over all ranks of the
    process group: the job's time is its slowest rank's."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


# ---------------------------------------------------------------------- GPU leg

def ffn_one_launch(inp) -> bool:
    """The library's automatic choice of the expert FFN's form for a contiguous
    batch: one launch when an expert's rows (M_total / G) are at most 128."""
    return inp.M_total // inp.G <= 128


def gemm_kernel_name(kind: str, inp, ue8m0: bool) -> str:
    """The GEMM kernel a step launches (the library's choice for the shape)."""
    if kind == "ffn":
        if ffn_one_launch(inp):
            return ("fp8_gemm_mx_kernel (both expert GEMMs in one launch: first GEMM with fused "
                    "SwiGLU + requantization, then second GEMM)")
        return "fp8_gemm_mx_kernel x2 (first GEMM with fused SwiGLU + requantization, second GEMM)"
    if kind == "kgrouped":
        return "fp8_gemm_mx_kernel (K-grouped, fp32 output)"
    thin = (kind == "dense" and inp.M <= 64) or (
        kind == "masked" and max(1, int(round(float(np.mean(inp.masked_m))))) <= 64)
    return "fp8_gemm_mx_kernel" if ue8m0 and not thin else "fp8_gemm_kernel"


class OperandSet:
    """Device buffers of one copy of a step's operands."""

    def __init__(self, torch, kind, inp, fg, x, w, B, SB, with_weight_quant: bool, extra=None):
        dev = "cuda"
        K, N = inp.K, inp.N
        self.x = x.clone()
        self.w = w.clone() if with_weight_quant else None
        self.extra = []
        if kind == "kgrouped":
            # both operands are per-step activations: x (dY^T) and x2 (X^T)
            x2 = extra
            self.x2 = x2.clone()
            M, N, T = inp.M, inp.N, inp.T
            self.A = torch.empty((M, T), dtype=torch.uint8, device=dev)
            self.SA = fg.empty_sfa(1, M, T, dev)
            self.B = torch.empty((N, T), dtype=torch.uint8, device=dev)
            self.SB = fg.empty_sfa(1, N, T, dev)
            self.D = torch.empty((inp.G, M, N), dtype=torch.float32, device=dev)
            self.extra = [self.x2]
            return
        self.B = B.clone()
        self.SB = SB.clone()
        if kind == "ffn":
            W2, SW2 = extra
            self.W2, self.SW2 = W2.clone(), SW2.clone()
            M, H, I = inp.M_total, inp.H, inp.I
            self.A = torch.empty((M, H), dtype=torch.uint8, device=dev)
            self.SA = fg.empty_sfa(1, M, H, dev)
            self.Hq = torch.empty((M, I), dtype=torch.uint8, device=dev)
            self.SH = fg.empty_sfa(1, M, I, dev)
            self.D = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
            # the one-kernel FFN's ready counters (cleared by every call)
            self.WS = fg.empty_ffn_workspace(fg.FG_LAYOUT_CONTIGUOUS, M, inp.G, dev)
            self.extra = [self.W2, self.SW2, self.Hq, self.SH]
            return
        if kind == "dense":
            G, M = 1, inp.M
            self.A = torch.empty((inp.M, K), dtype=torch.uint8, device=dev)
            self.D = torch.empty((inp.M, N), dtype=torch.bfloat16, device=dev)
        elif kind == "contiguous":
            G, M = 1, inp.M_total
            self.A = torch.empty((inp.M_total, K), dtype=torch.uint8, device=dev)
            self.D = torch.empty((inp.M_total, N), dtype=torch.bfloat16, device=dev)
        else:
            G, M = inp.G, inp.M_max
            self.A = torch.empty((inp.G, inp.M_max, K), dtype=torch.uint8, device=dev)
            self.D = torch.empty((inp.G, inp.M_max, N), dtype=torch.bfloat16, device=dev)
        self.SA = fg.empty_sfa(G, M, K, dev)

    def nbytes(self):
        ts = [self.x, self.B, self.SB, self.A, self.D, self.SA] + ([self.w] if self.w is not None else [])
        ts += self.extra
        return sum(t.numel() * t.element_size() for t in ts)


class Step:
    """The launches of one step over one of several operand sets.

    With `sets` > 1 the copies are used in turn, so that a step's weights and
    activations are not in L2 when it starts (their total exceeds L2)."""

    def __init__(self, fg, torch, kind, inp, with_weight_quant: bool, min_total_bytes: int,
                 ue8m0: bool = False):
        self.fg, self.torch, self.kind, self.inp = fg, torch, kind, inp
        self.with_wq = with_weight_quant
        self.ue8m0 = ue8m0
        sfx = "_ue8m0" if ue8m0 else ""
        self.q_token = getattr(fg, "per_token_cast_to_fp8" + sfx)
        self.q_block = getattr(fg, "per_block_cast_to_fp8" + sfx)
        self.g_dense = getattr(fg, "fp8_gemm_nt" + sfx)
        self.g_contig = getattr(fg, "fp8_grouped_gemm_contiguous" + sfx)
        self.g_masked = getattr(fg, "fp8_grouped_gemm_masked" + sfx)
        dev = "cuda"
        K, N = inp.K, inp.N

        def bf16(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

        extra = None
        if kind == "kgrouped":
            x, w = bf16(inp.a), None
            extra = bf16(inp.b)
            B = SB = None
            self.ks = torch.from_numpy(inp.ks).to(dev)
        elif kind == "ffn":
            # W1 [G][2I][H] in B/SB, W2 [G][H][I] alongside
            x, w = bf16(inp.a), bf16(inp.w1)
            B = torch.empty((inp.G, 2 * inp.I, inp.H), dtype=torch.uint8, device=dev)
            SB = fg.empty_sfb(inp.G, 2 * inp.I, inp.H, dev)
            self.q_block(w, B, SB)
            w2 = bf16(inp.w2)
            W2 = torch.empty((inp.G, inp.H, inp.I), dtype=torch.uint8, device=dev)
            SW2 = fg.empty_sfb(inp.G, inp.H, inp.I, dev)
            self.q_block(w2, W2, SW2)
            extra = (W2, SW2)
            del w2
        else:
            x, w = bf16(inp.a), bf16(inp.b)
            Gw = 1 if kind == "dense" else inp.G
            B = torch.empty((N, K) if kind == "dense" else (inp.G, N, K), dtype=torch.uint8, device=dev)
            SB = fg.empty_sfb(Gw, N, K, dev)
            self.q_block(w, B, SB)
        if kind in ("contiguous", "ffn"):
            self.mi = torch.from_numpy(inp.m_indices).to(dev)
        if kind == "masked":
            self.mm = torch.from_numpy(inp.masked_m).to(dev)
            self.expected_m = max(1, int(round(float(np.mean(inp.masked_m)))))
        first = OperandSet(torch, kind, inp, fg, x, w, B, SB, with_weight_quant, extra)
        per = first.nbytes()
        n = max(2, -(-min_total_bytes // per)) if min_total_bytes > 0 else 1
        self.sets = [first] + [OperandSet(torch, kind, inp, fg, x, w, B, SB, with_weight_quant, extra)
                               for _ in range(n - 1)]
        del x, w, B, SB
        self.set_bytes = per

    def quant_weights(self, o):
        self.q_block(o.w, o.B, o.SB)

    def quant_acts(self, o):
        self.q_token(o.x, o.A, o.SA)
        if self.kind == "kgrouped":
            self.q_token(o.x2, o.B, o.SB)

    def gemm(self, o):
        if self.kind == "kgrouped":
            self.fg.fp8_k_grouped_gemm_nt_ue8m0(o.A, o.SA[0], o.B, o.SB[0], o.D, self.ks)
        elif self.kind == "ffn":
            self.fg.fp8_moe_ffn_contiguous_ue8m0(o.A, o.SA, o.B, o.SB, o.W2, o.SW2, o.Hq, o.SH, o.D,
                                                 self.mi, ws=o.WS)
        elif self.kind == "dense":
            self.g_dense(o.A, o.SA, o.B, o.SB, o.D)
        elif self.kind == "contiguous":
            self.g_contig(o.A, o.SA, o.B, o.SB, o.D, self.mi)
        else:
            self.g_masked(o.A, o.SA, o.B, o.SB, o.D, self.mm, self.expected_m)

    def launches_per_step(self):
        """Kernels of this library per step: the activation quantizer and the
        GEMM; the FFN's two GEMMs are two kernels, or one in its one-launch
        form (whose counter reset is a memset, not a kernel); K-grouped: two
        quantizers and the GEMM."""
        n = 3 if self.kind == "kgrouped" else 2
        if self.kind == "ffn" and not ffn_one_launch(self.inp):
            n = 3
        return n + (1 if self.with_wq else 0)

    def run(self, i):
        o = self.sets[i % len(self.sets)]
        if self.with_wq:
            self.quant_weights(o)
        self.quant_acts(o)
        self.gemm(o)


def workload_config(kind: str, inp) -> dict:
    """The workload's sizes as they appear in the JSON line's `config` (the same
    keys in both arms, so the two lines describe the same problem)."""
    cfg = {"N": inp.N, "K": inp.K}
    if kind == "ffn":
        cfg = {"H": inp.H, "I": inp.I, "G": inp.G, "M_total": inp.M_total,
               "M_valid": int(inp.counts.sum())}
    elif kind == "kgrouped":
        cfg.update(M=inp.M, T=inp.T, G=inp.G, T_valid=int(inp.counts.sum()))
    elif kind == "dense":
        cfg["M"] = inp.M
    elif kind == "contiguous":
        cfg.update(G=inp.G, M_total=inp.M_total, M_valid=int(inp.counts.sum()))
    elif kind == "masked":
        cfg.update(G=inp.G, M_max=inp.M_max, M_valid=int(inp.masked_m.sum()))
    return cfg


def step_config(args, kind: str, inp, world: int, ue8m0: bool) -> dict:
    """The JSON line's `config`: what problem one step solves. Both arms build
    it with this function, so their lines carry the same config; how a step
    was timed goes into the separate `method` object."""
    return {"workload": args.workload, "kind": kind, **workload_config(kind, inp),
            "weights": "quantized inside every step" if args.with_weight_quant
                       else "quantized once before timing",
            "scales": ("power-of-two (UE8M0) scales, block-scaled tensor-core GEMM" if ue8m0 else
                       "fp32 scales amax/448, promoted per 128-wide K block"),
            "parallelism": "replicas" if world > 1 else "single GPU"}


def fp8_mma_rate():
    """The FP8 tensor-core rate this library's own MMA loop reached on this
    pool (workload peak_fp8_mma_16384), from its committed record, or None."""
    path = os.path.join(ROOT, "profiles", "fp8_mma_rate.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        return json.load(f).get("tflops")


def peaks_used(peaks: dict, source: str) -> dict:
    """The denominators a roofline fraction was taken against, with where they
    came from, so that the fraction can be recomputed."""
    d = {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
         "fp8_tflops": FP8_OVER_BF16 * peaks["bf16_tflops"],
         "fp8_rule": "%.1f x the bf16 burst figure" % FP8_OVER_BF16,
         "source": "MEASURED_PEAKS.json" if source == "measured" else "recipe fallback",
         "rated_fp8_tflops": RATED_FP8_TFLOPS, "rated_hbm_gbs": RATED_HBM_GBS}
    rate = fp8_mma_rate()
    if rate:
        d["fp8_mma_in_library_tflops"] = rate
    clk = peaks.get("clocks_under_load") or {}
    if clk.get("sm_mhz_median") is not None:
        d["sm_mhz_median_when_measured"] = clk["sm_mhz_median"]
    return d


def run_ours(args, rank, world, local_rank):
    import torch

    import moe_grouped_gemm_04_b200 as fg

    torch.cuda.set_device(local_rank)
    fg.load_library()
    kind = workloads.WORKLOADS[args.workload][0]
    inp = workloads.make(args.workload, seed=0)
    flops, alg_bytes = workloads.flops_and_bytes(kind, inp)
    rotate = args.l2 == "rotate"
    # the expert FFN and the K-grouped GEMM use power-of-two scales
    ue8m0 = args.scales == "ue8m0" or kind in ("ffn", "kgrouped")
    if kind in ("ffn", "kgrouped") and args.with_weight_quant:
        raise SystemExit("--with-weight-quant is not supported for the %s workload" % kind)
    step = Step(fg, torch, kind, inp, args.with_weight_quant,
                ROTATE_MIN_BYTES if rotate else 0, ue8m0)
    R = len(step.sets)
    stream = torch.cuda.current_stream()
    if not rotate:
        flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        flush_r = torch.ones(L2_FLUSH_BYTES // 8, dtype=torch.int64, device="cuda")

    def flush():
        flush_w.zero_()
        flush_r.sum()

    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod

    def barrier():
        if dist is not None:
            dist.barrier()

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def timed(body, K, graph=False):
        """Mean ms per iteration of body(i) over K iterations. rotate: one
        event pair around K back-to-back iterations (operand sets in turn),
        replayed from one CUDA graph when `graph`; flush: L2 flushed before
        every iteration, outside its event pair."""
        barrier()
        torch.cuda.synchronize()
        if rotate and graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                for i in range(K):
                    body(i)
            g.replay()  # untimed: the first replay uploads the graph
            torch.cuda.synchronize()
            barrier()
            torch.cuda.synchronize()
            e0, e1 = ev(), ev()
            s = torch.cuda.current_stream()
            e0.record(s)
            g.replay()
            e1.record(s)
            torch.cuda.synchronize()
            del g
            return e0.elapsed_time(e1) / K
        if rotate:
            e0, e1 = ev(), ev()
            e0.record(stream)
            for i in range(K):
                body(i)
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / K
        pairs = [(ev(), ev()) for _ in range(K)]
        for i in range(K):
            flush()
            pairs[i][0].record(stream)
            body(i)
            pairs[i][1].record(stream)
        torch.cuda.synchronize()
        return float(np.mean([x.elapsed_time(y) for x, y in pairs]))

    for i in range(max(args.warmup, R)):
        if not rotate:
            flush()
        step.run(i)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0

    K = args.steps
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)  # let the sampler see the timed region from its start
    use_graph = rotate and not args.no_graph
    ms = timed(step.run, K, use_graph)
    barrier()
    # the GEMM kernel alone (roofline); every set's activations are quantized.
    # Outputs start as a NaN sentinel so that the check below sees what the
    # timed launches wrote.
    for o in step.sets:
        o.D.view(torch.int16).fill_(SENTINEL_BF16)
    # The GEMM alone, as a burst: at most KERNEL_BURST launches back to back in
    # one CUDA graph. The roofline's denominators are burst figures (cuBLAS's
    # best single launches), and a longer uninterrupted GEMM-only loop can run
    # the tensor pipe into the power limit (sw_power_cap), which the timed
    # steps, with the quantizer between GEMMs, do not reach.
    n_burst = min(K, KERNEL_BURST)
    gms = timed(lambda i: step.gemm(step.sets[i % R]), n_burst, use_graph)
    barrier()
    clocks = sampler.stop()
    assert fg.get_device_status() == 0
    # the timed launches did the work: the last output the timed GEMM loop
    # wrote equals a fresh eager call, bit for bit (the kernels are deterministic)
    last = step.sets[(n_burst - 1) % R]
    timed_d = last.D.clone()
    last.D.view(torch.int16).fill_(SENTINEL_BF16)
    step.gemm(last)
    torch.cuda.synchronize()
    assert torch.equal(timed_d.view(torch.int16), last.D.view(torch.int16)), "timed output differs"

    # End to end through the public API from pinned host buffers: every step
    # uploads its activations, runs the quantizer and the GEMM, and reads its
    # output back. As in a serving loop the steps are pipelined on three
    # streams (upload, compute, download), so the upload of step i+1 and the
    # download of step i-1 overlap the compute of step i; each step uses its
    # own operand set, whose previous use (compute and read-back) must have
    # finished before the upload overwrites it. Timed between events on the
    # compute stream, which waits for the last download before the closing
    # event.
    e2e = None
    if not args.no_e2e:
        xh = step.sets[0].x.cpu().pin_memory()
        # (K-grouped: both operands are the step's inputs)
        x2h = step.sets[0].x2.cpu().pin_memory() if kind == "kgrouped" else None
        dh = [torch.empty(step.sets[0].D.shape, dtype=step.sets[0].D.dtype).pin_memory()
              for _ in range(2)]
        up, down = torch.cuda.Stream(), torch.cuda.Stream()

        # events are created once and re-recorded: set i % R's upload,
        # compute-done and download-done events (a wait sees the most recent
        # record)
        up_ev = [torch.cuda.Event() for _ in range(R)]
        done_ev = [torch.cuda.Event() for _ in range(R)]
        dl_ev = [torch.cuda.Event() for _ in range(R)]

        def e2e_loop(n):
            comp = torch.cuda.current_stream()
            e0, e1 = ev(), ev()
            e0.record(comp)
            up.wait_event(e0)
            down.wait_event(e0)
            for i in range(n):
                j = i % R
                o = step.sets[j]
                with torch.cuda.stream(up):
                    if i >= R:
                        # the set's previous step has been computed and read back
                        up.wait_event(dl_ev[j])
                    o.x.copy_(xh, non_blocking=True)
                    if x2h is not None:
                        o.x2.copy_(x2h, non_blocking=True)
                    up_ev[j].record(up)
                comp.wait_event(up_ev[j])
                step.run(i)
                done_ev[j].record(comp)
                with torch.cuda.stream(down):
                    down.wait_event(done_ev[j])
                    dh[i % 2].copy_(o.D, non_blocking=True)
                    dl_ev[j].record(down)
            comp.wait_stream(down)
            e1.record(comp)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n

        e2e_loop(max(3, args.warmup))
        barrier()
        torch.cuda.synchronize()
        e2e_ms = e2e_loop(K)
        barrier()
        e2e = {"ms": e2e_ms, "h2d": xh.numel() * xh.element_size() +
                                    (x2h.numel() * x2h.element_size() if x2h is not None else 0),
               "d2h": dh[0].numel() * dh[0].element_size()}

    # max over ranks
    if dist is not None:
        ms, gms, e2e_max = max_over_ranks(dist, [ms, gms, e2e["ms"] if e2e else 0.0], "cuda")
        if e2e:
            e2e["ms"] = e2e_max

    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    tensor_bound = flops / alg_bytes > (2 * peaks.get("bf16_tflops", 1590.0) * 1e12) / (peaks["hbm_gbs"] * 1e9)
    if tensor_bound:
        peak = FP8_OVER_BF16 * peaks["bf16_tflops"]
        achieved = flops / (gms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_rated": RATED_FP8_TFLOPS,
                "frac_rated": achieved / RATED_FP8_TFLOPS}
        if fp8_mma_rate():
            roof["peak_in_library"] = fp8_mma_rate()
            roof["frac_in_library"] = achieved / fp8_mma_rate()
        peak_note = "FP8 = %.1f x %s bf16 burst %.1f TFLOP/s (%s)" % (
            FP8_OVER_BF16, peak_src, peaks["bf16_tflops"], "MEASURED_PEAKS.json" if peak_src == "measured" else "recipe fallback")
    else:
        peak = peaks["hbm_gbs"]
        achieved = alg_bytes / (gms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_rated": RATED_HBM_GBS,
                "frac_rated": achieved / RATED_HBM_GBS}
        peak_note = "%s HBM copy bandwidth (%s)" % (peak_src, "MEASURED_PEAKS.json" if peak_src == "measured" else "recipe fallback")
    roof["traffic"] = traffic_for(args.workload, ue8m0)
    roof["kernel"] = gemm_kernel_name(kind, inp, ue8m0)
    roof["algorithmic_per_launch"] = {"flops": flops, "bytes": alg_bytes}
    roof["kernel_ms"] = gms
    roof["kernel_timing"] = ("%d GEMM-only launches back to back in one CUDA graph (a burst, like the "
                             "peaks' figures), CUDA events on the launching stream" % n_burst)
    roof["peak_source"] = peak_note
    roof["peaks_used"] = peaks_used(peaks, peak_src)

    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        threads = oracle.hardware_threads()
        fps, desc, secs = cpu_sample(inp, kind, args.cpu_seconds, threads, {}, ue8m0)
        cpu = {"value": fps / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": desc, "seconds": secs}

    value = world * flops / (ms * 1e-3) / 1e12
    cfg = step_config(args, kind, inp, world, ue8m0)
    method = {
        "l2": ("inputs larger than L2: %d operand sets of %.1f MB used in turn, steps back to back"
               % (R, step.set_bytes / 1e6)) if rotate else
              "flushed before every timed step (256 MiB write + 256 MiB read, outside the step events)",
        "launch": ("the K timed steps captured in one CUDA graph, replayed once untimed, "
                   "then once between the events") if use_graph else "eager launches from Python",
        "timing": "CUDA events on the launching stream, max over ranks"}
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8_e4m3", "data": "synthetic (seeded numpy, random weights)",
        "config": cfg, "method": method, "roofline": roof, "cpu_baseline": cpu,
        "gpu_launches": step.launches_per_step() * K,
        "clocks": clocks,
    }
    if e2e:
        out["e2e"] = {"value": world * flops / (e2e["ms"] * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                      "ms_per_step": e2e["ms"]}
    return out


DEQUANT_METRIC = "FP8 weight dequantization (e4m3 + 128x128 scales -> bf16) GB/s (device-timed)"


def time_graph_launches(launch, steps: int, local_rank: int, world: int):
    """launch(0 .. steps-1) captured in one CUDA graph, replayed once untimed
    (upload), then timed between one pair of CUDA events while the clocks are
    sampled. Returns (ms per launch, clock summary)."""
    import torch
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        for i in range(steps):
            launch(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del g
    return ms, sampler.stop()


def run_dequant(args, rank, world, local_rank):
    """The weight dequantizer alone: codes and block scales (quantized once on
    the GPU) -> bf16, on operand sets whose total exceeds L2, used in turn,
    K launches replayed from one CUDA graph between one pair of events."""
    import torch

    import moe_grouped_gemm_04_b200 as fg

    torch.cuda.set_device(local_rank)
    fg.load_library()
    inp = workloads.make(args.workload, seed=0)
    N, K = inp.N, inp.K
    _, alg_bytes = workloads.flops_and_bytes("dequant", inp)
    w = torch.from_numpy(np.ascontiguousarray(inp.b).view(np.int16)).cuda().view(torch.bfloat16)
    q0 = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    s0 = fg.empty_sfb(1, N, K, "cuda")
    fg.per_block_cast_to_fp8(w, q0, s0)
    per = int(alg_bytes)
    R = max(2, -(-ROTATE_MIN_BYTES // per))
    sets = [(q0.clone(), s0.clone(), torch.empty((N, K), dtype=torch.bfloat16, device="cuda"))
            for _ in range(R)]

    def launch(i):
        q, sc, x = sets[i % R]
        fg.per_block_dequant_to_bf16(q, sc, x)

    for i in range(max(args.warmup, R)):
        launch(i)
    torch.cuda.synchronize()
    steps = args.steps
    ms, clocks = time_graph_launches(launch, steps, local_rank, world)
    # the timed launches did the work: the last output equals a fresh call
    last = sets[(steps - 1) % R]
    timed_x = last[2].clone()
    last[2].view(torch.int16).fill_(SENTINEL_BF16)
    launch(steps - 1)
    torch.cuda.synchronize()
    assert torch.equal(timed_x.view(torch.int16), last[2].view(torch.int16)), "timed output differs"
    if world > 1:
        import torch.distributed as dist
        ms = max_over_ranks(dist, [ms], "cuda")[0]
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    cpu = None
    if not args.no_cpu_baseline:
        cpu = dequant_cpu_sample(inp, args.cpu_seconds)
    return {
        "metric": DEQUANT_METRIC, "value": world * gbs, "unit": "GB/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3->bf16",
        "data": "synthetic (seeded numpy, random weights)",
        "config": {"workload": args.workload, "kind": "dequant", "N": N, "K": K,
                   "l2": "inputs larger than L2: %d operand sets of %.1f MB used in turn" % (R, per / 1e6),
                   "launch": "K launches captured in one CUDA graph, replayed once untimed, then timed"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "kernel": "per_block_dequant_kernel", "kernel_ms": ms,
                     "algorithmic_per_launch": {"bytes": alg_bytes},
                     "peak_source": "%s HBM copy bandwidth" % peak_src},
        "cpu_baseline": cpu, "gpu_launches": steps, "clocks": clocks, "e2e": None,
    }


QUANT_METRIC = "FP8 activation quantization (bf16 -> e4m3 + per-token 1x128 scales) GB/s (device-timed)"


def run_quant(args, rank, world, local_rank):
    """The activation quantizer alone: bf16 activations -> e4m3 codes and
    per-token scales (amax / 448, or powers of two with --scales ue8m0), on
    operand sets whose total exceeds L2, used in turn, K launches replayed
    from one CUDA graph between one pair of events."""
    import torch

    import moe_grouped_gemm_04_b200 as fg

    torch.cuda.set_device(local_rank)
    fg.load_library()
    inp = workloads.make(args.workload, seed=0)
    M, K = inp.M, inp.K
    ue8m0 = args.scales == "ue8m0"
    cast = fg.per_token_cast_to_fp8_ue8m0 if ue8m0 else fg.per_token_cast_to_fp8
    _, alg_bytes = workloads.flops_and_bytes("quant", inp)
    x0 = torch.from_numpy(np.ascontiguousarray(inp.a).view(np.int16)).cuda().view(torch.bfloat16)
    per = int(alg_bytes)
    R = max(2, -(-ROTATE_MIN_BYTES // per))
    sets = [(x0.clone(), torch.empty((M, K), dtype=torch.uint8, device="cuda"),
             fg.empty_sfa(1, M, K, "cuda")) for _ in range(R)]

    def launch(i):
        x, q, sc = sets[i % R]
        cast(x, q, sc)

    for i in range(max(args.warmup, R)):
        launch(i)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    steps = args.steps
    ms, clocks = time_graph_launches(launch, steps, local_rank, world)
    # the timed launches did the work: the last outputs equal a fresh call's
    last = sets[(steps - 1) % R]
    timed_q, timed_s = last[1].clone(), last[2][..., :M].clone()
    last[1].fill_(0x7F)
    last[2].fill_(float("nan"))
    launch(steps - 1)
    torch.cuda.synchronize()
    assert torch.equal(timed_q, last[1]), "timed codes differ"
    assert torch.equal(timed_s.view(torch.int32), last[2][..., :M].view(torch.int32)), "timed scales differ"
    if world > 1:
        import torch.distributed as dist
        ms = max_over_ranks(dist, [ms], "cuda")[0]
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    cpu = None
    if not args.no_cpu_baseline:
        cpu = quant_cpu_sample(inp, args.cpu_seconds, ue8m0)
    return {
        "metric": QUANT_METRIC, "value": world * gbs, "unit": "GB/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3",
        "data": "synthetic (seeded numpy)",
        "config": {"workload": args.workload, "kind": "quant", "M": M, "K": K,
                   "scales": "power-of-two (UE8M0)" if ue8m0 else "fp32 amax/448",
                   "l2": "inputs larger than L2: %d operand sets of %.1f MB used in turn" % (R, per / 1e6),
                   "launch": "K launches captured in one CUDA graph, replayed once untimed, then timed"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "kernel": "per_token_cast_kernel", "kernel_ms": ms,
                     "algorithmic_per_launch": {"bytes": alg_bytes},
                     "peak_source": "%s HBM copy bandwidth" % peak_src},
        "cpu_baseline": cpu, "gpu_launches": steps, "clocks": clocks, "e2e": None,
    }


def quant_cpu_sample(inp, target_s: float, ue8m0: bool = False):
    """The oracle's activation quantizer on a bounded sample of rows."""
    import oracle
    threads = oracle.hardware_threads()
    rows = 16
    while True:
        t0 = time.perf_counter()
        oracle.per_token_cast(inp.a[:rows], threads=threads, ue8m0=ue8m0)
        dt = time.perf_counter() - t0
        if dt >= SAMPLE_STOP * target_s or rows >= inp.M:
            break
        rows = min(inp.M, rows * 2)
    passes = 1
    if dt < SAMPLE_STOP * target_s:
        passes, dt = repeat_for(
            lambda: oracle.per_token_cast(inp.a[:rows], threads=threads, ue8m0=ue8m0), target_s)
    byts = passes * (rows * inp.K * 3 + 4 * rows * (inp.K // 128))
    return {"value": byts / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": "%d of %d rows x K=%d, %d passes" % (rows, inp.M, inp.K, passes), "seconds": dt}


def dequant_cpu_sample(inp, target_s: float):
    """The oracle's dequantizer on a bounded sample of rows of the same weight."""
    import oracle
    threads = oracle.hardware_threads()
    q, s = oracle.per_block_cast(inp.b, threads=threads)
    rows = 128
    while True:
        t0 = time.perf_counter()
        oracle.per_block_dequant(q[:rows], s[:-(-rows // 128)], threads=threads)
        dt = time.perf_counter() - t0
        if dt >= SAMPLE_STOP * target_s or rows >= inp.N:
            break
        rows = min(inp.N, rows * 2)
    passes = 1
    if dt < SAMPLE_STOP * target_s:
        passes, dt = repeat_for(
            lambda: oracle.per_block_dequant(q[:rows], s[:-(-rows // 128)], threads=threads), target_s)
    byts = passes * (rows * inp.K * 3 + 4 * (-(-rows // 128)) * (inp.K // 128))
    return {"value": byts / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": "%d of %d rows x K=%d, %d passes" % (rows, inp.N, inp.K, passes), "seconds": dt}


EP_METRIC = ("Expert-parallel MoE layer (quantize, dispatch into the masked layout, masked FP8 GEMM, "
             "combine) TFLOP/s (device-timed)")


def run_ep(args, rank, world, local_rank):
    """The expert-parallel layer (moe_grouped_gemm_04_b200.ep) over the ranks
    of this run (one rank: its all-to-alls are local copies through NCCL),
    each step timed between CUDA events around one layer call (the layer
    reads its split sizes back to the host once, so steps are not captured
    in a graph); the masked GEMM of the layer timed alone on the layout the
    layer dispatched, K launches in one CUDA graph, for the roofline."""
    import datetime
    import socket

    import torch
    import torch.distributed as dist

    import moe_grouped_gemm_04_b200 as fg
    import moe_grouped_gemm_04_b200.ep as ep

    torch.cuda.set_device(local_rank)
    fg.load_library()
    created = False
    if not dist.is_initialized():
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        created = True
    try:
        inp = workloads.make(args.workload, seed=rank)
        E, k, N, K, M_max = inp.E, inp.k, inp.N, inp.K, inp.M_max
        G = E // world
        dev = "cuda"
        x = torch.from_numpy(np.ascontiguousarray(inp.x).view(np.int16)).to(dev).view(torch.bfloat16)
        topk = torch.from_numpy(inp.topk).to(dev)
        topk_w = torch.from_numpy(inp.topk_w).to(dev)
        wb = torch.from_numpy(np.ascontiguousarray(inp.w[rank * G:(rank + 1) * G]).view(np.int16)).to(dev)
        wq = torch.empty((G, N, K), dtype=torch.uint8, device=dev)
        ws = fg.empty_sfb(G, N, K, dev)
        fg.per_block_cast_to_fp8(wb.view(torch.bfloat16), wq, ws)
        del wb

        # a fixed capacity of every pair a rank has (T * k rows per destination:
        # nothing can be dropped), so the layer never reads counts back
        cap = inp.T * k

        def step(capacity):
            return ep.expert_parallel_masked_moe(x, topk, topk_w, wq, ws, E, M_max, capacity=capacity)

        def timed_steps(capacity):
            for _ in range(max(args.warmup, 3)):
                step(capacity)
            torch.cuda.synchronize()
            assert fg.get_device_status() == 0
            dist.barrier()
            pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(args.steps)]
            for e0, e1 in pairs:
                e0.record()
                step(capacity)
                e1.record()
            torch.cuda.synchronize()
            return float(np.mean([a.elapsed_time(b) for a, b in pairs]))

        sampler = ClockSampler(local_rank)
        sampler.start()
        time.sleep(0.3)
        ms = timed_steps(cap)
        ms_exact = timed_steps(None)
        # the layer's GEMM alone, on the layout this rank's dispatch produced
        h = ep.ep_dispatch(x, topk, E, M_max, capacity=cap)
        D = torch.empty((G, M_max, N), dtype=torch.bfloat16, device=dev)
        em = max(1, min(M_max, -(-inp.T * k // G)))
        gms, _ = time_graph_launches(lambda i: fg.fp8_grouped_gemm_masked(h.A, h.sfa, wq, ws, D, h.masked_m, em),
                                     args.steps, local_rank, 1)
        clocks = sampler.stop()
        assert fg.get_device_status() == 0
        mm = h.masked_m.cpu().numpy()
        rows = int(mm.sum())
        if world > 1:
            ms, gms, ms_exact = max_over_ranks(dist, [ms, gms, ms_exact], "cuda")
            rows_all = torch.tensor([float(rows)], device=dev)
            dist.all_reduce(rows_all)
            rows_total = int(rows_all.item())
        else:
            rows_total = rows
    finally:
        if created:
            dist.destroy_process_group()
    if rank != 0:
        return None
    flops = 2.0 * rows_total * N * K          # every rank's GEMM rows
    gemm_flops = 2.0 * rows * N * K           # this rank's GEMM (the roofline's kernel)
    experts = int((mm > 0).sum())
    gemm_bytes = float(experts * (N * K + 4 * (-(-N // 128)) * (K // 128)) + rows * (K + 4 * (K // 128))
                       + 2 * rows * N)
    peaks, peak_src = load_peaks()
    gbs = gemm_bytes / (gms * 1e-3) / 1e9
    return {
        "metric": EP_METRIC, "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3",
        "data": "synthetic (seeded numpy, random weights and uniform top-%d routing)" % k,
        "config": {"workload": args.workload, "kind": "ep", "experts": E, "experts_per_rank": G,
                   "tokens_per_rank": inp.T, "topk": k, "N": N, "K": K, "M_max": M_max,
                   "rows_this_rank": rows, "scales": "fp32 amax/448 (promoted masked GEMM)",
                   "exchange": "NCCL all_to_all_single (%d rank%s), fixed capacity of %d rows per "
                               "destination (no host read of the counts)" % (world, "" if world == 1 else "s", cap),
                   "exact_splits_ms_per_step": ms_exact,
                   "timing": "CUDA events around each layer call, eager launches",
                   "l2": "inputs larger than L2: the rank's expert weights (%.0f MB)" % (G * N * K / 1e6)},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "peak_rated": RATED_HBM_GBS,
                     "frac_rated": gbs / RATED_HBM_GBS, "traffic": None,
                     "kernel": "fp8_gemm_kernel (masked form)", "kernel_ms": gms,
                     "algorithmic_per_launch": {"flops": gemm_flops, "bytes": gemm_bytes},
                     "peak_source": "%s HBM copy bandwidth" % peak_src},
        # per layer call: quantizer, pair count, position and capacity, pack,
        # unpack, masked GEMM, gather, combine (NCCL's own copy kernels not counted)
        "cpu_baseline": None, "gpu_launches": 9 * args.steps, "clocks": clocks, "e2e": None,
    }


PEAK_METRIC = ("FP8 tensor-core rate (tcgen05.mma kind::f8f6f4, M=128 N=256 K=32, operands resident "
               "in shared memory) TFLOP/s (device-timed)")


def peak_expected(iters: int) -> np.ndarray:
    """The accumulator every CTA of the tensor-core rate kernel ends with
    (the formula its C-ABI declaration states): small integers, exact."""
    m = np.arange(128)[:, None]
    n = np.arange(256)[:, None]
    j = np.arange(16)[None, :]
    a = (2 * m + 3 * j) % 5 - 2
    b = (3 * n + 2 * j + n // 16) % 5 - 2
    return (8.0 * iters) * (a.astype(np.float64) @ b.T.astype(np.float64))


def run_peak(args, rank, world, local_rank):
    """The FP8 tensor-core rate: one CTA per SM issuing the GEMMs' MMA
    instruction back to back from resident operands, K launches replayed
    from one CUDA graph between one pair of events. The ceiling of every
    tensor-bound line, measured with this library's own instruction stream."""
    import torch

    import moe_grouped_gemm_04_b200 as fg

    torch.cuda.set_device(local_rank)
    fg.load_library()
    inp = workloads.make(args.workload)
    iters = inp.iters
    ctas = fg.fp8_mma_peak_ctas()
    out = torch.empty((ctas, 128, 256), dtype=torch.float32, device="cuda")

    def launch(i):
        fg.fp8_mma_peak(iters, out)

    for i in range(max(args.warmup, 3)):
        launch(i)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    out.fill_(float("nan"))
    steps = args.steps
    ms, clocks = time_graph_launches(launch, steps, local_rank, world)
    assert fg.get_device_status() == 0
    # every MMA ran: each CTA holds the exact accumulator
    got = out.cpu().numpy()
    assert np.array_equal(got, np.broadcast_to(peak_expected(iters).astype(np.float32), got.shape)), \
        "tensor-core rate kernel: accumulator differs"
    if world > 1:
        import torch.distributed as dist
        ms = max_over_ranks(dist, [ms], "cuda")[0]
    if rank != 0:
        return None
    flops = 2.0 * 128 * 256 * 128 * iters * ctas
    tflops = flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    anchor = FP8_OVER_BF16 * peaks["bf16_tflops"]
    return {
        "metric": PEAK_METRIC, "value": world * tflops, "unit": "TFLOP/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3",
        "data": "operands generated in shared memory by the kernel (small integers)",
        "config": {"workload": args.workload, "kind": "peak", "ctas": ctas, "iters": iters,
                   "mma": "128x256x32 kind::f8f6f4, fp32 accumulator in tensor memory",
                   "l2": "no memory operands (nothing to flush)",
                   "launch": "K launches captured in one CUDA graph, replayed once untimed, then timed"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": anchor, "unit": "TFLOP/s",
                     "frac": tflops / anchor, "peak_rated": RATED_FP8_TFLOPS,
                     "frac_rated": tflops / RATED_FP8_TFLOPS, "traffic": None,
                     "kernel": "fp8_mma_peak_kernel", "kernel_ms": ms,
                     "algorithmic_per_launch": {"flops": flops, "bytes": 0.0},
                     "peak_source": "FP8 = %.1f x %s bf16 burst %.1f TFLOP/s" % (
                         FP8_OVER_BF16, peak_src, peaks["bf16_tflops"]),
                     "peaks_used": peaks_used(peaks, peak_src)},
        "cpu_baseline": None, "gpu_launches": steps, "clocks": clocks, "e2e": None,
    }


def run_other_configs(args, rank, world, local_rank):
    """Each of OTHER_CONFIGS through run_ours with the same steps, warm-up and
    scales, device-timed only; rank 0 gets one summary per configuration."""
    import argparse as _ap

    import torch
    res = []
    for w in OTHER_CONFIGS:
        a = _ap.Namespace(**vars(args))
        a.workload, a.no_cpu_baseline, a.no_e2e = w, True, True
        r = run_ours(a, rank, world, local_rank)
        torch.cuda.empty_cache()
        if r is not None:
            roof = r["roofline"]
            res.append({"workload": w, "value": r["value"], "unit": r["unit"],
                        "ms_per_step": r["ms_per_step"], "kernel_ms": roof["kernel_ms"],
                        "roofline": {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac",
                                                          "frac_rated", "frac_in_library", "traffic")
                                     if k in roof},
                        "clocks": r.get("clocks")})
    return res


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm, on rank 0 only."""
    if rank != 0:
        return None
    import oracle
    kind = workloads.WORKLOADS[args.workload][0]
    inp = workloads.make(args.workload, seed=0)
    threads = oracle.hardware_threads()
    per_step = max(1.0, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    cache = {}
    ue8m0 = args.scales == "ue8m0" or kind in ("ffn", "kgrouped")
    for _ in range(args.warmup):
        cpu_sample(inp, kind, per_step, threads, cache, ue8m0)
    vals, descs, secs = [], [], []
    for _ in range(args.steps):
        fps, desc, s = cpu_sample(inp, kind, per_step, threads, cache, ue8m0)
        vals.append(fps)
        descs.append(desc)
        secs.append(s)
    value = float(np.mean(vals)) / 1e12
    ms = float(np.mean(secs)) * 1e3
    cfg = step_config(args, kind, inp, world, ue8m0)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy)",
        "config": cfg,
        "method": {"timing": "host wall clock (perf_counter) around each step's oracle calls; "
                             "each step is a bounded sample of the workload",
                   "threads": threads},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": descs[-1] if descs else ""},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    kind = workloads.WORKLOADS[args.workload][0]
    if args.impl == "reference" and kind == "ep":
        out = None
        if rank == 0:
            out = {"impl": "reference", "metric": EP_METRIC,
                   "unavailable": "the oracle has no all-to-all exchange; its masked GEMM is the "
                                  "masked_32x256x4096x7168 reference line"}
    elif args.impl == "reference" and kind == "peak":
        out = None
        if rank == 0:
            out = {"impl": "reference", "metric": PEAK_METRIC,
                   "unavailable": "the tensor-core rate workload measures the GPU itself; the oracle "
                                  "has no counterpart"}
    elif args.impl == "reference" and kind in ("dequant", "quant"):
        out = None
        if rank == 0:
            inp = workloads.make(args.workload, seed=0)
            if kind == "dequant":
                cpu = dequant_cpu_sample(inp, min(args.cpu_seconds, 5.0))
                metric, dtype = DEQUANT_METRIC, "f32->bf16"
            else:
                cpu = quant_cpu_sample(inp, min(args.cpu_seconds, 5.0), args.scales == "ue8m0")
                metric, dtype = QUANT_METRIC, "bf16->e4m3"
            out = {"impl": "reference", "metric": metric, "value": cpu["value"], "unit": "GB/s",
                   "n_gpus": world, "steps": 1, "warmup": 0, "higher_is_better": True,
                   "scaling": "weak", "vs_baseline": None, "dtype": dtype,
                   "data": "synthetic (seeded numpy)", "config": {"workload": args.workload},
                   "cpu_baseline": cpu,
                   "e2e": {"value": cpu["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}}
    elif args.impl == "reference":
        out = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime

            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local_rank))
        try:
            if kind == "dequant":
                out = run_dequant(args, rank, world, local_rank)
            elif kind == "quant":
                out = run_quant(args, rank, world, local_rank)
            elif kind == "peak":
                out = run_peak(args, rank, world, local_rank)
            elif kind == "ep":
                out = run_ep(args, rank, world, local_rank)
            else:
                out = run_ours(args, rank, world, local_rank)
                if args.workload == DEFAULT_WORKLOAD and not args.no_other_configs:
                    others = run_other_configs(args, rank, world, local_rank)
                    if out is not None:
                        out["other_configs"] = others
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
