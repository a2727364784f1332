"""Seeded synthetic inputs for the FP8 block-scaled GEMM workloads.

This module is shared by the CPU oracle's tests, the CUDA path's tests and the
benchmark. It holds none of the method's arithmetic: no quantization, no
scales, no products. It only draws random numbers, rounds them to the bf16
input format and lays them out in the shapes the workloads use.

Workloads (sizes from the DeepGEMM pages' serving scenarios: dense prefill and
decode shapes of DeepSeek-V3/R1, MoE grouped GEMM in contiguous and masked
layouts; the pages print no shape list, so these stand in for "all V3/R1
inference shapes"):

  dense_128x256x512        A ~ N(0,1), B ~ N(0,0.02)
  decode_64x4096x7168      A ~ N(0,1) with 1% of its rows (at least one) x30
  prefill_4096x7168x2048   A ~ N(0,1), B ~ N(0,0.02)
  prefill_4096x2112x7168   same, N not a multiple of 128
  contiguous_8x4096x7168   8 experts, token counts from top-8 routing of 4096
                           tokens over 256 experts (Gumbel-top-k on Zipf
                           s=1.1 weights over expert ids), experts 0..7,
                           each group padded to a multiple of 128, padding
                           rows zero, m_indices = -1 on padding rows
  masked_32x256x4096x7168  32 experts, capacity 256, masked_m ~ U{0..256}
  ffn_contiguous_8x7168x2048  expert FFN (DeepSeek-V3 expert shape: hidden
                           7168, intermediate 2048) on the contiguous
                           workload's 8 experts and token counts; W1 [8][4096][7168]
                           (gate rows, then up rows) and W2 [8][7168][2048]
                           ~ N(0, 0.02)
  quant_4096x7168          the activation quantizer alone, on the activations
                           of prefill_4096x2112x7168 (A ~ N(0,1))
  ep_32x512x8_4096x7168    expert-parallel layer (dispatch, masked GEMM, combine):
                           32 experts, 512 tokens ~ N(0,1) with K = 7168, each
                           routed to 8 distinct experts drawn uniformly
                           (Gumbel-top-k on equal weights), router weights
                           U(0,1) normalised per token, expert weights
                           [32][4096][7168] ~ N(0, 0.02), capacity M_max = 256
  peak_fp8_mma_16384       no inputs: the FP8 tensor-core rate, 16384 K blocks
                           of MMAs (128 x 256 x 128 each) per CTA from operands
                           the kernel generates in shared memory
  kgrouped_8x4096x7168     K-grouped weight-gradient GEMM of the contiguous
                           workload's experts: A = dY^T [4096][T] ~ N(0,1),
                           B = X^T [7168][T] ~ N(0,1), the experts' token
                           ranges (counts padded to 128, padding tokens zero)
                           stacked along T

Seeds: every tensor draws from its own ``numpy.random.default_rng(seed + i)``
with i = 0 for A, 1 for B (the FFN's W1), 2 for the routing, 3 for masked_m
and 5 for the FFN's W2.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

ALIGN_M = 128  # contiguous layout: each expert group starts on a 128-row boundary


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the raw 16-bit patterns as uint16. Inputs must be finite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    """bf16 bits of N(0, std^2) samples drawn in float32.

    Large tensors are drawn in slices along the first axis; the generator's
    stream is the same as one draw of the whole shape.
    """
    shape = tuple(shape)
    out = np.empty(shape, dtype=np.uint16)
    rows = shape[0] if shape else 1
    per_row = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    chunk = max(1, (1 << 26) // max(per_row, 1))
    flat = out.reshape(rows, per_row)
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        x = rng.standard_normal(size=(r1 - r0, per_row), dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        flat[r0:r1] = bf16_bits(x)
    return out


def zipf_top8_counts(seed: int, tokens: int = 4096, experts: int = 256,
                     topk: int = 8, s: float = 1.1) -> np.ndarray:
    """Per-expert token counts of top-k routing over Zipf(s) expert weights.

    Each token picks ``topk`` distinct experts by Gumbel-top-k on log weights
    w_i = (i+1)^-s (sampling without replacement proportionally to w).
    Returns counts for all ``experts`` experts.
    """
    rng = np.random.default_rng(seed + 2)
    logw = -s * np.log(np.arange(1, experts + 1, dtype=np.float64))
    g = rng.gumbel(size=(tokens, experts)) + logw[None, :]
    top = np.argpartition(-g, topk - 1, axis=1)[:, :topk]
    return np.bincount(top.ravel(), minlength=experts).astype(np.int64)


@dataclasses.dataclass
class DenseInputs:
    a: np.ndarray  # bf16 bits [M][K]
    b: np.ndarray  # bf16 bits [N][K]
    M: int
    N: int
    K: int


@dataclasses.dataclass
class ContiguousInputs:
    a: np.ndarray          # bf16 bits [M_total][K], padding rows zero
    b: np.ndarray          # bf16 bits [G][N][K]
    m_indices: np.ndarray  # int32 [M_total], expert id or -1 on padding rows
    counts: np.ndarray     # int64 [G] valid rows per expert
    M_total: int
    N: int
    K: int
    G: int


@dataclasses.dataclass
class MaskedInputs:
    a: np.ndarray         # bf16 bits [G][M_max][K]
    b: np.ndarray         # bf16 bits [G][N][K]
    masked_m: np.ndarray  # int32 [G]
    G: int
    M_max: int
    N: int
    K: int


def dense(M: int, N: int, K: int, seed: int = 0, outlier_frac: float = 0.0,
          outlier_scale: float = 30.0, a_std: float = 1.0,
          b_std: float = 0.02) -> DenseInputs:
    rng_a = np.random.default_rng(seed + 0)
    x = rng_a.standard_normal(size=(M, K), dtype=np.float32) * np.float32(a_std)
    if outlier_frac > 0.0 and M > 0:
        n_out = max(1, int(np.ceil(outlier_frac * M)))
        rows = rng_a.choice(M, size=n_out, replace=False)
        x[rows] *= np.float32(outlier_scale)
    a = bf16_bits(x)
    b = normal_bf16(np.random.default_rng(seed + 1), (N, K), b_std)
    return DenseInputs(a=a, b=b, M=M, N=N, K=K)


def contiguous_layout(counts: np.ndarray, align: int = ALIGN_M):
    """m_indices for groups stacked along M, each padded to ``align`` rows."""
    padded = [int(-(-int(c) // align) * align) for c in counts]
    M_total = int(sum(padded))
    m_indices = np.full(M_total, -1, dtype=np.int32)
    row = 0
    for g, (c, p) in enumerate(zip(counts, padded)):
        m_indices[row:row + int(c)] = g
        row += p
    return m_indices, M_total


def contiguous(N: int, K: int, counts: Optional[np.ndarray] = None, G: int = 8,
               seed: int = 0, a_std: float = 1.0, b_std: float = 0.02) -> ContiguousInputs:
    if counts is None:
        counts = zipf_top8_counts(seed)[:G]
    counts = np.asarray(counts, dtype=np.int64)
    G = len(counts)
    m_indices, M_total = contiguous_layout(counts)
    rng_a = np.random.default_rng(seed + 0)
    M_valid = int(counts.sum())
    xv = rng_a.standard_normal(size=(M_valid, K), dtype=np.float32) * np.float32(a_std)
    a = np.zeros((M_total, K), dtype=np.uint16)
    a[m_indices >= 0] = bf16_bits(xv)
    b = normal_bf16(np.random.default_rng(seed + 1), (G, N, K), b_std)
    return ContiguousInputs(a=a, b=b, m_indices=m_indices, counts=counts,
                            M_total=M_total, N=N, K=K, G=G)


@dataclasses.dataclass
class FfnInputs:
    a: np.ndarray          # bf16 bits [M_total][H], padding rows zero
    w1: np.ndarray         # bf16 bits [G][2I][H]: I gate rows, then I up rows
    w2: np.ndarray         # bf16 bits [G][H][I]
    m_indices: np.ndarray  # int32 [M_total]
    counts: np.ndarray     # int64 [G]
    M_total: int
    H: int
    I: int
    G: int

    @property
    def N(self) -> int:  # output columns (of the second GEMM)
        return self.H

    @property
    def K(self) -> int:  # contraction of the first GEMM
        return self.H


def ffn_contiguous(H: int, I: int, G: int = 8, seed: int = 0, a_std: float = 1.0,
                   w_std: float = 0.02) -> FfnInputs:
    c = contiguous(N=2 * I, K=H, G=G, seed=seed, a_std=a_std, b_std=w_std)
    w2 = normal_bf16(np.random.default_rng(seed + 5), (c.G, H, I), w_std)
    return FfnInputs(a=c.a, w1=c.b, w2=w2, m_indices=c.m_indices, counts=c.counts,
                     M_total=c.M_total, H=H, I=I, G=c.G)


@dataclasses.dataclass
class KGroupedInputs:
    a: np.ndarray       # bf16 bits [M][T] (the output gradient, transposed)
    b: np.ndarray       # bf16 bits [N][T] (the activations, transposed)
    ks: np.ndarray      # int32 [G] token counts, multiples of 128
    counts: np.ndarray  # int64 [G] valid tokens per expert (the rest are zero)
    M: int
    N: int
    T: int
    G: int

    @property
    def K(self) -> int:
        return self.T


def k_grouped(M: int, N: int, G: int = 8, seed: int = 0) -> KGroupedInputs:
    counts = zipf_top8_counts(seed)[:G].astype(np.int64)
    m_indices, T = contiguous_layout(counts)
    valid = m_indices >= 0
    a = np.zeros((M, T), np.uint16)
    b = np.zeros((N, T), np.uint16)
    a[:, valid] = normal_bf16(np.random.default_rng(seed + 0), (M, int(valid.sum())), 1.0)
    b[:, valid] = normal_bf16(np.random.default_rng(seed + 1), (N, int(valid.sum())), 1.0)
    ks = np.array([-(-int(c) // ALIGN_M) * ALIGN_M for c in counts], np.int32)
    return KGroupedInputs(a=a, b=b, ks=ks, counts=counts, M=M, N=N, T=int(T), G=G)


@dataclasses.dataclass
class DequantInputs:
    b: np.ndarray  # bf16 bits [N][K] (quantized once, then dequantized)
    N: int
    K: int


def dequant(N: int, K: int, seed: int = 0, b_std: float = 0.02) -> DequantInputs:
    return DequantInputs(b=normal_bf16(np.random.default_rng(seed + 1), (N, K), b_std), N=N, K=K)


@dataclasses.dataclass
class EpInputs:
    x: np.ndarray      # bf16 bits [T][K]
    topk: np.ndarray   # int32 [T][k] expert ids
    topk_w: np.ndarray  # fp32 [T][k] router weights
    w: np.ndarray      # bf16 bits [E][N][K]
    T: int
    E: int
    k: int
    N: int
    K: int
    M_max: int

    @property
    def counts(self) -> np.ndarray:
        return np.bincount(self.topk.ravel(), minlength=self.E).astype(np.int64)


def expert_parallel(T: int, E: int, k: int, N: int, K: int, M_max: int, seed: int = 0,
                    a_std: float = 1.0, b_std: float = 0.02) -> EpInputs:
    x = normal_bf16(np.random.default_rng(seed + 0), (T, K), a_std)
    w = normal_bf16(np.random.default_rng(seed + 1), (E, N, K), b_std)
    rng = np.random.default_rng(seed + 2)
    g = rng.gumbel(size=(T, E))
    topk = np.argpartition(-g, k - 1, axis=1)[:, :k].astype(np.int32)
    wt = rng.random((T, k)).astype(np.float32)
    wt /= wt.sum(axis=1, keepdims=True)
    return EpInputs(x=x, topk=topk, topk_w=wt, w=w, T=T, E=E, k=k, N=N, K=K, M_max=M_max)


@dataclasses.dataclass
class PeakInputs:
    iters: int  # K blocks per CTA and launch


@dataclasses.dataclass
class QuantInputs:
    a: np.ndarray  # bf16 bits [M][K]
    M: int
    K: int


def quant(M: int, K: int, seed: int = 0, a_std: float = 1.0) -> QuantInputs:
    """Activations alone: the same draw as a dense workload's A (no outliers)."""
    return QuantInputs(a=normal_bf16(np.random.default_rng(seed + 0), (M, K), a_std), M=M, K=K)


def masked(G: int, M_max: int, N: int, K: int, seed: int = 0,
           masked_m: Optional[np.ndarray] = None, a_std: float = 1.0,
           b_std: float = 0.02) -> MaskedInputs:
    a = normal_bf16(np.random.default_rng(seed + 0), (G, M_max, K), a_std)
    b = normal_bf16(np.random.default_rng(seed + 1), (G, N, K), b_std)
    if masked_m is None:
        masked_m = np.random.default_rng(seed + 3).integers(0, M_max + 1, size=G)
    masked_m = np.asarray(masked_m, dtype=np.int32)
    return MaskedInputs(a=a, b=b, masked_m=masked_m, G=G, M_max=M_max, N=N, K=K)


# Named workloads: name -> (kind, constructor kwargs)
WORKLOADS = {
    "dense_128x256x512": ("dense", dict(M=128, N=256, K=512)),
    "decode_64x4096x7168": ("dense", dict(M=64, N=4096, K=7168, outlier_frac=0.01)),
    "prefill_4096x7168x2048": ("dense", dict(M=4096, N=7168, K=2048)),
    "prefill_4096x2112x7168": ("dense", dict(M=4096, N=2112, K=7168)),
    "contiguous_8x4096x7168": ("contiguous", dict(N=4096, K=7168, G=8)),
    "masked_32x256x4096x7168": ("masked", dict(G=32, M_max=256, N=4096, K=7168)),
    # weight dequantization (e4m3 + 128x128 scales -> bf16) of a prefill weight
    "dequant_7168x2048": ("dequant", dict(N=7168, K=2048)),
    # activation quantization (bf16 -> e4m3 + per-token scales) of a prefill input
    "quant_4096x7168": ("quant", dict(M=4096, K=7168)),
    # expert FFN (first GEMM + SwiGLU + requantization, second GEMM)
    "ffn_contiguous_8x7168x2048": ("ffn", dict(H=7168, I=2048, G=8)),
    # K-grouped weight-gradient GEMM of the contiguous workload's experts
    "kgrouped_8x4096x7168": ("kgrouped", dict(M=4096, N=7168, G=8)),
    # the FP8 tensor-core rate (operands generated in shared memory)
    "peak_fp8_mma_16384": ("peak", dict(iters=16384)),
    # the expert-parallel layer around the masked GEMM
    "ep_32x512x8_4096x7168": ("ep", dict(T=512, E=32, k=8, N=4096, K=7168, M_max=256)),
}


def make(name: str, seed: int = 0):
    kind, kw = WORKLOADS[name]
    if kind == "dense":
        return dense(seed=seed, **kw)
    if kind == "contiguous":
        return contiguous(seed=seed, **kw)
    if kind == "dequant":
        return dequant(seed=seed, **kw)
    if kind == "quant":
        return quant(seed=seed, **kw)
    if kind == "ffn":
        return ffn_contiguous(seed=seed, **kw)
    if kind == "kgrouped":
        return k_grouped(seed=seed, **kw)
    if kind == "peak":
        return PeakInputs(**kw)
    if kind == "ep":
        return expert_parallel(seed=seed, **kw)
    return masked(seed=seed, **kw)


def flops_and_bytes(kind: str, inp) -> tuple:
    """Algorithmic FLOPs and HBM bytes of one GEMM call (valid rows only), or of
    one weight dequantization or activation quantization (bytes only).

    FLOPs = 2 * M_valid * N * K. Bytes = A (1 B/elt) + its fp32 scales (one per
    128 elements) + B (1 B/elt) and its fp32 scales (one per 128x128 block) for
    every expert with at least one valid row + D (2 B/elt) over valid rows.
    """
    if kind == "kgrouped":
        # FLOPs over the valid tokens; bytes: both operands and their per-row
        # scales over the padded token range, the fp32 output of every expert
        M, N, T = inp.M, inp.N, inp.T
        tv = int(inp.counts.sum())
        flops = 2.0 * M * N * tv
        byts = (M + N) * T + 4 * (M + N) * (T // 128) + 4 * inp.G * M * N
        return flops, float(byts)
    if kind == "quant":  # bf16 read; codes and one fp32 scale per 128 elements written
        return 0.0, float(3 * inp.M * inp.K + 4 * inp.M * (inp.K // 128))
    if kind == "ffn":
        # both GEMMs; bytes: X and its scales, W1 and W2 with their block
        # scales for every expert with a token, h written and read back with
        # its scales, Y
        H, I = inp.H, inp.I
        mv = int(inp.counts.sum())
        experts = int((inp.counts > 0).sum())
        flops = 2.0 * mv * (2 * I) * H + 2.0 * mv * H * I
        wbytes = experts * (3 * I * H + 4 * ((2 * I // 128) * (H // 128) + (H // 128) * (I // 128)))
        byts = mv * H + 4 * mv * (H // 128) + wbytes + 2 * (mv * I + 4 * mv * (I // 128)) + 2 * mv * H
        return flops, float(byts)
    N, K = inp.N, inp.K
    nb = -(-N // 128)
    kb = K // 128
    if kind == "dequant":  # no FLOPs; codes and scales read, bf16 written
        return 0.0, float(N * K + 4 * nb * kb + 2 * N * K)
    if kind == "dense":
        mv, experts = inp.M, 1
    elif kind == "contiguous":
        mv = int(inp.counts.sum())
        experts = int((inp.counts > 0).sum())
    else:
        mv = int(inp.masked_m.sum())
        experts = int((inp.masked_m > 0).sum())
    flops = 2.0 * mv * N * K
    byts = mv * K + 4 * mv * kb + experts * (N * K + 4 * nb * kb) + 2 * mv * N
    return flops, float(byts)
