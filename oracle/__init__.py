"""CPU oracle for the FP8 block-scaled GEMM (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package. The product library never calls
it, and it shares no code with the CUDA path. The arithmetic lives in
``fp8_oracle.cpp`` (plain C++, fp64 accumulation); this module only builds
that file with g++ and marshals numpy arrays through ctypes.

Layouts here are the logical ones: activation scales ``sa[..., m, kb]`` (token,
then 128-wide K block), weight scales ``sb[g, nb, kb]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib: Optional[ctypes.CDLL] = None

BLOCK = 128


def build(force: bool = False) -> str:
    """Compile fp8_oracle.cpp into liboracle.so (no fast-math, no FP contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
           "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I = ctypes.c_int
    I64 = ctypes.c_int64
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode_array.argtypes = [P, P, I64]
    lib.oracle_e4m3_encode_array.restype = None
    lib.oracle_per_token_cast.argtypes = [P, P, P, I, I, I, I, I]
    lib.oracle_per_block_cast.argtypes = [P, P, P, I, I, I, I, I]
    lib.oracle_per_block_dequant.argtypes = [P, P, P, I, I, I, I]
    lib.oracle_gemm_nt.argtypes = [P, P, P, P, P, I, I, I, I]
    lib.oracle_grouped_contiguous.argtypes = [P, P, P, P, P, P, I, I, I, I, I]
    lib.oracle_grouped_masked.argtypes = [P, P, P, P, P, P, I, I, I, I, I]
    lib.oracle_gemm_points.argtypes = [P, P, P, P, P, P, P, I64, P, I, I, I, I]
    lib.oracle_k_grouped.argtypes = [P, P, P, P, P, P, I, I, I, I, I]
    lib.oracle_k_grouped.restype = ctypes.c_int
    lib.oracle_exp_f32.argtypes = [ctypes.c_float]
    lib.oracle_exp_f32.restype = ctypes.c_float
    lib.oracle_silu_f32.argtypes = [ctypes.c_float]
    lib.oracle_silu_f32.restype = ctypes.c_float
    lib.oracle_swiglu.argtypes = [P, P, P, I64]
    lib.oracle_swiglu.restype = None
    lib.oracle_f64_to_bf16.argtypes = [P, P, I64]
    lib.oracle_f64_to_bf16.restype = None
    for f in ("oracle_per_token_cast", "oracle_per_block_cast", "oracle_gemm_nt",
              "oracle_grouped_contiguous", "oracle_grouped_masked", "oracle_gemm_points",
              "oracle_hardware_threads"):
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments (rc=%d)" % (what, rc))


def hardware_threads() -> int:
    return int(_load().oracle_hardware_threads())


def e4m3_decode(codes) -> np.ndarray:
    """Exact value of each e4m3 code (float64; NaN for 0x7F / 0xFF)."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    tab = np.array([lib.oracle_e4m3_decode(i) for i in range(256)], dtype=np.float64)
    return tab[c]


def e4m3_encode(values) -> np.ndarray:
    """Round float32 values to e4m3 codes (nearest, ties to even, saturating)."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(v), _ptr(out), v.size)
    return out


def per_token_cast(x_bf16: np.ndarray, threads: int = 0, ue8m0: bool = False):
    """x: bf16 bits [M][K] or [G][M][K] -> (codes like x, scales [..., M, K/128]).
    ue8m0: scales rounded up to powers of two (codes of x / s)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    squeeze = x.ndim == 2
    if squeeze:
        x = x[None]
    G, M, K = x.shape
    q = np.empty(x.shape, dtype=np.uint8)
    s = np.empty((G, M, K // BLOCK), dtype=np.float32)
    _check(_load().oracle_per_token_cast(_ptr(x), _ptr(q), _ptr(s), G, M, K, threads,
                                         int(ue8m0)), "per_token_cast")
    return (q[0], s[0]) if squeeze else (q, s)


def per_block_cast(x_bf16: np.ndarray, threads: int = 0, ue8m0: bool = False):
    """x: bf16 bits [N][K] or [G][N][K] -> (codes like x, scales [..., ceil(N/128), K/128]).
    ue8m0: scales rounded up to powers of two (codes of x / s)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    squeeze = x.ndim == 2
    if squeeze:
        x = x[None]
    G, N, K = x.shape
    NB = -(-N // BLOCK)
    q = np.empty(x.shape, dtype=np.uint8)
    s = np.empty((G, NB, K // BLOCK), dtype=np.float32)
    _check(_load().oracle_per_block_cast(_ptr(x), _ptr(q), _ptr(s), G, N, K, threads,
                                         int(ue8m0)), "per_block_cast")
    return (q[0], s[0]) if squeeze else (q, s)


def per_block_dequant(q: np.ndarray, s: np.ndarray, threads: int = 0) -> np.ndarray:
    """codes [N][K] or [G][N][K] with scales [..., ceil(N/128), K/128] -> bf16 bits like q:
    bf16(fp32(e4m3(q) * s)), both roundings to nearest even."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    squeeze = q.ndim == 2
    if squeeze:
        q, s = q[None], s[None]
    G, N, K = q.shape
    if s.shape != (G, -(-N // BLOCK), K // BLOCK):
        raise ValueError("scale shape %s does not match codes %s" % (s.shape, q.shape))
    x = np.empty(q.shape, dtype=np.uint16)
    _check(_load().oracle_per_block_dequant(_ptr(q), _ptr(s), _ptr(x), G, N, K, threads),
           "per_block_dequant")
    return x[0] if squeeze else x


def gemm_nt(qa, sa, qb, sb, threads: int = 0) -> np.ndarray:
    """D[m][n] (fp64) of the dense block-scaled GEMM."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    M, K = qa.shape
    N = qb.shape[0]
    assert qb.shape[1] == K and sa.shape == (M, K // BLOCK)
    assert sb.shape == (-(-N // BLOCK), K // BLOCK)
    out = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_gemm_nt(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), _ptr(out),
                                  M, N, K, threads), "gemm_nt")
    return out


def grouped_contiguous(qa, sa, qb, sb, m_indices, threads: int = 0) -> np.ndarray:
    """D[m][n] (fp64) of the contiguous grouped GEMM; NaN on padding rows."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    mi = np.ascontiguousarray(m_indices, dtype=np.int32)
    M_total, K = qa.shape
    G, N, _ = qb.shape
    out = np.empty((M_total, N), dtype=np.float64)
    _check(_load().oracle_grouped_contiguous(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), _ptr(mi),
                                             _ptr(out), M_total, N, K, G, threads),
           "grouped_contiguous")
    return out


def grouped_masked(qa, sa, qb, sb, masked_m, threads: int = 0) -> np.ndarray:
    """D[e][m][n] (fp64) of the masked grouped GEMM; NaN on rows >= masked_m[e]."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    mm = np.ascontiguousarray(masked_m, dtype=np.int32)
    G, M_max, K = qa.shape
    N = qb.shape[1]
    out = np.empty((G, M_max, N), dtype=np.float64)
    _check(_load().oracle_grouped_masked(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), _ptr(mm),
                                         _ptr(out), G, M_max, N, K, threads), "grouped_masked")
    return out


def gemm_points(qa, sa, qb, sb, a_rows, experts, cols, threads: int = 0) -> np.ndarray:
    """Selected outputs: element p = row a_rows[p] of (qa, sa) against row cols[p]
    of expert experts[p]. qa [R][K], sa [R][K/128], qb [G][N][K] (or [N][K]),
    sb [G][NB][KB] (or [NB][KB])."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8).reshape(-1, np.shape(qa)[-1])
    K = qa.shape[1]
    sa = np.ascontiguousarray(sa, dtype=np.float32).reshape(-1, K // BLOCK)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    if qb.ndim == 2:
        qb = qb[None]
        sb = sb[None]
    G, N, _ = qb.shape
    r = np.ascontiguousarray(a_rows, dtype=np.int64)
    e = np.ascontiguousarray(experts, dtype=np.int64)
    n = np.ascontiguousarray(cols, dtype=np.int64)
    assert r.shape == e.shape == n.shape
    assert r.size == 0 or int(r.max()) < qa.shape[0]
    out = np.empty(r.shape, dtype=np.float64)
    _check(_load().oracle_gemm_points(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), _ptr(r), _ptr(e),
                                      _ptr(n), r.size, _ptr(out), N, K, G, threads),
           "gemm_points")
    return out


# ---------------------------------------------------------------- expert FFN

def exp_f32(x) -> np.ndarray:
    """exp in fp32 by the oracle's fixed operation sequence (elementwise)."""
    lib = _load()
    x = np.asarray(x, np.float32)
    return np.array([lib.oracle_exp_f32(float(v)) for v in x.ravel()], np.float32).reshape(x.shape)


def silu_f32(x) -> np.ndarray:
    """silu(g) = g / (1 + exp(-g)) in fp32 (elementwise)."""
    lib = _load()
    x = np.asarray(x, np.float32)
    return np.array([lib.oracle_silu_f32(float(v)) for v in x.ravel()], np.float32).reshape(x.shape)


def swiglu(g_bits: np.ndarray, u_bits: np.ndarray) -> np.ndarray:
    """h = bf16(silu(gate) * up) for bf16 bit patterns of equal shape."""
    g = np.ascontiguousarray(g_bits, np.uint16)
    u = np.ascontiguousarray(u_bits, np.uint16)
    assert g.shape == u.shape
    h = np.empty_like(g)
    _load().oracle_swiglu(_ptr(g), _ptr(u), _ptr(h), g.size)
    return h


def f64_to_bf16(v: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of fp64 values (nearest even, one rounding)."""
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    _load().oracle_f64_to_bf16(_ptr(v), _ptr(out), v.size)
    return out


def moe_ffn_contiguous(xq, sx, w1q, sw1, w2q, sw2, m_indices, threads: int = 0):
    """Expert FFN on the contiguous layout with power-of-two scales: the first
    grouped GEMM (W1 rows: I gate rows, then I up rows), its result rounded to
    bf16, h = swiglu(gate, up), h quantized per token per 128 channels with
    power-of-two scales, the second grouped GEMM. Returns (gu_bits [M][2I],
    hq [M][I], sh [M][I/128], y fp64 [M][H]); rows with m_indices < 0 are
    undefined, as in the grouped GEMM (NaN values, NaN codes 0x7F), and are
    ignored by callers."""
    I = w1q.shape[1] // 2
    gu = f64_to_bf16(grouped_contiguous(xq, sx, w1q, sw1, m_indices, threads))
    h = swiglu(gu[:, :I], gu[:, I:])
    hq, sh = per_token_cast(h, threads=threads, ue8m0=True)
    y = grouped_contiguous(hq, sh, w2q, sw2, m_indices, threads)
    return gu, hq, sh, y


def moe_ffn_masked(xq, sx, w1q, sw1, w2q, sw2, masked_m, threads: int = 0):
    """The same chain on the masked layout ([G][M_max][...] slabs)."""
    G, M_max, _ = xq.shape
    I = w1q.shape[1] // 2
    y1 = grouped_masked(xq, sx, w1q, sw1, masked_m, threads)
    for e in range(G):  # rows past masked_m are not computed: their intermediate is zero
        y1[e, int(masked_m[e]):] = 0.0
    gu = f64_to_bf16(y1)
    h = swiglu(gu[..., :I], gu[..., I:])
    hq, sh = per_token_cast(h, threads=threads, ue8m0=True)
    y = grouped_masked(hq, sh, w2q, sw2, masked_m, threads)
    return gu, hq, sh, y


# ---------------------------------------------------------------- K-grouped GEMM

def k_grouped(qa, sa, qb, sb, ks, threads: int = 0) -> np.ndarray:
    """D[e][m][n] (fp64) of the K-grouped GEMM: qa [M][T], sa [M][T/128],
    qb [N][T], sb [N][T/128] (one scale per row per 128-token block on both
    sides), ks [G] token counts (multiples of 128, summing to T)."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    ks = np.ascontiguousarray(ks, dtype=np.int32)
    M, T = qa.shape
    N = qb.shape[0]
    G = ks.size
    assert qb.shape[1] == T and sa.shape == (M, T // BLOCK) and sb.shape == (N, T // BLOCK)
    out = np.empty((G, M, N), dtype=np.float64)
    _check(_load().oracle_k_grouped(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), _ptr(ks), _ptr(out),
                                    G, M, N, T, threads), "k_grouped")
    return out
