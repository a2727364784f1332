"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: the OCP E4M3
definition points, torch's independent float8_e4m3fn codec, hand-worked
fixtures, closed forms, integer special cases that reduce to a plain matmul,
and algebraic invariants (swap symmetry, grouping consistency, the relation
between block and token scales).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def torch_decode(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def torch_encode(values: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


ALL_CODES = np.arange(256, dtype=np.uint8)
FINITE_CODES = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


# ---------------------------------------------------------------- e4m3 codec

def test_decode_matches_ocp_definition_points():
    path = os.path.join(GOLDEN, "e4m3_ocp_points.txt")
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code_s, val_s = line.split()
        code = int(code_s, 16)
        got = float(oracle.e4m3_decode(np.array([code], np.uint8))[0])
        if val_s == "nan":
            assert math.isnan(got), hex(code)
        else:
            want = float(val_s)
            assert got == want and math.copysign(1, got) == math.copysign(1, want), hex(code)


def test_decode_all_codes_match_torch():
    ours = oracle.e4m3_decode(ALL_CODES)
    ref = torch_decode(ALL_CODES)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_encode_decode_roundtrip_every_finite_code():
    vals = oracle.e4m3_decode(FINITE_CODES).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), FINITE_CODES)


def test_encode_ties_go_to_even_code():
    pos = np.arange(0, 0x7F, dtype=np.uint8)  # 0x00 .. 0x7E, increasing values
    v = oracle.e4m3_decode(pos)
    mid = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (v[:-1] + v[1:]) / 2)  # exact in fp32
    got = oracle.e4m3_encode(mid)
    lo = pos[:-1]
    even = np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8)
    assert np.array_equal(got, even)
    assert np.array_equal(oracle.e4m3_encode(-mid), even | 0x80)


def test_encode_matches_torch_on_random_values():
    rng = np.random.default_rng(123)
    # log-uniform magnitudes from deep subnormal to the saturation midpoint
    mag = np.exp(rng.uniform(np.log(1e-5), np.log(463.9), size=200000)).astype(np.float32)
    sgn = np.where(rng.random(mag.size) < 0.5, -1, 1).astype(np.float32)
    vals = np.concatenate([mag * sgn, np.float32([0.0, -0.0, 464.0, -464.0])])
    assert np.array_equal(oracle.e4m3_encode(vals), torch_encode(vals))


def test_encode_saturates_at_448():
    vals = np.float32([448.0, 449.0, 464.0, 465.0, 1e6, 3e38, -500.0, -1e30])
    got = oracle.e4m3_encode(vals)
    assert np.array_equal(got, np.uint8([0x7E] * 6 + [0xFE] * 2))
    assert oracle.e4m3_encode(np.float32([np.nan]))[0] == 0x7F


# ---------------------------------------------------------------- quantizers

def _ulp_e4m3(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (e - 3))


def test_per_token_worked_example():
    path = os.path.join(GOLDEN, "per_token_worked_example.txt")
    x = np.zeros(128, np.float32)
    x[:4] = [3.5, -1.75, 0.5, 0.001]
    q, s = oracle.per_token_cast(workloads.bf16_bits(x)[None, :])
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b = line.split()
        if a == "scale":
            assert s[0, 0] == np.float32(float(b))
        else:
            assert q[0, int(a)] == int(b, 16), a


def test_per_token_invariants():
    rng = np.random.default_rng(7)
    M, K = 37, 512
    x = rng.standard_normal((M, K), dtype=np.float32)
    x[3] *= 30.0
    x[5, 128:256] = 0.0                      # an all-zero slice
    x[6, :128] *= 1e-6                       # a slice far below 1e-4 amax
    bits = workloads.bf16_bits(x)
    xf = workloads.bf16_to_f32(bits).astype(np.float64)
    q, s = oracle.per_token_cast(bits)
    assert q.shape == (M, K) and s.shape == (M, K // 128)
    deq = oracle.e4m3_decode(q).reshape(M, K // 128, 128)
    xs = xf.reshape(M, K // 128, 128)
    amax = np.abs(xs).max(axis=2)
    live = amax >= 1e-4
    # the scale is amax/448 (one fp32 rounding), floored at 1e-4/448
    np.testing.assert_allclose(s[live].astype(np.float64) * 448.0, amax[live], rtol=2 ** -23)
    assert np.all(s[~live] == np.float32(1e-4) / np.float32(448.0))
    # the element holding the slice's amax lands on +-448
    idx = np.abs(xs).argmax(axis=2)
    top = np.take_along_axis(deq, idx[..., None], axis=2)[..., 0]
    assert np.all(np.abs(top[live]) == 448.0)
    # reconstruction error: at most half an e4m3 ulp of x/s (plus fp32 slop)
    y = xs / s[..., None].astype(np.float64)
    err = np.abs(y - deq)
    assert np.all(err <= 0.5 * _ulp_e4m3(y) * (1 + 1e-6) + 1e-9)
    # the all-zero slice encodes to zero codes
    assert np.all(q[5, 128:256] == 0)


def test_slices_with_infinities_and_nan():
    """A slice holding +-inf has amax = inf, so its scale is +inf in both modes
    and every element maps to x / inf: finite elements to a zero code with
    their own sign, infinities (inf / inf) and NaN to the NaN code 0x7F. NaN
    elements do not raise the amax; a slice of NaN and finite values quantizes
    like its finite values."""
    x = np.zeros((2, 256), np.float32)
    x[0, :128] = np.linspace(-3.0, 3.0, 128, dtype=np.float32)
    x[0, 7], x[0, 9], x[0, 11] = np.inf, -np.inf, np.nan
    x[1, :128] = np.linspace(-1.0, 1.0, 128, dtype=np.float32)
    x[1, 40] = np.nan
    x[:, 128:] = np.linspace(0.5, 2.0, 128, dtype=np.float32)
    bits = workloads.bf16_bits(np.nan_to_num(x, nan=0.0, posinf=0.0, neginf=0.0))
    bits[0, 7], bits[0, 9], bits[0, 11], bits[1, 40] = 0x7F80, 0xFF80, 0x7FC0, 0x7FC0
    finite = workloads.bf16_to_f32(bits)
    for ue8m0 in (False, True):
        q, s = oracle.per_token_cast(bits, ue8m0=ue8m0)
        assert np.isposinf(s[0, 0])
        expect = np.where(np.signbit(finite[0, :128]), 0x80, 0x00).astype(np.uint8)
        expect[[7, 9, 11]] = 0x7F
        assert np.array_equal(q[0, :128], expect)
        # the NaN element alone is 0x7F; the rest quantizes as without it
        clean = bits[1:2, :128].copy()
        clean[0, 40] = 0
        qc, sc = oracle.per_token_cast(clean, ue8m0=ue8m0)
        assert s[1, 0] == sc[0, 0] and q[1, 40] == 0x7F
        rest = np.arange(128) != 40
        assert np.array_equal(q[1, :128][rest], qc[0][rest])
        # the other slices are untouched
        q2, s2 = oracle.per_token_cast(bits[:, 128:], ue8m0=ue8m0)
        assert np.array_equal(q[:, 128:], q2) and np.array_equal(s[:, 1:], s2)


def test_per_token_power_of_two_slices_are_exact():
    K = 256
    j = np.arange(-14, 2)                          # 16 powers of two, max 2
    vals = np.concatenate([2.0 ** j, -(2.0 ** j)]).astype(np.float32)
    x = np.tile(vals, K // vals.size + 1)[:K][None, :]
    q, s = oracle.per_token_cast(workloads.bf16_bits(x))
    want = 448.0 * x[0].astype(np.float64) / 2.0     # amax = 2 in every slice
    assert np.array_equal(oracle.e4m3_decode(q[0]), want)


def test_per_block_relates_to_per_token():
    """The block scale is the max of the 128 row scales of that block (amax is
    a max and the scale map is monotone); N tail blocks use only their rows."""
    rng = np.random.default_rng(11)
    for N in (256, 192, 64, 130):
        K = 384
        x = workloads.bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * 0.02)
        qb, sb = oracle.per_block_cast(x)
        _, st = oracle.per_token_cast(x)
        NB = -(-N // 128)
        assert sb.shape == (NB, K // 128)
        for nb in range(NB):
            rows = st[nb * 128:min(N, nb * 128 + 128)]
            assert np.array_equal(sb[nb], rows.max(axis=0))
        # a tail block quantizes exactly like a stand-alone matrix of its rows
        if N % 128:
            q2, s2 = oracle.per_block_cast(x[(NB - 1) * 128:])
            assert np.array_equal(q2, qb[(NB - 1) * 128:])
            assert np.array_equal(s2[0], sb[NB - 1])


def test_per_block_invariants_and_groups():
    rng = np.random.default_rng(5)
    G, N, K = 3, 256, 256
    x = workloads.bf16_bits(rng.standard_normal((G, N, K), dtype=np.float32) * 0.02)
    q, s = oracle.per_block_cast(x)
    for g in range(G):
        qg, sg = oracle.per_block_cast(x[g])
        assert np.array_equal(qg, q[g]) and np.array_equal(sg, s[g])
    xf = workloads.bf16_to_f32(x).astype(np.float64).reshape(G, 2, 128, 2, 128)
    amax = np.abs(xf).max(axis=(2, 4))
    np.testing.assert_allclose(s.astype(np.float64) * 448.0, amax, rtol=2 ** -23)
    deq = oracle.e4m3_decode(q).reshape(G, 2, 128, 2, 128)
    y = xf / s[:, :, None, :, None].astype(np.float64)
    assert np.all(np.abs(y - deq) <= 0.5 * _ulp_e4m3(y) * (1 + 1e-6) + 1e-9)


# ---------------------------------------------------------------- GEMM

def _expand_sa(sa):       # [M][KB] -> [M][K]
    return np.repeat(sa.astype(np.float64), 128, axis=1)


def _expand_sb(sb, N):    # [NB][KB] -> [N][K]
    return np.repeat(np.repeat(sb.astype(np.float64), 128, axis=0)[:N], 128, axis=1)


def _small_int_codes(rng, shape):
    vals = rng.integers(-2, 3, size=shape).astype(np.float32)
    return torch_encode(vals), vals.astype(np.int64)


def test_gemm_integer_case_unit_scales_is_integer_matmul():
    rng = np.random.default_rng(1)
    M, N, K = 40, 200, 256
    qa, ia = _small_int_codes(rng, (M, K))
    qb, ib = _small_int_codes(rng, (N, K))
    sa = np.ones((M, 2), np.float32)
    sb = np.ones((2, 2), np.float32)
    got = oracle.gemm_nt(qa, sa, qb, sb)
    assert np.array_equal(got, (ia @ ib.T).astype(np.float64))


def test_gemm_integer_case_power_of_two_scales_exact():
    rng = np.random.default_rng(2)
    M, N, K = 33, 160, 256
    qa, ia = _small_int_codes(rng, (M, K))
    qb, ib = _small_int_codes(rng, (N, K))
    sa = (2.0 ** rng.integers(-3, 3, size=(M, 2))).astype(np.float32)
    sb = (2.0 ** rng.integers(-3, 3, size=(2, 2))).astype(np.float32)
    got = oracle.gemm_nt(qa, sa, qb, sb)
    ref = (ia * _expand_sa(sa)) @ (ib * _expand_sb(sb, N)).T
    assert np.array_equal(got, ref)


def test_gemm_closed_form_all_ones():
    M, N, K = 5, 300, 640
    qa = np.full((M, K), 0x38, np.uint8)     # 1.0
    qb = np.full((N, K), 0x38, np.uint8)
    sa = np.full((M, K // 128), 0.375, np.float32)
    sb = np.full((3, K // 128), 0.0625, np.float32)
    got = oracle.gemm_nt(qa, sa, qb, sb)
    assert np.all(got == K * 0.375 * 0.0625)


def test_gemm_random_matches_scaled_operand_product():
    """The blocked definition equals one fp64 matmul of the scaled, dequantized
    operands (decoded by torch); a wrong block index or operand fails it."""
    rng = np.random.default_rng(3)
    M, N, K = 70, 300, 512
    xa = workloads.bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    xb = workloads.bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * 0.02)
    qa, sa = oracle.per_token_cast(xa)
    qb, sb = oracle.per_block_cast(xb)
    got = oracle.gemm_nt(qa, sa, qb, sb)
    ref = (torch_decode(qa) * _expand_sa(sa)) @ (torch_decode(qb) * _expand_sb(sb, N)).T
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_gemm_brute_force_long_double_tiny():
    rng = np.random.default_rng(4)
    M, N, K = 6, 9, 256
    qa = rng.integers(0, 256, size=(M, K)).astype(np.uint8)
    qb = rng.integers(0, 256, size=(N, K)).astype(np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x3F
    qb[(qb & 0x7F) == 0x7F] = 0x3F
    sa = rng.uniform(0.001, 0.01, size=(M, 2)).astype(np.float32)
    sb = rng.uniform(1e-4, 1e-3, size=(1, 2)).astype(np.float32)
    da = torch_decode(qa).astype(np.longdouble)
    db = torch_decode(qb).astype(np.longdouble)
    ref = np.zeros((M, N), np.longdouble)
    for m in range(M):
        for n in range(N):
            tot = np.longdouble(0)
            for k in range(K):
                tot += (da[m, k] * np.longdouble(sa[m, k // 128])) * (db[n, k] * np.longdouble(sb[n // 128, k // 128]))
            ref[m, n] = tot
    got = oracle.gemm_nt(qa, sa, qb, sb)
    np.testing.assert_allclose(got, ref.astype(np.float64), rtol=1e-13, atol=1e-300)


def test_gemm_swap_symmetry():
    """With activation scales constant over 128-row groups, gemm(A,B)^T equals
    gemm(B,A) with the two scale roles exchanged (the identity swapAB uses)."""
    rng = np.random.default_rng(6)
    M, N, K = 256, 384, 384
    qa = torch_encode(rng.standard_normal((M, K)).astype(np.float32) * 8)
    qb = torch_encode(rng.standard_normal((N, K)).astype(np.float32) * 8)
    sa_blk = rng.uniform(0.01, 0.02, size=(M // 128, K // 128)).astype(np.float32)
    sb = rng.uniform(0.001, 0.002, size=(N // 128, K // 128)).astype(np.float32)
    sa = np.repeat(sa_blk, 128, axis=0)
    sb_rows = np.repeat(sb, 128, axis=0)
    d = oracle.gemm_nt(qa, sa, qb, sb)
    dt = oracle.gemm_nt(qb, sb_rows, qa, sa_blk)
    assert np.array_equal(d.T, dt)


def test_grouped_forms_equal_per_expert_dense():
    rng = np.random.default_rng(8)
    N, K = 192, 256
    counts = np.array([130, 0, 5, 128])
    inp = workloads.contiguous(N, K, counts=counts, seed=3)
    qa, sa = oracle.per_token_cast(inp.a)
    qb, sb = oracle.per_block_cast(inp.b)
    out = oracle.grouped_contiguous(qa, sa, qb, sb, inp.m_indices)
    assert out.shape == (inp.M_total, N)
    assert np.all(np.isnan(out[inp.m_indices < 0]))
    for g in range(len(counts)):
        rows = np.nonzero(inp.m_indices == g)[0]
        if rows.size == 0:
            continue
        ref = oracle.gemm_nt(qa[rows], sa[rows], qb[g], sb[g])
        assert np.array_equal(out[rows], ref)

    G, M_max = 3, 80
    minp = workloads.masked(G, M_max, N, K, seed=4, masked_m=np.array([0, 80, 17]))
    qa3, sa3 = oracle.per_token_cast(minp.a)
    qb3, sb3 = oracle.per_block_cast(minp.b)
    out3 = oracle.grouped_masked(qa3, sa3, qb3, sb3, minp.masked_m)
    for e in range(G):
        mv = int(minp.masked_m[e])
        assert np.all(np.isnan(out3[e, mv:]))
        if mv:
            ref = oracle.gemm_nt(qa3[e, :mv], sa3[e, :mv], qb3[e], sb3[e])
            assert np.array_equal(out3[e, :mv], ref)


def test_points_equal_full_gemm():
    rng = np.random.default_rng(9)
    M, N, K, G = 50, 130, 384, 2
    xa = workloads.bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    xb = workloads.bf16_bits(rng.standard_normal((G, N, K), dtype=np.float32) * 0.02)
    qa, sa = oracle.per_token_cast(xa)
    qb, sb = oracle.per_block_cast(xb)
    r = rng.integers(0, M, 300)
    e = rng.integers(0, G, 300)
    n = rng.integers(0, N, 300)
    pts = oracle.gemm_points(qa, sa, qb, sb, r, e, n)
    full = [oracle.gemm_nt(qa, sa, qb[g], sb[g]) for g in range(G)]
    assert np.array_equal(pts, np.array([full[ei][ri, ni] for ri, ei, ni in zip(r, e, n)]))


def test_oracle_rejects_bad_sizes():
    with pytest.raises(ValueError):
        oracle.per_token_cast(np.zeros((4, 100), np.uint16))


# ---------------------------------------------------------------- weight dequantization

def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def _block_scales(s: np.ndarray, N: int) -> np.ndarray:
    """[G][NB][KB] block scales expanded to [G][N][K]."""
    return np.repeat(np.repeat(s, 128, axis=1)[:, :N], 128, axis=2)


def _finite_codes(rng, shape):
    q = rng.integers(0, 256, size=shape, dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x00
    return q


def test_dequant_power_of_two_scales_exact():
    """Power-of-two scales: product and bf16 rounding are exact, so every
    output is the code's value (torch's independent decoder) times the scale
    of its 128x128 block. N = 200 has a ragged last block; two groups."""
    rng = np.random.default_rng(3)
    G, N, K = 2, 200, 256
    q = _finite_codes(rng, (G, N, K))
    s = np.ldexp(1.0, rng.integers(-8, 8, size=(G, 2, 2))).astype(np.float32)
    got = _bf16_to_f64(oracle.per_block_dequant(q, s))
    assert np.array_equal(got, torch_decode(q) * _block_scales(s, N))


def test_dequant_matches_torch_casts():
    """General fp32 scales: torch's float8 decode, one float32 multiply and
    torch's round-to-nearest-even bfloat16 cast give the same bits."""
    rng = np.random.default_rng(4)
    G, N, K = 1, 300, 384
    q = _finite_codes(rng, (G, N, K))
    s = (rng.random((G, 3, 3)) * 0.01 + 1e-4).astype(np.float32)
    dec = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float32)
    want = (dec * torch.from_numpy(_block_scales(s, N).astype(np.float32))).to(torch.bfloat16)
    got = oracle.per_block_dequant(q, s)
    assert np.array_equal(got, want.view(torch.int16).numpy().view(np.uint16))


def test_dequant_block_indexing():
    """Every code 1.0 and a distinct power-of-two scale per block: each output
    equals its own block's scale (a swapped or shifted block index fails)."""
    G, N, K = 2, 300, 384
    q = np.full((G, N, K), 0x38, np.uint8)
    s = np.ldexp(1.0, np.arange(G * 3 * 3).reshape(G, 3, 3) - 9).astype(np.float32)
    got = _bf16_to_f64(oracle.per_block_dequant(q, s))
    for g in range(G):
        for nb in range(3):
            for kb in range(3):
                blk = got[g, nb * 128:min(N, nb * 128 + 128), kb * 128:kb * 128 + 128]
                assert np.all(blk == float(s[g, nb, kb]))


def test_dequant_inverts_quantizer():
    """dequant(per_block_cast(x)) is within half an e4m3 unit of x (relative
    2^-4, or 2^-10 * s in the subnormal range) plus the bf16 rounding."""
    rng = np.random.default_rng(5)
    x = workloads.bf16_bits(rng.standard_normal((300, 512), dtype=np.float32) * 0.02)
    q, s = oracle.per_block_cast(x)
    y = _bf16_to_f64(oracle.per_block_dequant(q, s))
    xv = _bf16_to_f64(x)
    sf = _block_scales(s[None], 300)[0].astype(np.float64)
    bound = 2.0 ** -4 * np.abs(xv) + 2.0 ** -10 * sf + 2.0 ** -8 * np.abs(y)
    assert np.all(np.abs(xv - y) <= bound)


def test_dequant_nan_code_gives_nan():
    q = np.zeros((128, 128), np.uint8)
    q[3, 5], q[7, 9] = 0x7F, 0xFF
    y = _bf16_to_f64(oracle.per_block_dequant(q, np.ones((1, 1), np.float32)))
    assert np.isnan(y[3, 5]) and np.isnan(y[7, 9])
    assert np.count_nonzero(np.isnan(y)) == 2


# ---------------------------------------------------------------- power-of-two (UE8M0) scales

def _ue8m0_input(rng, shape):
    x = rng.standard_normal(shape, dtype=np.float32)
    x[..., 0, :128] = 0.0                 # all-zero slice: amax floor
    x[..., 1, :] *= 1e-6                  # tiny row
    x[..., 2, :] *= 300.0                 # large row
    x[..., 3, 7] = 448.0 * 2.0 ** -5      # amax exactly 448 * 2^-5: scale exactly 2^-5
    x[..., 3, 8:128] = 0.0
    return workloads.bf16_bits(x)


def _smallest_pow2_at_least(r: np.ndarray) -> np.ndarray:
    m, e = np.frexp(r.astype(np.float64))          # r = m * 2^e, m in [0.5, 1)
    return np.where(m == 0.5, r.astype(np.float64), np.ldexp(1.0, e))


def test_ue8m0_token_scales_are_smallest_sufficient_powers_of_two():
    rng = np.random.default_rng(41)
    x = _ue8m0_input(rng, (2, 6, 512))
    q, s = oracle.per_token_cast(x, ue8m0=True)
    xv = _bf16_to_f64(x).astype(np.float32).reshape(2, 6, 4, 128)
    amax = np.maximum(np.abs(xv).max(axis=-1), np.float32(1e-4)).astype(np.float32)
    r = (amax / np.float32(448.0)).astype(np.float32)
    assert np.array_equal(s.astype(np.float64), _smallest_pow2_at_least(r))
    assert s[0, 3, 0] == 2.0 ** -5


def test_ue8m0_token_codes_are_x_over_s_rounded():
    """x / s is exact (s a power of two) and at most 448 in magnitude; the codes
    are torch's independent encoding of it."""
    rng = np.random.default_rng(42)
    x = _ue8m0_input(rng, (6, 384))
    q, s = oracle.per_token_cast(x, ue8m0=True)
    y = (_bf16_to_f64(x) / np.repeat(s, 128, axis=1)).astype(np.float32)
    assert np.all(np.abs(y) <= 448.0)
    assert np.array_equal(q, torch_encode(y))


def test_ue8m0_block_scales_and_codes():
    rng = np.random.default_rng(43)
    x = workloads.bf16_bits(rng.standard_normal((300, 256), dtype=np.float32) * 0.02)
    q, s = oracle.per_block_cast(x, ue8m0=True)
    xv = _bf16_to_f64(x)
    for nb in range(3):
        for kb in range(2):
            blk = xv[nb * 128:min(300, nb * 128 + 128), kb * 128:kb * 128 + 128].astype(np.float32)
            amax = np.float32(max(float(np.abs(blk).max()), 1e-4))
            want = _smallest_pow2_at_least(np.array([amax / np.float32(448.0)], np.float32))[0]
            assert s[nb, kb] == want
    y = (xv / _block_scales(s[None], 300)[0]).astype(np.float32)
    assert np.array_equal(q, torch_encode(y))


def test_ue8m0_round_trip_within_half_unit():
    rng = np.random.default_rng(44)
    x = workloads.bf16_bits(rng.standard_normal((256, 512), dtype=np.float32))
    q, s = oracle.per_block_cast(x, ue8m0=True)
    y = _bf16_to_f64(oracle.per_block_dequant(q, s))
    xv = _bf16_to_f64(x)
    sf = _block_scales(s[None], 256)[0].astype(np.float64)
    assert np.all(np.abs(xv - y) <= 2.0 ** -4 * np.abs(xv) + 2.0 ** -10 * sf + 2.0 ** -8 * np.abs(y))


# ---------------------------------------------------------------- expert FFN pieces

def _ulp32(x):
    x = np.abs(np.asarray(x, np.float32))
    return np.spacing(x).astype(np.float64)


def test_exp_f32_within_two_ulp_of_exp():
    """The fixed-sequence fp32 exp against the fp64 exp over its whole
    unclamped range (a wrong constant, a dropped Taylor term or a wrong
    exponent reassembly fails this)."""
    x = np.linspace(-87.0, 88.0, 40001).astype(np.float32)
    got = oracle.exp_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    err = np.abs(got - ref) / _ulp32(ref)
    assert err.max() <= 2.0, err.max()


def test_exp_f32_exact_points_and_clamp():
    assert oracle.exp_f32(np.float32(0.0)) == 1.0
    k = np.arange(-120, 121).astype(np.float32)
    x = (k.astype(np.float64) * np.log(2.0)).astype(np.float32)
    got = oracle.exp_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    assert np.all(np.abs(got - ref) <= 2 * _ulp32(ref))
    assert oracle.exp_f32(np.float32(200.0)) == oracle.exp_f32(np.float32(88.0))
    assert oracle.exp_f32(np.float32(-200.0)) == oracle.exp_f32(np.float32(-87.0))


def test_silu_identities():
    """silu(0) = 0; silu(x) - silu(-x) = x; silu(x) = x once exp(-x) is below
    half an ulp of 1; close to the fp64 formula."""
    assert oracle.silu_f32(np.float32(0.0)) == 0.0
    x = np.linspace(0.01, 15.0, 3001).astype(np.float32)
    d = oracle.silu_f32(x).astype(np.float64) - oracle.silu_f32(-x).astype(np.float64)
    assert np.all(np.abs(d - x) <= 4 * _ulp32(x))
    big = np.array([17.0, 20.0, 100.0, 3e4], np.float32)
    assert np.array_equal(oracle.silu_f32(big), big)
    xs = np.linspace(-30.0, 30.0, 6001).astype(np.float32)
    ref = xs.astype(np.float64) / (1.0 + np.exp(-xs.astype(np.float64)))
    got = oracle.silu_f32(xs).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 4 * _ulp32(ref) + 1e-45)


def _bf16_neighbours(v):
    """The two bf16 values around each fp64 v (from fp32 bit patterns)."""
    f = np.asarray(v, np.float64).astype(np.float32)
    b = f.view(np.uint32) & np.uint32(0xFFFF0000)
    lo = b.view(np.float32).astype(np.float64)
    hi = (b + np.uint32(0x10000)).view(np.float32).astype(np.float64)
    return lo, hi


def test_f64_to_bf16_single_rounding():
    """Hand cases (ties to even, subnormal, overflow) and random values against
    the nearest of the two neighbouring bf16 values (ties to even)."""
    cases = {1.0: 0x3F80, 1 + 2 ** -8: 0x3F80, 1 + 3 * 2 ** -8: 0x3F82, -2.5: 0xC020,
             1e-40: 0x0001, 3.39e38: 0x7F7F, 3.4e38: 0x7F80, 0.0: 0x0000}
    got = oracle.f64_to_bf16(np.array(list(cases)))
    assert got.tolist() == list(cases.values())
    rng = np.random.default_rng(21)
    v = rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))
    v = v[np.abs(v) > 1e-30]
    got = oracle.f64_to_bf16(v)
    gv = (got.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    lo, hi = _bf16_neighbours(np.abs(v))
    a = np.abs(v)
    nearest = np.where(a - lo < hi - a, lo, hi)
    tie = (a - lo) == (hi - a)
    even = np.where(((lo.astype(np.float32).view(np.uint32) >> 16) & 1) == 0, lo, hi)
    nearest = np.where(tie, even, nearest) * np.sign(v)
    assert np.array_equal(gv, nearest)


def test_swiglu_against_fp64_formula():
    """h = bf16(silu(g) * u): equal to the bf16 rounding of the fp64 formula
    except where the fp32 evaluation sits within a few ulp of a rounding
    boundary (then the neighbouring bf16 value)."""
    rng = np.random.default_rng(22)
    g = workloads.bf16_bits(rng.standard_normal(20000).astype(np.float32) * 3)
    u = workloads.bf16_bits(rng.standard_normal(20000).astype(np.float32))
    h = oracle.swiglu(g, u)
    gf = (g.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    uf = (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    ref = oracle.f64_to_bf16(gf / (1.0 + np.exp(-gf)) * uf)
    diff = np.abs(h.astype(np.int64) - ref.astype(np.int64))
    assert np.all(diff <= 1) and np.mean(diff == 0) > 0.999


def test_ffn_chain_closed_form():
    """All-ones operands: gate = 2, up = 1, so h = bf16(silu(2)) = 1.765625;
    its power-of-two scale is 2^-7 (1.7656/448 is just above 2^-8) and its code
    e4m3(226) = 224; with all-ones W2 at scale 2^-7 every output is
    I * 224 * 2^-7 * 2^-7 = 1.75 (I = 128)."""
    H = I = 128
    M = 5
    xq = np.full((M, H), 0x38, np.uint8)
    sx = np.full((M, 1), 2.0 ** -7, np.float32)
    w1q = np.full((1, 2 * I, H), 0x38, np.uint8)
    sw1 = np.array([[[2.0], [1.0]]], np.float32)  # gate block x2, up block x1
    w2q = np.full((1, H, I), 0x38, np.uint8)
    sw2 = np.full((1, 1, 1), 2.0 ** -7, np.float32)
    mi = np.zeros(M, np.int32)
    gu, hq, sh, y = oracle.moe_ffn_contiguous(xq, sx, w1q, sw1, w2q, sw2, mi)
    assert np.all(gu[:, :I] == 0x4000) and np.all(gu[:, I:] == 0x3F80)   # 2.0, 1.0
    assert np.all(sh == 2.0 ** -7)
    assert np.all(hq == oracle.e4m3_encode(np.float32(224.0)))
    assert np.all(y == 1.75)


def test_ffn_masked_matches_contiguous_per_expert():
    """The masked chain equals the contiguous chain on each expert's valid rows."""
    rng = np.random.default_rng(23)
    G, M_max, H, I = 2, 40, 256, 128
    mm = np.array([40, 17], np.int32)
    x = workloads.bf16_bits(rng.standard_normal((G, M_max, H)).astype(np.float32))
    xq, sx = oracle.per_token_cast(x, ue8m0=True)
    w1q, sw1 = oracle.per_block_cast(workloads.normal_bf16(rng, (G, 2 * I, H), 0.05), ue8m0=True)
    w2q, sw2 = oracle.per_block_cast(workloads.normal_bf16(rng, (G, H, I), 0.05), ue8m0=True)
    gu_m, hq_m, sh_m, y_m = oracle.moe_ffn_masked(xq, sx, w1q, sw1, w2q, sw2, mm)
    for e in range(G):
        v = int(mm[e])
        mi = np.full(v, e, np.int32)
        gu_c, hq_c, sh_c, y_c = oracle.moe_ffn_contiguous(xq[e, :v], sx[e, :v], w1q, sw1, w2q, sw2, mi)
        assert np.array_equal(gu_m[e, :v], gu_c)
        assert np.array_equal(hq_m[e, :v], hq_c)
        assert np.array_equal(y_m[e, :v], y_c)


# ---------------------------------------------------------------- K-grouped GEMM

def _kg_operands(rng, M, N, ks, ue8m0=True):
    T = int(sum(ks))
    a = workloads.bf16_bits(rng.standard_normal((M, T)).astype(np.float32))
    b = workloads.bf16_bits(rng.standard_normal((N, T)).astype(np.float32))
    qa, sa = oracle.per_token_cast(a, ue8m0=ue8m0)
    qb, sb = oracle.per_token_cast(b, ue8m0=ue8m0)
    return qa, sa, qb, sb


def test_k_grouped_single_group_is_the_dense_gemm():
    """One expert and B row scales constant over each 128-row block: the dense
    block-scaled GEMM (a swapped row/block index or operand fails this)."""
    rng = np.random.default_rng(41)
    M, N, T = 130, 256, 384
    qa, sa, qb, _ = _kg_operands(rng, M, N, [T])
    sbb = (2.0 ** rng.integers(-6, 3, size=(N // 128, T // 128))).astype(np.float32)
    sb_rows = np.repeat(sbb, 128, axis=0)
    d = oracle.k_grouped(qa, sa, qb, sb_rows, np.array([T], np.int32))
    ref = oracle.gemm_nt(qa, sa, qb, sbb)
    assert np.array_equal(d[0], ref)


def test_k_grouped_sums_to_the_whole_range():
    """Linearity: the experts' results add up to one GEMM over all tokens."""
    rng = np.random.default_rng(42)
    M, N = 64, 96
    ks = [256, 0, 128, 384]
    qa, sa, qb, sb = _kg_operands(rng, M, N, ks)
    d = oracle.k_grouped(qa, sa, qb, sb, np.array(ks, np.int32))
    whole = oracle.k_grouped(qa, sa, qb, sb, np.array([sum(ks)], np.int32))[0]
    rms = np.sqrt(np.mean(whole ** 2))
    assert np.max(np.abs(d.sum(axis=0) - whole)) <= 1e-12 * rms * len(ks)
    assert np.all(d[1] == 0.0)  # the empty expert


def test_k_grouped_brute_force_per_expert():
    """Each expert's result is the fp64 product of its decoded, scaled token
    slices (both scales indexed by row and 128-token block)."""
    rng = np.random.default_rng(43)
    M, N = 20, 24
    ks = [128, 256]
    qa, sa, qb, sb = _kg_operands(rng, M, N, ks)
    d = oracle.k_grouped(qa, sa, qb, sb, np.array(ks, np.int32))
    av = oracle.e4m3_decode(qa) * np.repeat(sa, 128, axis=1)
    bv = oracle.e4m3_decode(qb) * np.repeat(sb, 128, axis=1)
    t0 = 0
    for e, k in enumerate(ks):
        ref = av[:, t0:t0 + k] @ bv[:, t0:t0 + k].T
        assert np.allclose(d[e], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
        t0 += k


def test_k_grouped_integer_exact():
    """Entries in {-1, 0, 1} with power-of-two scales: exact (integer matmul)."""
    rng = np.random.default_rng(44)
    M, N = 33, 40
    ks = [128, 384]
    T = sum(ks)
    ia = rng.integers(-1, 2, size=(M, T))
    ib = rng.integers(-1, 2, size=(N, T))
    qa = oracle.e4m3_encode(ia.astype(np.float32))
    qb = oracle.e4m3_encode(ib.astype(np.float32))
    sa = (2.0 ** rng.integers(-3, 3, size=(M, T // 128))).astype(np.float32)
    sb = (2.0 ** rng.integers(-3, 3, size=(N, T // 128))).astype(np.float32)
    d = oracle.k_grouped(qa, sa, qb, sb, np.array(ks, np.int32))
    t0 = 0
    for e, k in enumerate(ks):
        ref = np.zeros((M, N))
        for tb in range(t0 // 128, (t0 + k) // 128):
            blk = slice(tb * 128, (tb + 1) * 128)
            ref += np.outer(sa[:, tb], sb[:, tb]) * (ia[:, blk] @ ib[:, blk].T)
        assert np.array_equal(d[e], ref)
        t0 += k


def test_k_grouped_rejects_bad_counts():
    qa = np.zeros((4, 256), np.uint8)
    sa = np.ones((4, 2), np.float32)
    with pytest.raises(ValueError):
        oracle.k_grouped(qa, sa, qa, sa, np.array([100, 156], np.int32))
    with pytest.raises(ValueError):
        oracle.k_grouped(qa, sa, qa, sa, np.array([128], np.int32))
