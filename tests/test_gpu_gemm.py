"""GPU GEMMs (dense, contiguous-grouped, masked-grouped) against the CPU
oracle through the C ABI.

Operands are quantized by the oracle on the CPU and uploaded, so these tests
isolate the GEMM kernels; the whole-path tests at the end quantize on the GPU
too. Every case, full-size workloads included, is compared element by element
over every valid output. The bar is
|gpu - ref| <= 2^-7 |ref| + 1e-3 rms(ref) per element and a global
1 - 2 sum(xy)/sum(x^2+y^2) < 1e-3; integer cases with power-of-two scales must
be exact.
"""
import numpy as np
import pytest

import oracle
import workloads
from helpers import (bf16_bits_to_f64, bf16_tensor, check_gemm, sa_to_mn_major,
                     tensor_bf16_bits, to_torch)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SENTINEL = 0xFFFF  # bf16 NaN pattern pre-filled into D


@pytest.fixture(scope="module")
def fg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_04_b200 as m
    m.load_library()
    return m


def _d_tensor(shape):
    return to_torch(np.full(shape, SENTINEL, np.uint16).view(np.int16)).view(torch.bfloat16)


def run_dense(fg, qa, sa, qb, sb):
    M, K = qa.shape
    N = qb.shape[0]
    A = to_torch(qa)
    B = to_torch(qb)
    SA = to_torch(sa_to_mn_major(sa))
    SB = to_torch(np.ascontiguousarray(sb, np.float32))
    D = _d_tensor((M, N))
    fg.fp8_gemm_nt(A, SA, B, SB, D)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    return tensor_bf16_bits(D)


def quantize_dense(inp):
    qa, sa = oracle.per_token_cast(inp.a)
    qb, sb = oracle.per_block_cast(inp.b)
    return qa, sa, qb, sb


# ------------------------------------------------------------------ exact cases

@pytest.mark.parametrize("M,N,K", [(200, 272, 256), (40, 384, 256), (128, 128, 128), (1, 256, 256)])
def test_dense_exact_integer_case(fg, M, N, K):
    """Entries in {-1,0,1}, power-of-two scales constant along K: every
    partial sum and the bf16 output are exact, so gpu == ref bitwise."""
    rng = np.random.default_rng(M + N + K)
    ia = rng.integers(-1, 2, size=(M, K)).astype(np.float32)
    ib = rng.integers(-1, 2, size=(N, K)).astype(np.float32)
    qa = oracle.e4m3_encode(ia)
    qb = oracle.e4m3_encode(ib)
    KB, NB = K // 128, -(-N // 128)
    sa = np.repeat((2.0 ** rng.integers(-4, 4, size=(M, 1))).astype(np.float32), KB, axis=1)
    sb = np.repeat((2.0 ** rng.integers(-4, 4, size=(NB, 1))).astype(np.float32), KB, axis=1)
    ref = oracle.gemm_nt(qa, sa, qb, sb)
    got = bf16_bits_to_f64(run_dense(fg, qa, sa, qb, sb))
    assert np.array_equal(got, ref)


def test_dense_closed_form_all_ones(fg):
    M, N, K = 96, 256, 1024
    qa = np.full((M, K), 0x38, np.uint8)
    qb = np.full((N, K), 0x38, np.uint8)
    sa = np.full((M, K // 128), 0.25, np.float32)
    sb = np.full((2, K // 128), 0.125, np.float32)
    got = bf16_bits_to_f64(run_dense(fg, qa, sa, qb, sb))
    assert np.all(got == K * 0.25 * 0.125)


# ------------------------------------------------------------------ dense parity

@pytest.mark.parametrize("M,N,K", [
    (128, 256, 512),     # dense_128x256x512
    (1, 4096, 512), (15, 256, 1024), (33, 512, 384), (63, 384, 1024), (64, 256, 2048),
    (65, 512, 256), (127, 128, 128), (200, 272, 640), (300, 2112, 384), (513, 1024, 256),
])
def test_dense_parity_small(fg, M, N, K):
    inp = workloads.dense(M, N, K, seed=M + 7 * N + K, outlier_frac=0.01)
    qa, sa, qb, sb = quantize_dense(inp)
    ref = oracle.gemm_nt(qa, sa, qb, sb)
    got = bf16_bits_to_f64(run_dense(fg, qa, sa, qb, sb))
    check_gemm(got, ref, "dense %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("M,N,K", [(64, 1024, 7168), (16, 2048, 1024), (30, 6144, 2048),
                                   (64, 18944, 512)])
def test_dense_split_k_parity_and_determinism(fg, M, N, K):
    """Shapes that split K across a cluster (4, 4, 2 and no split); the fixed
    reduction order makes repeated calls bitwise identical."""
    inp = workloads.dense(M, N, K, seed=5 + M, outlier_frac=0.01)
    qa, sa, qb, sb = quantize_dense(inp)
    ref = oracle.gemm_nt(qa, sa, qb, sb)
    a = run_dense(fg, qa, sa, qb, sb)
    b = run_dense(fg, qa, sa, qb, sb)
    assert np.array_equal(a, b)
    check_gemm(bf16_bits_to_f64(a), ref, "split-K %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("name", ["decode_64x4096x7168", "prefill_4096x7168x2048",
                                  "prefill_4096x2112x7168"])
def test_dense_full_size(fg, name):
    """Every output of the full-size dense shapes (the swapped split-K decode
    shape and both prefill shapes, one with a ragged N) against the oracle."""
    inp = workloads.make(name)
    qa, sa, qb, sb = quantize_dense(inp)
    got = run_dense(fg, qa, sa, qb, sb)
    ref = oracle.gemm_nt(qa, sa, qb, sb)
    check_gemm(bf16_bits_to_f64(got), ref, name)


# ------------------------------------------------------------------ contiguous

def run_contiguous(fg, qa, sa, qb, sb, m_indices):
    M_total, K = qa.shape
    G, N, _ = qb.shape
    D = _d_tensor((M_total, N))
    fg.fp8_grouped_gemm_contiguous(to_torch(qa), to_torch(sa_to_mn_major(sa)), to_torch(qb),
                                   to_torch(np.ascontiguousarray(sb, np.float32)), D,
                                   to_torch(m_indices.astype(np.int32)))
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    return tensor_bf16_bits(D)


@pytest.mark.parametrize("counts,N,K", [([130, 0, 5, 128], 192, 256), ([1], 128, 128),
                                        ([300, 257, 0, 0, 64], 2112, 384)])
def test_contiguous_parity_small(fg, counts, N, K):
    inp = workloads.contiguous(N, K, counts=np.array(counts), seed=len(counts) + N)
    qa, sa = oracle.per_token_cast(inp.a)
    qb, sb = oracle.per_block_cast(inp.b)
    ref = oracle.grouped_contiguous(qa, sa, qb, sb, inp.m_indices)
    got = run_contiguous(fg, qa, sa, qb, sb, inp.m_indices)
    valid = inp.m_indices >= 0
    check_gemm(bf16_bits_to_f64(got[valid]), ref[valid], "contiguous %s" % counts)
    assert np.all(got[~valid] == SENTINEL), "padding rows must stay unwritten"


def test_contiguous_padding_tiles_and_odd_runs(fg):
    """All-padding token tiles between groups, a group split into two runs,
    runs of odd length and groups meeting inside an aligned pair of token
    tiles: work is paired by expert, never across experts or padding."""
    N, K = 384, 256
    experts = [0, -1, 0, 1, 1, 1, -1, 2, 3, 3, 3]   # expert of each 128-row tile
    rows = [128, 0, 77, 128, 128, 5, 0, 128, 128, 128, 64]  # valid rows of each tile
    M_total = 128 * len(experts)
    m_indices = np.full(M_total, -1, np.int32)
    for t, (e, r) in enumerate(zip(experts, rows)):
        if e >= 0:
            m_indices[t * 128:t * 128 + r] = e
    rng = np.random.default_rng(11)
    a = np.zeros((M_total, K), np.uint16)
    valid = m_indices >= 0
    a[valid] = workloads.bf16_bits(rng.standard_normal((int(valid.sum()), K), dtype=np.float32))
    b = workloads.normal_bf16(np.random.default_rng(12), (4, N, K), 0.02)
    qa, sa = oracle.per_token_cast(a)
    qb, sb = oracle.per_block_cast(b)
    ref = oracle.grouped_contiguous(qa, sa, qb, sb, m_indices)
    got = run_contiguous(fg, qa, sa, qb, sb, m_indices)
    check_gemm(bf16_bits_to_f64(got[valid]), ref[valid], "contiguous padding tiles")
    assert np.all(got[~valid] == SENTINEL), "padding rows must stay unwritten"


def test_contiguous_full_size(fg):
    """Every valid output of the 8-expert contiguous workload against the
    oracle; padding rows stay unwritten."""
    inp = workloads.make("contiguous_8x4096x7168")
    qa, sa = oracle.per_token_cast(inp.a)
    qb, sb = oracle.per_block_cast(inp.b)
    got = run_contiguous(fg, qa, sa, qb, sb, inp.m_indices)
    ref = oracle.grouped_contiguous(qa, sa, qb, sb, inp.m_indices)
    valid = inp.m_indices >= 0
    check_gemm(bf16_bits_to_f64(got[valid]), ref[valid], "contiguous full")
    assert np.all(got[~valid] == SENTINEL)


# ------------------------------------------------------------------ masked

def run_masked(fg, qa, sa, qb, sb, masked_m, expected_m):
    G, M_max, K = qa.shape
    N = qb.shape[1]
    D = _d_tensor((G, M_max, N))
    fg.fp8_grouped_gemm_masked(to_torch(qa), to_torch(sa_to_mn_major(sa)), to_torch(qb),
                               to_torch(np.ascontiguousarray(sb, np.float32)), D,
                               to_torch(masked_m.astype(np.int32)), expected_m)
    torch.cuda.synchronize()
    status = fg.get_device_status()
    return tensor_bf16_bits(D), status


@pytest.mark.parametrize("masked_m,M_max,N,K,expected", [
    ([0, 80, 17], 80, 192, 256, 40),
    ([1, 256, 0, 129], 256, 256, 512, 128),
    ([64, 3, 0, 50], 64, 384, 384, 32),      # swapped tiles (expected <= 64)
    ([200, 7], 256, 2112, 256, 100),
])
def test_masked_parity_small(fg, masked_m, M_max, N, K, expected):
    G = len(masked_m)
    inp = workloads.masked(G, M_max, N, K, seed=G + N, masked_m=np.array(masked_m))
    qa, sa = oracle.per_token_cast(inp.a)
    qb, sb = oracle.per_block_cast(inp.b)
    ref = oracle.grouped_masked(qa, sa, qb, sb, inp.masked_m)
    # rows past masked_m hold e4m3 NaN codes: they must not reach valid outputs
    qa_nan = qa.copy()
    for e, mv in enumerate(masked_m):
        qa_nan[e, mv:] = 0x7F
    got, status = run_masked(fg, qa_nan, sa, qb, sb, inp.masked_m, expected)
    assert status == 0
    for e, mv in enumerate(masked_m):
        if mv:
            check_gemm(bf16_bits_to_f64(got[e, :mv]), ref[e, :mv], "masked e=%d" % e)
        assert np.all(got[e, mv:] == SENTINEL), "rows past masked_m must stay unwritten"


def test_masked_full_size(fg):
    """Every valid output of the 32-expert masked workload against the oracle;
    A rows past masked_m hold e4m3 NaN codes and their D rows stay unwritten."""
    inp = workloads.make("masked_32x256x4096x7168")
    qa, sa = oracle.per_token_cast(inp.a)
    qb, sb = oracle.per_block_cast(inp.b)
    qa_nan = qa.copy()
    for e, mv in enumerate(inp.masked_m):
        qa_nan[e, mv:] = 0x7F
    got, status = run_masked(fg, qa_nan, sa, qb, sb, inp.masked_m, 128)
    assert status == 0
    ref = oracle.grouped_masked(qa, sa, qb, sb, inp.masked_m)
    valid = np.arange(inp.M_max)[None, :] < np.asarray(inp.masked_m)[:, None]
    check_gemm(bf16_bits_to_f64(got[valid]), ref[valid], "masked full")
    assert np.all(got[~valid] == SENTINEL)


def test_masked_bad_count_sets_device_status(fg):
    G, M_max, N, K = 2, 64, 128, 128
    inp = workloads.masked(G, M_max, N, K, seed=1, masked_m=np.array([10, 64]))
    qa, sa = oracle.per_token_cast(inp.a)
    qb, sb = oracle.per_block_cast(inp.b)
    bad = np.array([10, 1000], np.int32)  # > M_max: clamped, status raised
    got, status = run_masked(fg, qa, sa, qb, sb, bad, 64)
    assert status == 2
    ref = oracle.grouped_masked(qa, sa, qb, sb, np.array([10, 64]))
    check_gemm(bf16_bits_to_f64(got[1]), ref[1], "clamped expert")


# ------------------------------------------------------------------ whole path

def test_whole_path_decode_gpu_quantized(fg):
    """bf16 in -> GPU quantizers -> GPU GEMM, against oracle quantizers + GEMM."""
    inp = workloads.make("decode_64x4096x7168")
    M, N, K = inp.M, inp.N, inp.K
    x = bf16_tensor(inp.a)
    w = bf16_tensor(inp.b)
    A = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    SA = fg.empty_sfa(1, M, K, "cuda")
    B = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    SB = fg.empty_sfb(1, N, K, "cuda")
    D = _d_tensor((M, N))
    fg.per_block_cast_to_fp8(w, B, SB)
    fg.per_token_cast_to_fp8(x, A, SA)
    fg.fp8_gemm_nt(A, SA, B, SB[0], D)
    torch.cuda.synchronize()
    qa, sa, qb, sb = quantize_dense(inp)
    ref = oracle.gemm_nt(qa, sa, qb, sb)
    check_gemm(bf16_bits_to_f64(tensor_bf16_bits(D)), ref, "whole path decode")


def test_gemm_argument_errors(fg):
    A = torch.zeros((64, 100), dtype=torch.uint8, device="cuda")
    with pytest.raises(fg.FP8GemmError) as ei:
        fg.fp8_gemm_nt(A, torch.zeros(64, device="cuda"), A, torch.zeros(4, device="cuda"),
                       torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda"))
    assert ei.value.status == fg.FG_ERR_INVALID_ARG


def test_bounded_wait_gives_up_and_reports(fg):
    fg.selftest_wait_timeout(2000)
    assert fg.get_device_status() == 1
    assert fg.get_device_status() == 0  # cleared
    # the context stays usable afterwards
    test_dense_closed_form_all_ones(fg)
