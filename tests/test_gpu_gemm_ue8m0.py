"""GPU GEMMs for power-of-two (UE8M0) scales against the CPU oracle, through
the C ABI: the block-scaled tensor-core kernel (scales applied inside the MMA,
the whole K range accumulated in tensor memory) for each weight-tile width,
and the automatic choice (which sends thin shapes to the promoted kernel).

Operands are quantized with power-of-two scales by the oracle on the CPU; the
whole-path test quantizes on the GPU. The acceptance bar is the one of the
other GEMM tests (per element |gpu - ref| <= 2^-7 |ref| + 1e-3 rms(ref),
global 1 - 2 sum(xy)/sum(x^2+y^2) < 1e-3); the integer case must equal the
bf16 rounding of the exact result.
"""
import numpy as np
import pytest

import oracle
import workloads
from helpers import (bf16_bits_to_f64, bf16_tensor, check_gemm, sa_to_mn_major,
                     tensor_bf16_bits, to_torch)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SENTINEL = 0xFFFF
# forced tiles: (weight rows, CTA pair); (0, False) = the automatic choice
TILES = [(128, False), (224, False), (256, False), (224, True), (192, True), (0, False)]


@pytest.fixture(scope="module")
def fg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_04_b200 as m
    m.load_library()
    yield m
    m.set_ue8m0_tile(0)


@pytest.fixture(params=TILES, ids=lambda t: ("p%d" if t[1] else "w%d") % t[0] if t[0] else "auto")
def width(request, fg):
    w, pair = request.param
    fg.set_ue8m0_tile(w, pair)
    yield w + (1000 if pair else 0)
    fg.set_ue8m0_tile(0)


def _d_tensor(shape):
    return to_torch(np.full(shape, SENTINEL, np.uint16).view(np.int16)).view(torch.bfloat16)


def _bf16_rne(x: np.ndarray) -> np.ndarray:
    """fp64 values exactly representable in fp32 -> nearest-even bf16, as fp64."""
    u = np.asarray(x, np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (r.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run_dense(fg, qa, sa, qb, sb):
    M, K = qa.shape
    N = qb.shape[0]
    D = _d_tensor((M, N))
    fg.fp8_gemm_nt_ue8m0(to_torch(qa), to_torch(sa_to_mn_major(sa)), to_torch(qb),
                         to_torch(np.ascontiguousarray(sb, np.float32)), D)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    return tensor_bf16_bits(D)


def quantize_dense(inp):
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=True)
    return qa, sa, qb, sb


# ------------------------------------------------------------------ exact case

@pytest.mark.parametrize("M,N,K", [(200, 272, 512), (128, 224, 384), (1, 256, 256),
                                   (129, 704, 512)])
def test_dense_exact_integer_case(fg, width, M, N, K):
    """Entries in {-1,0,1} and power-of-two scales varying along K and across
    rows and weight blocks: every product and every partial sum is exact in
    fp32 (magnitudes within 2^-8 .. 2^15), so the output must be the bf16
    rounding of the exact result, whatever the summation order."""
    rng = np.random.default_rng(M + N + K + width)
    qa = oracle.e4m3_encode(rng.integers(-1, 2, size=(M, K)).astype(np.float32))
    qb = oracle.e4m3_encode(rng.integers(-1, 2, size=(N, K)).astype(np.float32))
    KB, NB = K // 128, -(-N // 128)
    sa = (2.0 ** rng.integers(-4, 3, size=(M, KB))).astype(np.float32)
    sb = (2.0 ** rng.integers(-4, 3, size=(NB, KB))).astype(np.float32)
    ref = oracle.gemm_nt(qa, sa, qb, sb)
    got = bf16_bits_to_f64(run_dense(fg, qa, sa, qb, sb))
    assert np.array_equal(got, _bf16_rne(ref))


def test_dense_closed_form_all_ones(fg, width):
    M, N, K = 96, 480, 1024
    qa = np.full((M, K), 0x38, np.uint8)
    qb = np.full((N, K), 0x38, np.uint8)
    sa = np.full((M, K // 128), 0.25, np.float32)
    sb = np.full((4, K // 128), 0.125, np.float32)
    got = bf16_bits_to_f64(run_dense(fg, qa, sa, qb, sb))
    assert np.all(got == K * 0.25 * 0.125)


# ------------------------------------------------------------------ dense parity

@pytest.mark.parametrize("M,N,K", [
    (128, 256, 512), (1, 4096, 512), (65, 512, 256), (127, 128, 128), (200, 272, 640),
    (300, 2112, 384), (513, 1024, 256), (256, 16, 256), (384, 7168, 128),
])
def test_dense_parity_small(fg, width, M, N, K):
    inp = workloads.dense(M, N, K, seed=M + 7 * N + K, outlier_frac=0.01)
    qa, sa, qb, sb = quantize_dense(inp)
    ref = oracle.gemm_nt(qa, sa, qb, sb)
    a = run_dense(fg, qa, sa, qb, sb)
    check_gemm(bf16_bits_to_f64(a), ref, "ue8m0 dense %dx%dx%d w%d" % (M, N, K, width))
    # deterministic: one fixed accumulation order
    assert np.array_equal(a, run_dense(fg, qa, sa, qb, sb))


@pytest.mark.parametrize("name", ["prefill_4096x7168x2048", "prefill_4096x2112x7168",
                                  "decode_64x4096x7168"])
def test_dense_full_size_sampled(fg, name):
    inp = workloads.make(name)
    qa, sa, qb, sb = quantize_dense(inp)
    got = run_dense(fg, qa, sa, qb, sb)
    rng = np.random.default_rng(98)
    P = 20000
    r = rng.integers(0, inp.M, P)
    n = rng.integers(0, inp.N, P)
    r[:64] = inp.M - 1
    n[64:128] = inp.N - 1
    ref = oracle.gemm_points(qa, sa, qb, sb, r, np.zeros(P, np.int64), n)
    check_gemm(bf16_bits_to_f64(got[r, n]), ref, "ue8m0 " + name)


# ------------------------------------------------------------------ grouped forms

def run_contiguous(fg, qa, sa, qb, sb, m_indices):
    M_total, K = qa.shape
    G, N, _ = qb.shape
    D = _d_tensor((M_total, N))
    fg.fp8_grouped_gemm_contiguous_ue8m0(to_torch(qa), to_torch(sa_to_mn_major(sa)), to_torch(qb),
                                         to_torch(np.ascontiguousarray(sb, np.float32)), D,
                                         to_torch(m_indices.astype(np.int32)))
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    return tensor_bf16_bits(D)


@pytest.mark.parametrize("counts,N,K", [([130, 0, 5, 128], 192, 256), ([1], 128, 128),
                                        ([300, 257, 0, 0, 64], 2112, 384)])
def test_contiguous_parity_small(fg, width, counts, N, K):
    inp = workloads.contiguous(N, K, counts=np.array(counts), seed=len(counts) + N)
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=True)
    ref = oracle.grouped_contiguous(qa, sa, qb, sb, inp.m_indices)
    got = run_contiguous(fg, qa, sa, qb, sb, inp.m_indices)
    valid = inp.m_indices >= 0
    check_gemm(bf16_bits_to_f64(got[valid]), ref[valid], "ue8m0 contiguous %s" % counts)
    assert np.all(got[~valid] == SENTINEL), "padding rows must stay unwritten"


def test_contiguous_padding_tiles_and_odd_runs(fg, width):
    """Padding tiles between groups, an expert split into two runs, runs of
    odd length and groups meeting inside an aligned pair of token tiles: pair
    units join two tiles of one run only, and a unit's partner tile of
    another expert or of padding stores nothing."""
    N, K = 384, 512
    experts = [0, -1, 0, 1, 1, 1, -1, 2, 3, 3, 3, 0]   # expert of each 128-row tile
    rows = [128, 0, 77, 128, 128, 5, 0, 128, 128, 128, 64, 100]  # valid rows of each tile
    M_total = 128 * len(experts)
    m_indices = np.full(M_total, -1, np.int32)
    for t, (e, r) in enumerate(zip(experts, rows)):
        if e >= 0:
            m_indices[t * 128:t * 128 + r] = e
    rng = np.random.default_rng(13)
    a = np.zeros((M_total, K), np.uint16)
    valid = m_indices >= 0
    a[valid] = workloads.bf16_bits(rng.standard_normal((int(valid.sum()), K), dtype=np.float32))
    b = workloads.normal_bf16(np.random.default_rng(14), (4, N, K), 0.02)
    qa, sa = oracle.per_token_cast(a, ue8m0=True)
    qb, sb = oracle.per_block_cast(b, ue8m0=True)
    ref = oracle.grouped_contiguous(qa, sa, qb, sb, m_indices)
    got = run_contiguous(fg, qa, sa, qb, sb, m_indices)
    check_gemm(bf16_bits_to_f64(got[valid]), ref[valid], "ue8m0 contiguous padding tiles")
    assert np.all(got[~valid] == SENTINEL), "padding rows must stay unwritten"


def test_contiguous_full_size_sampled(fg):
    inp = workloads.make("contiguous_8x4096x7168")
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=True)
    got = run_contiguous(fg, qa, sa, qb, sb, inp.m_indices)
    valid_rows = np.nonzero(inp.m_indices >= 0)[0]
    rng = np.random.default_rng(8)
    P = 20000
    r = valid_rows[rng.integers(0, valid_rows.size, P)]
    n = rng.integers(0, inp.N, P)
    e = inp.m_indices[r].astype(np.int64)
    ref = oracle.gemm_points(qa, sa, qb, sb, r, e, n)
    check_gemm(bf16_bits_to_f64(got[r, n]), ref, "ue8m0 contiguous full")
    assert np.all(got[inp.m_indices < 0] == SENTINEL)


def run_masked(fg, qa, sa, qb, sb, masked_m, expected_m):
    G, M_max, K = qa.shape
    N = qb.shape[1]
    D = _d_tensor((G, M_max, N))
    fg.fp8_grouped_gemm_masked_ue8m0(to_torch(qa), to_torch(sa_to_mn_major(sa)), to_torch(qb),
                                     to_torch(np.ascontiguousarray(sb, np.float32)), D,
                                     to_torch(masked_m.astype(np.int32)), expected_m)
    torch.cuda.synchronize()
    return tensor_bf16_bits(D), fg.get_device_status()


@pytest.mark.parametrize("masked_m,M_max,N,K,expected", [
    ([0, 80, 17], 80, 192, 256, 40),
    ([1, 256, 0, 129], 256, 256, 512, 128),
    ([200, 7], 256, 2112, 256, 100),
])
def test_masked_parity_small(fg, width, masked_m, M_max, N, K, expected):
    G = len(masked_m)
    inp = workloads.masked(G, M_max, N, K, seed=G + N, masked_m=np.array(masked_m))
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=True)
    ref = oracle.grouped_masked(qa, sa, qb, sb, inp.masked_m)
    # rows past masked_m hold e4m3 NaN codes: they must not reach valid outputs
    qa_nan = qa.copy()
    for e, mv in enumerate(masked_m):
        qa_nan[e, mv:] = 0x7F
    got, status = run_masked(fg, qa_nan, sa, qb, sb, inp.masked_m, expected)
    assert status == 0
    for e, mv in enumerate(masked_m):
        if mv:
            check_gemm(bf16_bits_to_f64(got[e, :mv]), ref[e, :mv], "ue8m0 masked e=%d" % e)
        assert np.all(got[e, mv:] == SENTINEL), "rows past masked_m must stay unwritten"


def test_masked_full_size_sampled(fg):
    inp = workloads.make("masked_32x256x4096x7168")
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=True)
    got, status = run_masked(fg, qa, sa, qb, sb, inp.masked_m, 128)
    assert status == 0
    rows, experts = [], []
    for e, mv in enumerate(inp.masked_m):
        rows += [e * inp.M_max + m for m in range(mv)]
        experts += [e] * int(mv)
        assert np.all(got[e, mv:] == SENTINEL)
    rows = np.array(rows)
    experts = np.array(experts)
    rng = np.random.default_rng(4)
    P = 20000
    pick = rng.integers(0, rows.size, P)
    r, e = rows[pick], experts[pick]
    n = rng.integers(0, inp.N, P)
    ref = oracle.gemm_points(qa.reshape(-1, inp.K), sa.reshape(-1, inp.K // 128), qb, sb, r, e, n)
    check_gemm(bf16_bits_to_f64(got.reshape(-1, inp.N)[r, n]), ref, "ue8m0 masked full")


# ------------------------------------------------------------------ whole path

def test_whole_path_prefill_gpu_quantized(fg):
    """bf16 in -> GPU UE8M0 quantizers -> block-scaled GEMM, against the
    oracle's UE8M0 quantizers and GEMM on sampled outputs."""
    inp = workloads.make("prefill_4096x7168x2048")
    M, N, K = inp.M, inp.N, inp.K
    x = bf16_tensor(inp.a)
    w = bf16_tensor(inp.b)
    A = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    SA = fg.empty_sfa(1, M, K, "cuda")
    B = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    SB = fg.empty_sfb(1, N, K, "cuda")
    D = _d_tensor((M, N))
    fg.per_block_cast_to_fp8_ue8m0(w, B, SB)
    fg.per_token_cast_to_fp8_ue8m0(x, A, SA)
    fg.fp8_gemm_nt_ue8m0(A, SA, B, SB[0], D)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    qa, sa, qb, sb = quantize_dense(inp)
    rng = np.random.default_rng(5)
    P = 20000
    r = rng.integers(0, M, P)
    n = rng.integers(0, N, P)
    ref = oracle.gemm_points(qa, sa, qb, sb, r, np.zeros(P, np.int64), n)
    got = tensor_bf16_bits(D)
    check_gemm(bf16_bits_to_f64(got[r, n]), ref, "ue8m0 whole path prefill")
