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
def test_dense_full_size(fg, name):
    """Every output of the full-size dense shapes against the oracle."""
    inp = workloads.make(name)
    qa, sa, qb, sb = quantize_dense(inp)
    got = run_dense(fg, qa, sa, qb, sb)
    ref = oracle.gemm_nt(qa, sa, qb, sb)
    check_gemm(bf16_bits_to_f64(got), ref, "ue8m0 " + name)


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


def test_contiguous_full_size(fg):
    """Every valid output of the 8-expert contiguous workload."""
    inp = workloads.make("contiguous_8x4096x7168")
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=True)
    got = run_contiguous(fg, qa, sa, qb, sb, inp.m_indices)
    ref = oracle.grouped_contiguous(qa, sa, qb, sb, inp.m_indices)
    valid = inp.m_indices >= 0
    check_gemm(bf16_bits_to_f64(got[valid]), ref[valid], "ue8m0 contiguous full")
    assert np.all(got[~valid] == SENTINEL)


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


def test_masked_full_size(fg):
    """Every valid output of the 32-expert masked workload."""
    inp = workloads.make("masked_32x256x4096x7168")
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=True)
    got, status = run_masked(fg, qa, sa, qb, sb, inp.masked_m, 128)
    assert status == 0
    ref = oracle.grouped_masked(qa, sa, qb, sb, inp.masked_m)
    valid = np.arange(inp.M_max)[None, :] < np.asarray(inp.masked_m)[:, None]
    check_gemm(bf16_bits_to_f64(got[valid]), ref[valid], "ue8m0 masked full")
    assert np.all(got[~valid] == SENTINEL)


# ------------------------------------------------------------------ whole path

def test_whole_path_prefill_gpu_quantized(fg):
    """bf16 in -> GPU UE8M0 quantizers -> block-scaled GEMM, against the
    oracle's UE8M0 quantizers and GEMM on every output."""
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
    ref = oracle.gemm_nt(qa, sa, qb, sb)
    check_gemm(bf16_bits_to_f64(tensor_bf16_bits(D)), ref, "ue8m0 whole path prefill")


# ------------------------------------------------------------------ scale check

FG_DEVICE_BAD_SCALE = 5


def _dense_ue8m0_status(fg, qa, sa, qb, sb):
    M, K = qa.shape
    D = _d_tensor((M, qb.shape[0]))
    fg.fp8_gemm_nt_ue8m0(to_torch(qa), to_torch(sa_to_mn_major(sa)), to_torch(qb),
                         to_torch(np.ascontiguousarray(sb, np.float32)), D)
    torch.cuda.synchronize()
    return fg.get_device_status()


@pytest.mark.parametrize("which", ["token", "weight", "fp32 quantizer"])
def test_non_power_of_two_scale_is_reported(fg, which):
    """The block-scaled kernel keeps only a scale's exponent, so a scale with
    mantissa bits (one token scale, one weight-block scale, or the amax/448
    scales of the fp32 quantizers) cannot be applied: the call reports
    FG_DEVICE_BAD_SCALE instead of returning a silently rounded product."""
    inp = workloads.dense(256, 256, 512, seed=5)
    ue8m0 = which != "fp32 quantizer"
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=ue8m0)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=ue8m0)
    sa, sb = sa.copy(), sb.copy()
    if which == "token":
        sa[17, 2] *= np.float32(1.5)
    elif which == "weight":
        sb[1, 3] *= np.float32(1.25)
    assert _dense_ue8m0_status(fg, qa, sa, qb, sb) == FG_DEVICE_BAD_SCALE
    assert fg.get_device_status() == 0  # the read cleared it
    # the unmodified power-of-two scales pass the check
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=True)
    assert _dense_ue8m0_status(fg, qa, sa, qb, sb) == 0


def test_zero_and_negative_scales(fg):
    """Zero is accepted (it acts as 2^-127); a negative power of two is not a
    scale the kernel can apply (only the exponent field is used)."""
    inp = workloads.dense(256, 256, 256, seed=6)
    qa, sa = oracle.per_token_cast(inp.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(inp.b, ue8m0=True)
    sa = sa.copy()
    sa[3, 1] = 0.0
    assert _dense_ue8m0_status(fg, qa, sa, qb, sb) == 0
    sa[3, 1] = -0.5
    assert _dense_ue8m0_status(fg, qa, sa, qb, sb) == FG_DEVICE_BAD_SCALE


def test_scales_of_rows_never_stored_are_not_checked(fg):
    """Only the token scales of stored rows must be powers of two: masked rows
    past masked_m and contiguous padding rows may hold any scale."""
    G, M_max, N, K = 3, 256, 256, 256
    mm = np.array([200, 0, 131], np.int32)
    mi = workloads.masked(G, M_max, N, K, seed=9, masked_m=mm)
    qa, sa = oracle.per_token_cast(mi.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(mi.b, ue8m0=True)
    sa = sa.copy()
    for e in range(G):
        sa[e, mm[e]:, :] = np.float32(1.5)
    got, status = run_masked(fg, qa, sa, qb, sb, mm, 128)
    assert status == 0
    ref = oracle.grouped_masked(qa, sa, qb, sb, mm)
    for e in range(G):
        if mm[e]:
            check_gemm(bf16_bits_to_f64(got[e, :mm[e]]), ref[e, :mm[e]], "masked expert %d" % e)
    # ... and the same scale on a stored row is reported
    sa[0, 5, 0] = np.float32(1.5)
    _, status = run_masked(fg, qa, sa, qb, sb, mm, 128)
    assert status == FG_DEVICE_BAD_SCALE

    ci = workloads.contiguous(N, K, counts=np.array([130, 5]), seed=10)
    qa, sa = oracle.per_token_cast(ci.a, ue8m0=True)
    qb, sb = oracle.per_block_cast(ci.b, ue8m0=True)
    sa = sa.copy()
    sa[ci.m_indices < 0, :] = np.float32(3.0)
    got = run_contiguous(fg, qa, sa, qb, sb, ci.m_indices)  # asserts a clear status
    valid = ci.m_indices >= 0
    ref = oracle.grouped_contiguous(qa, sa, qb, sb, ci.m_indices)
    check_gemm(bf16_bits_to_f64(got[valid]), ref[valid], "contiguous padding scales")
