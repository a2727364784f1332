"""GPU quantizers against the CPU oracle: e4m3 bytes and fp32 scale bits must
be identical (bit-exact), on seeded inputs with ragged shapes, zero slices,
tiny values, outliers and N tails, through the C ABI."""
import numpy as np
import pytest

import oracle
import workloads
from helpers import bf16_tensor, sa_from_mn_major

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_04_b200 as m
    m.load_library()
    return m


def _special_rows(x: np.ndarray) -> np.ndarray:
    """Plant the edge cases the quantizer must get right."""
    x = x.copy()
    if x.shape[-2] > 4 and x.shape[-1] >= 256:
        x[..., 1, 128:256] = 0.0            # all-zero slice -> amax floor
        x[..., 2, :128] *= 1e-7             # amax far below the floor
        x[..., 3, :] *= 30.0                # outlier row
        x[..., 4, 5] = 1e-30                # deep underflow element
    return x


def gpu_per_token(fg, bits: np.ndarray):
    G, M, K = (1, *bits.shape) if bits.ndim == 2 else bits.shape
    x = bf16_tensor(bits.reshape(G, M, K))
    q = torch.empty((G, M, K), dtype=torch.uint8, device="cuda")
    s = torch.full((G, K // 128, fg.sfa_stride(M)), -1.0, dtype=torch.float32, device="cuda")
    fg.per_token_cast_to_fp8(x, q, s)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


def gpu_per_block(fg, bits: np.ndarray):
    G, N, K = (1, *bits.shape) if bits.ndim == 2 else bits.shape
    x = bf16_tensor(bits.reshape(G, N, K))
    q = torch.empty((G, N, K), dtype=torch.uint8, device="cuda")
    s = fg.empty_sfb(G, N, K, "cuda")
    fg.per_block_cast_to_fp8(x, q, s)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("G,M,K", [(1, 1, 128), (1, 63, 512), (1, 130, 384), (3, 80, 256),
                                   (1, 64, 7168), (2, 257, 1024),
                                   # rows of 9 and 15 slices: a full work item of 8
                                   # slices, then a partial one
                                   (1, 5, 1152), (2, 3, 1920)])
def test_per_token_bit_exact(fg, G, M, K):
    rng = np.random.default_rng(M * 1000 + K + G)
    x = _special_rows(rng.standard_normal((G, M, K), dtype=np.float32))
    bits = workloads.bf16_bits(x)
    q, s = gpu_per_token(fg, bits)
    qr, sr = oracle.per_token_cast(bits)
    assert np.array_equal(q, qr)
    assert np.array_equal(sa_from_mn_major(s, M).view(np.uint32), sr.view(np.uint32))


@pytest.mark.parametrize("G,N,K", [(1, 256, 512), (1, 2112, 768), (2, 130, 256), (1, 64, 128),
                                   (3, 384, 384)])
def test_per_block_bit_exact(fg, G, N, K):
    rng = np.random.default_rng(N * 1000 + K + G)
    x = _special_rows(rng.standard_normal((G, N, K), dtype=np.float32) * 0.02)
    bits = workloads.bf16_bits(x)
    q, s = gpu_per_block(fg, bits)
    qr, sr = oracle.per_block_cast(bits)
    assert np.array_equal(q, qr)
    assert np.array_equal(s.view(np.uint32), sr.view(np.uint32))


def test_quantizers_full_size_decode(fg):
    """decode_64x4096x7168: both operands at full size."""
    inp = workloads.make("decode_64x4096x7168")
    q, s = gpu_per_token(fg, inp.a)
    qr, sr = oracle.per_token_cast(inp.a)
    assert np.array_equal(q[0], qr)
    assert np.array_equal(sa_from_mn_major(s, inp.M)[0].view(np.uint32), sr.view(np.uint32))
    q, s = gpu_per_block(fg, inp.b)
    qr, sr = oracle.per_block_cast(inp.b)
    assert np.array_equal(q[0], qr)
    assert np.array_equal(s[0].view(np.uint32), sr.view(np.uint32))


def test_quantizers_full_size_prefill_tail(fg):
    """prefill_4096x2112x7168: N tail block of 64 rows, K = 7168."""
    inp = workloads.make("prefill_4096x2112x7168")
    q, s = gpu_per_block(fg, inp.b)
    qr, sr = oracle.per_block_cast(inp.b)
    assert np.array_equal(q[0], qr)
    assert np.array_equal(s[0].view(np.uint32), sr.view(np.uint32))
    q, s = gpu_per_token(fg, inp.a)
    qr, sr = oracle.per_token_cast(inp.a)
    assert np.array_equal(q[0], qr)
    assert np.array_equal(sa_from_mn_major(s, inp.M)[0].view(np.uint32), sr.view(np.uint32))


def test_per_token_zero_padding_rows(fg):
    """Contiguous-layout padding rows are zero: codes 0, scale 1e-4/448."""
    inp = workloads.contiguous(256, 512, counts=np.array([100, 3]), seed=2)
    q, s = gpu_per_token(fg, inp.a)
    pad = inp.m_indices < 0
    assert np.all(q[0][pad] == 0)
    sa = sa_from_mn_major(s, inp.M_total)[0]
    assert np.all(sa[pad] == np.float32(1e-4) / np.float32(448.0))
    qr, sr = oracle.per_token_cast(inp.a)
    assert np.array_equal(q[0], qr) and np.array_equal(sa.view(np.uint32), sr.view(np.uint32))


@pytest.mark.parametrize("ue8m0", [False, True])
def test_slices_with_infinities_and_nan_bit_exact(fg, ue8m0):
    """Infinities give the slice an infinite scale and zero codes (NaN for the
    infinities themselves); NaN elements map to 0x7F without raising the
    amax. Codes and scale bits equal the oracle's, per token and per block."""
    rng = np.random.default_rng(21)
    x = rng.standard_normal((130, 384), dtype=np.float32)
    bits = workloads.bf16_bits(x)
    bits[0, 7], bits[0, 9] = 0x7F80, 0xFF80      # +inf, -inf in slice (0, 0)
    bits[0, 11], bits[5, 200] = 0x7FC0, 0x7FC0   # NaN with and without an inf
    bits[129, 300] = 0xFF80                      # -inf in the N-tail block
    sfx = "_ue8m0" if ue8m0 else ""
    xt = bf16_tensor(bits[None])
    q = torch.empty((1, 130, 384), dtype=torch.uint8, device="cuda")
    s = torch.full((1, 3, fg.sfa_stride(130)), -1.0, dtype=torch.float32, device="cuda")
    getattr(fg, "per_token_cast_to_fp8" + sfx)(xt, q, s)
    qb = torch.empty((1, 130, 384), dtype=torch.uint8, device="cuda")
    sb = fg.empty_sfb(1, 130, 384, "cuda")
    getattr(fg, "per_block_cast_to_fp8" + sfx)(xt, qb, sb)
    torch.cuda.synchronize()
    qr, sr = oracle.per_token_cast(bits, ue8m0=ue8m0)
    assert np.array_equal(q.cpu().numpy()[0], qr)
    got_s = sa_from_mn_major(s.cpu().numpy(), 130)[0]
    assert np.array_equal(got_s.view(np.uint32), sr.view(np.uint32))
    assert np.isposinf(got_s[0, 0])
    qbr, sbr = oracle.per_block_cast(bits, ue8m0=ue8m0)
    assert np.array_equal(qb.cpu().numpy()[0], qbr)
    assert np.array_equal(sb.cpu().numpy()[0].view(np.uint32), sbr.view(np.uint32))


def test_quantizer_argument_errors(fg):
    x = torch.zeros((4, 100), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((4, 100), dtype=torch.uint8, device="cuda")
    s = torch.zeros(64, dtype=torch.float32, device="cuda")
    with pytest.raises(fg.FP8GemmError) as ei:
        fg.per_token_cast_to_fp8(x, q, s)
    assert ei.value.status == fg.FG_ERR_INVALID_ARG


# ---------------------------------------------------------------- weight dequantization

def gpu_dequant(fg, q: np.ndarray, s: np.ndarray) -> np.ndarray:
    qt = torch.from_numpy(np.ascontiguousarray(q)).cuda()
    st = torch.from_numpy(np.ascontiguousarray(s, np.float32)).cuda()
    x = torch.full(q.shape, -1.0, dtype=torch.bfloat16, device="cuda")
    fg.per_block_dequant_to_bf16(qt, st, x)
    torch.cuda.synchronize()
    return x.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("G,N,K", [(1, 256, 512), (2, 300, 384), (1, 2112, 768), (3, 64, 128)])
def test_per_block_dequant_bit_exact(fg, G, N, K):
    """Every finite code and scale bit pattern of the oracle's result."""
    rng = np.random.default_rng(N + K + G)
    q = rng.integers(0, 256, size=(G, N, K), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x41
    s = (rng.random((G, -(-N // 128), K // 128)) * 0.02 + 1e-5).astype(np.float32)
    assert np.array_equal(gpu_dequant(fg, q, s), oracle.per_block_dequant(q, s))


def test_per_block_dequant_round_trip_on_device(fg):
    """Weights quantized and dequantized on the GPU equal the oracle's chain;
    NaN codes come back as NaN."""
    rng = np.random.default_rng(21)
    bits = workloads.bf16_bits(rng.standard_normal((2, 2112, 512), dtype=np.float32) * 0.02)
    q, s = gpu_per_block(fg, bits)
    got = gpu_dequant(fg, q, s)
    assert np.array_equal(got, oracle.per_block_dequant(*oracle.per_block_cast(bits)))
    q[0, 7, 3] = 0x7F
    nan = gpu_dequant(fg, q, s)
    assert (nan[0, 7, 3] & 0x7F80) == 0x7F80 and (nan[0, 7, 3] & 0x007F) != 0


# ---------------------------------------------------------------- power-of-two (UE8M0) scales

@pytest.mark.parametrize("G,M,K", [(1, 1, 128), (1, 130, 384), (3, 80, 256), (1, 64, 7168)])
def test_per_token_ue8m0_bit_exact(fg, G, M, K):
    rng = np.random.default_rng(M * 3 + K + G)
    bits = workloads.bf16_bits(_special_rows(rng.standard_normal((G, M, K), dtype=np.float32)))
    x = bf16_tensor(bits)
    q = torch.empty((G, M, K), dtype=torch.uint8, device="cuda")
    s = torch.full((G, K // 128, fg.sfa_stride(M)), -1.0, dtype=torch.float32, device="cuda")
    fg.per_token_cast_to_fp8_ue8m0(x, q, s)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.per_token_cast(bits, ue8m0=True)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sa_from_mn_major(s.cpu().numpy(), M).view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("G,N,K", [(1, 256, 512), (2, 300, 384), (1, 2112, 768)])
def test_per_block_ue8m0_bit_exact(fg, G, N, K):
    rng = np.random.default_rng(N * 3 + K + G)
    bits = workloads.bf16_bits(rng.standard_normal((G, N, K), dtype=np.float32) * 0.02)
    x = bf16_tensor(bits)
    q = torch.empty((G, N, K), dtype=torch.uint8, device="cuda")
    s = fg.empty_sfb(G, N, K, "cuda")
    fg.per_block_cast_to_fp8_ue8m0(x, q, s)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.per_block_cast(bits, ue8m0=True)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
