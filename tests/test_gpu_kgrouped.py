"""The K-grouped GEMM (expert weight gradients: the contraction runs over each
expert's tokens, stacked along K) on the GPU against the CPU oracle, through
the C ABI. Operands are [rows][tokens] matrices quantized per row per 128
tokens with power-of-two scales (the oracle's UE8M0 per-token quantizer
applied to the transposed activations); the fp32 output is compared with the
GEMM bar and a tighter fp32 bound, the integer case exactly.
"""
import numpy as np
import pytest

import oracle
import workloads
from helpers import check_gemm, sa_to_mn_major, to_torch

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_04_b200 as m
    m.load_library()
    return m


def run(fg, qa, sa, qb, sb, ks):
    M, T = qa.shape
    N = qb.shape[0]
    G = len(ks)
    D = to_torch(np.full((G, M, N), np.nan, np.float32))
    fg.fp8_k_grouped_gemm_nt_ue8m0(to_torch(qa), to_torch(sa_to_mn_major(sa)[0]), to_torch(qb),
                                   to_torch(sa_to_mn_major(sb)[0]), D,
                                   to_torch(np.array(ks, np.int32)))
    torch.cuda.synchronize()
    return D.cpu().numpy().astype(np.float64), fg.get_device_status()


def operands(rng, M, N, ks):
    T = int(sum(ks))
    dy = workloads.bf16_bits(rng.standard_normal((M, T)).astype(np.float32))
    x = workloads.bf16_bits(rng.standard_normal((N, T)).astype(np.float32))
    qa, sa = oracle.per_token_cast(dy, ue8m0=True)
    qb, sb = oracle.per_token_cast(x, ue8m0=True)
    return qa, sa, qb, sb


@pytest.mark.parametrize("M,N,ks", [
    (128, 224, [256, 128]),          # single-CTA tiles
    (256, 448, [384, 0, 128, 256]),  # CTA pairs, an empty expert
    (200, 240, [128, 640]),          # M and N tails (partial token and weight tiles)
    (384, 96, [1024]),               # one expert, a long range, 3 token tiles (odd pair)
])
def test_k_grouped_parity(fg, M, N, ks):
    rng = np.random.default_rng(M + N + sum(ks))
    qa, sa, qb, sb = operands(rng, M, N, ks)
    got, status = run(fg, qa, sa, qb, sb, ks)
    assert status == 0
    ref = oracle.k_grouped(qa, sa, qb, sb, np.array(ks, np.int32))
    for e, k in enumerate(ks):
        if k == 0:
            assert np.all(got[e] == 0.0), "an expert without tokens gets zeros"
            continue
        check_gemm(got[e], ref[e], "k-grouped e=%d" % e)
        # fp32 accumulation: far inside the bf16 bar
        rms = np.sqrt(np.mean(ref[e] ** 2))
        assert np.max(np.abs(got[e] - ref[e])) <= 2.0 ** -12 * rms + 2.0 ** -14 * np.abs(ref[e]).max()


def test_k_grouped_integer_exact(fg):
    """Entries in {-1, 0, 1}, power-of-two scales varying by row and block:
    every product and partial sum is exact in fp32, so the result is exact."""
    rng = np.random.default_rng(51)
    M, N, ks = 160, 224, [256, 384]
    T = sum(ks)
    qa = oracle.e4m3_encode(rng.integers(-1, 2, size=(M, T)).astype(np.float32))
    qb = oracle.e4m3_encode(rng.integers(-1, 2, size=(N, T)).astype(np.float32))
    sa = (2.0 ** rng.integers(-3, 3, size=(M, T // 128))).astype(np.float32)
    sb = (2.0 ** rng.integers(-3, 3, size=(N, T // 128))).astype(np.float32)
    got, status = run(fg, qa, sa, qb, sb, ks)
    assert status == 0
    assert np.array_equal(got, oracle.k_grouped(qa, sa, qb, sb, np.array(ks, np.int32)))


def test_k_grouped_all_empty_and_bad_counts(fg):
    rng = np.random.default_rng(52)
    M, N = 128, 224
    qa, sa, qb, sb = operands(rng, M, N, [128])
    # T = 0 is allowed: every expert is empty (real buffers, T passed as 0)
    A = to_torch(np.zeros((M, 128), np.uint8))
    B = to_torch(np.zeros((N, 128), np.uint8))
    SA = to_torch(np.zeros((1, 128), np.float32))
    SB = to_torch(np.zeros((1, 224), np.float32))
    D = to_torch(np.full((2, M, N), np.nan, np.float32))
    ks0 = to_torch(np.zeros(2, np.int32))
    lib = fg.load_library()
    st = lib.fp8_k_grouped_gemm_nt_ue8m0(A.data_ptr(), SA.data_ptr(), B.data_ptr(), SB.data_ptr(),
                                         D.data_ptr(), ks0.data_ptr(), 2, M, N, 0,
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    assert np.all(D.cpu().numpy() == 0.0)
    # a count that is not a multiple of 128 is reported on the device
    got, status = run(fg, qa, sa, qb, sb, [100, 28])
    assert status == 4
