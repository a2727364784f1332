"""The tensor-core rate kernel (fg_fp8_mma_peak): every CTA's accumulator is
the exact integer its C-ABI declaration states, for a few launch lengths, and
bad arguments are refused before anything launches."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_04_b200 as m
    m.load_library()
    return m


def _expected(iters):
    # written out from the declaration: a[m][k] and b[n][k] over all 128 K of
    # a block (k % 16 picks the value), summed over `iters` blocks
    k = np.arange(128)
    a = (2 * np.arange(128)[:, None] + 3 * (k[None, :] % 16)) % 5 - 2
    n = np.arange(256)[:, None]
    b = (3 * n + 2 * (k[None, :] % 16) + n // 16) % 5 - 2
    return iters * (a.astype(np.int64) @ b.T.astype(np.int64))


@pytest.mark.parametrize("iters", [1, 15, 16, 17, 33, 1000])
def test_every_cta_holds_the_exact_accumulator(fg, iters):
    ctas = fg.fp8_mma_peak_ctas()
    assert ctas >= 1
    out = torch.full((ctas, 128, 256), float("nan"), device="cuda")
    fg.fp8_mma_peak(iters, out)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    got = out.cpu().numpy()
    want = _expected(iters).astype(np.float32)
    for c in range(ctas):
        assert np.array_equal(got[c], want), "CTA %d" % c


def test_largest_launch_stays_exact(fg):
    ctas = fg.fp8_mma_peak_ctas()
    out = torch.empty((ctas, 128, 256), device="cuda")
    fg.fp8_mma_peak(32768, out)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    assert np.array_equal(out[0].cpu().numpy(), _expected(32768).astype(np.float32))
    assert np.array_equal(out[-1].cpu().numpy(), _expected(32768).astype(np.float32))


def test_bad_arguments(fg):
    ctas = fg.fp8_mma_peak_ctas()
    out = torch.empty((ctas, 128, 256), device="cuda")
    for bad in (0, -1, 32769):
        with pytest.raises(fg.FP8GemmError):
            fg.fp8_mma_peak(bad, out)
    with pytest.raises(fg.FP8GemmError):
        fg.fp8_mma_peak(4, torch.empty((ctas, 128, 255), device="cuda"))
