"""The masked expert FFN entry point that allocates nothing
(fp8_moe_ffn_masked_ue8m0_noalloc), called through the C ABI, against the
entry point that takes a workspace.

Some callers are handed buffers for their inputs and outputs but may not
allocate any further device memory (a serving runtime that reserves the
GPU's memory at start-up, a plugin inside another framework's memory
manager). For them the no-allocation variant keeps its ready counters in a
fixed array of the library's own device memory instead of a workspace.

Every call shares that array, which keeps the previous call's counts: two
calls in a row must each clear what they use and give the same result. This
file runs last (pytest collects files in name order), so that a run stopping
at its first failure has run every other test first; it also passes alone in
a fresh process.
"""
import ctypes

import numpy as np
import pytest

import oracle
import workloads
from helpers import bf16_bits_to_f64, check_gemm, sa_to_mn_major, tensor_bf16_bits, to_torch

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SENT16 = 0xFFFF
SENT8 = 0x7F


@pytest.fixture(scope="module")
def fg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_04_b200 as m
    m.load_library()
    yield m
    m.set_ffn_mode(0)


def _outputs(G, M_max, H, I, fg):
    Hq = to_torch(np.full((G, M_max, I), SENT8, np.uint8))
    SH = to_torch(np.full((G, I // 128, fg.sfa_stride(M_max)), np.nan, np.float32))
    Y = to_torch(np.full((G, M_max, H), SENT16, np.uint16).view(np.int16)).view(torch.bfloat16)
    return Hq, SH, Y


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_no_alloc_ffn_matches_the_workspace_entry_point(fg):
    G, M_max, H, I = 4, 192, 256, 256
    masked_m = np.array([130, 0, 77, 192], np.int32)
    expected = 100
    rng = np.random.default_rng(2024)
    x = workloads.bf16_bits(rng.standard_normal((G, M_max, H)).astype(np.float32))
    xq, sx = oracle.per_token_cast(x, ue8m0=True)
    w1 = workloads.normal_bf16(rng, (G, 2 * I, H), 0.05)
    w2 = workloads.normal_bf16(rng, (G, H, I), 0.05)
    w1q, sw1 = oracle.per_block_cast(w1, ue8m0=True)
    w2q, sw2 = oracle.per_block_cast(w2, ue8m0=True)
    X, SX = to_torch(xq), to_torch(sa_to_mn_major(sx))
    W1, SW1, W2, SW2 = to_torch(w1q), to_torch(sw1), to_torch(w2q), to_torch(sw2)
    MM = to_torch(masked_m)

    # the existing entry point, in the same (one-launch) form, with a workspace
    fg.set_ffn_mode(1)
    Hq_ref, SH_ref, Y_ref = _outputs(G, M_max, H, I, fg)
    fg.fp8_moe_ffn_masked_ue8m0(X, SX, W1, SW1, W2, SW2, Hq_ref, SH_ref, Y_ref, MM, expected)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    fg.set_ffn_mode(0)
    y_ref = bf16_bits_to_f64(tensor_bf16_bits(Y_ref))
    hq_ref = Hq_ref.cpu().numpy()

    lib = fg.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):  # the second call finds the first call's counts in the array
        Hq, SH, Y = _outputs(G, M_max, H, I, fg)
        st = lib.fp8_moe_ffn_masked_ue8m0_noalloc(
            _p(X), _p(SX), _p(W1), _p(SW1), _p(W2), _p(SW2), _p(Hq), _p(SH), None, _p(Y), _p(MM),
            G, M_max, H, I, expected, stream)
        assert st == 0, lib.fg_last_error()
        torch.cuda.synchronize()
        assert fg.get_device_status() == 0
        y = bf16_bits_to_f64(tensor_bf16_bits(Y))
        hq = Hq.cpu().numpy()
        for e, v in enumerate(masked_m):
            if v:
                check_gemm(y[e, :v], y_ref[e, :v], "no-alloc FFN call %d expert %d" % (call, e))
                assert np.array_equal(hq[e, :v], hq_ref[e, :v]), "requantized activations differ"
            assert np.all(tensor_bf16_bits(Y)[e, v:] == SENT16), "rows past masked_m stay unwritten"


def test_no_alloc_ffn_rejects_problems_beyond_its_scratch(fg):
    """G * ceil(M_max / 128) above the fixed 4096 counters: a clear error,
    nothing launched (the pointers are never dereferenced)."""
    lib = fg.load_library()
    t = torch.zeros(16, dtype=torch.uint8, device="cuda")
    G, M_max = 1024, 1024  # 8192 token tiles
    st = lib.fp8_moe_ffn_masked_ue8m0_noalloc(*([_p(t)] * 11), G, M_max, 256, 256, 64, None)
    assert st == fg.FG_ERR_UNSUPPORTED
    assert b"4096" in lib.fg_last_error()
