"""The expert FFN (GEMM1 -> SwiGLU -> per-token UE8M0 requantization -> GEMM2)
on the GPU against the CPU oracle, through the C ABI.

For every case:
  * GU (the first GEMM's bf16 output) is within the GEMM tolerance of the
    oracle's first grouped GEMM;
  * the quantized activations and their scales are bit-exact with the
    oracle's SwiGLU and UE8M0 quantizer applied to the GPU's own GU values
    (the activation is a fixed sequence of IEEE operations on both sides);
  * Y is within the GEMM tolerance of the oracle's second grouped GEMM on the
    GPU's quantized activations, and of the oracle's whole chain;
  * rows that are not valid (padding, past masked_m) are left untouched.
"""
import numpy as np
import pytest

import oracle
import workloads
from helpers import bf16_bits_to_f64, check_gemm, sa_from_mn_major, sa_to_mn_major, tensor_bf16_bits, to_torch

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


@pytest.fixture(params=[1, 2], ids=["one-launch", "two-launches"])
def mode(request, fg):
    """Both forms of the FFN: one persistent launch, and two launches."""
    fg.set_ffn_mode(request.param)
    yield request.param
    fg.set_ffn_mode(0)


def _filled(shape, value, dtype):
    return to_torch(np.full(shape, value, dtype))


def _bf16(shape):
    return _filled(shape, SENT16, np.uint16).view(torch.int16).view(torch.bfloat16)


def _weights(rng, G, H, I):
    w1 = workloads.normal_bf16(rng, (G, 2 * I, H), 0.05)
    w2 = workloads.normal_bf16(rng, (G, H, I), 0.05)
    w1q, sw1 = oracle.per_block_cast(w1, ue8m0=True)
    w2q, sw2 = oracle.per_block_cast(w2, ue8m0=True)
    return w1q, sw1, w2q, sw2


def _check_requant(gu_rows, hq_rows, sh_rows, I, what):
    """Bit-exact: oracle SwiGLU + UE8M0 quantizer on the GPU's own GU rows."""
    h = oracle.swiglu(gu_rows[:, :I], gu_rows[:, I:])
    q, s = oracle.per_token_cast(h, ue8m0=True)
    assert np.array_equal(q, hq_rows), "%s: requantized codes differ" % what
    assert np.array_equal(s.view(np.uint32), sh_rows.view(np.uint32)), "%s: scales differ" % what


def run_contiguous(fg, xq, sx, w1q, sw1, w2q, sw2, mi):
    M, H = xq.shape
    G, I2, _ = w1q.shape
    I = I2 // 2
    Hq = _filled((M, I), SENT8, np.uint8)
    SH = _filled((I // 128, oracle_stride(M)), np.nan, np.float32)
    GU = _bf16((M, I2))
    Y = _bf16((M, H))
    fg.fp8_moe_ffn_contiguous_ue8m0(to_torch(xq), to_torch(sa_to_mn_major(sx)), to_torch(w1q),
                                    to_torch(sw1), to_torch(w2q), to_torch(sw2), Hq, SH, Y,
                                    to_torch(mi.astype(np.int32)), GU=GU)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    sh = sa_from_mn_major(SH.cpu().numpy()[None], M)[0]
    return tensor_bf16_bits(GU), Hq.cpu().numpy(), sh, tensor_bf16_bits(Y)


def oracle_stride(M):
    return (M + 3) // 4 * 4


@pytest.mark.parametrize("counts,H,I", [([130, 0, 200], 256, 256), ([1], 128, 128),
                                        ([300, 77, 128, 5], 512, 384)])
def test_ffn_contiguous_parity(fg, mode, counts, H, I):
    rng = np.random.default_rng(sum(counts) + H + I)
    G = len(counts)
    # groups stacked along M, each padded to 128 rows
    blocks = [-(-c // 128) * 128 for c in counts]
    M = sum(blocks)
    mi = np.full(M, -1, np.int32)
    r = 0
    for e, (c, b) in enumerate(zip(counts, blocks)):
        mi[r:r + c] = e
        r += b
    x = np.zeros((M, H), np.uint16)
    valid = mi >= 0
    x[valid] = workloads.bf16_bits(rng.standard_normal((int(valid.sum()), H)).astype(np.float32))
    xq, sx = oracle.per_token_cast(x, ue8m0=True)
    w1q, sw1, w2q, sw2 = _weights(rng, G, H, I)
    gu, hq, sh, y = run_contiguous(fg, xq, sx, w1q, sw1, w2q, sw2, mi)
    ref1 = oracle.grouped_contiguous(xq, sx, w1q, sw1, mi)
    check_gemm(bf16_bits_to_f64(gu[valid]), ref1[valid], "ffn GEMM1 %s" % counts)
    _check_requant(gu[valid], hq[valid], sh[valid], I, "ffn %s" % counts)
    ref2 = oracle.grouped_contiguous(hq * valid[:, None], sh, w2q, sw2, mi)
    check_gemm(bf16_bits_to_f64(y[valid]), ref2[valid], "ffn GEMM2 %s" % counts)
    _, _, _, yo = oracle.moe_ffn_contiguous(xq, sx, w1q, sw1, w2q, sw2, mi)
    check_gemm(bf16_bits_to_f64(y[valid]), yo[valid], "ffn end to end %s" % counts)
    assert np.all(y[~valid] == SENT16) and np.all(gu[~valid] == SENT16)
    assert np.all(hq[~valid] == SENT8)


def run_masked(fg, xq, sx, w1q, sw1, w2q, sw2, mm, expected_m):
    G, M_max, H = xq.shape
    I = w1q.shape[1] // 2
    Hq = _filled((G, M_max, I), SENT8, np.uint8)
    SH = _filled((G, I // 128, oracle_stride(M_max)), np.nan, np.float32)
    GU = _bf16((G, M_max, 2 * I))
    Y = _bf16((G, M_max, H))
    fg.fp8_moe_ffn_masked_ue8m0(to_torch(xq), to_torch(sa_to_mn_major(sx)), to_torch(w1q),
                                to_torch(sw1), to_torch(w2q), to_torch(sw2), Hq, SH, Y,
                                to_torch(mm.astype(np.int32)), expected_m, GU=GU)
    torch.cuda.synchronize()
    status = fg.get_device_status()
    sh = sa_from_mn_major(SH.cpu().numpy(), M_max)
    return tensor_bf16_bits(GU), Hq.cpu().numpy(), sh, tensor_bf16_bits(Y), status


@pytest.mark.parametrize("masked_m,M_max,H,I,expected", [
    ([0, 80, 17], 80, 256, 128, 40),           # single-CTA tiles
    ([256, 3, 0, 200], 256, 256, 256, 200),    # CTA pairs (expected rows > 128)
    ([130, 1], 192, 384, 128, 130),            # pairs whose second tile lies past M_max
])
def test_ffn_masked_parity(fg, mode, masked_m, M_max, H, I, expected):
    rng = np.random.default_rng(M_max + H + I)
    G = len(masked_m)
    mm = np.array(masked_m, np.int32)
    x = workloads.bf16_bits(rng.standard_normal((G, M_max, H)).astype(np.float32))
    xq, sx = oracle.per_token_cast(x, ue8m0=True)
    # rows past masked_m hold e4m3 NaN codes: they must not reach valid outputs
    xq_nan = xq.copy()
    for e, v in enumerate(masked_m):
        xq_nan[e, v:] = 0x7F
    w1q, sw1, w2q, sw2 = _weights(rng, G, H, I)
    gu, hq, sh, y, status = run_masked(fg, xq_nan, sx, w1q, sw1, w2q, sw2, mm, expected)
    assert status == 0
    gu_o, hq_o, sh_o, y_o = oracle.moe_ffn_masked(xq, sx, w1q, sw1, w2q, sw2, mm)
    for e, v in enumerate(masked_m):
        if v:
            ref1 = oracle.grouped_masked(xq[e:e + 1], sx[e:e + 1], w1q[e:e + 1], sw1[e:e + 1],
                                         np.array([v], np.int32))[0, :v]
            check_gemm(bf16_bits_to_f64(gu[e, :v]), ref1, "ffn masked GEMM1 e=%d" % e)
            _check_requant(gu[e, :v], hq[e, :v], sh[e, :v], I, "ffn masked e=%d" % e)
            ref2 = oracle.grouped_masked(hq[e:e + 1], sh[e:e + 1], w2q[e:e + 1], sw2[e:e + 1],
                                         np.array([v], np.int32))[0, :v]
            check_gemm(bf16_bits_to_f64(y[e, :v]), ref2, "ffn masked GEMM2 e=%d" % e)
            check_gemm(bf16_bits_to_f64(y[e, :v]), y_o[e, :v], "ffn masked end to end e=%d" % e)
        assert np.all(y[e, v:] == SENT16) and np.all(gu[e, v:] == SENT16)
        assert np.all(hq[e, v:] == SENT8)


def test_ffn_contiguous_deepseek_expert_shape(fg, mode):
    """An expert shape of the MoE layers (H = 7168, I = 2048) on the
    contiguous workload's token counts: every valid output of GU and Y, and the
    requantization of every valid row bit for bit."""
    inp = workloads.make("contiguous_8x4096x7168")
    H, I = 7168, 2048
    mi = inp.m_indices
    rng = np.random.default_rng(31)
    xq, sx = oracle.per_token_cast(inp.a, ue8m0=True)
    w1q, sw1, w2q, sw2 = _weights(rng, inp.G, H, I)
    gu, hq, sh, y = run_contiguous(fg, xq, sx, w1q, sw1, w2q, sw2, mi)
    valid = mi >= 0
    ref1 = oracle.grouped_contiguous(xq, sx, w1q, sw1, mi)
    check_gemm(bf16_bits_to_f64(gu[valid]), ref1[valid], "ffn GEMM1 full")
    del ref1
    _check_requant(gu[valid], hq[valid], sh[valid], I, "ffn full")
    ref2 = oracle.grouped_contiguous(hq * valid[:, None], sh, w2q, sw2, mi)
    check_gemm(bf16_bits_to_f64(y[valid]), ref2[valid], "ffn GEMM2 full")
    assert np.all(y[~valid] == SENT16)


def test_ffn_workspace_needs_no_initialisation(fg):
    fg.set_ffn_mode(1)  # the one-launch form reads the counters
    """The one-kernel FFN's second GEMM waits on ready counters in the
    workspace, which each call clears itself: a workspace holding garbage
    (counters that would read as complete) gives the same bits as a fresh
    one, and calls in a row reusing it do too."""
    counts = [300, 77, 128, 5]                    # odd runs: pair partners of other experts
    H, I = 256, 384
    rng = np.random.default_rng(77)
    G = len(counts)
    blocks = [-(-c // 128) * 128 for c in counts]
    M = sum(blocks)
    mi = np.full(M, -1, np.int32)
    r = 0
    for e, (c, b) in enumerate(zip(counts, blocks)):
        mi[r:r + c] = e
        r += b
    x = np.zeros((M, H), np.uint16)
    valid = mi >= 0
    x[valid] = workloads.bf16_bits(rng.standard_normal((int(valid.sum()), H)).astype(np.float32))
    xq, sx = oracle.per_token_cast(x, ue8m0=True)
    w1q, sw1, w2q, sw2 = _weights(rng, G, H, I)
    args = [to_torch(xq), to_torch(sa_to_mn_major(sx)), to_torch(w1q), to_torch(sw1),
            to_torch(w2q), to_torch(sw2)]
    mit = to_torch(mi)
    ws = fg.empty_ffn_workspace(fg.FG_LAYOUT_CONTIGUOUS, M, G)
    outs = []
    for fill in (0x00, 0x7F, 0x7F, 0xFF):
        ws.fill_(fill)
        Hq = _filled((M, I), SENT8, np.uint8)
        SH = _filled((I // 128, oracle_stride(M)), np.nan, np.float32)
        Y = _bf16((M, H))
        fg.fp8_moe_ffn_contiguous_ue8m0(*args, Hq, SH, Y, mit, ws=ws)
        torch.cuda.synchronize()
        assert fg.get_device_status() == 0
        outs.append((tensor_bf16_bits(Y), Hq.cpu().numpy(), SH.cpu().numpy()))
    for y, hq, sh in outs[1:]:
        assert np.array_equal(y, outs[0][0]) and np.array_equal(hq, outs[0][1])
        assert np.array_equal(sh.view(np.uint32), outs[0][2].view(np.uint32))
    _, _, _, yo = oracle.moe_ffn_contiguous(xq, sx, w1q, sw1, w2q, sw2, mi)
    check_gemm(bf16_bits_to_f64(outs[0][0][valid]), yo[valid], "ffn end to end, reused workspace")
    fg.set_ffn_mode(0)


def test_ffn_workspace_too_small(fg):
    xq = torch.zeros((256, 128), dtype=torch.uint8, device="cuda")
    sx = torch.ones((1, 256), dtype=torch.float32, device="cuda")
    w1 = torch.zeros((1, 256, 128), dtype=torch.uint8, device="cuda")
    sw1 = torch.ones((1, 2, 1), dtype=torch.float32, device="cuda")
    w2 = torch.zeros((1, 128, 128), dtype=torch.uint8, device="cuda")
    sw2 = torch.ones((1, 1, 1), dtype=torch.float32, device="cuda")
    Hq = torch.zeros((256, 128), dtype=torch.uint8, device="cuda")
    sh = torch.zeros((1, 256), dtype=torch.float32, device="cuda")
    Y = torch.zeros((256, 128), dtype=torch.bfloat16, device="cuda")
    mi = torch.zeros(256, dtype=torch.int32, device="cuda")
    ws = torch.zeros(4, dtype=torch.uint8, device="cuda")
    with pytest.raises(fg.FP8GemmError) as ei:
        fg.fp8_moe_ffn_contiguous_ue8m0(xq, sx, w1, sw1, w2, sw2, Hq, sh, Y, mi, ws=ws)
    assert ei.value.status == fg.FG_ERR_INVALID_ARG
