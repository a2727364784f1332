"""The seeded input generators and the algorithmic work counts (host logic).

The generators feed both the oracle and the CUDA path, so their recipe is
checked here on its own: bf16 rounding, the contiguous layout, the routing
counts, the decode outliers and the masked counts. The work counts are the
roofline numerator bench.py reports; they are checked against the terms of
their definition written out with the sizes of each workload.
"""
import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")


# ------------------------------------------------------------------ bf16

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(4096).astype(np.float32) * np.float32(s)
                        for s in (1e-30, 1e-3, 1.0, 7.0, 1e30)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(workloads.bf16_bits(x), want)


def test_bf16_rounding_ties_go_to_even():
    # 1 + 2^-8 lies halfway between bf16 1.0 (0x3F80) and 1.0078125 (0x3F81);
    # 1.0078125 + 2^-8 halfway between 0x3F81 and 0x3F82
    x = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x3F808001], np.uint32).view(np.float32)
    assert workloads.bf16_bits(x).tolist() == [0x3F80, 0x3F82, 0xBF80, 0x3F81]


def test_bf16_widening_is_exact_on_every_finite_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = workloads.bf16_to_f32(bits)
    finite = np.isfinite(f)
    assert np.array_equal(workloads.bf16_bits(f[finite]), bits[finite])
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(f.view(np.uint32)[finite], want.view(np.uint32)[finite])


# ------------------------------------------------------------------ layouts and recipes

def test_contiguous_layout_pads_each_group_to_128_rows():
    mi, M_total = workloads.contiguous_layout(np.array([130, 0, 5, 128]))
    assert M_total == 256 + 0 + 128 + 128
    want = np.full(M_total, -1, np.int32)
    want[0:130] = 0
    want[256:261] = 2
    want[384:512] = 3
    assert np.array_equal(mi, want)


def test_contiguous_inputs_zero_their_padding_rows():
    inp = workloads.contiguous(N=256, K=256, counts=np.array([130, 0, 5]), seed=3)
    valid = inp.m_indices >= 0
    assert inp.a.shape == (inp.M_total, 256) and inp.b.shape == (3, 256, 256)
    assert np.all(inp.a[~valid] == 0)
    assert np.all(np.any(inp.a[valid] != 0, axis=1))


def test_routing_counts_are_top8_of_256_with_zipf_weights():
    c = workloads.zipf_top8_counts(0)
    assert c.shape == (256,) and c.sum() == 4096 * 8
    assert c.max() <= 4096  # an expert is picked at most once per token
    # the hottest ids carry the most tokens (weights (i+1)^-1.1)
    assert c[0] == c.max() and c[0] > c[3] > c[7] > c[100]


def test_decode_inputs_have_one_outlier_row():
    inp = workloads.make("decode_64x4096x7168")
    assert inp.a.shape == (64, 7168) and inp.b.shape == (4096, 7168)
    rms = np.sqrt(np.mean(workloads.bf16_to_f32(inp.a).astype(np.float64) ** 2, axis=1))
    big = rms > 10.0
    assert big.sum() == 1  # ceil(1% of 64) rows scaled by 30
    assert abs(rms[big][0] - 30.0) < 1.5 and np.all(np.abs(rms[~big] - 1.0) < 0.1)
    sd = float(np.std(workloads.bf16_to_f32(inp.b[:512]).astype(np.float64)))
    assert abs(sd - 0.02) < 0.0005
    again = workloads.make("decode_64x4096x7168")
    assert np.array_equal(inp.a, again.a) and np.array_equal(inp.b, again.b)


def test_masked_counts_are_within_capacity_and_seeded():
    m = workloads.masked(G=32, M_max=64, N=128, K=128, seed=7)
    assert m.masked_m.dtype == np.int32 and m.masked_m.shape == (32,)
    assert np.all((m.masked_m >= 0) & (m.masked_m <= 64))
    assert np.array_equal(m.masked_m, workloads.masked(G=32, M_max=64, N=128, K=128, seed=7).masked_m)


def test_k_grouped_token_ranges():
    k = workloads.k_grouped(M=128, N=256, G=8, seed=0)
    counts = workloads.zipf_top8_counts(0)[:8]
    assert np.array_equal(k.counts, counts)
    assert np.all(k.ks % 128 == 0) and np.all(k.ks >= k.counts) and np.all(k.ks - k.counts < 128)
    assert k.T == int(k.ks.sum())
    # padding tokens of each expert's range are zero in both operands
    start = 0
    for c, n in zip(k.counts, k.ks):
        assert np.all(k.a[:, start + c:start + n] == 0) and np.all(k.b[:, start + c:start + n] == 0)
        start += n


# ------------------------------------------------------------------ algorithmic work

def test_work_counts_dense_shapes():
    d = workloads.make("decode_64x4096x7168")
    f, b = workloads.flops_and_bytes("dense", d)
    assert f == 2 * 64 * 4096 * 7168
    # A codes, A scales (one per 128), B codes, B scales (one per 128 x 128), D bf16
    assert b == 64 * 7168 + 4 * 64 * 56 + 4096 * 7168 + 4 * 32 * 56 + 2 * 64 * 4096 == 30364672
    p = workloads.DenseInputs(a=None, b=None, M=4096, N=2112, K=7168)
    f, b = workloads.flops_and_bytes("dense", p)
    assert f == 2 * 4096 * 2112 * 7168
    assert b == 4096 * 7168 + 4 * 4096 * 56 + 2112 * 7168 + 4 * 17 * 56 + 2 * 4096 * 2112


def test_work_counts_grouped_count_valid_rows_and_used_experts():
    c = workloads.ContiguousInputs(a=None, b=None, m_indices=None, counts=np.array([130, 0, 5]),
                                   M_total=512, N=256, K=384, G=3)
    f, b = workloads.flops_and_bytes("contiguous", c)
    assert f == 2 * 135 * 256 * 384
    # padding rows and the expert without tokens are not work
    assert b == 135 * 384 + 4 * 135 * 3 + 2 * (256 * 384 + 4 * 2 * 3) + 2 * 135 * 256
    m = workloads.MaskedInputs(a=None, b=None, masked_m=np.array([0, 3, 64, 0], np.int32),
                               G=4, M_max=64, N=128, K=256)
    f, b = workloads.flops_and_bytes("masked", m)
    assert f == 2 * 67 * 128 * 256
    assert b == 67 * 256 + 4 * 67 * 2 + 2 * (128 * 256 + 4 * 1 * 2) + 2 * 67 * 128


def test_quant_workload_is_the_prefill_activation():
    q = workloads.make("quant_4096x7168")
    d = workloads.dense(4096, 2112, 7168)
    assert np.array_equal(q.a, d.a)
    # bf16 read, e4m3 written, one fp32 scale per 128 elements written
    assert workloads.flops_and_bytes("quant", q) == (0.0, 4096 * 7168 * 3 + 4 * 4096 * 56)


def test_work_counts_dequant_ffn_and_k_grouped():
    q = workloads.DequantInputs(b=None, N=300, K=256)
    assert workloads.flops_and_bytes("dequant", q) == (0.0, 300 * 256 + 4 * 3 * 2 + 2 * 300 * 256)
    ffn = workloads.FfnInputs(a=None, w1=None, w2=None, m_indices=None, counts=np.array([10, 0]),
                              M_total=256, H=256, I=128, G=2)
    f, b = workloads.flops_and_bytes("ffn", ffn)
    assert f == 2 * 10 * 256 * 256 + 2 * 10 * 256 * 128
    w = 256 * 256 + 256 * 128 + 4 * (2 * 2 + 2 * 1)  # W1, W2 and their block scales, one expert
    h = 10 * 128 + 4 * 10 * 1                         # requantized activations and scales
    assert b == 10 * 256 + 4 * 10 * 2 + w + 2 * h + 2 * 10 * 256
    k = workloads.KGroupedInputs(a=None, b=None, ks=np.array([128, 256], np.int32),
                                 counts=np.array([100, 200]), M=64, N=96, T=384, G=2)
    f, b = workloads.flops_and_bytes("kgrouped", k)
    assert f == 2 * 64 * 96 * 300
    assert b == (64 + 96) * 384 + 4 * (64 + 96) * 3 + 4 * 2 * 64 * 96


def test_expert_parallel_inputs():
    """The expert-parallel workload's routing: k distinct experts per token
    (uniform Gumbel-top-k), router weights summing to one per token, and a
    seed that reproduces it; small sizes stand in for the bench's."""
    a = workloads.expert_parallel(T=64, E=16, k=4, N=128, K=256, M_max=64, seed=3)
    b = workloads.expert_parallel(T=64, E=16, k=4, N=128, K=256, M_max=64, seed=3)
    assert np.array_equal(a.topk, b.topk) and np.array_equal(a.x, b.x)
    assert a.topk.shape == (64, 4) and a.topk.dtype == np.int32
    assert all(len(set(r)) == 4 for r in a.topk.tolist())
    assert a.topk.min() >= 0 and a.topk.max() < 16
    assert np.allclose(a.topk_w.sum(axis=1), 1.0, atol=1e-6) and (a.topk_w > 0).all()
    assert a.counts.sum() == 64 * 4 and a.w.shape == (16, 128, 256)
    c = workloads.expert_parallel(T=64, E=16, k=4, N=128, K=256, M_max=64, seed=4)
    assert not np.array_equal(a.topk, c.topk)
