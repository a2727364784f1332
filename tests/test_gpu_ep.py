"""Expert-parallel dispatch and combine on the GPU: each kernel against its
plain CPU stand-in (tests/ep_reference.py; data movement bit for bit), and
the whole layer (quantize, dispatch, masked grouped GEMM, combine) on a
one-GPU NCCL group against the oracle. (Several GPUs are not available to
these tests; the exchange between ranks is covered on CPU gloo ranks by
tests/test_ep_cpu.py.)"""
import socket

import numpy as np
import pytest

import ep_reference
import oracle
import workloads
from helpers import bf16_bits_to_f64, check_gemm, tensor_bf16_bits, to_torch

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_04_b200 as m
    m.load_library()
    return m


def _topk(rng, T, k, E, drop=0.1):
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    topk[rng.random((T, k)) < drop] = -1
    return topk


def test_layout_and_pack(fg):
    rng = np.random.default_rng(1)
    T, k, E, K = 300, 4, 16, 384
    topk = _topk(rng, T, k, E)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, k), dtype=torch.int32, device="cuda")
    fg.ep_dispatch_layout(to_torch(topk), E, counts, pos)
    c_ref, p_ref = ep_reference.layout_ref(topk, E)
    assert np.array_equal(counts.cpu().numpy(), c_ref)
    assert np.array_equal(pos.cpu().numpy(), p_ref)
    # pack: rows and scales land in send order
    x = workloads.bf16_bits(rng.standard_normal((T, K)).astype(np.float32))
    q = torch.empty((T, K), dtype=torch.uint8, device="cuda")
    s = fg.empty_sfa(1, T, K, "cuda")
    fg.per_token_cast_to_fp8(to_torch(x.view(np.int16)).view(torch.bfloat16), q, s)
    P = int(c_ref.sum())
    send_q = torch.full((P, K), 0x7F, dtype=torch.uint8, device="cuda")
    send_s = torch.full((P, K // 128), float("nan"), device="cuda")
    fg.ep_dispatch_pack(q, s[0], pos, send_q, send_s)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    qn, sn = q.cpu().numpy(), s[0].cpu().numpy()
    want_q = np.zeros((P, K), np.uint8)
    want_s = np.zeros((P, K // 128), np.float32)
    for t in range(T):
        for j in range(k):
            if p_ref[t, j] >= 0:
                want_q[p_ref[t, j]] = qn[t]
                want_s[p_ref[t, j]] = sn[:, t]
    assert np.array_equal(send_q.cpu().numpy(), want_q)
    assert np.array_equal(send_s.cpu().numpy().view(np.uint32), want_s.view(np.uint32))


@pytest.mark.parametrize("C", [300, 37])  # 37: destinations with more pairs drop the rest
def test_layout_capacity(fg, C):
    rng = np.random.default_rng(11)
    T, k, E, W = 300, 4, 16, 4
    topk = _topk(rng, T, k, E)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, k), dtype=torch.int32, device="cuda")
    fg.ep_dispatch_layout_capacity(to_torch(topk), E, W, C, counts, pos)
    torch.cuda.synchronize()
    c_ref, p_ref = ep_reference.layout_capacity_ref(topk, E, W, C)
    dropped = bool(((p_ref < 0) & (topk >= 0)).any())
    assert fg.get_device_status() == (6 if dropped else 0)  # FG_DEVICE_EP_OVERFLOW
    assert dropped == (C == 37)
    assert np.array_equal(counts.cpu().numpy(), c_ref)
    assert np.array_equal(pos.cpu().numpy(), p_ref)


def test_unpack_capacity_skips_the_unused_rows(fg):
    rng = np.random.default_rng(12)
    W, G, K, C, M_max = 3, 4, 256, 30, 64
    recv_counts = rng.integers(0, 8, (W, G)).astype(np.int32)
    recv_counts[2] = 0  # a source that sent nothing
    recv_q = rng.integers(0, 0x7E, (W * C, K)).astype(np.uint8)
    recv_s = rng.random((W * C, K // 128)).astype(np.float32)
    A = torch.full((G, M_max, K), 0x7F, dtype=torch.uint8, device="cuda")
    sfa = torch.full((G, K // 128, fg.sfa_stride(M_max)), float("nan"), device="cuda")
    mm = torch.empty(G, dtype=torch.int32, device="cuda")
    slot = torch.empty(W * C, dtype=torch.int32, device="cuda")
    fg.ep_dispatch_unpack_masked_capacity(to_torch(recv_q), to_torch(recv_s), to_torch(recv_counts), C, A,
                                          sfa, mm, slot)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 0
    a_ref, sa_ref, mm_ref, slot_ref = ep_reference.unpack_capacity_ref(recv_q, recv_s, recv_counts, C, M_max)
    assert np.array_equal(mm.cpu().numpy(), mm_ref)
    assert np.array_equal(slot.cpu().numpy(), slot_ref)
    An, sn = A.cpu().numpy(), sfa.cpu().numpy()
    for g in range(G):
        v = mm_ref[g]
        assert np.array_equal(An[g, :v], a_ref[g, :v])
        assert np.array_equal(sn[g, :, :v].T.view(np.uint32), sa_ref[g, :v].view(np.uint32))


def test_layout_expert_out_of_range(fg):
    topk = np.array([[0, 7], [3, 1]], np.int32)  # 7 >= E
    counts = torch.empty(4, dtype=torch.int32, device="cuda")
    pos = torch.empty((2, 2), dtype=torch.int32, device="cuda")
    fg.ep_dispatch_layout(to_torch(topk), 4, counts, pos)
    torch.cuda.synchronize()
    assert fg.get_device_status() == 3  # FG_DEVICE_BAD_M_INDEX
    assert counts.cpu().tolist() == [1, 1, 0, 1]
    assert pos.cpu().tolist() == [[0, -1], [2, 1]]


@pytest.mark.parametrize("M_max", [64, 20])  # 20: some experts overflow
def test_unpack_gather(fg, M_max):
    rng = np.random.default_rng(2)
    W, G, K, N = 3, 4, 256, 136
    recv_counts = rng.integers(0, 12, (W, G)).astype(np.int32)
    recv_counts[1, 2] = 0
    R = int(recv_counts.sum())
    recv_q = rng.integers(0, 0x7E, (R, K)).astype(np.uint8)
    recv_s = rng.random((R, K // 128)).astype(np.float32)
    A = torch.full((G, M_max, K), 0x7F, dtype=torch.uint8, device="cuda")
    sfa = torch.full((G, K // 128, fg.sfa_stride(M_max)), float("nan"), device="cuda")
    mm = torch.empty(G, dtype=torch.int32, device="cuda")
    slot = torch.empty(R, dtype=torch.int32, device="cuda")
    fg.ep_dispatch_unpack_masked(to_torch(recv_q), to_torch(recv_s), to_torch(recv_counts), A, sfa, mm,
                                 slot)
    torch.cuda.synchronize()
    overflow = bool((recv_counts.sum(axis=0) > M_max).any())
    assert fg.get_device_status() == (6 if overflow else 0)  # FG_DEVICE_EP_OVERFLOW
    a_ref, sa_ref, mm_ref, slot_ref = ep_reference.unpack_ref(recv_q, recv_s, recv_counts, M_max)
    assert np.array_equal(mm.cpu().numpy(), mm_ref)
    assert np.array_equal(slot.cpu().numpy(), slot_ref)
    An, sn = A.cpu().numpy(), sfa.cpu().numpy()
    for g in range(G):
        v = mm_ref[g]
        assert np.array_equal(An[g, :v], a_ref[g, :v])
        assert np.array_equal(sn[g, :, :v].T.view(np.uint32), sa_ref[g, :v].view(np.uint32))
    # gather: D rows back in receive order, zeros for dropped rows
    D = workloads.bf16_bits(rng.standard_normal((G, M_max, N)).astype(np.float32))
    out = torch.full((R, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    fg.ep_combine_gather(to_torch(D.view(np.int16)).view(torch.bfloat16), slot, out)
    got = tensor_bf16_bits(out)
    flat = D.reshape(-1, N)
    for r in range(R):
        want = flat[slot_ref[r]] if slot_ref[r] >= 0 else np.zeros(N, np.uint16)
        assert np.array_equal(got[r], want), r


def test_combine(fg):
    rng = np.random.default_rng(3)
    T, k, P, N = 97, 3, 200, 264
    y = workloads.bf16_bits(rng.standard_normal((P, N)).astype(np.float32))
    pos = rng.integers(-1, P, (T, k)).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    fg.ep_combine_reduce(to_torch(y.view(np.int16)).view(torch.bfloat16), to_torch(pos), to_torch(w), out)
    got = tensor_bf16_bits(out)
    want = ep_reference.combine_ref(y, pos, w)
    # the kernel rounds each fp32 multiply-add once; the reference sums in
    # fp64 and rounds to fp32, the same unless that sum was inexact (terms of
    # far apart magnitudes): equal almost everywhere, never more than one
    # bf16 unit apart
    g, r = bf16_bits_to_f64(got), bf16_bits_to_f64(want)
    ulp = np.abs(r) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(g - r) <= ulp)
    assert (got == want).mean() > 0.999


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("capacity", [None, 300, 40])  # 40: some pairs dropped
def test_expert_parallel_layer_on_one_gpu(fg, capacity):
    """The whole layer through NCCL collectives on a one-GPU group: its output
    against the oracle's per-choice GEMM rows and combine (with a fixed
    capacity, of the routing without the pairs it drops)."""
    import datetime

    import torch.distributed as dist

    import moe_grouped_gemm_04_b200.ep as ep
    rng = np.random.default_rng(4)
    E, T, k, K, N, M_max = 8, 150, 2, 512, 256, 128
    w = workloads.normal_bf16(rng, (E, N, K), 0.05)
    wq, ws = oracle.per_block_cast(w)
    x = workloads.bf16_bits(rng.standard_normal((T, K)).astype(np.float32))
    topk = _topk(rng, T, k, E)
    wt = rng.random((T, k)).astype(np.float32)
    created = not dist.is_initialized()
    if created:
        dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _free_port(), rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=60),
                                device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        out = ep.expert_parallel_masked_moe(
            to_torch(x.view(np.int16)).view(torch.bfloat16), to_torch(topk), to_torch(wt), to_torch(wq),
            to_torch(np.ascontiguousarray(ws, np.float32)), E, M_max, capacity=capacity)
        torch.cuda.synchronize()
        assert fg.get_device_status() == (6 if capacity == 40 else 0)
    finally:
        if created:
            dist.destroy_process_group()
    if capacity is not None:
        _, pos = ep_reference.layout_capacity_ref(topk, E, 1, capacity)
        assert ((pos < 0) & (topk >= 0)).any() == (capacity == 40)
        topk = np.where(pos < 0, -1, topk).astype(np.int32)
    got = bf16_bits_to_f64(tensor_bf16_bits(out))
    want = bf16_bits_to_f64(ep_reference.expected_output(x, topk, wt, wq, ws))
    check_gemm(got, want, "expert-parallel layer")
