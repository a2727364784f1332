"""The expert-parallel layer's exchange protocol on two and four gloo CPU ranks.

Each rank runs moe_grouped_gemm_04_b200.ep.expert_parallel_masked_moe with
its own tokens and router choices (uneven counts, dropped choices, experts
with no tokens) and the CPU stand-ins of tests/ep_reference.py in place of
the CUDA kernels; the ranks exchange counts, rows, scales and results with
gloo all-to-all collectives. Every rank's output must equal, bit for bit,
the same computation done without any dispatch: each choice's oracle GEMM row
against its expert's weights, then the weighted combine."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))

torch = pytest.importorskip("torch")

E, K, N, k, M_max = 4, 256, 128, 2, 160  # M_max above any expert's rows (four ranks send up to ~110 to expert 1)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(rank):
    """Rank `rank`'s tokens, choices and weights; every rank draws the same
    expert weights."""
    import oracle
    import workloads
    w = workloads.normal_bf16(np.random.default_rng(7), (E, N, K), 0.05)
    wq, ws = oracle.per_block_cast(w)
    T = 20 + 5 * rank
    rng = np.random.default_rng(100 + rank)
    x = workloads.bf16_bits(rng.standard_normal((T, K)).astype(np.float32))
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    topk[rng.random((T, k)) < 0.15] = -1      # dropped choices
    topk[topk == 3] = 1                        # expert 3 (rank 1's second) gets no tokens
    for t in range(T):                         # keep a token's choices distinct
        if topk[t, 0] == topk[t, 1] and topk[t, 0] >= 0:
            topk[t, 1] = -1
    wt = rng.random((T, k)).astype(np.float32)
    return x, topk, wt, wq, ws


def _rank_main(rank, world, port, out_path, capacity=None):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, TESTS)
    import ep_reference
    import moe_grouped_gemm_04_b200.ep as ep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ep._ops = ep_reference.CpuOps  # the CUDA kernels' CPU stand-ins
        x, topk, wt, wq, ws = _case(rank)
        G = E // world
        xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
        out = ep.expert_parallel_masked_moe(
            xt, torch.from_numpy(topk), torch.from_numpy(wt),
            torch.from_numpy(np.ascontiguousarray(wq[rank * G:(rank + 1) * G])),
            torch.from_numpy(np.ascontiguousarray(ws[rank * G:(rank + 1) * G])), E, M_max,
            capacity=capacity)
        np.save(out_path % rank, out.view(torch.int16).numpy().view(np.uint16))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,capacity", [(2, None), (2, 40), (2, 9), (4, None), (4, 9)])
def test_dispatch_gemm_combine_on_gloo_ranks(tmp_path, world, capacity):
    """Exact splits (capacity None) and the fixed-capacity exchange (9 rows:
    some destinations have more pairs, which are dropped, and the output is
    that of the routing without them), on two ranks of two experts and four
    ranks of one."""
    import torch.multiprocessing as mp

    import ep_reference
    out = str(tmp_path / "rank%d.npy")
    mp.start_processes(_rank_main, args=(world, _free_port(), out, capacity), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        x, topk, wt, wq, ws = _case(rank)
        got = np.load(out % rank)
        if capacity is not None:
            _, pos = ep_reference.layout_capacity_ref(topk, E, world, capacity)
            topk = np.where(pos < 0, -1, topk).astype(np.int32)
        want = ep_reference.expected_output(x, topk, wt, wq, ws)
        assert got.shape == want.shape
        assert np.array_equal(got, want), "rank %d: %d outputs differ" % (rank, int((got != want).sum()))


def test_layout_reference_orders_pairs_by_expert():
    """The stand-in layout (which the GPU kernel is checked against): pairs of
    expert e occupy [sum of counts before e, + counts[e]) in (t, j) order."""
    import ep_reference
    topk = np.array([[2, 0], [0, -1], [2, 1], [5, 0]], np.int32)  # 5 >= E: no expert
    counts, pos = ep_reference.layout_ref(topk, 4)
    assert counts.tolist() == [3, 1, 2, 0]
    assert pos.tolist() == [[4, 0], [1, -1], [5, 3], [-1, 2]]


def test_capacity_layout_reference():
    """Fixed capacity: destination d's pairs from row d * C in expert order;
    pairs at position C or beyond in their destination's rows are dropped."""
    import ep_reference
    topk = np.array([[2, 0], [0, -1], [2, 1], [3, 0]], np.int32)  # E = 4, W = 2: G = 2
    counts, pos = ep_reference.layout_capacity_ref(topk, 4, 2, 3)
    assert counts.tolist() == [3, 0, 2, 1]  # the pairs sent
    # destination 0 (experts 0, 1): pairs (0,1) (1,0) (3,1) of expert 0, then (2,1) of expert 1
    #   -> positions 0, 1, 2, 3; 3 >= C is dropped
    # destination 1 (experts 2, 3): (0,0) (2,0) of expert 2, (3,0) of expert 3 -> rows 3, 4, 5
    assert pos.tolist() == [[3, 0], [1, -1], [4, -1], [5, 2]]
