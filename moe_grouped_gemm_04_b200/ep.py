"""Expert-parallel MoE layer around the masked grouped GEMM.

The masked layout ([G][M_max][K] per GPU with a per-expert valid-row count on
the device) is the one the grouped GEMM shares with the communication library
that moves tokens between the GPUs of an expert-parallel group ("DeepGEMM"
overview, section "约300行JIT核心", paragraph on MoE layouts); the tokens
travel over NVLink to the GPUs that hold their experts and the results travel
back (same page, section "swapAB与Mega MoE").

One call of `expert_parallel_masked_moe` on every rank of the group (or its
parts: `ep_dispatch` for steps 1-4, the masked GEMM, `ep_combine` for step 6):

  1. quantizes the rank's tokens per token per 128 channels (the library's
     quantizer: the rows travel as e4m3 codes with their scales, half the
     bytes of bf16);
  2. orders the (token, choice) pairs by expert (`ep_dispatch_layout`) and
     copies the rows into that order (`ep_dispatch_pack`), so that the pairs
     for rank d are one contiguous segment (rank d holds experts
     [d * G, (d + 1) * G));
  3. exchanges the per-expert counts, then the rows and their scales, with
     all-to-all collectives (NCCL over NVLink on GPUs);
  4. places the received rows into the masked layout and counts them per
     local expert on the device (`ep_dispatch_unpack_masked`);
  5. runs the masked grouped GEMM against the rank's expert weights;
  6. gathers the output rows back into receive order (`ep_combine_gather`),
     sends them back, and sums each token's choices weighted by the router
     (`ep_combine_reduce`: fp32, choices in order, one bf16 rounding).

Every step on the data runs in the library's CUDA kernels; this module only
allocates the buffers (torch device memory) and orders the kernels and the
collectives. The split sizes of the row exchange are read back to the host
(one synchronisation per call), as NCCL's all-to-all takes them on the host.
bf16 rows are exchanged as their bit patterns. No tensor-map or bulk
copy in this path reads another GPU's memory: the collectives copy the rows
into this GPU's memory before any kernel reads them.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import (FG_ERR_INVALID_ARG, FP8GemmError, empty_sfa, ep_combine_gather, ep_combine_reduce,
               ep_dispatch_layout, ep_dispatch_layout_capacity, ep_dispatch_pack,
               ep_dispatch_unpack_masked, ep_dispatch_unpack_masked_capacity,
               fp8_grouped_gemm_masked, per_token_cast_to_fp8)


class _LibraryOps:
    """The library calls the layer is made of (each a CUDA kernel)."""
    quantize = staticmethod(per_token_cast_to_fp8)
    layout = staticmethod(ep_dispatch_layout)
    pack = staticmethod(ep_dispatch_pack)
    unpack = staticmethod(ep_dispatch_unpack_masked)
    layout_capacity = staticmethod(ep_dispatch_layout_capacity)
    unpack_capacity = staticmethod(ep_dispatch_unpack_masked_capacity)
    gemm = staticmethod(fp8_grouped_gemm_masked)
    gather = staticmethod(ep_combine_gather)
    combine = staticmethod(ep_combine_reduce)


_ops = _LibraryOps


def _as_bits(t: torch.Tensor) -> torch.Tensor:
    """bf16 rows (an even number of columns) as int32 pairs of bit patterns,
    a type every collective backend moves."""
    return t.view(torch.int32) if t.dtype == torch.bfloat16 else t


class EpDispatch:
    """What ep_dispatch hands to the masked GEMM and to ep_combine: the masked
    layout of this rank's experts (A [G][M_max][K] e4m3, sfa in the MN-major
    layout, masked_m [G] on the device) and the bookkeeping of the exchange
    (each received row's slot in the layout, each own pair's position in the
    send order, and the split sizes of both all-to-alls)."""

    def __init__(self, A, sfa, masked_m, recv_slot, send_pos, send_sizes, recv_sizes, num_experts,
                 capacity=None, world=1):
        self.A, self.sfa, self.masked_m = A, sfa, masked_m
        self.recv_slot, self.send_pos = recv_slot, send_pos
        self.send_sizes, self.recv_sizes = send_sizes, recv_sizes
        self.num_experts = num_experts
        self.capacity, self.world = capacity, world

    @property
    def received(self) -> int:
        """Rows of the receive buffer (W * C with a fixed capacity)."""
        return self.world * self.capacity if self.capacity else sum(self.recv_sizes)

    @property
    def sent(self) -> int:
        return self.world * self.capacity if self.capacity else sum(self.send_sizes)


def ep_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, num_experts: int, M_max: int,
                group=None, capacity: Optional[int] = None) -> EpDispatch:
    """Steps 1-4 of the layer: quantize this rank's tokens, order the pairs by
    expert, exchange counts, rows and scales, and place the received rows into
    the masked layout of this rank's G = num_experts / world_size experts.

    capacity=None exchanges exactly the rows each pair of ranks has, which
    needs the split sizes on the host (one synchronisation). capacity=C
    exchanges C rows to and from every rank (pairs beyond C for one rank are
    dropped, FG_DEVICE_EP_OVERFLOW): equal splits known in advance, so
    nothing is read back and the layer never waits for the host."""
    W = dist.get_world_size(group)
    if num_experts % W != 0:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "num_experts %d is not a multiple of the group size %d"
                           % (num_experts, W))
    G = num_experts // W
    T, K = x.shape
    k = topk_idx.shape[1]
    dev = x.device
    KB = K // 128

    q = torch.empty((T, K), dtype=torch.uint8, device=dev)
    s = empty_sfa(1, T, K, dev)
    _ops.quantize(x, q, s)
    counts = torch.empty(num_experts, dtype=torch.int32, device=dev)
    send_pos = torch.empty((T, k), dtype=torch.int32, device=dev)
    if capacity is None:
        _ops.layout(topk_idx, num_experts, counts, send_pos)
    else:
        _ops.layout_capacity(topk_idx, num_experts, W, int(capacity), counts, send_pos)

    if capacity is not None:
        return _dispatch_capacity(x, q, s, topk_idx, counts, send_pos, num_experts, M_max, int(capacity),
                                  W, G, group)
    recv_counts = torch.empty((W, G), dtype=torch.int32, device=dev)
    dist.all_to_all_single(recv_counts.view(-1), counts, group=group)
    send_sizes = [int(v) for v in counts.view(W, G).sum(dim=1).tolist()]
    recv_sizes = [int(v) for v in recv_counts.sum(dim=1).tolist()]
    P, R = sum(send_sizes), sum(recv_sizes)
    send_q = torch.empty((P, K), dtype=torch.uint8, device=dev)
    send_s = torch.empty((P, KB), dtype=torch.float32, device=dev)
    _ops.pack(q, s[0], send_pos, send_q, send_s)
    recv_q = torch.empty((R, K), dtype=torch.uint8, device=dev)
    recv_s = torch.empty((R, KB), dtype=torch.float32, device=dev)
    dist.all_to_all_single(recv_q, send_q, recv_sizes, send_sizes, group=group)
    dist.all_to_all_single(recv_s, send_s, recv_sizes, send_sizes, group=group)

    A = torch.empty((G, M_max, K), dtype=torch.uint8, device=dev)
    sfa = empty_sfa(G, M_max, K, dev)
    masked_m = torch.empty(G, dtype=torch.int32, device=dev)
    recv_slot = torch.empty(R, dtype=torch.int32, device=dev)
    _ops.unpack(recv_q, recv_s, recv_counts, A, sfa, masked_m, recv_slot)
    return EpDispatch(A, sfa, masked_m, recv_slot, send_pos, send_sizes, recv_sizes, num_experts)


def _dispatch_capacity(x, q, s, topk_idx, counts, send_pos, num_experts, M_max, C, W, G, group):
    """ep_dispatch's exchange with C rows per rank each way (no host read)."""
    dev = x.device
    K = x.shape[1]
    KB = K // 128
    recv_counts = torch.empty((W, G), dtype=torch.int32, device=dev)
    dist.all_to_all_single(recv_counts.view(-1), counts, group=group)
    send_q = torch.empty((W * C, K), dtype=torch.uint8, device=dev)
    send_s = torch.empty((W * C, KB), dtype=torch.float32, device=dev)
    _ops.pack(q, s[0], send_pos, send_q, send_s)
    recv_q = torch.empty_like(send_q)
    recv_s = torch.empty_like(send_s)
    dist.all_to_all_single(recv_q, send_q, group=group)
    dist.all_to_all_single(recv_s, send_s, group=group)
    A = torch.empty((G, M_max, K), dtype=torch.uint8, device=dev)
    sfa = empty_sfa(G, M_max, K, dev)
    masked_m = torch.empty(G, dtype=torch.int32, device=dev)
    recv_slot = torch.empty(W * C, dtype=torch.int32, device=dev)
    _ops.unpack_capacity(recv_q, recv_s, recv_counts, C, A, sfa, masked_m, recv_slot)
    return EpDispatch(A, sfa, masked_m, recv_slot, send_pos, None, None, num_experts, capacity=C, world=W)


def ep_combine(D: torch.Tensor, h: EpDispatch, topk_w: torch.Tensor, group=None) -> torch.Tensor:
    """Step 6: gather the GEMM's output rows into receive order, send them back
    to their source ranks, and sum each token's choices weighted by the router
    (fp32, choices in order, one bf16 rounding). D: bf16 [G][M_max][N]."""
    dev = D.device
    N = D.shape[2]
    T = h.send_pos.shape[0]
    y_recv = torch.empty((h.received, N), dtype=torch.bfloat16, device=dev)
    _ops.gather(D, h.recv_slot, y_recv)
    y_send = torch.empty((h.sent, N), dtype=torch.bfloat16, device=dev)
    if h.capacity:
        dist.all_to_all_single(_as_bits(y_send), _as_bits(y_recv), group=group)
    else:
        dist.all_to_all_single(_as_bits(y_send), _as_bits(y_recv), h.send_sizes, h.recv_sizes, group=group)
    out = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    _ops.combine(y_send, h.send_pos, topk_w, out)
    return out


def expert_parallel_masked_moe(x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
                               w_local: torch.Tensor, sfb_local: torch.Tensor, num_experts: int,
                               M_max: int, group=None, expected_m: Optional[int] = None,
                               capacity: Optional[int] = None) -> torch.Tensor:
    """Routed expert GEMM over an expert-parallel group: ep_dispatch, the masked
    grouped GEMM with this rank's experts, ep_combine.

    x: bf16 [T][K] (this rank's tokens); topk_idx: int32 [T][k] global expert
    ids (negative = no expert); topk_w: fp32 [T][k] router weights; w_local:
    e4m3 [G][N][K] and sfb_local fp32 [G][ceil(N/128)][K/128], the weights of
    this rank's G = num_experts / world_size experts, quantized per 128 x 128
    block; M_max: rows per local expert in the masked layout (more are
    dropped, FG_DEVICE_EP_OVERFLOW); capacity: see ep_dispatch. Returns bf16
    [T][N]: out[t] = sum_j topk_w[t][j] * bf16((x_t quantized) W_{topk_idx[t][j]}^T).
    """
    W = dist.get_world_size(group)
    G = num_experts // W if num_experts % W == 0 else -1
    if G > 0 and w_local.shape[0] != G:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "w_local holds %d experts, this rank owns %d"
                           % (w_local.shape[0], G))
    h = ep_dispatch(x, topk_idx, num_experts, M_max, group, capacity)
    G = h.A.shape[0]
    N = w_local.shape[1]
    D = torch.empty((G, M_max, N), dtype=torch.bfloat16, device=x.device)
    if expected_m is None:
        # rows per local expert: what was received, or (fixed capacity, which
        # keeps the counts on the device) what uniform routing brings: every
        # rank's T * k pairs spread over W * G experts
        rows = h.received if h.capacity is None else topk_idx.numel()
        expected_m = max(1, min(M_max, -(-rows // G)))
    _ops.gemm(h.A, h.sfa, w_local, sfb_local, D, h.masked_m, expected_m)
    return ep_combine(D, h, topk_w, group)
