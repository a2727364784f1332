"""CPU stand-ins for the library calls of the expert-parallel layer
(moe_grouped_gemm_04_b200.ep), for tests only: each follows the contract its
kernel documents in include/fp8gemm.h, written plainly in numpy, and the GEMM
is the oracle's. The gloo tests swap them in for the CUDA kernels so that the
exchange protocol (counts, split sizes, orders) runs on CPU ranks; the GPU
tests compare the CUDA kernels with them.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads


def _np(t):
    return t.detach().cpu().numpy()


def layout_ref(topk: np.ndarray, E: int):
    """counts[E] and send_pos[P]: pairs ordered by expert, stably by p; -1 for
    pairs with no expert in [0, E)."""
    e = topk.reshape(-1).astype(np.int64)
    ok = (e >= 0) & (e < E)
    counts = np.bincount(e[ok], minlength=E).astype(np.int32)
    prefix = np.concatenate([[0], np.cumsum(counts)[:-1]])
    pos = np.full(e.size, -1, np.int32)
    rank = np.zeros(E, np.int64)
    for p in range(e.size):  # stable by p
        if ok[p]:
            pos[p] = prefix[e[p]] + rank[e[p]]
            rank[e[p]] += 1
    return counts, pos.reshape(topk.shape)


def layout_capacity_ref(topk: np.ndarray, E: int, W: int, C: int):
    """counts[E] of the pairs sent and send_pos with C rows per destination:
    d * C + the pair's position among destination d's pairs (by expert,
    stably by p), -1 for pairs with no expert and for pairs at position C or
    beyond (which the counts leave out)."""
    counts, pos = layout_ref(topk, E)
    G = E // W
    prefix = np.concatenate([[0], np.cumsum(counts)[:-1]])
    e = topk.reshape(-1).astype(np.int64)
    out = np.full(e.size, -1, np.int32)
    sent = np.zeros(E, np.int32)
    flat = pos.reshape(-1)
    for p in range(e.size):
        if flat[p] < 0:
            continue
        d = int(e[p]) // G
        i = int(flat[p]) - int(prefix[d * G])  # position within destination d's pairs
        if i < C:
            out[p] = d * C + i
            sent[e[p]] += 1
    return sent, out.reshape(topk.shape)


def unpack_capacity_ref(recv_q, recv_s, recv_counts, C, M_max):
    """unpack_ref for a W * C-row receive buffer, source s's rows from s * C."""
    W, G = recv_counts.shape
    K = recv_q.shape[1]
    rows = np.concatenate([recv_q[s * C:s * C + int(recv_counts[s].sum())] for s in range(W)])
    srows = np.concatenate([recv_s[s * C:s * C + int(recv_counts[s].sum())] for s in range(W)])
    A, sa, mm, slot_packed = unpack_ref(rows, srows, recv_counts, M_max)
    slot = np.full(W * C, -1, np.int32)
    r = 0
    for s in range(W):
        n = int(recv_counts[s].sum())
        slot[s * C:s * C + n] = slot_packed[r:r + n]
        r += n
    return A, sa, mm, slot


def unpack_ref(recv_q, recv_s, recv_counts, M_max):
    """Masked layout from the received rows (source by source, expert by
    expert): A [G][M_max][K], sa [G][M_max][KB] (logical), masked_m [G],
    recv_slot [R]."""
    W, G = recv_counts.shape
    R, K = recv_q.shape
    KB = K // 128
    A = np.zeros((G, M_max, K), np.uint8)
    sa = np.zeros((G, M_max, KB), np.float32)
    filled = np.zeros(G, np.int64)
    slot = np.full(R, -1, np.int32)
    r = 0
    for s in range(W):
        for g in range(G):
            for _ in range(int(recv_counts[s, g])):
                i = filled[g]
                filled[g] += 1
                if i < M_max:
                    A[g, i] = recv_q[r]
                    sa[g, i] = recv_s[r]
                    slot[r] = g * M_max + i
                r += 1
    return A, sa, np.minimum(filled, M_max).astype(np.int32), slot


def combine_ref(y_bits: np.ndarray, send_pos: np.ndarray, w: np.ndarray) -> np.ndarray:
    """bf16 bits of sum_j w[t][j] * y[send_pos[t][j]], j in order, in fp32,
    one bf16 rounding. Each step adds the product (exact in fp64: fp32 times
    bf16) to the fp32 accumulator in fp64 and rounds to fp32, which is the
    single-rounding multiply-add unless that fp64 sum itself rounds (terms of
    very different magnitudes)."""
    T, k = send_pos.shape
    N = y_bits.shape[1]
    yv = workloads.bf16_to_f32(y_bits).astype(np.float64)
    acc = np.zeros((T, N), np.float32)
    for j in range(k):
        pos = send_pos[:, j]
        ok = pos >= 0
        term = np.zeros((T, N), np.float64)
        term[ok] = w[ok, j].astype(np.float64)[:, None] * yv[pos[ok]]
        acc = (acc.astype(np.float64) + term).astype(np.float32)
    return workloads.bf16_bits(acc)


class CpuOps:
    """The layer's library calls on CPU torch tensors."""

    @staticmethod
    def quantize(x, q, s):
        bits = _np(x.view(torch.int16)).view(np.uint16)
        qq, sa = oracle.per_token_cast(bits)
        q.copy_(torch.from_numpy(qq))
        s.zero_()
        s[0, :, :sa.shape[0]] = torch.from_numpy(np.ascontiguousarray(sa.T))

    @staticmethod
    def layout(topk, E, counts, send_pos):
        c, p = layout_ref(_np(topk), E)
        counts.copy_(torch.from_numpy(c))
        send_pos.copy_(torch.from_numpy(p))

    @staticmethod
    def pack(q, s0, send_pos, send_q, send_s):
        qn, sn, pos = _np(q), _np(s0), _np(send_pos)
        T, k = pos.shape
        for t in range(T):
            for j in range(k):
                if pos[t, j] >= 0:
                    send_q[int(pos[t, j])] = torch.from_numpy(qn[t])
                    send_s[int(pos[t, j])] = torch.from_numpy(np.ascontiguousarray(sn[:, t]))

    @staticmethod
    def unpack(recv_q, recv_s, recv_counts, A, sfa, masked_m, recv_slot):
        M_max = A.shape[1]
        a, sa, mm, slot = unpack_ref(_np(recv_q), _np(recv_s), _np(recv_counts), M_max)
        A.copy_(torch.from_numpy(a))
        sfa.zero_()
        sfa[:, :, :M_max] = torch.from_numpy(np.ascontiguousarray(sa.transpose(0, 2, 1)))
        masked_m.copy_(torch.from_numpy(mm))
        recv_slot.copy_(torch.from_numpy(slot))

    @staticmethod
    def layout_capacity(topk, E, W, C, counts, send_pos):
        c, p = layout_capacity_ref(_np(topk), E, W, C)
        counts.copy_(torch.from_numpy(c))
        send_pos.copy_(torch.from_numpy(p))

    @staticmethod
    def unpack_capacity(recv_q, recv_s, recv_counts, C, A, sfa, masked_m, recv_slot):
        M_max = A.shape[1]
        a, sa, mm, slot = unpack_capacity_ref(_np(recv_q), _np(recv_s), _np(recv_counts), C, M_max)
        A.copy_(torch.from_numpy(a))
        sfa.zero_()
        sfa[:, :, :M_max] = torch.from_numpy(np.ascontiguousarray(sa.transpose(0, 2, 1)))
        masked_m.copy_(torch.from_numpy(mm))
        recv_slot.copy_(torch.from_numpy(slot))

    @staticmethod
    def gemm(A, sfa, w, sfb, D, masked_m, expected_m):
        M_max = A.shape[1]
        sa = np.ascontiguousarray(_np(sfa)[:, :, :M_max].transpose(0, 2, 1))
        mm = _np(masked_m)
        ref = oracle.grouped_masked(_np(A), sa, _np(w), _np(sfb), mm)
        bits = np.zeros(ref.shape, np.uint16)
        for g in range(ref.shape[0]):
            bits[g, :mm[g]] = oracle.f64_to_bf16(ref[g, :mm[g]])
        D.view(torch.int16).copy_(torch.from_numpy(bits.view(np.int16)))

    @staticmethod
    def gather(D, recv_slot, out):
        d = _np(D.view(torch.int16)).reshape(-1, D.shape[-1])
        slot = _np(recv_slot)
        o = np.zeros((slot.size, D.shape[-1]), np.int16)
        o[slot >= 0] = d[slot[slot >= 0]]
        out.view(torch.int16).copy_(torch.from_numpy(o))

    @staticmethod
    def combine(y, send_pos, w, out):
        bits = combine_ref(_np(y.view(torch.int16)).view(np.uint16), _np(send_pos), _np(w))
        out.view(torch.int16).copy_(torch.from_numpy(bits.view(np.int16)))


def expected_output(x_bits, topk, w, experts_q, experts_s):
    """What the layer must return for one rank's tokens, computed without any
    dispatch: for each choice, the oracle's GEMM row of the token against its
    expert, rounded to bf16, then the combine."""
    T, k = topk.shape
    qa, sa = oracle.per_token_cast(x_bits)
    N = experts_q.shape[1]
    rows = np.zeros((T * k, N), np.uint16)
    pos = np.full((T, k), -1, np.int32)
    for t in range(T):
        for j in range(k):
            e = int(topk[t, j])
            if e < 0:
                continue
            r = oracle.gemm_nt(qa[t:t + 1], sa[t:t + 1], experts_q[e], experts_s[e])
            rows[t * k + j] = oracle.f64_to_bf16(r)[0]
            pos[t, j] = t * k + j
    return combine_ref(rows, pos, w)
