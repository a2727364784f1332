"""Python binding of libfp8gemm.so, the B200 FP8 block-scaled GEMM library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/fp8gemm.h. Tensors are torch
tensors used as device memory; the calls run on the current torch CUDA stream
(or the stream passed in) and never synchronise the host. There is no CPU
fallback: if the library is missing or the device is not sm_100a, every call
raises.

The functions carry the C names:
  per_token_cast_to_fp8, per_block_cast_to_fp8, per_block_dequant_to_bf16,
  fp8_gemm_nt, fp8_grouped_gemm_contiguous, fp8_grouped_gemm_masked,
  per_token_cast_to_fp8_ue8m0, per_block_cast_to_fp8_ue8m0, and the GEMMs for
  power-of-two scales fp8_gemm_nt_ue8m0, fp8_grouped_gemm_contiguous_ue8m0,
  fp8_grouped_gemm_masked_ue8m0 (set_ue8m0_tile tunes them), and the expert FFN
  fp8_moe_ffn_contiguous_ue8m0, fp8_moe_ffn_masked_ue8m0, and the K-grouped
  (expert weight-gradient) GEMM fp8_k_grouped_gemm_nt_ue8m0
plus allocation helpers that return tensors in the layouts the kernels use.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8gemm.so")

FG_OK = 0
FG_ERR_INVALID_ARG = 1
FG_ERR_UNSUPPORTED = 2
FG_ERR_CUDA = 3
FG_ERR_DEVICE = 4

EXPORTED = (
    "fg_sfa_stride", "per_token_cast_to_fp8", "per_block_cast_to_fp8",
    "per_token_cast_to_fp8_ue8m0", "per_block_cast_to_fp8_ue8m0", "fp8_gemm_nt",
    "fp8_grouped_gemm_contiguous", "fp8_grouped_gemm_masked", "per_block_dequant_to_bf16",
    "fp8_gemm_nt_ue8m0", "fp8_grouped_gemm_contiguous_ue8m0", "fp8_grouped_gemm_masked_ue8m0",
    "fg_set_ue8m0_tile", "fg_set_ffn_mode", "fg_moe_ffn_workspace_bytes", "fp8_moe_ffn_contiguous_ue8m0",
    "fp8_moe_ffn_masked_ue8m0", "fp8_moe_ffn_masked_ue8m0_noalloc",
    "ep_dispatch_layout", "ep_dispatch_pack", "ep_dispatch_unpack_masked", "ep_combine_gather",
    "ep_combine_reduce", "ep_dispatch_layout_capacity", "ep_dispatch_unpack_masked_capacity",
    "fp8_k_grouped_gemm_nt_ue8m0",
    "fg_get_device_status", "fg_selftest_wait_timeout", "fg_status_string", "fg_last_error",
    "fg_fp8_mma_peak_ctas", "fg_fp8_mma_peak",
)


class FP8GemmError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (_status_name(status), message))
        self.status = status


_lib: Optional[ctypes.CDLL] = None


def load_library() -> ctypes.CDLL:
    """Load libfp8gemm.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise FP8GemmError(FG_ERR_UNSUPPORTED,
                           "%s is missing; build it with moe_grouped_gemm_04_b200/build.py" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.fg_sfa_stride.argtypes = [I]
    lib.fg_sfa_stride.restype = I
    lib.per_token_cast_to_fp8.argtypes = [P, P, P, I, I, I, P]
    lib.per_block_cast_to_fp8.argtypes = [P, P, P, I, I, I, P]
    lib.per_token_cast_to_fp8_ue8m0.argtypes = [P, P, P, I, I, I, P]
    lib.per_block_cast_to_fp8_ue8m0.argtypes = [P, P, P, I, I, I, P]
    lib.per_block_dequant_to_bf16.argtypes = [P, P, P, I, I, I, P]
    lib.fp8_gemm_nt.argtypes = [P, P, P, P, P, I, I, I, P]
    lib.fp8_grouped_gemm_contiguous.argtypes = [P, P, P, P, P, P, I, I, I, I, P]
    lib.fp8_grouped_gemm_masked.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P]
    lib.fp8_gemm_nt_ue8m0.argtypes = [P, P, P, P, P, I, I, I, P]
    lib.fp8_grouped_gemm_contiguous_ue8m0.argtypes = [P, P, P, P, P, P, I, I, I, I, P]
    lib.fp8_grouped_gemm_masked_ue8m0.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P]
    lib.fg_set_ue8m0_tile.argtypes = [I, I]
    Z = ctypes.c_size_t
    lib.fg_set_ffn_mode.argtypes = [I]
    lib.fg_moe_ffn_workspace_bytes.argtypes = [I, I, I]
    lib.fg_moe_ffn_workspace_bytes.restype = Z
    lib.fp8_moe_ffn_contiguous_ue8m0.argtypes = [P] * 11 + [I, I, I, I, P, Z, P]
    lib.fp8_moe_ffn_masked_ue8m0.argtypes = [P] * 11 + [I, I, I, I, I, P, Z, P]
    lib.fp8_moe_ffn_masked_ue8m0_noalloc.argtypes = [P] * 11 + [I, I, I, I, I, P]
    lib.ep_dispatch_layout.argtypes = [P, I, I, I, P, P, P]
    lib.ep_dispatch_pack.argtypes = [P, P, P, I, I, I, P, P, P]
    lib.ep_dispatch_unpack_masked.argtypes = [P, P, P, I, I, I, I, I, P, P, P, P, P]
    lib.ep_combine_gather.argtypes = [P, P, I, I, P, P]
    lib.ep_dispatch_layout_capacity.argtypes = [P, I, I, I, I, I, P, P, P]
    lib.ep_dispatch_unpack_masked_capacity.argtypes = [P, P, P, I, I, I, I, I, P, P, P, P, P]
    lib.ep_combine_reduce.argtypes = [P, P, P, I, I, I, P, P]
    lib.fp8_k_grouped_gemm_nt_ue8m0.argtypes = [P, P, P, P, P, P, I, I, I, I, P]
    lib.fg_get_device_status.argtypes = [P, ctypes.POINTER(I)]
    lib.fg_selftest_wait_timeout.argtypes = [I, P]
    lib.fg_status_string.argtypes = [I]
    lib.fg_status_string.restype = ctypes.c_char_p
    lib.fg_last_error.argtypes = []
    lib.fg_last_error.restype = ctypes.c_char_p
    lib.fg_fp8_mma_peak_ctas.argtypes = []
    lib.fg_fp8_mma_peak_ctas.restype = I
    lib.fg_fp8_mma_peak.argtypes = [I, P, P]
    for f in ("per_token_cast_to_fp8", "per_block_cast_to_fp8", "per_token_cast_to_fp8_ue8m0",
              "per_block_cast_to_fp8_ue8m0", "per_block_dequant_to_bf16",
              "fp8_gemm_nt",
              "fp8_grouped_gemm_contiguous", "fp8_grouped_gemm_masked",
              "fp8_gemm_nt_ue8m0", "fp8_grouped_gemm_contiguous_ue8m0",
              "fp8_grouped_gemm_masked_ue8m0", "fg_set_ue8m0_tile", "fg_set_ffn_mode",
              "fp8_moe_ffn_contiguous_ue8m0", "fp8_moe_ffn_masked_ue8m0",
              "fp8_moe_ffn_masked_ue8m0_noalloc",
              "ep_dispatch_layout", "ep_dispatch_pack", "ep_dispatch_unpack_masked",
              "ep_combine_gather", "ep_combine_reduce", "ep_dispatch_layout_capacity",
              "ep_dispatch_unpack_masked_capacity",
              "fp8_k_grouped_gemm_nt_ue8m0",
              "fg_get_device_status", "fg_selftest_wait_timeout", "fg_fp8_mma_peak"):
        getattr(lib, f).restype = I
    _lib = lib
    return lib


def _status_name(s: int) -> str:
    return {0: "FG_OK", 1: "FG_ERR_INVALID_ARG", 2: "FG_ERR_UNSUPPORTED", 3: "FG_ERR_CUDA",
            4: "FG_ERR_DEVICE"}.get(s, "FG_ERR_%d" % s)


def _check(status: int) -> None:
    if status != FG_OK:
        msg = load_library().fg_last_error()
        raise FP8GemmError(status, msg.decode() if msg else "")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise FP8GemmError(FG_ERR_INVALID_ARG, "tensor must be contiguous")
    return t.data_ptr()  # c_void_p argtypes take the integer address


# The raw handle of torch's current stream, read without building a Stream
# object (which costs several microseconds per call).
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream):
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None:
        return _raw_stream(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


# ---------------------------------------------------------------- layouts

def sfa_stride(M: int) -> int:
    """Row stride (floats) of the MN-major activation-scale layout."""
    return (M + 3) // 4 * 4


def empty_sfa(G: int, M: int, K: int, device) -> torch.Tensor:
    """Activation scales [G][K/128][stride(M)] (padding entries unused)."""
    return torch.empty((G, K // 128, sfa_stride(M)), dtype=torch.float32, device=device)


def empty_sfb(G: int, N: int, K: int, device) -> torch.Tensor:
    """Weight scales [G][ceil(N/128)][K/128]."""
    return torch.empty((G, -(-N // 128), K // 128), dtype=torch.float32, device=device)


# ---------------------------------------------------------------- entry points

def _token_cast(fn, x, q, sfa, stream):
    G, M, K = (1, *x.shape) if x.dim() == 2 else tuple(x.shape)
    if x.dtype != torch.bfloat16 or q.dtype != torch.uint8 or sfa.dtype != torch.float32:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "dtypes: x bf16, q uint8, sfa float32")
    if q.numel() != x.numel() or sfa.numel() < G * (K // 128) * sfa_stride(M):
        raise FP8GemmError(FG_ERR_INVALID_ARG, "output sizes do not match x")
    _check(fn(_ptr(x), _ptr(q), _ptr(sfa), G, M, K, _stream(stream)))


def _block_cast(fn, x, q, sfb, stream):
    G, N, K = (1, *x.shape) if x.dim() == 2 else tuple(x.shape)
    if x.dtype != torch.bfloat16 or q.dtype != torch.uint8 or sfb.dtype != torch.float32:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "dtypes: x bf16, q uint8, sfb float32")
    if q.numel() != x.numel() or sfb.numel() < G * (-(-N // 128)) * (K // 128):
        raise FP8GemmError(FG_ERR_INVALID_ARG, "output sizes do not match x")
    _check(fn(_ptr(x), _ptr(q), _ptr(sfb), G, N, K, _stream(stream)))


def per_token_cast_to_fp8(x: torch.Tensor, q: torch.Tensor, sfa: torch.Tensor,
                          stream=None) -> None:
    """x: bf16 [M][K] or [G][M][K] -> q (uint8, same shape), sfa [G][K/128][stride(M)]."""
    _token_cast(load_library().per_token_cast_to_fp8, x, q, sfa, stream)


def per_token_cast_to_fp8_ue8m0(x: torch.Tensor, q: torch.Tensor, sfa: torch.Tensor,
                                stream=None) -> None:
    """As per_token_cast_to_fp8 with power-of-two scales."""
    _token_cast(load_library().per_token_cast_to_fp8_ue8m0, x, q, sfa, stream)


def per_block_cast_to_fp8(x: torch.Tensor, q: torch.Tensor, sfb: torch.Tensor,
                          stream=None) -> None:
    """x: bf16 [N][K] or [G][N][K] -> q (uint8, same shape), sfb [G][ceil(N/128)][K/128]."""
    _block_cast(load_library().per_block_cast_to_fp8, x, q, sfb, stream)


def per_block_cast_to_fp8_ue8m0(x: torch.Tensor, q: torch.Tensor, sfb: torch.Tensor,
                                stream=None) -> None:
    """As per_block_cast_to_fp8 with power-of-two scales."""
    _block_cast(load_library().per_block_cast_to_fp8_ue8m0, x, q, sfb, stream)


def per_block_dequant_to_bf16(q: torch.Tensor, sfb: torch.Tensor, x: torch.Tensor,
                              stream=None) -> None:
    """q uint8 [N][K] or [G][N][K], sfb [G][ceil(N/128)][K/128] -> x bf16 (shape of q)."""
    G, N, K = (1, *q.shape) if q.dim() == 2 else tuple(q.shape)
    if q.dtype != torch.uint8 or x.dtype != torch.bfloat16 or sfb.dtype != torch.float32:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "dtypes: q uint8, sfb float32, x bf16")
    if x.numel() != q.numel() or sfb.numel() < G * (-(-N // 128)) * (K // 128):
        raise FP8GemmError(FG_ERR_INVALID_ARG, "sizes of sfb or x do not match q")
    _check(load_library().per_block_dequant_to_bf16(_ptr(q), _ptr(sfb), _ptr(x), G, N, K,
                                                    _stream(stream)))


def _gemm_nt(fn, A, sfa, B, sfb, D, stream):
    M, K = A.shape
    N = B.shape[0]
    if D.dtype != torch.bfloat16 or tuple(D.shape) != (M, N):
        raise FP8GemmError(FG_ERR_INVALID_ARG, "D must be bf16 [M][N]")
    _check(fn(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(D), M, N, K, _stream(stream)))


def _gemm_contiguous(fn, A, sfa, B, sfb, D, m_indices, stream):
    M_total, K = A.shape
    G, N, _ = B.shape
    if m_indices.dtype != torch.int32 or m_indices.numel() != M_total:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "m_indices must be int32 [M_total]")
    _check(fn(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(D), _ptr(m_indices), M_total, N, K, G,
              _stream(stream)))


def _gemm_masked(fn, A, sfa, B, sfb, D, masked_m, expected_m, stream):
    G, M_max, K = A.shape
    N = B.shape[1]
    if masked_m.dtype != torch.int32 or masked_m.numel() != G:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "masked_m must be int32 [G]")
    _check(fn(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(D), _ptr(masked_m), G, M_max, N, K,
              int(expected_m), _stream(stream)))


def fp8_gemm_nt(A: torch.Tensor, sfa: torch.Tensor, B: torch.Tensor, sfb: torch.Tensor,
                D: torch.Tensor, stream=None) -> None:
    """D[M][N] (bf16) = (A * sa)(B * sb)^T; A uint8 [M][K], B uint8 [N][K]."""
    _gemm_nt(load_library().fp8_gemm_nt, A, sfa, B, sfb, D, stream)


def fp8_grouped_gemm_contiguous(A: torch.Tensor, sfa: torch.Tensor, B: torch.Tensor,
                                sfb: torch.Tensor, D: torch.Tensor, m_indices: torch.Tensor,
                                stream=None) -> None:
    """A uint8 [M_total][K], B uint8 [G][N][K], m_indices int32 [M_total], D bf16 [M_total][N]."""
    _gemm_contiguous(load_library().fp8_grouped_gemm_contiguous, A, sfa, B, sfb, D, m_indices,
                     stream)


def fp8_grouped_gemm_masked(A: torch.Tensor, sfa: torch.Tensor, B: torch.Tensor,
                            sfb: torch.Tensor, D: torch.Tensor, masked_m: torch.Tensor,
                            expected_m: int, stream=None) -> None:
    """A uint8 [G][M_max][K], B uint8 [G][N][K], masked_m int32 [G], D bf16 [G][M_max][N]."""
    _gemm_masked(load_library().fp8_grouped_gemm_masked, A, sfa, B, sfb, D, masked_m, expected_m,
                 stream)


def fp8_gemm_nt_ue8m0(A: torch.Tensor, sfa: torch.Tensor, B: torch.Tensor, sfb: torch.Tensor,
                      D: torch.Tensor, stream=None) -> None:
    """fp8_gemm_nt with power-of-two scales (block-scaled tensor-core MMAs)."""
    _gemm_nt(load_library().fp8_gemm_nt_ue8m0, A, sfa, B, sfb, D, stream)


def fp8_grouped_gemm_contiguous_ue8m0(A: torch.Tensor, sfa: torch.Tensor, B: torch.Tensor,
                                      sfb: torch.Tensor, D: torch.Tensor,
                                      m_indices: torch.Tensor, stream=None) -> None:
    """fp8_grouped_gemm_contiguous with power-of-two scales."""
    _gemm_contiguous(load_library().fp8_grouped_gemm_contiguous_ue8m0, A, sfa, B, sfb, D,
                     m_indices, stream)


def fp8_grouped_gemm_masked_ue8m0(A: torch.Tensor, sfa: torch.Tensor, B: torch.Tensor,
                                  sfb: torch.Tensor, D: torch.Tensor, masked_m: torch.Tensor,
                                  expected_m: int, stream=None) -> None:
    """fp8_grouped_gemm_masked with power-of-two scales."""
    _gemm_masked(load_library().fp8_grouped_gemm_masked_ue8m0, A, sfa, B, sfb, D, masked_m,
                 expected_m, stream)


FG_LAYOUT_CONTIGUOUS = 0
FG_LAYOUT_MASKED = 1


def set_ffn_mode(mode: int) -> None:
    """Expert FFN form: 0 automatic, 1 one launch, 2 two launches."""
    _check(load_library().fg_set_ffn_mode(int(mode)))


def moe_ffn_workspace_bytes(layout: int, M: int, G: int) -> int:
    """Bytes of the workspace the expert FFN needs (M = M_total or M_max)."""
    return int(load_library().fg_moe_ffn_workspace_bytes(layout, M, G))


def empty_ffn_workspace(layout: int, M: int, G: int, device="cuda"):
    """A workspace for the expert FFN (its contents need no initialisation)."""
    n = max(moe_ffn_workspace_bytes(layout, M, G), 256)
    return torch.empty(n, dtype=torch.uint8, device=device)


def fp8_moe_ffn_contiguous_ue8m0(X, sfx, W1, sfw1, W2, sfw2, Hq, sfh, Y, m_indices, GU=None,
                                 ws=None, stream=None) -> None:
    """Expert FFN (contiguous layout): X uint8 [M_total][H], W1 uint8 [G][2I][H],
    W2 uint8 [G][H][I] -> Hq uint8 [M_total][I], sfh [I/128][stride], Y bf16
    [M_total][H] (and GU bf16 [M_total][2I] if given). ws: the workspace (a
    torch tensor; one is allocated when it is not given)."""
    M_total, H = X.shape
    G, I2, _ = W1.shape
    if m_indices.dtype != torch.int32 or m_indices.numel() != M_total:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "m_indices must be int32 [M_total]")
    if ws is None:
        ws = empty_ffn_workspace(FG_LAYOUT_CONTIGUOUS, M_total, G, X.device)
    _check(load_library().fp8_moe_ffn_contiguous_ue8m0(
        _ptr(X), _ptr(sfx), _ptr(W1), _ptr(sfw1), _ptr(W2), _ptr(sfw2), _ptr(Hq), _ptr(sfh),
        _ptr(GU), _ptr(Y), _ptr(m_indices), M_total, H, I2 // 2, G, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def fp8_moe_ffn_masked_ue8m0(X, sfx, W1, sfw1, W2, sfw2, Hq, sfh, Y, masked_m, expected_m,
                             GU=None, ws=None, stream=None) -> None:
    """Expert FFN (masked layout): X uint8 [G][M_max][H] -> Hq [G][M_max][I],
    sfh [G][I/128][stride], Y bf16 [G][M_max][H] (and GU [G][M_max][2I]).
    ws as for the contiguous form."""
    G, M_max, H = X.shape
    I2 = W1.shape[1]
    if masked_m.dtype != torch.int32 or masked_m.numel() != G:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "masked_m must be int32 [G]")
    if ws is None:
        ws = empty_ffn_workspace(FG_LAYOUT_MASKED, M_max, G, X.device)
    _check(load_library().fp8_moe_ffn_masked_ue8m0(
        _ptr(X), _ptr(sfx), _ptr(W1), _ptr(sfw1), _ptr(W2), _ptr(sfw2), _ptr(Hq), _ptr(sfh),
        _ptr(GU), _ptr(Y), _ptr(masked_m), G, M_max, H, I2 // 2, int(expected_m), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def fp8_moe_ffn_masked_ue8m0_noalloc(X, sfx, W1, sfw1, W2, sfw2, Hq, sfh, Y, masked_m, expected_m,
                                     GU=None, stream=None) -> None:
    """The masked expert FFN for callers that may not allocate device memory:
    no workspace (the library's own fixed scratch holds the ready counters;
    G * ceil(M_max / 128) <= 4096; calls that overlap on the GPU race on it)."""
    G, M_max, H = X.shape
    I2 = W1.shape[1]
    if masked_m.dtype != torch.int32 or masked_m.numel() != G:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "masked_m must be int32 [G]")
    _check(load_library().fp8_moe_ffn_masked_ue8m0_noalloc(
        _ptr(X), _ptr(sfx), _ptr(W1), _ptr(sfw1), _ptr(W2), _ptr(sfw2), _ptr(Hq), _ptr(sfh),
        _ptr(GU), _ptr(Y), _ptr(masked_m), G, M_max, H, I2 // 2, int(expected_m), _stream(stream)))


def ep_dispatch_layout(topk_idx, E, counts, send_pos, stream=None) -> None:
    """topk_idx int32 [T][k] -> counts int32 [E], send_pos int32 [T][k]."""
    T, k = topk_idx.shape
    _check(load_library().ep_dispatch_layout(_ptr(topk_idx), T, k, int(E), _ptr(counts),
                                             _ptr(send_pos), _stream(stream)))


def ep_dispatch_pack(q, sfa, send_pos, send_q, send_s, stream=None) -> None:
    """q uint8 [T][K], sfa MN-major [K/128][stride(T)], send_pos [T][k] ->
    send_q uint8 [P][K], send_s fp32 [P][K/128]."""
    T, K = q.shape
    k = send_pos.shape[1]
    _check(load_library().ep_dispatch_pack(_ptr(q), _ptr(sfa), _ptr(send_pos), T, k, K, _ptr(send_q),
                                           _ptr(send_s), _stream(stream)))


def ep_dispatch_unpack_masked(recv_q, recv_s, recv_counts, A, sfa, masked_m, recv_slot,
                              stream=None) -> None:
    """Received rows (source by source, local expert by local expert;
    recv_counts int32 [W][G]) -> masked layout A [G][M_max][K], sfa
    [G][K/128][stride(M_max)], masked_m [G], recv_slot [R]."""
    W, G = recv_counts.shape
    R = recv_q.shape[0]
    _, M_max, K = A.shape
    _check(load_library().ep_dispatch_unpack_masked(
        _ptr(recv_q), _ptr(recv_s), _ptr(recv_counts), W, G, R, M_max, K, _ptr(A), _ptr(sfa),
        _ptr(masked_m), _ptr(recv_slot), _stream(stream)))


def ep_dispatch_layout_capacity(topk_idx, E, W, C, counts, send_pos, stream=None) -> None:
    """As ep_dispatch_layout with C send rows per destination GPU (W GPUs of
    E / W experts): send_pos = d * C + position within destination d's rows."""
    T, k = topk_idx.shape
    _check(load_library().ep_dispatch_layout_capacity(_ptr(topk_idx), T, k, int(E), int(W), int(C),
                                                      _ptr(counts), _ptr(send_pos), _stream(stream)))


def ep_dispatch_unpack_masked_capacity(recv_q, recv_s, recv_counts, C, A, sfa, masked_m, recv_slot,
                                       stream=None) -> None:
    """As ep_dispatch_unpack_masked for W * C received rows, source s's from
    row s * C; recv_slot [W * C]."""
    W, G = recv_counts.shape
    _, M_max, K = A.shape
    _check(load_library().ep_dispatch_unpack_masked_capacity(
        _ptr(recv_q), _ptr(recv_s), _ptr(recv_counts), W, G, int(C), M_max, K, _ptr(A), _ptr(sfa),
        _ptr(masked_m), _ptr(recv_slot), _stream(stream)))


def ep_combine_gather(D, recv_slot, out, stream=None) -> None:
    """out [R][N] = rows recv_slot of D (bf16 [G][M_max][N]; zero where -1)."""
    R, N = out.shape
    _check(load_library().ep_combine_gather(_ptr(D), _ptr(recv_slot), R, N, _ptr(out),
                                            _stream(stream)))


def ep_combine_reduce(y, send_pos, topk_w, out, stream=None) -> None:
    """out [T][N] = bf16(sum_j topk_w[t][j] * y[send_pos[t][j]]) (fp32, j in order)."""
    T, k = send_pos.shape
    N = out.shape[1]
    _check(load_library().ep_combine_reduce(_ptr(y), _ptr(send_pos), _ptr(topk_w), T, k, N, _ptr(out),
                                            _stream(stream)))


def fp8_k_grouped_gemm_nt_ue8m0(A, sfa, B, sfb, D, ks, stream=None) -> None:
    """K-grouped GEMM (expert weight gradients): A uint8 [M][T], sfa [T/128][stride(M)],
    B uint8 [N][T], sfb [T/128][stride(N)], ks int32 [G] token counts (device),
    D float32 [G][M][N]."""
    M, T = A.shape
    N = B.shape[0]
    G = ks.numel()
    if ks.dtype != torch.int32:
        raise FP8GemmError(FG_ERR_INVALID_ARG, "ks must be int32 [G]")
    if D.dtype != torch.float32 or tuple(D.shape) != (G, M, N):
        raise FP8GemmError(FG_ERR_INVALID_ARG, "D must be float32 [G][M][N]")
    _check(load_library().fp8_k_grouped_gemm_nt_ue8m0(
        _ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(D), _ptr(ks), G, M, N, T, _stream(stream)))


def set_ue8m0_tile(width: int, pair: bool = False) -> None:
    """0 = automatic (default); else force weight tiles of `width` rows (128,
    224 or 256 single-CTA, or 224 or 192 as a CTA pair)."""
    _check(load_library().fg_set_ue8m0_tile(int(width), 1 if pair else 0))


def get_device_status(stream=None) -> int:
    """Synchronise the stream and read+clear the device status word (0 = clear)."""
    code = ctypes.c_int(0)
    st = load_library().fg_get_device_status(_stream(stream), ctypes.byref(code))
    if st not in (FG_OK, FG_ERR_DEVICE):
        _check(st)
    return int(code.value)


def selftest_wait_timeout(timeout_us: int, stream=None) -> None:
    _check(load_library().fg_selftest_wait_timeout(int(timeout_us), _stream(stream)))


def fp8_mma_peak_ctas() -> int:
    """CTAs of one fp8_mma_peak launch (the SM count of the current device)."""
    n = load_library().fg_fp8_mma_peak_ctas()
    if n <= 0:
        raise FP8GemmError(FG_ERR_UNSUPPORTED, load_library().fg_last_error().decode())
    return int(n)


def fp8_mma_peak(iters: int, out, stream=None) -> None:
    """The tensor-core rate kernel: `iters` K blocks of FP8 MMAs (M = 128,
    N = 256, K = 128 each) per CTA; out: fp32 [fp8_mma_peak_ctas()][128][256]
    on the device receives each CTA's exact integer accumulator."""
    ctas = fp8_mma_peak_ctas()
    if tuple(out.shape) != (ctas, 128, 256) or out.dtype != torch.float32 or not out.is_contiguous():
        raise FP8GemmError(FG_ERR_INVALID_ARG, "out must be contiguous fp32 [%d][128][256]" % ctas)
    _check(load_library().fg_fp8_mma_peak(int(iters), _ptr(out), _stream(stream)))

