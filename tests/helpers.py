"""Shared helpers for the GPU parity tests: layout conversion between the
oracle's logical scale layout and the library's MN-major layout, upload, and
the acceptance check."""
from __future__ import annotations

import numpy as np

# Acceptance bar for the GEMM outputs (bf16 D against the fp64 oracle):
#   per element  |gpu - ref| <= 2^-7 |ref| + 1e-3 rms(ref)
#   global       1 - 2 sum(xy) / sum(x^2 + y^2) < 1e-3
REL_TOL = 2.0 ** -7
RMS_TOL = 1e-3
GLOBAL_TOL = 1e-3


def sfa_stride(M: int) -> int:
    return (M + 3) // 4 * 4


def sa_to_mn_major(sa: np.ndarray) -> np.ndarray:
    """Oracle activation scales [G][M][KB] (or [M][KB]) -> [G][KB][stride(M)]."""
    if sa.ndim == 2:
        sa = sa[None]
    G, M, KB = sa.shape
    out = np.zeros((G, KB, sfa_stride(M)), dtype=np.float32)
    out[:, :, :M] = sa.transpose(0, 2, 1)
    return out


def sa_from_mn_major(sfa: np.ndarray, M: int) -> np.ndarray:
    """Library activation scales [G][KB][stride] -> [G][M][KB]."""
    return np.ascontiguousarray(sfa[:, :, :M].transpose(0, 2, 1))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits).view(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def to_torch(arr: np.ndarray, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(arr))
    return t.to(device)


def bf16_tensor(bits: np.ndarray, device="cuda"):
    import torch
    return to_torch(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16), device).view(torch.bfloat16)


def tensor_bf16_bits(t) -> np.ndarray:
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def check_gemm(gpu: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    """Assert the acceptance bar on matching 1-D/2-D arrays of valid outputs."""
    gpu = np.asarray(gpu, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    assert gpu.shape == ref.shape and ref.size > 0
    assert np.all(np.isfinite(gpu)), "%s: non-finite GPU output" % what
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = np.abs(gpu - ref)
    bound = REL_TOL * np.abs(ref) + RMS_TOL * rms
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), (
        "%s: %d of %d outside tolerance; worst at %d: gpu=%r ref=%r bound=%r"
        % (what, int((err > bound).sum()), err.size, worst, gpu[worst], ref[worst], bound[worst]))
    den = float(np.sum(gpu * gpu + ref * ref))
    glob = 1.0 - 2.0 * float(np.sum(gpu * ref)) / den if den > 0 else 0.0
    assert glob < GLOBAL_TOL, "%s: global difference %g" % (what, glob)
    return {"max_rel_err": float(np.max(err / np.maximum(np.abs(ref), 1e-30))),
            "global_diff": glob, "rms": rms}
