"""Shared helpers of the test suite (comparison metrics, buffer plumbing)."""
from __future__ import annotations

import hashlib

import numpy as np
import torch

# Layer-output tolerance (reading of "1e-2 max relative error normalised by
# the output RMS" for a bf16 output): max_i |out_i - ref_i| / max(|ref_i|, rms(ref))
# with ref the oracle's fp64 output before the bf16 cast.
OUT_TOL = 1e-2
# Expert outputs y (fp32 on the GPU) against the oracle's fp64 y, same metric.
Y_TOL = 1e-2


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (on the CPU)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(b) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rms_floor_err(out, ref64) -> float:
    """max |out - ref| / max(|ref|, rms(ref))."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref64, np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    den = np.maximum(np.abs(ref), rms if rms > 0 else 1.0)
    return float(np.max(np.abs(out - ref) / den))


def literal_rms_err(out, ref64) -> float:
    """max |out - ref| / rms(ref) (reported, not gated: bf16 half-ulp floor)."""
    ref = np.asarray(ref64, np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.max(np.abs(np.asarray(out, np.float64) - ref)) / rms)


def sha(t: torch.Tensor) -> str:
    return hashlib.sha256(t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes()).hexdigest()


def expert_weights_host(W1, W3, W2, experts):
    """Copy the weights of the given experts to host numpy (bit patterns)."""
    out = ({}, {}, {})
    for e in sorted(set(int(x) for x in experts)):
        for d, W in zip(out, (W1, W3, W2)):
            d[e] = bits(W[e])
    return out


def mx_tiled_offsets(R: int, K: int) -> np.ndarray:
    """Byte offsets [R, K/32] of the E8M0 scales of an [R, K] MXFP8 code matrix
    in the tiled layout the block-scaled tensor cores read (include/moe.h):
    512-byte atoms of 128 rows x 4 blocks of 32, the K-atoms of a 128-row
    block consecutive; inside an atom row r at (r % 32) * 16 + ((r // 32) % 4) * 4
    and block b at b % 4."""
    if R % 128 or K % 128:
        raise ValueError("R and K must be multiples of 128")
    r = np.arange(R, dtype=np.int64)[:, None]
    b = np.arange(K // 32, dtype=np.int64)[None, :]
    return ((r // 128) * (K // 128) + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + b % 4


def to_tiled(scales_rows: np.ndarray) -> np.ndarray:
    """Row-major scales [R, K/32] -> the tiled table (flat uint8, R*K/32 bytes)."""
    s = np.asarray(scales_rows, np.uint8)
    R, KB = s.shape
    out = np.zeros(R * KB, np.uint8)
    out[mx_tiled_offsets(R, KB * 32)] = s
    return out
