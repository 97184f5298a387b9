"""AWQ W4A16 linear (the second kernel family of the pages), restated in
numpy (float64) -- TEST INFRASTRUCTURE, like the rest of `oracle/`.

What the pages fix ("Bringing Nunchaku 4-bit diffusion inference to
Diffusers", Russian rendering, section "Technical details and hardware
support", and the Korean rendering's kernel-family list): awq_w4a16 layers
hold 4-bit (INT4) weights and use 16-bit activations; they serve the
memory-bound, precision-sensitive modulation / adaptive-normalization
projections of a diffusion transformer (e.g. FLUX's adanorm layers).

Readings of what the pages leave open (A1-A4):
  A1 format: AWQ's published storage format -- asymmetric INT4 per group of
     `group` (128) consecutive input channels of a weight row, one scale
     and one integer zero point per group.  The activation-aware scale
     search of AWQ is an offline tuning step; it is not part of the layer
     and is not reproduced (a searched per-channel scale would be folded
     into W before this step and into X by the caller).
  A2 scale and zero of a group whose range, widened to include 0, is
     [wmin, wmax] (wmin = min(0, min w), wmax = max(0, max w); including 0
     keeps it exactly representable, and a constant group then quantizes to
     itself instead of to the 1e-5 floor):
       s64   = max(wmax - wmin, 1e-5) / 15              (float64)
       scale = fp16_RN(s64)                             (stored)
       z     = clamp(rint(-wmin / scale), 0, 15)        (rint: ties to even)
     each weight: q = clamp(rint(w / scale) + z, 0, 15), the divisions in
     float64 of the stored fp16 scale.
  A3 dequantized weight: (q - z) * scale (exact in float32: a small integer
     times an fp16 value).
  A4 the layer: Y = X deq(W)^T + bias, X bf16 [M, K], in float64 here; the
     kernel accumulates in float32 and rounds Y once to bf16.

Pins: tests/test_oracle_awq.py.
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_bits_to_f64

AWQ_GROUP = 128


def fp16_round(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest fp16 value (ties to even), as float64.  numpy's
    float16 cast rounds to nearest even from float64 directly."""
    return np.asarray(x, np.float64).astype(np.float16).astype(np.float64)


def awq_quantize(W: np.ndarray, group: int = AWQ_GROUP):
    """Readings A1-A2.  W fp32 [N, K] (K % group == 0).  Returns
    (q uint8 [N, K] codes 0..15, z uint8 [N, K/group], scale_f16 uint16
    bit patterns [N, K/group])."""
    W = np.asarray(W, np.float32).astype(np.float64)
    N, K = W.shape
    assert K % group == 0
    G = W.reshape(N, K // group, group)
    wmin = np.minimum(G.min(axis=2), 0.0)
    wmax = np.maximum(G.max(axis=2), 0.0)
    s64 = np.maximum(wmax - wmin, 1e-5) / 15.0
    scale = fp16_round(s64)
    z = np.clip(np.rint(-wmin / scale), 0, 15)
    q = np.clip(np.rint(G / scale[:, :, None]) + z[:, :, None], 0, 15)
    scale_bits = scale.astype(np.float16).view(np.uint16)
    return q.reshape(N, K).astype(np.uint8), z.astype(np.uint8), scale_bits


def awq_dequantize(q: np.ndarray, z: np.ndarray, scale_bits: np.ndarray,
                   group: int = AWQ_GROUP) -> np.ndarray:
    """Reading A3: (q - z) * scale, float64 [N, K]."""
    N, K = q.shape
    scale = np.asarray(scale_bits, np.uint16).view(np.float16).astype(np.float64)
    Q = q.reshape(N, K // group, group).astype(np.float64)
    return ((Q - z[:, :, None].astype(np.float64)) * scale[:, :, None]).reshape(N, K)


def awq_linear_reference(X_bf16: np.ndarray, q, z, scale_bits, bias_bf16=None,
                         group: int = AWQ_GROUP) -> np.ndarray:
    """Reading A4: Y = X deq(W)^T + bias in float64, [M, N]."""
    Y = bf16_bits_to_f64(X_bf16) @ awq_dequantize(q, z, scale_bits, group).T
    if bias_bf16 is not None:
        Y = Y + bf16_bits_to_f64(bias_bf16)[None, :]
    return Y


def pack_nibbles_awq(q: np.ndarray) -> np.ndarray:
    """[N, K] codes -> [N, K/2] bytes, even k in the low nibble (the same
    order as the NVFP4 codes)."""
    q = np.asarray(q, np.uint8)
    return (q[:, 0::2] & 0xF) | ((q[:, 1::2] & 0xF) << 4)
