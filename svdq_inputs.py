"""Seeded synthetic inputs for the SVDQuant W4A4 linear layer.

This module only draws random tensors with the shapes and value
distributions of the Flux-shaped workloads; it holds none of the method's
arithmetic (no smoothing, no SVD, no quantization).  Both the CPU oracle
(`oracle/`) and the CUDA path (through the tests and `bench.py`) take their
inputs from here, so the two sides always see the same bits.

Recipe (every tensor is drawn from one `numpy.random.default_rng(seed)` in
the order written below, in float64, then cast):
  * X: standard normal (or Student-t with nu=3 divided by sqrt(3), i.e. unit
    variance) of shape [M, K]; `x_outliers` distinct channels chosen with
    `rng.choice(K, n, replace=False)` are multiplied by `x_scale`.  Cast
    float64 -> float32 (round to nearest even) -> bfloat16 (round to nearest
    even); bf16 tensors are carried as uint16 bit patterns.
  * W: normal(0, 0.02^2) of shape [N, K] (out x in, the PyTorch Linear
    layout); `w_outliers` distinct input columns are multiplied by 8.  Cast to
    float32.
  * bias: normal(0, 0.01^2) of shape [N], cast to bfloat16 like X.
For chained layers the weights of layer l+1 are drawn after those of layer l
from the same generator; the activations of later layers are produced by the
layers themselves.

Outlier counts follow "1% of channels" = round(0.01 * K) (31 of 3072) and
"0.5%" = round(0.005 * K) (15 of 3072, 61 of 12288).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit pattern (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    rounding = ((b >> 16) & 1) + 0x7FFF
    out = ((b + rounding) >> 16).astype(np.uint16)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit pattern (uint16) -> float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclass
class LayerSpec:
    name: str
    M: int
    K: int
    N: int
    r: int
    w_outliers: int
    w_scale: float = 8.0


@dataclass
class WorkloadSpec:
    """One workload: a list of linears (chained if `chain` is set)."""
    name: str
    seed: int
    layers: List[LayerSpec]
    x_dist: str = "normal"          # "normal" | "student_t3"
    x_outliers: int = 31
    x_scale: float = 30.0
    chain: Optional[str] = None      # None | "mlp" | "block"
    description: str = ""


def _pct(p: float, K: int) -> int:
    return int(round(p * K))


def workload_specs() -> Dict[str, WorkloadSpec]:
    """The five synthetic Flux-shaped workloads (and the sweep points of the
    rank / small-M workload as separate entries)."""
    H = 3072
    specs: Dict[str, WorkloadSpec] = {}
    specs["single_256"] = WorkloadSpec(
        "single_256", 0, [LayerSpec("linear", 256, H, H, 32, 16)],
        x_outliers=32, description="single svdq linear M=256 K=N=3072 r=32")
    specs["flux_qkv"] = WorkloadSpec(
        "flux_qkv", 1, [LayerSpec("qkv", 4608, H, 3 * H, 32, 16)],
        x_outliers=_pct(0.01, H),
        description="Flux fused QKV projection M=4608 K=3072 N=9216 r=32")
    specs["flux_mlp"] = WorkloadSpec(
        "flux_mlp", 2,
        [LayerSpec("fc1", 4608, H, 4 * H, 32, _pct(0.005, H)),
         LayerSpec("fc2", 4608, 4 * H, H, 32, _pct(0.005, 4 * H))],
        x_outliers=_pct(0.01, H), chain="mlp",
        description="Flux MLP pair fc1 3072->12288, GELU, fc2 12288->3072, M=4608 r=32")
    for r in (16, 32, 64, 128):
        specs[f"sweep_r{r}"] = WorkloadSpec(
            f"sweep_r{r}", 3, [LayerSpec("linear", 4608, H, H, r, 16)],
            x_dist="student_t3", x_outliers=_pct(0.01, H), x_scale=50.0,
            description=f"3072x3072 linear, Student-t activations, M=4608 r={r}")
    for M in (64, 512):
        specs[f"sweep_m{M}"] = WorkloadSpec(
            f"sweep_m{M}", 3, [LayerSpec("linear", M, H, H, 32, 16)],
            x_dist="student_t3", x_outliers=_pct(0.01, H), x_scale=50.0,
            description=f"3072x3072 linear, Student-t activations, M={M} r=32")
    specs["flux_block"] = WorkloadSpec(
        "flux_block", 4,
        [LayerSpec("qkv", 18432, H, 3 * H, 32, _pct(0.005, H)),
         LayerSpec("out", 18432, H, H, 32, _pct(0.005, H)),
         LayerSpec("fc1", 18432, H, 4 * H, 32, _pct(0.005, H)),
         LayerSpec("fc2", 18432, 4 * H, H, 32, _pct(0.005, 4 * H))],
        x_outliers=_pct(0.01, H), chain="block",
        description="Flux block linears at batch 4 (M=18432): qkv, out (V slice), fc1, GELU, fc2")
    return specs


@dataclass
class LayerTensors:
    spec: LayerSpec
    W: np.ndarray                  # float32 [N, K]
    bias_bf16: np.ndarray          # uint16 [N]


@dataclass
class Workload:
    spec: WorkloadSpec
    X_bf16: np.ndarray             # uint16 [M, K0]: the first layer's input
    layers: List[LayerTensors] = field(default_factory=list)


def draw_activations(rng: np.random.Generator, M: int, K: int, dist: str,
                     n_outliers: int, scale: float) -> np.ndarray:
    if dist == "normal":
        x = rng.standard_normal((M, K))
    elif dist == "student_t3":
        x = rng.standard_t(3.0, size=(M, K)) / np.sqrt(3.0)
    else:
        raise ValueError(dist)
    if n_outliers:
        ch = rng.choice(K, n_outliers, replace=False)
        x[:, ch] *= scale
    return f32_to_bf16_bits(x.astype(np.float32))


def draw_weight(rng: np.random.Generator, N: int, K: int, n_outliers: int,
                scale: float):
    w = rng.standard_normal((N, K)) * 0.02
    if n_outliers:
        cols = rng.choice(K, n_outliers, replace=False)
        w[:, cols] *= scale
    bias = rng.standard_normal(N) * 0.01
    return w.astype(np.float32), f32_to_bf16_bits(bias.astype(np.float32))


def make_workload(name: str, M: Optional[int] = None) -> Workload:
    """Draw the tensors of workload `name`.  `M` overrides the token count
    (rows of X) while keeping every other draw identical in distribution."""
    spec = workload_specs()[name]
    rng = np.random.default_rng(spec.seed)
    first = spec.layers[0]
    m = first.M if M is None else M
    X = draw_activations(rng, m, first.K, spec.x_dist, spec.x_outliers, spec.x_scale)
    wl = Workload(spec, X)
    for ls in spec.layers:
        W, b = draw_weight(rng, ls.N, ls.K, ls.w_outliers, ls.w_scale)
        wl.layers.append(LayerTensors(ls, W, b))
    return wl


def random_layer(seed: int, M: int, K: int, N: int, x_outliers: int = 4,
                 w_outliers: int = 2, dist: str = "normal",
                 x_scale: float = 30.0):
    """A small layer of arbitrary shape with the same value model, for
    ragged-shape parity cases."""
    rng = np.random.default_rng(seed)
    X = draw_activations(rng, M, K, dist, min(x_outliers, K), x_scale)
    W, b = draw_weight(rng, N, K, min(w_outliers, K), 8.0)
    return X, W, b


def channel_absmax(X_bf16: np.ndarray) -> np.ndarray:
    """Per-input-channel max |x| of a bf16 activation tensor (calibration
    statistics are the layer's own input)."""
    return np.abs(bf16_bits_to_f32(X_bf16)).max(axis=0).astype(np.float32)
