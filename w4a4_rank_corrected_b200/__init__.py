"""Python binding of libsvdq.so, the B200-native SVDQuant W4A4 (NVFP4) linear.

Argument marshalling only: every step of the layer runs inside the C/CUDA
library (include/svdq.h).  PyTorch is used for device memory and streams.
There is no fallback: if the library cannot be loaded, importing the
binding raises, and the GPU calls raise SvdqError on any non-OK status.

The functions keep the C names:
  svdq_pack_weight      host-side smoothing, SVD, residual NVFP4 packing
  svdq_quantize_act     activation kernel (+ fused low-rank down-projection)
  svdq_gemm             4-bit GEMM kernel (+ fused up-projection, bias)
  svdq_linear_forward   both kernels on one stream
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

__all__ = [
    "SvdqError", "PackedWeight", "DeviceWeight", "svdq_query_sizes", "svdq_pack_weight",
    "svdq_quantize_act", "svdq_gemm", "svdq_linear_forward", "svdq_act_workspace_bytes",
    "svdq_linear_forward_host", "svdq_linear_forward_static", "svdq_unswizzle_scales",
    "new_workspace", "svdq_gemm_gelu", "svdq_gemm_splitk", "svdq_gemm_workspace_bytes",
    "svdq_forward_workspace_bytes", "new_forward_workspace",
    "svdq_mlp_forward", "svdq_mlp_workspace_bytes", "new_mlp_workspace", "svdq_debug_gelu",
    "svdq_act_row_scales", "svdq_quantize_act_dynamic", "svdq_gemm_dynamic",
    "svdq_dyn_workspace_bytes", "svdq_linear_forward_dynamic", "svdq_awq_pack",
    "svdq_awq_linear", "svdq_awq_tile_codes", "AwqWeight",
    "svdq_device_error", "svdq_selftest_timeout", "svdq_debug_convert", "svdq_sf_tile_offset",
    "svdq_status_string", "SVDQW4A4Linear", "lib", "STATUS",
]

STATUS = {
    0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_UNSUPPORTED_ARCH",
    3: "SVDQ_ERR_MISALIGNED", 4: "SVDQ_ERR_WORKSPACE", 5: "SVDQ_ERR_CUDA",
    6: "SVDQ_ERR_TIMEOUT", 7: "SVDQ_ERR_NUMERIC",
}


class SvdqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({svdq_status_string(status)})")


class SvdqSizes(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("K", ctypes.c_int), ("r", ctypes.c_int),
                ("klr", ctypes.c_int), ("smooth_bytes", ctypes.c_size_t),
                ("l1_bytes", ctypes.c_size_t), ("l2_bytes", ctypes.c_size_t),
                ("l1_mma_bytes", ctypes.c_size_t), ("l2_mma_bytes", ctypes.c_size_t),
                ("codes_w_bytes", ctypes.c_size_t), ("sf_w_bytes", ctypes.c_size_t),
                ("bias_bytes", ctypes.c_size_t)]


class SvdqPackedHost(ctypes.Structure):
    _fields_ = [("smooth", ctypes.c_void_p), ("l1", ctypes.c_void_p), ("l2", ctypes.c_void_p),
                ("l1_mma", ctypes.c_void_p), ("l2_mma", ctypes.c_void_p),
                ("codes_w", ctypes.c_void_p), ("sf_w", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("amax_x", ctypes.c_float), ("amax_w", ctypes.c_float),
                ("g_x", ctypes.c_float), ("gs_x", ctypes.c_float), ("g_w", ctypes.c_float),
                ("alpha", ctypes.c_float), ("lr_scale", ctypes.c_float)]


class SvdqWeight(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("K", ctypes.c_int), ("r", ctypes.c_int),
                ("g_x", ctypes.c_float), ("gs_x", ctypes.c_float), ("g_w", ctypes.c_float),
                ("alpha", ctypes.c_float), ("lr_scale", ctypes.c_float), ("smooth", ctypes.c_void_p),
                ("l1_mma", ctypes.c_void_p), ("l2_mma", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("codes_w", ctypes.c_void_p),
                ("sf_w", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    path = _build.build()          # no-op when the in-tree library is current
    if not os.path.exists(path):
        raise ImportError(f"libsvdq.so missing at {path}")
    L = ctypes.CDLL(path)
    P, I, I64, SZ, F, U64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                             ctypes.c_float, ctypes.c_uint64)
    sig = {
        "svdq_status_string": (ctypes.c_char_p, [I]),
        "svdq_version": (ctypes.c_char_p, []),
        "svdq_query_sizes": (I, [I, I, I, ctypes.POINTER(SvdqSizes)]),
        "svdq_pack_weight": (I, [P, P, P, I, I, I, F, U64, ctypes.POINTER(SvdqPackedHost)]),
        "svdq_unswizzle_scales": (I, [P, I, I, P]),
        "svdq_linear_forward_host": (I, [ctypes.POINTER(SvdqWeight), P, I, I64, P, I64, P, P, P,
                                         SZ, P]),
        "svdq_sf_tile_offset": (I64, [I, I, I]),
        "svdq_act_workspace_bytes": (SZ, [I, I, I]),
        "svdq_quantize_act": (I, [ctypes.POINTER(SvdqWeight), P, I, I64, P, P, P, P]),
        "svdq_gemm": (I, [ctypes.POINTER(SvdqWeight), P, P, P, I, P, I64, P]),
        "svdq_gemm_workspace_bytes": (SZ, [I, I, I]),
        "svdq_gemm_splitk": (I, [ctypes.POINTER(SvdqWeight), P, P, P, I, P, I64, P, SZ, P]),
        "svdq_forward_workspace_bytes": (SZ, [ctypes.POINTER(SvdqWeight), I]),
        "svdq_linear_forward": (I, [ctypes.POINTER(SvdqWeight), P, I, I64, P, I64, P, SZ, P]),
        "svdq_linear_forward_static": (I, [ctypes.POINTER(SvdqWeight), P, I, I64, P, I64, P]),
        "svdq_device_error": (I, [P, ctypes.POINTER(I)]),
        "svdq_selftest_timeout": (I, [I, P]),
        "svdq_debug_convert": (I, [P, P, P, I64, P]),
        "svdq_debug_gelu": (I, [P, P, I64, P]),
        "svdq_awq_pack": (I, [P, I, I, I, P, P, P]),
        "svdq_awq_tile_codes": (I, [P, I, I, P]),
        "svdq_awq_linear": (I, [P, P, P, P, I, I, I, P, I, I64, P, I64, P]),
        "svdq_act_row_scales": (I, [ctypes.POINTER(SvdqWeight), P, I, I64, P, P]),
        "svdq_quantize_act_dynamic": (I, [ctypes.POINTER(SvdqWeight), P, I, I64, P, P, P, P, P]),
        "svdq_gemm_dynamic": (I, [ctypes.POINTER(SvdqWeight), P, P, P, P, I, P, I64, P]),
        "svdq_dyn_workspace_bytes": (SZ, [I, I, I]),
        "svdq_linear_forward_dynamic": (I, [ctypes.POINTER(SvdqWeight), P, I, I64, P, I64, P, SZ,
                                            P]),
        "svdq_gemm_gelu": (I, [ctypes.POINTER(SvdqWeight), P, P, P, I, P, I64, P]),
        "svdq_mlp_workspace_bytes": (SZ, [I, I, I, I, I]),
        "svdq_mlp_forward": (I, [ctypes.POINTER(SvdqWeight), ctypes.POINTER(SvdqWeight), P, I, I64,
                                 P, I64, P, I64, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def svdq_status_string(status: int) -> str:
    return lib.svdq_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != 0:
        raise SvdqError(status, what)


def svdq_query_sizes(N: int, K: int, r: int) -> SvdqSizes:
    out = SvdqSizes()
    _check(lib.svdq_query_sizes(N, K, r, ctypes.byref(out)), "svdq_query_sizes")
    return out


def svdq_sf_tile_offset(row: int, g: int, K: int) -> int:
    return int(lib.svdq_sf_tile_offset(row, g, K))


def svdq_act_workspace_bytes(M: int, K: int, r: int) -> int:
    return int(lib.svdq_act_workspace_bytes(M, K, r))


def new_workspace(M: int, K: int, r: int, device="cuda"):
    """A forward workspace of svdq_act_workspace_bytes(M, K, r) bytes (the
    minimum: the GEMM then never splits K)."""
    import torch
    return torch.empty(max(svdq_act_workspace_bytes(M, K, r), 256), dtype=torch.uint8,
                       device=device)


def svdq_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib.svdq_gemm_workspace_bytes(M, N, K))


def svdq_forward_workspace_bytes(w: "DeviceWeight", M: int) -> int:
    return int(lib.svdq_forward_workspace_bytes(ctypes.byref(w.struct), M))


def new_forward_workspace(w: "DeviceWeight", M: int, device="cuda"):
    """A forward workspace with room for the split-K partials when the layer
    has few output tiles (svdq_forward_workspace_bytes)."""
    import torch
    return torch.empty(max(svdq_forward_workspace_bytes(w, M), 256), dtype=torch.uint8,
                       device=device)


# ---------------------------------------------------------------- pack ----

@dataclass
class PackedWeight:
    """Host result of svdq_pack_weight (numpy arrays, bf16 as uint16)."""
    N: int
    K: int
    r: int
    klr: int
    smooth: np.ndarray       # fp32 [K]
    l1: np.ndarray           # bf16 [K, r]
    l2: np.ndarray           # bf16 [r, N]
    l1_mma: np.ndarray       # bf16 [2r, K]
    l2_mma: np.ndarray       # bf16 [N, klr]
    codes_w: np.ndarray      # u8 [N, K/2]
    sf_w: np.ndarray         # u8, MMA tiles
    bias: Optional[np.ndarray]  # bf16 [N] or None
    amax_x: float
    amax_w: float
    g_x: float
    gs_x: float
    g_w: float
    alpha: float
    lr_scale: float

    def to_device(self, device="cuda", bias_bf16: Optional[np.ndarray] = None) -> "DeviceWeight":
        """Device copies of the packed buffers.  The bias is the packed one
        unless `bias_bf16` is given."""
        import torch

        def up(a):
            return torch.from_numpy(np.ascontiguousarray(a)).to(device)

        t = {"smooth": up(self.smooth), "codes_w": up(self.codes_w), "sf_w": up(self.sf_w)}
        if self.r > 0:
            t["l1_mma"] = up(self.l1_mma.view(np.int16))
            t["l2_mma"] = up(self.l2_mma.view(np.int16))
        if bias_bf16 is None:
            bias_bf16 = self.bias
        if bias_bf16 is not None:
            t["bias"] = up(np.asarray(bias_bf16, np.uint16).view(np.int16))
        return DeviceWeight(self, t)


class DeviceWeight:
    """Device copies of a packed weight plus the C struct pointing at them."""

    def __init__(self, packed: PackedWeight, tensors: dict):
        self.packed = packed
        self.tensors = tensors
        s = SvdqWeight()
        s.N, s.K, s.r = packed.N, packed.K, packed.r
        s.g_x, s.gs_x, s.g_w = packed.g_x, packed.gs_x, packed.g_w
        s.alpha, s.lr_scale = packed.alpha, packed.lr_scale
        for name in ("smooth", "l1_mma", "l2_mma", "bias", "codes_w", "sf_w"):
            t = tensors.get(name)
            setattr(s, name, t.data_ptr() if t is not None else None)
        self.struct = s

    @property
    def N(self):
        return self.packed.N

    @property
    def K(self):
        return self.packed.K

    @property
    def r(self):
        return self.packed.r


def svdq_pack_weight(W: np.ndarray, x_absmax: np.ndarray, r: int, smooth_alpha: float = 0.5,
                     seed: int = 0, bias_bf16: Optional[np.ndarray] = None) -> PackedWeight:
    W = np.ascontiguousarray(W, dtype=np.float32)
    x_absmax = np.ascontiguousarray(x_absmax, dtype=np.float32)
    N, K = W.shape
    if x_absmax.shape != (K,):
        raise ValueError("x_absmax must have shape [K]")
    sz = svdq_query_sizes(N, K, r)
    smooth = np.empty(K, np.float32)
    l1 = np.empty((K, r), np.uint16)
    l2 = np.empty((r, N), np.uint16)
    l1m = np.empty((2 * r, K), np.uint16)
    l2m = np.empty((N, sz.klr), np.uint16)
    codes = np.empty((N, K // 2), np.uint8)
    sf = np.empty(sz.sf_w_bytes, np.uint8)
    bias_in = None
    bias = None
    if bias_bf16 is not None:
        bias_in = np.ascontiguousarray(bias_bf16, dtype=np.uint16)
        if bias_in.shape != (N,):
            raise ValueError("bias must have shape [N]")
        bias = np.empty(N, np.uint16)
    out = SvdqPackedHost()
    out.smooth = smooth.ctypes.data
    out.l1 = l1.ctypes.data if r else None
    out.l2 = l2.ctypes.data if r else None
    out.l1_mma = l1m.ctypes.data if r else None
    out.l2_mma = l2m.ctypes.data if r else None
    out.codes_w = codes.ctypes.data
    out.sf_w = sf.ctypes.data
    out.bias = bias.ctypes.data if bias is not None else None
    _check(lib.svdq_pack_weight(W.ctypes.data, x_absmax.ctypes.data,
                                bias_in.ctypes.data if bias_in is not None else None, N, K, r,
                                float(smooth_alpha), int(seed), ctypes.byref(out)),
           "svdq_pack_weight")
    return PackedWeight(N, K, r, sz.klr, smooth, l1, l2, l1m, l2m, codes, sf, bias,
                        float(out.amax_x), float(out.amax_w), float(out.g_x), float(out.gs_x),
                        float(out.g_w), float(out.alpha), float(out.lr_scale))


def svdq_unswizzle_scales(sf_mma: np.ndarray, rows: int, K: int) -> np.ndarray:
    """MMA tile layout -> row-major [rows, K/16] scales (host permutation)."""
    sf_mma = np.ascontiguousarray(sf_mma, dtype=np.uint8)
    need = ((rows + 127) // 128) * 128 * (K // 16)
    if sf_mma.size < need:
        raise ValueError("sf_mma smaller than round_up(rows, 128) * K/16 bytes")
    out = np.empty((rows, K // 16), np.uint8)
    _check(lib.svdq_unswizzle_scales(sf_mma.ctypes.data, rows, K, out.ctypes.data),
           "svdq_unswizzle_scales")
    return out


# ------------------------------------------------------------- forward ----

def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _act_shapes(M: int, K: int, r: int):
    klr = ((2 * r + 63) // 64) * 64
    sf_bytes = ((M + 127) // 128) * 128 * (K // 16)
    return klr, sf_bytes


def _check_x(X, K):
    import torch
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != K or X.stride(1) != 1:
        raise ValueError("X must be a bf16 [M, K] tensor with unit column stride")


def _keep_alive_on(stream, *tensors):
    """Tensors made here on torch's current stream but used by kernels on
    another stream: tell the caching allocator, so their memory is not
    handed to other work before that stream is done with it."""
    import torch
    if stream is None or stream == torch.cuda.current_stream():
        return
    for t in tensors:
        if t is not None:
            t.record_stream(stream)


def svdq_quantize_act(w: DeviceWeight, X, codes_x=None, sf_x=None, xl1=None, stream=None):
    """Returns (codes_x u8 [M, K/2], sf_x u8 tiles, xl1 bf16 [M, klr] or None)."""
    import torch
    _check_x(X, w.K)
    M = X.shape[0]
    klr, sf_bytes = _act_shapes(M, w.K, w.r)
    dev = X.device
    made = []
    if codes_x is None:
        codes_x = torch.empty((M, w.K // 2), dtype=torch.uint8, device=dev)
        made.append(codes_x)
    if sf_x is None:
        sf_x = torch.empty(sf_bytes, dtype=torch.uint8, device=dev)
        made.append(sf_x)
    if xl1 is None and w.r > 0:
        xl1 = torch.empty((M, klr), dtype=torch.bfloat16, device=dev)
        made.append(xl1)
    _check(lib.svdq_quantize_act(ctypes.byref(w.struct), X.data_ptr(), M, X.stride(0),
                                 codes_x.data_ptr(), sf_x.data_ptr(), _ptr(xl1),
                                 _stream_ptr(stream)), "svdq_quantize_act")
    _keep_alive_on(stream, *made)
    return codes_x, sf_x, xl1


def svdq_gemm(w: DeviceWeight, codes_x, sf_x, xl1, M: int, Y=None, stream=None):
    import torch
    made = []
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=codes_x.device)
        made.append(Y)
    _check(lib.svdq_gemm(ctypes.byref(w.struct), codes_x.data_ptr(), sf_x.data_ptr(),
                         _ptr(xl1), M, Y.data_ptr(), Y.stride(0), _stream_ptr(stream)),
           "svdq_gemm")
    _keep_alive_on(stream, *made)
    return Y


def svdq_linear_forward(w: DeviceWeight, X, Y=None, workspace=None, stream=None):
    import torch
    _check_x(X, w.K)
    M = X.shape[0]
    made = []
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
        made.append(Y)
    if workspace is None:
        workspace = new_forward_workspace(w, M, X.device)
        made.append(workspace)
    _check(lib.svdq_linear_forward(ctypes.byref(w.struct), X.data_ptr(), M, X.stride(0),
                                   Y.data_ptr(), Y.stride(0), workspace.data_ptr(),
                                   workspace.numel(), _stream_ptr(stream)),
           "svdq_linear_forward")
    _keep_alive_on(stream, *made)
    return Y


def svdq_gemm_splitk(w: DeviceWeight, codes_x, sf_x, xl1, M: int, Y=None, workspace=None,
                     stream=None):
    """svdq_gemm with K split across CTA pairs when the output has few tiles."""
    import torch
    made = []
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=codes_x.device)
        made.append(Y)
    need = svdq_gemm_workspace_bytes(M, w.N, w.K)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=codes_x.device)
        made.append(workspace)
    _check(lib.svdq_gemm_splitk(ctypes.byref(w.struct), codes_x.data_ptr(), sf_x.data_ptr(),
                                _ptr(xl1), M, Y.data_ptr(), Y.stride(0), _ptr(workspace),
                                0 if workspace is None else workspace.numel(),
                                _stream_ptr(stream)), "svdq_gemm_splitk")
    _keep_alive_on(stream, *made)
    return Y


def svdq_gemm_gelu(w: DeviceWeight, codes_x, sf_x, xl1, M: int, H=None, stream=None):
    """The GEMM with the MLP pair's GELU in its epilogue: H = GELU(layer output)."""
    import torch
    made = []
    if H is None:
        H = torch.empty((M, w.N), dtype=torch.bfloat16, device=codes_x.device)
        made.append(H)
    _check(lib.svdq_gemm_gelu(ctypes.byref(w.struct), codes_x.data_ptr(), sf_x.data_ptr(),
                              _ptr(xl1), M, H.data_ptr(), H.stride(0), _stream_ptr(stream)),
           "svdq_gemm_gelu")
    _keep_alive_on(stream, *made)
    return H


def svdq_mlp_workspace_bytes(M: int, K1: int, N1: int, r1: int, r2: int) -> int:
    return int(lib.svdq_mlp_workspace_bytes(M, K1, N1, r1, r2))


def new_mlp_workspace(M: int, w1: "DeviceWeight", w2: "DeviceWeight", device="cuda"):
    import torch
    return torch.empty(max(svdq_mlp_workspace_bytes(M, w1.K, w1.N, w1.r, w2.r), 256),
                       dtype=torch.uint8, device=device)


def svdq_mlp_forward(w1: DeviceWeight, w2: DeviceWeight, X, H=None, Y=None, workspace=None,
                     stream=None):
    """fc1 -> GELU (fused into fc1's epilogue) -> fc2.  Returns (H, Y)."""
    import torch
    _check_x(X, w1.K)
    M = X.shape[0]
    made = []
    if H is None:
        H = torch.empty((M, w1.N), dtype=torch.bfloat16, device=X.device)
        made.append(H)
    if Y is None:
        Y = torch.empty((M, w2.N), dtype=torch.bfloat16, device=X.device)
        made.append(Y)
    if workspace is None:
        workspace = new_mlp_workspace(M, w1, w2, X.device)
        made.append(workspace)
    _check(lib.svdq_mlp_forward(ctypes.byref(w1.struct), ctypes.byref(w2.struct), X.data_ptr(), M,
                                X.stride(0), H.data_ptr(), H.stride(0), Y.data_ptr(), Y.stride(0),
                                workspace.data_ptr(), workspace.numel(), _stream_ptr(stream)),
           "svdq_mlp_forward")
    _keep_alive_on(stream, *made)
    return H, Y


def svdq_debug_gelu(y_bf16):
    """The epilogue's GELU on a bf16 tensor (diagnostic)."""
    import torch
    y = y_bf16.contiguous()
    out = torch.empty_like(y)
    _check(lib.svdq_debug_gelu(y.data_ptr(), out.data_ptr(), y.numel(), _stream_ptr(None)),
           "svdq_debug_gelu")
    return out


# ------------------------------------------------ dynamic (per-token) ----

def svdq_act_row_scales(w: DeviceWeight, X, stream=None):
    """Per-row scales {g, gs, lr, alpha} (fp32 [M, 4]) of the dynamic mode."""
    import torch
    _check_x(X, w.K)
    M = X.shape[0]
    rs = torch.empty((M, 4), dtype=torch.float32, device=X.device)
    _check(lib.svdq_act_row_scales(ctypes.byref(w.struct), X.data_ptr(), M, X.stride(0),
                                   rs.data_ptr(), _stream_ptr(stream)), "svdq_act_row_scales")
    _keep_alive_on(stream, rs)
    return rs


def svdq_quantize_act_dynamic(w: DeviceWeight, X, row_scales, stream=None):
    """(codes_x, sf_x, xl1) with each row's own tensor scales."""
    import torch
    _check_x(X, w.K)
    M = X.shape[0]
    klr, sf_bytes = _act_shapes(M, w.K, w.r)
    codes_x = torch.empty((M, w.K // 2), dtype=torch.uint8, device=X.device)
    sf_x = torch.empty(sf_bytes, dtype=torch.uint8, device=X.device)
    xl1 = torch.empty((M, klr), dtype=torch.bfloat16, device=X.device) if w.r else None
    _check(lib.svdq_quantize_act_dynamic(ctypes.byref(w.struct), X.data_ptr(), M, X.stride(0),
                                         row_scales.data_ptr(), codes_x.data_ptr(),
                                         sf_x.data_ptr(), _ptr(xl1), _stream_ptr(stream)),
           "svdq_quantize_act_dynamic")
    _keep_alive_on(stream, codes_x, sf_x, xl1)
    return codes_x, sf_x, xl1


def svdq_gemm_dynamic(w: DeviceWeight, codes_x, sf_x, xl1, row_scales, M: int, Y=None,
                      stream=None):
    import torch
    made = []
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=codes_x.device)
        made.append(Y)
    _check(lib.svdq_gemm_dynamic(ctypes.byref(w.struct), codes_x.data_ptr(), sf_x.data_ptr(),
                                 _ptr(xl1), row_scales.data_ptr(), M, Y.data_ptr(), Y.stride(0),
                                 _stream_ptr(stream)), "svdq_gemm_dynamic")
    _keep_alive_on(stream, *made)
    return Y


def svdq_dyn_workspace_bytes(M: int, K: int, r: int) -> int:
    return int(lib.svdq_dyn_workspace_bytes(M, K, r))


def svdq_linear_forward_dynamic(w: DeviceWeight, X, Y=None, workspace=None, stream=None):
    """The layer with per-token activation scales."""
    import torch
    _check_x(X, w.K)
    M = X.shape[0]
    made = []
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
        made.append(Y)
    if workspace is None:
        workspace = torch.empty(max(svdq_dyn_workspace_bytes(M, w.K, w.r), 256),
                                dtype=torch.uint8, device=X.device)
        made.append(workspace)
    _check(lib.svdq_linear_forward_dynamic(ctypes.byref(w.struct), X.data_ptr(), M, X.stride(0),
                                           Y.data_ptr(), Y.stride(0), workspace.data_ptr(),
                                           workspace.numel(), _stream_ptr(stream)),
           "svdq_linear_forward_dynamic")
    _keep_alive_on(stream, *made)
    return Y


# --------------------------------------------------------- AWQ W4A16 ----

@dataclass
class AwqWeight:
    """A packed AWQ W4A16 weight (host numpy arrays) and, after to_device,
    its device copies."""
    N: int
    K: int
    group: int
    q: np.ndarray          # u8 [N, K/2], even k in the low nibble
    zeros: np.ndarray      # u8 [N, K/group]
    scales: np.ndarray     # fp16 bits [N, K/group]
    bias: Optional[np.ndarray] = None
    dev: Optional[dict] = None

    def to_device(self, device="cuda") -> "AwqWeight":
        """Device copies; the codes go up in the GPU layer's tiled layout."""
        import torch
        up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.dev = {"q": up(svdq_awq_tile_codes(self.q, self.N, self.K)), "zeros": up(self.zeros),
                    "scales": up(self.scales.view(np.int16)),
                    "bias": None if self.bias is None else up(np.asarray(self.bias, np.uint16).view(np.int16))}
        return self


def svdq_awq_pack(W: np.ndarray, group: int = 128, bias_bf16=None) -> AwqWeight:
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    q = np.empty((N, K // 2), np.uint8)
    z = np.empty((N, K // group), np.uint8)
    sc = np.empty((N, K // group), np.uint16)
    _check(lib.svdq_awq_pack(W.ctypes.data, N, K, group, q.ctypes.data, z.ctypes.data,
                             sc.ctypes.data), "svdq_awq_pack")
    return AwqWeight(N, K, group, q, z, sc, None if bias_bf16 is None else np.asarray(bias_bf16, np.uint16))


def svdq_awq_tile_codes(q_rowmajor: np.ndarray, N: int, K: int) -> np.ndarray:
    """[N, K/2] codes -> the GPU layer's tiled layout (ceil(N/16)*16*K/2 bytes)."""
    q_rowmajor = np.ascontiguousarray(q_rowmajor, dtype=np.uint8)
    if q_rowmajor.shape != (N, K // 2):
        raise ValueError("codes must have shape [N, K/2]")
    out = np.empty(((N + 15) // 16 * 16 * K // 2,), np.uint8)
    _check(lib.svdq_awq_tile_codes(q_rowmajor.ctypes.data, N, K, out.ctypes.data),
           "svdq_awq_tile_codes")
    return out


def svdq_awq_linear(w: AwqWeight, X, Y=None, stream=None):
    """Y = X dequant(W)^T + bias (bf16), 1 <= M <= 8."""
    import torch
    if w.dev is None:
        raise ValueError("AwqWeight.to_device() first")
    _check_x(X, w.K)
    M = X.shape[0]
    made = []
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
        made.append(Y)
    d = w.dev
    _check(lib.svdq_awq_linear(d["q"].data_ptr(), d["zeros"].data_ptr(), d["scales"].data_ptr(),
                               _ptr(d["bias"]), w.N, w.K, w.group, X.data_ptr(), M, X.stride(0),
                               Y.data_ptr(), Y.stride(0), _stream_ptr(stream)), "svdq_awq_linear")
    _keep_alive_on(stream, *made)
    return Y


SVDQ_STATIC_WORKSPACE_BYTES = 16 << 20


def svdq_linear_forward_static(w: DeviceWeight, X, Y=None, stream=None):
    """The forward with the library's own fixed device scratch: the C call
    allocates nothing (Y is allocated here only when not given).  M is
    limited to svdq_act_workspace_bytes(M, K, r) <= SVDQ_STATIC_WORKSPACE_BYTES;
    calls that overlap in time on one device share the scratch and race."""
    import torch
    _check_x(X, w.K)
    M = X.shape[0]
    made = []
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
        made.append(Y)
    _check(lib.svdq_linear_forward_static(ctypes.byref(w.struct), X.data_ptr(), M, X.stride(0),
                                          Y.data_ptr(), Y.stride(0), _stream_ptr(stream)),
           "svdq_linear_forward_static")
    _keep_alive_on(stream, *made)
    return Y


def svdq_linear_forward_host(w: DeviceWeight, X_host, Y_host, X_dev, Y_dev, workspace,
                             stream=None):
    """The host-buffer forward (C ABI svdq_linear_forward_host): X from host
    memory (pinned, for an asynchronous copy) to the device, the layer, Y
    back to host memory, all enqueued on `stream`.  X_dev [M, K], Y_dev
    [M, N] and the workspace are caller-owned device buffers."""
    _check_x(X_host, w.K)
    M = X_host.shape[0]
    if tuple(X_dev.shape) != (M, w.K) or tuple(Y_dev.shape) != (M, w.N) or \
            tuple(Y_host.shape) != (M, w.N) or not X_dev.is_contiguous() or \
            not Y_dev.is_contiguous() or Y_host.stride(1) != 1:
        raise ValueError("X_dev [M, K], Y_dev [M, N] contiguous; Y_host [M, N] row-major")
    _check(lib.svdq_linear_forward_host(ctypes.byref(w.struct), X_host.data_ptr(), M,
                                        X_host.stride(0), Y_host.data_ptr(), Y_host.stride(0),
                                        X_dev.data_ptr(), Y_dev.data_ptr(), workspace.data_ptr(),
                                        workspace.numel(), _stream_ptr(stream)),
           "svdq_linear_forward_host")
    return Y_host


class HostStreamer:
    """The host-buffer forward over a sequence of host batches (pinned X in,
    pinned Y out): each batch is one svdq_linear_forward_host call (upload,
    both kernels, download, in order on one stream); consecutive batches
    alternate between two streams with a device buffer set each, so the
    download of one batch overlaps the upload and kernels of the next.
    submit() only enqueues; synchronize() waits for all of it."""

    def __init__(self, w: DeviceWeight, M: int, device="cuda"):
        import torch
        self.w, self.M = w, M
        self.X = [torch.empty((M, w.K), dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.Y = [torch.empty((M, w.N), dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.ws = [new_forward_workspace(w, M, device) for _ in range(2)]
        self.streams = [torch.cuda.Stream(device=device) for _ in range(2)]
        self.n = 0

    def submit(self, X_host, Y_host):
        b = self.n & 1                 # buffer set b is only ever used on stream b
        svdq_linear_forward_host(self.w, X_host, Y_host, self.X[b], self.Y[b], self.ws[b],
                                 self.streams[b])
        self.n += 1

    def synchronize(self):
        for s in self.streams:
            s.synchronize()


def svdq_device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    st = lib.svdq_device_error(_stream_ptr(stream), ctypes.byref(code))
    if st not in (0, 6):
        raise SvdqError(st, "svdq_device_error")
    return code.value


def svdq_selftest_timeout(timeout_us: int, stream=None):
    _check(lib.svdq_selftest_timeout(int(timeout_us), _stream_ptr(stream)),
           "svdq_selftest_timeout")


def svdq_debug_convert(x):
    import torch
    x = x.contiguous()
    e2 = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    e4 = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    _check(lib.svdq_debug_convert(x.data_ptr(), e2.data_ptr(), e4.data_ptr(), x.numel(),
                                  _stream_ptr(None)), "svdq_debug_convert")
    return e2, e4


# ------------------------------------------------------------ module ----

def _linear_module_base():
    import torch
    return torch.nn.Module


class SVDQW4A4Linear(_linear_module_base()):
    """Drop-in analogue of the runtime layer the article names
    (SVDQW4A4Linear replaces nn.Linear): built from a float weight, a bias and
    calibration statistics; forward runs svdq_linear_forward."""

    def __init__(self, weight: np.ndarray, bias_bf16: Optional[np.ndarray], x_absmax: np.ndarray,
                 rank: int = 32, smooth_alpha: float = 0.5, seed: int = 0, device="cuda"):
        super().__init__()
        self.packed = svdq_pack_weight(weight, x_absmax, rank, smooth_alpha, seed, bias_bf16)
        self.dev = self.packed.to_device(device)
        self.in_features = self.packed.K
        self.out_features = self.packed.N
        self._ws = None

    def forward(self, X):
        import torch
        lead = X.shape[:-1]
        X2 = X.reshape(-1, X.shape[-1])
        M = X2.shape[0]
        need = svdq_forward_workspace_bytes(self.dev, M)
        if self._ws is None or self._ws.numel() < need or self._ws.device != X.device:
            self._ws = new_forward_workspace(self.dev, M, X.device)
        Y = svdq_linear_forward(self.dev, X2, workspace=self._ws)
        return Y.reshape(*lead, self.out_features)
