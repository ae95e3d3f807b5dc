"""Python binding of liborbitquant: argument marshalling only.

Every function has the name of the C entry point it calls
(include/orbitquant.h).  Torch tensors provide device memory and the current
stream; all compute runs in the library's CUDA kernels.  There is no fallback:
if the library is missing or no GPU is present the calls raise.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liborbitquant.so")

OQ_OK = 0
OQ_DTYPE_F32 = 0
OQ_DTYPE_BF16 = 1
OQ_FLAG_SIGNS = 1
OQ_FLAG_GAUSSIAN_MARGINAL = 2
OQ_FLAG_WEIGHT_ONLY_INT4 = 4
OQ_FLAG_FP8_CONTRACTION = 8
# oq_linear_fused decodes the weight codes once per call from this many tokens
# on (bf16 x, d_out % 256 == 0, a workspace of oq_linear_fused_workspace_size)
W16_MIN_T = 1024

# every symbol include/orbitquant.h declares
EXPORTS = (
    "oq_codebook_build", "oq_rotation_build", "oq_layer_create", "oq_layer_destroy", "oq_layer_get_info", "oq_layer_get_perm",
    "oq_rotate_quantize", "oq_weight_prepare", "oq_weight_save", "oq_weight_load", "oq_linear",
    "oq_linear_fused_workspace_size",
    "oq_linear_fused", "oq_linear_fused_decoded_workspace_size", "oq_linear_fused_decoded",
    "oq_rotate_quantize_levels", "oq_linear_levels", "oq_weight_levels", "oq_linear_decoded",
    "oq_linear_fused_static", "oq_linear_fused_host_workspace_size", "oq_linear_fused_host",
    "oq_poll_error", "oq_check_wait_timeout", "oq_last_error", "oq_status_string",
)


class OrbitQuantError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status}: {message}")
        self.status = status


class LibraryMissing(OrbitQuantError):
    pass


class CodebookC(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("bits", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("iterations", ctypes.c_int32), ("levels", ctypes.c_double * 256),
                ("thresholds", ctypes.c_double * 255), ("mse", ctypes.c_double)]


class LayerInfoC(ctypes.Structure):
    _fields_ = [("d_in", ctypes.c_int32), ("d_out", ctypes.c_int32), ("h", ctypes.c_int32),
                ("k", ctypes.c_int32), ("a_bits", ctypes.c_int32), ("w_bits", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("reserved", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("a_words_per_row", ctypes.c_int64), ("w_words_per_row", ctypes.c_int64),
                ("a_scale", ctypes.c_double), ("w_scale", ctypes.c_double)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load liborbitquant.so (raises LibraryMissing if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise LibraryMissing(-1, "load_library",
                             f"{path} not found; build it with `python -m quantized_linear_token_b200.build`")
    L = ctypes.CDLL(path)
    vp, i32, i64, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    sigs = {
        "oq_codebook_build": (i32, [i32, i32, i32, ctypes.POINTER(CodebookC)]),
        "oq_rotation_build": (i32, [i32, u64, i32, vp, vp]),
        "oq_layer_create": (i32, [i32, i32, u64, i32, i32, i32, ctypes.POINTER(vp)]),
        "oq_layer_destroy": (None, [vp]),
        "oq_layer_get_info": (i32, [vp, ctypes.POINTER(LayerInfoC)]),
        "oq_layer_get_perm": (i32, [vp, vp]),
        "oq_rotate_quantize": (i32, [vp, vp, i32, i64, vp, vp, vp]),
        "oq_weight_prepare": (i32, [vp, vp, i32, vp, vp, vp]),
        "oq_linear": (i32, [vp, vp, vp, i64, vp, vp, vp, i32, vp]),
        "oq_linear_fused_workspace_size": (sz, [vp, i64]),
        "oq_linear_fused": (i32, [vp, vp, i32, i64, vp, vp, vp, i32, vp, sz, vp]),
        "oq_rotate_quantize_levels": (i32, [vp, vp, i32, i64, vp, vp, vp]),
        "oq_linear_levels": (i32, [vp, vp, vp, i64, vp, vp, vp, i32, vp]),
        "oq_weight_levels": (i32, [vp, vp, vp, vp]),
        "oq_linear_fused_host_workspace_size": (ctypes.c_size_t, [vp, i32, i64]),
        "oq_linear_fused_host": (i32, [vp, vp, i32, i64, vp, vp, vp, i32, vp, ctypes.c_size_t, vp]),
        "oq_linear_decoded": (i32, [vp, vp, vp, i64, vp, vp, vp, i32, vp]),
        "oq_linear_fused_decoded_workspace_size": (sz, [vp, i64]),
        "oq_linear_fused_decoded": (i32, [vp, vp, i32, i64, vp, vp, vp, i32, vp, sz, vp]),
        "oq_linear_fused_static": (i32, [vp, vp, i32, i64, vp, vp, vp, vp]),
        "oq_weight_save": (i32, [vp, vp, vp, ctypes.c_char_p]),
        "oq_weight_load": (i32, [vp, ctypes.c_char_p, vp, vp]),
        "oq_poll_error": (i32, [vp]),
        "oq_check_wait_timeout": (i32, [vp, ctypes.c_uint32, vp]),
        "oq_last_error": (ctypes.c_char_p, []),
        "oq_status_string": (ctypes.c_char_p, [i32]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int, where: str):
    if status != OQ_OK:
        L = load_library()
        raise OrbitQuantError(status, where, L.oq_last_error().decode() or L.oq_status_string(status).decode())


# ------------------------------------------------------------------ host calls
def oq_codebook_build(d: int, bits: int, flags: int = 0) -> dict:
    """Lloyd-Max codebook C_{d,bits} as designed by the library (host)."""
    cb = CodebookC()
    _check(load_library().oq_codebook_build(d, bits, flags, ctypes.byref(cb)), "oq_codebook_build")
    L = 1 << bits
    return {"d": cb.d, "bits": cb.bits, "flags": cb.flags, "iterations": cb.iterations,
            "levels": np.array(cb.levels[:L]), "thresholds": np.array(cb.thresholds[:L - 1]), "mse": cb.mse}


def oq_rotation_build(d: int, seed: int, flags: int = 0):
    """(perm [d] uint32, signs [d] int8 or None) of the seeded rotation (host)."""
    perm = np.empty(d, dtype=np.uint32)
    signs = np.empty(d, dtype=np.int8) if flags & OQ_FLAG_SIGNS else None
    _check(load_library().oq_rotation_build(d, seed, flags, perm.ctypes.data,
                                            None if signs is None else signs.ctypes.data), "oq_rotation_build")
    return perm, signs


class Layer:
    """Owns an oq_layer* (the shared rotation, codebooks and device tables)."""

    def __init__(self, handle: int, lib):
        self._h = ctypes.c_void_p(handle)
        self._lib = lib
        info = LayerInfoC()
        _check(lib.oq_layer_get_info(self._h, ctypes.byref(info)), "oq_layer_get_info")
        self.d_in, self.d_out, self.h, self.k = info.d_in, info.d_out, info.h, info.k
        self.a_bits, self.w_bits, self.flags, self.seed = info.a_bits, info.w_bits, info.flags, info.seed
        self.a_words_per_row, self.w_words_per_row = info.a_words_per_row, info.w_words_per_row
        self.a_scale, self.w_scale = info.a_scale, info.w_scale

    @property
    def handle(self):
        return self._h

    def perm(self) -> np.ndarray:
        out = np.empty(self.d_in, dtype=np.uint32)
        _check(self._lib.oq_layer_get_perm(self._h, out.ctypes.data), "oq_layer_get_perm")
        return out

    def close(self):
        if self._h:
            self._lib.oq_layer_destroy(self._h)
            self._h = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def oq_layer_create(d_in: int, d_out: int, seed: int, a_bits: int, w_bits: int, flags: int = 0) -> Layer:
    L = load_library()
    h = ctypes.c_void_p()
    _check(L.oq_layer_create(d_in, d_out, seed, a_bits, w_bits, flags, ctypes.byref(h)), "oq_layer_create")
    return Layer(h.value, L)


# ------------------------------------------------------------------ device calls
def _torch():
    import torch
    return torch


def _stream(t):
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return OQ_DTYPE_BF16
    if t.dtype == torch.float32:
        return OQ_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}: use bfloat16 or float32")


def _dev(t, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def oq_rotate_quantize(layer: Layer, x, codes=None, s=None):
    """x [T, d_in] (bf16/fp32, CUDA) -> (codes [T, d_in*a_bits/32] int32 view of uint32, s [T] fp32)."""
    torch = _torch()
    T = x.shape[0]
    if x.dim() != 2 or x.shape[1] != layer.d_in:
        raise ValueError("x must be [T, d_in]")
    if codes is None:
        codes = torch.empty((T, layer.a_words_per_row), dtype=torch.int32, device=x.device)
    if s is None:
        s = torch.empty((T,), dtype=torch.float32, device=x.device)
    _check(load_library().oq_rotate_quantize(layer.handle, _dev(x, "x"), _dtype_code(x), T, _dev(codes, "codes"),
                                             _dev(s, "s"), _stream(x)), "oq_rotate_quantize")
    return codes, s


def oq_weight_prepare(layer: Layer, W, Wcodes=None, r=None):
    """W [d_out, d_in] (fp32/bf16, CUDA) -> (Wcodes [d_out, d_in*w_bits/32] int32, r [d_out] fp32)."""
    torch = _torch()
    if W.dim() != 2 or tuple(W.shape) != (layer.d_out, layer.d_in):
        raise ValueError("W must be [d_out, d_in]")
    if Wcodes is None:
        Wcodes = torch.empty((layer.d_out, layer.w_words_per_row), dtype=torch.int32, device=W.device)
    if r is None:
        r = torch.empty((layer.d_out,), dtype=torch.float32, device=W.device)
    _check(load_library().oq_weight_prepare(layer.handle, _dev(W, "W"), _dtype_code(W), _dev(Wcodes, "Wcodes"),
                                            _dev(r, "r"), _stream(W)), "oq_weight_prepare")
    return Wcodes, r


def _y_out(y, T: int, d_out: int, y_dtype, device):
    """The output tensor (given, or new of y_dtype: torch.float32 or
    torch.bfloat16) and its C dtype code."""
    torch = _torch()
    if y is None:
        y = torch.empty((T, d_out), dtype=torch.float32 if y_dtype is None else y_dtype, device=device)
    if y.dtype == torch.float32:
        return y, OQ_DTYPE_F32
    if y.dtype == torch.bfloat16:
        return y, OQ_DTYPE_BF16
    raise ValueError("y must be float32 or bfloat16")


def oq_linear(layer: Layer, codes, s, Wcodes, r, y=None, y_dtype=None):
    """(codes, s, Wcodes, r) -> y [T, d_out] fp32 (or bf16)."""
    T = codes.shape[0]
    y, ycode = _y_out(y, T, layer.d_out, y_dtype, codes.device)
    _check(load_library().oq_linear(layer.handle, _dev(codes, "codes"), _dev(s, "s"), T, _dev(Wcodes, "Wcodes"),
                                    _dev(r, "r"), _dev(y, "y"), ycode, _stream(codes)), "oq_linear")
    return y


def oq_linear_fused_workspace_size(layer: Layer, T: int) -> int:
    return int(load_library().oq_linear_fused_workspace_size(layer.handle, T))


def oq_linear_fused(layer: Layer, x, Wcodes, r, y=None, workspace=None, y_dtype=None):
    """x [T, d_in] -> y [T, d_out] fp32 (or bf16) in one call."""
    torch = _torch()
    T = x.shape[0]
    y, ycode = _y_out(y, T, layer.d_out, y_dtype, x.device)
    need = oq_linear_fused_workspace_size(layer, T)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=x.device)
    _check(load_library().oq_linear_fused(layer.handle, _dev(x, "x"), _dtype_code(x), T, _dev(Wcodes, "Wcodes"),
                                          _dev(r, "r"), _dev(y, "y"), ycode, _dev(workspace, "workspace"),
                                          workspace.numel() * workspace.element_size(), _stream(x)),
           "oq_linear_fused")
    return y


def oq_rotate_quantize_levels(layer: Layer, x, a16=None, s=None):
    """x [T, d_in] bf16 (CUDA) -> (a16 [T, d_in] fp16 levels of the codes, s [T] fp32):
    the first stage of the fused call's fp16 route."""
    torch = _torch()
    T = x.shape[0]
    if a16 is None:
        a16 = torch.empty((T, layer.d_in), dtype=torch.float16, device=x.device)
    if s is None:
        s = torch.empty((T,), dtype=torch.float32, device=x.device)
    _check(load_library().oq_rotate_quantize_levels(layer.handle, _dev(x, "x"), _dtype_code(x), T, _dev(a16, "a16"),
                                                    _dev(s, "s"), _stream(x)), "oq_rotate_quantize_levels")
    return a16, s


def oq_linear_levels(layer: Layer, a16, s, Wcodes, r, y=None, y_dtype=None):
    """(a16 fp16 levels, s, Wcodes, r) -> y [T, d_out] fp32 (or bf16): the
    second stage of the fused call's fp16 route."""
    T = a16.shape[0]
    y, ycode = _y_out(y, T, layer.d_out, y_dtype, a16.device)
    _check(load_library().oq_linear_levels(layer.handle, _dev(a16, "a16"), _dev(s, "s"), T, _dev(Wcodes, "Wcodes"),
                                           _dev(r, "r"), _dev(y, "y"), ycode, _stream(a16)), "oq_linear_levels")
    return y


def oq_weight_levels(layer: Layer, Wcodes, w16=None):
    """Wcodes [d_out, d_in*w_bits/32] -> w16 [d_out, d_in] fp16 levels of the
    weight codes (decoded once; the large-batch route's B operand)."""
    torch = _torch()
    if w16 is None:
        w16 = torch.empty((layer.d_out, layer.d_in), dtype=torch.float16, device=Wcodes.device)
    _check(load_library().oq_weight_levels(layer.handle, _dev(Wcodes, "Wcodes"), _dev(w16, "w16"), _stream(Wcodes)),
           "oq_weight_levels")
    return w16


def oq_linear_decoded(layer: Layer, a16, s, w16, r, y=None, y_dtype=None):
    """(a16, s, w16, r) -> y [T, d_out] fp32 (or bf16): the contraction of two
    fp16 level operands, both read by TMA."""
    T = a16.shape[0]
    y, ycode = _y_out(y, T, layer.d_out, y_dtype, a16.device)
    _check(load_library().oq_linear_decoded(layer.handle, _dev(a16, "a16"), _dev(s, "s"), T, _dev(w16, "w16"),
                                            _dev(r, "r"), _dev(y, "y"), ycode, _stream(a16)), "oq_linear_decoded")
    return y


def oq_linear_fused_decoded_workspace_size(layer: Layer, T: int) -> int:
    return int(load_library().oq_linear_fused_decoded_workspace_size(layer.handle, T))


def oq_linear_fused_decoded(layer: Layer, x, w16, r, y=None, workspace=None, y_dtype=None):
    """x [T, d_in] bf16 and the weights' fp16 levels w16 -> y [T, d_out]: the
    fused call's large-batch route after its weight decode (one kernel
    rotating, quantizing and contracting where the block size allows)."""
    torch = _torch()
    T = x.shape[0]
    y, ycode = _y_out(y, T, layer.d_out, y_dtype, x.device)
    if workspace is None:
        workspace = torch.empty((max(oq_linear_fused_decoded_workspace_size(layer, T), 1),), dtype=torch.uint8,
                                device=x.device)
    _check(load_library().oq_linear_fused_decoded(layer.handle, _dev(x, "x"), _dtype_code(x), T, _dev(w16, "w16"),
                                                  _dev(r, "r"), _dev(y, "y"), ycode, _dev(workspace, "workspace"),
                                                  workspace.numel() * workspace.element_size(), _stream(x)),
           "oq_linear_fused_decoded")
    return y


def oq_linear_fused_host_workspace_size(layer: Layer, x_dtype: int, T: int) -> int:
    return int(load_library().oq_linear_fused_host_workspace_size(layer.handle, x_dtype, T))


def _host(t, name: str):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def oq_linear_fused_host(layer: Layer, x_host, Wcodes, r, y_host=None, workspace=None, y_dtype=None):
    """x_host [T, d_in] bf16/fp32 in host memory (pinned for overlap) -> y_host
    [T, d_out] fp32 in host memory: copies in, the fused call and copies out,
    overlapped chunk by chunk, queued on the current stream of Wcodes' device.
    Synchronise that stream before reading y_host."""
    torch = _torch()
    T = x_host.shape[0]
    if x_host.dim() != 2 or x_host.shape[1] != layer.d_in:
        raise ValueError("x_host must be [T, d_in]")
    if y_host is None:
        y_host = torch.empty((T, layer.d_out), dtype=torch.float32 if y_dtype is None else y_dtype, pin_memory=True)
    if y_host.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("y_host must be float32 or bfloat16")
    ycode = OQ_DTYPE_F32 if y_host.dtype == torch.float32 else OQ_DTYPE_BF16
    code = _dtype_code(x_host)
    need = oq_linear_fused_host_workspace_size(layer, code, T)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=Wcodes.device)
    _check(load_library().oq_linear_fused_host(layer.handle, _host(x_host, "x_host"), code, T,
                                               _dev(Wcodes, "Wcodes"), _dev(r, "r"), _host(y_host, "y_host"), ycode,
                                               _dev(workspace, "workspace"),
                                               workspace.numel() * workspace.element_size(), _stream(Wcodes)),
           "oq_linear_fused_host")
    return y_host


def oq_linear_fused_static(layer: Layer, x, Wcodes, r, y=None):
    """x [T, d_in] -> y [T, d_out] fp32 without any device allocation by the
    library: its scratch is a fixed array the library reserves per GPU (see
    include/orbitquant.h).  Calls that overlap on the GPU race on it."""
    torch = _torch()
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, layer.d_out), dtype=torch.float32, device=x.device)
    _check(load_library().oq_linear_fused_static(layer.handle, _dev(x, "x"), _dtype_code(x), T,
                                                 _dev(Wcodes, "Wcodes"), _dev(r, "r"), _dev(y, "y"), _stream(x)),
           "oq_linear_fused_static")
    return y


def oq_weight_save(layer: Layer, Wcodes, r, path: str) -> None:
    """Write prepared weights (device Wcodes, r from oq_weight_prepare) to a file."""
    _check(load_library().oq_weight_save(layer.handle, _dev(Wcodes, "Wcodes"), _dev(r, "r"),
                                         os.fsencode(path)), "oq_weight_save")


def oq_weight_load(layer: Layer, path: str, Wcodes=None, r=None):
    """Read prepared weights saved for a layer with the same settings ->
    (Wcodes, r) on the current CUDA device."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device())
    if Wcodes is None:
        Wcodes = torch.empty((layer.d_out, layer.w_words_per_row), dtype=torch.int32, device=dev)
    if r is None:
        r = torch.empty((layer.d_out,), dtype=torch.float32, device=dev)
    _check(load_library().oq_weight_load(layer.handle, os.fsencode(path), _dev(Wcodes, "Wcodes"), _dev(r, "r")),
           "oq_weight_load")
    return Wcodes, r


def oq_poll_error(layer: Layer) -> None:
    _check(load_library().oq_poll_error(layer.handle), "oq_poll_error")


def oq_check_wait_timeout(layer: Layer, limit_us: int) -> None:
    """Launch the bounded-wait self-test on the current stream (its wait runs
    out after limit_us microseconds; oq_poll_error then raises)."""
    torch = _torch()
    _check(load_library().oq_check_wait_timeout(
        layer.handle, int(limit_us), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)),
        "oq_check_wait_timeout")
