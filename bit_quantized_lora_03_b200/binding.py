"""Thin Python binding of libqlora_nf4 (ctypes over the C ABI in include/qlora_nf4.h).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
PyTorch supplies device memory (including the caller-owned workspace) and the current stream.
There is no fallback: if the library is missing or the device is not an sm_100 GPU, the
calls raise.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

QLORA_OK = 0
QLORA_ERR_INVALID_ARG = -1
QLORA_ERR_BAD_SHAPE = -2
QLORA_ERR_MISALIGNED = -3
QLORA_ERR_WORKSPACE = -4
QLORA_ERR_CUDA = -5
QLORA_ERR_UNSUPPORTED_DEVICE = -6
QLORA_ERR_SCRATCH_LIMIT = -7
QLORA_STATIC_SCRATCH_BYTES = 8 << 20
QLORA_DEV_NONFINITE = 1
QLORA_DEV_TIMEOUT = 2
QLORA_DEV_LAUNCH = 4

# Every symbol the header declares, with its ctypes signature.
_PTR = ctypes.c_void_p
_I64 = ctypes.c_int64
SIGNATURES = {
    "qlora_nf4_codebook": (ctypes.c_int, [_PTR, _PTR]),
    "nf4_quantize": (ctypes.c_int, [_PTR, _PTR, _PTR]),
    "nf4_dequantize": (ctypes.c_int, [_PTR, _PTR, _PTR]),
    "qlora_linear_fwd": (ctypes.c_int, [_PTR, _I64, _PTR, _PTR, _PTR, _I64, ctypes.c_float,
                                        _PTR, _PTR, _PTR, ctypes.c_size_t, _PTR]),
    "qlora_linear_bwd": (ctypes.c_int, [_PTR, _PTR, _I64, _PTR, _PTR, _PTR, _I64, ctypes.c_float,
                                        _PTR, _PTR, _PTR, _PTR, _PTR, ctypes.c_size_t, _PTR]),
    "qlora_fwd_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _I64, _I64]),
    "qlora_bwd_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _I64, _I64]),
    "qlora_get_last_status": (ctypes.c_int, [_PTR]),
    "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qlora_set_gemv_max_ctas": (ctypes.c_int, [ctypes.c_int]),
    "qlora_selftest_wait_timeout": (ctypes.c_int, [_I64, _PTR]),
    "qlora_merge_adapters": (ctypes.c_int, [_PTR, _PTR, _PTR, _I64, ctypes.c_float, _PTR, _PTR]),
    "qlora_codebook": (ctypes.c_int, [ctypes.c_int, _PTR, _PTR]),
    "qlora_adamw_step": (ctypes.c_int, [_PTR, _PTR, _PTR, _PTR, _PTR, _I64, ctypes.c_float,
                                        ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                        ctypes.c_float, _I64, ctypes.c_uint, _PTR]),
    "qlora_adamw_step_multi": (ctypes.c_int, [ctypes.c_int, _PTR, _PTR, _PTR, _PTR, _PTR, _PTR,
                                              ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                              ctypes.c_float, ctypes.c_float, _I64, ctypes.c_uint,
                                              _PTR]),
    "qlora_quantize_codebook": (ctypes.c_int, [_PTR, _PTR, ctypes.c_int, _PTR]),
    "qlora_dequantize_codebook": (ctypes.c_int, [_PTR, ctypes.c_int, _PTR, _PTR]),
    "qlora_quantize_format": (ctypes.c_int, [_PTR, _PTR, ctypes.c_int, ctypes.c_int, _PTR]),
    "qlora_dequantize_format": (ctypes.c_int, [_PTR, ctypes.c_int, ctypes.c_int, _PTR, _PTR]),
    "qlora_profile_begin": (ctypes.c_int, [ctypes.c_int]),
    "qlora_profile_end": (ctypes.c_int, [_PTR, _PTR, ctypes.c_int]),
    "qlora_kernel_name": (ctypes.c_char_p, [ctypes.c_int]),
    "qlora_linear_fwd_noalloc": (ctypes.c_int, [_PTR, _I64, _PTR, _PTR, _PTR, _I64,
                                                ctypes.c_float, _PTR, _PTR, _PTR]),
    "qlora_linear_fwd_dropout": (ctypes.c_int, [_PTR, _I64, _PTR, _PTR, _PTR, _I64, ctypes.c_float,
                                                ctypes.c_float, ctypes.c_uint64, _PTR, _PTR, _PTR,
                                                _PTR, ctypes.c_size_t, _PTR]),
    "qlora_linear_bwd_dropout": (ctypes.c_int, [_PTR, _PTR, _I64, _PTR, _PTR, _PTR, _I64,
                                                ctypes.c_float, ctypes.c_float, ctypes.c_uint64,
                                                _PTR, _PTR, _PTR, _PTR, _PTR, _PTR, ctypes.c_size_t,
                                                _PTR]),
    "qlora_fwd_dropout_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _I64, _I64]),
    "qlora_bwd_dropout_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _I64, _I64]),
    "qlora_dropout_apply": (ctypes.c_int, [_PTR, _I64, _I64, ctypes.c_float, ctypes.c_uint64, _PTR,
                                           _PTR]),
}
KERNEL_KINDS = 8


class NF4WeightDesc(ctypes.Structure):
    """ctypes mirror of `nf4_weight`."""
    _fields_ = [("codes", _PTR), ("absmax_q8", _PTR), ("absmax_s2", _PTR),
                ("out_features", _I64), ("in_features", _I64)]


_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return _build.LIB_PATH


def lib() -> ctypes.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError(f"{path} is missing: build it with "
                                   "`python -m bit_quantized_lora_03_b200.build`")
            cdll = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(cdll, name)
                fn.restype = res
                fn.argtypes = args
            _lib = cdll
        return _lib


def status_string(code: int) -> str:
    return lib().qlora_status_string(int(code)).decode()


def _check(rc: int, what: str) -> None:
    if rc != QLORA_OK:
        raise RuntimeError(f"{what} failed: {status_string(rc)} ({rc})")


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


CODEBOOK_NF4, CODEBOOK_FP4, CODEBOOK_INT4 = 0, 1, 2
SCALES_U8, SCALES_S8, SCALES_E4M3 = 0, 1, 2


def codebook(codebook_id: int | None = None):
    """(levels[16], midpoints[15]) as derived by the library (host call, no GPU needed);
    the NF4 codebook unless another id is given."""
    lv = (ctypes.c_float * 16)()
    md = (ctypes.c_float * 15)()
    if codebook_id is None:
        _check(lib().qlora_nf4_codebook(ctypes.cast(lv, _PTR), ctypes.cast(md, _PTR)), "codebook")
    else:
        _check(lib().qlora_codebook(int(codebook_id), ctypes.cast(lv, _PTR), ctypes.cast(md, _PTR)),
               "codebook")
    return list(lv), list(md)


class PackedNF4:
    """A packed NF4 weight held in caller-owned torch device tensors (Wt is o x h)."""

    def __init__(self, out_features: int, in_features: int, device="cuda"):
        if in_features % 64:
            raise ValueError("in_features must be a multiple of 64")
        n = out_features * in_features
        self.out_features = out_features
        self.in_features = in_features
        self.codes = torch.empty(n // 2, dtype=torch.uint8, device=device)
        self.absmax_q8 = torch.empty(n // 64, dtype=torch.uint8, device=device)
        self.absmax_s2 = torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device=device)

    def desc(self) -> NF4WeightDesc:
        return NF4WeightDesc(self.codes.data_ptr(), self.absmax_q8.data_ptr(),
                             self.absmax_s2.data_ptr(), self.out_features, self.in_features)

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + self.absmax_q8.numel() + 4 * self.absmax_s2.numel()


def _require(t: torch.Tensor, dtype, shape, name: str) -> None:
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def nf4_quantize(Wt: torch.Tensor, out: PackedNF4 | None = None, stream=None,
                 codebook_id: int = CODEBOOK_NF4, scale_format: int = SCALES_U8) -> PackedNF4:
    """Quantize an fp32 CUDA weight Wt (o x h) to packed 4-bit codes with double-quantized
    scales (NF4 and unsigned 8-bit scales unless another codebook or scale format is given)."""
    o, h = Wt.shape
    _require(Wt, torch.float32, (o, h), "Wt")
    p = out if out is not None else PackedNF4(o, h, Wt.device)
    d = p.desc()
    if scale_format != SCALES_U8:
        _check(lib().qlora_quantize_format(Wt.data_ptr(), ctypes.byref(d), int(codebook_id),
                                           int(scale_format), _stream(stream)),
               "qlora_quantize_format")
    elif codebook_id == CODEBOOK_NF4:
        _check(lib().nf4_quantize(Wt.data_ptr(), ctypes.byref(d), _stream(stream)), "nf4_quantize")
    else:
        _check(lib().qlora_quantize_codebook(Wt.data_ptr(), ctypes.byref(d), int(codebook_id),
                                             _stream(stream)), "qlora_quantize_codebook")
    return p


def nf4_dequantize(p: PackedNF4, out: torch.Tensor | None = None, stream=None,
                   codebook_id: int = CODEBOOK_NF4, scale_format: int = SCALES_U8) -> torch.Tensor:
    """The bf16 weight Wt' (o x h) reconstructed from a packed weight (with the codebook and
    scale format it was packed with)."""
    if out is None:
        out = torch.empty(p.out_features, p.in_features, dtype=torch.bfloat16,
                          device=p.codes.device)
    _require(out, torch.bfloat16, (p.out_features, p.in_features), "out")
    d = p.desc()
    if scale_format != SCALES_U8:
        _check(lib().qlora_dequantize_format(ctypes.byref(d), int(codebook_id), int(scale_format),
                                             out.data_ptr(), _stream(stream)),
               "qlora_dequantize_format")
    elif codebook_id == CODEBOOK_NF4:
        _check(lib().nf4_dequantize(ctypes.byref(d), out.data_ptr(), _stream(stream)),
               "nf4_dequantize")
    else:
        _check(lib().qlora_dequantize_codebook(ctypes.byref(d), int(codebook_id), out.data_ptr(),
                                               _stream(stream)), "qlora_dequantize_codebook")
    return out


_ws_cache: dict = {}


def workspace(nbytes: int, device) -> torch.Tensor:
    """A cached caller-owned scratch buffer of at least nbytes on `device`."""
    key = (str(device), threading.get_ident())
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def fwd_workspace_bytes(t: int, h: int, o: int, r: int) -> int:
    return int(lib().qlora_fwd_workspace_bytes(t, h, o, r))


def bwd_workspace_bytes(t: int, h: int, o: int, r: int) -> int:
    return int(lib().qlora_bwd_workspace_bytes(t, h, o, r))


def qlora_linear_fwd(X: torch.Tensor, p: PackedNF4, L1: torch.Tensor, L2: torch.Tensor, s: float,
                     Y: torch.Tensor | None = None, sT: torch.Tensor | None = None,
                     want_sT: bool = True, ws: torch.Tensor | None = None, stream=None):
    """Y = X.W' + s.X.L1.L2. Returns (Y t x o bf16, sT t x r bf16 or None)."""
    t, h = X.shape
    o, r = p.out_features, L1.shape[1]
    _require(X, torch.bfloat16, (t, h), "X")
    _require(L1, torch.bfloat16, (h, r), "L1")
    _require(L2, torch.bfloat16, (r, o), "L2")
    if h != p.in_features:
        raise ValueError("X and W disagree on in_features")
    if Y is None:
        Y = torch.empty(t, o, dtype=torch.bfloat16, device=X.device)
    if sT is None and want_sT:
        sT = torch.empty(t, r, dtype=torch.bfloat16, device=X.device)
    need = fwd_workspace_bytes(t, h, o, r)
    if ws is None:
        ws = workspace(need, X.device)
    d = p.desc()
    rc = lib().qlora_linear_fwd(X.data_ptr(), t, ctypes.byref(d), L1.data_ptr(), L2.data_ptr(), r,
                                float(s), Y.data_ptr(), _ptr(sT), ws.data_ptr(), ws.numel(),
                                _stream(stream))
    _check(rc, "qlora_linear_fwd")
    return Y, sT


def qlora_linear_bwd(dY: torch.Tensor, X: torch.Tensor, p: PackedNF4, L1: torch.Tensor,
                     L2: torch.Tensor, s: float, sT: torch.Tensor | None = None,
                     dX: torch.Tensor | None = None, dL1: torch.Tensor | None = None,
                     dL2: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                     stream=None):
    """Returns (dX t x h bf16, dL1 h x r fp32, dL2 r x o fp32); W gets no gradient."""
    t, h = X.shape
    o, r = p.out_features, L1.shape[1]
    _require(dY, torch.bfloat16, (t, o), "dY")
    _require(X, torch.bfloat16, (t, h), "X")
    _require(L1, torch.bfloat16, (h, r), "L1")
    _require(L2, torch.bfloat16, (r, o), "L2")
    if sT is not None:
        _require(sT, torch.bfloat16, (t, r), "sT")
    dev = X.device
    dX = torch.empty(t, h, dtype=torch.bfloat16, device=dev) if dX is None else dX
    dL1 = torch.empty(h, r, dtype=torch.float32, device=dev) if dL1 is None else dL1
    dL2 = torch.empty(r, o, dtype=torch.float32, device=dev) if dL2 is None else dL2
    need = bwd_workspace_bytes(t, h, o, r)
    if ws is None:
        ws = workspace(need, dev)
    d = p.desc()
    rc = lib().qlora_linear_bwd(dY.data_ptr(), X.data_ptr(), t, ctypes.byref(d), L1.data_ptr(),
                                L2.data_ptr(), r, float(s), _ptr(sT), dX.data_ptr(),
                                dL1.data_ptr(), dL2.data_ptr(), ws.data_ptr(), ws.numel(),
                                _stream(stream))
    _check(rc, "qlora_linear_bwd")
    return dX, dL1, dL2


def _dropout_args(dropout_p: float, seed: int):
    p32 = float(dropout_p)
    if not (0.0 <= p32 < 1.0):
        raise ValueError("dropout probability must lie in [0, 1)")
    return ctypes.c_float(p32), ctypes.c_uint64(int(seed) & 0xFFFFFFFFFFFFFFFF)


def qlora_dropout_apply(X: torch.Tensor, dropout_p: float, seed: int,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """X (.) M for the LoRA-dropout keep mask M of (dropout_p, seed); dropped elements are +0."""
    t, h = X.shape
    _require(X, torch.bfloat16, (t, h), "X")
    out = torch.empty_like(X) if out is None else out
    _require(out, torch.bfloat16, (t, h), "out")
    pf, sd = _dropout_args(dropout_p, seed)
    _check(lib().qlora_dropout_apply(X.data_ptr(), t, h, pf, sd, out.data_ptr(), _stream(stream)),
           "qlora_dropout_apply")
    return out


def dropout_mask_bytes(t: int, h: int) -> int:
    """Bytes of a keep mask stored as bits (bit e mod 8 of byte e / 8)."""
    return t * h // 8


def qlora_linear_fwd_dropout(X: torch.Tensor, p: PackedNF4, L1: torch.Tensor, L2: torch.Tensor,
                             s: float, dropout_p: float, seed: int, Y: torch.Tensor | None = None,
                             sT: torch.Tensor | None = None, want_sT: bool = True,
                             mask: torch.Tensor | None = None, want_mask: bool = False,
                             ws: torch.Tensor | None = None, stream=None):
    """Y = X.W' + s.((X (.) M / (1 - p)).L1).L2 with the keep mask M of (dropout_p, seed).
    Returns (Y, sT or None, mask bits or None); pass the mask to the backward to spare it the
    generator calls."""
    t, h = X.shape
    o, r = p.out_features, L1.shape[1]
    _require(X, torch.bfloat16, (t, h), "X")
    _require(L1, torch.bfloat16, (h, r), "L1")
    _require(L2, torch.bfloat16, (r, o), "L2")
    if h != p.in_features:
        raise ValueError("X and W disagree on in_features")
    Y = torch.empty(t, o, dtype=torch.bfloat16, device=X.device) if Y is None else Y
    if sT is None and want_sT:
        sT = torch.empty(t, r, dtype=torch.bfloat16, device=X.device)
    if mask is None and want_mask:
        mask = torch.empty(dropout_mask_bytes(t, h), dtype=torch.uint8, device=X.device)
    if mask is not None:
        _require(mask, torch.uint8, (dropout_mask_bytes(t, h),), "mask")
    if ws is None:
        ws = workspace(int(lib().qlora_fwd_dropout_workspace_bytes(t, h, o, r)), X.device)
    pf, sd = _dropout_args(dropout_p, seed)
    d = p.desc()
    rc = lib().qlora_linear_fwd_dropout(X.data_ptr(), t, ctypes.byref(d), L1.data_ptr(),
                                        L2.data_ptr(), r, float(s), pf, sd, Y.data_ptr(), _ptr(sT),
                                        _ptr(mask), ws.data_ptr(), ws.numel(), _stream(stream))
    _check(rc, "qlora_linear_fwd_dropout")
    return Y, sT, mask


def qlora_linear_bwd_dropout(dY: torch.Tensor, X: torch.Tensor, p: PackedNF4, L1: torch.Tensor,
                             L2: torch.Tensor, s: float, dropout_p: float, seed: int,
                             sT: torch.Tensor | None = None, mask: torch.Tensor | None = None,
                             dX: torch.Tensor | None = None,
                             dL1: torch.Tensor | None = None, dL2: torch.Tensor | None = None,
                             ws: torch.Tensor | None = None, stream=None):
    """Gradients for qlora_linear_fwd_dropout with the same (dropout_p, seed) (and, optionally,
    the forward's mask bits)."""
    t, h = X.shape
    o, r = p.out_features, L1.shape[1]
    _require(dY, torch.bfloat16, (t, o), "dY")
    _require(X, torch.bfloat16, (t, h), "X")
    _require(L1, torch.bfloat16, (h, r), "L1")
    _require(L2, torch.bfloat16, (r, o), "L2")
    if sT is not None:
        _require(sT, torch.bfloat16, (t, r), "sT")
    if mask is not None:
        _require(mask, torch.uint8, (dropout_mask_bytes(t, h),), "mask")
    dev = X.device
    dX = torch.empty(t, h, dtype=torch.bfloat16, device=dev) if dX is None else dX
    dL1 = torch.empty(h, r, dtype=torch.float32, device=dev) if dL1 is None else dL1
    dL2 = torch.empty(r, o, dtype=torch.float32, device=dev) if dL2 is None else dL2
    if ws is None:
        ws = workspace(int(lib().qlora_bwd_dropout_workspace_bytes(t, h, o, r)), dev)
    pf, sd = _dropout_args(dropout_p, seed)
    d = p.desc()
    rc = lib().qlora_linear_bwd_dropout(dY.data_ptr(), X.data_ptr(), t, ctypes.byref(d),
                                        L1.data_ptr(), L2.data_ptr(), r, float(s), pf, sd, _ptr(sT),
                                        _ptr(mask), dX.data_ptr(), dL1.data_ptr(), dL2.data_ptr(),
                                        ws.data_ptr(), ws.numel(), _stream(stream))
    _check(rc, "qlora_linear_bwd_dropout")
    return dX, dL1, dL2


class KernelProfile:
    """Per-kernel device time and launch counts, from CUDA events the library records around
    each of its launches while the profile is open (``with KernelProfile() as p: ...``)."""

    def __init__(self, capacity: int = 65536):
        self.capacity = capacity
        self.ms = {}
        self.launches = {}
        self.recorded = 0

    def __enter__(self):
        _check(lib().qlora_profile_begin(self.capacity), "qlora_profile_begin")
        return self

    def __exit__(self, *exc):
        ms = (ctypes.c_double * KERNEL_KINDS)()
        n = (ctypes.c_int64 * KERNEL_KINDS)()
        rc = lib().qlora_profile_end(ctypes.cast(ms, _PTR), ctypes.cast(n, _PTR), KERNEL_KINDS)
        if rc < 0:
            raise RuntimeError(f"qlora_profile_end: {status_string(rc)}")
        self.recorded = rc
        for k in range(KERNEL_KINDS):
            name = lib().qlora_kernel_name(k).decode()
            self.ms[name] = ms[k]
            self.launches[name] = n[k]
        return False


def merge_adapters(p: PackedNF4, L1: torch.Tensor, L2: torch.Tensor, s: float,
                   out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Wt_merged (o x h fp32) = W'^T + s.(L1.L2)^T: the adapters merged into the dequantized
    base (re-quantize it with nf4_quantize for a merged packed weight)."""
    o, h, r = p.out_features, p.in_features, L1.shape[1]
    _require(L1, torch.bfloat16, (h, r), "L1")
    _require(L2, torch.bfloat16, (r, o), "L2")
    if out is None:
        out = torch.empty(o, h, dtype=torch.float32, device=L1.device)
    _require(out, torch.float32, (o, h), "out")
    d = p.desc()
    _check(lib().qlora_merge_adapters(ctypes.byref(d), L1.data_ptr(), L2.data_ptr(), r,
                                      float(s), out.data_ptr(), _stream(stream)),
           "qlora_merge_adapters")
    return out


ADAMW_PREFETCH = 1


def adamw_step_ptr(p: int, p16: int, g: int, m: int, v: int, n: int, lr: float, beta1: float,
                   beta2: float, eps: float, weight_decay: float, step: int, flags: int = 0,
                   stream=None) -> None:
    """qlora_adamw_step on raw device (or unified-memory) pointers."""
    _check(lib().qlora_adamw_step(p, p16, g, m, v, int(n), float(lr), float(beta1), float(beta2),
                                  float(eps), float(weight_decay), int(step), int(flags),
                                  _stream(stream)),
           "qlora_adamw_step")


def adamw_step(p: torch.Tensor, g: torch.Tensor, m: torch.Tensor, v: torch.Tensor, step: int,
               lr: float = 1e-4, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
               weight_decay: float = 0.0, p16: torch.Tensor | None = None, stream=None) -> None:
    """One fused AdamW step on fp32 CUDA tensors of equal shape (in place); p16, if given, gets
    the bf16 copy of the updated parameters."""
    for t, name in ((p, "p"), (g, "g"), (m, "m"), (v, "v")):
        _require(t, torch.float32, p.shape, name)
    if p16 is not None:
        _require(p16, torch.bfloat16, p.shape, "p16")
    adamw_step_ptr(p.data_ptr(), p16.data_ptr() if p16 is not None else 0, g.data_ptr(),
                   m.data_ptr(), v.data_ptr(), p.numel(), lr, beta1, beta2, eps, weight_decay,
                   step, 0, stream)


ADAMW_MAX_TENSORS = 64


def adamw_step_multi_ptr(params, params_bf16, grads, m, v, counts, lr: float, beta1: float,
                         beta2: float, eps: float, weight_decay: float, step: int, flags: int = 0,
                         stream=None) -> None:
    """qlora_adamw_step_multi on lists of raw device pointers (params_bf16 may be None, or hold
    0 for tensors without a bf16 copy) and parameter counts."""
    n = len(params)
    if not (len(grads) == len(m) == len(v) == len(counts) == n) or (
            params_bf16 is not None and len(params_bf16) != n):
        raise ValueError("adamw_step_multi: pointer lists of different lengths")
    P = ctypes.c_void_p * max(n, 1)
    p16 = P(*params_bf16) if params_bf16 is not None else None
    _check(lib().qlora_adamw_step_multi(
        n, P(*params), p16, P(*grads), P(*m), P(*v), (ctypes.c_int64 * max(n, 1))(*counts),
        float(lr), float(beta1), float(beta2), float(eps), float(weight_decay), int(step),
        int(flags), _stream(stream)), "qlora_adamw_step_multi")


def adamw_step_multi(params, grads, ms, vs, step: int, lr: float = 1e-4, beta1: float = 0.9,
                     beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
                     params_bf16=None, stream=None) -> None:
    """One fused AdamW step over several fp32 CUDA tensors in one launch (in place); each
    tensor's grad and moments match its shape; params_bf16, if given, is a list holding a bf16
    tensor (or None) per parameter tensor."""
    for p, g, m, v in zip(params, grads, ms, vs, strict=True):
        for t, name in ((p, "p"), (g, "g"), (m, "m"), (v, "v")):
            _require(t, torch.float32, p.shape, name)
    ptr16 = None
    if params_bf16 is not None:
        ptr16 = []
        for p, q in zip(params, params_bf16, strict=True):
            if q is not None:
                _require(q, torch.bfloat16, p.shape, "p16")
            ptr16.append(q.data_ptr() if q is not None else 0)
    adamw_step_multi_ptr([p.data_ptr() for p in params], ptr16, [g.data_ptr() for g in grads],
                         [m.data_ptr() for m in ms], [v.data_ptr() for v in vs],
                         [p.numel() for p in params], lr, beta1, beta2, eps, weight_decay, step, 0,
                         stream)


def selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Launch the bounded-wait self-test (a wait nothing completes, given up after limit_ns)."""
    _check(lib().qlora_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "qlora_selftest_wait_timeout")


def set_gemv_max_ctas(n: int) -> int:
    """Cap the decode GEMV's CTA count (n <= 0: one per SM); returns the previous cap."""
    return int(lib().qlora_set_gemv_max_ctas(int(n)))


def last_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(lib().qlora_get_last_status(_stream(stream)))
