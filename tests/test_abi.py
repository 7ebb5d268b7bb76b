"""The C-ABI library loads without a GPU, exports every function include/qlora_nf4.h declares,
derives the same NF4 codebook as the oracle, and rejects bad arguments on the host before
touching CUDA (these calls never launch anything)."""

import ctypes
import os
import re

import numpy as np
import pytest

from bit_quantized_lora_03_b200 import binding as B
from bit_quantized_lora_03_b200 import build as build_mod
from oracle import nf4_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_header_declares_the_four_calls_and_helpers():
    names = declared_functions()
    for required in ["nf4_quantize", "nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd",
                     "qlora_get_last_status", "qlora_status_string"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) <= set(B.SIGNATURES), "binding signatures must cover the header"


def test_library_links_no_gpu_driver():
    out = os.popen(f"ldd {build_mod.LIB_PATH}").read()
    assert "libcuda.so" not in out and "libcudart.so" not in out


def test_codebook_matches_oracle_bit_exactly(lib):
    lv, md = B.codebook()
    assert np.array_equal(np.array(lv, np.float32), O.nf4_codebook())
    assert np.array_equal(np.array(md, np.float32), O.nf4_midpoints())
    assert lib.qlora_nf4_codebook(None, None) == B.QLORA_ERR_INVALID_ARG


def test_status_strings(lib):
    for code in [0, -1, -2, -3, -4, -5, -6, 1, 2, 3, 12345]:
        s = B.status_string(code)
        assert isinstance(s, str) and s


def test_workspace_sizes(lib):
    # t > 16: a t x r bf16 region per rank-r product (sT; sU and a recomputed sT)
    assert lib.qlora_fwd_workspace_bytes(4096, 4096, 4096, 64) >= 4096 * 64 * 2
    assert lib.qlora_bwd_workspace_bytes(4096, 4096, 4096, 64) >= 2 * 4096 * 64 * 2
    # the decode path also keeps a t x o fp32 accumulator
    assert lib.qlora_fwd_workspace_bytes(16, 4096, 11008, 16) >= 16 * 11008 * 4
    assert lib.qlora_fwd_workspace_bytes(0, 4096, 4096, 64) == 0
    assert lib.qlora_fwd_workspace_bytes(8, 100, 4096, 64) == 0      # h % 64 != 0
    assert lib.qlora_fwd_workspace_bytes(8, 4096, 4096, 24) == 0     # r % 16 != 0
    assert lib.qlora_bwd_workspace_bytes(8, 4096, 4096, 512) == 0    # r > 256


def _desc(codes=0x1000, q8=0x2000, s2=0x3000, o=128, h=128):
    return B.NF4WeightDesc(codes, q8, s2, o, h)


def test_host_validation_rejects_before_launch(lib):
    d = _desc()
    assert lib.nf4_quantize(None, ctypes.byref(d), None) == B.QLORA_ERR_INVALID_ARG
    assert lib.nf4_quantize(0x1000, None, None) == B.QLORA_ERR_INVALID_ARG
    bad_h = _desc(h=100)
    assert lib.nf4_quantize(0x1000, ctypes.byref(bad_h), None) == B.QLORA_ERR_BAD_SHAPE
    zero_o = _desc(o=0)
    assert lib.nf4_quantize(0x1000, ctypes.byref(zero_o), None) == B.QLORA_ERR_BAD_SHAPE
    for mis in (_desc(codes=0x1001), _desc(q8=0x2008), _desc(s2=0x3004)):
        assert lib.nf4_quantize(0x1000, ctypes.byref(mis), None) == B.QLORA_ERR_MISALIGNED
    assert lib.nf4_quantize(0x1004, ctypes.byref(d), None) == B.QLORA_ERR_MISALIGNED
    null_codes = _desc(codes=0)
    assert lib.nf4_dequantize(ctypes.byref(null_codes), 0x1000, None) == B.QLORA_ERR_INVALID_ARG
    assert lib.nf4_dequantize(ctypes.byref(d), None, None) == B.QLORA_ERR_INVALID_ARG
    assert lib.nf4_dequantize(ctypes.byref(d), 0x1008, None) == B.QLORA_ERR_MISALIGNED

    P = 0x10000
    fwd = lib.qlora_linear_fwd
    assert fwd(None, 4, ctypes.byref(d), P, P, 16, 1.0, P, None, P, 1 << 30, None) == B.QLORA_ERR_INVALID_ARG
    assert fwd(P, 0, ctypes.byref(d), P, P, 16, 1.0, P, None, P, 1 << 30, None) == B.QLORA_ERR_INVALID_ARG
    assert fwd(P, 4, ctypes.byref(d), P, P, 24, 1.0, P, None, P, 1 << 30, None) == B.QLORA_ERR_INVALID_ARG
    assert fwd(P, 4, ctypes.byref(d), P, P, 16, float("nan"), P, None, P, 1 << 30, None) == B.QLORA_ERR_INVALID_ARG
    d_o = _desc(o=100)
    assert fwd(P, 4, ctypes.byref(d_o), P, P, 16, 1.0, P, None, P, 1 << 30, None) == B.QLORA_ERR_BAD_SHAPE
    assert fwd(P + 2, 4, ctypes.byref(d), P, P, 16, 1.0, P, None, P, 1 << 30, None) == B.QLORA_ERR_MISALIGNED
    assert fwd(P, 4, ctypes.byref(d), P, P, 16, 1.0, P, None, None, 0, None) == B.QLORA_ERR_WORKSPACE
    assert fwd(P, 4, ctypes.byref(d), P, P, 16, 1.0, P, None, P, 16, None) == B.QLORA_ERR_WORKSPACE

    bwd = lib.qlora_linear_bwd
    assert bwd(P, P, 4, ctypes.byref(d), P, P, 16, 1.0, None, P, P, None, P, 1 << 30, None) == B.QLORA_ERR_INVALID_ARG
    assert bwd(P, P, 4, ctypes.byref(d), P, P, 16, 1.0, None, P, P, P + 4, P, 1 << 30, None) == B.QLORA_ERR_MISALIGNED
    assert bwd(P, P, 4, ctypes.byref(d), P, P, 16, 1.0, None, P, P, P, P, 8, None) == B.QLORA_ERR_WORKSPACE


@pytest.mark.parametrize("cb", [0, 1, 2])
def test_codebooks_match_oracle_bit_exactly(lib, cb):
    lv, md = B.codebook(cb)
    want = O.codebook_levels(cb)
    assert np.array_equal(np.array(lv, np.float32).view(np.uint32), want.view(np.uint32))
    assert np.array_equal(np.array(md, np.float32).view(np.uint32), O.nf4_midpoints(want).view(np.uint32))


def test_unknown_codebook_is_rejected(lib):
    lv = (ctypes.c_float * 16)()
    assert lib.qlora_codebook(3, ctypes.cast(lv, ctypes.c_void_p), None) == B.QLORA_ERR_INVALID_ARG
    assert lib.qlora_codebook(-1, ctypes.cast(lv, ctypes.c_void_p), None) == B.QLORA_ERR_INVALID_ARG


def test_scale_format_argument_checks(lib):
    d = _desc()
    q = ctypes.byref(d)
    P = 0x10000
    for fmt in (-1, 3, 99):
        assert lib.qlora_quantize_format(P, q, 0, fmt, None) == B.QLORA_ERR_INVALID_ARG
        assert lib.qlora_dequantize_format(q, 0, fmt, P, None) == B.QLORA_ERR_INVALID_ARG
    assert lib.qlora_quantize_format(P, q, 3, B.SCALES_S8, None) == B.QLORA_ERR_INVALID_ARG
    assert lib.qlora_quantize_format(None, q, 0, B.SCALES_E4M3, None) == B.QLORA_ERR_INVALID_ARG
    assert lib.qlora_quantize_format(P + 4, q, 0, B.SCALES_E4M3, None) == B.QLORA_ERR_MISALIGNED
    assert lib.qlora_dequantize_format(q, 0, B.SCALES_S8, P + 2, None) == B.QLORA_ERR_MISALIGNED
    bad_h = _desc(h=100)
    assert lib.qlora_dequantize_format(ctypes.byref(bad_h), 0, B.SCALES_S8, P, None) == B.QLORA_ERR_BAD_SHAPE


def test_adamw_argument_checks(lib):
    f = lib.qlora_adamw_step
    p = ctypes.c_void_p(16)   # never dereferenced: the checks run before anything else
    ok = dict(lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0)

    def call(n=64, step=1, lr=ok["lr"], b1=ok["b1"], b2=ok["b2"], eps=ok["eps"], ptr=p):
        return f(ptr, None, ptr, ptr, ptr, n, lr, b1, b2, eps, ok["wd"], step, 0, None)
    assert call(n=6) == B.QLORA_ERR_INVALID_ARG          # n % 4 != 0
    assert call(step=0) == B.QLORA_ERR_INVALID_ARG
    assert call(eps=0.0) == B.QLORA_ERR_INVALID_ARG
    assert call(b1=1.0) == B.QLORA_ERR_INVALID_ARG
    assert call(lr=float("nan")) == B.QLORA_ERR_INVALID_ARG
    assert call(ptr=None) == B.QLORA_ERR_INVALID_ARG
    assert call(ptr=ctypes.c_void_p(20)) == B.QLORA_ERR_MISALIGNED


def test_adamw_multi_argument_checks(lib):
    f = lib.qlora_adamw_step_multi
    P = ctypes.c_void_p * 2
    good = P(16, 32)
    counts = (ctypes.c_int64 * 2)(64, 128)

    def call(n=2, params=good, grads=good, cnt=counts, step=1, eps=1e-8):
        return f(n, params, None, grads, good, good, cnt, 1e-3, 0.9, 0.999, eps, 0.0, step, 0, None)
    assert call(n=0) == B.QLORA_ERR_INVALID_ARG
    assert call(n=65) == B.QLORA_ERR_INVALID_ARG
    assert call(params=None) == B.QLORA_ERR_INVALID_ARG
    assert call(step=0) == B.QLORA_ERR_INVALID_ARG
    assert call(eps=0.0) == B.QLORA_ERR_INVALID_ARG
    assert call(grads=P(16, 0)) == B.QLORA_ERR_INVALID_ARG                  # a null entry
    assert call(cnt=(ctypes.c_int64 * 2)(64, 6)) == B.QLORA_ERR_INVALID_ARG  # count % 4 != 0
    assert call(cnt=(ctypes.c_int64 * 2)(64, 0)) == B.QLORA_ERR_INVALID_ARG
    assert call(params=P(16, 36)) == B.QLORA_ERR_MISALIGNED


def test_dropout_workspace_and_argument_checks(lib):
    # the dropout calls hold X (.) M (t x h bf16), and the backward also the mask as bits,
    # in front of the plain workspace
    for t, h, o, r in ((4096, 4096, 11008, 64), (5, 320, 576, 16), (300, 640, 320, 48)):
        xd = (t * h * 2 + 255) // 256 * 256
        assert lib.qlora_fwd_dropout_workspace_bytes(t, h, o, r) == xd + lib.qlora_fwd_workspace_bytes(t, h, o, r)
        bits = (t * h // 8 + 255) // 256 * 256
        assert lib.qlora_bwd_dropout_workspace_bytes(t, h, o, r) == xd + bits + lib.qlora_bwd_workspace_bytes(t, h, o, r)
    assert lib.qlora_fwd_dropout_workspace_bytes(8, 100, 4096, 64) == 0
    assert lib.qlora_bwd_dropout_workspace_bytes(8, 4096, 4096, 512) == 0

    d = _desc()
    P = 0x10000
    big = 1 << 30
    fwd = lib.qlora_linear_fwd_dropout
    for p in (-0.1, 1.0, 2.0, float("nan"), float("inf")):
        assert fwd(P, 4, ctypes.byref(d), P, P, 16, 1.0, p, 1, P, None, None, P, big, None) == B.QLORA_ERR_INVALID_ARG
    # s / (1 - p) must stay finite
    assert fwd(P, 4, ctypes.byref(d), P, P, 16, 3e38, 0.5, 1, P, None, None, P, big, None) == B.QLORA_ERR_INVALID_ARG
    assert fwd(P, 4, ctypes.byref(d), P, P, 16, 1.0, 0.1, 1, P, None, None, P, 1024, None) == B.QLORA_ERR_WORKSPACE
    assert fwd(P + 2, 4, ctypes.byref(d), P, P, 16, 1.0, 0.1, 1, P, None, None, P, big, None) == B.QLORA_ERR_MISALIGNED
    bwd = lib.qlora_linear_bwd_dropout
    assert bwd(P, P, 4, ctypes.byref(d), P, P, 16, 1.0, 1.0, 1, None, None, P, P, P, P, big, None) == B.QLORA_ERR_INVALID_ARG
    assert bwd(P, P, 4, ctypes.byref(d), P, P, 16, 1.0, 0.1, 1, None, None, P, P, None, P, big, None) == B.QLORA_ERR_INVALID_ARG
    assert bwd(P, P, 4, ctypes.byref(d), P, P, 16, 1.0, 0.1, 1, None, None, P, P, P, P, 8, None) == B.QLORA_ERR_WORKSPACE
    # a mask buffer must be 16-byte aligned
    assert fwd(P, 4, ctypes.byref(d), P, P, 16, 1.0, 0.1, 1, P, None, P + 4, P, big, None) == B.QLORA_ERR_MISALIGNED
    assert bwd(P, P, 4, ctypes.byref(d), P, P, 16, 1.0, 0.1, 1, None, P + 4, P, P, P, P, big, None) == B.QLORA_ERR_MISALIGNED
    app = lib.qlora_dropout_apply
    assert app(None, 4, 128, 0.1, 1, P, None) == B.QLORA_ERR_INVALID_ARG
    assert app(P, 4, 128, 1.0, 1, P, None) == B.QLORA_ERR_INVALID_ARG
    assert app(P, 4, 100, 0.1, 1, P, None) == B.QLORA_ERR_BAD_SHAPE
    assert app(P, 0, 128, 0.1, 1, P, None) == B.QLORA_ERR_BAD_SHAPE
    assert app(P, 4, 128, 0.1, 1, P + 8, None) == B.QLORA_ERR_MISALIGNED
    assert app(P, 4, 128, 0.1, 1, P + 16, None) == B.QLORA_ERR_INVALID_ARG   # partial overlap
    with pytest.raises(ValueError):
        B._dropout_args(1.0, 0)


def test_noalloc_forward_rejects_oversized_shapes_on_the_host(lib):
    """The allocation-free forward refuses, before any CUDA call, a shape whose workspace
    would not fit its fixed scratch array, and leaves invalid shapes to the forward's own
    checks (these arguments are never dereferenced)."""
    P = 0x10000
    big = _desc(o=1024, h=1024)
    t, r = 32768, 256                    # sT alone is 32768 x 256 bf16 = 16 MiB
    assert lib.qlora_fwd_workspace_bytes(t, 1024, 1024, r) > B.QLORA_STATIC_SCRATCH_BYTES
    f = lib.qlora_linear_fwd_noalloc
    assert f(P, t, ctypes.byref(big), P, P, r, 1.0, P, None, None) == B.QLORA_ERR_SCRATCH_LIMIT
    assert f(P, 4, None, P, P, 16, 1.0, P, None, None) == B.QLORA_ERR_INVALID_ARG
    assert f(P, 4, ctypes.byref(_desc(h=100)), P, P, 16, 1.0, P, None, None) == B.QLORA_ERR_BAD_SHAPE


def test_binding_fails_loudly_without_the_library(monkeypatch):
    """No CPU or library fallback: with the library missing every call raises, and a host
    tensor is refused rather than computed on the CPU."""
    import torch
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "library_path", lambda: os.path.join(ROOT, "no-such-dir", "lib.so"))
    with pytest.raises(RuntimeError, match="missing"):
        B.lib()
    with pytest.raises((RuntimeError, ValueError)):
        B.nf4_quantize(torch.zeros(4, 64))
    with pytest.raises((RuntimeError, ValueError)):
        B.nf4_dequantize(B.PackedNF4(4, 64, "cpu"))
