"""Helpers shared by the GPU parity tests (not collected as tests)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as O

TOL = 2e-2   # max |gpu - oracle| <= TOL * RMS(oracle), the bound stated for products


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_quantized_lora_03_b200 import build
    build.build()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def assert_close_rms(got, ref, name: str, tol: float = TOL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    mx, rms = O.max_err_vs_rms(got, ref)
    assert mx <= tol * rms, f"{name}: max|err| {mx:.4g} > {tol} * RMS {rms:.4g} ({mx / max(rms, 1e-300):.4g})"
    return mx / max(rms, 1e-300)


def oracle_packed_rows(Wt: np.ndarray, rows) -> np.ndarray:
    """Oracle dequantized rows of a large Wt, quantizing only the scale groups that cover them.

    A row's values depend on its own blocks and on the 8-bit scale groups (256 consecutive
    blocks) those blocks fall in, so the oracle quantizes exactly those groups."""
    o, h = Wt.shape
    nbr = h // 64
    out = []
    flat = Wt.reshape(-1)
    for j in rows:
        b0, b1 = j * nbr, (j + 1) * nbr
        g0, g1 = b0 // 256, (b1 - 1) // 256 + 1
        lo, hi = g0 * 256 * 64, min(g1 * 256 * 64, flat.size)
        chunk = flat[lo:hi].reshape(1, -1)
        p = O.nf4_quantize(chunk)
        deq = O.nf4_dequantize(p).reshape(-1)
        out.append(deq[j * h - lo:(j + 1) * h - lo])
    return np.stack(out)
