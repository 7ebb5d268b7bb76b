"""Pins of the oracle's adapted linear layer (forward and backward) and storage arithmetic.

Products: Y = X.W' + s.X.L1.L2 ("QLoRA: Efficient Finetuning of Quantized LLMs", "The
algebra"; "QLoRA in LLMs" section 3), gradients reach the adapters through the frozen base,
which gets none ("One training step, from input to update"; "QLoRA in LLMs" section 4).
Checked against: explicit loops (special cases s = 0, L2 = 0, W = 0), the adjoint identity,
bilinearity in the adapters, finite differences, and torch.autograd in float64.

Storage: the pages' ledger numbers ("A worked memory budget for 65 billion weights",
"2. Double quantization", "04 Work through an example") and the byte count of the real
packed format.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(t=3, h=64, o=128, r=16, seed=0):
    rng = np.random.default_rng(seed)
    X = O.bf16_round(rng.standard_normal((t, h)).astype(np.float32))
    Wt = O.nf4_dequantize(O.nf4_quantize((rng.standard_normal((o, h)) * 0.02).astype(np.float32)))
    L1 = O.bf16_round((rng.standard_normal((h, r)) * 0.01).astype(np.float32))
    L2 = O.bf16_round((rng.standard_normal((r, o)) * 0.01).astype(np.float32))
    dY = O.bf16_round(rng.standard_normal((t, o)).astype(np.float32))
    return X, Wt, L1, L2, dY


def _loop_matmul(A, B):
    n, k = A.shape
    k2, m = B.shape
    assert k == k2
    out = np.zeros((n, m))
    for i in range(n):
        for j in range(m):
            acc = 0.0
            for p in range(k):
                acc += float(A[i, p]) * float(B[p, j])
            out[i, j] = acc
    return out


def test_shapes():
    X, Wt, L1, L2, dY = _case()
    Y, sT = O.qlora_linear_fwd(X, Wt, L1, L2, 2.0)
    dX, dL1, dL2, sU = O.qlora_linear_bwd(dY, X, Wt, L1, L2, 2.0)
    assert Y.shape == (3, 128) and sT.shape == (3, 16)
    assert dX.shape == (3, 64) and dL1.shape == (64, 16) and dL2.shape == (16, 128)
    assert sU.shape == (3, 16)


def test_special_cases_reduce_to_plain_products():
    X, Wt, L1, L2, _ = _case(t=2, h=64, o=8, r=16, seed=1)
    base = _loop_matmul(X, Wt.T)                       # X . W' with W' = Wt^T (h x o)
    Y0, _ = O.qlora_linear_fwd(X, Wt, L1, L2, 0.0)
    assert np.allclose(Y0, base, rtol=0, atol=1e-12)
    Yz, _ = O.qlora_linear_fwd(X, Wt, L1, np.zeros_like(L2), 3.0)
    assert np.allclose(Yz, base, rtol=0, atol=1e-12)
    Yw, sT = O.qlora_linear_fwd(X, np.zeros_like(Wt), L1, L2, 3.0)
    lora = 3.0 * _loop_matmul(_loop_matmul(X, L1), L2)
    assert np.allclose(Yw, lora, rtol=0, atol=1e-14)
    assert np.allclose(sT, 3.0 * _loop_matmul(X, L1), rtol=0, atol=1e-13)


def test_single_token_is_a_gemv():
    X, Wt, L1, L2, _ = _case(t=1, h=64, o=16, r=16, seed=2)
    Y, _ = O.qlora_linear_fwd(X, Wt, L1, L2, 2.0)
    for j in range(16):
        ref = sum(float(X[0, k]) * float(Wt[j, k]) for k in range(64))
        ref += 2.0 * sum(sum(float(X[0, k]) * float(L1[k, c]) for k in range(64)) * float(L2[c, j])
                         for c in range(16))
        assert abs(Y[0, j] - ref) < 1e-12


def test_adjoint_identity():
    X, Wt, L1, L2, dY = _case(t=5, h=128, o=192, r=32, seed=3)
    s = 0.25
    Y, _ = O.qlora_linear_fwd(X, Wt, L1, L2, s)
    dX, _, _, _ = O.qlora_linear_bwd(dY, X, Wt, L1, L2, s)
    lhs = float(np.sum(dX * X.astype(np.float64)))
    rhs = float(np.sum(dY.astype(np.float64) * Y))
    assert abs(lhs - rhs) <= 1e-10 * (abs(rhs) + 1)


def test_bilinearity_in_the_adapters():
    X, Wt, L1, L2, dY = _case(t=4, h=64, o=128, r=16, seed=4)
    s = 2.0
    _, dL1, dL2, _ = O.qlora_linear_bwd(dY, X, Wt, L1, L2, s)
    lora = s * (X.astype(np.float64) @ L1 @ L2)
    ref = float(np.sum(dY.astype(np.float64) * lora))
    a = float(np.sum(dL1 * L1.astype(np.float64)))
    b = float(np.sum(dL2 * L2.astype(np.float64)))
    assert abs(a - ref) <= 1e-10 * (abs(ref) + 1e-30)
    assert abs(b - ref) <= 1e-10 * (abs(ref) + 1e-30)


def test_finite_differences():
    X, Wt, L1, L2, dY = _case(t=3, h=64, o=64, r=16, seed=5)
    X, L1, L2 = (a.astype(np.float64) for a in (X, L1, L2))
    s = 0.7
    dX, dL1, dL2, _ = O.qlora_linear_bwd(dY, X, Wt, L1, L2, s)

    def loss(X_, L1_, L2_):
        Y, _ = O.qlora_linear_fwd(X_, Wt, L1_, L2_, s)
        return float(np.sum(dY.astype(np.float64) * Y))

    rng = np.random.default_rng(6)
    eps = 1e-6
    for arr, grad, idx in [(X, dX, 0), (L1, dL1, 1), (L2, dL2, 2)]:
        D = rng.standard_normal(arr.shape)
        args_p = [X, L1, L2]
        args_m = [X, L1, L2]
        args_p[idx] = arr + eps * D
        args_m[idx] = arr - eps * D
        fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        an = float(np.sum(grad * D))
        assert abs(fd - an) <= 1e-6 * (abs(an) + 1e-3), (idx, fd, an)


def test_backward_against_torch_autograd_float64():
    X, Wt, L1, L2, dY = _case(t=6, h=128, o=64, r=16, seed=7)
    s = 0.25
    tX = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    tW = torch.tensor(Wt, dtype=torch.float64, requires_grad=False)
    tL1 = torch.tensor(L1, dtype=torch.float64, requires_grad=True)
    tL2 = torch.tensor(L2, dtype=torch.float64, requires_grad=True)
    T = tX @ tL1
    T.retain_grad()
    Y = tX @ tW.T + s * T @ tL2
    Y.backward(torch.tensor(dY, dtype=torch.float64))
    dX, dL1, dL2, sU = O.qlora_linear_bwd(dY, X, Wt, L1, L2, s)
    Yo, sT = O.qlora_linear_fwd(X, Wt, L1, L2, s)
    assert np.allclose(Yo, Y.detach().numpy(), rtol=1e-12, atol=1e-12)
    # the saved rank-r intermediates: sT = s.X.L1 and sU = dY-gradient of T = s.dY.L2^T
    assert np.allclose(sT, s * T.detach().numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(sU, T.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dX, tX.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dL1, tL1.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dL2, tL2.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert tW.grad is None          # the frozen base receives no gradient


def test_row_helpers_match_full_products():
    X, Wt, L1, L2, dY = _case(t=9, h=64, o=128, r=16, seed=8)
    rows = [0, 4, 8]
    Y, _ = O.qlora_linear_fwd(X, Wt, L1, L2, 1.5)
    dX, _, _, _ = O.qlora_linear_bwd(dY, X, Wt, L1, L2, 1.5)
    assert np.array_equal(O.qlora_linear_fwd_rows(rows, X, Wt, L1, L2, 1.5), Y[rows])
    assert np.allclose(O.qlora_linear_bwd_dx_rows(rows, dY, Wt, L1, L2, 1.5), dX[rows],
                       rtol=0, atol=1e-13)


def test_tolerance_helper():
    ref = np.array([3.0, -4.0])
    got = np.array([3.1, -4.0])
    mx, rms = O.max_err_vs_rms(got, ref)
    assert math.isclose(mx, 0.1, rel_tol=1e-12) and math.isclose(rms, math.sqrt(12.5))


def test_lora_parameter_count():
    g = json.load(open(os.path.join(GOLDEN, "lora_param_count.json")))
    adapter = g["h"] * g["r"] + g["r"] * g["o"]
    full = g["h"] * g["o"]
    assert adapter == g["adapter_params"] and full == g["full_params"]
    assert full // adapter == g["ratio"] and full % adapter == 0


def test_storage_ledger():
    g = json.load(open(os.path.join(GOLDEN, "storage_ledger.json")))
    assert g["block_size"]["value"] == O.BLOCK and g["scales_per_second_level_block"]["value"] == O.GROUP
    no_dq = O.scale_bits_per_weight(False)
    dq = O.scale_bits_per_weight(True)
    assert no_dq == g["scale_bits_no_dq"]["value"]
    assert round(dq, 3) == g["scale_bits_dq"]["value"]
    assert round(no_dq - dq, 2) == g["bits_saved"]["value"]
    s7 = g["llama7b"]
    assert O.weight_storage_bytes(s7["params"], 16) / 1e9 == s7["gb_16bit"]
    assert O.weight_storage_bytes(s7["params"], 4) / 1e9 == s7["gb_4bit"]
    assert O.weight_storage_bytes(s7["params"], 32) / 1e9 == s7["gb_fp32"]
    assert O.weight_storage_bytes(s7["params"], 8) / 1e9 == s7["gb_8bit"]
    s65 = g["llama65b"]
    assert O.weight_storage_bytes(s65["params"], 16) / 1e9 == s65["gb_16bit"]
    assert O.weight_storage_bytes(s65["params"], 4) / 1e9 == s65["gb_4bit"]
    assert round(O.weight_storage_bytes(s65["params"], 4 + dq) / 1e9, 1) == s65["gb_4bit_dq"]
    assert round(O.weight_storage_bytes(s65["params"], dq) / 1e9) == s65["gb_dq_scales"]
    assert round(O.weight_storage_bytes(s65["params"], no_dq) / 1e9, 1) == s65["gb_scales_no_dq"]
    assert round(O.weight_storage_bytes(s65["params"], no_dq - dq) / 1e9) == s65["gb_saved"]
    ex = g["ratio_example"]
    for other, ratio in [(ex["other_small_gb"], ex["ratio_small"]),
                         (ex["other_large_gb"], ex["ratio_large"])]:
        r = (s7["gb_16bit"] + other) / (s7["gb_4bit"] + other)
        assert round(r, 3) == ratio
    raw = g["raw_bytes_per_param"]
    assert O.weight_storage_bytes(1, 16) == raw["bits16"] and O.weight_storage_bytes(1, 4) == raw["bits4"]


@pytest.mark.parametrize("o,h", [(1, 64), (3, 128), (64, 4096), (5, 64 * 300)])
def test_packed_format_byte_count(o, h):
    W = (np.random.default_rng(o + h).standard_normal((o, h)) * 0.02).astype(np.float32)
    p = O.nf4_quantize(W)
    n = o * h
    real = p.codes.nbytes + p.absmax_q8.nbytes + p.absmax_s2.nbytes
    assert real == O.packed_bytes(n)
    assert p.codes.size == n // 2 and p.absmax_q8.size == n // 64
    assert p.absmax_s2.size == -(-n // (64 * 256))


def test_packed_bits_per_weight_tends_to_4_127():
    n = 64 * 256 * 1000
    bits = O.packed_bytes(n) * 8 / n
    assert abs(bits - (4 + O.scale_bits_per_weight(True))) < 1e-12
    assert round(bits, 3) == 4.127
