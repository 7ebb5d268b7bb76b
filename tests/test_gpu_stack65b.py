"""The 65B-shaped stack at full size (80 layers x 7 linears, 33.4 GB packed, t = 2048, r = 64),
one forward+backward step exactly as the bench runs it, checked against the oracle on three
linears: layer 0 q_proj (8192 x 8192), layer 40 up_proj (h 8192 -> o 22016) and layer 79
down_proj (h 22016 -> o 8192).

Per checked linear: sT, dL1 and dL2 in full (they do not involve W); seeded samples of Y
(tokens x output columns, from the oracle's own dequantization of the scale groups covering
those rows of Wt, regenerated from the same device seed); and dX as seeded full rows against
the oracle's dequantization of the whole weight (8192 x 8192 for q_proj, 22016 x 8192 and
8192 x 22016 for up_proj and down_proj: about 180 M weights each)."""

import numpy as np
import pytest
import torch

from bit_quantized_lora_03_b200 import binding as B
from bit_quantized_lora_03_b200 import inputs
from oracle import nf4_oracle as O

from gpu_util import assert_close_rms, f32, require_gpu

pytestmark = pytest.mark.gpu

CHECKED = {(0, 0): "full_dx", (40, 5): "full_dx", (79, 6): "full_dx"}


@pytest.fixture(scope="module")
def stack_step():
    require_gpu()
    if torch.cuda.get_device_properties(0).total_memory < 60 * 2**30:
        pytest.skip("needs ~40 GB of device memory")
    from bit_quantized_lora_03_b200.stack65b import Stack65B
    st = Stack65B(torch.device("cuda"))
    kept = st.step(keep=set(CHECKED))
    torch.cuda.synchronize()
    assert B.last_status() == 0
    out = {"X": {k: f32(v) for k, v in st.X.items()}, "dY": {k: f32(v) for k, v in st.dY.items()},
           "s": st.s, "t": st.t, "packed": st.packed_bytes}
    for (layer, i) in CHECKED:
        _, _, h, o, p, L1, L2, sT, dL1, dL2 = st.linear(layer, i)
        out[(layer, i)] = {"h": h, "o": o, "L1": f32(L1), "L2": f32(L2), "sT": f32(sT),
                           "dL1": f32(dL1), "dL2": f32(dL2),
                           "Y": f32(kept[(layer, i, "Y")]), "dX": f32(kept[(layer, i, "dX")])}
    del st, kept
    torch.cuda.empty_cache()
    return out


def test_stack65b_size(stack_step):
    n = inputs.STACK65B_LAYERS * sum(h * o for _, h, o in inputs.LLAMA65B_LINEARS)
    assert n == 64_760_053_760
    assert stack_step["packed"] == sum(
        O.packed_bytes(h * o) for _, h, o in inputs.LLAMA65B_LINEARS) * inputs.STACK65B_LAYERS


@pytest.mark.parametrize("key", sorted(CHECKED))
def test_stack65b_linear(stack_step, key):
    d = stack_step[key]
    h, o, s = d["h"], d["o"], stack_step["s"]
    X, dY = stack_step["X"][h], stack_step["dY"][o]
    L1, L2 = d["L1"], d["L2"]
    X64, dY64 = X.astype(np.float64), dY.astype(np.float64)
    T = X64 @ L1
    U = dY64 @ L2.T
    assert_close_rms(d["sT"], s * T, "sT")
    assert_close_rms(d["dL1"], s * (X64.T @ U), "dL1")
    assert_close_rms(d["dL2"], s * (T.T @ dY64), "dL2")

    rng = np.random.default_rng(key[0] * 7 + key[1])
    cols = np.unique(np.concatenate([[0, o - 1], rng.choice(o, 62, replace=False)]))
    toks = np.unique(np.concatenate([[0, stack_step["t"] - 1], rng.choice(stack_step["t"], 30, replace=False)]))
    Wt = inputs.stack65b_weight(key[0], key[1], torch.device("cuda"))
    Wt_host = Wt.cpu().numpy()
    del Wt
    torch.cuda.empty_cache()
    Wdq = O.nf4_dequantize(O.nf4_quantize(Wt_host))
    del Wt_host
    Y_ref = X64[toks] @ Wdq[cols].astype(np.float64).T + s * (T[toks] @ L2[:, cols])
    assert_close_rms(d["Y"][np.ix_(toks, cols)], Y_ref, "Y samples")
    assert_close_rms(d["dX"][toks], O.qlora_linear_bwd_dx_rows(toks, dY, Wdq, L1, L2, s), "dX rows")
