"""GPU parity of qlora_merge_adapters against the oracle ("QLoRA in LLMs" §11): the merged
weight W' + s.L1.L2 (stored orientation, fp32) element by element within the stated fp32
bound, including N tiles with a ragged last tile, every rank class and a zero adapter (then
exactly W'); and the merged weight, re-quantized, used as a plain NF4 linear."""

import numpy as np
import pytest
import torch

from bit_quantized_lora_03_b200 import binding as B
from bit_quantized_lora_03_b200 import inputs
from oracle import nf4_oracle as O

from gpu_util import assert_close_rms, f32, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _merge_case(o, h, r, s, seed):
    li = inputs.random_linear(8, h, o, r, s, seed=seed, with_grad=False)
    p = B.nf4_quantize(li.Wt.cuda())
    Wm = B.merge_adapters(p, li.L1.cuda(), li.L2.cuda(), s)
    assert B.last_status() == 0
    Wdq = O.nf4_dequantize(O.nf4_quantize(li.Wt.numpy()))
    ref = O.merge_adapters(Wdq, f32(li.L1), f32(li.L2), s)
    bound = O.merge_error_bound(Wdq, f32(li.L1), f32(li.L2), s)
    return li, p, Wm, Wdq, ref, bound


@pytest.mark.parametrize("o,h,r,s", [
    (64, 64, 16, 2.0),          # one tile, smallest shapes
    (320, 576, 48, 0.5),        # ragged M tile (320 = 2.5 x 128) and N tile (576 = 2 x 256 + 64)
    (640, 1024, 64, 0.25),      # several tiles each way
    (192, 256, 256, 1.0),       # the largest rank (four K-steps)
])
def test_merge_matches_oracle(o, h, r, s):
    li, p, Wm, Wdq, ref, bound = _merge_case(o, h, r, s, seed=o + h + r)
    got = f32(Wm).astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"max excess {np.max(err - bound):.3g}"


def test_zero_adapter_merges_to_the_dequantized_weight():
    li = inputs.random_linear(8, 320, 192, 16, 1.0, seed=9, with_grad=False)
    p = B.nf4_quantize(li.Wt.cuda())
    Wm = B.merge_adapters(p, torch.zeros_like(li.L1).cuda(), li.L2.cuda(), 1.0)
    deq = B.nf4_dequantize(p).float()
    assert torch.equal(Wm, deq)


def test_requantized_merge_as_a_plain_linear():
    """Merged then re-quantized, the weight is an ordinary NF4 linear (s = 0): its output is
    the oracle's product with the oracle's own quantization of the GPU's merged weight, and it
    stays close to the unmerged layer (the drift the pages warn about is one more round of
    4-bit quantization error)."""
    li, p, Wm, Wdq, ref, bound = _merge_case(320, 576, 32, 1.0, seed=21)
    pm = B.nf4_quantize(Wm)
    X = li.X.cuda()
    L1z = torch.zeros_like(li.L1).cuda()
    L2z = torch.zeros_like(li.L2).cuda()
    Ym, _ = B.qlora_linear_fwd(X, pm, L1z, L2z, 0.0)
    assert B.last_status() == 0
    Wm_dq = O.nf4_dequantize(O.nf4_quantize(f32(Wm)))
    Ym_ref, _ = O.qlora_linear_fwd(f32(li.X), Wm_dq, f32(L1z), f32(L2z), 0.0)
    assert_close_rms(f32(Ym), Ym_ref, "merged, re-quantized Y")
    Yu, _ = O.qlora_linear_fwd(f32(li.X), Wdq, f32(li.L1), f32(li.L2), li.s)
    drift = np.sqrt(np.mean((Ym_ref - Yu) ** 2)) / np.sqrt(np.mean(Yu ** 2))
    assert 0.0 < drift < 0.25, drift
