"""Every output and the workspace of the C-ABI calls sit between guard bytes: 4 KB on each side
filled with 0xA5 before the call. After the call the guards must be unchanged (no kernel
writes outside the buffers it was given) and the outputs must still match the oracle.

This stands in for a memory checker on ragged shapes, where tile edges, partial scale groups
and split-K reductions are most likely to overrun: a partial last scale group in the
quantizer, the decode GEMV (t <= 16, its sums and counters in the workspace) and the tcgen05
path (t > 16, ragged in t, o and r)."""

import numpy as np
import pytest
import torch

from bit_quantized_lora_03_b200 import binding as B
from bit_quantized_lora_03_b200 import inputs
from oracle import nf4_oracle as O

from gpu_util import assert_close_rms, f32, require_gpu

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side; a multiple of 256 keeps every view 16-byte aligned
FILL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


class Guarded:
    """A device tensor of `shape` and `dtype` inside a larger buffer whose guard bytes on
    both sides hold FILL."""

    def __init__(self, shape, dtype):
        el = torch.tensor([], dtype=dtype).element_size()
        n = int(np.prod(shape))
        self.nbytes = n * el
        self.raw = torch.full((GUARD + self.nbytes + GUARD,), FILL, dtype=torch.uint8,
                              device="cuda")
        self.t = self.raw[GUARD:GUARD + self.nbytes].view(dtype).view(shape)

    def check(self, name):
        torch.cuda.synchronize()
        head = self.raw[:GUARD].cpu().numpy()
        tail = self.raw[GUARD + self.nbytes:].cpu().numpy()
        assert np.all(head == FILL), f"{name}: bytes written before the buffer"
        assert np.all(tail == FILL), f"{name}: bytes written after the buffer"


def _guarded_pack(o, h):
    p = B.PackedNF4(o, h, "cuda")
    g = {"codes": Guarded(p.codes.shape, torch.uint8),
         "q8": Guarded(p.absmax_q8.shape, torch.uint8),
         "s2": Guarded(p.absmax_s2.shape, torch.float32)}
    p.codes, p.absmax_q8, p.absmax_s2 = g["codes"].t, g["q8"].t, g["s2"].t
    return p, g


@pytest.mark.parametrize("o,h", [(257, 192), (5, 64 * 300)])
def test_quantize_and_dequantize_stay_inside_their_buffers(o, h):
    W = inputs.weight_f32(o, h, 31)
    p, g = _guarded_pack(o, h)
    B.nf4_quantize(W.cuda(), out=p)
    out = Guarded((o, h), torch.bfloat16)
    B.nf4_dequantize(p, out=out.t)
    assert B.last_status() == 0
    for name, gb in g.items():
        gb.check(name)
    out.check("dequantized weight")
    ref = O.nf4_quantize(W.numpy())
    assert np.array_equal(p.codes.cpu().numpy(), ref.codes)
    assert np.array_equal(out.t.view(torch.int16).cpu().numpy().view(np.uint16),
                          O.nf4_dequantize_bits(ref))


def _oracle(li):
    return O.nf4_dequantize(O.nf4_quantize(li.Wt.numpy()))


@pytest.mark.parametrize("t", [7, 16])
def test_decode_forward_stays_inside_its_buffers(t):
    """The decode GEMV (t <= 16): Y, sT and the workspace holding its fp32 sums and tile
    counters (cleared by the call itself: the guard fill inside the workspace is overwritten
    as the call needs)."""
    h, o, r = 320, 576, 16
    li = inputs.random_linear(t, h, o, r, 2.0, seed=500 + t, with_grad=False)
    p = B.nf4_quantize(li.Wt.cuda())
    Y, sT = Guarded((t, o), torch.bfloat16), Guarded((t, r), torch.bfloat16)
    ws = Guarded((B.fwd_workspace_bytes(t, h, o, r),), torch.uint8)
    B.qlora_linear_fwd(li.X.cuda(), p, li.L1.cuda(), li.L2.cuda(), li.s, Y=Y.t, sT=sT.t, ws=ws.t)
    assert B.last_status() == 0
    for name, gb in (("Y", Y), ("sT", sT), ("workspace", ws)):
        gb.check(name)
    Y_ref, sT_ref = O.qlora_linear_fwd(f32(li.X), _oracle(li), f32(li.L1), f32(li.L2), li.s)
    assert_close_rms(f32(Y.t), Y_ref, "Y")
    assert_close_rms(f32(sT.t), sT_ref, "sT")


@pytest.mark.parametrize("t,h,o,r,s", [(300, 320, 576, 48, 0.5), (257, 640, 320, 80, 1.0)])
def test_forward_and_backward_stay_inside_their_buffers(t, h, o, r, s):
    """The tcgen05 path with ragged t, o and r: Y, sT, dX, dL1, dL2 and both workspaces."""
    li = inputs.random_linear(t, h, o, r, s, seed=600 + t)
    p = B.nf4_quantize(li.Wt.cuda())
    X, L1, L2, dY = li.X.cuda(), li.L1.cuda(), li.L2.cuda(), li.dY.cuda()
    Y, sT = Guarded((t, o), torch.bfloat16), Guarded((t, r), torch.bfloat16)
    wsf = Guarded((B.fwd_workspace_bytes(t, h, o, r),), torch.uint8)
    B.qlora_linear_fwd(X, p, L1, L2, li.s, Y=Y.t, sT=sT.t, ws=wsf.t)
    dX = Guarded((t, h), torch.bfloat16)
    dL1, dL2 = Guarded((h, r), torch.float32), Guarded((r, o), torch.float32)
    wsb = Guarded((B.bwd_workspace_bytes(t, h, o, r),), torch.uint8)
    B.qlora_linear_bwd(dY, X, p, L1, L2, li.s, sT=sT.t, dX=dX.t, dL1=dL1.t, dL2=dL2.t, ws=wsb.t)
    assert B.last_status() == 0
    for name, gb in (("Y", Y), ("sT", sT), ("forward workspace", wsf), ("dX", dX),
                     ("dL1", dL1), ("dL2", dL2), ("backward workspace", wsb)):
        gb.check(name)
    Wdq = _oracle(li)
    Y_ref, sT_ref = O.qlora_linear_fwd(f32(li.X), Wdq, f32(li.L1), f32(li.L2), li.s)
    dX_ref, dL1_ref, dL2_ref, _ = O.qlora_linear_bwd(f32(li.dY), f32(li.X), Wdq, f32(li.L1),
                                                    f32(li.L2), li.s)
    assert_close_rms(f32(Y.t), Y_ref, "Y")
    assert_close_rms(f32(sT.t), sT_ref, "sT")
    assert_close_rms(f32(dX.t), dX_ref, "dX")
    assert_close_rms(f32(dL1.t), dL1_ref, "dL1")
    assert_close_rms(f32(dL2.t), dL2_ref, "dL2")
