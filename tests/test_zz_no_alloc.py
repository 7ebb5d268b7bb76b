"""The allocation-free forward entry point against the regular one.

qlora_linear_fwd_noalloc serves callers that are given only input and output buffers and
cannot allocate device memory (no workspace to pass, or cudaMalloc's device-wide
synchronisation is not acceptable); it uses a scratch array that lives in the library's
device image instead of a caller workspace. This test calls it through the C ABI twice in a
row per shape and compares each result with qlora_linear_fwd (caller workspace) within the
tolerance the parity tests use. It lives in its own file so that pytest collects it last.
"""

import ctypes

import pytest
import torch

from bit_quantized_lora_03_b200 import binding as B
from bit_quantized_lora_03_b200 import inputs

from gpu_util import assert_close_rms, f32, require_gpu

pytestmark = pytest.mark.gpu


def _noalloc(X, p, L1, L2, s, Y, sT):
    d = p.desc()
    stream = torch.cuda.current_stream().cuda_stream
    return B.lib().qlora_linear_fwd_noalloc(X.data_ptr(), X.shape[0], ctypes.byref(d),
                                            L1.data_ptr(), L2.data_ptr(), L1.shape[1], float(s),
                                            Y.data_ptr(), sT.data_ptr(), stream)


@pytest.mark.parametrize("t,h,o,r,s", [
    (4, 320, 576, 16, 2.0),        # decode GEMV path (scratch holds a t x o fp32 accumulator)
    (300, 320, 576, 48, 0.5),      # tcgen05 GEMM path
    (4096, 4096, 4096, 64, 0.25),  # training shape
])
def test_noalloc_matches_workspace_forward_twice(t, h, o, r, s):
    require_gpu()
    li = inputs.random_linear(t, h, o, r, s, seed=900 + t, with_grad=False)
    dev = torch.device("cuda")
    p = B.nf4_quantize(li.Wt.to(dev))
    X, L1, L2 = li.X.to(dev), li.L1.to(dev), li.L2.to(dev)
    Y_ref, sT_ref = B.qlora_linear_fwd(X, p, L1, L2, s)
    torch.cuda.synchronize()
    for call in range(2):
        Y = torch.full((t, o), float("nan"), dtype=torch.bfloat16, device=dev)
        sT = torch.full((t, r), float("nan"), dtype=torch.bfloat16, device=dev)
        assert _noalloc(X, p, L1, L2, s, Y, sT) == B.QLORA_OK
        assert B.last_status() == 0
        assert_close_rms(f32(Y), f32(Y_ref), f"Y (call {call + 1})")
        assert_close_rms(f32(sT), f32(sT_ref), f"sT (call {call + 1})")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    require_gpu()
    t, h, o, r = 32768, 1024, 1024, 256      # sT alone is 32768 * 256 * 2 bytes = 16 MiB > 8 MiB
    assert B.fwd_workspace_bytes(t, h, o, r) > B.QLORA_STATIC_SCRATCH_BYTES
    dev = torch.device("cuda")
    p = B.PackedNF4(o, h, dev)
    X = torch.zeros(t, h, dtype=torch.bfloat16, device=dev)
    L1 = torch.zeros(h, r, dtype=torch.bfloat16, device=dev)
    L2 = torch.zeros(r, o, dtype=torch.bfloat16, device=dev)
    Y = torch.empty(t, o, dtype=torch.bfloat16, device=dev)
    sT = torch.empty(t, r, dtype=torch.bfloat16, device=dev)
    assert _noalloc(X, p, L1, L2, 1.0, Y, sT) == B.QLORA_ERR_SCRATCH_LIMIT
