"""GPU parity of qlora_adamw_step (the adapters' update) against the oracle's fp64 AdamW over
several steps, its bf16 copy bit for bit, and the same step with the optimizer state in unified
memory (the pages' paged optimizer), also after that state was moved to host memory."""

import ctypes

import numpy as np
import pytest
import torch

from bit_quantized_lora_03_b200 import binding as B
from oracle import nf4_oracle as O

from gpu_util import require_gpu

pytestmark = pytest.mark.gpu

HP = dict(lr=2e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _grads(n, k, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(n, generator=g) * (0.1 * (i + 1)) for i in range(k)]


def test_adamw_matches_oracle_over_steps():
    require_gpu()
    n = 4096 * 64 + 1024        # an L1 of h = 4096, r = 64, plus a tail
    g0 = torch.Generator().manual_seed(5)
    p0 = torch.randn(n, generator=g0) * 0.01
    p, m, v = p0.cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    p16 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    pr, mr, vr = p0.double().numpy(), np.zeros(n), np.zeros(n)
    for t, g in enumerate(_grads(n, 4, 6), start=1):
        B.adamw_step(p, g.cuda(), m, v, t, p16=p16, **HP)
        # the library takes fp32 hyper-parameters: the oracle gets the same fp32 values
        f = {k: float(np.float32(x)) for k, x in HP.items()}
        pr, mr, vr = O.adamw_step(pr, g.double().numpy(), mr, vr, t, f["lr"], f["beta1"],
                                  f["beta2"], f["eps"], f["weight_decay"])
    assert B.last_status() == 0
    # fp32 evaluation of sums of signed terms: a few ulps of each value, plus a floor of 1e-6
    # of the tensor's largest magnitude for entries that pass near zero (for p that floor,
    # ~5e-8, is far below one step of lr = 2e-3)
    for got, ref, name in ((p, pr, "p"), (m, mr, "m"), (v, vr, "v")):
        err = np.abs(got.double().cpu().numpy() - ref)
        floor = 1e-6 * np.max(np.abs(ref))
        assert np.all(err <= 4e-6 * np.abs(ref) + floor), f"{name}: max excess {np.max(err - 4e-6 * np.abs(ref) - floor)}"
    assert torch.equal(p16, p.to(torch.bfloat16))


def _managed(nbytes):
    from cuda.bindings import runtime as rt
    err, ptr = rt.cudaMallocManaged(nbytes, rt.cudaMemAttachGlobal)
    assert err == rt.cudaError_t.cudaSuccess
    return int(ptr)


def test_adamw_with_state_in_unified_memory():
    require_gpu()
    from cuda.bindings import runtime as rt
    n = 8192
    m_ptr, v_ptr = _managed(4 * n), _managed(4 * n)
    try:
        ctypes.memset(m_ptr, 0, 4 * n)      # unified memory is host-writable
        ctypes.memset(v_ptr, 0, 4 * n)
        g0 = torch.Generator().manual_seed(9)
        p0 = torch.randn(n, generator=g0) * 0.01
        p_a, p_b = p0.cuda(), p0.cuda()
        m_b, v_b = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
        for t, g in enumerate(_grads(n, 3, 10), start=1):
            gd = g.cuda()
            if t >= 2:   # page the state out to host memory; the step brings it back
                for ptr in (m_ptr, v_ptr):
                    assert rt.cudaMemPrefetchAsync(ptr, 4 * n, rt.cudaCpuDeviceId, 0)[0] == rt.cudaError_t.cudaSuccess
            # step 2 prefetches the paged-out state back; step 3 lets it migrate on first touch
            B.adamw_step_ptr(p_a.data_ptr(), 0, gd.data_ptr(), m_ptr, v_ptr, n, HP["lr"],
                             HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t,
                             flags=B.ADAMW_PREFETCH if t == 2 else 0)
            B.adamw_step(p_b, gd, m_b, v_b, t, **HP)
        assert B.last_status() == 0
        torch.cuda.synchronize()
        assert torch.equal(p_a, p_b)
        m_host = np.ctypeslib.as_array((ctypes.c_float * n).from_address(m_ptr)).copy()
        assert np.array_equal(m_host, m_b.cpu().numpy())
    finally:
        rt.cudaFree(m_ptr)
        rt.cudaFree(v_ptr)
