"""GPU parity of qlora_adamw_step (the adapters' update) against the oracle's fp64 AdamW over
several steps, its bf16 copy bit for bit, and the same step with the optimizer state in unified
memory (the pages' paged optimizer), also after that state was moved to host memory; and
qlora_adamw_step_multi (all adapters in one launch) against the single-tensor call, bit for bit,
and against the oracle."""

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


def _check_against_oracle(got, ref, name):
    err = np.abs(got.double().cpu().numpy() - ref)
    floor = 1e-6 * np.max(np.abs(ref))
    assert np.all(err <= 4e-6 * np.abs(ref) + floor), f"{name}: max excess {np.max(err - 4e-6 * np.abs(ref) - floor)}"


def test_adamw_multi_matches_single_and_oracle():
    """The 14 adapter tensors of one LLaMA-7B layer at r = 64 (L1 h x r and L2 r x o of seven
    linears), scaled down in h and o by 8 so the oracle stays quick, plus two tiny tensors of
    4 and 8 parameters: one multi-tensor launch per step equals 16 single-tensor launches bit
    for bit (p, m, v and the bf16 copies), over three steps."""
    require_gpu()
    shapes = []
    for h, o in ((512, 512),) * 4 + ((512, 1376),) * 2 + ((1376, 512),):
        shapes += [(h, 64), (64, o)]
    shapes += [(4,), (8,)]
    g0 = torch.Generator().manual_seed(21)
    p0 = [torch.randn(*sh, generator=g0) * 0.02 for sh in shapes]
    pa = [x.cuda() for x in p0]
    pb = [x.cuda() for x in p0]
    ma, va = [torch.zeros_like(x) for x in pa], [torch.zeros_like(x) for x in pa]
    mb, vb = [torch.zeros_like(x) for x in pb], [torch.zeros_like(x) for x in pb]
    qa = [torch.empty_like(x, dtype=torch.bfloat16) if k % 3 else None for k, x in enumerate(pa)]
    qb = [torch.empty_like(x, dtype=torch.bfloat16) if k % 3 else None for k, x in enumerate(pb)]
    ref = [(x.double().numpy().ravel(), np.zeros(x.numel()), np.zeros(x.numel())) for x in p0]
    f = {k: float(np.float32(x)) for k, x in HP.items()}
    for t in range(1, 4):
        gs = [torch.randn(*sh, generator=g0) * 0.1 for sh in shapes]
        gd = [g.cuda() for g in gs]
        B.adamw_step_multi(pa, gd, ma, va, t, params_bf16=qa, **HP)
        for k in range(len(shapes)):
            B.adamw_step(pb[k], gd[k], mb[k], vb[k], t, p16=qb[k], **HP)
        ref = [O.adamw_step(pr, g.double().numpy().ravel(), mr, vr, t, f["lr"], f["beta1"],
                            f["beta2"], f["eps"], f["weight_decay"])
               for (pr, mr, vr), g in zip(ref, gs)]
    assert B.last_status() == 0
    torch.cuda.synchronize()
    for k in range(len(shapes)):
        assert torch.equal(pa[k], pb[k]) and torch.equal(ma[k], mb[k]) and torch.equal(va[k], vb[k])
        if qa[k] is not None:
            assert torch.equal(qa[k], qb[k])
            assert torch.equal(qa[k], pa[k].to(torch.bfloat16))
        for got, r, name in zip((pa[k], ma[k], va[k]), ref[k], "pmv"):
            _check_against_oracle(got.reshape(-1), r, f"{name}[{k}]")
