"""Grouped-/multi-query attention parity (unite.ai page, "FlashAttention-2"
item 3): CUDA path through fa_forward_gqa / fa_backward_gqa vs the fp64
oracle's grouped-query functions."""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_31_b200 import binding
from io_aware_exact_31_b200.workloads import bf16_bits

from _parity import TOL_GRAD_REL, TOL_LSE, TOL_O, grad_rel_err, o_error, record

pytestmark = pytest.mark.gpu


def _inputs(B, H, Hkv, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda h: torch.randn(B, h, N, d, generator=g).to(torch.bfloat16)  # noqa: E731
    return mk(H), mk(Hkv), mk(Hkv), mk(H)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,Hkv", [(8, 1), (8, 2), (6, 3), (4, 4)])
@pytest.mark.parametrize("causal,N", [(False, 300), (True, 257), (True, 640)])
def test_gqa_forward_backward(H, Hkv, causal, N, d):
    B = 2
    Q, K, V, dO = _inputs(B, H, Hkv, N, d, seed=H * 100 + Hkv + N)
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (t.cuda() for t in (Q, K, V, dO))
    o, lse = binding.forward(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=causal, scale=scale)
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"
    assert dk.shape == K.shape and dv.shape == V.shape
    bits = [bf16_bits(t) for t in (Q, K, V, dO)]
    O_ref, L_ref = oracle.attention_forward_gqa(*bits[:3], scale, causal)
    _, eo = o_error(o.double().cpu().numpy(), O_ref)
    el = float(np.max(np.abs(lse.double().cpu().numpy() - L_ref)))
    record(lse=el)
    assert eo <= TOL_O and el <= TOL_LSE, (eo, el)
    refs = oracle.attention_backward_gqa(*bits, scale, causal)
    for name, gr, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        e = grad_rel_err(gr, r)
        assert e <= TOL_GRAD_REL, f"{name}: {e:.3e}"


def test_gqa_rejects_bad_head_counts():
    q = torch.zeros(1, 6, 16, 64, device="cuda", dtype=torch.bfloat16)
    k = torch.zeros(1, 4, 16, 64, device="cuda", dtype=torch.bfloat16)
    lse = torch.zeros(1, 6, 16, device="cuda")
    lib = binding.load_library()
    st = lib.fa_forward_gqa(q.data_ptr(), k.data_ptr(), k.data_ptr(), q.data_ptr(),
                            lse.data_ptr(), 1, 6, 4, 16, 64, 0.125, 0, None)
    assert st == binding.FA_ERR_INVALID_ARG
