"""Padded batches (padding mask of downcodes.com "triton transformer", BERT
example): CUDA path through fa_forward_varlen / fa_backward_varlen vs the
fp64 oracle's padded functions."""
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
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,Hkv,N,seqlens", [
    (2, 2, 300, [300, 129, 1]),
    (4, 2, 600, [0, 600, 257]),
    (2, 1, 513, [128, 500, 513]),
])
def test_varlen_forward_backward(H, Hkv, N, seqlens, causal, d):
    B = len(seqlens)
    Q, K, V, dO = _inputs(B, H, Hkv, N, d, seed=N + sum(seqlens))
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (t.cuda() for t in (Q, K, V, dO))
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    o, lse = binding.forward(q, k, v, causal=causal, scale=scale, seqlens=sl)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=causal, scale=scale, seqlens=sl)
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"
    bits = [bf16_bits(t) for t in (Q, K, V, dO)]
    O_ref, L_ref = oracle.attention_forward_varlen(*bits[:3], seqlens, scale, causal)
    _, eo = o_error(o.double().cpu().numpy(), O_ref)
    el = float(np.max(np.abs(lse.double().cpu().numpy() - L_ref)))
    record(lse=el)
    assert eo <= TOL_O and el <= TOL_LSE, (eo, el)
    refs = oracle.attention_backward_varlen(*bits, seqlens, scale, causal)
    for name, gr, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        e = grad_rel_err(gr, r)
        assert e <= TOL_GRAD_REL, f"{name}: {e:.3e}"
    # padding tokens: exactly zero outputs and gradients
    for b, n in enumerate(seqlens):
        assert torch.all(o[b, :, n:] == 0) and torch.all(lse[b, :, n:] == 0)
        assert torch.all(dq[b, :, n:] == 0)
        assert torch.all(dk[b, :, n:] == 0) and torch.all(dv[b, :, n:] == 0)


def test_full_lengths_equal_unpadded_path():
    B, H, N, d = 2, 2, 333, 64
    Q, K, V, dO = _inputs(B, H, H, N, d, seed=5)
    q, k, v, do = (t.cuda() for t in (Q, K, V, dO))
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    o1, l1 = binding.forward(q, k, v, causal=True, seqlens=sl)
    o2, l2 = binding.forward(q, k, v, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    g1 = binding.backward(q, k, v, o1, do, l1, causal=True, seqlens=sl)
    g2 = binding.backward(q, k, v, o2, do, l2, causal=True)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
