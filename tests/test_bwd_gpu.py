"""Backward parity: CUDA path (through the C ABI) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

from io_aware_exact_31_b200 import binding
from io_aware_exact_31_b200.workloads import WORKLOADS

from _parity import check_backward, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 255, 300])
def test_small(N, causal, d):
    check_backward(1, 2, N, d, causal, seed=N + d)


@pytest.mark.parametrize("d", [64, 128])
def test_multi_block(d):
    check_backward(2, 2, 700, d, True, seed=11)
    check_backward(1, 3, 520, d, False, seed=12)


def test_b4_h16_n2048_d64_causal_sampled_heads():
    """The full backward workload; the oracle checks 16 of its 64 heads: the
    first and last head of every batch (the first and last CTAs of each
    batch's key blocks) and eight more drawn at random."""
    w = WORKLOADS["b4_h16_n2048_d64_causal_bwd"]
    ends = [(b, h) for b in range(w.B) for h in (0, w.H - 1)]
    rest = [(b, h) for b in range(w.B) for h in range(1, w.H - 1)]
    r = np.random.default_rng(2)
    pick = [rest[i] for i in sorted(r.choice(len(rest), size=8, replace=False))]
    check_backward(w.B, w.H, w.N, w.d, w.causal, heads=ends + pick)


def test_b4_h16_n2048_d128_causal_sampled_heads():
    """The backward at head dimension 128 on the same shape (the benchmark's
    --bwd-d 128 run): the first and last head of every batch."""
    w = WORKLOADS["b4_h16_n2048_d64_causal_bwd"]
    heads = [(b, h) for b in range(w.B) for h in (0, w.H - 1)]
    check_backward(w.B, w.H, w.N, 128, True, seed=0, heads=heads)


def test_autograd_wrapper_matches_raw():
    x = inputs(1, 2, 200, 64, seed=13, with_dO=True)
    q, k, v, do = (x[n].cuda() for n in ("Q", "K", "V", "dO"))
    qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
    out = binding.attention(qr, kr, vr, causal=True)
    out.backward(do)
    o, lse = binding.forward(q, k, v, causal=True)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=True)
    assert torch.equal(out.detach(), o)
    assert torch.equal(kr.grad, dk) and torch.equal(vr.grad, dv)
    assert (qr.grad.float() - dq.float()).abs().max() <= 1e-2 * dq.float().abs().max()


def test_workspace_too_small_rejected():
    x = inputs(1, 1, 128, 64, seed=14, with_dO=True)
    q, k, v, do = (x[n].cuda() for n in ("Q", "K", "V", "dO"))
    o, lse = binding.forward(q, k, v)
    ws = torch.empty(16, device="cuda", dtype=torch.uint8)
    with pytest.raises(binding.FaError) as e:
        binding.backward(q, k, v, o, do, lse, workspace=ws)
    assert e.value.status == binding.FA_ERR_INVALID_ARG
