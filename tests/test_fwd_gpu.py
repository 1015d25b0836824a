"""Forward parity: CUDA path (through the C ABI) vs the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_31_b200 import binding
from io_aware_exact_31_b200.workloads import WORKLOADS, bf16_bits

from _parity import (TOL_GRAD_REL, TOL_LSE, TOL_O, check_forward_full, check_forward_sampled,
                     fwd_errors, gpu_forward, grad_rel_err, inputs)

pytestmark = pytest.mark.gpu


def test_tiny_workload():
    w = WORKLOADS["tiny_n256_d64"]
    check_forward_full(w.B, w.H, w.N, w.d, w.causal)


def test_transformer_h8_n1024_d64_causal():
    w = WORKLOADS["transformer_h8_n1024_d64_causal"]
    check_forward_full(w.B, w.H, w.N, w.d, w.causal)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 3, 17, 127, 128, 129, 255, 256, 257, 300, 513])
def test_ragged_lengths(N, causal, d):
    check_forward_full(1, 2, N, d, causal, seed=N)


@pytest.mark.parametrize("d", [64, 128])
def test_many_heads_small_n(d):
    check_forward_full(3, 5, 64, d, False, seed=3)
    check_forward_full(3, 5, 200, d, True, seed=4)


@pytest.mark.parametrize("d", [64, 128])
def test_multi_block_wide_scores(d):
    # scaled inputs: scores with std ~4, exercises the running-max rescale
    check_forward_full(2, 3, 1000, d, False, seed=5, input_scale=2.0)
    check_forward_full(2, 3, 777, d, True, seed=6, input_scale=2.0)


def test_b4_h16_n4096_d128_sampled():
    w = WORKLOADS["b4_h16_n4096_d128"]
    check_forward_sampled(w.B, w.H, w.N, w.d, w.causal, n_random=4)


def test_h16_n16384_d128_causal_x2_sampled():
    w = WORKLOADS["h16_n16384_d128_causal_x2"]
    check_forward_sampled(w.B, w.H, w.N, w.d, w.causal, input_scale=w.input_scale, n_random=4)


def test_b4_h16_n2048_d64_causal_sampled():
    """The forward of the forward + backward workload, every CTA checked."""
    w = WORKLOADS["b4_h16_n2048_d64_causal_bwd"]
    check_forward_sampled(w.B, w.H, w.N, w.d, w.causal, n_random=4)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("p_drop", [0.0, 0.1])
def test_late_dominant_key(d, causal, p_drop):
    """One key in a late block (key 700 = 64 * ones) whose scores exceed the
    earlier blocks' by up to ~2^250 for a quarter of the rows: the running
    reference must move (rescale, or at d = 64 the redo of a block that
    outgrows a reference taken without its row max) and O, LSE and the
    gradients still match the oracle."""
    B, H, N = 1, 2, 1024
    x = inputs(B, H, N, d, seed=31, with_dO=True)
    x["K"][:, :, 700, :] = 64.0
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("Q", "K", "V", "dO"))
    o, lse = binding.forward(q, k, v, causal=causal, scale=scale, dropout_p=p_drop, seed=5)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=causal, scale=scale,
                                  dropout_p=p_drop, seed=5)
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"
    bits = [bf16_bits(x[n]) for n in ("Q", "K", "V", "dO")]
    if p_drop > 0:
        O_ref, L_ref = oracle.attention_forward_dropout(*bits[:3], scale, causal, p_drop, 5, 0)
        refs = oracle.attention_backward_dropout(*bits, scale, causal, p_drop, 5, 0)
    else:
        O_ref, L_ref = oracle.attention_forward(*bits[:3], scale, causal)
        refs = oracle.attention_backward(*bits, scale, causal)
    eo, el = fwd_errors(o, lse, O_ref, L_ref)
    assert eo <= TOL_O and el <= TOL_LSE, f"max|dO|={eo:.3e} max|dLSE|={el:.3e}"
    for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        e = grad_rel_err(g, r)
        assert e <= TOL_GRAD_REL, f"{name}: {e:.3e}"


def test_deterministic():
    x = inputs(2, 4, 1100, 128, seed=7)
    o1, l1 = gpu_forward(x, True, 1 / math.sqrt(128))
    o2, l2 = gpu_forward(x, True, 1 / math.sqrt(128))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_guard_bands_untouched():
    B, H, N, d = 1, 3, 333, 64
    x = inputs(B, H, N, d, seed=8)
    q, k, v = (x[n].cuda() for n in ("Q", "K", "V"))
    pad = 4096
    obuf = torch.full((pad + B * H * N * d + pad,), -7.0, device="cuda", dtype=torch.bfloat16)
    lbuf = torch.full((pad + B * H * N + pad,), -7.0, device="cuda", dtype=torch.float32)
    o = obuf[pad:pad + B * H * N * d].view(B, H, N, d)
    lse = lbuf[pad:pad + B * H * N].view(B, H, N)
    binding.forward(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert (obuf[:pad] == -7).all() and (obuf[-pad:] == -7).all()
    assert (lbuf[:pad] == -7).all() and (lbuf[-pad:] == -7).all()
    assert torch.isfinite(o.float()).all()


def test_non_default_stream():
    x = inputs(1, 2, 300, 128, seed=9)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        q, k, v = (x[n].cuda() for n in ("Q", "K", "V"))
        o, lse = binding.forward(q, k, v, causal=False)
    s.synchronize()
    o_ref, l_ref = gpu_forward(x, False, 1 / math.sqrt(128))
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_invalid_args_on_device():
    q = torch.zeros(1, 1, 16, 64, device="cuda", dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 16, device="cuda")
    st = binding.forward_raw(q.data_ptr() + 2, q.data_ptr(), q.data_ptr(), q.data_ptr(),
                             lse.data_ptr(), 1, 1, 16, 64, 0.125, 0)
    assert st == binding.FA_ERR_INVALID_ARG
    st = binding.forward_raw(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(),
                             lse.data_ptr(), 1, 1, 16, 80, 0.125, 0)
    assert st == binding.FA_ERR_UNSUPPORTED
