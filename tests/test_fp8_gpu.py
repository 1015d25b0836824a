"""FP8 (E4M3) forward parity: fa_forward_fp8 vs the fp64 oracle evaluated on
the dequantised inputs.

The pages give no FP8 tolerance, so the band is derived from the arithmetic:
the E4M3 products and their fp32 sums in S are exact up to fp32 rounding;
P is rounded to E4M3, |p~ - p| <= 2^-4 p + 2^-10 (relative half-ulp of the
3-bit mantissa; half the subnormal spacing 2^-9 below 2^-6); O is divided by
the sum of the same rounded weights, so exactly
    O - O_ref = sum_j (p~_j - p_j) (v_j - O_ref) / sum_j p~_j .
With w_j the softmax weights and p_j >= 2^-8 w_j / w_max (the kernel keeps
its running max within 2^8 of the true one), per element
    |O - O_ref| <= 2^-4 sum_j w_j |v_j - O_ref| + 2^-10 w_max sum_j |v_j - O_ref|
to first order; the test allows 10 % on top for the second-order terms, plus
the bf16 rounding of O.  LSE is computed from the unrounded p: 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_31_b200 import binding

from _parity import TOL_LSE, bf16_rounding_distance, record

pytestmark = pytest.mark.gpu


def _quant(x):
    """Per-tensor E4M3 quantisation: (fp8 tensor, dequant scale)."""
    s = float(x.abs().max()) / 448.0
    return (x / s).to(torch.float8_e4m3fn), s


def _fp8_band(Qd, Kd, Vd, O_ref, scale, causal):
    B, H, N, d = Qd.shape
    G = H // Kd.shape[1]
    Kr = np.repeat(Kd, G, axis=1)
    Vr = np.repeat(Vd, G, axis=1)
    S = scale * np.einsum("bhid,bhjd->bhij", Qd, Kr)
    if causal:
        S = np.where(np.triu(np.ones((N, N), bool), 1), -np.inf, S)
    W = np.exp(S - S.max(-1, keepdims=True))
    W /= W.sum(-1, keepdims=True)
    dev = np.abs(Vr[:, :, None, :, :] - O_ref[:, :, :, None, :])  # [B,H,i,j,d]
    if causal:
        dev = dev * np.tril(np.ones((N, N)))[None, None, :, :, None]
    t1 = np.einsum("bhij,bhijd->bhid", W, dev)
    t2 = W.max(-1)[..., None] * dev.sum(3)
    return 1.1 * (2.0 ** -4 * t1 + 2.0 ** -10 * t2) + bf16_rounding_distance(O_ref)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,Hkv,N", [(1, 2, 2, 300), (1, 4, 2, 700), (2, 1, 1, 129)])
def test_fp8_forward(B, H, Hkv, N, causal):
    d = 128
    g = torch.Generator().manual_seed(N + H)
    q = torch.randn(B, H, N, d, generator=g)
    k = torch.randn(B, Hkv, N, d, generator=g)
    v = torch.randn(B, Hkv, N, d, generator=g)
    (q8, sq), (k8, sk), (v8, sv) = _quant(q), _quant(k), _quant(v)
    scale = 1.0 / math.sqrt(d)
    o, lse = binding.forward_fp8(q8.cuda(), k8.cuda(), v8.cuda(), sq, sk, sv, causal=causal,
                                 scale=scale)
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"
    Qd, Kd, Vd = (t.double().numpy() * s for t, s in ((q8, sq), (k8, sk), (v8, sv)))
    O_ref, L_ref = oracle.attention_forward_gqa(Qd, Kd, Vd, scale, causal)
    err = np.abs(o.double().cpu().numpy() - O_ref)
    band = _fp8_band(Qd, Kd, Vd, O_ref, scale, causal)
    worst = float(np.max(err / band))
    assert worst <= 1.0, f"error/band max {worst:.3f} (max abs err {err.max():.3e})"
    el = float(np.max(np.abs(lse.double().cpu().numpy() - L_ref)))
    assert el <= TOL_LSE, el
    assert torch.isfinite(o.float()).all()


def test_fp8_rejects_unsupported():
    z = torch.zeros(1, 1, 16, 64, device="cuda", dtype=torch.float8_e4m3fn)
    with pytest.raises(binding.FaError) as e:
        binding.forward_fp8(z, z, z, 1.0, 1.0, 1.0)
    assert e.value.status == binding.FA_ERR_UNSUPPORTED
    z = torch.zeros(1, 1, 16, 128, device="cuda", dtype=torch.float8_e4m3fn)
    with pytest.raises(binding.FaError) as e:
        binding.forward_fp8(z, z, z, 0.0, 1.0, 1.0)
    assert e.value.status == binding.FA_ERR_INVALID_ARG


def test_fp8_forward_full_size_sampled():
    """The bench's E4M3 workload (4x16x4096x128, per-tensor quantisation of the
    seeded inputs, the launch bench.py times) on sampled rows of every head,
    with the band of the module docstring computed row by row."""
    from io_aware_exact_31_b200.workloads import WORKLOADS, workload_inputs
    from _parity import sample_rows
    w = WORKLOADS["b4_h16_n4096_d128"]
    x = workload_inputs(w, seed=0)
    (q8, sq), (k8, sk), (v8, sv) = (_quant(x[n].float()) for n in ("Q", "K", "V"))
    o, lse = binding.forward_fp8(q8.cuda(), k8.cuda(), v8.cuda(), sq, sk, sv, causal=w.causal,
                                 scale=w.scale)
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"
    Qd, Kd, Vd = (t.double().numpy() * s for t, s in ((q8, sq), (k8, sk), (v8, sv)))
    rows = sample_rows(w.B, w.H, w.N, n_random=2)
    O_ref, L_ref = oracle.attention_forward_rows(Qd, Kd, Vd, w.scale, w.causal, rows)
    o_rows = o.reshape(-1, w.d)[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    l_rows = lse.reshape(-1)[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    Kh, Vh = Kd.reshape(-1, w.N, w.d), Vd.reshape(-1, w.N, w.d)
    worst = 0.0
    for k, rid in enumerate(rows):
        bh, i = divmod(int(rid), w.N)
        srow = w.scale * (Kh[bh] @ Qd.reshape(-1, w.d)[rid])
        wts = np.exp(srow - srow.max())
        wts /= wts.sum()
        dev = np.abs(Vh[bh] - O_ref[k])
        band = (1.1 * (2.0 ** -4 * (wts @ dev) + 2.0 ** -10 * wts.max() * dev.sum(0)) +
                bf16_rounding_distance(O_ref[k]))
        worst = max(worst, float(np.max(np.abs(o_rows[k] - O_ref[k]) / band)))
    el = float(np.max(np.abs(l_rows - L_ref)))
    record(o_raw=float(np.max(np.abs(o_rows - O_ref))), fp8_err_over_band=worst, lse=el,
           rows_checked=rows.size)
    assert worst <= 1.0, f"error/band max {worst:.3f}"
    assert el <= TOL_LSE
