"""Attention dropout (attn_dropout of downcodes.com "triton transformer",
usage section): the CUDA path through fa_forward_dropout / fa_backward_dropout
against the fp64 oracle with the same Philox-4x32 (7-round) keep mask.

Two kinds of check:
  * mask read-back, bit-exact: with Q = 0 every score is 0, so every weight
    is exactly 1 and O_i = sum_j z_ij v_j / (n_i q) (n_i visible keys, q the
    keep probability).
    A one-hot V (column c <- key c of one chunk) makes O[i, c] non-zero
    exactly where z_ij = 1.  Likewise a one-hot dO exposes z through dV in the
    backward (which regenerates the mask on its own).
  * parity on random inputs: O and LSE within the forward bands, dQ/dK/dV
    within the gradient band, including grouped-query heads and padding.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_31_b200 import binding
from io_aware_exact_31_b200.workloads import bf16_bits

from _parity import TOL_GRAD_REL, TOL_LSE, TOL_O, grad_rel_err, o_error, record

pytestmark = pytest.mark.gpu


def _ok():
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"


def _visible(B, N, causal, seqlens):
    """[B, 1, N(query), N(key)] bool: key j visible to query i."""
    lens = seqlens if seqlens is not None else [N] * B
    j = np.arange(N)
    m = (j[None, None, :] < np.array(lens)[:, None, None]) & (j[None, :, None] < np.array(lens)[:, None, None])
    if causal:
        m = m & np.tril(np.ones((N, N), bool))[None]
    return m[:, None]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,Hkv,N,p,seqlens", [
    (2, 2, 2, 300, 0.3, None),
    (1, 4, 1, 200, 0.7, None),
    (2, 2, 1, 260, 0.1, [260, 131]),
])
def test_forward_mask_readback(B, H, Hkv, N, p, seqlens, causal, d):
    seed, offset = 0x5DEECE66D + N, 11
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(B, Hkv, N, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).cuda()
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda") if seqlens else None
    got = np.zeros((B, H, N, N), bool)
    o_kept = []
    for c0 in range(0, N, d):  # key chunk [c0, c0 + d) -> columns 0 .. d-1
        v = torch.zeros(B, Hkv, N, d)
        w = min(d, N - c0)
        v[:, :, c0:c0 + w, :w] = torch.eye(w)
        o, _ = binding.forward(q, k, v.to(torch.bfloat16).cuda(), causal=causal, scale=0.125,
                               seqlens=sl, dropout_p=p, seed=seed, offset=offset)
        _ok()
        oc = o[..., :w].float().cpu().numpy()
        got[..., c0:c0 + w] = oc != 0
        o_kept.append(oc)
    vis = _visible(B, N, causal, seqlens)
    want = oracle.dropout_keep_mask(B, H, N, p, seed, offset) & vis
    mism = np.argwhere(got != want)
    assert mism.size == 0, f"{len(mism)} keep bits differ, first (b,h,i,j) = {mism[:5].tolist()}"
    # kept weights are 1 / (n_i q) up to the bf16 rounding of O, with the keep
    # probability q = t / 2^8, t = floor((1 - p) 2^8 + 1/2)
    n_i = vis.sum(-1)  # [B,1,N]
    vals = np.concatenate(o_kept, axis=-1)[..., :N]
    q_keep = math.floor((1.0 - p) * 2.0 ** 8 + 0.5) / 2.0 ** 8
    expect = np.where(want, 1.0 / (np.maximum(n_i, 1)[..., None] * q_keep), 0.0)
    assert np.allclose(vals, expect, rtol=2 ** -8, atol=0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_mask_readback(causal, d):
    """dV_j[c] = sum_i Pd_ij dO_i[c]; with Q = 0 (P_ij = 1 / n_i) and dO one-hot
    on query i = chunk start + c, dV_j[c] != 0 exactly where z_ij = 1."""
    B, H, N, p, seed, offset = 1, 2, 300, 0.4, 2024, 3
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    g = torch.Generator().manual_seed(2)
    k, v = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(2))
    o, lse = binding.forward(q, k, v, causal=causal, scale=0.125, dropout_p=p, seed=seed,
                             offset=offset)
    got = np.zeros((B, H, N, N), bool)  # [b, h, query, key]
    for c0 in range(0, N, d):
        w = min(d, N - c0)
        do = torch.zeros(B, H, N, d)
        do[:, :, c0:c0 + w, :w] = torch.eye(w)
        _, _, dv = binding.backward(q, k, v, o, do.to(torch.bfloat16).cuda(), lse, causal=causal,
                                    scale=0.125, dropout_p=p, seed=seed, offset=offset)
        _ok()
        got[:, :, c0:c0 + w, :] = np.swapaxes(dv[..., :w].float().cpu().numpy() != 0, -1, -2)
    want = oracle.dropout_keep_mask(B, H, N, p, seed, offset) & _visible(B, N, causal, None)
    mism = np.argwhere(got != want)
    assert mism.size == 0, f"{len(mism)} keep bits differ, first (b,h,i,j) = {mism[:5].tolist()}"


def _inputs(B, H, Hkv, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda h: torch.randn(B, h, N, d, generator=g).to(torch.bfloat16)  # noqa: E731
    return mk(H), mk(Hkv), mk(Hkv), mk(H)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,Hkv,N,p,seqlens", [
    (1, 2, 2, 300, 0.1, None),
    (2, 4, 2, 257, 0.5, None),
    (2, 2, 1, 400, 0.25, [400, 190]),
])
def test_dropout_parity(B, H, Hkv, N, p, seqlens, causal, d):
    Q, K, V, dO = _inputs(B, H, Hkv, N, d, seed=N + d)
    scale = 1.0 / math.sqrt(d)
    seed, offset = 123456789 + N, 7
    q, k, v, do = (t.cuda() for t in (Q, K, V, dO))
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda") if seqlens else None
    o, lse = binding.forward(q, k, v, causal=causal, scale=scale, seqlens=sl, dropout_p=p,
                             seed=seed, offset=offset)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=causal, scale=scale, seqlens=sl,
                                  dropout_p=p, seed=seed, offset=offset)
    _ok()
    bits = [bf16_bits(t) for t in (Q, K, V, dO)]
    O_ref, L_ref = oracle.attention_forward_dropout(*bits[:3], scale, causal, p, seed, offset,
                                                    seqlens=seqlens)
    _, eo = o_error(o.double().cpu().numpy(), O_ref)
    el = float(np.max(np.abs(lse.double().cpu().numpy() - L_ref)))
    record(lse=el)
    assert eo <= TOL_O and el <= TOL_LSE, (eo, el)
    refs = oracle.attention_backward_dropout(*bits, scale, causal, p, seed, offset,
                                             seqlens=seqlens)
    for name, gr, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        e = grad_rel_err(gr, r)
        assert e <= TOL_GRAD_REL, f"{name}: {e:.3e}"


def test_dropout_zero_is_the_plain_path_and_masks_are_reproducible():
    B, H, N, d = 1, 2, 333, 128
    Q, K, V, _ = _inputs(B, H, H, N, d, seed=9)
    q, k, v = (t.cuda() for t in (Q, K, V))
    o0, l0 = binding.forward(q, k, v, causal=True)
    o1, l1 = binding.forward(q, k, v, causal=True, dropout_p=0.0, seed=99)
    lib = binding.load_library()
    o2, l2 = torch.empty_like(o0), torch.empty_like(l0)
    st = lib.fa_forward_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(),
                                l2.data_ptr(), None, B, H, H, N, d, 1.0 / math.sqrt(d), 1, 0.0,
                                99, 0, binding._stream_handle(None))
    assert st == binding.FA_OK
    assert torch.equal(o0, o1) and torch.equal(o0, o2) and torch.equal(l0, l2)
    # p below 2^-9 rounds to keep probability 1: the plain path as well
    o3, l3 = binding.forward(q, k, v, causal=True, dropout_p=1e-3, seed=99)
    assert torch.equal(o0, o3) and torch.equal(l0, l3)
    a, la = binding.forward(q, k, v, causal=True, dropout_p=0.2, seed=5, offset=1)
    b, lb = binding.forward(q, k, v, causal=True, dropout_p=0.2, seed=5, offset=1)
    c, _ = binding.forward(q, k, v, causal=True, dropout_p=0.2, seed=5, offset=2)
    _ok()
    assert torch.equal(a, b) and torch.equal(la, l0) and not torch.equal(a, c)


def test_dropout_rejects_bad_probability():
    z = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    for p in (1.0, -0.1, float("nan"), 1.5, 1.0 - 2.0 ** -17):
        with pytest.raises(binding.FaError) as e:
            binding.forward(z, z, z, dropout_p=p, seed=1)
        assert e.value.status == binding.FA_ERR_INVALID_ARG
        with pytest.raises(binding.FaError) as e:
            o, lse = torch.zeros_like(z), torch.zeros(1, 1, 16, device="cuda")
            binding.backward(z, z, z, o, z, lse, dropout_p=p, seed=1)
        assert e.value.status == binding.FA_ERR_INVALID_ARG


def test_autograd_wrapper_regenerates_the_mask():
    B, H, N, d = 1, 2, 200, 64
    Q, K, V, dO = _inputs(B, H, H, N, d, seed=3)
    q, k, v = (t.cuda().requires_grad_() for t in (Q, K, V))
    out = binding.attention(q, k, v, causal=True, dropout_p=0.3, seed=77, offset=4)
    out.backward(dO.cuda())
    o, lse = binding.forward(q.detach(), k.detach(), v.detach(), causal=True, dropout_p=0.3,
                             seed=77, offset=4)
    dq, dk, dv = binding.backward(q.detach(), k.detach(), v.detach(), o, dO.cuda(), lse,
                                  causal=True, dropout_p=0.3, seed=77, offset=4)
    _ok()
    assert torch.equal(out.detach(), o)
    for a, b in ((q.grad, dq), (k.grad, dk), (v.grad, dv)):
        assert (a.float() - b.float()).abs().max() <= 2e-2 * b.float().abs().max()


def test_dropout_forward_full_size_sampled():
    """The bench's dropout workload (4x16x4096x128, p = 0.1, its seed and
    offset, the launch bench.py times) on sampled rows of every head."""
    from io_aware_exact_31_b200.workloads import WORKLOADS, workload_inputs
    from _parity import sample_rows
    w = WORKLOADS["b4_h16_n4096_d128"]
    x = workload_inputs(w, seed=0)
    q, k, v = (x[n].cuda() for n in ("Q", "K", "V"))
    o, lse = binding.forward(q, k, v, causal=w.causal, scale=w.scale, dropout_p=0.1, seed=1234,
                             offset=0)
    _ok()
    rows = sample_rows(w.B, w.H, w.N, n_random=2)
    O_ref, L_ref = oracle.attention_forward_dropout_rows(
        *(bf16_bits(x[n]) for n in ("Q", "K", "V")), w.scale, w.causal, 0.1, 1234, 0, rows)
    o_rows = o.reshape(-1, w.d)[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    l_rows = lse.reshape(-1)[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    _, eo = o_error(o_rows, O_ref)
    el = float(np.max(np.abs(l_rows - L_ref)))
    record(lse=el)
    assert eo <= TOL_O and el <= TOL_LSE, (eo, el)


def test_dropout_backward_full_size_sampled_heads():
    """The bench's dropout backward workload (4x16x2048x64 causal, p = 0.1, its
    seed) on two whole heads: each head's gradient depends only on that head
    and, through the keep-mask counter, on its index b*H + h."""
    from io_aware_exact_31_b200.workloads import WORKLOADS, workload_inputs
    w = WORKLOADS["b4_h16_n2048_d64_causal_bwd"]
    x = workload_inputs(w, seed=0)
    q, k, v, do = (x[n].cuda() for n in ("Q", "K", "V", "dO"))
    o, lse = binding.forward(q, k, v, causal=True, scale=w.scale, dropout_p=0.1, seed=99)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=True, scale=w.scale, dropout_p=0.1,
                                  seed=99)
    _ok()
    heads = [0, 2 * w.H + 11]
    refs = oracle.attention_backward_dropout_heads(
        *(bf16_bits(x[n]) for n in ("Q", "K", "V", "dO")), w.scale, True, 0.1, 99, 0, heads)
    for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        for bh in heads:
            b, h = divmod(bh, w.H)
            e = grad_rel_err(g[b, h], r[b, h])
            assert e <= TOL_GRAD_REL, f"{name} head {bh}: {e:.3e}"
