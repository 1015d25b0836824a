"""Full-size parity of the extension workloads the benchmark times: grouped-query
and padded batches on the 4x16x4096x128 forward and on the 4x16x2048x64 causal
forward + backward, and the deterministic backward of the latter.  Shapes,
entry points and input seeds are those of the benchmark's timed calls (rank
0); the fp64 oracle checks sampled rows or whole heads (heads are independent)
under the standard bands."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_31_b200 import binding
from io_aware_exact_31_b200.workloads import WORKLOADS, bf16_bits, workload_inputs

from _parity import (TOL_GRAD_REL, TOL_LSE, TOL_O, grad_rel_err, o_error, record,
                     sample_rows)

pytestmark = pytest.mark.gpu

HEADLINE = WORKLOADS["b4_h16_n4096_d128"]
FWDBWD = WORKLOADS["b4_h16_n2048_d64_causal_bwd"]


def _gen(shape, seed):
    """The benchmark's input generator for these workloads: i.i.d. N(0, 1)
    from a seeded CPU generator, rounded to bf16 (kept on the CPU here)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def _ok():
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"


def _fwd_compare(o, lse, O_ref, L_ref):
    _, eo = o_error(o.double().cpu().numpy(), O_ref)
    el = float(np.max(np.abs(lse.double().cpu().numpy() - L_ref)))
    record(lse=el)
    assert eo <= TOL_O and el <= TOL_LSE, f"max|dO|={eo:.3e} max|dLSE|={el:.3e}"


def test_headline_grouped_query_sampled_rows():
    """4x16x4096x128 with 2 K/V heads (8 query heads each), every CTA of every
    head checked on sampled rows against the plain oracle on K/V repeated per
    query head (query head h reads K/V head h // 8)."""
    w, hkv = HEADLINE, 2
    Q = _gen((w.B, w.H, w.N, w.d), 10)
    K, V = _gen((w.B, hkv, w.N, w.d), 11), _gen((w.B, hkv, w.N, w.d), 12)
    o, lse = binding.forward(Q.cuda(), K.cuda(), V.cuda(), causal=w.causal, scale=w.scale)
    _ok()
    g = w.H // hkv
    Kx, Vx = K.repeat_interleave(g, dim=1), V.repeat_interleave(g, dim=1)
    rows = sample_rows(w.B, w.H, w.N, n_random=2)
    O_ref, L_ref = oracle.attention_forward_rows(bf16_bits(Q), bf16_bits(Kx), bf16_bits(Vx),
                                                 w.scale, w.causal, rows)
    idx = torch.from_numpy(rows).cuda()
    _fwd_compare(o.reshape(-1, w.d)[idx], lse.reshape(-1)[idx], O_ref, L_ref)
    record(rows_checked=rows.size)


def test_headline_padded_heads():
    """4x16x4096x128 with real lengths 4096/3072/2048/1024: two whole heads per
    batch against the oracle, and exact zeros on every padding row."""
    w = HEADLINE
    lens = [w.N, 3 * w.N // 4, w.N // 2, w.N // 4]
    Q = _gen((w.B, w.H, w.N, w.d), 10)
    K, V = _gen((w.B, w.H, w.N, w.d), 13), _gen((w.B, w.H, w.N, w.d), 14)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = binding.forward(Q.cuda(), K.cuda(), V.cuda(), causal=w.causal, scale=w.scale,
                             seqlens=sl)
    _ok()
    for b, n in enumerate(lens):
        assert not o[b, :, n:].any() and not lse[b, :, n:].any(), f"batch {b} padding"
        hs = [b, w.H - 1 - b]
        sub = lambda t: t[b:b + 1, hs].contiguous()  # noqa: E731
        O_ref, L_ref = oracle.attention_forward_varlen(
            *(bf16_bits(sub(t)) for t in (Q, K, V)), [n], w.scale, w.causal)
        _fwd_compare(o[b:b + 1, hs], lse[b:b + 1, hs], O_ref, L_ref)
    record(heads_checked=2 * w.B)


def _grad_check(pairs):
    errs = {}
    for name, g, r in pairs:
        errs[name] = max(errs.get(name, 0.0), grad_rel_err(g, r))
    for name, e in errs.items():
        assert e <= TOL_GRAD_REL, f"{name} rel err {e:.3e} (all: {errs})"


def test_fwdbwd_grouped_query_groups():
    """4x16x2048x64 causal with 4 K/V heads: forward and backward of three
    whole groups (four query heads and their K/V head) against the oracle."""
    w, hkv = FWDBWD, 4
    Q, dO = _gen((w.B, w.H, w.N, w.d), 20), _gen((w.B, w.H, w.N, w.d), 21)
    K, V = _gen((w.B, hkv, w.N, w.d), 22), _gen((w.B, hkv, w.N, w.d), 23)
    q, k, v, do = (t.cuda() for t in (Q, K, V, dO))
    o, lse = binding.forward(q, k, v, causal=True, scale=w.scale)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=True, scale=w.scale)
    _ok()
    g = w.H // hkv
    for b, kv in [(0, 0), (1, 3), (3, 2)]:
        hs = slice(kv * g, (kv + 1) * g)
        bits = [bf16_bits(t[b:b + 1, hs].contiguous()) for t in (Q,)] + \
               [bf16_bits(t[b:b + 1, kv:kv + 1].contiguous()) for t in (K, V)] + \
               [bf16_bits(dO[b:b + 1, hs].contiguous())]
        O_ref, L_ref = oracle.attention_forward_gqa(*bits[:3], w.scale, True)
        _fwd_compare(o[b:b + 1, hs], lse[b:b + 1, hs], O_ref, L_ref)
        dQ_ref, dK_ref, dV_ref = oracle.attention_backward_gqa(*bits, w.scale, True)
        _grad_check([("dQ", dq[b:b + 1, hs], dQ_ref), ("dK", dk[b:b + 1, kv:kv + 1], dK_ref),
                     ("dV", dv[b:b + 1, kv:kv + 1], dV_ref)])
    record(groups_checked=3)


def test_fwdbwd_padded_heads():
    """4x16x2048x64 causal with real lengths 2048/1536/1024/512: forward and
    backward of one whole head per batch against the oracle, and exact zeros
    on every padding row of O, LSE, dQ, dK and dV."""
    w = FWDBWD
    lens = [w.N, 3 * w.N // 4, w.N // 2, w.N // 4]
    Q, dO = _gen((w.B, w.H, w.N, w.d), 20), _gen((w.B, w.H, w.N, w.d), 21)
    K, V = _gen((w.B, w.H, w.N, w.d), 24), _gen((w.B, w.H, w.N, w.d), 25)
    q, k, v, do = (t.cuda() for t in (Q, K, V, dO))
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = binding.forward(q, k, v, causal=True, scale=w.scale, seqlens=sl)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=True, scale=w.scale, seqlens=sl)
    _ok()
    for b, n in enumerate(lens):
        for t in (o, lse, dq, dk, dv):
            assert not t[b, :, n:].any(), f"batch {b}: padding rows not zero"
        h = (5 * b + 3) % w.H
        bits = [bf16_bits(t[b:b + 1, h:h + 1].contiguous()) for t in (Q, K, V, dO)]
        O_ref, L_ref = oracle.attention_forward_varlen(*bits[:3], [n], w.scale, True)
        _fwd_compare(o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], O_ref, L_ref)
        refs = oracle.attention_backward_varlen(*bits, [n], w.scale, True)
        _grad_check([(nm, g[b:b + 1, h:h + 1], r)
                     for nm, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs)])
    record(heads_checked=w.B)


def test_fwdbwd_deterministic_heads():
    """The deterministic backward of the 4x16x2048x64 causal workload: two
    whole heads against the oracle, and the same bits on a second run."""
    w = FWDBWD
    x = workload_inputs(w, seed=0)
    q, k, v, do = (x[n].cuda() for n in ("Q", "K", "V", "dO"))
    o, lse = binding.forward(q, k, v, causal=True, scale=w.scale)
    g1 = binding.backward(q, k, v, o, do, lse, causal=True, scale=w.scale, deterministic=True)
    g2 = binding.backward(q, k, v, o, do, lse, causal=True, scale=w.scale, deterministic=True)
    _ok()
    for a, b2 in zip(g1, g2):
        assert torch.equal(a, b2)
    for (b, h) in [(0, w.H - 1), (w.B - 1, 0)]:
        bits = [bf16_bits(x[n][b:b + 1, h:h + 1].contiguous()) for n in ("Q", "K", "V", "dO")]
        refs = oracle.attention_backward(*bits, w.scale, True)
        _grad_check([(nm, g[b:b + 1, h:h + 1], r)
                     for nm, g, r in zip(("dQ", "dK", "dV"), g1, refs)])
    record(heads_checked=2)
