"""Randomised parity sweep: forward and backward of the CUDA path against the
fp64 oracle on configurations that combine the features -- grouped-query
heads, padded batches (zero-length batches included), attention dropout,
causal masking, both head dimensions, ragged N and widened score ranges --
drawn from a fixed seed, so every run checks the same cases."""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_31_b200 import binding
from io_aware_exact_31_b200.workloads import bf16_bits

from _parity import TOL_GRAD_REL, TOL_LSE, TOL_O, grad_rel_err, o_error, record

pytestmark = pytest.mark.gpu

HEADS = [(1, 1), (2, 1), (2, 2), (4, 1), (4, 2), (4, 4), (6, 3), (6, 2)]


def _cases(n=24, seed=2026):
    r = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        B = int(r.integers(1, 4))
        H, Hkv = HEADS[int(r.integers(len(HEADS)))]
        N = int(r.integers(1, 601))
        d = int(r.choice([64, 128]))
        causal = bool(r.integers(2))
        seqlens = None
        if r.random() < 0.35:
            seqlens = [int(r.integers(0, N + 1)) for _ in range(B)]
            seqlens[int(r.integers(B))] = N  # at least one full batch
            if B > 1 and r.random() < 0.3:
                seqlens[0] = 0
        p = float(r.choice([0.1, 0.3, 0.6])) if r.random() < 0.3 else 0.0
        xs = 2.0 if r.random() < 0.3 else 1.0
        out.append((B, H, Hkv, N, d, causal, seqlens, p, xs))
    # Two fixed combinations the draw above does not happen to contain: a
    # zero-length batch, and dropout together with padding.
    out.append((3, 4, 2, 333, 64, True, [0, 333, 120], 0.2, 1.0))
    out.append((2, 6, 3, 129, 128, False, [129, 1], 0.5, 2.0))
    return out


def _id(c):
    B, H, Hkv, N, d, causal, seqlens, p, xs = c
    return (f"B{B}H{H}k{Hkv}N{N}d{d}{'c' if causal else ''}"
            f"{'v' if seqlens else ''}{f'p{p}' if p else ''}{'x2' if xs != 1 else ''}")


@pytest.mark.parametrize("case", _cases(), ids=_id)
def test_random_configuration_matches_oracle(case):
    B, H, Hkv, N, d, causal, seqlens, p, xs = case
    g = torch.Generator().manual_seed(N * 131 + d + H)
    mk = lambda h: (torch.randn(B, h, N, d, generator=g) * xs).to(torch.bfloat16)  # noqa: E731
    Q, K, V, dO = mk(H), mk(Hkv), mk(Hkv), mk(H)
    scale = 1.0 / math.sqrt(d)
    seed, offset = 1000 + N, 3
    q, k, v, do = (t.cuda() for t in (Q, K, V, dO))
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda") if seqlens else None
    o, lse = binding.forward(q, k, v, causal=causal, scale=scale, seqlens=sl, dropout_p=p,
                             seed=seed, offset=offset)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=causal, scale=scale, seqlens=sl,
                                  dropout_p=p, seed=seed, offset=offset)
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"

    bits = [bf16_bits(t) for t in (Q, K, V, dO)]
    O_ref, L_ref = oracle.attention_forward_dropout(*bits[:3], scale, causal, p, seed, offset,
                                                    seqlens=seqlens)
    _, eo = o_error(o.double().cpu().numpy(), O_ref)
    el = float(np.max(np.abs(lse.double().cpu().numpy() - L_ref)))
    record(lse=el)
    assert eo <= TOL_O and el <= TOL_LSE, f"max|dO|={eo:.3e} max|dLSE|={el:.3e}"
    refs = oracle.attention_backward_dropout(*bits, scale, causal, p, seed, offset,
                                             seqlens=seqlens)
    for name, gr, ref in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        e = grad_rel_err(gr, ref)
        assert e <= TOL_GRAD_REL, f"{name}: rel err {e:.3e}"
