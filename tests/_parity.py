"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare with the fp64 oracle on the same seeded bf16 inputs."""
import math
import os

import numpy as np
import torch

import oracle
from io_aware_exact_31_b200 import binding
from io_aware_exact_31_b200.workloads import bf16_bits, make_inputs

# Acceptance bands: max |O - O_ref| <= 2e-2 beyond the bf16 rounding of O_ref
# (see o_error), max |LSE - LSE_ref| <= 1e-3, and
# max |dX - dX_ref| / max |dX_ref| <= 5e-2 for dX in dQ, dK, dV.
TOL_O = 2e-2
TOL_LSE = 1e-3
TOL_GRAD_REL = 5e-2


# Largest errors seen by each test of this session, kept so that the raw
# max |O - O_ref| (which the bands do not bound by themselves, see o_error) is
# on record beside the banded figure.  conftest.py prints the table at the
# end of the run and writes it as JSON to $FA_PARITY_RECORD when that is set.
RECORD = {}


def record(**errs):
    test = os.environ.get("PYTEST_CURRENT_TEST", "(outside pytest)").split(" ")[0]
    rec = RECORD.setdefault(test, {})
    for k, v in errs.items():
        rec[k] = max(rec.get(k, 0.0), float(v))


def inputs(B, H, N, d, seed=0, input_scale=1.0, with_dO=False):
    return make_inputs(B, H, N, d, seed=seed, input_scale=input_scale, with_dO=with_dO)


def gpu_forward(x, causal, scale):
    q, k, v = (x[n].cuda() for n in ("Q", "K", "V"))
    o, lse = binding.forward(q, k, v, causal=causal, scale=scale)
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"
    return o, lse


def bf16_rounding_distance(O_ref):
    """|bf16(O_ref) - O_ref| elementwise: the error any bf16 output must carry
    (up to 1/32 where |O_ref| >= 8, beyond the 2e-2 band by itself)."""
    t = torch.from_numpy(np.ascontiguousarray(O_ref))
    return np.abs(t.to(torch.bfloat16).double().numpy() - O_ref)


def o_error(o_gpu, O_ref):
    """(raw max |O - O_ref|, max of |O - O_ref| beyond the output rounding).
    The O band applies to the second: O is delivered in bf16, so the error is
    measured on top of the distance from O_ref to its nearest bf16 value."""
    diff = np.abs(o_gpu - O_ref)
    raw = float(np.max(diff)) if diff.size else 0.0
    adj = float(np.max(diff - bf16_rounding_distance(O_ref))) if diff.size else 0.0
    record(o_raw=raw, o_beyond_bf16=adj)
    return raw, adj


def fwd_errors(o, lse, O_ref, L_ref):
    _, eo = o_error(o.double().cpu().numpy(), O_ref)
    el = float(np.max(np.abs(lse.double().cpu().numpy() - L_ref)))
    record(lse=el)
    return eo, el


def check_forward_full(B, H, N, d, causal, seed=0, input_scale=1.0):
    x = inputs(B, H, N, d, seed, input_scale)
    scale = 1.0 / math.sqrt(d)
    o, lse = gpu_forward(x, causal, scale)
    O_ref, L_ref = oracle.attention_forward(bf16_bits(x["Q"]), bf16_bits(x["K"]),
                                            bf16_bits(x["V"]), scale, causal)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    eo, el = fwd_errors(o, lse, O_ref, L_ref)
    assert eo <= TOL_O and el <= TOL_LSE, f"max|dO|={eo:.3e} max|dLSE|={el:.3e}"
    return eo, el


def sample_rows(B, H, N, n_random, seed=1):
    """Row ids bh*N+i, stratified so that every CTA of the launch is checked:
    per head, the first and last row of every 128-row tile and one random row
    inside it, plus n_random random rows of the head."""
    r = np.random.default_rng(seed)
    rows = []
    for bh in range(B * H):
        pick = set()
        for t0 in range(0, N, 128):
            t1 = min(t0 + 128, N)
            pick.update((t0, t1 - 1, int(r.integers(t0, t1))))
        pick.update(int(v) for v in r.choice(N, size=min(n_random, N), replace=False))
        rows.extend(bh * N + i for i in sorted(pick))
    return np.array(rows, np.int64)


def check_forward_sampled(B, H, N, d, causal, input_scale=1.0, n_random=8, seed=0):
    x = inputs(B, H, N, d, seed, input_scale)
    scale = 1.0 / math.sqrt(d)
    o, lse = gpu_forward(x, causal, scale)
    rows = sample_rows(B, H, N, n_random)
    O_ref, L_ref = oracle.attention_forward_rows(bf16_bits(x["Q"]), bf16_bits(x["K"]),
                                                 bf16_bits(x["V"]), scale, causal, rows)
    o_rows = o.reshape(-1, d)[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    l_rows = lse.reshape(-1)[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    _, eo = o_error(o_rows, O_ref)
    el = float(np.max(np.abs(l_rows - L_ref)))
    record(lse=el, rows_checked=rows.size)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert eo <= TOL_O and el <= TOL_LSE, f"max|dO|={eo:.3e} max|dLSE|={el:.3e}"
    return eo, el


def grad_rel_err(g, ref):
    """max |g - ref| / max |ref|; the denominator is floored at 1.0 for
    gradients that vanish identically (N = 1 gives dQ = dK = 0)."""
    g = g.double().cpu().numpy()
    denom = float(np.max(np.abs(ref)))
    e = float(np.max(np.abs(g - ref))) / (denom if denom > 0 else 1.0)
    record(grad_rel=e)
    return e


def check_backward(B, H, N, d, causal, seed=0, heads=None):
    """GPU forward + backward; oracle backward on all heads or on `heads`
    (list of (b, h)); each head's gradient depends only on that head."""
    x = inputs(B, H, N, d, seed, with_dO=True)
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("Q", "K", "V", "dO"))
    o, lse = binding.forward(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = binding.backward(q, k, v, o, do, lse, causal=causal, scale=scale)
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    errs = {}
    for name, g in (("dQ", dq), ("dK", dk), ("dV", dv)):
        assert torch.isfinite(g.float()).all(), f"{name} not finite"
    for (b, h) in sel:
        sl = lambda t: t[b:b + 1, h:h + 1].contiguous()  # noqa: E731
        ref = oracle.attention_backward(*(bf16_bits(sl(x[n])) for n in ("Q", "K", "V", "dO")),
                                        scale, causal)
        for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
            e = grad_rel_err(g[b:b + 1, h:h + 1], r)
            errs[name] = max(errs.get(name, 0.0), e)
    record(heads_checked=len(sel), **errs)
    for name, e in errs.items():
        assert e <= TOL_GRAD_REL, f"{name} rel err {e:.3e} (all: {errs})"
    return errs
