"""fa_backward_noalloc: the backward pass for callers that cannot allocate
device memory (code under an allocator that owns the whole GPU, or a
latency-critical path that cannot take a cudaMalloc's synchronisation).  Its
scratch is a fixed array inside the library instead of a caller workspace.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test.  Checked against the regular
fa_backward entry point on the same inputs, within the backward band the
parity tests use, on two calls in a row with different shapes, so that what
the first call leaves in the shared array cannot leak into the second; and
once directly against the fp64 oracle, so that a fault shared by both entry
points would not pass unseen.
"""
import ctypes
import math

import pytest
import torch

import oracle
from io_aware_exact_31_b200 import binding
from io_aware_exact_31_b200.workloads import bf16_bits

from _parity import TOL_GRAD_REL, grad_rel_err, inputs

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, k, v, o, do, lse, dq, dk, dv, causal, scale):
    B, H, N, d = q.shape
    return lib.fa_backward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                   dv.data_ptr(), B, H, N, d, scale, int(causal),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _rel(a, b):
    a, b = a.float(), b.float()
    return float((a - b).abs().max()) / max(float(b.abs().max()), 1e-30)


@pytest.mark.parametrize("first,second", [
    ((2, 3, 700, 64, True, 21), (1, 2, 300, 128, False, 22)),
    ((4, 16, 2048, 64, True, 23), (1, 1, 129, 64, False, 24)),
])
def test_noalloc_matches_fa_backward_on_two_calls(first, second):
    lib = binding.load_library()
    for (B, H, N, d, causal, seed) in (first, second):
        assert binding.backward_workspace_bytes(B, H, N, d) <= binding.NOALLOC_MAX_SCRATCH_BYTES
        x = inputs(B, H, N, d, seed=seed, with_dO=True)
        q, k, v, do = (x[n].cuda() for n in ("Q", "K", "V", "dO"))
        scale = 1.0 / math.sqrt(d)
        o, lse = binding.forward(q, k, v, causal=causal, scale=scale)
        ref = binding.backward(q, k, v, o, do, lse, causal=causal, scale=scale)
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        st = _noalloc(lib, q, k, v, o, do, lse, *got, causal, scale)
        assert st == binding.FA_OK, binding.status_str(st)
        st, site = binding.check_device_error()
        assert st == binding.FA_OK, f"device error {site:#x}"
        for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
            assert torch.isfinite(g.float()).all(), name
            e = _rel(g, r)
            assert e <= TOL_GRAD_REL, f"{name}: rel diff {e:.3e} vs fa_backward"


def test_noalloc_matches_the_oracle():
    lib = binding.load_library()
    B, H, N, d, causal = 1, 2, 333, 64, True
    x = inputs(B, H, N, d, seed=25, with_dO=True)
    q, k, v, do = (x[n].cuda() for n in ("Q", "K", "V", "dO"))
    scale = 1.0 / math.sqrt(d)
    o, lse = binding.forward(q, k, v, causal=causal, scale=scale)
    got = [torch.full_like(q, float("nan")) for _ in range(3)]
    st = _noalloc(lib, q, k, v, o, do, lse, *got, causal, scale)
    assert st == binding.FA_OK, binding.status_str(st)
    st, site = binding.check_device_error()
    assert st == binding.FA_OK, f"device error {site:#x}"
    refs = oracle.attention_backward(*(bf16_bits(x[n]) for n in ("Q", "K", "V", "dO")), scale,
                                     causal)
    for name, g, r in zip(("dQ", "dK", "dV"), got, refs):
        e = grad_rel_err(g, r)
        assert e <= TOL_GRAD_REL, f"{name}: rel err {e:.3e} vs the oracle"


def test_noalloc_rejects_problems_beyond_its_array():
    lib = binding.load_library()
    B, H, N, d = 1, 1, 300_000, 128
    assert binding.backward_workspace_bytes(B, H, N, d) > binding.NOALLOC_MAX_SCRATCH_BYTES
    t = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    p = t.data_ptr()
    st = lib.fa_backward_noalloc(p, p, p, p, p, p, p, p, p, B, H, N, d, 0.1, 0,
                                 ctypes.c_void_p(0))
    assert st == binding.FA_ERR_UNSUPPORTED
