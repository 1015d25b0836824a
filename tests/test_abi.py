"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/fa.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re
import subprocess

import pytest

from io_aware_exact_31_b200 import binding
from io_aware_exact_31_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return binding.load_library()


def declared_functions():
    with open(os.path.join(ROOT, "include", "fa.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    assert set(binding.EXPORTS) <= set(names), names


def test_noalloc_limit_matches_the_header():
    """The binding's copy of the no-allocation backward's array size is the
    header's FA_BACKWARD_NOALLOC_MAX_SCRATCH_BYTES."""
    with open(os.path.join(ROOT, "include", "fa.h")) as f:
        m = re.search(r"#define\s+FA_BACKWARD_NOALLOC_MAX_SCRATCH_BYTES\s+\(([^)]*)\)", f.read())
    assert m, "macro not found"
    expr = m.group(1).replace("u", "")
    assert re.fullmatch(r"[0-9* ]+", expr), expr
    value = 1
    for factor in expr.split("*"):
        value *= int(factor)
    assert value == binding.NOALLOC_MAX_SCRATCH_BYTES


def test_every_declared_function_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fa_[a-z_0-9]+)\b", out))
    for name in declared_functions():
        assert name in exported, f"{name} declared in include/fa.h but not exported"
        assert hasattr(lib, name)


def test_library_does_not_link_the_oracle(lib):
    out = subprocess.run(["nm", "-D", binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    assert "oracle_" not in out


def test_status_strings(lib):
    for st in range(5):
        assert lib.fa_status_str(st)
    assert lib.fa_version() >= 100


def _fwd(lib, q=16, k=16, v=16, o=16, lse=16, B=1, H=1, N=8, d=64, scale=0.125, causal=0):
    return lib.fa_forward(q, k, v, o, lse, B, H, N, d, scale, causal, None)


def test_forward_rejects_bad_arguments_without_a_device(lib):
    assert _fwd(lib, q=None) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, lse=None) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, v=24) == binding.FA_ERR_INVALID_ARG          # not 16-byte aligned
    assert _fwd(lib, N=0) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, B=-1) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=-1.0) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("inf")) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, d=96) == binding.FA_ERR_UNSUPPORTED
    assert _fwd(lib, d=256) == binding.FA_ERR_UNSUPPORTED
    assert _fwd(lib, B=1 << 20, H=1 << 10, N=4096) == binding.FA_ERR_UNSUPPORTED


def test_backward_rejects_bad_arguments_without_a_device(lib):
    p = [16] * 10

    def bwd(ptrs=p, ws=1 << 30, B=1, H=1, N=8, d=64, scale=0.125):
        return lib.fa_backward(*ptrs, ws, B, H, N, d, scale, 0, None)

    assert bwd(ptrs=[None] + p[1:]) == binding.FA_ERR_INVALID_ARG
    assert bwd(ptrs=p[:9] + [None]) == binding.FA_ERR_INVALID_ARG
    assert bwd(ptrs=p[:3] + [8] + p[4:]) == binding.FA_ERR_INVALID_ARG
    assert bwd(ws=16) == binding.FA_ERR_INVALID_ARG
    assert bwd(d=32) == binding.FA_ERR_UNSUPPORTED
    assert bwd(N=0) == binding.FA_ERR_INVALID_ARG


def test_workspace_size_formula(lib):
    # D and LSE2 (fp32) plus the fp32 dQ accumulator, rows padded to 128 per
    # head, then one int32 counter per 128-row query block padded to 256 bytes
    assert lib.fa_backward_workspace_bytes(2, 3, 200, 64) == 2 * 3 * 256 * (4 + 4 + 64 * 4) + 256
    assert lib.fa_backward_workspace_bytes(1, 1, 128, 128) == 128 * (8 + 512) + 256
    assert lib.fa_backward_workspace_bytes(4, 16, 2048, 64) == (
        4 * 16 * 2048 * (8 + 256) + 4 * 16 * 16 * 4)
    assert lib.fa_backward_workspace_bytes(1, 1, 0, 64) == 0


def test_package_exports_resolve():
    """Every public name resolves lazily, before and without loading the library."""
    import importlib
    import sys
    for mod in [m for m in sys.modules if m.startswith("io_aware_exact_31_b200")]:
        del sys.modules[mod]
    pkg = importlib.import_module("io_aware_exact_31_b200")
    for name in pkg.__all__:
        assert getattr(pkg, name) is not None, name


def test_extended_entry_points_reject_bad_arguments_without_a_device(lib):
    """The documented INVALID_ARG / UNSUPPORTED cases of the grouped, padded,
    dropout, E4M3, deterministic, no-alloc and self-test entry points, all
    returned before any device is touched."""
    INV, UNS = binding.FA_ERR_INVALID_ARG, binding.FA_ERR_UNSUPPORTED
    a = [16] * 5  # aligned fake pointers: Q, K, V, O, LSE

    # grouped-query: H_kv must divide H
    assert lib.fa_forward_gqa(*a, 1, 6, 4, 8, 64, 0.125, 0, None) == INV
    assert lib.fa_forward_gqa(*a, 1, 4, 0, 8, 64, 0.125, 0, None) == INV
    # padded batches: seqlens must be 4-byte aligned
    assert lib.fa_forward_varlen(*a, 18, 1, 2, 2, 8, 64, 0.125, 0, None) == INV
    # dropout: p in [0, 1 - 2^-9]
    for pd in (1.0, -0.1, float("nan"), 1.0 - 2.0 ** -17):
        assert lib.fa_forward_dropout(*a, None, 1, 2, 2, 8, 64, 0.125, 0, pd, 1, 0, None) == INV
    assert lib.fa_forward_dropout(None, *a[1:], None, 1, 2, 2, 8, 64, 0.125, 0, 0.1, 1, 0,
                                  None) == INV
    # E4M3: finite positive descales; d = 128 only
    for ds in (0.0, -1.0, float("nan"), float("inf")):
        assert lib.fa_forward_fp8(*a, ds, 1.0, 1.0, 1, 2, 2, 8, 128, 0.125, 0, None) == INV
        assert lib.fa_forward_fp8(*a, 1.0, 1.0, ds, 1, 2, 2, 8, 128, 0.125, 0, None) == INV
    assert lib.fa_forward_fp8(*a, 1.0, 1.0, 1.0, 1, 2, 2, 8, 64, 0.125, 0, None) == UNS
    # backward with dropout: bad p, workspace too small
    p10 = [16] * 10
    assert lib.fa_backward_dropout(*p10, 1 << 30, None, 1, 2, 2, 8, 64, 0.125, 0, 1.0, 1, 0,
                                   None) == INV
    assert lib.fa_backward_dropout(*p10, 16, None, 1, 2, 2, 8, 64, 0.125, 0, 0.1, 1, 0,
                                   None) == INV
    # deterministic backward: the same argument checks as the dropout backward
    assert lib.fa_backward_deterministic(*p10, 1 << 30, None, 1, 2, 2, 8, 64, 0.125, 0, 1.0, 1,
                                         0, None) == INV
    assert lib.fa_backward_deterministic(*p10, 16, None, 1, 2, 2, 8, 64, 0.125, 0, 0.0, 1, 0,
                                         None) == INV
    assert lib.fa_backward_deterministic(*p10, 1 << 30, None, 1, 6, 4, 8, 64, 0.125, 0, 0.0, 1,
                                         0, None) == INV
    assert lib.fa_backward_deterministic(*p10, 1 << 30, None, 1, 2, 2, 8, 80, 0.125, 0, 0.0, 1,
                                         0, None) == UNS
    # no-alloc backward: problems beyond its built-in array are UNSUPPORTED
    p9 = [16] * 9
    assert lib.fa_backward_noalloc(*p9, 64, 16, 4096, 128, 0.088, 1, None) == UNS
    assert lib.fa_backward_noalloc(None, *p9[1:], 1, 1, 8, 64, 0.125, 0, None) == INV
    # bounded-wait self-test: limit must be in (0, 1 s]
    assert lib.fa_selftest_bounded_wait(0, None) == INV
    assert lib.fa_selftest_bounded_wait(2_000_000_000, None) == INV


def test_python_entry_points_reject_host_tensors():
    """No CPU fallback: every Python entry point refuses tensors that are not
    contiguous bf16 CUDA tensors before anything is launched."""
    import torch
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.forward(q, q, q)
    with pytest.raises(ValueError):
        binding.backward(q, q, q, q, q, torch.zeros(1, 2, 8))
    with pytest.raises(ValueError):
        binding.attention(q, q, q)
    with pytest.raises(ValueError):
        binding.forward(q.float(), q.float(), q.float())
