"""Failure detection on the GPU without faulting it: a bounded wait runs out
on a barrier nothing arrives at, the kernel records a timeout code and
returns, the host reads FA_ERR_TIMEOUT, and the context stays usable."""
import math

import pytest
import torch

from io_aware_exact_31_b200 import binding

from _parity import check_forward_full

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    st, site = binding.selftest_bounded_wait(20_000_000)  # 20 ms
    assert st == binding.FA_ERR_TIMEOUT
    assert site == 0x163
    # the error word is cleared by the read
    assert binding.check_device_error() == (binding.FA_OK, 0)


def test_context_usable_after_timeout():
    binding.selftest_bounded_wait(5_000_000)
    check_forward_full(1, 2, 300, 64, True, seed=31)
    assert binding.check_device_error() == (binding.FA_OK, 0)


def test_selftest_rejects_unbounded_limits():
    lib = binding.load_library()
    assert lib.fa_selftest_bounded_wait(0, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_selftest_bounded_wait(2_000_000_000, None) == binding.FA_ERR_INVALID_ARG
