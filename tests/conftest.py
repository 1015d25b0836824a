import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Print the largest errors each parity test saw (raw max |O - O_ref|,
    the same beyond the bf16 rounding of O_ref, |LSE| error, gradient
    relative errors), and write them as JSON to $FA_PARITY_RECORD if set."""
    mod = sys.modules.get("_parity")
    rec = getattr(mod, "RECORD", None) if mod else None
    if not rec:
        return
    cols = ["o_raw", "o_beyond_bf16", "fp8_err_over_band", "lse", "grad_rel", "dQ", "dK", "dV", "rows_checked",
            "heads_checked"]
    tr = terminalreporter
    tr.write_sep("-", "parity errors per test (max over the test's checks)")
    tr.write_line("test | " + " | ".join(cols))
    for test in sorted(rec):
        r = rec[test]
        tr.write_line(test + " | " + " | ".join(
            ("%.3e" % r[c] if c not in ("rows_checked", "heads_checked") else "%d" % r[c])
            if c in r else "-" for c in cols))
    path = os.environ.get("FA_PARITY_RECORD")
    if path:
        import json
        with open(path, "w") as f:
            json.dump(rec, f, indent=1, sort_keys=True)
