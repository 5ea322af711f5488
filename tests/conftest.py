import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Totals of the GPU parity comparisons (tests/gpu_harness.py REPORTS):
    how many units matched exactly, how many differed only in ways the
    parity rules allow (near-cutoff pages, ambiguous query bits), and how the
    attention outputs were checked."""
    try:
        from gpu_harness import QUALITY, REPORTS
    except Exception:  # noqa: BLE001 - the harness needs torch + CUDA
        return
    if QUALITY:
        terminalreporter.write_sep("-", "selection quality (diagnostic): recall of the exact top-k by logit")
        for q in QUALITY:
            terminalreporter.write_line(str(q))
    if not REPORTS:
        return
    keys = ["units", "units_exact", "units_explained", "near_cutoff_pages", "tok_set_diff",
            "q_ambiguous", "attn_vs_oracle", "attn_vs_oracle_on_gpu_idx"]
    tot = {k: sum(r[k] for r in REPORTS) for k in keys}
    worst = max(r["attn_max_err"] for r in REPORTS)
    terminalreporter.write_sep("-", "GPU parity totals")
    terminalreporter.write_line(", ".join(f"{k}={v}" for k, v in tot.items()) +
                                f", attention max-abs error={worst:.2e} over {len(REPORTS)} comparisons")
    for r in REPORTS:
        if r["units_explained"]:
            terminalreporter.write_line(f"  {r['name']}: {r['units_explained']} of {r['units']} units differ "
                                        f"within the rules ({r['near_cutoff_pages']} near-cutoff pages, "
                                        f"{r['tok_set_diff']} tokens, {r['q_ambiguous']} ambiguous query bits)")
