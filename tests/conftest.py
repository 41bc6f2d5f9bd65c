import os
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running parity case")


def pytest_terminal_summary(terminalreporter):
    """One JSON line per GPU parity case: routing decisions and selected
    blocks excused by the 1e-4 exemption rule (counted, as the parity
    protocol requires), query blocks whose attention was compared, and the
    attention errors; the totals come last."""
    import json
    try:
        import parity_util
    except ImportError:
        return
    reps = parity_util.SESSION_REPORTS
    if not reps:
        return
    terminalreporter.write_sep("-", "parity exemptions (1e-4 rule) per case")
    for r in reps:
        terminalreporter.write_line(json.dumps(r, default=float))
    tot = {"cases": len(reps), "heads": sum(r["heads"] for r in reps),
           "exempt_routes": sum(r["exempt_routes"] for r in reps),
           "exempt_blocks": sum(r["exempt_blocks"] for r in reps),
           "exempt_differing": sum(r.get("exempt_differing", 0) for r in reps),
           "routes_differing": sum(r.get("routes_differing", 0) for r in reps),
           "qblocks_compared": sum(r["qblocks_compared"] for r in reps),
           "attn_max_abs": max(r["attn_max_abs"] for r in reps)}
    terminalreporter.write_line("parity totals: " + json.dumps(tot, default=float))
