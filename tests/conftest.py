import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_terminal_summary(terminalreporter):
    """Whole-layer output errors against the oracle (relative Frobenius and max-abs), the
    worst per case, when the session ran any GPU parity check."""
    mp = sys.modules.get("moe_parity")
    rep = getattr(mp, "LAYER_REPORT", None) if mp is not None else None
    if not rep:
        return
    worst = {}
    for r in rep:
        w = worst.setdefault(r["case"], dict(r))
        if r["rel_fro"] > w["rel_fro"]:
            w.update(rel_fro=r["rel_fro"])
        w["max_abs"] = max(w["max_abs"], r["max_abs"])
    full = [w for w in worst.values() if w["case"].startswith("full:")]
    tr = terminalreporter
    tr.write_line(f"layer output vs oracle: {len(rep)} checks over {len(worst)} cases, worst "
                  f"rel-Frobenius {max(w['rel_fro'] for w in worst.values()):.3g}, worst max-abs "
                  f"{max(w['max_abs'] for w in worst.values()):.3g}")
    for w in full:
        tr.write_line(f"  {w['case']}: {w['tokens']} tokens, rel-Frobenius {w['rel_fro']:.3g} "
                      f"(tol {w['tol']:g}), max-abs {w['max_abs']:.3g} (max |out| "
                      f"{w['max_abs_ref']:.3g})")
