"""Shared pytest set-up: the ``gpu`` marker and import paths.

Tests marked ``gpu`` need a CUDA device and the built library; everything else
runs on the CPU (``pytest -m "not gpu"``).
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built libgdr.so")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the parity margins of every comparison the GPU tests made: max |err|, the
    reference RMS and the fraction of the allowed bound used (1.0 = at the bound)."""
    try:
        from gpu_helpers import RECORDS
    except Exception:  # the helpers import the oracle; nothing to report without them
        return
    if not RECORDS:
        return
    tr = terminalreporter
    tr.section("parity margins (fraction of the bound used, worst first)")
    worst = sorted(RECORDS, key=lambda r: -r[4])
    for test, name, err, rms, used in worst[:40]:
        tr.write_line(f"{used:7.3f}  max|err| {err:.3e}  RMS {rms:.3e}  err/RMS {err / rms if rms else 0:.2e}  "
                      f"{test} :: {name}")
    tr.write_line(f"{len(RECORDS)} comparisons; worst fraction {worst[0][4]:.3f}")
    out = os.environ.get("GDR_PARITY_REPORT")
    if out:
        import json
        with open(out, "w") as f:
            json.dump([dict(test=t, name=n, max_err=e, rms=r, used=u) for t, n, e, r, u in RECORDS],
                      f, indent=0)
