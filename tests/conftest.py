"""Shared test configuration.

``-m gpu`` tests need a B200 and the built CUDA library; everything else runs
on CPU.  The CPU oracle (``oracle/``) is test infrastructure and is imported
only from tests, the smoke check and the benchmark's CPU arms.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a) and the built libtfq.so")
    config.addinivalue_line("markers", "slow: full-size parity cases (minutes)")


def pytest_report_header(config):
    override = os.environ.get("TFQ_ORACLE_LIB")
    if override:
        return f"oracle library override (TFQ_ORACLE_LIB): {override}"
    return None


@pytest.fixture(autouse=True)
def _no_oracle_override_under_gpu_parity(request):
    """The GPU parity tests compare against the built oracle only: with
    TFQ_ORACLE_LIB set (the mutation test's way of loading a planted
    mistake) they fail instead of checking against another library."""
    if request.node.get_closest_marker("gpu") is not None and os.environ.get("TFQ_ORACLE_LIB"):
        pytest.fail("TFQ_ORACLE_LIB is set: GPU parity tests run only against the built oracle")


def pytest_terminal_summary(terminalreporter):
    """The GEMM parity figures of the run: per tolerance check, the outputs
    compared, E_max = max |y - y_ref|, E_rel = ||y - y_ref|| / ||y_ref|| and the
    worst ratio of error to the bound 2^-7 |y_ref| + 1e-3 rms(y_ref)."""
    gpu = sys.modules.get("tests._gpu")
    records = getattr(gpu, "PARITY_RECORDS", None)
    if not records:
        return
    tr = terminalreporter
    tr.section("GEMM tolerance checks (the oracle unless the label names another reference)")
    tr.write_line(f"{'check':<48} {'outputs':>11} {'E_max':>10} {'E_rel':>10} {'err/bound':>9}")
    for what, n, e_max, e_rel, worst in records:
        tr.write_line(f"{what[:48]:<48} {n:>11} {e_max:>10.3e} {e_rel:>10.3e} {worst:>9.3f}")
    tr.write_line(f"{len(records)} checks; worst err/bound {max(r[4] for r in records):.3f}")
