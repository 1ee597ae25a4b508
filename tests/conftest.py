"""Shared pytest setup: the ``gpu`` marker, repo-root imports, and a summary
of the parity margins the GPU tests record (printed even under ``-q``)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# (what, elements compared, max |gpu - ref|, worst err / bound), appended by
# tests.test_gpu_parity.assert_attention_close
PARITY_RECORDS = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not PARITY_RECORDS:
        return
    terminalreporter.section("attention parity margins (full-size and named workloads)")
    for what, n, max_abs, worst in PARITY_RECORDS:
        terminalreporter.write_line(
            f"{what:<44s} elements {n:>10d}  max|err| {max_abs:.3e}  worst err/bound {worst:.4f}")
