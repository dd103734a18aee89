import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter):
    """One line on the selection masks of the GPU parity tests: entries
    compared with the oracle, entries inside the 1e-4 band around the row
    threshold, and disagreements (allowed only there)."""
    mod = sys.modules.get("parity_util")
    if mod is None or not mod.SESSION["mask_entries"]:
        return
    s = mod.SESSION
    terminalreporter.write_line(
        f"mask parity: {s['mask_entries']} entries compared, {s['in_band']} within 1e-4 of the threshold, "
        f"{s['band_mismatch']} in-band disagreements; {s['count_rows']} per-row counts checked against the oracle")
