import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """The parity margins: the largest err/limit ratios of the comparisons that ran."""
    from helpers import RATIOS
    if not RATIOS:
        return
    tr = terminalreporter
    tr.section("parity margins (worst err / limit per comparison, largest first)")
    for what, dtype, worst in sorted(RATIOS, key=lambda r: -r[2])[:25]:
        tr.write_line(f"{worst:7.3f}  {dtype:4s}  {what}")
    tr.write_line(f"{len(RATIOS)} comparisons")
