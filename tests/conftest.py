import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_terminal_summary(terminalreporter):
    parity = sys.modules.get("tests.parity")
    rows = getattr(parity, "HEADROOM", None) if parity else None
    if not rows:
        return
    terminalreporter.write_line("largest errors seen / bounds (scaled by max(1, |ref|)):")
    for name, (mx, mxb, mean, meanb) in sorted(rows.items()):
        terminalreporter.write_line(f"  {name}: max {mx:.3e} of {mxb:.0e} ({100 * mx / mxb:.0f} %), "
                                    f"mean {mean:.3e} of {meanb:.0e} ({100 * mean / meanb:.0f} %)")
