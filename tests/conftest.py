import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Report the routing-weight errors the GPU parity tests measured."""
    mod = sys.modules.get("parity_util")
    st = getattr(mod, "ROUTING_WEIGHT_STATS", None)
    if st and st["checks"]:
        terminalreporter.write_line(
            f"routing weights: {st['tokens']} tokens in {st['checks']} checks, largest relative "
            f"error {st['max_rel']:.3e}, largest ratio to the per-token bound {st['max_ratio']:.3f}")
