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
    log = getattr(mod, "PARITY_LOG", None)
    if log:
        w = terminalreporter.write_line
        w(f"output parity: {len(log)} comparisons (max abs / bound, rel Frobenius / bound)")
        worst = max(log, key=lambda r: max(r[1] / r[2], r[3] / r[4]))
        w(f"  largest share of a bound: {worst[0]}: {worst[1]:.3e} / {worst[2]:.3e}, "
          f"{worst[3]:.3e} / {worst[4]:.0e}")
        for what, ma, mb, rel, rb in log:
            if "whole" in what or "sampled" in what:
                w(f"  {what}: {ma:.3e} / {mb:.3e}, {rel:.3e} / {rb:.0e}")
    st = getattr(mod, "ROUTING_WEIGHT_STATS", None)
    if st and st["checks"]:
        terminalreporter.write_line(
            f"routing weights: {st['tokens']} tokens in {st['checks']} checks, largest relative "
            f"error {st['max_rel']:.3e}, largest ratio to the per-token bound {st['max_ratio']:.3f}")
