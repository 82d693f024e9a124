import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """The parity maxima every GPU comparison recorded (tests/gpu_common.py): per workload,
    the output error against the oracle it is held to, and the LSE error against the pure
    and the staged fp64 oracle."""
    mod = sys.modules.get("tests.gpu_common")
    log = getattr(mod, "PARITY_LOG", None)
    if not log:
        return

    def f(v):
        return "-" if v is None else f"{v:.3e}"

    terminalreporter.write_sep("-", "parity maxima (out vs oracle; lse vs pure / staged oracle)")
    for r in log:
        terminalreporter.write_line(f"{r['what'][:70]:<70} out max {f(r.get('out_max'))} mean {f(r.get('out_mean'))}"
                                    f"  lse pure {f(r.get('lse_pure'))} staged {f(r.get('lse_staged'))}")
