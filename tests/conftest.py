import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")

TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_sessionfinish(session, exitstatus):
    """With FFTCONV_PARITY_LOG=<path>, write every parity check's errors as JSON lines."""
    path = os.environ.get("FFTCONV_PARITY_LOG")
    if not path:
        return
    try:
        import json
        import parity
    except Exception:
        return
    with open(path, "w") as f:
        for what, dtype, rel, mx, rms, n in parity.RECORD:
            f.write(json.dumps({"check": what, "dtype": dtype, "rel_l2": rel, "max_abs": mx, "rms_ref": rms,
                                "n": n}) + "\n")
