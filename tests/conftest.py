import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionfinish(session, exitstatus):
    """Writes the observed agreement of the parity checks (kvc_testutil.OBSERVED)
    to the file named by KVC_PARITY_LOG, if set."""
    path = os.environ.get("KVC_PARITY_LOG")
    if not path:
        return
    try:
        import json

        import kvc_testutil
    except Exception:
        return
    with open(path, "w") as f:
        json.dump(kvc_testutil.OBSERVED, f, indent=0)
