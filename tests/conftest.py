import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Per-test error figures of the parity tests (max-abs / relative-L2 against the
# oracle), written as JSON to $FA_PARITY_REPORT at the end of the session when
# that variable is set, so the margins below each tolerance can be read back.
_PARITY = {}


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionfinish(session, exitstatus):
    path = os.environ.get("FA_PARITY_REPORT")
    if path and _PARITY:
        os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
        with open(path, "w") as f:
            json.dump(_PARITY, f, indent=1, sort_keys=True)


@pytest.fixture
def parity_record(request):
    """parity_record(name=value, ...) stores error figures under the test's id."""
    def record(**kw):
        _PARITY.setdefault(request.node.nodeid, {}).update(kw)
    return record


def has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # pragma: no cover
        return False


@pytest.fixture(scope="session")
def lib():
    """The C-ABI library, built in-tree if it is missing or stale (unless
    FA_B200_LIBRARY names another build to load)."""
    from io_aware_exact_20_b200 import build as _build
    if not os.environ.get("FA_B200_LIBRARY"):
        _build.ensure_built()
    import io_aware_exact_20_b200 as fa
    return fa
