import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


@pytest.fixture(params=["per_item", "persistent"])
def bwd_kernel(request):
    """Runs the test once with each form of the attention backward kernel
    forced (process-wide), and restores the window-size dispatch after."""
    import windowed_attention_implicit_b200 as R
    from windowed_attention_implicit_b200 import _abi
    which = {"per_item": _abi.RIB_BWD_PER_ITEM, "persistent": _abi.RIB_BWD_PERSISTENT}
    R.rib_set_bwd_kernel(which[request.param])
    yield request.param
    R.rib_set_bwd_kernel(_abi.RIB_BWD_AUTO)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_sessionfinish(session, exitstatus):
    """With RIB_PARITY_LOG set, every parity comparison of the run (absolute
    and normalised error figures) is written there as JSON lines."""
    path = os.environ.get("RIB_PARITY_LOG")
    if not path:
        return
    try:
        from tests.rib_testlib import RECORDS
    except Exception:  # pragma: no cover
        return
    import json
    with open(path, "w") as f:
        for r in RECORDS:
            f.write(json.dumps(r) + "\n")
