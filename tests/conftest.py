import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")


def pytest_collection_modifyitems(config, items):
    # a GPU test that runs on a host without a GPU fails loudly instead of
    # silently falling back; selecting `-m "not gpu"` skips them.
    pass


def pytest_sessionfinish(session, exitstatus):
    """Writes the worst parity figures the GPU comparisons saw (largest
    intermediate-scale difference, smallest share of identical codes, largest
    output errors) to the JSON file named by MOE_PARITY_STATS, if set."""
    path = os.environ.get("MOE_PARITY_STATS")
    # the helpers are imported as `tests.gpu_helpers` and as `gpu_helpers`:
    # two module objects, each with its own figures
    found = (sys.modules.get("tests.gpu_helpers"), sys.modules.get("gpu_helpers"))
    mods = list({id(m): m for m in found if m is not None}.values())
    if not path or not mods:
        return
    import json
    st = dict(mods[0].STATS)
    for m in mods[1:]:
        for key, v in m.STATS.items():
            st[key] = min(st[key], v) if key.endswith("_min") else (
                st[key] + v if key == "calls" else max(st[key], v))
    with open(path, "w") as f:
        json.dump(st, f, indent=1)


@pytest.fixture(scope="session")
def oracle():
    import oracle as _o
    _o.build()
    return _o
