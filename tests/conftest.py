import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: CPU test taking more than ~30 s")


_cache = {}


@pytest.fixture(scope="session")
def workload_data():
    """Seeded synthetic inputs of a named workload, generated once per session."""
    import synth

    def get(name):
        if name not in _cache:
            _cache[name] = synth.make(synth.WORKLOADS[name])
        return _cache[name]

    return get
