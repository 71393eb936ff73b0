import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def _build_library():
    """Compile libpaged_kv.so in-tree if it is missing or older than its
    sources (nvcc cross-compiles; no GPU needed)."""
    import importlib.util
    path = os.path.join(ROOT, "paged_kv_cache_371_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_pkv_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    _build_library()


def read_golden(name):
    """Parse a golden fixture: '#' comments, 'key: values' lines or bare rows."""
    rows, keyed = [], []
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                keyed.append((k.strip(), v.split()))
            else:
                rows.append(line.split())
    return rows, keyed


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.lib()
