import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def build_library():
    """Compile libmoe_b200.so when its sources are newer.  build.py is loaded
    by path: the package itself refuses to import until the library exists."""
    import importlib.util
    path = os.path.join(ROOT, "int4_expert_grouped_b200", "build.py")
    spec = importlib.util.spec_from_file_location("moe_libbuild", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="session")
def built_library():
    return build_library()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    # gpu tests cannot run without a GPU; fail loudly instead of skipping when
    # a GPU is present but the library is missing (handled in the tests).
    pass
