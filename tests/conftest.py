import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")


def pytest_sessionstart(session):
    # compile the in-tree library if a source is newer than it (no-op otherwise)
    import importlib
    importlib.import_module("llama_decoder_only_b200.build").build()
