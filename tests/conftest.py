import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_sessionstart(session):
    # the tests exercise the CUDA library and the C oracle as built from the
    # current sources: (re)build either when it is missing or older than them
    from lora_adapter_execution_b200 import build as cuda_build
    import oracle
    cuda_build.build()
    oracle.build()
