import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    # temporary files of the tests (tmp_path) stay inside the repository
    if not config.option.basetemp:
        config.option.basetemp = os.path.join(ROOT, "tests", "_tmp")
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")
