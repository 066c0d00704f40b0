import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def toy_cfg():
    from workloads import get_config
    return get_config("toy")


@pytest.fixture(scope="session")
def toy_layer(toy_cfg):
    from workloads import make_layer
    return make_layer(toy_cfg)


@pytest.fixture(scope="session")
def toy_codec(toy_cfg, toy_layer):
    import oracle
    return oracle.calibrate(toy_cfg, toy_layer["H_calib"], toy_layer["W_K"], toy_layer["W_V"])
