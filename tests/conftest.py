import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long CPU test")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


# The Qwen3-8B-shaped model of the GPU tests, drawn once per session (about a minute of
# host time and 19.4 GB): host arrays for the oracle, device tensors for the library.
@pytest.fixture(scope="session")
def qwen_host_weights():
    import synth
    return synth.make_weights(synth.QWEN3_8B, 11, 12)


@pytest.fixture(scope="session")
def qwen_device_weights(qwen_host_weights):
    from shared_kv_draft_b200 import orthrus
    return {k: orthrus.upload(v) for k, v in qwen_host_weights.items()}
