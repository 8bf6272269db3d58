import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    """The index builder's device tests run after every head test (a stable sort keeps the rest in
    file order), so that under -x a builder failure cannot hide a head result."""
    items.sort(key=lambda item: os.path.basename(str(item.fspath)) == "test_kmeans_gpu.py")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def fh():
    """The CUDA binding; builds the library if it is missing or stale."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_retrieval_classification_b200 import _build
    _build.build()
    from clustered_retrieval_classification_b200 import flashhead
    flashhead.load()
    return flashhead


@pytest.fixture(scope="session")
def llama_host():
    """The Llama-3.2-1B-shaped synthetic index (v=128256, d=2048, c=8016, p=512) and 64 queries,
    built once per session on the host."""
    from clustered_retrieval_classification_b200 import synth
    cfg = synth.CONFIGS["llama"]
    return synth.make_index(cfg), synth.make_queries(cfg, 64)


@pytest.fixture(scope="session")
def gemma_host():
    """The Gemma-3-1B-shaped synthetic index with INT4 Stage-1 centroids (v=262144, d=1152,
    c=16384, p=1024) and 32 queries, built once per session on the host."""
    from clustered_retrieval_classification_b200 import synth
    cfg = synth.CONFIGS["gemma"]
    return synth.make_index(cfg), synth.make_queries(cfg, 32)
