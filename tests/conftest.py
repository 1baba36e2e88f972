import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a) and the CUDA library")


# Order of the GPU test files: the routing parity first, then the rows built on routing, so
# that under -x a failure in a later row cannot hide an earlier row's results.  The test of
# the allocation-free entry point runs last of all.
GPU_FILE_ORDER = ("test_gpu_parity", "test_gpu_train_stats", "test_gpu_dispatch", "test_gpu_variant_cluster",
                  "test_gpu_training_backward", "test_gpu_variant_dispatch", "test_gpu_fullrank", "test_gpu_wait_timeout",
                  "test_zz_no_alloc")


def pytest_collection_modifyitems(config, items):
    rank = {name: i for i, name in enumerate(GPU_FILE_ORDER)}

    def file_rank(item):
        mod = getattr(item, "module", None)
        return rank.get(mod.__name__.rsplit(".", 1)[-1] if mod is not None else "", -1)

    items.sort(key=file_rank)  # stable: the other files keep their order, ahead of these
    # GPU tests are selected with -m gpu; without a GPU they are skipped instead of failing.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
