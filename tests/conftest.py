import gc
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200) and the built CUDA library")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def pytest_collection_modifyitems(config, items):
    # GPU tests cannot run without a device: skip them loudly instead of failing
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(autouse=True)
def pool_guard_blocks(request):
    """GPU tests: every pool destroyed during the test (closed, or collected
    at its end) must leave the guard blocks around its own K/V buffers
    untouched, i.e. no kernel or copy wrote outside the pool."""
    if "gpu" not in request.keywords:
        yield
        return
    import pagedattention_decode_02_b200 as pk
    changed = []
    close = pk.Pool.close

    def checked_close(self):
        if self.handle:
            try:
                if not pk.kv_pool_check_guards(self):
                    changed.append((self.num_blocks, self.block_size, self.head_dim, self.dtype))
            except Exception:
                pass   # no device to check on (e.g. a pool of another device)
        close(self)

    pk.Pool.close = checked_close
    try:
        yield
        gc.collect()
    finally:
        pk.Pool.close = close
    assert not changed, f"guard blocks changed around pools {changed}"
