import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")


@pytest.fixture(params=[2, 1], ids=["pair_kernel", "block_kernel"])
def attn_kernel(request):
    """Runs a GPU attention test with each head_dim-128 kernel in every mode: 2 = one CTA per query-block
    pair, 1 = one CTA per query block (head_dim 64 always uses the latter)."""
    from int8_kv_cache_action_b200 import _nomas as N
    prev = N.nomas_set_attn_kernel(request.param)
    yield request.param
    N.nomas_set_attn_kernel(prev)
