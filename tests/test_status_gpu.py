"""Bounded waits: a wait that nothing will ever satisfy runs out, records ETA_DEV_TIMEOUT and returns;
the context stays usable afterwards.  No fault, trap or hang is involved."""
import pytest
import torch

import exact_tiled_attention_43_b200 as eta

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_bounded_and_reported():
    assert eta.status() == 0
    eta.set_wait_timeout_ns(20_000_000)  # 20 ms
    try:
        eta.selftest_wait_timeout()
        assert eta.status() == eta.ETA_DEV_TIMEOUT
    finally:
        eta.set_wait_timeout_ns(0)  # default
    # the context still works
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
    assert eta.status() == 0
