"""The bounded-wait path: a kernel that waits on a barrier nothing completes
gives up after the wait limit, records WP_ERR_TIMEOUT in the device status
word and returns; the context stays usable. No fault, trap or hang."""
import pytest
import torch

import rope_period_truncated_b200 as wp

pytestmark = pytest.mark.gpu


def test_wait_limit_reports_timeout_and_context_survives():
    assert wp.wp_device_status() == wp.WP_OK
    prev = wp.wp_set_wait_limit(200_000)  # ~0.1 ms of SM clock
    try:
        wp.wp_wait_probe()
        assert wp.wp_device_status() == wp.WP_ERR_TIMEOUT
        assert wp.wp_device_status() == wp.WP_OK  # reading clears it
    finally:
        wp.wp_set_wait_limit(prev)
    # the context still runs real work
    q = torch.randn(1, 256, 2, 64, device="cuda").to(torch.bfloat16)
    k = torch.randn(1, 256, 2, 64, device="cuda").to(torch.bfloat16)
    o, _ = wp.wp_prefill(q, k, k, None)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert wp.wp_device_status() == wp.WP_OK
