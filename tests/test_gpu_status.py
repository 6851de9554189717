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


def test_prefill_writes_nan_rows_while_status_is_set():
    """After a timeout the status word stays set until it is read; prefill
    calls in between skip their work and write NaN to every O row and LSE
    entry (no stale outputs). Once the word is read and cleared, the same
    call computes normally."""
    assert wp.wp_device_status() == wp.WP_OK
    g = torch.Generator().manual_seed(11)
    q = torch.randn(1, 300, 4, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(1, 300, 2, 128, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(1, 300, 2, 128, generator=g).to(torch.bfloat16).cuda()
    prev = wp.wp_set_wait_limit(200_000)
    try:
        wp.wp_wait_probe()  # sets the status word; not read yet
    finally:
        wp.wp_set_wait_limit(prev)
    for mode, cut in [(wp.MODE_GROUPED, None), (wp.MODE_CHANNEL, None)]:
        o = torch.zeros_like(q)  # finite: any row left unwritten would show
        lse = torch.zeros(1, 4, 300, dtype=torch.float32, device="cuda")
        wp.wp_prefill(q, k, v, cut, mode, out=o, lse=lse)
        torch.cuda.synchronize()
        assert torch.isnan(o.float()).all(), f"mode {mode}: some O entries are not NaN"
        assert torch.isnan(lse).all(), f"mode {mode}: some LSE entries are not NaN"
    assert wp.wp_device_status() == wp.WP_ERR_TIMEOUT
    o, lse = wp.wp_prefill(q, k, v, None)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert wp.wp_device_status() == wp.WP_OK
