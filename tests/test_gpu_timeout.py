"""Failure detection on the device: a bounded barrier wait that runs out.

The kernels of the library wait on shared-memory barriers with a time limit; when a wait
expires the kernel raises a device error flag and returns instead of spinning forever, and
omq_sync_check reports OMQ_ERR_TIMEOUT. Here a probe kernel waits, with that same wait, on a
barrier that nothing completes, under a short limit: the wait must give up, the status must
say so, the flag must clear, and the context must stay usable for the next call."""
import time

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


def test_expired_wait_reports_timeout_and_context_stays_usable(omq, cuda_device):
    default = omq.wait_limit_ns()
    assert default == 2_000_000_000
    omq.set_wait_limit_ns(50_000_000)            # 50 ms
    try:
        assert omq.wait_limit_ns() == 50_000_000
        omq.wait_probe(True)                     # completed barrier: no error
        omq.sync_check()
        t0 = time.perf_counter()
        omq.wait_probe(False)                    # nothing completes the barrier
        with pytest.raises(omq.OmqError) as err:
            omq.sync_check()
        waited = time.perf_counter() - t0
        assert err.value.status == 9             # OMQ_ERR_TIMEOUT
        assert 0.04 <= waited < 5.0
        omq.sync_check()                         # the flag was cleared by the report
        # the context still runs real work correctly
        W = (torch.randn(64, 256, device=cuda_device) * 0.02).to(torch.bfloat16)
        gl = torch.full((64, 2), 4.0, device=cuda_device)
        out = omq.lwc_quant(W, gl, gl.clone(), bits=4, group=128)
        torch.cuda.synchronize()
        omq.sync_check()
        assert torch.isfinite(out["W_hat"].float()).all()
    finally:
        omq.set_wait_limit_ns(default)
    assert omq.wait_limit_ns() == default


def test_wait_limit_is_range_checked(omq, cuda_device):
    with pytest.raises(omq.OmqError):
        omq.set_wait_limit_ns(10)
    with pytest.raises(omq.OmqError):
        omq.set_wait_limit_ns(10**12)
