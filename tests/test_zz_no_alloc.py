"""omq_fq_linear_fwd_noalloc gives what omq_fq_linear_fwd gives.

The no-allocation entry point is for hosts that cannot lend this library device scratch
memory, for example a framework whose memory pool owns every device allocation and gives
plug-ins no allocation hook, or a runtime that forbids device allocation after start-up.
Its scratch (the per-tile partial sums of the squared error) is a fixed array inside the
library, shared by all calls on a device. Two calls in a row, on different problems, must
each match the workspace-based entry point on the same inputs. This file is collected last,
so a run that stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from tests.gpu_common import close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


def _problem(seed, M, N, K, dtype, dev):
    g = torch.Generator().manual_seed(seed)
    Xq = torch.randn(M, K, generator=g).to(dtype)
    W = (torch.randn(N, K, generator=g) * 0.02).to(dtype)
    B = torch.randn(N, generator=g) * 0.1
    Yref = (Xq.double() @ W.double().T + B.double() + 0.05 * torch.randn(M, N, generator=g,
                                                                        dtype=torch.float64))
    return (Xq.to(dev), W.to(dev), B.to(dev), Yref.float().to(dev))


@pytest.mark.parametrize("calls", [[(11, 520, 600, 384, "bf16"), (12, 136, 264, 512, "bf16")],
                                   [(13, 200, 328, 320, "f32"), (14, 72, 136, 256, "f32")]],
                         ids=["bf16", "f32"])
def test_noalloc_forward_matches_workspace_forward(omq, cuda_device, calls):
    """Both entry points run the same kernels, tile order and fixed-order loss reduction, so
    their results agree bit for bit. The first call of each pair is the larger problem: its
    partial sums fill more slots of the shared array than the second call uses, so a second
    call that read a slot it did not write would show up as a different loss."""
    for seed, M, N, K, name in calls:       # two calls in a row share the fixed scratch
        dtype = torch.bfloat16 if name == "bf16" else torch.float32
        Xq, W, B, Yref = _problem(seed, M, N, K, dtype, cuda_device)
        got = omq.fq_linear_fwd_noalloc(Xq, W, Yref, B_tilde=B)
        want = omq.fq_linear_fwd(Xq, W, B_tilde=B, Y_ref=Yref)
        torch.cuda.synchronize()
        omq.sync_check()
        for key in ("Y", "dY"):
            assert torch.equal(got[key], want[key]), key
        # and both agree with a plain product within the tests' tolerance for the dtype
        ok, err = close(got["Y"].float().cpu().numpy(),
                        (Xq.double() @ W.double().T + B.double()).cpu().numpy(), name)
        assert ok, err
        lg, lw = got["loss"].item(), want["loss"].item()
        assert np.isfinite(lg) and lw > 0
        assert lg == lw


def test_noalloc_rejects_problems_beyond_its_scratch(omq, cuda_device):
    import ctypes
    # 2 x ceil(16512/256) x 128 = 16640 partial sums > 16384 slots: rejected on the host
    # before any buffer is touched, so one small tensor stands in for every pointer
    buf = torch.zeros(64, dtype=torch.float32, device=cuda_device)
    p = ctypes.c_void_p(buf.data_ptr())
    st = omq._lib.omq_fq_linear_fwd_noalloc(p, p, omq.OMQ_BF16, 128 * 129, 256 * 128, 64, None,
                                            p, None, p, p, None)
    assert st == 2
    st = omq._lib.omq_fq_linear_fwd_noalloc(p, p, omq.OMQ_BF16, 128, 256, 64, None, None, None,
                                            p, p, None)
    assert st == 1
    omq.sync_check()
