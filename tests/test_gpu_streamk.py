"""The tcgen05 GEMM's stream-K tail schedule.

When the last wave of whole 256 x 256 tiles would leave many of the 74 CTA pairs idle and
the contraction is long, the last whole wave and the tail are dealt out as equal runs of
k-blocks: a tile of that region
is finished by one pair or by two, the second adding the first's stored partial
accumulator. Here the forward GEMM (bias + residual + loss epilogue) on shapes that take
that schedule is checked against a binary64 product of the same 16-bit operands (only the
float32 summation order differs), with ragged tiles, and for run-to-run bitwise
reproducibility (the sum of two partials does not depend on which pair arrives second).
"""
import numpy as np
import pytest
import torch

from tests.gpu_common import frob_rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


# (M, N, K), contractions of at least 128 k-blocks of 64 and at least two waves of tiles (the
# schedule's thresholds): 160 tiles (two waves + 12: one whole wave ahead of the region, the
# down_proj forward), 304 tiles (4 waves + 8), ragged rows, columns and depth
SHAPES = [(2048, 5120, 13824), (4096, 4864, 8192), (2000, 5096, 8200), (2304, 4352, 8192)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_stream_k_forward_matches_fp64_product(omq, cuda_device, M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    Xq = torch.randn(M, K, generator=g).to(torch.float16)
    W = (torch.randn(N, K, generator=g) * 0.05).to(torch.float16)
    B = torch.randn(N, generator=g) * 0.1
    ref = Xq.double() @ W.double().T + B.double()
    Yref = (ref + 0.01 * torch.randn(M, N, generator=g, dtype=torch.float64)).float()
    dev = cuda_device
    args = (Xq.to(dev), W.to(dev))
    kw = dict(B_tilde=B.to(dev), Y_ref=Yref.to(dev))
    a = omq.fq_linear_fwd(*args, **kw)
    b = omq.fq_linear_fwd(*args, **kw)
    torch.cuda.synchronize()
    omq.sync_check()
    # float32 accumulation of K exact products: relative error about sqrt(K) 2^-24 (a
    # missing or misplaced partial would be of order one)
    assert frob_rel(a["Y"].cpu().numpy(), ref.numpy()) <= 3 * np.sqrt(K) * 2.0 ** -24
    # the epilogue on the GPU's own Y: the residual rounded once to float16, the loss from
    # float32 squares summed in a fixed order
    res = a["Y"].double().cpu().numpy() - Yref.double().numpy()
    assert frob_rel(a["dY"].float().cpu().numpy(), res) <= 2.0 ** -11
    loss = float((res ** 2).mean())
    assert abs(a["loss"].item() - loss) <= 1e-5 * loss
    for key in ("Y", "dY", "loss"):
        assert torch.equal(a[key], b[key]), key
