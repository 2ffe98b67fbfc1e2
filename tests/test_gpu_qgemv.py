"""omq_qgemv (inference with the folded weights) against the oracle: the oracle folds a seeded
weight (codes, h, z), the same packed codes go to the GPU, and y = x dequant(W)^T is compared
with the oracle's binary64 product of x and the dequantized weight (c - z) h. Float32
accumulation over K: max relative error 1e-5 of the largest output."""
import numpy as np
import pytest
import torch

from oracle import omniquant as om
from post_quantization_lwc_b200 import synth
from tests.gpu_common import max_rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


CASES = [  # M tokens, N, K, group, bits
    (1, 264, 512, 128, 4),
    (3, 136, 768, 256, 2),
    (8, 200, 256, 64, 8),
    (5, 72, 384, 384, 4),
    (1, 4096, 4096, 128, 4),     # LLaMA-7B q_proj, g128 (the fold of the bench workload)
    (4, 11008, 4096, 4096, 4),   # LLaMA-7B gate/up, per channel
    (7, 4096, 4096, 128, 2),     # more than four tokens: two launches (4 + 3)
]


@pytest.mark.parametrize("M,N,K,G,bits", CASES)
def test_qgemv_matches_dequantized_product(omq, cuda_device, M, N, K, G, bits):
    gen = torch.Generator().manual_seed(N + K + bits)
    W = synth.make_weight(gen, N, K, "bf16")
    gl, bl = synth.random_logits(N + 1, N, K // G, 1.0, 5.0)
    x = torch.randn(M, K, generator=gen).to(torch.bfloat16)
    packed, h, z = om.fold_pack(synth.as_f32_numpy(W), None, gl.numpy(), bl.numpy(), bits, G)
    y = omq.qgemv(x.to(cuda_device), torch.from_numpy(packed).to(cuda_device),
                  torch.from_numpy(h).to(cuda_device), torch.from_numpy(z).to(cuda_device), G,
                  bits)
    torch.cuda.synchronize()
    omq.sync_check()
    codes = om.unpack_codes(packed, bits, K).astype(np.float32)
    Wd = ((codes.reshape(N, K // G, G) - z.astype(np.float32)[:, :, None]) *
          h[:, :, None]).reshape(N, K)
    want = synth.as_f32_numpy(x).astype(np.float64) @ Wd.astype(np.float64).T
    assert max_rel(y.cpu().numpy(), want) <= 1e-5


def test_qgemv_rejects_bad_shapes(omq):
    lib = omq._lib
    P = 256
    assert lib.omq_qgemv(P, 1, 9, 256, P, P, P, 16, 128, 4, P, None) == 2      # 9 tokens
    assert lib.omq_qgemv(P, 0, 1, 256, P, P, P, 16, 128, 3, P, None) == 8      # 3 bits, f32 x
    assert lib.omq_qgemv(P, 1, 1, 256, P, P, P, 16, 128, 9, P, None) == 5      # 9 bits
    assert lib.omq_qgemv(P, 1, 1, 256, P, P, P, 16, 16, 4, P, None) == 2       # group < 32
    assert lib.omq_qgemv(None, 1, 1, 256, P, P, P, 16, 128, 4, P, None) == 1
