"""omq_qgemm (tensor-core product with the folded weights, the codes expanded inside the GEMM)
against the oracle: the oracle folds a seeded weight into packed codes, h and z (2 to 8 bits,
groups of 32 to whole rows), the same packed bytes go to the GPU, and y = x dequant(W)^T is
compared with binary64 products:
  - with the dequantized weight (c - z) h rounded once to the activations' 16-bit type, the
    operand the tensor cores multiply: within the float32 accumulation bound
    3 sqrt(K) 2^-24 (Frobenius), so a wrong code, shift, zero point or group shows;
  - with the binary32 dequantized weight: within the 16-bit GEMM tolerance 2e-2.
The 3-, 5-, 6- and 7-bit decode path of omq_qgemv, which runs the same kernel, is checked the
same way."""
import numpy as np
import pytest
import torch

from oracle import omniquant as om
from post_quantization_lwc_b200 import synth
from tests.gpu_common import TOL_BF16_FROB, dtype_round, frob_rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


def _fold(N, K, G, bits, seed):
    gen = torch.Generator().manual_seed(seed)
    W = synth.make_weight(gen, N, K, "bf16")
    gl, bl = synth.random_logits(seed + 1, N, K // G, 1.0, 5.0)
    packed, h, z = om.fold_pack(synth.as_f32_numpy(W), None, gl.numpy(), bl.numpy(), bits, G)
    codes = om.unpack_codes(packed, bits, K).astype(np.float32)
    Wd = ((codes.reshape(N, K // G, G) - z.astype(np.float32)[:, :, None]) *
          h[:, :, None]).reshape(N, K).astype(np.float32)
    return packed, h, z, Wd, gen


CASES = [  # M tokens, N, K, group, bits, x dtype
    (16, 264, 512, 128, 4, "f16"),
    (200, 136, 768, 64, 3, "bf16"),
    (37, 520, 1024, 32, 5, "f16"),
    (300, 264, 640, 640, 6, "f16"),
    (64, 128, 384, 96, 7, "bf16"),
    (513, 200, 256, 64, 8, "f16"),
    (96, 1032, 1024, 128, 2, "f16"),
    (2048, 4096, 4096, 128, 4, "f16"),     # LLaMA-7B q_proj prefill, g128 (the q_proj fold)
]


@pytest.mark.parametrize("M,N,K,G,bits,xdt", CASES)
def test_qgemm_matches_dequantized_product(omq, cuda_device, M, N, K, G, bits, xdt):
    packed, h, z, Wd, gen = _fold(N, K, G, bits, 7 * N + K + bits)
    tdt = torch.float16 if xdt == "f16" else torch.bfloat16
    x = torch.randn(M, K, generator=gen).to(tdt)
    bias = torch.randn(N, generator=gen) * 0.1
    dev = cuda_device
    y = omq.qgemm(x.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(h).to(dev),
                  torch.from_numpy(z).to(dev), G, bits, bias=bias.to(dev))
    torch.cuda.synchronize()
    omq.sync_check()
    x64 = x.double().numpy()
    exact16 = x64 @ dtype_round(Wd, xdt).astype(np.float64).T + bias.double().numpy()
    assert frob_rel(y.cpu().numpy(), exact16) <= 3 * np.sqrt(K) * 2.0 ** -24
    exact = x64 @ Wd.astype(np.float64).T + bias.double().numpy()
    assert frob_rel(y.cpu().numpy(), exact) <= TOL_BF16_FROB


@pytest.mark.parametrize("M,bits", [(1, 3), (4, 5), (8, 6), (2, 7)])
def test_qgemv_straddling_bits(omq, cuda_device, M, bits):
    N, K, G = 264, 512, 128
    packed, h, z, Wd, gen = _fold(N, K, G, bits, 31 * M + bits)
    x = torch.randn(M, K, generator=gen).to(torch.bfloat16)
    dev = cuda_device
    y = omq.qgemv(x.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(h).to(dev),
                  torch.from_numpy(z).to(dev), G, bits)
    torch.cuda.synchronize()
    omq.sync_check()
    exact16 = x.double().numpy() @ dtype_round(Wd, "bf16").astype(np.float64).T
    assert frob_rel(y.cpu().numpy(), exact16) <= 3 * np.sqrt(K) * 2.0 ** -24
