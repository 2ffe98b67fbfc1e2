"""Pins of the oracle's LET, AdamW and packing against closed forms and library routines."""
import numpy as np
import pytest
import torch

from oracle import omniquant as om
from post_quantization_lwc_b200 import synth


def test_let_is_exact_with_quantization_off():
    """[ICLR] section LET: [(X-delta)/s][s.W]^T + [B + W delta] equals X W^T + B."""
    gen = torch.Generator().manual_seed(21)
    X = torch.randn(32, 64, generator=gen).numpy()
    X[:, 5] *= 40
    W = (torch.randn(16, 64, generator=gen) * 0.02).numpy()
    B = torch.randn(16, generator=gen).numpy()
    s, d = synth.random_let(3, 64)
    s, d = s.numpy(), d.numpy()
    Y = om.reference_output(X, W, B)
    Xt = om.let_act(X, s, d).astype(np.float64)
    Wt = om.let_weight(W, s).astype(np.float64)
    Bt = om.let_bias(W, B, d)
    Y2 = Xt @ Wt.T + Bt[None, :]
    # binary32 X~ and W~ carry one rounding each (~6e-8 relative per element)
    assert np.abs(Y2 - Y).max() <= 1e-5 * np.abs(Y).max()
    # in binary64 the identity is exact up to rounding of the sums
    X64, W64 = X.astype(np.float64), W.astype(np.float64)
    s64, d64 = s.astype(np.float64), d.astype(np.float64)
    Y3 = ((X64 - d64) / s64) @ (W64 * s64).T + (B + W64 @ d64)[None, :]
    assert np.abs(Y3 - Y).max() <= 1e-12 * np.abs(Y).max()


def test_let_bias_uses_original_weight():
    W = np.array([[1.0, 2.0], [3.0, -1.0]], np.float32)
    d = np.array([0.5, -2.0], np.float32)
    np.testing.assert_array_equal(om.let_bias(W, np.zeros(2, np.float32), d), [-3.5, 3.5])
    np.testing.assert_array_equal(om.let_weight(W, np.array([2.0, 0.5], np.float32)),
                                  [[2.0, 1.0], [6.0, -0.5]])
    np.testing.assert_array_equal(om.let_act(np.array([[1.0, 1.0]], np.float32),
                                             np.array([2.0, 0.5], np.float32), d),
                                  [[0.25, 6.0]])


def test_adamw_matches_torch():
    gen = torch.Generator().manual_seed(4)
    p0 = torch.randn(50, generator=gen, dtype=torch.float64)
    p = p0.clone().requires_grad_(True)
    opt = torch.optim.AdamW([p], lr=5e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0)
    q, m, v = p0.numpy().copy(), np.zeros(50), np.zeros(50)
    for t in range(1, 6):
        g = torch.randn(50, generator=gen, dtype=torch.float64)
        opt.zero_grad()
        p.grad = g.clone()
        opt.step()
        q, m, v = om.adamw_step(q, g.numpy(), m, v, t, 5e-3)
    np.testing.assert_allclose(q, p.detach().numpy(), rtol=1e-14, atol=1e-15)


def test_adamw_weight_decay_matches_torch():
    p = torch.tensor([1.0, -2.0, 3.0], dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([p], lr=1e-2, weight_decay=0.1)
    p.grad = torch.tensor([0.1, 0.2, -0.3], dtype=torch.float64)
    opt.step()
    q, _, _ = om.adamw_step([1.0, -2.0, 3.0], [0.1, 0.2, -0.3], [0, 0, 0], [0, 0, 0], 1, 1e-2,
                            weight_decay=0.1)
    np.testing.assert_allclose(q, p.detach().numpy(), rtol=1e-14)


def test_pack_hand_examples():
    # 4 bits: element 0 in the low nibble of byte 0
    c4 = np.array([[1, 2, 3, 4, 15, 0]], np.uint8)
    assert om.pack_codes(c4, 4).tolist() == [[0x21, 0x43, 0x0F]]
    # 2 bits: four codes per byte, element 0 in bits 0-1
    c2 = np.array([[1, 2, 3, 0, 3, 3, 3, 3]], np.uint8)
    assert om.pack_codes(c2, 2).tolist() == [[1 | 2 << 2 | 3 << 4, 0xFF]]
    assert om.pack_codes(np.array([[7, 200]], np.uint8), 8).tolist() == [[7, 200]]
    # 3 bits: codes 1..7, 0 are the bit string 001 010 011 100 101 110 111 000 written from
    # the least-significant end: byte 0 = 11|010|001, byte 1 = 0|101|100|0, byte 2 = 000|111|11
    c3 = np.array([[1, 2, 3, 4, 5, 6, 7, 0]], np.uint8)
    assert om.pack_codes(c3, 3).tolist() == [[0xD1, 0x58, 0x1F]]
    # 6 bits: 0x3F, 0x01, 0x20, 0x15 -> 111111 | 000001 | 100000 | 010101 from the low end:
    # byte 0 = 01|111111, byte 1 = 0000|0000, byte 2 = 010101|10
    c6 = np.array([[0x3F, 0x01, 0x20, 0x15]], np.uint8)
    assert om.pack_codes(c6, 6).tolist() == [[0x7F, 0x00, 0x56]]
    with pytest.raises(ValueError):
        om.pack_codes(np.zeros((1, 3), np.uint8), 4)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
def test_pack_roundtrip(bits):
    gen = np.random.default_rng(bits)
    c = gen.integers(0, 2 ** bits, size=(7, 64)).astype(np.uint8)
    assert np.array_equal(om.unpack_codes(om.pack_codes(c, bits), bits, 64), c)


def test_fold_pack_dequant_equals_fake_quant():
    """Codes unpacked from the fold give back the fake-quant weights bit for bit."""
    cfg = synth.scaled(synth.CONFIGS["llama7b_qproj_w4a16g128"], 8, 512, 16)
    inp = synth.make_inputs(cfg)
    W = synth.as_f32_numpy(inp.W)
    gl, bl = synth.random_logits(5, 16, 4)
    s, _ = synth.random_let(6, 512)
    packed, h, z = om.fold_pack(W, s.numpy(), gl.numpy(), bl.numpy(), 4, 128)
    _, enc, _, _ = om.lwc_quant(W, s.numpy(), gl.numpy(), bl.numpy(), 4, 128)
    c = om.unpack_codes(packed, 4, 512).astype(np.float32).reshape(16, 4, 128)
    deq = (c - z.astype(np.float32)[:, :, None]) * h[:, :, None]
    assert np.array_equal(deq.reshape(16, 512).view(np.uint32), enc.deq.view(np.uint32))
