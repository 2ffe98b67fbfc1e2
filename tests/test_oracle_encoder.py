"""Pins of the oracle's LWC / activation encoder against facts fixed outside the oracle."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import omniquant as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_affine_example():
    """The tutorial's affine example ([3, 1, -2, 3], 4 bits) mapped to the LWC convention."""
    with open(os.path.join(GOLDEN, "affine_worked_example.json")) as f:
        ex = json.load(f)
    x = np.array([ex["x"]], dtype=np.float32)
    one = np.ones((1, 1), np.float32)
    enc = om.encode_affine(x, one, one, ex["bits"], 4)
    assert enc.h[0, 0] == np.float32(ex["expected_h"])
    assert int(enc.z_i32[0, 0]) == ex["expected_z"]
    assert enc.codes_u8[0].tolist() == ex["expected_codes"]
    # the page's signed codes shifted into [0, 15]; its zero point shifted likewise
    shift = -ex["page_signed_qmin"]
    assert [c + shift for c in ex["page_signed_codes"]] == ex["expected_codes"]
    assert ex["page_signed_zero_point"] + shift == ex["expected_z"]
    # the page's scale is the reciprocal of h
    assert abs(1.0 / float(enc.h[0, 0]) - ex["page_scale_reciprocal"]) < 1e-6
    np.testing.assert_allclose(enc.deq[0], ex["expected_dequant"], rtol=0, atol=1e-6)


def test_sigmoid_init_value():
    # logits +4 give clipping strength 1/(1+e^-4) = 0.98201379...
    assert om.sigmoid32(4.0) == np.float32(0.9820137900379085)
    assert om.sigmoid32(0.0) == np.float32(0.5)


def test_bf16_round_matches_torch():
    gen = torch.Generator().manual_seed(11)
    x = torch.randn(100000, generator=gen) * 3
    # add exact ties: values whose low 16 bits are 0x8000
    ties = (torch.arange(1, 1001, dtype=torch.int32) << 16 | 0x8000).view(torch.float32)
    x = torch.cat([x, ties, -ties])
    ours = om.bf16_round(x.numpy())
    ref = x.to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def _torch_fq(V, h, z, bits, group):
    """torch's affine fake-quant with the same scale / zero point, per group (axis 0)."""
    R, C = V.shape
    ng = C // group
    v = torch.from_numpy(V.reshape(R * ng, group).copy())
    return torch.fake_quantize_per_channel_affine(
        v, torch.from_numpy(h.reshape(-1).copy()), torch.from_numpy(z.reshape(-1).astype(np.int32)),
        0, 0, 2 ** bits - 1).numpy().reshape(R, C)


@pytest.mark.parametrize("bits,group", [(4, 64), (2, 64), (4, 256), (3, 32), (8, 128)])
def test_minmax_special_case_matches_torch(bits, group):
    """gamma = beta = 1 is MinMax ([ICLR] section LWC): same values as torch's affine
    fake-quant given h and z, away from rounding ties (torch multiplies by 1/scale)."""
    gen = torch.Generator().manual_seed(bits * 100 + group)
    V = (torch.randn(32, 256, generator=gen) * 0.02).numpy()
    one = np.ones((32, 256 // group), np.float32)
    enc = om.encode_affine(V, one, one, bits, group)
    # with gamma = beta = 1 the zero point lies in [0, Q] whenever min < 0 < max
    assert (enc.z >= 0).all() and (enc.z <= 2 ** bits - 1).all()
    assert enc.inrange.all()          # MinMax never clips
    ref = _torch_fq(V, enc.h, enc.z, bits, group)
    u = V.reshape(32, -1, group) / enc.h[:, :, None]
    safe = (np.abs(u - np.floor(u) - 0.5) > 1e-4).reshape(32, 256)
    assert safe.mean() > 0.99
    np.testing.assert_allclose(enc.deq[safe], ref[safe], rtol=0, atol=1e-7)
    # and MinMax keeps min and max representable to within one rounding
    np.testing.assert_allclose(enc.h, (enc.vmax - enc.vmin) / (2 ** bits - 1), rtol=1e-6)


def test_per_token_act_quant_matches_torch():
    gen = torch.Generator().manual_seed(5)
    X = torch.randn(16, 128, generator=gen)
    X[:, 3] *= 50
    Xn = X.numpy()
    enc = om.act_quant(Xn, 4)
    assert enc.h.shape == (16, 1)
    ref = _torch_fq(Xn, enc.h, enc.z, 4, 128)
    u = Xn / enc.h
    safe = np.abs(u - np.floor(u) - 0.5) > 1e-4
    np.testing.assert_allclose(enc.deq[safe], ref[safe], rtol=0, atol=1e-6)
    assert om.act_quant(Xn, 16) is None


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_dequant_error_bound_and_code_range(bits):
    """codes in [0, Q]; |deq - V| <= h/2 (+ one rounding) wherever the value is not clipped."""
    gen = torch.Generator().manual_seed(7 + bits)
    V = (torch.randn(64, 128, generator=gen) * 0.05).numpy()
    g = om.sigmoid32(torch.empty(64, 2).uniform_(-1, 5, generator=gen).numpy())
    b = om.sigmoid32(torch.empty(64, 2).uniform_(-1, 5, generator=gen).numpy())
    enc = om.encode_affine(V, g, b, bits, 64)
    Q = 2 ** bits - 1
    assert enc.codes.min() >= 0 and enc.codes.max() <= Q
    assert np.all(enc.codes == np.round(enc.codes))
    hh = np.repeat(enc.h, 64, axis=1)
    err = np.abs(enc.deq.astype(np.float64) - V.astype(np.float64))
    bound = hh / 2 * (1 + 1e-5) + 4 * np.spacing(np.abs(V).max())
    assert np.all(err[enc.inrange] <= bound[enc.inrange])
    # the clipped elements sit beyond the kept range
    clipped = ~enc.inrange
    assert clipped.any()
    hi = np.repeat(enc.codes, 1, axis=1)[clipped]
    assert set(np.unique(hi).tolist()) <= {0.0, float(Q)}


def test_clipping_is_monotone_in_strength():
    """Smaller gamma (upper strength) never clips fewer elements at the top."""
    gen = torch.Generator().manual_seed(3)
    V = (torch.randn(8, 256, generator=gen) * 0.02).numpy()
    one = np.ones((8, 1), np.float32)
    prev = -1
    for gval in [1.0, 0.9, 0.8, 0.6, 0.4]:
        enc = om.encode_affine(V, one * np.float32(gval), one, 4, 256)
        n_top = int((enc.codes == 15).sum())
        assert n_top >= prev
        prev = n_top


def test_constant_group_uses_floor():
    V = np.full((1, 8), 0.25, np.float32)
    one = np.ones((1, 1), np.float32)
    enc = om.encode_affine(V, one, one, 4, 8)
    assert enc.h[0, 0] == np.float32(1e-8)
    assert enc.h_raw[0, 0] == 0
    assert (enc.codes >= 0).all() and (enc.codes <= 15).all()
