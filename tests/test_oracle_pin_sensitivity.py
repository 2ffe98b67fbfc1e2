"""The pins must fail on plausible mistakes. Each case plants one mistake in a copy of an
oracle function (on the CPU) and checks that the corresponding pin rejects it."""
import numpy as np
import pytest

from oracle import omniquant as om
from tests import test_oracle_ste as ste


def _drop_zero_point_path(dDeq, V, enc, g, b):
    # planted mistake: the zero point's dependence on h, b and min is ignored
    enc2 = om.Encoded(**{**enc.__dict__})
    dV, dg, db = _orig_backward(dDeq, V, enc2, g, b)
    R, C = enc.codes.shape
    G = enc.group
    inr = enc.inrange.reshape(R, C // G, G)
    dD = np.asarray(dDeq, np.float64).reshape(R, C // G, G)
    Gz = (dD * np.where(inr, 0.0, -enc.h.astype(np.float64)[:, :, None])).sum(2)
    m = enc.vmin.astype(np.float64)
    h = enc.h.astype(np.float64)
    return dV, dg, db + Gz * m / h   # removes the -Gz*m/h term of db


def _flip_clip_slope(dDeq, V, enc, g, b):
    enc2 = om.Encoded(**{**enc.__dict__})
    enc2.codes = enc.codes[:, ::-1].copy() if enc.codes.shape[1] > 1 else enc.codes
    return _orig_backward(dDeq, V, enc2, g, b)


_orig_backward = om.encode_backward


@pytest.mark.parametrize("mutant", [_drop_zero_point_path, _flip_clip_slope])
def test_ste_pin_rejects_mutant(monkeypatch, mutant):
    monkeypatch.setattr(om, "encode_backward", mutant)
    failures = 0
    for case in [(1, 4, 8, 4, 4), (2, 4, 8, 4, 2), (5, 8, 8, 4, 2)]:
        try:
            ste.test_encoder_ste_matches_autograd(*case)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_let_pin_rejects_sign_error(monkeypatch):
    from tests import test_oracle_let_adamw_pack as letp
    real = om.let_bias
    monkeypatch.setattr(om, "let_bias", lambda W, B, d: real(W, B, None if d is None else -d))
    with pytest.raises(AssertionError):
        letp.test_let_is_exact_with_quantization_off()


def test_step_pin_rejects_transposed_operand(monkeypatch):
    real = om.calib_step

    def bad(*a, **k):
        r = real(*a, **k)
        if r.d_delta is not None:
            r.d_delta = r.d_delta[::-1].copy()
        return r
    monkeypatch.setattr(om, "calib_step", bad)
    with pytest.raises(AssertionError):
        ste.test_full_step_matches_autograd(4, True, 4)
