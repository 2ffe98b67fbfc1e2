"""Pins of the oracle's multi-step procedures: the calibration loop of one linear layer
(oracle/omniquant.py `calibrate`) and of one block (oracle/block.py `block_calibrate`).

"【ICLR 2024】OmniQuant ...", section 实验证据: the learnable parameters are trained with AdamW
(no weight decay) at 5e-3 for the LWC logits and 1e-2 for the LET vectors, one calibration
sample per step, epochs over the samples in order. The pin is an independent statement of that
loop: torch.optim.AdamW (two parameter groups at the two rates) driving the float64 autograd
statements of the step already pinned in tests/test_oracle_ste.py and
tests/test_oracle_block.py, over several steps and, for the block, two samples and two epochs.
Past the first step AdamW's bias corrections no longer cancel, so a wrong correction, a
parameter updated at the other group's rate, an update applied before every gradient of the
step is taken, or samples visited out of order all change the trajectory at the 1e-3 level;
the two sides agree to rounding (1e-6).
"""
import numpy as np
import pytest
import torch

from oracle import block as ob
from oracle import omniquant as om
from tests.test_oracle_block import SHAPES, _autograd_block, make_case
from tests.test_oracle_ste import _autograd_step

# the rates the page gives (section 实验证据), restated here rather than read from the oracle
LR_LWC, LR_LET = 5e-3, 1e-2


def _torch_adamw(params, lrs):
    groups = [{"params": [p], "lr": lr} for p, lr in zip(params, lrs)]
    return torch.optim.AdamW(groups, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0)


def _linear_case(seed, abits, let, group, M=6, K=8, N=4):
    gen = torch.Generator().manual_seed(seed)
    W = (torch.randn(N, K, generator=gen) * 0.1).numpy()
    X = torch.randn(M, K, generator=gen).numpy()
    X[:, 1] *= 6.0
    B = (torch.randn(N, generator=gen) * 0.1).numpy()
    Yref = X.astype(np.float64) @ W.T.astype(np.float64) + B
    gl = torch.empty(N, K // group).uniform_(0.5, 3.0, generator=gen).numpy().astype(np.float32)
    bl = torch.empty(N, K // group).uniform_(0.5, 3.0, generator=gen).numpy().astype(np.float32)
    s = (0.7 + 0.6 * torch.rand(K, generator=gen)).numpy().astype(np.float32)
    d = (0.2 * torch.randn(K, generator=gen)).numpy().astype(np.float32)
    return X, W, B, Yref, gl, bl, s, d


def _torch_calibrate(X, W, B, Yref, gl, bl, s, d, bits, group, abits, let, steps):
    """The loop with torch's AdamW on binary64 master parameters; each step's forward and
    gradient are taken at the parameters rounded to binary32, as the oracle and the device
    hold them."""
    P = [torch.from_numpy(np.asarray(a, np.float64).copy()) for a in (gl, bl, s, d)]
    opt = _torch_adamw(P, [LR_LWC, LR_LWC, LR_LET, LR_LET])
    losses = []
    for _ in range(steps):
        cur = [p.detach().numpy().astype(np.float32) for p in P]
        loss, dgl, dbl, ds, dd, _ = _autograd_step(X, W, B, Yref, *cur, bits, group, abits, let)
        losses.append(loss)
        grads = [dgl, dbl, ds if let else None, dd if let else None]
        for p, g in zip(P, grads):
            p.grad = None if g is None else torch.from_numpy(np.asarray(g, np.float64))
        opt.step()
    return losses, [p.detach().numpy() for p in P]


@pytest.mark.parametrize("abits,let,group", [(16, True, 4), (4, True, 8), (16, False, 8),
                                             (4, False, 4)])
def test_linear_calibrate_matches_torch_adamw(abits, let, group):
    bits, steps = 4, 5
    X, W, B, Yref, gl, bl, s, d = _linear_case(300 + abits + group, abits, let, group)
    losses, ogl, obl, os_, od = om.calibrate(X, W, B, Yref, gl, bl, s, d, bits, group, abits,
                                             let, steps)
    tl, (tgl, tbl, ts, td) = _torch_calibrate(X, W, B, Yref, gl, bl, s, d, bits, group, abits,
                                              let, steps)
    np.testing.assert_allclose(losses, tl, rtol=1e-6, atol=0)
    for got, want in ((ogl, tgl), (obl, tbl), (os_, ts), (od, td)):
        np.testing.assert_allclose(got.astype(np.float64), want, rtol=0, atol=2e-6)
    # the parameters moved by several learning-rate steps, so the comparison has teeth
    assert np.abs(ogl.astype(np.float64) - gl).max() > 2 * LR_LWC
    if let:
        assert np.abs(os_.astype(np.float64) - s).max() > 2 * LR_LET
    else:
        np.testing.assert_array_equal(os_, s)


def _torch_block_calibrate(sh, xs, W, theta0, epochs):
    split = sum(n for name, n in ob.theta_layout(sh) if name.startswith(("gamma", "beta")))
    lwc = torch.from_numpy(theta0[:split].astype(np.float64))
    let = torch.from_numpy(theta0[split:].astype(np.float64))
    opt = _torch_adamw([lwc, let], [LR_LWC, LR_LET])
    y_refs = [ob.block_reference(sh, x, W) for x in xs]
    losses = []
    for _ in range(epochs):
        for x, y_ref in zip(xs, y_refs):
            theta = np.concatenate([lwc.numpy(), let.numpy()]).astype(np.float32)
            loss, grad, _ = _autograd_block(sh, x, W, theta, y_ref)
            losses.append(loss)
            lwc.grad = torch.from_numpy(grad[:split].astype(np.float64))
            let.grad = torch.from_numpy(grad[split:].astype(np.float64))
            opt.step()
            # the parameter vector is held in binary32 between steps
            with torch.no_grad():
                lwc.copy_(lwc.float().double())
                let.copy_(let.float().double())
    return np.array(losses), np.concatenate([lwc.numpy(), let.numpy()]).astype(np.float32)


@pytest.mark.parametrize("si", [0, 2])
def test_block_calibrate_matches_torch_adamw(si):
    sh = SHAPES[si]
    x0, W, theta = make_case(sh, 500 + si)
    x1, _, _ = make_case(sh, 600 + si)
    losses, theta_n, outs = ob.block_calibrate(sh, [x0, x1], W, theta, 2)
    tl, ttheta = _torch_block_calibrate(sh, [x0, x1], W, theta, 2)
    assert len(losses) == 4
    np.testing.assert_allclose(losses, tl, rtol=1e-6, atol=0)
    np.testing.assert_allclose(theta_n, ttheta, rtol=0, atol=2e-6)
    assert np.abs(theta_n.astype(np.float64) - theta).max() > 2 * LR_LET
    # the samples' quantized outputs are the forward at the final parameters
    for x, y in zip((x0, x1), outs):
        _, _, ay = _autograd_block(sh, x, W, theta_n, ob.block_reference(sh, x, W))
        np.testing.assert_allclose(y, ay, rtol=1e-5, atol=1e-5)


# ---- planted mistakes: each must make the pins above fail

_true_adamw = om.adamw_step


def _adamw_no_bias_correction_after_first(p, grad, m, v, step, lr, **kw):
    return _true_adamw(p, grad, m, v, 1, lr, **kw)


def _adamw_coupled_decay(p, grad, m, v, step, lr, **kw):
    return _true_adamw(p, grad, m, v, step, lr, weight_decay=0.01)


@pytest.mark.parametrize("mutant", ["bias_correction", "let_rate", "decay"])
def test_linear_pin_rejects_mutant(monkeypatch, mutant):
    if mutant == "bias_correction":
        monkeypatch.setattr(om, "adamw_step", _adamw_no_bias_correction_after_first)
    elif mutant == "let_rate":
        monkeypatch.setattr(om, "LR_LET", LR_LWC)
    else:
        monkeypatch.setattr(om, "adamw_step", _adamw_coupled_decay)
    with pytest.raises(AssertionError):
        test_linear_calibrate_matches_torch_adamw(16, True, 4)


@pytest.mark.parametrize("mutant", ["bias_correction", "let_rate", "sample_order"])
def test_block_pin_rejects_mutant(monkeypatch, mutant):
    if mutant == "bias_correction":
        monkeypatch.setattr(om, "adamw_step", _adamw_no_bias_correction_after_first)
    elif mutant == "let_rate":
        sh = SHAPES[0]
        x0, W, theta = make_case(sh, 500)
        x1, _, _ = make_case(sh, 600)
        losses, theta_n, _ = ob.block_calibrate(sh, [x0, x1], W, theta, 2, lr_let=LR_LWC)
        tl, ttheta = _torch_block_calibrate(sh, [x0, x1], W, theta, 2)
        assert np.abs(theta_n - ttheta).max() > 1e-4
        return
    else:
        real = ob.block_calibrate

        def reversed_samples(sh, xs, W, theta0, epochs, **kw):
            return real(sh, list(reversed(xs)), W, theta0, epochs, **kw)
        monkeypatch.setattr(ob, "block_calibrate", reversed_samples)
    with pytest.raises(AssertionError):
        test_block_calibrate_matches_torch_adamw(0)
