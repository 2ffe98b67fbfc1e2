"""Pins of the oracle's hand-derived STE chain rule against an independent float64 autograd
statement of the same forward (rounding written as x + (round(x) - x).detach()), on tiny
inputs that exercise every branch: in range, clipped low, clipped high, extremal elements,
ties at the max, and the activation quantizer."""
import numpy as np
import pytest
import torch

from oracle import omniquant as om


def _ste_round(x):
    return x + (torch.round(x) - x).detach()


def _autograd_encode(V, g, b, bits, group):
    """deq(V; g, b) in float64 torch, differentiable in V, g, b (STE through round)."""
    R, C = V.shape
    Vg = V.view(R, C // group, group)
    Q = float(2 ** bits - 1)
    M = Vg.amax(-1)
    m = Vg.amin(-1)
    h = ((g * M - b * m) / Q).clamp(min=1e-8)
    z = -_ste_round(b * m / h)
    q = _ste_round(Vg / h[..., None]) + z[..., None]
    c = q.clamp(0.0, Q)
    return ((c - z[..., None]) * h[..., None]).reshape(R, C)


def _case(seed, R, C, spread=(-1.0, 3.0), scale=0.05):
    gen = torch.Generator().manual_seed(seed)
    V = (torch.randn(R, C, generator=gen) * scale).to(torch.float32)
    gl = torch.empty(R, C).uniform_(*spread, generator=gen)
    bl = torch.empty(R, C).uniform_(*spread, generator=gen)
    dD = torch.randn(R, C, generator=gen, dtype=torch.float64)
    return V, gl, bl, dD


@pytest.mark.parametrize("seed,R,C,group,bits", [
    (0, 4, 4, 4, 4), (1, 4, 8, 4, 4), (2, 4, 8, 4, 2), (3, 6, 12, 6, 3), (4, 4, 16, 16, 4),
    (5, 8, 8, 4, 2)])
def test_encoder_ste_matches_autograd(seed, R, C, group, bits):
    V, gl, bl, dD = _case(seed, R, C)
    ng = C // group
    gl, bl = gl[:, :ng].contiguous().float(), bl[:, :ng].contiguous().float()
    g = om.sigmoid32(gl.numpy())
    b = om.sigmoid32(bl.numpy())
    enc = om.encode_affine(V.numpy(), g, b, bits, group)
    dV, dg, db = om.encode_backward(dD.numpy(), V.numpy(), enc, g, b)

    Vt = V.double().requires_grad_(True)
    gt = torch.from_numpy(g.astype(np.float64)).requires_grad_(True)
    bt = torch.from_numpy(b.astype(np.float64)).requires_grad_(True)
    deq = _autograd_encode(Vt, gt, bt, bits, group)
    # the float64 statement must take the same integer decisions as the binary32 encoder
    np.testing.assert_allclose(deq.detach().numpy(), enc.deq, rtol=0, atol=1e-6)
    (deq * dD).sum().backward()
    # tolerance: the oracle's h is binary32 (one rounding, 6e-8 relative); u = V/h is up to
    # ~2^bits, so r - u and the group sums carry ~1e-6 absolute differences. A dropped term or
    # a sign error changes these gradients at the 1e-1 level.
    np.testing.assert_allclose(dV, Vt.grad.numpy(), rtol=1e-5, atol=2e-5)
    np.testing.assert_allclose(dg, gt.grad.numpy(), rtol=1e-5, atol=2e-5)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-5, atol=2e-5)


def test_cases_cover_every_branch():
    """The parametrised cases above contain clipped-low, clipped-high and in-range values."""
    seen = set()
    for seed, R, C, group, bits in [(0, 4, 4, 4, 4), (1, 4, 8, 4, 4), (2, 4, 8, 4, 2),
                                    (3, 6, 12, 6, 3), (4, 4, 16, 16, 4), (5, 8, 8, 4, 2)]:
        V, gl, bl, _ = _case(seed, R, C)
        ng = C // group
        g = om.sigmoid32(gl[:, :ng].numpy())
        b = om.sigmoid32(bl[:, :ng].numpy())
        enc = om.encode_affine(V.numpy(), g, b, bits, group)
        q = enc.r + np.repeat(enc.z, group, axis=1)
        seen |= {"low"} if (q < 0).any() else set()
        seen |= {"high"} if (q > 2 ** bits - 1).any() else set()
        seen |= {"in"} if enc.inrange.any() else set()
    assert seen == {"low", "high", "in"}


def test_ties_at_max_split_equally():
    V = torch.tensor([[0.3, -0.1, 0.3, 0.05, -0.2, 0.1, 0.3, 0.0]], dtype=torch.float32)
    g = om.sigmoid32(np.array([[1.0]], np.float32))
    b = om.sigmoid32(np.array([[2.0]], np.float32))
    enc = om.encode_affine(V.numpy(), g, b, 4, 8)
    assert enc.nmax[0, 0] == 3
    dD = torch.linspace(-1, 1, 8, dtype=torch.float64)[None, :]
    dV, dg, db = om.encode_backward(dD.numpy(), V.numpy(), enc, g, b)
    Vt = V.double().requires_grad_(True)
    gt = torch.from_numpy(g.astype(np.float64)).requires_grad_(True)
    bt = torch.from_numpy(b.astype(np.float64)).requires_grad_(True)
    (_autograd_encode(Vt, gt, bt, 4, 8) * dD).sum().backward()
    np.testing.assert_allclose(dV, Vt.grad.numpy(), rtol=1e-5, atol=2e-5)
    np.testing.assert_allclose(dg, gt.grad.numpy(), rtol=1e-5, atol=2e-5)


def _autograd_step(X, W, B, Yref, gl, bl, s, d, bits, group, abits, let):
    """The whole fake-quant linear + MSE in float64 autograd."""
    Xd = torch.from_numpy(X.astype(np.float64))
    Wd = torch.from_numpy(W.astype(np.float64))
    glt = torch.from_numpy(gl.astype(np.float64)).requires_grad_(True)
    blt = torch.from_numpy(bl.astype(np.float64)).requires_grad_(True)
    st = torch.from_numpy(s.astype(np.float64)).requires_grad_(True)
    dt = torch.from_numpy(d.astype(np.float64)).requires_grad_(True)
    if let:
        Wt = Wd * st[None, :]
        Xt = (Xd - dt[None, :]) / st[None, :]
        Bt = torch.from_numpy(B.astype(np.float64)) + Wd @ dt
    else:
        Wt, Xt, Bt = Wd, Xd, torch.from_numpy(B.astype(np.float64))
    What = _autograd_encode(Wt, torch.sigmoid(glt), torch.sigmoid(blt), bits, group)
    if abits < 16:
        one = torch.ones(Xt.shape[0], 1, dtype=torch.float64)
        Xq = _autograd_encode(Xt, one, one, abits, Xt.shape[1])
    else:
        Xq = Xt
    Y = Xq @ What.T + Bt[None, :]
    loss = ((Y - torch.from_numpy(Yref)) ** 2).mean()
    loss.backward()
    ds = None if st.grad is None else st.grad.numpy()
    dd = None if dt.grad is None else dt.grad.numpy()
    return loss.item(), glt.grad.numpy(), blt.grad.numpy(), ds, dd, Y


@pytest.mark.parametrize("abits,let,group", [(16, False, 8), (16, True, 4), (4, True, 8),
                                             (4, True, 4), (3, False, 8)])
def test_full_step_matches_autograd(abits, let, group):
    gen = torch.Generator().manual_seed(100 + abits + group)
    M, K, N, bits = 5, 8, 4, 4
    W = (torch.randn(N, K, generator=gen) * 0.1).numpy()
    X = torch.randn(M, K, generator=gen).numpy()
    X[:, 2] *= 8.0
    B = (torch.randn(N, generator=gen) * 0.1).numpy()
    Yref = (X.astype(np.float64) @ W.T.astype(np.float64) + B)
    gl = torch.empty(N, K // group).uniform_(0.0, 3.0, generator=gen).numpy()
    bl = torch.empty(N, K // group).uniform_(0.0, 3.0, generator=gen).numpy()
    s = (0.5 + torch.rand(K, generator=gen)).numpy()
    d = (0.3 * torch.randn(K, generator=gen)).numpy()
    r = om.calib_step(X, W, B, Yref, gl, bl, s, d, bits, group, abits, let)
    loss, dgl, dbl, ds, dd, Y = _autograd_step(X, W, B, Yref, gl, bl, s, d, bits, group,
                                               abits, let)
    # same forward (binary32 encoder decisions) as the float64 statement
    np.testing.assert_allclose(r.Y, Y.detach().numpy(), rtol=1e-5, atol=1e-6)
    assert abs(r.loss - loss) <= 1e-5 * abs(loss)
    np.testing.assert_allclose(r.d_gamma_logit, dgl, rtol=1e-4, atol=1e-9)
    np.testing.assert_allclose(r.d_beta_logit, dbl, rtol=1e-4, atol=1e-9)
    if let:
        np.testing.assert_allclose(r.d_s, ds, rtol=1e-4, atol=1e-8)
        np.testing.assert_allclose(r.d_delta, dd, rtol=1e-4, atol=1e-8)


def test_mse_gradient_matches_autograd():
    gen = torch.Generator().manual_seed(9)
    Y = torch.randn(7, 5, generator=gen, dtype=torch.float64, requires_grad=True)
    Yr = torch.randn(7, 5, generator=gen, dtype=torch.float64)
    loss = torch.nn.functional.mse_loss(Y, Yr)
    loss.backward()
    L, dY = om.mse_loss(Y.detach().numpy(), Yr.numpy())
    assert abs(L - loss.item()) < 1e-14
    np.testing.assert_allclose(dY, Y.grad.numpy(), rtol=1e-13)
