"""Pins of the block oracle (oracle/block.py) against what the pages and the mathematics fix.

- The hand-derived backward against an independent float64 autograd statement of the
  fake-quantized block (rounding as x + (round(x) - x).detach(); torch amax / amin for the
  ranges, which split gradients equally between ties), on tiny sizes, per-channel and
  grouped LWC, A4 and A16.
- "【ICLR 2024】OmniQuant ...", section LET: with the quantizers off, the channel-wise
  scaling / shifting of every linear's input, the affinity scaling Q / s_a, s_a K and the
  output projection's transform acting on V leave the block's output unchanged.
- Causality: the output of token t does not depend on later tokens.
- RoPE: rotations preserve norms and q_m . k_n depends only on m - n.
- RMSNorm output has unit mean square (up to eps); causal softmax rows sum to one.
- Planted mistakes in the oracle's backward make the autograd pin fail.
"""
import numpy as np
import pytest
import torch

from oracle import block as ob
from oracle import omniquant as om


def _ste_round(x):
    return x + (torch.round(x) - x).detach()


def _encode(V, g, b, bits, group):
    R, C = V.shape
    Vg = V.reshape(R, C // group, group)
    Q = float(2 ** bits - 1)
    M = Vg.amax(-1)
    m = Vg.amin(-1)
    h = ((g * M - b * m) / Q).clamp(min=1e-8)
    z = -_ste_round(b * m / h)
    q = _ste_round(Vg / h[..., None]) + z[..., None]
    return ((q.clamp(0.0, Q) - z[..., None]) * h[..., None]).reshape(R, C)


def _act(V, abits, width):
    if abits >= 16:
        return V
    one = torch.ones(V.shape[0], V.shape[1] // width, dtype=V.dtype)
    return _encode(V, one, one, abits, width)


def _f32(t):
    """Round to binary32 where a kernel stores binary32 (gradient passes through)."""
    return t.float().double()


def _rope(X, cos, sin, H):
    # binary32 rotation, one rounding per operation
    M, D = X.shape
    Dh = D // H
    Xh = X.float().reshape(M, H, Dh)
    lo, hi = Xh[:, :, :Dh // 2], Xh[:, :, Dh // 2:]
    c = torch.from_numpy(cos)[:, None, :]
    s = torch.from_numpy(sin)[:, None, :]
    return torch.cat([lo * c - hi * s, hi * c + lo * s], dim=2).reshape(M, D).double()


def _autograd_block(sh, x, W, theta, y_ref):
    """The whole fake-quantized block and its MSE in float64 autograd (written independently
    of the oracle's stage functions)."""
    parts = ob.theta_split(sh, theta.astype(np.float32))
    P = {k: torch.from_numpy(v.astype(np.float64)).requires_grad_(True) for k, v in parts.items()}
    Wd = {k: torch.from_numpy(np.asarray(v, np.float64)) for k, v in W.items()}
    M, D, H, I, A = sh.M, sh.D, sh.H, sh.I, sh.abits
    Dh = D // H
    cos, sin = ob.rope_table(M, Dh)

    def wq(name, s):
        Wn = Wd[name]
        Wt = Wn * s[None, :] if s is not None else Wn
        if sh.wbits >= 16:
            return Wt
        K = Wn.shape[1]
        G = sh.group_of(K)
        g = torch.sigmoid(P["gamma_" + name]).float().double().reshape(Wn.shape[0], K // G)
        b = torch.sigmoid(P["beta_" + name]).float().double().reshape(Wn.shape[0], K // G)
        return _encode(Wt.float().double(), g, b, sh.wbits, G)

    def norm(t):
        return t / torch.sqrt((t * t).mean(1, keepdim=True) + 1e-6)

    def let(t32, s, d):
        # binary32 (X - delta) / s
        return ((t32.float() - d.float()[None, :]) / s.float()[None, :]).double()

    xt = torch.from_numpy(np.asarray(x, np.float64))
    a = _f32(norm(xt))
    qa = _act(let(a, P["s1"], P["delta1"]), A, D)
    qkv = _f32(qa @ wq("qkv", P["s1"]).T + Wd["qkv"] @ P["delta1"])
    q, k, v = qkv[:, :D], qkv[:, D:2 * D], qkv[:, 2 * D:]
    qt = (_rope(q, cos, sin, H).float() / P["s_a"].float()[None, :]).double()
    kt = (_rope(k, cos, sin, H).float() * P["s_a"].float()[None, :]).double()
    vt = let(v, P["s_o"], P["delta_o"])
    Qq, Qk, Qv = _act(qt, A, Dh), _act(kt, A, Dh), _act(vt, A, Dh)
    hq = Qq.reshape(M, H, Dh).transpose(0, 1)
    hk = Qk.reshape(M, H, Dh).transpose(0, 1)
    hv = Qv.reshape(M, H, Dh).transpose(0, 1)
    S = hq @ hk.transpose(1, 2) / np.sqrt(Dh)
    mask = torch.tril(torch.ones(M, M, dtype=torch.bool))
    Pm = torch.softmax(S.masked_fill(~mask, float("-inf")), dim=-1)
    O = _f32((Pm @ hv).transpose(0, 1).reshape(M, D))
    o_out = _act(O, A, D) @ wq("o", P["s_o"]).T + Wd["o"] @ P["delta_o"]
    x2 = xt + o_out
    bn = _f32(norm(x2))
    qb = _act(let(bn, P["s2"], P["delta2"]), A, D)
    gu = _f32(qb @ wq("gu", P["s2"]).T + Wd["gu"] @ P["delta2"])
    m = _f32(torch.nn.functional.silu(gu[:, :I]) * gu[:, I:])
    y = x2 + _act(m, A, I) @ wq("d", None).T
    loss = ((y - torch.from_numpy(y_ref)) ** 2).mean()
    loss.backward()
    grads = {}
    for name, _ in ob.theta_layout(sh):
        gr = P[name].grad
        grads[name] = np.zeros(P[name].shape) if gr is None else gr.numpy()
    return loss.item(), ob.theta_join(sh, grads), y.detach().numpy()


def make_case(sh, seed, let_spread=0.3):
    gen = torch.Generator().manual_seed(seed)
    M, D, I = sh.M, sh.D, sh.I
    x = torch.randn(M, D, generator=gen)
    x[:, 1] *= 6.0                                  # one outlier channel
    W = {"qkv": torch.randn(3 * D, D, generator=gen) * 0.2,
         "o": torch.randn(D, D, generator=gen) * 0.2,
         "gu": torch.randn(2 * I, D, generator=gen) * 0.2,
         "d": torch.randn(D, I, generator=gen) * 0.2}
    W = {k: v.to(torch.bfloat16).float().numpy() for k, v in W.items()}
    parts = {}
    for name, n in ob.theta_layout(sh):
        if name.startswith(("gamma", "beta")):
            parts[name] = torch.empty(n).uniform_(0.5, 4.0, generator=gen).numpy()
        elif name.startswith("delta"):
            parts[name] = (let_spread * torch.randn(n, generator=gen)).numpy()
        else:
            parts[name] = (1.0 + let_spread * (torch.rand(n, generator=gen) - 0.5)).numpy()
    theta = ob.theta_join(sh, parts).astype(np.float32)
    return x.numpy(), W, theta


def _rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300)


SHAPES = [
    ob.BlockShape(M=6, D=16, H=2, I=24, wbits=4, abits=4),
    ob.BlockShape(M=5, D=16, H=2, I=24, wbits=4, abits=16),
    ob.BlockShape(M=7, D=32, H=4, I=16, wbits=3, abits=4, group=8),
    ob.BlockShape(M=4, D=16, H=1, I=32, wbits=2, abits=8, group=8),
]


@pytest.mark.parametrize("si", range(len(SHAPES)))
def test_block_backward_matches_autograd(si):
    sh = SHAPES[si]
    x, W, theta = make_case(sh, 40 + si)
    y_ref = ob.block_reference(sh, x, W)
    loss, grad, st, _ = ob.block_step(sh, x, W, theta, y_ref)
    aloss, agrad, ay = _autograd_block(sh, x, W, theta, y_ref)
    # the same integer decisions: identical forward up to rounding order
    np.testing.assert_allclose(st["y"], ay, rtol=1e-6, atol=1e-6)
    assert abs(loss - aloss) <= 1e-6 * aloss
    # per parameter tensor; a dropped term or a sign error moves these at the 1e-1 level.
    # Unquantized Q and K make the affinity scaling exactly invariant: d s_a is then zero
    # up to rounding on both sides.
    scale = np.linalg.norm(agrad)
    off = 0
    for name, n in ob.theta_layout(sh):
        g, ag = grad[off:off + n], agrad[off:off + n]
        off += n
        if name == "s_a" and sh.abits >= 16:
            assert np.linalg.norm(g) < 1e-6 * scale and np.linalg.norm(ag) < 1e-6 * scale
            continue
        if np.linalg.norm(ag) == 0:
            assert np.linalg.norm(g) == 0, name
            continue
        assert _rel(g, ag) < 2e-5, (name, _rel(g, ag))


def test_every_parameter_gets_a_gradient():
    sh = SHAPES[0]
    x, W, theta = make_case(sh, 40)
    _, grad, _, _ = ob.block_step(sh, x, W, theta, ob.block_reference(sh, x, W))
    off = 0
    for name, n in ob.theta_layout(sh):
        assert np.abs(grad[off:off + n]).max() > 0, name
        off += n


@pytest.mark.parametrize("seed", [0, 1])
def test_transforms_leave_unquantized_block_unchanged(seed):
    sh = ob.BlockShape(M=9, D=32, H=2, I=40, wbits=16, abits=16)
    x, W, theta = make_case(sh, 70 + seed, let_spread=0.8)
    th = ob.theta_split(sh, theta)
    y = ob.block_forward(sh, x, W, th)["y"]
    y_ref = ob.block_reference(sh, x, W)
    # binary32 storage of the intermediates is the only difference
    assert _rel(y, y_ref) < 1e-6


def test_transform_pin_rejects_wrong_affinity_direction(monkeypatch):
    real = ob.stage_attn_prep

    def bad(qkv32, cos, sin, s_a, s_o, delta_o, H, abits):
        # planted: K divided by s_a like Q (instead of s_a K): the affinities change
        ap = real(qkv32, cos, sin, s_a, s_o, delta_o, H, abits)
        ap["kt"] = ap["kr"] / np.asarray(s_a, np.float32)[None, :]
        ap["Qk"] = ap["kt"]
        return ap
    monkeypatch.setattr(ob, "stage_attn_prep", bad)
    with pytest.raises(AssertionError):
        test_transforms_leave_unquantized_block_unchanged(0)


def test_causal():
    sh = SHAPES[0]
    x, W, theta = make_case(sh, 5)
    th = ob.theta_split(sh, theta)
    y0 = ob.block_forward(sh, x, W, th)["y"]
    x1 = x.copy()
    x1[4:] = np.random.default_rng(1).standard_normal(x1[4:].shape).astype(np.float32)
    y1 = ob.block_forward(sh, x1, W, th)["y"]
    np.testing.assert_allclose(y1[:4], y0[:4], rtol=1e-12, atol=1e-12)
    assert np.abs(y1[4:] - y0[4:]).max() > 1e-3


def test_rope_relative_position_and_norm():
    M, Dh = 40, 16
    cos, sin = ob.rope_table(M, Dh)
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, Dh)).astype(np.float32)
    k = rng.standard_normal((1, Dh)).astype(np.float32)
    Q = ob.rope32(np.repeat(q, M, 0), cos, sin, 1).astype(np.float64)
    K = ob.rope32(np.repeat(k, M, 0), cos, sin, 1).astype(np.float64)
    np.testing.assert_allclose(np.linalg.norm(Q, axis=1), np.linalg.norm(q), rtol=1e-6)
    for d in (0, 3, 11):
        dots = np.array([Q[m + d] @ K[m] for m in range(0, M - d)])
        np.testing.assert_allclose(dots, dots[0], rtol=1e-4, atol=1e-5)
    # position 0 is the identity; the first pair at position 1 turns by exactly 1 radian
    np.testing.assert_array_equal(Q[0], q[0])
    np.testing.assert_allclose(cos[1, 0], np.cos(1.0), rtol=1e-7)
    # rope_backward is the transpose of the rotation
    dQ = rng.standard_normal((M, Dh))
    X = rng.standard_normal((M, Dh)).astype(np.float32)
    lhs = (ob.rope32(X, cos, sin, 1).astype(np.float64) * dQ).sum()
    rhs = (X.astype(np.float64) * ob.rope_backward(dQ, cos, sin, 1)).sum()
    assert abs(lhs - rhs) < 1e-5 * abs(lhs)


def test_rms_norm_and_softmax_invariants():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 64)) * 3.0
    n, rstd = ob.rms_norm(x)
    ms = (n * n).mean(1)
    np.testing.assert_allclose(ms, (x * x).mean(1) / ((x * x).mean(1) + 1e-6), rtol=1e-12)
    P = ob.causal_softmax(rng.standard_normal((2, 6, 6)))
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=1e-12)
    assert (P[:, np.triu_indices(6, 1)[0], np.triu_indices(6, 1)[1]] == 0).all()
    np.testing.assert_array_equal(P[:, 0, 0], 1.0)


def _mutant_drop_rowsum(dO, P, Qq, Qk, Qv, H):
    q, k, v = (ob.heads(np.asarray(t, np.float64), H) for t in (Qq, Qk, Qv))
    do = ob.heads(np.asarray(dO, np.float64), H)
    dv = np.einsum("hmn,hmd->hnd", P, do)
    dP = np.einsum("hmd,hnd->hmn", do, v)
    dS = P * dP / np.sqrt(q.shape[-1])     # planted: the softmax's rowsum term is dropped
    return (ob.unheads(np.einsum("hmn,hnd->hmd", dS, k)),
            ob.unheads(np.einsum("hmn,hmd->hnd", dS, q)), ob.unheads(dv))


def _mutant_rope_sign(dXr, cos, sin, H):
    return _real_rope_bwd(dXr, cos, -sin, H)   # planted: forward rotation used backward


_real_rope_bwd = ob.rope_backward


def _mutant_rms(dn, n, rstd):
    return rstd[:, None] * np.asarray(dn, np.float64)   # planted: the mean term is dropped


@pytest.mark.parametrize("name,mutant", [("stage_attention_backward", _mutant_drop_rowsum),
                                         ("rope_backward", _mutant_rope_sign),
                                         ("rms_backward", _mutant_rms)])
def test_block_pin_rejects_mutant(monkeypatch, name, mutant):
    monkeypatch.setattr(ob, name, mutant)
    with pytest.raises(AssertionError):
        test_block_backward_matches_autograd(0)


def test_stage_functions_compose():
    """The forward stages called one by one on the stored tensors give block_forward's y."""
    sh = SHAPES[0]
    x, W, theta = make_case(sh, 8)
    th = ob.theta_split(sh, theta)
    st = ob.block_forward(sh, x, W, th)
    ap = ob.stage_attn_prep(st["qkv32"], st["cos"], st["sin"], th["s_a"], th["s_o"],
                            th["delta_o"], sh.H, sh.abits)
    np.testing.assert_array_equal(ap["Qq"], st["Qq"])
    P, O = ob.stage_attention(ap["Qq"], ap["Qk"], ap["Qv"], sh.H)
    np.testing.assert_array_equal(O.astype(np.float32), st["O32"])
    assert om.F32 is np.float32


def test_block_calibrate_is_steps_then_adamw():
    """One epoch over one sample: the loss of block_step, then AdamW from zero moments (whose
    first step moves every parameter by -lr sign(g) up to eps: the bias corrections cancel)."""
    sh = SHAPES[1]
    x, W, theta = make_case(sh, 77)
    losses, theta1, _ = ob.block_calibrate(sh, [x], W, theta, 1)
    loss, g, _, _ = ob.block_step(sh, x, W, theta, ob.block_reference(sh, x, W))
    assert losses[0] == loss
    split = sum(n for name, n in ob.theta_layout(sh) if name.startswith(("gamma", "beta")))
    lr = np.where(np.arange(theta.size) < split, om.LR_LWC, om.LR_LET)
    step = lr * g / (np.abs(g) + 1e-8)
    np.testing.assert_allclose(theta1, (theta - step).astype(np.float32), rtol=0, atol=1e-6)
