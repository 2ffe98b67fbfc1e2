"""CPU oracle of OmniQuant's block-wise calibration step on one LLaMA-shaped transformer block.

TEST INFRASTRUCTURE, like ``oracle.omniquant`` (whose encoder, STE and LET primitives this
module composes): only tests/, __graft_entry__.smoke() and the CPU-baseline leg of bench.py
may import or run it, and it imports nothing from the product.

What it computes, and where the pages define it ([ICLR] = "【ICLR 2024】OmniQuant:
Omnidirectionally Calibrated Quantization for Large Language Models", onecrewdev.com):
  - section 框架: the objective is the block output's reconstruction error against the
    full-precision block, over Theta1 = {gamma, beta} (LWC) and Theta2 = {delta, s, s_a} (LET).
  - section LET: every linear's input takes X~ = (X - delta)/s with W~ = s W, B~ = B + delta W,
    except the FFN's second linear (its input follows the nonlinearity); the attention
    affinity takes Q~ = Q / s_a and K~ = s_a K, which leaves softmax(Q K^T) unchanged; Q, K
    and V are quantized; V's own transform is the inverse of the output projection's LET
    (so the o_proj shift and scale act on V, exact because each row of the softmax sums to
    one); the softmax output stays in full precision.
  - section LWC and 实验证据: the weight and per-token activation quantizers, as in
    ``oracle.omniquant``.

The block (readings of what the pages leave open, each listed in the design notes):
    a   = RMSNorm(x)                      (eps 1e-6, weight 1)
    qa  = Q_a((a - delta1)/s1)            per token
    [q, k, v] = qa W^_qkv^T + W_qkv delta1     (W~_qkv = s1 W_qkv; W_qkv rows: q, k, v)
    q~  = RoPE(q) / s_a,  k~ = RoPE(k) s_a,  v~ = (v - delta_o)/s_o
    Qq, Qk, Qv = Q_a(.) per (token, head) row of Dh values
    P_h = softmax(causal(Qq_h Qk_h^T / sqrt(Dh)))     full precision
    O   = [P_h Qv_h]_h
    x2  = x + Q_a(O) W^_o^T + W_o delta_o              (W~_o = s_o W_o; Q_a per token)
    b   = RMSNorm(x2);  qb = Q_a((b - delta2)/s2)
    [gate, up] = qb W^_gu^T + W_gu delta2              (W_gu rows: gate, up)
    m   = SiLU(gate) up;  qm = Q_a(m)     (no LET)
    y   = x2 + qm W^_d^T
    L   = mean (y - y*)^2,  y* = the same block with every quantizer and transform removed.
RoPE is the rotate-half form (pairs (i, i + Dh/2)), base 10000, positions 0 .. M-1.

Precision follows ``oracle.omniquant``: the value path and every gradient are binary64; each
tensor that a kernel stores in binary32 and then encodes (a, b, q, k, v, O, m) is rounded to
binary32, and the transforms applied to it before the encoder (LET, RoPE, s_a) run in
binary32, one rounding per operation, in a fixed order:
    x_r[i] = x[i] c - x[i + Dh/2] s,  x_r[i + Dh/2] = x[i + Dh/2] c + x[i] s
    q~ = q_r / s_a,  k~ = k_r s_a,  v~ = (v - delta_o) / s_o
with c, s the binary64 cosine and sine of position * 10000^(-2i/Dh), each rounded once.

Pins (tests/test_oracle_block.py): the hand-derived backward against a float64 autograd
statement of the block on tiny sizes; LET, affinity and V/o transforms leave the unquantized
block's output unchanged; causality; RoPE's relative-position property and norm
preservation; RMSNorm output RMS; the stage functions compose to ``block_step``.
``block_calibrate`` against torch.optim.AdamW driving that autograd statement over two samples
and two epochs (tests/test_oracle_calibrate.py).
"""
from __future__ import annotations

import dataclasses

import numpy as np

from oracle import omniquant as om

F32 = np.float32
F64 = np.float64


@dataclasses.dataclass(frozen=True)
class BlockShape:
    M: int            # tokens
    D: int            # hidden size
    H: int            # heads
    I: int            # FFN intermediate size
    wbits: int = 4
    abits: int = 4
    group: int = 0    # 0: per output channel (one group per weight row)
    eps: float = 1e-6
    rope_base: float = 10000.0

    @property
    def Dh(self) -> int:
        return self.D // self.H

    def group_of(self, K: int) -> int:
        return K if self.group == 0 else self.group


# Parameter vector layout: one float32 vector holds every learnable tensor of the block.
# LWC logits are one per (row, group) of each weight; LET vectors are one per channel.
def theta_layout(sh: BlockShape):
    """Ordered (name, length) pairs of the parameter vector."""
    D, I = sh.D, sh.I
    ng = lambda rows, K: rows * (K // sh.group_of(K))  # noqa: E731
    return [
        ("gamma_qkv", ng(3 * D, D)), ("beta_qkv", ng(3 * D, D)),
        ("gamma_o", ng(D, D)), ("beta_o", ng(D, D)),
        ("gamma_gu", ng(2 * I, D)), ("beta_gu", ng(2 * I, D)),
        ("gamma_d", ng(D, I)), ("beta_d", ng(D, I)),
        ("s1", D), ("delta1", D), ("s_a", D), ("s_o", D), ("delta_o", D),
        ("s2", D), ("delta2", D),
    ]


def theta_split(sh: BlockShape, theta):
    out, off = {}, 0
    for name, n in theta_layout(sh):
        out[name] = np.asarray(theta[off:off + n])
        off += n
    return out


def theta_join(sh: BlockShape, parts) -> np.ndarray:
    return np.concatenate([np.asarray(parts[n], F64).reshape(-1) for n, _ in theta_layout(sh)])


# ----------------------------------------------------------------------------- primitives

def rms_norm(x):
    """RMSNorm with unit weight, binary64: x / sqrt(mean(x^2) + eps) per row.

    Returns (normalized [M, D], rstd [M])."""
    x = np.asarray(x, F64)
    rstd = 1.0 / np.sqrt((x * x).mean(axis=1) + 1e-6)
    return x * rstd[:, None], rstd


def rope_table(M: int, Dh: int, base: float = 10000.0):
    """cos and sin of position * base^(-2i/Dh), i < Dh/2, in binary64, each rounded once to
    binary32: [M, Dh/2] each."""
    i = np.arange(Dh // 2, dtype=F64)
    inv = base ** (-2.0 * i / Dh)
    ang = np.arange(M, dtype=F64)[:, None] * inv[None, :]
    return np.cos(ang).astype(F32), np.sin(ang).astype(F32)


def rope32(X, cos, sin, H: int):
    """Rotate-half RoPE of every head of X [M, H*Dh] in binary32 (the fixed order above)."""
    X = np.asarray(X, F32)
    M, D = X.shape
    Dh = D // H
    half = Dh // 2
    Xh = X.reshape(M, H, Dh)
    lo, hi = Xh[:, :, :half], Xh[:, :, half:]
    c, s = cos[:, None, :], sin[:, None, :]
    out = np.empty_like(Xh)
    out[:, :, :half] = lo * c - hi * s
    out[:, :, half:] = hi * c + lo * s
    return out.reshape(M, D)


def rope_backward(dXr, cos, sin, H: int):
    """Gradient through the rotation (its transpose), binary64."""
    dXr = np.asarray(dXr, F64)
    M, D = dXr.shape
    Dh = D // H
    half = Dh // 2
    d = dXr.reshape(M, H, Dh)
    dlo, dhi = d[:, :, :half], d[:, :, half:]
    c, s = cos.astype(F64)[:, None, :], sin.astype(F64)[:, None, :]
    out = np.empty_like(d)
    out[:, :, :half] = dlo * c + dhi * s
    out[:, :, half:] = dhi * c - dlo * s
    return out.reshape(M, D)


def act_encode(V32, abits: int, width: int):
    """Activation fake-quant: MinMax affine (gamma = beta = 1) over each run of ``width``
    values along a row (width = row length: per token; width = Dh: per (token, head)).
    Returns (dequantized float32, Encoded or None when abits == 16)."""
    V32 = np.asarray(V32, F32)
    if abits >= 16:
        return V32.copy(), None
    R, C = V32.shape
    one = np.ones((R, C // width), F32)
    enc = om.encode_affine(V32, one, one, abits, width)
    return enc.deq, enc


def act_backward(dDeq, V32, enc):
    """Straight-through gradient of ``act_encode`` (identity when not quantized)."""
    if enc is None:
        return np.asarray(dDeq, F64)
    R, C = enc.codes.shape
    one = np.ones((R, C // enc.group), F32)
    dV, _, _ = om.encode_backward(dDeq, V32, enc, one, one)
    return dV


def causal_softmax(S):
    """Row softmax of S [H, M, M] with the entries above the diagonal removed (binary64)."""
    S = np.asarray(S, F64)
    M = S.shape[-1]
    mask = np.tril(np.ones((M, M), dtype=bool))
    Sm = np.where(mask, S, -np.inf)
    Sm = Sm - Sm.max(axis=-1, keepdims=True)
    E = np.exp(Sm)
    return E / E.sum(axis=-1, keepdims=True)


def silu(x):
    x = np.asarray(x, F64)
    return x / (1.0 + np.exp(-x))


def weight_quant(W, s, gl, bl, bits: int, group: int):
    """LWC weight side: (W~ float32, Encoded or None, g, b, W^ float32)."""
    if bits >= 16:
        Wt = om.let_weight(W, s)
        return Wt, None, None, None, Wt
    Wt, enc, g, b = om.lwc_quant(W, s, gl.reshape(W.shape[0], -1), bl.reshape(W.shape[0], -1),
                                 bits, group)
    return Wt, enc, g, b, enc.deq


# ----------------------------------------------------------------------------- stages

def stage_norm_let_quant(x, s, delta, abits: int):
    """RMSNorm, then the linear's LET and per-token act quant.

    Returns (n32 = RMSNorm(x) rounded to binary32, rstd, nt32 = (n32 - delta)/s in binary32,
    Encoded or None, Q_a(nt32) float32)."""
    n, rstd = rms_norm(x)
    n32 = n.astype(F32)
    nt32 = om.let_act(n32, s, delta)
    deq, enc = act_encode(nt32, abits, nt32.shape[1])
    return n32, rstd, nt32, enc, deq


def stage_attn_prep(qkv32, cos, sin, s_a, s_o, delta_o, H: int, abits: int):
    """RoPE on q and k, the affinity LET (q / s_a, k s_a), the o_proj LET on v ((v - delta_o)
    / s_o), and the per-(token, head) act quant of the three. binary32 throughout.

    Returns dict with qr, kr (rotated), qt, kt, vt (transformed), enc_q/k/v, Qq, Qk, Qv."""
    qkv32 = np.asarray(qkv32, F32)
    M, D3 = qkv32.shape
    D = D3 // 3
    Dh = D // H
    q, k, v = qkv32[:, :D], qkv32[:, D:2 * D], qkv32[:, 2 * D:]
    qr = rope32(q, cos, sin, H)
    kr = rope32(k, cos, sin, H)
    sa = np.asarray(s_a, F32)[None, :]
    qt = qr / sa
    kt = kr * sa
    vt = om.let_act(v, s_o, delta_o)
    Qq, eq = act_encode(qt, abits, Dh)
    Qk, ek = act_encode(kt, abits, Dh)
    Qv, ev = act_encode(vt, abits, Dh)
    return dict(qr=qr, kr=kr, qt=qt, kt=kt, vt=vt, enc_q=eq, enc_k=ek, enc_v=ev, Qq=Qq, Qk=Qk,
                Qv=Qv)


def heads(X, H: int):
    """[M, H*Dh] -> [H, M, Dh]."""
    X = np.asarray(X)
    M, D = X.shape
    return X.reshape(M, H, D // H).transpose(1, 0, 2)


def unheads(Xh):
    """[H, M, Dh] -> [M, H*Dh]."""
    H, M, Dh = Xh.shape
    return np.ascontiguousarray(Xh.transpose(1, 0, 2)).reshape(M, H * Dh)


def stage_attention(Qq, Qk, Qv, H: int):
    """P_h = causal softmax(Qq_h Qk_h^T / sqrt(Dh)), O = [P_h Qv_h]. binary64.
    Returns (P [H, M, M], O [M, D])."""
    q, k, v = (heads(np.asarray(t, F64), H) for t in (Qq, Qk, Qv))
    Dh = q.shape[-1]
    S = np.einsum("hmd,hnd->hmn", q, k) / np.sqrt(Dh)
    P = causal_softmax(S)
    O = unheads(np.einsum("hmn,hnd->hmd", P, v))
    return P, O


def stage_attention_backward(dO, P, Qq, Qk, Qv, H: int):
    """Gradients of O = [P_h Qv_h] through the softmax to the quantized Q, K, V (binary64):
    dQv_h = P_h^T dO_h, dP_h = dO_h Qv_h^T, dS = P (dP - rowsum(P dP)) / sqrt(Dh),
    dQq_h = dS Qk_h, dQk_h = dS^T Qq_h. Returns (dQq, dQk, dQv) [M, D]."""
    q, k, v = (heads(np.asarray(t, F64), H) for t in (Qq, Qk, Qv))
    do = heads(np.asarray(dO, F64), H)
    Dh = q.shape[-1]
    dv = np.einsum("hmn,hmd->hnd", P, do)
    dP = np.einsum("hmd,hnd->hmn", do, v)
    dS = P * (dP - (P * dP).sum(axis=-1, keepdims=True)) / np.sqrt(Dh)
    dq = np.einsum("hmn,hnd->hmd", dS, k)
    dk = np.einsum("hmn,hmd->hnd", dS, q)
    return unheads(dq), unheads(dk), unheads(dv)


def rms_backward(dn, n, rstd):
    """Gradient of n = x * rstd(x) (unit weight): dx = rstd (dn - n mean(dn n)). binary64."""
    dn = np.asarray(dn, F64)
    n = np.asarray(n, F64)
    return rstd[:, None] * (dn - n * (dn * n).mean(axis=1, keepdims=True))


def let_grads(dWt, W, dXt, Xt32, s, dBt):
    """LET parameter gradients of one linear ([ICLR] section LET, chain rule):
    W~ = W s: ds += sum_n dW~ W;  X~ = (X - delta)/s: ds -= sum_m dX~ X~ / s,
    ddelta -= sum_m dX~ / s;  B~ = B + W delta: ddelta += W^T dB~.
    Any of the three sides may be None."""
    K = (W if W is not None else Xt32).shape[1]
    s64 = np.ones(K) if s is None else np.asarray(s, F64)
    ds = np.zeros(K)
    dd = np.zeros(K)
    if dWt is not None:
        ds += (np.asarray(dWt, F64) * np.asarray(W, F64)).sum(axis=0)
    if dXt is not None:
        ds -= (dXt * np.asarray(Xt32, F64)).sum(axis=0) / s64
        dd -= dXt.sum(axis=0) / s64
    if dBt is not None:
        dd += np.asarray(W, F64).T @ dBt
    return ds, dd


# ----------------------------------------------------------------------------- the step

WEIGHTS = ("qkv", "o", "gu", "d")          # [3D, D], [D, D], [2I, D], [D, I]


def _weights_quant(sh: BlockShape, W, th):
    """LWC (with the LET scale of each linear's input) of the four weights."""
    D, I = sh.D, sh.I
    let_s = {"qkv": th["s1"], "o": th["s_o"], "gu": th["s2"], "d": None}
    out = {}
    for name in WEIGHTS:
        Wn = np.asarray(W[name], F32)
        K = Wn.shape[1]
        assert K == (I if name == "d" else D)
        out[name] = weight_quant(Wn, let_s[name], th["gamma_" + name], th["beta_" + name],
                                 sh.wbits, sh.group_of(K))
    return out


def block_forward(sh: BlockShape, x, W, th, y_ref=None):
    """Forward of the fake-quantized block (the formulas in the module docstring).

    x: [M, D]; W: dict of the four weights (float32 values); th: theta_split(...) dict.
    Returns a dict of every intermediate (float32 where a kernel stores binary32), with the
    loss when y_ref is given."""
    M, D, H, I, A = sh.M, sh.D, sh.H, sh.I, sh.abits
    x64 = np.asarray(x, F64)
    cos, sin = rope_table(M, sh.Dh, sh.rope_base)
    wq = _weights_quant(sh, W, th)
    st = dict(cos=cos, sin=sin, wq=wq)
    a32, rstd1, at32, enc_a, qa = stage_norm_let_quant(x64, th["s1"], th["delta1"], A)
    st.update(a32=a32, rstd1=rstd1, at32=at32, enc_a=enc_a, qa=qa)
    Bt_qkv = om.let_bias(W["qkv"], None, th["delta1"])
    qkv = qa.astype(F64) @ wq["qkv"][4].astype(F64).T + Bt_qkv[None, :]
    qkv32 = qkv.astype(F32)
    st.update(Bt_qkv=Bt_qkv, qkv32=qkv32)
    ap = stage_attn_prep(qkv32, cos, sin, th["s_a"], th["s_o"], th["delta_o"], H, A)
    st.update(ap)
    P, O = stage_attention(ap["Qq"], ap["Qk"], ap["Qv"], H)
    O32 = O.astype(F32)
    Qo, enc_o = act_encode(O32, A, D)
    st.update(P=P, O32=O32, Qo=Qo, enc_o=enc_o)
    Bt_o = om.let_bias(W["o"], None, th["delta_o"])
    o_out = Qo.astype(F64) @ wq["o"][4].astype(F64).T + Bt_o[None, :]
    x2 = x64 + o_out
    st.update(Bt_o=Bt_o, o_out=o_out, x2=x2)
    b32, rstd2, bt32, enc_b, qb = stage_norm_let_quant(x2, th["s2"], th["delta2"], A)
    st.update(b32=b32, rstd2=rstd2, bt32=bt32, enc_b=enc_b, qb=qb)
    Bt_gu = om.let_bias(W["gu"], None, th["delta2"])
    gu = qb.astype(F64) @ wq["gu"][4].astype(F64).T + Bt_gu[None, :]
    gu32 = gu.astype(F32)
    m32 = (silu(gu32[:, :I]) * gu32[:, I:].astype(F64)).astype(F32)
    qm, enc_m = act_encode(m32, A, I)
    st.update(Bt_gu=Bt_gu, gu32=gu32, m32=m32, qm=qm, enc_m=enc_m)
    d_out = qm.astype(F64) @ wq["d"][4].astype(F64).T
    y = x2 + d_out
    st.update(d_out=d_out, y=y)
    if y_ref is not None:
        st["loss"], st["dy"] = om.mse_loss(y, y_ref)
    return st


def _lwc_grads(dWhat, wq_entry):
    """STE through one weight's LWC: (dW~, d gamma logit, d beta logit) in binary64."""
    Wt, enc, g, b, _ = wq_entry
    if enc is None:
        z = np.zeros(0)
        return np.asarray(dWhat, F64), z, z
    dWt, dg, db = om.encode_backward(dWhat, Wt, enc, g, b)
    g64, b64 = g.astype(F64), b.astype(F64)
    return dWt, (dg * g64 * (1 - g64)).reshape(-1), (db * b64 * (1 - b64)).reshape(-1)


def block_backward(sh: BlockShape, W, th, st):
    """Straight-through backward of ``block_forward`` (chain rule through every stage, each
    quantizer's gradient from oracle.omniquant.encode_backward). Returns the dict of
    parameter gradients (names of theta_layout) plus the intermediate gradients."""
    D, H, I = sh.D, sh.H, sh.I
    wq = st["wq"]
    g = {}
    dy = st["dy"]
    # down projection (no LET)
    dWh_d = dy.T @ st["qm"].astype(F64)
    _, g["gamma_d"], g["beta_d"] = _lwc_grads(dWh_d, wq["d"])
    dqm = dy @ wq["d"][4].astype(F64)
    dm = act_backward(dqm, st["m32"], st["enc_m"])
    # SwiGLU: m = silu(gate) up
    gate = st["gu32"][:, :I].astype(F64)
    up = st["gu32"][:, I:].astype(F64)
    sg = 1.0 / (1.0 + np.exp(-gate))
    dgu = np.concatenate([dm * up * sg * (1.0 + gate * (1.0 - sg)), dm * gate * sg], axis=1)
    # gate / up projection (LET s2, delta2)
    dWh_gu = dgu.T @ st["qb"].astype(F64)
    dWt_gu, g["gamma_gu"], g["beta_gu"] = _lwc_grads(dWh_gu, wq["gu"])
    dqb = dgu @ wq["gu"][4].astype(F64)
    dbt = act_backward(dqb, st["bt32"], st["enc_b"])
    g["s2"], g["delta2"] = let_grads(dWt_gu, W["gu"], dbt, st["bt32"], th["s2"], dgu.sum(axis=0))
    db = dbt / np.asarray(th["s2"], F64)[None, :]
    b64 = st["x2"] * st["rstd2"][:, None]
    dx2 = dy + rms_backward(db, b64, st["rstd2"])
    # output projection (its LET acts on V)
    dWh_o = dx2.T @ st["Qo"].astype(F64)
    dWt_o, g["gamma_o"], g["beta_o"] = _lwc_grads(dWh_o, wq["o"])
    dQo = dx2 @ wq["o"][4].astype(F64)
    dO = act_backward(dQo, st["O32"], st["enc_o"])
    # attention
    dQq, dQk, dQv = stage_attention_backward(dO, st["P"], st["Qq"], st["Qk"], st["Qv"], H)
    dqt = act_backward(dQq, st["qt"], st["enc_q"])
    dkt = act_backward(dQk, st["kt"], st["enc_k"])
    dvt = act_backward(dQv, st["vt"], st["enc_v"])
    sa = np.asarray(th["s_a"], F64)[None, :]
    g["s_a"] = (dkt * st["kr"].astype(F64)).sum(axis=0) - (dqt * st["qt"].astype(F64)).sum(
        axis=0) / sa[0]
    g["s_o"], g["delta_o"] = let_grads(dWt_o, W["o"], dvt, st["vt"], th["s_o"], dx2.sum(axis=0))
    dq = rope_backward(dqt / sa, st["cos"], st["sin"], H)
    dk = rope_backward(dkt * sa, st["cos"], st["sin"], H)
    dv = dvt / np.asarray(th["s_o"], F64)[None, :]
    dqkv = np.concatenate([dq, dk, dv], axis=1)
    # q / k / v projection (LET s1, delta1)
    dWh_qkv = dqkv.T @ st["qa"].astype(F64)
    dWt_qkv, g["gamma_qkv"], g["beta_qkv"] = _lwc_grads(dWh_qkv, wq["qkv"])
    dqa = dqkv @ wq["qkv"][4].astype(F64)
    dat = act_backward(dqa, st["at32"], st["enc_a"])
    g["s1"], g["delta1"] = let_grads(dWt_qkv, W["qkv"], dat, st["at32"], th["s1"],
                                     dqkv.sum(axis=0))
    inter = dict(dm=dm, dgu=dgu, dbt=dbt, dx2=dx2, dO=dO, dQq=dQq, dQk=dQk, dQv=dQv, dqkv=dqkv,
                 dat=dat)
    return g, inter


def block_reference(sh: BlockShape, x, W):
    """The full-precision block y* (no quantizer, no transform), binary64."""
    M, D, H, I = sh.M, sh.D, sh.H, sh.I
    Dh = sh.Dh
    x64 = np.asarray(x, F64)
    Wd = {k: np.asarray(v, F64) for k, v in W.items()}
    a, _ = rms_norm(x64)
    qkv = a @ Wd["qkv"].T
    cos, sin = rope_table(M, Dh, sh.rope_base)
    c, s = cos.astype(F64)[:, None, :], sin.astype(F64)[:, None, :]

    def rot(X):
        Xh = X.reshape(M, H, Dh)
        lo, hi = Xh[:, :, :Dh // 2], Xh[:, :, Dh // 2:]
        return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=2).reshape(M, D)

    q, k, v = rot(qkv[:, :D]), rot(qkv[:, D:2 * D]), qkv[:, 2 * D:]
    _, O = stage_attention(q, k, v, H)
    x2 = x64 + O @ Wd["o"].T
    b, _ = rms_norm(x2)
    gu = b @ Wd["gu"].T
    m = silu(gu[:, :I]) * gu[:, I:]
    return x2 + m @ Wd["d"].T


def block_step(sh: BlockShape, x, W, theta, y_ref):
    """One calibration step: (loss, gradient vector in theta_layout order, forward state,
    intermediate gradients)."""
    th = theta_split(sh, np.asarray(theta, F32))
    st = block_forward(sh, x, W, th, y_ref)
    g, inter = block_backward(sh, W, th, st)
    if sh.wbits >= 16:
        for name in WEIGHTS:
            n = dict(theta_layout(sh))["gamma_" + name]
            g["gamma_" + name] = np.zeros(n)
            g["beta_" + name] = np.zeros(n)
    return st["loss"], theta_join(sh, g), st, inter


def block_calibrate(sh: BlockShape, xs, W, theta0, epochs: int, lr_lwc: float = om.LR_LWC,
                    lr_let: float = om.LR_LET):
    """One block's calibration ([ICLR] sections 框架, 实验证据): targets y*_i = the
    full-precision block on each sample's input, then `epochs` passes over the samples in
    order, each a block_step followed by AdamW (LWC logits at lr_lwc, LET vectors at lr_let;
    the parameters kept in binary32 between steps, as a device vector holds them). Returns
    (per-step losses, final theta float32, the samples' quantized block outputs float32)."""
    theta = np.asarray(theta0, F32).copy()
    n_lwc = dict(theta_layout(sh))
    split = sum(n for name, n in theta_layout(sh) if name.startswith(("gamma", "beta")))
    assert split == sum(n_lwc[k] for k in n_lwc if k.startswith(("gamma", "beta")))
    m = np.zeros(theta.size)
    v = np.zeros(theta.size)
    y_refs = [block_reference(sh, x, W) for x in xs]
    losses = []
    t = 0
    for _ in range(epochs):
        for x, y_ref in zip(xs, y_refs):
            t += 1
            loss, g, _, _ = block_step(sh, x, W, theta, y_ref)
            losses.append(loss)
            p1, m[:split], v[:split] = om.adamw_step(theta[:split], g[:split], m[:split],
                                                     v[:split], t, lr_lwc)
            p2, m[split:], v[split:] = om.adamw_step(theta[split:], g[split:], m[split:],
                                                     v[split:], t, lr_let)
            theta = np.concatenate([p1, p2]).astype(F32)
    th = theta_split(sh, theta)
    outs = [block_forward(sh, x, W, th)["y"].astype(F32) for x in xs]
    return np.array(losses), theta, outs
