"""CPU oracle of the OmniQuant calibration step for one fake-quantized linear layer.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the CPU-baseline leg of
bench.py may import or run this module. The product (the libomq CUDA library and its
Python binding) never calls it, and this module imports nothing from the product: the two
share only the seeded input recipes, which hold no quantization arithmetic.

What it computes, and where the pages define it:

  [ICLR] "【ICLR 2024】OmniQuant: Omnidirectionally Calibrated Quantization for Large
         Language Models" (onecrewdev.com paper reading)
           - section 框架 (block-wise objective, frozen W, learnable Theta1={gamma,beta},
             Theta2={delta,s,s_a})
           - section LWC (W_q = clamp(round(W/h)+z, 0, 2^N-1), h = (gamma max W - beta min W)
             /(2^N-1), z = -round(beta min W / h); gamma, beta in [0,1] through a sigmoid;
             gamma = beta = 1 is MinMax)
           - section LET (Y = [(X-delta)/s] [s*W] + [B + delta W];
             Y = Q_a(X~) Q_w(W~) + B~)
           - section 实验证据 (AdamW, zero weight decay, LWC lr 5e-3, LET lr 1e-2,
             per-channel weights or group 128, per-token activations)
  [AFF]  "LLM quantization tutorial" (devpress.csdn.net), section 2.2 仿射量化: the affine
         (scale, zero-point) worked example on [3, 1, -2, 3].
  [EDGE] "OmniQuant：端侧大模型低比特量化的新思路与实战" (bjdmk.com.cn), section 2.2: the
         straight-through estimator carries gradients past rounding.

Precision. Gradients and the forward value path are binary64. The encoder that decides
integers (h, z, codes, clip decisions) runs in IEEE binary32 with one rounding per
operation in a fixed order, because a kernel can reproduce that bit for bit:
    W~ = W*s;  h = ((g*M) - (b*m)) / Q;  h = max(h, 1e-8);  t = (b*m)/h;  z = -rint(t)
    u = W~/h;  q = rint(u) + z;  c = clamp(q, 0, Q);  W^ = (c - z)*h
numpy float32 arithmetic rounds after every operation and never fuses a multiply-add.

Readings where the pages are silent (each also listed in the design notes):
  - round() is round-half-to-even.
  - h is floored at 1e-8; the gradient reaches h's inputs only where the unfloored h >= 1e-8.
  - z is not clamped (codes are). It is stored as int32.
  - g = sigmoid(gamma_logit) is evaluated in binary64 and rounded once to binary32.
  - min/max are plain (zero is not forced into the range) and are differentiated: their
    gradient goes to the extremal elements, split equally between ties.
  - clamp passes the gradient where 0 <= q <= Q (inclusive), blocks it outside.
  - the activation quantizer is the same affine MinMax rule per token with gamma = beta = 1
    and nothing learnable.
  - the loss is the mean squared error over all M*N outputs.
  - AdamW uses beta1 = 0.9, beta2 = 0.999, eps = 1e-8 (the library defaults; the pages give
    only "AdamW, zero weight decay").

Pins (tests/test_oracle_*.py): the worked affine example; gamma = beta = 1 against
torch.fake_quantize_per_channel_affine; LET equivalence with quantization off; the
dequantization error bound; the STE chain against an independent float64 autograd
statement on tiny inputs; AdamW against torch.optim.AdamW; pack/unpack round trips and a
hand-packed byte example; the multi-step loop ``calibrate`` against torch.optim.AdamW (two
parameter groups at the page's two rates) driving that autograd statement for five steps,
where the bias corrections no longer cancel (tests/test_oracle_calibrate.py).
"""
from __future__ import annotations

import dataclasses

import numpy as np

F32 = np.float32
H_MIN = F32(1e-8)
Z_LIMIT = 2 ** 30


# ----------------------------------------------------------------------------- primitives

def sigmoid32(logit) -> np.ndarray:
    """Clipping strength in [0, 1] from a logit ([ICLR] section LWC: "sigmoid parameterised").

    Evaluated in binary64 and rounded once to binary32.
    """
    x = np.asarray(logit, dtype=np.float64)
    return (1.0 / (1.0 + np.exp(-x))).astype(F32)


def bf16_round(x) -> np.ndarray:
    """Round binary32 values to bfloat16 (nearest, ties to even); returned widened to float32.

    Used only to state what a bfloat16 output tensor must hold bit for bit.
    """
    a = np.ascontiguousarray(np.asarray(x, dtype=F32))
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(a)
    out = r.astype(np.uint32).view(F32).copy()
    out[nan] = np.nan
    return out


# ----------------------------------------------------------------------------- LET

def let_weight(W, s) -> np.ndarray:
    """W~ = s (.) W: column k of W [N, K] scaled by s[k] ([ICLR] section LET). binary32."""
    W = np.asarray(W, dtype=F32)
    if s is None:
        return W.copy()
    return W * np.asarray(s, dtype=F32)[None, :]


def let_act(X, s, delta) -> np.ndarray:
    """X~ = (X - delta) / s per input channel ([ICLR] section LET). binary32."""
    X = np.asarray(X, dtype=F32)
    if s is None and delta is None:
        return X.copy()
    d = np.zeros(X.shape[1], F32) if delta is None else np.asarray(delta, F32)
    sv = np.ones(X.shape[1], F32) if s is None else np.asarray(s, F32)
    return (X - d[None, :]) / sv[None, :]


def let_bias(W, B, delta) -> np.ndarray:
    """B~ = B + delta W, i.e. B~[n] = B[n] + sum_k delta[k] W[n, k], with the ORIGINAL W
    ([ICLR] section LET). binary64."""
    W64 = np.asarray(W, dtype=np.float64)
    out = np.zeros(W64.shape[0]) if B is None else np.asarray(B, dtype=np.float64).copy()
    if delta is not None:
        out = out + W64 @ np.asarray(delta, dtype=np.float64)
    return out


# ----------------------------------------------------------------------------- encoder

@dataclasses.dataclass
class Encoded:
    """Result of the affine encoder on a [R, C] array split into groups of G along C."""
    group: int
    bits: int
    h: np.ndarray        # [R, C/G] float32 (floored)
    h_raw: np.ndarray    # [R, C/G] float32 (before the floor)
    z: np.ndarray        # [R, C/G] float32 integral value (unclamped zero point)
    vmax: np.ndarray     # [R, C/G] float32
    vmin: np.ndarray     # [R, C/G] float32
    nmax: np.ndarray     # [R, C/G] ties at the max
    nmin: np.ndarray     # [R, C/G] ties at the min
    r: np.ndarray        # [R, C] float32 rint(u)
    inrange: np.ndarray  # [R, C] bool, 0 <= q <= Q
    codes: np.ndarray    # [R, C] float32 integral value in [0, Q]
    deq: np.ndarray      # [R, C] float32 (c - z) * h

    @property
    def z_i32(self) -> np.ndarray:
        return np.clip(self.z, -Z_LIMIT, Z_LIMIT).astype(np.int32)

    @property
    def codes_u8(self) -> np.ndarray:
        return self.codes.astype(np.uint8)


def encode_affine(V, g, b, bits: int, group: int) -> Encoded:
    """LWC uniform affine encoder with clipping strengths g (upper) and b (lower).

    [ICLR] section LWC: per group, h = (g*max V - b*min V)/(2^N - 1), z = -round(b*min V/h),
    codes = clamp(round(V/h) + z, 0, 2^N - 1). The dequantized value is (codes - z)*h.
    With g = b = 1 this is MinMax asymmetric quantization ([AFF] section 2.2).
    V is [R, C] binary32, g and b are [R, C/G] binary32.
    """
    V = np.asarray(V, dtype=F32)
    R, C = V.shape
    if C % group:
        raise ValueError("group must divide the row length")
    ng = C // group
    Vg = V.reshape(R, ng, group)
    g = np.broadcast_to(np.asarray(g, dtype=F32), (R, ng))
    b = np.broadcast_to(np.asarray(b, dtype=F32), (R, ng))
    Q = F32(2 ** bits - 1)
    vmax = Vg.max(axis=2)
    vmin = Vg.min(axis=2)
    h_raw = (g * vmax - b * vmin) / Q
    h = np.maximum(h_raw, H_MIN)
    t = (b * vmin) / h
    z = -np.rint(t)
    u = Vg / h[:, :, None]
    r = np.rint(u)
    q = r + z[:, :, None]
    inr = (q >= F32(0)) & (q <= Q)
    c = np.clip(q, F32(0), Q)
    deq = (c - z[:, :, None]) * h[:, :, None]
    nmax = (Vg == vmax[:, :, None]).sum(axis=2)
    nmin = (Vg == vmin[:, :, None]).sum(axis=2)
    return Encoded(group=group, bits=bits, h=h, h_raw=h_raw, z=z, vmax=vmax, vmin=vmin,
                   nmax=nmax, nmin=nmin, r=r.reshape(R, C), inrange=inr.reshape(R, C),
                   codes=c.reshape(R, C), deq=deq.reshape(R, C))


def encode_backward(dDeq, V, enc: Encoded, g, b):
    """Straight-through gradient of deq = (clamp(round(V/h)+z, 0, Q) - z)*h.

    round' = 1 ([EDGE] section 2.2); the formula of [ICLR] section LWC is differentiated as
    written, through h and z into g, b and the group's max and min:
      in range : d deq/dV = 1, d deq/dh = round(u) - u, d deq/dz = 0
      clipped  : d deq/dV = 0, d deq/dh = c - z,        d deq/dz = -h
      G_h = sum dDeq * d deq/dh,  G_z = sum dDeq * d deq/dz   (per group)
      z = -round(t), t = b*m/h:  dz/dh = t/h,  dz/db = -m/h,  dz/dm = -b/h
      h = (g*M - b*m)/Q:  dh/dg = M/Q, dh/db = -m/Q, dh/dM = g/Q, dh/dm = -b/Q
    Returns (dV [R, C], dg [R, C/G], db [R, C/G]) in binary64.
    """
    G = enc.group
    R, C = enc.codes.shape
    ng = C // G
    Q = float(2 ** enc.bits - 1)
    dD = np.asarray(dDeq, dtype=np.float64).reshape(R, ng, G)
    Vg = np.asarray(V, dtype=F32).reshape(R, ng, G)
    V64 = Vg.astype(np.float64)
    h = enc.h.astype(np.float64)
    z = enc.z.astype(np.float64)
    g = np.broadcast_to(np.asarray(g, dtype=F32), (R, ng)).astype(np.float64)
    b = np.broadcast_to(np.asarray(b, dtype=F32), (R, ng)).astype(np.float64)
    M = enc.vmax.astype(np.float64)
    m = enc.vmin.astype(np.float64)
    u = V64 / h[:, :, None]
    r = enc.r.reshape(R, ng, G).astype(np.float64)
    inr = enc.inrange.reshape(R, ng, G)
    c = enc.codes.reshape(R, ng, G).astype(np.float64)

    d_dh = np.where(inr, r - u, c - z[:, :, None])
    d_dz = np.where(inr, 0.0, -h[:, :, None])
    Gh = (dD * d_dh).sum(axis=2)
    Gz = (dD * d_dz).sum(axis=2)
    t = b * m / h
    dh = Gh + Gz * t / h
    dh = np.where(enc.h_raw >= H_MIN, dh, 0.0)   # the floor blocks h's own gradient
    dg = dh * M / Q
    db = -dh * m / Q - Gz * m / h
    dM = dh * g / Q
    dm = -dh * b / Q - Gz * b / h
    at_max = Vg == enc.vmax[:, :, None]
    at_min = Vg == enc.vmin[:, :, None]
    dV = (dD * inr
          + at_max * (dM / enc.nmax)[:, :, None]
          + at_min * (dm / enc.nmin)[:, :, None])
    return dV.reshape(R, C), dg, db


# ----------------------------------------------------------------------------- quantizers

def lwc_quant(W, s, gamma_logit, beta_logit, bits: int, group: int):
    """Weight side: W~ = s (.) W, then LWC with g = sigmoid(gamma), b = sigmoid(beta).

    Returns (W~ float32 [N, K], Encoded, g, b)."""
    Wt = let_weight(W, s)
    g = sigmoid32(gamma_logit)
    b = sigmoid32(beta_logit)
    return Wt, encode_affine(Wt, g, b, bits, group), g, b


def act_quant(Xt, abits: int):
    """Per-token activation fake-quant ([ICLR] section 实验证据: "activations per-token"):
    MinMax affine over each row of X~ (gamma = beta = 1). None when abits == 16."""
    if abits >= 16:
        return None
    Xt = np.asarray(Xt, dtype=F32)
    one = np.ones((Xt.shape[0], 1), F32)
    return encode_affine(Xt, one, one, abits, Xt.shape[1])


# ----------------------------------------------------------------------------- forward

def mse_loss(Y, Yref):
    """L = mean((Y - Y*)^2) over all outputs and dL/dY = 2 (Y - Y*) / (M N)."""
    Y = np.asarray(Y, dtype=np.float64)
    diff = Y - np.asarray(Yref, dtype=np.float64)
    n = diff.size
    return float((diff * diff).sum() / n), 2.0 * diff / n


def reference_output(X, W, B):
    """Full-precision target Y* = X W^T + B ([ICLR] section 框架: F(W, X)). binary64."""
    Y = np.asarray(X, np.float64) @ np.asarray(W, np.float64).T
    if B is not None:
        Y = Y + np.asarray(B, np.float64)[None, :]
    return Y


@dataclasses.dataclass
class StepResult:
    loss: float
    Y: np.ndarray            # [M, N] binary64
    dY: np.ndarray           # [M, N] binary64
    Wt: np.ndarray           # W~ [N, K] float32
    wenc: Encoded
    Xt: np.ndarray           # X~ [M, K] float32
    aenc: Encoded | None
    Xq: np.ndarray           # Q_a(X~) (or X~) [M, K] float32
    Bt: np.ndarray           # B~ [N] binary64
    d_gamma_logit: np.ndarray
    d_beta_logit: np.ndarray
    d_s: np.ndarray | None
    d_delta: np.ndarray | None
    d_Bt: np.ndarray


def calib_step(X, W, B, Yref, gamma_logit, beta_logit, s, delta, bits: int, group: int,
               abits: int, let: bool, need_backward: bool = True) -> StepResult:
    """One forward + backward of the fake-quantized linear ([ICLR] sections LET, LWC, 框架).

    Forward:  W~ = s.W, X~ = (X-delta)/s, B~ = B + W delta,
              Y = Q_a(X~) Q_w(W~)^T + B~, L = mean (Y - Y*)^2.
    Backward (STE): gradients of L with respect to the gamma/beta logits, and to s, delta
    when LET is learnable.
    """
    s_eff = s if let else None
    d_eff = delta if let else None
    Wt, wenc, g, b = lwc_quant(W, s_eff, gamma_logit, beta_logit, bits, group)
    Xt = let_act(X, s_eff, d_eff)
    aenc = act_quant(Xt, abits)
    Xq = Xt if aenc is None else aenc.deq
    Bt = let_bias(W, B, d_eff)
    Xq64 = Xq.astype(np.float64)
    What64 = wenc.deq.astype(np.float64)
    Y = Xq64 @ What64.T + Bt[None, :]
    loss, dY = mse_loss(Y, Yref)
    res = StepResult(loss=loss, Y=Y, dY=dY, Wt=Wt, wenc=wenc, Xt=Xt, aenc=aenc, Xq=Xq, Bt=Bt,
                     d_gamma_logit=None, d_beta_logit=None, d_s=None, d_delta=None,
                     d_Bt=None)
    if not need_backward:
        return res

    dWhat = dY.T @ Xq64                       # [N, K]
    dWt, dg, db = encode_backward(dWhat, Wt, wenc, g, b)
    g64, b64 = g.astype(np.float64), b.astype(np.float64)
    res.d_gamma_logit = dg * g64 * (1.0 - g64)
    res.d_beta_logit = db * b64 * (1.0 - b64)
    res.d_Bt = dY.sum(axis=0)                 # [N]
    if let:
        dXq = dY @ What64                     # [M, K]
        if aenc is None:
            dXt = dXq
        else:
            one = np.ones((Xt.shape[0], 1), F32)
            dXt, _, _ = encode_backward(dXq, Xt, aenc, one, one)
        s64 = np.asarray(s, np.float64)
        W64 = np.asarray(W, np.float64)
        Xt64 = Xt.astype(np.float64)
        # W~ = W s:   dL/ds_k += sum_n dW~[n,k] W[n,k]
        # X~ = (X - delta)/s:  dX~/ds = -X~/s,  dX~/ddelta = -1/s
        # B~ = B + W delta:    dL/ddelta_k += sum_n dB~[n] W[n,k]
        res.d_s = (dWt * W64).sum(axis=0) - (dXt * Xt64).sum(axis=0) / s64
        res.d_delta = -dXt.sum(axis=0) / s64 + W64.T @ res.d_Bt
    return res


# ----------------------------------------------------------------------------- AdamW

def adamw_step(p, grad, m, v, step: int, lr: float, beta1=0.9, beta2=0.999, eps=1e-8,
               weight_decay=0.0):
    """AdamW ([ICLR] section 实验证据: "AdamW, zero weight decay"). ``step`` counts from 1.

    Decoupled decay p *= (1 - lr wd); m = b1 m + (1-b1) g; v = b2 v + (1-b2) g^2;
    p -= lr/(1 - b1^t) * m / (sqrt(v)/sqrt(1 - b2^t) + eps). Returns new (p, m, v), binary64.
    """
    p = np.asarray(p, np.float64) * (1.0 - lr * weight_decay)
    g = np.asarray(grad, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    bc1 = 1.0 - beta1 ** step
    bc2 = 1.0 - beta2 ** step
    p = p - (lr / bc1) * m / (np.sqrt(v) / np.sqrt(bc2) + eps)
    return p, m, v


LR_LWC = 5e-3   # [ICLR] section 实验证据
LR_LET = 1e-2


# ----------------------------------------------------------------------------- fold / pack

def pack_codes(codes, bits: int) -> np.ndarray:
    """Row-major bit packing: element k of a row occupies bits k*bits .. k*bits + bits - 1 of
    the row's little-endian bit string, i.e. it starts in byte (k*bits)//8 at bit offset
    (k*bits) % 8, least-significant bits first; a 3-, 5-, 6- or 7-bit code may straddle two
    bytes.
    Supports bits 2 to 8 with a row length whose bits fill whole bytes."""
    c = np.asarray(codes).astype(np.uint64)
    R, C = c.shape
    if not 2 <= bits <= 8 or (C * bits) % 8:
        raise ValueError("unsupported packing")
    out = np.zeros((R, C * bits // 8), dtype=np.uint64)
    for k in range(C):
        pos = k * bits
        byte, off = pos // 8, pos % 8
        v = c[:, k] << np.uint64(off)                     # at most 10 bits
        out[:, byte] |= v & np.uint64(0xFF)
        if off + bits > 8:
            out[:, byte + 1] |= v >> np.uint64(8)
    return out.astype(np.uint8)


def unpack_codes(packed, bits: int, C: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).astype(np.uint64)
    mask = np.uint64((1 << bits) - 1)
    out = np.zeros((p.shape[0], C), dtype=np.uint64)
    for k in range(C):
        pos = k * bits
        byte, off = pos // 8, pos % 8
        v = p[:, byte] >> np.uint64(off)
        if off + bits > 8:
            v |= p[:, byte + 1] << np.uint64(8 - off)
        out[:, k] = v & mask
    return out.astype(np.uint8)


def fold_pack(W, s, gamma_logit, beta_logit, bits: int, group: int):
    """Fold learned Theta into deployable weights ([ICLR] section 框架: learned parameters
    fold back into the weights): codes of W~ = s.W at the learned clipping, packed, with
    h and z. Returns (packed uint8 [N, K*bits/8], h float32, z int32)."""
    _, enc, _, _ = lwc_quant(W, s, gamma_logit, beta_logit, bits, group)
    return pack_codes(enc.codes_u8, bits), enc.h.copy(), enc.z_i32


# ----------------------------------------------------------------------------- driver

def calibrate(X, W, B, Yref, gamma_logit, beta_logit, s, delta, bits, group, abits, let,
              steps: int):
    """The step iterated with AdamW (LWC lr 5e-3 on the logits, LET lr 1e-2 on s, delta).
    Returns the per-step losses and the final parameters (pinned over several steps against
    torch.optim.AdamW driving an independent autograd statement of the step)."""
    gl = np.asarray(gamma_logit, np.float64)
    bl = np.asarray(beta_logit, np.float64)
    sv = np.asarray(s, np.float64)
    dv = np.asarray(delta, np.float64)
    mom = {k: np.zeros_like(a) for k, a in (("g", gl), ("b", bl), ("s", sv), ("d", dv))}
    var = {k: np.zeros_like(a) for k, a in (("g", gl), ("b", bl), ("s", sv), ("d", dv))}
    losses = []
    for t in range(1, steps + 1):
        r = calib_step(X, W, B, Yref, gl.astype(F32), bl.astype(F32), sv.astype(F32),
                       dv.astype(F32), bits, group, abits, let)
        losses.append(r.loss)
        gl, mom["g"], var["g"] = adamw_step(gl, r.d_gamma_logit, mom["g"], var["g"], t, LR_LWC)
        bl, mom["b"], var["b"] = adamw_step(bl, r.d_beta_logit, mom["b"], var["b"], t, LR_LWC)
        if let:
            sv, mom["s"], var["s"] = adamw_step(sv, r.d_s, mom["s"], var["s"], t, LR_LET)
            dv, mom["d"], var["d"] = adamw_step(dv, r.d_delta, mom["d"], var["d"], t, LR_LET)
    return losses, gl.astype(F32), bl.astype(F32), sv.astype(F32), dv.astype(F32)
