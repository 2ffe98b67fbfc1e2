"""GPU parity of the transformer-block step (omq_block_step through the C ABI) against the
block oracle (oracle/block.py), stage by stage.

Each stage of the GPU step is checked against the oracle's statement of that stage applied
to the GPU's own inputs to it (read from the workspace), so that every comparison isolates
one stage: integer decisions (weight and activation codes) must match bit for bit, values
within the tolerances below. The whole step is also compared end to end with the oracle run
on its own (loss and every parameter gradient) where the chain has no activation quantizer
to amplify rounding differences (abits = 16).

The step's GEMM operands are float16, and the gradients between stages are stored unscaled
(in units of the residual y - y*: gradients of (M D / 2) L); the tests multiply them by
2 / (M D) before comparing.

Tolerances (Frobenius-normalised unless stated):
  stages whose inputs are the same 16-bit values on both sides (float32 accumulation only):
      1e-5 (GEMM outputs), 1e-4 (gradients through the STE, float32 sums)
  stages that store a float16 result:  2e-3 (float16 rounding is 2^-11 relative per element)
  gradients through the attention backward, whose probabilities and score gradient the GPU
  rounds to float16 as GEMM operands: 5e-3
  end to end: the loss and every parameter gradient within 2e-2 (E2E_TOL)
"""
import numpy as np
import pytest
import torch

from oracle import block as ob
from oracle import omniquant as om
from post_quantization_lwc_b200 import synth
from tests.gpu_common import frob_rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


# End to end, every gradient is proportional to the residual y - y*, a small difference of
# the block's output and the target, and the GPU forms y from float16 GEMM operands at six
# linears and two attention products; the gradients then cross up to six more stages that
# round a GEMM operand to float16. The 16-bit GEMM tolerance holds for the whole chain.
E2E_TOL = 2e-2

CASES = [
    # (M, H, I, group, wbits, abits): several GEMM tiles with ragged tails in M and I
    (264, 2, 352, 0, 4, 4),
    (200, 2, 288, 32, 3, 8),
    (136, 1, 160, 0, 4, 16),
]


def _f(t):
    return t.detach().float().cpu().numpy()


class Run:
    def __init__(self, omq, dev, M, H, I, group, wbits, abits, seed=0):
        cfg = synth.scaled_block(synth.BLOCK_CONFIGS["llama7b_block_w4a4"], M, H, I,
                                 seed=500 + seed, group=group, wbits=wbits, abits=abits,
                                 w_std=0.05)
        self.sh = ob.BlockShape(M=M, D=128 * H, H=H, I=I, wbits=wbits, abits=abits,
                                group=group)
        inp = synth.make_block_inputs(cfg)
        self.x = _f(inp.x)
        self.W = {k: _f(v) for k, v in inp.W.items()}
        self.theta = synth.random_block_theta(700 + seed, ob.theta_layout(self.sh)).numpy()
        self.th = ob.theta_split(self.sh, self.theta)
        self.y_ref = ob.block_reference(self.sh, self.x, self.W).astype(np.float32)
        blk = omq.Block(M, 128 * H, H, I, group=group, wbits=wbits, abits=abits, device=dev)
        for name, n in ob.theta_layout(self.sh):
            assert blk.theta_slices[name][1] == n, name
        blk.load({k: v.to(dev) for k, v in inp.W.items()}, torch.from_numpy(self.theta).to(dev))
        self.loss = blk.step(inp.x.to(dev), torch.from_numpy(self.y_ref).to(dev), update=False)
        torch.cuda.synchronize()
        omq.sync_check()
        self.blk = blk
        self.gtheta = _f(blk.d_theta)

    def buf(self, name, *shape):
        return _f(self.blk.buffer(name)).reshape(*shape)

    def gbuf(self, name, *shape):
        """A stored stage gradient, scaled to dL (the step keeps them in units of res)."""
        M, D = self.sh.M, self.sh.D
        return self.buf(name, *shape).astype(np.float64) * (2.0 / (M * D))

    def grad(self, name):
        o, n = self.blk.theta_slices[name]
        return self.gtheta[o:o + n]


@pytest.fixture(scope="module", params=range(len(CASES)), ids=lambda i: "M{}_H{}_I{}_g{}_w{}a{}".format(*CASES[i]))
def run(request, omq, cuda_device):
    return Run(omq, cuda_device, *CASES[request.param], seed=request.param)


def _bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def _f16(x):
    """The float16 operand the step stores for the binary32 value x (round to nearest even)."""
    return np.asarray(x, np.float32).astype(np.float16).astype(np.float32)


def _lower(M):
    """j <= i: the probabilities the step computes (the float32 rows hold nothing above)."""
    return np.tril(np.ones((M, M), dtype=bool))


def _span(M, tile=256):
    """j < the end of row i's 256-column tile: what the 16-bit probability and score-gradient
    rows hold (zero between the diagonal and the tile's end); the causal GEMMs read no more."""
    i = np.arange(M)[:, None]
    return np.arange(M)[None, :] < np.minimum((i // tile + 1) * tile, M)


def test_forward_stages(run):
    sh, th, W = run.sh, run.th, run.W
    M, D, H, I, A = sh.M, sh.D, sh.H, sh.I, sh.abits
    # rotary table: the binary64 cos / sin rounded once
    cos, sin = ob.rope_table(M, 128)
    rope = run.buf("rope", 2, M, 64)
    assert np.array_equal(_bits(rope[0]), _bits(cos)) and np.array_equal(_bits(rope[1]), _bits(sin))
    # weights: LWC codes through the BF16 Ŵ, bit for bit
    wq = ob._weights_quant(sh, W, th)
    for name, shape in (("qkv", (3 * D, D)), ("o", (D, D)), ("gu", (2 * I, D)), ("d", (D, I))):
        got = run.buf("what_" + name, *shape)
        assert np.array_equal(_bits(got), _bits(_f16(wq[name][4]))), name
    # RMSNorm, then LET + per-token quant of the GPU's a
    a = run.buf("a", M, D)
    n_ref, _ = ob.rms_norm(run.x)
    assert frob_rel(a, n_ref) < 1e-6
    qa_ref, _ = ob.act_encode(om.let_act(a, th["s1"], th["delta1"]), A, D)
    assert np.array_equal(_bits(run.buf("qa", M, D)), _bits(_f16(qa_ref)))
    # q | k | v from the GPU's operands
    qa, Wq = run.buf("qa", M, D), run.buf("what_qkv", 3 * D, D)
    qkv_ref = qa.astype(np.float64) @ Wq.astype(np.float64).T + om.let_bias(W["qkv"], None,
                                                                            th["delta1"])
    qkv = run.buf("qkv", M, 3 * D)
    assert frob_rel(qkv, qkv_ref) < 1e-5
    # RoPE, affinity LET, V transform and the per-head quantizer: bit for bit
    ap = ob.stage_attn_prep(qkv, cos, sin, th["s_a"], th["s_o"], th["delta_o"], H, A)
    qqkv = run.buf("qqkv", M, 3 * D)
    want = np.concatenate([ap["Qq"], ap["Qk"], ap["Qv"]], axis=1)
    assert np.array_equal(_bits(qqkv), _bits(_f16(want)))
    # causal softmax and P V
    Qq, Qk, Qv = qqkv[:, :D], qqkv[:, D:2 * D], qqkv[:, 2 * D:]
    P_ref, _ = ob.stage_attention(Qq, Qk, Qv, H)
    low, span = _lower(M), _span(M)
    P = np.where(low, run.buf("p", H, M, M), 0.0)
    assert frob_rel(P, P_ref) < 1e-5
    P16 = run.buf("p16", H, M, M)
    assert np.array_equal(_bits(P16[:, span]), _bits(_f16(P.astype(np.float32))[:, span]))
    P16 = np.where(span, P16, 0.0)
    O_ref = ob.unheads(np.einsum("hmn,hnd->hmd", P16.astype(np.float64), ob.heads(Qv, H)))
    O = run.buf("o", M, D)
    assert frob_rel(O, O_ref) < 1e-5
    Qo_ref, _ = ob.act_encode(O, A, D)
    assert np.array_equal(_bits(run.buf("qo", M, D)), _bits(_f16(Qo_ref)))
    # o_proj + residual, RMSNorm, LET + quant
    x2_ref = run.x.astype(np.float64) + run.buf("qo", M, D).astype(np.float64) @ run.buf(
        "what_o", D, D).astype(np.float64).T + om.let_bias(W["o"], None, th["delta_o"])
    x2 = run.buf("x2", M, D)
    assert frob_rel(x2, x2_ref) < 1e-5
    b = run.buf("b", M, D)
    assert frob_rel(b, ob.rms_norm(x2)[0]) < 1e-6
    qb_ref, _ = ob.act_encode(om.let_act(b, th["s2"], th["delta2"]), A, D)
    assert np.array_equal(_bits(run.buf("qb", M, D)), _bits(_f16(qb_ref)))
    # gate / up, SwiGLU, quant
    gu_ref = run.buf("qb", M, D).astype(np.float64) @ run.buf("what_gu", 2 * I, D).astype(
        np.float64).T + om.let_bias(W["gu"], None, th["delta2"])
    gu = run.buf("gu", M, 2 * I)
    assert frob_rel(gu, gu_ref) < 1e-5
    mid = run.buf("mid", M, I)
    assert frob_rel(mid, ob.silu(gu[:, :I]) * gu[:, I:]) < 1e-5
    qm_ref, _ = ob.act_encode(mid, A, I)
    assert np.array_equal(_bits(run.buf("qm", M, I)), _bits(_f16(qm_ref)))
    # down + residual, loss
    y = x2.astype(np.float64) + run.buf("qm", M, I).astype(np.float64) @ run.buf(
        "what_d", D, I).astype(np.float64).T
    res_ref = y - run.y_ref
    assert frob_rel(run.buf("res", M, D), res_ref) < 2e-3
    loss_ref = float((res_ref ** 2).mean())
    assert abs(run.loss.item() - loss_ref) <= 1e-4 * loss_ref


def _lwc_grad_check(run, name, dWhat):
    sh, th, W = run.sh, run.th, run.W
    wq = ob._weights_quant(sh, W, th)
    dWt, dgl, dbl = ob._lwc_grads(dWhat, wq[name])
    assert frob_rel(run.grad("gamma_" + name), dgl) < 1e-4, name
    assert frob_rel(run.grad("beta_" + name), dbl) < 1e-4, name
    return dWt


def test_backward_stages(run):
    sh, th, W = run.sh, run.th, run.W
    M, D, H, I, A = sh.M, sh.D, sh.H, sh.I, sh.abits
    f64 = np.float64
    gscale = 2.0 / (M * D)
    dy = gscale * run.buf("res", M, D).astype(f64)
    # down projection: LWC gradients and dL/dm through the act quantizer's STE
    _lwc_grad_check(run, "d", dy.T @ run.buf("qm", M, I).astype(f64))
    mid = run.buf("mid", M, I)
    _, enc_m = ob.act_encode(mid, A, I)
    dm_ref = ob.act_backward(dy @ run.buf("what_d", D, I).astype(f64), mid, enc_m)
    dm = run.gbuf("dmid", M, I)
    assert frob_rel(dm, dm_ref) < 1e-4
    # SwiGLU backward
    gu = run.buf("gu", M, 2 * I).astype(f64)
    g, u = gu[:, :I], gu[:, I:]
    sg = 1 / (1 + np.exp(-g))
    dgu_ref = np.concatenate([dm * u * sg * (1 + g * (1 - sg)), dm * g * sg], axis=1)
    dgu = run.gbuf("dgu", M, 2 * I)
    assert frob_rel(dgu, dgu_ref) < 2e-3
    # gate / up projection: LWC gradients, dL/db, s2 / delta2
    dWt_gu = _lwc_grad_check(run, "gu", dgu.T @ run.buf("qb", M, D).astype(f64))
    b = run.buf("b", M, D)
    bt = om.let_act(b, th["s2"], th["delta2"])
    _, enc_b = ob.act_encode(bt, A, D)
    dbt = ob.act_backward(dgu @ run.buf("what_gu", 2 * I, D).astype(f64), bt, enc_b)
    assert frob_rel(run.gbuf("db", M, D), dbt / th["s2"].astype(f64)) < 1e-4
    ds2, dd2 = ob.let_grads(dWt_gu, W["gu"], dbt, bt, th["s2"], dgu.sum(0))
    assert frob_rel(run.grad("s2"), ds2) < 1e-4
    assert frob_rel(run.grad("delta2"), dd2) < 1e-4
    # RMSNorm backward with the residual path
    x2 = run.buf("x2", M, D).astype(f64)
    _, rstd2 = ob.rms_norm(x2)
    dx2_ref = dy + ob.rms_backward(run.gbuf("db", M, D), b, rstd2)
    dx2 = run.gbuf("dx2", M, D)
    assert frob_rel(dx2, dx2_ref) < 2e-3
    # output projection: LWC gradients and dL/dO
    dWt_o = _lwc_grad_check(run, "o", dx2.T @ run.buf("qo", M, D).astype(f64))
    O = run.buf("o", M, D)
    _, enc_o = ob.act_encode(O, A, D)
    dO_ref = ob.act_backward(dx2 @ run.buf("what_o", D, D).astype(f64), O, enc_o)
    dO = run.gbuf("do", M, D)
    assert frob_rel(dO, dO_ref) < 2e-3
    # attention backward (probabilities from the GPU's float32 P)
    qqkv = run.buf("qqkv", M, 3 * D)
    P = np.where(_lower(M), run.buf("p", H, M, M), 0.0)
    dQq, dQk, dQv = ob.stage_attention_backward(dO, P, qqkv[:, :D],
                                                qqkv[:, D:2 * D], qqkv[:, 2 * D:], H)
    dqq = run.gbuf("dqqkv", M, 3 * D)
    assert frob_rel(dqq[:, 2 * D:], dQv) < 2e-2
    assert frob_rel(dqq[:, :D], dQq) < 2e-2
    assert frob_rel(dqq[:, D:2 * D], dQk) < 2e-2
    # head quantizers' STE, affinity / V transforms, RoPE transpose (from the GPU's dQ)
    cos, sin = ob.rope_table(M, 128)
    ap = ob.stage_attn_prep(run.buf("qkv", M, 3 * D), cos, sin, th["s_a"], th["s_o"],
                            th["delta_o"], H, A)
    dqt = ob.act_backward(dqq[:, :D], ap["qt"], ap["enc_q"])
    dkt = ob.act_backward(dqq[:, D:2 * D], ap["kt"], ap["enc_k"])
    dvt = ob.act_backward(dqq[:, 2 * D:], ap["vt"], ap["enc_v"])
    sa, so = th["s_a"].astype(f64), th["s_o"].astype(f64)
    dqkv_ref = np.concatenate([ob.rope_backward(dqt / sa, cos, sin, H),
                               ob.rope_backward(dkt * sa, cos, sin, H), dvt / so], axis=1)
    dqkv = run.gbuf("dqkv", M, 3 * D)
    assert frob_rel(dqkv, dqkv_ref) < 2e-3
    t_k, t_q = (dkt * ap["kr"]).sum(0), (dqt * ap["qt"]).sum(0) / sa
    dsa = t_k - t_q
    # the two sums cancel exactly without quantized Q, K (the affinity transform is then an
    # invariance): bound the difference by the size of the sums, not of the result
    scale = max(np.linalg.norm(dsa), 1e-2 * (np.linalg.norm(t_k) + np.linalg.norm(t_q)))
    assert np.linalg.norm(run.grad("s_a") - dsa) < 1e-4 * scale
    ds_o, dd_o = ob.let_grads(dWt_o, W["o"], dvt, ap["vt"], th["s_o"], dx2.sum(0))
    assert frob_rel(run.grad("s_o"), ds_o) < 1e-4
    assert frob_rel(run.grad("delta_o"), dd_o) < 1e-4
    # q / k / v projection: LWC gradients, s1 / delta1
    dWt_qkv = _lwc_grad_check(run, "qkv", dqkv.T @ run.buf("qa", M, D).astype(f64))
    a = run.buf("a", M, D)
    at = om.let_act(a, th["s1"], th["delta1"])
    _, enc_a = ob.act_encode(at, A, D)
    dat = ob.act_backward(dqkv @ run.buf("what_qkv", 3 * D, D).astype(f64), at, enc_a)
    ds1, dd1 = ob.let_grads(dWt_qkv, W["qkv"], dat, at, th["s1"], dqkv.sum(0))
    assert frob_rel(run.grad("s1"), ds1) < 1e-4
    assert frob_rel(run.grad("delta1"), dd1) < 1e-4


# The activation quantizers in the order the block's forward applies them.
ACT_ORDER = ("qa", "q", "k", "v", "qo", "qb", "qm")


def _gpu_quantizer_inputs(run):
    """Each activation quantizer's input as the GPU step formed it: its stored stage input put
    through the oracle's own formula for that stage (the forward stage test shows these match
    the GPU bit for bit)."""
    sh, th = run.sh, run.th
    M, D, H, I = sh.M, sh.D, sh.H, sh.I
    cos, sin = ob.rope_table(M, 128)
    ap = ob.stage_attn_prep(run.buf("qkv", M, 3 * D), cos, sin, th["s_a"], th["s_o"],
                            th["delta_o"], H, sh.abits)
    return {"qa": om.let_act(run.buf("a", M, D), th["s1"], th["delta1"]),
            "q": ap["qt"], "k": ap["kt"], "v": ap["vt"], "qo": run.buf("o", M, D),
            "qb": om.let_act(run.buf("b", M, D), th["s2"], th["delta2"]),
            "qm": run.buf("mid", M, I)}


def _levels(enc):
    """Signed level c - z of every element (deq = level * h)."""
    R, C = enc.codes.shape
    G = C // enc.h.shape[1]
    return enc.codes.astype(np.float64) - np.repeat(enc.z.astype(np.float64), G, axis=1)


def test_end_to_end_against_oracle(run, monkeypatch):
    """The whole step against the oracle run on its own inputs: the loss and every parameter
    gradient within the 16-bit GEMM tolerance (E2E_TOL).

    With quantized activations the two sides' quantizer inputs differ by upstream rounding
    (float16 GEMM operands against binary64 products), and an input that lies that close to
    a rounding boundary takes the neighbouring level on one side: both results are correct
    roundings of the same value. Such level flips are counted and each is checked to be
    one: the levels differ by one and the two sides' quotients V / h lie on either side of
    the boundary between them. The oracle run then takes the GPU's level at exactly those
    elements (every other value, range, scale and zero point stays its own), so that the
    comparison measures the arithmetic, not the choice between two valid roundings."""
    sh = run.sh
    M, D, I = sh.M, sh.D, sh.I
    report = {}
    if sh.abits < 16:
        gpu_in = _gpu_quantizer_inputs(run)
        width = {"qa": D, "q": 128, "k": 128, "v": 128, "qo": D, "qb": D, "qm": I}
        real = ob.act_encode
        calls = []

        def conditioned(V32, abits, w):
            deq, enc = real(V32, abits, w)
            name = ACT_ORDER[len(calls)]
            calls.append(name)
            assert w == width[name], name
            _, enc_g = real(gpu_in[name], abits, w)     # the GPU's own encoding
            lv_o, lv_g = _levels(enc), _levels(enc_g)
            flip = lv_o != lv_g
            R, C = enc.codes.shape
            G = C // enc.h.shape[1]
            u_o = np.asarray(V32, np.float64) / np.repeat(enc.h.astype(np.float64), G, axis=1)
            u_g = np.asarray(gpu_in[name], np.float64) / np.repeat(
                enc_g.h.astype(np.float64), G, axis=1)
            mid = 0.5 * (lv_o + lv_g)
            valid = (np.abs(lv_o - lv_g) == 1) & ((u_o - mid) * (u_g - mid) <= 0)
            report[name] = (float(flip.mean()), int((flip & ~valid).sum()))
            if flip.any():
                z = np.repeat(enc.z, G, axis=1)
                Q = np.float32(2 ** abits - 1)
                r = np.where(flip, lv_g, enc.r).astype(np.float32)
                q = r + z
                enc.r = r
                enc.inrange = (q >= 0) & (q <= Q)
                enc.codes = np.clip(q, np.float32(0), Q)
                enc.deq = ((enc.codes - z) * np.repeat(enc.h, G, axis=1)).astype(np.float32)
            return enc.deq, enc

        monkeypatch.setattr(ob, "act_encode", conditioned)
    loss, grad, st, inter = ob.block_step(sh, run.x, run.W, run.theta, run.y_ref)
    monkeypatch.undo()
    if report:
        print("activation level flips (fraction, not explained):",
              {k: f"{v[0]:.2e}/{v[1]}" for k, v in report.items()})
        assert sorted(report) == sorted(ACT_ORDER)
        assert all(bad == 0 for _, bad in report.values()), report
        # a wrong h or z would move most levels of a row, not a fraction of them
        assert max(f for f, _ in report.values()) <= 1.5e-3 * (2 ** sh.abits - 1), report
    assert abs(run.loss.item() - loss) <= E2E_TOL * loss
    off = 0
    errs = {}
    for name, n in ob.theta_layout(sh):
        g = grad[off:off + n]
        off += n
        err = frob_rel(run.grad(name), g)
        if name == "s_a":
            # d s_a is the difference of two sums that cancel exactly when Q and K are not
            # quantized (the affinity scaling is then an invariance) and nearly at 8 bits:
            # its error is bounded by the size of the two sums
            dkt = ob.act_backward(inter["dQk"], st["kt"], st["enc_k"])
            dqt = ob.act_backward(inter["dQq"], st["qt"], st["enc_q"])
            t_k = (dkt * st["kr"]).sum(0)
            t_q = (dqt * st["qt"]).sum(0) / run.th["s_a"].astype(np.float64)
            size = np.linalg.norm(t_k) + np.linalg.norm(t_q)
            err = np.linalg.norm(run.grad(name) - g) / max(np.linalg.norm(g), 1e-2 * size)
        errs[name] = err
    print("end-to-end gradient errors:", {k: f"{v:.2e}" for k, v in errs.items()})
    assert max(errs.values()) < E2E_TOL, errs


def test_reference_block(omq, cuda_device):
    """omq_block_reference: the full-precision block (BF16 GEMM operands)."""
    M, H, I = 136, 2, 160
    cfg = synth.scaled_block(synth.BLOCK_CONFIGS["llama7b_block_w4a4"], M, H, I, seed=900)
    sh = ob.BlockShape(M=M, D=128 * H, H=H, I=I)
    inp = synth.make_block_inputs(cfg)
    blk = omq.Block(M, 128 * H, H, I, device=cuda_device)
    blk.load({k: v.to(cuda_device) for k, v in inp.W.items()},
             torch.zeros(blk.P, device=cuda_device))
    y = blk.reference(inp.x.to(cuda_device))
    torch.cuda.synchronize()
    omq.sync_check()
    y_ref = ob.block_reference(sh, _f(inp.x), {k: _f(v) for k, v in inp.W.items()})
    assert frob_rel(_f(y), y_ref) < 2e-2
    # the residual stream dominates y: check the block's own contribution too
    assert frob_rel(_f(y) - _f(inp.x), y_ref - _f(inp.x)) < 2e-2


def test_block_rejects_bad_dims(omq):
    with pytest.raises(ValueError):
        omq.Block(100, 256, 2, 352, device="cuda")       # M not a multiple of 8
    with pytest.raises(ValueError):
        omq.Block(128, 200, 2, 352, device="cuda")       # D != 128 H
