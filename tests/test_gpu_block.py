"""GPU parity of the transformer-block step (omq_block_step through the C ABI) against the
block oracle (oracle/block.py), stage by stage.

Each stage of the GPU step is checked against the oracle's statement of that stage applied
to the GPU's own inputs to it (read from the workspace), so that every comparison isolates
one stage: integer decisions (weight and activation codes) must match bit for bit, values
within the tolerances below. The whole step is also compared end to end with the oracle run
on its own (loss and every parameter gradient) where the chain has no activation quantizer
to amplify rounding differences (abits = 16).

Tolerances (Frobenius-normalised unless stated):
  stages whose inputs are the same BF16 values on both sides (float32 accumulation only):
      1e-5 (GEMM outputs), 1e-4 (gradients through the STE, float32 sums)
  stages that store a BF16 result:  1e-2 (BF16 rounding is 2^-9 relative per element)
  gradients through the attention backward, whose probabilities and score gradient the GPU
  rounds to BF16 as GEMM operands: 2e-2
  end to end (abits 16): the loss 2e-2, the gradients E2E_TOL (see there)
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
# the block's output and the target, and the GPU forms y from BF16 GEMM operands at six
# linears and two attention products; the gradients then cross up to six more stages that
# round a GEMM operand to BF16 (dL/dres, dL/d[gate|up], dL/dx2, dL/dO, the probabilities and
# the score gradient, dL/d[q|k|v]). Each stage is held to its own bound above; end to end
# the measured errors are 1e-2 to 3e-2 (every parameter alike, not one stage), hence:
E2E_TOL = 5e-2

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

    def grad(self, name):
        o, n = self.blk.theta_slices[name]
        return self.gtheta[o:o + n]


@pytest.fixture(scope="module", params=range(len(CASES)), ids=lambda i: "M{}_H{}_I{}_g{}_w{}a{}".format(*CASES[i]))
def run(request, omq, cuda_device):
    return Run(omq, cuda_device, *CASES[request.param], seed=request.param)


def _bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


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
        assert np.array_equal(_bits(got), _bits(om.bf16_round(wq[name][4]))), name
    # RMSNorm, then LET + per-token quant of the GPU's a
    a = run.buf("a", M, D)
    n_ref, _ = ob.rms_norm(run.x)
    assert frob_rel(a, n_ref) < 1e-6
    qa_ref, _ = ob.act_encode(om.let_act(a, th["s1"], th["delta1"]), A, D)
    assert np.array_equal(_bits(run.buf("qa", M, D)), _bits(om.bf16_round(qa_ref)))
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
    assert np.array_equal(_bits(qqkv), _bits(om.bf16_round(want)))
    # causal softmax and P V
    Qq, Qk, Qv = qqkv[:, :D], qqkv[:, D:2 * D], qqkv[:, 2 * D:]
    P_ref, _ = ob.stage_attention(Qq, Qk, Qv, H)
    low, span = _lower(M), _span(M)
    P = np.where(low, run.buf("p", H, M, M), 0.0)
    assert frob_rel(P, P_ref) < 1e-5
    P16 = run.buf("p16", H, M, M)
    assert np.array_equal(_bits(P16[:, span]), _bits(om.bf16_round(P.astype(np.float32))[:, span]))
    P16 = np.where(span, P16, 0.0)
    O_ref = ob.unheads(np.einsum("hmn,hnd->hmd", P16.astype(np.float64), ob.heads(Qv, H)))
    O = run.buf("o", M, D)
    assert frob_rel(O, O_ref) < 1e-5
    Qo_ref, _ = ob.act_encode(O, A, D)
    assert np.array_equal(_bits(run.buf("qo", M, D)), _bits(om.bf16_round(Qo_ref)))
    # o_proj + residual, RMSNorm, LET + quant
    x2_ref = run.x.astype(np.float64) + run.buf("qo", M, D).astype(np.float64) @ run.buf(
        "what_o", D, D).astype(np.float64).T + om.let_bias(W["o"], None, th["delta_o"])
    x2 = run.buf("x2", M, D)
    assert frob_rel(x2, x2_ref) < 1e-5
    b = run.buf("b", M, D)
    assert frob_rel(b, ob.rms_norm(x2)[0]) < 1e-6
    qb_ref, _ = ob.act_encode(om.let_act(b, th["s2"], th["delta2"]), A, D)
    assert np.array_equal(_bits(run.buf("qb", M, D)), _bits(om.bf16_round(qb_ref)))
    # gate / up, SwiGLU, quant
    gu_ref = run.buf("qb", M, D).astype(np.float64) @ run.buf("what_gu", 2 * I, D).astype(
        np.float64).T + om.let_bias(W["gu"], None, th["delta2"])
    gu = run.buf("gu", M, 2 * I)
    assert frob_rel(gu, gu_ref) < 1e-5
    mid = run.buf("mid", M, I)
    assert frob_rel(mid, ob.silu(gu[:, :I]) * gu[:, I:]) < 1e-5
    qm_ref, _ = ob.act_encode(mid, A, I)
    assert np.array_equal(_bits(run.buf("qm", M, I)), _bits(om.bf16_round(qm_ref)))
    # down + residual, loss
    y = x2.astype(np.float64) + run.buf("qm", M, I).astype(np.float64) @ run.buf(
        "what_d", D, I).astype(np.float64).T
    res_ref = y - run.y_ref
    assert frob_rel(run.buf("res", M, D), res_ref) < 1e-2
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
    dm = run.buf("dmid", M, I)
    assert frob_rel(dm, dm_ref) < 1e-4
    # SwiGLU backward
    gu = run.buf("gu", M, 2 * I).astype(f64)
    g, u = gu[:, :I], gu[:, I:]
    sg = 1 / (1 + np.exp(-g))
    dgu_ref = np.concatenate([dm * u * sg * (1 + g * (1 - sg)), dm * g * sg], axis=1)
    dgu = run.buf("dgu", M, 2 * I).astype(f64)
    assert frob_rel(dgu, dgu_ref) < 1e-2
    # gate / up projection: LWC gradients, dL/db, s2 / delta2
    dWt_gu = _lwc_grad_check(run, "gu", dgu.T @ run.buf("qb", M, D).astype(f64))
    b = run.buf("b", M, D)
    bt = om.let_act(b, th["s2"], th["delta2"])
    _, enc_b = ob.act_encode(bt, A, D)
    dbt = ob.act_backward(dgu @ run.buf("what_gu", 2 * I, D).astype(f64), bt, enc_b)
    assert frob_rel(run.buf("db", M, D), dbt / th["s2"].astype(f64)) < 1e-4
    ds2, dd2 = ob.let_grads(dWt_gu, W["gu"], dbt, bt, th["s2"], dgu.sum(0))
    assert frob_rel(run.grad("s2"), ds2) < 1e-4
    assert frob_rel(run.grad("delta2"), dd2) < 1e-4
    # RMSNorm backward with the residual path
    x2 = run.buf("x2", M, D).astype(f64)
    _, rstd2 = ob.rms_norm(x2)
    dx2_ref = dy + ob.rms_backward(run.buf("db", M, D), b, rstd2)
    dx2 = run.buf("dx2", M, D).astype(f64)
    assert frob_rel(dx2, dx2_ref) < 1e-2
    # output projection: LWC gradients and dL/dO
    dWt_o = _lwc_grad_check(run, "o", dx2.T @ run.buf("qo", M, D).astype(f64))
    O = run.buf("o", M, D)
    _, enc_o = ob.act_encode(O, A, D)
    dO_ref = ob.act_backward(dx2 @ run.buf("what_o", D, D).astype(f64), O, enc_o)
    dO = run.buf("do", M, D).astype(f64)
    assert frob_rel(dO, dO_ref) < 1e-2
    # attention backward (probabilities from the GPU's float32 P)
    qqkv = run.buf("qqkv", M, 3 * D)
    P = np.where(_lower(M), run.buf("p", H, M, M), 0.0)
    dQq, dQk, dQv = ob.stage_attention_backward(dO, P, qqkv[:, :D],
                                                qqkv[:, D:2 * D], qqkv[:, 2 * D:], H)
    dqq = run.buf("dqqkv", M, 3 * D)
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
    dqkv = run.buf("dqkv", M, 3 * D).astype(f64)
    assert frob_rel(dqkv, dqkv_ref) < 1e-2
    dsa = (dkt * ap["kr"]).sum(0) - (dqt * ap["qt"]).sum(0) / sa
    assert frob_rel(run.grad("s_a"), dsa) < 1e-4
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


def test_end_to_end_against_oracle(run):
    """The whole step against the oracle run on its own inputs (no GPU intermediate)."""
    sh = run.sh
    loss, grad, _, _ = ob.block_step(sh, run.x, run.W, run.theta, run.y_ref)
    assert abs(run.loss.item() - loss) <= 2e-2 * loss
    if sh.abits < 16:
        pytest.skip("with quantized activations the stage checks above are the parity "
                    "test: rounding-level differences upstream flip activation codes")
    off = 0
    errs = {}
    for name, n in ob.theta_layout(sh):
        g = grad[off:off + n]
        off += n
        if name == "s_a":     # exactly invariant without quantized Q, K: both sides ~0
            assert np.linalg.norm(run.grad(name)) <= 1e-3 * np.linalg.norm(grad)
            continue
        errs[name] = frob_rel(run.grad(name), g)
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
