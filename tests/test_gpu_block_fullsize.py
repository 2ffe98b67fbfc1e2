"""Full-size parity of the transformer-block step: the LLaMA-7B block workload (M = 2048
tokens, D = 4096, 32 heads, I = 11008, per-channel W4A4) through omq_block_step, the call and
launch configuration bench.py times, checked stage by stage on sampled tokens, heads and
weight rows that the block oracle (oracle/block.py) computes one by one from the GPU's own
inputs to each stage. Tolerances as in tests/test_gpu_block.py.

The target y* is a seeded synthetic array (the input plus noise), so no expected value comes
from the GPU; the check of the loss uses every token.
"""
import numpy as np
import pytest
import torch

from oracle import block as ob
from oracle import omniquant as om
from post_quantization_lwc_b200 import synth
from tests.gpu_common import frob_rel

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

TOKENS = [0, 1, 255, 256, 1031, 2047]      # first / tile edges / last
HEADS = [0, 17, 31]
ROWS = {"qkv": [0, 4095, 4096, 12287], "o": [0, 2048, 4095], "gu": [0, 11007, 11008, 22015],
        "d": [0, 4095]}


def _f(t):
    return t.detach().float().cpu().numpy()


def _bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


@pytest.fixture(scope="module")
def run(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq
    cfg = synth.BLOCK_CONFIGS["llama7b_block_w4a4"]
    sh = ob.BlockShape(M=cfg.M, D=cfg.D, H=cfg.H, I=cfg.I, wbits=cfg.wbits, abits=cfg.abits,
                       group=cfg.group)
    inp = synth.make_block_inputs(cfg)
    theta = synth.random_block_theta(4242, ob.theta_layout(sh)).numpy()
    gen = torch.Generator().manual_seed(4243)
    y_ref = (inp.x.float() + 0.05 * torch.randn(cfg.M, cfg.D, generator=gen)).numpy()
    blk = omq.Block(cfg.M, cfg.D, cfg.H, cfg.I, group=cfg.group, wbits=cfg.wbits,
                    abits=cfg.abits, device=cuda_device)
    blk.load({k: v.to(cuda_device) for k, v in inp.W.items()},
             torch.from_numpy(theta).to(cuda_device))
    loss = blk.step(inp.x.to(cuda_device), torch.from_numpy(y_ref).to(cuda_device), update=False)
    torch.cuda.synchronize()
    omq.sync_check()

    class R:
        pass
    r = R()
    r.sh, r.blk, r.y_ref, r.loss = sh, blk, y_ref, loss.item()
    r.x = _f(inp.x)
    r.W = {k: _f(v) for k, v in inp.W.items()}
    r.th = ob.theta_split(sh, theta.astype(np.float32))
    r.grad = _f(blk.d_theta)
    return r


def buf(r, name, *shape):
    return _f(r.blk.buffer(name)).reshape(*shape)


def gbuf(r, name, *shape):
    """A stored stage gradient scaled to dL (the step keeps them in units of y - y*)."""
    return buf(r, name, *shape).astype(np.float64) * (2.0 / (r.sh.M * r.sh.D))


def _f16(x):
    """The float16 operand the step stores for the binary32 value x (round to nearest even)."""
    return np.asarray(x, np.float32).astype(np.float16).astype(np.float32)


def grad(r, name):
    o, n = r.blk.theta_slices[name]
    return r.grad[o:o + n]


def test_weights_sampled_rows(run):
    r, sh = run, run.sh
    D, I = sh.D, sh.I
    s_of = {"qkv": r.th["s1"], "o": r.th["s_o"], "gu": r.th["s2"], "d": None}
    shapes = {"qkv": (3 * D, D), "o": (D, D), "gu": (2 * I, D), "d": (D, I)}
    for name, rows in ROWS.items():
        W = r.W[name][rows]
        gl = r.th["gamma_" + name][rows]
        bl = r.th["beta_" + name][rows]
        _, enc, _, _ = om.lwc_quant(W, s_of[name], gl[:, None], bl[:, None], sh.wbits, W.shape[1])
        got = buf(r, "what_" + name, *shapes[name])[rows]
        assert np.array_equal(_bits(got), _bits(_f16(enc.deq))), name


def test_forward_sampled_tokens(run):
    r, sh = run, run.sh
    M, D, H, I, A = sh.M, sh.D, sh.H, sh.I, sh.abits
    t = TOKENS
    th, W = r.th, r.W
    a = buf(r, "a", M, D)
    assert frob_rel(a[t], ob.rms_norm(r.x[t])[0]) < 1e-6
    qa_ref, _ = ob.act_encode(om.let_act(a[t], th["s1"], th["delta1"]), A, D)
    qa = buf(r, "qa", M, D)
    assert np.array_equal(_bits(qa[t]), _bits(_f16(qa_ref)))
    Wq = buf(r, "what_qkv", 3 * D, D).astype(np.float64)
    qkv = buf(r, "qkv", M, 3 * D)
    qkv_ref = qa[t].astype(np.float64) @ Wq.T + om.let_bias(W["qkv"], None, th["delta1"])
    assert frob_rel(qkv[t], qkv_ref) < 1e-5
    cos, sin = ob.rope_table(M, 128)
    rope = buf(r, "rope", 2, M, 64)
    assert np.array_equal(_bits(rope[0]), _bits(cos)) and np.array_equal(_bits(rope[1]), _bits(sin))
    ap = ob.stage_attn_prep(qkv[t], cos[t], sin[t], th["s_a"], th["s_o"], th["delta_o"], H, A)
    qqkv = buf(r, "qqkv", M, 3 * D)
    want = np.concatenate([ap["Qq"], ap["Qk"], ap["Qv"]], axis=1)
    assert np.array_equal(_bits(qqkv[t]), _bits(_f16(want)))
    # causal softmax rows of sampled (head, query), from the GPU's quantized Q, K
    P = r.blk.buffer("p").view(H, M, M)
    P16 = r.blk.buffer("p16").view(H, M, M)
    for h in HEADS:
        q = qqkv[:, h * 128:(h + 1) * 128].astype(np.float64)
        k = qqkv[:, D + h * 128:D + (h + 1) * 128].astype(np.float64)
        for i in t:
            sc = k[:i + 1] @ q[i] / np.sqrt(128.0)
            p = np.exp(sc - sc.max())
            p /= p.sum()
            assert frob_rel(_f(P[h, i, :i + 1]), p) < 1e-5
            span = min((i // 256 + 1) * 256, M)
            p16 = _f(P16[h, i, :span])
            assert np.array_equal(_bits(p16[:i + 1]), _bits(_f16(_f(P[h, i, :i + 1]))))
            assert (p16[i + 1:] == 0).all()
    # O on sampled tokens from the GPU's float16 probabilities and Qv
    O = buf(r, "o", M, D)
    qv = qqkv[:, 2 * D:].astype(np.float64)
    for i in t:
        o_ref = np.concatenate([_f(P16[h, i, :]).astype(np.float64) @ qv[:, h * 128:(h + 1) * 128]
                                for h in range(H)])
        assert frob_rel(O[i], o_ref) < 1e-5
    Qo_ref, _ = ob.act_encode(O[t], A, D)
    qo = buf(r, "qo", M, D)
    assert np.array_equal(_bits(qo[t]), _bits(_f16(Qo_ref)))
    x2 = buf(r, "x2", M, D)
    x2_ref = r.x[t].astype(np.float64) + qo[t].astype(np.float64) @ buf(
        r, "what_o", D, D).astype(np.float64).T + om.let_bias(W["o"], None, th["delta_o"])
    assert frob_rel(x2[t], x2_ref) < 1e-5
    b = buf(r, "b", M, D)
    assert frob_rel(b[t], ob.rms_norm(x2[t])[0]) < 1e-6
    qb_ref, _ = ob.act_encode(om.let_act(b[t], th["s2"], th["delta2"]), A, D)
    qb = buf(r, "qb", M, D)
    assert np.array_equal(_bits(qb[t]), _bits(_f16(qb_ref)))
    gu = buf(r, "gu", M, 2 * I)
    gu_ref = qb[t].astype(np.float64) @ buf(r, "what_gu", 2 * I, D).astype(np.float64).T + \
        om.let_bias(W["gu"], None, th["delta2"])
    assert frob_rel(gu[t], gu_ref) < 1e-5
    mid = buf(r, "mid", M, I)
    assert frob_rel(mid[t], ob.silu(gu[t, :I]) * gu[t, I:]) < 1e-5
    qm_ref, _ = ob.act_encode(mid[t], A, I)
    assert np.array_equal(_bits(buf(r, "qm", M, I)[t]), _bits(_f16(qm_ref)))


def test_loss_all_tokens(run):
    r, sh = run, run.sh
    M, D, I = sh.M, sh.D, sh.I
    y = buf(r, "x2", M, D).astype(np.float64) + buf(r, "qm", M, I).astype(np.float64) @ buf(
        r, "what_d", D, I).astype(np.float64).T
    res = y - r.y_ref
    loss_ref = float((res ** 2).mean())
    assert abs(r.loss - loss_ref) <= 1e-4 * loss_ref
    assert frob_rel(buf(r, "res", M, D), res) < 2e-3


def test_backward_sampled(run):
    r, sh = run, run.sh
    M, D, H, I, A = sh.M, sh.D, sh.H, sh.I, sh.abits
    t = TOKENS
    th, W = r.th, r.W
    f64 = np.float64
    gscale = 2.0 / (M * D)
    res = buf(r, "res", M, D).astype(f64)
    dy = gscale * res
    # LWC logit gradients of sampled weight rows: dW^[n, :] over all tokens
    wq = {name: ob.weight_quant(W[name][rows], s, th["gamma_" + name][rows],
                                th["beta_" + name][rows], sh.wbits, W[name].shape[1])
          for name, rows, s in (("d", ROWS["d"], None), ("gu", ROWS["gu"], th["s2"]),
                                ("o", ROWS["o"], th["s_o"]), ("qkv", ROWS["qkv"], th["s1"]))}
    dgu = gbuf(r, "dgu", M, 2 * I)
    dx2 = gbuf(r, "dx2", M, D)
    dqkv = gbuf(r, "dqkv", M, 3 * D)
    upstream = {"d": (dy, "qm", I), "gu": (dgu, "qb", D), "o": (dx2, "qo", D),
                "qkv": (dqkv, "qa", D)}
    for name, (dY, xq_name, K) in upstream.items():
        rows = ROWS[name]
        xq = buf(r, xq_name, M, K).astype(f64)
        dWh = dY[:, rows].T @ xq
        _, dgl, dbl = ob._lwc_grads(dWh, wq[name])
        assert frob_rel(grad(r, "gamma_" + name)[rows], dgl) < 1e-4, name
        assert frob_rel(grad(r, "beta_" + name)[rows], dbl) < 1e-4, name
    # down projection -> dL/dm on sampled tokens
    mid = buf(r, "mid", M, I)
    _, enc_m = ob.act_encode(mid[t], A, I)
    dm_ref = ob.act_backward(dy[t] @ buf(r, "what_d", D, I).astype(f64), mid[t], enc_m)
    assert frob_rel(gbuf(r, "dmid", M, I)[t], dm_ref) < 1e-4
    gu = buf(r, "gu", M, 2 * I).astype(f64)
    g, u = gu[t, :I], gu[t, I:]
    sg = 1 / (1 + np.exp(-g))
    dm = gbuf(r, "dmid", M, I)[t]
    assert frob_rel(dgu[t], np.concatenate([dm * u * sg * (1 + g * (1 - sg)), dm * g * sg], 1)) < 2e-3
    b = buf(r, "b", M, D)
    bt = om.let_act(b[t], th["s2"], th["delta2"])
    _, enc_b = ob.act_encode(bt, A, D)
    dbt = ob.act_backward(dgu[t] @ buf(r, "what_gu", 2 * I, D).astype(f64), bt, enc_b)
    db = gbuf(r, "db", M, D)
    assert frob_rel(db[t], dbt / th["s2"].astype(f64)) < 1e-4
    _, rstd2 = ob.rms_norm(buf(r, "x2", M, D)[t])
    assert frob_rel(dx2[t], dy[t] + ob.rms_backward(db[t], b[t], rstd2)) < 2e-3
    O = buf(r, "o", M, D)
    _, enc_o = ob.act_encode(O[t], A, D)
    dO_ref = ob.act_backward(dx2[t] @ buf(r, "what_o", D, D).astype(f64), O[t], enc_o)
    dO = gbuf(r, "do", M, D)
    assert frob_rel(dO[t], dO_ref) < 2e-3
    # attention backward of sampled heads, over all tokens of the head
    qqkv = buf(r, "qqkv", M, 3 * D).astype(f64)
    dqq = gbuf(r, "dqqkv", M, 3 * D)
    Pb = r.blk.buffer("p").view(H, M, M)
    low = np.tril(np.ones((M, M), dtype=bool))
    for h in HEADS:
        c = slice(h * 128, (h + 1) * 128)
        P = np.where(low, _f(Pb[h]).astype(f64), 0.0)
        q, k, v = qqkv[:, c], qqkv[:, D:][:, c], qqkv[:, 2 * D:][:, c]
        do = dO[:, c]
        dP = do @ v.T
        dS = P * (dP - (P * dP).sum(1, keepdims=True)) / np.sqrt(128.0)
        assert frob_rel(dqq[:, 2 * D:][:, c], P.T @ do) < 2e-2
        assert frob_rel(dqq[:, c], dS @ k) < 2e-2
        assert frob_rel(dqq[:, D:][:, c], dS.T @ q) < 2e-2
    # head STE and transposed transforms on sampled tokens
    cos, sin = ob.rope_table(M, 128)
    ap = ob.stage_attn_prep(buf(r, "qkv", M, 3 * D)[t], cos[t], sin[t], th["s_a"], th["s_o"],
                            th["delta_o"], H, A)
    dq_t = dqq[t]
    dqt = ob.act_backward(dq_t[:, :D], ap["qt"], ap["enc_q"])
    dkt = ob.act_backward(dq_t[:, D:2 * D], ap["kt"], ap["enc_k"])
    dvt = ob.act_backward(dq_t[:, 2 * D:], ap["vt"], ap["enc_v"])
    sa, so = th["s_a"].astype(f64), th["s_o"].astype(f64)
    want = np.concatenate([ob.rope_backward(dqt / sa, cos[t], sin[t], H),
                           ob.rope_backward(dkt * sa, cos[t], sin[t], H), dvt / so], axis=1)
    assert frob_rel(dqkv[t], want) < 2e-3
