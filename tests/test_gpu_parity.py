"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs, element by element. Integer and fixed-order binary32 results bit for bit; floats
within the tolerances stated in tests/gpu_common.py."""
import numpy as np
import pytest
import torch

from oracle import omniquant as om
from post_quantization_lwc_b200 import synth
from tests.gpu_common import (SMALL_CASES, TORCH, close, dtype_round, frob_rel, max_rel,
                              operand, oracle_step, prepare)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


def _np(t):
    return t.detach().float().cpu().numpy()


def _dev(p, dev):
    g = lambda t: t.to(dev).contiguous()
    return dict(W=g(p.W), X=g(p.X), B=g(p.B), gl=g(p.gl), bl=g(p.bl), s=g(p.s), d=g(p.delta),
                Yref=torch.from_numpy(p.Yref).to(dev))


def _gpu_forward(omq, p, d):
    """The step's forward with the step's operand type (float16 for 16-bit storage)."""
    c = p.case
    s = d["s"] if c.let else None
    op = TORCH[operand(c.dtype)]
    lw = omq.lwc_quant(d["W"], d["gl"], d["bl"], c.bits, c.group, s=s, codes=True,
                       hat_dtype=op)
    la = omq.let_apply(d["X"], c.abits, s=s, delta=d["d"] if c.let else None, W=d["W"],
                       B=d["B"], want_bias=True, xq_dtype=op)
    fw = omq.fq_linear_fwd(la["Xq"], lw["W_hat"], B_tilde=la["B_tilde"], Y_ref=d["Yref"])
    return lw, la, fw


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: c.name)
def test_lwc_quant_bit_exact(omq, cuda_device, case):
    p = prepare(case)
    d = _dev(p, cuda_device)
    s = d["s"] if case.let else None
    out = omq.lwc_quant(d["W"], d["gl"], d["bl"], case.bits, case.group, s=s, codes=True)
    torch.cuda.synchronize()
    omq.sync_check()
    Wt, enc, _, _ = om.lwc_quant(synth.as_f32_numpy(p.W), p.s.numpy() if case.let else None,
                                 p.gl.numpy(), p.bl.numpy(), case.bits, case.group)
    assert np.array_equal(out["h"].cpu().numpy().view(np.uint32), enc.h.view(np.uint32))
    assert np.array_equal(out["z"].cpu().numpy(), enc.z_i32)
    assert np.array_equal(out["codes"].cpu().numpy(), enc.codes_u8)
    assert np.array_equal(_np(out["W_hat"]).view(np.uint32),
                          dtype_round(enc.deq, case.dtype).view(np.uint32))
    vmax, vmin, nmax, nmin = (x.cpu().numpy() for x in omq.range_fields(out["grp_range"]))
    assert np.array_equal(vmax, enc.vmax.reshape(-1))
    assert np.array_equal(vmin, enc.vmin.reshape(-1))
    assert np.array_equal(nmax, enc.nmax.reshape(-1))
    assert np.array_equal(nmin, enc.nmin.reshape(-1))
    # the cases exercise clipping on both sides
    assert (enc.codes == 0).any() and (enc.codes == 2 ** case.bits - 1).any()


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: c.name)
def test_let_apply(omq, cuda_device, case):
    p = prepare(case)
    d = _dev(p, cuda_device)
    s = d["s"] if case.let else None
    dl = d["d"] if case.let else None
    out = omq.let_apply(d["X"], case.abits, s=s, delta=dl, W=d["W"], B=d["B"], want_bias=True)
    torch.cuda.synchronize()
    Xt = om.let_act(synth.as_f32_numpy(p.X), p.s.numpy() if case.let else None,
                    p.delta.numpy() if case.let else None)
    aenc = om.act_quant(Xt, case.abits)
    want = Xt if aenc is None else aenc.deq
    assert np.array_equal(_np(out["Xq"]).view(np.uint32),
                          dtype_round(want, case.dtype).view(np.uint32))
    if aenc is not None:
        assert np.array_equal(out["h_a"].cpu().numpy().view(np.uint32),
                              aenc.h.reshape(-1).view(np.uint32))
        assert np.array_equal(out["z_a"].cpu().numpy(), aenc.z_i32.reshape(-1))
        vmax, vmin, nmax, nmin = (x.cpu().numpy() for x in omq.range_fields(out["tok_range"]))
        assert np.array_equal(vmax, aenc.vmax.reshape(-1))
        assert np.array_equal(nmin, aenc.nmin.reshape(-1))
    Bt = om.let_bias(synth.as_f32_numpy(p.W), p.B.numpy(), p.delta.numpy() if case.let else None)
    assert max_rel(_np(out["B_tilde"]), Bt) <= 1e-5


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: c.name)
def test_forward_loss(omq, cuda_device, case):
    p = prepare(case)
    d = _dev(p, cuda_device)
    lw, la, fw = _gpu_forward(omq, p, d)
    torch.cuda.synchronize()
    omq.sync_check()
    r = oracle_step(p, need_backward=False)
    ok, e = close(_np(fw["Y"]), r.Y, case.dtype)
    assert ok, f"Y rel err {e}"
    # dY holds the residual Y - Y*; the oracle's dL/dY is 2 (Y - Y*) / (M N)
    ok, e = close(_np(fw["dY"]), r.dY * (case.M * case.N / 2.0), case.dtype)
    assert ok, f"dY rel err {e}"
    assert abs(fw["loss"].item() - r.loss) <= (1e-4 if case.dtype == "f32" else 2e-2) * r.loss
    # the GEMM itself: fp64 product of the oracle's operands in the operand dtype; only the
    # fp32 accumulation order differs
    Xq = dtype_round(r.Xq, operand(case.dtype)).astype(np.float64)
    Wq = dtype_round(r.wenc.deq, operand(case.dtype)).astype(np.float64)
    Y_tight = Xq @ Wq.T + r.Bt[None, :]
    assert frob_rel(_np(fw["Y"]), Y_tight) <= 2e-6


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: c.name)
def test_backward_gradients(omq, cuda_device, case):
    p = prepare(case)
    d = _dev(p, cuda_device)
    lw, la, fw = _gpu_forward(omq, p, d)
    s = d["s"] if case.let else None
    g = omq.fq_linear_bwd(X=d["X"], W=d["W"], gamma_logit=d["gl"], beta_logit=d["bl"], Xq=la["Xq"],
                          W_hat=lw["W_hat"], h=lw["h"], z=lw["z"], grp_range=lw["grp_range"],
                          dY=fw["dY"], bits=case.bits, group=case.group, abits=case.abits, s=s,
                          delta=d["d"] if case.let else None, h_a=la["h_a"], z_a=la["z_a"],
                          tok_range=la["tok_range"], want_let=case.let, want_dBt=True)
    torch.cuda.synchronize()
    omq.sync_check()
    r = oracle_step(p)
    for name, got, want in (("d_gamma_logit", g["d_gamma_logit"], r.d_gamma_logit),
                            ("d_beta_logit", g["d_beta_logit"], r.d_beta_logit),
                            ("d_B_tilde", g["d_B_tilde"], r.d_Bt)):
        ok, e = close(_np(got), want, case.dtype)
        assert ok, f"{name} rel err {e}"
    if case.let:
        for name, got, want in (("d_s", g["d_s"], r.d_s), ("d_delta", g["d_delta"], r.d_delta)):
            ok, e = close(_np(got), want, case.dtype)
            assert ok, f"{name} rel err {e}"


@pytest.mark.parametrize("case", SMALL_CASES[:4], ids=lambda c: c.name)
def test_backward_is_bitwise_reproducible(omq, cuda_device, case):
    p = prepare(case)
    d = _dev(p, cuda_device)
    outs = []
    for _ in range(2):
        lw, la, fw = _gpu_forward(omq, p, d)
        s = d["s"] if case.let else None
        g = omq.fq_linear_bwd(X=d["X"], W=d["W"], gamma_logit=d["gl"], beta_logit=d["bl"],
                              Xq=la["Xq"], W_hat=lw["W_hat"], h=lw["h"], z=lw["z"],
                              grp_range=lw["grp_range"], dY=fw["dY"], bits=case.bits,
                              group=case.group, abits=case.abits, s=s,
                              delta=d["d"] if case.let else None, h_a=la["h_a"], z_a=la["z_a"],
                              tok_range=la["tok_range"], want_let=case.let)
        outs.append((fw["loss"].clone(), {k: v.clone() for k, v in g.items() if v is not None}))
    assert torch.equal(outs[0][0], outs[1][0])
    for k in outs[0][1]:
        assert torch.equal(outs[0][1][k], outs[1][1][k]), k


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: c.name)
def test_calib_step_through_one_call(omq, cuda_device, case):
    """omq_calib_step (the path bench.py times): loss, gradients and the AdamW update."""
    p = prepare(case)
    d = _dev(p, cuda_device)
    dt = torch.float32 if case.dtype == "f32" else torch.bfloat16
    lc = omq.LinearCalibration(M=case.M, N=case.N, K=case.K, group=case.group, bits=case.bits,
                               abits=case.abits, let=case.let, dtype=dt, device=cuda_device)
    lc.load(d["W"], d["gl"], d["bl"], s=d["s"], delta=d["d"], B=d["B"])
    loss = lc.step(d["X"], d["Yref"])
    torch.cuda.synchronize()
    omq.sync_check()
    r = oracle_step(p)
    assert abs(loss.item() - r.loss) <= (1e-4 if case.dtype == "f32" else 2e-2) * r.loss
    ok, e = close(_np(lc.d_gamma), r.d_gamma_logit, case.dtype)
    assert ok, e
    # AdamW step 1 moves a parameter by lr * g / (|g| + eps): about lr * sign(g) once |g| >> eps.
    # Two gradients g1 = g, g2 = g (1 + r) of the same sign give moves that differ by about
    # lr * eps * |r| / |g|: below 1e-10 for |g| > 1e-6, so there the updates agree to 1e-5
    # (binary32 rounding of the parameter) unless the sign differs. bf16 GEMM operands bound
    # the gradient's error in norm (2e-2 of ||g||), not per element, so the sign is only
    # reliable well above the noise: elements with |g| > 0.1 rms(g) must agree (99%). The
    # AdamW arithmetic itself is pinned separately; this checks the step's wiring.
    def check_update(new_gpu, old, grad_oracle, lr):
        moved = _np(new_gpu) - old
        assert np.abs(moved).max() <= lr * 1.0001
        want, _, _ = om.adamw_step(old, grad_oracle, 0, 0, 1, lr)
        rms = np.sqrt(np.mean(np.square(grad_oracle)))
        big = np.abs(grad_oracle) > max(1e-6, 0.1 * rms)
        assert big.any()
        agree = np.abs(_np(new_gpu)[big] - want[big]) <= 1e-5
        assert agree.mean() >= 0.99

    check_update(lc.gamma_logit, p.gl.numpy(), r.d_gamma_logit, om.LR_LWC)
    check_update(lc.beta_logit, p.bl.numpy(), r.d_beta_logit, om.LR_LWC)
    if case.let:
        ok, e = close(_np(lc.d_s), r.d_s, case.dtype)
        assert ok, e
        check_update(lc.s, p.s.numpy(), r.d_s, om.LR_LET)
        check_update(lc.delta, p.delta.numpy(), r.d_delta, om.LR_LET)


@pytest.mark.parametrize("case", [c for c in SMALL_CASES if c.dtype != "f32"],
                         ids=lambda c: c.name)
def test_calib_step_group_records(omq, cuda_device, case):
    """The step's group records: ranges bit for bit; the tie counts as the oracle's with LET
    (the extremes' gradient shares need them) and 0 without (nothing reads them there)."""
    p = prepare(case)
    d = _dev(p, cuda_device)
    lc = omq.LinearCalibration(M=case.M, N=case.N, K=case.K, group=case.group, bits=case.bits,
                               abits=case.abits, let=case.let, dtype=torch.bfloat16,
                               device=cuda_device)
    lc.load(d["W"], d["gl"], d["bl"], s=d["s"], delta=d["d"], B=d["B"])
    lc.step(d["X"], d["Yref"])
    torch.cuda.synchronize()
    omq.sync_check()
    s = p.s.numpy() if case.let else None
    _, enc, _, _ = om.lwc_quant(p.W.float().numpy(), s, p.gl.numpy(), p.bl.numpy(), case.bits,
                                case.group)
    vmax, vmin, nmax, nmin = (x.cpu().numpy() for x in omq.range_fields(lc.grp_range))
    assert np.array_equal(vmax, enc.vmax.reshape(-1))
    assert np.array_equal(vmin, enc.vmin.reshape(-1))
    if case.let:
        assert np.array_equal(nmax, enc.nmax.reshape(-1))
        assert np.array_equal(nmin, enc.nmin.reshape(-1))
    else:
        assert not nmax.any() and not nmin.any()


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: c.name)
def test_fold_pack_bit_exact(omq, cuda_device, case):
    p = prepare(case)
    d = _dev(p, cuda_device)
    s = d["s"] if case.let else None
    packed, h, z = omq.fold_pack(d["W"], d["gl"], d["bl"], case.bits, case.group, s=s)
    torch.cuda.synchronize()
    want, wh, wz = om.fold_pack(synth.as_f32_numpy(p.W), p.s.numpy() if case.let else None,
                                p.gl.numpy(), p.bl.numpy(), case.bits, case.group)
    assert np.array_equal(packed.cpu().numpy(), want)
    assert np.array_equal(h.cpu().numpy().view(np.uint32), wh.view(np.uint32))
    assert np.array_equal(z.cpu().numpy(), wz)


@pytest.mark.parametrize("M,N,K,dtype", [(1024, 8192, 128, torch.bfloat16),
                                         (600, 2824, 200, torch.float16),
                                         (4096, 2048, 64, torch.float16)])
def test_gemm_many_tiles_per_cta(omq, cuda_device, M, N, K, dtype):
    """More output tiles than SMs: every CTA cycles through both accumulator buffers."""
    gen = torch.Generator().manual_seed(M + N + K)
    Xq = torch.randn(M, K, generator=gen).to(dtype)
    W = (torch.randn(N, K, generator=gen) * 0.05).to(dtype)
    B = torch.randn(N, generator=gen) * 0.1
    Yref = torch.randn(M, N, generator=gen)
    out = omq.fq_linear_fwd(Xq.to(cuda_device), W.to(cuda_device), B_tilde=B.to(cuda_device),
                            Y_ref=Yref.to(cuda_device))
    torch.cuda.synchronize()
    omq.sync_check()
    Y64 = Xq.double().numpy() @ W.double().numpy().T + B.double().numpy()[None, :]
    assert frob_rel(_np(out["Y"]), Y64) <= 2e-6
    loss64 = float(np.mean((Y64 - Yref.double().numpy()) ** 2))
    assert abs(out["loss"].item() - loss64) <= 1e-5 * loss64
    R64 = Y64 - Yref.double().numpy()              # the residual stored as dY
    assert frob_rel(_np(out["dY"]), R64) <= 1e-2


def test_adamw_matches_oracle(omq, cuda_device):
    gen = torch.Generator().manual_seed(8)
    p0 = torch.randn(10007, generator=gen)
    p, m, v = p0.clone().to(cuda_device), torch.zeros(10007, device=cuda_device), torch.zeros(
        10007, device=cuda_device)
    q, mq, vq = p0.numpy().astype(np.float64), np.zeros(10007), np.zeros(10007)
    for t in range(1, 4):
        g = torch.randn(10007, generator=gen)
        omq.adamw_step(p, g.to(cuda_device), m, v, 5e-3, t, weight_decay=0.01)
        q, mq, vq = om.adamw_step(q, g.numpy(), mq, vq, t, 5e-3, weight_decay=0.01)
    torch.cuda.synchronize()
    assert np.abs(_np(p) - q).max() <= 1e-6 * np.abs(q).max()


def test_degenerate_inputs(omq, cuda_device):
    """Constant groups (h floored), an all-zero weight row, single-token activations."""
    N, K, G = 8, 64, 32
    W = torch.randn(N, K, generator=torch.Generator().manual_seed(3)) * 0.02
    W[0] = 0.25          # constant row: max == min
    W[1] = 0.0           # zero row
    W[2, :G] = -0.5      # constant first group
    gl = torch.full((N, K // G), 4.0)
    bl = torch.full((N, K // G), 4.0)
    dev = cuda_device
    out = omq.lwc_quant(W.to(dev), gl.to(dev), bl.to(dev), 4, G, codes=True)
    torch.cuda.synchronize()
    _, enc, _, _ = om.lwc_quant(W.numpy(), None, gl.numpy(), bl.numpy(), 4, G)
    assert np.array_equal(out["codes"].cpu().numpy(), enc.codes_u8)
    assert np.array_equal(out["z"].cpu().numpy(), enc.z_i32)
    assert np.array_equal(out["h"].cpu().numpy().view(np.uint32), enc.h.view(np.uint32))
    assert enc.h[0, 0] == np.float32(1e-8)
    X = torch.randn(1, K, generator=torch.Generator().manual_seed(4))
    la = omq.let_apply(X.to(dev), 4)
    torch.cuda.synchronize()
    aenc = om.act_quant(X.numpy(), 4)
    assert np.array_equal(_np(la["Xq"]), aenc.deq)


def test_rejected_call_enqueues_nothing(omq, cuda_device):
    W = torch.zeros(16, 250, device=cuda_device)
    gl = torch.zeros(16, 2, device=cuda_device)
    with pytest.raises(omq.OmqError) as e:
        omq.lwc_quant(W, gl, gl, 4, 125)
    assert e.value.status == 2
    omq.sync_check()
