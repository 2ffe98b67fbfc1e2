"""Full-size parity: one calibration step of each single-layer workload through
omq_calib_step (the call bench.py times), against the oracle's whole step on the same seeded
inputs, element by element:

- the weight quantizer in full: every h, z and fake-quantized weight bit for bit;
- the activation quantizer in full (gate/up, W4A4): every per-token h_a, z_a and quantized
  activation bit for bit;
- the forward residual Y - Y* over all M x N outputs and the loss, within the 16-bit GEMM
  tolerance (2e-2 relative, Frobenius);
- every gradient the step produces (LWC logits, and s, delta with LET) within that tolerance;
- the fold to packed integer codes (int4 for q_proj, int2 for down_proj) bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import omniquant as om
from post_quantization_lwc_b200 import synth
from tests.gpu_common import TOL_BF16_FROB, dtype_round, frob_rel

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


def _bits_equal(a, b):
    a = np.ascontiguousarray(np.asarray(a, np.float32))
    b = np.ascontiguousarray(np.asarray(b, np.float32))
    return a.shape == b.shape and np.array_equal(a.view(np.uint32), b.view(np.uint32))


def _run(omq, cfg, dev):
    inp = synth.make_inputs(cfg)
    lc = omq.LinearCalibration(M=cfg.m_tokens, N=cfg.n_out, K=cfg.k_in, group=cfg.group,
                               bits=cfg.bits, abits=cfg.abits, let=cfg.let,
                               dtype=torch.bfloat16, device=dev)
    lc.load(inp.W.to(dev), inp.gamma_logit.to(dev), inp.beta_logit.to(dev), s=inp.s.to(dev),
            delta=inp.delta.to(dev), B=inp.B.to(dev))
    X = synth.as_f32_numpy(inp.X)
    W = synth.as_f32_numpy(inp.W)
    Yref = om.reference_output(X, W, inp.B.numpy()).astype(np.float32)
    loss = lc.step(inp.X.to(dev), torch.from_numpy(Yref).to(dev)).item()
    torch.cuda.synchronize()
    omq.sync_check()
    r = om.calib_step(X, W, inp.B.numpy(), Yref, inp.gamma_logit.numpy(),
                      inp.beta_logit.numpy(), inp.s.numpy(), inp.delta.numpy(), cfg.bits,
                      cfg.group, cfg.abits, cfg.let)
    return inp, W, Yref, lc, loss, r


def _check_step(lc, loss, r, Yref, cfg):
    op = "f16" if lc.op_dtype == torch.float16 else "bf16"      # the step's GEMM operand type
    # weight quantizer: h, z and the 16-bit GEMM operand W^ bit for bit
    assert _bits_equal(lc.h.cpu().numpy(), r.wenc.h)
    assert np.array_equal(lc.z.cpu().numpy(), r.wenc.z_i32)
    assert _bits_equal(lc.W_hat.float().cpu().numpy(), dtype_round(r.wenc.deq, op))
    # activation side: the 16-bit operand X~ / Q_a(X~) and, when quantized, h_a, z_a
    if lc.Xq is not None:
        assert _bits_equal(lc.Xq.float().cpu().numpy(), dtype_round(r.Xq, op))
    if cfg.abits < 16:
        assert _bits_equal(lc.h_a.cpu().numpy(), r.aenc.h.reshape(-1))
        assert np.array_equal(lc.z_a.cpu().numpy(), r.aenc.z_i32.reshape(-1))
    # forward: the residual Y - Y* everywhere, and the loss
    res = r.Y - Yref.astype(np.float64)
    assert frob_rel(lc.dY.float().cpu().numpy(), res) <= TOL_BF16_FROB
    assert abs(loss - r.loss) <= TOL_BF16_FROB * r.loss
    # every gradient of the step
    grads = [(lc.d_gamma, r.d_gamma_logit, "d_gamma"), (lc.d_beta, r.d_beta_logit, "d_beta")]
    if cfg.let:
        grads += [(lc.d_s, r.d_s, "d_s"), (lc.d_delta, r.d_delta, "d_delta")]
    for got, want, name in grads:
        e = frob_rel(got.cpu().numpy(), want)
        assert e <= TOL_BF16_FROB, (name, e)


def _check_fold(omq, cfg, inp, W, dev):
    s = inp.s if cfg.let else None
    gp, gh, gz = omq.fold_pack(inp.W.to(dev), inp.gamma_logit.to(dev), inp.beta_logit.to(dev),
                               cfg.bits, cfg.group, s=None if s is None else s.to(dev))
    torch.cuda.synchronize()
    packed, h, z = om.fold_pack(W, None if s is None else s.numpy(), inp.gamma_logit.numpy(),
                                inp.beta_logit.numpy(), cfg.bits, cfg.group)
    assert np.array_equal(gp.cpu().numpy(), packed)
    assert _bits_equal(gh.cpu().numpy(), h)
    assert np.array_equal(gz.cpu().numpy(), z)


def test_llama7b_qproj_w4a16g128_full_step_and_int4_fold(omq, cuda_device):
    cfg = synth.CONFIGS["llama7b_qproj_w4a16g128"]
    inp, W, Yref, lc, loss, r = _run(omq, cfg, cuda_device)
    _check_step(lc, loss, r, Yref, cfg)
    _check_fold(omq, cfg, inp, W, cuda_device)


def test_llama7b_gateup_w4a4_full_step(omq, cuda_device):
    cfg = synth.CONFIGS["llama7b_gateup_w4a4"]
    inp, W, Yref, lc, loss, r = _run(omq, cfg, cuda_device)
    assert cfg.abits == 4 and cfg.let
    _check_step(lc, loss, r, Yref, cfg)


def test_llama13b_down_w2a16g64_full_step_and_int2_fold(omq, cuda_device):
    cfg = synth.CONFIGS["llama13b_down_w2a16g64"]
    inp, W, Yref, lc, loss, r = _run(omq, cfg, cuda_device)
    assert cfg.bits == 2 and not cfg.let
    _check_step(lc, loss, r, Yref, cfg)
    _check_fold(omq, cfg, inp, W, cuda_device)
