"""Block-sequential calibration (omq_block_calibrate, omq_block_quant_forward and the stack
driver post_quantization_lwc_b200/calibrate.py) on a two-block stack.

- The library's calibration loop equals the same steps issued one at a time (bit for bit).
- Each block's next-block inputs are the fake-quantized block's outputs at its final theta.
- Against the oracle running the same procedure on its own (oracle.block.block_calibrate):
  the first step's loss within 2e-2 and both loss trajectories decreasing; the folded codes
  of each weight bit for bit given the final theta (the integer decisions of the fold).
"""
import numpy as np
import pytest
import torch

from oracle import block as ob
from oracle import omniquant as om
from post_quantization_lwc_b200 import synth

pytestmark = pytest.mark.gpu

M, H, I, S, EPOCHS = 136, 1, 160, 2, 3


def _f(t):
    return t.detach().float().cpu().numpy()


@pytest.fixture(scope="module")
def setup(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import calibrate, omq
    sh = ob.BlockShape(M=M, D=128 * H, H=H, I=I, wbits=4, abits=16)
    blocks_in = []
    for b in range(2):
        cfg = synth.scaled_block(synth.BLOCK_CONFIGS["llama7b_block_w4a4"], M, H, I,
                                 seed=600 + b, wbits=4, abits=16, w_std=0.05)
        inp = synth.make_block_inputs(cfg)
        theta = synth.init_block_theta(cfg, ob.theta_layout(sh))
        blocks_in.append((inp, theta))
    gen = torch.Generator().manual_seed(610)
    x0 = blocks_in[0][0].x
    xs = torch.stack([x0, (x0.float() + 0.3 * torch.randn(M, 128 * H, generator=gen)).to(
        torch.bfloat16)])
    blocks = []
    for inp, theta in blocks_in:
        blk = omq.Block(M, 128 * H, H, I, wbits=4, abits=16, device=cuda_device)
        blk.load({k: v.to(cuda_device) for k, v in inp.W.items()}, theta.to(cuda_device))
        blocks.append(blk)
    results, out = calibrate.calibrate_stack(blocks, xs.to(cuda_device), EPOCHS)
    torch.cuda.synchronize()
    omq.sync_check()
    return dict(omq=omq, sh=sh, blocks_in=blocks_in, xs=xs, blocks=blocks, results=results,
                out=out, dev=cuda_device)


def test_loop_equals_single_steps(setup):
    omq, dev = setup["omq"], setup["dev"]
    inp, theta = setup["blocks_in"][0]
    blk = omq.Block(M, 128 * H, H, I, wbits=4, abits=16, device=dev)
    blk.load({k: v.to(dev) for k, v in inp.W.items()}, theta.to(dev))
    xs = setup["xs"].to(dev)
    ys = torch.stack([blk.reference(xs[i]) for i in range(S)])
    losses = []
    for _ in range(EPOCHS):
        for i in range(S):
            losses.append(blk.step(xs[i], ys[i]).clone())
    torch.cuda.synchronize()
    first = setup["blocks"][0]
    assert torch.equal(blk.theta, first.theta)
    assert torch.equal(torch.stack(losses).flatten(), setup["results"][0].losses)


def test_next_block_inputs_are_quantized_outputs(setup):
    # the stack's output equals the last block's fake-quantized forward of its inputs
    blocks, dev = setup["blocks"], setup["dev"]
    xs = setup["xs"].to(dev)
    mid = torch.stack([blocks[0].quant_forward(xs[i], dtype=torch.bfloat16) for i in range(S)])
    last = torch.stack([blocks[1].quant_forward(mid[i], dtype=torch.bfloat16) for i in range(S)])
    torch.cuda.synchronize()
    assert torch.equal(last, setup["out"])


def test_against_oracle_procedure(setup):
    sh, dev = setup["sh"], setup["dev"]
    xs = [_f(setup["xs"][i]) for i in range(S)]
    for b, (inp, theta) in enumerate(setup["blocks_in"]):
        W = {k: _f(v) for k, v in inp.W.items()}
        losses, theta_o, outs = ob.block_calibrate(sh, xs, W, theta.numpy(), EPOCHS)
        gpu_losses = _f(setup["results"][b].losses)
        assert abs(gpu_losses[0] - losses[0]) <= 2e-2 * losses[0], (b, gpu_losses[0], losses[0])
        # calibration lowers the loss on both sides (the mean of the last epoch vs the first)
        for ls in (losses, gpu_losses):
            assert ls[-S:].mean() < ls[:S].mean(), (b, ls)
        # fold of the GPU's final theta: codes, h, z bit for bit
        blk = setup["blocks"][b]
        th = ob.theta_split(sh, _f(blk.theta))
        s_of = {"qkv": "s1", "o": "s_o", "gu": "s2", "d": None}
        for name, (packed, h, z) in setup["results"][b].folded.items():
            s = th[s_of[name]] if s_of[name] else None
            want, wh, wz = om.fold_pack(W[name], s, th["gamma_" + name][:, None],
                                        th["beta_" + name][:, None], 4, W[name].shape[1])
            assert np.array_equal(packed.cpu().numpy(), want), (b, name)
            assert np.array_equal(h.cpu().numpy().view(np.uint32), wh.view(np.uint32)), (b, name)
            assert np.array_equal(z.cpu().numpy(), wz), (b, name)
        # the oracle's next inputs (its own procedure), BF16 like the stack's
        xs = [om.bf16_round(o) for o in outs]
