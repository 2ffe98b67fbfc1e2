"""Data-parallel block calibration on one rank: DataParallelBlock (gradient-only block step,
the exchange, then the library's AdamW on the two parameter segments) must reproduce the
block step that updates in place, and the library's own calibration loop, bit for bit."""
import numpy as np
import pytest
import torch

from post_quantization_lwc_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


M, H, I = 128, 2, 160


def _blocks(omq, dev, n=2):
    cfg = synth.scaled_block(synth.BLOCK_CONFIGS["llama7b_block_w4a4"], M, H, I, seed=950,
                             w_std=0.05)
    inp = synth.make_block_inputs(cfg)
    out = []
    for _ in range(n):
        blk = omq.Block(M, 128 * H, H, I, device=dev)
        names = [(k, blk.theta_slices[k][1]) for k in omq.THETA]
        theta = synth.random_block_theta(951, names)
        blk.load({k: v.to(dev) for k, v in inp.W.items()}, theta.to(dev))
        out.append(blk)
    gen = torch.Generator().manual_seed(952)
    xs = torch.randn(3, M, 128 * H, generator=gen).to(torch.bfloat16).to(dev)
    ys = torch.stack([out[0].reference(xs[i]).clone() for i in range(3)])
    torch.cuda.synchronize()
    return out, xs, ys


def _same(a, b):
    return np.array_equal(a.cpu().numpy().view(np.uint32), b.cpu().numpy().view(np.uint32))


def test_one_rank_step_matches_the_in_place_update(omq, cuda_device):
    from post_quantization_lwc_b200.data_parallel import DataParallelBlock
    (a, b), xs, ys = _blocks(omq, cuda_device)
    dp = DataParallelBlock(b)
    for i in range(3):
        la = a.step(xs[i], ys[i]).clone()
        lb = dp.step(xs[i], ys[i]).clone()
        torch.cuda.synchronize()
        omq.sync_check()
        assert _same(la, lb)
    assert a.t == b.t == 3
    for name in ("theta", "adam_m", "adam_v", "d_theta"):
        assert _same(getattr(a, name), getattr(b, name)), name
    # the parameters moved
    assert not _same(a.theta, _blocks(omq, cuda_device, 1)[0][0].theta)


def test_one_rank_calibrate_matches_the_library_loop(omq, cuda_device):
    from post_quantization_lwc_b200.data_parallel import DataParallelBlock
    (a, b), xs, ys = _blocks(omq, cuda_device)
    la = a.calibrate(xs, ys, 2)
    lb = DataParallelBlock(b).calibrate(xs, ys, 2)
    torch.cuda.synchronize()
    omq.sync_check()
    assert _same(la, lb)
    assert _same(a.theta, b.theta)
    assert _same(a.adam_v, b.adam_v)


def test_side_stream_step_matches_the_in_place_update(omq, cuda_device):
    """The step given a stream that is not the current one: kernels, exchange and update all
    run on that stream, so the result is bitwise the in-place step's."""
    from post_quantization_lwc_b200.data_parallel import DataParallelBlock
    (a, b), xs, ys = _blocks(omq, cuda_device)
    dp = DataParallelBlock(b)
    side = torch.cuda.Stream(device=cuda_device)
    side.wait_stream(torch.cuda.current_stream())
    for i in range(3):
        la = a.step(xs[i], ys[i]).clone()
        lb = dp.step(xs[i], ys[i], stream=side)
        side.synchronize()
        lb = lb.clone()
        torch.cuda.synchronize()
        omq.sync_check()
        assert _same(la, lb)
    for name in ("theta", "adam_m", "adam_v", "d_theta"):
        assert _same(getattr(a, name), getattr(b, name)), name
