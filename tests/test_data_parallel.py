"""The exchange of data-parallel block calibration on 2 gloo ranks (host, no GPU): each rank
takes its own calibration sample, the oracle gives the block's loss and parameter gradient on
it, and allreduce_mean_ must leave both ranks holding bitwise the mean of the two gradient
vectors and losses, which is the gradient of the block objective averaged over the two
samples ("【ICLR 2024】OmniQuant: ...", section 框架: a mean over calibration samples)."""
import datetime
import os
import socket
import tempfile

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import block as ob

SHAPE = dict(M=6, D=16, H=2, I=24, wbits=4, abits=4)


def _shared(sh):
    """Weights and parameters every rank holds (one seed)."""
    gen = torch.Generator().manual_seed(11)
    D, I = sh.D, sh.I
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
            parts[name] = (0.3 * torch.randn(n, generator=gen)).numpy()
        else:
            parts[name] = (1.0 + 0.3 * (torch.rand(n, generator=gen) - 0.5)).numpy()
    return W, ob.theta_join(sh, parts).astype(np.float32)


def _sample(sh, r):
    gen = torch.Generator().manual_seed(100 + r)
    x = torch.randn(sh.M, sh.D, generator=gen)
    x[:, 1] *= 6.0
    return x.numpy()


def _grad(sh, W, theta, r):
    x = _sample(sh, r)
    loss, g, _, _ = ob.block_step(sh, x, W, theta, ob.block_reference(sh, x, W))
    return np.float32(loss), np.asarray(g, np.float32)


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from post_quantization_lwc_b200.data_parallel import allreduce_mean_, world_size
        assert world_size() == world
        sh = ob.BlockShape(**SHAPE)
        W, theta = _shared(sh)
        loss, g = _grad(sh, W, theta, rank)
        gt, lt = torch.from_numpy(g.copy()), torch.tensor([loss])
        allreduce_mean_([gt, lt])
        np.save(os.path.join(out, f"g{rank}.npy"), gt.numpy())
        np.save(os.path.join(out, f"l{rank}.npy"), lt.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_gradient_mean_over_two_gloo_ranks():
    world = 2
    with tempfile.TemporaryDirectory() as out:
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        g = [np.load(os.path.join(out, f"g{r}.npy")) for r in range(world)]
        lo = [np.load(os.path.join(out, f"l{r}.npy")) for r in range(world)]
    sh = ob.BlockShape(**SHAPE)
    W, theta = _shared(sh)
    per = [_grad(sh, W, theta, r) for r in range(world)]
    want_g = (torch.from_numpy(per[0][1]) + torch.from_numpy(per[1][1])) / world
    want_l = (torch.tensor([per[0][0]]) + torch.tensor([per[1][0]])) / world
    for r in range(world):
        assert np.array_equal(g[r].view(np.uint32), want_g.numpy().view(np.uint32))
        assert np.array_equal(lo[r].view(np.uint32), want_l.numpy().view(np.uint32))
    # the two samples give different gradients, so the exchange did something
    assert not np.array_equal(per[0][1], per[1][1])


def test_single_process_is_a_no_op():
    from post_quantization_lwc_b200.data_parallel import allreduce_mean_, world_size
    assert world_size() == 1
    t = torch.arange(5, dtype=torch.float32)
    allreduce_mean_([t])
    assert torch.equal(t, torch.arange(5, dtype=torch.float32))
