"""Block-sequential calibration of a stack of transformer blocks through libomq.

"【ICLR 2024】OmniQuant: ...", section 框架: blocks are calibrated one after another; block k
is fitted to the full-precision block's output on the calibration samples, then its quantized
weights compute the inputs of block k + 1; section 实验证据: AdamW, batch size 1, a number
of epochs over the samples (20 in the paper, 40 for W2A16). Both sides of block k's
objective see the same input, the output of the already calibrated blocks before it.

This module only sequences library calls (omq_block_reference, omq_block_calibrate,
omq_block_quant_forward, omq_fold_pack) and allocates their buffers; every computation runs
in libomq.
"""
from __future__ import annotations

import dataclasses

import torch

from post_quantization_lwc_b200 import omq


@dataclasses.dataclass
class BlockResult:
    losses: torch.Tensor          # [epochs * S] per-step losses (device)
    folded: dict                  # weight name -> (packed codes, h, z)


def calibrate_stack(blocks, xs, epochs: int, stream=None):
    """Calibrate `blocks` (omq.Block objects with weights and initial theta loaded) in order.

    xs: [S, M, D] BF16 device tensor, the first block's input for each calibration sample.
    Returns (list of BlockResult, the last block's quantized outputs [S, M, D] BF16)."""
    S = xs.shape[0]
    results = []
    for blk in blocks:
        d = blk.dims
        ys = torch.empty(S, d.M, d.D, dtype=torch.float32, device=blk.device)
        for i in range(S):
            blk.reference(xs[i], out=ys[i], stream=stream)
        losses = blk.calibrate(xs, ys, epochs, stream=stream)
        nxt = torch.empty_like(xs)
        for i in range(S):
            blk.quant_forward(xs[i], out=nxt[i], stream=stream)
        results.append(BlockResult(losses=losses, folded=blk.fold(stream=stream)))
        xs = nxt
    return results, xs
