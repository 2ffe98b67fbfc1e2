"""Shared helpers of the GPU parity tests: cases, tolerances and oracle runs."""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from oracle import omniquant as om
from post_quantization_lwc_b200 import synth

# Tolerances. Integer work (codes, zero points) and values with one fixed binary32
# operation order (h, W^, Xq, ranges) must match bit for bit. Floating-point results:
#   float32 storage:  max |gpu - oracle| / max |oracle| <= 1e-4
#   16-bit storage:   ||gpu - oracle||_F / ||oracle||_F <= 2e-2   (16-bit GEMM operands, fp32
#                     accumulation; the step uses float16 operands, rounding 2^-11 relative)
TOL_F32_MAXREL = 1e-4
TOL_BF16_FROB = 2e-2


def frob_rel(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def max_rel(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    mb = np.abs(b).max()
    return float(np.abs(a - b).max() / (mb if mb > 0 else 1.0))


def close(a, b, dtype: str) -> tuple[bool, float]:
    if dtype == "f32":
        e = max_rel(a, b)
        return e <= TOL_F32_MAXREL, e
    e = frob_rel(a, b)
    return e <= TOL_BF16_FROB, e


@dataclasses.dataclass(frozen=True)
class Case:
    name: str
    M: int
    K: int
    N: int
    group: int
    bits: int
    abits: int
    let: bool
    dtype: str
    base: str          # synth recipe the inputs follow
    seed: int = 0

    def cfg(self):
        c = synth.scaled(synth.CONFIGS[self.base], self.M, self.K, self.N, group=self.group,
                         seed=1000 + self.seed, name=self.name)
        return dataclasses.replace(c, bits=self.bits, abits=self.abits, let=self.let,
                                   dtype=self.dtype)


# Small cases: several 256 x 256 output tiles with ragged tails in every GEMM dimension
# (M, N, K not multiples of 256 / 64 / 32), both LWC launch shapes (group <= 256 power of
# two, and larger or irregular groups), the weight-side STE both inside the dW^ GEMM's
# epilogue (16-bit operands, groups a multiple of 32, per-channel included) and as its own
# kernels (fp32 operands, groups of 16), every weight / activation bit width the configs use.
SMALL_CASES = [
    Case("f32_w4a16_perchannel", 64, 256, 256, 256, 4, 16, False, "f32", "tiny_w4a16", 0),
    Case("f32_w4a8_g32_let", 72, 320, 136, 32, 4, 8, True, "f32", "llama7b_gateup_w4a4", 1),
    Case("bf16_w4a16_g128_let", 200, 384, 328, 128, 4, 16, True, "bf16",
         "llama7b_qproj_w4a16g128", 2),
    Case("bf16_w4a4_perchannel_let", 136, 512, 264, 512, 4, 4, True, "bf16",
         "llama7b_gateup_w4a4", 3),
    Case("bf16_w2a16_g64", 72, 448, 200, 64, 2, 16, False, "bf16", "llama13b_down_w2a16g64", 4),
    Case("bf16_w3a6_g96_let", 160, 288, 136, 96, 3, 6, True, "bf16", "llama7b_gateup_w4a4", 5),
    Case("bf16_w8a16_g256", 128, 768, 512, 256, 8, 16, False, "bf16", "llama7b_qproj_w4a16g128",
         6),
    Case("bf16_w4a8_g32_let", 96, 416, 264, 32, 4, 8, True, "bf16", "llama7b_gateup_w4a4", 7),
    Case("bf16_w4a16_g16_let", 80, 272, 200, 16, 4, 16, True, "bf16", "llama7b_qproj_w4a16g128",
         8),
    Case("f32_w4a4_perchannel_let", 72, 320, 136, 320, 4, 4, True, "f32", "llama7b_gateup_w4a4",
         9),
    Case("bf16_w6a6_g64_let", 96, 320, 136, 64, 6, 6, True, "bf16", "llama7b_gateup_w4a4", 10),
    # groups of 32 without LET; K = 224 leaves the last epilogue warp of a column tile one
    # 32-column chunk
    Case("bf16_w3a16_g32", 96, 224, 264, 32, 3, 16, False, "bf16", "llama13b_down_w2a16g64", 11),
]


@dataclasses.dataclass
class Prepared:
    case: Case
    W: torch.Tensor
    X: torch.Tensor
    B: torch.Tensor
    gl: torch.Tensor
    bl: torch.Tensor
    s: torch.Tensor
    delta: torch.Tensor
    Yref: np.ndarray     # float32, computed by the oracle


def prepare(case: Case) -> Prepared:
    cfg = case.cfg()
    inp = synth.make_inputs(cfg)
    gl, bl = synth.random_logits(case.seed + 77, case.N, case.K // case.group, -1.0, 5.0)
    if case.let:
        s, d = synth.random_let(case.seed + 99, case.K)
    else:
        s, d = inp.s, inp.delta
    B = torch.randn(case.N, generator=torch.Generator().manual_seed(case.seed + 5)) * 0.1
    Yref = om.reference_output(synth.as_f32_numpy(inp.X), synth.as_f32_numpy(inp.W),
                               B.numpy()).astype(np.float32)
    return Prepared(case, inp.W, inp.X, B.float(), gl, bl, s, d, Yref)


def oracle_step(p: Prepared, need_backward=True):
    c = p.case
    return om.calib_step(synth.as_f32_numpy(p.X), synth.as_f32_numpy(p.W), p.B.numpy(), p.Yref,
                         p.gl.numpy(), p.bl.numpy(), p.s.numpy(), p.delta.numpy(), c.bits,
                         c.group, c.abits, c.let, need_backward=need_backward)


def dtype_round(x, dtype: str):
    """What a tensor stored in `dtype` must hold for the binary32 value x (numpy's float16
    conversion rounds to nearest even, like the kernels)."""
    if dtype == "bf16":
        return om.bf16_round(x)
    if dtype == "f16":
        return np.asarray(x, np.float32).astype(np.float16).astype(np.float32)
    return np.asarray(x, np.float32)


def operand(dtype: str) -> str:
    """GEMM operand type the step uses for a storage type (float16 for 16-bit storage)."""
    return "f32" if dtype == "f32" else "f16"


TORCH = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
