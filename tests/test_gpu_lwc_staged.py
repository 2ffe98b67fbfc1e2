"""GPU parity of the row-staged LWC launch shape (16-bit W and W^, groups of 32 to 256
columns or one group per row, no integer codes requested) against the oracle, bit for bit:
W^, h, z and the group ranges with their tie counts. The shapes cover both buffer modes
(two staged rows per warp, and one for long rows), grouped rows staged in several pieces
(whole rows a warp with B~, single pieces dealt out without it), persistent warps with
several rows each, a ragged last 256-column segment, constant / zero rows and groups, ties at both
extremes and clipping on both sides. The same pass's B~ = B + W delta is checked through
the calibration step against the exact sum, within the binary32 summation bound."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import omniquant as om
from tests.gpu_common import dtype_round

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def omq(cuda_device):
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


@dataclasses.dataclass(frozen=True)
class StagedCase:
    name: str
    N: int
    K: int
    group: int          # == K: one group per row
    wdt: str
    hat: str
    let: bool
    bits: int = 4
    seed: int = 0


TORCH = {"bf16": torch.bfloat16, "f16": torch.float16}

CASES = [
    # one group per row, 2 rows per warp, two staged buffers
    StagedCase("bf16_row_k512_persistent", 2500, 512, 512, "bf16", "f16", True, 4, 1),
    # one group per row, one staged buffer (long rows)
    StagedCase("f16_row_k6144_single", 40, 6144, 6144, "f16", "f16", True, 4, 2),
    # groups of 128, ragged last segment (K = 33 * 128)
    StagedCase("bf16_g128_k4224_ragged", 300, 4224, 128, "bf16", "bf16", True, 4, 3),
    # groups of 64, 2 rows per warp, no LET
    StagedCase("f16_g64_k448_persistent", 2600, 448, 64, "f16", "bf16", False, 2, 4),
    StagedCase("bf16_g32_k1024", 200, 1024, 32, "bf16", "f16", True, 3, 5),
    StagedCase("bf16_g256_k2304", 150, 2304, 256, "bf16", "bf16", True, 8, 6),
    # groups of 128, one staged buffer
    StagedCase("bf16_g128_k6144_single", 64, 6144, 128, "bf16", "f16", False, 4, 7),
    # grouped rows longer than one staged piece (2048 columns): 7 pieces with a ragged last
    # one (K = 6.75 pieces), B~ summed across the pieces of a row; the down_proj row length
    StagedCase("bf16_g64_k13824_pieces", 700, 13824, 64, "bf16", "bf16", True, 2, 8),
    StagedCase("f16_g32_k2304_two_pieces", 900, 2304, 32, "f16", "f16", True, 4, 9),
    # without B~ the (row, piece) items are dealt out one by one: 3 pieces a row (the last
    # 256 columns), 15000 items, several per warp and a partial last round
    StagedCase("bf16_g128_k4352_items", 5000, 4352, 128, "bf16", "bf16", False, 3, 10),
]


def make_inputs(c: StagedCase):
    """Seeded weights with outlier columns, constant / zero rows and groups, and ties at both
    extremes of W~ = s W planted in the first group of rows 3..39; logits spanning strong to
    no clipping; a LET scale around 1, equal on column pairs (2k, 2k+1) so that a planted pair
    stays tied after scaling."""
    rng = np.random.default_rng(4000 + c.seed)
    W = rng.standard_normal((c.N, c.K)).astype(np.float32) * 0.02
    W[:, rng.choice(c.K, size=max(1, c.K // 64), replace=False)] *= 8.0
    G = c.group
    W[0] = 0.25                       # constant row
    W[1] = 0.0                        # zero row
    W[2, :G] = -0.5                   # constant first group
    W = torch.from_numpy(W).to(TORCH[c.wdt]).float().numpy()
    s = None
    if c.let:
        s = np.repeat(np.exp(rng.uniform(-0.5, 0.5, c.K // 2)), 2).astype(np.float32)
    sc = s[:G] if s is not None else 1.0
    for n in range(3, min(c.N, 40)):
        j = int(np.argmax(W[n, :G] * sc))
        W[n, j ^ 1] = W[n, j]
        j = int(np.argmin(W[n, :G] * sc))
        W[n, j ^ 1] = W[n, j]
    Wt = torch.from_numpy(W).to(TORCH[c.wdt])
    ng = c.K // G
    gl = rng.uniform(0.5, 5.0, (c.N, ng)).astype(np.float32)
    bl = rng.uniform(0.5, 5.0, (c.N, ng)).astype(np.float32)
    gl[::7] = 12.0                    # no clipping (strength ~ 1)
    return Wt, gl, bl, s


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_lwc_staged_bit_exact(omq, cuda_device, case):
    Wt, gl, bl, s = make_inputs(case)
    dev = cuda_device
    out = omq.lwc_quant(Wt.to(dev), torch.from_numpy(gl).to(dev), torch.from_numpy(bl).to(dev),
                        case.bits, case.group,
                        s=torch.from_numpy(s).to(dev) if s is not None else None,
                        hat_dtype=TORCH[case.hat])
    torch.cuda.synchronize()
    omq.sync_check()
    _, enc, _, _ = om.lwc_quant(Wt.float().numpy(), s, gl, bl, case.bits, case.group)
    assert np.array_equal(out["h"].cpu().numpy().view(np.uint32), enc.h.view(np.uint32))
    assert np.array_equal(out["z"].cpu().numpy(), enc.z_i32)
    want = dtype_round(enc.deq, case.hat)
    got = out["W_hat"].float().cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    vmax, vmin, nmax, nmin = (x.cpu().numpy() for x in omq.range_fields(out["grp_range"]))
    assert np.array_equal(vmax, enc.vmax.reshape(-1))
    assert np.array_equal(vmin, enc.vmin.reshape(-1))
    assert np.array_equal(nmax, enc.nmax.reshape(-1))
    assert np.array_equal(nmin, enc.nmin.reshape(-1))
    # the planted ties, the degenerate groups and clipping on both sides all occur
    assert (enc.nmax > 1).any() and (enc.nmin > 1).any()
    assert (enc.nmax[3:40, 0] > 1).all() and (enc.nmin[3:40, 0] > 1).all()
    assert (enc.codes == 0).any() and (enc.codes == 2 ** case.bits - 1).any()


@pytest.mark.parametrize("case", [CASES[0], CASES[2], CASES[4], CASES[7]], ids=lambda c: c.name)
def test_calib_step_fused_bias(omq, cuda_device, case):
    """B~ = B + W delta from the LWC pass of omq_calib_step (W~ = s W, LET on), with W^, h and
    z of the same pass bit for bit. (The step takes N a multiple of 8.)"""
    case = dataclasses.replace(case, N=case.N // 8 * 8)
    Wt, gl, bl, s = make_inputs(case)
    dev = cuda_device
    rng = np.random.default_rng(77 + case.seed)
    M = 96
    delta = rng.standard_normal(case.K).astype(np.float32) * 0.1
    B = rng.standard_normal(case.N).astype(np.float32) * 0.05
    X = torch.from_numpy(rng.standard_normal((M, case.K)).astype(np.float32)).to(TORCH[case.wdt])
    Yref = torch.from_numpy(rng.standard_normal((M, case.N)).astype(np.float32))
    lc = omq.LinearCalibration(M=M, N=case.N, K=case.K, group=case.group, bits=case.bits,
                               abits=16, let=True, dtype=TORCH[case.wdt], device=dev)
    lc.load(Wt.to(dev), torch.from_numpy(gl).to(dev), torch.from_numpy(bl).to(dev),
            s=torch.from_numpy(s).to(dev), delta=torch.from_numpy(delta).to(dev),
            B=torch.from_numpy(B).to(dev))
    lc.step(X.to(dev), Yref.to(dev))
    torch.cuda.synchronize()
    omq.sync_check()
    W64 = Wt.double().numpy()
    exact = B.astype(np.float64) + W64 @ delta.astype(np.float64)
    bound = case.K * 2.0 ** -24 * (np.abs(B) + np.abs(W64) @ np.abs(delta).astype(np.float64))
    err = np.abs(lc.B_tilde.cpu().numpy().astype(np.float64) - exact)
    assert (err <= bound + 1e-30).all(), float((err / np.maximum(bound, 1e-30)).max())
    _, enc, _, _ = om.lwc_quant(Wt.float().numpy(), s, gl, bl, case.bits, case.group)
    assert np.array_equal(lc.h.cpu().numpy().view(np.uint32), enc.h.view(np.uint32))
    assert np.array_equal(lc.z.cpu().numpy(), enc.z_i32)
    want = dtype_round(enc.deq, "f16" if lc.op_dtype == torch.float16 else "bf16")
    assert np.array_equal(lc.W_hat.float().cpu().numpy().view(np.uint32), want.view(np.uint32))
