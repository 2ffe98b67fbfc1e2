"""Seeded synthetic inputs for the fake-quantized linear calibration step.

This module holds only random-number recipes (shapes, distributions, outlier structure). It
contains none of the quantization arithmetic, and it is shared by the CUDA path's tests and
benchmark and by the CPU oracle's tests, which must see identical arrays.

The recipes stand in for the pages' calibration data (128 random 2048-token WikiText2
segments on LLaMA weights, per "【ICLR 2024】OmniQuant: Omnidirectionally Calibrated
Quantization for Large Language Models", section 实验证据), which are not available here.
They reproduce the two features the method is built around: weight tails (a few large
weights stretch a row's min/max; section LWC) and systematic per-channel activation outliers
(a few fixed channels carry large values; section LET).

All draws use one CPU ``torch.Generator`` seeded per layer, in a fixed order, so any process
regenerates the same tensors bit for bit.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class LinearConfig:
    """One calibration workload: a linear layer Y = X W^T + B with its quantizer settings.

    W is [n_out, k_in] (PyTorch layout), X is [m_tokens, k_in]. ``group`` is the LWC group
    length along k_in (``group == k_in`` means one group per output row, "per-channel").
    ``abits == 16`` disables activation quantization. ``let`` turns the learnable equivalent
    transformation on (s, delta learnable); otherwise s = 1, delta = 0 and both are frozen.
    """
    name: str
    m_tokens: int
    k_in: int
    n_out: int
    bits: int
    group: int
    abits: int
    let: bool
    dtype: str            # "f32" or "bf16": storage type of W and X
    x_kind: str           # "outlier_fixed", "outlier_uniform" or "sparse_relu"
    x_outlier_frac: float
    x_outlier_scale: tuple  # (lo, hi) multiplier range; lo == hi for a fixed multiplier
    x_outlier_count: int  # used when > 0 instead of x_outlier_frac
    let_init: str         # "identity" (s=1, delta=0) or "stats" (s from max|X|, max|W|; delta=mean X)
    steps: int
    seed: int
    logit_init: float = 4.0

    @property
    def n_groups(self) -> int:
        return self.k_in // self.group


# The four single-linear workloads. Sizes follow LLaMA-7B q_proj (4096x4096), LLaMA-7B
# gate/up (4096 -> 11008) and LLaMA-13B down_proj (13824 -> 5120) with 2048 tokens, the
# pages' calibration segment length.
CONFIGS = {
    "tiny_w4a16": LinearConfig(
        name="tiny_w4a16", m_tokens=64, k_in=256, n_out=256, bits=4, group=256, abits=16,
        let=False, dtype="f32", x_kind="outlier_fixed", x_outlier_frac=0.0,
        x_outlier_scale=(50.0, 50.0), x_outlier_count=4, let_init="identity", steps=1, seed=0),
    "llama7b_qproj_w4a16g128": LinearConfig(
        name="llama7b_qproj_w4a16g128", m_tokens=2048, k_in=4096, n_out=4096, bits=4,
        group=128, abits=16, let=True, dtype="bf16", x_kind="outlier_uniform",
        x_outlier_frac=0.01, x_outlier_scale=(20.0, 100.0), x_outlier_count=0,
        let_init="identity", steps=20, seed=1),
    "llama7b_gateup_w4a4": LinearConfig(
        name="llama7b_gateup_w4a4", m_tokens=2048, k_in=4096, n_out=11008, bits=4,
        group=4096, abits=4, let=True, dtype="bf16", x_kind="outlier_fixed",
        x_outlier_frac=0.01, x_outlier_scale=(50.0, 50.0), x_outlier_count=0,
        let_init="stats", steps=20, seed=2),
    "llama13b_down_w2a16g64": LinearConfig(
        name="llama13b_down_w2a16g64", m_tokens=2048, k_in=13824, n_out=5120, bits=2,
        group=64, abits=16, let=False, dtype="bf16", x_kind="sparse_relu",
        x_outlier_frac=0.0, x_outlier_scale=(1.0, 1.0), x_outlier_count=0,
        let_init="identity", steps=20, seed=3),
}


def scaled(cfg: LinearConfig, m_tokens: int, k_in: int, n_out: int, group: int | None = None,
           seed: int | None = None, name: str | None = None) -> LinearConfig:
    """The same recipe at another size (for parity tests that the oracle finishes quickly)."""
    g = group if group is not None else (k_in if cfg.group == cfg.k_in else cfg.group)
    return dataclasses.replace(cfg, m_tokens=m_tokens, k_in=k_in, n_out=n_out, group=g,
                               seed=cfg.seed if seed is None else seed,
                               name=name or f"{cfg.name}@{m_tokens}x{k_in}x{n_out}")


def _student_t3(gen: torch.Generator, n: int) -> torch.Tensor:
    """Student-t with 3 degrees of freedom: Z / sqrt(chi2_3 / 3)."""
    z = torch.randn(n, generator=gen, dtype=torch.float64)
    chi = torch.randn(n, 3, generator=gen, dtype=torch.float64).pow(2).sum(1)
    return z / torch.sqrt(chi / 3.0)


def _storage(t: torch.Tensor, dtype: str) -> torch.Tensor:
    return t.to(torch.float32) if dtype == "f32" else t.to(torch.bfloat16)


@dataclasses.dataclass
class LinearInputs:
    """CPU tensors of one workload. W, X in the storage dtype; everything else float32."""
    cfg: LinearConfig
    W: torch.Tensor          # [N, K]
    X: torch.Tensor          # [M, K]
    B: torch.Tensor          # [N] float32
    gamma_logit: torch.Tensor  # [N, K/G] float32
    beta_logit: torch.Tensor   # [N, K/G] float32
    s: torch.Tensor          # [K] float32
    delta: torch.Tensor      # [K] float32


def make_weight(gen: torch.Generator, n_out: int, k_in: int, dtype: str) -> torch.Tensor:
    """W ~ N(0, 0.02) with 0.5% of entries (uniform, without replacement) replaced by
    Student-t(3) x 0.1 heavy-tail values."""
    numel = n_out * k_in
    w = torch.randn(numel, generator=gen, dtype=torch.float64) * 0.02
    n_tail = max(1, int(round(0.005 * numel)))
    idx = torch.randperm(numel, generator=gen)[:n_tail]
    w[idx] = _student_t3(gen, n_tail) * 0.1
    return _storage(w.view(n_out, k_in), dtype)


def make_activation(gen: torch.Generator, cfg: LinearConfig) -> torch.Tensor:
    m, k = cfg.m_tokens, cfg.k_in
    if cfg.x_kind == "sparse_relu":
        # post-nonlinearity input of a down projection: 70% zeros, else |N(0,1)|
        x = torch.randn(m, k, generator=gen, dtype=torch.float64).abs()
        keep = torch.rand(m, k, generator=gen, dtype=torch.float64) >= 0.7
        x = x * keep
        return _storage(x, cfg.dtype)
    x = torch.randn(m, k, generator=gen, dtype=torch.float64)
    n_out = cfg.x_outlier_count if cfg.x_outlier_count > 0 else max(1, int(math.floor(cfg.x_outlier_frac * k)))
    chans = torch.randperm(k, generator=gen)[:n_out]
    lo, hi = cfg.x_outlier_scale
    if cfg.x_kind == "outlier_uniform":
        mult = lo + (hi - lo) * torch.rand(n_out, generator=gen, dtype=torch.float64)
    else:
        mult = torch.full((n_out,), lo, dtype=torch.float64)
    x[:, chans] *= mult
    return _storage(x, cfg.dtype)


def make_inputs(cfg: LinearConfig) -> LinearInputs:
    """Generate one workload's tensors in a fixed draw order: W, then X, then (LET init)."""
    gen = torch.Generator().manual_seed(cfg.seed)
    W = make_weight(gen, cfg.n_out, cfg.k_in, cfg.dtype)
    X = make_activation(gen, cfg)
    B = torch.zeros(cfg.n_out, dtype=torch.float32)   # LLaMA linears carry no bias
    ng = cfg.n_groups
    gl = torch.full((cfg.n_out, ng), cfg.logit_init, dtype=torch.float32)
    bl = torch.full((cfg.n_out, ng), cfg.logit_init, dtype=torch.float32)
    if cfg.let_init == "stats":
        # smoothing-style start: s_c = max|X_c|^0.5 / max|W_c|^0.5, delta_c = mean_m X[m, c]
        xf = X.to(torch.float64)
        wf = W.to(torch.float64)
        amax_x = xf.abs().amax(0).clamp_min(1e-5)
        amax_w = wf.abs().amax(0).clamp_min(1e-5)
        s = (amax_x.sqrt() / amax_w.sqrt()).to(torch.float32)
        delta = xf.mean(0).to(torch.float32)
    else:
        s = torch.ones(cfg.k_in, dtype=torch.float32)
        delta = torch.zeros(cfg.k_in, dtype=torch.float32)
    return LinearInputs(cfg=cfg, W=W, X=X, B=B, gamma_logit=gl, beta_logit=bl, s=s, delta=delta)


def random_logits(gen_seed: int, n_out: int, n_groups: int, lo: float = -1.0, hi: float = 5.0):
    """Spread gamma/beta logits (for tests that need clipping on both sides)."""
    gen = torch.Generator().manual_seed(gen_seed)
    gl = lo + (hi - lo) * torch.rand(n_out, n_groups, generator=gen)
    bl = lo + (hi - lo) * torch.rand(n_out, n_groups, generator=gen)
    return gl.to(torch.float32), bl.to(torch.float32)


def random_let(gen_seed: int, k_in: int):
    """A non-trivial LET state (s in [0.5, 2], delta ~ N(0, 0.3)) for tests."""
    gen = torch.Generator().manual_seed(gen_seed)
    s = 0.5 + 1.5 * torch.rand(k_in, generator=gen)
    d = 0.3 * torch.randn(k_in, generator=gen)
    return s.to(torch.float32), d.to(torch.float32)


def as_f32_numpy(t: torch.Tensor):
    """Exact float32 numpy copy of a CPU tensor (bf16 widens exactly)."""
    return t.detach().to(torch.float32).cpu().numpy()


# ------------------------------------------------------------------ one transformer block

@dataclasses.dataclass(frozen=True)
class BlockConfig:
    """One block-calibration workload: a LLaMA-shaped block (M tokens, hidden D = 128 H,
    H heads, FFN size I), LWC group (0 = per output channel), weight / activation bits."""
    name: str
    M: int
    D: int
    H: int
    I: int
    group: int
    wbits: int
    abits: int
    seed: int
    x_outlier_frac: float = 0.01
    x_outlier_scale: float = 50.0
    w_std: float = 0.02
    logit_init: float = 4.0


BLOCK_CONFIGS = {
    # LLaMA-7B block: q/k/v/o 4096 x 4096, gate/up 4096 -> 11008, down 11008 -> 4096,
    # 32 heads of 128, 2048 tokens, per-channel W4A4
    "llama7b_block_w4a4": BlockConfig(name="llama7b_block_w4a4", M=2048, D=4096, H=32,
                                      I=11008, group=0, wbits=4, abits=4, seed=4),
}


def scaled_block(cfg: BlockConfig, M: int, H: int, I: int, seed: int | None = None,
                 name: str | None = None, **kw) -> BlockConfig:
    """The same recipe at another size."""
    return dataclasses.replace(cfg, M=M, D=128 * H, H=H, I=I,
                               seed=cfg.seed if seed is None else seed,
                               name=name or f"{cfg.name}@{M}x{128 * H}x{I}", **kw)


@dataclasses.dataclass
class BlockInputs:
    cfg: BlockConfig
    x: torch.Tensor            # [M, D] bf16
    W: dict                    # qkv [3D, D], o [D, D], gu [2I, D], d [D, I], bf16


def make_block_inputs(cfg: BlockConfig) -> BlockInputs:
    """Weights ~ N(0, w_std) (rows of q, k, v, o, gate, up, down in that order), then the
    block input x ~ N(0, 1) with a fixed 1% of channels (first of a seeded permutation)
    scaled by x_outlier_scale."""
    gen = torch.Generator().manual_seed(cfg.seed)
    D, I, M = cfg.D, cfg.I, cfg.M

    def w(n, k):
        return (torch.randn(n, k, generator=gen, dtype=torch.float64) * cfg.w_std).to(
            torch.bfloat16)
    W = {"qkv": w(3 * D, D), "o": w(D, D), "gu": w(2 * I, D), "d": w(D, I)}
    x = torch.randn(M, D, generator=gen, dtype=torch.float64)
    n_out = max(1, int(math.floor(cfg.x_outlier_frac * D)))
    chans = torch.randperm(D, generator=gen)[:n_out]
    x[:, chans] *= cfg.x_outlier_scale
    return BlockInputs(cfg=cfg, x=x.to(torch.bfloat16), W=W)


def random_block_theta(gen_seed: int, names_counts, spread: float = 0.3,
                       logit_range=(1.0, 5.0)):
    """A non-trivial parameter vector for tests: logits uniform in logit_range, s in
    1 +- spread/2, delta ~ N(0, spread / 3). names_counts: ordered (name, length) pairs."""
    gen = torch.Generator().manual_seed(gen_seed)
    parts = []
    for name, n in names_counts:
        if name.startswith(("gamma", "beta")):
            lo, hi = logit_range
            parts.append(lo + (hi - lo) * torch.rand(n, generator=gen))
        elif name.startswith("delta"):
            parts.append(spread / 3 * torch.randn(n, generator=gen))
        else:
            parts.append(1.0 + spread * (torch.rand(n, generator=gen) - 0.5))
    return torch.cat(parts).to(torch.float32)


def init_block_theta(cfg: BlockConfig, names_counts):
    """The starting point of calibration: logits logit_init, s = 1, delta = 0, s_a = 1."""
    parts = []
    for name, n in names_counts:
        if name.startswith(("gamma", "beta")):
            parts.append(torch.full((n,), cfg.logit_init))
        elif name.startswith("delta"):
            parts.append(torch.zeros(n))
        else:
            parts.append(torch.ones(n))
    return torch.cat(parts).to(torch.float32)
