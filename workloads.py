"""Seeded synthetic inputs for the diffusion-LLM decode step (mask-only logits + unmasking).

This module only draws random numbers and lays out masks and windows.  It holds none of
the method's arithmetic (no compaction, no logits, no softmax, no top-k), so that both the
CUDA path and the CPU oracle can take their inputs from it without sharing any code that
computes a result.

Workloads (shapes and distributions follow the Mosaic page, "Mosaic: Unlocking
Long-Context Inference for Diffusion LLMs via Global Memory Planning and Dynamic Peak
Taming", Abstract and Fig. 3 (128k context, mask-ratio sweep), and the Sparse-dLLM page,
"More Results" (32-token blocks)):

  cfg0   B=1 L=256    d=256  V=4096    Bernoulli(0.5) mask            k=8
  cfg1   B=1 L=4096   d=4096 V=126464  last 1024 positions masked     k=32
  cfg2   B=1 L=32768  d=4096 V=126464  Bernoulli(0.9) mask            k=64
  cfg3x  B=1 L=131072 d=4096 V=126464  Bernoulli(r), r=0.1/0.5/0.9    k=128
  cfg1_m64  cfg1's shapes with only the last 64 positions masked (few rows: W streaming
         from HBM bounds the step, not the tensor cores)
  cfg4   B=8 L=8192   d=2048 V=151936  semi-autoregressive blocks of 32: sequence b's
         current block is block 32*b+16; it and every later position are masked, earlier
         ones are not; unmask candidates are the positions of the current block; k=4
  cfg4_block  cfg4 with logits for the current block's masked rows only (Sparse-dLLM
         page, "Experiment": block-wise decoding needs the current block only)

Random draws, in this order, from one ``torch.Generator`` (CPU) seeded with ``seed``:
W ~ N(0, 0.02^2) [V, d] in fp32, then H ~ N(0, 1) [B*L, d] in fp32, then for Bernoulli
masks U ~ Uniform[0,1) [B, L] with mask = U < r.  H and W are rounded to bfloat16
(round-to-nearest-even, ``Tensor.to(torch.bfloat16)``); both the GPU path and the oracle
see exactly those bfloat16 values.  With one seed the r-sweep of cfg3 shares W, H and U,
so its masks are nested.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    L: int
    d: int
    V: int
    k: int
    mask: str            # "bernoulli" | "suffix" | "semi_ar"
    r: float = 0.0       # Bernoulli mask ratio
    n_suffix: int = 0    # masked suffix length ("suffix")
    block: int = 32      # semi-autoregressive block length ("semi_ar")
    block_only: bool = False   # logits for the masked rows of the current block only
    w_std: float = 0.02
    h_std: float = 1.0
    description: str = ""


CONFIGS: dict[str, Config] = {
    "cfg0": Config("cfg0", B=1, L=256, d=256, V=4096, k=8, mask="bernoulli", r=0.5,
                   description="B1 L256 d256 V4096, Bernoulli(0.5) mask, k=8"),
    "cfg1": Config("cfg1", B=1, L=4096, d=4096, V=126464, k=32, mask="suffix", n_suffix=1024,
                   description="B1 L4096 d4096 V126464, prompt 3072 + 1024 masked, k=32"),
    "cfg2": Config("cfg2", B=1, L=32768, d=4096, V=126464, k=64, mask="bernoulli", r=0.9,
                   description="B1 L32768 d4096 V126464, Bernoulli(0.9) mask, k=64"),
    "cfg3_r0.1": Config("cfg3_r0.1", B=1, L=131072, d=4096, V=126464, k=128, mask="bernoulli",
                        r=0.1, description="B1 L131072 d4096 V126464, Bernoulli(0.1), k=128"),
    "cfg3_r0.5": Config("cfg3_r0.5", B=1, L=131072, d=4096, V=126464, k=128, mask="bernoulli",
                        r=0.5, description="B1 L131072 d4096 V126464, Bernoulli(0.5), k=128"),
    "cfg3_r0.9": Config("cfg3_r0.9", B=1, L=131072, d=4096, V=126464, k=128, mask="bernoulli",
                        r=0.9, description="B1 L131072 d4096 V126464, Bernoulli(0.9), k=128"),
    # supplementary, HBM-bound point: cfg1's shapes with only the last 64 positions masked
    "cfg1_m64": Config("cfg1_m64", B=1, L=4096, d=4096, V=126464, k=32, mask="suffix",
                       n_suffix=64, description="B1 L4096 d4096 V126464, last 64 masked, k=32"),
    "cfg4": Config("cfg4", B=8, L=8192, d=2048, V=151936, k=4, mask="semi_ar", block=32,
                   description="B8 L8192 d2048 V151936, 32-token blocks, current block "
                               "32b+16 and later masked, window = current block, k=4"),
    # cfg4 decoded block-wise with current-block-only logits: 8 x 32 rows (few rows, so
    # streaming W from HBM and the tensor cores bound the step about equally)
    "cfg4_block": Config("cfg4_block", B=8, L=8192, d=2048, V=151936, k=4, mask="semi_ar",
                         block=32, block_only=True,
                         description="B8 L8192 d2048 V151936, cfg4's mask and windows, logits "
                                     "for the current 32-token block only (256 rows), k=4"),
}


def get_config(name: str, **overrides) -> Config:
    """A named workload, optionally with fields replaced (used for small ragged cases)."""
    cfg = CONFIGS[name]
    if overrides:
        cfg = dataclasses.replace(cfg, **overrides)
    return cfg


def custom_config(B, L, d, V, k, mask="bernoulli", r=0.5, n_suffix=0, block=32,
                  name="custom", block_only=False) -> Config:
    return Config(name, B=B, L=L, d=d, V=V, k=k, mask=mask, r=r, n_suffix=n_suffix,
                  block=block, block_only=block_only)


def _bernoulli_mask(g: torch.Generator, B: int, L: int, r: float) -> torch.Tensor:
    u = torch.rand(B, L, generator=g, dtype=torch.float32)
    return (u < r).to(torch.uint8)


def semi_ar_block(cfg: Config, b: int) -> int:
    """Index of sequence b's current block (32*b + 16, clamped into the sequence)."""
    n_blocks = cfg.L // cfg.block
    return min(32 * b + 16, n_blocks - 1)


def make_mask(cfg: Config, g: torch.Generator | None = None) -> torch.Tensor:
    """The uint8 mask [B, L] (1 = position holds [MASK] and needs a prediction)."""
    if cfg.mask == "bernoulli":
        assert g is not None
        return _bernoulli_mask(g, cfg.B, cfg.L, cfg.r)
    m = torch.zeros(cfg.B, cfg.L, dtype=torch.uint8)
    if cfg.mask == "suffix":
        if cfg.n_suffix > 0:
            m[:, cfg.L - cfg.n_suffix:] = 1
    elif cfg.mask == "semi_ar":
        for b in range(cfg.B):
            m[b, semi_ar_block(cfg, b) * cfg.block:] = 1
    else:
        raise ValueError(f"unknown mask kind {cfg.mask!r}")
    return m


def make_windows(cfg: Config) -> tuple[np.ndarray, np.ndarray] | tuple[None, None]:
    """Per-sequence unmask window [lo, hi) (positions), or (None, None) for no window."""
    if cfg.mask != "semi_ar":
        return None, None
    lo = np.array([semi_ar_block(cfg, b) * cfg.block for b in range(cfg.B)], dtype=np.int32)
    hi = lo + cfg.block
    return lo, hi


def make_inputs(cfg: Config, seed: int = 0) -> dict:
    """All inputs of one decode step, on the CPU.

    Returns H (bf16 [B*L, d]), W (bf16 [V, d]), M (uint8 [B, L]), k, and the window arrays
    win_lo / win_hi (int32 [B] or None).
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    W = (torch.randn(cfg.V, cfg.d, generator=g, dtype=torch.float32) * cfg.w_std).to(torch.bfloat16)
    H = (torch.randn(cfg.B * cfg.L, cfg.d, generator=g, dtype=torch.float32) * cfg.h_std).to(torch.bfloat16)
    M = make_mask(cfg, g)
    lo, hi = make_windows(cfg)
    return dict(cfg=cfg, H=H, W=W, M=M, k=cfg.k, win_lo=lo, win_hi=hi, seed=seed)


def make_sweep_inputs(names: list[str], seed: int = 0) -> dict:
    """Inputs of several workloads that differ only in their Bernoulli mask ratio (the cfg3
    sweep): W and H are drawn once, and each mask is drawn from the generator state that
    follows H, exactly as ``make_inputs`` would for that workload alone."""
    cfgs = [CONFIGS[n] for n in names]
    c0 = cfgs[0]
    for c in cfgs[1:]:
        assert (c.B, c.L, c.d, c.V) == (c0.B, c0.L, c0.d, c0.V) and c.mask == "bernoulli"
    g = torch.Generator(device="cpu").manual_seed(seed)
    W = (torch.randn(c0.V, c0.d, generator=g, dtype=torch.float32) * c0.w_std).to(torch.bfloat16)
    H = (torch.randn(c0.B * c0.L, c0.d, generator=g, dtype=torch.float32) * c0.h_std).to(torch.bfloat16)
    state = g.get_state()
    out = {}
    for c in cfgs:
        g.set_state(state)
        out[c.name] = dict(cfg=c, H=H, W=W, M=make_mask(c, g), k=c.k, win_lo=None, win_hi=None,
                           seed=seed)
    return out


def sample_rows(count: int, n: int = 512, seed: int = 0) -> np.ndarray:
    """A seeded sample of compacted row numbers in [0, count), ascending."""
    if count <= n:
        return np.arange(count, dtype=np.int64)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(count, size=n, replace=False)).astype(np.int64)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bfloat16 bit patterns of a CPU tensor as a uint16 NumPy array (no rounding)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
