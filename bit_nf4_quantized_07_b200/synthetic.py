"""Seeded synthetic workloads shared by the tests, the smoke check and the
benchmark.  This module holds shapes, seeds and random draws only: none of the
method's arithmetic lives here, so both the CUDA path and the CPU oracle can be
fed from it without sharing any computation.

Draws are float32 from NumPy ``Generator(PCG64(seed))``; BF16 tensors are the
round-to-nearest cast of those draws done by torch.  Seeds are
``1000 * config_index + tensor_index`` with tensor indices W0=1, X=2, A=3, B=4,
dY=5.  Gaussian weights stand in for pretrained LLM weights, which the method
assumes to be roughly zero-centred normal (deck "3 QLoRA Finetuning", card 2).
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np

W0, X_, A_, B_, DY = 1, 2, 3, 4, 5


@dataclass(frozen=True)
class LinearConfig:
    name: str
    index: int
    dout: int
    din: int
    n: int
    r: int
    s: float
    w_sigma: float
    ab_sigma: float
    outlier_rate: float = 0.0     # fraction of W0 entries multiplied by 10
    backward: bool = True

    @property
    def numel(self) -> int:
        return self.dout * self.din

    def fwd_flops(self) -> int:
        """Algorithmic forward FLOPs: 2n(dout*din + r*din + dout*r)."""
        return 2 * self.n * (self.dout * self.din + self.r * self.din + self.dout * self.r)

    def bwd_flops(self) -> int:
        """Algorithmic backward FLOPs (dX, G, dA, dB): 2n(dout*din + 2r*dout + 2r*din)."""
        return 2 * self.n * (self.dout * self.din + 2 * self.r * self.dout + 2 * self.r * self.din)


PR1 = LinearConfig("pr1_512x512_n64_r8", 0, 512, 512, 64, 8, 2.0, 0.02, 0.02)
DECODE = {b: LinearConfig(f"decode_4096x4096_n{b}_r16", 1, 4096, 4096, b, 16, 2.0, 0.02, 0.01,
                          backward=False) for b in (1, 4, 16)}
PREFILL = LinearConfig("prefill_11008x4096_n2048_r16", 2, 11008, 4096, 2048, 16, 2.0, 0.02, 0.02)
LARGE = LinearConfig("large_28672x8192_n4096_r64", 3, 28672, 8192, 4096, 64, 1.0, 0.015, 0.02,
                     outlier_rate=0.001)

#: Quantize sweep: every linear of a 32-layer d=4096, ffn=11008 decoder.
SWEEP_LAYERS = 32
SWEEP_SHAPES: Tuple[Tuple[str, int, int], ...] = (
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))
SWEEP_SIGMA = 0.02
SWEEP_INDEX = 4


def sweep_params() -> int:
    return SWEEP_LAYERS * sum(r * c for _, r, c in SWEEP_SHAPES)


def seed_of(cfg_index: int, tensor: int) -> int:
    return 1000 * cfg_index + tensor


def normal_f32(shape, sigma: float, seed: int) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(seed))
    x = g.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return x


def weight_f32(cfg: LinearConfig) -> np.ndarray:
    """W0 [dout][din] float32 ~ N(0, sigma^2); with ``outlier_rate`` > 0 a
    Bernoulli-chosen fraction of the entries is multiplied by 10."""
    w = normal_f32((cfg.dout, cfg.din), cfg.w_sigma, seed_of(cfg.index, W0))
    if cfg.outlier_rate > 0:
        g = np.random.Generator(np.random.PCG64(seed_of(cfg.index, W0) + 100))
        mask = g.random(size=w.shape, dtype=np.float32) < np.float32(cfg.outlier_rate)
        w[mask] *= np.float32(10.0)
    return w


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest BF16 cast (torch's), returned as uint16 bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def activations_bf16(cfg: LinearConfig):
    """(X [n][din], A [r][din], B [dout][r], dY [n][dout]) as BF16 bits."""
    X = to_bf16_bits(normal_f32((cfg.n, cfg.din), 1.0, seed_of(cfg.index, X_)))
    A = to_bf16_bits(normal_f32((cfg.r, cfg.din), cfg.ab_sigma, seed_of(cfg.index, A_)))
    B = to_bf16_bits(normal_f32((cfg.dout, cfg.r), cfg.ab_sigma, seed_of(cfg.index, B_)))
    dY = to_bf16_bits(normal_f32((cfg.n, cfg.dout), 1.0, seed_of(cfg.index, DY)))
    return X, A, B, dY


def custom(name: str, dout: int, din: int, n: int, r: int, s: float = 2.0,
           w_sigma: float = 0.02, ab_sigma: float = 0.02, index: int = 9,
           outlier_rate: float = 0.0) -> LinearConfig:
    """A config of arbitrary shape for parity cases (ragged tails, edge sizes)."""
    return LinearConfig(name, index, dout, din, n, r, s, w_sigma, ab_sigma, outlier_rate)
