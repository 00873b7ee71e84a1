"""Seeded synthetic inputs for the BitLinear / H-BitLinear forward.

This module is the one piece the CUDA path and the CPU oracle share: it draws the inputs and
holds none of the method's arithmetic (no quantisation, transform or product).  Every array is
drawn in float32 with numpy's PCG64 generator and rounded once to bf16 (round to nearest even)
by torch on the CPU; bf16 values are returned as uint16 bit patterns so that numpy code can
use them directly (``to_torch_bf16`` views them as a torch bf16 tensor).

Distributions follow the pages' description of the layers' inputs (BitNet v2 write-up, the
paragraphs on Figures 1-3: the inputs of Wo and Wdown are sharp, mostly near zero, with a few
outlier channels; the inputs of the other projections are close to Gaussian):

* latent weights  W ~ N(0, 0.02)                                    [N, K]
* ``tiny``        X ~ Laplace(0, 0.05), 4 channels scaled by 50      [16, 256]
* ``sharp``       X ~ Laplace(0, b), b = 0.02 / ln 10 so P(|x| < 0.02) = 0.9, and
                  floor(K / 100) channels scaled by 50 (at least one)
* ``gaussian``    X ~ N(0, 1)
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

# Sub-stream ids so that X and W are independent and each reproducible on its own.
_STREAM_X = 1
_STREAM_W = 2
_STREAM_CH = 3


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream)])


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even) and return the uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_torch_bf16(bits: np.ndarray) -> torch.Tensor:
    """View uint16 bf16 bit patterns as a (CPU) torch bf16 tensor without copying values."""
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(
        torch.bfloat16)


def latent_weights(N: int, K: int, seed: int = 0, std: float = 0.02) -> np.ndarray:
    """Latent weights W ~ N(0, std) as bf16 bits [N, K]."""
    w = _rng(seed, _STREAM_W).standard_normal((N, K), dtype=np.float32)
    w *= np.float32(std)
    return f32_to_bf16_bits(w)


def _outlier_channels(K: int, count: int, seed: int) -> np.ndarray:
    return np.sort(_rng(seed, _STREAM_CH).choice(K, size=count, replace=False))


def laplace_activations(M: int, K: int, scale: float, n_outlier: int, factor: float = 50.0,
                        seed: int = 0, row0: int = 0) -> np.ndarray:
    """X ~ Laplace(0, scale) with ``n_outlier`` channels multiplied by ``factor``.

    Rows are drawn in blocks of 256 from per-block streams, so rows [row0, row0 + M) of a
    large matrix can be regenerated without drawing the rows before them.
    """
    ch = _outlier_channels(K, n_outlier, seed) if n_outlier > 0 else np.empty(0, np.int64)
    out = np.empty((M, K), dtype=np.float32)
    blk = 256
    first = row0 // blk
    last = (row0 + M + blk - 1) // blk
    for b in range(first, last):
        rows = _rng(seed, 1000 + b).laplace(0.0, scale, size=(blk, K)).astype(np.float32)
        lo = max(row0, b * blk)
        hi = min(row0 + M, (b + 1) * blk)
        out[lo - row0:hi - row0] = rows[lo - b * blk:hi - b * blk]
    if ch.size:
        out[:, ch] *= np.float32(factor)
    return f32_to_bf16_bits(out)


SHARP_SCALE = 0.02 / math.log(10.0)   # P(|x| < 0.02) = 1 - exp(-0.02 / b) = 0.9


def sharp_activations(M: int, K: int, seed: int = 0, row0: int = 0) -> np.ndarray:
    """Outlier-heavy inputs of Wo / Wdown: 90 % of |x| < 0.02, 1 % of channels x50."""
    return laplace_activations(M, K, SHARP_SCALE, max(1, K // 100), 50.0, seed, row0)


def tiny_activations(M: int = 16, K: int = 256, seed: int = 0) -> np.ndarray:
    return laplace_activations(M, K, 0.05, 4, 50.0, seed)


def gaussian_activations(M: int, K: int, seed: int = 0, row0: int = 0) -> np.ndarray:
    out = np.empty((M, K), dtype=np.float32)
    blk = 256
    for b in range(row0 // blk, (row0 + M + blk - 1) // blk):
        rows = _rng(seed, 1000 + b).standard_normal((blk, K), dtype=np.float32)
        lo = max(row0, b * blk)
        hi = min(row0 + M, (b + 1) * blk)
        out[lo - row0:hi - row0] = rows[lo - b * blk:hi - b * blk]
    return f32_to_bf16_bits(out)


@dataclass(frozen=True)
class Workload:
    """One layer shape of the pages' workloads."""
    name: str
    M: int          # tokens
    K: int          # input features
    N: int          # output features
    hadamard: bool  # H-BitLinear (True) or plain BitLinear (False)
    act_bits: int   # 8 or 4
    dist: str       # "tiny" | "sharp" | "gaussian"

    def activations(self, seed: int = 0, rows: int | None = None, row0: int = 0) -> np.ndarray:
        M = self.M if rows is None else rows
        if self.dist == "tiny":
            return tiny_activations(M, self.K, seed)
        if self.dist == "sharp":
            return sharp_activations(M, self.K, seed, row0)
        if self.dist == "gaussian":
            return gaussian_activations(M, self.K, seed, row0)
        raise ValueError(self.dist)

    def weights(self, seed: int = 0) -> np.ndarray:
        return latent_weights(self.N, self.K, seed)

    @property
    def ops(self) -> int:
        """Integer operations of the product, 2 * M * N * K."""
        return 2 * self.M * self.N * self.K


WORKLOADS = {
    # 16 tokens of a 256-wide H-BitLinear layer, INT8 activations.
    "tiny": Workload("tiny", 16, 256, 256, True, 8, "tiny"),
    # Attention output projection Wo of a 2B-class model (hidden 2048), 4096 tokens.
    "wo_2048": Workload("wo_2048", 4096, 2048, 2048, True, 8, "sharp"),
    # FFN down projection Wdown 8192 -> 2048, 8192 tokens, INT4 activations.
    "wdown_8192": Workload("wdown_8192", 8192, 8192, 2048, True, 4, "sharp"),
    # 7B-scale prefill: down projection (H-BitLinear, INT4) and up projection (BitLinear, INT8).
    "down_7b": Workload("down_7b", 16384, 16384, 4096, True, 4, "sharp"),
    "up_7b": Workload("up_7b", 16384, 4096, 16384, False, 8, "gaussian"),
}
for _m in (1, 8, 32, 64):
    WORKLOADS[f"decode_m{_m}_k8192"] = Workload(f"decode_m{_m}_k8192", _m, 8192, 2048, True, 8,
                                                "sharp")
    WORKLOADS[f"decode_m{_m}_k2048"] = Workload(f"decode_m{_m}_k2048", _m, 2048, 8192, True, 8,
                                                "sharp")
