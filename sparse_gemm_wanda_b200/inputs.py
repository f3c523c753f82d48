"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the method: it only draws random tensors and
random tile maps.  Every tensor is drawn on the CPU with ``torch.Generator``
seeded from the workload's seed, drawn in fp32 and rounded to bf16 (RNE).

Recipe (Llama-shaped stand-ins for real weights and calibration text, which are
not used):

* weights ``W[N, K] ~ N(0, 0.02)``;
* activations ``X[T, K] ~ N(0, 1)`` with outlier channels scaled by 20; the
  outlier set is ``randperm(K)[:round(0.01 K)]`` drawn from the workload seed
  (3 channels for the tiny 256-wide case), shared by calibration and input
  activations of the same width;
* random tile maps mark exactly ``n_sparse`` tiles 2:4, the set being
  ``randperm(n_tiles)[:n_sparse]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BASE_SEED = 1234


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def outlier_channels(K: int, seed: int, count: int | None = None) -> torch.Tensor:
    if count is None:
        count = int(round(0.01 * K))
    return torch.randperm(K, generator=_gen(seed * 7 + 1))[:count]


def weight(N: int, K: int, seed: int, std: float = 0.02) -> torch.Tensor:
    w = torch.randn(N, K, generator=_gen(seed * 7 + 2), dtype=torch.float32) * std
    return w.to(torch.bfloat16)


def activations(T: int, K: int, seed: int, outliers: torch.Tensor | None,
                role: int = 0, scale: float = 20.0) -> torch.Tensor:
    x = torch.randn(T, K, generator=_gen(seed * 7 + 3 + 1000 * role), dtype=torch.float32)
    if outliers is not None and outliers.numel():
        x[:, outliers] *= scale
    return x.to(torch.bfloat16)


def activations_chunked(T: int, K: int, seed: int, outliers: torch.Tensor | None,
                        role: int = 0, chunk: int = 16384, out: torch.Tensor | None = None
                        ) -> torch.Tensor:
    """Large activation sets drawn in blocks of ``chunk`` tokens.

    Block c is ``activations(rows, K, seed, outliers, role + 100000 * c)``, so
    the first block of a set equals the unchunked draw of the same role and
    peak host memory stays at one fp32 block.
    """
    if out is None:
        out = torch.empty((T, K), dtype=torch.bfloat16)
    for c, t0 in enumerate(range(0, T, chunk)):
        rows = min(chunk, T - t0)
        out[t0:t0 + rows] = activations(rows, K, seed, outliers, role=role + 100000 * c)
    return out


def random_map(n_tiles: int, n_sparse: int, seed: int) -> torch.Tensor:
    """Bitmap words (int32 holding the uint32 bit patterns) with exactly n_sparse bits set.

    Bit t % 32 of word t // 32 is set for a 2:4 tile.
    """
    chosen = torch.randperm(n_tiles, generator=_gen(seed * 7 + 5))[:n_sparse]
    words = [0] * ((n_tiles + 31) // 32)
    for t in chosen.tolist():
        words[t // 32] |= 1 << (t % 32)
    words = [w - (1 << 32) if w >= (1 << 31) else w for w in words]
    return torch.tensor(words, dtype=torch.int32)


@dataclass
class Matrix:
    """One linear layer W[N, K]; layers with the same ``group`` read the same
    input activations (q/k/v share one input, gate/up another)."""
    name: str
    N: int
    K: int
    group: str = ""

    @property
    def input_group(self) -> str:
        return self.group or f"in{self.K}"


@dataclass
class Workload:
    """One of the named workloads; sizes only, tensors are drawn on demand."""
    name: str
    index: int
    matrices: list
    tile_n: int
    tile_k: int
    calib_tokens: int | None
    tokens: list
    fractions: list
    map_rule: str  # "random" or "loss"
    outlier_count: int | None = None
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def seed(self) -> int:
        return BASE_SEED + self.index


def workloads() -> dict:
    """The five named workloads (tiny check, decode, prefill sweep, 13B prefill, block)."""
    L7 = [Matrix("q", 4096, 4096, "attn_in"), Matrix("k", 4096, 4096, "attn_in"),
          Matrix("v", 4096, 4096, "attn_in"), Matrix("o", 4096, 4096, "attn_out"),
          Matrix("gate", 11008, 4096, "mlp_in"), Matrix("up", 11008, 4096, "mlp_in"),
          Matrix("down", 4096, 11008, "mlp_mid")]
    return {
        "tiny": Workload("tiny", 0, [Matrix("w", 256, 256)], 64, 64, 64, [8], [0.5], "random",
                         outlier_count=3,
                         notes="W 256x256, 64x64 tiles, 8 of 16 tiles 2:4, Xcal 64x256, X 8x256"),
        "llama7b-decode": Workload("llama7b-decode", 1,
                                   [Matrix("attn", 4096, 4096), Matrix("mlp_up", 11008, 4096)],
                                   128, 128, 2048, [1, 4, 16], [0.5], "loss",
                                   notes="decode GEMV, map by lowest Wanda tile loss, f=0.5"),
        "llama7b-prefill": Workload("llama7b-prefill", 2,
                                    [Matrix("mlp_up", 11008, 4096), Matrix("mlp_down", 4096, 11008)],
                                    128, 128, None, [2048], [0.0, 0.25, 0.5, 0.75, 1.0], "random",
                                    notes="prefill sweep; 2:4 patterns from Wanda with X as calibration"),
        "llama13b-prefill": Workload("llama13b-prefill", 3,
                                     [Matrix("mlp_up", 13824, 5120), Matrix("mlp_down", 5120, 13824)],
                                     128, 128, None, [4096], [1.0, 0.75], "random",
                                     notes="13B-shaped prefill, f=1 and seeded random f=0.75"),
        "llama7b-block": Workload("llama7b-block", 4, L7, 128, 128, 128 * 2048,
                                  [1, 8, 64, 512, 4096], [0.6], "loss",
                                  notes="full decoder block at 30% target sparsity"),
    }


def n_sparse_tiles(fraction: float, n_tiles: int) -> int:
    """The count of 2:4 tiles a seeded random map of this fraction gets."""
    return int(math.floor(fraction * n_tiles))
