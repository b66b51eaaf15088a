"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and nothing else: no packing, dequantizing or
dot products live here, so the CUDA path and the oracle meet only on its
outputs.  Every draw comes from ``numpy.random.default_rng([seed, layer, proj])``.

Distributions (the pages give none for the weights they ship; these stand in
for the trained Phi-3-mini / Llama-7B q4 checkpoints the pages run):

* packed weights -- uniform uint32 words, which is the same distribution as
  eight independent uniform 4-bit codes in [0, 15] per word;
* scales -- uniform on [0.005, 0.02], rounded to fp16;
* activations -- standard normal, rounded to fp16.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

import numpy as np

GROUP = 32

# projection ids used as the third seed word
PROJ_QKV, PROJ_O, PROJ_GATE_UP, PROJ_DOWN, PROJ_LM_HEAD = 0, 1, 2, 3, 4


def rng(seed: int, layer: int = 0, proj: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(layer), int(proj)])


def weights(g: np.random.Generator, n_rows: int, K: int) -> Tuple[np.ndarray, np.ndarray]:
    """(qw uint32 [n_rows][K/8], scales fp16 [n_rows][K/32])."""
    if K % GROUP:
        raise ValueError("K must be a multiple of 32")
    qw = g.integers(0, 2**32, size=(n_rows, K // 8), dtype=np.uint32)
    scales = g.uniform(0.005, 0.02, size=(n_rows, K // GROUP)).astype(np.float16)
    return qw, scales


def activations(g: np.random.Generator, M: int, K: int) -> np.ndarray:
    """x fp16 [M][K], iid N(0, 1)."""
    return g.standard_normal((M, K)).astype(np.float16)


def problem(seed: int, n_rows: int, K: int, M: int = 1, layer: int = 0, proj: int = 0):
    """One projection's inputs: (qw, scales, x)."""
    g = rng(seed, layer, proj)
    qw, s = weights(g, n_rows, K)
    x = activations(g, M, K)
    return qw, s, x


@dataclass(frozen=True)
class Proj:
    """One projection of a decode weight pass.

    kind: "gemv" (fp16 y), "gate_up" (fused SiLU(gate)*up, weight has 2*n_out
    rows) or "lm_head" (f32 logits + argmax)."""
    name: str
    kind: str
    K: int
    n_out: int
    proj_id: int

    @property
    def n_rows(self) -> int:
        return 2 * self.n_out if self.kind == "gate_up" else self.n_out

    def weight_bytes(self) -> int:
        return self.n_rows * self.K // 2 + self.n_rows * (self.K // GROUP) * 2


def phi3_mini_layer() -> List[Proj]:
    """Phi-3-mini decoder layer shapes (hidden 3072, FFN 8192)."""
    return [Proj("qkv", "gemv", 3072, 9216, PROJ_QKV),
            Proj("o", "gemv", 3072, 3072, PROJ_O),
            Proj("gate_up", "gate_up", 3072, 8192, PROJ_GATE_UP),
            Proj("down", "gemv", 8192, 3072, PROJ_DOWN)]


def phi3_mini_lm_head() -> Proj:
    return Proj("lm_head", "lm_head", 3072, 32064, PROJ_LM_HEAD)


def llama7b_layer() -> List[Proj]:
    """Llama-7B decoder layer shapes (hidden 4096, FFN 11008)."""
    return [Proj("qkv", "gemv", 4096, 12288, PROJ_QKV),
            Proj("o", "gemv", 4096, 4096, PROJ_O),
            Proj("gate_up", "gate_up", 4096, 11008, PROJ_GATE_UP),
            Proj("down", "gemv", 11008, 4096, PROJ_DOWN)]


def llama7b_lm_head() -> Proj:
    return Proj("lm_head", "lm_head", 4096, 32000, PROJ_LM_HEAD)


def proj_inputs(seed: int, layer: int, p: Proj, M: int = 1):
    """(qw, scales, x) for projection p of layer `layer`."""
    return problem(seed, p.n_rows, p.K, M=M, layer=layer, proj=p.proj_id)
