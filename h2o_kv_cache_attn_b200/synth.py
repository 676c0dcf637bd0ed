"""Seeded synthetic inputs (queries, keys, values) for chunked cache attention.

This module draws random numbers and rounds them to the input dtype; it holds
none of the attention, scoring or eviction arithmetic.  The same bytes feed the
CUDA path and the CPU oracle: tests draw on one side and copy to the other.

Recipe (per layer, per chunk c covering tokens P = c*S .. P+S-1):

* q, k, v ~ N(0, 1) drawn in float32 by torch's Philox-based generator seeded
  from (seed, layer, chunk, tensor id) through numpy's SeedSequence;
* with heavy hitters on, the keys of 1% of token positions (chosen once per
  sequence by a uniform draw < 0.01) are multiplied by 4 for every batch row and
  KV head before rounding;
* the result is rounded to the input dtype (bf16 round-to-nearest-even, or kept
  as float32).

Draws on a CUDA generator and on the CPU generator give different numbers for
the same seed (both follow the recipe); a test that compares two paths always
hands both the same tensor.
"""

from __future__ import annotations

import numpy as np
import torch

from .configs import Workload

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _seed(*parts: int) -> int:
    ss = np.random.SeedSequence([int(p) & 0xFFFFFFFF for p in parts])
    return int(ss.generate_state(1, np.uint64)[0] & np.uint64(0x7FFF_FFFF_FFFF_FFFF))


def heavy_hitter_mask(seed: int, n_tokens: int) -> np.ndarray:
    """Boolean [n_tokens]: positions whose keys are scaled x4."""
    rng = np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, 0x48483031])))
    return rng.random(n_tokens) < 0.01


class ChunkSource:
    """Draws the (q, k, v) of each chunk of one layer of a workload."""

    def __init__(self, wl: Workload, layer: int = 0, device: str | torch.device = "cpu"):
        self.wl = wl
        self.layer = layer
        self.device = torch.device(device)
        self.hh = heavy_hitter_mask(wl.seed + layer, wl.seq_len) if wl.heavy_hitters else None
        self.kv_in_dtype = torch.float32 if wl.kv_dtype == "f32" else torch.bfloat16

    def _normal(self, shape, chunk: int, which: int) -> torch.Tensor:
        g = torch.Generator(device=self.device)
        g.manual_seed(_seed(self.wl.seed, self.layer, chunk, which))
        return torch.randn(shape, generator=g, device=self.device, dtype=torch.float32)

    def chunk(self, c: int):
        wl = self.wl
        S = wl.chunk_len(c)
        P = c * wl.chunk
        q = self._normal((wl.B, wl.Hq, S, wl.d), c, 0)
        k = self._normal((wl.B, wl.Hk, S, wl.d), c, 1)
        v = self._normal((wl.B, wl.Hk, S, wl.d), c, 2)
        if self.hh is not None:
            sel = torch.from_numpy(self.hh[P:P + S]).to(self.device)
            if bool(sel.any()):
                k[:, :, sel, :] *= 4.0
        return (q.to(_TORCH_DTYPE[wl.q_dtype]), k.to(self.kv_in_dtype), v.to(self.kv_in_dtype))
