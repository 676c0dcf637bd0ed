"""Drive one attention layer's cache through a sequence, chunk by chunk.

Per chunk c (tokens P = c*S .. P+S-1), in the order the paper gives ("Learning
how to Forget", §A.1: the chunk's keys and values are written into the cache
before SDPA runs):

  1. h2o_evict_insert: fold the previous chunk's summed weights into the H2O
     scores, pick S slots per (b, h_k) and write the chunk's keys/values;
  2. attn_chunk_with_scoresum: SDPA of the chunk's queries over the cache,
     returning y, the row log-sum-exp and the summed weights w.

After the last chunk, h2o_evict_insert with S = 0 folds the last w in.  A
replay run (§3.2: decisions read back from a replay log) passes the logged slots
to ``step`` and writes them with h2o_insert_at instead of step 1's choice.
"""

from __future__ import annotations

import torch

from .binding import CacheShape, KVCache
from .configs import Workload


class LayerRunner:
    def __init__(self, wl: Workload, device="cuda", with_wq: bool = False, with_lse: bool = True):
        self.wl = wl
        self.device = torch.device(device)
        self.cache = KVCache(CacheShape(wl.B, wl.Hq, wl.Hk, wl.d, wl.capacity, wl.chunk,
                                        wl.q_dtype, wl.kv_dtype), self.device)
        qt = torch.float32 if wl.q_dtype == "f32" else torch.bfloat16
        S = wl.chunk
        self.y = torch.empty((wl.B, wl.Hq, S, wl.d), dtype=qt, device=self.device)
        self.lse = torch.empty((wl.B, wl.Hq, S), dtype=torch.float32, device=self.device) if with_lse else None
        # two w buffers: the previous chunk's weights are read while the new ones are written
        self.w = [torch.zeros((wl.B, wl.Hk, wl.capacity), dtype=torch.float32, device=self.device)
                  for _ in range(2)]
        self.wq = torch.empty((wl.B, wl.Hq, wl.capacity), dtype=torch.float32,
                              device=self.device) if with_wq else None
        self.slots = torch.empty((wl.B, wl.Hk, S), dtype=torch.int32, device=self.device)
        self.chunk_index = 0
        self.P = 0

    def w_prev(self):
        return None if self.chunk_index == 0 else self.w[(self.chunk_index - 1) % 2]

    def w_cur(self):
        return self.w[self.chunk_index % 2]

    def step(self, q, k, v, stream=None, slots_in=None):
        """Process one chunk whose inputs are already on the device.  With
        ``slots_in`` ([B, H_k, S] int32) the chunk is written to those slots
        instead of the ones the policy would choose (replay of a logged
        decision); the slots then returned are slots_in."""
        S = q.shape[2]
        y = self.y[:, :, :S] if S == self.wl.chunk else torch.empty_like(q)
        lse = None
        if self.lse is not None:
            lse = self.lse[:, :, :S] if S == self.wl.chunk else torch.empty(q.shape[:3], dtype=torch.float32, device=self.device)
        if S != self.wl.chunk:
            y = y.contiguous()
        slots = self.slots[:, :, :S] if S == self.wl.chunk else torch.empty((self.wl.B, self.wl.Hk, S), dtype=torch.int32, device=self.device)
        if slots_in is None:
            self.cache.evict_insert(self.w_prev(), k, v, S, self.P, slots, stream)
        else:
            self.cache.insert_at(self.w_prev(), k, v, S, self.P, slots_in, None, stream)
            slots = slots_in
        self.cache.attend(q, S, self.P, y, lse, self.w_cur(), self.wq, stream)
        self.last = (y, lse, self.w_cur(), self.wq, slots)
        self.chunk_index += 1
        self.P += S
        return self.last

    def finish(self, stream=None):
        """Fold the last chunk's weights into the scores."""
        if self.chunk_index:
            self.cache.evict_insert(self.w_prev(), None, None, 0, self.P, None, stream)

    def reset(self, stream=None):
        self.cache.reset(stream)
        self.chunk_index = 0
        self.P = 0
