"""A stack of independent attention layers advanced chunk by chunk together.

"Learning how to Forget" (§A.5.1, loop orderings) runs the layers of a model over
one chunk of tokens before the next chunk; each layer keeps its own cache and the
policy acts per (batch row, KV head) (§3.1), so the caches of different layers
never interact.  Per chunk this driver makes the chunk's inputs for every layer of
this rank (outside the timed region), runs one batched eviction over all of them
(h2o_evict_insert_many) and then each layer's attention.  Ranks take layers
round-robin (dist.layers_for_rank) and exchange nothing; the job's time is the
slowest rank's.

The steps and the clock are passed in, so the same driver runs the CUDA library
(device events) and, in the multi-process CPU tests, a stand-in step.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable, Sequence


@dataclass
class StackTimes:
    """Per-chunk times (ms) of one pass of this rank's layers over the sequence."""

    evict_ms: list = field(default_factory=list)  # one batched eviction per chunk
    attn_ms: list = field(default_factory=list)   # all of this rank's attention calls per chunk
    chunk_len: list = field(default_factory=list)

    @property
    def total_ms(self) -> float:
        return float(sum(self.evict_ms) + sum(self.attn_ms))


def run_stack(layers: Sequence[int], n_chunks: int, chunk_len: Callable[[int], int],
              make_inputs: Callable[[int, int], object],
              evict: Callable[[int, dict], None],
              attend: Callable[[int, int, object], None],
              finish: Callable[[], None],
              clock) -> StackTimes:
    """One pass over n_chunks chunks for `layers`.

    make_inputs(layer, c) -> the chunk's inputs for that layer (untimed);
    evict(c, {layer: inputs}) -> the batched eviction/insert of chunk c;
    attend(layer, c, inputs) -> that layer's attention for chunk c;
    finish() -> the fold of the last chunk's weights (timed with the last chunk).
    clock.mark() -> a token at the current point of the work; clock.sync() waits for
    the work; clock.ms(a, b) -> the time between two tokens (after sync)."""
    marks = []
    for c in range(n_chunks):
        inputs = {layer: make_inputs(layer, c) for layer in layers}
        t0 = clock.mark()
        evict(c, inputs)
        t1 = clock.mark()
        for layer in layers:
            attend(layer, c, inputs[layer])
        if c == n_chunks - 1:
            finish()
        t2 = clock.mark()
        marks.append((t0, t1, t2))
    clock.sync()
    out = StackTimes()
    for c, (t0, t1, t2) in enumerate(marks):
        out.evict_ms.append(clock.ms(t0, t1))
        out.attn_ms.append(clock.ms(t1, t2))
        out.chunk_len.append(chunk_len(c))
    return out
