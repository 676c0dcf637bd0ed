"""Named synthetic workloads for one attention layer with a fixed-capacity cache.

The shapes follow the setting of "Learning how to Forget: Fine-tuning for
Long-Context Sparse Attention" (§4 and §A.6.2: a Qwen3-4B-shaped model with 32
query heads, 8 KV heads, head dimension 128, cache length 16384 or 32768 and
chunk sizes 1024 / 2048 over 64K / 128K-token sequences).  All data is synthetic.
"""

from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int            # batch
    Hq: int           # query heads
    Hk: int           # KV heads (H_q = H_k * q_g)
    d: int            # head dimension
    capacity: int     # cache slots N_C
    seq_len: int      # tokens per sequence N
    chunk: int        # chunk size S
    q_dtype: str      # "f32" | "bf16"
    kv_dtype: str     # "f32" | "bf16" | "i8" | "i4"
    layers: int = 1   # independent attention layers
    heavy_hitters: bool = False  # 1% of key positions scaled x4
    seed: int = 1234

    @property
    def q_g(self) -> int:
        return self.Hq // self.Hk

    @property
    def n_chunks(self) -> int:
        return -(-self.seq_len // self.chunk)

    def chunk_len(self, c: int) -> int:
        return min(self.chunk, self.seq_len - c * self.chunk)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads: a tiny fp32 layer, the 64K/16K and 128K/32K bf16 layers,
# an int8 cache and the batch-4, 36-layer int4 stack.
TINY_F32 = Workload("tiny_h2o_fp32_c256_n1024_s128", B=1, Hq=4, Hk=2, d=64, capacity=256,
                    seq_len=1024, chunk=128, q_dtype="f32", kv_dtype="f32", seed=0)
QWEN_64K = Workload("qwen3_4b_layer_64k_c16384_s2048_bf16", B=1, Hq=32, Hk=8, d=128,
                    capacity=16384, seq_len=65536, chunk=2048, q_dtype="bf16",
                    kv_dtype="bf16", heavy_hitters=True)
QWEN_128K = Workload("qwen3_4b_layer_128k_c32768_s1024_bf16", B=1, Hq=32, Hk=8, d=128,
                     capacity=32768, seq_len=131072, chunk=1024, q_dtype="bf16",
                     kv_dtype="bf16", heavy_hitters=True)
QWEN_INT8 = Workload("qwen3_4b_layer_128k_c16384_s2048_int8", B=1, Hq=32, Hk=8, d=128,
                     capacity=16384, seq_len=131072, chunk=2048, q_dtype="bf16",
                     kv_dtype="i8", heavy_hitters=True)
STACK_INT4 = Workload("qwen3_4b_stack36_b4_128k_c32768_s2048_int4", B=4, Hq=32, Hk=8, d=128,
                      capacity=32768, seq_len=131072, chunk=2048, q_dtype="bf16",
                      kv_dtype="i4", layers=36)

WORKLOADS = {w.name: w for w in (TINY_F32, QWEN_64K, QWEN_128K, QWEN_INT8, STACK_INT4)}
SHORT = {"tiny": TINY_F32, "64k": QWEN_64K, "128k": QWEN_128K, "int8": QWEN_INT8,
         "int4stack": STACK_INT4}
