"""The synthetic workloads: shapes and generator settings, nothing else.

Each entry names a workload by what it is. The attention-layer shape of the
large ones follows a Qwen3-4B attention layer (32 query heads, 8 KV heads,
head_dim 128, RoPE base 1e6); the tiny one is an fp32 case small enough for
the CPU oracle to finish in seconds.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_kv_heads: int
    group: int            # query heads per KV head (GQA group size G)
    head_dim: int
    branching: int        # b
    k: int                # selections per level
    length: int           # tokens cached before the decode steps (or prefilled in total)
    bf16: bool
    centroids: int        # Gaussian-mixture components per KV head
    run_min: int          # token-run length range of the mixture layout
    run_max: int
    sigma_noise: float = 0.3
    rope_base: float = 1e6
    seed: int = 0
    decode_steps: int = 0  # append-one-token + decode steps after the build
    queries: int = 0       # decode queries against a fixed cache (no append)
    chunk: int = 0         # prefill chunk length (0: not a prefill workload)

    @property
    def n_q_heads(self) -> int:
        return self.n_kv_heads * self.group

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


_QWEN = dict(n_kv_heads=8, group=4, head_dim=128, branching=64, k=16, bf16=True, centroids=1024, run_min=32,
             run_max=2048)

WORKLOADS = {
    "tiny_f32": Workload(name="tiny_f32", batch=1, n_kv_heads=1, group=4, head_dim=64, branching=16, k=4,
                         length=4096, bf16=False, centroids=32, run_min=64, run_max=256, queries=8),
    "decode_131k": Workload(name="decode_131k", batch=1, length=131072, decode_steps=256, **_QWEN),
    "decode_524k_b4": Workload(name="decode_524k_b4", batch=4, length=524288, decode_steps=256, **_QWEN),
    "prefill_131k": Workload(name="prefill_131k", batch=1, length=131072, chunk=4096, **_QWEN),
    "decode_2m": Workload(name="decode_2m", batch=1, length=2097152, decode_steps=128, **_QWEN),
    "decode_524k_b1": Workload(name="decode_524k_b1", batch=1, length=524288, decode_steps=256, **_QWEN),
    "prefill_524k": Workload(name="prefill_524k", batch=1, length=524288, chunk=4096, **_QWEN),
}
