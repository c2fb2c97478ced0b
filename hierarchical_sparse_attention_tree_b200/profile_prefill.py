"""One chunked-prefill call on a 131072-token tree (Qwen3-4B layer shape,
bf16, b = 64, k = 16, chunk 4096), for profiling the prefill kernels:

    python -m hierarchical_sparse_attention_tree_b200.profile_prefill [reps]

A warm-up call, then `reps` timed calls (CUDA events, L2 flushed before each).
"""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from hierarchical_sparse_attention_tree_b200 import RecsaLayer  # noqa: E402


def main(reps: int = 2) -> None:
    w = synth.WORKLOADS["prefill_131k"]
    B, H, Hq, D, C, Lt = w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim, w.chunk, w.length
    s0 = Lt - C
    bf = torch.bfloat16
    K, V, runs = synth.cache_arrays(w, Lt)
    Q = synth.prefill_queries(w.seed, 0, s0, Lt, H, w.group, D, w.centroids, w.sigma_noise, runs[0], True)
    Wp = synth.workload_pooler(w)
    layer = RecsaLayer(B, H, Hq, D, w.branching, w.k, Lt, torch.from_numpy(Wp).view(bf).cuda(), dtype=bf,
                       max_chunk=C)
    layer.k_cache.copy_(torch.from_numpy(K).view(bf))
    layer.v_cache.copy_(torch.from_numpy(V).view(bf))
    layer.ctx.build_tree([s0])
    q = torch.from_numpy(Q).view(bf).cuda().unsqueeze(0)
    kc = torch.from_numpy(np.ascontiguousarray(K[:, :, s0:].transpose(0, 2, 1, 3))).view(bf).cuda()
    vc = torch.from_numpy(np.ascontiguousarray(V[:, :, s0:].transpose(0, 2, 1, 3))).view(bf).cuda()
    out = torch.empty_like(q)
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    layer.prefill(q, kc, vc, out)
    torch.cuda.synchronize()
    for _ in range(reps):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        layer.prefill(q, kc, vc, out)
        e1.record()
        torch.cuda.synchronize()
        print(f"prefill chunk of {C} at s = {s0}: {e0.elapsed_time(e1):.2f} ms")
    layer.check()
    layer.close()


if __name__ == "__main__":
    main(int(sys.argv[1]) if len(sys.argv) > 1 else 2)
