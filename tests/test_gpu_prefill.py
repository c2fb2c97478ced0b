"""Chunked prefill through the C ABI vs the fp64 oracle (needs a B200).

Token t of a chunk [s, s+C) attends the tree over the s cached tokens and the
chunk's own tokens s..t. The oracle descends over the GPU's stored node
arrays (read as data, "staged") with the chunk prefix as its local tokens;
selections must match exactly except near ties (oracle margin < 1e-4),
outputs within max-abs 2e-2 (bf16 I/O, fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity
from tests.test_gpu_parity import make_layer, run_decode, check_units, per_seq_queries, small

pytestmark = pytest.mark.gpu


def prefill_queries(w, runs, total):
    return [synth.prefill_queries(w.seed, b, 0, total, w.n_kv_heads, w.group, w.head_dim, w.centroids,
                                  w.sigma_noise, runs[b], w.bf16) for b in range(w.batch)]


def check_chunk(layer, w, K, V, Q, s, C, gout, gsel, tokens, rep):
    G, tol = w.group, 2e-2
    for b in range(w.batch):
        J, _ = oracle.levels(s, w.branching)
        for h in range(w.n_kv_heads):
            tK, tV = parity.gpu_tree_unit(layer, b, h, J, s) if s > 0 else ([None], [None])
            for t in tokens:
                if t >= C:
                    continue
                qu = synth.as_f32(np.ascontiguousarray(Q[b][s + t, h * G:(h + 1) * G]))
                ref = oracle.query(tK, tV, K[b, h], V[b, h], s, qu, w.head_dim, w.branching, w.k, G, w.rope_base,
                                   Kloc=K[b, h, s:s + t + 1], Vloc=V[b, h, s:s + t + 1])
                rep["queries"] += 1
                tie = parity.first_tie_level(ref)
                rep["near_ties"] += 1 if tie else 0
                differs = False
                for j in range(ref["J"], 0, -1):
                    got = [x for x in gsel[b, t, h, j - 1].tolist() if x >= 0]
                    want = [x for x in ref["sel"][j - 1].tolist() if x >= 0]
                    if got != want:
                        assert j <= tie, (s, t, b, h, j, got, want)  # exact above the first near tie
                        differs = True
                        break
                if differs:
                    rep["near_tie_sel_diff"] += 1
                    continue
                assert (gsel[b, t, h, ref["J"]:] == -1).all()
                err = np.abs(gout[b, t, h * G:(h + 1) * G] - ref["out"]).max()
                rep["max_abs"] = max(rep["max_abs"], float(err))
                assert err <= tol, (s, t, b, h, err)
                rep["checked"] += 1


def run_prefill(w, total, chunk, tokens_for, max_chunks_checked=None):
    K, V, runs = synth.cache_arrays(w, total)
    Q = prefill_queries(w, runs, total)
    layer, Wp = make_layer(w, total, max_chunk=chunk)
    J_cap, _ = layer.tree_shape()
    rep = parity.new_report()
    Kd, Vd = parity.to_dev(K, True), parity.to_dev(V, True)
    ci = 0
    for s in range(0, total, chunk):
        C = min(chunk, total - s)
        q = torch.stack([parity.to_dev(Q[b][s:s + C], True) for b in range(w.batch)])
        kc = Kd[:, :, s:s + C].permute(0, 2, 1, 3).contiguous()
        vc = Vd[:, :, s:s + C].permute(0, 2, 1, 3).contiguous()
        sel = torch.full((w.batch, C, w.n_kv_heads, J_cap, w.k), -7, dtype=torch.int32, device="cuda")
        out = layer.prefill(q, kc, vc, sel_out=sel)
        torch.cuda.synchronize()
        layer.check()
        toks = tokens_for(ci, C)
        if toks and (max_chunks_checked is None or ci in max_chunks_checked):
            check_chunk(layer, w, K, V, Q, s, C, parity.to_f64(out), sel.cpu().numpy(), toks, rep)
        layer.append(kc, vc)
        ci += 1
    torch.cuda.synchronize()
    layer.check()
    assert layer.lengths() == [total] * w.batch
    return layer, K, V, runs, Wp, rep


def test_prefill_small_multichunk():
    """Several chunks (the last one ragged) over a tree that grows by appends."""
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=128, branching=8, k=3)
    _, _, _, _, _, rep = run_prefill(w, 700, 128, lambda ci, C: sorted(set(range(0, C, 9)) | {C - 1}))
    parity.record("test_prefill_small_multichunk", "bf16 700 tokens, chunks of 128, b=8 k=3", "staged", rep)
    assert rep["checked"] > 300, rep


@pytest.mark.parametrize("D,G", [(64, 2), (128, 1), (64, 8), (128, 8)])
def test_prefill_shapes(D, G):
    w = small(batch=1, n_kv_heads=2, group=G, head_dim=D, branching=4, k=2)
    _, _, _, _, _, rep = run_prefill(w, 300, 64, lambda ci, C: list(range(0, C, 5)) + [C - 1])
    parity.record("test_prefill_shapes", f"bf16 d={D} G={G} 300 tokens, chunks of 64, b=4 k=2", "staged", rep)
    assert rep["checked"] > 100, rep


def test_prefill_first_chunk_is_causal_attention():
    """No tree before the first chunk: token t attends tokens 0..t only."""
    w = small(batch=1, n_kv_heads=1, group=4, head_dim=128, branching=16, k=4)
    _, _, _, _, _, rep = run_prefill(w, 200, 200, lambda ci, C: list(range(C)))
    assert rep["checked"] == 200, rep


def test_prefill_then_decode():
    """A cache filled by prefill + chunk appends decodes like the oracle."""
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=128, branching=8, k=3)
    total = 1100
    layer, K, V, runs, Wp, _ = run_prefill(w, total, 256, lambda ci, C: [])
    lengths = [total] * w.batch
    q = per_seq_queries(w, runs, 0, lengths)
    gout, gsel, grows = run_decode(layer, w, q)
    check_units(layer, w, K, V, Wp, lengths, q, gout, gsel, grows)


def test_prefill_131k_sampled():
    """The 131072-token chunked prefill workload (4096-token chunks, b = 64,
    k = 16): every chunk runs, sampled tokens of three chunks are checked."""
    w = synth.WORKLOADS["prefill_131k"]
    _, _, _, _, _, rep = run_prefill(w, w.length, w.chunk, lambda ci, C: [0, 1, 517, 2048, C - 1],
                                     max_chunks_checked={0, 1, 31})
    parity.record("test_prefill_131k_sampled", w.name, "staged", rep)
    assert rep["checked"] >= 40, rep


@pytest.mark.parametrize("k", [16, 40])
def test_prefill_selection_paths(k):
    """b = 64 over trees of 12K to 65K tokens: level-1 candidate lists of about
    190, 320, 640 and 1024 (the selection's 8, 16 and 32 keys-per-lane paths,
    and, with k = 40 > 32, the register path without the lane-maximum cut)."""
    w = small(batch=1, n_kv_heads=2, group=4, head_dim=128, branching=64, k=k)
    _, _, _, _, _, rep = run_prefill(w, 17 * 4096, 4096, lambda ci, C: [0, 1, 2047, C - 1],
                                     max_chunks_checked={3, 5, 10, 16})
    parity.record("test_prefill_selection_paths", f"bf16 69632 tokens, chunks of 4096, b=64 k={k}", "staged", rep)
    assert rep["checked"] >= 24, rep
