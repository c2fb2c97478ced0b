"""Paged token cache through the C ABI (recsa_init_paged; needs a B200).

The tokens live in a shared pool of fixed pages addressed through a
per-sequence page table (pages handed out in shuffled order, so no sequence
is contiguous in the pool). The tree, the descent and the softmax must be
exactly what the contiguous cache gives: checked against the fp64 oracle
(staged and free-running, as in test_gpu_parity) and against a contiguous
context fed the same tokens.
"""
import numpy as np
import pytest
import torch

import synth
from hierarchical_sparse_attention_tree_b200 import RecsaError, RecsaLayer
from hierarchical_sparse_attention_tree_b200 import recsa as R
from tests import parity
from tests.test_gpu_parity import check_nodes, check_units, per_seq_queries, record_all, run_decode, small

pytestmark = pytest.mark.gpu


def paged_layer(w, capacity, page_size, seed=0, spare=5, max_chunk=0):
    """A layer over a pool with every sequence's pages assigned up front, in
    a shuffled order, plus a few spare pages."""
    max_pages = -(-capacity // page_size)
    num_pages = w.batch * max_pages + spare
    perm = np.random.default_rng(seed).permutation(num_pages)[:w.batch * max_pages]
    table = perm.reshape(w.batch, max_pages).astype(np.int32)
    Wp = synth.workload_pooler(w)
    layer = RecsaLayer(w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim, w.branching, w.k, capacity,
                       parity.to_dev(Wp, w.bf16), dtype=torch.bfloat16 if w.bf16 else torch.float32,
                       rope_base=w.rope_base, max_chunk=max_chunk, page_size=page_size, num_pages=num_pages,
                       page_table=table)
    return layer, Wp, table


@pytest.mark.parametrize("bf16", [True, False])
def test_paged_ragged_decode_matches_oracle(bf16):
    w = small(batch=3, n_kv_heads=2, group=4, head_dim=128, branching=8, k=3, bf16=bf16)
    lengths = [1, 517, 3001]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp, _ = paged_layer(w, 4096, 64)
    layer.load(parity.to_dev(K, bf16), parity.to_dev(V, bf16), lengths)
    for b, L in enumerate(lengths):  # the pool holds each sequence's tokens, in order, through its table
        kt, vt = layer.tokens(b, L)
        assert torch.equal(kt, parity.to_dev(K[b, :, :L], bf16)) and torch.equal(vt, parity.to_dev(V[b, :, :L], bf16))
    check_nodes(layer, w, K, V, Wp, lengths)
    reps = None
    for s in range(3):
        q = per_seq_queries(w, runs, s, lengths)
        gout, gsel, grows = run_decode(layer, w, q)
        reps = check_units(layer, w, K, V, Wp, lengths, q, gout, gsel, grows, free_exact=not bf16, reports=reps)
    record_all("test_paged_ragged_decode_matches_oracle", f"paged {'bf16' if bf16 else 'fp32'} lengths 1/517/3001",
               reps)
    layer.check()


def test_paged_fused_steps_across_pages():
    """Fused append + decode steps that fill one page and open the next:
    the paged context matches a contiguous one bit for bit (node arrays,
    selections, rows) and to rounding in the outputs, then the oracle."""
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=128, branching=8, k=3)
    start, steps, P = [58, 121], 12, 64
    cap = max(start) + steps
    K, V, runs = synth.cache_arrays(w, cap)
    Kd, Vd = parity.to_dev(K, True), parity.to_dev(V, True)
    paged, Wp, _ = paged_layer(w, cap, P, seed=3)
    flat = RecsaLayer(w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim, w.branching, w.k, cap,
                      parity.to_dev(Wp, True), dtype=torch.bfloat16, rope_base=w.rope_base)
    K0, V0 = Kd.clone(), Vd.clone()
    for b in range(w.batch):
        K0[b, :, start[b]:] = 0
        V0[b, :, start[b]:] = 0
    paged.load(K0, V0, start)
    flat.load(K0.clone(), V0.clone(), start)
    J_cap, _ = paged.tree_shape()
    pos = list(start)
    for s in range(steps):
        kn = torch.stack([Kd[b, :, pos[b]:pos[b] + 1] for b in range(w.batch)]).permute(0, 2, 1, 3).contiguous()
        vn = torch.stack([Vd[b, :, pos[b]:pos[b] + 1] for b in range(w.batch)]).permute(0, 2, 1, 3).contiguous()
        pos = [x + 1 for x in pos]
        q = parity.to_dev(per_seq_queries(w, runs, s, pos), True)
        res = []
        for layer in (paged, flat):
            sel = torch.full((w.batch, w.n_kv_heads, J_cap, w.k), -7, dtype=torch.int32, device="cuda")
            rows = torch.zeros((w.batch, w.n_kv_heads, 2), dtype=torch.int64, device="cuda")
            res.append((layer.append_decode(kn, vn, q, sel_out=sel, rows_out=rows), sel, rows))
        torch.cuda.synchronize()
        assert torch.equal(res[0][1], res[1][1]) and torch.equal(res[0][2], res[1][2]), s
        assert torch.equal(res[0][0], res[1][0]), s  # the same launch shape: bit for bit
    paged.check()
    flat.check()
    for j in range(1, J_cap + 1):
        for x, y in zip(paged.level(j), flat.level(j)):
            assert torch.equal(x, y), j
    for b in range(w.batch):
        kt, vt = paged.tokens(b, pos[b])
        assert torch.equal(kt, Kd[b, :, :pos[b]]) and torch.equal(vt, Vd[b, :, :pos[b]])
    q_np = per_seq_queries(w, runs, steps - 1, pos)
    gout, gsel, grows = parity.to_f64(res[0][0]), res[0][1].cpu().numpy(), res[0][2].cpu().numpy()
    check_units(paged, w, K, V, Wp, pos, q_np, gout, gsel, grows)


def test_paged_chunked_prefill_matches_contiguous():
    """Chunked prefill and chunk appends through the page table give the
    contiguous cache's selections and outputs."""
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=128, branching=8, k=3)
    total, C, P = 520, 128, 64
    K, V, runs = synth.cache_arrays(w, total)
    Q = [synth.prefill_queries(w.seed, b, 0, total, w.n_kv_heads, w.group, w.head_dim, w.centroids, w.sigma_noise,
                               runs[b], True) for b in range(w.batch)]
    paged, Wp, _ = paged_layer(w, total, P, seed=7, max_chunk=C)
    flat = RecsaLayer(w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim, w.branching, w.k, total,
                      parity.to_dev(Wp, True), dtype=torch.bfloat16, rope_base=w.rope_base, max_chunk=C)
    Kd, Vd = parity.to_dev(K, True), parity.to_dev(V, True)
    J_cap, _ = paged.tree_shape()
    for s0 in range(0, total, C):
        Cc = min(C, total - s0)
        q = torch.stack([parity.to_dev(Q[b][s0:s0 + Cc], True) for b in range(w.batch)])
        kc = Kd[:, :, s0:s0 + Cc].permute(0, 2, 1, 3).contiguous()
        vc = Vd[:, :, s0:s0 + Cc].permute(0, 2, 1, 3).contiguous()
        outs = []
        for layer in (paged, flat):
            sel = torch.full((w.batch, Cc, w.n_kv_heads, J_cap, w.k), -7, dtype=torch.int32, device="cuda")
            outs.append((layer.prefill(q, kc, vc, sel_out=sel), sel))
            layer.append(kc, vc)
        torch.cuda.synchronize()
        assert torch.equal(outs[0][1], outs[1][1]), s0
        diff = (outs[0][0].float() - outs[1][0].float()).abs().max().item()
        assert diff <= 1e-2, (s0, diff)  # atomic accumulation order may differ
    paged.check()
    for j in range(1, J_cap + 1):
        for x, y in zip(paged.level(j), flat.level(j)):
            assert torch.equal(x, y), j


def test_paged_bad_page_id_is_reported():
    """A page table entry outside the pool is reported through the device
    error word; the kernels read page 0 instead of leaving the pool."""
    w = small(batch=1, n_kv_heads=1, group=4, head_dim=64, branching=8, k=2, bf16=False)
    K, V, runs = synth.cache_arrays(w, 200)
    layer, _, table = paged_layer(w, 256, 64)
    layer.load(parity.to_dev(K, False), parity.to_dev(V, False), [200])
    layer.check()
    # the next token (position 200) goes to page 3 of the sequence: point
    # that entry past the pool, then append it (the append writes that row)
    layer.page_table[0, 200 // 64] = int(layer.k_cache.shape[0]) + 100
    kn = parity.to_dev(K[:, :, 199:200], False).permute(0, 2, 1, 3).contiguous()
    layer.append_decode(kn, kn, parity.to_dev(per_seq_queries(w, runs, 0, [201]), False))
    with pytest.raises(RecsaError) as e:
        layer.check()
    assert e.value.status == R.ERR_DEVICE
