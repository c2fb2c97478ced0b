"""The LSA-style variant through the C ABI (needs a B200): recsa_cluster_load
orders every unit's tokens hierarchically by the learned latent directions,
places them in the cache in that order and builds the tree; recsa_decode
then runs over the clustered tree.

Checked against the fp64 oracle: the order itself bit for bit
(oracle.cluster_order, whose pins are in test_oracle_cluster.py), the cache
rows (the source rows in that order, bit for bit), every tree level
(check_nodes over the reordered tokens) and decode outputs and selections
(check_units over the reordered cache, staged and free). Source: the "Latent
Sparse Attention" abstract (keys clustered hierarchically in a learned latent
space, queries scoring the hierarchy of clusters), reading R20.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from hierarchical_sparse_attention_tree_b200 import RecsaLayer
from hierarchical_sparse_attention_tree_b200.recsa import ERR_CAPACITY, ERR_UNSUPPORTED, RecsaError
from tests import parity
from tests.test_gpu_parity import check_nodes, check_units, make_layer, per_seq_queries, record_all, run_decode, small

pytestmark = pytest.mark.gpu


def _directions(layer, w, seed):
    J_cap, _ = layer.tree_shape()
    return synth.plain(903, seed, (J_cap, w.head_dim), 0.0, 1.0, False)


def _bits(t: torch.Tensor) -> np.ndarray:
    """A device tensor in the arrays' storage format (bf16 as int16 bits)."""
    t = t.contiguous()
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t).cpu().numpy()


def _reordered(A, perm, lengths):
    """A [B][H][L][d] with the first lengths[b] rows of every unit in the
    order perm gives (the rest unchanged)."""
    out = A.copy()
    for b, L in enumerate(lengths):
        for h in range(A.shape[1]):
            out[b, h, :L] = A[b, h, perm[b, h, :L]]
    return out


def _load_and_check_order(w, lengths, cap, seed):
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp = make_layer(w, cap)
    Z = _directions(layer, w, seed)
    perm_d = layer.load_clustered(parity.to_dev(K, w.bf16), parity.to_dev(V, w.bf16), lengths, torch.from_numpy(Z))
    torch.cuda.synchronize()
    layer.check()
    perm = perm_d.cpu().numpy()
    for b, L in enumerate(lengths):
        for h in range(w.n_kv_heads):
            ref = oracle.cluster_order(K[b, h], L, w.branching, Z)
            assert np.array_equal(perm[b, h, :L], ref), (b, h)
            assert (perm[b, h, L:] == -1).all()
    Kp, Vp = _reordered(K, perm, lengths), _reordered(V, perm, lengths)
    for b, L in enumerate(lengths):  # the cache holds the reordered rows, bit for bit
        kc, vc = layer.tokens(b, L)
        assert np.array_equal(_bits(kc), Kp[b, :, :L]) and np.array_equal(_bits(vc), Vp[b, :, :L])
    return layer, Wp, Kp, Vp, runs


@pytest.mark.parametrize("bf16,D,G,b,lengths", [(True, 128, 4, 8, [517, 3001]), (False, 64, 2, 5, [1, 777]),
                                                (True, 64, 8, 16, [4097, 300])])
def test_cluster_load_matches_oracle(bf16, D, G, b, lengths):
    w = small(batch=len(lengths), n_kv_heads=2, group=G, head_dim=D, branching=b, k=3, bf16=bf16)
    layer, Wp, Kp, Vp, runs = _load_and_check_order(w, lengths, 4608, seed=b)
    check_nodes(layer, w, Kp, Vp, Wp, lengths)
    q_np = per_seq_queries(w, runs, 0, lengths)
    gout, gsel, grows = run_decode(layer, w, q_np)
    reps = check_units(layer, w, Kp, Vp, Wp, lengths, q_np, gout, gsel, grows, free_exact=not bf16)
    record_all("test_cluster_load_matches_oracle",
               f"{'bf16' if bf16 else 'fp32'} d={D} G={G} b={b} lengths {'/'.join(map(str, lengths))}, clustered",
               reps)


def test_cluster_load_131k():
    """131072 tokens x 4 KV heads, b = 64, k = 16: the sort's global passes
    (524288 records) and a two-level clustering; every unit's order checked,
    the nodes and decode on sampled units."""
    L = 131072
    w = small(batch=1, n_kv_heads=4, group=4, head_dim=128, branching=64, k=16, bf16=True, length=L)
    layer, Wp, Kp, Vp, runs = _load_and_check_order(w, [L], L, seed=1)
    check_nodes(layer, w, Kp, Vp, Wp, [L], units=[(0, 2)])
    q_np = per_seq_queries(w, runs, 0, [L])
    gout, gsel, grows = run_decode(layer, w, q_np)
    reps = check_units(layer, w, Kp, Vp, Wp, [L], q_np, gout, gsel, grows, units=[(0, 0), (0, 3)])
    record_all("test_cluster_load_131k", "bf16 131072 tokens x 4 KV heads b=64 k=16, clustered", reps)


def test_cluster_load_errors():
    w = small(batch=1, n_kv_heads=1, group=4, head_dim=128, branching=8, k=3)
    K, V, _ = synth.cache_arrays(w, 64)
    layer, _ = make_layer(w, 64)
    Z = torch.from_numpy(_directions(layer, w, 2))
    with pytest.raises(RecsaError) as e:
        layer.load_clustered(parity.to_dev(K, True), parity.to_dev(V, True), [65], Z)  # longer than the source
    assert e.value.status == ERR_CAPACITY
    W = synth.workload_pooler(w)
    paged = RecsaLayer(1, 1, 4, 128, 8, 3, 64, parity.to_dev(W, True), dtype=torch.bfloat16, page_size=32,
                       num_pages=2, page_table=[[0, 1]])
    with pytest.raises(RecsaError) as e:
        paged.load_clustered(parity.to_dev(K, True), parity.to_dev(V, True), [64], Z)
    assert e.value.status == ERR_UNSUPPORTED
