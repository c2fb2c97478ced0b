"""Decode-query gradients through the C ABI against the fp64 oracle (needs a B200).

recsa_decode_backward + recsa_tree_backward give dq, every cached token's dk
and dv, and the pooler's dW for the selections the forward made. The oracle
(oracle.query_grad, pinned by finite differences and by autograd on the
dense case) runs over the GPU's stored node arrays (staged, as the forward
parity tests), with the same selections (asserted, per unit).

Tolerance: the GPU recomputes the logits and accumulates everything in fp32
(sums of at most a few thousand terms, plus atomic sums over the tree for dW),
so its relative error is of order 1e-6. Every gradient row (a query head's dq,
a token's dk or dv) must match the oracle's to 1e-3 of that row's norm plus
1e-6 of the largest row norm, and dW to 1e-4 of its norm: a dropped or
doubled term, a wrong rotation, a wrong subtree count moves rows by 1e-2 or
more.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from hierarchical_sparse_attention_tree_b200 import RecsaError
from hierarchical_sparse_attention_tree_b200 import recsa as R
from tests import parity
from tests.test_gpu_parity import make_layer, per_seq_queries, run_decode, small
from tests.test_gpu_paged import paged_layer

pytestmark = pytest.mark.gpu


def _rows_close(gpu, ref, what, rel=1e-3, floor=1e-6):
    gpu, ref = np.asarray(gpu, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    gpu2, ref2 = gpu.reshape(-1, gpu.shape[-1]), ref.reshape(-1, ref.shape[-1])
    err = np.linalg.norm(gpu2 - ref2, axis=1)
    nrm = np.linalg.norm(ref2, axis=1)
    bound = rel * nrm + floor * max(nrm.max(), 1e-30)
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, (what, int(bad.size), int(bad[0]), float(err[bad[0]]), float(nrm[bad[0]]))


def _dout(w, seed):
    return synth.plain(77, seed, (w.batch, w.n_q_heads, w.head_dim), 0.0, 1.0, w.bf16)


def _oracle_unit(layer, w, K, V, Wf, lengths, b, h, q_np, dout_np, gsel):
    """Oracle gradient of unit (b, h) over the GPU's node arrays; also checks
    that the oracle's staged descent makes the GPU's selections."""
    L = lengths[b]
    J, _ = oracle.levels(L, w.branching)
    tK, tV = parity.gpu_tree_unit(layer, b, h, J, L)
    qu = parity.q_unit(q_np, b, h, w.group)
    du = parity.q_unit(dout_np, b, h, w.group).astype(np.float64)
    ref = parity.oracle_query(tK, tV, K, V, b, h, L, qu, w)
    assert np.array_equal(ref["sel"], gsel[b, h, :J]), ("selection differs", b, h, ref["margin"])
    return oracle.query_grad(tK, tV, K[b, h], V[b, h], L, qu, du, Wf, w.head_dim, w.branching, w.k, w.group,
                             w.rope_base)


def _token_grads(layer, b, h, L):
    """Gradient rows of sequence b, KV head h, tokens [0, L) (through the page
    table when paged), as fp64 numpy [L][d]."""
    if not layer.page_size:
        return parity.to_f64(layer.dk[b, h, :L]), parity.to_f64(layer.dv[b, h, :L])
    P = layer.page_size
    pages = [int(x) for x in layer.page_table[b, :-(-L // P)].cpu()]
    dk = torch.cat([layer.dk[pg, h] for pg in pages], dim=0)[:L]
    dv = torch.cat([layer.dv[pg, h] for pg in pages], dim=0)[:L]
    return parity.to_f64(dk), parity.to_f64(dv)


def _check_layer(layer, w, K, V, Wf, lengths, queries, extra_dk=None):
    """queries: list of (q_np, dout_np, gsel, dq_gpu) already back-propagated
    into the layer; compares dq per query and the summed dk, dv, dW."""
    dW = np.zeros((w.head_dim, w.head_dim))
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            L = lengths[b]
            dK = np.zeros((L, w.head_dim))
            dV = np.zeros((L, w.head_dim))
            for q_np, dout_np, gsel, dq in queries:
                g = _oracle_unit(layer, w, K, V, Wf, lengths, b, h, q_np, dout_np, gsel)
                _rows_close(dq[b, h * w.group:(h + 1) * w.group], g["dq"], ("dq", b, h))
                dK += g["dK"]
                dV += g["dV"]
                dW += g["dW"]
            gk, gv = _token_grads(layer, b, h, L)
            _rows_close(gk, dK, ("dk", b, h))
            _rows_close(gv, dV, ("dv", b, h))
    gdw = parity.to_f64(layer.dw)
    assert np.linalg.norm(gdw - dW) <= 1e-4 * np.linalg.norm(dW) + 1e-12, (np.linalg.norm(gdw - dW),
                                                                           np.linalg.norm(dW))
    if not layer.page_size:  # rows past each sequence's length get nothing
        for b in range(w.batch):
            assert not layer.dk[b, :, lengths[b]:].any() and not layer.dv[b, :, lengths[b]:].any()


@pytest.mark.parametrize("bf16,D,G", [(True, 128, 4), (True, 64, 2), (False, 128, 8), (False, 64, 1)])
def test_decode_backward_matches_oracle(bf16, D, G):
    w = small(batch=2, n_kv_heads=2, group=G, head_dim=D, branching=8, k=3, bf16=bf16)
    lengths = [517, 3001]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp = make_layer(w, 4096)
    layer.load(parity.to_dev(K, bf16), parity.to_dev(V, bf16), lengths)
    q_np = per_seq_queries(w, runs, 0, lengths)
    _, gsel, _ = run_decode(layer, w, q_np)
    dout_np = _dout(w, 1)
    J_cap, _ = layer.tree_shape()
    layer.zero_grad()
    sel = torch.from_numpy(gsel).cuda()
    dq = layer.decode_backward(parity.to_dev(q_np, bf16), parity.to_dev(dout_np, bf16), sel)
    layer.tree_backward()
    torch.cuda.synchronize()
    layer.check()
    _check_layer(layer, w, K, V, synth.as_f32(Wp), lengths, [(q_np, dout_np, gsel, parity.to_f64(dq))])


@pytest.mark.parametrize("bf16,D,b", [(True, 128, 5), (False, 64, 12), (True, 64, 3)])
def test_backward_mixed_parents_matches_oracle(bf16, D, b):
    """Branching factors that are not multiples of the propagation's
    eight-node pass: passes whose nodes have different parents (the general
    path) next to passes under one parent (the shared path), on every level."""
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=D, branching=b, k=3, bf16=bf16)
    lengths = [777, 2050]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp = make_layer(w, 4096)
    layer.load(parity.to_dev(K, bf16), parity.to_dev(V, bf16), lengths)
    q_np = per_seq_queries(w, runs, 0, lengths)
    _, gsel, _ = run_decode(layer, w, q_np)
    dout_np = _dout(w, 2)
    layer.zero_grad()
    dq = layer.decode_backward(parity.to_dev(q_np, bf16), parity.to_dev(dout_np, bf16), torch.from_numpy(gsel).cuda())
    layer.tree_backward()
    torch.cuda.synchronize()
    layer.check()
    _check_layer(layer, w, K, V, synth.as_f32(Wp), lengths, [(q_np, dout_np, gsel, parity.to_f64(dq))])


@pytest.mark.parametrize("bf16,D", [(True, 128), (False, 64)])
def test_backward_token_sweep_alignment(bf16, D):
    """dk, dv that start 16 bytes past a 32-byte boundary (allowed by the
    ABI) take the 64/128-bit token sweep; aligned ones the 256-bit sweep.
    The two give the same dk, dv bit for bit (one add per element) and the
    same dW up to the order of the key sums; the unaligned run is also
    checked against the oracle."""
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=D, branching=8, k=3, bf16=bf16)
    lengths = [517, 3001]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp = make_layer(w, 4096)
    layer.load(parity.to_dev(K, bf16), parity.to_dev(V, bf16), lengths)
    q_np = per_seq_queries(w, runs, 0, lengths)
    _, gsel, _ = run_decode(layer, w, q_np)
    dout_np = _dout(w, 3)
    q, dout, sel = parity.to_dev(q_np, bf16), parity.to_dev(dout_np, bf16), torch.from_numpy(gsel).cuda()
    layer.zero_grad()
    layer.decode_backward(q, dout, sel)
    layer.tree_backward()
    torch.cuda.synchronize()
    layer.check()
    dk_a, dv_a, dw_a = layer.dk.clone(), layer.dv.clone(), layer.dw.clone()
    assert layer.dk.data_ptr() % 32 == 0 and layer.dv.data_ptr() % 32 == 0
    n = layer.dk.numel()
    bufs = [torch.zeros(n + 4, dtype=torch.float32, device="cuda") for _ in range(2)]
    layer.dk = bufs[0][4:].view(dk_a.shape)
    layer.dv = bufs[1][4:].view(dv_a.shape)
    assert layer.dk.data_ptr() % 32 == 16 and layer.dv.data_ptr() % 32 == 16
    layer.dw.zero_()
    dq = layer.decode_backward(q, dout, sel)
    layer.tree_backward()
    torch.cuda.synchronize()
    layer.check()
    assert torch.equal(layer.dk, dk_a) and torch.equal(layer.dv, dv_a)
    assert torch.allclose(layer.dw, dw_a, rtol=1e-5, atol=1e-6 * dw_a.abs().max().item())
    _check_layer(layer, w, K, V, synth.as_f32(Wp), lengths, [(q_np, dout_np, gsel, parity.to_f64(dq))])


def test_backward_sums_queries_and_clears_accumulators():
    """Two queries back-propagated before one tree pass give the sum of their
    gradients; a second tree pass adds nothing (the accumulators were cleared)."""
    w = small(batch=1, n_kv_heads=2, group=4, head_dim=128, branching=8, k=2)
    lengths = [2000]
    K, V, runs = synth.cache_arrays(w, 2000)
    layer, Wp = make_layer(w, 2048)
    layer.load(parity.to_dev(K, True), parity.to_dev(V, True), lengths)
    layer.zero_grad()
    qs = []
    for s in range(2):
        q_np = per_seq_queries(w, runs, s, lengths)
        _, gsel, _ = run_decode(layer, w, q_np)
        dout_np = _dout(w, 10 + s)
        dq = layer.decode_backward(parity.to_dev(q_np, True), parity.to_dev(dout_np, True),
                                   torch.from_numpy(gsel).cuda())
        qs.append((q_np, dout_np, gsel, parity.to_f64(dq)))
    layer.tree_backward()
    torch.cuda.synchronize()
    _check_layer(layer, w, K, V, synth.as_f32(Wp), lengths, qs)
    before = (layer.dk.clone(), layer.dv.clone(), layer.dw.clone())
    layer.tree_backward()
    torch.cuda.synchronize()
    assert torch.equal(before[0], layer.dk) and torch.equal(before[1], layer.dv) and torch.equal(before[2], layer.dw)
    layer.check()


@pytest.mark.parametrize("L", [1, 7, 8, 9, 64, 65, 200])
def test_backward_edge_lengths(L):
    """One token, one node, a ragged second node, exactly b^2, every level
    kept (nothing summarised: dW must be zero)."""
    w = small(batch=1, n_kv_heads=1, group=2, head_dim=64, branching=8, k=3, bf16=False)
    K, V, runs = synth.cache_arrays(w, L)
    layer, Wp = make_layer(w, 256)
    layer.load(parity.to_dev(K, False), parity.to_dev(V, False), [L])
    q_np = per_seq_queries(w, runs, 0, [L])
    _, gsel, _ = run_decode(layer, w, q_np)
    dout_np = _dout(w, 3)
    layer.zero_grad()
    dq = layer.decode_backward(parity.to_dev(q_np, False), parity.to_dev(dout_np, False),
                               torch.from_numpy(gsel).cuda())
    layer.tree_backward()
    torch.cuda.synchronize()
    layer.check()
    _check_layer(layer, w, K, V, synth.as_f32(Wp), [L], [(q_np, dout_np, gsel, parity.to_f64(dq))])
    J, n = oracle.levels(L, w.branching)
    if max(n[1:]) <= w.k:  # nothing dropped: no summary, no gradient for W
        assert not layer.dw.any()


def test_backward_paged_matches_oracle():
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=128, branching=8, k=3)
    lengths = [700, 1500]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp, _ = paged_layer(w, 2048, 64)
    layer.load(parity.to_dev(K, True), parity.to_dev(V, True), lengths)
    q_np = per_seq_queries(w, runs, 0, lengths)
    _, gsel, _ = run_decode(layer, w, q_np)
    dout_np = _dout(w, 4)
    layer.zero_grad()
    dq = layer.decode_backward(parity.to_dev(q_np, True), parity.to_dev(dout_np, True), torch.from_numpy(gsel).cuda())
    layer.tree_backward()
    torch.cuda.synchronize()
    layer.check()
    _check_layer(layer, w, K, V, synth.as_f32(Wp), lengths, [(q_np, dout_np, gsel, parity.to_f64(dq))])


def test_backward_rejects_bad_selections():
    """Selections that are not a valid descent are flagged in the device
    error word; that unit gets a zero dq and adds nothing; others are exact."""
    w = small(batch=2, n_kv_heads=1, group=4, head_dim=128, branching=8, k=3)
    lengths = [900, 900]
    K, V, runs = synth.cache_arrays(w, 900)
    layer, Wp = make_layer(w, 1024)
    layer.load(parity.to_dev(K, True), parity.to_dev(V, True), lengths)
    q_np = per_seq_queries(w, runs, 0, lengths)
    _, gsel, _ = run_decode(layer, w, q_np)
    bad = gsel.copy()
    bad[1, 0, 0, :] = bad[1, 0, 0, ::-1]  # level-1 selections out of order
    layer.zero_grad()
    dq = layer.decode_backward(parity.to_dev(q_np, True), parity.to_dev(_dout(w, 5), True),
                               torch.from_numpy(bad).cuda())
    layer.tree_backward()
    with pytest.raises(RecsaError) as e:
        layer.check()
    assert e.value.status == R.ERR_DEVICE
    assert not dq[1].any() and not layer.dk[1].any() and not layer.dv[1].any()
    assert dq[0].abs().sum() > 0
    with pytest.raises(RecsaError):
        layer.ctx.decode_backward(parity.to_dev(q_np, True), parity.to_dev(_dout(w, 5), True),
                                  torch.from_numpy(gsel).cuda(), dq, layer.dk, layer.dv, layer._bwd_scratch[:256])
