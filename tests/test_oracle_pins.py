"""Pins of the fp64 oracle against what the pages and mathematics fix.

Method pages: "Recursive Sparse Attention" (arXiv 2611.07232) abstract, and
the kongchang.com RecSA article ("Core Idea", "Position Encoding").
Each test targets a plausible mistake in the oracle: a wrong RoPE sign or
index, a transposed pooler, a dropped or double-counted entry, a wrong node
range, a wrong query position.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import brute_recsa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F64 = oracle.STORE_F64


def _rand(seed, shape, scale=1.0):
    return synth.plain(123, seed, shape, 0.0, scale).astype(np.float32)


def _dense_numpy(K, V, q, base):
    """Textbook causal RoPE attention of the last position over all tokens,
    written with explicit 2x2 rotation blocks per pair (i, i+d/2)."""
    T, d = K.shape
    h = d // 2
    inv = np.array([base ** (-2.0 * i / d) for i in range(h)])

    def rot(x, p):
        c, s = np.cos(p * inv), np.sin(p * inv)
        return np.concatenate([x[:h] * c - x[h:] * s, x[h:] * c + x[:h] * s])

    out = []
    for g in range(q.shape[0]):
        qr = rot(q[g].astype(np.float64), T - 1)
        lg = np.array([qr @ rot(K[t].astype(np.float64), t) for t in range(T)]) / math.sqrt(d)
        w = np.exp(lg - lg.max())
        out.append((w / w.sum()) @ V.astype(np.float64))
    return np.array(out)


def _dense_sdpa(K, V, q, base):
    """torch SDPA (float64, CPU) on keys/queries rotated with torch.polar."""
    T, d = K.shape
    h = d // 2
    theta = base ** (-torch.arange(h, dtype=torch.float64) * 2 / d)

    def rot(x, pos):
        z = torch.complex(x[..., :h], x[..., h:])
        z = z * torch.polar(torch.ones_like(pos[:, None] * theta), pos[:, None] * theta)
        return torch.cat([z.real, z.imag], dim=-1)

    Kt = torch.from_numpy(K.astype(np.float64))
    Vt = torch.from_numpy(V.astype(np.float64))
    qt = torch.from_numpy(q.astype(np.float64))
    kr = rot(Kt, torch.arange(T, dtype=torch.float64))
    qr = rot(qt, torch.full((q.shape[0],), float(T - 1), dtype=torch.float64))
    o = torch.nn.functional.scaled_dot_product_attention(qr[:, None, :], kr[None].expand(q.shape[0], T, d),
                                                         Vt[None].expand(q.shape[0], T, d))
    return o[:, 0, :].numpy()


# ---------------------------------------------------------------- levels

@pytest.mark.parametrize("T,b,expect", [
    (4096, 16, [4096, 256, 16]),            # the tiny fp32 workload's shape
    (131072, 64, [131072, 2048, 32]),
    (524288, 64, [524288, 8192, 128, 2]),
    (2097152, 64, [2097152, 32768, 512, 8]),
    (1, 4, [1, 1]), (4, 4, [4, 1]), (5, 4, [5, 2]), (17, 4, [17, 5, 2]),
])
def test_levels(T, b, expect):
    J, n = oracle.levels(T, b)
    assert n == expect and J == len(expect) - 1


# ----------------------------------------------------------- hand cases

def test_hand_examples():
    cases = json.load(open(os.path.join(GOLDEN, "hand_examples.json")))["cases"]
    s1, r2 = math.sin(1.0), math.sqrt(2.0)
    expected = {
        "identity_pooler_sign": (np.exp(-s1 / r2) * np.array([0.5, 0.5]) + np.exp(0.25 / r2) * np.array([2, -1]))
        / (np.exp(-s1 / r2) + np.exp(0.25 / r2)),
        "nonsymmetric_pooler": (np.exp(-s1 / r2) * np.array([0.5, 0.5]) + np.array([2, -1]))
        / (np.exp(-s1 / r2) + 1.0),
    }
    for c in cases:
        K = np.array(c["K"], dtype=np.float32)
        V = np.array(c["V"], dtype=np.float32)
        W = np.array(c["W"], dtype=np.float32)
        q = np.array(c["q"], dtype=np.float32)
        tree = oracle.build_tree(K, V, 3, 2, 2, W, F64)
        r = oracle.query_tree(tree, K, V, q, k=1, G=1, rope_base=1e6)
        assert r["J"] == 1
        assert list(r["sel"][0]) == c["selected_level1"], c["name"]
        np.testing.assert_allclose(r["out"][0], expected[c["name"]], rtol=0, atol=1e-14)


# ------------------------------------------------- (a) dense equivalence

@pytest.mark.parametrize("T,b", [(1, 2), (7, 2), (64, 2), (64, 16), (7, 16), (300, 3), (4096, 16)])
def test_dense_equivalence(T, b):
    """With k >= every level's size nothing is dropped: every candidate index
    equals its token position and the output is dense causal RoPE attention."""
    d, G, base = 16, 2, 1e4
    K, V, q = _rand(1, (T, d)), _rand(2, (T, d)), _rand(3, (G, d))
    W = _rand(4, (d, d), 1 / math.sqrt(d))
    J, n = oracle.levels(T, b)
    k = max(n[1:])
    tree = oracle.build_tree(K, V, T, d, b, W, F64)
    r = oracle.query_tree(tree, K, V, q, k=k, G=G, rope_base=base)
    assert r["v_rows"] == T and all((m == np.inf) for m in r["margin"])
    ref_np = _dense_numpy(K, V, q, base)
    ref_sdpa = _dense_sdpa(K, V, q, base)
    np.testing.assert_allclose(r["out"], ref_np, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["out"], ref_sdpa, rtol=0, atol=1e-12)


def test_dense_equivalence_prefill_first_chunk():
    """A chunk with no tree before it is plain causal attention over the chunk."""
    d, G, base, C = 16, 2, 1e6, 40
    K, V, q = _rand(5, (C, d)), _rand(6, (C, d)), _rand(7, (C, G, d))
    for t in (0, 1, 17, C - 1):
        r = oracle.query([None], [None], K[:0], V[:0], 0, q[t], d, 4, 2, G, base, Kloc=K[:t + 1], Vloc=V[:t + 1])
        np.testing.assert_allclose(r["out"], _dense_numpy(K[:t + 1], V[:t + 1], q[t], base), atol=1e-12)


# ----------------------------------------------- (b) exact subtree means

@pytest.mark.parametrize("T,b", [(1, 2), (100, 3), (4096, 16), (1000, 7)])
def test_subtree_means(T, b):
    d = 8
    K, V = _rand(8, (T, d)), _rand(9, (T, d))
    W = _rand(10, (d, d))
    tree = oracle.build_tree(K, V, T, d, b, W, F64)
    J, n = oracle.levels(T, b)
    for j in range(1, J + 1):
        span = b ** j
        for m in range(n[j]):
            lo, hi = m * span, min((m + 1) * span, T)
            np.testing.assert_allclose(tree.V[j][m], V[lo:hi].astype(np.float64).mean(0), rtol=1e-12, atol=1e-13)


def test_storage_rounding():
    """Nearest-even to bf16 and fp32 at the points where nodes are stored."""
    vals = [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1.0 + 2 ** -9, 3.0 + 2 ** -7 + 2 ** -30]
    want = [1.0, 1 + 2 ** -6, -1.0, 1.0, 3.0 + 2 ** -6]
    for v, w in zip(vals, want):
        assert oracle.round_store(v, oracle.STORE_BF16) == w
    x = _rand(11, (2000,)).astype(np.float64) * 3.7
    x = x + 1e-3 * _rand(12, (2000,))
    got = np.array([oracle.round_store(v, oracle.STORE_BF16) for v in x])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert (got == ref).all()
    got32 = np.array([oracle.round_store(v, oracle.STORE_F32) for v in x])
    assert (got32 == x.astype(np.float32).astype(np.float64)).all()


def test_stored_nodes_rounded_once():
    """bf16 storage: values are the rounded exact means; keys are W times the
    mean of the rounded child keys, then rounded."""
    T, b, d = 70, 4, 8
    K, V = _rand(13, (T, d)), _rand(14, (T, d))
    W = _rand(15, (d, d))
    t64 = oracle.build_tree(K, V, T, d, b, W, F64)
    t16 = oracle.build_tree(K, V, T, d, b, W, oracle.STORE_BF16)
    J, n = oracle.levels(T, b)
    rb = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64)).to(torch.bfloat16).double().numpy()  # noqa
    for j in range(1, J + 1):
        np.testing.assert_array_equal(t16.V[j][:n[j]], rb(t64.V[j][:n[j]]))
        below = K.astype(np.float64) if j == 1 else t16.K[j - 1]
        for m in range(n[j]):
            mean = below[m * b:min((m + 1) * b, n[j - 1])].mean(0)
            np.testing.assert_array_equal(t16.K[j][m], rb(W.astype(np.float64) @ mean))


# --------------------------------------------------------- (c) read bound

@pytest.mark.parametrize("T,b,k", [(4096, 16, 4), (5000, 8, 3), (20000, 4, 2), (999, 10, 5), (65, 64, 16)])
def test_read_bound(T, b, k):
    d, G = 8, 2
    K, V = _rand(16, (T, d)), _rand(17, (T, d))
    W = _rand(18, (d, d))
    tree = oracle.build_tree(K, V, T, d, b, W, F64)
    J, n = oracle.levels(T, b)
    depth = J + 1
    for s in range(4):
        q = _rand(100 + s, (G, d), 2.0)
        r = oracle.query_tree(tree, K, V, q, k=k, G=G, rope_base=1e6)
        assert r["k_rows"] <= k * b * depth and r["v_rows"] <= k * b * depth
        # every candidate beyond the first k per level is a summary; tokens all enter
        assert r["k_rows"] == r["v_rows"] + sum(len([x for x in row if x >= 0]) for row in r["sel"])
    D = 1
    while b ** D < T:
        D += 1
    assert depth == max(2, D)


# ------------------------------------------------------- (d) brute force

def _case(L, b, k, G, d, seed, nloc=0):
    K, V = _rand(seed, (L + nloc, d)), _rand(seed + 1, (L + nloc, d))
    W = _rand(seed + 2, (d, d), 1 / math.sqrt(d))
    q = _rand(seed + 3, (G, d), 1.5)
    return K, V, W, q


@pytest.mark.parametrize("b,k,G", list(itertools.product([2, 3, 4], [1, 2, 3], [1, 2])))
def test_brute_force_sweep(b, k, G):
    d, base = 8, 1e3
    skipped = 0
    for L in range(1, 81):
        K, V, W, q = _case(L, b, k, G, d, 1000 * b + 100 * k + 10 * G + L)
        levels = brute_recsa.build(K[:L], V[:L], W, b)
        if brute_recsa.min_margin(levels, q, k, base) < 1e-9:
            skipped += 1
            continue
        want, picked = brute_recsa.query(levels, q, k, base)
        tree = oracle.build_tree(K, V, L, d, b, W, F64)
        r = oracle.query_tree(tree, K, V, q, k=k, G=G, rope_base=base)
        np.testing.assert_allclose(r["out"], want, rtol=0, atol=1e-12, err_msg=f"L={L}")
        assert r["J"] == len(levels) - 1
        # selected sets, top level first, as token ranges
        for j, rng in zip(range(r["J"], 0, -1), picked):
            ids = [x for x in r["sel"][j - 1] if x >= 0]
            assert [(m * b ** j, min((m + 1) * b ** j, L)) for m in ids] == rng
    assert skipped <= 2


@pytest.mark.parametrize("b,k", [(2, 1), (3, 2), (4, 3)])
def test_brute_force_prefill(b, k):
    """Tree over [0, s) plus the chunk's causal tokens after the level-0 list."""
    d, G, base = 8, 2, 1e3
    for s, nloc in [(0, 5), (1, 3), (9, 4), (40, 7), (77, 1)]:
        K, V, W, q = _case(s, b, k, G, d, 7 * s + nloc + b, nloc=nloc)
        local = [(K[s + i], V[s + i]) for i in range(nloc)]
        if s:
            levels = brute_recsa.build(K[:s], V[:s], W, b)
            if brute_recsa.min_margin(levels, q, k, base) < 1e-9:
                continue
            want, _ = brute_recsa.query(levels, q, k, base, local=local)
            tree = oracle.build_tree(K, V, s, d, b, W, F64)
            r = oracle.query_tree(tree, K, V, q, k=k, G=G, rope_base=base, Kloc=K[s:], Vloc=V[s:])
        else:
            want = _dense_numpy(K[:nloc], V[:nloc], q, base)
            r = oracle.query([None], [None], K[:0], V[:0], 0, q, d, b, k, G, base, Kloc=K, Vloc=V)
        np.testing.assert_allclose(r["out"], want, rtol=0, atol=1e-12)


# ------------------------------------------------------ (e) invariants

def test_constant_values():
    T, b, k, d, G = 3000, 8, 3, 8, 4
    K = _rand(20, (T, d))
    V = np.tile(np.linspace(-1, 1, d, dtype=np.float32), (T, 1))
    W = _rand(21, (d, d))
    tree = oracle.build_tree(K, V, T, d, b, W, F64)
    r = oracle.query_tree(tree, K, V, _rand(22, (G, d)), k=k, G=G, rope_base=1e6)
    np.testing.assert_allclose(r["out"], np.tile(V[0], (G, 1)), atol=1e-12)


def test_gqa_sum_selection():
    """Selection ranks by the sum of the group's logits: duplicating one head
    G times gives the single-head result for every head."""
    T, b, k, d = 2000, 8, 2, 8
    K, V, W = _rand(23, (T, d)), _rand(24, (T, d)), _rand(25, (d, d))
    q1 = _rand(26, (1, d), 2.0)
    tree = oracle.build_tree(K, V, T, d, b, W, F64)
    r1 = oracle.query_tree(tree, K, V, q1, k=k, G=1, rope_base=1e6)
    r3 = oracle.query_tree(tree, K, V, np.repeat(q1, 3, 0), k=k, G=3, rope_base=1e6)
    np.testing.assert_allclose(r3["out"], np.repeat(r1["out"], 3, 0), atol=1e-12)
    assert (r3["sel"] == r1["sel"]).all()


@pytest.mark.parametrize("storage", [oracle.STORE_F32, oracle.STORE_BF16])
def test_refresh_equals_rebuild(storage):
    """Adding tokens and refreshing the affected nodes equals a full build."""
    T0, b, d = 1000, 8, 8
    K, V, W = _rand(27, (5000, d)), _rand(28, (5000, d)), _rand(29, (d, d))
    cap = 5000
    inc = oracle.Tree(d, b, cap, storage).build(K, V, T0, W)
    for T in [1001, 1002, 1024, 1025, 4095, 4096, 4097, 5000]:
        inc.build(K, V, T, W, t_from=inc.T)
        full = oracle.Tree(d, b, cap, storage).build(K, V, T, W)
        J, n = oracle.levels(T, b)
        for j in range(1, inc.J_keep + 1):
            m = -(-T // b ** j)
            np.testing.assert_array_equal(inc.K[j][:m], full.K[j][:m])
            np.testing.assert_array_equal(inc.V[j][:m], full.V[j][:m])


def test_decode_equals_chunk_form_when_nothing_dropped():
    """With k covering every level, the decode descent and the prefill form
    (the same rows as a chunk's causal tokens after an empty tree) both put
    every token at its own position, so they agree."""
    d, G, b, k = 8, 2, 4, 64
    K, V, q = _rand(30, (50, d)), _rand(31, (50, d)), _rand(32, (G, d))
    W = _rand(33, (d, d))
    tree = oracle.build_tree(K, V, 50, d, b, W, F64)
    dec = oracle.query_tree(tree, K, V, q, k=k, G=G, rope_base=1e6)
    pre = oracle.query([None], [None], K[:0], V[:0], 0, q, d, b, k, G, 1e6, Kloc=K, Vloc=V)
    np.testing.assert_allclose(dec["out"], pre["out"], atol=1e-12)


def test_pool_level_matches_build():
    """Pooling a level from given child keys reproduces the build's keys."""
    T, b, d = 700, 5, 8
    K, V, W = _rand(34, (T, d)), _rand(35, (T, d)), _rand(36, (d, d))
    for storage in (F64, oracle.STORE_BF16):
        tree = oracle.build_tree(K, V, T, d, b, W, storage)
        J, n = oracle.levels(T, b)
        np.testing.assert_array_equal(oracle.pool_level(K.astype(np.float64), b, W, storage), tree.K[1][:n[1]])
        for j in range(2, J + 1):
            np.testing.assert_array_equal(oracle.pool_level(tree.K[j - 1][:n[j - 1]], b, W, storage),
                                          tree.K[j][:n[j]])
