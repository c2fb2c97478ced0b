"""Pins of the oracle's decode-query gradient (oracle.query_grad).

Method pages: "Recursive Sparse Attention" (arXiv 2611.07232) abstract (the
tree of means, the pooled keys, unselected candidates as summaries) and the
kongchang.com RecSA article ("Core Idea", "Position Encoding"). The selection
is a discrete choice, so the gradient is the one of the output with the
selections held fixed; node storage in fp64 makes rounding the identity.

Pins, each independent of the gradient code:
  * central finite differences of the oracle's own forward (tree rebuilt from
    perturbed tokens / pooler, query repeated) along random directions in
    every input and along single coordinates, at shapes where summaries of
    several levels, ragged last nodes and direct tokens all take part;
  * with nothing dropped the output is dense causal RoPE attention, whose
    gradient torch autograd gives (and the pooler gets none);
  * a single token (the whole cache is one exact entry) reduces to the
    same dense check with T = 1.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

F64 = oracle.STORE_F64


def _rand(seed, shape, scale=1.0):
    return synth.plain(321, seed, shape, 0.0, scale).astype(np.float32)


def _forward(K, V, W, q, T, d, b, k, G, base):
    tree = oracle.build_tree(K, V, T, d, b, W, F64)
    r = oracle.query_tree(tree, K, V, q, k=k, G=G, rope_base=base)
    return r["out"], r["sel"], tree, r


def _grad(K, V, W, q, dout, T, d, b, k, G, base):
    tree = oracle.build_tree(K, V, T, d, b, W, F64)
    return oracle.query_grad(tree.K, tree.V, K, V, T, q, dout, W, d, b, k, G, base)


def _step(x, u, h):
    """x + h u and x - h u as float32 arrays, with the steps really taken
    (float32 rounding of the shifted inputs is measured, not assumed)."""
    xp = (x.astype(np.float64) + h * u).astype(np.float32)
    xm = (x.astype(np.float64) - h * u).astype(np.float32)
    return xp, xm, xp.astype(np.float64) - xm.astype(np.float64)


CASES = [  # T, b, k, G, d
    (37, 4, 1, 1, 8),     # J = 3, ragged nodes at every level
    (300, 4, 2, 3, 8),    # J = 4, several summaries per level
    (130, 5, 2, 2, 16),   # b not a power of two
    (9, 2, 1, 2, 4),      # deep binary tree
]


@pytest.mark.parametrize("T,b,k,G,d", CASES)
@pytest.mark.parametrize("which", ["K", "V", "W", "q"])
def test_directional_finite_difference(T, b, k, G, d, which):
    base = 100.0
    K, V, q = _rand(1, (T, d)), _rand(2, (T, d)), _rand(3, (G, d))
    W = _rand(4, (d, d), 1.3 / math.sqrt(d))
    dout = _rand(5, (G, d)).astype(np.float64)
    args = dict(K=K, V=V, W=W, q=q)
    out, sel, _, r = _forward(K, V, W, q, T, d, b, k, G, base)
    assert np.all(r["margin"] > 1e-3), "pick inputs without a near tie"
    g = _grad(K, V, W, q, dout, T, d, b, k, G, base)
    grads = dict(K=g["dK"], V=g["dV"], W=g["dW"], q=g["dq"])
    rng = np.random.default_rng(hash((T, b, k, G, d, which)) % 2**32)
    u = rng.standard_normal(args[which].shape)
    xp, xm, delta = _step(args[which], u, 1e-3)
    fp = _forward(**{**args, which: xp}, T=T, d=d, b=b, k=k, G=G, base=base)
    fm = _forward(**{**args, which: xm}, T=T, d=d, b=b, k=k, G=G, base=base)
    assert np.array_equal(fp[1], sel) and np.array_equal(fm[1], sel), "the step changed a selection"
    fd = float(np.sum(dout * (fp[0] - fm[0])))
    an = float(np.sum(grads[which] * delta))
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, fd, an)


def test_coordinate_finite_difference():
    """Single coordinates: a token under an unselected node (reached only
    through summaries), a token read directly, the pooler's corners, one
    query coordinate of the second head."""
    T, b, k, G, d, base = 300, 4, 2, 3, 8, 100.0
    K, V, q = _rand(1, (T, d)), _rand(2, (T, d)), _rand(3, (G, d))
    W = _rand(4, (d, d), 1.3 / math.sqrt(d))
    dout = _rand(5, (G, d)).astype(np.float64)
    _, sel, _, r = _forward(K, V, W, q, T, d, b, k, G, base)
    g = _grad(K, V, W, q, dout, T, d, b, k, G, base)
    # first token whose level-1 node was not selected (reached through summaries only)
    t_sum = next(t for t in range(T) if t // b not in sel[0])
    lo = sel[0][0] * b
    t_direct = lo  # first token under the first selected level-1 node
    picks = [("K", (t_sum, 1)), ("V", (t_sum, 2)), ("K", (t_direct, 0)), ("V", (t_direct, 5)),
             ("W", (0, 0)), ("W", (d - 1, 2)), ("q", (1, 3))]
    grads = dict(K=g["dK"], V=g["dV"], W=g["dW"], q=g["dq"])
    args = dict(K=K, V=V, W=W, q=q)
    for which, idx in picks:
        u = np.zeros(args[which].shape)
        u[idx] = 1.0
        xp, xm, delta = _step(args[which], u, 2e-3)
        fp = _forward(**{**args, which: xp}, T=T, d=d, b=b, k=k, G=G, base=base)
        fm = _forward(**{**args, which: xm}, T=T, d=d, b=b, k=k, G=G, base=base)
        fd = float(np.sum(dout * (fp[0] - fm[0]))) / delta[idx]
        assert abs(fd - grads[which][idx]) <= 1e-6 * max(1.0, abs(fd)), (which, idx, fd, grads[which][idx])
    # summaries reach the first token: its key gradient is not zero
    assert np.abs(g["dK"][t_sum]).max() > 0 and np.abs(g["dV"][t_sum]).max() > 0


def _dense_torch_grads(K, V, q, dout, base):
    """torch autograd through dense causal RoPE attention of the last
    position (rotations written as complex multiplications)."""
    T, d = K.shape
    h = d // 2
    theta = base ** (-torch.arange(h, dtype=torch.float64) * 2 / d)
    Kt = torch.tensor(K, dtype=torch.float64, requires_grad=True)
    Vt = torch.tensor(V, dtype=torch.float64, requires_grad=True)
    qt = torch.tensor(q, dtype=torch.float64, requires_grad=True)

    def rot(x, pos):
        z = torch.complex(x[..., :h], x[..., h:]) * torch.polar(torch.ones(len(pos), h, dtype=torch.float64),
                                                                 pos[:, None] * theta)
        return torch.cat([z.real, z.imag], dim=-1)

    kr = rot(Kt, torch.arange(T, dtype=torch.float64))
    qr = rot(qt, torch.full((q.shape[0],), float(T - 1), dtype=torch.float64))
    p = torch.softmax(qr @ kr.T / math.sqrt(d), dim=-1)
    out = p @ Vt
    (out * torch.tensor(dout)).sum().backward()
    return Kt.grad.numpy(), Vt.grad.numpy(), qt.grad.numpy()


@pytest.mark.parametrize("T,b", [(1, 2), (7, 2), (64, 4), (200, 16)])
def test_dense_equivalence(T, b):
    d, G, base = 16, 2, 1e4
    K, V, q = _rand(11, (T, d)), _rand(12, (T, d)), _rand(13, (G, d))
    W = _rand(14, (d, d), 1 / math.sqrt(d))
    dout = _rand(15, (G, d)).astype(np.float64)
    J, n = oracle.levels(T, b)
    g = _grad(K, V, W, q, dout, T, d, b, max(n[1:]), G, base)
    dK, dV, dq = _dense_torch_grads(K, V, q, dout, base)
    np.testing.assert_allclose(g["dK"], dK, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dV"], dV, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dq"], dq, rtol=0, atol=1e-12)
    assert not g["dW"].any()


def test_gradient_linear_in_dout():
    """Every gradient is linear in the output gradient."""
    T, b, k, G, d, base = 37, 4, 1, 1, 8, 100.0
    K, V, q = _rand(1, (T, d)), _rand(2, (T, d)), _rand(3, (G, d))
    W = _rand(4, (d, d), 1.3 / math.sqrt(d))
    dout = _rand(5, (G, d)).astype(np.float64)
    g1 = _grad(K, V, W, q, dout, T, d, b, k, G, base)
    g2 = _grad(K, V, W, q, 2 * dout, T, d, b, k, G, base)
    for key in ("dK", "dV", "dW", "dq"):
        np.testing.assert_allclose(g2[key], 2 * g1[key], rtol=1e-13, atol=1e-15)


# ------------------------------------------------------- prefill queries
# A prefill query of a chunk sees the tree over the tokens before the chunk
# plus the chunk's own causal tokens, which follow the level-0 candidates in
# the index order (reading R9); the gradient reaches those local tokens too.


def _forward_local(K, V, W, q, Kl, Vl, T, d, b, k, G, base):
    if T > 0:
        tree = oracle.build_tree(K, V, T, d, b, W, F64)
        r = oracle.query(tree.K, tree.V, K, V, T, q, d, b, k, G, base, Kloc=Kl, Vloc=Vl)
    else:
        r = oracle.query([None], [None], K, V, 0, q, d, b, k, G, base, Kloc=Kl, Vloc=Vl)
    return r["out"], r["sel"], r


def _grad_local(K, V, W, q, Kl, Vl, dout, T, d, b, k, G, base):
    if T > 0:
        tree = oracle.build_tree(K, V, T, d, b, W, F64)
        tK, tV = tree.K, tree.V
    else:
        tK = tV = [None]
    return oracle.query_grad(tK, tV, K, V, T, q, dout, W, d, b, k, G, base, Kloc=Kl, Vloc=Vl)


LOCAL_CASES = [  # T, nloc, b, k, G, d
    (37, 5, 4, 1, 1, 8),
    (300, 9, 4, 2, 3, 8),
    (130, 4, 5, 2, 2, 16),
    (0, 7, 4, 2, 2, 8),   # the first chunk: no tree, the chunk's causal tokens only
]


@pytest.mark.parametrize("T,nloc,b,k,G,d", LOCAL_CASES)
@pytest.mark.parametrize("which", ["K", "V", "W", "q", "Kl", "Vl"])
def test_prefill_directional_finite_difference(T, nloc, b, k, G, d, which):
    if T == 0 and which in ("K", "V", "W"):
        pytest.skip("no tree: nothing depends on these")
    base = 100.0
    K, V = _rand(21, (max(T, 1), d)), _rand(22, (max(T, 1), d))
    Kl, Vl, q = _rand(23, (nloc, d)), _rand(24, (nloc, d)), _rand(25, (G, d))
    W = _rand(26, (d, d), 1.3 / math.sqrt(d))
    dout = _rand(27, (G, d)).astype(np.float64)
    args = dict(K=K, V=V, W=W, q=q, Kl=Kl, Vl=Vl)
    out, sel, r = _forward_local(**args, T=T, d=d, b=b, k=k, G=G, base=base)
    assert np.all(r["margin"] > 1e-3), "pick inputs without a near tie"
    g = _grad_local(**args, dout=dout, T=T, d=d, b=b, k=k, G=G, base=base)
    grads = dict(K=g["dK"], V=g["dV"], W=g["dW"], q=g["dq"], Kl=g["dKloc"], Vl=g["dVloc"])
    rng = np.random.default_rng(hash((T, nloc, b, k, G, d, which)) % 2**32)
    u = rng.standard_normal(args[which].shape)
    if which in ("K", "V"):
        u[T:] = 0.0
    xp, xm, delta = _step(args[which], u, 1e-3)
    fp = _forward_local(**{**args, which: xp}, T=T, d=d, b=b, k=k, G=G, base=base)
    fm = _forward_local(**{**args, which: xm}, T=T, d=d, b=b, k=k, G=G, base=base)
    assert np.array_equal(fp[1], sel) and np.array_equal(fm[1], sel), "the step changed a selection"
    fd = float(np.sum(dout * (fp[0] - fm[0])))
    an = float(np.sum(grads[which] * delta[:grads[which].shape[0]]))
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, fd, an)


@pytest.mark.parametrize("T,nloc,b", [(0, 1, 2), (0, 12, 4), (50, 7, 4), (200, 33, 16)])
def test_prefill_dense_equivalence(T, nloc, b):
    """Nothing dropped (k at least every level's size): the prefill query is
    dense causal RoPE attention over the tokens before the chunk followed by
    the chunk's own tokens, so its gradients are torch autograd's of that, and
    the pooler gets none."""
    d, G, base = 16, 2, 1e4
    K, V = _rand(31, (max(T, 1), d)), _rand(32, (max(T, 1), d))
    Kl, Vl, q = _rand(33, (nloc, d)), _rand(34, (nloc, d)), _rand(35, (G, d))
    W = _rand(36, (d, d), 1 / math.sqrt(d))
    dout = _rand(37, (G, d)).astype(np.float64)
    kmax = max(oracle.levels(T, b)[1][1:]) if T > 0 else 1
    g = _grad_local(K, V, W, q, Kl, Vl, dout, T, d, b, kmax, G, base)
    dK, dV, dq = _dense_torch_grads(np.concatenate([K[:T], Kl]), np.concatenate([V[:T], Vl]), q, dout, base)
    np.testing.assert_allclose(g["dK"], dK[:T], rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dV"], dV[:T], rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dKloc"], dK[T:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dVloc"], dV[T:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dq"], dq, rtol=0, atol=1e-12)
    assert not g["dW"].any()


def test_prefill_chunk_gradient_is_dense_causal():
    """A whole chunk: query i of the chunk sees the tree over the T earlier
    tokens and the chunk's tokens 0..i. With nothing dropped, the gradients
    summed over the chunk's queries are torch autograd's of dense causal RoPE
    attention of the chunk's queries over all T + C tokens."""
    T, C, b, d, G, base = 50, 6, 4, 16, 2, 1e4
    K, V = _rand(41, (T, d)), _rand(42, (T, d))
    Kc, Vc = _rand(43, (C, d)), _rand(44, (C, d))
    Q = _rand(45, (C, G, d))
    W = _rand(46, (d, d), 1 / math.sqrt(d))
    dO = _rand(47, (C, G, d)).astype(np.float64)
    kmax = max(oracle.levels(T, b)[1][1:])
    dK, dV, dKc, dVc = np.zeros((T, d)), np.zeros((T, d)), np.zeros((C, d)), np.zeros((C, d))
    dQ = np.zeros((C, G, d))
    for i in range(C):
        g = _grad_local(K, V, W, Q[i], Kc[:i + 1], Vc[:i + 1], dO[i], T, d, b, kmax, G, base)
        dK += g["dK"]
        dV += g["dV"]
        dKc[:i + 1] += g["dKloc"]
        dVc[:i + 1] += g["dVloc"]
        dQ[i] = g["dq"]
        assert not g["dW"].any()
    # dense causal attention of the chunk's queries (positions T .. T + C - 1)
    h = d // 2
    theta = base ** (-torch.arange(h, dtype=torch.float64) * 2 / d)
    X = torch.tensor(np.concatenate([K, Kc]), dtype=torch.float64, requires_grad=True)
    Y = torch.tensor(np.concatenate([V, Vc]), dtype=torch.float64, requires_grad=True)
    Qt = torch.tensor(Q, dtype=torch.float64, requires_grad=True)

    def rot(x, pos):
        z = torch.complex(x[..., :h], x[..., h:]) * torch.polar(torch.ones_like(pos[..., None] * theta),
                                                                 pos[..., None] * theta)
        return torch.cat([z.real, z.imag], dim=-1)

    n = T + C
    kr = rot(X, torch.arange(n, dtype=torch.float64))
    pos_q = (T + torch.arange(C, dtype=torch.float64))[:, None].expand(C, G)
    qr = rot(Qt, pos_q)
    s = torch.einsum("cgd,nd->cgn", qr, kr) / math.sqrt(d)
    mask = torch.arange(n)[None, :] > (T + torch.arange(C))[:, None]
    s = s.masked_fill(mask[:, None, :], float("-inf"))
    out = torch.einsum("cgn,nd->cgd", torch.softmax(s, dim=-1), Y)
    (out * torch.tensor(dO)).sum().backward()
    np.testing.assert_allclose(dK, X.grad[:T].numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dV, Y.grad[:T].numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dKc, X.grad[T:].numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dVc, Y.grad[T:].numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dQ, Qt.grad.numpy(), rtol=0, atol=1e-12)
