"""Brute-force RecSA reference for tiny inputs (pins the oracle; tests only).

Written independently of the oracle: the tree is built by explicit
recursion, grouping each level's node objects b at a time and carrying the
token range of every node; there is no node-index arithmetic. RoPE is written
with complex numbers (each pair (x_i, x_{i+d/2}) is one complex coordinate
rotated by e^{i p theta_i}), and the descent sorts Python objects.

Method: "Recursive Sparse Attention" (arXiv 2611.07232) abstract; the
kongchang.com article on RecSA, "Core Idea" and "Position Encoding". The same
readings of open points as the oracle (top level = first level with at most
b nodes, query at position n-1 among n candidates, ties to the earlier node).
"""
from __future__ import annotations

import numpy as np


class Node:
    __slots__ = ("lo", "hi", "children", "key", "value")

    def __init__(self, lo, hi, children, key, value):
        self.lo, self.hi, self.children, self.key, self.value = lo, hi, children, key, value


def build(K, V, W, b):
    """Levels of Node objects, bottom (tokens) first."""
    level = [Node(t, t + 1, [], K[t].astype(np.float64), V[t].astype(np.float64)) for t in range(len(K))]
    levels = [level]
    while True:
        parents = []
        for start in range(0, len(level), b):
            group = level[start:start + b]
            lo, hi = group[0].lo, group[-1].hi
            value = np.mean(np.asarray(V[lo:hi], dtype=np.float64), axis=0)
            key = np.asarray(W, dtype=np.float64) @ np.mean([c.key for c in group], axis=0)
            parents.append(Node(lo, hi, group, key, value))
        levels.append(parents)
        level = parents
        if len(level) <= b:
            return levels


def _rot(x, p, base):
    d = len(x)
    h = d // 2
    theta = base ** (-(np.arange(h) * 2.0) / d)
    return (x[:h] + 1j * x[h:]) * np.exp(1j * p * theta)


def _dot(u, v):
    return float(np.real(np.sum(np.conj(u) * v)))


def query(levels, q, k, base, local=None):
    """q: [G][d]. local: optional list of (key, value) rows appended after the
    level-0 candidates. Returns (out [G][d], [selected lo-sorted token ranges
    per level, top first])."""
    G, d = q.shape
    scale = 1.0 / np.sqrt(d)
    entries = []  # (logits[G], value)
    chosen_log = []
    cands = list(levels[-1])
    for _lev in range(len(levels) - 1, 0, -1):
        P = len(cands) - 1
        qr = [_rot(q[g].astype(np.float64), P, base) for g in range(G)]
        scored = []
        for i, node in enumerate(cands):
            kr = _rot(node.key, i, base)
            lg = [_dot(qr[g], kr) * scale for g in range(G)]
            scored.append((sum(lg), node, lg))
        ranked = sorted(scored, key=lambda s: (-s[0], s[1].lo))
        keep = ranked[:min(k, len(ranked))]
        keep_ids = {id(s[1]) for s in keep}
        for s in scored:
            if id(s[1]) not in keep_ids:
                entries.append((s[2], s[1].value))
        picked = sorted((s[1] for s in keep), key=lambda n: n.lo)
        chosen_log.append([(n.lo, n.hi) for n in picked])
        cands = [c for n in picked for c in n.children]
    rows = [(c.key, c.value) for c in cands] + list(local or [])
    P = len(rows) - 1
    qr = [_rot(q[g].astype(np.float64), P, base) for g in range(G)]
    for i, (kk, vv) in enumerate(rows):
        kr = _rot(np.asarray(kk, dtype=np.float64), i, base)
        entries.append(([_dot(qr[g], kr) * scale for g in range(G)], np.asarray(vv, dtype=np.float64)))
    out = np.zeros((G, d))
    for g in range(G):
        lg = np.array([e[0][g] for e in entries])
        w = np.exp(lg - lg.max())
        w /= w.sum()
        out[g] = sum(wi * e[1] for wi, e in zip(w, entries))
    return out, chosen_log


def min_margin(levels, q, k, base):
    """Smallest gap between the k-th and (k+1)-th selection scores over the
    descent (inf if nothing is dropped): a guard against comparing a near tie."""
    G, d = q.shape
    scale = 1.0 / np.sqrt(d)
    best = np.inf
    cands = list(levels[-1])
    for _lev in range(len(levels) - 1, 0, -1):
        P = len(cands) - 1
        qr = [_rot(q[g].astype(np.float64), P, base) for g in range(G)]
        sc = sorted(((sum(_dot(qr[g], _rot(n.key, i, base)) * scale for g in range(G)), n)
                     for i, n in enumerate(cands)), key=lambda s: (-s[0], s[1].lo))
        if len(sc) > k:
            best = min(best, sc[k - 1][0] - sc[k][0])
        keep = sorted((s[1] for s in sc[:k]), key=lambda n: n.lo)
        cands = [c for n in keep for c in n.children]
    return best
