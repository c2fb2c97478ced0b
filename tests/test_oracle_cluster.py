"""Pins of the oracle's LSA-style clustered order (oracle.cluster_order).

The order is pinned by what it must be, not by retyping it: a permutation;
for every level j, inside every block of b^(j+1) positions, consecutive
blocks of b^j positions follow one another in (z_j, token index) order, with
z_j = <Z_j, k_t> computed here by numpy; inside a level-1 block the tokens are
in (z_1, index) order; with every direction equal to one coordinate axis the
order is numpy's stable argsort along it; identical keys keep the token order.
Source: the "Latent Sparse Attention" abstract (keys clustered hierarchically
in a learned latent space, queries scoring the hierarchy of clusters) and the
reading R20 of recsa_oracle.c.
"""
import numpy as np
import pytest

import oracle
import synth


def _keys(seed, T, d, bf16=False):
    return synth.plain(901, seed, (T, d), 0.0, 1.0, bf16)


def _dirs(seed, J, d):
    return synth.plain(902, seed, (J, d), 0.0, 1.0, False)


def _check_partition(K, T, b, Z, perm):
    Kf = synth.as_f32(K).astype(np.float64)[:T]
    assert sorted(perm.tolist()) == list(range(T))
    J, _ = oracle.levels(T, b)
    for j in range(1, J + 1):
        z = Kf @ Z[j - 1].astype(np.float64)
        key = [(z[t], t) for t in perm]
        S, s = b ** (j + 1), b ** j
        for p0 in range(0, T, S):
            blocks = [key[c0:min(c0 + s, p0 + S, T)] for c0 in range(p0, min(p0 + S, T), s)]
            for lo, hi in zip(blocks, blocks[1:]):
                assert max(lo) < min(hi), (j, p0)
        if j == 1:  # inside a level-1 node: (z_1, index) order
            for c0 in range(0, T, b):
                run = key[c0:c0 + b]
                assert run == sorted(run)


@pytest.mark.parametrize("T,b,d", [(1, 4, 8), (3, 4, 8), (4, 4, 8), (5, 4, 8), (300, 4, 16), (1000, 8, 16),
                                   (4097, 16, 32), (777, 5, 12)])
def test_cluster_order_is_a_nested_sorted_partition(T, b, d):
    J, _ = oracle.levels(T, b)
    K = _keys(T, T, d)
    Z = _dirs(T, max(J, 1), d)
    perm = oracle.cluster_order(K, T, b, Z)
    _check_partition(K, T, b, Z, perm)


def test_cluster_order_bf16_keys():
    T, b, d = 2000, 8, 16
    J, _ = oracle.levels(T, b)
    K = _keys(5, T, d, bf16=True)
    Z = _dirs(5, J, d)
    _check_partition(K, T, b, Z, oracle.cluster_order(K, T, b, Z))


def test_cluster_order_along_one_axis_is_argsort():
    """Every level splitting along the same coordinate axis: each level
    refines the order of the one above, so the whole order is one stable
    argsort of that coordinate."""
    T, b, d = 1500, 6, 10
    J, _ = oracle.levels(T, b)
    K = _keys(7, T, d)
    Z = np.zeros((J, d), np.float32)
    Z[:, 3] = 1.0
    perm = oracle.cluster_order(K, T, b, Z)
    assert np.array_equal(perm, np.argsort(K[:, 3], kind="stable"))


def test_cluster_order_ties_keep_token_order():
    T, b, d = 500, 4, 8
    J, _ = oracle.levels(T, b)
    K = np.ones((T, d), np.float32)
    Z = _dirs(9, J, d)
    assert np.array_equal(oracle.cluster_order(K, T, b, Z), np.arange(T))
    # negative zero and zero are one latent value: ties again
    K[::2, :] = 0.0
    K[1::2, :] = -0.0
    assert np.array_equal(oracle.cluster_order(K, T, b, Z), np.arange(T))


def test_cluster_order_single_level():
    """T <= b: one level, one block: the order is the argsort of z_1 (ties by
    index)."""
    T, b, d = 7, 8, 5
    K = _keys(11, T, d)
    Z = _dirs(11, 1, d)
    z = K.astype(np.float64) @ Z[0].astype(np.float64)
    assert np.array_equal(oracle.cluster_order(K, T, b, Z), np.lexsort((np.arange(T), z)))
