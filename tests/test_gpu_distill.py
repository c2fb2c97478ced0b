"""One distillation step of the pooler through the C ABI (needs a B200).

recsa_distill_step: forward (selections kept), squared error against dense
attention outputs, the pooler's gradient, a gradient-descent update of the
fp32 master pooler and a rebuild of every node key under it. Checked
against the fp64 oracle (its decode output and its gradient, oracle.query
and oracle.query_grad, over the GPU's node arrays before the step), against
a fresh build with the new pooler, and for a falling loss over steps.

The dense targets come from a plain float64 torch computation of causal
RoPE attention of the last position (test data, independent of both paths).
Tolerances as for the backward: fp32 arithmetic with sums of a few thousand
terms, relative error ~1e-6; the loss to 1e-4 relative, dW to 1e-3 of its
norm.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity
from tests.test_gpu_parity import make_layer, per_seq_queries, small

pytestmark = pytest.mark.gpu


def dense_targets(w, K, V, lengths, q_np):
    """Dense causal RoPE attention of the last position, [B][H_q][d] float64."""
    d, G, h2 = w.head_dim, w.group, w.head_dim // 2
    theta = w.rope_base ** (-torch.arange(h2, dtype=torch.float64) * 2 / d)

    def rot(x, pos):
        z = torch.complex(x[..., :h2], x[..., h2:]) * torch.polar(torch.ones(len(pos), h2, dtype=torch.float64),
                                                                   pos[:, None] * theta)
        return torch.cat([z.real, z.imag], dim=-1)

    out = np.zeros((w.batch, w.n_q_heads, d))
    for b in range(w.batch):
        L = lengths[b]
        for h in range(w.n_kv_heads):
            Kt = torch.from_numpy(synth.as_f32(np.ascontiguousarray(K[b, h, :L])).astype(np.float64))
            Vt = torch.from_numpy(synth.as_f32(np.ascontiguousarray(V[b, h, :L])).astype(np.float64))
            qu = torch.from_numpy(parity.q_unit(q_np, b, h, G).astype(np.float64))
            kr = rot(Kt, torch.arange(L, dtype=torch.float64))
            qr = rot(qu, torch.full((G,), float(L - 1), dtype=torch.float64))
            p = torch.softmax(qr @ kr.T / math.sqrt(d), dim=-1)
            out[b, h * G:(h + 1) * G] = (p @ Vt).numpy()
    return out


def oracle_step(layer, w, K, V, Wf, lengths, q_np, target, trees):
    """Loss and dW of one step by the oracle over the given node arrays."""
    n = w.batch * w.n_q_heads * w.head_dim
    loss, dW = 0.0, np.zeros((w.head_dim, w.head_dim))
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            L = lengths[b]
            tK, tV = trees[(b, h)]
            qu = parity.q_unit(q_np, b, h, w.group)
            ref = parity.oracle_query(tK, tV, K, V, b, h, L, qu, w)
            assert all(m > parity.NEAR_TIE for m in ref["margin"]), "a near tie: pick another seed"
            diff = ref["out"] - target[b, h * w.group:(h + 1) * w.group]
            loss += float((diff ** 2).sum()) / n
            g = oracle.query_grad(tK, tV, K[b, h], V[b, h], L, qu, 2 * diff / n, Wf, w.head_dim, w.branching, w.k,
                                  w.group, w.rope_base)
            dW += g["dW"]
    return loss, dW


@pytest.mark.parametrize("bf16,D,b", [(False, 64, 8), (True, 128, 8), (True, 128, 5)])
def test_distill_step_matches_oracle_and_rebuild(bf16, D, b):
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=D, branching=b, k=3, bf16=bf16)
    lengths = [600, 1500]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp = make_layer(w, 2048)
    layer.load(parity.to_dev(K, bf16), parity.to_dev(V, bf16), lengths)
    q_np = per_seq_queries(w, runs, 0, lengths)
    target = dense_targets(w, K, V, lengths, q_np)
    J_cap, _ = layer.tree_shape()
    trees = {(b, h): parity.gpu_tree_unit(layer, b, h, oracle.levels(lengths[b], w.branching)[0], lengths[b])
             for b in range(w.batch) for h in range(w.n_kv_heads)}
    Wf = synth.as_f32(Wp)
    loss_o, dW_o = oracle_step(layer, w, K, V, Wf, lengths, q_np, target, trees)
    lr = 0.05 * np.linalg.norm(Wf) / np.linalg.norm(dW_o)
    dw = torch.zeros((D, D), dtype=torch.float32, device="cuda")
    loss = layer.distill_step(parity.to_dev(q_np, bf16), torch.from_numpy(target).float().cuda(), lr, dw_out=dw)
    torch.cuda.synchronize()
    layer.check()
    assert abs(loss.item() - loss_o) <= 1e-4 * loss_o, (loss.item(), loss_o)
    gdw = parity.to_f64(dw)
    assert np.linalg.norm(gdw - dW_o) <= 1e-3 * np.linalg.norm(dW_o), (np.linalg.norm(gdw - dW_o),
                                                                       np.linalg.norm(dW_o))
    w_new = parity.to_f64(layer.w_master)
    # w - lr dW in fp32 with the GPU's dW: within 0.1 % of the largest step
    assert np.all(np.abs(w_new - (Wf - lr * dW_o)) <= 1e-3 * lr * np.abs(dW_o).max() + 1e-6 * np.abs(Wf) + 1e-7)
    # the tree was rebuilt under the new pooler: the same nodes as a fresh build with it
    fresh = type(layer)(w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim, w.branching, w.k, 2048,
                        layer.w_master.to(torch.bfloat16 if bf16 else torch.float32),
                        dtype=torch.bfloat16 if bf16 else torch.float32, rope_base=w.rope_base)
    fresh.load(parity.to_dev(K, bf16), parity.to_dev(V, bf16), lengths)
    torch.cuda.synchronize()
    for j in range(1, J_cap + 1):
        for x, y in zip(layer.level(j), fresh.level(j)):
            assert torch.equal(x, y), j


def test_distill_loss_falls():
    """Small gradient steps lower the squared error against dense attention
    (fp32 storage, so that a small change of the pooler reaches the tree;
    steps of 0.1 % of |W|)."""
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=64, branching=8, k=3, bf16=False)
    lengths = [1200, 1700]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp = make_layer(w, 2048)
    layer.load(parity.to_dev(K, False), parity.to_dev(V, False), lengths)
    q_np = per_seq_queries(w, runs, 0, lengths)
    q = parity.to_dev(q_np, False)
    target = torch.from_numpy(dense_targets(w, K, V, lengths, q_np)).float().cuda()
    dw = torch.zeros((w.head_dim, w.head_dim), dtype=torch.float32, device="cuda")
    loss0 = layer.distill_step(q, target, 0.0, dw_out=dw).item()  # lr 0: the loss and gradient only
    lr = 1e-3 * layer.w_master.norm().item() / dw.norm().item()
    losses = [loss0]
    for _ in range(6):
        losses.append(layer.distill_step(q, target, lr).item())
    layer.check()
    # the step returns the loss before its update: losses[i + 1] is the loss after i updates
    assert losses[1] == pytest.approx(loss0, rel=1e-6)
    # the first update lowers it (first order, the selections held); later a
    # selection may flip and move it either way, but the trend is down
    assert losses[2] < losses[1] and losses[-1] < losses[1], losses
