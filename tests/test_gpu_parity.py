"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Bars: selections bit-exact except near ties (oracle margin < 1e-4, counted);
outputs within max-abs 1e-4 (fp32) / 2e-2 (bf16 I/O, fp32 accumulation);
node arrays within 1e-5 relative (fp32) / 1 ulp (bf16); rows read equal.
"staged" runs the oracle's descent over the GPU's stored node arrays (read
as data), so selection is checked independently of 1-ulp node rounding;
"free" runs the oracle on its own tree.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from hierarchical_sparse_attention_tree_b200 import RecsaError, RecsaLayer
from hierarchical_sparse_attention_tree_b200 import recsa as R
from tests import parity

pytestmark = pytest.mark.gpu

W_TINY = synth.WORKLOADS["tiny_f32"]


def small(**kw):
    base = dict(name="small", batch=1, n_kv_heads=1, group=4, head_dim=128, branching=8, k=3, length=1000,
                bf16=True, centroids=16, run_min=16, run_max=64)
    base.update(kw)
    return synth.Workload(**base)


def make_layer(w, capacity, max_chunk=0):
    W = synth.workload_pooler(w)
    return RecsaLayer(w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim, w.branching, w.k, capacity,
                      parity.to_dev(W, w.bf16), dtype=torch.bfloat16 if w.bf16 else torch.float32,
                      rope_base=w.rope_base, max_chunk=max_chunk), W


def per_seq_queries(w, runs, step, lengths):
    return np.stack([synth.decode_query(w.seed, b, step, lengths[b], w.n_kv_heads, w.group, w.head_dim, w.centroids,
                                        w.sigma_noise, runs[b], w.bf16)[0] for b in range(w.batch)])


def run_decode(layer, w, q_np):
    B, H, G, D = w.batch, w.n_kv_heads, w.group, w.head_dim
    J_cap, _ = layer.tree_shape()
    q = parity.to_dev(q_np, w.bf16)
    sel = torch.full((B, H, J_cap, w.k), -7, dtype=torch.int32, device="cuda")
    rows = torch.zeros((B, H, 2), dtype=torch.int64, device="cuda")
    out = layer.decode(q, sel_out=sel, rows_out=rows)
    torch.cuda.synchronize()
    layer.check()
    return parity.to_f64(out), sel.cpu().numpy(), rows.cpu().numpy()


def check_units(layer, w, K, V, Wp, lengths, q_np, gout, gsel, grows, units=None, staged=True, free=True,
                free_exact=None, reports=None):
    """Checks the listed units of one decode against the oracle.

    staged: the oracle descends over the GPU's stored node arrays (read as
    data). Selections must be exact above the first near tie; outputs and
    rows read are compared wherever all levels agree.
    free: the oracle descends over its own tree (fp64 arithmetic rounded
    once). Node keys may then differ by one storage ulp from the GPU's; where
    that alone changes the oracle's selection (staged and free oracle
    disagree) the unit is counted as a node-rounding flip. Everywhere else
    the GPU must select exactly what the free oracle selects, with outputs
    within the tolerance. free_exact: no flips allowed either (fp32)."""
    G = w.group
    tol = 2e-2 if w.bf16 else 1e-4
    storage = parity.storage_of(w.bf16)
    reports = reports or {"staged": parity.new_report(), "free": parity.new_report()}
    units = units or [(b, h) for b in range(w.batch) for h in range(w.n_kv_heads)]
    for b, h in units:
        L = lengths[b]
        J, _ = oracle.levels(L, w.branching)
        qu = parity.q_unit(q_np, b, h, G)
        ref_staged, staged_ok = None, True
        if staged:
            tK, tV = parity.gpu_tree_unit(layer, b, h, J, L)
            ref_staged = parity.oracle_query(tK, tV, K, V, b, h, L, qu, w)
            reports["staged"]["queries"] += 1
            staged_ok = parity.check_decode(gout, gsel, grows, ref_staged, b, h, G, tol, reports["staged"])
        if free:
            tree = oracle.build_tree(K[b, h], V[b, h], L, w.head_dim, w.branching, synth.as_f32(Wp), storage)
            ref = oracle.query_tree(tree, K[b, h], V[b, h], qu, w.k, G, w.rope_base)
            rep = reports["free"]
            rep["queries"] += 1
            if ref_staged is not None and not parity.same_selection(ref_staged, ref):
                rep["node_rounding_flips"] += 1
                continue
            if not staged_ok:  # a near tie the GPU resolved the other way
                rep["near_tie_sel_diff"] += 1
                continue
            parity.check_decode(gout, gsel, grows, ref, b, h, G, tol, rep)
    st, fr = reports["staged"], reports["free"]
    if staged:
        assert st["sel_mismatch"] == 0, st
        assert st["checked"] + st["near_tie_sel_diff"] == st["queries"], st
    if free:
        assert fr["sel_mismatch"] == 0, fr
        if free_exact:
            assert fr["node_rounding_flips"] == 0 and fr["near_tie_sel_diff"] == 0, fr
    return reports


def record_all(test, config, reps, modes=("staged", "free")):
    for m in modes:
        parity.record(test, config, m, reps[m])


def check_nodes(layer, w, K, V, Wp, lengths, units=None):
    """GPU node arrays vs the oracle, every kept level. Values: the oracle's
    exact subtree means, rounded once. Keys: the oracle's pooler applied to
    the mean of the children as the GPU stored them (level 1: the tokens), so
    a 1-ulp rounding difference one level down is not compounded."""
    storage = parity.storage_of(w.bf16)
    J_cap, _ = layer.tree_shape()
    units = units or [(b, h) for b in range(w.batch) for h in range(w.n_kv_heads)]
    Wf = synth.as_f32(Wp)
    off = 0
    for b, h in units:
        L = lengths[b]
        if L == 0:
            continue
        tree = oracle.Tree(w.head_dim, w.branching, L, storage, J_keep=J_cap).build(K[b, h], V[b, h], L, Wf)
        below = synth.as_f32(K[b, h, :L]).astype(np.float64)
        vtok = synth.as_f32(V[b, h, :L])
        for j in range(1, J_cap + 1):
            n = -(-L // w.branching ** j)
            kj, vj, sj = layer.level(j)
            gk = parity.to_f64(kj[b, h, :n])
            okk, nk = parity.compare_nodes(gk, oracle.pool_level(below, w.branching, Wf, storage), w.bf16,
                                           atol=parity.pooled_key_bound(below, w.branching, Wf))
            okv, nv = parity.compare_nodes(parity.to_f64(vj[b, h, :n]), tree.V[j][:n], w.bf16,
                                           atol=parity.mean_value_bound(vtok, w.branching ** j))
            assert okk and okv, (b, h, j, nk, nv)
            off += nk + nv
            below = gk
    return off


# ---------------------------------------------------------------- tiny fp32


def test_tiny_f32_build_and_decode():
    """The tiny fp32 workload: L=4096, one KV head, G=4, d=64, b=16, k=4
    (levels 4096 -> 256 -> 16), 8 decode queries against a fixed cache."""
    w = W_TINY
    K, V, runs = synth.cache_arrays(w, w.length)
    layer, Wp = make_layer(w, w.length)
    layer.load(parity.to_dev(K, False), parity.to_dev(V, False), [w.length])
    assert layer.tree_shape()[0] == 2
    check_nodes(layer, w, K, V, Wp, [w.length])
    reps = None
    for s in range(w.queries):
        q = per_seq_queries(w, runs, s, [w.length])
        gout, gsel, grows = run_decode(layer, w, q)
        reps = check_units(layer, w, K, V, Wp, [w.length], q, gout, gsel, grows, free_exact=True, reports=reps)
        assert grows[0, 0, 0] <= w.k * w.branching * 3
    record_all("test_tiny_f32_build_and_decode", w.name, reps)
    assert reps["staged"]["checked"] >= 6, reps


# -------------------------------------------------- bf16, several units


@pytest.mark.parametrize("D,G", [(128, 4), (64, 2), (128, 1), (64, 8), (128, 8)])
def test_bf16_ragged_batch(D, G):
    w = small(batch=3, n_kv_heads=2, group=G, head_dim=D, branching=8, k=3)
    lengths = [1, 517, 3001]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp = make_layer(w, 4096)
    layer.load(parity.to_dev(K, True), parity.to_dev(V, True), lengths)
    check_nodes(layer, w, K, V, Wp, lengths)
    reps = None
    for s in range(3):
        q = per_seq_queries(w, runs, s, lengths)
        gout, gsel, grows = run_decode(layer, w, q)
        reps = check_units(layer, w, K, V, Wp, lengths, q, gout, gsel, grows, reports=reps)
    record_all("test_bf16_ragged_batch", f"bf16 d={D} G={G} lengths 1/517/3001 b=8 k=3", reps)


def test_query_stats_report_depth_and_rows():
    """recsa_query_stats returns, per unit, the depth the last decode
    descended (J + 1) and the K / V rows it read (the same counts as
    rows_out, which the parity checks compare with the oracle's)."""
    w = small(batch=3, n_kv_heads=2, group=4, head_dim=128, branching=8, k=3)
    lengths = [1, 517, 3001]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp = make_layer(w, 4096)
    assert layer.query_stats() == ([0] * 6, [0] * 6, [0] * 6)
    layer.load(parity.to_dev(K, True), parity.to_dev(V, True), lengths)
    q = per_seq_queries(w, runs, 0, lengths)
    gout, gsel, grows = run_decode(layer, w, q)
    depth, kr, vr = layer.query_stats()
    for b in range(w.batch):
        J, _ = oracle.levels(lengths[b], w.branching)
        for h in range(w.n_kv_heads):
            u = b * w.n_kv_heads + h
            assert depth[u] == J + 1
            assert (kr[u], vr[u]) == tuple(grows[b, h])


@pytest.mark.parametrize("k,L", [(24, 20000), (40, 200000)])
def test_large_k_selection(k, L):
    """k > 16: the CTA and cluster top-k are merged by rank search; at
    L = 200000 (b = 64, k = 40) a CTA holds 320 level-1 rows, more than 32 per
    warp, so each warp ranks its rows instead of sorting them in registers."""
    w = small(batch=1, n_kv_heads=2, group=4, head_dim=128, branching=64, k=k)
    K, V, runs = synth.cache_arrays(w, L)
    layer, Wp = make_layer(w, L)
    layer.load(parity.to_dev(K, True), parity.to_dev(V, True), [L])
    reps = None
    for s in range(2):
        q = per_seq_queries(w, runs, s, [L])
        gout, gsel, grows = run_decode(layer, w, q)
        reps = check_units(layer, w, K, V, Wp, [L], q, gout, gsel, grows, free=False, reports=reps)
    record_all("test_large_k_selection", f"bf16 L={L} b=64 k={k}", reps, modes=("staged",))


def test_f32_d128_matches_free_oracle():
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=128, branching=16, k=4, bf16=False)
    lengths = [4100, 700]
    K, V, runs = synth.cache_arrays(w, max(lengths))
    layer, Wp = make_layer(w, 8192)
    layer.load(parity.to_dev(K, False), parity.to_dev(V, False), lengths)
    check_nodes(layer, w, K, V, Wp, lengths)
    reps = None
    for s in range(3):
        q = per_seq_queries(w, runs, s, lengths)
        gout, gsel, grows = run_decode(layer, w, q)
        reps = check_units(layer, w, K, V, Wp, lengths, q, gout, gsel, grows, free_exact=True, reports=reps)
    record_all("test_f32_d128_matches_free_oracle", "fp32 d=128 lengths 4100/700 b=16 k=4", reps)


@pytest.mark.parametrize("L", [1, 2, 7, 8, 9, 63, 64, 65, 511, 512, 513])
def test_edge_lengths(L):
    """Single token, exactly b and b^2 tokens, one past (a new level)."""
    w = small(batch=1, n_kv_heads=1, group=4, head_dim=64, branching=8, k=2, bf16=False)
    K, V, runs = synth.cache_arrays(w, L)
    layer, Wp = make_layer(w, 600)
    layer.load(parity.to_dev(K, False), parity.to_dev(V, False), [L])
    check_nodes(layer, w, K, V, Wp, [L])
    q = per_seq_queries(w, runs, 0, [L])
    gout, gsel, grows = run_decode(layer, w, q)
    check_units(layer, w, K, V, Wp, [L], q, gout, gsel, grows, free_exact=True)


def test_dense_equivalence_on_gpu():
    """k covering every level keeps everything: the GPU output equals dense
    causal RoPE attention (the oracle reaches the same case)."""
    w = small(batch=1, n_kv_heads=2, group=4, head_dim=64, branching=16, k=64, bf16=False)
    L = 1000
    K, V, runs = synth.cache_arrays(w, L)
    layer, Wp = make_layer(w, L)
    layer.load(parity.to_dev(K, False), parity.to_dev(V, False), [L])
    q = per_seq_queries(w, runs, 0, [L])
    gout, gsel, grows = run_decode(layer, w, q)
    assert (grows[0, :, 1] == L).all()  # every token enters the softmax
    check_units(layer, w, K, V, Wp, [L], q, gout, gsel, grows, free_exact=True)


# ---------------------------------------------------------------- append


@pytest.mark.parametrize("bf16", [False, True])
def test_append_matches_rebuild_bitwise(bf16):
    """Token-by-token and chunked appends leave exactly the node arrays a
    fresh build over the same tokens produces."""
    w = small(batch=2, n_kv_heads=2, group=2, head_dim=64, branching=4, k=2, bf16=bf16)
    start = [30, 61]
    plan = [1] * 40 + [7, 1, 64, 3, 1, 16]
    total = sum(plan)
    cap = max(start) + total
    K, V, runs = synth.cache_arrays(w, cap)
    Kd, Vd = parity.to_dev(K, bf16), parity.to_dev(V, bf16)
    inc, Wp = make_layer(w, cap)
    K0, V0 = Kd.clone(), Vd.clone()
    for b in range(w.batch):  # the cache holds only the first start[b] tokens
        K0[b, :, start[b]:] = 0
        V0[b, :, start[b]:] = 0
    inc.load(K0, V0, start)
    # the appended tokens come from the generator: sequence b, positions start[b] + ...
    pos = list(start)
    for n in plan:
        kn = torch.stack([Kd[b, :, pos[b]:pos[b] + n] for b in range(w.batch)]).permute(0, 2, 1, 3).contiguous()
        vn = torch.stack([Vd[b, :, pos[b]:pos[b] + n] for b in range(w.batch)]).permute(0, 2, 1, 3).contiguous()
        inc.append(kn, vn)
        pos = [p + n for p in pos]
        full, _ = make_layer(w, cap)
        full.load(Kd, Vd, pos)
        torch.cuda.synchronize()
        J_cap, rows = inc.tree_shape()
        for j in range(1, J_cap + 1):
            for a, b_ in zip(inc.level(j), full.level(j)):
                for s in range(w.batch):
                    n_j = -(-pos[s] // w.branching ** j)
                    assert torch.equal(a[s, :, :n_j], b_[s, :, :n_j]), (n, j, s)
        full.close()
    assert inc.lengths() == pos
    inc.check()
    for b in range(w.batch):  # the appended rows landed after each sequence's tokens
        assert torch.equal(inc.k_cache[b, :, :pos[b]], Kd[b, :, :pos[b]])
        assert torch.equal(inc.v_cache[b, :, :pos[b]], Vd[b, :, :pos[b]])
    check_nodes(inc, w, K, V, Wp, pos)
    q = per_seq_queries(w, runs, 0, pos)
    gout, gsel, grows = run_decode(inc, w, q)
    check_units(inc, w, K, V, Wp, pos, q, gout, gsel, grows, free_exact=not bf16)


@pytest.mark.parametrize("bf16,branching,k,start,steps", [
    (False, 4, 2, [30, 61], 40),
    (True, 4, 2, [30, 61], 40),
    # first scored level of 960 candidates: the appending CTA keeps a share of
    # the rows and refreshes the right-edge row in its tile after the append
    (True, 64, 16, [61400, 61439], 3),
])
def test_fused_append_decode(bf16, branching, k, start, steps):
    """recsa_append_decode (one launch per step) leaves the node arrays and
    returns the selections and row counts of recsa_append then recsa_decode,
    bit for bit, across node and level boundaries (sequence 1 grows from 61
    past 64 = b^3 tokens). The outputs agree to rounding: the fused launch
    splits the first level's rows differently over the cluster, so the
    per-CTA softmax sums are added in another order. The last step also
    matches the oracle."""
    w = small(batch=2, n_kv_heads=2, group=4, head_dim=128, branching=branching, k=k, bf16=bf16)
    cap = max(start) + steps
    K, V, runs = synth.cache_arrays(w, cap)
    Kd, Vd = parity.to_dev(K, bf16), parity.to_dev(V, bf16)
    fused, Wp = make_layer(w, cap)
    split, _ = make_layer(w, cap)
    K0, V0 = Kd.clone(), Vd.clone()
    for b in range(w.batch):
        K0[b, :, start[b]:] = 0
        V0[b, :, start[b]:] = 0
    fused.load(K0.clone(), V0.clone(), start)
    split.load(K0.clone(), V0.clone(), start)
    J_cap, _ = fused.tree_shape()
    pos = list(start)
    for s in range(steps):
        kn = torch.stack([Kd[b, :, pos[b]:pos[b] + 1] for b in range(w.batch)]).permute(0, 2, 1, 3).contiguous()
        vn = torch.stack([Vd[b, :, pos[b]:pos[b] + 1] for b in range(w.batch)]).permute(0, 2, 1, 3).contiguous()
        pos = [p + 1 for p in pos]
        q_np = per_seq_queries(w, runs, s, pos)
        q = parity.to_dev(q_np, bf16)
        outs = []
        for layer in (fused, split):
            sel = torch.full((w.batch, w.n_kv_heads, J_cap, w.k), -7, dtype=torch.int32, device="cuda")
            rows = torch.zeros((w.batch, w.n_kv_heads, 2), dtype=torch.int64, device="cuda")
            if layer is fused:
                out = layer.append_decode(kn, vn, q, sel_out=sel, rows_out=rows)
            else:
                layer.append(kn, vn)
                out = layer.decode(q, sel_out=sel, rows_out=rows)
            outs.append((out, sel, rows))
        torch.cuda.synchronize()
        assert torch.equal(outs[0][1], outs[1][1]) and torch.equal(outs[0][2], outs[1][2]), s
        diff = (outs[0][0].float() - outs[1][0].float()).abs().max().item()
        assert diff <= (1e-2 if bf16 else 1e-5), (s, diff)
    fused.check()
    split.check()
    assert fused.lengths() == pos == split.lengths()
    for j in range(1, J_cap + 1):
        for x, y in zip(fused.level(j), split.level(j)):
            for b in range(w.batch):
                n_j = -(-pos[b] // w.branching ** j)
                assert torch.equal(x[b, :, :n_j], y[b, :, :n_j]), (j, b)
    for b in range(w.batch):
        assert torch.equal(fused.k_cache[b, :, :pos[b]], Kd[b, :, :pos[b]])
        assert torch.equal(fused.v_cache[b, :, :pos[b]], Vd[b, :, :pos[b]])
    gout, gsel, grows = parity.to_f64(outs[0][0]), outs[0][1].cpu().numpy(), outs[0][2].cpu().numpy()
    check_units(fused, w, K, V, Wp, pos, q_np, gout, gsel, grows, free_exact=not bf16)


def test_capacity_and_argument_errors():
    w = small(batch=1, n_kv_heads=1, group=4, head_dim=64, branching=4, k=2, bf16=False)
    K, V, _ = synth.cache_arrays(w, 20)
    layer, _ = make_layer(w, 20)
    with pytest.raises(RecsaError) as e:
        layer.decode(torch.zeros(1, 4, 64, device="cuda"))
    assert e.value.status == R.ERR_INVALID_ARG  # no tokens yet
    layer.load(parity.to_dev(K, False), parity.to_dev(V, False), [18])
    kn = torch.zeros(1, 3, 1, 64, device="cuda")
    with pytest.raises(RecsaError) as e:
        layer.append(kn, kn)
    assert e.value.status == R.ERR_CAPACITY
    assert layer.lengths() == [18]
    with pytest.raises(RecsaError) as e:
        layer.ctx.build_tree([21])
    assert e.value.status == R.ERR_CAPACITY
    layer.check()


# ------------------------------------------------------- full-size decode


def _full_size(name, steps, units):
    """Build the workload's tree, then `steps` append + decode steps; every
    sampled unit's node arrays are checked against the oracle after the
    build and after the last step, and every step's decode of the sampled
    units in staged and free mode."""
    w = synth.WORKLOADS[name]
    L0 = w.length
    cap = L0 + steps
    K, V, runs = synth.cache_arrays(w, cap)
    layer, Wp = make_layer(w, cap)
    Kd, Vd = parity.to_dev(K, True), parity.to_dev(V, True)
    layer.load(Kd, Vd, [L0] * w.batch)
    check_nodes(layer, w, K, V, Wp, [L0] * w.batch, units=units)
    lengths = [L0] * w.batch
    reps = None
    for s in range(steps):
        kn = Kd[:, :, lengths[0]:lengths[0] + 1].permute(0, 2, 1, 3).contiguous()
        vn = Vd[:, :, lengths[0]:lengths[0] + 1].permute(0, 2, 1, 3).contiguous()
        lengths = [x + 1 for x in lengths]
        q = per_seq_queries(w, runs, s, lengths)
        # the fused step (one launch), as the benchmark runs it
        J_cap, _ = layer.tree_shape()
        sel = torch.full((w.batch, w.n_kv_heads, J_cap, w.k), -7, dtype=torch.int32, device="cuda")
        rows = torch.zeros((w.batch, w.n_kv_heads, 2), dtype=torch.int64, device="cuda")
        out = layer.append_decode(kn, vn, parity.to_dev(q, True), sel_out=sel, rows_out=rows)
        torch.cuda.synchronize()
        layer.check()
        reps = check_units(layer, w, K, V, Wp, lengths, q, parity.to_f64(out), sel.cpu().numpy(),
                           rows.cpu().numpy(), units=units, reports=reps)
    check_nodes(layer, w, K, V, Wp, lengths, units=units)
    record_all(f"_full_size[{name}]", name, reps)
    depth, kr, vr = layer.query_stats()
    parity.record(f"_full_size[{name}]", name, "reads",
                  {"depth": max(depth), "k_rows_mean": float(np.mean(kr)), "v_rows_mean": float(np.mean(vr)),
                   "bound_k_b_depth": w.k * w.branching * max(depth)})
    assert max(kr) <= w.k * w.branching * max(depth) and max(vr) <= w.k * w.branching * max(depth)
    layer.close()
    return reps


def test_decode_131k_sampled():
    """Qwen3-4B-shaped layer at L=131072 (b=64, k=16): build, then fused
    append + decode steps; sampled KV heads checked against the oracle."""
    _full_size("decode_131k", 3, [(0, 0), (0, 5)])


def test_decode_524k_batch4_sampled():
    """The 524K, batch-4 decode workload in the benchmark's launch shape."""
    _full_size("decode_524k_b4", 2, [(0, 0), (1, 3), (3, 7)])


def test_decode_2m_sampled():
    """L = 2097152 (about 8.6 GB of keys and values for the layer; levels
    2097152 -> 32768 -> 512 -> 8, b = 64, k = 16): full build, fused steps,
    sampled KV heads in staged and free mode. The rows each query reads grow
    with the depth, not with L."""
    reps = _full_size("decode_2m", 2, [(0, 0), (0, 6)])
    assert reps["staged"]["checked"] >= 2


# ----------------------------------------------------- dense comparator


@pytest.mark.parametrize("dtype,D,G,L", [(torch.bfloat16, 128, 4, 70000), (torch.float32, 64, 2, 999),
                                         (torch.bfloat16, 64, 8, 5)])
def test_dense_decode_comparator(dtype, D, G, L):
    B, H = 2, 3
    g = torch.Generator(device="cuda").manual_seed(0)
    Kc = torch.randn(B, H, L + 3, D, device="cuda", generator=g).to(dtype)
    Vc = torch.randn(B, H, L + 3, D, device="cuda", generator=g).to(dtype)
    q = torch.randn(B, H * G, D, device="cuda", generator=g).to(dtype)
    out = torch.empty_like(q)
    scratch = torch.empty(R.dense_decode_scratch_bytes(B, H * G, D), dtype=torch.uint8, device="cuda")
    R.dense_decode(Kc, Vc, q, out, L, scratch)
    qf = q.float().view(B, H, G, D)
    s = torch.einsum("bhgd,bhtd->bhgt", qf, Kc[:, :, :L].float()) / D ** 0.5
    ref = torch.einsum("bhgt,bhtd->bhgd", torch.softmax(s, -1), Vc[:, :, :L].float()).reshape(B, H * G, D)
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    assert (out.float() - ref).abs().max().item() <= tol
