#!/usr/bin/env python
"""RecSA decode benchmark on B200.

Workload (default): one Qwen3-4B-shaped attention layer (32 query heads, 8 KV
heads, head_dim 128, bf16), L = 524288 cached tokens per sequence, batch 4,
branching 64, k = 16. One step = append one token to every sequence and
one decode query per sequence, one launch (recsa_append_decode). Inputs are
seeded synthetic data (Gaussian-mixture keys in token runs, N(0,1) values,
queries aimed at a planted run, random pooler) resident in HBM before timing.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch of
independent sequences (weak scaling, no collective on the data path); the
step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "RecSA layer decode query-tok/s & prefill tok/s at 524K; % of HBM roofline"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="recsa", choices=["recsa", "reference"])
    ap.add_argument("--workload", default="decode_524k_b4")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-distill", action="store_true")
    ap.add_argument("--no-cluster", action="store_true")
    ap.add_argument("--prefill-workload", default="prefill_524k")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the chunked prefill (profiling): no decode, no baselines")
    ap.add_argument("--prefill-last", type=int, default=0,
                    help="build the tree over all but the last N chunks at once, then prefill only those N")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="time limit of the oracle CPU-baseline sample (seconds)")
    ap.add_argument("--settle-s", type=float, default=0.3, help="decode-only launches before timing (clock sampling)")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source for this workload (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)[kernel]
        if d.get("workload") != workload:
            return None
        src = b"".join(open(os.path.join(ROOT, f), "rb").read() for f in d["sources"])
        if hashlib.sha256(src).hexdigest()[:16] != d["source_sha"]:
            return None
        return d["bytes_per_launch"]
    except Exception:
        return None


class ClockSampler:
    """Polls NVML every 10 ms (SM clock, max SM clock, throttle reasons) from
    a thread while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device_index: int):
        self.sm, self.reasons, self.max_sm = [], set(), None
        self.stop_flag = threading.Event()
        self.err = None
        try:
            import pynvml

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = pynvml
            self.max_sm = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        except Exception as e:  # no NVML: report why
            self.err = str(e)
            self.t = None

    def _poll(self):
        while not self.stop_flag.is_set():
            try:
                self.sm.append(float(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(0.01)

    def stop(self):
        if self.t is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        self.stop_flag.set()
        self.t.join(timeout=2)
        return {"sm_mhz": statistics.median(self.sm) if self.sm else None, "sm_max_mhz": self.max_sm,
                "reasons": sorted(self.reasons), "samples": len(self.sm)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world, local, backend: str = "nccl"):
    if world > 1:
        import torch.distributed as dist

        if backend == "nccl":
            dist.barrier(device_ids=[local])
        else:
            dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time: every rank's number is reduced with MAX."""
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_sequences(rank: int, batch: int) -> int:
    """First generator sequence id of this rank's batch: ranks hold disjoint,
    independent sequences (weak scaling, no collective on the data path)."""
    return rank * batch


def aggregate_rate(world: int, batch: int, steps: int, max_seconds: float) -> float:
    """Whole-job query tokens per second: every rank's batch per step, over
    the slowest rank's time."""
    return world * batch * steps / max_seconds


# --------------------------------------------------------- oracle baseline


def oracle_decode_steps(w, K, V, Wp, runs, length0, n_steps, limit_s, seq_ids, threads):
    """The fp64 oracle doing the decode workload's steps for the given
    sequences, every (sequence, KV head) unit in parallel on `threads` host
    threads: per step and per unit, refresh the nodes the new token touched,
    then one query. The trees are built and every step's queries generated
    before the timed loop. Stops at n_steps or after limit_s seconds.
    Returns (steps done, seconds, query tokens, threads used)."""
    import oracle

    storage = oracle.STORE_BF16 if w.bf16 else oracle.STORE_F32
    Wf = synth.as_f32(Wp)
    units = [(b, h) for b in seq_ids for h in range(w.n_kv_heads)]
    used = min(threads, len(units))
    pool = oracle.pool(used)
    trees = dict(zip(units, pool.map(
        lambda bh: oracle.Tree(w.head_dim, w.branching, length0 + n_steps + 1, storage).build(
            K[bh[0], bh[1]], V[bh[0], bh[1]], length0, Wf), units)))
    G = w.group
    qs = {}
    for s in range(n_steps):
        for b in seq_ids:
            q, _ = synth.decode_query(w.seed, b, s, length0 + s + 1, w.n_kv_heads, G, w.head_dim, w.centroids,
                                      w.sigma_noise, runs[b], w.bf16)
            for h in range(w.n_kv_heads):
                qs[(s, b, h)] = synth.as_f32(np.ascontiguousarray(q[h * G:(h + 1) * G]))
    t0 = time.perf_counter()
    done = 0
    for s in range(n_steps):
        L = length0 + s + 1

        def unit(bh, L=L, s=s):
            b, h = bh
            tr = trees[bh]
            tr.build(K[b, h], V[b, h], L, Wf, t_from=L - 1)
            return oracle.query_tree(tr, K[b, h], V[b, h], qs[(s, b, h)], w.k, G, w.rope_base)

        list(pool.map(unit, units))
        done += 1
        if time.perf_counter() - t0 > limit_s:
            break
    dt = time.perf_counter() - t0
    pool.shutdown()
    return done, dt, done * len(seq_ids), used


def run_reference(args, w, world, rank):
    """Reference arm: the fp64 CPU oracle on the same workload and metric
    (every sequence of the batch, every KV head, on all host cores)."""
    if rank != 0:
        return
    threads = os.cpu_count() or 1
    L0 = w.length
    K, V, runs = synth.cache_arrays(w, L0 + args.warmup + args.steps + 1)
    Wp = synth.workload_pooler(w)
    seqs = list(range(w.batch))
    if args.warmup:
        oracle_decode_steps(w, K, V, Wp, runs, L0, args.warmup, 60.0, seqs, threads)
    done, dt, toks, used = oracle_decode_steps(w, K, V, Wp, runs, L0 + args.warmup, args.steps, 150.0, seqs,
                                               threads)
    v = toks / dt
    line = {"metric": METRIC, "impl": "reference", "value": v, "unit": "query-tok/s", "n_gpus": args.gpus,
            "steps": done, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(done, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "L": L0, "batch": w.batch, "n_q_heads": w.n_q_heads,
                       "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "branching": w.branching, "k": w.k},
            "cpu_baseline": {"value": v, "unit": "query-tok/s", "cores": used, "kind": "oracle",
                             "sample": f"{done} decode steps of all {w.batch} sequences x {w.n_kv_heads} KV heads: "
                                       "right-edge node refresh + one query per unit, fp64 (queries generated "
                                       "before timing)"},
            "e2e": {"value": v, "unit": "query-tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ prefill


def prefill_flops(rows_sum_k: int, rows_sum_v: int, n_tokens_local: int, G: int, D: int) -> float:
    """Algorithmic flops of a chunked prefill, from the kernel's own row
    counts: per (token, query head), 2d per key row scored (node keys and
    cached tokens), 2d per value row weighted into the output (summaries,
    cached tokens and the chunk's own tokens), and 2d per chunk token for its
    causal score. rows_sum_k / rows_sum_v are summed over (token, KV head);
    n_tokens_local = sum over (token, KV head) of the chunk tokens it sees."""
    return 2.0 * D * G * (rows_sum_k + rows_sum_v + n_tokens_local)


def measure_prefill(wname, dev, flush, peaks, last_chunks=0, with_dense=True):
    """Chunked prefill of one sequence: every chunk runs recsa_prefill then
    recsa_append (the tree grows after each chunk). last_chunks > 0: the tree
    over all but the last N chunks is built at once (recsa_build_tree) and
    only those N chunks are prefilled. Returns the timings, the prefill's
    tensor roofline and a dense causal prefill of the same length (torch
    SDPA) for comparison."""
    from hierarchical_sparse_attention_tree_b200 import RecsaLayer

    w = synth.WORKLOADS[wname]
    B, H, Hq, D, C, Ltot, G = w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim, w.chunk, w.length, w.group
    bf = torch.bfloat16
    t0 = time.perf_counter()
    K, V, runs = synth.cache_arrays(w, Ltot)
    s_first = 0 if not last_chunks else max(0, Ltot - last_chunks * C)
    Q = [synth.prefill_queries(w.seed, b, s_first, Ltot, H, G, D, w.centroids, w.sigma_noise, runs[b], True)
         for b in range(B)]
    Wp = synth.workload_pooler(w)
    gen_s = time.perf_counter() - t0
    layer = RecsaLayer(B, H, Hq, D, w.branching, w.k, Ltot, torch.from_numpy(Wp).view(bf).to(dev), dtype=bf,
                       rope_base=w.rope_base, max_chunk=C, device=dev)
    kd = torch.from_numpy(np.ascontiguousarray(K.transpose(0, 2, 1, 3))).view(bf).to(dev)  # [B][L][H][D]
    vd = torch.from_numpy(np.ascontiguousarray(V.transpose(0, 2, 1, 3))).view(bf).to(dev)
    qd = torch.stack([torch.from_numpy(x).view(bf) for x in Q]).to(dev)                      # [B][L - s_first][Hq][D]
    if s_first:
        layer.k_cache[:, :, :s_first].copy_(torch.from_numpy(K[:, :, :s_first]).view(bf))
        layer.v_cache[:, :, :s_first].copy_(torch.from_numpy(V[:, :, :s_first]).view(bf))
        layer.ctx.build_tree([s_first] * B)
    del K, V, Q
    out = torch.empty((B, C, Hq, D), dtype=bf, device=dev)
    rows = torch.zeros((B, C, H, 2), dtype=torch.int64, device=dev)
    rows_sum = torch.zeros(2, dtype=torch.int64, device=dev)
    starts = list(range(s_first, Ltot, C))
    n_chunks = len(starts)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_chunks)]
    stream = torch.cuda.current_stream(dev)
    # one warm-up chunk on a throw-away layer of the same shape
    warm = RecsaLayer(B, H, Hq, D, w.branching, w.k, 2 * C, torch.from_numpy(Wp).view(bf).to(dev), dtype=bf,
                      rope_base=w.rope_base, max_chunk=C, device=dev)
    for s0 in (0, C):  # the first chunk's queries, the tree growing over the sequence's first tokens
        sl = slice(s0, s0 + C)
        warm.prefill(qd[:, :C].contiguous(), kd[:, sl].contiguous(), vd[:, sl].contiguous(), out)
        warm.append(kd[:, sl].contiguous(), vd[:, sl].contiguous())
    torch.cuda.synchronize(dev)
    warm.close()
    chunks = [(qd[:, s0 - s_first:s0 - s_first + C].contiguous(), kd[:, s0:s0 + C].contiguous(),
               vd[:, s0:s0 + C].contiguous()) for s0 in starts]
    torch.cuda.synchronize(dev)
    n_local = 0
    for i, (qc, kc, vc) in enumerate(chunks):
        Cc = qc.shape[1]
        flush.fill_(5.0)
        ev[i][0].record(stream)
        layer.prefill(qc, kc, vc, out[:, :Cc], rows_out=rows[:, :Cc])
        ev[i][1].record(stream)
        layer.append(kc, vc)
        ev[i][2].record(stream)
        rows_sum += rows[:, :Cc].sum(dim=(0, 1, 2))
        n_local += B * H * Cc * (Cc + 1) // 2
    torch.cuda.synchronize(dev)
    layer.check()
    pre_ms = [e[0].elapsed_time(e[1]) for e in ev]
    app_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = sum(pre_ms) + sum(app_ms)
    rk, rv = (int(x) for x in rows_sum.tolist())
    flops = prefill_flops(rk, rv, n_local, G, D)
    del chunks
    layer.close()
    ntok = B * (Ltot - s_first)
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    achieved = flops / (sum(pre_ms) / 1e3) / 1e12
    res = {"workload": wname, "tokens": ntok, "chunk": C, "chunks": n_chunks, "first_chunk_start": s_first,
           "tok_s": ntok / (total_ms / 1e3), "ms_total": total_ms, "ms_per_chunk": total_ms / n_chunks,
           "build_share": sum(app_ms) / total_ms, "prefill_ms_per_chunk": sum(pre_ms) / n_chunks,
           "append_ms_per_chunk": sum(app_ms) / n_chunks, "input_gen_s": gen_s, "l2": "flushed before each chunk",
           "roofline": {"kernel": "recsa_prefill (all its launches)", "bound": "tensor", "achieved": achieved,
                        "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                        "peak_source": "bf16_tflops_sustained",
                        "algorithmic_flops": flops, "key_rows": rk, "value_rows": rv}}
    if not with_dense:
        return res
    # dense causal prefill of the same length (torch SDPA, GQA): the faster of
    # two timed runs after a warm-up
    try:
        if s_first:
            raise RuntimeError("dense comparator needs the whole sequence's queries")
        qt = qd.transpose(1, 2)                   # [B][Hq][L][D]
        kt = kd.transpose(1, 2)
        vt = vd.transpose(1, 2)
        sdpa = torch.nn.functional.scaled_dot_product_attention
        sdpa(qt[:, :, :C], kt[:, :, :C], vt[:, :, :C], is_causal=True, enable_gqa=True)
        torch.cuda.synchronize(dev)
        runs_ms = []
        for _ in range(2):
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            sdpa(qt, kt, vt, is_causal=True, enable_gqa=True)
            b_.record(stream)
            torch.cuda.synchronize(dev)
            runs_ms.append(a_.elapsed_time(b_))
        dms = min(runs_ms)
        dflops = 4.0 * B * Hq * D * Ltot * Ltot / 2
        res["dense_sdpa"] = {"ms": dms, "runs_ms": runs_ms, "tok_s": B * Ltot / (dms / 1e3),
                             "tflops": dflops / (dms / 1e3) / 1e12, "recsa_speedup": dms / total_ms}
    except Exception as e:  # the comparator is optional
        res["dense_sdpa"] = {"error": str(e)[:200]}
    return res


def measure_backward(layer, w, q, dev, flush, peaks, kv_host, cpu_threads, with_cpu):
    """Gradients of one decode query per sequence over the layer's current
    tree (recsa_decode_backward, then recsa_tree_backward), each timed with
    CUDA events over 10 runs (L2 flushed before each), with the propagation's
    HBM roofline; and the fp64 oracle's gradient of one query per unit on a
    sample of units, on the host cores."""
    B, H, Hq, D, G = w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim, w.group
    es = 2
    stream = torch.cuda.current_stream(dev)
    J_cap, _ = layer.tree_shape()
    sel = torch.full((B, H, J_cap, w.k), -1, dtype=torch.int32, device=dev)
    layer.decode(q, sel_out=sel)
    _, _, v_rows = layer.query_stats()
    dout = torch.from_numpy(synth.plain(91, 0, (B, Hq, D), 0.0, 1.0, True)).view(torch.bfloat16).to(dev)
    layer.zero_grad()
    dq = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    for _ in range(3):
        layer.decode_backward(q, dout, sel, dq)
        layer.tree_backward()
    t_dec, t_tree = [], []
    for _ in range(10):
        for fn, acc in ((lambda: layer.decode_backward(q, dout, sel, dq), t_dec), (layer.tree_backward, t_tree)):
            flush.fill_(7.0)
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b_.record(stream)
            torch.cuda.synchronize(dev)
            acc.append(a.elapsed_time(b_))
    layer.check()
    lengths = layer.lengths()
    b = w.branching
    # propagation: every token's key read and dk, dv read-modify-written
    # (fp32); per level the node accumulators read, the inner levels' h and
    # s written and their children's keys read; the accumulators cleared
    tree_bytes = 0
    for L in lengths:
        tree_bytes += H * L * (D * es + 4 * D * 4)
        for j in range(1, J_cap + 1):
            nj = -(-L // b ** j)
            tree_bytes += H * nj * 2 * D * 4 * 2  # accumulators read + cleared
            if j >= 2:
                tree_bytes += H * (nj * 2 * D * 4 + (-(-L // b ** (j - 1))) * D * es)
    entries = int(sum(v_rows))
    dec_bytes = entries * (2 * D * es + 4 * D * 4) + B * Hq * D * (2 * es + 4)
    hbm = float(peaks["hbm_gbs"])
    dec_ms, tree_ms = statistics.median(t_dec), statistics.median(t_tree)
    res = {"decode_backward_us": dec_ms * 1e3, "tree_backward_ms": tree_ms,
           "queries": B * Hq, "entries": entries,
           "roofline": {"kernel": "bwd_prop_kernel (all levels)", "bound": "hbm",
                        "achieved": tree_bytes / (tree_ms / 1e3) / 1e9, "peak": hbm, "unit": "GB/s",
                        "frac": tree_bytes / (tree_ms / 1e3) / 1e9 / hbm, "algorithmic_bytes": tree_bytes,
                        "traffic": kernel_traffic("bwd_prop_kernel", w.name)},
           "entry_gbs": dec_bytes / (dec_ms / 1e3) / 1e9,
           "how": "one decode query per sequence (its selections from recsa_decode), dout ~ N(0,1) bf16; "
                  "recsa_decode_backward and recsa_tree_backward timed separately, median of 10, L2 flushed"}
    del layer.dk, layer.dv, layer.dw, layer._bwd_scratch
    layer.dk = None
    torch.cuda.empty_cache()
    if with_cpu:
        import oracle

        L0 = w.length
        units = [(bb, h) for bb in range(B) for h in range(H)][:max(1, min(cpu_threads, B * H))]
        Wf = synth.as_f32(synth.workload_pooler(w))
        storage = oracle.STORE_BF16
        pool = oracle.pool(len(units))
        qh = q.view(torch.int16).cpu().numpy()
        dh = dout.float().cpu().numpy().astype(np.float64)

        def prep(bh):
            bb, h = bh
            tr = oracle.Tree(D, b, L0, storage).build(kv_host[0][bb, h], kv_host[1][bb, h], L0, Wf)
            return tr

        trees = list(pool.map(prep, units))

        def grad(i):
            bb, h = units[i]
            qu = synth.as_f32(np.ascontiguousarray(qh[bb, h * G:(h + 1) * G]))
            return oracle.query_grad(trees[i].K, trees[i].V, kv_host[0][bb, h], kv_host[1][bb, h], L0, qu,
                                     dh[bb, h * G:(h + 1) * G], Wf, D, b, w.k, G, w.rope_base)

        t0 = time.perf_counter()
        list(pool.map(grad, range(len(units))))
        dt = time.perf_counter() - t0
        pool.shutdown()
        res["cpu_baseline"] = {"value": len(units) * G / dt, "unit": "query-gradients/s", "cores": len(units),
                               "kind": "oracle",
                               "sample": f"oracle.query_grad of one query per unit on {len(units)} units "
                                         f"(L = {L0}) in parallel, trees built before timing"}
        res["gpu_query_gradients_s"] = B * Hq / ((dec_ms + tree_ms) / 1e3)
    return res


def distill_token_pass_bytes(H, lengths, D, b, J_cap, es):
    """Bytes of the distillation step's passes over every token, which
    dominate it: the pooler-only propagation (every token's key read; per
    level the node accumulators read and cleared, the inner levels' h and s
    written and their children's keys read) and the rebuild of every level
    (the tokens' keys and values read, the level-1 keys, values and fp32 value
    sums written; each upper level reading its children's keys and value sums
    and writing its own). The decode, loss, entry gradients and update (about
    0.1 GB at 524K x 4) are not counted."""
    total = 0
    for L in lengths:
        total += H * L * D * es
        for j in range(1, J_cap + 1):
            nj = -(-L // b ** j)
            total += H * nj * 2 * D * 4 * 2
            if j >= 2:
                total += H * (nj * 2 * D * 4 + (-(-L // b ** (j - 1))) * D * es)
        total += H * (2 * L * D * es + (-(-L // b)) * D * (2 * es + 4))
        for j in range(2, J_cap + 1):
            nj, nprev = -(-L // b ** j), -(-L // b ** (j - 1))
            total += H * (nprev * D * (es + 4) + nj * D * (2 * es + 4))
    return total


def measure_distill(layer, w, q, dev, flush, build_ms, peaks, kv_host, cpu_threads, with_cpu):
    """One distillation step of the pooler (recsa_distill_step: forward,
    squared error, the pooler's gradient, update, tree rebuild) on the
    layer's current cache, median of 5 after 2 warm-ups, L2 flushed before
    each. The dense targets are synthetic N(0, 0.1^2) stand-ins (the step's
    cost does not depend on them); lr = 0 leaves the pooler, so the tree the
    rest of the run uses is unchanged. Beside it, the oracle doing the same
    step (tree build, query, gradient) for a sample of units on the host."""
    B, H, Hq, D, G = w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim, w.group
    stream = torch.cuda.current_stream(dev)
    target = torch.from_numpy(synth.plain(92, 0, (B, Hq, D), 0.0, 0.1)).to(dev)
    for _ in range(2):
        layer.distill_step(q, target, 0.0)
    ts = []
    for _ in range(5):
        flush.fill_(8.0)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        loss = layer.distill_step(q, target, 0.0)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        ts.append(a.elapsed_time(b_))
    layer.check()
    ms = statistics.median(ts)
    pass_bytes = distill_token_pass_bytes(H, layer.lengths(), D, w.branching, layer.tree_shape()[0], 2)
    hbm = float(peaks["hbm_gbs"])
    res = {"step_ms": ms, "tree_rebuild_ms_alone": build_ms, "queries": B * Hq, "loss": float(loss.item()),
           "roofline": {"kernel": "recsa_distill_step (its passes over every token)", "bound": "hbm",
                        "achieved": pass_bytes / (ms / 1e3) / 1e9, "peak": hbm, "unit": "GB/s",
                        "frac": pass_bytes / (ms / 1e3) / 1e9 / hbm, "algorithmic_bytes": pass_bytes,
                        "traffic": None},
           "how": "recsa_distill_step on the decode workload's cache, one query per sequence, synthetic targets, "
                  "lr 0; median of 5, L2 flushed"}
    del layer._distill_scratch
    layer._distill_scratch = None
    torch.cuda.empty_cache()
    if with_cpu:
        import oracle

        L0, b = w.length, w.branching
        units = [(bb, h) for bb in range(B) for h in range(H)][:max(1, min(cpu_threads, B * H))]
        Wf = synth.as_f32(synth.workload_pooler(w))
        qh = q.view(torch.int16).cpu().numpy()
        th = target.cpu().numpy().astype(np.float64)
        n = B * Hq * D

        def unit(bh):
            bb, h = bh
            Kt, Vt = kv_host[0][bb, h], kv_host[1][bb, h]
            tr = oracle.Tree(D, b, L0, oracle.STORE_BF16).build(Kt, Vt, L0, Wf)
            qu = synth.as_f32(np.ascontiguousarray(qh[bb, h * G:(h + 1) * G]))
            r = oracle.query_tree(tr, Kt, Vt, qu, w.k, G, w.rope_base)
            diff = r["out"] - th[bb, h * G:(h + 1) * G]
            return oracle.query_grad(tr.K, tr.V, Kt, Vt, L0, qu, 2 * diff / n, Wf, D, b, w.k, G, w.rope_base)["dW"]

        pool = oracle.pool(len(units))
        t0 = time.perf_counter()
        list(pool.map(unit, units))
        dt = time.perf_counter() - t0
        pool.shutdown()
        res["cpu_baseline"] = {"value": len(units) / dt, "unit": "units/s", "cores": len(units), "kind": "oracle",
                               "sample": f"the step's tree build, query and gradient for {len(units)} units "
                                         f"(L = {L0}) in parallel (the update itself omitted)"}
        res["gpu_units_s"] = B * H / (ms / 1e3)
    return res


def measure_cluster(layer, w, q, dev, flush, peaks, kv_host, steps, cpu_threads, with_cpu):
    """LSA-style variant on the decode workload's tokens: recsa_cluster_load
    (the clustered order of every unit's first L tokens under seeded learned
    directions, the rows placed in that order, the tree built), median of 3
    after a warm-up, L2 flushed; then decode steps (recsa_decode) over the
    clustered tree. Roofline of the clustering: the bytes its kernels move by
    design (per level the key rows read and the records written, every pass of
    the sorting network reading and writing all records, the rows placed)
    against the measured copy bandwidth. Beside it, the oracle computing the
    same order for a sample of units on the host cores."""
    B, H, D = w.batch, w.n_kv_heads, w.head_dim
    L0, b = w.length, w.branching
    stream = torch.cuda.current_stream(dev)
    J_cap, _ = layer.tree_shape()
    Z = torch.from_numpy(synth.plain(903, 0, (J_cap, D), 0.0, 1.0, False)).to(dev)
    ksrc = layer.k_cache[:, :, :L0].contiguous()
    vsrc = layer.v_cache[:, :, :L0].contiguous()
    perm = torch.empty((B, H, layer.cfg.capacity), dtype=torch.int32, device=dev)
    scratch = torch.empty(layer.ctx.cluster_scratch_bytes(), dtype=torch.uint8, device=dev)
    layer.ctx.cluster_load(ksrc, vsrc, [L0] * B, Z, perm, scratch)
    ts = []
    for _ in range(3):
        flush.fill_(6.0)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        layer.ctx.cluster_load(ksrc, vsrc, [L0] * B, Z, perm, scratch)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        ts.append(a.elapsed_time(b_))
    layer.check()
    ms = statistics.median(ts)
    # the sorting network's own traffic (records of 24 bytes, all levels)
    J, _ = oracle_levels(L0, b)
    n = B * H * L0
    n_pad, TILE, es = 1024, 1024, 2
    while n_pad < n:
        n_pad <<= 1
    lg = n_pad.bit_length() - 1
    # first tile launch; per stage: the global distances two per pass, then a tile launch
    passes = 1 + sum((s_ - 10 + 1) // 2 + 1 for s_ in range(11, lg + 1))
    level_bytes = n * D * es + n_pad * 24 * 2 + passes * n_pad * 48
    cl_bytes = J * level_bytes + n * (4 * D * es + 4)
    gbs = cl_bytes / (ms / 1e3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    # decode over the clustered tree (the fused append would add its token
    # outside the clustered order; decode alone, on the clustered cache)
    out = torch.empty((B, w.n_q_heads, D), dtype=torch.bfloat16, device=dev)
    rows = torch.zeros((B, H, 2), dtype=torch.int64, device=dev)
    for _ in range(3):
        layer.decode(q, out)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for i in range(steps):
        flush.fill_(7.0)
        evs[i][0].record(stream)
        layer.decode(q, out, rows_out=rows if i == 0 else None)
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    layer.check()
    dms = [e[0].elapsed_time(e[1]) for e in evs]
    rows_np = rows.cpu().numpy()
    res = {"workload": f"{B} sequences x {H} KV heads x {L0} tokens (the decode workload's keys), b = {b}",
           "cluster_ms": ms, "levels": J, "records": n,
           "roofline": {"kernel": "recsa_cluster_load (all its launches)", "bound": "hbm", "achieved": gbs,
                        "peak": hbm, "unit": "GB/s", "frac": gbs / hbm, "algorithmic_bytes": cl_bytes,
                        "sort_passes_per_level": passes, "traffic": None},
           "decode_ms": sum(dms) / steps, "decode_query_tok_s": B / (sum(dms) / steps / 1e3),
           "rows_per_query": {"k_rows": float(rows_np[..., 0].mean()), "v_rows": float(rows_np[..., 1].mean())},
           "how": "recsa_cluster_load median of 3 (L2 flushed), then recsa_decode steps over the clustered tree"}
    del ksrc, vsrc, scratch
    torch.cuda.empty_cache()
    if with_cpu:
        import oracle

        units = [(bb, h) for bb in range(B) for h in range(H)][:max(1, min(cpu_threads, B * H))]
        Zh = Z.cpu().numpy()
        pool = oracle.pool(len(units))
        t0 = time.perf_counter()
        list(pool.map(lambda bh: oracle.cluster_order(kv_host[0][bh[0], bh[1]], L0, b, Zh), units))
        dt = time.perf_counter() - t0
        pool.shutdown()
        res["cpu_baseline"] = {"value": len(units) * L0 / dt, "unit": "tokens/s", "cores": len(units), "kind": "oracle",
                               "sample": f"oracle.cluster_order of {len(units)} units (L = {L0}) in parallel"}
        res["gpu_tokens_s"] = n / (ms / 1e3)
    return res


def oracle_levels(T, b):
    """Levels of the tree over T tokens (the first j >= 1 with
    ceil(T / b^j) <= b) and the level sizes."""
    n, j = [T], 0
    while True:
        j += 1
        n.append(-(-n[-1] // b))
        if n[-1] <= b:
            return j, n


# -------------------------------------------------------------------- main


def main():
    args = parse()
    world, rank, local = dist_setup(args.gpus)
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w, world, rank)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return

    from hierarchical_sparse_attention_tree_b200 import RecsaLayer, dense_decode, dense_decode_scratch_bytes

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = measured_peaks()
    if args.prefill_only:  # profiling: the chunked prefill alone, one JSON line of its own
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        res = measure_prefill(args.prefill_workload, dev, flush, peaks, last_chunks=args.prefill_last,
                              with_dense=not args.no_dense)
        if rank == 0:
            print(json.dumps({"prefill": res, "peak_source": peak_src}), flush=True)
        return
    B, H, Hq, D = w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim
    L0 = w.length
    W_, K_ = args.warmup, args.steps
    n_total = 2 * W_ + 3 * K_ + 30  # decode steps, split and append steps, e2e loops
    cap = L0 + n_total
    seq_off = rank_sequences(rank, B)
    bf = torch.bfloat16

    # ---- inputs: host (pinned), then resident in HBM
    t_gen = time.perf_counter()
    # the cache (4.3 GB of keys and values per rank at 524K x 4) is uploaded
    # once, outside every timed region: pageable host memory, so that eight
    # ranks do not pin 70 GB; the per-step inputs below are pinned
    Kh = torch.empty((B, H, cap, D), dtype=torch.int16)
    Vh = torch.empty((B, H, cap, D), dtype=torch.int16)
    _, _, runs = synth.cache_arrays(w, cap, seq_offset=seq_off, out=(Kh.numpy(), Vh.numpy()))
    Wp = synth.workload_pooler(w)
    q_h = torch.from_numpy(np.stack([synth.decode_queries(w, runs, s, L0 + s + 1, seq_off) for s in range(n_total)]))
    q_h = q_h.view(bf).pin_memory()                                        # [S][B][Hq][D]
    kn_h = Kh[:, :, L0:L0 + n_total].permute(2, 0, 1, 3).contiguous().view(bf).unsqueeze(2).pin_memory()
    vn_h = Vh[:, :, L0:L0 + n_total].permute(2, 0, 1, 3).contiguous().view(bf).unsqueeze(2).pin_memory()
    gen_s = time.perf_counter() - t_gen                                    # kn_h: [S][B][1][H][D]

    layer = RecsaLayer(B, H, Hq, D, w.branching, w.k, cap, torch.from_numpy(Wp).view(bf).to(dev), dtype=bf,
                       rope_base=w.rope_base, device=dev)
    layer.k_cache[:, :, :L0].copy_(Kh[:, :, :L0].view(bf))
    layer.v_cache[:, :, :L0].copy_(Vh[:, :, :L0].view(bf))
    q_d, kn_d, vn_d = q_h.to(dev), kn_h.to(dev), vn_h.to(dev)
    out = torch.empty((B, Hq, D), dtype=bf, device=dev)
    rows = torch.zeros((K_, B, H, 2), dtype=torch.int64, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    # ---- tree build, timed on its own: a first build (which also loads the
    # kernels), then the same build again, timed (same result), L2 flushed
    layer.ctx.build_tree([L0] * B)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush.fill_(1.0)
    e0.record(stream)
    layer.ctx.build_tree([L0] * B)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    layer.check()
    build_ms = e0.elapsed_time(e1)
    es = 2  # bf16
    n1 = -(-L0 // w.branching)
    build_bytes = B * H * (2 * L0 * D * es + n1 * D * (2 * es + 4))
    for j in range(2, layer.tree_shape()[0] + 1):
        nj = -(-L0 // w.branching ** j)
        nprev = -(-L0 // w.branching ** (j - 1))
        build_bytes += B * H * (nprev * D * (es + 4) + nj * D * (2 * es + 4))

    # ---- device-resident decode steps: warm-up, then K timed steps. One
    # step = append one token per sequence + one decode query per sequence,
    # one launch (recsa_append_decode), bracketed by two events.
    def step(s, ev=None, rows_out=None):
        if ev is not None:
            ev[0].record(stream)
        layer.append_decode(kn_d[s], vn_d[s], q_d[s], out, rows_out=rows_out)
        if ev is not None:
            ev[1].record(stream)

    s_idx = 0
    for _ in range(W_):
        flush.fill_(float(s_idx))
        step(s_idx)
        s_idx += 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_)]
    torch.cuda.synchronize(dev)
    # clock sampling starts with ~0.3 s of decode-only launches (the tree is not
    # changed), so the samples see this load; then the timed region
    clocks = ClockSampler(dev.index)
    t_settle = time.perf_counter()
    while time.perf_counter() - t_settle < args.settle_s:
        for _ in range(32):
            layer.decode(q_d[s_idx], out)
        torch.cuda.synchronize(dev)
    barrier(world, local)
    torch.cuda.synchronize(dev)
    t_wall = time.perf_counter()
    for i in range(K_):
        flush.fill_(float(s_idx))
        step(s_idx, evs[i], rows[i])
        s_idx += 1
    torch.cuda.synchronize(dev)
    wall_s = time.perf_counter() - t_wall
    barrier(world, local)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    layer.check()
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    total_s = max_over_ranks(sum(step_ms) / 1e3, world)
    value = aggregate_rate(world, B, K_, total_s)
    rows_np = rows.cpu().numpy()  # K and V rows each fused step's descent read

    # ---- for the record: the decode kernel alone (K launches on the current
    # tree), the append alone, and the step as two launches
    dev_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_)]
    for i in range(K_):
        flush.fill_(3.0)
        dev_ev[i][0].record(stream)
        layer.decode(q_d[i % n_total], out)
        dev_ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    layer.check()
    dec_ms = [e[0].elapsed_time(e[1]) for e in dev_ev]
    split_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(16)]
    for i in range(16):
        flush.fill_(5.0)
        split_ev[i][0].record(stream)
        layer.append(kn_d[s_idx], vn_d[s_idx])
        layer.decode(q_d[s_idx], out)
        split_ev[i][1].record(stream)
        s_idx += 1
    torch.cuda.synchronize(dev)
    split_ms = [e[0].elapsed_time(e[1]) for e in split_ev]
    # append alone, for the record (appends K more tokens)
    app_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(8)]
    for i in range(8):
        flush.fill_(4.0)
        app_ev[i][0].record(stream)
        layer.append(kn_d[s_idx], vn_d[s_idx])
        app_ev[i][1].record(stream)
        s_idx += 1
    torch.cuda.synchronize(dev)
    app_ms = [e[0].elapsed_time(e[1]) for e in app_ev]

    # roofline of the fused step kernel: algorithmic bytes per launch = the
    # gathered K/V rows + q + out, plus the append (new token row; per level
    # the right-edge node K, V, fp32 value sum written and prefix sums read
    # and written; the pooler once)
    J_cap = layer.tree_shape()[0]
    app_bytes = B * H * (2 * D * es + J_cap * D * (2 * es + 4 + 16)) + D * D * es
    dec_bytes = int(rows_np.sum()) * D * es + K_ * (2 * B * Hq * D * es + app_bytes)
    dec_bytes_per_launch = dec_bytes / K_
    hbm = float(peaks["hbm_gbs"])
    dec_avg_s = sum(step_ms) / K_ / 1e3
    achieved = dec_bytes_per_launch / dec_avg_s / 1e9

    # ---- end to end through the public API: every step's q, k_new, v_new
    # arrive as one pinned host record and cross in one copy; the output goes
    # back to pinned host memory. Double-buffered: step s+1's record uploads
    # on a side stream while step s's kernel runs, and step s's output copies
    # back on a third stream. Timed from the first upload to the last
    # download (events on the compute stream, which waits for the others),
    # with no L2 flush between steps (a flush would sit inside the region);
    # the same loop with device-resident inputs and no copies is timed the
    # same way beside it.
    e2e = None
    if not args.no_e2e:
        nq, nkv = q_h[0].numel(), kn_h[0].numel()
        rec_h = torch.cat([q_h.reshape(n_total, -1), kn_h.reshape(n_total, -1), vn_h.reshape(n_total, -1)],
                          dim=1).pin_memory()
        rec_d = [torch.empty(nq + 2 * nkv, dtype=bf, device=dev) for _ in range(2)]
        views = [(r[:nq].view(q_d[0].shape), r[nq:nq + nkv].view(kn_d[0].shape), r[nq + nkv:].view(vn_d[0].shape))
                 for r in rec_d]
        outs = [torch.empty((B, Hq, D), dtype=bf, device=dev) for _ in range(2)]
        out_h = [torch.empty((B, Hq, D), dtype=bf).pin_memory() for _ in range(2)]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_loop(s0, n, copies=True):
            ready = [torch.cuda.Event() for _ in range(2)]
            used = [torch.cuda.Event() for _ in range(2)]
            copied = [torch.cuda.Event() for _ in range(2)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            up.wait_event(t0)
            down.wait_event(t0)
            if copies:
                with torch.cuda.stream(up):
                    rec_d[0].copy_(rec_h[s0], non_blocking=True)
                    ready[0].record(up)
            for i in range(n):
                cur, nxt = i % 2, (i + 1) % 2
                if copies:
                    if i + 1 < n:
                        with torch.cuda.stream(up):
                            if i >= 1:
                                up.wait_event(used[nxt])  # step i - 1 is done with that record
                            rec_d[nxt].copy_(rec_h[s0 + i + 1], non_blocking=True)
                            ready[nxt].record(up)
                    stream.wait_event(ready[cur])
                    if i >= 2:
                        stream.wait_event(copied[cur])  # step i - 2's output is back on the host
                    qb, kb, vb = views[cur]
                    layer.append_decode(kb, vb, qb, outs[cur])
                    used[cur].record(stream)
                    with torch.cuda.stream(down):
                        down.wait_event(used[cur])
                        out_h[cur].copy_(outs[cur], non_blocking=True)
                        copied[cur].record(down)
                else:
                    layer.append_decode(kn_d[s0 + i], vn_d[s0 + i], q_d[s0 + i], outs[cur])
            stream.wait_stream(up)
            stream.wait_stream(down)
            t1.record(stream)
            return t0, t1

        e2e_loop(s_idx, W_)
        s_idx += W_
        torch.cuda.synchronize(dev)
        barrier(world, local)
        t0, t1 = e2e_loop(s_idx, K_)
        s_idx += K_
        torch.cuda.synchronize(dev)
        barrier(world, local)
        e2e_s = max_over_ranks(t0.elapsed_time(t1) / 1e3, world)
        torch.cuda.synchronize(dev)
        t0, t1 = e2e_loop(s_idx, K_, copies=False)
        s_idx += K_
        torch.cuda.synchronize(dev)
        same_loop_s = max_over_ranks(t0.elapsed_time(t1) / 1e3, world)
        e2e = {"value": aggregate_rate(world, B, K_, e2e_s), "unit": "query-tok/s",
               "h2d_bytes_per_step": int(rec_h[0].numel() * es), "d2h_bytes_per_step": int(out_h[0].numel() * es),
               "device_same_loop": aggregate_rate(world, B, K_, same_loop_s),
               "how": "per step: one pinned host record [q | k_new | v_new] copied in (side stream, one step "
                      "ahead), recsa_append_decode, the output copied back to pinned host memory (third stream); "
                      "timed from the first upload to the last download, no L2 flush between steps; "
                      "device_same_loop = the same loop on device-resident inputs, no copies"}
        layer.check()

    # ---- dense flash-decode comparator on the same cache
    dense = None
    if not args.no_dense:
        Ld = layer.lengths()[0]
        scratch = torch.empty(dense_decode_scratch_bytes(B, Hq, D), dtype=torch.uint8, device=dev)
        dout = torch.empty_like(out)
        for _ in range(3):
            dense_decode(layer.k_cache, layer.v_cache, q_d[0], dout, Ld, scratch)
        dms = []
        for _ in range(10):
            flush.fill_(2.0)
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            dense_decode(layer.k_cache, layer.v_cache, q_d[0], dout, Ld, scratch)
            b_.record(stream)
            torch.cuda.synchronize(dev)
            dms.append(a.elapsed_time(b_))
        dmed = statistics.median(dms)
        dbytes = 2 * B * H * Ld * D * es
        dense = {"ms": dmed, "query_tok_s": B / (dmed / 1e3), "gbs": dbytes / (dmed / 1e3) / 1e9,
                 "frac_hbm": dbytes / (dmed / 1e3) / 1e9 / hbm, "length": Ld,
                 "recsa_step_speedup": dmed / (sum(step_ms) / K_)}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, one GPU only):
    # decode steps of every sequence and KV head, on all host cores
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        Kn, Vn = Kh.numpy(), Vh.numpy()
        done, dt, toks, used = oracle_decode_steps(w, Kn, Vn, Wp, runs, L0, 64, args.cpu_seconds, list(range(B)),
                                                   threads)
        cpu = {"value": toks / dt, "unit": "query-tok/s", "cores": used, "kind": "oracle",
               "sample": f"{done} decode steps of all {B} sequences x {H} KV heads ({B * H} units in parallel): "
                         "refresh of the nodes the new token touched + one query per unit, fp64; trees built and "
                         "queries generated before timing"}

    backward = None
    if not args.no_backward:
        backward = measure_backward(layer, w, q_d[0], dev, flush, peaks, (Kh.numpy(), Vh.numpy()),
                                    os.cpu_count() or 1, rank == 0 and world == 1 and not args.no_cpu_baseline)

    distill = None
    if not args.no_distill:
        distill = measure_distill(layer, w, q_d[0], dev, flush, build_ms, peaks, (Kh.numpy(), Vh.numpy()),
                                  os.cpu_count() or 1, rank == 0 and world == 1 and not args.no_cpu_baseline)

    cluster = None
    if not args.no_cluster:
        cluster = measure_cluster(layer, w, q_d[0], dev, flush, peaks, (Kh.numpy(), Vh.numpy()), 32,
                                  os.cpu_count() or 1, rank == 0 and world == 1 and not args.no_cpu_baseline)

    prefill = None
    if not args.no_prefill:
        prefill = measure_prefill(args.prefill_workload, dev, flush, peaks)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "query-tok/s", "n_gpus": world, "steps": K_, "warmup": W_,
            "ms_per_step": 1e3 * total_s / K_, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "L": L0, "batch_per_gpu": B, "n_q_heads": Hq, "n_kv_heads": H,
                       "head_dim": D, "branching": w.branching, "k": w.k,
                       "step": "recsa_append_decode: append 1 token/seq + 1 decode query/seq, one launch",
                       "l2": "flushed between steps (256 MB write, outside the events)",
                       "value_is": "decode query-tok/s; prefill tok/s under 'prefill'"},
            "roofline": {"kernel": "decode_kernel", "bound": "hbm", "achieved": achieved, "peak": hbm,
                         "unit": "GB/s", "frac": achieved / hbm, "peak_source": peak_src,
                         "traffic": kernel_traffic("decode_kernel", w.name),
                         "algorithmic_bytes_per_launch": dec_bytes_per_launch, "launch_ms": dec_avg_s * 1e3},
            "append_ms": sum(app_ms) / len(app_ms), "decode_ms": sum(dec_ms) / K_,
            "split_step_ms": sum(split_ms) / len(split_ms),
            "rows_per_query": {"k_rows": float(rows_np[..., 0].mean()), "v_rows": float(rows_np[..., 1].mean())},
            "build_tree": {"ms": build_ms, "gbs": build_bytes / (build_ms / 1e3) / 1e9,
                           "frac_hbm": build_bytes / (build_ms / 1e3) / 1e9 / hbm},
            "e2e": e2e, "gpu_launches": K_, "clocks": clk, "dense_decode": dense, "cpu_baseline": cpu,
            "wall_s_timed_loop": wall_s, "input_gen_s": gen_s, "prefill": prefill, "backward": backward,
            "distill": distill, "cluster": cluster,
        }
        print(json.dumps(line), flush=True)
    layer.close()
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
