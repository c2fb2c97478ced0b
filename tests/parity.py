"""Helpers that compare the CUDA path with the fp64 oracle (tests only)."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
import synth

NEAR_TIE = 1e-4  # oracle margin S_(k) - S_(k+1) below which a query is a near tie


def to_dev(a: np.ndarray, bf16: bool, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if bf16:
        t = t.view(torch.bfloat16)
    return t.to(device)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def storage_of(bf16: bool) -> int:
    return oracle.STORE_BF16 if bf16 else oracle.STORE_F32


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(x)
    a = np.where(a < 2.0 ** -126, 2.0 ** -126, a)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def compare_nodes(gpu: np.ndarray, ref: np.ndarray, bf16: bool, atol=0.0):
    """Returns (ok, n_differing). bf16: |diff| <= 1 ulp of the larger
    magnitude + atol; fp32: |diff| <= 2^-20 |ref| + atol. atol carries the
    fp32 rounding bound of the GPU's own arithmetic where it matters."""
    diff = np.abs(gpu - ref)
    if bf16:
        ulp = bf16_ulp(np.maximum(np.abs(gpu), np.abs(ref)))
        return bool((diff <= ulp * 1.0000001 + atol).all()), int((diff > 0).sum())
    ok = diff <= 2.0 ** -20 * np.abs(ref) + atol
    return bool(ok.all()), int((~ok).sum())


def pooled_key_bound(below: np.ndarray, b: int, W: np.ndarray) -> np.ndarray:
    """fp32 rounding bound of W * mean(children) computed in fp32 with d-term
    sums: 2 d 2^-24 * sum_c |W_rc| |mean_c| per output (Higham's gamma_d,
    doubled for the mean)."""
    n, d = below.shape
    groups = -(-n // b)
    means = np.stack([np.abs(below[m * b:(m + 1) * b]).mean(0) for m in range(groups)])
    return 2 * (d + b) * 2.0 ** -24 * (means @ np.abs(W.astype(np.float64)).T)


def mean_value_bound(V_tok: np.ndarray, span: int) -> np.ndarray:
    """Rounding allowance of an fp32 running sum of cnt token values divided
    by cnt: 8 sqrt(cnt) 2^-24 rms(v) per node (the random-walk size of the
    sum's rounding errors, with margin; a dropped or doubled token moves the
    mean by about rms(v)/cnt, far above this for cnt <= 2^20)."""
    L = V_tok.shape[0]
    n = -(-L // span)
    out = np.empty((n, 1))
    for m in range(n):
        blk = V_tok[m * span:min((m + 1) * span, L)].astype(np.float64)
        out[m, 0] = 8 * np.sqrt(len(blk)) * 2.0 ** -24 * np.sqrt((blk ** 2).mean())
    return out


def unit_tokens(K: np.ndarray, b: int, h: int, L: int):
    return K[b, h, :L]


def gpu_tree_unit(layer, b: int, h: int, J: int, L: int):
    """GPU node arrays of one unit, levels 1..J, as fp64 numpy (rows < n_j)."""
    Ks, Vs = [None], [None]
    for j in range(1, J + 1):
        n = -(-L // layer.cfg.branching ** j)
        kj, vj, _ = layer.level(j)
        Ks.append(to_f64(kj[b, h, :n]))
        Vs.append(to_f64(vj[b, h, :n]))
    return Ks, Vs


def oracle_query(tree_K, tree_V, K, V, b, h, L, q_unit, w, Kloc=None, Vloc=None):
    """q_unit: [G][d] float32."""
    return oracle.query(tree_K, tree_V, K[b, h], V[b, h], L, q_unit, w.head_dim, w.branching, w.k, w.group,
                        w.rope_base, Kloc, Vloc)


def q_unit(q: np.ndarray, b: int, h: int, G: int) -> np.ndarray:
    """Query heads of KV head h of sequence b, as float32 [G][d]."""
    return synth.as_f32(np.ascontiguousarray(q[b, h * G:(h + 1) * G]))


def first_tie_level(ref):
    """Highest level whose oracle margin S_(k) - S_(k+1) is below NEAR_TIE
    (the descent runs from level J down), or 0 if there is none. Selections
    at that level and below may legitimately differ from the oracle's."""
    for j in range(ref["J"], 0, -1):
        if ref["margin"][j - 1] < NEAR_TIE:
            return j
    return 0


def check_decode(gpu_out, gpu_sel, gpu_rows, ref, b, h, G, tol, report):
    """Compares one unit's decode with an oracle result. Levels above the
    first near tie must select exactly what the oracle selects; at and below
    it a different selection is counted as a near tie and the output is not
    compared. Where every level agrees (near tie or not) the output and the
    rows read are compared too."""
    J = ref["J"]
    tie = first_tie_level(ref)
    if tie:
        report["near_ties"] += 1
    for j in range(J, 0, -1):
        got = [x for x in gpu_sel[b, h, j - 1].tolist() if x >= 0]
        want = [x for x in ref["sel"][j - 1].tolist() if x >= 0]
        if got != want:
            if j <= tie:
                report["near_tie_sel_diff"] += 1
                return False
            report["sel_mismatch"] += 1
            report.setdefault("first_mismatch", (b, h, j, got, want))
            return False
    assert (gpu_sel[b, h, J:] == -1).all()
    err = np.abs(gpu_out[b, h * G:(h + 1) * G] - ref["out"]).max()
    report["max_abs"] = max(report["max_abs"], float(err))
    assert err <= tol, (b, h, err)
    assert tuple(gpu_rows[b, h]) == expected_rows(ref), (gpu_rows[b, h], expected_rows(ref))
    report["checked"] += 1
    return True


def same_selection(ref_a, ref_b):
    """True if two oracle results keep the same nodes at every level."""
    if ref_a["J"] != ref_b["J"]:
        return False
    return all((ref_a["sel"][j] == ref_b["sel"][j]).all() for j in range(ref_a["J"]))


def expected_rows(ref):
    """(K rows, V rows) the CUDA path reads for this query: the oracle's
    counts, less the top levels that keep every candidate (at most k of them:
    margin = inf), whose keys need not be read because nothing is selected
    among them."""
    skipped = 0
    for j in range(ref["J"], 0, -1):
        if not np.isinf(ref["margin"][j - 1]):
            break
        skipped += int((ref["sel"][j - 1] >= 0).sum())
    return ref["k_rows"] - skipped, ref["v_rows"]


def new_report():
    return {"queries": 0, "checked": 0, "near_ties": 0, "near_tie_sel_diff": 0, "sel_mismatch": 0,
            "node_rounding_flips": 0, "max_abs": 0.0}


def merge_reports(total, rep):
    for key, v in rep.items():
        if key == "max_abs":
            total[key] = max(total[key], v)
        elif isinstance(v, int):
            total[key] = total.get(key, 0) + v
    return total


def record(test: str, config: str, mode: str, rep) -> None:
    """Appends one parity count record (JSON line) to the file named by
    RECSA_PARITY_REPORT, if set: near ties and free-running mismatches are
    counted and kept, not only printed."""
    path = os.environ.get("RECSA_PARITY_REPORT")
    line = {"test": test, "config": config, "mode": mode,
            **{k: v for k, v in rep.items() if k != "first_mismatch"}}
    print(json.dumps(line))
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(line) + "\n")
