"""fp64 CPU oracle for RecSA tree sparse attention — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package. It shares no code with the CUDA path.
The arithmetic lives in ``recsa_oracle.c`` (plain C, fp64); this module
compiles it and marshals numpy arrays. ctypes drops the GIL during each call,
so independent queries run in parallel from a thread pool.

Method source: "Recursive Sparse Attention: Million-Token Length
Extrapolation at Logarithmic Cost" (arXiv 2611.07232), abstract, and the
kongchang.com article on RecSA ("Core Idea", "Position Encoding"); the
readings of open points are listed in ``recsa_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "recsa_oracle.c")
_HDR = os.path.join(_HERE, "recsa_oracle.h")
_LIB = os.path.join(_HERE, "liborecsa.so")
_lock = threading.Lock()
_lib = None

MAXLEV = 40
STORE_F32, STORE_BF16, STORE_F64 = 0, 1, 2


def build(force: bool = False) -> str:
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            i32, i64, dbl, vp = ctypes.c_int, ctypes.c_longlong, ctypes.c_double, ctypes.c_void_p
            lib.orc_levels.restype = i32
            lib.orc_levels.argtypes = [i64, i32, vp]
            lib.orc_round.restype = dbl
            lib.orc_round.argtypes = [dbl, i32]
            lib.orc_build.restype = i32
            lib.orc_build.argtypes = [vp, vp, i32, i64, i32, i32, vp, i32, i64, i32, vp, vp]
            lib.orc_pool_level.restype = i32
            lib.orc_pool_level.argtypes = [vp, i64, i32, i32, vp, i32, vp]
            lib.orc_query_grad.restype = i32
            lib.orc_query_grad.argtypes = [i32, i32, i32, i32, dbl, i64, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp,
                                           vp]
            lib.orc_query_grad_local.restype = i32
            lib.orc_query_grad_local.argtypes = [i32, i32, i32, i32, dbl, i64, vp, vp, vp, vp, i32, vp, vp, i64, vp,
                                                 vp, vp, vp, vp, vp, vp, vp, vp]
            lib.orc_cluster_order.restype = i32
            lib.orc_cluster_order.argtypes = [vp, i32, i64, i32, i32, vp, vp]
            lib.orc_query.restype = i32
            lib.orc_query.argtypes = [i32, i32, i32, i32, dbl, i64, vp, vp, vp, vp, i32, vp, vp, i64, vp, vp, vp, vp,
                                      vp]
            _lib = lib
    return _lib


def _tok(a: np.ndarray):
    """(array, tok_dtype): float32 rows or bf16 bit patterns (int16)."""
    if a.dtype == np.int16:
        return np.ascontiguousarray(a), 1
    return np.ascontiguousarray(a, dtype=np.float32), 0


def levels(T: int, b: int):
    """(J, [n_0, ..., n_J]) for the tree over T tokens."""
    n = np.zeros(MAXLEV + 1, dtype=np.int64)
    J = _load().orc_levels(T, b, n.ctypes.data)
    return J, [int(x) for x in n[: J + 1]]


def round_store(x: float, storage: int) -> float:
    return _load().orc_round(x, storage)


def pool_level(child_keys, b: int, W, storage: int) -> np.ndarray:
    """Keys of the level above, pooled from the given child keys (rows as
    stored): the pooler applied to the mean of each node's children."""
    ck = np.ascontiguousarray(child_keys, dtype=np.float64)
    n, d = ck.shape
    Wf = np.ascontiguousarray(W, dtype=np.float32)
    out = np.zeros((-(-n // b), d))
    if _load().orc_pool_level(ck.ctypes.data, n, d, b, Wf.ctypes.data, storage, out.ctypes.data) != 0:
        raise ValueError("bad arguments")
    return out


def _ptr_array(arrs):
    p = (ctypes.c_void_p * (MAXLEV + 1))()
    for j, a in enumerate(arrs):
        p[j] = a.ctypes.data if a is not None else None
    return p


class Tree:
    """Node arrays (fp64, as stored) of one unit's tree, levels 1..J_keep,
    sized for `capacity` tokens."""

    def __init__(self, d: int, b: int, capacity: int, storage: int, J_keep: int = 0):
        self.d, self.b, self.storage = d, b, storage
        Jc, _ = levels(max(capacity, 1), b)
        self.J_keep = max(J_keep, Jc)
        self.K = [None]
        self.V = [None]
        n = max(capacity, 1)
        for _j in range(1, self.J_keep + 1):
            n = (n + b - 1) // b
            self.K.append(np.zeros((n, d)))
            self.V.append(np.zeros((n, d)))
        self.T = 0

    def build(self, Ktok, Vtok, T, W, t_from=0):
        """(Re)compute the nodes over tokens [0, T); t_from > 0 refreshes only
        the nodes whose tokens reach past t_from."""
        kt, dt = _tok(Ktok)
        vt, _ = _tok(Vtok)
        Wf = np.ascontiguousarray(W, dtype=np.float32)
        r = _load().orc_build(kt.ctypes.data, vt.ctypes.data, dt, T, self.d, self.b, Wf.ctypes.data, self.storage,
                              t_from, self.J_keep, _ptr_array(self.K), _ptr_array(self.V))
        if r < 0:
            raise MemoryError("oracle build failed")
        self.T = T
        return self


def build_tree(Ktok, Vtok, T, d, b, W, storage, capacity=None):
    return Tree(d, b, capacity or T, storage).build(Ktok, Vtok, T, W)


def query(tree_K, tree_V, Ktok, Vtok, T, q, d, b, k, G, rope_base, Kloc=None, Vloc=None):
    """One query of one unit. tree_K/tree_V: per-level node arrays (index 0
    unused), fp64 [>= n_j][d]. Ktok/Vtok: level-0 rows. Kloc/Vloc: local
    causal rows (prefill), or None. q: [G][d].
    Returns dict(out [G][d], sel [J][k], margin [J], k_rows, v_rows, J)."""
    lib = _load()
    kt, dt = _tok(Ktok)
    vt, _ = _tok(Vtok)
    nloc = 0
    kl = vl = None
    if Kloc is not None and len(Kloc):
        kl, dt2 = _tok(Kloc)
        vl, _ = _tok(Vloc)
        if dt2 != dt:
            raise ValueError("local tokens must have the cache's dtype")
        nloc = kl.shape[0]
    Jt, _ = levels(T, b)
    qf = np.ascontiguousarray(q, dtype=np.float32)
    if qf.dtype != np.float32:
        raise TypeError
    out = np.zeros((G, d))
    sel = np.full((max(Jt, 1), k), -1, dtype=np.int32)
    margin = np.zeros(max(Jt, 1))
    rows = np.zeros(2, dtype=np.int64)
    Kp = [None] + [np.ascontiguousarray(x, dtype=np.float64) for x in tree_K[1:Jt + 1]]
    Vp = [None] + [np.ascontiguousarray(x, dtype=np.float64) for x in tree_V[1:Jt + 1]]
    J = lib.orc_query(d, b, k, G, rope_base, T, _ptr_array(Kp), _ptr_array(Vp), kt.ctypes.data, vt.ctypes.data, dt,
                      kl.ctypes.data if kl is not None else None, vl.ctypes.data if vl is not None else None, nloc,
                      qf.ctypes.data, out.ctypes.data, sel.ctypes.data, margin.ctypes.data, rows.ctypes.data)
    if J < 0:
        raise ValueError("oracle query rejected its arguments")
    return dict(out=out, sel=sel[:J], margin=margin[:J], k_rows=int(rows[0]), v_rows=int(rows[1]), J=J)


def query_grad(tree_K, tree_V, Ktok, Vtok, T, q, dout, W, d, b, k, G, rope_base, Kloc=None, Vloc=None):
    """Gradients of one query with the selections held fixed: a decode query,
    or (Kloc, Vloc given) a prefill query with its chunk's own causal tokens.
    Returns dict(dq [G][d], dK [T][d], dV [T][d], dW [d][d]) in fp64, and
    dKloc, dVloc [nloc][d] for the local tokens."""
    if Kloc is not None and len(Kloc):
        return _query_grad_local(tree_K, tree_V, Ktok, Vtok, T, q, dout, W, d, b, k, G, rope_base, Kloc, Vloc)
    lib = _load()
    kt, dt = _tok(Ktok)
    vt, _ = _tok(Vtok)
    Jt, _ = levels(T, b)
    qf = np.ascontiguousarray(q, dtype=np.float32)
    do = np.ascontiguousarray(dout, dtype=np.float64)
    Wf = np.ascontiguousarray(W, dtype=np.float32)
    dq = np.zeros((G, d))
    dK = np.zeros((T, d))
    dV = np.zeros((T, d))
    dW = np.zeros((d, d))
    Kp = [None] + [np.ascontiguousarray(x, dtype=np.float64) for x in tree_K[1:Jt + 1]]
    Vp = [None] + [np.ascontiguousarray(x, dtype=np.float64) for x in tree_V[1:Jt + 1]]
    J = lib.orc_query_grad(d, b, k, G, rope_base, T, _ptr_array(Kp), _ptr_array(Vp), kt.ctypes.data, vt.ctypes.data,
                           dt, Wf.ctypes.data, qf.ctypes.data, do.ctypes.data, dq.ctypes.data, dK.ctypes.data,
                           dV.ctypes.data, dW.ctypes.data)
    if J < 0:
        raise ValueError("oracle gradient rejected its arguments")
    return dict(dq=dq, dK=dK, dV=dV, dW=dW, J=J)


def cluster_order(Ktok, T: int, b: int, Z) -> np.ndarray:
    """LSA-style clustered order of tokens [0, T) (reading R20 in
    recsa_oracle.c): int32 [T], the token index at each position. Ktok: the
    unit's keys [>= T][d] (float32, or bf16 bit patterns as int16); Z: the
    learned directions, float32 [>= levels(T, b)][d]."""
    lib = _load()
    Kt, dt = _tok(Ktok)
    Zf = np.ascontiguousarray(Z, dtype=np.float32)
    d = Kt.shape[-1]
    perm = np.zeros(T, dtype=np.int32)
    J = lib.orc_cluster_order(Kt.ctypes.data, dt, T, d, b, Zf.ctypes.data, perm.ctypes.data)
    if J < 0:
        raise ValueError("oracle clustered order rejected its arguments")
    return perm


def _query_grad_local(tree_K, tree_V, Ktok, Vtok, T, q, dout, W, d, b, k, G, rope_base, Kloc, Vloc):
    lib = _load()
    kt, dt = _tok(Ktok)
    vt, _ = _tok(Vtok)
    kl, dt2 = _tok(Kloc)
    vl, _ = _tok(Vloc)
    if dt2 != dt:
        raise ValueError("local tokens must have the cache's dtype")
    nloc = kl.shape[0]
    Jt, _ = levels(T, b)
    qf = np.ascontiguousarray(q, dtype=np.float32)
    do = np.ascontiguousarray(dout, dtype=np.float64)
    Wf = np.ascontiguousarray(W, dtype=np.float32)
    dq = np.zeros((G, d))
    dK, dV = np.zeros((max(T, 1), d)), np.zeros((max(T, 1), d))
    dKl, dVl = np.zeros((nloc, d)), np.zeros((nloc, d))
    dW = np.zeros((d, d))
    Kp = [None] + [np.ascontiguousarray(x, dtype=np.float64) for x in tree_K[1:Jt + 1]]
    Vp = [None] + [np.ascontiguousarray(x, dtype=np.float64) for x in tree_V[1:Jt + 1]]
    J = lib.orc_query_grad_local(d, b, k, G, rope_base, T, _ptr_array(Kp), _ptr_array(Vp), kt.ctypes.data,
                                 vt.ctypes.data, dt, kl.ctypes.data, vl.ctypes.data, nloc, Wf.ctypes.data,
                                 qf.ctypes.data, do.ctypes.data, dq.ctypes.data, dK.ctypes.data, dV.ctypes.data,
                                 dKl.ctypes.data, dVl.ctypes.data, dW.ctypes.data)
    if J < 0:
        raise ValueError("oracle gradient rejected its arguments")
    return dict(dq=dq, dK=dK[:T], dV=dV[:T], dW=dW, dKloc=dKl, dVloc=dVl, J=J)


def query_tree(tree: Tree, Ktok, Vtok, q, k, G, rope_base, Kloc=None, Vloc=None, T=None):
    return query(tree.K, tree.V, Ktok, Vtok, tree.T if T is None else T, q, tree.d, tree.b, k, G, rope_base, Kloc,
                 Vloc)


def pool(n_threads: int | None = None) -> ThreadPoolExecutor:
    """Thread pool for independent oracle calls (ctypes releases the GIL)."""
    return ThreadPoolExecutor(max_workers=n_threads or os.cpu_count() or 1)
