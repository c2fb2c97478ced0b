"""Seeded synthetic inputs for the RecSA tree-attention workloads.

Data generation only: nothing in this package computes any part of the
attention method. The arrays it returns feed both the CUDA library and the
CPU oracle. The generator itself is ``synth.c`` (counter-based splitmix64 and
Box-Muller, see its header); this module compiles it on first use and wraps it
with numpy.

bf16 arrays are returned as ``np.int16`` holding the bf16 bit patterns (numpy
has no bf16 type); ``bf16_to_f32`` widens them exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .workloads import WORKLOADS, Workload  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile libsynth.so next to its source (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            u64, i32, i64, dbl, vp = (ctypes.c_uint64, ctypes.c_int, ctypes.c_longlong, ctypes.c_double,
                                      ctypes.c_void_p)
            lib.synth_splitmix64_at.restype = u64
            lib.synth_splitmix64_at.argtypes = [u64, u64]
            lib.synth_uniform_at.restype = dbl
            lib.synth_uniform_at.argtypes = [u64, u64]
            lib.synth_normal_at.restype = dbl
            lib.synth_normal_at.argtypes = [u64, u64]
            lib.synth_stream.restype = u64
            lib.synth_stream.argtypes = [u64, u64, u64]
            lib.synth_runs.restype = i64
            lib.synth_runs.argtypes = [u64, i32, i64, i32, i32, vp, i64]
            lib.synth_keys.restype = None
            lib.synth_keys.argtypes = [u64, i32, i32, i32, i32, dbl, vp, i64, i64, i64, i64, i32, vp, i32]
            lib.synth_values.restype = None
            lib.synth_values.argtypes = [u64, i32, i32, i32, i64, i64, i64, i32, vp, i32]
            lib.synth_decode_query.restype = i64
            lib.synth_decode_query.argtypes = [u64, i32, i64, i64, i32, i32, i32, i32, dbl, vp, i64, i32, vp]
            lib.synth_prefill_queries.restype = None
            lib.synth_prefill_queries.argtypes = [u64, i32, i64, i64, i32, i32, i32, i32, dbl, vp, i64, i32, vp,
                                                  i32]
            lib.synth_pooler.restype = None
            lib.synth_pooler.argtypes = [u64, i32, i32, vp]
            lib.synth_plain.restype = None
            lib.synth_plain.argtypes = [u64, u64, i64, dbl, dbl, i32, vp]
            _lib = lib
    return _lib


def _threads(n: int | None) -> int:
    return n if n else max(1, os.cpu_count() or 1)


def _alloc(shape, bf16: bool):
    return np.empty(shape, dtype=np.int16 if bf16 else np.float32)


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (np.int16) to float32."""
    return (a.view(np.uint16).astype(np.uint32) << 16).view(np.float32)


def as_f32(a: np.ndarray) -> np.ndarray:
    return bf16_to_f32(a) if a.dtype == np.int16 else a


def splitmix64_at(base: int, i: int) -> int:
    return _load().synth_splitmix64_at(base, i)


def uniform_at(base: int, i: int) -> float:
    return _load().synth_uniform_at(base, i)


def normal_at(base: int, i: int) -> float:
    return _load().synth_normal_at(base, i)


def stream(seed: int, tag: int, a: int) -> int:
    return _load().synth_stream(seed, tag, a)


def runs(seed: int, seq: int, length: int, run_min: int, run_max: int) -> np.ndarray:
    """Starts of the runs covering [0, length), with `length` appended."""
    cap = length // max(run_min, 1) + 2
    out = np.empty(cap + 1, dtype=np.int64)
    n = _load().synth_runs(seed, seq, length, run_min, run_max, _ptr(out), cap)
    if n < 0:
        raise RuntimeError("run table overflow")
    return out[: n + 1].copy()


def keys(seed, seq, H, d, M, sigma, run_start, t0, t1, bf16, out=None, head_stride=None, nthreads=None):
    """Keys [H][t1-t0][d] of one sequence (or written into `out` with the
    given head stride in elements)."""
    if out is None:
        out = _alloc((H, t1 - t0, d), bf16)
        head_stride = (t1 - t0) * d
    rs = np.ascontiguousarray(run_start, dtype=np.int64)
    _load().synth_keys(seed, seq, H, d, M, sigma, _ptr(rs), len(rs) - 1, t0, t1, head_stride, int(bf16), _ptr(out),
                       _threads(nthreads))
    return out


def values(seed, seq, H, d, t0, t1, bf16, out=None, head_stride=None, nthreads=None):
    if out is None:
        out = _alloc((H, t1 - t0, d), bf16)
        head_stride = (t1 - t0) * d
    _load().synth_values(seed, seq, H, d, t0, t1, head_stride, int(bf16), _ptr(out), _threads(nthreads))
    return out


def decode_query(seed, seq, step, length, H, G, d, M, sigma, run_start, bf16):
    """Decode query [H*G][d] for `step`, aimed at a run that starts before
    `length`. Returns (query, planted run index)."""
    out = _alloc((H * G, d), bf16)
    rs = np.ascontiguousarray(run_start, dtype=np.int64)
    run = _load().synth_decode_query(seed, seq, step, length, H, G, d, M, sigma, _ptr(rs), len(rs) - 1, int(bf16),
                                     _ptr(out))
    return out, int(run)


def prefill_queries(seed, seq, t0, t1, H, G, d, M, sigma, run_start, bf16, nthreads=None):
    """Prefill queries [t1-t0][H*G][d]: each token aims at its own run."""
    out = _alloc((t1 - t0, H * G, d), bf16)
    rs = np.ascontiguousarray(run_start, dtype=np.int64)
    _load().synth_prefill_queries(seed, seq, t0, t1, H, G, d, M, sigma, _ptr(rs), len(rs) - 1, int(bf16), _ptr(out),
                                  _threads(nthreads))
    return out


def pooler(seed: int, d: int, bf16: bool) -> np.ndarray:
    out = _alloc((d, d), bf16)
    _load().synth_pooler(seed, d, int(bf16), _ptr(out))
    return out


def plain(seed: int, a: int, shape, mean=0.0, scale=1.0, bf16=False) -> np.ndarray:
    """Unstructured N(mean, scale^2) array of the given shape."""
    out = _alloc(shape, bf16)
    _load().synth_plain(seed, a, out.size, mean, scale, int(bf16), _ptr(out))
    return out


def cache_arrays(w, length: int, nthreads=None, seq_offset: int = 0, out=None):
    """Keys and values [B][H][length][d] of a workload (np.int16 bf16 bits or
    float32) and each sequence's run table. Sequence b uses generator
    sequence id seq_offset + b. `out` = (K, V) preallocated arrays, optional."""
    B, H, d = w.batch, w.n_kv_heads, w.head_dim
    K, V = out if out is not None else (_alloc((B, H, length, d), w.bf16), _alloc((B, H, length, d), w.bf16))
    run_tables = []
    for b in range(B):
        s = seq_offset + b
        rs = runs(w.seed, s, length, w.run_min, w.run_max)
        run_tables.append(rs)
        keys(w.seed, s, H, d, w.centroids, w.sigma_noise, rs, 0, length, w.bf16, out=K[b], head_stride=length * d,
             nthreads=nthreads)
        values(w.seed, s, H, d, 0, length, w.bf16, out=V[b], head_stride=length * d, nthreads=nthreads)
    return K, V, run_tables


def decode_queries(w, run_tables, step: int, length: int, seq_offset: int = 0):
    """Decode queries [B][H*G][d] for `step` with `length` cached tokens."""
    qs = [decode_query(w.seed, seq_offset + b, step, length, w.n_kv_heads, w.group, w.head_dim, w.centroids,
                       w.sigma_noise, run_tables[b], w.bf16)[0] for b in range(w.batch)]
    return np.stack(qs)


def workload_pooler(w):
    return pooler(w.seed, w.head_dim, w.bf16)
