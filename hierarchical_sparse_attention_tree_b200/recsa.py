"""ctypes binding of librecsa.so (C ABI in include/recsa.h).

Argument marshalling only: every step of the method runs in the library's
CUDA kernels. PyTorch provides device memory and streams. If the shared
library is missing this module raises; there is no other code path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librecsa.so")

OK, ERR_INVALID_ARG, ERR_CAPACITY, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE = range(6)
F32, BF16 = 0, 1
_TORCH_DTYPE = {F32: torch.float32, BF16: torch.bfloat16}

EXPORTS = [
    "recsa_workspace_bytes", "recsa_init", "recsa_init_paged", "recsa_build_tree", "recsa_append", "recsa_decode", "recsa_append_decode",
    "recsa_prefill_scratch_bytes", "recsa_prefill", "recsa_get_lengths", "recsa_tree_shape", "recsa_level_arrays",
    "recsa_query_stats", "recsa_check_device", "recsa_last_error", "recsa_destroy", "recsa_dense_decode_scratch_bytes",
    "recsa_dense_decode", "recsa_dense_decode_static", "recsa_backward_scratch_bytes", "recsa_decode_backward",
    "recsa_tree_backward", "recsa_distill_scratch_bytes", "recsa_distill_step", "recsa_cluster_scratch_bytes",
    "recsa_cluster_load",
]


class RecsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"recsa status {status}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_kv_heads", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("branching", ctypes.c_int), ("k", ctypes.c_int),
                ("capacity", ctypes.c_longlong), ("max_chunk", ctypes.c_int), ("rope_base", ctypes.c_double),
                ("dtype", ctypes.c_int)]


_lib = None


def lib():
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m hierarchical_sparse_attention_tree_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
        P = ctypes.POINTER
        sig = {
            "recsa_workspace_bytes": (sz, [P(Config)]),
            "recsa_init": (i32, [P(vp), P(Config), vp, vp, vp, sz, vp, vp]),
            "recsa_init_paged": (i32, [P(vp), P(Config), vp, vp, i64, i32, vp, i32, vp, sz, vp, vp]),
            "recsa_build_tree": (i32, [vp, P(i64), vp]),
            "recsa_append": (i32, [vp, vp, vp, i32, vp]),
            "recsa_decode": (i32, [vp, vp, vp, vp, vp, vp]),
            "recsa_backward_scratch_bytes": (sz, [P(Config)]),
            "recsa_decode_backward": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "recsa_tree_backward": (i32, [vp, vp, vp, vp, vp, sz, vp]),
            "recsa_distill_scratch_bytes": (sz, [P(Config)]),
            "recsa_distill_step": (i32, [vp, vp, vp, ctypes.c_float, vp, vp, vp, vp, sz, vp]),
            "recsa_cluster_scratch_bytes": (sz, [P(Config)]),
            "recsa_cluster_load": (i32, [vp, vp, vp, i64, P(i64), vp, vp, vp, sz, vp]),
            "recsa_append_decode": (i32, [vp, vp, vp, vp, vp, vp, vp, vp]),
            "recsa_prefill_scratch_bytes": (sz, [P(Config), i32]),
            "recsa_prefill": (i32, [vp, vp, vp, vp, i32, vp, vp, vp, vp, sz, vp]),
            "recsa_query_stats": (i32, [vp, P(i32), P(i64), P(i64), vp]),
            "recsa_get_lengths": (i32, [vp, P(i64)]),
            "recsa_tree_shape": (i32, [vp, P(i32), P(i64)]),
            "recsa_level_arrays": (i32, [vp, i32, P(vp), P(vp), P(vp)]),
            "recsa_check_device": (i32, [vp, vp]),
            "recsa_last_error": (ctypes.c_char_p, []),
            "recsa_destroy": (None, [vp]),
            "recsa_dense_decode_scratch_bytes": (sz, [i32, i32, i32]),
            "recsa_dense_decode": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i64, i64, i32, vp, sz, vp]),
            "recsa_dense_decode_static": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i64, i64, i32, vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != OK:
        raise RecsaError(status, lib().recsa_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return BF16
    if dtype == torch.float32:
        return F32
    raise ValueError(f"unsupported dtype {dtype}")


def make_config(batch, n_kv_heads, n_q_heads, head_dim, branching, k, capacity, dtype=torch.bfloat16,
                rope_base=1e6, max_chunk=0) -> Config:
    return Config(batch, n_kv_heads, n_q_heads, head_dim, branching, k, capacity, max_chunk, rope_base,
                  dtype_code(dtype))


def workspace_bytes(cfg: Config) -> int:
    n = lib().recsa_workspace_bytes(ctypes.byref(cfg))
    if n == 0:
        _check(ERR_INVALID_ARG)
    return n


class _DevArray:
    """Exposes a raw device pointer to torch.as_tensor (no copy)."""

    _TYPESTR = {torch.float32: "<f4", torch.int16: "<i2", torch.int32: "<i4", torch.int64: "<i8"}

    def __init__(self, ptr: int, shape, dtype: torch.dtype):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": self._TYPESTR[dtype], "data": (ptr, False),
                                         "version": 3}


def _view(ptr: int, shape, dtype: torch.dtype) -> torch.Tensor:
    if dtype == torch.bfloat16:
        return torch.as_tensor(_DevArray(ptr, shape, torch.int16), device="cuda").view(torch.bfloat16)
    return torch.as_tensor(_DevArray(ptr, shape, dtype), device="cuda")


class Context:
    """One recsa_ctx. The caller's cache and workspace tensors are kept alive
    by this object."""

    def __init__(self, cfg: Config, k_cache: torch.Tensor, v_cache: torch.Tensor, workspace: torch.Tensor,
                 pooler_w: torch.Tensor, stream=None, page_table: torch.Tensor | None = None, page_size: int = 0):
        """Contiguous cache: k_cache, v_cache [B][H_kv][capacity][d]. Paged:
        k_cache, v_cache are the page pools [num_pages][H_kv][page_size][d]
        and page_table the device int32 [B][max_pages] table."""
        self.cfg = cfg
        self._keep = (k_cache, v_cache, workspace, page_table)
        h = ctypes.c_void_p()
        if page_table is None:
            _check(lib().recsa_init(ctypes.byref(h), ctypes.byref(cfg), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(pooler_w),
                                    _stream(stream)))
        else:
            _check(lib().recsa_init_paged(ctypes.byref(h), ctypes.byref(cfg), _ptr(k_cache), _ptr(v_cache),
                                          k_cache.shape[0], page_size, _ptr(page_table), page_table.shape[1],
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _ptr(pooler_w), _stream(stream)))
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            lib().recsa_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def build_tree(self, lengths, stream=None):
        arr = (ctypes.c_longlong * self.cfg.batch)(*[int(x) for x in lengths])
        _check(lib().recsa_build_tree(self.handle, arr, _stream(stream)))

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None):
        n = k_new.shape[1]
        _check(lib().recsa_append(self.handle, _ptr(k_new), _ptr(v_new), n, _stream(stream)))

    def decode(self, q, out, sel_out=None, rows_out=None, stream=None):
        _check(lib().recsa_decode(self.handle, _ptr(q), _ptr(out), _ptr(sel_out), _ptr(rows_out), _stream(stream)))

    def append_decode(self, k_new, v_new, q, out, sel_out=None, rows_out=None, stream=None):
        _check(lib().recsa_append_decode(self.handle, _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(out), _ptr(sel_out),
                                         _ptr(rows_out), _stream(stream)))

    def append_decode_ptrs(self, k_new: int, v_new: int, q: int, out: int, sel_out=None, rows_out=None,
                           stream=None):
        """recsa_append_decode on raw addresses: device memory, or pinned host
        memory mapped into the device's address space (the kernel then reads
        the inputs and writes the output over the bus)."""
        vp = ctypes.c_void_p
        _check(lib().recsa_append_decode(self.handle, vp(k_new), vp(v_new), vp(q), vp(out), _ptr(sel_out),
                                         _ptr(rows_out), _stream(stream)))

    def prefill(self, q, k, v, out, sel_out=None, scratch=None, rows_out=None, stream=None):
        C = q.shape[1]
        nbytes = 0 if scratch is None else scratch.numel() * scratch.element_size()
        _check(lib().recsa_prefill(self.handle, _ptr(q), _ptr(k), _ptr(v), C, _ptr(out), _ptr(sel_out),
                                   _ptr(rows_out), _ptr(scratch), nbytes, _stream(stream)))

    def backward_scratch_bytes(self) -> int:
        return lib().recsa_backward_scratch_bytes(ctypes.byref(self.cfg))

    def decode_backward(self, q, dout, sel, dq, dk, dv, scratch, stream=None):
        _check(lib().recsa_decode_backward(self.handle, _ptr(q), _ptr(dout), _ptr(sel), _ptr(dq), _ptr(dk), _ptr(dv),
                                           _ptr(scratch), scratch.numel() * scratch.element_size(),
                                           _stream(stream)))

    def tree_backward(self, dk, dv, dw, scratch, stream=None):
        _check(lib().recsa_tree_backward(self.handle, _ptr(dk), _ptr(dv), _ptr(dw), _ptr(scratch),
                                         scratch.numel() * scratch.element_size(), _stream(stream)))

    def cluster_scratch_bytes(self) -> int:
        return lib().recsa_cluster_scratch_bytes(ctypes.byref(self.cfg))

    def cluster_load(self, k_src, v_src, lengths, Z, perm, scratch, stream=None):
        arr = (ctypes.c_longlong * self.cfg.batch)(*[int(x) for x in lengths])
        _check(lib().recsa_cluster_load(self.handle, _ptr(k_src), _ptr(v_src), int(k_src.shape[2]), arr, _ptr(Z),
                                        _ptr(perm), _ptr(scratch), scratch.numel() * scratch.element_size(),
                                        _stream(stream)))

    def distill_scratch_bytes(self) -> int:
        return lib().recsa_distill_scratch_bytes(ctypes.byref(self.cfg))

    def distill_step(self, q, target, lr, w_master, scratch, loss=None, dw_out=None, stream=None):
        _check(lib().recsa_distill_step(self.handle, _ptr(q), _ptr(target), float(lr), _ptr(w_master), _ptr(loss),
                                        _ptr(dw_out), _ptr(scratch), scratch.numel() * scratch.element_size(),
                                        _stream(stream)))

    def query_stats(self, stream=None):
        """(depth, k_rows, v_rows) of the last decode, per (sequence, KV head)
        unit, as lists of B * H_kv host integers."""
        n = self.cfg.batch * self.cfg.n_kv_heads
        d, kr, vr = (ctypes.c_int * n)(), (ctypes.c_longlong * n)(), (ctypes.c_longlong * n)()
        _check(lib().recsa_query_stats(self.handle, d, kr, vr, _stream(stream)))
        return list(d), list(kr), list(vr)

    def prefill_scratch_bytes(self, C: int) -> int:
        return lib().recsa_prefill_scratch_bytes(ctypes.byref(self.cfg), C)

    def lengths(self):
        arr = (ctypes.c_longlong * self.cfg.batch)()
        _check(lib().recsa_get_lengths(self.handle, arr))
        return list(arr)

    def tree_shape(self):
        j = ctypes.c_int()
        _check(lib().recsa_tree_shape(self.handle, ctypes.byref(j), None))
        rows = (ctypes.c_longlong * (j.value + 1))()
        _check(lib().recsa_tree_shape(self.handle, ctypes.byref(j), rows))
        return j.value, list(rows)

    def level(self, j: int):
        """(keys, values, value_sums) of level j as device tensor views
        [B][H_kv][rows][d]."""
        kp, vp, sp = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib().recsa_level_arrays(self.handle, j, ctypes.byref(kp), ctypes.byref(vp), ctypes.byref(sp)))
        _, rows = self.tree_shape()
        shape = (self.cfg.batch, self.cfg.n_kv_heads, rows[j], self.cfg.head_dim)
        dt = _TORCH_DTYPE[self.cfg.dtype]
        return _view(kp.value, shape, dt), _view(vp.value, shape, dt), _view(sp.value, shape, torch.float32)

    def check_device(self, stream=None):
        _check(lib().recsa_check_device(self.handle, _stream(stream)))


def dense_decode_scratch_bytes(batch, n_q_heads, head_dim) -> int:
    return lib().recsa_dense_decode_scratch_bytes(batch, n_q_heads, head_dim)


def dense_decode(k_cache, v_cache, q, out, length, scratch, stream=None):
    B, H, Ls, D = k_cache.shape
    Hq = q.shape[1]
    _check(lib().recsa_dense_decode(_ptr(k_cache), _ptr(v_cache), _ptr(q), _ptr(out), B, H, Hq, D, length, Ls,
                                    dtype_code(k_cache.dtype), _ptr(scratch),
                                    scratch.numel() * scratch.element_size(), _stream(stream)))


def dense_decode_static(k_cache, v_cache, q, out, length, stream=None):
    """recsa_dense_decode without a scratch argument: for callers that cannot
    allocate device memory (the library's fixed 8 MiB device array is used)."""
    B, H, Ls, D = k_cache.shape
    Hq = q.shape[1]
    _check(lib().recsa_dense_decode_static(_ptr(k_cache), _ptr(v_cache), _ptr(q), _ptr(out), B, H, Hq, D, length, Ls,
                                           dtype_code(k_cache.dtype), _stream(stream)))
