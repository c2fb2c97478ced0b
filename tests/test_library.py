"""The C-ABI library loads on a CPU-only host, exports every symbol its
header declares, and rejects bad arguments on the host before touching a
device."""
import ctypes
import os
import re

import pytest

from hierarchical_sparse_attention_tree_b200 import recsa as R

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "recsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(recsa_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    lib = R.lib()
    names = declared_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(R.EXPORTS) == names


def test_workspace_sizes():
    cfg = R.make_config(4, 8, 32, 128, 64, 16, 524288 + 512)
    n = R.workspace_bytes(cfg)
    # three levels of bf16 keys/values plus fp32 value sums: a few percent of the 8.6 GB cache
    assert 0.25e9 < n < 0.3e9
    tiny = R.make_config(1, 1, 4, 64, 16, 4, 4096, dtype=__import__("torch").float32)
    assert R.workspace_bytes(tiny) > 2 * 256 * 64 * 4


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 96, R.ERR_UNSUPPORTED), ("branching", 1, R.ERR_INVALID_ARG), ("k", 0, R.ERR_INVALID_ARG),
    ("n_q_heads", 12, R.ERR_INVALID_ARG), ("n_q_heads", 24, R.ERR_UNSUPPORTED), ("capacity", 0, R.ERR_INVALID_ARG),
    ("rope_base", 1.0, R.ERR_INVALID_ARG), ("k", 65, R.ERR_INVALID_ARG),
])
def test_bad_config_rejected(field, value, status):
    cfg = R.make_config(1, 8, 32, 128, 64, 16, 1024)
    setattr(cfg, field, value)
    assert R.lib().recsa_workspace_bytes(ctypes.byref(cfg)) == 0
    assert R.lib().recsa_last_error()
    h = ctypes.c_void_p()
    st = R.lib().recsa_init(ctypes.byref(h), ctypes.byref(cfg), None, None, None, 0, None, None)
    assert st == status and not h.value


def test_null_buffers_rejected():
    cfg = R.make_config(1, 8, 32, 128, 64, 16, 1024)
    h = ctypes.c_void_p()
    assert R.lib().recsa_init(ctypes.byref(h), ctypes.byref(cfg), None, None, None, 0, None, None) == R.ERR_INVALID_ARG
    assert b"NULL" in R.lib().recsa_last_error()
    assert R.lib().recsa_build_tree(None, None, None) == R.ERR_INVALID_ARG
    assert R.lib().recsa_decode(None, None, None, None, None, None) == R.ERR_INVALID_ARG
    assert R.lib().recsa_dense_decode_scratch_bytes(4, 32, 128) == 4 * 32 * 256 * 130 * 4


def test_query_stats_rejects_null_context():
    assert R.lib().recsa_query_stats(None, None, None, None, None) == R.ERR_INVALID_ARG


def test_decode_shared_memory_limit_checked_at_init():
    """k * b candidates whose decode tiles cannot fit the 227 KB of shared
    memory a CTA may use are refused when the context is created, before any
    device call (the buffers below are never touched)."""
    cfg = R.make_config(1, 8, 32, 128, 64, 64, 1 << 20)  # 4096 candidates per level
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced
    st = R.lib().recsa_init(ctypes.byref(h), ctypes.byref(cfg), fake, fake, fake, 0, fake, None)
    assert st == R.ERR_UNSUPPORTED and not h.value
    assert b"shared memory" in R.lib().recsa_last_error()


def test_paged_init_checks_page_geometry():
    """recsa_init_paged refuses a page size that is not a multiple of the
    branching factor and a page table too small for the capacity, before any
    device call (the buffers below are never touched)."""
    cfg = R.make_config(1, 8, 32, 128, 64, 16, 4096)
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)
    st = R.lib().recsa_init_paged(ctypes.byref(h), ctypes.byref(cfg), fake, fake, 64, 96, fake, 64, fake, 1 << 40,
                                  fake, None)
    assert st == R.ERR_INVALID_ARG and b"multiple of branching" in R.lib().recsa_last_error()
    st = R.lib().recsa_init_paged(ctypes.byref(h), ctypes.byref(cfg), fake, fake, 64, 64, fake, 8, fake, 1 << 40,
                                  fake, None)
    assert st == R.ERR_INVALID_ARG and b"cover the capacity" in R.lib().recsa_last_error()


def test_backward_scratch_and_null_arguments():
    """The backward scratch holds two fp32 rows per tree node (about 2/b of
    the fp32 token gradients) plus small per-call arrays; NULL arguments
    are rejected on the host."""
    cfg = R.make_config(4, 8, 32, 128, 64, 16, 524288)
    n = R.lib().recsa_backward_scratch_bytes(ctypes.byref(cfg))
    nodes = 4 * 8 * (8192 + 128 + 2) * 128 * 4 * 2
    assert nodes <= n < nodes + 16 * 2 ** 20
    bad = R.make_config(1, 8, 32, 96, 64, 16, 1024)
    assert R.lib().recsa_backward_scratch_bytes(ctypes.byref(bad)) == 0
    assert R.lib().recsa_decode_backward(None, None, None, None, None, None, None, None, 0, None) == R.ERR_INVALID_ARG
    assert R.lib().recsa_tree_backward(None, None, None, None, None, 0, None) == R.ERR_INVALID_ARG


def test_distill_scratch_and_null_arguments():
    cfg = R.make_config(4, 8, 32, 128, 64, 16, 524288)
    n = R.lib().recsa_distill_scratch_bytes(ctypes.byref(cfg))
    assert n >= R.lib().recsa_backward_scratch_bytes(ctypes.byref(cfg)) + 3 * 4 * 32 * 128 * 4
    assert R.lib().recsa_distill_step(None, None, None, ctypes.c_float(0.1), None, None, None, None, 0,
                                      None) == R.ERR_INVALID_ARG


def test_cluster_scratch_and_null_arguments():
    """The clustered order's scratch: one 24-byte record per token of every
    unit at capacity, padded to a power of two (at least one 1024-record
    tile), plus the sequences' start offsets; NULL arguments are rejected on
    the host."""
    tail = 256  # [B + 1] offsets, one 256-byte-aligned block
    cfg = R.make_config(4, 8, 32, 128, 64, 16, 524288)
    assert R.lib().recsa_cluster_scratch_bytes(ctypes.byref(cfg)) == (1 << 24) * 24 + tail
    cfg = R.make_config(4, 8, 32, 128, 64, 16, 524289)
    assert R.lib().recsa_cluster_scratch_bytes(ctypes.byref(cfg)) == (1 << 25) * 24 + tail
    cfg = R.make_config(1, 1, 4, 64, 8, 3, 10)
    assert R.lib().recsa_cluster_scratch_bytes(ctypes.byref(cfg)) == 1024 * 24 + tail
    bad = R.make_config(1, 8, 32, 96, 64, 16, 1024)
    assert R.lib().recsa_cluster_scratch_bytes(ctypes.byref(bad)) == 0
    lengths = (ctypes.c_longlong * 1)(10)
    assert R.lib().recsa_cluster_load(None, None, None, 10, lengths, None, None, None, 0, None) == R.ERR_INVALID_ARG
