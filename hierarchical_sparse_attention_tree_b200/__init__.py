"""RecSA (Recursive Sparse Attention) tree sparse attention for one attention
layer on B200 (sm_100a): tree build and append, per-query top-k descent and
shared-softmax gather attention, behind the C ABI of librecsa.so."""
from .recsa import (BF16, F32, Config, Context, RecsaError, dense_decode, dense_decode_scratch_bytes,  # noqa: F401
                    lib, make_config, workspace_bytes)
from .layer import RecsaLayer  # noqa: F401
