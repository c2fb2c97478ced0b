"""The scratch-free dense decode entry point (recsa_dense_decode_static).

For callers that hold only their input and output buffers and may not
allocate device memory (so they cannot hand the library a scratch buffer),
the library keeps one fixed 8 MiB device array for the partial results. This
checks, through the C ABI, that two calls in a row give what the scratch-taking
entry point gives, and that a call too large for the fixed array is refused
on the host. Collected last on purpose: it runs after every other test.
"""
import pytest
import torch

from hierarchical_sparse_attention_tree_b200 import recsa as R

pytestmark = pytest.mark.gpu


def _inputs(seed, B, H, G, D, L, dtype):
    g = torch.Generator(device="cuda").manual_seed(seed)
    Kc = torch.randn(B, H, L + 5, D, device="cuda", generator=g).to(dtype)
    Vc = torch.randn(B, H, L + 5, D, device="cuda", generator=g).to(dtype)
    q = torch.randn(B, H * G, D, device="cuda", generator=g).to(dtype)
    return Kc, Vc, q


@pytest.mark.parametrize("dtype,D,G,L", [(torch.bfloat16, 128, 4, 40000), (torch.float32, 64, 2, 777)])
def test_static_scratch_matches_allocating_entry_point(dtype, D, G, L):
    B, H = 4, 8
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    for call, seed in enumerate((11, 12)):  # two calls in a row share the fixed array
        Kc, Vc, q = _inputs(seed, B, H, G, D, L, dtype)
        ref = torch.empty_like(q)
        scratch = torch.empty(R.dense_decode_scratch_bytes(B, H * G, D), dtype=torch.uint8, device="cuda")
        R.dense_decode(Kc, Vc, q, ref, L, scratch)
        out = torch.full_like(q, float("nan"))
        R.dense_decode_static(Kc, Vc, q, out, L)
        torch.cuda.synchronize()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= tol, (call, err)


def test_static_scratch_refuses_oversized_call():
    B, H, G, D = 130, 16, 8, 128  # B * H_q = 16640 > 16131
    Kc = torch.zeros(1, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(R.RecsaError) as e:
        R.lib()  # the call below is refused on the host before any pointer is used
        st = R.lib().recsa_dense_decode_static(Kc.data_ptr(), Kc.data_ptr(), Kc.data_ptr(), Kc.data_ptr(), B, H,
                                               H * G, D, 1, 1, R.BF16, None)
        R._check(st)
    assert e.value.status == R.ERR_CAPACITY
    assert "fixed scratch" in str(e.value)
