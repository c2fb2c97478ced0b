"""The benchmark's byte bookkeeping for the rooflines that compose several
kernels (host arithmetic only)."""
import bench


def test_distill_token_pass_bytes_by_hand():
    """One unit of 16 tokens, b = 4, d = 2, bf16, two levels (4 nodes, 1 node):
    propagation: token keys 16*2*2 = 64; level 1: accumulators (2 arrays of
    4 fp32 rows) read and cleared 4*2*2*4*2 = 128; level 2: 1*2*2*4*2 = 32,
    its h and s written 1*2*2*4 = 16 and its 4 children's keys read 4*2*2 = 16;
    rebuild: level 1 reads 2*16*2*2 = 128 and writes 4 rows of (key, value,
    fp32 sum) 4*2*(2+2+4) = 64; level 2 reads 4 children's keys and fp32 sums
    4*2*(2+4) = 48 and writes 1*2*(2+2+4) = 16. Total 512."""
    assert bench.distill_token_pass_bytes(1, [16], 2, 4, 2, 2) == 512


def test_distill_token_pass_bytes_scales_with_units():
    one = bench.distill_token_pass_bytes(1, [1000], 8, 8, 3, 2)
    assert bench.distill_token_pass_bytes(4, [1000], 8, 8, 3, 2) == 4 * one
    assert bench.distill_token_pass_bytes(1, [1000, 1000], 8, 8, 3, 2) == 2 * one
