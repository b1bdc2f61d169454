"""The seeded workloads on the CPU: the padded-length recipe is deterministic
and in range, and the counted FLOPs credit exactly the unmasked (query, key)
pairs (brute-force count over explicit masks), keeping the n*m/2 convention
for unpadded causal workloads."""
import numpy as np

import synth


def _brute_pairs(n, m, causal, L):
    keep = np.arange(m)[None, :] < L
    if causal:
        keep = keep & (np.arange(m)[None, :] <= np.arange(n)[:, None])
    else:
        keep = np.broadcast_to(keep, (n, m))
    return int(keep.sum())


def test_padded_lengths_deterministic_and_in_range():
    w = synth.workload("padded_b8h16_n1024_d64")
    a, b = w.key_len(), w.key_len()
    assert a == b and len(a) == w.B
    assert all(w.pad_min <= L <= w.m for L in a)
    assert len(set(a)) > 1                      # a real mix of lengths


def test_unpadded_flops_keep_the_convention():
    w = synth.workload("causal_b2h32_n4096_d128")
    assert w.key_len() is None
    assert w.bwd_flops() == 2.5 * 4 * w.B * w.H * w.n * w.m * w.d / 2
    w = synth.workload("cross_b8h16_n512_m2048_d64")
    assert w.bwd_flops() == 2.5 * 4 * w.B * w.H * w.n * w.m * w.d


def test_padded_flops_count_unmasked_pairs():
    for causal in (False, True):
        w = synth.make_small(3, 2, 37, 37, 8, 8, "bf16", causal, seed=1, lengths=(5, 37, 1))
        pairs = [_brute_pairs(w.n, w.m, causal, L) for L in w.key_len()]
        assert w.bwd_flops() == 2.5 * 4 * w.H * w.d * sum(pairs)
        assert w.fwd_flops() == 4 * w.H * w.d * sum(pairs)
        for b, p in enumerate(pairs):
            assert w.head_bwd_flops(b) == 2.5 * 4 * w.d * p
