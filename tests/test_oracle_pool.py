"""The spawned-process pool that the GPU parity tests use for the oracle's
containers of many streams gives the same digests as direct oracle calls."""
import hashlib

import kvgen
import oracle
from oracle_pool import oracle_digests, oracle_digests_and_histograms


def test_pool_digests_equal_direct_oracle_calls():
    xs = [kvgen.mixed_small(1000 + 37 * i, seed=900 + i) for i in range(9)] + [kvgen.uniform_u16(4097, seed=7)]
    assert oracle_digests(xs, workers=3) == [hashlib.sha256(oracle.encode(x)).hexdigest() for x in xs]


def test_pool_generates_and_histograms_like_direct_calls():
    args = [(1, 0, 0, 40), (1, 0, 1, 40), (3, 1, 0, 24)]
    got = oracle_digests_and_histograms(kvgen.contiguous_tensor, args, workers=2)
    for (dig, hist), a in zip(got, args):
        x = kvgen.contiguous_tensor(*a)
        assert dig == hashlib.sha256(oracle.encode(x)).hexdigest()
        assert hist == [int(v) for v in oracle.histogram(x)]
