"""The spawned-process pool that the GPU parity tests use for the oracle's
containers of many streams gives the same digests as direct oracle calls."""
import hashlib

import kvgen
import oracle
from oracle_pool import oracle_digests


def test_pool_digests_equal_direct_oracle_calls():
    xs = [kvgen.mixed_small(1000 + 37 * i, seed=900 + i) for i in range(9)] + [kvgen.uniform_u16(4097, seed=7)]
    assert oracle_digests(xs, workers=3) == [hashlib.sha256(oracle.encode(x)).hexdigest() for x in xs]
