"""The top-k's second read classifies scores by comparing them with float bounds of the 12-bit
order-key buckets instead of forming each score's key; dsa_test_topk_bucket_floor is the host
build of that bound.  Checked here (no GPU) against the order-key definition written out in
numpy: for every bucket b and every score v of a set that holds the special values, the floats
at and next to every bucket edge and random bit patterns, (key(v) >> 20) >= b exactly when
v >= bound(b)."""
import numpy as np

import sparse_attention_15_b200 as dsa


def order_key(v):
    """The top-k's order: -0.0 counts as +0.0; the sign bit set for v >= 0, every bit flipped
    for v < 0 (unsigned comparison of keys is the float order)."""
    u = v.astype(np.float32).view(np.uint32).copy()
    u[(u << 1) == 0] = 0
    return np.where((u & 0x80000000) != 0, ~u, u | 0x80000000).astype(np.uint32)


def floats_of_keys(keys):
    """The float whose key is `keys` (the inverse of order_key away from -0.0)."""
    keys = keys.astype(np.uint32)
    bits = np.where((keys & 0x80000000) != 0, keys ^ 0x80000000, ~keys).astype(np.uint32)
    return bits.view(np.float32)


def test_bucket_bounds_match_the_key_definition(lib):
    rng = np.random.default_rng(0)
    specials = np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, -1e-45, 3.4028235e38,
                         -3.4028235e38, 1.1754944e-38, -1.1754944e-38, 1.0, -1.0], np.float32)
    edges = ((np.arange(4097, dtype=np.int64)[:, None] << 20) +
             np.array([-2, -1, 0, 1], dtype=np.int64)[None, :]).ravel() % (1 << 32)
    rand = rng.integers(0, 1 << 32, 20000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    v = np.concatenate([specials, floats_of_keys(edges), rand])
    v = v[~np.isnan(v)]
    bucket = order_key(v) >> 20
    for b in range(4097):
        f = np.float32(dsa.dsa_test_topk_bucket_floor(b))
        assert np.array_equal(bucket >= b, v >= f), f"bucket {b}: bound {f!r}"
    # the bounds themselves: -inf for the buckets of NaN images and -inf, NaN past +inf's
    assert dsa.dsa_test_topk_bucket_floor(0) == -np.inf
    assert dsa.dsa_test_topk_bucket_floor(2048) == 0.0
    assert dsa.dsa_test_topk_bucket_floor(0xFF8) == np.inf
    assert np.isnan(dsa.dsa_test_topk_bucket_floor(0xFF9))
