"""Pins of the oracle's reading of the chunk-paged KV cache: the page table
gathers back, token by token, to the cache it describes, and a decode step on
a shuffled pool equals the decode step on the contiguous cache."""
import numpy as np

from oracle.oracle import Oracle, Rows, gather_pages


def _scatter(cache, table, n_pages, rng):
    """Pool [n_pages, H, C, d] holding cache chunk (b, c) at page table[b, c];
    unused pages hold noise."""
    B, H, N, d = cache.shape
    C = 64
    pool = rng.standard_normal((n_pages, H, C, d))
    for b in range(B):
        for i in range(N):
            pool[table[b, i // C], :, i % C, :] = cache[b, :, i, :]
    return pool


def test_gather_matches_the_table_token_by_token():
    rng = np.random.default_rng(3)
    B, H, N, d = 2, 3, 256, 8
    cache = rng.standard_normal((B, H, N, d))
    n_pages = B * (N // 64) + 5
    table = rng.permutation(n_pages)[: B * (N // 64)].reshape(B, N // 64)
    pool = _scatter(cache, table, n_pages, rng)
    back = gather_pages(pool, table)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                assert np.array_equal(back[b, h, i], pool[table[b, i // 64], h, i % 64])
    assert np.array_equal(back, cache)


def test_decode_on_a_shuffled_pool_equals_the_contiguous_decode():
    rng = np.random.default_rng(4)
    B, Hq, Hkv, N, d, K = 2, 4, 2, 1024, 16, 3
    nc = N // 64
    q = rng.standard_normal((B, Hq, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    lq = rng.standard_normal((B, Hkv, nc, d))
    n_pages = B * nc + 3
    table = rng.permutation(n_pages)[: B * nc].reshape(B, nc)
    kg = gather_pages(_scatter(k, table, n_pages, rng), table)
    vg = gather_pages(_scatter(v, table, n_pages, rng), table)
    o = Oracle(B, Hq, Hkv, N, d, 64, K)
    seqlens = np.array([N, 700], np.int32)
    kp, bp = o.summary(k, lq)
    kp_g, bp_g = o.summary(kg, lq)
    assert np.array_equal(kp, kp_g) and np.array_equal(bp, bp_g)
    ref = o.decode(q, k, v, kp, bp, seqlens)
    got = o.decode(q, kg, vg, kp_g, bp_g, seqlens)
    assert np.array_equal(ref["ids"], got["ids"])
    assert np.array_equal(ref["O"], got["O"])
