"""Pins of the test-side page pool helpers (CPU): element-by-element placement checked by
explicit loops, gather undoes scatter, unused pages stay empty."""
import numpy as np

from tests import paging


def _setup(seed=0):
    rng = np.random.default_rng(seed)
    B, Hkv, page_tokens, per, d = 3, 2, 64, 4, 128
    T_cap = per * page_tokens
    num_pages = B * per + 5
    tb = paging.token_bytes(d, 2, 4, d)
    planes = [rng.integers(0, 256, B * Hkv * T_cap * n, dtype=np.uint8) for n in tb]
    table = paging.random_table(rng, B, per, num_pages)
    return B, Hkv, page_tokens, T_cap, num_pages, tb, planes, table


def test_token_bytes_of_the_planes():
    assert paging.token_bytes(128, 2, 2, 128) == [32, 4, 32, 4]
    assert paging.token_bytes(64, 4, 2, 32) == [32, 8, 16, 8]


def test_scatter_places_every_slot_by_the_table():
    B, Hkv, pt, T_cap, npg, tb, planes, table = _setup()
    pools = paging.scatter(planes, table, Hkv, T_cap, pt, npg, tb)
    for plane, pool, n in zip(planes, pools, tb):
        for b in range(B):
            for h in range(Hkv):
                for t in range(0, T_cap, 7):
                    src = ((b * Hkv + h) * T_cap + t) * n
                    dst = ((int(table[b, t // pt]) * Hkv + h) * pt + t % pt) * n
                    assert np.array_equal(plane[src:src + n], pool[dst:dst + n])


def test_gather_undoes_scatter_and_unused_pages_stay_zero():
    B, Hkv, pt, T_cap, npg, tb, planes, table = _setup(1)
    pools = paging.scatter(planes, table, Hkv, T_cap, pt, npg, tb)
    back = paging.gather(pools, table, Hkv, pt, tb)
    for a, b in zip(planes, back):
        assert np.array_equal(a, b)
    unused = sorted(set(range(npg)) - set(table.reshape(-1).tolist()))
    assert len(unused) == 5
    for pool, n in zip(pools, tb):
        p = pool.reshape(npg, -1)
        assert not p[unused].any()


def test_random_table_uses_distinct_pages():
    rng = np.random.default_rng(2)
    t = paging.random_table(rng, 4, 3, 20)
    assert t.shape == (4, 3) and len(set(t.reshape(-1).tolist())) == 12
    assert t.min() >= 0 and t.max() < 20
