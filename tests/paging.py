"""Page pools for the paged cache layout (data movement only, no arithmetic of the method).

A contiguous plane holds per (sequence b, KV head h) T_cap token slots of `tb` bytes
([B][Hkv][T_cap][tb]; a value-code plane's 16-slot tiles are 16 consecutive slots). A
pool holds num_pages pages of page_tokens slots per KV head ([num_pages][Hkv]
[page_tokens][tb]); position t of sequence b lives in page table[b][t // page_tokens] at
slot t % page_tokens. `scatter` moves contiguous planes into a pool, `gather` back.
"""
import numpy as np


def token_bytes(d, bits_k, bits_v, group):
    """Bytes per token slot of the four planes (k_codes, k_sz, v_codes, v_sz)."""
    ng = d // group
    return [d * bits_k // 8, 4 * ng, d * bits_v // 8, 4 * ng]


def random_table(rng, B, pages_per_seq, num_pages):
    """A block table using distinct pages, drawn without replacement from the pool."""
    assert num_pages >= B * pages_per_seq
    return rng.permutation(num_pages)[:B * pages_per_seq].reshape(B, pages_per_seq).astype(np.int32)


def scatter(planes, table, Hkv, T_cap, page_tokens, num_pages, tbytes):
    """Contiguous planes (flat uint8) -> pools (flat uint8); unused pages are zero."""
    B, per = table.shape
    assert per * page_tokens == T_cap
    pools = []
    for plane, tb in zip(planes, tbytes):
        src = np.asarray(plane).view(np.uint8).reshape(B, Hkv, per, page_tokens, tb)
        pool = np.zeros((num_pages, Hkv, page_tokens, tb), np.uint8)
        pool[table.reshape(-1)] = src.transpose(0, 2, 1, 3, 4).reshape(B * per, Hkv, page_tokens, tb)
        pools.append(pool.reshape(-1))
    return pools


def gather(pools, table, Hkv, page_tokens, tbytes):
    """Pools (flat uint8) -> contiguous planes (flat uint8) for the sequences of `table`."""
    B, per = table.shape
    planes = []
    for pool, tb in zip(pools, tbytes):
        p = np.asarray(pool).view(np.uint8).reshape(-1, Hkv, page_tokens, tb)
        got = p[table.reshape(-1)].reshape(B, per, Hkv, page_tokens, tb).transpose(0, 2, 1, 3, 4)
        planes.append(np.ascontiguousarray(got).reshape(-1))
    return planes
