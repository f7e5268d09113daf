"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry
point include/kvq.h declares, sizes planes as the layout says, and rejects bad arguments
before launching anything."""
import ctypes as C
import os
import re

import pytest

import decode_attention_post_b200 as kvq
from decode_attention_post_b200 import kvq as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    L = kvq.load()
    names = _header_functions()
    assert {"kvq_quantize_append", "kvq_decode_attention", "kvq_bf16_decode"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    L = kvq.load()
    for s in range(6):
        assert L.kvq_status_string(s)
    assert L.kvq_status_string(99) == b"unknown status"


def _desc(B=2, Hkv=2, T_cap=128, d=128, bits_k=2, bits_v=2, group=128, alpha=0.01,
          ptr=0x1000):
    qp = K._QParams(bits_k, bits_v, group, alpha)
    return K._Cache(B, Hkv, T_cap, d, qp, ptr, ptr, ptr, ptr), qp


def test_plane_bytes_follow_layout():
    L = kvq.load()
    desc, _ = _desc(B=3, Hkv=2, T_cap=192, d=128, bits_k=4, bits_v=2)
    tok = 3 * 2 * 192
    want = [tok * 64, tok * 4, tok * 32, tok * 4]
    assert [L.kvq_cache_plane_bytes(C.byref(desc), w) for w in range(4)] == want
    assert L.kvq_cache_plane_bytes(C.byref(desc), 7) == 0
    # 2-bit, group 128: 2.25 bits per element including the float16 (s, z)
    desc, _ = _desc(bits_k=2)
    kb = L.kvq_cache_plane_bytes(C.byref(desc), 0) + L.kvq_cache_plane_bytes(C.byref(desc), 1)
    assert kb * 8 / (2 * 2 * 128 * 128) == 2.25


def _paged_desc(page_tokens=64, num_pages=10, table=0x8000, T_cap=128, **kw):
    desc, qp = _desc(T_cap=T_cap, **kw)
    desc.block_table = table
    desc.page_tokens = page_tokens
    desc.num_pages = num_pages
    return desc, qp


def test_paged_plane_bytes_are_pool_sizes():
    L = kvq.load()
    desc, _ = _paged_desc(page_tokens=128, num_pages=7, T_cap=256, B=3, Hkv=2, bits_k=4,
                          bits_v=2)
    tok = 7 * 2 * 128                                  # pages x heads x slots per page
    want = [tok * 64, tok * 4, tok * 32, tok * 4]
    assert [L.kvq_cache_plane_bytes(C.byref(desc), w) for w in range(4)] == want
    bad, _ = _paged_desc(page_tokens=96)
    assert L.kvq_cache_plane_bytes(C.byref(bad), 0) == 0


@pytest.mark.parametrize("mut", [
    dict(page_tokens=0), dict(page_tokens=96), dict(page_tokens=256),   # not a divisor of T_cap
    dict(num_pages=0), dict(table=0x8002),                              # misaligned table
])
def test_paged_cache_validation(mut):
    desc, qp = _paged_desc(**mut)
    assert _append(desc, qp) == 1
    assert kvq.load().kvq_last_error()
    assert _decode(desc) == 1


def test_paged_cache_accepted_shapes():
    # argument checks pass (n = 0 is a no-op: nothing is launched)
    desc, qp = _paged_desc(page_tokens=64, num_pages=4)
    assert _append(desc, qp, n=0) == 0
    desc, qp = _paged_desc(page_tokens=128, num_pages=1)
    assert _append(desc, qp, n=0) == 0


def _append(desc, qp, n=4, dtype=0, k=0x2000, pos=0x3000):
    L = kvq.load()
    return L.kvq_quantize_append(k, k, dtype, None, None, C.byref(qp), C.byref(desc), pos, n,
                                 None, None)


@pytest.mark.parametrize("mut,status", [
    (dict(bits_k=3), 2), (dict(bits_v=8), 2), (dict(group=48), 1), (dict(group=256), 1),
    (dict(d=96, group=32), 2), (dict(T_cap=100), 1), (dict(B=0), 1), (dict(alpha=0.6), 1),
    (dict(alpha=0.2), 2),            # clip index 25 > 8
    (dict(ptr=0x1004), 1),           # misaligned planes
])
def test_append_rejects_bad_cache(mut, status):
    desc, qp = _desc(**mut)
    assert _append(desc, qp) == status
    assert kvq.load().kvq_last_error()


def test_append_argument_errors():
    L = kvq.load()
    desc, qp = _desc()
    other = K._QParams(2, 2, 128, 0.02)
    assert L.kvq_quantize_append(0x2000, 0x2000, 0, None, None, C.byref(other), C.byref(desc),
                                 0x3000, 4, None, None) == 1          # qp != cache qp
    assert _append(desc, qp, n=-1) == 1
    assert _append(desc, qp, n=129) == 3                              # > T_cap
    assert _append(desc, qp, dtype=7) == 1
    assert _append(desc, qp, k=0) == 1                                # NULL input
    assert _append(desc, qp, n=0) == 0                                # no-op, nothing launched
    assert L.kvq_quantize_append(0x2000, 0x2000, 0, None, None, C.byref(qp), None, 0x3000, 4,
                                 None, None) == 1


def _decode(desc, Hq=8, max_seqlen=64, ws=0x4000, ws_bytes=1 << 30, q=0x5000, out=0x6000,
            qd=1, od=1):
    L = kvq.load()
    return L.kvq_decode_attention(q, qd, Hq, None, C.byref(desc), 0x7000, max_seqlen, out, od,
                                  ws, ws_bytes, None, None)


def test_decode_argument_errors():
    desc, _ = _desc()
    assert _decode(desc, Hq=7) == 1            # not a multiple of Hkv
    assert _decode(desc, Hq=6) == 2            # G = 3 not implemented
    assert _decode(desc, Hq=4) == 2            # G = 2 not implemented
    assert _decode(desc, max_seqlen=129) == 3  # > T_cap
    assert _decode(desc, max_seqlen=-1) == 1
    assert _decode(desc, ws=0) == 4
    assert _decode(desc, ws=0x4010) == 4       # not 256-byte aligned
    assert _decode(desc, ws_bytes=16) == 4
    assert _decode(desc, q=0) == 1
    assert _decode(desc, qd=5) == 1
    d2, _ = _desc(group=64)
    assert _decode(d2) == 2                    # decode implements group == d


def _window_decode(desc, win, Hq=8, max_seqlen=64, qd=1, ws_bytes=1 << 30):
    L = kvq.load()
    return L.kvq_decode_attention_window(0x5000, qd, Hq, None, C.byref(desc),
                                         None if win is None else C.byref(win), 0x7000,
                                         max_seqlen, 0x6000, 1, 0x4000, ws_bytes, None, None)


def _win(S_sink=4, S_keep=32, S_flush=64, ks=0x9000, vs=0x9000, kr=0xA000, vr=0xA000):
    return K._Window(S_sink, S_keep, S_flush, ks, vs, kr, vr, None)


def test_window_decode_argument_errors():
    desc, _ = _desc(T_cap=128)
    assert _window_decode(desc, None) == 1                        # no window
    assert _window_decode(desc, _win(S_flush=0)) == 1
    assert _window_decode(desc, _win(S_sink=-1)) == 1
    assert _window_decode(desc, _win(S_keep=-2)) == 1
    assert _window_decode(desc, _win(S_sink=1024, S_keep=1024, S_flush=64)) == 2   # > 2048
    assert _window_decode(desc, _win(ks=0)) == 1                  # sink buffer missing
    assert _window_decode(desc, _win(kr=0)) == 1                  # recent buffer missing
    assert _window_decode(desc, _win(), qd=0) == 2                # float32 queries
    # the quantized middle of max_seqlen must fit the cache: 4 + 32 + 128 fits, + 64 not
    assert _window_decode(desc, _win(), max_seqlen=4 + 32 + 192 + 63) == 3
    assert _window_decode(desc, _win(), ws_bytes=16) == 4
    # 16-byte copies of window rows and float4 reads of T_v: misaligned buffers refused
    assert _window_decode(desc, _win(kr=0xA008)) == 1
    assert _window_decode(desc, _win(vs=0x9004)) == 1
    w = _win()
    w.T_v = 0xB004
    assert _window_decode(desc, w) == 1
    assert kvq.load().kvq_last_error()


def _window_append(desc, qp, win, dtype=1, n=1, k=0x5000, seqlens=0x7000):
    L = kvq.load()
    return L.kvq_window_append(k, 0x6000, dtype, None, None, C.byref(qp), C.byref(desc),
                               None if win is None else C.byref(win), seqlens, n, None, None)


def test_window_append_argument_errors():
    desc, qp = _desc(T_cap=128)
    assert _window_append(desc, qp, None) == 1                     # no window
    assert _window_append(desc, qp, _win(S_flush=0)) == 1
    assert _window_append(desc, qp, _win(S_sink=1024, S_keep=1024, S_flush=64)) == 2
    assert _window_append(desc, qp, _win(kr=0)) == 1
    assert _window_append(desc, qp, _win(), dtype=0) == 2          # float32 tokens
    assert _window_append(desc, qp, _win(), n=-1) == 1
    assert _window_append(desc, qp, _win(), k=0) == 1
    assert _window_append(desc, qp, _win(), seqlens=0) == 1
    assert _window_append(desc, qp, _win(), k=0x5002) == 1         # misaligned
    other = K._QParams(4, 2, 128, 0.01)
    assert _window_append(desc, other, _win()) == 1                # qparams differ
    assert _window_append(desc, qp, _win(), n=0, k=0) == 0         # nothing to do
    assert kvq.load().kvq_last_error() == b""


def test_window_quantized_middle_matches_the_oracle_reading():
    import oracle
    # the library's host-side reading (through the capacity check) equals the oracle's:
    # max_seqlen whose middle is exactly T_cap passes the shape checks, one batch more fails
    desc, _ = _desc(T_cap=128)
    for S_sink, S_keep, S_flush in [(4, 32, 64), (0, 0, 64), (64, 128, 128), (3, 5, 16)]:
        win = _win(S_sink, S_keep, S_flush)
        L_ok = S_sink + S_keep + 128 + S_flush - 1
        assert oracle.window_quantized(L_ok, S_sink, S_keep, S_flush) == 128
        assert _window_decode(desc, win, max_seqlen=L_ok, ws_bytes=16) == 4   # shape ok
        assert oracle.window_quantized(L_ok + 1, S_sink, S_keep, S_flush) > 128
        assert _window_decode(desc, win, max_seqlen=L_ok + 1, ws_bytes=16) == 3


def test_workspace_sizes_positive_and_monotone():
    L = kvq.load()
    desc, _ = _desc(B=4, Hkv=8, T_cap=16384)
    a = L.kvq_decode_workspace_bytes(C.byref(desc), 32, 1024)
    b = L.kvq_decode_workspace_bytes(C.byref(desc), 32, 16384)
    assert 0 < a <= b
    assert L.kvq_decode_workspace_bytes(C.byref(desc), 31, 1024) == 0
    assert L.kvq_bf16_decode_workspace_bytes(4, 32, 8, 128, 16384) > 0
    assert L.kvq_bf16_decode_workspace_bytes(4, 32, 8, 96, 16384) == 0


def test_workspace_never_shrinks_across_a_split_boundary():
    """With 32 (sequence, KV head) pairs the split target is 74 (148 SMs x 4 CTAs x 4 waves
    / 32): 74 blocks of 64 tokens give 74 splits and 75 blocks only 38. The workspace must
    not shrink at that boundary, so that a size query for any longer max_seqlen (e.g.
    T_cap, as the windowed decode allows) covers every shorter call."""
    L = kvq.load()
    desc, _ = _desc(B=4, Hkv=8, T_cap=16384)
    sizes = [L.kvq_decode_workspace_bytes(C.byref(desc), 32, m)
             for m in range(64, 16385, 64)]
    assert all(0 < a <= b for a, b in zip(sizes, sizes[1:]))
    assert L.kvq_decode_workspace_bytes(C.byref(desc), 32, 74 * 64) == \
        L.kvq_decode_workspace_bytes(C.byref(desc), 32, 75 * 64)


def test_window_decode_accepts_a_workspace_sized_for_t_cap():
    """The header's promise: kvq_decode_workspace_bytes(cache, Hq, m) for any m >= the
    quantized middle of max_seqlen (m = T_cap always) is enough. The windowed decode needs
    the size for its quantized middle, one byte less is rejected (KVQ_ERR_WORKSPACE, 4)
    before anything is launched; the T_cap size is at least that."""
    import oracle
    L = kvq.load()
    desc, _ = _desc(B=4, Hkv=8, T_cap=16384)
    ws_cap = L.kvq_decode_workspace_bytes(C.byref(desc), 32, 16384)
    for S_sink, S_keep, S_flush in [(0, 0, 64), (4, 60, 64), (64, 256, 128)]:
        for mid_blocks in (1, 37, 74, 75, 149, 255):
            max_seqlen = S_sink + S_keep + mid_blocks * 64
            qmax = oracle.window_quantized(max_seqlen, S_sink, S_keep, S_flush)
            need = L.kvq_decode_workspace_bytes(C.byref(desc), 32, qmax)
            assert 0 < need <= ws_cap
            r = _window_decode(desc, _win(S_sink, S_keep, S_flush), Hq=32,
                               max_seqlen=max_seqlen, ws_bytes=need - 1)
            assert r == 4, (S_sink, S_keep, S_flush, mid_blocks)


def test_bf16_decode_argument_errors():
    L = kvq.load()
    args = dict(q=0x1000, Hq=32, k=0x2000, v=0x3000, B=2, Hkv=8, T_cap=128, d=128,
                seqlens=0x4000, max_seqlen=64, out=0x5000, ws=0x6000, ws_bytes=1 << 30)

    def call(**kw):
        a = dict(args, **kw)
        return L.kvq_bf16_decode(a["q"], a["Hq"], a["k"], a["v"], a["B"], a["Hkv"], a["T_cap"],
                                 a["d"], a["seqlens"], a["max_seqlen"], a["out"], a["ws"],
                                 a["ws_bytes"], None, None)
    assert call(k=0) == 1
    assert call(T_cap=100) == 1
    assert call(d=80) == 2
    assert call(Hq=16) == 2
    assert call(max_seqlen=200) == 3
    assert call(ws_bytes=8) == 4
    assert call(k=0x2008) == 1


def test_binding_requires_cuda_tensors():
    import torch
    qp = kvq.QParams()
    with pytest.raises(TypeError):
        kvq.KVCache(1, 1, 64, 128, qp, [torch.zeros(8, dtype=torch.uint8)] * 4)


def _vq_desc(B=2, Hkv=2, T_cap=128, d=128, ptr=0x1000):
    return K._VQCache(B, Hkv, T_cap, d, ptr, ptr, ptr, ptr)


def test_vq_plane_bytes_follow_layout():
    L = kvq.load()
    desc = _vq_desc(B=3, Hkv=2, T_cap=192, d=128)
    tok = 3 * 2 * 192
    assert [L.kvq_vq_plane_bytes(C.byref(desc), w) for w in range(4)] == \
        [tok * 32, tok * 2, tok * 32, tok * 2]
    assert L.kvq_vq_plane_bytes(C.byref(desc), 9) == 0


def test_vq_argument_errors():
    L = kvq.load()
    desc = _vq_desc()

    def append(**kw):
        a = dict(k=0x5000, v=0x5000, dt=1, ck=0x7000, cv=0x7000, pos=0x6000, n=4)
        a.update(kw)
        return L.kvq_vq_append(a["k"], a["v"], a["dt"], None, None, a["ck"], a["cv"],
                               C.byref(desc), a["pos"], a["n"], None, None)
    assert append(ck=0) == 1
    assert append(ck=0x7008) == 1                       # misaligned codebook
    assert append(dt=3) == 1
    assert append(n=-1) == 1
    assert append(n=1000) == 3
    assert append(k=0) == 1
    assert append(n=0, k=0) == 0

    def decode(ws_bytes=16, **kw):
        a = dict(q=0x5000, Hq=8, ck=0x7000, cv=0x7000, seq=0x6000, mx=64, out=0x8000)
        a.update(kw)
        return L.kvq_vq_decode_attention(a["q"], 1, a["Hq"], None, a["ck"], a["cv"],
                                         C.byref(desc), a["seq"], a["mx"], a["out"], 1, 0x9000,
                                         ws_bytes, None, None)
    assert decode(Hq=6) == 2                            # G = 3
    assert decode(mx=200) == 3
    assert decode(cv=0) == 1
    assert decode(out=0) == 1
    assert decode() == 4                                # workspace too small
    assert 0 < L.kvq_vq_decode_workspace_bytes(C.byref(desc), 8, 64) <= \
        L.kvq_vq_decode_workspace_bytes(C.byref(desc), 8, 128)
    bad = _vq_desc(d=96)
    assert L.kvq_vq_decode_workspace_bytes(C.byref(bad), 8, 64) == 0
