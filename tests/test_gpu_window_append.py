"""GPU tests of the write side of the full-precision window ("WUSH-KV: KV Cache
Quantization with Data-Adaptive Transforms", section 4.4), through the C ABI:
kvq_window_append over a serving loop (a prefill per sequence, then one token per step),
checked three ways --
  * the sink and the recent ring hold exactly the bfloat16 tokens of the window positions;
  * the quantized middle (cache positions [0, Q)) is byte-identical to kvq_quantize_append
    of the same tokens through the same float32 path;
  * kvq_decode_attention_window over that state matches the oracle's windowed decode of
    the whole token history (relative L2 <= 1e-3, max-abs <= 5e-3).
"""
import numpy as np
import pytest
import torch

import decode_attention_post_b200 as kvq
import oracle
from tests import synth
from tests.test_gpu_parity import assert_close, host_cache_from, qp_of, t_, upload_cache

pytestmark = pytest.mark.gpu

DEV = "cuda"


class WindowState:
    """Device buffers of a windowed cache and the token history on the host."""

    def __init__(self, cfg, B, T_cap, S_sink, S_keep, S_flush):
        self.cfg, self.B, self.S_sink, self.S_keep, self.S_flush = cfg, B, S_sink, S_keep, S_flush
        self.R = S_keep + S_flush
        self.cache = kvq.KVCache.allocate(B, cfg.Hkv, T_cap, cfg.d, qp_of(cfg))
        z = lambda n: torch.zeros((B, cfg.Hkv, n, cfg.d), dtype=torch.bfloat16, device=DEV)
        self.ks, self.vs = (z(S_sink), z(S_sink)) if S_sink else (None, None)
        self.kr, self.vr = z(self.R), z(self.R)
        self.err = torch.zeros(1, dtype=torch.int32, device=DEV)
        self.len = np.zeros(B, np.int32)
        Tk, Tv, Tit = synth.transforms(cfg)
        self.Tk_h, self.Tv_h, self.Tit_h = Tk, Tv, Tit
        self.Tk, self.Tv, self.Tit = t_(Tk), t_(Tv), t_(Tit)
        self.hist_k = [np.zeros((0, cfg.Hkv, cfg.d), np.uint16) for _ in range(B)]
        self.hist_v = [np.zeros((0, cfg.Hkv, cfg.d), np.uint16) for _ in range(B)]

    def append(self, kb, vb, seqs=None):
        """kb, vb: bf16 bits [B'][n][Hkv][d] for the sequences `seqs` (default all)."""
        seqs = list(range(self.B)) if seqs is None else seqs
        if len(seqs) == self.B:
            cache, bufs = self.cache, (self.ks, self.vs, self.kr, self.vr)
        else:
            assert len(seqs) == 1
            b = seqs[0]
            cache = self.cache.view_sequence(b)
            bufs = tuple(None if x is None else x[b:b + 1] for x in (self.ks, self.vs, self.kr, self.vr))
        lens = t_(self.len[seqs].copy())
        kvq.window_append(t_(kb), t_(vb), self.Tk, self.Tv, qp_of(self.cfg), cache, self.S_sink,
                          self.S_keep, self.S_flush, *bufs, lens, dev_err=self.err)
        n = kb.shape[1]
        for j, b in enumerate(seqs):
            self.hist_k[b] = np.concatenate([self.hist_k[b], kb[j]])
            self.hist_v[b] = np.concatenate([self.hist_v[b], vb[j]])
            self.len[b] += n

    def Q(self, L):
        return oracle.window_quantized(int(L), self.S_sink, self.S_keep, self.S_flush)


def _tokens(cfg, b, t0, t1):
    return (synth.as_dtype(synth.keys(cfg, b, t0, t1), "bf16"),
            synth.as_dtype(synth.values(cfg, b, t0, t1), "bf16"))


def _run_loop(cfg, prefill, steps, S_sink, S_keep, S_flush):
    B = len(prefill)
    T_cap = 64 * ((max(prefill) + steps + 63) // 64 + 1)
    st = WindowState(cfg, B, T_cap, S_sink, S_keep, S_flush)
    for b, n in enumerate(prefill):
        if n:
            kb, vb = _tokens(cfg, b, 0, n)
            st.append(kb[None], vb[None], seqs=[b])
    for _ in range(steps):
        ks, vs = zip(*[_tokens(cfg, b, int(st.len[b]), int(st.len[b]) + 1) for b in range(B)])
        st.append(np.stack(ks), np.stack(vs))
    torch.cuda.synchronize()
    assert st.err.item() == 0
    return st


LOOPS = [
    # (config, prefill lengths, single-token steps, S_sink, S_keep, S_flush)
    (2, [150, 70, 3], 140, 4, 32, 64),      # flushes from new tokens (prefill) and from the ring
    (2, [0, 129, 64], 70, 0, 0, 64),        # no window: batches of 64 quantized as they fill
    (4, [200, 9], 90, 8, 24, 32),           # GQA 8, d 64
]


@pytest.mark.parametrize("ci,prefill,steps,S_sink,S_keep,S_flush", LOOPS)
def test_window_append_serving_loop(ci, prefill, steps, S_sink, S_keep, S_flush):
    cfg = synth.CONFIGS[ci]
    st = _run_loop(cfg, prefill, steps, S_sink, S_keep, S_flush)
    B, R = len(prefill), st.R
    ks = None if st.ks is None else st.ks.view(torch.int16).cpu().numpy().view(np.uint16)
    vs = None if st.vs is None else st.vs.view(torch.int16).cpu().numpy().view(np.uint16)
    kr = st.kr.view(torch.int16).cpu().numpy().view(np.uint16)
    vr = st.vr.view(torch.int16).cpu().numpy().view(np.uint16)
    # ---- sink and ring hold the window positions exactly
    for b in range(B):
        L, Q = int(st.len[b]), st.Q(st.len[b])
        for t in range(min(S_sink, L)):
            assert np.array_equal(ks[b, :, t], st.hist_k[b][t]), (b, t)
            assert np.array_equal(vs[b, :, t], st.hist_v[b][t]), (b, t)
        for t in range(S_sink + Q, L):
            assert np.array_equal(kr[b, :, t % R], st.hist_k[b][t]), (b, t)
            assert np.array_equal(vr[b, :, t % R], st.hist_v[b][t]), (b, t)
    # ---- quantized middle == direct quantize-append of the same tokens (float32 path:
    #      chunks of at most 64 tokens of one sequence)
    Qmax = max(st.Q(L) for L in st.len)
    ref = kvq.KVCache.allocate(B, cfg.Hkv, st.cache.T_cap, cfg.d, qp_of(cfg))
    for b in range(B):
        Q = st.Q(st.len[b])
        for c0 in range(0, Q, 64):
            c1 = min(Q, c0 + 64)
            kb = np.ascontiguousarray(st.hist_k[b][S_sink + c0:S_sink + c1])[None]
            vb = np.ascontiguousarray(st.hist_v[b][S_sink + c0:S_sink + c1])[None]
            kvq.quantize_append(t_(kb), t_(vb), st.Tk, st.Tv, qp_of(cfg), ref.view_sequence(b),
                                t_(np.array([c0], np.int32)))
    torch.cuda.synchronize()
    ng = cfg.d // cfg.group
    per_tok = [cfg.d * cfg.bits_k // 8, 4 * ng, cfg.d * cfg.bits_v // 8, 4 * ng]
    for p_got, p_ref, w in zip((st.cache.k_codes, st.cache.k_sz, st.cache.v_codes, st.cache.v_sz),
                               (ref.k_codes, ref.k_sz, ref.v_codes, ref.v_sz), per_tok):
        g = p_got.view(B, cfg.Hkv, st.cache.T_cap * w).cpu().numpy()
        r = p_ref.view(B, cfg.Hkv, st.cache.T_cap * w).cpu().numpy()
        for b in range(B):
            Q = st.Q(st.len[b])
            assert np.array_equal(g[b, :, :Q * w], r[b, :, :Q * w]), b
    assert Qmax > 0
    # ---- the oracle quantizes every position of the history itself; the GPU's quantized
    #      middle matches its codes end to end (<= 0.1% of codes off by one, s/z <= 1 ulp)
    Lmax = int(st.len.max())
    Tfull = 64 * ((Lmax + 63) // 64)
    kall = np.zeros((B, Tfull, cfg.Hkv, cfg.d), np.uint16)
    vall = np.zeros_like(kall)
    for b in range(B):
        kall[b, :st.len[b]], vall[b, :st.len[b]] = st.hist_k[b], st.hist_v[b]
    ofull = oracle.Cache(B, cfg.Hkv, Tfull, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    oracle.quantize_append(kall, vall, st.Tk_h, st.Tv_h, cfg.bits_k, cfg.bits_v, cfg.group,
                           cfg.clip_alpha, ofull, np.zeros(B, np.int32))
    gh = host_cache_from(st.cache, cfg)
    diff = total = 0
    for b in range(B):
        Q = st.Q(st.len[b])
        for h in range(cfg.Hkv):
            if Q == 0:
                continue
            gk, gv, gks, gvs = gh.unpack_tokens(b, h, 0, Q)
            ok_, ov, oks, ovs = ofull.unpack_tokens(b, h, S_sink, Q)
            for x, y in ((gk, ok_), (gv, ov)):
                dlt = x.astype(np.int32) - y.astype(np.int32)
                assert np.abs(dlt).max() <= 1
                diff += np.count_nonzero(dlt)
                total += dlt.size
            for x, y in ((gks, oks), (gvs, ovs)):
                assert np.abs(x.astype(np.int32) - y.astype(np.int32)).max() <= 1
    assert diff <= 1e-3 * total, diff / total
    # ---- decode parity over the same cache: the oracle's quantized middle at cache
    #      positions [0, Q), the sink and ring as kvq_window_append left them (checked
    #      above to be the exact tokens), against the oracle's windowed decode
    Tc = st.cache.T_cap
    om = oracle.Cache(B, cfg.Hkv, Tc, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    for b in range(B):
        Q = st.Q(st.len[b])
        for h in range(cfg.Hkv):
            if Q:
                om.pack_tokens(b, h, 0, *ofull.unpack_tokens(b, h, S_sink, Q))
    gc = upload_cache(om, cfg)
    q = synth.as_dtype(synth.queries(cfg.with_(B=B)), "bf16")
    want = oracle.window_decode(q, st.Tit_h, st.Tv_h, kall, vall, ofull, st.len, S_sink, S_keep,
                                S_flush)
    out = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.float32, device=DEV)
    ws = torch.empty(kvq.decode_workspace_bytes(gc, cfg.Hq, Tc), dtype=torch.uint8, device=DEV)
    kvq.decode_attention_window(t_(q), st.Tit, gc, S_sink, S_keep, S_flush, st.ks, st.vs,
                                st.kr, st.vr, st.Tv, t_(st.len), Lmax, out, ws, dev_err=st.err)
    torch.cuda.synchronize()
    assert st.err.item() == 0
    assert_close(out.cpu().numpy(), want, where=f"window append {S_sink}/{S_keep}/{S_flush}")
    # ---- and end to end over the GPU's own state: the same attention up to the code
    #      differences checked above (a sanity bound: with 2-bit codes one flipped code
    #      moves its value by a whole step, so this is looser than the parity bar)
    kvq.decode_attention_window(t_(q), st.Tit, st.cache, S_sink, S_keep, S_flush, st.ks, st.vs,
                                st.kr, st.vr, st.Tv, t_(st.len), Lmax, out, ws, dev_err=st.err)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert np.linalg.norm(got - want) <= 1e-2 * np.linalg.norm(want)


def test_window_append_out_of_range_is_flagged_and_skipped():
    """A sequence whose quantized middle would pass T_cap is skipped whole (cache, sink and
    ring untouched) and flagged; the other sequence is appended."""
    cfg = synth.CONFIGS[2]
    st = WindowState(cfg, 2, 64, 4, 8, 16)
    st.len[:] = [4 + 8 + 80 - 1, 10]          # Q = 64 now; one more token makes Q = 80 > 64
    kb, vb = zip(*[_tokens(cfg, b, 0, 1) for b in range(2)])
    before = st.kr.clone()
    kvq.window_append(t_(np.stack(kb)), t_(np.stack(vb)), st.Tk, st.Tv, qp_of(cfg), st.cache, 4,
                      8, 16, st.ks, st.vs, st.kr, st.vr, t_(st.len), dev_err=st.err)
    torch.cuda.synchronize()
    assert st.err.item() & kvq.KVQ_DEVERR_POS_RANGE
    assert torch.equal(st.kr[0], before[0])
    assert not torch.equal(st.kr[1], before[1])          # position 10 -> ring slot 10 % 24
