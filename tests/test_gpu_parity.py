"""GPU parity: the CUDA library against the float64 oracle, through the C ABI.

* quantize-append: bit-exact codes, scales, zero-points and packing when both sides see
  the same transformed inputs; end to end (transform on the GPU in float32) at most 0.1%
  of codes differ, each by +-1, and s/z by at most one float16 ulp;
* decode: against the oracle's attention over the same cache (built by the oracle),
  relative L2 <= 1e-3 and max-abs <= 5e-3 with float32 output; bfloat16 output within
  one bfloat16 ulp of the rounded oracle;
* the uncompressed bf16 comparator against the oracle's bf16 attention;
* sizes span several 64-token blocks and splits with ragged tails, plus the full
  workload shapes on sampled heads.
"""
import os

import numpy as np
import pytest
import torch

import decode_attention_post_b200 as kvq
import oracle
from tests import paging, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"
REL_L2, MAX_ABS = 1e-3, 5e-3


def t_(a, dtype=None):
    """numpy -> CUDA tensor (bf16 bit patterns become torch.bfloat16)."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def bf16_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def qp_of(cfg):
    return kvq.QParams(cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha)


def planes_to_host(cache):
    return [p.cpu().numpy() for p in (cache.k_codes, cache.k_sz, cache.v_codes, cache.v_sz)]


def upload_cache(ocache, cfg):
    gc = kvq.KVCache.allocate(ocache.B, ocache.Hkv, ocache.T_cap, ocache.d, qp_of(cfg))
    for dst, src in zip((gc.k_codes, gc.k_sz, gc.v_codes, gc.v_sz), ocache.planes()):
        dst.copy_(torch.from_numpy(src.view(np.uint8)))
    return gc


def host_cache_from(gc, cfg):
    oc = oracle.Cache(gc.B, gc.Hkv, gc.T_cap, gc.d, cfg.bits_k, cfg.bits_v, cfg.group)
    kc, ksz, vc, vsz = planes_to_host(gc)
    oc.k_codes[:] = kc
    oc.k_sz[:] = ksz.view(np.uint16)
    oc.v_codes[:] = vc
    oc.v_sz[:] = vsz.view(np.uint16)
    return oc


def small(cfg, **kw):
    return cfg.with_(**kw)


def gpu_append(cfg, k, v, Tk, Tv, pos, cache=None):
    if cache is None:
        cache = kvq.KVCache.allocate(k.shape[0], cfg.Hkv, cfg.T_cap, cfg.d, qp_of(cfg))
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    kvq.quantize_append(t_(k), t_(v), None if Tk is None else t_(Tk),
                        None if Tv is None else t_(Tv), qp_of(cfg), cache,
                        t_(np.asarray(pos, np.int32)), dev_err=err)
    torch.cuda.synchronize()
    return cache, int(err.item())


def gpu_decode(cfg, q, M, cache, seqlens, max_seqlen=None, out_dtype=torch.float32, Hq=None):
    B = q.shape[0]
    Hq = q.shape[1]
    max_seqlen = int(max(seqlens)) if max_seqlen is None else max_seqlen
    ws = torch.empty(kvq.decode_workspace_bytes(cache, Hq, max_seqlen), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty((B, Hq, cfg.d), dtype=out_dtype, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    kvq.decode_attention(t_(q), None if M is None else t_(M), cache,
                         t_(np.asarray(seqlens, np.int32)), max_seqlen, out, ws, dev_err=err)
    torch.cuda.synchronize()
    return out, int(err.item())


def assert_close(got, want, rel=REL_L2, mx=MAX_ABS, where=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.isfinite(got).all(), where
    err = got - want
    rl2 = np.linalg.norm(err) / max(np.linalg.norm(want), 1e-30)
    assert rl2 <= rel and np.abs(err).max() <= mx, f"{where} rel-L2 {rl2:.3e} max-abs {np.abs(err).max():.3e}"
    return rl2


def assert_bf16_output(out_bf16, out_f32, want_f64, where=""):
    """bfloat16 output path: bit-identical to round-to-nearest-even of the same kernel's
    float32 output (which assert_close checks against the oracle), and every element
    within half a bfloat16 ulp plus the max-abs bound of the oracle."""
    g = synth.bf16_bits_to_f32(bf16_bits(out_bf16)).astype(np.float64)
    ref = bf16_bits(out_f32.to(torch.bfloat16))
    assert np.array_equal(bf16_bits(out_bf16), ref), f"{where}: bf16 output != rn(f32 output)"
    w = np.asarray(want_f64, np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(w), 1e-30))) - 7)
    bad = np.abs(g - w) > 0.5 * ulp + MAX_ABS
    assert not bad.any(), f"{where}: {np.count_nonzero(bad)} elements beyond rounding + {MAX_ABS}"


# ======================================================================== append

APPEND_CASES = [
    # (config, B, n, pos list, dtype)
    (synth.CONFIGS[0], 1, 2048, [0], "f32"),
    (small(synth.CONFIGS[1], T_cap=256), 3, 77, [0, 64, 179], "bf16"),
    (small(synth.CONFIGS[3], T_cap=128), 2, 45, [3, 80], "bf16"),
    (small(synth.CONFIGS[4], T_cap=256), 2, 130, [0, 126], "bf16"),
    (small(synth.CONFIGS[1], T_cap=64, group=64), 2, 9, [1, 50], "f32"),
    (small(synth.CONFIGS[1], T_cap=64, group=32, bits_k=4, bits_v=4, clip_alpha=0.1), 1, 33, [7], "f32"),
]


def _inputs(cfg, B, n, dtype, seed=0):
    c = cfg.with_(B=B)
    k, v = synth.kv_batch(c, 0, n)
    return synth.as_dtype(k, dtype), synth.as_dtype(v, dtype)


@pytest.mark.parametrize("cfg,B,n,pos,dtype", APPEND_CASES)
def test_append_identity_transform_bit_exact(cfg, B, n, pos, dtype):
    k, v = _inputs(cfg, B, n, dtype)
    oc = oracle.Cache(B, cfg.Hkv, cfg.T_cap, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    oracle.quantize_append(k, v, None, None, cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha,
                           oc, pos)
    gc, err = gpu_append(cfg, k, v, None, None, pos)
    assert err == 0
    for name, a, b in zip(("k_codes", "k_sz", "v_codes", "v_sz"), planes_to_host(gc), oc.planes()):
        assert np.array_equal(a, b.view(np.uint8)), name


@pytest.mark.parametrize("cfg,B,n,pos,dtype", APPEND_CASES[:4])
def test_append_same_transformed_inputs_bit_exact(cfg, B, n, pos, dtype):
    """Both sides quantize the oracle's float32 transformed keys/values."""
    k, v = _inputs(cfg, B, n, dtype)
    Tk, Tv, _ = synth.transforms(cfg)
    oc = oracle.Cache(B, cfg.Hkv, cfg.T_cap, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    kt, vt = oracle.quantize_append(k, v, Tk, Tv, cfg.bits_k, cfg.bits_v, cfg.group,
                                    cfg.clip_alpha, oc, pos, return_transformed=True)
    gc, err = gpu_append(cfg, kt, vt, None, None, pos)
    assert err == 0
    for name, a, b in zip(("k_codes", "k_sz", "v_codes", "v_sz"), planes_to_host(gc), oc.planes()):
        assert np.array_equal(a, b.view(np.uint8)), name


def _compare_codes_end_to_end(gc, oc, cfg, B, pos, n):
    g = host_cache_from(gc, cfg)
    total = diff = 0
    for b in range(B):
        for h in range(cfg.Hkv):
            gk, gv, gks, gvs = g.unpack_tokens(b, h, pos[b], n)
            ok_, ov, oks, ovs = oc.unpack_tokens(b, h, pos[b], n)
            for a, c in ((gk, ok_), (gv, ov)):
                dlt = a.astype(np.int32) - c.astype(np.int32)
                assert np.abs(dlt).max() <= 1
                diff += np.count_nonzero(dlt)
                total += dlt.size
            for a, c in ((gks, oks), (gvs, ovs)):
                da = np.abs(a.astype(np.int32) - c.astype(np.int32))   # f16 bit patterns
                assert da.max() <= 1                                    # same sign, <= 1 ulp
    return diff / total


@pytest.mark.parametrize("cfg,B,n,pos,dtype", APPEND_CASES[:4])
def test_append_with_transform_end_to_end(cfg, B, n, pos, dtype):
    k, v = _inputs(cfg, B, n, dtype)
    Tk, Tv, _ = synth.transforms(cfg)
    oc = oracle.Cache(B, cfg.Hkv, cfg.T_cap, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    oracle.quantize_append(k, v, Tk, Tv, cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha, oc, pos)
    gc, err = gpu_append(cfg, k, v, Tk, Tv, pos)
    assert err == 0
    frac = _compare_codes_end_to_end(gc, oc, cfg, B, pos, n)
    assert frac <= 1e-3, frac


MMA_APPEND_CASES = [
    # (d, bits_k, bits_v, group, clip_alpha, B, n, pos): bf16 chunks of >= 256 tokens take
    # the tensor-core transform path; kappa 0, 1 and the general kappa >= 2 path
    (64, 2, 2, 64, 0.01, 3, 130, [0, 200, 64]),
    (128, 2, 2, 128, 0.01, 2, 300, [0, 212]),
    (128, 4, 2, 128, 0.005, 1, 512, [0]),
    (128, 4, 4, 32, 0.1, 2, 140, [5, 300]),
    (64, 2, 4, 64, 0.05, 2, 160, [96, 0]),
    (64, 4, 2, 32, 0.05, 2, 200, [0, 64]),     # d 64, group 32, kappa 1, 4-bit keys
    (64, 2, 2, 32, 0.01, 1, 300, [0]),          # d 64, group 32, kappa 0
]


@pytest.mark.parametrize("d,bk,bv,group,alpha,B,n,pos", MMA_APPEND_CASES)
def test_append_tensor_core_path_with_identity_matrix_bit_exact(d, bk, bv, group, alpha, B, n, pos):
    """T = I passed as a matrix: bf16 inputs times the identity on tensor cores reproduce
    the inputs exactly, so clipping, quantization and packing of the tensor-core path must
    equal the oracle's (T = None) bit for bit."""
    cfg = synth.Config(97, "mma", B=B, Hq=4 * 2, Hkv=2, d=d, T_cap=512, bits_k=bk, bits_v=bv,
                       group=group, clip_alpha=alpha, in_dtype="bf16", q_dtype="bf16",
                       out_dtype="bf16", seq_lo=1, seq_hi=1)
    k, v = _inputs(cfg, B, n, "bf16")
    eye = np.broadcast_to(np.eye(d, dtype=np.float32), (cfg.Hkv, d, d)).copy()
    oc = oracle.Cache(B, cfg.Hkv, cfg.T_cap, d, bk, bv, group)
    oracle.quantize_append(k, v, None, None, bk, bv, group, alpha, oc, pos)
    gc, err = gpu_append(cfg, k, v, eye, eye, pos)
    assert err == 0
    for name, a, b in zip(("k_codes", "k_sz", "v_codes", "v_sz"), planes_to_host(gc), oc.planes()):
        assert np.array_equal(a, b.view(np.uint8)), name


@pytest.mark.parametrize("d,bk,bv,group,alpha,B,n,pos", MMA_APPEND_CASES[:3])
def test_append_tensor_core_path_end_to_end(d, bk, bv, group, alpha, B, n, pos):
    cfg = synth.Config(96, "mma", B=B, Hq=8, Hkv=2, d=d, T_cap=512, bits_k=bk, bits_v=bv,
                       group=group, clip_alpha=alpha, in_dtype="bf16", q_dtype="bf16",
                       out_dtype="bf16", seq_lo=1, seq_hi=1)
    k, v = _inputs(cfg, B, n, "bf16")
    Tk, Tv, _ = synth.transforms(cfg)
    oc = oracle.Cache(B, cfg.Hkv, cfg.T_cap, d, bk, bv, group)
    oracle.quantize_append(k, v, Tk, Tv, bk, bv, group, alpha, oc, pos)
    gc, err = gpu_append(cfg, k, v, Tk, Tv, pos)
    assert err == 0
    frac = _compare_codes_end_to_end(gc, oc, cfg, B, pos, n)
    assert frac <= 1e-3, frac


def test_append_out_of_range_sequence_is_skipped_and_flagged():
    cfg = small(synth.CONFIGS[1], T_cap=64)
    k, v = _inputs(cfg, 2, 10, "f32")
    gc, err = gpu_append(cfg, k, v, None, None, [60, 5])      # 60 + 10 > 64
    assert err & kvq.KVQ_DEVERR_POS_RANGE
    host = host_cache_from(gc, cfg)
    kc, _, ksz, _ = host.unpack_tokens(0, 0, 0, 64)
    assert not kc.any() and not ksz.any()                    # sequence 0 untouched
    kc1, _, _, _ = host.unpack_tokens(1, 0, 5, 10)
    assert kc1.any()


def test_append_single_tokens_accumulate():
    """Decode-time appends one token at a time land exactly where a chunk append puts them."""
    cfg = small(synth.CONFIGS[1], T_cap=64)
    k, v = _inputs(cfg, 2, 20, "bf16")
    Tk, Tv, _ = synth.transforms(cfg)
    whole, _ = gpu_append(cfg, k, v, Tk, Tv, [0, 0])
    step = kvq.KVCache.allocate(2, cfg.Hkv, cfg.T_cap, cfg.d, qp_of(cfg))
    for i in range(20):
        gpu_append(cfg, np.ascontiguousarray(k[:, i:i + 1]), np.ascontiguousarray(v[:, i:i + 1]),
                   Tk, Tv, [i, i], cache=step)
    for a, b in zip(planes_to_host(whole), planes_to_host(step)):
        assert np.array_equal(a, b)


# ======================================================================== decode

def oracle_built_cache(cfg, B, T_fill, with_T=True):
    """Oracle-quantized cache holding T_fill synthetic tokens per sequence."""
    c = cfg.with_(B=B)
    k, v = synth.kv_batch(c, 0, T_fill)
    k, v = synth.as_dtype(k, cfg.in_dtype), synth.as_dtype(v, cfg.in_dtype)
    Tk, Tv, Tit = synth.transforms(cfg)
    oc = oracle.Cache(B, cfg.Hkv, cfg.T_cap, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    oracle.quantize_append(k, v, Tk if with_T else None, Tv if with_T else None, cfg.bits_k,
                           cfg.bits_v, cfg.group, cfg.clip_alpha, oc, [0] * B)
    return oc, (Tit if with_T else None)


DECODE_CASES = [
    # (name, cfg, B, seqlens)
    ("cfg0", synth.CONFIGS[0], 1, [2048]),
    ("gqa4-ragged", small(synth.CONFIGS[2], T_cap=1024), 3, [1000, 1, 577]),
    ("gqa4-k4v2", small(synth.CONFIGS[3], T_cap=1280), 2, [1280, 700]),
    ("gqa8-d64", small(synth.CONFIGS[4], T_cap=768), 2, [768, 333]),
    ("gqa4-v4", small(synth.CONFIGS[1], T_cap=512, bits_v=4), 2, [512, 129]),
    ("gqa8-d128", small(synth.CONFIGS[1], T_cap=640, Hq=64), 2, [640, 321]),
    ("gqa8-d128-k4v4", small(synth.CONFIGS[1], T_cap=384, Hq=64, bits_k=4, bits_v=4), 2,
     [384, 70]),
]


@pytest.mark.parametrize("name,cfg,B,seql", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_matches_oracle(name, cfg, B, seql):
    oc, M = oracle_built_cache(cfg, B, cfg.T_cap)
    gc = upload_cache(oc, cfg)
    q = synth.as_dtype(synth.queries(cfg.with_(B=B)), cfg.q_dtype)
    want = oracle.decode(q, M, oc, np.array(seql, np.int32))
    out, err = gpu_decode(cfg, q, M, gc, seql)
    assert err == 0
    assert_close(out.cpu().numpy(), want, where=name)
    out16, _ = gpu_decode(cfg, q, M, gc, seql, out_dtype=torch.bfloat16)
    assert_bf16_output(out16, out, want, where=name)


@pytest.mark.parametrize("splits", ["1", "2", "5", "16", "200"])
def test_decode_split_invariance(splits, monkeypatch):
    cfg = small(synth.CONFIGS[2], T_cap=1024)
    oc, M = oracle_built_cache(cfg, 2, 1024)
    gc = upload_cache(oc, cfg)
    q = synth.as_dtype(synth.queries(cfg.with_(B=2)), cfg.q_dtype)
    seql = [1024, 517]
    want = oracle.decode(q, M, oc, np.array(seql, np.int32))
    monkeypatch.setenv("KVQ_DECODE_SPLITS", splits)
    out, err = gpu_decode(cfg, q, M, gc, seql)
    assert err == 0
    assert_close(out.cpu().numpy(), want, where=f"splits={splits}")


def test_decode_wait_timeout_is_flagged_and_the_context_stays_usable(monkeypatch):
    """Failure path of the bounded pipeline waits, made to run out without a fault: the
    test hook KVQ_TEST_STALL_NS makes every decode warp first wait 1 ms on a barrier that
    nothing arrives at. Each warp then takes the timeout path (waits for its own copies
    in flight, skips its blocks) and the call flags KVQ_DEVERR_WAIT_TIMEOUT. The next
    call without the hook gives the oracle's result, so the context is intact."""
    cfg = small(synth.CONFIGS[2], T_cap=1024)
    oc, M = oracle_built_cache(cfg, 2, 1024)
    gc = upload_cache(oc, cfg)
    q = synth.as_dtype(synth.queries(cfg.with_(B=2)), cfg.q_dtype)
    seql = [1024, 517]
    want = oracle.decode(q, M, oc, np.array(seql, np.int32))
    monkeypatch.setenv("KVQ_TEST_STALL_NS", "1000000")
    _, err = gpu_decode(cfg, q, M, gc, seql)
    assert err & kvq.KVQ_DEVERR_WAIT_TIMEOUT
    monkeypatch.delenv("KVQ_TEST_STALL_NS")
    out, err = gpu_decode(cfg, q, M, gc, seql)
    assert err == 0
    assert_close(out.cpu().numpy(), want, where="after the timeout test")


@pytest.mark.parametrize("splits", ["1", "3", "100"])
def test_decode_many_short_sequences(splits, monkeypatch):
    # short, empty and capacity-length sequences side by side, each split count
    cfg = small(synth.CONFIGS[1], T_cap=256)
    seql = [5, 0, 64, 200, 0, 0, 1, 130, 256, 65]
    oc, M = oracle_built_cache(cfg, len(seql), 256)
    gc = upload_cache(oc, cfg)
    q = synth.as_dtype(synth.queries(cfg.with_(B=len(seql))), cfg.q_dtype)
    want = oracle.decode(q, M, oc, np.array(seql, np.int32))
    monkeypatch.setenv("KVQ_DECODE_SPLITS", splits)
    out, err = gpu_decode(cfg, q, M, gc, seql, max_seqlen=256)
    assert err == 0
    assert not out[1].any() and not out[4].any() and not out[5].any()
    assert_close(out.cpu().numpy(), want, where=f"splits={splits}")


def test_decode_edge_lengths():
    cfg = small(synth.CONFIGS[1], T_cap=320)
    seql = [0, 1, 63, 64, 65, 128, 319, 320]
    oc, M = oracle_built_cache(cfg, len(seql), 320)
    gc = upload_cache(oc, cfg)
    q = synth.as_dtype(synth.queries(cfg.with_(B=len(seql))), "bf16")
    want = oracle.decode(q, M, oc, np.array(seql, np.int32))
    out, err = gpu_decode(cfg, q, M, gc, seql, max_seqlen=320)
    assert err == 0
    assert not out[0].any()                                  # empty sequence -> zeros
    assert_close(out.cpu().numpy(), want, where="edges")
    # max_seqlen below capacity, and every sequence empty
    out, err = gpu_decode(cfg, q, M, gc, [0] * len(seql), max_seqlen=0)
    assert err == 0 and not out.any()


@pytest.mark.parametrize("qscale", [1e-30, 1e-6, 1e3, 1e12])
def test_decode_query_magnitude(qscale):
    # the key product runs on q~ as per-head 16-bit fixed point: its exponent must follow
    # the query's magnitude from tiny to huge (softmax over near-equal or one-hot logits)
    cfg = small(synth.CONFIGS[2], T_cap=512)
    seql = [512, 300]
    oc, M = oracle_built_cache(cfg, 2, 512)
    gc = upload_cache(oc, cfg)
    q = synth.queries(cfg.with_(B=2)).astype(np.float64)
    q[:, ::3] *= 1e-3                                   # heads of very different sizes
    q = synth.as_dtype((q * qscale).astype(np.float32), "f32")
    want = oracle.decode(q, M, oc, np.array(seql, np.int32))
    out, err = gpu_decode(cfg, q, M, gc, seql)
    assert err == 0
    assert_close(out.cpu().numpy(), want, where=f"qscale={qscale}")


def test_decode_seqlen_beyond_max_is_clamped_and_flagged():
    cfg = small(synth.CONFIGS[1], T_cap=256)
    oc, M = oracle_built_cache(cfg, 1, 256)
    gc = upload_cache(oc, cfg)
    q = synth.as_dtype(synth.queries(cfg.with_(B=1)), "bf16")
    out, err = gpu_decode(cfg, q, M, gc, [250], max_seqlen=128)
    assert err & kvq.KVQ_DEVERR_SEQLEN_CLAMPED
    want = oracle.decode(q, M, oc, np.array([128], np.int32))
    assert_close(out.cpu().numpy(), want, where="clamped")


def test_decode_identity_transform_and_fp32_query():
    cfg = small(synth.CONFIGS[0], T_cap=512)
    oc, _ = oracle_built_cache(cfg, 1, 512, with_T=False)
    gc = upload_cache(oc, cfg)
    q = synth.queries(cfg.with_(B=1))
    want = oracle.decode(q, None, oc, np.array([500], np.int32))
    out, err = gpu_decode(cfg, q, None, gc, [500])
    assert err == 0
    assert_close(out.cpu().numpy(), want, where="identity")


def test_end_to_end_gpu_append_then_decode():
    """GPU append -> GPU decode against oracle append -> oracle decode (independent
    caches; the rare +-1 code flips move the output far less than the tolerance)."""
    cfg = small(synth.CONFIGS[2], T_cap=512)
    B = 2
    k, v = synth.kv_batch(cfg.with_(B=B), 0, 512)
    k, v = synth.as_dtype(k, "bf16"), synth.as_dtype(v, "bf16")
    Tk, Tv, Tit = synth.transforms(cfg)
    oc = oracle.Cache(B, cfg.Hkv, cfg.T_cap, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    oracle.quantize_append(k, v, Tk, Tv, 2, 2, 128, cfg.clip_alpha, oc, [0, 0])
    gc, err = gpu_append(cfg, k, v, Tk, Tv, [0, 0])
    q = synth.as_dtype(synth.queries(cfg.with_(B=B)), "bf16")
    seql = [512, 300]
    want = oracle.decode(q, Tit, oc, np.array(seql, np.int32))
    out, err2 = gpu_decode(cfg, q, Tit, gc, seql)
    assert err == 0 and err2 == 0
    assert_close(out.cpu().numpy(), want, rel=5e-3, mx=5e-2, where="e2e")


# ======================================================================== full size

def _random_full_cache(cfg, seql):
    oc = oracle.Cache.for_config(cfg)
    for b in range(cfg.B):
        n = int(seql[b])
        n16 = (n + 15) // 16 * 16
        kc, vc, ks, kz, vs, vz = synth.random_cache_fields(cfg, b, n16)
        f = lambda a: a.astype(np.float16).view(np.uint16)
        for h in range(cfg.Hkv):
            oc.pack_tokens(b, h, 0, kc[h], vc[h], np.stack([f(ks[h]), f(kz[h])], -1),
                           np.stack([f(vs[h]), f(vz[h])], -1))
    return oc


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_decode_full_size_sampled(idx):
    """Full workload shape, bench launch configuration; oracle on sampled heads."""
    cfg = synth.CONFIGS[idx]
    seql = synth.seqlens(cfg)
    oc = _random_full_cache(cfg, seql)
    gc = upload_cache(oc, cfg)
    q = synth.as_dtype(synth.queries(cfg), cfg.q_dtype)
    _, _, Tit = synth.transforms(cfg)
    out, err = gpu_decode(cfg, q, Tit, gc, seql, max_seqlen=cfg.T_cap)
    out16, err16 = gpu_decode(cfg, q, Tit, gc, seql, max_seqlen=cfg.T_cap,
                              out_dtype=torch.bfloat16)
    assert err == 0 and err16 == 0
    rng = np.random.default_rng(idx)
    sel = np.stack([rng.integers(0, cfg.B, 12), rng.integers(0, cfg.Hq, 12)], 1).astype(np.int32)
    sel[0] = [0, 0]
    sel[1] = [cfg.B - 1, cfg.Hq - 1]
    sel = np.unique(sel, axis=0)
    want = oracle.decode(q, Tit, oc, seql, sel=sel)
    got = out.cpu().numpy()
    for b, h in sel:
        assert_close(got[b, h], want[b, h], where=f"cfg{idx} b{b} h{h}")
        assert_bf16_output(out16[b, h], out[b, h], want[b, h], where=f"cfg{idx} b{b} h{h} bf16")
    assert np.isfinite(got).all()
    assert np.array_equal(bf16_bits(out16), bf16_bits(out.to(torch.bfloat16)))


def test_window_decode_full_size_sampled():
    """The batch-64 / 12K-16K shape with the bench's window (S_sink 64, S_keep 256, S_flush
    128) in the bench's launch configuration: random quantized middles from cache position
    0, random bfloat16 sink and ring rows (the unused ring slots hold NaN bit patterns);
    the oracle's windowed decode on sampled sequences, each run on its own."""
    cfg = synth.CONFIGS[2]
    S_sink, S_keep, S_flush = 64, 256, 128
    R = S_keep + S_flush
    B, Hkv, d, T = cfg.B, cfg.Hkv, cfg.d, cfg.T_cap
    seql = synth.seqlens(cfg)
    Qs = [oracle.window_quantized(int(L), S_sink, S_keep, S_flush) for L in seql]
    gpu_c = oracle.Cache.for_config(cfg)
    ks = np.full((B, Hkv, S_sink, d), 0x7FC1, np.uint16)
    vs = ks.copy()
    kr = np.full((B, Hkv, R, d), 0x7FC1, np.uint16)
    vr = kr.copy()
    f16 = lambda a: a.astype(np.float16).view(np.uint16)
    win = {}
    for b in range(B):
        L, Q = int(seql[b]), Qs[b]
        kc, vc, k_s, k_z, v_s, v_z = synth.random_cache_fields(cfg, b, (Q + 15) // 16 * 16)
        for h in range(Hkv):
            gpu_c.pack_tokens(b, h, 0, kc[h], vc[h], np.stack([f16(k_s[h]), f16(k_z[h])], -1),
                              np.stack([f16(v_s[h]), f16(v_z[h])], -1))
        pos = list(range(min(S_sink, L))) + list(range(S_sink + Q, L))
        kw, vw = synth.window_tokens(cfg, b, len(pos))
        kw, vw = synth.as_dtype(kw, "bf16"), synth.as_dtype(vw, "bf16")
        for j, t in enumerate(pos):
            if t < S_sink:
                ks[b, :, t], vs[b, :, t] = kw[:, j], vw[:, j]
            else:
                kr[b, :, t % R], vr[b, :, t % R] = kw[:, j], vw[:, j]
        win[b] = (pos, kw, vw, (kc, vc, k_s, k_z, v_s, v_z))
    gc = upload_cache(gpu_c, cfg)
    q = synth.as_dtype(synth.queries(cfg), "bf16")
    _, Tv, Tit = synth.transforms(cfg)
    out = torch.empty((B, cfg.Hq, d), dtype=torch.float32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(kvq.decode_workspace_bytes(gc, cfg.Hq, T), dtype=torch.uint8, device=DEV)
    kvq.decode_attention_window(t_(q), t_(Tit), gc, S_sink, S_keep, S_flush, t_(ks), t_(vs),
                                t_(kr), t_(vr), t_(Tv), t_(seql.astype(np.int32)), T, out, ws,
                                dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    for b in (0, int(np.argmax(seql)), B - 1):
        L, Q = int(seql[b]), Qs[b]
        pos, kw, vw, (kc, vc, k_s, k_z, v_s, v_z) = win[b]
        one = oracle.Cache(1, Hkv, T, d, cfg.bits_k, cfg.bits_v, cfg.group)
        for h in range(Hkv):
            one.pack_tokens(0, h, S_sink, kc[h][:Q], vc[h][:Q],
                            np.stack([f16(k_s[h][:Q]), f16(k_z[h][:Q])], -1),
                            np.stack([f16(v_s[h][:Q]), f16(v_z[h][:Q])], -1))
        k_all = np.zeros((1, T, Hkv, d), np.uint16)
        v_all = np.zeros_like(k_all)
        for j, t in enumerate(pos):
            k_all[0, t], v_all[0, t] = kw[:, j], vw[:, j]
        want = oracle.window_decode(q[b:b + 1], Tit, Tv, k_all, v_all, one,
                                    np.array([L], np.int32), S_sink, S_keep, S_flush)
        assert_close(got[b:b + 1], want, where=f"window full size b{b}")


def test_append_full_size_sampled_config4():
    """32768-token chunk append of the GPT-OSS-like shape; oracle on sampled tokens."""
    cfg = synth.CONFIGS[4]
    n = cfg.append_n
    k, v = synth.kv_batch(cfg, 0, n)
    kb, vb = synth.as_dtype(k, "bf16"), synth.as_dtype(v, "bf16")
    Tk, Tv, _ = synth.transforms(cfg)
    gc, err = gpu_append(cfg, kb, vb, Tk, Tv, [0] * cfg.B)
    assert err == 0
    hc = host_cache_from(gc, cfg)
    rng = np.random.default_rng(4)
    diff = total = 0
    for b, i in zip(rng.integers(0, cfg.B, 24), rng.integers(0, n, 24)):
        i = int(i) // 16 * 16
        oc = oracle.Cache(1, cfg.Hkv, 16, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
        oracle.quantize_append(np.ascontiguousarray(kb[b:b + 1, i:i + 16]),
                               np.ascontiguousarray(vb[b:b + 1, i:i + 16]), Tk, Tv, cfg.bits_k,
                               cfg.bits_v, cfg.group, cfg.clip_alpha, oc, [0])
        for h in range(cfg.Hkv):
            gk, gv, gks, gvs = hc.unpack_tokens(int(b), h, i, 16)
            ok_, ov, oks, ovs = oc.unpack_tokens(0, h, 0, 16)
            for a, c in ((gk, ok_), (gv, ov)):
                d_ = a.astype(np.int32) - c.astype(np.int32)
                assert np.abs(d_).max() <= 1
                diff += np.count_nonzero(d_)
                total += d_.size
            for a, c in ((gks, oks), (gvs, ovs)):
                assert np.abs(a.astype(np.int32) - c.astype(np.int32)).max() <= 1
    assert diff / total <= 1e-3


# ======================================================================== bf16 comparator

@pytest.mark.parametrize("G,d", [(4, 128), (8, 64)])
def test_bf16_decode_matches_oracle(G, d):
    rng = np.random.default_rng(G + d)
    B, Hkv, T_cap = 3, 2, 320
    Hq = G * Hkv
    q = synth.f32_to_bf16_bits(rng.standard_normal((B, Hq, d)).astype(np.float32))
    K = synth.f32_to_bf16_bits((rng.standard_normal((B, Hkv, T_cap, d)) * 2).astype(np.float32))
    V = synth.f32_to_bf16_bits(rng.standard_normal((B, Hkv, T_cap, d)).astype(np.float32))
    # poison the unused tail: the kernel must never read past seqlen into its result
    seql = np.array([320, 1, 150], np.int32)
    K[2, :, 150:] = 0x7FC0
    V[2, :, 150:] = 0x7FC0
    want = oracle.bf16_decode(q, K, V, seql, Hkv)
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    for splits in ("1", "3", "40"):
        os.environ["KVQ_DECODE_SPLITS"] = splits
        try:
            ws = torch.empty(kvq.bf16_decode_workspace_bytes(B, Hq, Hkv, d, T_cap),
                             dtype=torch.uint8, device=DEV)
            kvq.bf16_decode(t_(q), t_(K), t_(V), t_(seql), T_cap, out, ws, dev_err=err)
        finally:
            del os.environ["KVQ_DECODE_SPLITS"]
        torch.cuda.synchronize()
        assert err.item() == 0
        g = synth.bf16_bits_to_f32(bf16_bits(out)).astype(np.float64)
        # bf16 output of a float32 computation: rounding plus the float32-path tolerance
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7)
        assert np.all(np.abs(g - want) <= 0.5 * ulp + MAX_ABS), splits
        rl2 = np.linalg.norm(g - want) / np.linalg.norm(want)
        assert rl2 <= 3e-3, (splits, rl2)      # bf16 rounding alone is about 1.5e-3


# ----------------------------------------------------------------------------- paged cache


def _paged(cfg, B, page_tokens, extra_pages, seed):
    per = cfg.T_cap // page_tokens
    num_pages = B * per + extra_pages
    table = paging.random_table(np.random.default_rng(seed), B, per, num_pages)
    tb = paging.token_bytes(cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    return table, num_pages, tb


def paged_upload(oc, cfg, page_tokens, extra_pages=5, seed=0):
    """The oracle's contiguous planes moved into a shuffled page pool on the GPU."""
    table, num_pages, tb = _paged(cfg, oc.B, page_tokens, extra_pages, seed)
    pools = paging.scatter([p.view(np.uint8) for p in oc.planes()], table, oc.Hkv, oc.T_cap,
                           page_tokens, num_pages, tb)
    gc = kvq.KVCache.allocate_paged(num_pages, page_tokens, t_(table), oc.Hkv, oc.d, qp_of(cfg))
    for dst, src in zip((gc.k_codes, gc.k_sz, gc.v_codes, gc.v_sz), pools):
        dst.copy_(torch.from_numpy(src))
    return gc


@pytest.mark.parametrize("page_tokens", [64, 256])
def test_paged_decode_matches_oracle(page_tokens):
    cfg = small(synth.CONFIGS[2], T_cap=1024)
    seql = [1000, 1, 577]
    oc, M = oracle_built_cache(cfg, 3, 1024)
    gc = paged_upload(oc, cfg, page_tokens, seed=page_tokens)
    q = synth.as_dtype(synth.queries(cfg.with_(B=3)), cfg.q_dtype)
    want = oracle.decode(q, M, oc, np.array(seql, np.int32))
    out, err = gpu_decode(cfg, q, M, gc, seql)
    assert err == 0
    assert_close(out.cpu().numpy(), want, where=f"paged {page_tokens}")


@pytest.mark.parametrize("cfg,B,n,pos,dtype,with_T", [
    (small(synth.CONFIGS[1], T_cap=512), 3, 1, [0, 100, 511], "bf16", True),    # decode-time
    (small(synth.CONFIGS[1], T_cap=512), 3, 77, [0, 64, 435], "f32", False),
    (small(synth.CONFIGS[4], T_cap=512), 2, 300, [0, 212], "bf16", True),       # tensor cores
])
def test_paged_append_matches_contiguous_bytes(cfg, B, n, pos, dtype, with_T):
    """An append into a shuffled page pool, gathered back, is byte-identical to the same
    append into contiguous planes (which the oracle pins), and leaves unused pages empty."""
    k, v = _inputs(cfg, B, n, dtype)
    Tk, Tv, _ = synth.transforms(cfg) if with_T else (None, None, None)
    ref, err = gpu_append(cfg, k, v, Tk, Tv, pos)
    assert err == 0
    if not with_T:
        oc = oracle.Cache(B, cfg.Hkv, cfg.T_cap, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
        oracle.quantize_append(k, v, None, None, cfg.bits_k, cfg.bits_v, cfg.group,
                               cfg.clip_alpha, oc, pos)
        for a, b in zip(planes_to_host(ref), oc.planes()):
            assert np.array_equal(a, b.view(np.uint8))
    page_tokens = 128
    table, num_pages, tb = _paged(cfg, B, page_tokens, 4, n)
    gc = kvq.KVCache.allocate_paged(num_pages, page_tokens, t_(table), cfg.Hkv, cfg.d,
                                    qp_of(cfg))
    gc, err = gpu_append(cfg, k, v, Tk, Tv, pos, cache=gc)
    assert err == 0
    back = paging.gather(planes_to_host(gc), table, cfg.Hkv, page_tokens, tb)
    for name, a, b in zip(("k_codes", "k_sz", "v_codes", "v_sz"), back, planes_to_host(ref)):
        assert np.array_equal(a, b), name
    unused = sorted(set(range(num_pages)) - set(table.reshape(-1).tolist()))
    for pool in planes_to_host(gc):
        assert not pool.reshape(num_pages, -1)[unused].any()


def test_paged_out_of_range_page_is_flagged():
    cfg = small(synth.CONFIGS[2], T_cap=256)
    seql = [256, 130]
    oc, M = oracle_built_cache(cfg, 2, 256)
    gc = paged_upload(oc, cfg, 64, extra_pages=0)
    gc.block_table[1, 1] = gc.num_pages + 3                 # outside the pool
    q = synth.as_dtype(synth.queries(cfg.with_(B=2)), cfg.q_dtype)
    out, err = gpu_decode(cfg, q, M, gc, seql)
    assert err & 0x10
    k, v = _inputs(cfg, 2, 1, "bf16")
    _, err = gpu_append(cfg, k, v, None, None, [0, 70], cache=gc)   # 70 -> page entry [1][1]
    assert err & 0x10


# ----------------------------------------------------------------------------- full-precision window


def _round64(x):
    return max(64, (x + 63) // 64 * 64)


@pytest.mark.parametrize("ci,S_sink,S_keep,S_flush,seql,variant", [
    (2, 4, 32, 64, [300, 20, 97], ""),    # quantized middles; one sequence entirely in the window
    (2, 0, 0, 64, [256, 128, 64], ""),    # no window: every position quantized
    (2, 64, 128, 128, [700, 300, 0], ""), # an empty sequence
    (4, 8, 64, 64, [500, 71], ""),        # GQA 8, d 64
    # ring slots and sink rows that hold no window position filled with NaN bit patterns:
    # they must not reach the result
    (2, 16, 48, 64, [40, 250, 129], "nan"),
    (3, 16, 64, 64, [400, 150], "nan"),   # 4-bit keys, 2-bit values
    # identity transforms with no T_v for the window (the window's values are used as given)
    (2, 4, 32, 64, [300, 97], "ident"),
])
def test_window_decode_matches_oracle(ci, S_sink, S_keep, S_flush, seql, variant):
    cfg = synth.CONFIGS[ci]
    B, T = len(seql), _round64(max(seql))
    c = cfg.with_(B=B, T_cap=T)
    k, v = synth.kv_batch(c, 0, T)                       # [B][T][Hkv][d] float32
    kb, vb = synth.as_dtype(k, "bf16"), synth.as_dtype(v, "bf16")
    Tk, Tv, Tit = synth.transforms(cfg)
    if variant == "ident":
        Tk = np.broadcast_to(np.eye(cfg.d, dtype=Tk.dtype), Tk.shape).copy()
        Tv, Tit = Tk.copy(), Tk.copy()
    q = synth.as_dtype(synth.queries(c), "bf16")
    # oracle: every position quantized at its own position; the window decode reads the
    # middle from there and the rest in full precision
    ofull = oracle.Cache(B, cfg.Hkv, T, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    oracle.quantize_append(kb, vb, Tk, Tv, cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha,
                           ofull, np.zeros(B, np.int32))
    want = oracle.window_decode(q, Tit, Tv, kb, vb, ofull, np.array(seql, np.int32), S_sink,
                                S_keep, S_flush)
    # GPU: the quantized middle of each sequence from cache position 0 (the oracle's codes
    # for the same tokens), sink and recent ring in bfloat16
    Qs = [oracle.window_quantized(L, S_sink, S_keep, S_flush) for L in seql]
    Tc = _round64(max(Qs))
    oc = oracle.Cache(B, cfg.Hkv, Tc, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    for b, Qb in enumerate(Qs):
        if Qb == 0:
            continue
        one = oracle.Cache(1, cfg.Hkv, Tc, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
        oracle.quantize_append(np.ascontiguousarray(kb[b:b + 1, S_sink:S_sink + Qb]),
                               np.ascontiguousarray(vb[b:b + 1, S_sink:S_sink + Qb]), Tk, Tv,
                               cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha, one, [0])
        for dst, src in zip(oc.planes(), one.planes()):
            n = src.size
            dst[b * n:(b + 1) * n] = src
    gc = upload_cache(oc, cfg)
    R = S_keep + S_flush
    fill = 0x7FC1 if variant == "nan" else 0             # a bfloat16 NaN
    ks = np.full((B, cfg.Hkv, max(S_sink, 1), cfg.d), fill, np.uint16)
    vs = np.full_like(ks, fill)
    kr = np.full((B, cfg.Hkv, R, cfg.d), fill, np.uint16)
    vr = np.full_like(kr, fill)
    for b, L in enumerate(seql):
        for t in range(min(S_sink, L)):
            ks[b, :, t], vs[b, :, t] = kb[b, t], vb[b, t]
        for t in range(S_sink + Qs[b], L):
            kr[b, :, t % R], vr[b, :, t % R] = kb[b, t], vb[b, t]
    out = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.float32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(kvq.decode_workspace_bytes(gc, cfg.Hq, Tc), dtype=torch.uint8, device=DEV)
    kvq.decode_attention_window(t_(q), t_(Tit), gc, S_sink, S_keep, S_flush,
                                t_(ks) if S_sink else None, t_(vs) if S_sink else None,
                                t_(kr), t_(vr), None if variant == "ident" else t_(Tv),
                                t_(np.array(seql, np.int32)), max(seql), out, ws, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    for b, L in enumerate(seql):
        if L == 0:
            assert not got[b].any()
    assert_close(got, want, where=f"window {S_sink}/{S_keep}/{S_flush}")
