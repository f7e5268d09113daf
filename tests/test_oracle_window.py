"""Pins of the oracle's full-precision window ("WUSH-KV: KV Cache Quantization with
Data-Adaptive Transforms", section 4.4): the quantized-middle length by hand-worked
cases, and the windowed decode against independently pinned functions -- the plain
quantized decode (everything quantized), the bfloat16 attention (nothing quantized),
and lossless quantization (inputs on the quantizer's grid: every window gives the
full-precision result)."""
import numpy as np
import pytest

import oracle
from tests import synth


@pytest.mark.parametrize("L,S_sink,S_keep,S_flush,Q", [
    # S_sink = 4, S_keep = 8, S_flush = 16: L - 12 eligible, floored to whole batches
    (0, 4, 8, 16, 0), (5, 4, 8, 16, 0), (12, 4, 8, 16, 0), (27, 4, 8, 16, 0),
    (28, 4, 8, 16, 16), (43, 4, 8, 16, 16), (44, 4, 8, 16, 32), (45, 4, 8, 16, 32),
    (60, 4, 8, 16, 48),
    # no window: every complete batch is quantized
    (64, 0, 0, 64, 64), (100, 0, 0, 64, 64), (100, 0, 0, 1, 100),
    # sink only / keep only
    (10, 10, 0, 2, 0), (11, 10, 0, 2, 0), (12, 10, 0, 2, 2), (9, 0, 9, 3, 0), (12, 0, 9, 3, 3),
])
def test_window_quantized_length(L, S_sink, S_keep, S_flush, Q):
    assert oracle.window_quantized(L, S_sink, S_keep, S_flush) == Q


def test_window_quantized_rejects_bad_arguments():
    for args in [(-1, 0, 0, 1), (5, -1, 0, 1), (5, 0, -1, 1), (5, 0, 0, 0)]:
        with pytest.raises(ValueError):
            oracle.window_quantized(*args)


def _setup(seed, B=2, Hkv=2, G=2, d=64, T=96, grid=False):
    rng = np.random.default_rng(seed)
    Hq = G * Hkv
    if grid:
        # values on the quantizer's grid z + c s with z = -0.5, s = 0.25, codes 0..3, each
        # group (= one token-head, g = d) holding at least one 0 and one 3: with clip index
        # 0 the quantizer finds lo = z, hi = z + 3 s and reproduces every value exactly
        c = rng.integers(0, 4, size=(B, T, Hkv, d))
        c[..., 0], c[..., 1] = 0, 3
        k = (-0.5 + 0.25 * c).astype(np.float32)
        c = rng.integers(0, 4, size=(B, T, Hkv, d))
        c[..., 0], c[..., 1] = 0, 3
        v = (-0.5 + 0.25 * c).astype(np.float32)
    else:
        k = rng.standard_normal((B, T, Hkv, d)).astype(np.float32)
        v = rng.standard_normal((B, T, Hkv, d)).astype(np.float32)
    q = rng.standard_normal((B, Hq, d)).astype(np.float32)
    kb, vb, qb = synth.f32_to_bf16_bits(k), synth.f32_to_bf16_bits(v), synth.f32_to_bf16_bits(q)
    return kb, vb, qb, Hkv


def _quantize_all(kb, vb, Hkv, T_k=None, T_v=None, alpha=0.0):
    B, T, _, d = kb.shape
    oc = oracle.Cache(B, Hkv, T, d, 2, 2, d)
    oracle.quantize_append(kb, vb, T_k, T_v, 2, 2, d, alpha, oc, np.zeros(B, np.int32))
    return oc


def _bf16_attention(qb, kb, vb, seql, Hkv):
    K = np.ascontiguousarray(kb.transpose(0, 2, 1, 3))      # [B][Hkv][T][d]
    V = np.ascontiguousarray(vb.transpose(0, 2, 1, 3))
    return oracle.bf16_decode(qb, K, V, seql, Hkv)


def test_everything_quantized_equals_quantized_decode():
    kb, vb, qb, Hkv = _setup(1)
    cfg = synth.CONFIGS[4].with_(Hkv=Hkv, Hq=4, d=64)
    Tk, Tv, Tit = synth.transforms(cfg)
    oc = _quantize_all(kb, vb, Hkv, Tk, Tv, 0.01)
    seql = np.array([96, 64], np.int32)                    # multiples of S_flush
    got = oracle.window_decode(qb, Tit, Tv, kb, vb, oc, seql, 0, 0, 32)
    want = oracle.decode(qb, Tit, oc, seql)
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_nothing_quantized_equals_value_transformed_bf16_attention():
    kb, vb, qb, Hkv = _setup(2)
    cfg = synth.CONFIGS[4].with_(Hkv=Hkv, Hq=4, d=64)
    Tk, Tv, Tit = synth.transforms(cfg)
    oc = _quantize_all(kb, vb, Hkv, Tk, Tv, 0.01)
    seql = np.array([40, 17], np.int32)
    for S_sink, S_keep in [(40, 0), (0, 40), (8, 32), (100, 100)]:
        got = oracle.window_decode(qb, Tit, Tv, kb, vb, oc, seql, S_sink, S_keep, 16)
        plain = _bf16_attention(qb, kb, vb, seql, Hkv)         # untransformed values
        G = qb.shape[1] // Hkv
        want = np.einsum("hij,bhgj->bhgi", Tv.astype(np.float64),
                         plain.reshape(2, Hkv, G, 64)).reshape(plain.shape)
        assert np.allclose(got, want, rtol=0, atol=1e-12), (S_sink, S_keep)


@pytest.mark.parametrize("S_sink,S_keep,S_flush", [(0, 0, 1), (4, 8, 16), (16, 0, 32), (0, 24, 8)])
def test_lossless_quantization_makes_the_window_invisible(S_sink, S_keep, S_flush):
    kb, vb, qb, Hkv = _setup(3, grid=True)
    oc = _quantize_all(kb, vb, Hkv)                        # identity transforms, clip index 0
    seql = np.array([96, 53], np.int32)
    got = oracle.window_decode(qb, None, None, kb, vb, oc, seql, S_sink, S_keep, S_flush)
    want = _bf16_attention(qb, kb, vb, seql, Hkv)
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_window_changes_the_result_between_the_extremes():
    kb, vb, qb, Hkv = _setup(4)
    oc = _quantize_all(kb, vb, Hkv, alpha=0.01)
    seql = np.array([96, 96], np.int32)
    full = oracle.window_decode(qb, None, None, kb, vb, oc, seql, 0, 96, 16)
    quant = oracle.window_decode(qb, None, None, kb, vb, oc, seql, 0, 0, 16)
    mixed = oracle.window_decode(qb, None, None, kb, vb, oc, seql, 8, 24, 16)
    ef, eq = np.linalg.norm(mixed - full), np.linalg.norm(mixed - quant)
    assert ef > 0 and eq > 0
    assert np.linalg.norm(quant - full) > max(ef, eq) * 0.5


# ---------------------------------------------------------------- mixed windows
#
# A sequence with a sink, a quantized middle and a non-empty recent part is checked
# against three pieces computed independently of oracle.window_decode: the quantized
# middle through oracle.decode_partial (pinned in test_oracle.py against brute-force
# attention), and the sink and the recent positions by a plain numpy softmax in float64
# with the query as given and T_v applied to the values. oracle.merge (pinned by split
# invariance) joins them.

def _numpy_partial(q_f64, K_f64, V_f64, Tv_h):
    """(m, l, o) of one query over full-precision rows K, V [n][d] (T_v applied)."""
    if K_f64.shape[0] == 0:
        return -np.inf, 0.0, np.zeros(q_f64.shape[0])
    d = q_f64.shape[0]
    logits = (K_f64 @ q_f64) / np.sqrt(d)
    m = logits.max()
    p = np.exp(logits - m)
    o = p @ V_f64
    if Tv_h is not None:
        o = Tv_h.astype(np.float64) @ o
    return m, p.sum(), o


def _bf16_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("seed,S_sink,S_keep,S_flush,lens", [
    (11, 4, 8, 16, (96, 53)),      # Q = 80 and 32; recent 12 and 17 positions
    (12, 16, 0, 32, (96, 81)),     # Q = 64 and 64; recent 16 and 1
    (13, 1, 24, 8, (96, 40)),      # Q = 64 and 8; recent 31 and 31
    (14, 7, 5, 3, (95, 17)),       # odd sizes: Q = 81 and 3
])
def test_mixed_window_equals_merge_of_independent_pieces(seed, S_sink, S_keep, S_flush, lens):
    kb, vb, qb, Hkv = _setup(seed)
    cfg = synth.CONFIGS[4].with_(Hkv=Hkv, Hq=4, d=64)
    Tk, Tv, Tit = synth.transforms(cfg)
    oc = _quantize_all(kb, vb, Hkv, Tk, Tv, 0.01)
    seql = np.array(lens, np.int32)
    got = oracle.window_decode(qb, Tit, Tv, kb, vb, oc, seql, S_sink, S_keep, S_flush)
    B, Hq, d = qb.shape
    G = Hq // Hkv
    checked = 0
    for b in range(B):
        L = int(seql[b])
        Q = oracle.window_quantized(L, S_sink, S_keep, S_flush)
        assert 0 < Q and S_sink + Q < L            # all three pieces are present
        for hq in range(Hq):
            h = hq // G
            qv = _bf16_f64(qb[b, hq])
            sink = _numpy_partial(qv, _bf16_f64(kb[b, :S_sink, h]), _bf16_f64(vb[b, :S_sink, h]),
                                  Tv[h])
            mid = oracle.decode_partial(qb, Tit, oc, b, hq, S_sink, S_sink + Q)
            rec = _numpy_partial(qv, _bf16_f64(kb[b, S_sink + Q:L, h]),
                                 _bf16_f64(vb[b, S_sink + Q:L, h]), Tv[h])
            want = oracle.merge([sink[0], mid[0], rec[0]], [sink[1], mid[1], rec[1]],
                                np.stack([sink[2], mid[2], rec[2]]))
            assert np.allclose(got[b, hq], want, rtol=1e-12, atol=1e-12), (b, hq)
            checked += 1
    assert checked == B * Hq


def _marker_setup(d=64, L=12, T=16):
    """One sequence, one KV head, two query heads. Cache token t dequantizes to 100 e_t
    for its value (code 1 at dim t, s = 100, z = 0) and to 0 for its key (s = z = 0);
    the full-precision value of position t is e_t."""
    kc = np.zeros((T, d), np.uint8)
    vc = np.zeros((T, d), np.uint8)
    for t in range(T):
        vc[t, t] = 1
    f16 = lambda x: np.float16(x).view(np.uint16)
    ksz = np.zeros((T, 1, 2), np.uint16)
    vsz = np.zeros((T, 1, 2), np.uint16)
    vsz[:, 0, 0] = f16(100.0)
    oc = oracle.Cache(1, 1, T, d, 2, 2, d)
    oc.pack_tokens(0, 0, 0, kc, vc, ksz, vsz)
    v = np.zeros((1, T, 1, d), np.float32)
    for t in range(T):
        v[0, t, 0, t] = 1.0
    return oc, v


def test_hand_sized_window_value_positions():
    """S_sink = 2, S_keep = 3, S_flush = 2, L = 12: 7 positions are eligible, so the
    quantized middle is the 6 positions {2, 3, 4, 5, 6, 7}; the full-precision positions
    are {0, 1} and {8, 9, 10, 11}. With q = 0 every position has weight 1/12, so
    12 * out[j] is 100 at a quantized position j and 1 at a full-precision one."""
    d, L = 64, 12
    oc, v = _marker_setup(d, L)
    k = np.zeros_like(v)
    q = np.zeros((1, 2, d), np.float32)
    got = oracle.window_decode(q, None, None, k, v, oc, np.array([L], np.int32), 2, 3, 2)
    quantized = [2, 3, 4, 5, 6, 7]
    full_precision = [0, 1, 8, 9, 10, 11]
    want = np.zeros(d)
    want[quantized] = 100.0
    want[full_precision] = 1.0
    for hq in range(2):
        assert np.allclose(L * got[0, hq], want, rtol=0, atol=1e-12)


def test_hand_sized_window_key_positions():
    """Same window. Full-precision keys are 1 in dim 0 and the query is 8 * 40 in dim 0
    (logit 40 after 1/sqrt(64)); quantized keys dequantize to 0 (logit 0). The softmax
    then sits on the six full-precision positions {0, 1, 8, 9, 10, 11} (each weight 1/6,
    the quantized ones e^-40 smaller), and the output is e_t / 6 over those positions."""
    d, L = 64, 12
    oc, v = _marker_setup(d, L)
    k = np.zeros_like(v)
    k[0, :, 0, 0] = 1.0
    q = np.zeros((1, 2, d), np.float32)
    q[0, :, 0] = 8.0 * 40.0
    got = oracle.window_decode(q, None, None, k, v, oc, np.array([L], np.int32), 2, 3, 2)
    want = np.zeros(d)
    want[[0, 1, 8, 9, 10, 11]] = 1.0 / 6.0
    for hq in range(2):
        assert np.allclose(got[0, hq], want, rtol=0, atol=1e-12)
