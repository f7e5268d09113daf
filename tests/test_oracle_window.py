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
