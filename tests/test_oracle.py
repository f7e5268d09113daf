"""Pins for the float64 CPU oracle: each check ties it to something other than itself.

* hand-worked quantizer examples and hand-derived layout positions (tests/golden/);
* the numbers the pages print for bits per element (tests/golden/);
* float16 rounding against numpy's independent implementation;
* T = I reduces to textbook clipped affine quantization (numpy order statistics,
  nearest reconstruction level in float64);
* the reconstruction error bound of an affine quantizer;
* exact preservation of q.k under (T^{-T} q).(T k) with quantization off
  (WUSH-KV summary, section 1 / section 4.2: query-side compensation);
* brute force attention on tiny inputs, its special cases, and split invariance;
* an exhaustive pack/unpack round trip and an independent little-endian bit stream.
"""
import itertools
import os

import numpy as np
import pytest

import oracle
from tests import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


# ----------------------------------------------------------------- golden fixtures

def test_quantizer_hand_worked_examples():
    n = 0
    for bits, kap, xs, sh, zh, codes, packed in _rows("quantizer_hand_worked.txt"):
        x = np.array([float(v) for v in xs.split()], np.float32)
        c, s, z = oracle.quantize_group(x, int(bits), int(kap))
        assert s == int(sh, 16), (xs, hex(s))
        assert z == int(zh, 16), (xs, hex(z))
        assert c.tolist() == [int(v) for v in codes.split()]
        row = oracle.pack_k_row(c, int(bits))
        assert row.tolist() == [int(v, 16) for v in packed.split()]
        n += 1
    assert n == 5


def test_v_tile_hand_derived_positions():
    n = 0
    for d, bits, tok, dim, byte, bit in _rows("v_tile_positions.txt"):
        assert oracle.v_code_pos(int(d), int(bits), int(tok), int(dim)) == (int(byte), int(bit))
        n += 1
    assert n == 14


def test_bits_per_element_matches_pages():
    """2-bit codes + float16 (s, z) per 128 dims = 2.25 bits/element, the QuaRot figure
    on the NOVA-KV page; the nominal reduction vs 16-bit is 8x (WUSH-KV section 5.3)."""
    table = {name: float(v) for name, v in _rows("storage_bits_per_element.txt")}
    for bits, want in ((2, table["QuaRot"]), (4, 4.25)):
        c = oracle.Cache(1, 1, 16, 128, bits, bits, 128)
        per_tok_head = (c.k_codes.nbytes + c.k_sz.nbytes) / 16
        assert per_tok_head * 8 / 128 == want
    assert table["BF16 (uncompressed)"] / 2 == table["nominal reduction 16->2 bit"]
    # 16-bit cache vs this layout: about 7.1x, below the nominal 8x because of metadata
    assert abs(16 / 2.25 - 7.111) < 1e-3


def test_kappa_examples():
    assert oracle.kappa(0.01, 128) == 1       # floor(0.01*127) = 1
    assert oracle.kappa(0.005, 128) == 0      # floor(0.635) = 0
    assert oracle.kappa(0.01, 64) == 0        # floor(0.63) = 0
    assert oracle.kappa(0.0, 128) == 0
    assert oracle.kappa(0.1, 128) == 12


# ----------------------------------------------------------------- float16

def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(5)
    u = rng.integers(0, 2 ** 32, size=40000, dtype=np.uint64).astype(np.uint32)
    x = u.view(np.float32)
    x = x[np.isfinite(x)]
    special = np.array([0.0, -0.0, 1.0, 65504.0, 65519.99, 65520.0, 1e30, 2 ** -24, 2 ** -25,
                        3 * 2 ** -26, 2 ** -25 * 1.0000001, 2 ** -14, 2 ** -14 * (1 - 2 ** -11),
                        1 + 2 ** -11, 1 + 3 * 2 ** -11, 0.1, -0.2, 1 / 3, 5.960464477539063e-08,
                        6.097555160522461e-05], np.float32)
    small = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 12, 20000))).astype(np.float32)
    x = np.concatenate([x, special, -special, small])
    got = oracle.f32_to_f16_bits(x)
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(got[~nan], want[~nan])
    back = oracle.f16_bits_to_f64(got[~nan])
    assert np.array_equal(back, want[~nan].view(np.float16).astype(np.float64))


# ----------------------------------------------------------------- quantizer pins

def _textbook(x, bits, alpha):
    """Clipped affine quantizer written the textbook way: numpy order statistics and the
    nearest reconstruction level z + c*s (float64), no division."""
    lo = np.float32(np.quantile(x.astype(np.float64), alpha, method="lower"))
    hi = np.float32(np.quantile(x.astype(np.float64), 1 - alpha, method="higher"))
    qmax = (1 << bits) - 1
    s = np.float32(np.float32(hi - lo) / np.float32(qmax)).astype(np.float16)
    z = np.float16(lo)
    levels = float(z) + np.arange(qmax + 1) * float(s)
    c = np.argmin(np.abs(x.astype(np.float64)[:, None] - levels[None, :]), axis=1)
    return c, s, z


@pytest.mark.parametrize("bits,g,alpha", [(2, 128, 0.01), (4, 128, 0.005), (2, 64, 0.01),
                                          (4, 32, 0.1), (2, 8, 0.15)])
def test_identity_transform_is_textbook_clipped_affine(bits, g, alpha):
    rng = np.random.default_rng(bits * 1000 + g)
    kap = oracle.kappa(alpha, g)
    checked = 0
    for trial in range(300):
        x = (rng.standard_normal(g) * rng.lognormal(0, 1)).astype(np.float32)
        if trial % 7 == 0:
            x[rng.integers(g)] *= 50
        c, sh, zh = oracle.quantize_group(x, bits, kap)
        ct, st, zt = _textbook(x, bits, alpha)
        assert sh == st.view(np.uint16) and zh == zt.view(np.uint16)
        # near-ties in the reconstruction domain may legitimately round either way
        s, z = float(st), float(zt)
        y = (x.astype(np.float64) - z) / s
        fr = np.abs(y - np.floor(y) - 0.5)
        ok = fr > 1e-4
        assert np.array_equal(c[ok], ct[ok])
        checked += ok.sum()
    assert checked > 300 * g * 0.99


@pytest.mark.parametrize("bits", [2, 4])
def test_reconstruction_error_bound(bits):
    rng = np.random.default_rng(77 + bits)
    qmax = (1 << bits) - 1
    for _ in range(400):
        g = 64
        x = (rng.standard_normal(g) * 3 + rng.uniform(-5, 5)).astype(np.float32)
        c, sh, zh = oracle.quantize_group(x, bits, oracle.kappa(0.03, g))
        s = float(np.uint16(sh).view(np.float16))
        z = float(np.uint16(zh).view(np.float16))
        xh = z + c.astype(np.float64) * s
        inside = (x >= z) & (x <= z + qmax * s)
        err = np.abs(x.astype(np.float64) - xh)
        assert np.all(err[inside] <= s / 2 * (1 + 2 ** -20))
        assert np.all(np.isin(c[~inside], [0, qmax]))
        assert np.all((c[x < z] == 0)) and np.all(c[x > z + qmax * s] == qmax)


def test_codes_are_nearest_level_brute_force_tiny():
    """Brute force on tiny groups: every code is the level c minimising
    |f32(f32(x - z)/s) - c| over all 2^b levels, ties to the even level."""
    rng = np.random.default_rng(3)
    for bits in (2, 4):
        qmax = (1 << bits) - 1
        for g in (4, 8):
            for _ in range(500):
                x = np.round(rng.standard_normal(g) * 4, rng.integers(0, 3)).astype(np.float32)
                c, sh, zh = oracle.quantize_group(x, bits, 0)
                s = np.uint16(sh).view(np.float16).astype(np.float32)
                z = np.uint16(zh).view(np.float16).astype(np.float32)
                if s == 0:
                    assert not c.any()
                    continue
                y = (x - z) / s            # numpy float32 IEEE ops
                for i in range(g):
                    dist = [abs(float(y[i]) - L) for L in range(qmax + 1)]
                    best = min(dist)
                    cands = [L for L in range(qmax + 1) if dist[L] == best]
                    want = cands[0] if len(cands) == 1 else [L for L in cands if L % 2 == 0][0]
                    if y[i] > qmax:
                        want = qmax
                    assert c[i] == want, (x, y, c)


# ----------------------------------------------------------------- transform pins

def test_query_compensation_preserves_qk():
    cfg = synth.CONFIGS[0]
    T, Tit = synth.transforms_f64(cfg)
    rng = np.random.default_rng(11)
    cond = 10.0
    for _ in range(50):
        q = rng.standard_normal(cfg.d)
        k = rng.standard_normal(cfg.d) * 5
        qt = oracle.matvec(Tit[0], q)
        kt = oracle.matvec(T[0], k)
        assert abs(qt @ kt - q @ k) <= 1e-12 * np.linalg.norm(q) * np.linalg.norm(k) * cond * 10
    # the closed form really is the inverse transpose
    assert np.abs(T[0].T @ Tit[0] - np.eye(cfg.d)).max() < 1e-12
    s = np.linalg.svd(T[0], compute_uv=False)
    assert s.max() / s.min() <= 10.0 + 1e-9


def test_append_applies_transform_then_rounds_to_f32():
    cfg = synth.CONFIGS[0].with_(T_cap=32, seq_lo=32, seq_hi=32)
    Tk, Tv, _ = synth.transforms(cfg)
    k, v = synth.kv_batch(cfg, 0, 16)
    cache = oracle.Cache.for_config(cfg)
    kt, vt = oracle.quantize_append(k, v, Tk, Tv, 2, 2, 128, 0.01, cache, [0],
                                    return_transformed=True)
    want_k = np.einsum("hij,bnhj->bnhi", Tk.astype(np.float64), k.astype(np.float64))
    want_v = np.einsum("hij,bnhj->bnhi", Tv.astype(np.float64), v.astype(np.float64))
    assert np.array_equal(kt, want_k.astype(np.float32)) or \
        np.abs(kt - want_k).max() <= 2 ** -22 * np.abs(want_k).max()
    assert np.abs(vt - want_v).max() <= 2 ** -22 * np.abs(want_v).max()


def test_append_identity_matches_groupwise_quantizer_and_layout():
    cfg = synth.CONFIGS[0].with_(T_cap=64, group=64)
    rng = np.random.default_rng(2)
    k = rng.standard_normal((1, 20, 1, 128)).astype(np.float32)
    v = rng.standard_normal((1, 20, 1, 128)).astype(np.float32)
    cache = oracle.Cache(1, 1, 64, 128, 4, 2, 64)
    oracle.quantize_append(k, v, None, None, 4, 2, 64, 0.05, cache, [7])
    kc, vc, ksz, vsz = cache.unpack_tokens(0, 0, 7, 20)
    kap = oracle.kappa(0.05, 64)
    for i in range(20):
        for gr in range(2):
            c, s, z = oracle.quantize_group(k[0, i, 0, gr * 64:(gr + 1) * 64], 4, kap)
            assert np.array_equal(kc[i, gr * 64:(gr + 1) * 64], c)
            assert (ksz[i, gr, 0], ksz[i, gr, 1]) == (s, z)
            c, s, z = oracle.quantize_group(v[0, i, 0, gr * 64:(gr + 1) * 64], 2, kap)
            assert np.array_equal(vc[i, gr * 64:(gr + 1) * 64], c)
    # positions outside [7, 27) untouched
    kc0, vc0, ksz0, _ = cache.unpack_tokens(0, 0, 0, 7)
    assert not kc0.any() and not vc0.any() and not ksz0.any()


def test_append_bf16_inputs_read_exactly():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 3, 2, 64)).astype(np.float32)
    xb = synth.f32_to_bf16_bits(x)
    xf = synth.bf16_bits_to_f32(xb)
    c1 = oracle.Cache(2, 2, 16, 64, 2, 2, 64)
    c2 = oracle.Cache(2, 2, 16, 64, 2, 2, 64)
    oracle.quantize_append(xb, xb, None, None, 2, 2, 64, 0.01, c1, [0, 5])
    oracle.quantize_append(xf, xf, None, None, 2, 2, 64, 0.01, c2, [0, 5])
    for a, b in zip(c1.planes(), c2.planes()):
        assert np.array_equal(a, b)


# ----------------------------------------------------------------- layout pins

def test_k_row_is_little_endian_bitstream_exhaustive():
    for bits, d in ((2, 8), (4, 4)):
        for codes in itertools.product(range(1 << bits), repeat=d):
            codes = np.array(codes, np.uint8)
            row = oracle.pack_k_row(np.concatenate([codes, np.zeros(64 - d, np.uint8)]), bits)
            # independent: expand each code to its bits (LSB first) and pack LSB-first
            bitsarr = ((codes[:, None] >> np.arange(bits)) & 1).astype(np.uint8).ravel()
            want = np.packbits(bitsarr, bitorder="little")
            assert np.array_equal(row[:len(want)], want)
            back = oracle.unpack_k_row(row, 64, bits)[:d]
            assert np.array_equal(back, codes)
    assert oracle.pack_k_row(np.array([0, 1, 2, 3] + [0] * 60, np.uint8), 2)[0] == 0xE4
    assert oracle.pack_k_row(np.array([1, 2] + [0] * 62, np.uint8), 4)[0] == 0x21


@pytest.mark.parametrize("d,bits", [(128, 2), (64, 2), (128, 4), (64, 4)])
def test_v_tile_layout_is_a_bijection_and_round_trips(d, bits):
    seen = set()
    for tok in range(16):
        for j in range(d):
            by, bi = oracle.v_code_pos(d, bits, tok, j)
            assert 0 <= by < oracle.v_tile_bytes(d, bits) and bi % bits == 0 and bi + bits <= 8
            for k in range(bits):
                seen.add(by * 8 + bi + k)
    assert len(seen) == oracle.v_tile_bytes(d, bits) * 8
    rng = np.random.default_rng(d + bits)
    for _ in range(20):
        codes = rng.integers(0, 1 << bits, size=(16, d), dtype=np.uint8)
        tile = oracle.pack_v_tile(codes, bits)
        assert np.array_equal(oracle.unpack_v_tile(tile, d, bits), codes)


# ----------------------------------------------------------------- attention pins

def _fields_cache(cfg, n_tok, seed):
    """Cache holding random fields; returns (cache, khat, vhat) with khat/vhat float64
    [B][Hkv][n][d] computed directly from the drawn fields (not from the planes)."""
    rng = np.random.default_rng(seed)
    c = oracle.Cache.for_config(cfg)
    ng = cfg.d // cfg.group
    kh = np.zeros((cfg.B, cfg.Hkv, n_tok, cfg.d))
    vh = np.zeros((cfg.B, cfg.Hkv, n_tok, cfg.d))
    for b in range(cfg.B):
        for h in range(cfg.Hkv):
            kc = rng.integers(0, 1 << cfg.bits_k, (n_tok, cfg.d), dtype=np.uint8)
            vc = rng.integers(0, 1 << cfg.bits_v, (n_tok, cfg.d), dtype=np.uint8)
            ks = rng.uniform(0.1, 1.5, (n_tok, ng)).astype(np.float16)
            kz = rng.uniform(-3, 0, (n_tok, ng)).astype(np.float16)
            vs = rng.uniform(0.1, 1.5, (n_tok, ng)).astype(np.float16)
            vz = rng.uniform(-3, 0, (n_tok, ng)).astype(np.float16)
            ksz = np.stack([ks.view(np.uint16), kz.view(np.uint16)], -1)
            vsz = np.stack([vs.view(np.uint16), vz.view(np.uint16)], -1)
            c.pack_tokens(b, h, 0, kc, vc, ksz, vsz)
            rep = lambda a: np.repeat(a.astype(np.float64), cfg.group, axis=1)
            kh[b, h] = rep(kz) + kc * rep(ks)
            vh[b, h] = rep(vz) + vc * rep(vs)
    return c, kh, vh


def _two_pass(q, M, kh, vh, n, d):
    qt = q if M is None else M @ q
    logits = (kh[:n] @ qt) / np.sqrt(d)
    p = np.exp(logits - logits.max())
    return (p[:, None] * vh[:n]).sum(0) / p.sum()


@pytest.mark.parametrize("bits_k,bits_v,group", [(2, 2, 64), (4, 2, 64), (2, 4, 32)])
def test_decode_brute_force_tiny(bits_k, bits_v, group):
    cfg = synth.Config(99, "tiny", B=2, Hq=4, Hkv=2, d=64, T_cap=16, bits_k=bits_k,
                       bits_v=bits_v, group=group, clip_alpha=0.0, in_dtype="f32",
                       q_dtype="f32", out_dtype="f32", seq_lo=1, seq_hi=8)
    c, kh, vh = _fields_cache(cfg, 8, seed=bits_k * 10 + bits_v)
    rng = np.random.default_rng(0)
    q = rng.standard_normal((2, 4, 64)).astype(np.float32)
    M = (np.eye(64) + 0.1 * rng.standard_normal((2, 64, 64))).astype(np.float32)
    seql = np.array([8, 5], np.int32)
    out = oracle.decode(q, M, c, seql)
    for b in range(2):
        for hq in range(4):
            h = hq // 2                                 # contiguous GQA grouping
            want = _two_pass(q[b, hq].astype(np.float64), M[h].astype(np.float64), kh[b, h],
                             vh[b, h], seql[b], 64)
            np.testing.assert_allclose(out[b, hq], want, rtol=1e-12, atol=1e-12)


def test_decode_special_cases():
    cfg = synth.Config(98, "tiny", B=1, Hq=2, Hkv=1, d=64, T_cap=32, bits_k=2, bits_v=2,
                       group=64, clip_alpha=0.0, in_dtype="f32", q_dtype="f32",
                       out_dtype="f32", seq_lo=1, seq_hi=32)
    c, kh, vh = _fields_cache(cfg, 32, seed=9)
    q = np.zeros((1, 2, 64), np.float32)
    # q = 0: uniform attention, the mean of the dequantized values
    out = oracle.decode(q, None, c, np.array([20], np.int32))
    np.testing.assert_allclose(out[0, 0], vh[0, 0, :20].mean(0), rtol=1e-12, atol=1e-13)
    # one token: exactly that token's value
    q1 = np.random.default_rng(1).standard_normal((1, 2, 64)).astype(np.float32)
    out = oracle.decode(q1, None, c, np.array([1], np.int32))
    np.testing.assert_allclose(out[0, 1], vh[0, 0, 0], rtol=1e-14)
    # empty sequence: zeros
    out = oracle.decode(q1, None, c, np.array([0], np.int32))
    assert not out.any()
    # one dominant logit: the output is (almost) that token's value
    qd = (kh[0, 0, 13] - kh[0, 0].mean(0)).astype(np.float32)[None, None, :] * 40
    qd = np.concatenate([qd, qd], 1)
    logits = kh[0, 0] @ qd[0, 0].astype(np.float64) / 8.0
    top = np.argsort(logits)[::-1]
    assert logits[top[0]] - logits[top[1]] > 30          # one logit dominates
    out = oracle.decode(qd, None, c, np.array([32], np.int32))
    np.testing.assert_allclose(out[0, 0], vh[0, 0, top[0]], atol=1e-9)


def test_split_merge_invariance():
    cfg = synth.CONFIGS[0].with_(T_cap=256, d=128)
    c, _, _ = _fields_cache(cfg, 256, seed=21)
    q = np.random.default_rng(8).standard_normal((1, 4, 128)).astype(np.float32) * 3
    _, _, M = synth.transforms(cfg)
    full = oracle.decode(q, M, c, np.array([250], np.int32))
    rng = np.random.default_rng(12)
    for hq in range(4):
        for _ in range(5):
            cuts = np.sort(rng.choice(np.arange(1, 250), size=rng.integers(1, 9), replace=False))
            edges = [0, *cuts.tolist(), 250]
            parts = [oracle.decode_partial(q, M, c, 0, hq, a, b) for a, b in zip(edges, edges[1:])]
            parts.append(oracle.decode_partial(q, M, c, 0, hq, 250, 250))   # empty split
            m = [p[0] for p in parts]
            l = [p[1] for p in parts]
            o = np.stack([p[2] for p in parts])
            merged = oracle.merge(m, l, o)
            np.testing.assert_allclose(merged, full[0, hq], rtol=1e-12, atol=1e-13)


def test_sampled_heads_equal_full_decode():
    cfg = synth.CONFIGS[0].with_(T_cap=64, B=2, Hq=4, Hkv=2)
    c, _, _ = _fields_cache(cfg, 64, seed=5)
    q = np.random.default_rng(2).standard_normal((2, 4, 128)).astype(np.float32)
    seql = np.array([64, 33], np.int32)
    full = oracle.decode(q, None, c, seql)
    sel = np.array([[1, 3], [0, 2], [1, 3], [1, 3], [0, 2]], np.int32)   # duplicates allowed
    part = oracle.decode(q, None, c, seql, sel=sel)
    for b, h in sel:
        assert np.array_equal(part[b, h], full[b, h])
    assert np.isnan(part[0, 0]).all()


def test_bf16_comparator_brute_force():
    rng = np.random.default_rng(6)
    B, Hq, Hkv, d, T = 2, 4, 2, 64, 16
    q = synth.f32_to_bf16_bits(rng.standard_normal((B, Hq, d)).astype(np.float32))
    K = synth.f32_to_bf16_bits(rng.standard_normal((B, Hkv, T, d)).astype(np.float32))
    V = synth.f32_to_bf16_bits(rng.standard_normal((B, Hkv, T, d)).astype(np.float32))
    seql = np.array([16, 3], np.int32)
    out = oracle.bf16_decode(q, K, V, seql, Hkv)
    f = lambda a: synth.bf16_bits_to_f32(a).astype(np.float64)
    for b in range(B):
        for hq in range(Hq):
            want = _two_pass(f(q[b, hq]), None, f(K[b, hq // 2]), f(V[b, hq // 2]), seql[b], d)
            np.testing.assert_allclose(out[b, hq], want, rtol=1e-12, atol=1e-13)


def test_end_to_end_chain_against_numpy_restatement():
    """Transform -> clipped affine quantize -> pack -> decode with T^{-T} q, checked
    against a numpy chain: textbook quantizer on the oracle's float32 transformed keys
    and values, then plain float64 attention with the compensated queries."""
    cfg = synth.CONFIGS[0].with_(T_cap=96)
    Tk, Tv, Tit = synth.transforms(cfg)
    k, v = synth.kv_batch(cfg, 0, 96)
    q = synth.queries(cfg)
    cache = oracle.Cache.for_config(cfg)
    kt, vt = oracle.quantize_append(k, v, Tk, Tv, 2, 2, 128, 0.01, cache, [0],
                                    return_transformed=True)
    np.testing.assert_allclose(kt[0, :, 0], k[0, :, 0].astype(np.float64) @ Tk[0].T.astype(np.float64),
                               rtol=0, atol=1e-5 * np.abs(kt).max())
    kc, vc, _, _ = cache.unpack_tokens(0, 0, 0, 96)

    def restate(x, codes_oracle):
        out = np.empty((x.shape[0], x.shape[1]))
        for t in range(x.shape[0]):
            c, s, z = _textbook(x[t], 2, 0.01)
            y = (x[t].astype(np.float64) - float(z)) / float(s)
            near = np.abs(y - np.floor(y) - 0.5) <= 1e-4
            c = np.where(near, codes_oracle[t], c)
            out[t] = float(z) + c * float(s)
        return out

    kh = restate(kt[0, :, 0], kc)
    vh = restate(vt[0, :, 0], vc)
    out = oracle.decode(q, Tit, cache, np.array([90], np.int32))
    for hq in range(4):
        want = _two_pass(q[0, hq].astype(np.float64), Tit[0].astype(np.float64), kh, vh, 90, 128)
        np.testing.assert_allclose(out[0, hq], want, rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------- QuEST INT quantizer
# ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms", section 4.3)

def test_quest_hand_worked_examples():
    n = 0
    for bits, xs, sh, zh, codes, packed in _rows("quest_hand_worked.txt"):
        x = np.array([float(v) for v in xs.split()], np.float32)
        c, s, z = oracle.quantize_group_quest(x, int(bits))
        assert s == int(sh, 16), (xs, hex(s))
        assert z == int(zh, 16), (xs, hex(z))
        assert c.tolist() == [int(v) for v in codes.split()]
        assert oracle.pack_k_row(c, int(bits)).tolist() == [int(v, 16) for v in packed.split()]
        n += 1
    assert n == 4


@pytest.mark.parametrize("bits", [2, 4])
def test_quest_step_minimises_the_gaussian_mse(bits):
    """The step constant is the uniform step with the least mean squared error for a unit
    Gaussian, found here by numerical integration and minimisation (independent of the
    oracle and of any table): 2^b levels at (c - (2^b - 1)/2) step, cells split at the
    midpoints, the outer cells open."""
    from scipy import integrate, optimize, stats
    N = 1 << bits

    def mse(step):
        levels = (np.arange(N) - (N - 1) / 2) * step
        edges = np.concatenate([[-np.inf], (levels[:-1] + levels[1:]) / 2, [np.inf]])
        tot = 0.0
        for c in range(N):
            f = lambda x, y=levels[c]: (x - y) ** 2 * stats.norm.pdf(x)
            tot += integrate.quad(f, edges[c], edges[c + 1])[0]
        return tot
    best = optimize.minimize_scalar(mse, bounds=(0.05, 2.0), method="bounded",
                                    options={"xatol": 1e-7}).x
    assert abs(best - oracle.quest_delta(bits)) < 5e-4, best


@pytest.mark.parametrize("bits,mse_opt", [(2, 0.1188), (4, 0.01154)])
def test_quest_gaussian_mse_is_the_textbook_optimum(bits, mse_opt):
    """On unit-Gaussian groups of 128 the quantizer's mean squared error is close to the
    optimal uniform quantizer's (Max 1960: 0.1188 for 4 levels, 0.01154 for 16); the
    per-group RMS keeps it a few percent lower (a sample's largest values sit closer to
    its own RMS, fewer overload errors). A grid shifted by half a step, a missing clip or
    a wrong RMS moves it far outside 6%."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3000, 128)).astype(np.float32)
    err = 0.0
    for row in x:
        c, sh, zh = oracle.quantize_group_quest(row, bits)
        s, z = oracle.f16_bits_to_f64([sh, zh])
        err += np.sum((row.astype(np.float64) - (z + c * s)) ** 2)
    mse = err / x.size
    assert abs(mse - mse_opt) / mse_opt < 0.06, mse


@pytest.mark.parametrize("bits", [2, 4])
def test_quest_grid_and_error_bound(bits):
    """Levels sit symmetrically (up to the float16 zero-point) around 0 with step
    delta_b * rms; entries inside the grid are within s/2 of their reconstruction, entries
    outside clip to the outer level."""
    rng = np.random.default_rng(6 + bits)
    qmax = (1 << bits) - 1
    for _ in range(200):
        g = int(rng.choice([32, 64, 128]))
        x = (rng.standard_normal(g) * rng.lognormal(0, 2)).astype(np.float32)
        c, sh, zh = oracle.quantize_group_quest(x, bits)
        s, z = oracle.f16_bits_to_f64([sh, zh])
        rms = np.float32(np.sqrt(np.mean(x.astype(np.float64) ** 2)))
        s_ref = np.float32(rms * np.float32(oracle.quest_delta(bits)))
        assert abs(s - s_ref) <= s_ref * 2.0 ** -11                      # f16 rounding of s
        assert abs(z + qmax / 2 * s) <= abs(z) * 2.0 ** -11 + 1e-30     # z = -(2^b-1)/2 s
        xh = z + c * s
        inside = (x >= z) & (x <= z + qmax * s)
        assert np.all(np.abs(x[inside] - xh[inside]) <= s / 2 * (1 + 2.0 ** -20))
        assert np.all(c[x < z] == 0) and np.all(c[x > z + qmax * s] == qmax)


def test_quest_scale_invariance():
    """Scaling a group by a power of two scales s_h and z_h by it and keeps every code."""
    rng = np.random.default_rng(9)
    for bits in (2, 4):
        for _ in range(50):
            x = rng.standard_normal(64).astype(np.float32)
            c0, s0, z0 = oracle.quantize_group_quest(x, bits)
            c1, s1, z1 = oracle.quantize_group_quest(x * np.float32(8.0), bits)
            a0, b0 = oracle.f16_bits_to_f64([s0, z0])
            a1, b1 = oracle.f16_bits_to_f64([s1, z1])
            assert np.array_equal(c0, c1) and a1 == 8 * a0 and b1 == 8 * b0


def test_quest_append_uses_the_groupwise_quantizer():
    """quantize_append with quantizer 1 stores exactly the QuEST codes and (s, z) of each
    transformed token group."""
    rng = np.random.default_rng(10)
    k = rng.standard_normal((1, 5, 2, 128)).astype(np.float32)
    v = rng.standard_normal((1, 5, 2, 128)).astype(np.float32)
    oc = oracle.Cache(1, 2, 64, 128, 4, 2, 128)
    oracle.quantize_append(k, v, None, None, 4, 2, 128, 0.0, oc, [3], quantizer=1)
    for h in range(2):
        kc, vc, ksz, vsz = oc.unpack_tokens(0, h, 3, 5)
        for i in range(5):
            c, s, z = oracle.quantize_group_quest(k[0, i, h], 4)
            assert kc[i].tolist() == c.tolist() and ksz[i, 0].tolist() == [s, z]
            c, s, z = oracle.quantize_group_quest(v[0, i, h], 2)
            assert vc[i].tolist() == c.tolist() and vsz[i, 0].tolist() == [s, z]
