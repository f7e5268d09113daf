"""float64 CPU oracle for transformed-KV quantize-append and decode attention.

TEST INFRASTRUCTURE: only tests/, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg may import this package. The product (``decode_attention_post_b200``)
never imports it and shares no code with it. See ``kvq_oracle.c`` for the definitions
and the passages of the pages they follow.

Every function here is a thin numpy <-> C marshalling wrapper.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None

P = C.c_void_p
I = C.c_int
F = C.c_float


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        L.oracle_f32_to_f16.argtypes = [F]
        L.oracle_f32_to_f16.restype = C.c_uint16
        L.oracle_f16_to_f64.argtypes = [C.c_uint16]
        L.oracle_f16_to_f64.restype = C.c_double
        L.oracle_kappa.argtypes = [F, I]
        L.oracle_kappa.restype = I
        L.oracle_matvec.argtypes = [P, P, I, P]
        L.oracle_quantize_group.argtypes = [P, I, I, I, P, P, P]
        L.oracle_pack_k_row.argtypes = [P, I, I, P]
        L.oracle_unpack_k_row.argtypes = [P, I, I, P]
        L.oracle_pack_v_token.argtypes = [P, I, I, I, P]
        L.oracle_unpack_v_token.argtypes = [P, I, I, I, P]
        L.oracle_quantize_append.argtypes = [P, P, I, P, P, I, I, I, I, I, I, I, F, I, P,
                                             P, P, P, P, P, P]
        L.oracle_quantize_append.restype = I
        L.oracle_quantize_append_q.argtypes = [P, P, I, P, P, I, I, I, I, I, I, I, F, I, I, P,
                                               P, P, P, P, P, P]
        L.oracle_quantize_append_q.restype = I
        L.oracle_quantize_group_quest.argtypes = [P, I, I, P, P, P]
        L.oracle_quest_delta.argtypes = [I]
        L.oracle_quest_delta.restype = F
        L.oracle_pack_tokens.argtypes = [I] * 11 + [P] * 8
        L.oracle_pack_tokens.restype = I
        L.oracle_unpack_tokens.argtypes = [I] * 11 + [P] * 8
        L.oracle_unpack_tokens.restype = I
        L.oracle_decode.argtypes = [P, I, I, I, I, I, P, I, I, I, I, P, P, P, P, P, P, I, P]
        L.oracle_decode.restype = I
        L.oracle_decode_partial.argtypes = [P, I, I, I, I, I, P, I, I, I, I, P, P, P, P,
                                            I, I, I, I, P, P, P]
        L.oracle_decode_partial.restype = I
        L.oracle_merge.argtypes = [I, P, P, P, I, P]
        L.oracle_bf16_decode.argtypes = [P, I, I, I, I, P, P, I, P, P, I, P]
        L.oracle_bf16_decode.restype = I
        L.oracle_v_code_pos.argtypes = [I, I, I, I, P, P]
        L.oracle_k_code_pos.argtypes = [I, I, I, P, P]
        L.oracle_window_quantized.argtypes = [I, I, I, I]
        L.oracle_window_quantized.restype = I
        L.oracle_window_decode.argtypes = [P, I, I, I, I, I, P, P, P, P, I, I, I, I, I,
                                           P, P, P, P, P, I, I, I, P]
        L.oracle_window_decode.restype = I
        L.oracle_vq_encode.argtypes = [P, I, P, P, P]
        L.oracle_vq_append.argtypes = [P, P, I, P, P, P, P, I, I, I, I, I, P, P, P, P, P, P, P]
        L.oracle_vq_append.restype = I
        L.oracle_vq_decode.argtypes = [P, I, I, I, I, I, P, P, P, I, P, P, P, P, P, P, I, P]
        L.oracle_vq_decode.restype = I
        L.oracle_set_threads.argtypes = [I]
        L.oracle_get_threads.restype = I
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _dt(a) -> int:
    """0 = float32 array, 1 = bfloat16 bit patterns (uint16 array)."""
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {a.dtype}")


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


# ------------------------------------------------------------------ scalars

def f32_to_f16_bits(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32).ravel()
    L = lib()
    return np.array([L.oracle_f32_to_f16(float(v)) for v in x], dtype=np.uint16)


def f16_bits_to_f64(h) -> np.ndarray:
    h = np.asarray(h, dtype=np.uint16).ravel()
    L = lib()
    return np.array([L.oracle_f16_to_f64(int(v)) for v in h], dtype=np.float64)


def kappa(clip_alpha: float, group: int) -> int:
    return int(lib().oracle_kappa(float(clip_alpha), int(group)))


def matvec(T, x) -> np.ndarray:
    """float64 T @ x for a single d-vector (T None = identity)."""
    x = _c(x, np.float64)
    d = x.shape[0]
    Tc = None if T is None else _c(T, np.float64)
    out = np.empty(d, np.float64)
    lib().oracle_matvec(_p(Tc), _p(x), d, _p(out))
    return out


def quantize_group(x, bits: int, kap: int):
    """Codes (uint8 [g]), s_h, z_h (float16 bit patterns) of one group of float32 values."""
    x = _c(x, np.float32)
    codes = np.empty(x.shape[0], np.uint8)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    lib().oracle_quantize_group(_p(x), x.shape[0], bits, kap, _p(codes), _p(s), _p(z))
    return codes, int(s[0]), int(z[0])


def quest_delta(bits: int) -> float:
    """The QuEST INT step in units of the group RMS (float32)."""
    return float(lib().oracle_quest_delta(int(bits)))


def quantize_group_quest(x, bits: int):
    """QuEST INT codes (uint8 [g]), s_h, z_h (float16 bit patterns) of one group."""
    x = _c(x, np.float32)
    codes = np.empty(x.shape[0], np.uint8)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    lib().oracle_quantize_group_quest(_p(x), x.shape[0], bits, _p(codes), _p(s), _p(z))
    return codes, int(s[0]), int(z[0])


# ------------------------------------------------------------------ layout

def k_row_bytes(d: int, bits: int) -> int:
    return d * bits // 8


def v_tile_bytes(d: int, bits: int) -> int:
    return 16 * d * bits // 8


def v_code_pos(d: int, bits: int, tok: int, j: int):
    """(byte, bit) of code (token tok of its 16-token tile, dim j) inside the V tile."""
    by = C.c_size_t(0)
    bi = C.c_int(0)
    lib().oracle_v_code_pos(d, bits, tok, j, C.byref(by), C.byref(bi))
    return int(by.value), int(bi.value)


def k_code_pos(d: int, bits: int, j: int):
    by = C.c_size_t(0)
    bi = C.c_int(0)
    lib().oracle_k_code_pos(d, bits, j, C.byref(by), C.byref(bi))
    return int(by.value), int(bi.value)


def pack_k_row(codes, bits: int) -> np.ndarray:
    codes = _c(codes, np.uint8)
    d = codes.shape[0]
    row = np.zeros(k_row_bytes(d, bits), np.uint8)
    lib().oracle_pack_k_row(_p(codes), d, bits, _p(row))
    return row


def unpack_k_row(row, d: int, bits: int) -> np.ndarray:
    row = _c(row, np.uint8)
    out = np.empty(d, np.uint8)
    lib().oracle_unpack_k_row(_p(row), d, bits, _p(out))
    return out


def pack_v_tile(codes16, bits: int) -> np.ndarray:
    """codes16: uint8 [16][d] -> one V tile."""
    codes16 = _c(codes16, np.uint8)
    d = codes16.shape[1]
    tile = np.zeros(v_tile_bytes(d, bits), np.uint8)
    for t in range(16):
        lib().oracle_pack_v_token(_p(np.ascontiguousarray(codes16[t])), d, bits, t, _p(tile))
    return tile


def unpack_v_tile(tile, d: int, bits: int) -> np.ndarray:
    tile = _c(tile, np.uint8)
    out = np.empty((16, d), np.uint8)
    row = np.empty(d, np.uint8)
    for t in range(16):
        lib().oracle_unpack_v_token(_p(tile), d, bits, t, _p(row))
        out[t] = row
    return out


class Cache:
    """Host copy of the four cache planes plus their shape parameters."""

    def __init__(self, B, Hkv, T_cap, d, bits_k, bits_v, group):
        self.B, self.Hkv, self.T_cap, self.d = B, Hkv, T_cap, d
        self.bits_k, self.bits_v, self.group = bits_k, bits_v, group
        ng = d // group
        self.k_codes = np.zeros(B * Hkv * T_cap * d * bits_k // 8, np.uint8)
        self.v_codes = np.zeros(B * Hkv * T_cap * d * bits_v // 8, np.uint8)
        self.k_sz = np.zeros(B * Hkv * T_cap * ng * 2, np.uint16)
        self.v_sz = np.zeros(B * Hkv * T_cap * ng * 2, np.uint16)

    @classmethod
    def for_config(cls, cfg, T_cap=None, B=None):
        return cls(cfg.B if B is None else B, cfg.Hkv, cfg.T_cap if T_cap is None else T_cap,
                   cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)

    def planes(self):
        return self.k_codes, self.k_sz, self.v_codes, self.v_sz

    def _shape(self):
        return [self.B, self.Hkv, self.T_cap, self.d, self.bits_k, self.bits_v, self.group]

    def pack_tokens(self, b, h, t0, kc, vc, ksz, vsz):
        """Store codes uint8 [n][d] and (s, z) float16 bits uint16 [n][ng][2]."""
        kc, vc = _c(kc, np.uint8), _c(vc, np.uint8)
        ksz, vsz = _c(ksz, np.uint16), _c(vsz, np.uint16)
        n = kc.shape[0]
        r = lib().oracle_pack_tokens(*self._shape(), b, h, t0, n, _p(kc), _p(vc), _p(ksz),
                                     _p(vsz), _p(self.k_codes), _p(self.k_sz),
                                     _p(self.v_codes), _p(self.v_sz))
        if r:
            raise ValueError("oracle_pack_tokens: bad arguments")

    def unpack_tokens(self, b, h, t0, n):
        ng = self.d // self.group
        kc = np.empty((n, self.d), np.uint8)
        vc = np.empty((n, self.d), np.uint8)
        ksz = np.empty((n, ng, 2), np.uint16)
        vsz = np.empty((n, ng, 2), np.uint16)
        r = lib().oracle_unpack_tokens(*self._shape(), b, h, t0, n, _p(self.k_codes),
                                       _p(self.k_sz), _p(self.v_codes), _p(self.v_sz),
                                       _p(kc), _p(vc), _p(ksz), _p(vsz))
        if r:
            raise ValueError("oracle_unpack_tokens: bad arguments")
        return kc, vc, ksz, vsz

    def dequant(self, b, h, t0, n):
        """float64 (khat, vhat) [n][d] of tokens [t0, t0+n) of (b, h)."""
        kc, vc, ksz, vsz = self.unpack_tokens(b, h, t0, n)
        f = lambda a: a.view(np.float16).astype(np.float64)
        g = self.group
        ks, kz = np.repeat(f(ksz[..., 0]), g, axis=1), np.repeat(f(ksz[..., 1]), g, axis=1)
        vs, vz = np.repeat(f(vsz[..., 0]), g, axis=1), np.repeat(f(vsz[..., 1]), g, axis=1)
        return kz + kc * ks, vz + vc * vs


# ------------------------------------------------------------------ write path

def quantize_append(k, v, T_k, T_v, bits_k, bits_v, group, clip_alpha, cache: Cache, pos,
                    return_transformed=False, quantizer=0):
    """k, v: [B][n][Hkv][d] float32 or bf16 bits; T_k/T_v float32 [Hkv][d][d] or None.
    quantizer 0 = percentile-clipped affine, 1 = QuEST INT (clip_alpha unused)."""
    dt = _dt(k)
    assert _dt(v) == dt
    k, v = np.ascontiguousarray(k), np.ascontiguousarray(v)
    B, n, Hkv, d = k.shape
    Tk = None if T_k is None else _c(T_k, np.float32)
    Tv = None if T_v is None else _c(T_v, np.float32)
    pos = _c(pos, np.int32)
    kt = np.empty((B, n, Hkv, d), np.float32) if return_transformed else None
    vt = np.empty((B, n, Hkv, d), np.float32) if return_transformed else None
    r = lib().oracle_quantize_append_q(_p(k), _p(v), dt, _p(Tk), _p(Tv), B, n, Hkv, d, bits_k,
                                     bits_v, group, float(clip_alpha), int(quantizer),
                                     cache.T_cap, _p(pos),
                                     _p(cache.k_codes), _p(cache.k_sz), _p(cache.v_codes),
                                     _p(cache.v_sz), _p(kt), _p(vt))
    if r:
        raise ValueError("oracle_quantize_append: bad arguments")
    return (kt, vt) if return_transformed else None


# ------------------------------------------------------------------ read path

def decode(q, M, cache: Cache, seqlens, Hq=None, sel=None) -> np.ndarray:
    """float64 [B][Hq][d] decode attention (entries not in sel are NaN)."""
    dt = _dt(q)
    q = np.ascontiguousarray(q)
    B, Hq_, d = q.shape
    Mc = None if M is None else _c(M, np.float32)
    seqlens = _c(seqlens, np.int32)
    out = np.full((B, Hq_, d), np.nan, np.float64)
    selc = None if sel is None else _c(sel, np.int32).reshape(-1, 2)
    nsel = 0 if selc is None else selc.shape[0]
    r = lib().oracle_decode(_p(q), dt, B, Hq_, cache.Hkv, d, _p(Mc), cache.T_cap, cache.bits_k,
                            cache.bits_v, cache.group, _p(cache.k_codes), _p(cache.k_sz),
                            _p(cache.v_codes), _p(cache.v_sz), _p(seqlens), _p(selc), nsel,
                            _p(out))
    if r:
        raise ValueError("oracle_decode: bad arguments")
    return out


def decode_partial(q, M, cache: Cache, b, hq, t0, t1):
    """(m, l, o[d]) of query head (b, hq) over tokens [t0, t1)."""
    dt = _dt(q)
    q = np.ascontiguousarray(q)
    B, Hq, d = q.shape
    Mc = None if M is None else _c(M, np.float32)
    m = np.zeros(1)
    l = np.zeros(1)
    o = np.zeros(d)
    r = lib().oracle_decode_partial(_p(q), dt, B, Hq, cache.Hkv, d, _p(Mc), cache.T_cap,
                                    cache.bits_k, cache.bits_v, cache.group,
                                    _p(cache.k_codes), _p(cache.k_sz), _p(cache.v_codes),
                                    _p(cache.v_sz), b, hq, t0, t1, _p(m), _p(l), _p(o))
    if r:
        raise ValueError("oracle_decode_partial: bad arguments")
    return float(m[0]), float(l[0]), o


def merge(ms, ls, os_) -> np.ndarray:
    ms, ls = _c(ms, np.float64), _c(ls, np.float64)
    os_ = _c(os_, np.float64)
    n, d = os_.shape
    out = np.zeros(d)
    lib().oracle_merge(n, _p(ms), _p(ls), _p(os_), d, _p(out))
    return out


def bf16_decode(q_bits, K_bits, V_bits, seqlens, Hkv, sel=None) -> np.ndarray:
    """Uncompressed comparator over bf16 K, V [B][Hkv][T_cap][d]; q [B][Hq][d] bf16 bits."""
    q = _c(q_bits, np.uint16)
    K, V = _c(K_bits, np.uint16), _c(V_bits, np.uint16)
    B, Hq, d = q.shape
    T_cap = K.shape[2]
    seqlens = _c(seqlens, np.int32)
    out = np.full((B, Hq, d), np.nan)
    selc = None if sel is None else _c(sel, np.int32).reshape(-1, 2)
    nsel = 0 if selc is None else selc.shape[0]
    r = lib().oracle_bf16_decode(_p(q), B, Hq, Hkv, d, _p(K), _p(V), T_cap, _p(seqlens),
                                 _p(selc), nsel, _p(out))
    if r:
        raise ValueError("oracle_bf16_decode: bad arguments")
    return out


def window_quantized(L, S_sink, S_keep, S_flush) -> int:
    """Quantized middle length Q of a sequence of L positions (full-precision window)."""
    r = lib().oracle_window_quantized(int(L), int(S_sink), int(S_keep), int(S_flush))
    if r < 0:
        raise ValueError("oracle_window_quantized: bad arguments")
    return r


def window_decode(q, M, Tv, k_all, v_all, cache: Cache, seqlens, S_sink, S_keep,
                  S_flush) -> np.ndarray:
    """float64 [B][Hq][d] decode with a full-precision window: positions [S_sink,
    S_sink + Q) from the quantized cache, the others from k_all, v_all [B][T_cap][Hkv][d]
    (float32 or bf16 bits) with T_v [Hkv][d][d] (or None) applied to their values."""
    dq, din = _dt(q), _dt(k_all)
    assert _dt(v_all) == din
    q = np.ascontiguousarray(q)
    k_all, v_all = np.ascontiguousarray(k_all), np.ascontiguousarray(v_all)
    B, Hq, d = q.shape
    assert k_all.shape == (B, cache.T_cap, cache.Hkv, d)
    Mc = None if M is None else _c(M, np.float32)
    Tvc = None if Tv is None else _c(Tv, np.float32)
    seqlens = _c(seqlens, np.int32)
    out = np.full((B, Hq, d), np.nan, np.float64)
    r = lib().oracle_window_decode(_p(q), dq, B, Hq, cache.Hkv, d, _p(Mc), _p(Tvc),
                                   _p(k_all), _p(v_all), din, cache.T_cap, cache.bits_k,
                                   cache.bits_v, cache.group, _p(cache.k_codes),
                                   _p(cache.k_sz), _p(cache.v_codes), _p(cache.v_sz),
                                   _p(seqlens), int(S_sink), int(S_keep), int(S_flush),
                                   _p(out))
    if r:
        raise ValueError("oracle_window_decode: bad arguments")
    return out


def build_cache_from_fields(cfg, fields_per_b, tokens):
    """Cache whose first `tokens` positions hold the given codes/scales/zeros.

    fields_per_b(b) -> (kc, vc, ks, kz, vs, vz) as drawn by tests.synth.random_cache_fields.
    """
    c = Cache.for_config(cfg)
    for b in range(cfg.B):
        kc, vc, ks, kz, vs, vz = fields_per_b(b)
        ksz = np.stack([ks.astype(np.float16).view(np.uint16), kz.astype(np.float16).view(np.uint16)], -1)
        vsz = np.stack([vs.astype(np.float16).view(np.uint16), vz.astype(np.float16).view(np.uint16)], -1)
        for h in range(cfg.Hkv):
            c.pack_tokens(b, h, 0, kc[h], vc[h], ksz[h], vsz[h])
    return c


# ------------------------------------------------------------------ NOVA-KV vector quantization

VQ_DIM, VQ_SIZE = 4, 256


def vq_encode(x, cb):
    """(idx uint8 [d/4], gain float16 bits) of one transformed token x [d] (float32) with
    codebook cb [256][4] float16 bits."""
    x = _c(x, np.float32)
    cb = _c(cb, np.uint16)
    d = x.shape[0]
    idx = np.empty(d // VQ_DIM, np.uint8)
    g = np.zeros(1, np.uint16)
    lib().oracle_vq_encode(_p(x), d, _p(cb), _p(idx), _p(g))
    return idx, int(g[0])


class VQCache:
    """Host planes of a vector-quantized cache: indices [B][Hkv][T_cap][d/4] uint8 and
    gains [B][Hkv][T_cap] float16 bits, for keys and values."""

    def __init__(self, B, Hkv, T_cap, d):
        self.B, self.Hkv, self.T_cap, self.d = B, Hkv, T_cap, d
        self.k_idx = np.zeros(B * Hkv * T_cap * (d // VQ_DIM), np.uint8)
        self.v_idx = np.zeros_like(self.k_idx)
        self.k_gain = np.zeros(B * Hkv * T_cap, np.uint16)
        self.v_gain = np.zeros_like(self.k_gain)

    def planes(self):
        return self.k_idx, self.k_gain, self.v_idx, self.v_gain


def vq_append(k, v, T_k, T_v, cb_k, cb_v, cache: VQCache, pos, return_transformed=False):
    """k, v [B][n][Hkv][d] float32 or bf16 bits; T_k, T_v [Hkv][d][d] float32 or None;
    codebooks [Hkv][256][4] float16 bits."""
    dt = _dt(k)
    k, v = np.ascontiguousarray(k), np.ascontiguousarray(v)
    B, n, Hkv, d = k.shape
    Tk = None if T_k is None else _c(T_k, np.float32)
    Tv = None if T_v is None else _c(T_v, np.float32)
    ck, cv = _c(cb_k, np.uint16), _c(cb_v, np.uint16)
    pos = _c(pos, np.int32)
    kt = np.empty((B, n, Hkv, d), np.float32) if return_transformed else None
    vt = np.empty((B, n, Hkv, d), np.float32) if return_transformed else None
    r = lib().oracle_vq_append(_p(k), _p(v), dt, _p(Tk), _p(Tv), _p(ck), _p(cv), B, n, Hkv, d,
                               cache.T_cap, _p(pos), _p(cache.k_idx), _p(cache.k_gain),
                               _p(cache.v_idx), _p(cache.v_gain), _p(kt), _p(vt))
    if r:
        raise ValueError("oracle_vq_append: bad arguments")
    return (kt, vt) if return_transformed else None


def vq_decode(q, M, cb_k, cb_v, cache: VQCache, seqlens, sel=None) -> np.ndarray:
    dt = _dt(q)
    q = np.ascontiguousarray(q)
    B, Hq, d = q.shape
    Mc = None if M is None else _c(M, np.float32)
    ck, cv = _c(cb_k, np.uint16), _c(cb_v, np.uint16)
    seqlens = _c(seqlens, np.int32)
    out = np.full((B, Hq, d), np.nan, np.float64)
    selc = None if sel is None else _c(sel, np.int32).reshape(-1, 2)
    nsel = 0 if selc is None else selc.shape[0]
    r = lib().oracle_vq_decode(_p(q), dt, B, Hq, cache.Hkv, d, _p(Mc), _p(ck), _p(cv),
                               cache.T_cap, _p(cache.k_idx), _p(cache.k_gain), _p(cache.v_idx),
                               _p(cache.v_gain), _p(seqlens), _p(selc), nsel, _p(out))
    if r:
        raise ValueError("oracle_vq_decode: bad arguments")
    return out
