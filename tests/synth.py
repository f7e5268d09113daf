"""Seeded synthetic inputs for the transformed-KV quantize-append and decode path.

This module is shared by the oracle tests, the GPU parity tests, ``bench.py`` and
``__graft_entry__.smoke()``. It only *draws* inputs; it contains none of the method's
arithmetic (no key/value transform application, no clipping, no quantization, no
attention). Everything is numpy ``PCG64`` with ``seed = 1000 * cfg + stream``.

Workload shapes follow the decode workloads the pages discuss: Qwen3-8B-shaped GQA
(32 query heads / 8 KV heads, head_dim 128) at 16K context with batch 16 and 64, one
long-context case at 128K, and a GPT-OSS-20B-like small-head case (64/8 heads,
head_dim 64). The models and datasets themselves are not available, so these
generators stand in for their post-RoPE key, value and query activations:

* pre-RoPE keys per KV head: Gaussian, channel std ~ lognormal(0, 0.5), plus four
  outlier channels per head with 10x std and mean +3 (the channel-structured keys
  that motivate post-RoPE transforms in WUSH-KV, section 1 and section 4.2);
  rotate-half RoPE (pairs i, i + d/2) with base 1e6 at positions 0..T-1;
* values and queries N(0, 1);
* per-KV-head transforms T = Q1 diag(sigma) Q2 with Haar-orthogonal Q1, Q2 and
  log sigma ~ N(0, 0.5) clamped to +-ln(10)/2 (condition number <= 10), and the
  query-side matrix T^{-T} = Q1 diag(1/sigma) Q2 in closed form.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

STREAM_K, STREAM_V, STREAM_Q, STREAM_TK, STREAM_TV, STREAM_SEQ, STREAM_CACHE = 1, 2, 3, 4, 5, 6, 7
STREAM_CODEBOOK = 8
STREAM_WINDOW, STREAM_VQ = 9, 10


@dataclasses.dataclass(frozen=True)
class Config:
    """One synthetic workload."""
    idx: int
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T_cap: int                 # cache capacity per sequence (tokens)
    bits_k: int
    bits_v: int
    group: int
    clip_alpha: float
    in_dtype: str              # 'f32' or 'bf16' for keys/values fed to the append
    q_dtype: str               # 'f32' or 'bf16'
    out_dtype: str             # 'f32' or 'bf16'
    seq_lo: int                # seqlens drawn uniform in [seq_lo, seq_hi]
    seq_hi: int
    append_n: int = 0          # tokens per sequence in a chunk append (0: the whole context)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    0: Config(0, "tiny-gqa4-d128-ctx2048-f32", B=1, Hq=4, Hkv=1, d=128, T_cap=2048,
              bits_k=2, bits_v=2, group=128, clip_alpha=0.01, in_dtype="f32",
              q_dtype="f32", out_dtype="f32", seq_lo=2048, seq_hi=2048),
    1: Config(1, "qwen3-8b-b16-ctx16k-2bit", B=16, Hq=32, Hkv=8, d=128, T_cap=16384,
              bits_k=2, bits_v=2, group=128, clip_alpha=0.01, in_dtype="bf16",
              q_dtype="bf16", out_dtype="bf16", seq_lo=16384, seq_hi=16384),
    2: Config(2, "qwen3-8b-b64-ctx16k-ragged-2bit", B=64, Hq=32, Hkv=8, d=128, T_cap=16384,
              bits_k=2, bits_v=2, group=128, clip_alpha=0.01, in_dtype="bf16",
              q_dtype="bf16", out_dtype="bf16", seq_lo=12288, seq_hi=16384),
    3: Config(3, "qwen3-8b-b4-ctx128k-k4v2", B=4, Hq=32, Hkv=8, d=128, T_cap=131072,
              bits_k=4, bits_v=2, group=128, clip_alpha=0.005, in_dtype="bf16",
              q_dtype="bf16", out_dtype="bf16", seq_lo=131072, seq_hi=131072),
    4: Config(4, "gptoss20b-like-b8-gqa8-d64-append32k", B=8, Hq=64, Hkv=8, d=64,
              T_cap=32768, bits_k=2, bits_v=2, group=64, clip_alpha=0.01, in_dtype="bf16",
              q_dtype="bf16", out_dtype="bf16", seq_lo=16384, seq_hi=32768,
              append_n=32768),
}


def _rng(cfg: Config, stream: int, *sub: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([1000 * cfg.idx + stream, *sub])))


# ----------------------------------------------------------------------------- dtypes

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def as_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 array -> array in the config dtype ('f32' float32, 'bf16' uint16 bits)."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(x)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------- draws

def seqlens(cfg: Config) -> np.ndarray:
    """int32 [B], uniform in [seq_lo, seq_hi]."""
    if cfg.seq_lo == cfg.seq_hi:
        return np.full(cfg.B, cfg.seq_lo, dtype=np.int32)
    return _rng(cfg, STREAM_SEQ).integers(cfg.seq_lo, cfg.seq_hi + 1, size=cfg.B).astype(np.int32)


def key_channel_stats(cfg: Config):
    """Per KV head channel (mean, std) of the pre-RoPE keys: float64 [Hkv][d] each."""
    r = _rng(cfg, STREAM_K, 0)
    std = r.lognormal(0.0, 0.5, size=(cfg.Hkv, cfg.d))
    mean = np.zeros((cfg.Hkv, cfg.d))
    for h in range(cfg.Hkv):
        out = r.choice(cfg.d, size=4, replace=False)
        std[h, out] *= 10.0
        mean[h, out] = 3.0
    return mean, std


def _rope(x: np.ndarray, pos: np.ndarray, base: float = 1e6) -> np.ndarray:
    """Rotate-half RoPE of x [n][H][d] (float64) at integer positions pos [n]."""
    d = x.shape[-1]
    half = d // 2
    inv_freq = base ** (-2.0 * np.arange(half) / d)
    ang = pos[:, None].astype(np.float64) * inv_freq[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def keys(cfg: Config, b: int, t0: int, t1: int) -> np.ndarray:
    """Post-RoPE keys of sequence b at positions [t0, t1): float32 [t1-t0][Hkv][d].

    Token t of sequence b is drawn from its own counter-keyed stream chunk so that any
    sub-range is reproducible without drawing the rest of the sequence.
    """
    mean, std = key_channel_stats(cfg)
    out = np.empty((t1 - t0, cfg.Hkv, cfg.d), dtype=np.float32)
    CH = 4096
    for c0 in range((t0 // CH) * CH, t1, CH):
        r = _rng(cfg, STREAM_K, 1, b, c0 // CH)
        z = r.standard_normal((CH, cfg.Hkv, cfg.d))
        pre = mean[None] + std[None] * z
        pos = np.arange(c0, c0 + CH)
        post = _rope(pre, pos)
        lo, hi = max(c0, t0), min(c0 + CH, t1)
        out[lo - t0:hi - t0] = post[lo - c0:hi - c0]
    return out


def values(cfg: Config, b: int, t0: int, t1: int) -> np.ndarray:
    """Values of sequence b at positions [t0, t1): float32 N(0,1) [t1-t0][Hkv][d]."""
    out = np.empty((t1 - t0, cfg.Hkv, cfg.d), dtype=np.float32)
    CH = 4096
    for c0 in range((t0 // CH) * CH, t1, CH):
        r = _rng(cfg, STREAM_V, b, c0 // CH)
        z = r.standard_normal((CH, cfg.Hkv, cfg.d), dtype=np.float32)
        lo, hi = max(c0, t0), min(c0 + CH, t1)
        out[lo - t0:hi - t0] = z[lo - c0:hi - c0]
    return out


def kv_batch(cfg: Config, t0: int, t1: int):
    """Keys and values for all sequences at positions [t0, t1): float32 [B][n][Hkv][d]."""
    k = np.stack([keys(cfg, b, t0, t1) for b in range(cfg.B)])
    v = np.stack([values(cfg, b, t0, t1) for b in range(cfg.B)])
    return k, v


def queries(cfg: Config, step: int = 0) -> np.ndarray:
    """Post-RoPE queries of one decode step: float32 N(0,1) [B][Hq][d]."""
    return _rng(cfg, STREAM_Q, step).standard_normal((cfg.B, cfg.Hq, cfg.d)).astype(np.float32)


def _haar(r: np.random.Generator, d: int) -> np.ndarray:
    a = r.standard_normal((d, d))
    q, rr = np.linalg.qr(a)
    return q * np.sign(np.diag(rr))[None, :]


def transforms(cfg: Config):
    """(T_k, T_v, T_k^{-T}) as float32 [Hkv][d][d] row-major.

    T = Q1 diag(sigma) Q2; because Q1, Q2 are orthogonal, T^{-T} = Q1 diag(1/sigma) Q2.
    """
    lim = math.log(10.0) / 2.0
    out = {}
    for name, stream in (("k", STREAM_TK), ("v", STREAM_TV)):
        r = _rng(cfg, stream)
        T = np.empty((cfg.Hkv, cfg.d, cfg.d))
        Tit = np.empty((cfg.Hkv, cfg.d, cfg.d))
        for h in range(cfg.Hkv):
            q1, q2 = _haar(r, cfg.d), _haar(r, cfg.d)
            ls = np.clip(r.normal(0.0, 0.5, size=cfg.d), -lim, lim)
            T[h] = (q1 * np.exp(ls)[None, :]) @ q2
            Tit[h] = (q1 * np.exp(-ls)[None, :]) @ q2
        out[name] = (T, Tit)
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)
    return f(out["k"][0]), f(out["v"][0]), f(out["k"][1])


def transforms_f64(cfg: Config):
    """Same draws as :func:`transforms`, kept in float64: (T_k, T_k^{-T})."""
    lim = math.log(10.0) / 2.0
    r = _rng(cfg, STREAM_TK)
    T = np.empty((cfg.Hkv, cfg.d, cfg.d))
    Tit = np.empty((cfg.Hkv, cfg.d, cfg.d))
    for h in range(cfg.Hkv):
        q1, q2 = _haar(r, cfg.d), _haar(r, cfg.d)
        ls = np.clip(r.normal(0.0, 0.5, size=cfg.d), -lim, lim)
        T[h] = (q1 * np.exp(ls)[None, :]) @ q2
        Tit[h] = (q1 * np.exp(-ls)[None, :]) @ q2
    return T, Tit


def random_cache_fields(cfg: Config, b: int, tokens: int):
    """Uniform random cache contents for one sequence (all KV heads).

    Returns (k_codes, v_codes, k_s, k_z, v_s, v_z): codes uint8 [Hkv][tokens][d] in
    [0, 2^bits), scales float32 positive and zero-points float32, both exactly
    representable in float16. Used to exercise the decode at full size without
    running the quantizer.
    """
    r = _rng(cfg, STREAM_CACHE, b)
    ng = cfg.d // cfg.group
    kc = r.integers(0, 1 << cfg.bits_k, size=(cfg.Hkv, tokens, cfg.d), dtype=np.uint8)
    vc = r.integers(0, 1 << cfg.bits_v, size=(cfg.Hkv, tokens, cfg.d), dtype=np.uint8)
    f16 = lambda a: a.astype(np.float16).astype(np.float32)
    ks = f16(r.uniform(0.05, 2.0, size=(cfg.Hkv, tokens, ng)))
    kz = f16(r.uniform(-4.0, 0.0, size=(cfg.Hkv, tokens, ng)))
    vs = f16(r.uniform(0.2, 1.5, size=(cfg.Hkv, tokens, ng)))
    vz = f16(r.uniform(-2.5, -0.5, size=(cfg.Hkv, tokens, ng)))
    return kc, vc, ks, kz, vs, vz


def codebooks(cfg: Config):
    """Synthetic vector-quantization codebooks (codebook training is out of scope): for
    keys and values, per KV head, 256 four-dimensional codewords drawn N(0, 1) and rounded
    to float16 (the encoder scales tokens to unit RMS first). Returns (cb_k, cb_v) as
    float16 bit patterns uint16 [Hkv][256][4]."""
    r = _rng(cfg, STREAM_CODEBOOK)
    out = []
    for _ in range(2):
        c = r.standard_normal((cfg.Hkv, 256, 4)).astype(np.float16)
        out.append(np.ascontiguousarray(c).view(np.uint16))
    return out[0], out[1]


def window_tokens(cfg: Config, b: int, n: int) -> tuple:
    """Full-precision window tokens of sequence b for full-size tests: keys and values
    float32 N(0, 1) [Hkv][n][d] (callers round them to bfloat16)."""
    r = _rng(cfg, STREAM_WINDOW, b)
    return (r.standard_normal((cfg.Hkv, n, cfg.d)).astype(np.float32),
            r.standard_normal((cfg.Hkv, n, cfg.d)).astype(np.float32))


def random_vq_planes(cfg: Config, b: int, tokens: int) -> tuple:
    """Uniform random vector-quantized cache contents of sequence b (all KV heads), to
    exercise the VQ decode at full size without running the encoder: indices uint8
    [Hkv][tokens][d/4], gains float16 bits uint16 [Hkv][tokens] in [0.5, 1.5) (keys, then
    values)."""
    r = _rng(cfg, STREAM_VQ, b)
    g = lambda: r.uniform(0.5, 1.5, size=(cfg.Hkv, tokens)).astype(np.float16).view(np.uint16)
    ki = r.integers(0, 256, size=(cfg.Hkv, tokens, cfg.d // 4), dtype=np.uint8)
    kg = g()
    vi = r.integers(0, 256, size=(cfg.Hkv, tokens, cfg.d // 4), dtype=np.uint8)
    vg = g()
    return ki, kg, vi, vg
