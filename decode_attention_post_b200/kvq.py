"""ctypes binding of include/kvq.h. Argument marshalling only.

Every function takes torch tensors that already live on a CUDA device (the caller owns
them), checks dtype/shape/contiguity, and calls the C entry point of the same name on
the current CUDA stream (or the stream given). A non-OK status raises KvqError with the
library's own message. If ``libkvq.so`` is missing the first call raises: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libkvq.so")
_lib = None

KVQ_F32, KVQ_BF16 = 0, 1
KVQ_QUANT_PERCENTILE, KVQ_QUANT_QUEST = 0, 1
KVQ_DEVERR_SEQLEN_CLAMPED = 0x1
KVQ_DEVERR_POS_RANGE = 0x2
KVQ_DEVERR_NONFINITE = 0x4
KVQ_DEVERR_WAIT_TIMEOUT = 0x8
KVQ_DEVERR_PAGE_RANGE = 0x10

_P, _I, _F, _S = C.c_void_p, C.c_int, C.c_float, C.c_size_t


class _QParams(C.Structure):
    _fields_ = [("bits_k", _I), ("bits_v", _I), ("group", _I), ("clip_alpha", _F),
                ("quantizer", _I)]


class _Cache(C.Structure):
    _fields_ = [("B", _I), ("Hkv", _I), ("T_cap", _I), ("d", _I), ("qp", _QParams),
                ("k_codes", _P), ("k_sz", _P), ("v_codes", _P), ("v_sz", _P),
                ("block_table", _P), ("page_tokens", _I), ("num_pages", _I)]


class _Window(C.Structure):
    _fields_ = [("S_sink", _I), ("S_keep", _I), ("S_flush", _I), ("k_sink", _P),
                ("v_sink", _P), ("k_recent", _P), ("v_recent", _P), ("T_v", _P)]


class _VQCache(C.Structure):
    _fields_ = [("B", _I), ("Hkv", _I), ("T_cap", _I), ("d", _I), ("k_idx", _P),
                ("k_gain", _P), ("v_idx", _P), ("v_gain", _P)]


class KvqError(RuntimeError):
    def __init__(self, status: int, func: str, detail: str):
        self.status = status
        super().__init__(f"{func}: status {status}: {detail}")


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libkvq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m decode_attention_post_b200.build`")
    L = C.CDLL(_LIB_PATH)
    L.kvq_status_string.restype = C.c_char_p
    L.kvq_status_string.argtypes = [_I]
    L.kvq_last_error.restype = C.c_char_p
    L.kvq_cache_plane_bytes.restype = _S
    L.kvq_cache_plane_bytes.argtypes = [C.POINTER(_Cache), _I]
    L.kvq_quantize_append.restype = _I
    L.kvq_quantize_append.argtypes = [_P, _P, _I, _P, _P, C.POINTER(_QParams), C.POINTER(_Cache),
                                      _P, _I, _P, _P]
    L.kvq_decode_workspace_bytes.restype = _S
    L.kvq_decode_workspace_bytes.argtypes = [C.POINTER(_Cache), _I, _I]
    L.kvq_decode_attention.restype = _I
    L.kvq_decode_attention.argtypes = [_P, _I, _I, _P, C.POINTER(_Cache), _P, _I, _P, _I, _P, _S,
                                       _P, _P]
    L.kvq_decode_attention_noalloc.restype = _I
    L.kvq_decode_attention_window.argtypes = [_P, _I, _I, _P, C.POINTER(_Cache),
                                              C.POINTER(_Window), _P, _I, _P, _I, _P, _S,
                                              _P, _P]
    L.kvq_decode_attention_window.restype = _I
    L.kvq_window_append.argtypes = [_P, _P, _I, _P, _P, C.POINTER(_QParams), C.POINTER(_Cache),
                                    C.POINTER(_Window), _P, _I, _P, _P]
    L.kvq_window_append.restype = _I
    L.kvq_vq_plane_bytes.restype = _S
    L.kvq_vq_plane_bytes.argtypes = [C.POINTER(_VQCache), _I]
    L.kvq_vq_append.restype = _I
    L.kvq_vq_append.argtypes = [_P, _P, _I, _P, _P, _P, _P, C.POINTER(_VQCache), _P, _I, _P, _P]
    L.kvq_vq_decode_workspace_bytes.restype = _S
    L.kvq_vq_decode_workspace_bytes.argtypes = [C.POINTER(_VQCache), _I, _I]
    L.kvq_vq_decode_attention.restype = _I
    L.kvq_vq_decode_attention.argtypes = [_P, _I, _I, _P, _P, _P, C.POINTER(_VQCache), _P, _I,
                                          _P, _I, _P, _S, _P, _P]
    L.kvq_decode_attention_noalloc.argtypes = [_P, _I, _I, _P, C.POINTER(_Cache), _P, _I, _P,
                                               _I, _P, _P]
    L.kvq_bf16_decode_workspace_bytes.restype = _S
    L.kvq_bf16_decode_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
    L.kvq_bf16_decode.restype = _I
    L.kvq_bf16_decode.argtypes = [_P, _I, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _S, _P, _P]
    _lib = L
    return L


def _check(status: int, func: str):
    if status != 0:
        L = load()
        raise KvqError(status, func, L.kvq_last_error().decode() or
                       L.kvq_status_string(status).decode())


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _dt(t) -> int:
    if t.dtype == torch.float32:
        return KVQ_F32
    if t.dtype == torch.bfloat16:
        return KVQ_BF16
    raise TypeError(f"expected float32 or bfloat16, got {t.dtype}")


def _cuda(name, t, dtype=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


@dataclasses.dataclass(frozen=True)
class QParams:
    """kvq_qparams: quantizer KVQ_QUANT_PERCENTILE (clip_alpha used) or KVQ_QUANT_QUEST."""
    bits_k: int = 2
    bits_v: int = 2
    group: int = 128
    clip_alpha: float = 0.01
    quantizer: int = KVQ_QUANT_PERCENTILE

    def _c(self):
        return _QParams(self.bits_k, self.bits_v, self.group, self.clip_alpha, self.quantizer)


class KVCache:
    """The four cache planes (caller-owned device memory) plus their shape.

    ``KVCache.allocate`` asks the library for each plane's size and allocates it with
    torch; ``KVCache(planes=...)`` wraps existing uint8 tensors. With ``block_table``
    (int32 [B][T_cap/page_tokens] on the device) the planes are page pools of
    ``num_pages`` pages (``KVCache.allocate_paged``).
    """

    def __init__(self, B, Hkv, T_cap, d, qp: QParams, planes, block_table=None,
                 page_tokens=0, num_pages=0):
        self.B, self.Hkv, self.T_cap, self.d, self.qp = B, Hkv, T_cap, d, qp
        self.k_codes, self.k_sz, self.v_codes, self.v_sz = planes
        for name, t in zip(("k_codes", "k_sz", "v_codes", "v_sz"), planes):
            _cuda(name, t, torch.uint8)
        _cuda("block_table", block_table, torch.int32)
        self.block_table, self.page_tokens, self.num_pages = block_table, page_tokens, num_pages
        self._desc = _Cache(B, Hkv, T_cap, d, qp._c(), _ptr(self.k_codes), _ptr(self.k_sz),
                            _ptr(self.v_codes), _ptr(self.v_sz), _ptr(block_table),
                            page_tokens if block_table is not None else 0,
                            num_pages if block_table is not None else 0)

    @staticmethod
    def plane_bytes(B, Hkv, T_cap, d, qp: QParams, page_tokens=0, num_pages=0):
        """Plane sizes; with page_tokens > 0, those of a pool of num_pages pages."""
        paged = page_tokens > 0
        desc = _Cache(B, Hkv, T_cap, d, qp._c(), None, None, None, None,
                      C.c_void_p(16) if paged else None, page_tokens, num_pages)
        return [int(load().kvq_cache_plane_bytes(C.byref(desc), w)) for w in range(4)]

    @classmethod
    def allocate(cls, B, Hkv, T_cap, d, qp: QParams, device="cuda", zero=True):
        sizes = cls.plane_bytes(B, Hkv, T_cap, d, qp)
        if min(sizes) <= 0:
            raise ValueError("invalid cache shape")
        make = torch.zeros if zero else torch.empty
        planes = [make(n, dtype=torch.uint8, device=device) for n in sizes]
        return cls(B, Hkv, T_cap, d, qp, planes)

    @classmethod
    def allocate_paged(cls, num_pages, page_tokens, block_table, Hkv, d, qp: QParams,
                       device="cuda", zero=True):
        """A pool of num_pages pages; block_table int32 [B][pages per sequence] on the
        device gives the page of every page_tokens positions of every sequence."""
        B, per_seq = block_table.shape
        T_cap = per_seq * page_tokens
        sizes = cls.plane_bytes(B, Hkv, T_cap, d, qp, page_tokens, num_pages)
        if min(sizes) <= 0:
            raise ValueError("invalid paged cache shape")
        make = torch.zeros if zero else torch.empty
        planes = [make(n, dtype=torch.uint8, device=device) for n in sizes]
        return cls(B, Hkv, T_cap, d, qp, planes, block_table, page_tokens, num_pages)

    def view_sequence(self, b: int) -> "KVCache":
        """The same cache restricted to sequence b (a B = 1 view of its planes)."""
        if self.block_table is not None:
            return KVCache(1, self.Hkv, self.T_cap, self.d, self.qp,
                           (self.k_codes, self.k_sz, self.v_codes, self.v_sz),
                           self.block_table[b:b + 1], self.page_tokens, self.num_pages)
        per = [p.numel() // self.B for p in (self.k_codes, self.k_sz, self.v_codes, self.v_sz)]
        planes = [p[b * n:(b + 1) * n] for p, n in zip((self.k_codes, self.k_sz, self.v_codes,
                                                         self.v_sz), per)]
        return KVCache(1, self.Hkv, self.T_cap, self.d, self.qp, planes)

    @property
    def desc(self):
        return self._desc

    def nbytes(self):
        return sum(p.numel() for p in (self.k_codes, self.k_sz, self.v_codes, self.v_sz))


def cache_plane_bytes(cache: KVCache, which: int) -> int:
    return int(load().kvq_cache_plane_bytes(C.byref(cache.desc), which))


def quantize_append(k_post_rope, v, T_k, T_v, qp: QParams, cache: KVCache, pos, n=None,
                    dev_err=None, stream=None):
    """kvq_quantize_append: k, v [B][n][Hkv][d] float32/bfloat16; T_k, T_v [Hkv][d][d]
    float32 or None; pos int32 [B] on the device."""
    L = load()
    _cuda("k_post_rope", k_post_rope)
    _cuda("v", v, k_post_rope.dtype)
    _cuda("T_k", T_k, torch.float32)
    _cuda("T_v", T_v, torch.float32)
    _cuda("pos", pos, torch.int32)
    _cuda("dev_err", dev_err, torch.int32)
    if n is None:
        n = k_post_rope.shape[1]
    qpc = qp._c()
    _check(L.kvq_quantize_append(_ptr(k_post_rope), _ptr(v), _dt(k_post_rope), _ptr(T_k),
                                 _ptr(T_v), C.byref(qpc), C.byref(cache.desc), _ptr(pos), int(n),
                                 _ptr(dev_err), _stream(stream)), "kvq_quantize_append")


def decode_workspace_bytes(cache: KVCache, Hq: int, max_seqlen: int) -> int:
    return int(load().kvq_decode_workspace_bytes(C.byref(cache.desc), int(Hq), int(max_seqlen)))


def decode_attention(q, Tk_invT, cache: KVCache, seqlens, max_seqlen: int, out, workspace,
                     dev_err=None, stream=None):
    """kvq_decode_attention: q [B][Hq][d] float32/bfloat16; Tk_invT [Hkv][d][d] float32 or
    None; seqlens int32 [B]; out [B][Hq][d] float32/bfloat16; workspace uint8 tensor."""
    L = load()
    _cuda("q", q)
    _cuda("Tk_invT", Tk_invT, torch.float32)
    _cuda("seqlens", seqlens, torch.int32)
    _cuda("out", out)
    _cuda("workspace", workspace, torch.uint8)
    _cuda("dev_err", dev_err, torch.int32)
    Hq = q.shape[1]
    _check(L.kvq_decode_attention(_ptr(q), _dt(q), int(Hq), _ptr(Tk_invT), C.byref(cache.desc),
                                  _ptr(seqlens), int(max_seqlen), _ptr(out), _dt(out),
                                  _ptr(workspace), workspace.numel(), _ptr(dev_err),
                                  _stream(stream)), "kvq_decode_attention")


def decode_attention_window(q, Tk_invT, cache: KVCache, S_sink: int, S_keep: int,
                            S_flush: int, k_sink, v_sink, k_recent, v_recent, T_v, seqlens,
                            max_seqlen: int, out, workspace, dev_err=None, stream=None):
    """kvq_decode_attention_window: decode with a full-precision window. q bfloat16
    [B][Hq][d]; k_sink, v_sink bfloat16 [B][Hkv][S_sink][d] (None when S_sink = 0);
    k_recent, v_recent bfloat16 [B][Hkv][S_keep + S_flush][d] (position t at slot
    t % (S_keep + S_flush)); T_v float32 [Hkv][d][d] or None; seqlens int32 [B] whole
    lengths; the cache holds the quantized middle from its position 0."""
    L = load()
    _cuda("q", q)
    _cuda("Tk_invT", Tk_invT, torch.float32)
    for name, t in (("k_sink", k_sink), ("v_sink", v_sink), ("k_recent", k_recent),
                    ("v_recent", v_recent)):
        _cuda(name, t, torch.bfloat16)
    _cuda("T_v", T_v, torch.float32)
    _cuda("seqlens", seqlens, torch.int32)
    _cuda("out", out)
    _cuda("workspace", workspace, torch.uint8)
    _cuda("dev_err", dev_err, torch.int32)
    win = _Window(int(S_sink), int(S_keep), int(S_flush), _ptr(k_sink), _ptr(v_sink),
                  _ptr(k_recent), _ptr(v_recent), _ptr(T_v))
    _check(L.kvq_decode_attention_window(_ptr(q), _dt(q), int(q.shape[1]), _ptr(Tk_invT),
                                         C.byref(cache.desc), C.byref(win), _ptr(seqlens),
                                         int(max_seqlen), _ptr(out), _dt(out), _ptr(workspace),
                                         workspace.numel(), _ptr(dev_err), _stream(stream)),
           "kvq_decode_attention_window")


def window_append(k_new, v_new, T_k, T_v, qp: QParams, cache: KVCache, S_sink: int,
                  S_keep: int, S_flush: int, k_sink, v_sink, k_recent, v_recent, seqlens,
                  n=None, dev_err=None, stream=None):
    """kvq_window_append: append n bfloat16 tokens k_new, v_new [B][n][Hkv][d] to sequences
    of seqlens (int32 [B], lengths before the call; not updated) with a full-precision
    window: sink k_sink, v_sink [B][Hkv][S_sink][d] (None when S_sink = 0), recent ring
    k_recent, v_recent [B][Hkv][S_keep + S_flush][d], positions leaving the window
    quantized into the cache at position t - S_sink."""
    L = load()
    _cuda("k_new", k_new, torch.bfloat16)
    _cuda("v_new", v_new, torch.bfloat16)
    _cuda("T_k", T_k, torch.float32)
    _cuda("T_v", T_v, torch.float32)
    for name, t in (("k_sink", k_sink), ("v_sink", v_sink), ("k_recent", k_recent),
                    ("v_recent", v_recent)):
        _cuda(name, t, torch.bfloat16)
    _cuda("seqlens", seqlens, torch.int32)
    _cuda("dev_err", dev_err, torch.int32)
    if n is None:
        n = k_new.shape[1]
    win = _Window(int(S_sink), int(S_keep), int(S_flush), _ptr(k_sink), _ptr(v_sink),
                  _ptr(k_recent), _ptr(v_recent), None)
    qpc = qp._c()
    _check(L.kvq_window_append(_ptr(k_new), _ptr(v_new), KVQ_BF16, _ptr(T_k), _ptr(T_v),
                               C.byref(qpc), C.byref(cache.desc), C.byref(win), _ptr(seqlens),
                               int(n), _ptr(dev_err), _stream(stream)), "kvq_window_append")


NOALLOC_SCRATCH_BYTES = 8 << 20


def decode_attention_noalloc(q, Tk_invT, cache: KVCache, seqlens, max_seqlen: int, out,
                             dev_err=None, stream=None):
    """kvq_decode_attention_noalloc: as decode_attention, with the library's fixed
    device scratch array instead of a caller workspace (for callers that cannot
    allocate device memory; calls must not overlap on the GPU)."""
    L = load()
    _cuda("q", q)
    _cuda("Tk_invT", Tk_invT, torch.float32)
    _cuda("seqlens", seqlens, torch.int32)
    _cuda("out", out)
    _cuda("dev_err", dev_err, torch.int32)
    _check(L.kvq_decode_attention_noalloc(_ptr(q), _dt(q), int(q.shape[1]), _ptr(Tk_invT),
                                          C.byref(cache.desc), _ptr(seqlens), int(max_seqlen),
                                          _ptr(out), _dt(out), _ptr(dev_err), _stream(stream)),
           "kvq_decode_attention_noalloc")


def bf16_decode_workspace_bytes(B, Hq, Hkv, d, max_seqlen) -> int:
    return int(load().kvq_bf16_decode_workspace_bytes(int(B), int(Hq), int(Hkv), int(d),
                                                      int(max_seqlen)))


def bf16_decode(q, k, v, seqlens, max_seqlen: int, out, workspace, dev_err=None, stream=None):
    """kvq_bf16_decode: q, out [B][Hq][d] bf16; k, v [B][Hkv][T_cap][d] bf16."""
    L = load()
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _cuda(name, t, torch.bfloat16)
    _cuda("seqlens", seqlens, torch.int32)
    _cuda("workspace", workspace, torch.uint8)
    _cuda("dev_err", dev_err, torch.int32)
    B, Hq, d = q.shape
    _, Hkv, T_cap, _ = k.shape
    _check(L.kvq_bf16_decode(_ptr(q), int(Hq), _ptr(k), _ptr(v), int(B), int(Hkv), int(T_cap),
                             int(d), _ptr(seqlens), int(max_seqlen), _ptr(out), _ptr(workspace),
                             workspace.numel(), _ptr(dev_err), _stream(stream)), "kvq_bf16_decode")


# ------------------------------------------------------------------ vector-quantized cache

class VQCache:
    """kvq_vq_cache: index planes [B][Hkv][T_cap][d/4] uint8 and gain planes
    [B][Hkv][T_cap] float16 (stored as uint8 tensors), caller-owned device memory."""

    def __init__(self, B, Hkv, T_cap, d, planes):
        self.B, self.Hkv, self.T_cap, self.d = B, Hkv, T_cap, d
        self.k_idx, self.k_gain, self.v_idx, self.v_gain = planes
        for name, t in zip(("k_idx", "k_gain", "v_idx", "v_gain"), planes):
            _cuda(name, t, torch.uint8)
        self._desc = _VQCache(B, Hkv, T_cap, d, _ptr(self.k_idx), _ptr(self.k_gain),
                              _ptr(self.v_idx), _ptr(self.v_gain))

    @classmethod
    def allocate(cls, B, Hkv, T_cap, d, device="cuda", zero=True):
        desc = _VQCache(B, Hkv, T_cap, d, None, None, None, None)
        sizes = [int(load().kvq_vq_plane_bytes(C.byref(desc), w)) for w in range(4)]
        if min(sizes) <= 0:
            raise ValueError("invalid VQ cache shape")
        make = torch.zeros if zero else torch.empty
        return cls(B, Hkv, T_cap, d, [make(n, dtype=torch.uint8, device=device) for n in sizes])

    @property
    def desc(self):
        return self._desc


def vq_append(k, v, T_k, T_v, cb_k, cb_v, cache: VQCache, pos, n=None, dev_err=None,
              stream=None):
    """kvq_vq_append: k, v [B][n][Hkv][d] float32/bfloat16; T_k, T_v [Hkv][d][d] float32 or
    None; codebooks cb_k, cb_v [Hkv][256][4] float16; pos int32 [B]."""
    L = load()
    _cuda("k", k)
    _cuda("v", v, k.dtype)
    _cuda("T_k", T_k, torch.float32)
    _cuda("T_v", T_v, torch.float32)
    _cuda("cb_k", cb_k, torch.float16)
    _cuda("cb_v", cb_v, torch.float16)
    _cuda("pos", pos, torch.int32)
    _cuda("dev_err", dev_err, torch.int32)
    if n is None:
        n = k.shape[1]
    _check(L.kvq_vq_append(_ptr(k), _ptr(v), _dt(k), _ptr(T_k), _ptr(T_v), _ptr(cb_k),
                           _ptr(cb_v), C.byref(cache.desc), _ptr(pos), int(n), _ptr(dev_err),
                           _stream(stream)), "kvq_vq_append")


def vq_decode_workspace_bytes(cache: VQCache, Hq: int, max_seqlen: int) -> int:
    return int(load().kvq_vq_decode_workspace_bytes(C.byref(cache.desc), int(Hq),
                                                    int(max_seqlen)))


def vq_decode_attention(q, Tk_invT, cb_k, cb_v, cache: VQCache, seqlens, max_seqlen: int, out,
                        workspace, dev_err=None, stream=None):
    """kvq_vq_decode_attention: q [B][Hq][d] float32/bfloat16, out [B][Hq][d]."""
    L = load()
    _cuda("q", q)
    _cuda("Tk_invT", Tk_invT, torch.float32)
    _cuda("cb_k", cb_k, torch.float16)
    _cuda("cb_v", cb_v, torch.float16)
    _cuda("seqlens", seqlens, torch.int32)
    _cuda("out", out)
    _cuda("workspace", workspace, torch.uint8)
    _cuda("dev_err", dev_err, torch.int32)
    _check(L.kvq_vq_decode_attention(_ptr(q), _dt(q), int(q.shape[1]), _ptr(Tk_invT),
                                     _ptr(cb_k), _ptr(cb_v), C.byref(cache.desc), _ptr(seqlens),
                                     int(max_seqlen), _ptr(out), _dt(out), _ptr(workspace),
                                     workspace.numel(), _ptr(dev_err), _stream(stream)),
           "kvq_vq_decode_attention")
