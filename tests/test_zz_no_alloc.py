"""The allocation-free decode entry point, through the C ABI.

For callers that cannot allocate device memory (an engine owning all of it, or a hot
loop that forbids cudaMalloc), kvq_decode_attention_noalloc uses a fixed scratch array
declared by the library. This test checks it against kvq_decode_attention with a
caller workspace on two calls in a row (the second after the first left its scratch
contents behind), and that a shape needing more scratch than the array holds is
rejected before launching. The file name makes pytest collect it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import decode_attention_post_b200 as kvq
from decode_attention_post_b200 import kvq as K
from tests import synth

pytestmark = pytest.mark.gpu

REL_L2, MAX_ABS = 1e-3, 5e-3


def _setup(cfg, B, seed):
    qp = kvq.QParams(cfg.bits_k, cfg.bits_v, cfg.group, cfg.clip_alpha)
    cache = kvq.KVCache.allocate(B, cfg.Hkv, cfg.T_cap, cfg.d, qp)
    k, v = synth.kv_batch(cfg.with_(B=B), 0, cfg.T_cap)
    Tk, Tv, Tit = synth.transforms(cfg)
    g = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    kvq.quantize_append(g(k).bfloat16(), g(v).bfloat16(), g(Tk), g(Tv), qp, cache,
                        torch.zeros(B, dtype=torch.int32, device="cuda"))
    rng = np.random.default_rng(seed)
    q = g(rng.standard_normal((B, cfg.Hq, cfg.d)).astype(np.float32)).bfloat16()
    seql = g(rng.integers(1, cfg.T_cap + 1, size=B).astype(np.int32))
    return cache, q, g(Tit), seql


def _reference(cache, q, M, seql, T_cap):
    ws = torch.empty(kvq.decode_workspace_bytes(cache, q.shape[1], T_cap), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    kvq.decode_attention(q, M, cache, seql, T_cap, out, ws)
    return out


def _noalloc_via_c_abi(cache, q, M, seql, T_cap):
    L = K.load()
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.kvq_decode_attention_noalloc(
        C.c_void_p(q.data_ptr()), K.KVQ_BF16, q.shape[1], C.c_void_p(M.data_ptr()),
        C.byref(cache.desc), C.c_void_p(seql.data_ptr()), T_cap, C.c_void_p(out.data_ptr()),
        K.KVQ_F32, C.c_void_p(err.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, L.kvq_last_error()
    torch.cuda.synchronize()
    assert err.item() == 0
    return out


def _close(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    rl2 = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rl2 <= REL_L2 and np.abs(a - b).max() <= MAX_ABS, rl2


def test_noalloc_matches_workspace_entry_point_twice():
    cfg = synth.CONFIGS[1].with_(T_cap=512)
    cache, q, M, seql = _setup(cfg, 3, seed=1)
    for call in range(2):                       # second call reuses stale scratch
        if call == 1:
            q = torch.flip(q, dims=[1]).contiguous()
            seql = torch.clamp(seql - 37, min=0)
        want = _reference(cache, q, M, seql, cfg.T_cap)
        got = _noalloc_via_c_abi(cache, q, M, seql, cfg.T_cap)
        _close(got, want)


def test_noalloc_other_shape_after_first():
    cfg = synth.CONFIGS[4].with_(T_cap=256)     # GQA 8, head_dim 64
    cache, q, M, seql = _setup(cfg, 2, seed=2)
    want = _reference(cache, q, M, seql, cfg.T_cap)
    got = _noalloc_via_c_abi(cache, q, M, seql, cfg.T_cap)
    _close(got, want)


def test_noalloc_rejects_scratch_beyond_maximum():
    L = K.load()
    qp = kvq.QParams()
    big = kvq.KVCache.allocate(256, 8, 64, 128, qp)       # tiny planes, many pairs
    need = kvq.decode_workspace_bytes(big, 32, 64)
    assert need > kvq.kvq.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((256, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((256, 32, 128), dtype=torch.bfloat16, device="cuda")
    seql = torch.full((256,), 64, dtype=torch.int32, device="cuda")
    st = L.kvq_decode_attention_noalloc(
        C.c_void_p(q.data_ptr()), K.KVQ_BF16, 32, None, C.byref(big.desc),
        C.c_void_p(seql.data_ptr()), 64, C.c_void_p(out.data_ptr()), K.KVQ_BF16, None, None)
    assert st == 4                                        # KVQ_ERR_WORKSPACE, nothing launched
    assert b"scratch" in L.kvq_last_error()
