"""GPU parity of the QuEST INT quantizer ("WUSH-KV: KV Cache Quantization with
Data-Adaptive Transforms", section 4.3: each token's channels as one group, RMS-based
clipped levels), through the C ABI with kvq_qparams.quantizer = KVQ_QUANT_QUEST:
  * both append paths (float32 CUDA-core, bf16 tensor-core) byte-identical to the oracle
    when both sides quantize the same inputs;
  * end to end with the transforms: at most 0.1% of codes differ, each by +-1, s/z by at
    most one float16 ulp;
  * the decode over a QuEST-quantized cache (same format) against the oracle's attention.
"""
import numpy as np
import pytest
import torch

import decode_attention_post_b200 as kvq
import oracle
from tests import synth
from tests.test_gpu_parity import (DEV, _compare_codes_end_to_end, _inputs, assert_close,
                                   gpu_decode, planes_to_host, t_, upload_cache)

pytestmark = pytest.mark.gpu


def qp_quest(cfg):
    return kvq.QParams(cfg.bits_k, cfg.bits_v, cfg.group, 0.0, kvq.KVQ_QUANT_QUEST)


def gpu_append_quest(cfg, k, v, Tk, Tv, pos, B):
    cache = kvq.KVCache.allocate(B, cfg.Hkv, cfg.T_cap, cfg.d, qp_quest(cfg))
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    kvq.quantize_append(t_(k), t_(v), None if Tk is None else t_(Tk),
                        None if Tv is None else t_(Tv), qp_quest(cfg), cache,
                        t_(np.asarray(pos, np.int32)), dev_err=err)
    torch.cuda.synchronize()
    return cache, int(err.item())


def oracle_append_quest(cfg, k, v, Tk, Tv, pos, B, **kw):
    oc = oracle.Cache(B, cfg.Hkv, cfg.T_cap, cfg.d, cfg.bits_k, cfg.bits_v, cfg.group)
    r = oracle.quantize_append(k, v, Tk, Tv, cfg.bits_k, cfg.bits_v, cfg.group, 0.0, oc, pos,
                               quantizer=1, **kw)
    return oc, r


CASES = [
    # (config, B, n, pos, dtype): float32 path (f32 inputs or short bf16 appends) and the
    # tensor-core path (bf16 chunks of >= 256 tokens with a transform matrix)
    (synth.CONFIGS[0].with_(T_cap=512), 1, 300, [100], "f32"),
    (synth.CONFIGS[1].with_(T_cap=256), 3, 77, [0, 64, 179], "bf16"),
    (synth.CONFIGS[3].with_(T_cap=128), 2, 45, [3, 80], "bf16"),
    (synth.CONFIGS[4].with_(T_cap=512), 2, 300, [0, 126], "bf16"),
    (synth.CONFIGS[1].with_(T_cap=512, bits_k=4, bits_v=4), 2, 280, [7, 200], "bf16"),
]


@pytest.mark.parametrize("cfg,B,n,pos,dtype", CASES)
def test_quest_append_identity_bit_exact(cfg, B, n, pos, dtype):
    """T = I: given as NULL (float32 path) or, for bf16 chunks, as an identity matrix so
    that the tensor-core path runs (bf16 times I is exact)."""
    k, v = _inputs(cfg, B, n, dtype)
    oc, _ = oracle_append_quest(cfg, k, v, None, None, pos, B)
    eye = None
    if dtype == "bf16" and B * n >= 256:
        eye = np.broadcast_to(np.eye(cfg.d, dtype=np.float32), (cfg.Hkv, cfg.d, cfg.d)).copy()
    gc, err = gpu_append_quest(cfg, k, v, eye, eye, pos, B)
    assert err == 0
    for name, a, b in zip(("k_codes", "k_sz", "v_codes", "v_sz"), planes_to_host(gc), oc.planes()):
        assert np.array_equal(a, b.view(np.uint8)), name


@pytest.mark.parametrize("cfg,B,n,pos,dtype", CASES[:3])
def test_quest_append_same_transformed_inputs_bit_exact(cfg, B, n, pos, dtype):
    k, v = _inputs(cfg, B, n, dtype)
    Tk, Tv, _ = synth.transforms(cfg)
    oc, (kt, vt) = oracle_append_quest(cfg, k, v, Tk, Tv, pos, B, return_transformed=True)
    gc, err = gpu_append_quest(cfg, kt, vt, None, None, pos, B)
    assert err == 0
    for name, a, b in zip(("k_codes", "k_sz", "v_codes", "v_sz"), planes_to_host(gc), oc.planes()):
        assert np.array_equal(a, b.view(np.uint8)), name


@pytest.mark.parametrize("cfg,B,n,pos,dtype", CASES)
def test_quest_append_with_transform_end_to_end(cfg, B, n, pos, dtype):
    k, v = _inputs(cfg, B, n, dtype)
    Tk, Tv, _ = synth.transforms(cfg)
    oc, _ = oracle_append_quest(cfg, k, v, Tk, Tv, pos, B)
    gc, err = gpu_append_quest(cfg, k, v, Tk, Tv, pos, B)
    assert err == 0
    frac = _compare_codes_end_to_end(gc, oc, cfg, B, pos, n)
    assert frac <= 1e-3, frac


@pytest.mark.parametrize("ci,T,seql", [(2, 1024, [1024, 333]), (4, 768, [768, 65])])
def test_quest_cache_decode_matches_oracle(ci, T, seql):
    cfg = synth.CONFIGS[ci].with_(T_cap=T)
    B = len(seql)
    k, v = synth.kv_batch(cfg.with_(B=B), 0, T)
    k, v = synth.as_dtype(k, "bf16"), synth.as_dtype(v, "bf16")
    Tk, Tv, Tit = synth.transforms(cfg)
    oc, _ = oracle_append_quest(cfg, k, v, Tk, Tv, [0] * B, B)
    gc = upload_cache(oc, cfg)
    gc = kvq.KVCache(B, cfg.Hkv, T, cfg.d, qp_quest(cfg),
                     (gc.k_codes, gc.k_sz, gc.v_codes, gc.v_sz))
    q = synth.as_dtype(synth.queries(cfg.with_(B=B)), "bf16")
    want = oracle.decode(q, Tit, oc, np.array(seql, np.int32))
    out, err = gpu_decode(cfg, q, Tit, gc, seql)
    assert err == 0
    assert_close(out.cpu().numpy(), want, where=f"quest decode cfg{ci}")
