"""GPU parity of the vector-quantized cache ("Spend Bits Where Queries Look", NOVA-KV
project page: codebook lookup plus one multiply on the read path), through the C ABI:
  * kvq_vq_append: indices and gains identical to the oracle's when both sides code the
    same transformed inputs (the nearest-codeword rule is float32 with a fixed order);
    end to end with the transforms at most 0.1% of the indices differ and gains by at
    most one float16 ulp;
  * kvq_vq_decode_attention over the oracle's VQ cache against the oracle's attention:
    relative L2 <= 1e-3, max-abs <= 5e-3 (float32 output), bf16 output = rn(float32).
"""
import numpy as np
import pytest
import torch

import decode_attention_post_b200 as kvq
import oracle
from tests import synth
from tests.test_gpu_parity import DEV, assert_bf16_output, assert_close, t_

pytestmark = pytest.mark.gpu


def f16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.float16)).to(DEV)


def upload_vq(oc):
    gc = kvq.VQCache.allocate(oc.B, oc.Hkv, oc.T_cap, oc.d)
    for dst, src in zip((gc.k_idx, gc.k_gain, gc.v_idx, gc.v_gain), oc.planes()):
        dst.copy_(torch.from_numpy(src.view(np.uint8)))
    return gc


def gpu_vq_append(cfg, k, v, Tk, Tv, pos, B):
    cb_k, cb_v = synth.codebooks(cfg)
    gc = kvq.VQCache.allocate(B, cfg.Hkv, cfg.T_cap, cfg.d)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    kvq.vq_append(t_(k), t_(v), None if Tk is None else t_(Tk), None if Tv is None else t_(Tv),
                  f16_dev(cb_k), f16_dev(cb_v), gc, t_(np.asarray(pos, np.int32)), dev_err=err)
    torch.cuda.synchronize()
    return gc, int(err.item())


def host(gc):
    return [p.cpu().numpy() for p in (gc.k_idx, gc.k_gain, gc.v_idx, gc.v_gain)]


APPEND = [
    (synth.CONFIGS[0].with_(T_cap=256), 1, 200, [17], "f32"),
    (synth.CONFIGS[2].with_(T_cap=128), 3, 40, [0, 64, 88], "bf16"),
    (synth.CONFIGS[4].with_(T_cap=128), 2, 70, [5, 50], "bf16"),
]


@pytest.mark.parametrize("cfg,B,n,pos,dtype", APPEND)
def test_vq_append_same_inputs_bit_exact(cfg, B, n, pos, dtype):
    k, v = synth.kv_batch(cfg.with_(B=B), 0, n)
    k, v = synth.as_dtype(k, dtype), synth.as_dtype(v, dtype)
    Tk, Tv, _ = synth.transforms(cfg)
    cb_k, cb_v = synth.codebooks(cfg)
    # identity transform on both sides
    oc = oracle.VQCache(B, cfg.Hkv, cfg.T_cap, cfg.d)
    oracle.vq_append(k, v, None, None, cb_k, cb_v, oc, pos)
    gc, err = gpu_vq_append(cfg, k, v, None, None, pos, B)
    assert err == 0
    for name, a, b in zip(("k_idx", "k_gain", "v_idx", "v_gain"), host(gc), oc.planes()):
        assert np.array_equal(a, b.view(np.uint8)), name
    # the oracle's float32 transformed tokens coded by both
    oc2 = oracle.VQCache(B, cfg.Hkv, cfg.T_cap, cfg.d)
    kt, vt = oracle.vq_append(k, v, Tk, Tv, cb_k, cb_v, oc2, pos, return_transformed=True)
    gc2, err = gpu_vq_append(cfg, kt, vt, None, None, pos, B)
    assert err == 0
    for name, a, b in zip(("k_idx", "k_gain", "v_idx", "v_gain"), host(gc2), oc2.planes()):
        assert np.array_equal(a, b.view(np.uint8)), name


@pytest.mark.parametrize("cfg,B,n,pos,dtype", APPEND)
def test_vq_append_end_to_end(cfg, B, n, pos, dtype):
    k, v = synth.kv_batch(cfg.with_(B=B), 0, n)
    k, v = synth.as_dtype(k, dtype), synth.as_dtype(v, dtype)
    Tk, Tv, _ = synth.transforms(cfg)
    cb_k, cb_v = synth.codebooks(cfg)
    oc = oracle.VQCache(B, cfg.Hkv, cfg.T_cap, cfg.d)
    oracle.vq_append(k, v, Tk, Tv, cb_k, cb_v, oc, pos)
    gc, err = gpu_vq_append(cfg, k, v, Tk, Tv, pos, B)
    assert err == 0
    g = host(gc)
    diff = total = 0
    for a, b in ((g[0], oc.k_idx), (g[2], oc.v_idx)):
        diff += np.count_nonzero(a != b)
        total += a.size
    assert diff <= 1e-3 * total, diff / total
    for a, b in ((g[1], oc.k_gain), (g[3], oc.v_gain)):
        assert np.abs(a.view(np.uint16).astype(np.int32) - b.astype(np.int32)).max() <= 1


def gpu_vq_decode(cfg, q, M, gc, seql, out_dtype=torch.float32, mx=None):
    cb_k, cb_v = synth.codebooks(cfg)
    B, Hq = q.shape[0], q.shape[1]
    mx = int(max(seql)) if mx is None else mx
    ws = torch.empty(kvq.vq_decode_workspace_bytes(gc, Hq, mx), dtype=torch.uint8, device=DEV)
    out = torch.empty((B, Hq, cfg.d), dtype=out_dtype, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    kvq.vq_decode_attention(t_(q), None if M is None else t_(M), f16_dev(cb_k), f16_dev(cb_v),
                            gc, t_(np.asarray(seql, np.int32)), mx, out, ws, dev_err=err)
    torch.cuda.synchronize()
    return out, int(err.item())


def oracle_vq_cache(cfg, B, T):
    k, v = synth.kv_batch(cfg.with_(B=B), 0, T)
    k, v = synth.as_dtype(k, "bf16"), synth.as_dtype(v, "bf16")
    Tk, Tv, Tit = synth.transforms(cfg)
    cb_k, cb_v = synth.codebooks(cfg)
    oc = oracle.VQCache(B, cfg.Hkv, cfg.T_cap, cfg.d)
    oracle.vq_append(k, v, Tk, Tv, cb_k, cb_v, oc, [0] * B)
    return oc, Tit, cb_k, cb_v


DECODE = [
    ("gqa4-d128", synth.CONFIGS[2].with_(T_cap=1024), [1024, 333, 1]),
    ("gqa8-d64", synth.CONFIGS[4].with_(T_cap=768), [768, 65]),
    ("gqa8-d128", synth.CONFIGS[1].with_(T_cap=512, Hq=64), [512, 63]),
    ("gqa4-d64", synth.CONFIGS[4].with_(T_cap=256, Hq=32), [256, 129, 0]),
]


@pytest.mark.parametrize("name,cfg,seql", DECODE, ids=[c[0] for c in DECODE])
def test_vq_decode_matches_oracle(name, cfg, seql):
    B = len(seql)
    oc, Tit, cb_k, cb_v = oracle_vq_cache(cfg, B, cfg.T_cap)
    gc = upload_vq(oc)
    q = synth.as_dtype(synth.queries(cfg.with_(B=B)), "bf16")
    want = oracle.vq_decode(q, Tit, cb_k, cb_v, oc, np.array(seql, np.int32))
    out, err = gpu_vq_decode(cfg, q, Tit, gc, seql)
    assert err == 0
    got = out.cpu().numpy()
    for b, L in enumerate(seql):
        if L == 0:
            assert not got[b].any()
    assert_close(got, want, where=name)
    out16, _ = gpu_vq_decode(cfg, q, Tit, gc, seql, out_dtype=torch.bfloat16)
    assert_bf16_output(out16, out, want, where=name)


@pytest.mark.parametrize("splits", ["1", "3", "50"])
def test_vq_decode_split_invariance(splits, monkeypatch):
    cfg = synth.CONFIGS[2].with_(T_cap=1024)
    oc, Tit, cb_k, cb_v = oracle_vq_cache(cfg, 2, 1024)
    gc = upload_vq(oc)
    q = synth.as_dtype(synth.queries(cfg.with_(B=2)), "bf16")
    seql = [1024, 700]
    want = oracle.vq_decode(q, Tit, cb_k, cb_v, oc, np.array(seql, np.int32))
    monkeypatch.setenv("KVQ_DECODE_SPLITS", splits)
    out, err = gpu_vq_decode(cfg, q, Tit, gc, seql)
    assert err == 0
    assert_close(out.cpu().numpy(), want, where=f"vq splits={splits}")


def test_vq_decode_full_size_sampled():
    """The batch-64 / 12K-16K shape in the bench's launch configuration over random indices
    and gains; the oracle on sampled (sequence, head) outputs."""
    cfg = synth.CONFIGS[2]
    B, Hkv, d, T = cfg.B, cfg.Hkv, cfg.d, cfg.T_cap
    seql = synth.seqlens(cfg)
    oc = oracle.VQCache(B, Hkv, T, d)
    ki_all = oc.k_idx.reshape(B, Hkv, T, d // 4)
    vi_all = oc.v_idx.reshape(B, Hkv, T, d // 4)
    kg_all = oc.k_gain.reshape(B, Hkv, T)
    vg_all = oc.v_gain.reshape(B, Hkv, T)
    for b in range(B):
        n = int(seql[b])
        ki, kg, vi, vg = synth.random_vq_planes(cfg, b, n)
        ki_all[b, :, :n], kg_all[b, :, :n], vi_all[b, :, :n], vg_all[b, :, :n] = ki, kg, vi, vg
    gc = upload_vq(oc)
    q = synth.as_dtype(synth.queries(cfg), "bf16")
    _, _, Tit = synth.transforms(cfg)
    cb_k, cb_v = synth.codebooks(cfg)
    out, err = gpu_vq_decode(cfg, q, Tit, gc, seql, mx=T)
    assert err == 0
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    rng = np.random.default_rng(2)
    sel = np.stack([rng.integers(0, B, 10), rng.integers(0, cfg.Hq, 10)], 1).astype(np.int32)
    sel[0] = [0, 0]
    sel[1] = [B - 1, cfg.Hq - 1]
    sel = np.unique(sel, axis=0)
    want = oracle.vq_decode(q, Tit, cb_k, cb_v, oc, seql, sel=sel)
    for b, h in sel:
        assert_close(got[b, h], want[b, h], where=f"vq full size b{b} h{h}")
