// Host side of the C ABI declared in include/kvq.h: argument validation, workspace
// sizing, split selection and kernel dispatch. Nothing here allocates device memory.
#include "kvq_common.cuh"
#include "decode_shapes.h"

#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

namespace kvq {

cudaError_t append_launch(const void *k, const void *v, int in_bf16, const float *Tk,
                          const float *Tv, int B, int n, const kvq_cache *c, int kappa,
                          const int32_t *pos, int32_t *dev_err, cudaStream_t st);
cudaError_t window_flush_launch(const void *k_new, const void *v_new, const float *Tk,
                                const float *Tv, int B, int n_new, const kvq_cache *c, int kappa,
                                const void *ring_k, const void *ring_v, const int32_t *len,
                                int S_sink, int S_keep, int S_flush, int32_t *dev_err,
                                cudaStream_t st);
cudaError_t launch_window_store(const void *k_new, const void *v_new, int B, int n, int Hkv,
                                int d, const int32_t *len, int S_sink, int S_keep, int S_flush,
                                int T_cap, void *k_sink, void *v_sink, void *k_ring, void *v_ring,
                                cudaStream_t st);
cudaError_t launch_vq_append(const void *k, const void *v, int in_bf16, const float *Tk,
                             const float *Tv, const void *cb_k, const void *cb_v, int B, int n,
                             const kvq_vq_cache *c, const int32_t *pos, int32_t *dev_err,
                             cudaStream_t st);
int vq_resident_ctas(int d, int G);
cudaError_t launch_bf16_decode(const void *q, int Hq, const void *k, const void *v, int B,
                               int Hkv, int T_cap, int d, const int32_t *seqlens, int max_seqlen,
                               void *out, void *ws, int nsplit, int split_tokens,
                               int32_t *dev_err, cudaStream_t st);

static thread_local char g_last_error[512];

void set_error(const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
}

static bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

static int kappa_of(float alpha, int group)
{
    double k = floor((double)alpha * (double)(group - 1));
    return k < 0 ? 0 : (int)k;
}

// What the append kernels take as their clip parameter: the order-statistic index of the
// percentile quantizer, or kQuestClip for the QuEST INT quantizer.
static int clip_param(const kvq_qparams *qp)
{
    return qp->quantizer == KVQ_QUANT_QUEST ? kQuestClip : kappa_of(qp->clip_alpha, qp->group);
}

static kvq_status check_qparams(const kvq_qparams *qp, int d)
{
    if (!qp)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "qparams is NULL");
    if ((qp->bits_k != 2 && qp->bits_k != 4) || (qp->bits_v != 2 && qp->bits_v != 4))
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "bits_k=%d bits_v=%d: only 2 and 4 are implemented",
                 qp->bits_k, qp->bits_v);
    if (qp->group <= 0 || d % qp->group || qp->group % 32)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "group=%d must divide d=%d and be a multiple of 32",
                 qp->group, d);
    if (qp->quantizer != KVQ_QUANT_PERCENTILE && qp->quantizer != KVQ_QUANT_QUEST)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "quantizer=%d is not KVQ_QUANT_PERCENTILE or KVQ_QUANT_QUEST",
                 qp->quantizer);
    if (qp->quantizer == KVQ_QUANT_QUEST)
        return KVQ_OK;                         // clip_alpha is not used
    if (!(qp->clip_alpha >= 0.f) || !(qp->clip_alpha < 0.5f))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "clip_alpha=%g must be in [0, 0.5)", (double)qp->clip_alpha);
    const int kap = kappa_of(qp->clip_alpha, qp->group);
    if (2 * kap >= qp->group)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "clip index %d leaves no range in a group of %d", kap,
                 qp->group);
    if (kap > 8)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "clip index %d > 8 is not implemented", kap);
    return KVQ_OK;
}

static kvq_status check_cache(const kvq_cache *c)
{
    if (!c)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (c->B <= 0 || c->Hkv <= 0 || c->T_cap <= 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "cache B=%d Hkv=%d T_cap=%d must be positive", c->B, c->Hkv,
                 c->T_cap);
    if (c->T_cap % kCapAlign)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "T_cap=%d must be a multiple of %d", c->T_cap, kCapAlign);
    if (c->d != 64 && c->d != 128)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "d=%d: only 64 and 128 are implemented", c->d);
    kvq_status s = check_qparams(&c->qp, c->d);
    if (s != KVQ_OK)
        return s;
    if (!c->k_codes || !c->k_sz || !c->v_codes || !c->v_sz)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "a cache plane pointer is NULL");
    if (!aligned(c->k_codes, 16) || !aligned(c->k_sz, 16) || !aligned(c->v_codes, 16) ||
        !aligned(c->v_sz, 16))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "cache planes must be 16-byte aligned");
    if (c->block_table) {
        if (c->page_tokens <= 0 || c->page_tokens % kDecodeBlock || c->T_cap % c->page_tokens)
            KVQ_FAIL(KVQ_ERR_INVALID_ARG,
                     "page_tokens=%d must be a positive multiple of %d dividing T_cap=%d",
                     c->page_tokens, kDecodeBlock, c->T_cap);
        if (c->num_pages <= 0)
            KVQ_FAIL(KVQ_ERR_INVALID_ARG, "num_pages=%d must be positive", c->num_pages);
        if (!aligned(c->block_table, 4))
            KVQ_FAIL(KVQ_ERR_INVALID_ARG, "block_table must be 4-byte aligned");
    }
    return KVQ_OK;
}

static bool same_qp(const kvq_qparams *a, const kvq_qparams *b)
{
    return a->bits_k == b->bits_k && a->bits_v == b->bits_v && a->group == b->group &&
           a->quantizer == b->quantizer &&
           (a->quantizer == KVQ_QUANT_QUEST || a->clip_alpha == b->clip_alpha);
}

static int num_sms()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0) {
        cudaGetLastError();
        return 148;
    }
    return sms;
}

// Target number of splits per (sequence, KV head), before clamping to the blocks of the
// sequence. With `resident` CTAs per SM there are slots = SMs * resident places. When
// there are at least two slots per (sequence, KV head) pair, floor(slots / pairs) splits
// fill one wave with long CTAs (the per-CTA prologue, ring fill and merge are paid once
// per split; measured on B200: batch 4 x 128K 0.144 -> 0.096 ms, batch 16 x 16K
// 0.073 -> 0.055 ms against 4 waves). With fewer, about 4 waves: the short last splits of
// ragged sequences then fill the tail (batch 64 x U[12K, 16K]: 5 splits best).
// KVQ_DECODE_SPLITS overrides it (tuning).
static long target_splits(int B, int Hkv, int resident, bool window = false)
{
    const long pairs = (long)B * Hkv;
    const long slots = (long)num_sms() * (resident > 0 ? resident : kDecodeMinBlocks);
    long ns = slots >= 2 * pairs ? slots / pairs : (4 * slots + pairs - 1) / pairs;
    // a windowed decode adds one window split per pair: when the splits fill one wave,
    // leave room in it for the window splits (never more splits than without a window)
    if (window && slots >= 2 * pairs)
        ns = (slots - pairs) / pairs;
    if (const char *e = getenv("KVQ_DECODE_SPLITS"))
        ns = atol(e);
    return ns < 1 ? 1 : ns;
}

static int blocks_of(int max_seqlen)
{
    return max_seqlen > 0 ? (max_seqlen + kDecodeBlock - 1) / kDecodeBlock : 1;
}

// Splits along the tokens; each split is a whole number of 64-token blocks. The count
// is ceil(blocks / ceil(blocks / ns)) with ns = min(target, blocks), which is at most ns;
// it is not monotonic in max_seqlen (75 blocks over 74 target splits give 38 splits).
static int choose_splits(int B, int Hkv, int max_seqlen, int *split_tokens, int resident,
                         bool window = false)
{
    const int blocks = blocks_of(max_seqlen);
    long ns = target_splits(B, Hkv, resident, window);
    if (ns > blocks)
        ns = blocks;
    const int bps = (int)((blocks + ns - 1) / ns);
    *split_tokens = bps * kDecodeBlock;
    return (blocks + bps - 1) / bps;
}

// Split partial slots the workspace holds: min(target, blocks), an upper bound of
// choose_splits that never decreases as max_seqlen grows, so a workspace sized for a
// longer max_seqlen always serves a shorter one.
static int split_slots(int B, int Hkv, int max_seqlen, int resident)
{
    const long ns = target_splits(B, Hkv, resident);
    const int blocks = blocks_of(max_seqlen);
    return (int)(ns < blocks ? ns : blocks);
}

static size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

static DecodeWorkspace decode_layout(int B, int Hkv, int Hq, int d, int nslots)
{
    const int G = Hq / Hkv;
    DecodeWorkspace w;
    size_t off = 0;
    w.qfrag = off;
    off += up256((size_t)B * Hkv * decode_qfrag_words(d, G) * 4);
    w.qscale = off;
    off += up256((size_t)B * Hq * 4);
    w.qw = off;
    off += up256((size_t)B * Hq * 4);
    w.part = off;                              // nslots split slots + 1 window slot
    off += up256((size_t)B * Hkv * (nslots + 1) * G * (d + 2) * 4);
    w.ticket = off;
    off += up256((size_t)B * Hkv * 4);
    w.total = off;
    return w;
}

static kvq_status check_decode_shape(const kvq_cache *c, int Hq, int max_seqlen)
{
    kvq_status s = check_cache(c);
    if (s != KVQ_OK)
        return s;
    if (Hq <= 0 || Hq % c->Hkv)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d", Hq, c->Hkv);
    const int G = Hq / c->Hkv;
    if (G != 4 && G != 8)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "query heads per KV head G=%d: 4 and 8 are implemented", G);
    if (c->qp.group != c->d)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "decode implements group == d (got group=%d, d=%d)",
                 c->qp.group, c->d);
    if (max_seqlen < 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "max_seqlen=%d is negative", max_seqlen);
    if (max_seqlen > c->T_cap)
        KVQ_FAIL(KVQ_ERR_CAPACITY, "max_seqlen=%d exceeds T_cap=%d", max_seqlen, c->T_cap);
    return KVQ_OK;
}

}  // namespace kvq

using namespace kvq;

extern "C" {

const char *kvq_status_string(kvq_status s)
{
    switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "cache capacity exceeded";
    case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case KVQ_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char *kvq_last_error(void) { return g_last_error; }

size_t kvq_cache_plane_bytes(const kvq_cache *c, int which)
{
    if (!c || c->B <= 0 || c->Hkv <= 0 || c->T_cap <= 0 || c->d <= 0 || c->qp.group <= 0 ||
        c->d % c->qp.group)
        return 0;
    size_t tok = (size_t)c->B * c->Hkv * c->T_cap;
    if (c->block_table) {
        if (c->page_tokens <= 0 || c->page_tokens % kDecodeBlock || c->num_pages <= 0)
            return 0;
        tok = (size_t)c->num_pages * c->Hkv * c->page_tokens;
    }
    switch (which) {
    case 0: return tok * c->d * c->qp.bits_k / 8;
    case 1: return tok * (c->d / c->qp.group) * 4;
    case 2: return tok * c->d * c->qp.bits_v / 8;
    case 3: return tok * (c->d / c->qp.group) * 4;
    }
    return 0;
}

kvq_status kvq_quantize_append(const void *k, const void *v, kvq_dtype in_dtype, const float *T_k,
                               const float *T_v, const kvq_qparams *qp, kvq_cache *cache,
                               const int32_t *pos, int n, int32_t *dev_err, kvq_stream_t stream)
{
    g_last_error[0] = 0;
    kvq_status s = check_cache(cache);
    if (s != KVQ_OK)
        return s;
    s = check_qparams(qp, cache->d);
    if (s != KVQ_OK)
        return s;
    if (!same_qp(qp, &cache->qp))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "qparams differ from the cache's qparams");
    if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "in_dtype=%d is not KVQ_F32 or KVQ_BF16", (int)in_dtype);
    if (n < 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "n=%d is negative", n);
    if (n > cache->T_cap)
        KVQ_FAIL(KVQ_ERR_CAPACITY, "n=%d exceeds T_cap=%d", n, cache->T_cap);
    if (n == 0)
        return KVQ_OK;
    if (!k || !v || !pos)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "k, v and pos must not be NULL");
    cudaError_t e = append_launch(k, v, in_dtype == KVQ_BF16, T_k, T_v, cache->B, n, cache,
                                clip_param(qp), pos, dev_err,
                                (cudaStream_t)stream);
    if (e != cudaSuccess)
        KVQ_FAIL(KVQ_ERR_CUDA, "append launch: %s", cudaGetErrorString(e));
    return KVQ_OK;
}

size_t kvq_decode_workspace_bytes(const kvq_cache *c, int Hq, int max_seqlen)
{
    if (check_decode_shape(c, Hq, max_seqlen) != KVQ_OK)
        return 0;
    const int res = decode_resident_ctas(c->d, Hq / c->Hkv, c->qp.bits_k, c->qp.bits_v);
    return decode_layout(c->B, c->Hkv, Hq, c->d, split_slots(c->B, c->Hkv, max_seqlen, res)).total;
}

// Shared by the plain and the windowed decode: argument checks beyond the cache shape,
// workspace carving and launch. `win` (nullable) describes the full-precision window and
// `qmax` is the longest quantized run the cache holds for max_seqlen.
static kvq_status decode_common(const void *q, kvq_dtype q_dtype, int Hq, const float *Tk_invT,
                                const kvq_cache *c, const int32_t *seqlens, int max_seqlen,
                                int qmax, void *out, kvq_dtype out_dtype, void *workspace,
                                size_t ws_bytes, int32_t *dev_err, kvq_stream_t stream,
                                const kvq_window *win)
{
    kvq_status s = check_decode_shape(c, Hq, qmax);
    if (s != KVQ_OK)
        return s;
    if (!q || !seqlens || !out)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "q, seqlens and out must not be NULL");
    if ((q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) ||
        (out_dtype != KVQ_F32 && out_dtype != KVQ_BF16))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "q_dtype/out_dtype must be KVQ_F32 or KVQ_BF16");
    int split_tokens = 0;
    const int res = decode_resident_ctas(c->d, Hq / c->Hkv, c->qp.bits_k, c->qp.bits_v);
    const int ns = choose_splits(c->B, c->Hkv, qmax, &split_tokens, res, win != nullptr);
    const int nslots = split_slots(c->B, c->Hkv, qmax, res);     // >= ns
    const DecodeWorkspace w = decode_layout(c->B, c->Hkv, Hq, c->d, nslots);
    if (!workspace || !aligned(workspace, 256))
        KVQ_FAIL(KVQ_ERR_WORKSPACE, "workspace must be a 256-byte aligned device buffer");
    if (ws_bytes < w.total)
        KVQ_FAIL(KVQ_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, w.total);
    unsigned char *ws = (unsigned char *)workspace;
    DecodeLaunch L;
    L.p.k_codes = (const uint8_t *)c->k_codes;
    L.p.k_sz = (const uint32_t *)c->k_sz;
    L.p.v_codes = (const uint8_t *)c->v_codes;
    L.p.v_sz = (const uint32_t *)c->v_sz;
    L.p.seqlens = seqlens;
    L.p.B = c->B;
    L.p.Hkv = c->Hkv;
    L.p.Hq = Hq;
    L.p.T_cap = c->T_cap;
    L.p.max_seqlen = max_seqlen;
    L.p.nsplit = ns;
    L.p.split_tokens = split_tokens;
    L.p.qfrag = (const uint32_t *)(ws + w.qfrag);
    L.p.qscale = (const float *)(ws + w.qscale);
    L.p.qw = (const float *)(ws + w.qw);
    L.p.part = (float *)(ws + w.part);
    L.p.ticket = (int *)(ws + w.ticket);
    L.p.out = out;
    L.p.out_bf16 = out_dtype == KVQ_BF16;
    L.p.dev_err = dev_err;
    L.p.block_table = c->block_table;
    L.p.page_tokens = c->page_tokens;
    L.p.num_pages = c->num_pages;
    L.p.part_slots = nslots + 1;
    L.p.win_sink = win ? win->S_sink : 0;
    L.p.win_keep = win ? win->S_keep : 0;
    L.p.win_flush = win ? win->S_flush : 0;
    L.p.stall_test_ns = 0;
    if (const char *e = getenv("KVQ_TEST_STALL_NS"))
        L.p.stall_test_ns = atoll(e);
    L.q = q;
    L.q_bf16 = q_dtype == KVQ_BF16;
    L.M = Tk_invT;
    L.d = c->d;
    L.G = Hq / c->Hkv;
    L.bits_k = c->qp.bits_k;
    L.bits_v = c->qp.bits_v;
    L.p.win_q = win ? q : nullptr;
    L.p.k_sink = win ? win->k_sink : nullptr;
    L.p.v_sink = win ? win->v_sink : nullptr;
    L.p.k_recent = win ? win->k_recent : nullptr;
    L.p.v_recent = win ? win->v_recent : nullptr;
    L.p.win_Tv = win ? win->T_v : nullptr;
    cudaError_t e = launch_decode(L, (cudaStream_t)stream);
    if (e != cudaSuccess)
        KVQ_FAIL(KVQ_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return KVQ_OK;
}

kvq_status kvq_decode_attention(const void *q, kvq_dtype q_dtype, int Hq, const float *Tk_invT,
                                const kvq_cache *c, const int32_t *seqlens, int max_seqlen,
                                void *out, kvq_dtype out_dtype, void *workspace, size_t ws_bytes,
                                int32_t *dev_err, kvq_stream_t stream)
{
    g_last_error[0] = 0;
    return decode_common(q, q_dtype, Hq, Tk_invT, c, seqlens, max_seqlen, max_seqlen, out,
                         out_dtype, workspace, ws_bytes, dev_err, stream, nullptr);
}

// Window parameters shared by the windowed decode and the windowed append.
static kvq_status check_window(const kvq_window *win)
{
    if (!win)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "window is NULL");
    if (win->S_sink < 0 || win->S_keep < 0 || win->S_flush <= 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "window S_sink=%d S_keep=%d S_flush=%d: need >= 0, >= 0, > 0",
                 win->S_sink, win->S_keep, win->S_flush);
    if ((long)win->S_sink + win->S_keep + win->S_flush > 2048)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "window of %ld positions: at most 2048 are implemented",
                 (long)win->S_sink + win->S_keep + win->S_flush);
    if ((win->S_sink > 0 && (!win->k_sink || !win->v_sink)) || !win->k_recent || !win->v_recent)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "a window buffer is NULL");
    return KVQ_OK;
}

kvq_status kvq_window_append(const void *k_new, const void *v_new, kvq_dtype in_dtype,
                             const float *T_k, const float *T_v, const kvq_qparams *qp,
                             kvq_cache *cache, const kvq_window *win, const int32_t *seqlens,
                             int n, int32_t *dev_err, kvq_stream_t stream)
{
    g_last_error[0] = 0;
    kvq_status s = check_cache(cache);
    if (s != KVQ_OK)
        return s;
    s = check_qparams(qp, cache->d);
    if (s != KVQ_OK)
        return s;
    if (!same_qp(qp, &cache->qp))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "qparams differ from the cache's qparams");
    s = check_window(win);
    if (s != KVQ_OK)
        return s;
    if (in_dtype != KVQ_BF16)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "the windowed append takes bfloat16 keys and values");
    if (n < 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "n=%d is negative", n);
    if (n == 0)
        return KVQ_OK;
    if (!k_new || !v_new || !seqlens)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "k_new, v_new and seqlens must not be NULL");
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(win->k_recent, 16) ||
        !aligned(win->v_recent, 16) ||
        (win->S_sink > 0 && (!aligned(win->k_sink, 16) || !aligned(win->v_sink, 16))))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "bfloat16 token and window buffers must be 16-byte aligned");
    if ((long)cache->B * n > 0x7fffffffL / 4)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "B * n = %ld new tokens in one call is too many",
                 (long)cache->B * n);
    cudaStream_t st = (cudaStream_t)stream;
    // the flush reads ring slots that the store below may overwrite: flush first
    cudaError_t e = window_flush_launch(k_new, v_new, T_k, T_v, cache->B, n, cache,
                                        clip_param(qp), win->k_recent,
                                        win->v_recent, seqlens, win->S_sink, win->S_keep,
                                        win->S_flush, dev_err, st);
    if (e != cudaSuccess)
        KVQ_FAIL(KVQ_ERR_CUDA, "window flush launch: %s", cudaGetErrorString(e));
    e = launch_window_store(k_new, v_new, cache->B, n, cache->Hkv, cache->d, seqlens,
                            win->S_sink, win->S_keep, win->S_flush, cache->T_cap, win->k_sink,
                            win->v_sink, win->k_recent, win->v_recent, st);
    if (e != cudaSuccess)
        KVQ_FAIL(KVQ_ERR_CUDA, "window store launch: %s", cudaGetErrorString(e));
    return KVQ_OK;
}

kvq_status kvq_decode_attention_window(const void *q, kvq_dtype q_dtype, int Hq,
                                       const float *Tk_invT, const kvq_cache *c,
                                       const kvq_window *win, const int32_t *seqlens,
                                       int max_seqlen, void *out, kvq_dtype out_dtype,
                                       void *workspace, size_t ws_bytes, int32_t *dev_err,
                                       kvq_stream_t stream)
{
    g_last_error[0] = 0;
    kvq_status ws = check_window(win);
    if (ws != KVQ_OK)
        return ws;
    if (q_dtype != KVQ_BF16)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "the windowed decode takes bfloat16 queries");
    if (!aligned(win->k_recent, 16) || !aligned(win->v_recent, 16) ||
        (win->S_sink > 0 && (!aligned(win->k_sink, 16) || !aligned(win->v_sink, 16))) ||
        (win->T_v && !aligned(win->T_v, 16)) || !aligned(q, 4))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG,
                 "window buffers and T_v must be 16-byte aligned, q 4-byte aligned");
    if (max_seqlen < 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "max_seqlen=%d must be >= 0", max_seqlen);
    const int qmax = window_quantized(max_seqlen, win->S_sink, win->S_keep, win->S_flush);
    return decode_common(q, q_dtype, Hq, Tk_invT, c, seqlens, max_seqlen, qmax, out, out_dtype,
                         workspace, ws_bytes, dev_err, stream, win);
}

// ------------------------------------------------------------------ vector-quantized cache

static kvq_status check_vq_cache(const kvq_vq_cache *c)
{
    if (!c)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "cache is NULL");
    if (c->B <= 0 || c->Hkv <= 0 || c->T_cap <= 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "cache B=%d Hkv=%d T_cap=%d must be positive", c->B, c->Hkv,
                 c->T_cap);
    if (c->T_cap % kCapAlign)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "T_cap=%d must be a multiple of %d", c->T_cap, kCapAlign);
    if (c->d != 64 && c->d != 128)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "d=%d: only 64 and 128 are implemented", c->d);
    if (!c->k_idx || !c->k_gain || !c->v_idx || !c->v_gain)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "a cache plane pointer is NULL");
    if (!aligned(c->k_idx, 16) || !aligned(c->k_gain, 16) || !aligned(c->v_idx, 16) ||
        !aligned(c->v_gain, 16))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "cache planes must be 16-byte aligned");
    return KVQ_OK;
}

static kvq_status check_codebooks(const void *cb_k, const void *cb_v)
{
    if (!cb_k || !cb_v)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "codebooks must not be NULL");
    if (!aligned(cb_k, 16) || !aligned(cb_v, 16))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "codebooks must be 16-byte aligned");
    return KVQ_OK;
}

size_t kvq_vq_plane_bytes(const kvq_vq_cache *c, int which)
{
    if (!c || c->B <= 0 || c->Hkv <= 0 || c->T_cap <= 0 || c->d <= 0 || c->d % KVQ_VQ_DIM)
        return 0;
    const size_t tok = (size_t)c->B * c->Hkv * c->T_cap;
    switch (which) {
    case 0:
    case 2: return tok * (c->d / KVQ_VQ_DIM);
    case 1:
    case 3: return tok * 2;
    }
    return 0;
}

kvq_status kvq_vq_append(const void *k, const void *v, kvq_dtype in_dtype, const float *T_k,
                         const float *T_v, const void *cb_k, const void *cb_v,
                         kvq_vq_cache *cache, const int32_t *pos, int n, int32_t *dev_err,
                         kvq_stream_t stream)
{
    g_last_error[0] = 0;
    kvq_status s = check_vq_cache(cache);
    if (s != KVQ_OK)
        return s;
    s = check_codebooks(cb_k, cb_v);
    if (s != KVQ_OK)
        return s;
    if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "in_dtype=%d is not KVQ_F32 or KVQ_BF16", (int)in_dtype);
    if (n < 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "n=%d is negative", n);
    if (n > cache->T_cap)
        KVQ_FAIL(KVQ_ERR_CAPACITY, "n=%d exceeds T_cap=%d", n, cache->T_cap);
    if (n == 0)
        return KVQ_OK;
    if (!k || !v || !pos)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "k, v and pos must not be NULL");
    if ((T_k && !aligned(T_k, 16)) || (T_v && !aligned(T_v, 16)))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "transforms must be 16-byte aligned");
    cudaError_t e = launch_vq_append(k, v, in_dtype == KVQ_BF16, T_k, T_v, cb_k, cb_v, cache->B,
                                     n, cache, pos, dev_err, (cudaStream_t)stream);
    if (e != cudaSuccess)
        KVQ_FAIL(KVQ_ERR_CUDA, "vq append launch: %s", cudaGetErrorString(e));
    return KVQ_OK;
}

// The VQ decode's workspace: the scalar decode's sections (query prologue outputs, split
// partials, tickets) plus q~ itself (float32 [B][Hq][d]) at the end.
static kvq_status vq_shape(const kvq_vq_cache *c, int Hq, int max_seqlen)
{
    kvq_status s = check_vq_cache(c);
    if (s != KVQ_OK)
        return s;
    if (Hq <= 0 || Hq % c->Hkv)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d", Hq, c->Hkv);
    const int G = Hq / c->Hkv;
    if (G != 4 && G != 8)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "query heads per KV head G=%d: 4 and 8 are implemented", G);
    if (max_seqlen < 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "max_seqlen=%d is negative", max_seqlen);
    if (max_seqlen > c->T_cap)
        KVQ_FAIL(KVQ_ERR_CAPACITY, "max_seqlen=%d exceeds T_cap=%d", max_seqlen, c->T_cap);
    return KVQ_OK;
}

static size_t vq_workspace(const kvq_vq_cache *c, int Hq, int max_seqlen, size_t *qt_off)
{
    const DecodeWorkspace w =
        decode_layout(c->B, c->Hkv, Hq, c->d,
                      split_slots(c->B, c->Hkv, max_seqlen, vq_resident_ctas(c->d, Hq / c->Hkv)));
    *qt_off = w.total;
    return w.total + up256((size_t)c->B * Hq * c->d * 4);
}

size_t kvq_vq_decode_workspace_bytes(const kvq_vq_cache *c, int Hq, int max_seqlen)
{
    if (vq_shape(c, Hq, max_seqlen) != KVQ_OK)
        return 0;
    size_t qt_off;
    return vq_workspace(c, Hq, max_seqlen, &qt_off);
}

kvq_status kvq_vq_decode_attention(const void *q, kvq_dtype q_dtype, int Hq, const float *Tk_invT,
                                   const void *cb_k, const void *cb_v, const kvq_vq_cache *c,
                                   const int32_t *seqlens, int max_seqlen, void *out,
                                   kvq_dtype out_dtype, void *workspace, size_t ws_bytes,
                                   int32_t *dev_err, kvq_stream_t stream)
{
    g_last_error[0] = 0;
    kvq_status s = vq_shape(c, Hq, max_seqlen);
    if (s != KVQ_OK)
        return s;
    s = check_codebooks(cb_k, cb_v);
    if (s != KVQ_OK)
        return s;
    if (!q || !seqlens || !out)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "q, seqlens and out must not be NULL");
    if ((q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) ||
        (out_dtype != KVQ_F32 && out_dtype != KVQ_BF16))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "q_dtype/out_dtype must be KVQ_F32 or KVQ_BF16");
    size_t qt_off;
    const size_t need = vq_workspace(c, Hq, max_seqlen, &qt_off);
    if (!workspace || !aligned(workspace, 256))
        KVQ_FAIL(KVQ_ERR_WORKSPACE, "workspace must be a 256-byte aligned device buffer");
    if (ws_bytes < need)
        KVQ_FAIL(KVQ_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
    int split_tokens = 0;
    const int res = vq_resident_ctas(c->d, Hq / c->Hkv);
    const int ns = choose_splits(c->B, c->Hkv, max_seqlen, &split_tokens, res);
    const int nslots = split_slots(c->B, c->Hkv, max_seqlen, res);
    const DecodeWorkspace w = decode_layout(c->B, c->Hkv, Hq, c->d, nslots);
    unsigned char *ws = (unsigned char *)workspace;
    VqLaunch V;
    DecodeLaunch &L = V.L;
    memset(&L.p, 0, sizeof(L.p));
    L.p.seqlens = seqlens;
    L.p.B = c->B;
    L.p.Hkv = c->Hkv;
    L.p.Hq = Hq;
    L.p.T_cap = c->T_cap;
    L.p.max_seqlen = max_seqlen;
    L.p.nsplit = ns;
    L.p.split_tokens = split_tokens;
    L.p.qfrag = (const uint32_t *)(ws + w.qfrag);
    L.p.qscale = (const float *)(ws + w.qscale);
    L.p.qw = (const float *)(ws + w.qw);
    L.p.part = (float *)(ws + w.part);
    L.p.ticket = (int *)(ws + w.ticket);
    L.p.out = out;
    L.p.out_bf16 = out_dtype == KVQ_BF16;
    L.p.dev_err = dev_err;
    L.p.part_slots = nslots + 1;
    L.q = q;
    L.q_bf16 = q_dtype == KVQ_BF16;
    L.M = Tk_invT;
    L.d = c->d;
    L.G = Hq / c->Hkv;
    L.bits_k = 2;
    L.bits_v = 2;
    V.qt = (float *)(ws + qt_off);
    V.k_idx = (const uint8_t *)c->k_idx;
    V.v_idx = (const uint8_t *)c->v_idx;
    V.k_gain = (const uint16_t *)c->k_gain;
    V.v_gain = (const uint16_t *)c->v_gain;
    V.cb_k = (const uint16_t *)cb_k;
    V.cb_v = (const uint16_t *)cb_v;
    cudaError_t e = launch_vq_decode(V, (cudaStream_t)stream);
    if (e != cudaSuccess)
        KVQ_FAIL(KVQ_ERR_CUDA, "vq decode launch: %s", cudaGetErrorString(e));
    return KVQ_OK;
}

size_t kvq_bf16_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int max_seqlen)
{
    if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv || (d != 64 && d != 128) || max_seqlen < 0)
        return 0;
    const int G = Hq / Hkv;
    if (G != 4 && G != 8)
        return 0;
    int split_tokens = 0;
    const int ns = choose_splits(B, Hkv, max_seqlen, &split_tokens, kDecodeMinBlocks);
    return up256((size_t)B * Hkv * ns * G * (d + 2) * 4) + up256((size_t)B * Hkv * 4);
}

kvq_status kvq_bf16_decode(const void *q, int Hq, const void *k, const void *v, int B, int Hkv,
                           int T_cap, int d, const int32_t *seqlens, int max_seqlen, void *out,
                           void *workspace, size_t ws_bytes, int32_t *dev_err, kvq_stream_t stream)
{
    g_last_error[0] = 0;
    if (!q || !k || !v || !seqlens || !out)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "q, k, v, seqlens and out must not be NULL");
    if (B <= 0 || Hkv <= 0 || T_cap <= 0 || Hq <= 0 || Hq % Hkv)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "bad shape B=%d Hq=%d Hkv=%d T_cap=%d", B, Hq, Hkv, T_cap);
    if (T_cap % kCapAlign)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "T_cap=%d must be a multiple of %d", T_cap, kCapAlign);
    if (d != 64 && d != 128)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "d=%d: only 64 and 128 are implemented", d);
    const int G = Hq / Hkv;
    if (G != 4 && G != 8)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "query heads per KV head G=%d: 4 and 8 are implemented", G);
    if (max_seqlen < 0)
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "max_seqlen=%d is negative", max_seqlen);
    if (max_seqlen > T_cap)
        KVQ_FAIL(KVQ_ERR_CAPACITY, "max_seqlen=%d exceeds T_cap=%d", max_seqlen, T_cap);
    if (!aligned(k, 16) || !aligned(v, 16))
        KVQ_FAIL(KVQ_ERR_INVALID_ARG, "k and v must be 16-byte aligned");
    const size_t need = kvq_bf16_decode_workspace_bytes(B, Hq, Hkv, d, max_seqlen);
    if (!workspace || !aligned(workspace, 256))
        KVQ_FAIL(KVQ_ERR_WORKSPACE, "workspace must be a 256-byte aligned device buffer");
    if (ws_bytes < need)
        KVQ_FAIL(KVQ_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
    int split_tokens = 0;
    const int ns = choose_splits(B, Hkv, max_seqlen, &split_tokens, kDecodeMinBlocks);
    cudaError_t e = launch_bf16_decode(q, Hq, k, v, B, Hkv, T_cap, d, seqlens, max_seqlen, out,
                                       workspace, ns, split_tokens, dev_err, (cudaStream_t)stream);
    if (e != cudaSuccess)
        KVQ_FAIL(KVQ_ERR_CUDA, "bf16 decode launch: %s", cudaGetErrorString(e));
    return KVQ_OK;
}

}  // extern "C"
