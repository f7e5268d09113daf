/*
 * kvq.h -- C ABI of a B200 (sm_100a) library for decode attention over a transformed,
 * percentile-clipped, affine-quantized 2/4-bit KV cache, and for the quantize-append
 * step that fills that cache.
 *
 * The method (WUSH-KV, with AATC and NOVA-KV as related transform-coding work):
 *  - "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms" (paperlayer
 *    summary), section 1 and section 4.2: a dense d x d key transform per KV head is
 *    applied after RoPE to every new key, and each query is compensated with T_k^{-T}
 *    so that query-key products are preserved; a per-KV-head value transform is folded
 *    into the projection weights on a real model (applied explicitly here), so the
 *    attention output stays in the value-transform domain.
 *  - same page, section 5.3 (downstream setup) and the abstract: OSCAR-style
 *    percentile-clipped affine quantization of the transformed cache at 2 bits.
 *  - same page, section 4.1: grouped-query attention; several query heads read one
 *    KV head. Query head hq reads KV head hq / (Hq / Hkv).
 *  - "Spend Bits Where Queries Look" (NOVA-KV project page), "Three requirements",
 *    items 2 and 3: the cache is read at every decode step, and every token occupies
 *    the same number of bits.
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers owned by the caller (allocated, e.g., by
 *    PyTorch). The library allocates no memory and keeps no state between calls; it
 *    is safe to call from several host threads on different streams.
 *  - Work is enqueued on `stream` (NULL = the legacy default stream) and runs
 *    asynchronously; pointers must stay valid until it completes.
 *  - Argument errors are detected on the host before anything is launched and
 *    return a kvq_status other than KVQ_OK. A failed launch returns KVQ_ERR_CUDA.
 *    kvq_last_error() gives a one-line description (thread-local).
 *  - Problems that depend on device data are never fatal: the kernels clamp or skip
 *    and OR a bit into *dev_err (a device int32, nullable): see KVQ_DEVERR_*.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

struct CUstream_st;                        /* the CUDA runtime's cudaStream_t target */
typedef struct CUstream_st *kvq_stream_t;  /* pass a cudaStream_t here */

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,   /* null pointer, inconsistent sizes or parameters */
    KVQ_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels implement */
    KVQ_ERR_CAPACITY = 3,      /* host-known length exceeds the cache capacity */
    KVQ_ERR_WORKSPACE = 4,     /* workspace missing, too small or misaligned */
    KVQ_ERR_CUDA = 5           /* a CUDA launch or query failed */
} kvq_status;

typedef enum { KVQ_F32 = 0, KVQ_BF16 = 1 } kvq_dtype;

/* Bits in *dev_err (device int32, OR-ed, never cleared by the library). */
#define KVQ_DEVERR_SEQLEN_CLAMPED 0x1   /* seqlens[b] < 0 or > max_seqlen: clamped */
#define KVQ_DEVERR_POS_RANGE      0x2   /* pos[b] < 0 or pos[b] + n > T_cap: sequence skipped */
#define KVQ_DEVERR_NONFINITE      0x4   /* a group had a non-finite clip range: codes 0 */
#define KVQ_DEVERR_WAIT_TIMEOUT   0x8   /* a bounded pipeline wait (about 1 s) gave up: the
                                           output is invalid; the warp waited for its own
                                           copies in flight and stopped. For tests of this
                                           path, the environment variable KVQ_TEST_STALL_NS
                                           (read at every decode call) makes each decode warp
                                           first wait that many ns on a barrier nothing
                                           arrives at and then take the same path. */
#define KVQ_DEVERR_PAGE_RANGE     0x10  /* a block-table entry outside [0, num_pages): the
                                           append skips the token, the decode reads page 0 */

/*
 * Quantizer parameters. Two quantizers write the same cache format (x^ = z_h + c s_h):
 *
 * quantizer = KVQ_QUANT_PERCENTILE (0): OSCAR-style percentile-clipped affine quantizer
 * (WUSH-KV summary, section 5.3). For a group of `group` consecutive dims of one token,
 * with kappa = floor(clip_alpha * (group - 1)) computed in double on the host:
 *   lo = x_(kappa), hi = x_(group-1-kappa)          order statistics, 0-indexed ascending
 *   s  = f32(f32(hi - lo) / (2^bits - 1))           IEEE float32 division
 *   s_h = f16_rn(s), z_h = f16_rn(lo)               stored as the pair (s_h, z_h)
 *   c  = clamp(rint(f32(f32(x - z_h) / s_h)), 0, 2^bits - 1), rint ties-to-even;
 *        s_h == 0 gives c = 0 for the whole group.
 * Dequantization is x^ = z_h + c * s_h. Supported: 0 <= kappa <= 8 and 2*kappa < group.
 *
 * quantizer = KVQ_QUANT_QUEST (1): QuEST INT, RMS-based clipped levels (WUSH-KV summary,
 * section 4.3; each token's group of channels quantized on its own). The page gives no
 * constants; this library's reading is a symmetric uniform grid of 2^bits levels whose
 * step is delta_b times the group RMS, delta_b the uniform step of least mean squared
 * error for a unit Gaussian (0.9957 at 2 bits, 0.3352 at 4 bits):
 *   rms = f32(sqrt(sum_j x_j^2 / group))            sum of squares in float64
 *   s   = f32(rms * delta_b),  s_h = f16_rn(s),  z_h = f16_rn(-(2^bits - 1)/2 * s_h)
 *   c   = clamp(rint(f32(f32(x - z_h) / s_h)), 0, 2^bits - 1)  as above.
 * clip_alpha is not used.
 *
 * Supported: bits_k, bits_v in {2, 4}; group divides d and is a multiple of 32.
 */
#define KVQ_QUANT_PERCENTILE 0
#define KVQ_QUANT_QUEST      1
typedef struct {
    int bits_k;
    int bits_v;
    int group;
    float clip_alpha;
    int quantizer;              /* KVQ_QUANT_PERCENTILE or KVQ_QUANT_QUEST */
} kvq_qparams;

/*
 * Quantized cache (fixed width per token). Four caller-owned device planes:
 *  k_codes [B][Hkv][T_cap][d*bits_k/8] bytes: one row per token, element j at bit
 *          bits_k*j of the row (little-endian bit stream).
 *  v_codes [B][Hkv][T_cap/16][16*d*bits_v/8] bytes: 16-token tiles laid out for the
 *          P.V contraction. Tile = 32 lane chunks of d*bits_v/16 bytes; chunk L holds
 *          tokens {t, t+4, t+8, t+12} (t = L % 4) at dims {8n + L/4}; inside it,
 *          32-bit little-endian words, word p*W + r (W = d*bits_v/128, p = 0, 1)
 *          holding token t+4p in its low 16 bits and token t+4p+8 in its high 16
 *          bits, dim 8*(E*r + s) + L/4 at bit offset bits_v*s of the half (E = 16/bits_v).
 *          Each token owns whole bytes, so single-token appends need no read-modify-write.
 *  k_sz, v_sz [B][Hkv][T_cap][d/group] pairs of float16 (s_h, z_h), s_h first (4 bytes).
 * T_cap must be a multiple of 64; d must be 64 or 128. All planes 16-byte aligned.
 * qp must equal the parameters passed to kvq_quantize_append.
 *
 * Paged layout (optional; the serving layout of a block table, NOVA-KV page, "Three
 * requirements", item 3: fixed-width tokens make pages of equal size). With
 * block_table != NULL the planes are pools of num_pages pages of page_tokens positions:
 *  k_codes [num_pages][Hkv][page_tokens][d*bits_k/8], v_codes [num_pages][Hkv]
 *  [page_tokens/16][16*d*bits_v/8], k_sz, v_sz [num_pages][Hkv][page_tokens][d/group],
 * each page holding every KV head of page_tokens consecutive positions of one sequence.
 * block_table is device int32 [B][T_cap/page_tokens]: position t of sequence b lives in
 * page block_table[b][t / page_tokens] at slot t % page_tokens. page_tokens must be a
 * multiple of 64 dividing T_cap; T_cap is the per-sequence capacity. The table is read
 * on the device at every call (it may change between calls); an entry outside
 * [0, num_pages) sets KVQ_DEVERR_PAGE_RANGE. block_table == NULL: contiguous planes as
 * above, page_tokens and num_pages ignored.
 */
typedef struct {
    int B;
    int Hkv;
    int T_cap;
    int d;
    kvq_qparams qp;
    void *k_codes;
    void *k_sz;
    void *v_codes;
    void *v_sz;
    const int32_t *block_table; /* NULL = contiguous; else device [B][T_cap/page_tokens] */
    int page_tokens;            /* paged: positions per page, a multiple of 64 */
    int num_pages;              /* paged: pages in each pool plane */
} kvq_cache;

/* Size in bytes of plane `which` (0 k_codes, 1 k_sz, 2 v_codes, 3 v_sz); 0 if invalid.
 * Paged caches: the size of the page pool (num_pages pages). */
KVQ_API size_t kvq_cache_plane_bytes(const kvq_cache *cache, int which);

/*
 * Write path: transform, clip, quantize and append n new tokens per sequence.
 * (WUSH-KV summary, section 4.2: key transform after RoPE, value transform; section 5.3:
 * percentile-clipped affine quantizer; NOVA-KV page, item 3: fixed-width store.)
 *   k_post_rope, v: [B][n][Hkv][d] in_dtype (float32 or bfloat16), post-RoPE keys and values.
 *   T_k, T_v: [Hkv][d][d] float32 row-major, x~_i = sum_j T[i][j] x_j; NULL = identity.
 *   qp: must equal cache->qp.  pos: device int32 [B], first position written per sequence.
 *   n >= 0 tokens per sequence (n == 0 is a no-op). Token i of sequence b goes to position
 *   pos[b] + i; a sequence whose range leaves [0, T_cap) is skipped and flagged in dev_err.
 * The transformed values are computed in float32 (fused multiply-add); for identical
 * transformed inputs the codes, scales and zero-points equal the float64 definition
 * above bit for bit.
 */
KVQ_API kvq_status kvq_quantize_append(const void *k_post_rope, const void *v, kvq_dtype in_dtype,
                               const float *T_k, const float *T_v, const kvq_qparams *qp,
                               kvq_cache *cache, const int32_t *pos, int n, int32_t *dev_err,
                               kvq_stream_t stream);

/* Workspace bytes kvq_decode_attention needs for this cache shape, Hq query heads and
 * sequences of at most max_seqlen tokens (0 if the arguments are invalid). The size never
 * decreases as max_seqlen grows, so a workspace sized for T_cap serves every call. */
KVQ_API size_t kvq_decode_workspace_bytes(const kvq_cache *cache, int Hq, int max_seqlen);

/*
 * Read path: one decode step of grouped-query attention over the quantized cache.
 * (WUSH-KV summary, sections 1, 4.1, 4.2; NOVA-KV page, "Three requirements" item 2.)
 *   q: [B][Hq][d] q_dtype (float32 or bfloat16), post-RoPE queries; Hq % Hkv == 0.
 *   Tk_invT: [Hkv][d][d] float32 row-major, M = T_k^{-T}; q~ = M q (NULL = identity).
 *   seqlens: device int32 [B], tokens attended per sequence (0..max_seqlen; positions
 *            [0, seqlens[b]) must hold appended tokens). max_seqlen <= T_cap.
 *   out: [B][Hq][d] out_dtype: softmax_t(q~ . k^_t / sqrt(d)) v^_t, in the value-transform
 *        domain; 0 for an empty sequence.
 *   workspace: device buffer of at least kvq_decode_workspace_bytes(...) bytes,
 *              256-byte aligned, used as scratch (contents need not be initialised).
 * Computed as a split-K flash decode: scores on int8 tensor cores (key codes against q~
 * as per-head 16-bit fixed point, exact int32 accumulation), float32 online softmax, P.V
 * on float16 tensor cores with float32 accumulation, then a merge of the splits.
 * Paged caches (block_table != NULL) are read through the block table.
 */
KVQ_API kvq_status kvq_decode_attention(const void *q, kvq_dtype q_dtype, int Hq, const float *Tk_invT,
                                const kvq_cache *cache, const int32_t *seqlens, int max_seqlen,
                                void *out, kvq_dtype out_dtype, void *workspace,
                                size_t ws_bytes, int32_t *dev_err, kvq_stream_t stream);

/* Workspace bytes kvq_bf16_decode needs (0 if the arguments are invalid). */
KVQ_API size_t kvq_bf16_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int max_seqlen);

/*
 * Uncompressed comparator: the same decode attention over bfloat16 keys and values
 * [B][Hkv][T_cap][d] (no transform, no quantization); q, out [B][Hq][d] bfloat16.
 * d in {64, 128}; T_cap a multiple of 64. Same workspace and error conventions.
 */
KVQ_API kvq_status kvq_bf16_decode(const void *q, int Hq, const void *k, const void *v, int B, int Hkv,
                           int T_cap, int d, const int32_t *seqlens, int max_seqlen, void *out,
                           void *workspace, size_t ws_bytes, int32_t *dev_err,
                           kvq_stream_t stream);

/*
 * Full-precision window (WUSH-KV summary, section 4.4): the first S_sink positions and
 * the newest S_keep positions of a sequence stay in full precision; the positions between
 * are quantized in batches of S_flush. With L positions the quantized middle is
 * [S_sink, S_sink + Q), Q = S_flush * floor(max(0, L - S_sink - S_keep) / S_flush)
 * (the flush runs after every append). The caller keeps:
 *   k_sink, v_sink:     bfloat16 [B][Hkv][S_sink][d], positions 0..S_sink-1 as given;
 *   k_recent, v_recent: bfloat16 [B][Hkv][S_keep + S_flush][d], position t >= S_sink + Q
 *                       at slot t % (S_keep + S_flush), as given (post-RoPE keys);
 *   the quantized cache holding position S_sink + i at cache position i (i < Q), written
 *   by kvq_quantize_append when a batch is flushed.
 * T_v: [Hkv][d][d] float32 (NULL = identity), applied to the full-precision values so
 * that the whole output is in the value-transform domain.
 */
typedef struct {
    int S_sink;
    int S_keep;
    int S_flush;                /* > 0 */
    void *k_sink;               /* read by the decode, written by kvq_window_append */
    void *v_sink;
    void *k_recent;
    void *v_recent;
    const float *T_v;
} kvq_window;

/*
 * Decode with a full-precision window: seqlens[b] = L (all positions of sequence b,
 * L <= max_seqlen); full-precision positions attend with the query as given (q . k,
 * = (T_k^{-T} q) . (T_k k)), quantized ones as in kvq_decode_attention; one softmax over
 * all L positions. q must be bfloat16. The window buffers and T_v must be 16-byte aligned
 * and q 4-byte aligned (KVQ_ERR_INVALID_ARG otherwise). The quantized middle of max_seqlen
 * positions must fit the cache (Q(max_seqlen) <= T_cap); S_sink + S_keep + S_flush <= 2048.
 * Ring slots that hold no window position are never read into the result, whatever their
 * contents. Workspace:
 * kvq_decode_workspace_bytes(cache, Hq, m) for any m >= Q(max_seqlen) (m = T_cap always
 * suffices, as that size never decreases with m). Other arguments and errors as in
 * kvq_decode_attention.
 */
KVQ_API kvq_status kvq_decode_attention_window(const void *q, kvq_dtype q_dtype, int Hq,
                                               const float *Tk_invT, const kvq_cache *cache,
                                               const kvq_window *window,
                                               const int32_t *seqlens, int max_seqlen,
                                               void *out, kvq_dtype out_dtype, void *workspace,
                                               size_t ws_bytes, int32_t *dev_err,
                                               kvq_stream_t stream);

/*
 * Write path with a full-precision window (WUSH-KV summary, section 4.4): append n new
 * tokens to every sequence and quantize the positions that leave the window, so that the
 * state afterwards is the one kvq_decode_attention_window reads for L + n positions.
 *   k_new, v_new: bfloat16 [B][n][Hkv][d], post-RoPE keys and values of positions
 *                 [L_b, L_b + n), L_b = seqlens[b] (device int32 [B], lengths BEFORE the
 *                 call; the library does not update them).
 *   window: S_sink, S_keep, S_flush and the sink / recent-ring buffers (written here);
 *           T_v is not used (the values go through T_v in the quantizer).
 *   T_k, T_v, qp, cache: as in kvq_quantize_append.
 * Per sequence: new positions t < S_sink are copied to the sink; the positions
 * [S_sink + Q(L_b), S_sink + Q(L_b + n)) (Q as above) are transformed, clipped, quantized
 * and written at cache positions [Q(L_b), Q(L_b + n)), each read from the recent ring
 * (t < L_b) or from the new tokens (t >= L_b); the new positions still in the window
 * (t >= S_sink + Q(L_b + n)) are copied to ring slot t % (S_keep + S_flush). The flush
 * reading is the one of the windowed decode: after every append, the oldest S_flush
 * eligible positions are quantized while at least S_flush are eligible. The quantization
 * uses the float32 CUDA-core transform; its codes equal those of kvq_quantize_append on
 * the same tokens through that path (fewer than 256 tokens in one call).
 * A sequence with L_b < 0 or Q(L_b + n) > T_cap is skipped and flagged
 * (KVQ_DEVERR_POS_RANGE). All bf16 buffers 16-byte aligned. n == 0 is a no-op.
 */
KVQ_API kvq_status kvq_window_append(const void *k_new, const void *v_new, kvq_dtype in_dtype,
                                     const float *T_k, const float *T_v, const kvq_qparams *qp,
                                     kvq_cache *cache, const kvq_window *window,
                                     const int32_t *seqlens, int n, int32_t *dev_err,
                                     kvq_stream_t stream);

/*
 * Vector-quantized cache ("Spend Bits Where Queries Look", NOVA-KV project page: keys and
 * values transformed and encoded once on the write path into a fixed-width cache; the
 * read path is a codebook lookup plus one multiply; equal-size codebooks keep every token
 * the same width). This library's reading (the page fixes neither the sub-vector size nor
 * the codebook layout): the d transformed coefficients of a token form d/4 groups of 4
 * consecutive coefficients, each coded by an 8-bit index into a codebook of 256 float16
 * codewords of 4 coefficients (one codebook per KV head for keys, one for values, shared
 * by the groups), and the token carries a float16 gain g, so x^_group = g * C[idx].
 * 2 bits per coefficient plus 16 bits per token (2.125 bits per element at d = 128).
 *  k_idx, v_idx   [B][Hkv][T_cap][d/4] uint8
 *  k_gain, v_gain [B][Hkv][T_cap] float16
 *  codebooks      cb_k, cb_v: [Hkv][256][4] float16 (device), caller-owned like the transforms
 * T_cap a multiple of 64; d 64 or 128; planes 16-byte aligned.
 */
#define KVQ_VQ_DIM  4
#define KVQ_VQ_SIZE 256
typedef struct {
    int B;
    int Hkv;
    int T_cap;
    int d;
    void *k_idx;
    void *k_gain;
    void *v_idx;
    void *v_gain;
} kvq_vq_cache;

/* Size of plane `which` (0 k_idx, 1 k_gain, 2 v_idx, 3 v_gain); 0 if invalid. */
KVQ_API size_t kvq_vq_plane_bytes(const kvq_vq_cache *cache, int which);

/*
 * VQ write path: x~ = T x per KV head (float32), then per token the gain
 * g = f16(f32(sqrt(sum_j x~_j^2 / d))) (sum in float64) and per group of 4 the codeword
 * nearest to the group after scaling by g, in float32 with a fixed operation order (an
 * integer decision, reproduced exactly by the reference): e_m = f32(x~_m - f32(g c_m)),
 * dist = f32(e_0 e_0), dist = fmaf(e_m, e_m, dist) for m = 1..3; the smallest dist wins,
 * ties to the lowest index; g == 0 codes index 0. k, v: [B][n][Hkv][d] float32 or
 * bfloat16; T_k, T_v as kvq_quantize_append (NULL = identity); pos: device int32 [B].
 * Out-of-range sequences are skipped and flagged as in kvq_quantize_append.
 */
KVQ_API kvq_status kvq_vq_append(const void *k, const void *v, kvq_dtype in_dtype,
                                 const float *T_k, const float *T_v, const void *cb_k,
                                 const void *cb_v, kvq_vq_cache *cache, const int32_t *pos,
                                 int n, int32_t *dev_err, kvq_stream_t stream);

/* Workspace bytes kvq_vq_decode_attention needs (0 if the arguments are invalid); never
 * decreases as max_seqlen grows. */
KVQ_API size_t kvq_vq_decode_workspace_bytes(const kvq_vq_cache *cache, int Hq, int max_seqlen);

/*
 * VQ read path: softmax_t(q~ . k^_t / sqrt(d)) v^_t with q~ = Tk_invT q and
 * k^_t = g^K_t C_K[idx], v^_t = g^V_t C_V[idx] (codebook lookup plus one multiply), in the
 * value-transform domain. Codewords are expanded into float16 tiles in shared memory and
 * both contractions run on float16 tensor cores (q~ and the softmax weights as float16
 * hi/lo pairs), float32 online softmax, split-K with the same merge as
 * kvq_decode_attention. Arguments and errors as kvq_decode_attention; G in {4, 8}.
 */
KVQ_API kvq_status kvq_vq_decode_attention(const void *q, kvq_dtype q_dtype, int Hq,
                                           const float *Tk_invT, const void *cb_k,
                                           const void *cb_v, const kvq_vq_cache *cache,
                                           const int32_t *seqlens, int max_seqlen, void *out,
                                           kvq_dtype out_dtype, void *workspace,
                                           size_t ws_bytes, int32_t *dev_err,
                                           kvq_stream_t stream);

/*
 * Allocation-free decode (no counterpart in the paper; an addition for callers that
 * cannot allocate device memory). Same arguments and result as kvq_decode_attention
 * minus the workspace: an inference engine that has reserved nearly all device memory
 * for its own KV pool, or a latency-critical serving loop that forbids cudaMalloc
 * (it synchronises the device), can call this instead. The scratch lives in a fixed
 * array that the library declares in device memory:
 *  - every GPU that loads the library holds KVQ_NOALLOC_SCRATCH_BYTES for it until exit;
 *  - if kvq_decode_workspace_bytes(cache, Hq, max_seqlen) exceeds that size the call
 *    returns KVQ_ERR_WORKSPACE without launching;
 *  - all calls on a device share the array and it keeps the last call's contents (each
 *    call re-initialises what must start at zero); calls whose kernels overlap on the
 *    GPU (e.g. on unordered streams) race on it and must be avoided;
 *  - the first call on each device looks up the array's address (once per device, that
 *    device current); make that first call before any stream capture.
 * No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define KVQ_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
KVQ_API kvq_status kvq_decode_attention_noalloc(const void *q, kvq_dtype q_dtype, int Hq,
                                                const float *Tk_invT, const kvq_cache *cache,
                                                const int32_t *seqlens, int max_seqlen,
                                                void *out, kvq_dtype out_dtype,
                                                int32_t *dev_err, kvq_stream_t stream);

/* Static description of a status code. */
KVQ_API const char *kvq_status_string(kvq_status status);

/* Detail of the last non-OK status returned on this host thread ("" if none). */
KVQ_API const char *kvq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
