// Write path: per-KV-head transform, percentile clipping, affine quantization and
// fixed-width store of new tokens ("WUSH-KV: KV Cache Quantization with Data-Adaptive
// Transforms", sections 4.2 and 5.3; "Spend Bits Where Queries Look", "Three
// requirements", item 3).
//
// CUDA-core float32 path. One CTA owns one KV head and one of {K, V} and walks tiles
// of 32 tokens of the flattened (sequence, new token) list:
//   1. T_h is staged transposed (row stride d+1, conflict-free) in shared memory once
//      per CTA; the tile's inputs are staged as float32.
//   2. Each warp transforms 4 tokens: lane l owns output dims l + 32r, so the d x d
//      product is register-tiled 4 tokens x d/32 dims with fused multiply-add.
//   3. Per group, the order statistics x_(kappa) and x_(g-1-kappa) come from kappa+1
//      rounds of a warp-wide min (max) with removal of one instance (exact, ties safe);
//      for the QuEST INT quantizer, the group RMS from a float64 sum of squares.
//   4. Scale and zero-point use IEEE float32 division (__fdiv_rn); codes use the
//      correctly rounded quotient from a reciprocal and one correction, ties to even, so
//      they match the definition bit for bit.
//   5. Codes are packed in registers by OR-reductions over lanes and written as whole
//      32-bit words (K rows) or whole 16-bit halves (V tiles); every token owns whole
//      bytes, so no read-modify-write is needed even for single-token appends. The
//      token slot comes from the contiguous layout or, for a paged cache, the block table.
#include "kvq_common.cuh"
#include "kvq_ptx.cuh"

#include <stdlib.h>

namespace kvq {

namespace {

constexpr int kAppendThreads = 256;
constexpr int kAppendWarps = kAppendThreads / 32;

// TPW tokens per warp: 4 for bulk appends (register tiling amortises the T reads),
// 1 for small ones (decode-time appends), so that more warps share the work.
template <int D, int TPW>
struct AppendSmem {
    static constexpr int kTokPerTile = kAppendWarps * TPW;
    float Tt[D * (D + 1)];          // Tt[j*(D+1) + i] = T[i][j]
    float X[kTokPerTile][D];
};

// kappa+1 rounds of "take the warp-wide extreme and remove one instance".
// vals: this lane's NV values of the group; returns the kappa-th smallest (MAX=false)
// or kappa-th largest (MAX=true) of the 32*NV values.
template <int NV, bool MAX>
__device__ __forceinline__ float order_stat(const float (&vals)[NV], int kappa, int lane)
{
    uint32_t removed = 0;
    float m = 0.f;
    for (int it = 0; it <= kappa; ++it) {
        float best = MAX ? -INFINITY : INFINITY;
        int bi = -1;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            if (removed & (1u << i))
                continue;
            float x = vals[i];
            bool better = MAX ? (x > best) : (x < best);
            if (bi < 0 || better) {
                best = x;
                bi = i;
            }
        }
        m = best;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            float o = __shfl_xor_sync(0xffffffffu, m, off);
            m = MAX ? fmaxf(m, o) : fminf(m, o);
        }
        uint32_t holders = __ballot_sync(0xffffffffu, bi >= 0 && best == m);
        if (holders == 0)                       // only non-finite values left
            break;
        if (lane == __ffs(holders) - 1)
            removed |= 1u << bi;
    }
    return m;
}

// Where flattened token (b, i) of the call comes from and goes to.
//  plain append (ring_k == nullptr): input row (b, i) of in[B][n][Hkv][D], written at cache
//    position pos[b] + i; the sequence is out of range unless 0 <= pos[b], pos[b] + n <= T_cap.
//  window flush (kvq_window_append, WUSH-KV section 4.4): sequence b had len[b] positions
//    and receives n_new more; the call quantizes the positions that leave the
//    full-precision window, [S_sink + Q(len), S_sink + Q(len + n_new)) with Q the
//    quantized-middle length, i.e. i < Q(len + n_new) - Q(len) (larger i: nothing to do).
//    Position t = S_sink + Q(len) + i comes from the recent ring (slot t % R of
//    ring[B][Hkv][R][D]) when t < len, else from the new tokens (row t - len of
//    in[B][n_new][Hkv][D]); it is written at cache position Q(len) + i. Out of range
//    unless Q(len + n_new) <= T_cap.
struct TokenMap {
    const void *ring_k, *ring_v;
    const int32_t *len;
    int S_sink, S_keep, S_flush, R, n_new;
};

struct TokenSlot {
    bool active;        // the token is written by this call
    bool bad_range;     // its sequence is out of range (flagged once, skipped)
    int first;          // i == 0 of its sequence
    size_t src;         // element offset of its input row
    const void *base;   // buffer holding the row
    int dst;            // cache position
};

__device__ __forceinline__ TokenSlot token_slot(const TokenMap &tm, const void *in, int which,
                                                const int32_t *pos, int b, int i, int n, int h,
                                                int Hkv, int D, int T_cap)
{
    TokenSlot ts;
    ts.first = i == 0;
    if (!tm.ring_k) {
        const int p0 = pos[b];
        ts.bad_range = p0 < 0 || (long)p0 + n > T_cap;
        ts.active = !ts.bad_range;
        ts.base = in;
        ts.src = (((size_t)b * n + i) * Hkv + h) * D;
        ts.dst = p0 + i;
        return ts;
    }
    const int L = tm.len[b];
    const int qo = L < 0 ? 0 : window_quantized(L, tm.S_sink, tm.S_keep, tm.S_flush);
    const int qn = L < 0 ? 0 : window_quantized(L + tm.n_new, tm.S_sink, tm.S_keep, tm.S_flush);
    ts.bad_range = L < 0 || qn > T_cap;
    ts.active = !ts.bad_range && i < qn - qo;
    const int t = tm.S_sink + qo + i;
    if (t < L) {
        ts.base = which ? tm.ring_v : tm.ring_k;
        ts.src = (((size_t)b * Hkv + h) * tm.R + t % tm.R) * D;
    } else {
        ts.base = in;
        ts.src = (((size_t)b * tm.n_new + (t - L)) * Hkv + h) * D;
    }
    ts.dst = qo + i;
    return ts;
}

// Quantize one token held by a warp (lane l holds dims l + 32 r in vals[r]) and store it
// at cache row `row`: per group the clip range (order statistics, or the RMS for the QuEST
// INT quantizer, kappa == kQuestClip), the float16 scale and zero-point, and the codes
// c = clamp(rint((x - z) / s), 0, qmax) from the correctly rounded quotient (div_rn: a
// reciprocal and one correction), so the codes are those of the definition bit for bit
// (rint as the float32 addition of 1.5 * 2^23 to the clamped quotient, ties to even). The K row
// (whole 32-bit words) or the token's halves of its V tile are packed in registers by
// OR-reductions over the lanes that share a word or half. bits is 2 or 4.
constexpr float kRoundMagic = 12582912.0f;      // 1.5 * 2^23

template <int D>
__device__ __forceinline__ void quantize_store_token(const float (&vals)[D / 32], int lane,
                                                     int which, int bits, int group, int kappa,
                                                     long long row, uint8_t *k_codes,
                                                     uint32_t *k_sz, uint8_t *v_codes,
                                                     uint32_t *v_sz, int32_t *dev_err)
{
    constexpr int R = D / 32;
    const int ng = D / group;
    const int qmax = (1 << bits) - 1;
    uint32_t cq[R];
#pragma unroll
    for (int r = 0; r < R; ++r)
        cq[r] = 0;
    for (int gr = 0; gr < ng; ++gr) {
        // group gr covers dims [gr*group, (gr+1)*group), i.e. r in [r0, r0+nr);
        // dims outside the group are padded with +-inf so they are never picked.
        const int r0 = gr * group / 32, nr = group / 32;
        __half sh, zh;
        bool finite;
        if (kappa == kQuestClip) {
            // QuEST INT: s = f32(rms * delta_b), z = -(2^b - 1)/2 * s_h; the sum of
            // squares in float64 (each square exact), reduced over the warp
            double ss = 0.0;
#pragma unroll
            for (int r = 0; r < R; ++r)
                if (r >= r0 && r < r0 + nr)
                    ss = fma((double)vals[r], (double)vals[r], ss);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float rms = __double2float_rn(sqrt(ss / (double)group));
            const float s = __fmul_rn(rms, quest_delta(bits));
            sh = __float2half_rn(s);
            zh = __float2half_rn(__fmul_rn(-0.5f * (float)qmax, __half2float(sh)));
            finite = isfinite(s);
        } else {
            float vmin[R], vmax[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const bool ing = r >= r0 && r < r0 + nr;
                vmin[r] = ing ? vals[r] : INFINITY;
                vmax[r] = ing ? vals[r] : -INFINITY;
            }
            const float lo = order_stat<R, false>(vmin, kappa, lane);
            const float hi = order_stat<R, true>(vmax, kappa, lane);
            const float range = __fsub_rn(hi, lo);
            // range / qmax correctly rounded (div_rn; tiny or non-finite ranges, outside
            // its conditions, by IEEE division)
            const float s = (range >= 0x1p-100f && range <= 0x1p+100f)
                                ? div_rn(range, (float)qmax, __frcp_rn((float)qmax))
                                : __fdiv_rn(range, (float)qmax);
            sh = __float2half_rn(s);
            zh = __float2half_rn(lo);
            finite = isfinite(range) && isfinite(s);
        }
        const float sf = __half2float(sh), zf = __half2float(zh);
        if (!finite && lane == 0)
            flag(dev_err, KVQ_DEVERR_NONFINITE);
        const bool zero = !finite || sf == 0.f;
        const float rc = zero ? 0.f : __frcp_rn(sf);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            if (r < r0 || r >= r0 + nr || zero)
                continue;
            // the correctly rounded quotient, clamped, rounded to nearest even
            const float y = fminf(fmaxf(div_rn(__fsub_rn(vals[r], zf), sf, rc), 0.f),
                                  (float)qmax);
            cq[r] = (uint32_t)(__float_as_int(__fadd_rn(y, kRoundMagic)) - 0x4B400000);
        }
        if (lane == 0) {
            uint32_t pair = (uint32_t)__half_as_ushort(sh) |
                            ((uint32_t)__half_as_ushort(zh) << 16);
            (which ? v_sz : k_sz)[row * ng + gr] = pair;
        }
    }
    if (!which) {
        // K row: word (32 r + l) / cpw holds lane l's code r at bit bits * (l % cpw)
        const int cpw = 32 / bits;
        uint32_t w[R];
#pragma unroll
        for (int r = 0; r < R; ++r)
            w[r] = cq[r] << (bits * (lane & (cpw - 1)));
        for (int off = 1; off < cpw; off <<= 1)
#pragma unroll
            for (int r = 0; r < R; ++r)
                w[r] |= __shfl_xor_sync(0xffffffffu, w[r], off);
        if ((lane & (cpw - 1)) == 0) {
            uint32_t *dst = reinterpret_cast<uint32_t *>(k_codes + row * (D * bits / 8));
#pragma unroll
            for (int r = 0; r < R; ++r)
                dst[r * (32 / cpw) + lane / cpw] = w[r];
        }
    } else {
        // V tile half (gq, rr) holds dims gq + 8 (E rr + s2), s2 < E = 16 / bits: lane l's
        // code r is dim l + 32 r, i.e. gq = l % 8, E rr + s2 = 4 r + l / 8, so rr = r / 2
        // (2-bit) or r (4-bit); OR-reduced over the lanes with the same gq
        uint32_t hv[R];
#pragma unroll
        for (int r = 0; r < R; ++r)
            hv[r] = 0;
        if (bits == 2) {
#pragma unroll
            for (int r = 0; r < R; ++r)
                hv[r >> 1] |= cq[r] << (2 * (4 * (r & 1) + (lane >> 3)));
        } else {
#pragma unroll
            for (int r = 0; r < R; ++r)
                hv[r] = cq[r] << (4 * (lane >> 3));
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            hv[r] |= __shfl_xor_sync(0xffffffffu, hv[r], 8);
            hv[r] |= __shfl_xor_sync(0xffffffffu, hv[r], 16);
        }
        if (lane < 8) {
            const int W = D * bits / 128;                // halves per gq: D / (8 E)
            unsigned char *tile_base =
                v_codes + (size_t)(row / kTileTokens) * (kTileTokens * D * bits / 8);
            const int tok = (int)(row % kTileTokens);
#pragma unroll
            for (int rr = 0; rr < R; ++rr)
                if (rr < W)
                    *reinterpret_cast<uint16_t *>(tile_base +
                                                  v_half_offset(D, bits, tok, lane, rr)) =
                        (uint16_t)hv[rr];
        }
    }
}

template <int D, int TPW>
__global__ void __launch_bounds__(kAppendThreads)
append_fp32_kernel(const void *__restrict__ k_in, const void *__restrict__ v_in, int in_bf16,
                   const float *__restrict__ Tk, const float *__restrict__ Tv, int B, int n,
                   int Hkv, int T_cap, int bits_k, int bits_v, int group, int kappa,
                   uint8_t *__restrict__ k_codes, uint32_t *__restrict__ k_sz,
                   uint8_t *__restrict__ v_codes, uint32_t *__restrict__ v_sz,
                   const int32_t *__restrict__ pos, int32_t *dev_err, PageMap pm, TokenMap tm)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ int tile_active;
    using Smem = AppendSmem<D, TPW>;
    constexpr int kTokPerWarp = TPW;
    constexpr int kTokPerTile = Smem::kTokPerTile;
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);

    const int h = blockIdx.y;
    const int which = blockIdx.z;               // 0 = keys, 1 = values
    const void *in = which ? v_in : k_in;
    const float *T = which ? Tv : Tk;
    const int bits = which ? bits_v : bits_k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long total = (long)B * n;
    const long tiles = (total + kTokPerTile - 1) / kTokPerTile;
    constexpr int R = D / 32;                   // dims per lane

    // T_h staged transposed; a window flush stages it only once the CTA meets a tile with
    // work (most CTAs of a decode-time flush have none)
    auto stage_T = [&]() {
        // 16 independent float4 loads in flight per thread, then transposed stores
        const float4 *Th4 = reinterpret_cast<const float4 *>(T + (size_t)h * D * D);
        constexpr int N4 = D * D / 4 / kAppendThreads;
#pragma unroll 16
        for (int it = 0; it < N4; ++it) {
            const int idx4 = threadIdx.x + kAppendThreads * it;
            const float4 v4 = Th4[idx4];
            const int i = (4 * idx4) / D, j = (4 * idx4) % D;
            sm.Tt[(j + 0) * (D + 1) + i] = v4.x;
            sm.Tt[(j + 1) * (D + 1) + i] = v4.y;
            sm.Tt[(j + 2) * (D + 1) + i] = v4.z;
            sm.Tt[(j + 3) * (D + 1) + i] = v4.w;
        }
    };
    bool T_staged = false;
    if (T && !tm.ring_k) {
        stage_T();
        T_staged = true;
    }

    for (long tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const long u0 = tile * kTokPerTile;
        __syncthreads();                        // previous tile's readers are done
        if (tm.ring_k) {
            // window flush: most sequences flush nothing in a call; skip tiles without work
            if (threadIdx.x == 0)
                tile_active = 0;
            __syncthreads();
            if (threadIdx.x < kTokPerTile && u0 + threadIdx.x < total) {
                const long u = u0 + threadIdx.x;
                const TokenSlot ts = token_slot(tm, in, which, pos, (int)(u / n), (int)(u % n), n,
                                                h, Hkv, D, T_cap);
                if (ts.active || (ts.bad_range && ts.first))
                    tile_active = 1;
            }
            __syncthreads();
            if (!tile_active)
                continue;
            if (T && !T_staged) {               // uniform: every thread saw tile_active
                stage_T();
                T_staged = true;
            }
        }
#pragma unroll
        for (int it = 0; it < (kTokPerTile * D + kAppendThreads - 1) / kAppendThreads; ++it) {
            const int idx = threadIdx.x + kAppendThreads * it;
            if (idx >= kTokPerTile * D)
                break;
            const int tk = idx / D, j = idx % D;
            const long u = u0 + tk;
            float x = 0.f;
            if (u < total) {
                const TokenSlot ts = token_slot(tm, in, which, pos, (int)(u / n), (int)(u % n), n,
                                                h, Hkv, D, T_cap);
                if (ts.active)
                    x = load_in(ts.base, in_bf16, ts.src + j);
            }
            sm.X[tk][j] = x;
        }
        __syncthreads();

        // ---- transform: 4 tokens x R dims per lane
        float acc[kTokPerWarp][R];
        const int t0 = warp * kTokPerWarp;
        if (T) {
#pragma unroll
            for (int q = 0; q < kTokPerWarp; ++q)
#pragma unroll
                for (int r = 0; r < R; ++r)
                    acc[q][r] = 0.f;
#pragma unroll 4
            for (int j = 0; j < D; ++j) {
                float tv[R];
#pragma unroll
                for (int r = 0; r < R; ++r)
                    tv[r] = sm.Tt[j * (D + 1) + lane + 32 * r];
#pragma unroll
                for (int q = 0; q < kTokPerWarp; ++q) {
                    float xq = sm.X[t0 + q][j];
#pragma unroll
                    for (int r = 0; r < R; ++r)
                        acc[q][r] = fmaf(tv[r], xq, acc[q][r]);
                }
            }
        } else {
#pragma unroll
            for (int q = 0; q < kTokPerWarp; ++q)
#pragma unroll
                for (int r = 0; r < R; ++r)
                    acc[q][r] = sm.X[t0 + q][lane + 32 * r];
        }

        // ---- quantize and store, one token at a time per warp
#pragma unroll
        for (int q = 0; q < kTokPerWarp; ++q) {
            const long u = u0 + t0 + q;
            if (u >= total)
                break;
            const int b = (int)(u / n), i = (int)(u % n);
            const TokenSlot ts = token_slot(tm, in, which, pos, b, i, n, h, Hkv, D, T_cap);
            if (ts.bad_range) {
                if (ts.first && lane == 0)
                    flag(dev_err, KVQ_DEVERR_POS_RANGE);
                continue;
            }
            if (!ts.active)
                continue;
            const int t = ts.dst;
            const long long row = cache_row(pm, b, h, Hkv, T_cap, t);
            if (row < 0) {
                if (lane == 0)
                    flag(dev_err, KVQ_DEVERR_PAGE_RANGE);
                continue;
            }
            quantize_store_token<D>(acc[q], lane, which, bits, group, kappa, row,
                                    k_codes, k_sz, v_codes, v_sz, dev_err);
        }
    }
}

// ---------------------------------------------------------------- short bf16 appends

// Decode-time appends (a few tokens per sequence, bfloat16, both transforms) and window
// flushes: 16-token tiles, one warp per 8 output dims (D / 8 warps). Warp w computes output
// dims [8w, 8w + 8) of the tile on mma.sync (bf16, float32 accumulate): its fragments of
// T = T_hi + T_lo (two bfloat16 pieces, 16 significant bits) come straight from global
// memory (L2) into registers once per CTA, so no CTA stages the whole transform in shared
// memory. The tile's inputs are staged in shared memory by asynchronous copies issued
// before the transform loads (ldmatrix A operands), the transformed tile goes back to
// shared memory, and each warp quantizes and stores 16 / (D / 8) of its tokens.
constexpr int kSmallTile = 16;

template <int D>
struct SmallCfg {
    static constexpr int WARPS = D / 8;              // 16 at d = 128, 8 at d = 64
    static constexpr int TPW = kSmallTile / WARPS;   // tokens each warp quantizes
    static_assert(kSmallTile % WARPS == 0, "whole tokens per warp");
};

template <int D>
struct SmallSmem {
    static constexpr int XS = D + 8;                 // bf16 per staged input row
    static constexpr int YS = D + 4;                 // float per transformed row
    __nv_bfloat16 X[kSmallTile * XS];
    float Y[kSmallTile * YS];
};

template <int D>
__global__ void __launch_bounds__(SmallCfg<D>::WARPS * 32)
append_small_kernel(const __nv_bfloat16 *__restrict__ k_in, const __nv_bfloat16 *__restrict__ v_in,
                    const float *__restrict__ Tk, const float *__restrict__ Tv, int B, int n,
                    int Hkv, int T_cap, int bits_k, int bits_v, int group, int kappa,
                    uint8_t *__restrict__ k_codes, uint32_t *__restrict__ k_sz,
                    uint8_t *__restrict__ v_codes, uint32_t *__restrict__ v_sz,
                    const int32_t *__restrict__ pos, int32_t *dev_err, PageMap pm, TokenMap tm)
{
    constexpr int NW = SmallCfg<D>::WARPS, NTW = 1;  // one n-tile (8 output dims) per warp
    constexpr int KS = D / 16;
    using Sm = SmallSmem<D>;
    __shared__ __align__(16) Sm sm;
    __shared__ int tile_active;

    const int h = blockIdx.y, which = blockIdx.z;
    const void *in = which ? (const void *)v_in : (const void *)k_in;
    const float *T = (which ? Tv : Tk) + (size_t)h * D * D;
    const int bits = which ? bits_v : bits_k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    // B * n < 2^29 on every path here (short appends, bounded window flushes): 32-bit
    // token indices, so the divisions by n stay 32-bit
    const int total = B * n;
    const int tiles = (total + kSmallTile - 1) / kSmallTile;

    uint32_t bhi[NTW][KS][2], blo[NTW][KS][2];
    bool have_b = false;
    auto load_b = [&]() {
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
            const float *row = T + (size_t)(8 * (warp * NTW + nt) + g) * D;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const float2 f = *reinterpret_cast<const float2 *>(row + 16 * ks + 8 * half + 2 * t);
                    const __nv_bfloat162 hi2 = __floats2bfloat162_rn(f.x, f.y);
                    const float2 hf = __bfloat1622float2(hi2);
                    const __nv_bfloat162 lo2 = __floats2bfloat162_rn(f.x - hf.x, f.y - hf.y);
                    bhi[nt][ks][half] = *reinterpret_cast<const uint32_t *>(&hi2);
                    blo[nt][ks][half] = *reinterpret_cast<const uint32_t *>(&lo2);
                }
        }
        have_b = true;
    };

    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int u0 = tile * kSmallTile;
        __syncthreads();                             // the previous tile's readers are done
        if (tm.ring_k) {
            // window flush: skip tiles without a token to write (most of a decode step)
            if (threadIdx.x == 0)
                tile_active = 0;
            __syncthreads();
            if (threadIdx.x < kSmallTile && u0 + threadIdx.x < total) {
                const int u = u0 + (int)threadIdx.x;
                const TokenSlot ts = token_slot(tm, in, which, pos, u / n, u % n, n,
                                                h, Hkv, D, T_cap);
                if (ts.active || (ts.bad_range && ts.first))
                    tile_active = 1;
            }
            __syncthreads();
            if (!tile_active)
                continue;
        }
        // ---- stage the tile's inputs (16-byte asynchronous copies; inactive rows are zero),
        //      issued before the transform fragments so that both loads are in flight
        for (int c = threadIdx.x; c < kSmallTile * (D / 8); c += NW * 32) {
            const int rr = c / (D / 8), ch = c % (D / 8);
            const int u = u0 + rr;
            const __nv_bfloat16 *src = nullptr;
            if (u < total) {
                const TokenSlot ts = token_slot(tm, in, which, pos, u / n, u % n, n,
                                                h, Hkv, D, T_cap);
                if (ts.active)
                    src = reinterpret_cast<const __nv_bfloat16 *>(ts.base) + ts.src + 8 * ch;
            }
            cp_async16(sm.X + rr * Sm::XS + 8 * ch, src ? (const void *)src : in, src ? 16 : 0);
        }
        cp_async_commit();
        if (!have_b)
            load_b();
        cp_async_wait<0>();
        __syncthreads();
        // ---- X~ = X . (T_hi + T_lo)^T, this warp's output dims
        float acc[NTW][4];
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            uint32_t a[4];
            ldmatrix_x4(a, sm.X + (lane & 15) * Sm::XS + 16 * ks + 8 * (lane >> 4));
#pragma unroll
            for (int nt = 0; nt < NTW; ++nt) {
                mma_bf16(acc[nt], a[0], a[1], a[2], a[3], bhi[nt][ks][0], bhi[nt][ks][1]);
                mma_bf16(acc[nt], a[0], a[1], a[2], a[3], blo[nt][ks][0], blo[nt][ks][1]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
            const int col = 8 * (warp * NTW + nt) + 2 * t;
            *reinterpret_cast<float2 *>(sm.Y + g * Sm::YS + col) = make_float2(acc[nt][0], acc[nt][1]);
            *reinterpret_cast<float2 *>(sm.Y + (g + 8) * Sm::YS + col) =
                make_float2(acc[nt][2], acc[nt][3]);
        }
        __syncthreads();
        // ---- quantize and store: warp w takes tokens TPW w .. TPW w + TPW - 1 of the tile
#pragma unroll
        for (int q = 0; q < SmallCfg<D>::TPW; ++q) {
            const int rr = SmallCfg<D>::TPW * warp + q;
            const int u = u0 + rr;
            if (u >= total)
                break;
            const int b = u / n, i = u % n;
            const TokenSlot ts = token_slot(tm, in, which, pos, b, i, n, h, Hkv, D, T_cap);
            if (ts.bad_range) {
                if (ts.first && lane == 0)
                    flag(dev_err, KVQ_DEVERR_POS_RANGE);
                continue;
            }
            if (!ts.active)
                continue;
            const long long row = cache_row(pm, b, h, Hkv, T_cap, ts.dst);
            if (row < 0) {
                if (lane == 0)
                    flag(dev_err, KVQ_DEVERR_PAGE_RANGE);
                continue;
            }
            float vals[D / 32];
#pragma unroll
            for (int r = 0; r < D / 32; ++r)
                vals[r] = sm.Y[rr * Sm::YS + lane + 32 * r];
            quantize_store_token<D>(vals, lane, which, bits, group, kappa, row,
                                    k_codes, k_sz, v_codes, v_sz, dev_err);
        }
    }
}

template <int D>
cudaError_t launch_append_small(const void *k, const void *v, const float *Tk, const float *Tv,
                                int B, int n, const kvq_cache *c, int kappa, const int32_t *pos,
                                int32_t *dev_err, cudaStream_t st, const TokenMap &tm = TokenMap{})
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long tiles = ((long)B * n + kSmallTile - 1) / kSmallTile;
    // one tile per CTA while that fills the GPU; a flush (most tiles empty) or a long
    // chunk walks the tiles grid-stride with about two CTAs per SM
    long want = (2L * sms + 2L * c->Hkv - 1) / (2L * c->Hkv);
    long gx = tiles;
    if (tm.ring_k || tiles > 4 * want)
        gx = tiles < want ? tiles : want;
    if (gx < 1)
        gx = 1;
    dim3 grid((unsigned)gx, (unsigned)c->Hkv, 2);
    append_small_kernel<D><<<grid, SmallCfg<D>::WARPS * 32, 0, st>>>(
        (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, Tk, Tv, B, n, c->Hkv, c->T_cap,
        c->qp.bits_k, c->qp.bits_v, c->qp.group, kappa, (uint8_t *)c->k_codes, (uint32_t *)c->k_sz,
        (uint8_t *)c->v_codes, (uint32_t *)c->v_sz, pos, dev_err,
        PageMap{c->block_table, c->page_tokens, c->num_pages}, tm);
    return cudaGetLastError();
}

template <int D, int TPW>
cudaError_t launch_append_fp32(const void *k, const void *v, int in_bf16, const float *Tk,
                               const float *Tv, int B, int n, const kvq_cache *c, int kappa,
                               const int32_t *pos, int32_t *dev_err, cudaStream_t st,
                               const TokenMap &tm = TokenMap{})
{
    using Smem = AppendSmem<D, TPW>;
    const size_t smem = sizeof(Smem);
    static int attr_set = 0;                // once per process (before any graph capture)
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(append_fp32_kernel<D, TPW>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        attr_set = 1;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long total = (long)B * n;
    const long tiles = (total + Smem::kTokPerTile - 1) / Smem::kTokPerTile;
    long want = (2L * sms + 2L * c->Hkv - 1) / (2L * c->Hkv);   // ~2 CTAs per SM overall
    if (want < 1)
        want = 1;
    // at least 8 tiles per CTA once the T staging cost matters
    long gx = tiles < want ? tiles : want;
    if (tm.ring_k)                          // window flush: most tiles have no work
        gx = tiles < want * 4 ? tiles : want * 4;
    else if (tiles > want * 8)
        gx = (tiles + 7) / 8 < 65535 ? (tiles + 7) / 8 : 65535;
    dim3 grid((unsigned)gx, (unsigned)c->Hkv, 2);
    append_fp32_kernel<D, TPW><<<grid, kAppendThreads, smem, st>>>(
        k, v, in_bf16, Tk, Tv, B, n, c->Hkv, c->T_cap, c->qp.bits_k, c->qp.bits_v, c->qp.group,
        kappa, (uint8_t *)c->k_codes, (uint32_t *)c->k_sz, (uint8_t *)c->v_codes,
        (uint32_t *)c->v_sz, pos, dev_err, PageMap{c->block_table, c->page_tokens, c->num_pages},
        tm);
    return cudaGetLastError();
}

}  // namespace

// Window flush of kvq_window_append: the positions leaving the full-precision window
// (from the recent ring or the n_new new tokens) through the short tensor-core kernel
// (both transforms given) or the float32 CUDA-core kernel; the flattened list holds
// S_flush * ceil(n_new / S_flush) entries per sequence, the most any sequence can flush
// in one call.
cudaError_t window_flush_launch(const void *k_new, const void *v_new, const float *Tk,
                                const float *Tv, int B, int n_new, const kvq_cache *c, int kappa,
                                const void *ring_k, const void *ring_v, const int32_t *len,
                                int S_sink, int S_keep, int S_flush, int32_t *dev_err,
                                cudaStream_t st)
{
    TokenMap tm;
    tm.ring_k = ring_k;
    tm.ring_v = ring_v;
    tm.len = len;
    tm.S_sink = S_sink;
    tm.S_keep = S_keep;
    tm.S_flush = S_flush;
    tm.R = S_keep + S_flush;
    tm.n_new = n_new;
    const long nmax = (long)S_flush * ((n_new + S_flush - 1) / S_flush);
    if (nmax > 0x7fffffffL / (B > 0 ? B : 1))
        return cudaErrorInvalidValue;
    if (Tk && Tv) {                     // bf16 tokens (ring and new) through the tensor cores
        if (c->d == 64)
            return launch_append_small<64>(k_new, v_new, Tk, Tv, B, (int)nmax, c, kappa, nullptr,
                                           dev_err, st, tm);
        return launch_append_small<128>(k_new, v_new, Tk, Tv, B, (int)nmax, c, kappa, nullptr,
                                        dev_err, st, tm);
    }
    if (c->d == 64)
        return launch_append_fp32<64, 4>(k_new, v_new, 1, Tk, Tv, B, (int)nmax, c, kappa, nullptr,
                                         dev_err, st, tm);
    return launch_append_fp32<128, 4>(k_new, v_new, 1, Tk, Tv, B, (int)nmax, c, kappa, nullptr,
                                      dev_err, st, tm);
}

cudaError_t append_tc(const void *k, const void *v, const float *Tk, const float *Tv, int B, int n,
                      const kvq_cache *c, int clip, const int32_t *pos, int32_t *dev_err,
                      cudaStream_t st);

// bfloat16 inputs with both transforms: chunks of 256 tokens or more go to the tcgen05
// tensor-core kernel (which counts tokens in 32 bits), shorter (decode-time) appends to
// the short mma.sync kernel; float32 inputs, identity transforms, unaligned inputs and
// chunks beyond 2^31 tokens use the float32 CUDA-core kernel.
cudaError_t append_launch(const void *k, const void *v, int in_bf16, const float *Tk,
                          const float *Tv, int B, int n, const kvq_cache *c, int kappa,
                          const int32_t *pos, int32_t *dev_err, cudaStream_t st)
{
    const long tokens = (long)B * n;
    const bool a16 = ((uintptr_t)k % 16 == 0) && ((uintptr_t)v % 16 == 0) &&
                     ((uintptr_t)Tk % 16 == 0) && ((uintptr_t)Tv % 16 == 0);
    if (in_bf16 && Tk && Tv && a16 && tokens >= 256 && tokens <= 0x7fffff00L)
        return append_tc(k, v, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
    if (in_bf16 && Tk && Tv && a16 && tokens < 256) {
        if (c->d == 64)
            return launch_append_small<64>(k, v, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
        return launch_append_small<128>(k, v, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
    }
    const bool small = tokens <= 2048;
    if (c->d == 64)
        return small ? launch_append_fp32<64, 1>(k, v, in_bf16, Tk, Tv, B, n, c, kappa, pos, dev_err, st)
                     : launch_append_fp32<64, 4>(k, v, in_bf16, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
    return small ? launch_append_fp32<128, 1>(k, v, in_bf16, Tk, Tv, B, n, c, kappa, pos, dev_err, st)
                 : launch_append_fp32<128, 4>(k, v, in_bf16, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
}

}  // namespace kvq
