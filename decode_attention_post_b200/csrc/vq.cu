// Vector-quantized cache ("Spend Bits Where Queries Look: KV Cache Vector Quantization with
// Attention-Preserving Transforms", NOVA-KV project page): keys and values are transformed
// and encoded once on the write path into a fixed-width cache; the read path is a codebook
// lookup plus one multiply. Groups of 4 transformed coefficients carry an 8-bit index into
// a 256-word float16 codebook (one per KV head for keys, one for values); each token
// carries a float16 gain: x^_group = g * C[idx].
//
//  vq_append_kernel   write path. CTA = (KV head, one of {K, V}, token slice), 8 warps, T
//                     staged transposed in shared memory once per CTA, the codebook as
//                     float32. A warp encodes one token: lane i computes transformed dims
//                     4i..4i+3 (d = 128; d = 64: two lanes per group, each scanning half
//                     of the codebook), the gain from a float64 sum of squares, then the
//                     nearest scaled codeword by the float32 distance with the fixed
//                     operation order of the definition (ties to the lowest index).
//  vq_decode_kernel   read path. CTA = (KV head, sequence, split), 4 warps, launched as a
//                     programmatic dependent of the query prologue (which writes q~). Each
//                     warp streams 64-token blocks (key indices, key gains, value indices,
//                     value gains) through a 2-stage bulk-copy ring; per 16 tokens it
//                     expands the key codewords into a float16 tile in shared memory,
//                     S = Ktile . q~ on float16 mma.sync (q~ as hi/lo pieces, float32
//                     accumulate), logits = g_t S / sqrt(d), float32 online softmax, then
//                     expands the value codewords and O^T += Vtile^T . P'^T with
//                     P' = p g^V (float16 hi/lo, laid out by movmatrix). Warps merge in
//                     shared memory, splits in the last CTA of the pair.
#include "kvq_common.cuh"
#include "kvq_ptx.cuh"
#include "decode_shapes.h"

#include <math.h>
#include <type_traits>

namespace kvq {

namespace {

constexpr int kVqDim = KVQ_VQ_DIM;
constexpr int kVqSize = KVQ_VQ_SIZE;
constexpr float kVqLog2e = 1.4426950408889634f;
constexpr float kVqLazy = 4.0f;

// ---------------------------------------------------------------- write path

constexpr int kVqAppendWarps = 8;

template <int D>
struct VqAppendSmem {
    float Tt[D * (D + 4)];              // Tt[j][i] = T[i][j], row stride D + 4
    float4 cb[kVqSize];                 // codebook as float32
    float x[kVqAppendWarps][D];         // the warp's input token
};

template <int D>
__global__ void __launch_bounds__(kVqAppendWarps * 32)
vq_append_kernel(const void *__restrict__ k_in, const void *__restrict__ v_in, int in_bf16,
                 const float *__restrict__ Tk, const float *__restrict__ Tv,
                 const uint16_t *__restrict__ cb_k, const uint16_t *__restrict__ cb_v, int B,
                 int n, int Hkv, int T_cap, uint8_t *__restrict__ k_idx,
                 uint16_t *__restrict__ k_gain, uint8_t *__restrict__ v_idx,
                 uint16_t *__restrict__ v_gain, const int32_t *__restrict__ pos,
                 int32_t *dev_err)
{
    using Sm = VqAppendSmem<D>;
    constexpr int NGRP = D / kVqDim;                // groups per token: 32 or 16
    constexpr int LPG = 32 / NGRP;                  // lanes per group: 1 or 2
    constexpr int CAND = kVqSize / LPG;             // codewords scanned per lane
    extern __shared__ __align__(16) unsigned char vq_smem[];
    Sm &sm = *reinterpret_cast<Sm *>(vq_smem);

    const int h = blockIdx.y, which = blockIdx.z;
    const void *in = which ? v_in : k_in;
    const float *T = which ? Tv : Tk;
    const uint16_t *cb = (which ? cb_v : cb_k) + (size_t)h * kVqSize * kVqDim;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (T) {
        for (int c = threadIdx.x; c < D * D / 4; c += kVqAppendWarps * 32) {
            const int i = c / (D / 4), j = 4 * (c % (D / 4));
            const float4 t4 = reinterpret_cast<const float4 *>(T + ((size_t)h * D + i) * D)[j / 4];
            sm.Tt[(j + 0) * (D + 4) + i] = t4.x;
            sm.Tt[(j + 1) * (D + 4) + i] = t4.y;
            sm.Tt[(j + 2) * (D + 4) + i] = t4.z;
            sm.Tt[(j + 3) * (D + 4) + i] = t4.w;
        }
    }
    for (int c = threadIdx.x; c < kVqSize; c += kVqAppendWarps * 32) {
        const uint2 w = reinterpret_cast<const uint2 *>(cb)[c];
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&w.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&w.y));
        sm.cb[c] = make_float4(a.x, a.y, b.x, b.y);
    }
    __syncthreads();

    const long total = (long)B * n;
    const int grp = lane / LPG, half = lane % LPG;
    for (long u = (long)blockIdx.x * kVqAppendWarps + warp; u < total;
         u += (long)gridDim.x * kVqAppendWarps) {
        const int b = (int)(u / n), i = (int)(u % n);
        const int p0 = pos[b];
        if (p0 < 0 || (long)p0 + n > T_cap) {
            if (i == 0 && lane == 0)
                flag(dev_err, KVQ_DEVERR_POS_RANGE);
            continue;
        }
        for (int j = lane; j < D; j += 32)
            sm.x[warp][j] = load_in(in, in_bf16, (((size_t)b * n + i) * Hkv + h) * D + j);
        __syncwarp();
        // ---- this lane's transformed dims 4 grp .. 4 grp + 3 (both lanes of a pair compute them)
        float xt[kVqDim];
        if (T) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
            for (int j = 0; j < D; ++j) {
                const float xj = sm.x[warp][j];
                const float4 t4 = *reinterpret_cast<const float4 *>(&sm.Tt[j * (D + 4) + 4 * grp]);
                acc.x = fmaf(t4.x, xj, acc.x);
                acc.y = fmaf(t4.y, xj, acc.y);
                acc.z = fmaf(t4.z, xj, acc.z);
                acc.w = fmaf(t4.w, xj, acc.w);
            }
            xt[0] = acc.x;
            xt[1] = acc.y;
            xt[2] = acc.z;
            xt[3] = acc.w;
        } else {
#pragma unroll
            for (int m = 0; m < kVqDim; ++m)
                xt[m] = sm.x[warp][4 * grp + m];
        }
        __syncwarp();
        // ---- gain: g = f16(f32(sqrt(sum x~^2 / d))), the sum in float64 over the groups
        double ss = 0.0;
        if (half == 0) {
#pragma unroll
            for (int m = 0; m < kVqDim; ++m)
                ss = fma((double)xt[m], (double)xt[m], ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const __half gh = __float2half_rn(__double2float_rn(sqrt(ss / (double)D)));
        const float g = __half2float(gh);
        // ---- nearest scaled codeword, ties to the lowest index
        int best = 0;
        float bestd = INFINITY;
        if (g != 0.f) {
            for (int c = half * CAND; c < (half + 1) * CAND; ++c) {
                const float4 w = sm.cb[c];
                const float e0 = __fsub_rn(xt[0], __fmul_rn(g, w.x));
                const float e1 = __fsub_rn(xt[1], __fmul_rn(g, w.y));
                const float e2 = __fsub_rn(xt[2], __fmul_rn(g, w.z));
                const float e3 = __fsub_rn(xt[3], __fmul_rn(g, w.w));
                float dist = __fmul_rn(e0, e0);
                dist = __fmaf_rn(e1, e1, dist);
                dist = __fmaf_rn(e2, e2, dist);
                dist = __fmaf_rn(e3, e3, dist);
                if (dist < bestd) {
                    bestd = dist;
                    best = c;
                }
            }
        }
        if (LPG == 2) {
            // merge the two halves: the lower half's codewords come first
            const float od = __shfl_xor_sync(0xffffffffu, bestd, 1);
            const int ob = __shfl_xor_sync(0xffffffffu, best, 1);
            const bool take = half == 0 ? (od < bestd) : !(bestd < od);
            if (take) {
                bestd = od;
                best = ob;
            }
        }
        const size_t slot = ((size_t)b * Hkv + h) * T_cap + p0 + i;
        if (half == 0)
            (which ? v_idx : k_idx)[slot * NGRP + grp] = (uint8_t)best;
        if (lane == 0)
            (which ? v_gain : k_gain)[slot] = __half_as_ushort(gh);
    }
}

// ---------------------------------------------------------------- read path

constexpr int kVqWarps = 4;
constexpr int kVqStages = 2;
constexpr int kVqBlock = 64;                    // tokens per ring stage
constexpr int kVqSub = 16;                      // tokens per MMA sub-tile

template <int D, int G>
struct VqCfg {
    static constexpr int NGRP = D / kVqDim;
    static constexpr int IDX_BYTES = kVqBlock * NGRP;       // one plane's indices of a block
    static constexpr int GAIN_BYTES = kVqBlock * 2;
    static constexpr int STAGE = 2 * IDX_BYTES + 2 * GAIN_BYTES;
    static constexpr int TS = D + 8;                        // float16 per tile row
    static constexpr int TILE = kVqSub * TS * 2;            // bytes of one expanded tile
    static constexpr int NT = (2 * G) / 8;                  // n-tiles of (hi, lo) x G columns
    static constexpr int KS = D / 16;                       // k-steps over the dims
    static constexpr int MT = D / 16;                       // m-tiles of the value product
    static constexpr int RING = kVqWarps * kVqStages * STAGE;
    static constexpr int TILES = kVqWarps * 2 * TILE;       // key and value tile per warp
    static constexpr int CB = 2 * kVqSize * kVqDim * 2;     // both codebooks, float16
    static constexpr int MERGE = kVqWarps * G * (D + 2) * 4;
    static constexpr int MAIN = RING + TILES + CB;
    static constexpr int SMEM = (MAIN > MERGE ? MAIN : MERGE) + kVqWarps * kVqStages * 8 + 16;
    static_assert(STAGE % 16 == 0 && TILE % 16 == 0, "alignment");
};

// Expand the codewords of 16 tokens (indices idx [16][NGRP], one byte each) into the
// float16 tile [16][TS]: entry (token, group) -> C[idx] at columns 4 group .. 4 group + 3.
// Lane work item = 4 consecutive groups of one token: one 32-bit index load, four
// codeword loads, two 16-byte stores; fully unrolled so that the loads overlap.
template <int D>
__device__ __forceinline__ void expand_tile(const uint8_t *idx, const uint2 *cb, __half *tile,
                                            int lane)
{
    constexpr int NGRP = D / kVqDim, TS = D + 8, QUADS = kVqSub * NGRP / 4;
    static_assert(QUADS % 32 == 0, "whole warp iterations");
    uint32_t iw[QUADS / 32];
#pragma unroll
    for (int m = 0; m < QUADS / 32; ++m)
        iw[m] = reinterpret_cast<const uint32_t *>(idx)[lane + 32 * m];
#pragma unroll
    for (int m = 0; m < QUADS / 32; ++m) {
        const int e4 = lane + 32 * m;                   // quad of groups 4 e4 .. 4 e4 + 3
        const int tok = (4 * e4) / NGRP, grp = (4 * e4) % NGRP;
        const uint2 w0 = cb[iw[m] & 0xFF], w1 = cb[(iw[m] >> 8) & 0xFF];
        const uint2 w2 = cb[(iw[m] >> 16) & 0xFF], w3 = cb[iw[m] >> 24];
        uint4 *dst = reinterpret_cast<uint4 *>(tile + tok * TS + kVqDim * grp);
        dst[0] = make_uint4(w0.x, w0.y, w1.x, w1.y);
        dst[1] = make_uint4(w2.x, w2.y, w3.x, w3.y);
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kVqWarps * 32)
vq_decode_kernel(const uint8_t *__restrict__ k_idx, const uint16_t *__restrict__ k_gain,
                 const uint8_t *__restrict__ v_idx, const uint16_t *__restrict__ v_gain,
                 const uint16_t *__restrict__ cb_k, const uint16_t *__restrict__ cb_v,
                 const float *__restrict__ qt, const int32_t *__restrict__ seqlens, int B,
                 int Hkv, int Hq, int T_cap, int max_seqlen, int nsplit, int split_tokens,
                 int part_slots, float *__restrict__ part, int *__restrict__ ticket, void *out,
                 int out_bf16, int32_t *dev_err)
{
    using C = VqCfg<D, G>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *ring = smem_raw;
    __half *tiles = reinterpret_cast<__half *>(smem_raw + C::RING);
    uint2 *cbs = reinterpret_cast<uint2 *>(smem_raw + C::RING + C::TILES);   // [2][256]
    uint64_t *bars_all = reinterpret_cast<uint64_t *>(
        smem_raw + (C::MAIN > C::MERGE ? C::MAIN : C::MERGE));
    int *flag_smem = reinterpret_cast<int *>(bars_all + kVqWarps * kVqStages);

    const int h = blockIdx.x, b = blockIdx.y, sigma = blockIdx.z;
    const int lane = threadIdx.x & 31;
    const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
    const int g = lane >> 2, t = lane & 3;
    const size_t pair = (size_t)b * Hkv + h;

    int seqlen = seqlens[b];
    if (seqlen < 0 || seqlen > max_seqlen) {
        if (sigma == 0 && h == 0 && threadIdx.x == 0)
            flag(dev_err, KVQ_DEVERR_SEQLEN_CLAMPED);
        seqlen = seqlen < 0 ? 0 : max_seqlen;
    }
    const int t_begin = sigma * split_tokens;
    if (t_begin >= seqlen)
        return;                                 // the prologue wrote empty sequences' zeros
    const int t_end = min(t_begin + split_tokens, seqlen);
    const int nsplit_b = (seqlen + split_tokens - 1) / split_tokens;
    const int nblk = (t_end - t_begin + kVqBlock - 1) / kVqBlock;
    const int my_nblk = nblk > warp ? (nblk - warp + kVqWarps - 1) / kVqWarps : 0;
    unsigned char *wring = ring + warp * kVqStages * C::STAGE;
    uint64_t *bars = bars_all + warp * kVqStages;
    __half *ktile = tiles + (size_t)warp * 2 * kVqSub * C::TS;
    __half *vtile = ktile + kVqSub * C::TS;

    if (lane == 0) {
        for (int s = 0; s < kVqStages; ++s)
            mbar_init(&bars[s], 1);
        mbar_fence_init();
    }
    __syncwarp();
    auto issue = [&](int jj, int s) {
        const int tok0 = t_begin + (warp + jj * kVqWarps) * kVqBlock;
        unsigned char *st = wring + s * C::STAGE;
        if (lane == 0) {
            const size_t row0 = pair * T_cap + tok0;
            mbar_arrive_expect_tx_relaxed(&bars[s], C::STAGE);
            bulk_g2s(st, k_idx + row0 * C::NGRP, C::IDX_BYTES, &bars[s]);
            bulk_g2s(st + C::IDX_BYTES, k_gain + row0, C::GAIN_BYTES, &bars[s]);
            bulk_g2s(st + C::IDX_BYTES + C::GAIN_BYTES, v_idx + row0 * C::NGRP, C::IDX_BYTES,
                     &bars[s]);
            bulk_g2s(st + 2 * C::IDX_BYTES + C::GAIN_BYTES, v_gain + row0, C::GAIN_BYTES,
                     &bars[s]);
        }
        __syncwarp();
    };
    for (int jj = 0; jj < kVqStages && jj < my_nblk; ++jj)
        issue(jj, jj);
    // both codebooks of this KV head (float16, 8 bytes a codeword)
    for (int c = threadIdx.x; c < 2 * kVqSize; c += kVqWarps * 32) {
        const uint16_t *src = (c < kVqSize ? cb_k : cb_v) + ((size_t)h * kVqSize + c % kVqSize) * kVqDim;
        cbs[c] = *reinterpret_cast<const uint2 *>(src);
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");     // q~ from the prologue

    // q~ of the G heads as the B operand of S = K . q~: column n = 2 head' + piece of
    // n-tile nt (head' = 4 nt + n/2), piece 0 = float16(q~), 1 = float16(q~ - that)
    uint32_t qB[C::NT][C::KS][2];
    {
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            const int head = 4 * nt + g / 2, piece = g & 1;
            const float *qh = qt + ((size_t)b * Hq + h * G + head) * D;
#pragma unroll
            for (int ks = 0; ks < C::KS; ++ks)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float2 f = *reinterpret_cast<const float2 *>(qh + 16 * ks + 8 * hh + 2 * t);
                    const __half2 hi = __floats2half2_rn(f.x, f.y);
                    const float2 hf = __half22float2(hi);
                    const __half2 lo = __floats2half2_rn(f.x - hf.x, f.y - hf.y);
                    const __half2 v = piece ? lo : hi;
                    qB[nt][ks][hh] = *reinterpret_cast<const uint32_t *>(&v);
                }
        }
    }
    const float sc = kVqLog2e * rsqrtf((float)D);

    float m_run[C::NT], l_run[C::NT];
    float O[C::MT][C::NT][4];
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
        m_run[nt] = -INFINITY;
        l_run[nt] = 0.f;
#pragma unroll
        for (int m = 0; m < C::MT; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                O[m][nt][i] = 0.f;
    }
    bool timed_out = false;

    for (int jj = 0; jj < my_nblk; ++jj) {
        const int s = jj % kVqStages;
        if (!mbar_wait_bounded(&bars[s], (jj / kVqStages) & 1)) {
            timed_out = true;
            for (int k2 = jj + 1; k2 < jj + kVqStages && k2 < my_nblk; ++k2)
                mbar_wait_bounded(&bars[k2 % kVqStages], (k2 / kVqStages) & 1);
            break;
        }
        const unsigned char *st = wring + s * C::STAGE;
        const uint8_t *kid = st;
        const uint16_t *kg = reinterpret_cast<const uint16_t *>(st + C::IDX_BYTES);
        const uint8_t *vid = st + C::IDX_BYTES + C::GAIN_BYTES;
        const uint16_t *vg = reinterpret_cast<const uint16_t *>(st + 2 * C::IDX_BYTES + C::GAIN_BYTES);
        const int tok0 = t_begin + (warp + jj * kVqWarps) * kVqBlock;
        for (int stt = 0; stt < kVqBlock / kVqSub; ++stt) {
            if (tok0 + kVqSub * stt >= t_end)
                break;
            const int ta = kVqSub * stt + g, tb = ta + 8;          // this lane's two tokens
            const bool va = tok0 + ta < t_end, vb = tok0 + tb < t_end;
            // ---- keys: expand, S[16 x 2G] = Ktile . q~
            expand_tile<D>(kid + kVqSub * stt * C::NGRP, cbs, ktile, lane);
            __syncwarp();
            float S[C::NT][4];
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    S[nt][i] = 0.f;
#pragma unroll
            for (int ks = 0; ks < C::KS; ++ks) {
                uint32_t a[4];
                ldmatrix_x4(a, ktile + (lane & 15) * C::TS + 16 * ks + 8 * (lane >> 4));
#pragma unroll
                for (int nt = 0; nt < C::NT; ++nt)
                    mma_f16(S[nt], a[0], a[1], a[2], a[3], qB[nt][ks][0], qB[nt][ks][1]);
            }
            // ---- logits (log2 units): g_t (hi + lo) / sqrt(d); online softmax per head
            const float ga = __half2float(__ushort_as_half(kg[ta])) * sc;
            const float gb = __half2float(__ushort_as_half(kg[tb])) * sc;
            float la[C::NT], lb[C::NT];
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt) {
                la[nt] = va ? ga * (S[nt][0] + S[nt][1]) : -INFINITY;
                lb[nt] = vb ? gb * (S[nt][2] + S[nt][3]) : -INFINITY;
                float bm = fmaxf(la[nt], lb[nt]);
                bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
                bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
                bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
                if (bm > m_run[nt] + kVqLazy) {
                    const float alpha = ex2(m_run[nt] - bm);
                    l_run[nt] *= alpha;
#pragma unroll
                    for (int m = 0; m < C::MT; ++m)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            O[m][nt][i] *= alpha;
                    m_run[nt] = bm;
                }
            }
            // ---- P' = p g^V as float16 (hi, lo): rows = tokens, columns (hi, lo) of head t;
            //      one 8x8 transpose per row half makes the B operand of the value product
            // masked tokens: gain 0 (cache bytes past the length may hold any bit pattern)
            const float gva = va ? __half2float(__ushort_as_half(vg[ta])) : 0.f;
            const float gvb = vb ? __half2float(__ushort_as_half(vg[tb])) : 0.f;
            uint32_t pb[C::NT][2];
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt) {
                const float pa = ex2(la[nt] - m_run[nt]), pbv = ex2(lb[nt] - m_run[nt]);
                l_run[nt] += pa + pbv;
                const float wa = pa * gva, wb = pbv * gvb;
                const __half ha = __float2half_rn(wa), hb = __float2half_rn(wb);
                const __half2 ra = __halves2half2(ha, __float2half_rn(wa - __half2float(ha)));
                const __half2 rb = __halves2half2(hb, __float2half_rn(wb - __half2float(hb)));
                pb[nt][0] = movmatrix_trans(*reinterpret_cast<const uint32_t *>(&ra));
                pb[nt][1] = movmatrix_trans(*reinterpret_cast<const uint32_t *>(&rb));
            }
            // ---- values: expand, O^T[d x 2G] += Vtile^T . P'^T
            expand_tile<D>(vid + kVqSub * stt * C::NGRP, cbs + kVqSize, vtile, lane);
            __syncwarp();
#pragma unroll
            for (int m = 0; m < C::MT; ++m) {
                // matrices (dims 16m + 8(q&1) .. +7) x (tokens 8(q>>1) .. +7), q = lane / 8
                const int q = lane >> 3;
                uint32_t a[4];
                ldmatrix_x4_trans(a, vtile + (8 * (q >> 1) + (lane & 7)) * C::TS + 16 * m + 8 * (q & 1));
#pragma unroll
                for (int nt = 0; nt < C::NT; ++nt)
                    mma_f16(O[m][nt], a[0], a[1], a[2], a[3], pb[nt][0], pb[nt][1]);
            }
            __syncwarp();                       // the tiles are rewritten by the next sub-tile
        }
        if (jj + kVqStages < my_nblk)
            issue(jj + kVqStages, s);
    }
    if (timed_out && lane == 0)
        flag(dev_err, KVQ_DEVERR_WAIT_TIMEOUT);

#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1)
            l_run[nt] += __shfl_xor_sync(0xffffffffu, l_run[nt], off);

    __syncthreads();                            // every warp is done with the ring and tiles
    if (lane == 0)
        for (int s = 0; s < kVqStages; ++s)
            mbar_inval(&bars[s]);
    float *mw = reinterpret_cast<float *>(smem_raw);     // [W][G]
    float *lw = mw + kVqWarps * G;                       // [W][G]
    float *ow = lw + kVqWarps * G;                       // [W][G][D]
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
        const int head = 4 * nt + t;
        if (g == 0) {
            mw[warp * G + head] = m_run[nt];
            lw[warp * G + head] = l_run[nt];
        }
#pragma unroll
        for (int m = 0; m < C::MT; ++m) {
            // rows g and g+8 of m-tile m are dims 16m + g and 16m + g + 8; columns 2t (hi)
            // and 2t+1 (lo) of head t
            ow[(warp * G + head) * D + 16 * m + g] = O[m][nt][0] + O[m][nt][1];
            ow[(warp * G + head) * D + 16 * m + g + 8] = O[m][nt][2] + O[m][nt][3];
        }
    }
    __syncthreads();

    const int nmerge = nsplit_b;
    float *mypart = part + (pair * part_slots + sigma) * (size_t)(G * (D + 2));
    for (int idx = threadIdx.x; idx < G * D; idx += kVqWarps * 32) {
        const int head = idx / D, dim = idx % D;
        float Mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kVqWarps; ++w)
            Mx = fmaxf(Mx, mw[w * G + head]);
        float L = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < kVqWarps; ++w) {
            const float mwv = mw[w * G + head];
            if (mwv == -INFINITY)
                continue;
            const float wt = ex2(mwv - Mx);
            L = fmaf(wt, lw[w * G + head], L);
            o = fmaf(wt, ow[(w * G + head) * D + dim], o);
        }
        if (nmerge == 1) {
            const size_t oi = ((size_t)b * Hq + h * G + head) * D + dim;
            const float r = o / L;
            if (out_bf16)
                reinterpret_cast<__nv_bfloat16 *>(out)[oi] = __float2bfloat16_rn(r);
            else
                reinterpret_cast<float *>(out)[oi] = r;
        } else {
            mypart[head * (D + 2) + 2 + dim] = o;
            if (dim == 0) {
                mypart[head * (D + 2)] = Mx;
                mypart[head * (D + 2) + 1] = L;
            }
        }
    }
    if (nmerge == 1)
        return;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int last = (atomicAdd(&ticket[pair], 1) == nmerge - 1);
        __threadfence();
        *flag_smem = last;
    }
    __syncthreads();
    if (!*flag_smem)
        return;
    const float *pall = part + pair * part_slots * (size_t)(G * (D + 2));
    for (int idx = threadIdx.x; idx < G * D; idx += kVqWarps * 32) {
        const int head = idx / D, dim = idx % D;
        float Mx = -INFINITY;
        for (int i = 0; i < nmerge; ++i)
            Mx = fmaxf(Mx, __ldcg(pall + (size_t)i * G * (D + 2) + head * (D + 2)));
        float L = 0.f, o = 0.f;
        for (int i = 0; i < nmerge; ++i) {
            const float *pp = pall + (size_t)i * G * (D + 2) + head * (D + 2);
            const float wt = ex2(__ldcg(pp) - Mx);
            L = fmaf(wt, __ldcg(pp + 1), L);
            o = fmaf(wt, __ldcg(pp + 2 + dim), o);
        }
        const size_t oi = ((size_t)b * Hq + h * G + head) * D + dim;
        const float r = o / L;
        if (out_bf16)
            reinterpret_cast<__nv_bfloat16 *>(out)[oi] = __float2bfloat16_rn(r);
        else
            reinterpret_cast<float *>(out)[oi] = r;
    }
}

template <int D>
cudaError_t launch_vq_append_t(const void *k, const void *v, int in_bf16, const float *Tk,
                               const float *Tv, const void *cb_k, const void *cb_v, int B, int n,
                               const kvq_vq_cache *c, const int32_t *pos, int32_t *dev_err,
                               cudaStream_t st)
{
    const int smem = (int)sizeof(VqAppendSmem<D>);
    static unsigned long long attr = 0;
    cudaError_t e = ensure_dynamic_smem(vq_append_kernel<D>, smem, attr);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long tokens = (long)B * n;
    long gx = (tokens + kVqAppendWarps - 1) / kVqAppendWarps;
    const long cap = (2L * sms + 2L * c->Hkv - 1) / (2L * c->Hkv) * 4;
    if (gx > cap)
        gx = cap;
    if (gx < 1)
        gx = 1;
    vq_append_kernel<D><<<dim3((unsigned)gx, (unsigned)c->Hkv, 2), kVqAppendWarps * 32, smem, st>>>(
        k, v, in_bf16, Tk, Tv, (const uint16_t *)cb_k, (const uint16_t *)cb_v, B, n, c->Hkv,
        c->T_cap, (uint8_t *)c->k_idx, (uint16_t *)c->k_gain, (uint8_t *)c->v_idx,
        (uint16_t *)c->v_gain, pos, dev_err);
    return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_vq_decode_t(const VqLaunch &V, cudaStream_t st)
{
    using C = VqCfg<D, G>;
    static unsigned long long attr = 0;
    cudaError_t e = ensure_dynamic_smem(vq_decode_kernel<D, G>, C::SMEM, attr);
    if (e != cudaSuccess)
        return e;
    e = launch_qprep_qt(V.L, V.qt, st);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(V.L.p.Hkv, V.L.p.B, V.L.p.nsplit);
    cfg.blockDim = dim3(kVqWarps * 32);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr1[1];
    attr1[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr1[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr1;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, vq_decode_kernel<D, G>, V.k_idx, V.k_gain, V.v_idx, V.v_gain,
                              V.cb_k, V.cb_v, (const float *)V.qt, V.L.p.seqlens, V.L.p.B,
                              V.L.p.Hkv, V.L.p.Hq, V.L.p.T_cap, V.L.p.max_seqlen, V.L.p.nsplit,
                              V.L.p.split_tokens, V.L.p.part_slots, V.L.p.part, V.L.p.ticket,
                              V.L.p.out, V.L.p.out_bf16, V.L.p.dev_err);
}

}  // namespace

cudaError_t launch_vq_append(const void *k, const void *v, int in_bf16, const float *Tk,
                             const float *Tv, const void *cb_k, const void *cb_v, int B, int n,
                             const kvq_vq_cache *c, const int32_t *pos, int32_t *dev_err,
                             cudaStream_t st)
{
    if (c->d == 64)
        return launch_vq_append_t<64>(k, v, in_bf16, Tk, Tv, cb_k, cb_v, B, n, c, pos, dev_err, st);
    return launch_vq_append_t<128>(k, v, in_bf16, Tk, Tv, cb_k, cb_v, B, n, c, pos, dev_err, st);
}

// Resident VQ decode CTAs per SM (shared memory bound; at most 4).
int vq_resident_ctas(int d, int G)
{
    int smem = VqCfg<128, 4>::SMEM;
    if (d == 128 && G == 8)
        smem = VqCfg<128, 8>::SMEM;
    else if (d == 64 && G == 4)
        smem = VqCfg<64, 4>::SMEM;
    else if (d == 64 && G == 8)
        smem = VqCfg<64, 8>::SMEM;
    const int fit = (227 * 1024) / (smem + 1024);
    return fit < 1 ? 1 : (fit > 4 ? 4 : fit);
}

cudaError_t launch_vq_decode(const VqLaunch &V, cudaStream_t st)
{
    const int d = V.L.d, G = V.L.G;
    if (d == 128 && G == 4)
        return launch_vq_decode_t<128, 4>(V, st);
    if (d == 128 && G == 8)
        return launch_vq_decode_t<128, 8>(V, st);
    if (d == 64 && G == 4)
        return launch_vq_decode_t<64, 4>(V, st);
    if (d == 64 && G == 8)
        return launch_vq_decode_t<64, 8>(V, st);
    return cudaErrorInvalidValue;
}

}  // namespace kvq
