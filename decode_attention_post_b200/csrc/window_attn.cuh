// Full-precision window of the read path ("WUSH-KV: KV Cache Quantization with
// Data-Adaptive Transforms", section 4.4): attention over the positions a sequence keeps
// in full precision -- the first S_sink positions and those after the quantized middle --
// as one more partial (running max, sum of weights, weighted sum of values) next to the
// splits of the quantized middle. It runs as one more split CTA of the decode grid, so it
// overlaps the quantized splits and joins their merge.
//
// The CTA's 4 warps serve the G query heads of one (KV head, sequence). The window is the
// sink rows present plus every slot of the recent ring, each slot masked by the position
// it holds (the softmax does not depend on the order). Each warp takes 16-row tiles: key
// and value rows staged in shared memory by 16-byte asynchronous copies, S = K q on bf16
// tensor cores (the query as given, bf16, exact: q . k = (T_k^{-T} q) . (T_k k)), logits
// in log2 units, float32 online softmax, O^T += V^T P^T with P as bf16 (hi, lo) pairs; the
// warps merge in shared memory and T_v is applied once to the merged sum, so that o is in
// the value-transform domain like the quantized values.
#pragma once

#include "kvq_common.cuh"
#include "kvq_ptx.cuh"
#include "decode_shapes.h"

#include <math.h>

namespace kvq {
namespace win {

constexpr int kThreads = kDecodeWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSub = 16;                        // window rows per MMA tile
constexpr float kLazy = 4.0f;

template <int D, int G>
struct Smem {
    static constexpr int TS = D + 8;            // bf16 per staged row (ldmatrix conflict-free)
    static constexpr int TILE = kSub * TS;      // bf16 of one staged 16-row tile
    static constexpr int NT = (2 * G) / 8;      // n-tiles of the value product ((hi, lo) x G)
    static constexpr int KS = D / 16;
    static constexpr int MT = D / 16;
    // per warp: K and V tiles; after the loop the same space holds the warps' partials
    // (MERGE bytes), the merged sum x[G][D] and (m, l) per head; T_v o goes to offset 0
    static constexpr int TILES = kDecodeWarps * 2 * TILE * 2;
    static constexpr int MERGE = kDecodeWarps * G * (D + 2) * 4;
    static constexpr int FIN = G * D * 4 + 2 * G * 4;
    static constexpr int BYTES = TILES > MERGE + FIN ? TILES : MERGE + FIN;
    static_assert(G <= 8, "one n-tile of the key product");
    static_assert(G * D * 4 <= MERGE, "T_v o fits below the merged sum");
};

// Row w of the window: w < nsink is sink row w; otherwise ring slot w - nsink, valid when
// the position it holds is in [rec0, L) (slot s holds the position t in [L - R, L) with
// t = s mod R; the others are flushed or not yet written).
struct Rows {
    const __nv_bfloat16 *sink, *ring;           // [S_sink][D] and [R][D] of this (seq, head)
    int nsink, R, L, rec0;
};

__device__ __forceinline__ bool row_of(const Rows &wr, int w, int D, const __nv_bfloat16 **row)
{
    if (w < wr.nsink) {
        *row = wr.sink + (size_t)w * D;
        return true;
    }
    const int s = w - wr.nsink;
    const int t = wr.L - wr.R + (((s - (wr.L - wr.R)) % wr.R) + wr.R) % wr.R;
    *row = wr.ring + (size_t)s * D;
    return t >= wr.rec0 && t < wr.L;
}

// Attention of the G query heads of KV head h of sequence b (length L > 0, Q positions
// quantized) over its window. Leaves in shared memory o[G][D] = T_v sum_t p_t v_t and
// stat[G][2] = (m, l) in log2 units (l = sum_t 2^(logit_t - m)), returned through *o_out
// and *stat_out; ends with a CTA barrier. Uses Smem<D, G>::BYTES bytes at smem.
template <int D, int G>
__device__ __forceinline__ void attend(const DecodeParams &P, int b, int h, int L, int Q,
                                       unsigned char *smem, const float **o_out,
                                       const float **stat_out)
{
    using C = Smem<D, G>;
    __nv_bfloat16 *tiles = reinterpret_cast<__nv_bfloat16 *>(smem);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int R = P.win_keep + P.win_flush;
    const size_t pair = (size_t)b * P.Hkv + h;
    Rows kr, vr;
    kr.nsink = vr.nsink = min(P.win_sink, L);
    kr.R = vr.R = R;
    kr.L = vr.L = L;
    kr.rec0 = vr.rec0 = P.win_sink + Q;
    kr.sink = reinterpret_cast<const __nv_bfloat16 *>(P.k_sink) + pair * P.win_sink * D;
    vr.sink = reinterpret_cast<const __nv_bfloat16 *>(P.v_sink) + pair * P.win_sink * D;
    kr.ring = reinterpret_cast<const __nv_bfloat16 *>(P.k_recent) + pair * R * D;
    vr.ring = reinterpret_cast<const __nv_bfloat16 *>(P.v_recent) + pair * R * D;
    // rows to scan: the sink rows present, then every ring slot (masked by position)
    const int nrows = kr.nsink + (L > kr.rec0 ? R : 0);
    const int ntiles = (nrows + kSub - 1) / kSub;
    const float sc = kLog2e * rsqrtf((float)D);
    __nv_bfloat16 *ktile = tiles + (size_t)warp * 2 * C::TILE;
    __nv_bfloat16 *vtile = ktile + C::TILE;

    // q of the G heads (bf16, exact) as the B operand of S = K . q: column n = head n
    uint32_t qB[C::KS][2];
#pragma unroll
    for (int ks = 0; ks < C::KS; ++ks)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t v = 0;
            if (g < G)
                v = *reinterpret_cast<const uint32_t *>(
                    reinterpret_cast<const __nv_bfloat16 *>(P.win_q) +
                    ((size_t)b * P.Hq + h * G + g) * D + 16 * ks + 8 * hh + 2 * t);
            qB[ks][hh] = v;
        }

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

    for (int tt = warp; tt < ntiles; tt += kDecodeWarps) {
        const int w0 = tt * kSub;
        // ---- stage the tile's key and value rows (16-byte copies). Rows past the end and
        //      ring slots not holding a window position are zero-filled: their weight is 0,
        //      and a never-written slot may hold any bit pattern (0 * NaN would not be 0).
        for (int c = lane; c < 2 * kSub * (D / 8); c += 32) {
            const int which = c / (kSub * (D / 8)), cc = c % (kSub * (D / 8));
            const int rr = cc / (D / 8), ch = cc % (D / 8);
            const __nv_bfloat16 *row = nullptr;
            bool ok = false;
            if (w0 + rr < nrows)
                ok = row_of(which ? vr : kr, w0 + rr, D, &row);
            __nv_bfloat16 *dst = (which ? vtile : ktile) + rr * C::TS + 8 * ch;
            cp_async16(dst, ok ? row + 8 * ch : kr.ring, ok ? 16 : 0);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
        // validity of this lane's two rows (g and g + 8 of the tile)
        const __nv_bfloat16 *dummy;
        const bool va = w0 + g < nrows && row_of(kr, w0 + g, D, &dummy);
        const bool vb = w0 + g + 8 < nrows && row_of(kr, w0 + g + 8, D, &dummy);
        // ---- S[16 x G] = Ktile . q
        float S[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
            uint32_t a[4];
            ldmatrix_x4(a, ktile + (lane & 15) * C::TS + 16 * ks + 8 * (lane >> 4));
            mma_bf16(S, a[0], a[1], a[2], a[3], qB[ks][0], qB[ks][1]);
        }
        // The key product's accumulator has row g, columns 2t, 2t+1 = heads 2t, 2t+1; the
        // value product wants head 4 nt + t on this lane. Its logits come from the quad
        // lane holding that head.
        float la[C::NT], lb[C::NT];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            const int head = 4 * nt + t;
            const int src = (lane & ~3) | (head >> 1);
            const float sa0 = __shfl_sync(0xffffffffu, S[0], src);
            const float sa1 = __shfl_sync(0xffffffffu, S[1], src);
            const float sb0 = __shfl_sync(0xffffffffu, S[2], src);
            const float sb1 = __shfl_sync(0xffffffffu, S[3], src);
            la[nt] = va ? sc * ((head & 1) ? sa1 : sa0) : -INFINITY;
            lb[nt] = vb ? sc * ((head & 1) ? sb1 : sb0) : -INFINITY;
            float bm = fmaxf(la[nt], lb[nt]);
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
            if (bm > m_run[nt] + kLazy) {
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
        // ---- P as bf16 (hi, lo) pairs, rows = window rows, columns (hi, lo) of head
        //      4nt + t; 8x8 transposes make the B operand of the value product
        uint32_t pb[C::NT][2];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            // no valid row seen yet: every logit so far is -inf and every weight 0
            const float mr = m_run[nt] == -INFINITY ? 0.f : m_run[nt];
            const float pa = ex2(la[nt] - mr), pbv = ex2(lb[nt] - mr);
            l_run[nt] += pa + pbv;
            const __nv_bfloat16 ha = __float2bfloat16_rn(pa), hb = __float2bfloat16_rn(pbv);
            const __nv_bfloat162 ra2 =
                __halves2bfloat162(ha, __float2bfloat16_rn(pa - __bfloat162float(ha)));
            const __nv_bfloat162 rb2 =
                __halves2bfloat162(hb, __float2bfloat16_rn(pbv - __bfloat162float(hb)));
            pb[nt][0] = movmatrix_trans(*reinterpret_cast<const uint32_t *>(&ra2));
            pb[nt][1] = movmatrix_trans(*reinterpret_cast<const uint32_t *>(&rb2));
        }
        // ---- O^T[D x 2G] += Vtile^T . P^T
#pragma unroll
        for (int m = 0; m < C::MT; ++m) {
            const int q = lane >> 3;
            uint32_t a[4];
            ldmatrix_x4_trans(a, vtile + (8 * (q >> 1) + (lane & 7)) * C::TS + 16 * m + 8 * (q & 1));
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt)
                mma_bf16(O[m][nt], a[0], a[1], a[2], a[3], pb[nt][0], pb[nt][1]);
        }
        __syncwarp();                                   // the tiles are refilled next
    }
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1)
            l_run[nt] += __shfl_xor_sync(0xffffffffu, l_run[nt], off);

    // ---- merge the warps (log2-scaled (m, l, o) in shared memory)
    __syncthreads();
    float *mw = reinterpret_cast<float *>(smem);        // [W][G]
    float *lw = mw + kDecodeWarps * G;                  // [W][G]
    float *ow = lw + kDecodeWarps * G;                  // [W][G][D]
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
        const int head = 4 * nt + t;
        if (g == 0) {
            mw[warp * G + head] = m_run[nt];
            lw[warp * G + head] = l_run[nt];
        }
#pragma unroll
        for (int m = 0; m < C::MT; ++m) {
            ow[(warp * G + head) * D + 16 * m + g] = O[m][nt][0] + O[m][nt][1];
            ow[(warp * G + head) * D + 16 * m + g + 8] = O[m][nt][2] + O[m][nt][3];
        }
    }
    __syncthreads();
    float *x = reinterpret_cast<float *>(smem + C::MERGE);   // [G][D]
    float *stat = x + G * D;                                 // [G][2]
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int head = idx / D, dim = idx % D;
        float Mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w)
            Mx = fmaxf(Mx, mw[w * G + head]);
        float Lsum = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
            const float mwv = mw[w * G + head];
            if (mwv == -INFINITY)
                continue;
            const float wt = ex2(mwv - Mx);
            Lsum = fmaf(wt, lw[w * G + head], Lsum);
            o = fmaf(wt, ow[(w * G + head) * D + dim], o);
        }
        x[idx] = o;
        if (dim == 0) {
            stat[2 * head] = Mx;
            stat[2 * head + 1] = Lsum;
        }
    }
    __syncthreads();
    *stat_out = stat;
    if (!P.win_Tv) {
        *o_out = x;
        return;
    }
    // ---- o = T_v x: thread per output row i (two threads per row when d = 64, each with
    //      half of the heads); the row is read once, x by broadcast
    constexpr int TPR = kThreads / D;
    constexpr int HPT = G / TPR;
    const int i = threadIdx.x % D, h0 = (threadIdx.x / D) * HPT;
    const float4 *row = reinterpret_cast<const float4 *>(P.win_Tv + ((size_t)h * D + i) * D);
    float acc[HPT];
#pragma unroll
    for (int hh = 0; hh < HPT; ++hh)
        acc[hh] = 0.f;
#pragma unroll 4
    for (int j4 = 0; j4 < D / 4; ++j4) {
        const float4 tr = __ldg(row + j4);
#pragma unroll
        for (int hh = 0; hh < HPT; ++hh) {
            const float4 xv = reinterpret_cast<const float4 *>(x + (h0 + hh) * D)[j4];
            acc[hh] = fmaf(tr.x, xv.x, acc[hh]);
            acc[hh] = fmaf(tr.y, xv.y, acc[hh]);
            acc[hh] = fmaf(tr.z, xv.z, acc[hh]);
            acc[hh] = fmaf(tr.w, xv.w, acc[hh]);
        }
    }
    float *o = reinterpret_cast<float *>(smem);              // [G][D], over the dead merge area
#pragma unroll
    for (int hh = 0; hh < HPT; ++hh)
        o[(h0 + hh) * D + i] = acc[hh];
    __syncthreads();
    *o_out = o;
}

}  // namespace win
}  // namespace kvq
