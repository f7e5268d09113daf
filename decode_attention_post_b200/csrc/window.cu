// Full-precision window of the read path ("WUSH-KV: KV Cache Quantization with
// Data-Adaptive Transforms", section 4.4): attention over the positions a sequence keeps
// in full precision -- the first S_sink positions and those after the quantized middle --
// as one more partial (running max, sum of weights, weighted sum of values) next to the
// splits of the quantized middle, merged by the decode kernel's last split.
//
// One CTA per (KV head, sequence), 4 warps, for the G query heads of the KV head. The
// window is the sink rows present plus every slot of the recent ring, each slot masked by
// the position it holds (the softmax does not depend on the order). Each warp takes
// 16-row tiles: key and value rows staged in shared memory by 16-byte asynchronous
// copies, S = K q on bf16 tensor cores (the query as given, bf16, exact: q . k =
// (T_k^{-T} q) . (T_k k)), logits in log2 units, float32 online softmax, O^T += V^T P^T
// with P as bf16 (hi, lo) pairs; the warps merge in shared memory, T_v is applied once to
// the merged sum so that o is in the value-transform domain like the quantized values.
// When nothing of the sequence is quantized the partial is the whole attention and o / l
// is written as the output.
//
// Ordering with the decode grid that follows: that grid is a programmatic dependent of
// this kernel and its last split reads this partial and counts this kernel's ticket
// increment. This kernel therefore never issues griddepcontrol.launch_dependents: the
// dependent grid's griddepcontrol.wait then returns only after this grid has completed
// and its writes are visible.
#include "kvq_common.cuh"
#include "kvq_ptx.cuh"
#include "decode_shapes.h"

#include <math.h>

namespace kvq {

namespace {

constexpr int kWinWarps = 4;
constexpr int kWinThreads = kWinWarps * 32;
constexpr float kWinLog2e = 1.4426950408889634f;
constexpr int kWinSub = 16;                     // window rows per MMA tile
constexpr float kWinLazy = 4.0f;

template <int D, int G>
struct WinCfg {
    static constexpr int TS = D + 8;            // bf16 per staged row (ldmatrix conflict-free)
    static constexpr int TILE = kWinSub * TS;   // bf16 of one staged 16-row tile
    static constexpr int NT = (2 * G) / 8;      // n-tiles of the value product ((hi, lo) x G)
    static constexpr int NTK = 1;               // n-tiles of the key product (G <= 8 columns)
    static constexpr int KS = D / 16;
    static constexpr int MT = D / 16;
    // per warp: K and V tiles; after the loop the same space holds the warps' partials
    static constexpr int TILES = kWinWarps * 2 * TILE * 2;
    static constexpr int MERGE = kWinWarps * G * (D + 2) * 4;
    static constexpr int SMEM = (TILES > MERGE ? TILES : MERGE) + G * D * 4 + 2 * G * 4;
};

// Row w of the window: w < nsink is sink row w; otherwise ring slot w - nsink, valid when
// the position it holds is in [rec0, L) (slot s holds the position t in [L - R, L) with
// t = s mod R; the others are flushed or not yet written).
struct WinRows {
    const __nv_bfloat16 *sink, *ring;           // [S_sink][D] and [R][D] of this (seq, head)
    int nsink, R, L, rec0;
};

__device__ __forceinline__ bool win_row(const WinRows &wr, int w, int D, const __nv_bfloat16 **row)
{
    if (w < wr.nsink) {
        *row = wr.sink + (size_t)w * D;
        return true;
    }
    const int s = w - wr.nsink;
    int t = wr.L - wr.R + (((s - (wr.L - wr.R)) % wr.R) + wr.R) % wr.R;
    *row = wr.ring + (size_t)s * D;
    return t >= wr.rec0 && t < wr.L;
}

template <int D, int G>
__global__ void __launch_bounds__(kWinThreads) window_kernel(WindowParams W)
{
    using C = WinCfg<D, G>;
    extern __shared__ __align__(16) unsigned char wsm_raw[];
    __nv_bfloat16 *tiles = reinterpret_cast<__nv_bfloat16 *>(wsm_raw);
    float *ofin = reinterpret_cast<float *>(wsm_raw + (C::TILES > C::MERGE ? C::TILES : C::MERGE));
    const int h = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int R = W.S_keep + W.S_flush;

    int L = W.seqlens[b];
    L = L < 0 ? 0 : (L > W.max_seqlen ? W.max_seqlen : L);
    if (L == 0)
        return;                                         // the q prologue wrote zeros
    const int Q = window_quantized(L, W.S_sink, W.S_keep, W.S_flush);
    const size_t pair = (size_t)b * W.Hkv + h;
    WinRows kr, vr;
    kr.nsink = vr.nsink = min(W.S_sink, L);
    kr.R = vr.R = R;
    kr.L = vr.L = L;
    kr.rec0 = vr.rec0 = W.S_sink + Q;
    kr.sink = reinterpret_cast<const __nv_bfloat16 *>(W.k_sink) + pair * W.S_sink * D;
    vr.sink = reinterpret_cast<const __nv_bfloat16 *>(W.v_sink) + pair * W.S_sink * D;
    kr.ring = reinterpret_cast<const __nv_bfloat16 *>(W.k_recent) + pair * R * D;
    vr.ring = reinterpret_cast<const __nv_bfloat16 *>(W.v_recent) + pair * R * D;
    // rows to scan: the sink rows present, then every ring slot (masked by position)
    const int nrows = kr.nsink + (L > kr.rec0 ? R : 0);
    const int ntiles = (nrows + kWinSub - 1) / kWinSub;
    const float sc = kWinLog2e * rsqrtf((float)D);
    __nv_bfloat16 *ktile = tiles + (size_t)warp * 2 * C::TILE;
    __nv_bfloat16 *vtile = ktile + C::TILE;

    // q of the G heads (bf16, exact) as the B operand of S = K . q: column n = head n
    uint32_t qB[C::NTK][C::KS][2];
#pragma unroll
    for (int nt = 0; nt < C::NTK; ++nt) {
        const int head = 8 * nt + g;
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t v = 0;
                if (head < G)
                    v = *reinterpret_cast<const uint32_t *>(
                        reinterpret_cast<const __nv_bfloat16 *>(W.q) +
                        ((size_t)b * W.Hq + h * G + head) * D + 16 * ks + 8 * hh + 2 * t);
                qB[nt][ks][hh] = v;
            }
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

    for (int tt = warp; tt < ntiles; tt += kWinWarps) {
        const int w0 = tt * kWinSub;
        // ---- stage the tile's key and value rows (16-byte copies). Rows past the end and
        //      ring slots not holding a window position are zero-filled: their weight is 0,
        //      and a never-written slot may hold any bit pattern (0 * NaN would not be 0).
        for (int c = lane; c < 2 * kWinSub * (D / 8); c += 32) {
            const int which = c / (kWinSub * (D / 8)), cc = c % (kWinSub * (D / 8));
            const int rr = cc / (D / 8), ch = cc % (D / 8);
            const __nv_bfloat16 *row = nullptr;
            bool ok = false;
            if (w0 + rr < nrows)
                ok = win_row(which ? vr : kr, w0 + rr, D, &row);
            __nv_bfloat16 *dst = (which ? vtile : ktile) + rr * C::TS + 8 * ch;
            cp_async16(dst, ok ? row + 8 * ch : kr.ring, ok ? 16 : 0);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
        // validity of this lane's two rows (g and g + 8 of the tile)
        const __nv_bfloat16 *dummy;
        const bool va = w0 + g < nrows && win_row(kr, w0 + g, D, &dummy);
        const bool vb = w0 + g + 8 < nrows && win_row(kr, w0 + g + 8, D, &dummy);
        // ---- S[16 x G] = Ktile . q
        float S[C::NTK][4];
#pragma unroll
        for (int nt = 0; nt < C::NTK; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                S[nt][i] = 0.f;
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
            uint32_t a[4];
            ldmatrix_x4(a, ktile + (lane & 15) * C::TS + 16 * ks + 8 * (lane >> 4));
#pragma unroll
            for (int nt = 0; nt < C::NTK; ++nt)
                mma_bf16(S[nt], a[0], a[1], a[2], a[3], qB[nt][ks][0], qB[nt][ks][1]);
        }
        // The key product's accumulator has row g, columns 2t, 2t+1 = heads 2t, 2t+1 (G <= 8:
        // one n-tile); the value product wants head 4 nt + t on this lane. Its logits come
        // from the quad lane holding that head.
        float la[C::NT], lb[C::NT];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            const int head = 4 * nt + t;
            const int src = (lane & ~3) | ((head & 7) >> 1);
            const float sa0 = __shfl_sync(0xffffffffu, S[0][0], src);
            const float sa1 = __shfl_sync(0xffffffffu, S[0][1], src);
            const float sb0 = __shfl_sync(0xffffffffu, S[0][2], src);
            const float sb1 = __shfl_sync(0xffffffffu, S[0][3], src);
            la[nt] = va ? sc * ((head & 1) ? sa1 : sa0) : -INFINITY;
            lb[nt] = vb ? sc * ((head & 1) ? sb1 : sb0) : -INFINITY;
            float bm = fmaxf(la[nt], lb[nt]);
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
            if (bm > m_run[nt] + kWinLazy) {
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
    float *mw = reinterpret_cast<float *>(wsm_raw);
    float *lw = mw + kWinWarps * G;
    float *ow = lw + kWinWarps * G;
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
    float *stat = ofin + G * D;                         // [G][2]
    for (int idx = threadIdx.x; idx < G * D; idx += kWinThreads) {
        const int head = idx / D, dim = idx % D;
        float Mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWinWarps; ++w)
            Mx = fmaxf(Mx, mw[w * G + head]);
        float Lsum = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < kWinWarps; ++w) {
            const float mwv = mw[w * G + head];
            if (mwv == -INFINITY)
                continue;
            const float wt = ex2(mwv - Mx);
            Lsum = fmaf(wt, lw[w * G + head], Lsum);
            o = fmaf(wt, ow[(w * G + head) * D + dim], o);
        }
        ofin[idx] = o;
        if (dim == 0) {
            stat[2 * head] = Mx;
            stat[2 * head + 1] = Lsum;
        }
    }
    __syncthreads();
    // ---- o = T_v (sum p v), then the partial (or the output); thread per (head, dim i)
    const float *Tv = W.T_v ? W.T_v + (size_t)h * D * D : nullptr;
    float *part = W.part + (pair * W.part_slots + W.slot) * (size_t)(G * (D + 2));
    for (int idx = threadIdx.x; idx < G * D; idx += kWinThreads) {
        const int head = idx / D, i = idx % D;
        float o = ofin[idx];
        if (Tv) {
            const float4 *row = reinterpret_cast<const float4 *>(Tv + (size_t)i * D);
            const float4 *oh = reinterpret_cast<const float4 *>(ofin + head * D);
            float acc = 0.f;
#pragma unroll 8
            for (int j4 = 0; j4 < D / 4; ++j4) {
                const float4 tr = row[j4], ov = oh[j4];
                acc = fmaf(tr.x, ov.x, acc);
                acc = fmaf(tr.y, ov.y, acc);
                acc = fmaf(tr.z, ov.z, acc);
                acc = fmaf(tr.w, ov.w, acc);
            }
            o = acc;
        }
        if (Q == 0) {
            const size_t oi = ((size_t)b * W.Hq + h * G + head) * D + i;
            const float r = o / stat[2 * head + 1];
            if (W.out_bf16)
                reinterpret_cast<__nv_bfloat16 *>(W.out)[oi] = __float2bfloat16_rn(r);
            else
                reinterpret_cast<float *>(W.out)[oi] = r;
        } else {
            part[head * (D + 2) + 2 + i] = o;
            if (i == 0) {
                part[head * (D + 2)] = stat[2 * head];
                part[head * (D + 2) + 1] = stat[2 * head + 1];
            }
        }
    }
    if (Q > 0) {
        // count this partial in the pair's ticket: the decode kernel's last split merges it
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            atomicAdd(&W.ticket[pair], 1);
        }
    }
}

template <int D, int G>
cudaError_t launch_window_t(const WindowParams &W, cudaStream_t st)
{
    static unsigned long long attr_done = 0;
    cudaError_t e = ensure_dynamic_smem(window_kernel<D, G>, WinCfg<D, G>::SMEM, attr_done);
    if (e != cudaSuccess)
        return e;
    window_kernel<D, G><<<dim3(W.Hkv, W.B), kWinThreads, WinCfg<D, G>::SMEM, st>>>(W);
    return cudaGetLastError();
}

// Full-precision store of kvq_window_append: new token i of sequence b is position
// t = len[b] + i; it goes to the sink (t < S_sink) or to the recent ring slot t % R
// (t >= S_sink + Q(len + n), i.e. still in the window after this call's flush). Positions
// flushed by this call are not stored (the flush kernel, launched before, read them from
// the ring or the new tokens). A sequence whose flush is out of range is left untouched.
// One thread per 16-byte chunk of a (sequence, token, KV head, K or V) row.
template <int D>
__global__ void __launch_bounds__(256)
window_store_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new, int B,
                    int n, int Hkv, const int32_t *__restrict__ len, int S_sink, int S_keep,
                    int S_flush, int T_cap, uint4 *k_sink, uint4 *v_sink, uint4 *k_ring,
                    uint4 *v_ring)
{
    constexpr int CH = D / 8;                       // 16-byte chunks per bf16 row
    const int R = S_keep + S_flush;
    const long total = (long)B * n * Hkv * 2 * CH;
    for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long)gridDim.x * blockDim.x) {
        const int c = (int)(idx % CH);
        long r = idx / CH;
        const int which = (int)(r % 2);
        r /= 2;
        const int h = (int)(r % Hkv);
        r /= Hkv;
        const int i = (int)(r % n);
        const int b = (int)(r / n);
        const int L = len[b];
        if (L < 0)
            continue;
        const int qn = window_quantized(L + n, S_sink, S_keep, S_flush);
        if (qn > T_cap)
            continue;
        const int t = L + i;
        const uint4 val = (which ? v_new : k_new)[(((size_t)b * n + i) * Hkv + h) * CH + c];
        if (t < S_sink)
            (which ? v_sink : k_sink)[(((size_t)b * Hkv + h) * S_sink + t) * CH + c] = val;
        else if (t >= S_sink + qn)
            (which ? v_ring : k_ring)[(((size_t)b * Hkv + h) * R + t % R) * CH + c] = val;
    }
}

}  // namespace

cudaError_t launch_window_store(const void *k_new, const void *v_new, int B, int n, int Hkv,
                                int d, const int32_t *len, int S_sink, int S_keep, int S_flush,
                                int T_cap, void *k_sink, void *v_sink, void *k_ring, void *v_ring,
                                cudaStream_t st)
{
    const long total = (long)B * n * Hkv * 2 * (d / 8);
    if (total <= 0)
        return cudaSuccess;
    const long blocks = (total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096;
    auto u4 = [](const void *p) { return reinterpret_cast<const uint4 *>(p); };
    auto m4 = [](void *p) { return reinterpret_cast<uint4 *>(p); };
    if (d == 64)
        window_store_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(
            u4(k_new), u4(v_new), B, n, Hkv, len, S_sink, S_keep, S_flush, T_cap, m4(k_sink),
            m4(v_sink), m4(k_ring), m4(v_ring));
    else
        window_store_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(
            u4(k_new), u4(v_new), B, n, Hkv, len, S_sink, S_keep, S_flush, T_cap, m4(k_sink),
            m4(v_sink), m4(k_ring), m4(v_ring));
    return cudaGetLastError();
}

cudaError_t launch_window(const WindowParams &W, cudaStream_t st)
{
    const int G = W.Hq / W.Hkv;
    if (W.d == 128 && G == 4)
        return launch_window_t<128, 4>(W, st);
    if (W.d == 128 && G == 8)
        return launch_window_t<128, 8>(W, st);
    if (W.d == 64 && G == 4)
        return launch_window_t<64, 4>(W, st);
    if (W.d == 64 && G == 8)
        return launch_window_t<64, 8>(W, st);
    return cudaErrorInvalidValue;
}

}  // namespace kvq
