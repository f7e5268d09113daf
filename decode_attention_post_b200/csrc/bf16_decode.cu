// Uncompressed comparator: the same grouped-query decode attention over bfloat16 keys
// and values [B][Hkv][T_cap][d], no transform and no quantization. It is the baseline
// the quantized path is measured against (a 16-bit cache, the "BF16 (uncompressed)"
// row of the NOVA-KV page's results table, is 7.1x larger than the 2-bit layout).
//
// Same split-K structure as the quantized decode: CTA = (split, KV head, sequence),
// 4 warps, each warp streams 16-token blocks through a private 3-stage ring. Rows are
// brought in by per-row cp.async.bulk copies (one per lane) into rows padded by 16
// bytes so that ldmatrix reads are free of bank conflicts. Q.K: S^T[16 tok x 8] from
// ldmatrix K fragments and the bfloat16 query; P.V: O^T[d x 2G] from ldmatrix.trans
// V fragments and P split into bfloat16 hi/lo pieces.
#include "kvq_common.cuh"
#include "kvq_ptx.cuh"
#include "decode_shapes.h"

namespace kvq {

namespace {

constexpr int kBWarps = 4;
constexpr int kBStages = 3;
constexpr int kBBlk = 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 4.0f;

template <int D, int G>
struct BCfg {
    static constexpr int RSTRIDE = D * 2 + 16;           // bytes per padded row
    static constexpr int STAGE = 2 * kBBlk * RSTRIDE;    // K rows then V rows
    static constexpr int KSTEPS = D / 16;
    static constexpr int MT = D / 16;
    static constexpr int NTQ = (G + 7) / 8;              // n-tiles of the score product
    static constexpr int NTP = (2 * G) / 8;              // n-tiles of (hi, lo) P columns
    static constexpr int PSTRIDE = kBBlk + 8;            // halves per P^T column
    static constexpr int PBUF = 2 * G * PSTRIDE * 2;
    static constexpr int RING = kBWarps * kBStages * STAGE;
    static constexpr int MERGE = kBWarps * G * (D + 2) * 4;
    static constexpr int SMEM = (RING > MERGE ? RING : MERGE) + kBWarps * PBUF +
                                kBWarps * kBStages * 8 + 16;
};

template <int D, int G>
__global__ void __launch_bounds__(kBWarps * 32, 2)
bf16_decode_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ K,
                   const __nv_bfloat16 *__restrict__ V, int B, int Hq, int Hkv, int T_cap,
                   const int32_t *__restrict__ seqlens, int max_seqlen, __nv_bfloat16 *out,
                   float *part, int *ticket, int nsplit, int split_tokens, int32_t *dev_err)
{
    using C = BCfg<D, G>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *ring = smem_raw;
    __nv_bfloat16 *pbuf_all =
        reinterpret_cast<__nv_bfloat16 *>(smem_raw + (C::RING > C::MERGE ? C::RING : C::MERGE));
    uint64_t *bars_all = reinterpret_cast<uint64_t *>(reinterpret_cast<unsigned char *>(pbuf_all) +
                                                      kBWarps * C::PBUF);
    int *flag_smem = reinterpret_cast<int *>(bars_all + kBWarps * kBStages);

    const int sigma = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const size_t pair = (size_t)b * Hkv + h;

    int seqlen = seqlens[b];
    if (seqlen < 0 || seqlen > max_seqlen) {
        if (sigma == 0 && h == 0 && threadIdx.x == 0)
            flag(dev_err, KVQ_DEVERR_SEQLEN_CLAMPED);
        seqlen = seqlen < 0 ? 0 : max_seqlen;
    }
    const int t_begin = sigma * split_tokens;
    if (t_begin >= seqlen) {
        if (sigma == 0)
            for (int idx = threadIdx.x; idx < G * D; idx += kBWarps * 32)
                out[((size_t)b * Hq + h * G + idx / D) * D + idx % D] = __float2bfloat16_rn(0.f);
        return;
    }
    const int t_end = min(t_begin + split_tokens, seqlen);
    const int nsplit_b = (seqlen + split_tokens - 1) / split_tokens;
    const int nblk = (t_end - t_begin + kBBlk - 1) / kBBlk;
    const int my_nblk = nblk > warp ? (nblk - warp + kBWarps - 1) / kBWarps : 0;

    unsigned char *wring = ring + warp * kBStages * C::STAGE;
    __nv_bfloat16 *pbuf = pbuf_all + warp * (C::PBUF / 2);
    uint64_t *bars = bars_all + warp * kBStages;
    const __nv_bfloat16 *Kp = K + pair * (size_t)T_cap * D;
    const __nv_bfloat16 *Vp = V + pair * (size_t)T_cap * D;

    if (lane == 0) {
        for (int s = 0; s < kBStages; ++s)
            mbar_init(&bars[s], 1);
        mbar_fence_init();
    }
    __syncwarp();

    // Every lane takes part: lane i < 16 brings K row i, lane i >= 16 V row i-16.
    // Rows past the end of the sequence are zero-filled instead of copied.
    auto issue = [&](int jj, int s) {
        const int tok0 = t_begin + (warp + jj * kBWarps) * kBBlk;
        const int nvalid = min(kBBlk, t_end - tok0);
        unsigned char *st = wring + s * C::STAGE;
        if (lane == 0)
            mbar_arrive_expect_tx(&bars[s], 2u * nvalid * D * 2);
        __syncwarp();
        const int r = lane & 15;
        unsigned char *dst = st + (lane >> 4) * kBBlk * C::RSTRIDE + r * C::RSTRIDE;
        if (r < nvalid) {
            const __nv_bfloat16 *src = (lane < 16 ? Kp : Vp) + (size_t)(tok0 + r) * D;
            bulk_g2s(dst, src, D * 2, &bars[s]);
        } else {
            for (int i = 0; i < D * 2; i += 16)
                *reinterpret_cast<uint4 *>(dst + i) = make_uint4(0, 0, 0, 0);
        }
    };
    for (int jj = 0; jj < kBStages && jj < my_nblk; ++jj)
        issue(jj, jj);

    // query operand: B[k = dim][n = head], zero columns past G
    uint32_t qB[C::NTQ][C::KSTEPS][2];
#pragma unroll
    for (int nt = 0; nt < C::NTQ; ++nt) {
        const int head = 8 * nt + g;
        const __nv_bfloat16 *qv = q + ((size_t)b * Hq + h * G + (head < G ? head : 0)) * D;
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks) {
            uint32_t v0 = *reinterpret_cast<const uint32_t *>(qv + 16 * ks + 2 * t);
            uint32_t v1 = *reinterpret_cast<const uint32_t *>(qv + 16 * ks + 2 * t + 8);
            qB[nt][ks][0] = head < G ? v0 : 0u;
            qB[nt][ks][1] = head < G ? v1 : 0u;
        }
    }
    const float sl2 = kLog2e * rsqrtf((float)D);
    const bool owner = 2 * t < G;               // threads whose score columns are heads
    const int hp = owner ? 2 * t : 0;

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float O[C::MT][C::NTP][4];
#pragma unroll
    for (int m = 0; m < C::MT; ++m)
#pragma unroll
        for (int nt = 0; nt < C::NTP; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                O[m][nt][i] = 0.f;

    // zero the P^T buffer once: columns of non-owner threads stay zero
    for (int i = lane; i < C::PBUF / 4; i += 32)
        reinterpret_cast<uint32_t *>(pbuf)[i] = 0u;
    __syncwarp();

    bool timed_out = false;
    for (int jj = 0; jj < my_nblk; ++jj) {
        const int s = jj % kBStages;
        if (!mbar_wait_bounded(&bars[s], (jj / kBStages) & 1)) {
            timed_out = true;
            for (int k2 = jj + 1; k2 < jj + kBStages && k2 < my_nblk; ++k2)
                mbar_wait_bounded(&bars[k2 % kBStages], (k2 / kBStages) & 1);
            break;
        }
        __syncwarp();                           // zero-filled rows are visible
        const unsigned char *Ks = wring + s * C::STAGE;
        const unsigned char *Vs = Ks + kBBlk * C::RSTRIDE;
        const int tok0 = t_begin + (warp + jj * kBWarps) * kBBlk;

        float S[C::NTQ][4];
#pragma unroll
        for (int nt = 0; nt < C::NTQ; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                S[nt][i] = 0.f;
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks) {
            uint32_t a[4];
            ldmatrix_x4(a, Ks + (lane & 15) * C::RSTRIDE + (16 * ks + 8 * (lane >> 4)) * 2);
#pragma unroll
            for (int nt = 0; nt < C::NTQ; ++nt)
                mma_bf16(S[nt], a[0], a[1], a[2], a[3], qB[nt][ks][0], qB[nt][ks][1]);
        }
        // thread holds tokens g (c0, c1) and g+8 (c2, c3) for heads 2t, 2t+1 (G <= 8)
        float L2[2][2];
        float bm[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
            for (int tk = 0; tk < 2; ++tk) {
                const bool valid = tok0 + g + 8 * tk < t_end;
                L2[tk][hh] = valid ? S[0][2 * tk + hh] * sl2 : -INFINITY;
            }
            bm[hh] = fmaxf(L2[0][hh], L2[1][hh]);
            bm[hh] = fmaxf(bm[hh], __shfl_xor_sync(0xffffffffu, bm[hh], 4));
            bm[hh] = fmaxf(bm[hh], __shfl_xor_sync(0xffffffffu, bm[hh], 8));
            bm[hh] = fmaxf(bm[hh], __shfl_xor_sync(0xffffffffu, bm[hh], 16));
            // G == 4: lanes t >= 2 hold the lo-piece output columns of the heads owned
            // by lane t ^ 2 and follow that lane's running max
            const float from_owner = __shfl_xor_sync(0xffffffffu, bm[hh], 2);
            if (!owner)
                bm[hh] = from_owner;
            if (bm[hh] > m_run[hh] + kLazy) {
                const float alpha = ex2(m_run[hh] - bm[hh]);
                l_run[hh] *= alpha;
#pragma unroll
                for (int m = 0; m < C::MT; ++m)
#pragma unroll
                    for (int nt = 0; nt < C::NTP; ++nt) {
                        O[m][nt][hh] *= alpha;
                        O[m][nt][2 + hh] *= alpha;
                    }
                m_run[hh] = bm[hh];
            }
        }
        if (owner) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int tk = 0; tk < 2; ++tk) {
                    const float p = ex2(L2[tk][hh] - m_run[hh]);
                    l_run[hh] += p;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(p);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
                    pbuf[(hp + hh) * C::PSTRIDE + g + 8 * tk] = hi;
                    pbuf[(G + hp + hh) * C::PSTRIDE + g + 8 * tk] = lo;
                }
        }
        __syncwarp();
        uint32_t pb[C::NTP][2];
#pragma unroll
        for (int nt = 0; nt < C::NTP; ++nt) {
            const __nv_bfloat16 *pc = pbuf + (8 * nt + g) * C::PSTRIDE + 2 * t;
            pb[nt][0] = *reinterpret_cast<const uint32_t *>(pc);
            pb[nt][1] = *reinterpret_cast<const uint32_t *>(pc + 8);
        }
        const int vrow = (lane & 7) + 8 * (lane >> 4);
        const int vcol = 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int m = 0; m < C::MT; ++m) {
            uint32_t a[4];
            ldmatrix_x4_trans(a, Vs + vrow * C::RSTRIDE + (16 * m + vcol) * 2);
#pragma unroll
            for (int nt = 0; nt < C::NTP; ++nt)
                mma_bf16(O[m][nt], a[0], a[1], a[2], a[3], pb[nt][0], pb[nt][1]);
        }
        __syncwarp();
        if (jj + kBStages < my_nblk) {
            fence_proxy_async_smem();
            issue(jj + kBStages, s);
        }
    }
    if (timed_out && lane == 0)
        flag(dev_err, KVQ_DEVERR_WAIT_TIMEOUT);

#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1)
            l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], off);
    // O^T columns: (hi, lo) x G -> thread t holds columns 2t, 2t+1 of every n-tile
    __syncthreads();
    for (int s = 0; s < kBStages && lane == 0; ++s)
        mbar_inval(&bars[s]);
    float *mw = reinterpret_cast<float *>(ring);
    float *lw = mw + kBWarps * G;
    float *ow = lw + kBWarps * G;
    for (int i = threadIdx.x; i < kBWarps * G * D; i += kBWarps * 32)
        ow[i] = 0.f;
    __syncthreads();
    // each (column piece) adds into its head; hi and lo land in the same slot
#pragma unroll
    for (int nt = 0; nt < C::NTP; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int col = 8 * nt + 2 * t + hh;
            const int head = col % G;
#pragma unroll
            for (int m = 0; m < C::MT; ++m) {
                atomicAdd(&ow[(warp * G + head) * D + 16 * m + g], O[m][nt][hh]);
                atomicAdd(&ow[(warp * G + head) * D + 16 * m + 8 + g], O[m][nt][2 + hh]);
            }
        }
    if (owner && g == 0)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            mw[warp * G + hp + hh] = m_run[hh];
            lw[warp * G + hp + hh] = l_run[hh];
        }
    __syncthreads();

    float *mypart = part + (pair * nsplit + sigma) * (size_t)(G * (D + 2));
    for (int idx = threadIdx.x; idx < G * D; idx += kBWarps * 32) {
        const int head = idx / D, dim = idx % D;
        float Mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kBWarps; ++w)
            Mx = fmaxf(Mx, mw[w * G + head]);
        float L = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < kBWarps; ++w) {
            const float mwv = mw[w * G + head];
            if (mwv == -INFINITY)
                continue;
            const float wt = ex2(mwv - Mx);
            L = fmaf(wt, lw[w * G + head], L);
            o = fmaf(wt, ow[(w * G + head) * D + dim], o);
        }
        if (nsplit_b == 1) {
            out[((size_t)b * Hq + h * G + head) * D + dim] = __float2bfloat16_rn(o / L);
        } else {
            mypart[head * (D + 2) + 2 + dim] = o;
            if (dim == 0) {
                mypart[head * (D + 2)] = Mx;
                mypart[head * (D + 2) + 1] = L;
            }
        }
    }
    if (nsplit_b == 1)
        return;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        *flag_smem = (atomicAdd(&ticket[pair], 1) == nsplit_b - 1);
    __syncthreads();
    if (!*flag_smem)
        return;
    __threadfence();
    const float *pall = part + pair * nsplit * (size_t)(G * (D + 2));
    for (int idx = threadIdx.x; idx < G * D; idx += kBWarps * 32) {
        const int head = idx / D, dim = idx % D;
        float Mx = -INFINITY;
        for (int sg = 0; sg < nsplit_b; ++sg)
            Mx = fmaxf(Mx, __ldcg(pall + (size_t)sg * G * (D + 2) + head * (D + 2)));
        float L = 0.f, o = 0.f;
        for (int sg = 0; sg < nsplit_b; ++sg) {
            const float *pp = pall + (size_t)sg * G * (D + 2) + head * (D + 2);
            const float wt = ex2(__ldcg(pp) - Mx);
            L = fmaf(wt, __ldcg(pp + 1), L);
            o = fmaf(wt, __ldcg(pp + 2 + dim), o);
        }
        out[((size_t)b * Hq + h * G + head) * D + dim] = __float2bfloat16_rn(o / L);
    }
}

template <int D, int G>
cudaError_t launch_t(const void *q, int Hq, const void *k, const void *v, int B, int Hkv,
                     int T_cap, const int32_t *seqlens, int max_seqlen, void *out, void *ws,
                     int nsplit, int split_tokens, int32_t *dev_err, cudaStream_t st)
{
    using C = BCfg<D, G>;
    const size_t part_bytes = ((size_t)B * Hkv * nsplit * G * (D + 2) * 4 + 255) & ~(size_t)255;
    int *ticket = reinterpret_cast<int *>(static_cast<unsigned char *>(ws) + part_bytes);
    cudaError_t e = cudaMemsetAsync(ticket, 0, (size_t)B * Hkv * 4, st);
    if (e != cudaSuccess)
        return e;
    static int attr_set = 0;
    if (!attr_set) {
        e = cudaFuncSetAttribute(bf16_decode_kernel<D, G>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess)
            return e;
        attr_set = 1;
    }
    dim3 grid(nsplit, Hkv, B);
    bf16_decode_kernel<D, G><<<grid, kBWarps * 32, C::SMEM, st>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, B, Hq, Hkv,
        T_cap, seqlens, max_seqlen, (__nv_bfloat16 *)out, (float *)ws, ticket, nsplit,
        split_tokens, dev_err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bf16_decode(const void *q, int Hq, const void *k, const void *v, int B,
                               int Hkv, int T_cap, int d, const int32_t *seqlens, int max_seqlen,
                               void *out, void *ws, int nsplit, int split_tokens,
                               int32_t *dev_err, cudaStream_t st)
{
    const int G = Hq / Hkv;
#define KVQ_B16(DD, GG)                                                                        \
    if (d == DD && G == GG)                                                                    \
        return launch_t<DD, GG>(q, Hq, k, v, B, Hkv, T_cap, seqlens, max_seqlen, out, ws, nsplit, \
                                split_tokens, dev_err, st);
    KVQ_B16(128, 4)
    KVQ_B16(128, 8)
    KVQ_B16(64, 4)
    KVQ_B16(64, 8)
#undef KVQ_B16
    return cudaErrorInvalidValue;
}

}  // namespace kvq
