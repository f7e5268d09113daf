// Write path for chunks of bfloat16 keys/values: the token-block x d x d transform on
// tensor cores, then clipping, affine quantization and the fixed-width store
// ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms", sections 4.2 and 5.3;
// "Spend Bits Where Queries Look", "Three requirements", item 3).
//
// CTA = (KV head, one of {K, V}), 4 warps, grid-stride over 16-token tiles of the
// flattened (sequence, new token) list. Per CTA, T is staged once in shared memory as two
// bfloat16 pieces T = T_hi + T_lo (16 significant bits; rows padded by 16 bytes so that
// ldmatrix is free of bank conflicts). Per tile (one warp):
//   X~[16 tok x d] = X[16 x d] . (T_hi + T_lo)^T on mma.sync m16n8k16 (bf16, f32 acc);
//   the inputs are bfloat16, so X is exact and only T is split.
//   Each token's d values sit in the 4 lanes of a quad: order statistics by a quad-wide
//   min/max (kappa = 0) or a top-2 merge (kappa = 1) or kappa+1 extraction rounds; the
//   QuEST INT quantizer takes the group RMS from a float64 sum of squares instead.
//   s = f32(f32(hi - lo) / qmax), s_h = f16(s), z_h = f16(lo), as the definition; codes
//   c = clamp(rint(f32(x - z)/s)) computed as (x - z) * rcp_rn(s), which differs from the
//   IEEE quotient by under 2 ulp; a value within 2^-20 of a rounding tie is recomputed
//   with IEEE division, so the codes are those of the definition bit for bit.
//   Codes are packed in registers: a K-row word from the quad's 4 lanes (two xor
//   shuffles), a V-tile half from one lane (it holds every column of that half), and
//   stored whole.
#include "kvq_common.cuh"
#include "kvq_ptx.cuh"

namespace kvq {

namespace {

constexpr int kMmaWarps = 4;

template <int D>
struct MmaSmem {
    static constexpr int TS = D + 8;       // bf16 per staged row
    __nv_bfloat16 Thi[D * TS];
    __nv_bfloat16 Tlo[D * TS];
    __nv_bfloat16 X[kMmaWarps][2][16 * TS];      // double-buffered input rows
};

__device__ __forceinline__ void quad_minmax(float &mn, float &mx)
{
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
}

// Merge (a1 <= a2) with (b1 <= b2): the two smallest of the four.
__device__ __forceinline__ void merge2_min(float &a1, float &a2, float b1, float b2)
{
    const float lo = fminf(a1, b1);
    const float hi = fminf(fmaxf(a1, b1), fminf(a2, b2));
    a1 = lo;
    a2 = hi;
}

// kappa-th smallest (MAX = false) / largest of the values of one quad (4 lanes x NV),
// by kappa+1 rounds of "quad-wide extreme, then remove one instance" (general kappa).
template <int NV, bool MAX>
__device__ __forceinline__ float quad_order_stat(const float (&vals)[NV], int kappa, int lane)
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
            const float x = vals[i];
            if (bi < 0 || (MAX ? (x > best) : (x < best))) {
                best = x;
                bi = i;
            }
        }
        m = best;
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            const float o = __shfl_xor_sync(0xffffffffu, m, off);
            m = MAX ? fmaxf(m, o) : fminf(m, o);
        }
        const uint32_t quad = 0xFu << (lane & ~3);
        const uint32_t holders = __ballot_sync(0xffffffffu, bi >= 0 && best == m) & quad;
        if (holders && lane == __ffs(holders) - 1)
            removed |= 1u << bi;
    }
    return m;
}

// K row: little-endian bit stream, column j at bit BITS*j. A 32-bit word holds 32/BITS
// columns, i.e. 2 (2-bit) or 1 (4-bit) n-tiles of 8 columns; lane t of the quad holds
// columns 8nt + 2t + {0, 1} of every n-tile, so the quad's 4 lanes together hold a word:
// partial words are OR-ed over the quad and lane t stores words t, t+4, ...
template <int D, int BITS, int NV>
__device__ __forceinline__ void store_k_row(const uint32_t (&cq)[NV], uint32_t *dst, int t, bool ok)
{
    constexpr int WORDS = D * BITS / 32, TPW = 4 / BITS;
#pragma unroll
    for (int w = 0; w < WORDS; ++w) {
        uint32_t part = 0;
#pragma unroll
        for (int q = 0; q < TPW; ++q) {
            const int nt = w * TPW + q;
            part |= cq[2 * nt] << (BITS * (8 * q + 2 * t));
            part |= cq[2 * nt + 1] << (BITS * (8 * q + 2 * t + 1));
        }
        part |= __shfl_xor_sync(0xffffffffu, part, 1);
        part |= __shfl_xor_sync(0xffffffffu, part, 2);
        if (ok && (w & 3) == t)
            dst[w] = part;
    }
}

// V tile halves of one token: half (gq, rr) holds dims 8(E rr + s) + gq at bits BITS*s,
// E = 16/BITS. Lane t holds gq = 2t and 2t+1 of every n-tile, so both are local.
template <int D, int BITS, int NV>
__device__ __forceinline__ void store_v_halves(const uint32_t (&cq)[NV], unsigned char *tile_base,
                                               int tok, int t)
{
    constexpr int E = 16 / BITS, W = D * BITS / 128;
#pragma unroll
    for (int odd = 0; odd < 2; ++odd)
#pragma unroll
        for (int rr = 0; rr < W; ++rr) {
            uint32_t val = 0;
#pragma unroll
            for (int s2 = 0; s2 < E; ++s2)
                val |= cq[2 * (E * rr + s2) + odd] << (BITS * s2);
            *reinterpret_cast<uint16_t *>(tile_base + v_half_offset(D, BITS, tok, 2 * t + odd, rr)) =
                (uint16_t)val;
        }
}

template <int D>
__global__ void __launch_bounds__(kMmaWarps * 32)
append_mma_kernel(const __nv_bfloat16 *__restrict__ k_in, const __nv_bfloat16 *__restrict__ v_in,
                  const float *__restrict__ Tk, const float *__restrict__ Tv, int B, int n,
                  int Hkv, int T_cap, int bits_k, int bits_v, int group, int kappa,
                  uint8_t *__restrict__ k_codes, uint32_t *__restrict__ k_sz,
                  uint8_t *__restrict__ v_codes, uint32_t *__restrict__ v_sz,
                  const int32_t *__restrict__ pos, int32_t *dev_err, PageMap pm)
{
    using Sm = MmaSmem<D>;
    constexpr int TS = Sm::TS, NT = D / 8, NV = 2 * NT;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Sm &sm = *reinterpret_cast<Sm *>(smem_raw);

    const int h = blockIdx.y, which = blockIdx.z;
    const __nv_bfloat16 *in = which ? v_in : k_in;
    const float *T = which ? Tv : Tk;
    const int bits = which ? bits_v : bits_k;
    const int qmax = (1 << bits) - 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const long total = (long)B * n;
    const long tiles = (total + 15) / 16;
    const int ng = D / group;

    // ---- T -> bf16 hi/lo pieces, rows padded (T row i = output dim i)
    {
        const float4 *T4 = reinterpret_cast<const float4 *>(T + (size_t)h * D * D);
        constexpr int N4 = D * D / 4 / (kMmaWarps * 32);
#pragma unroll 8
        for (int it = 0; it < N4; ++it) {
            const int idx4 = threadIdx.x + kMmaWarps * 32 * it;
            const float4 v4 = T4[idx4];
            const int i = (4 * idx4) / D, j = (4 * idx4) % D;
            const float xs[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat16 hi = __float2bfloat16_rn(xs[e]);
                sm.Thi[i * TS + j + e] = hi;
                sm.Tlo[i * TS + j + e] = __float2bfloat16_rn(xs[e] - __bfloat162float(hi));
            }
        }
    }
    __syncthreads();

    constexpr int CH = D / 8;                         // 16-byte chunks per input row
    // cp.async the 16 input rows of `tile` into buffer `buf` (rows past the end zero-fill)
    auto fetch = [&](long tile, int buf) {
        __nv_bfloat16 *Xb = sm.X[warp][buf];
#pragma unroll
        for (int c = lane; c < 16 * CH; c += 32) {
            const int r = c / CH, ch = c % CH;
            const long u = tile * 16 + r;
            const __nv_bfloat16 *src = in;
            uint32_t bytes = 0;
            if (u < total) {
                const long b = u / n, i = u % n;
                src = in + (((size_t)b * n + i) * Hkv + h) * D + 8 * ch;
                bytes = 16;
            }
            cp_async16(Xb + r * TS + 8 * ch, src, bytes);
        }
        cp_async_commit();
    };
    const long stride = (long)gridDim.x * kMmaWarps;
    long tile = (long)blockIdx.x * kMmaWarps + warp;
    int buf = 0;
    if (tile < tiles)
        fetch(tile, 0);
    for (; tile < tiles; tile += stride, buf ^= 1) {
        const long u0 = tile * 16;
        if (tile + stride < tiles) {
            fetch(tile + stride, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        const __nv_bfloat16 *X = sm.X[warp][buf];

        // ---- X~ = X . T^T on tensor cores
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[nt][i] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[4];
            ldmatrix_x4(a, X + (lane & 15) * TS + 16 * ks + 8 * (lane >> 4));
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                const int trow = 16 * np + 8 * ((lane >> 4) & 1) + (lane & 7);
                const int tcol = 16 * ks + 8 * ((lane >> 3) & 1);
                uint32_t bh[4], bl[4];
                ldmatrix_x4(bh, sm.Thi + trow * TS + tcol);
                ldmatrix_x4(bl, sm.Tlo + trow * TS + tcol);
                mma_bf16(acc[2 * np], a[0], a[1], a[2], a[3], bh[0], bh[1]);
                mma_bf16(acc[2 * np + 1], a[0], a[1], a[2], a[3], bh[2], bh[3]);
                mma_bf16(acc[2 * np], a[0], a[1], a[2], a[3], bl[0], bl[1]);
                mma_bf16(acc[2 * np + 1], a[0], a[1], a[2], a[3], bl[2], bl[3]);
            }
        }

        // ---- sequence and position of the tile's first token (one division per tile)
        int b0, i0;
        if (total <= 0x7fffffffL) {
            const unsigned uu = (unsigned)u0, nn = (unsigned)n;
            b0 = (int)(uu / nn);
            i0 = (int)(uu - (unsigned)b0 * nn);
        } else {
            b0 = (int)(u0 / n);
            i0 = (int)(u0 - (long)b0 * n);
        }

        // ---- per token (rows g and g+8): clip range, scale/zero, codes, packed stores
#pragma unroll
        for (int tk = 0; tk < 2; ++tk) {
            const int r = g + 8 * tk;
            const long u = u0 + r;
            bool ok = u < total;
            int b = b0, i = i0 + r, p0 = 0;
            while (i >= n) {                          // the tile may run into later sequences
                i -= n;
                ++b;
            }
            long long row = 0;                        // token slot in the planes
            if (ok) {
                p0 = pos[b];
                if (p0 < 0 || (long)p0 + n > T_cap) {
                    if (i == 0 && t == 0)
                        flag(dev_err, KVQ_DEVERR_POS_RANGE);
                    ok = false;
                } else {
                    row = cache_row(pm, b, h, Hkv, T_cap, p0 + i);
                    if (row < 0) {
                        if (t == 0)
                            flag(dev_err, KVQ_DEVERR_PAGE_RANGE);
                        ok = false;
                        row = 0;
                    }
                }
            }
            // this lane's values of the token: columns 8nt + 2t + {0, 1}
            float x[NV];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                x[2 * nt] = acc[nt][2 * tk];
                x[2 * nt + 1] = acc[nt][2 * tk + 1];
            }
            uint32_t cq[NV];                          // codes of this lane's columns
            for (int gr = 0; gr < ng; ++gr) {
                const int c0 = gr * group, c1 = c0 + group;    // columns of this group
                float lo = 0.f, hi = 0.f;
                float quest_s = 0.f;
                if (kappa == kQuestClip) {
                    // QuEST INT: float64 sum of squares of the group over the quad
                    double ss = 0.0;
#pragma unroll
                    for (int e = 0; e < NV; ++e) {
                        const int col = 8 * (e >> 1) + 2 * t + (e & 1);
                        if (col >= c0 && col < c1)
                            ss = fma((double)x[e], (double)x[e], ss);
                    }
                    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
                    const float rms = __double2float_rn(sqrt(ss / (double)group));
                    quest_s = __fmul_rn(rms, quest_delta(bits));
                } else if (kappa == 0) {
                    lo = INFINITY;
                    hi = -INFINITY;
#pragma unroll
                    for (int e = 0; e < NV; ++e) {
                        const int col = 8 * (e >> 1) + 2 * t + (e & 1);
                        if (col >= c0 && col < c1) {
                            lo = fminf(lo, x[e]);
                            hi = fmaxf(hi, x[e]);
                        }
                    }
                    quad_minmax(lo, hi);
                } else if (kappa == 1) {
                    float m1 = INFINITY, m2 = INFINITY, M1 = -INFINITY, M2 = -INFINITY;
#pragma unroll
                    for (int e = 0; e < NV; ++e) {
                        const int col = 8 * (e >> 1) + 2 * t + (e & 1);
                        if (col >= c0 && col < c1) {
                            const float v = x[e];
                            m2 = fminf(m2, fmaxf(m1, v));
                            m1 = fminf(m1, v);
                            M2 = fmaxf(M2, fminf(M1, v));
                            M1 = fmaxf(M1, v);
                        }
                    }
#pragma unroll
                    for (int off = 1; off <= 2; off <<= 1) {
                        const float o1 = __shfl_xor_sync(0xffffffffu, m1, off);
                        const float o2 = __shfl_xor_sync(0xffffffffu, m2, off);
                        const float O1 = __shfl_xor_sync(0xffffffffu, M1, off);
                        const float O2 = __shfl_xor_sync(0xffffffffu, M2, off);
                        merge2_min(m1, m2, o1, o2);
                        float nM1 = -M1, nM2 = -M2;
                        merge2_min(nM1, nM2, -O1, -O2);
                        M1 = -nM1;
                        M2 = -nM2;
                    }
                    lo = m2;
                    hi = M2;
                } else {
                    float vmin[NV], vmax[NV];
#pragma unroll
                    for (int e = 0; e < NV; ++e) {
                        const int col = 8 * (e >> 1) + 2 * t + (e & 1);
                        const bool in_g = col >= c0 && col < c1;
                        vmin[e] = in_g ? x[e] : INFINITY;
                        vmax[e] = in_g ? x[e] : -INFINITY;
                    }
                    lo = quad_order_stat<NV, false>(vmin, kappa, lane);
                    hi = quad_order_stat<NV, true>(vmax, kappa, lane);
                }
                __half sh, zh;
                bool finite;
                if (kappa == kQuestClip) {
                    sh = __float2half_rn(quest_s);
                    zh = __float2half_rn(__fmul_rn(-0.5f * (float)qmax, __half2float(sh)));
                    finite = isfinite(quest_s);
                } else {
                    const float range = __fsub_rn(hi, lo);
                    const float s = __fdiv_rn(range, (float)qmax);
                    sh = __float2half_rn(s);
                    zh = __float2half_rn(lo);
                    finite = isfinite(range) && isfinite(s);
                }
                const float sf = __half2float(sh), zf = __half2float(zh);
                if (ok && !finite && t == 0)
                    flag(dev_err, KVQ_DEVERR_NONFINITE);
                const bool zero = !finite || sf == 0.f;
                const float rc = zero ? 0.f : __frcp_rn(sf);
#pragma unroll
                for (int e = 0; e < NV; ++e) {
                    const int col = 8 * (e >> 1) + 2 * t + (e & 1);
                    if (col < c0 || col >= c1)
                        continue;
                    int c = 0;
                    if (!zero) {
                        const float dlt = __fsub_rn(x[e], zf);
                        float y = __fmul_rn(dlt, rc);
                        float k = rintf(y);
                        // within 2^-20 relative of a tie: take the IEEE quotient
                        if (fabsf(y - k) >= 0.5f - 9.5367431640625e-07f * fmaxf(fabsf(y), 1.f)) {
                            y = __fdiv_rn(dlt, sf);
                            k = rintf(y);
                        }
                        c = (int)fminf(fmaxf(k, 0.f), (float)qmax);
                    }
                    cq[e] = (uint32_t)c;
                }
                if (ok && t == 0) {
                    const uint32_t pair = (uint32_t)__half_as_ushort(sh) |
                                          ((uint32_t)__half_as_ushort(zh) << 16);
                    (which ? v_sz : k_sz)[row * ng + gr] = pair;
                }
            }

            // ---- packed stores, built in registers
            if (!which) {
                uint32_t *dst = reinterpret_cast<uint32_t *>(k_codes + row * (D * bits / 8));
                if (bits == 2)
                    store_k_row<D, 2>(cq, dst, t, ok);
                else
                    store_k_row<D, 4>(cq, dst, t, ok);
            } else if (ok) {
                unsigned char *tile_base =
                    v_codes + (size_t)(row / kTileTokens) * (kTileTokens * D * bits / 8);
                const int tok = (int)(row % kTileTokens);
                if (bits == 2)
                    store_v_halves<D, 2>(cq, tile_base, tok, t);
                else
                    store_v_halves<D, 4>(cq, tile_base, tok, t);
            }
        }
        __syncwarp();
    }
}

template <int D>
cudaError_t launch_mma(const void *k, const void *v, const float *Tk, const float *Tv, int B,
                       int n, const kvq_cache *c, int kappa, const int32_t *pos, int32_t *dev_err,
                       cudaStream_t st)
{
    const size_t smem = sizeof(MmaSmem<D>);
    static int attr_set = 0;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(append_mma_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        attr_set = 1;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long tiles = ((long)B * n + 15) / 16;
    const int per_sm = D == 64 ? 4 : 2;               // resident CTAs per SM (registers, shared memory)
    long gx = ((long)sms * per_sm + 2L * c->Hkv - 1) / (2L * c->Hkv);
    const long need = (tiles + kMmaWarps - 1) / kMmaWarps;
    if (gx > need)
        gx = need;
    if (gx < 1)
        gx = 1;
    dim3 grid((unsigned)gx, (unsigned)c->Hkv, 2);
    append_mma_kernel<D><<<grid, kMmaWarps * 32, smem, st>>>(
        (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, Tk, Tv, B, n, c->Hkv, c->T_cap,
        c->qp.bits_k, c->qp.bits_v, c->qp.group, kappa, (uint8_t *)c->k_codes,
        (uint32_t *)c->k_sz, (uint8_t *)c->v_codes, (uint32_t *)c->v_sz, pos, dev_err,
        PageMap{c->block_table, c->page_tokens, c->num_pages});
    return cudaGetLastError();
}

}  // namespace

cudaError_t append_mma(const void *k, const void *v, const float *Tk, const float *Tv, int B,
                       int n, const kvq_cache *c, int kappa, const int32_t *pos, int32_t *dev_err,
                       cudaStream_t st)
{
    if (c->d == 64)
        return launch_mma<64>(k, v, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
    return launch_mma<128>(k, v, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
}

}  // namespace kvq
