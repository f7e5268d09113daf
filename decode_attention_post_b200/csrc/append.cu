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
//      rounds of a warp-wide min (max) with removal of one instance (exact, ties safe).
//   4. Scale, zero-point and codes use IEEE float32 division (__fdiv_rn) and rintf
//      (ties to even), so they match the float64 definition bit for bit.
//   5. Codes are gathered through shared memory and written as whole 32-bit words
//      (K rows) or whole 16-bit halves (V tiles); every token owns whole bytes, so
//      no read-modify-write is needed even for single-token appends. The token slot
//      comes from the contiguous layout or, for a paged cache, the block table.
#include "kvq_common.cuh"

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
    uint8_t codes[kAppendWarps][D];
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

template <int D, int TPW>
__global__ void __launch_bounds__(kAppendThreads)
append_fp32_kernel(const void *__restrict__ k_in, const void *__restrict__ v_in, int in_bf16,
                   const float *__restrict__ Tk, const float *__restrict__ Tv, int B, int n,
                   int Hkv, int T_cap, int bits_k, int bits_v, int group, int kappa,
                   uint8_t *__restrict__ k_codes, uint32_t *__restrict__ k_sz,
                   uint8_t *__restrict__ v_codes, uint32_t *__restrict__ v_sz,
                   const int32_t *__restrict__ pos, int32_t *dev_err, PageMap pm)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
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
    const int ng = D / group;
    const int qmax = (1 << bits) - 1;

    if (T) {
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
    }

    for (long tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const long u0 = tile * kTokPerTile;
        __syncthreads();                        // previous tile's readers are done
#pragma unroll
        for (int it = 0; it < (kTokPerTile * D + kAppendThreads - 1) / kAppendThreads; ++it) {
            const int idx = threadIdx.x + kAppendThreads * it;
            if (idx >= kTokPerTile * D)
                break;
            const int tk = idx / D, j = idx % D;
            const long u = u0 + tk;
            float x = 0.f;
            if (u < total) {
                const long b = u / n, i = u % n;
                x = load_in(in, in_bf16, (((size_t)b * n + i) * Hkv + h) * D + j);
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
            const int p0 = pos[b];
            if (p0 < 0 || (long)p0 + n > T_cap) {
                if (i == 0 && lane == 0)
                    flag(dev_err, KVQ_DEVERR_POS_RANGE);
                continue;
            }
            const int t = p0 + i;
            const long long row = cache_row(pm, b, h, Hkv, T_cap, t);
            if (row < 0) {
                if (lane == 0)
                    flag(dev_err, KVQ_DEVERR_PAGE_RANGE);
                continue;
            }
            for (int gr = 0; gr < ng; ++gr) {
                // group gr covers dims [gr*group, (gr+1)*group), i.e. r in [r0, r0+nr);
                // dims outside the group are padded with +-inf so they are never picked.
                const int r0 = gr * group / 32, nr = group / 32;
                float vmin[R], vmax[R];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const bool ing = r >= r0 && r < r0 + nr;
                    vmin[r] = ing ? acc[q][r] : INFINITY;
                    vmax[r] = ing ? acc[q][r] : -INFINITY;
                }
                const float lo = order_stat<R, false>(vmin, kappa, lane);
                const float hi = order_stat<R, true>(vmax, kappa, lane);
                const float range = __fsub_rn(hi, lo);
                const float s = __fdiv_rn(range, (float)qmax);
                const __half sh = __float2half_rn(s);
                const __half zh = __float2half_rn(lo);
                const float sf = __half2float(sh), zf = __half2float(zh);
                const bool finite = isfinite(range) && isfinite(s);
                if (!finite && lane == 0)
                    flag(dev_err, KVQ_DEVERR_NONFINITE);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (r < r0 || r >= r0 + nr)
                        continue;
                    int c = 0;
                    if (finite && sf != 0.f) {
                        float y = __fdiv_rn(__fsub_rn(acc[q][r], zf), sf);
                        float cr = rintf(y);
                        cr = fminf(fmaxf(cr, 0.f), (float)qmax);
                        c = (int)cr;
                    }
                    sm.codes[warp][lane + 32 * r] = (uint8_t)c;
                }
                if (lane == 0) {
                    uint32_t pair = (uint32_t)__half_as_ushort(sh) |
                                    ((uint32_t)__half_as_ushort(zh) << 16);
                    (which ? v_sz : k_sz)[row * ng + gr] = pair;
                }
            }
            __syncwarp();
            if (!which) {
                const int words = D * bits / 32, cpw = 32 / bits;
                if (lane < words) {
                    uint32_t w = 0;
                    for (int e = 0; e < cpw; ++e)
                        w |= (uint32_t)sm.codes[warp][lane * cpw + e] << (bits * e);
                    reinterpret_cast<uint32_t *>(k_codes + row * (D * bits / 8))[lane] = w;
                }
            } else {
                const int E = 16 / bits, halves = D / E;
                if (lane < halves) {
                    const int gq = lane & 7, r = lane >> 3;
                    uint32_t hv = 0;
                    for (int s2 = 0; s2 < E; ++s2)
                        hv |= (uint32_t)sm.codes[warp][8 * (E * r + s2) + gq] << (bits * s2);
                    const size_t tile_base =
                        (size_t)(row / kTileTokens) * (kTileTokens * D * bits / 8);
                    const int off = v_half_offset(D, bits, (int)(row % kTileTokens), gq, r);
                    *reinterpret_cast<uint16_t *>(v_codes + tile_base + off) = (uint16_t)hv;
                }
            }
            __syncwarp();
        }
    }
}

template <int D, int TPW>
cudaError_t launch_append_fp32(const void *k, const void *v, int in_bf16, const float *Tk,
                               const float *Tv, int B, int n, const kvq_cache *c, int kappa,
                               const int32_t *pos, int32_t *dev_err, cudaStream_t st)
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
    if (tiles > want * 8)
        gx = (tiles + 7) / 8 < 65535 ? (tiles + 7) / 8 : 65535;
    dim3 grid((unsigned)gx, (unsigned)c->Hkv, 2);
    append_fp32_kernel<D, TPW><<<grid, kAppendThreads, smem, st>>>(
        k, v, in_bf16, Tk, Tv, B, n, c->Hkv, c->T_cap, c->qp.bits_k, c->qp.bits_v, c->qp.group,
        kappa, (uint8_t *)c->k_codes, (uint32_t *)c->k_sz, (uint8_t *)c->v_codes,
        (uint32_t *)c->v_sz, pos, dev_err, PageMap{c->block_table, c->page_tokens, c->num_pages});
    return cudaGetLastError();
}

}  // namespace

cudaError_t append_mma(const void *k, const void *v, const float *Tk, const float *Tv, int B,
                       int n, const kvq_cache *c, int kappa, const int32_t *pos, int32_t *dev_err,
                       cudaStream_t st);

// Chunks of bfloat16 inputs with both transforms go to the tensor-core kernel; float32
// inputs, identity transforms, small (decode-time) appends and unaligned inputs use the
// float32 CUDA-core kernel.
cudaError_t append_launch(const void *k, const void *v, int in_bf16, const float *Tk,
                          const float *Tv, int B, int n, const kvq_cache *c, int kappa,
                          const int32_t *pos, int32_t *dev_err, cudaStream_t st)
{
    const long tokens = (long)B * n;
    const bool a16 = ((uintptr_t)k % 16 == 0) && ((uintptr_t)v % 16 == 0) &&
                     ((uintptr_t)Tk % 16 == 0) && ((uintptr_t)Tv % 16 == 0);
    if (in_bf16 && Tk && Tv && a16 && tokens >= 256)
        return append_mma(k, v, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
    const bool small = tokens <= 2048;
    if (c->d == 64)
        return small ? launch_append_fp32<64, 1>(k, v, in_bf16, Tk, Tv, B, n, c, kappa, pos, dev_err, st)
                     : launch_append_fp32<64, 4>(k, v, in_bf16, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
    return small ? launch_append_fp32<128, 1>(k, v, in_bf16, Tk, Tv, B, n, c, kappa, pos, dev_err, st)
                 : launch_append_fp32<128, 4>(k, v, in_bf16, Tk, Tv, B, n, c, kappa, pos, dev_err, st);
}

}  // namespace kvq
