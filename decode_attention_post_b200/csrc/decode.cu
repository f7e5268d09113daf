// Read path: one decode step of grouped-query attention over the transformed,
// clipped, affine-quantized cache ("WUSH-KV: KV Cache Quantization with Data-Adaptive
// Transforms", sections 1, 4.1, 4.2; "Spend Bits Where Queries Look", "Three
// requirements", item 2: the whole cache is read at every step, so this path is bound
// by HBM bandwidth).
//
// Two kernels per call:
//  qprep   q~ = T_k^{-T} q for every query head (float32), and from it the tensor-core
//          operand fragments (q~ as 16-bit fixed point, two int8 pieces), the logit
//          scale and sum(q~) per head.
//  decode  split-K flash decode. CTA = (KV head, sequence, split), 4 warps; launched as a
//          programmatic dependent of qprep, it requests its first cache blocks before
//          waiting for qprep. Each warp streams 64-token blocks (K codes, K scale/zero,
//          V codes, V scale/zero) with cp.async.bulk into a private 2-stage shared-memory
//          ring (mbarrier completion, bounded waits), and per block:
//            S^T[16 tok x (hi,lo)*G] = Kcodes[16 tok x d] . q_int[d x 2G]  (mma int8,
//                    int32 accumulate: exact)
//            logit = log2(e)/sqrt(d) * (s_t * q~.c_t + z_t * sum q~)       (affine dequant
//                    folded per token: x^ = z + c s)
//            online softmax in float32 (lazy rescale), P' = p * s^v_t split f16 hi/lo
//            O^T[d x (hi,lo)*G] += Vcodes^T[d x 16 tok] . P'^T[16 tok x 2G]  (mma f16)
//          and sum_t p_t z^v_t for the value zero-points.
//          Warps merge in shared memory; splits merge in the last CTA to finish a
//          (sequence, KV head) (atomic ticket, no spin-wait).
//
// Codes reach the tensor cores without unpacking. Keys: masking field position k of
// every byte of a 32-bit word leaves four uint8 operands c * 2^(bits*k); one int8 MMA per
// field position, with the int32 accumulator multiplied by 2^bits between positions,
// sums every code with the same weight. Values: a 2-bit (4-bit) field masked in place is
// the float16 subnormal c * 2^(bits*k) * 2^-24; the per-position factor is compensated
// per output dim. Tensor cores take float16 subnormals exactly.
#include "kvq_common.cuh"
#include "kvq_ptx.cuh"
#include "decode_shapes.h"
#include "window_attn.cuh"

#include <math.h>
#include <type_traits>

namespace kvq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 4.0f;     // rescale the running sums only when the max grows by > 2^4
constexpr int kQprepSeqs = 2;     // sequences per q-prologue CTA (one T_k^{-T} load serves
                                  // 8 G query vectors)

template <int D, int G, int BK, int BV>
struct Cfg {
    static constexpr int KCH = D * BK / 256 > 0 ? D * BK / 256 : 1;  // int8 k-chunks per field
    static constexpr int KS = (8 / BK) * KCH;        // int8 k-steps of the Q.K contraction
    static constexpr int MT = D / 16;                // m-tiles (output dims) of P.V
    static constexpr int NT = (2 * G) / 8;           // n-tiles of (hi, lo) x G columns
    static constexpr int ROWK = D * BK / 8;          // bytes per K row (token)
    static constexpr int WPT = D * BK / 128;         // K words per thread per token
    static constexpr int CPBK = 8 / BK;              // code fields per byte (K)
    static constexpr int CPBV = 8 / BV;
    static constexpr int EV = 16 / BV;               // V codes per 16-bit half
    static constexpr int WV = D * BV / 128;          // V words per token pair in a chunk
    static constexpr int VCH = D * BV / 16;          // bytes per V lane chunk
    static constexpr int VTILE = 16 * D * BV / 8;    // bytes per 16-token V tile
    static constexpr int KC_BYTES = kDecodeBlock * ROWK;
    static constexpr int SZ_BYTES = kDecodeBlock * 4;
    static constexpr int VC_BYTES = kDecodeBlock * D * BV / 8;
    static constexpr int STAGE = KC_BYTES + SZ_BYTES + VC_BYTES + SZ_BYTES;
    static constexpr int QFRAG = NT * KS * 32 * 2;
    static constexpr int RING = kDecodeWarps * kDecodeStages * STAGE;
    static constexpr int MERGE = kDecodeWarps * G * (D + 2) * 4;
    // the ring, the merge area after it, or the window split's tiles and sums
    static constexpr int AREA0 = RING > MERGE ? RING : MERGE;
    static constexpr int WIN = win::Smem<D, G>::BYTES;
    static constexpr int AREA = ((AREA0 > WIN ? AREA0 : WIN) + 15) / 16 * 16;
    // area, stage barriers, one test-hook barrier per warp, merge flag
    static constexpr int SMEM = AREA + kDecodeWarps * (kDecodeStages + 1) * 8 + 16;
    // resident CTAs per SM the register budget targets: kDecodeMinBlocks, or fewer when
    // shared memory (227 KB per SM, 1 KB reserved per CTA) holds fewer
    static constexpr int SMEM_FIT = (227 * 1024) / (SMEM + 1024);
    // d = 128 with G = 8 keeps 64 output accumulators and 32 query-fragment registers per
    // thread: it needs the register budget of 3 CTAs per SM
    static constexpr int REG_FIT = (D == 128 && G == 8) ? 3 : kDecodeMinBlocks;
    static constexpr int MINB = SMEM_FIT < REG_FIT ? SMEM_FIT : REG_FIT;
    static_assert(MINB >= 1, "decode CTA does not fit in shared memory");
    static_assert(STAGE % 16 == 0, "stage alignment");
    static_assert(MERGE % 16 == 0, "merge area alignment");
    static_assert(NT >= 1 && (2 * G) % 8 == 0, "G must be a multiple of 4");
};

// ---------------------------------------------------------------- operand extraction

// Value operand: the float16 pair (token t+4p, token t+4p+8) of output dim 8n + g.
template <int BV, int CPB, int EV, int WV>
__device__ __forceinline__ uint32_t ext_v(const uint32_t *vw, int p, int n)
{
    constexpr uint32_t M = ((1u << BV) - 1u) * 0x00010001u;
    const int r = n / EV, s = n % EV, beta = s / CPB, k = s % CPB;
    const uint32_t w = beta ? (vw[p * WV + r] >> 8) : vw[p * WV + r];
    return w & (M << (BV * k));
}

template <int N>
__device__ __forceinline__ void lds_words(uint32_t (&w)[N], const unsigned char *p)
{
    if constexpr (N == 1) {
        w[0] = *reinterpret_cast<const uint32_t *>(p);
    } else if constexpr (N == 2) {
        uint2 v = *reinterpret_cast<const uint2 *>(p);
        w[0] = v.x;
        w[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < N / 4; ++i) {
            uint4 v = reinterpret_cast<const uint4 *>(p)[i];
            w[4 * i] = v.x;
            w[4 * i + 1] = v.y;
            w[4 * i + 2] = v.z;
            w[4 * i + 3] = v.w;
        }
    }
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t u)
{
    __half2 h = *reinterpret_cast<__half2 *>(&u);
    return __half22float2(h);
}

// ---------------------------------------------------------------- q prologue

// One CTA per (KV head, chunk of `bb` sequences), kQprepThreads threads. M_h is staged in
// shared memory with one cp.async round trip (row stride D+4 floats: the float4 reads of
// row i by 8 consecutive threads fall in distinct banks), the q vectors as qs[j][v].
// Thread (i, part) accumulates output dim i of every vector over one of JP slices of j;
// the slices are summed in shared memory. From q~ = M q (float32) it derives
//   eq  = per head, the power-of-two exponent that brings max|q~| to 2^14..32512,
//   q_int = rint(q~ 2^eq) = 256 hi + lo (int8 hi, lo),
//   frag[nt][ks][lane][2] = int8 hi/lo pieces of q_int laid out as the B operand of the
//                           int8 Q.K product (k-step = field position x k-chunk); n-tile
//                           nt holds heads 4nt..4nt+3, column 2h' = hi and 2h'+1 = lo,
//   cs  = log2(e) / sqrt(d) / (2^(BK*(CPB-1)) 2^eq), per head,
//   w_h = log2(e) / sqrt(d) * sum_j q~_hj,
// zeroes the split-merge ticket of each (sequence, KV head), and writes the zero output
// of every empty sequence. It lets the dependent decode launch start at once: the decode
// kernel requests its first cache blocks, then waits for this grid.
constexpr int kQprepThreads = 256;

template <int D, int G>
struct QprepSmem {
    static constexpr int NVMAX = kQprepSeqs * G;
    static constexpr int JP = kQprepThreads / D;     // slices of the j range
    static constexpr int MSTRIDE = D + 4;
    static constexpr int BYTES = (D * MSTRIDE + D * NVMAX + JP * NVMAX * D + NVMAX) * 4;
};

template <int D, int G, int BK>
__global__ void __launch_bounds__(kQprepThreads)
qprep_kernel(const void *__restrict__ q, int q_bf16, const float *__restrict__ M, int B, int Hq,
             int Hkv, int bb, const int32_t *__restrict__ seqlens, int max_seqlen, void *out,
             int out_bf16, uint32_t *__restrict__ qfrag, float *__restrict__ qscale,
             float *__restrict__ qw, int *__restrict__ ticket, float *__restrict__ qt_out)
{
    constexpr int CPB = 8 / BK, NT = (2 * G) / 8, WPT = D * BK / 128;
    constexpr int KCH = WPT >= 2 ? WPT / 2 : 1, KS = CPB * KCH;
    using S = QprepSmem<D, G>;
    constexpr int NVMAX = S::NVMAX, JP = S::JP, JL = D / JP;
    extern __shared__ __align__(16) float qsm[];
    float *Ms = qsm;                              // [D][D+4]
    float *qs = Ms + D * S::MSTRIDE;              // [D][NVMAX]
    float *pt = qs + D * NVMAX;                   // [JP][NVMAX][D]; slice 0 ends up as q~
    int *eqv = reinterpret_cast<int *>(pt + JP * NVMAX * D);   // [NVMAX] per-head exponent

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int h = blockIdx.x;
    const int b0 = blockIdx.y * bb;
    const int nb = min(bb, B - b0);
    const int NV = nb * G;
    const int tid = threadIdx.x;
    if (M) {
        const float *Mh = M + (size_t)h * D * D;
#pragma unroll
        for (int k = 0; k < D * D / 4 / kQprepThreads; ++k) {
            const int f = tid + k * kQprepThreads, r = f / (D / 4), c = 4 * (f % (D / 4));
            cp_async16(Ms + r * S::MSTRIDE + c, Mh + (size_t)r * D + c, 16);
        }
        cp_async_commit();
    }
    for (int idx = tid; idx < NVMAX * D; idx += kQprepThreads) {
        const int v = idx / D, j = idx % D;
        const int bi = v / G, gg = v % G;
        qs[j * NVMAX + v] =
            v < NV ? load_in(q, q_bf16, ((size_t)(b0 + bi) * Hq + h * G + gg) * D + j) : 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();
    {
        const int i = tid % D, jp = tid / D;          // jp is warp-uniform (D >= 64)
        float acc[NVMAX];
#pragma unroll
        for (int v = 0; v < NVMAX; ++v)
            acc[v] = 0.f;
        if (M) {
            const float4 *Mrow = reinterpret_cast<const float4 *>(Ms + i * S::MSTRIDE + jp * JL);
#pragma unroll 2
            for (int j4 = 0; j4 < JL / 4; ++j4) {
                const float4 m = Mrow[j4];
                const float mj[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const float4 *x =
                        reinterpret_cast<const float4 *>(qs + (jp * JL + 4 * j4 + jj) * NVMAX);
#pragma unroll
                    for (int v4 = 0; v4 < NVMAX / 4; ++v4) {
                        const float4 xv = x[v4];
                        acc[4 * v4] = fmaf(mj[jj], xv.x, acc[4 * v4]);
                        acc[4 * v4 + 1] = fmaf(mj[jj], xv.y, acc[4 * v4 + 1]);
                        acc[4 * v4 + 2] = fmaf(mj[jj], xv.z, acc[4 * v4 + 2]);
                        acc[4 * v4 + 3] = fmaf(mj[jj], xv.w, acc[4 * v4 + 3]);
                    }
                }
            }
        } else if (jp == 0) {
#pragma unroll
            for (int v = 0; v < NVMAX; ++v)
                acc[v] = qs[i * NVMAX + v];
        }
#pragma unroll
        for (int v = 0; v < NVMAX; ++v)
            pt[(jp * NVMAX + v) * D + i] = acc[v];
    }
    __syncthreads();
    if (JP > 1) {
        for (int idx = tid; idx < NV * D; idx += kQprepThreads) {
            float x = pt[idx];
#pragma unroll
            for (int jp = 1; jp < JP; ++jp)
                x += pt[jp * NVMAX * D + idx];
            pt[idx] = x;
        }
        __syncthreads();
    }
    const float *qt = pt;                         // [NVMAX][D]
    if (qt_out) {                                 // q~ itself, for the vector-quantized decode
        for (int idx = tid; idx < NV * D; idx += kQprepThreads) {
            const int v = idx / D, j = idx % D;
            qt_out[((size_t)(b0 + v / G) * Hq + h * G + v % G) * D + j] = qt[idx];
        }
    }
    // per sequence: max |q~| over its G heads; per head: sum of q~
    const int warp = tid >> 5, lane = tid & 31;
    const float sm = rsqrtf((float)D);
    for (int v = warp; v < NV; v += kQprepThreads / 32) {
        float s = 0.f, a = 0.f;
        for (int j = lane; j < D; j += 32) {
            const float x = qt[v * D + j];
            s += x;
            a = fmaxf(a, fabsf(x));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            s += __shfl_xor_sync(0xffffffffu, s, off);
            a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        }
        if (lane == 0) {
            const int bi = v / G, gg = v % G;
            const size_t hq = (size_t)(b0 + bi) * Hq + h * G + gg;
            qw[hq] = kLog2e * sm * s;
            // q_int = rint(q~ 2^eq) with max |q_int| <= 127 * 256, so that q_int = 256 hi + lo
            // with int8 hi and lo: 2^15 when the mantissa of max|q~| allows it, else 2^14
            int ex = 0;
            const float m = a > 0.f ? frexpf(a, &ex) : 0.f;   // a = m 2^ex, m in [0.5, 1)
            const int eq = a > 0.f ? (m <= 0.9921875f ? 15 - ex : 14 - ex) : 0;
            eqv[v] = eq;
            // S = 2^(BK*(CPB-1)) * sum_j c_j q_int_j; cs = log2e * sm / (2^(BK*(CPB-1)) 2^eq)
            qscale[hq] = kLog2e * sm * ldexpf(1.f, -eq - BK * (CPB - 1));
        }
    }
    __syncthreads();
    for (int bi = 0; bi < nb; ++bi) {
        const size_t pair = (size_t)(b0 + bi) * Hkv + h;
        if (tid == 0)
            ticket[pair] = 0;
        uint32_t *fr = qfrag + pair * (size_t)(NT * KS * 64);
        for (int idx = tid; idx < NT * KS * 64; idx += kQprepThreads) {
            const int rho = idx & 1, ln = (idx >> 1) & 31, ks = (idx >> 6) % KS;
            const int nt = (idx >> 6) / KS;
            const int k = ks / KCH, c = ks % KCH;               // field position, k-chunk
            const int g = ln >> 2, t = ln & 3;
            const int head = 4 * nt + g / 2, piece = g & 1;     // columns (hi, lo) per head
            const float *qv = qt + (bi * G + head) * D;
            const float qs2 = ldexpf(1.f, eqv[bi * G + head]);
            uint32_t packed = 0;
            if (WPT >= 2 || rho == 0) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // key slot 16 rho + 4t + j <-> byte 4 WPT t + 8c + 4 rho + j, field k
                    const int byte = WPT >= 2 ? 4 * WPT * t + 8 * c + 4 * rho + j : 4 * t + j;
                    const int qi = (int)rintf(qv[CPB * byte + k] * qs2);
                    const int hi = (qi + 128) >> 8, lo = qi - 256 * hi;   // qi = 256 hi + lo
                    packed |= (uint32_t)(uint8_t)(int8_t)(piece ? lo : hi) << (8 * j);
                }
            }
            fr[idx] = packed;
        }
        // an empty sequence (after clamping to [0, max_seqlen]) attends to nothing: zeros
        const int sl = seqlens[b0 + bi];
        if (sl <= 0 || max_seqlen == 0) {
            for (int idx = tid; idx < G * D; idx += kQprepThreads) {
                const size_t o = ((size_t)(b0 + bi) * Hq + h * G) * D + idx;
                if (out_bf16)
                    reinterpret_cast<__nv_bfloat16 *>(out)[o] = __float2bfloat16_rn(0.f);
                else
                    reinterpret_cast<float *>(out)[o] = 0.f;
            }
        }
    }
}

// ---------------------------------------------------------------- main decode

// The last CTA of a (sequence, KV head) to finish -- a split or the window split --
// merges every partial of the pair: slots 0 .. nsplit_b - 1 hold the splits, the last slot
// the window's. The barrier orders every thread's partial stores before thread 0's
// device-scope fence and ticket; the merging CTA's thread 0 fences after its ticket and
// the barrier orders that before every thread's loads.
template <int D, int G>
__device__ __forceinline__ void merge_if_last(const DecodeParams &P, size_t pair, int b, int h,
                                              int nmerge, int nsplit_b, int *flag_smem)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int last = (atomicAdd(&P.ticket[pair], 1) == nmerge - 1);
        __threadfence();
        *flag_smem = last;
    }
    __syncthreads();
    if (!*flag_smem)
        return;
    const float *pall = P.part + pair * P.part_slots * (size_t)(G * (D + 2));
    for (int idx = threadIdx.x; idx < G * D; idx += kDecodeWarps * 32) {
        const int head = idx / D, dim = idx % D;
        float Mx = -INFINITY;
        for (int i = 0; i < nmerge; ++i) {
            const int sg = i < nsplit_b ? i : P.part_slots - 1;
            Mx = fmaxf(Mx, __ldcg(pall + (size_t)sg * G * (D + 2) + head * (D + 2)));
        }
        float L = 0.f, o = 0.f;
        for (int i = 0; i < nmerge; ++i) {
            const int sg = i < nsplit_b ? i : P.part_slots - 1;
            const float *pp = pall + (size_t)sg * G * (D + 2) + head * (D + 2);
            const float m = __ldcg(pp);
            if (m == -INFINITY)
                continue;                       // a partial that saw no position
            const float wt = ex2(m - Mx);
            L = fmaf(wt, __ldcg(pp + 1), L);
            o = fmaf(wt, __ldcg(pp + 2 + dim), o);
        }
        const size_t oi = ((size_t)b * P.Hq + h * G + head) * D + dim;
        const float r = o / L;
        if (P.out_bf16)
            reinterpret_cast<__nv_bfloat16 *>(P.out)[oi] = __float2bfloat16_rn(r);
        else
            reinterpret_cast<float *>(P.out)[oi] = r;
    }
}

// WIN: the grid has one more split per pair, the full-precision window's (slice z = 0);
// a separate instantiation, so that the plain decode carries none of its code.
template <int D, int G, int BK, int BV, bool WIN>
__global__ void __launch_bounds__(kDecodeWarps * 32, (Cfg<D, G, BK, BV>::MINB)) decode_kernel(DecodeParams P)
{
    using C = Cfg<D, G, BK, BV>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *ring = smem_raw;
    uint64_t *bars_all = reinterpret_cast<uint64_t *>(smem_raw + C::AREA);
    uint64_t *stall_bars = bars_all + kDecodeWarps * kDecodeStages;
    int *flag_smem = reinterpret_cast<int *>(stall_bars + kDecodeWarps);

    // with a window, grid slice z = 0 is the window split (often the pair's longest CTA: it
    // starts first) and z = 1 + sigma the quantized split sigma
    const int h = blockIdx.x, b = blockIdx.y, sigma = (int)blockIdx.z - (WIN ? 1 : 0);
    const int lane = threadIdx.x & 31;
    // the warp index through a broadcast shuffle: the compiler then knows it is the same
    // in every lane, keeps the ring and copy addresses in uniform registers and issues the
    // bulk copies from them directly
    const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
    const int g = lane >> 2, t = lane & 3;
    // Tokens of a 16-token sub-tile held in accumulator rows g and g+8: row 2i holds token
    // i and row 2i+1 token i+8 (i < 4), row 8+2i token i+4 and row 9+2i token i+12. After
    // the 8x8 transposes the value product then sees key slot 2t = token t, 2t+1 = t+8,
    // 2t+8 = t+4, 2t+9 = t+12 -- the token order of the value-code tiles.
    const int ta = (g >> 1) + 8 * (g & 1), tb = ta + 4;
    const size_t pair = (size_t)b * P.Hkv + h;

    int seqlen = P.seqlens[b];
    if (seqlen < 0 || seqlen > P.max_seqlen) {
        if (blockIdx.z == 0 && h == 0 && threadIdx.x == 0)
            flag(P.dev_err, KVQ_DEVERR_SEQLEN_CLAMPED);
        seqlen = seqlen < 0 ? 0 : P.max_seqlen;
    }
    constexpr bool windowed = WIN;
    const int L_all = seqlen;
    if (windowed)                               // the cache holds the quantized middle only
        seqlen = window_quantized(seqlen, P.win_sink, P.win_keep, P.win_flush);
    const int nsplit_b = (seqlen + P.split_tokens - 1) / P.split_tokens;
    const int nmerge = nsplit_b + (windowed ? 1 : 0);   // partials merged for the pair
    if (WIN && sigma < 0) {
        // ---- the window split: its partial in the last slot, or the output when nothing
        //      of the sequence is quantized
        if (L_all == 0)
            return;                             // the prologue wrote zeros
        const float *o, *stat;
        win::attend<D, G>(P, b, h, L_all, seqlen, smem_raw, &o, &stat);
        float *part = P.part + (pair * P.part_slots + P.part_slots - 1) * (size_t)(G * (D + 2));
        for (int idx = threadIdx.x; idx < G * D; idx += kDecodeWarps * 32) {
            const int head = idx / D, dim = idx % D;
            if (nmerge == 1) {
                const size_t oi = ((size_t)b * P.Hq + h * G + head) * D + dim;
                const float r = o[idx] / stat[2 * head + 1];
                if (P.out_bf16)
                    reinterpret_cast<__nv_bfloat16 *>(P.out)[oi] = __float2bfloat16_rn(r);
                else
                    reinterpret_cast<float *>(P.out)[oi] = r;
            } else {
                part[head * (D + 2) + 2 + dim] = o[idx];
                if (dim == 0) {
                    part[head * (D + 2)] = stat[2 * head];
                    part[head * (D + 2) + 1] = stat[2 * head + 1];
                }
            }
        }
        if (nmerge == 1)
            return;
        asm volatile("griddepcontrol.wait;" ::: "memory");   // the prologue zeroed the ticket
        merge_if_last<D, G>(P, pair, b, h, nmerge, nsplit_b, flag_smem);
        return;
    }
    const int t_begin = sigma * P.split_tokens;
    if (t_begin >= seqlen)
        return;                                 // nothing here (the prologue zeroes empty ones)
    const int t_end = min(t_begin + P.split_tokens, seqlen);
    const int nblk = (t_end - t_begin + kDecodeBlock - 1) / kDecodeBlock;
    const int my_nblk = nblk > warp ? (nblk - warp + kDecodeWarps - 1) / kDecodeWarps : 0;

    unsigned char *wring = ring + warp * kDecodeStages * C::STAGE;
    uint64_t *bars = bars_all + warp * kDecodeStages;

    const PageMap pm{P.block_table, P.page_tokens, P.num_pages};

    if (lane == 0) {
        for (int s = 0; s < kDecodeStages; ++s)
            mbar_init(&bars[s], 1);
        mbar_init(&stall_bars[warp], 1);
        mbar_fence_init();
    }
    __syncwarp();

    // Block jj of this warp into stage s: lane 0 announces the stage's bytes and issues the
    // four bulk copies (K codes, K scale/zero, V codes, V scale/zero) of the block's 64
    // token slots (contiguous, or one page-aligned run of a page: page_tokens is a
    // multiple of 64). Called by the whole warp.
    auto issue = [&](int jj, int s) {
        const int tok0 = t_begin + (warp + jj * kDecodeWarps) * kDecodeBlock;
        unsigned char *st = wring + s * C::STAGE;
        if (lane == 0) {
            long long row0;
            if (!pm.table) {
                row0 = (long long)pair * P.T_cap + tok0;
            } else {
                row0 = cache_row(pm, b, h, P.Hkv, P.T_cap, tok0);
                if (row0 < 0) {                 // out-of-range page: flagged, read page 0
                    flag(P.dev_err, KVQ_DEVERR_PAGE_RANGE);
                    row0 = (long long)h * pm.page_tokens + tok0 % pm.page_tokens;
                }
            }
            mbar_arrive_expect_tx_relaxed(&bars[s], C::STAGE);
            bulk_g2s(st, P.k_codes + row0 * C::ROWK, C::KC_BYTES, &bars[s]);
            bulk_g2s(st + C::KC_BYTES, P.k_sz + row0, C::SZ_BYTES, &bars[s]);
            bulk_g2s(st + C::KC_BYTES + C::SZ_BYTES, P.v_codes + row0 * (D * BV / 8),
                     C::VC_BYTES, &bars[s]);
            bulk_g2s(st + C::KC_BYTES + C::SZ_BYTES + C::VC_BYTES, P.v_sz + row0, C::SZ_BYTES,
                     &bars[s]);
        }
        __syncwarp();
    };
    for (int jj = 0; jj < kDecodeStages && jj < my_nblk; ++jj)
        issue(jj, jj);
    // everything below reads what the q prologue writes
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // q~ operand fragments and per-head constants
    uint32_t qB[C::NT][C::KS][2];
    {
        const uint32_t *fr = P.qfrag + pair * (size_t)C::QFRAG;
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
            for (int ks = 0; ks < C::KS; ++ks) {
                uint2 v = reinterpret_cast<const uint2 *>(fr)[(nt * C::KS + ks) * 32 + lane];
                qB[nt][ks][0] = v.x;
                qB[nt][ks][1] = v.y;
            }
    }
    // Thread (g, t) owns head 4nt + t of every n-tile nt (columns 2t = hi, 2t+1 = lo) and
    // tokens g, g+8 of every 16-token sub-tile.
    float cs[C::NT], wq[C::NT];
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
        cs[nt] = P.qscale[(size_t)b * P.Hq + h * G + 4 * nt + t];
        wq[nt] = P.qw[(size_t)b * P.Hq + h * G + 4 * nt + t];
    }

    float m_run[C::NT], l_run[C::NT], lz_run[C::NT];
    float O[C::MT][C::NT][4];
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
        m_run[nt] = -INFINITY;
        l_run[nt] = 0.f;
        lz_run[nt] = 0.f;
#pragma unroll
        for (int m = 0; m < C::MT; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                O[m][nt][i] = 0.f;
    }
    bool timed_out = false;
    if (P.stall_test_ns > 0 && my_nblk > 0) {
        // failure-path test hook: a bounded wait on a barrier that nothing arrives at; on
        // giving up, the same path as a real timeout -- wait (bounded, normal limit) for
        // this warp's copies in flight, skip the blocks, flag the error
        if (!mbar_wait_bounded(&stall_bars[warp], 0, (uint64_t)P.stall_test_ns)) {
            timed_out = true;
            for (int k2 = 0; k2 < kDecodeStages && k2 < my_nblk; ++k2)
                mbar_wait_bounded(&bars[k2], 0);
        }
    }

    // One 64-token block. FULL: every token is below t_end (no per-token masking).
    auto block = [&](const unsigned char *st, int tok0, auto full_tag) {
        constexpr bool FULL = decltype(full_tag)::value;
        const uint32_t *kszw = reinterpret_cast<const uint32_t *>(st + C::KC_BYTES);
        const uint32_t *vszw =
            reinterpret_cast<const uint32_t *>(st + C::KC_BYTES + C::SZ_BYTES + C::VC_BYTES);

        // ---- scores S^T for 4 sub-tiles on int8 MMAs. A k-step takes one field position k
        //      of every code byte, masked in place (uint8 c * 2^(BK k)); the field steps are
        //      accumulated Horner-style (x 2^BK between them), so each score is the exact
        //      integer 2^(BK(CPB-1)) * sum_j c_j q_int_j. Accumulator rows g and g+8 hold
        //      tokens ta and tb of the sub-tile (see below).
        int S[4][C::NT][4];
        uint32_t kw[4][2][C::WPT];
#pragma unroll
        for (int stt = 0; stt < 4; ++stt) {
            const unsigned char *kt = st + stt * 16 * C::ROWK + t * 4 * C::WPT;
            lds_words<C::WPT>(kw[stt][0], kt + ta * C::ROWK);
            lds_words<C::WPT>(kw[stt][1], kt + tb * C::ROWK);
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    S[stt][nt][i] = 0;
        }
#pragma unroll
        for (int k = 0; k < C::CPBK; ++k) {
            if (k > 0) {
#pragma unroll
                for (int stt = 0; stt < 4; ++stt)
#pragma unroll
                    for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            S[stt][nt][i] *= (1 << BK);
            }
            const uint32_t M = (((1u << BK) - 1u) * 0x01010101u) << (BK * k);
#pragma unroll
            for (int c = 0; c < C::KCH; ++c)
#pragma unroll
                for (int stt = 0; stt < 4; ++stt) {
                    if constexpr (C::WPT >= 2) {
                        const uint32_t a0 = kw[stt][0][2 * c] & M, a1 = kw[stt][1][2 * c] & M;
                        const uint32_t a2 = kw[stt][0][2 * c + 1] & M, a3 = kw[stt][1][2 * c + 1] & M;
#pragma unroll
                        for (int nt = 0; nt < C::NT; ++nt)
                            imma_k32(S[stt][nt], a0, a1, a2, a3, qB[nt][k * C::KCH + c][0],
                                     qB[nt][k * C::KCH + c][1]);
                    } else {
                        const uint32_t a0 = kw[stt][0][0] & M, a1 = kw[stt][1][0] & M;
#pragma unroll
                        for (int nt = 0; nt < C::NT; ++nt)
                            imma_k16(S[stt][nt], a0, a1, qB[nt][k][0]);
                    }
                }
        }

        // ---- logits (log2 units): hi + lo columns, then the per-token affine terms
        float L2[4][2][C::NT];
        float bm[C::NT];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt)
            bm[nt] = -INFINITY;
#pragma unroll
        for (int stt = 0; stt < 4; ++stt)
#pragma unroll
            for (int tk = 0; tk < 2; ++tk) {
                const int tl = 16 * stt + (tk ? tb : ta);
                const float2 sz = half2_bits_to_float2(kszw[tl]);
                const bool valid = FULL || (tok0 + tl < t_end);
#pragma unroll
                for (int nt = 0; nt < C::NT; ++nt) {
                    // columns hi, lo of the head: q_int = 256 hi + lo (exact in int32)
                    const float v = (float)(S[stt][nt][2 * tk] * 256 + S[stt][nt][2 * tk + 1]);
                    float l2 = fmaf(sz.x * cs[nt], v, sz.y * wq[nt]);
                    if constexpr (!FULL)
                        l2 = valid ? l2 : -INFINITY;
                    L2[stt][tk][nt] = l2;
                    bm[nt] = fmaxf(bm[nt], l2);
                }
            }
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            bm[nt] = fmaxf(bm[nt], __shfl_xor_sync(0xffffffffu, bm[nt], 4));
            bm[nt] = fmaxf(bm[nt], __shfl_xor_sync(0xffffffffu, bm[nt], 8));
            bm[nt] = fmaxf(bm[nt], __shfl_xor_sync(0xffffffffu, bm[nt], 16));
            if (bm[nt] > m_run[nt] + kLazy) {
                const float alpha = ex2(m_run[nt] - bm[nt]);
                l_run[nt] *= alpha;
                lz_run[nt] *= alpha;
#pragma unroll
                for (int m = 0; m < C::MT; ++m)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        O[m][nt][i] *= alpha;
                m_run[nt] = bm[nt];
            }
        }

        // ---- P' = p * s^v as float16 (hi, lo) pairs in the accumulator layout (row = token,
        //      columns 2t, 2t+1 = hi, lo of head 4nt+t); one 8x8 transpose per row half turns
        //      them into the B operand of the value product
        uint32_t pb[4][C::NT][2];
#pragma unroll
        for (int stt = 0; stt < 4; ++stt) {
            const float2 vz0 = half2_bits_to_float2(vszw[16 * stt + ta]);
            const float2 vz1 = half2_bits_to_float2(vszw[16 * stt + tb]);
            bool v0 = true, v1 = true;
            if constexpr (!FULL) {
                v0 = tok0 + 16 * stt + ta < t_end;
                v1 = tok0 + 16 * stt + tb < t_end;
            }
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt) {
                const float p0 = ex2(L2[stt][0][nt] - m_run[nt]);
                const float p1 = ex2(L2[stt][1][nt] - m_run[nt]);
                l_run[nt] += p0 + p1;
                float pp0 = p0 * vz0.x, pp1 = p1 * vz1.x;
                float z0 = p0 * vz0.y, z1 = p1 * vz1.y;
                if constexpr (!FULL) {
                    pp0 = v0 ? pp0 : 0.f;
                    pp1 = v1 ? pp1 : 0.f;
                    z0 = v0 ? z0 : 0.f;
                    z1 = v1 ? z1 : 0.f;
                }
                lz_run[nt] += z0 + z1;
                const __half2 hi = __floats2half2_rn(pp0, pp1);
                const float2 hif = __half22float2(hi);
                const __half2 lo = __floats2half2_rn(pp0 - hif.x, pp1 - hif.y);
                const __half2 ra = __lows2half2(hi, lo), rb = __highs2half2(hi, lo);
                pb[stt][nt][0] = movmatrix_trans(*reinterpret_cast<const uint32_t *>(&ra));
                pb[stt][nt][1] = movmatrix_trans(*reinterpret_cast<const uint32_t *>(&rb));
            }
        }

        // ---- O^T += Vcodes^T . P'^T
#pragma unroll
        for (int stt = 0; stt < 4; ++stt) {
            uint32_t vw[2 * C::WV];
            lds_words<2 * C::WV>(vw, st + C::KC_BYTES + C::SZ_BYTES + stt * C::VTILE + lane * C::VCH);
#pragma unroll
            for (int m = 0; m < C::MT; ++m) {
                const uint32_t a0 = ext_v<BV, C::CPBV, C::EV, C::WV>(vw, 0, 2 * m);
                const uint32_t a1 = ext_v<BV, C::CPBV, C::EV, C::WV>(vw, 0, 2 * m + 1);
                const uint32_t a2 = ext_v<BV, C::CPBV, C::EV, C::WV>(vw, 1, 2 * m);
                const uint32_t a3 = ext_v<BV, C::CPBV, C::EV, C::WV>(vw, 1, 2 * m + 1);
#pragma unroll
                for (int nt = 0; nt < C::NT; ++nt)
                    mma_f16(O[m][nt], a0, a1, a2, a3, pb[stt][nt][0], pb[stt][nt][1]);
            }
        }
        __syncwarp();
    };

    for (int jj = 0; !timed_out && jj < my_nblk; ++jj) {
        const int s = jj % kDecodeStages;
        if (!mbar_wait_bounded(&bars[s], (jj / kDecodeStages) & 1)) {
            timed_out = true;
            // wait (bounded) for this warp's copies still in flight, then stop
            for (int k2 = jj + 1; k2 < jj + kDecodeStages && k2 < my_nblk; ++k2)
                mbar_wait_bounded(&bars[k2 % kDecodeStages], (k2 / kDecodeStages) & 1);
            break;
        }
        const unsigned char *st = wring + s * C::STAGE;
        const int tok0 = t_begin + (warp + jj * kDecodeWarps) * kDecodeBlock;
        if (tok0 + kDecodeBlock <= t_end)
            block(st, tok0, std::true_type{});
        else
            block(st, tok0, std::false_type{});
        // every lane has consumed the stage (its values are in registers) before the
        // warp-synchronous refill below
        if (jj + kDecodeStages < my_nblk)
            issue(jj + kDecodeStages, s);
    }
    if (timed_out && lane == 0)
        flag(P.dev_err, KVQ_DEVERR_WAIT_TIMEOUT);

    // ---- per-warp reduction across the 8 lanes sharing a head (same t)
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l_run[nt] += __shfl_xor_sync(0xffffffffu, l_run[nt], off);
            lz_run[nt] += __shfl_xor_sync(0xffffffffu, lz_run[nt], off);
        }

    __syncthreads();                             // all warps are done with the ring
    if (lane == 0) {
        for (int s = 0; s < kDecodeStages; ++s)
            mbar_inval(&bars[s]);
        mbar_inval(&stall_bars[warp]);
    }
    float *mw = reinterpret_cast<float *>(ring);                 // [W][G]
    float *lw = mw + kDecodeWarps * G;                           // [W][G]
    float *ow = lw + kDecodeWarps * G;                           // [W][G][D]
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
        const int head = 4 * nt + t;
        if (g == 0) {
            mw[warp * G + head] = m_run[nt];
            lw[warp * G + head] = l_run[nt];
        }
#pragma unroll
        for (int m = 0; m < C::MT; ++m) {
            // rows g (n = 2m) and g+8 (n = 2m+1); value-field factor 2^(BV*(n % CPB));
            // columns 2t (hi) and 2t+1 (lo) of the same head
            const int n0 = 2 * m, n1 = 2 * m + 1;
            const float f0 = __int_as_float((127 + 24 - BV * (n0 % C::CPBV)) << 23);
            const float f1 = __int_as_float((127 + 24 - BV * (n1 % C::CPBV)) << 23);
            ow[(warp * G + head) * D + 8 * n0 + g] =
                fmaf(O[m][nt][0] + O[m][nt][1], f0, lz_run[nt]);
            ow[(warp * G + head) * D + 8 * n1 + g] =
                fmaf(O[m][nt][2] + O[m][nt][3], f1, lz_run[nt]);
        }
    }
    __syncthreads();

    // ---- merge warps; either finish the output or store this split's partial
    float *part = P.part + (pair * P.part_slots + sigma) * (size_t)(G * (D + 2));
    for (int idx = threadIdx.x; idx < G * D; idx += kDecodeWarps * 32) {
        const int head = idx / D, dim = idx % D;
        float Mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w)
            Mx = fmaxf(Mx, mw[w * G + head]);
        float L = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
            const float mwv = mw[w * G + head];
            if (mwv == -INFINITY)
                continue;
            const float wt = ex2(mwv - Mx);
            L = fmaf(wt, lw[w * G + head], L);
            o = fmaf(wt, ow[(w * G + head) * D + dim], o);
        }
        if (nmerge == 1) {
            const size_t oi = ((size_t)b * P.Hq + h * G + head) * D + dim;
            const float r = o / L;
            if (P.out_bf16)
                reinterpret_cast<__nv_bfloat16 *>(P.out)[oi] = __float2bfloat16_rn(r);
            else
                reinterpret_cast<float *>(P.out)[oi] = r;
        } else {
            part[head * (D + 2) + 2 + dim] = o;
            if (dim == 0) {
                part[head * (D + 2)] = Mx;
                part[head * (D + 2) + 1] = L;
            }
        }
    }
    if (nmerge == 1)
        return;
    merge_if_last<D, G>(P, pair, b, h, nmerge, nsplit_b, flag_smem);
}

template <int D, int G, int BK, int BV>
cudaError_t launch_decode_t(const DecodeLaunch &L, cudaStream_t st)
{
    using C = Cfg<D, G, BK, BV>;
    using QS = QprepSmem<D, G>;
    static unsigned long long qprep_attr = 0, decode_attr = 0, decode_win_attr = 0;
    cudaError_t e = ensure_dynamic_smem(qprep_kernel<D, G, BK>, QS::BYTES, qprep_attr);
    if (e != cudaSuccess)
        return e;
    const bool win = L.p.win_flush > 0;
    e = win ? ensure_dynamic_smem(decode_kernel<D, G, BK, BV, true>, C::SMEM, decode_win_attr)
            : ensure_dynamic_smem(decode_kernel<D, G, BK, BV, false>, C::SMEM, decode_attr);
    if (e != cudaSuccess)
        return e;
    // q prologue
    {
        dim3 grid(L.p.Hkv, (L.p.B + kQprepSeqs - 1) / kQprepSeqs);
        qprep_kernel<D, G, BK><<<grid, kQprepThreads, QS::BYTES, st>>>(
            L.q, L.q_bf16, L.M, L.p.B, L.p.Hq, L.p.Hkv, kQprepSeqs, L.p.seqlens, L.p.max_seqlen,
            L.p.out, L.p.out_bf16, const_cast<uint32_t *>(L.p.qfrag),
            const_cast<float *>(L.p.qscale), const_cast<float *>(L.p.qw), L.p.ticket, nullptr);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    // decode: CTA (KV head, sequence, split), splits slowest so that the short last
    // splits of the sequences run last; with a full-precision window its split comes first
    // (slice z = 0); a programmatic dependent of qprep
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(L.p.Hkv, L.p.B, L.p.nsplit + (win ? 1 : 0));
    cfg.blockDim = dim3(kDecodeWarps * 32);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return win ? cudaLaunchKernelEx(&cfg, decode_kernel<D, G, BK, BV, true>, L.p)
               : cudaLaunchKernelEx(&cfg, decode_kernel<D, G, BK, BV, false>, L.p);
}

template <int D, int G>
cudaError_t launch_qprep_qt_t(const DecodeLaunch &L, float *qt_out, cudaStream_t st)
{
    using QS = QprepSmem<D, G>;
    static unsigned long long attr = 0;
    cudaError_t e = ensure_dynamic_smem(qprep_kernel<D, G, 2>, QS::BYTES, attr);
    if (e != cudaSuccess)
        return e;
    dim3 grid(L.p.Hkv, (L.p.B + kQprepSeqs - 1) / kQprepSeqs);
    qprep_kernel<D, G, 2><<<grid, kQprepThreads, QS::BYTES, st>>>(
        L.q, L.q_bf16, L.M, L.p.B, L.p.Hq, L.p.Hkv, kQprepSeqs, L.p.seqlens, L.p.max_seqlen,
        L.p.out, L.p.out_bf16, const_cast<uint32_t *>(L.p.qfrag), const_cast<float *>(L.p.qscale),
        const_cast<float *>(L.p.qw), L.p.ticket, qt_out);
    return cudaGetLastError();
}

}  // namespace

size_t decode_qfrag_words(int d, int G) { return (size_t)((2 * G) / 8) * (d / 16) * 64; }

// Resident decode CTAs per SM of the instantiation for (d, G, bits_k, bits_v) (registers
// and shared memory), for the host's split count.
int decode_resident_ctas(int d, int G, int bk, int bv)
{
#define KVQ_RES(DD, GG, KK, VV)                                        \
    if (d == DD && G == GG && bk == KK && bv == VV)                    \
        return Cfg<DD, GG, KK, VV>::MINB;
    KVQ_RES(128, 4, 2, 2)
    KVQ_RES(128, 4, 4, 2)
    KVQ_RES(128, 4, 2, 4)
    KVQ_RES(128, 4, 4, 4)
    KVQ_RES(128, 8, 2, 2)
    KVQ_RES(128, 8, 4, 2)
    KVQ_RES(128, 8, 2, 4)
    KVQ_RES(128, 8, 4, 4)
    KVQ_RES(64, 4, 2, 2)
    KVQ_RES(64, 4, 4, 2)
    KVQ_RES(64, 4, 2, 4)
    KVQ_RES(64, 4, 4, 4)
    KVQ_RES(64, 8, 2, 2)
    KVQ_RES(64, 8, 4, 2)
    KVQ_RES(64, 8, 2, 4)
    KVQ_RES(64, 8, 4, 4)
#undef KVQ_RES
    return kDecodeMinBlocks;
}

// The query prologue alone, also writing q~ (float32 [B][Hq][d]) to qt_out: the first
// kernel of the vector-quantized decode (it also zeroes the merge tickets and writes the
// zero output of empty sequences).
cudaError_t launch_qprep_qt(const DecodeLaunch &L, float *qt_out, cudaStream_t st)
{
    if (L.d == 128 && L.G == 4)
        return launch_qprep_qt_t<128, 4>(L, qt_out, st);
    if (L.d == 128 && L.G == 8)
        return launch_qprep_qt_t<128, 8>(L, qt_out, st);
    if (L.d == 64 && L.G == 4)
        return launch_qprep_qt_t<64, 4>(L, qt_out, st);
    if (L.d == 64 && L.G == 8)
        return launch_qprep_qt_t<64, 8>(L, qt_out, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeLaunch &L, cudaStream_t st)
{
    const int d = L.d, G = L.G, bk = L.bits_k, bv = L.bits_v;
#define KVQ_DISPATCH(DD, GG, KK, VV)                                   \
    if (d == DD && G == GG && bk == KK && bv == VV)                    \
        return launch_decode_t<DD, GG, KK, VV>(L, st);
    KVQ_DISPATCH(128, 4, 2, 2)
    KVQ_DISPATCH(128, 4, 4, 2)
    KVQ_DISPATCH(128, 4, 2, 4)
    KVQ_DISPATCH(128, 4, 4, 4)
    KVQ_DISPATCH(128, 8, 2, 2)
    KVQ_DISPATCH(128, 8, 4, 2)
    KVQ_DISPATCH(128, 8, 2, 4)
    KVQ_DISPATCH(128, 8, 4, 4)
    KVQ_DISPATCH(64, 4, 2, 2)
    KVQ_DISPATCH(64, 4, 4, 2)
    KVQ_DISPATCH(64, 4, 2, 4)
    KVQ_DISPATCH(64, 4, 4, 4)
    KVQ_DISPATCH(64, 8, 2, 2)
    KVQ_DISPATCH(64, 8, 4, 2)
    KVQ_DISPATCH(64, 8, 2, 4)
    KVQ_DISPATCH(64, 8, 4, 4)
#undef KVQ_DISPATCH
    return cudaErrorInvalidValue;
}

}  // namespace kvq
