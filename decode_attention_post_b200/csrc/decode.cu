// Read path: one decode step of grouped-query attention over the transformed,
// clipped, affine-quantized cache ("WUSH-KV: KV Cache Quantization with Data-Adaptive
// Transforms", sections 1, 4.1, 4.2; "Spend Bits Where Queries Look", "Three
// requirements", item 2: the whole cache is read at every step, so this path is bound
// by HBM bandwidth).
//
// Two kernels per call:
//  qprep   q~ = T_k^{-T} q for every query head (float32), and from it the tensor-core
//          operand fragments, the logit scale and sum(q~) per head.
//  decode  split-K flash decode. CTA = (split, KV head, sequence), 4 warps. Each warp
//          streams 64-token blocks (K codes, K scale/zero, V codes, V scale/zero) with
//          cp.async.bulk into a private 3-stage shared-memory ring (mbarrier completion,
//          bounded waits), and per block:
//            S^T[16 tok x (hi,lo)*G] = Kcodes[16 tok x d] . q~'[d x 2G]   (mma f16, f32 acc)
//            logit = log2(e)/sqrt(d) * (s_t * q~.c_t + z_t * sum q~)       (affine dequant
//                    folded per token: x^ = z + c s)
//            online softmax in float32 (lazy rescale), P' = p * s^v_t split f16 hi/lo
//            O^T[d x (hi,lo)*G] += Vcodes^T[d x 16 tok] . P'^T[16 tok x 2G]
//          and sum_t p_t z^v_t for the value zero-points.
//          Warps merge in shared memory; splits merge in the last CTA to finish a
//          (sequence, KV head) (atomic ticket, no spin-wait).
//
// Codes reach the tensor cores without a float conversion: a 2-bit (4-bit) code field
// masked in place inside a 32-bit word is the float16 subnormal c * 2^(bits*k) * 2^-24,
// where k is its field position inside the byte. The per-position factor 2^(bits*k) is
// compensated in the q~ operand (keys) or per output dim (values), so every product
// carries the same power-of-two scale. Tensor cores take float16 subnormals exactly.
#include "kvq_common.cuh"
#include "kvq_ptx.cuh"
#include "decode_shapes.h"

#include <math.h>

namespace kvq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 4.0f;     // rescale the running sums only when the max grows by > 2^4

template <int D, int G, int BK, int BV>
struct Cfg {
    static constexpr int KSTEPS = D / 16;            // k-steps of the Q.K contraction
    static constexpr int MT = D / 16;                // m-tiles (output dims) of P.V
    static constexpr int NT = (2 * G) / 8;           // n-tiles of (hi, lo) x G columns
    static constexpr int COLS = 2 * G;
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
    static constexpr int PSTRIDE = kDecodeBlock + 8; // halves per P'^T column (padded)
    static constexpr int PBUF = COLS * PSTRIDE * 2;  // bytes per warp
    static constexpr int QFRAG = NT * KSTEPS * 32 * 2;
    static constexpr int RING = kDecodeWarps * kDecodeStages * STAGE;
    static constexpr int MERGE = kDecodeWarps * G * (D + 2) * 4;
    static constexpr int SMEM = (RING > MERGE ? RING : MERGE) + kDecodeWarps * PBUF +
                                kDecodeWarps * kDecodeStages * 8 + 16;
    static_assert(STAGE % 16 == 0, "stage alignment");
    static_assert(NT >= 1 && (2 * G) % 8 == 0, "G must be a multiple of 4");
};

// ---------------------------------------------------------------- operand extraction

// Key operand: extraction e (0 .. d/8-1) of this thread's WPT words of one token.
// Word e / (2 CPB), byte-half beta = (e / CPB) % 2, field k = e % CPB. The float16
// pair holds dims (4w+beta)*CPB + k (low) and (4w+2+beta)*CPB + k (high), w the
// token-row word index, each scaled by 2^(BK*k) * 2^-24.
template <int BK, int CPB>
__device__ __forceinline__ uint32_t ext_k(const uint32_t *kw, int e)
{
    constexpr uint32_t M = ((1u << BK) - 1u) * 0x00010001u;
    const int wl = e / (2 * CPB), beta = (e / CPB) & 1, k = e % CPB;
    const uint32_t w = beta ? (kw[wl] >> 8) : kw[wl];
    return w & (M << (BK * k));
}

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

// One CTA per (KV head, chunk of `bb` sequences). Computes q~ = M q in float32, then
//   eq  = power-of-two exponent bringing max|q~| * 2^(BK*(CPB-1)) to about 2^14,
//   frag[nt][ks][lane][2] = float16 hi/lo pieces of q~ * 2^eq * 2^(BK*(CPB-1-k)) laid
//                           out as the B operand of the Q.K product,
//   cs  = log2(e) / sqrt(d) / F with F = 2^(eq + BK*(CPB-1) - 24) the product scale,
//   w_h = log2(e) / sqrt(d) * sum_j q~_hj,
// and zeroes the split-merge ticket of the (sequence, KV head).
template <int D, int G, int BK>
__global__ void __launch_bounds__(256)
qprep_kernel(const void *__restrict__ q, int q_bf16, const float *__restrict__ M, int B, int Hq,
             int Hkv, int bb, uint32_t *__restrict__ qfrag, float *__restrict__ qscale,
             float *__restrict__ qw, int *__restrict__ ticket)
{
    constexpr int CPB = 8 / BK, KSTEPS = D / 16, NT = (2 * G) / 8, WPT = D * BK / 128;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float *Mt = reinterpret_cast<float *>(smem_raw);                 // [D][D+1] or unused
    float *qs = Mt + (M ? D * (D + 1) : 0);                            // [bb*G][D]
    float *qt = qs + bb * G * D;                                       // [bb*G][D]
    float *red = qt + bb * G * D;                                      // [bb][2]

    const int h = blockIdx.x;
    const int b0 = blockIdx.y * bb;
    const int nb = min(bb, B - b0);
    const int tid = threadIdx.x;
    if (tid < bb)
        red[tid] = 0.f;

    if (M) {
        const float *Mh = M + (size_t)h * D * D;
        for (int idx = tid; idx < D * D; idx += 256) {
            int i = idx / D, j = idx % D;
            Mt[j * (D + 1) + i] = Mh[idx];
        }
    }
    for (int idx = tid; idx < nb * G * D; idx += 256) {
        int v = idx / D, j = idx % D;
        int bi = v / G, gg = v % G;
        qs[idx] = load_in(q, q_bf16, ((size_t)(b0 + bi) * Hq + h * G + gg) * D + j);
    }
    __syncthreads();
    for (int idx = tid; idx < nb * G * D; idx += 256) {
        int v = idx / D, i = idx % D;
        float acc;
        if (M) {
            acc = 0.f;
            const float *qv = qs + v * D;
#pragma unroll 8
            for (int j = 0; j < D; ++j)
                acc = fmaf(Mt[j * (D + 1) + i], qv[j], acc);
        } else {
            acc = qs[idx];
        }
        qt[idx] = acc;
    }
    __syncthreads();
    // per sequence: max |q~| over its G heads; per head: sum of q~
    const int warp = tid >> 5, lane = tid & 31;
    const float sm = rsqrtf((float)D);
    for (int v = warp; v < nb * G; v += 8) {
        float s = 0.f, a = 0.f;
        for (int j = lane; j < D; j += 32) {
            float x = qt[v * D + j];
            s += x;
            a = fmaxf(a, fabsf(x));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            s += __shfl_xor_sync(0xffffffffu, s, off);
            a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        }
        if (lane == 0) {
            int bi = v / G, gg = v % G;
            qw[(size_t)(b0 + bi) * Hq + h * G + gg] = kLog2e * sm * s;
            atomicMax(reinterpret_cast<int *>(&red[bi]), __float_as_int(a));   // a >= 0
        }
    }
    __syncthreads();
    for (int bi = 0; bi < nb; ++bi) {
        const size_t pair = (size_t)(b0 + bi) * Hkv + h;
        const float amax = red[bi];
        int ex = 0;
        if (amax > 0.f)
            frexpf(amax, &ex);                         // amax <= 2^ex
        const int eq = amax > 0.f ? 14 - BK * (CPB - 1) - ex : 0;
        if (tid == 0) {
            // F = 2^(eq + BK*(CPB-1) - 24); cs = log2e * sm / F
            qscale[pair] = kLog2e * sm * ldexpf(1.f, 24 - eq - BK * (CPB - 1));
            ticket[pair] = 0;
        }
        uint32_t *fr = qfrag + pair * (size_t)(NT * KSTEPS * 64);
        for (int idx = tid; idx < NT * KSTEPS * 64; idx += 256) {
            const int rho = idx & 1, ln = (idx >> 1) & 31, ks = (idx >> 6) % KSTEPS;
            const int nt = (idx >> 6) / KSTEPS;
            const int g = ln >> 2, t = ln & 3;
            const int col = 8 * nt + g, head = col % G, piece = col / G;
            const int e = 2 * ks + rho;
            const int w = WPT * t + e / (2 * CPB), beta = (e / CPB) & 1, k = e % CPB;
            const int dlo = (4 * w + beta) * CPB + k, dhi = (4 * w + 2 + beta) * CPB + k;
            const float scale = ldexpf(1.f, eq + BK * (CPB - 1 - k));
            const float *qv = qt + (bi * G + head) * D;
            uint32_t packed = 0;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const float val = qv[half ? dhi : dlo] * scale;
                const __half hi = __float2half_rn(val);
                const __half pc = piece ? __float2half_rn(val - __half2float(hi)) : hi;
                packed |= (uint32_t)__half_as_ushort(pc) << (16 * half);
            }
            fr[idx] = packed;
        }
    }
}

// ---------------------------------------------------------------- main decode

template <int D, int G, int BK, int BV>
__global__ void __launch_bounds__(kDecodeWarps * 32, 3) decode_kernel(DecodeParams P)
{
    using C = Cfg<D, G, BK, BV>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *ring = smem_raw;
    __half *pbuf_all = reinterpret_cast<__half *>(smem_raw + (C::RING > C::MERGE ? C::RING : C::MERGE));
    uint64_t *bars_all = reinterpret_cast<uint64_t *>(reinterpret_cast<unsigned char *>(pbuf_all) +
                                                      kDecodeWarps * C::PBUF);
    int *flag_smem = reinterpret_cast<int *>(bars_all + kDecodeWarps * kDecodeStages);

    const int sigma = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const size_t pair = (size_t)b * P.Hkv + h;

    int seqlen = P.seqlens[b];
    if (seqlen < 0 || seqlen > P.max_seqlen) {
        if (sigma == 0 && h == 0 && threadIdx.x == 0)
            flag(P.dev_err, KVQ_DEVERR_SEQLEN_CLAMPED);
        seqlen = seqlen < 0 ? 0 : P.max_seqlen;
    }
    const int t_begin = sigma * P.split_tokens;
    if (t_begin >= seqlen) {
        if (sigma == 0) {                       // empty sequence: the output is 0
            for (int idx = threadIdx.x; idx < G * D; idx += kDecodeWarps * 32) {
                const size_t o = ((size_t)b * P.Hq + h * G + idx / D) * D + idx % D;
                if (P.out_bf16)
                    reinterpret_cast<__nv_bfloat16 *>(P.out)[o] = __float2bfloat16_rn(0.f);
                else
                    reinterpret_cast<float *>(P.out)[o] = 0.f;
            }
        }
        return;
    }
    const int t_end = min(t_begin + P.split_tokens, seqlen);
    const int nsplit_b = (seqlen + P.split_tokens - 1) / P.split_tokens;
    const int nblk = (t_end - t_begin + kDecodeBlock - 1) / kDecodeBlock;
    const int my_nblk = nblk > warp ? (nblk - warp + kDecodeWarps - 1) / kDecodeWarps : 0;

    unsigned char *wring = ring + warp * kDecodeStages * C::STAGE;
    __half *pbuf = pbuf_all + warp * (C::PBUF / 2);
    uint64_t *bars = bars_all + warp * kDecodeStages;

    const uint8_t *kc = P.k_codes + pair * (size_t)P.T_cap * C::ROWK;
    const uint8_t *ksz = reinterpret_cast<const uint8_t *>(P.k_sz + pair * (size_t)P.T_cap);
    const uint8_t *vc = P.v_codes + pair * (size_t)P.T_cap * (D * BV / 8);
    const uint8_t *vsz = reinterpret_cast<const uint8_t *>(P.v_sz + pair * (size_t)P.T_cap);

    if (lane == 0) {
        for (int s = 0; s < kDecodeStages; ++s)
            mbar_init(&bars[s], 1);
        mbar_fence_init();
    }
    __syncwarp();

    auto issue = [&](int jj, int s) {
        const int tok0 = t_begin + (warp + jj * kDecodeWarps) * kDecodeBlock;
        unsigned char *st = wring + s * C::STAGE;
        mbar_arrive_expect_tx(&bars[s], C::STAGE);
        bulk_g2s(st, kc + (size_t)tok0 * C::ROWK, C::KC_BYTES, &bars[s]);
        bulk_g2s(st + C::KC_BYTES, ksz + (size_t)tok0 * 4, C::SZ_BYTES, &bars[s]);
        bulk_g2s(st + C::KC_BYTES + C::SZ_BYTES, vc + (size_t)tok0 * (D * BV / 8), C::VC_BYTES,
                 &bars[s]);
        bulk_g2s(st + C::KC_BYTES + C::SZ_BYTES + C::VC_BYTES, vsz + (size_t)tok0 * 4,
                 C::SZ_BYTES, &bars[s]);
    };
    if (lane == 0)
        for (int jj = 0; jj < kDecodeStages && jj < my_nblk; ++jj)
            issue(jj, jj);

    // q~ operand fragments and per-head constants
    uint32_t qB[C::NT][C::KSTEPS][2];
    {
        const uint32_t *fr = P.qfrag + pair * (size_t)C::QFRAG;
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
            for (int ks = 0; ks < C::KSTEPS; ++ks) {
                uint2 v = reinterpret_cast<const uint2 *>(fr)[(nt * C::KSTEPS + ks) * 32 + lane];
                qB[nt][ks][0] = v.x;
                qB[nt][ks][1] = v.y;
            }
    }
    const int hp = (2 * t) % G;                 // this thread's head pair (hp, hp+1)
    const float cs = P.qscale[pair];
    const float wq0 = P.qw[(size_t)b * P.Hq + h * G + hp];
    const float wq1 = P.qw[(size_t)b * P.Hq + h * G + hp + 1];

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f}, lz_run[2] = {0.f, 0.f};
    float O[C::MT][C::NT][4];
#pragma unroll
    for (int m = 0; m < C::MT; ++m)
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                O[m][nt][i] = 0.f;

    constexpr int TPT = (G == 4) ? 1 : 2;       // tokens per thread per 16-token sub-tile
    bool timed_out = false;

    for (int jj = 0; jj < my_nblk; ++jj) {
        const int s = jj % kDecodeStages;
        if (!mbar_wait_bounded(&bars[s], (jj / kDecodeStages) & 1)) {
            timed_out = true;
            // wait (bounded) for this warp's copies still in flight, then stop
            for (int k2 = jj + 1; k2 < jj + kDecodeStages && k2 < my_nblk; ++k2)
                mbar_wait_bounded(&bars[k2 % kDecodeStages], (k2 / kDecodeStages) & 1);
            break;
        }
        const unsigned char *st = wring + s * C::STAGE;
        const uint32_t *kszw = reinterpret_cast<const uint32_t *>(st + C::KC_BYTES);
        const uint32_t *vszw =
            reinterpret_cast<const uint32_t *>(st + C::KC_BYTES + C::SZ_BYTES + C::VC_BYTES);
        const int tok0 = t_begin + (warp + jj * kDecodeWarps) * kDecodeBlock;

        // ---- scores S^T for 4 sub-tiles of 16 tokens
        float S[4][C::NT][4];
#pragma unroll
        for (int stt = 0; stt < 4; ++stt) {
            const unsigned char *kt = st + stt * 16 * C::ROWK + t * 4 * C::WPT;
            uint32_t kw0[C::WPT], kw1[C::WPT];
            lds_words<C::WPT>(kw0, kt + g * C::ROWK);
            lds_words<C::WPT>(kw1, kt + (g + 8) * C::ROWK);
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    S[stt][nt][i] = 0.f;
#pragma unroll
            for (int ks = 0; ks < C::KSTEPS; ++ks) {
                const uint32_t a0 = ext_k<BK, C::CPBK>(kw0, 2 * ks);
                const uint32_t a1 = ext_k<BK, C::CPBK>(kw1, 2 * ks);
                const uint32_t a2 = ext_k<BK, C::CPBK>(kw0, 2 * ks + 1);
                const uint32_t a3 = ext_k<BK, C::CPBK>(kw1, 2 * ks + 1);
#pragma unroll
                for (int nt = 0; nt < C::NT; ++nt)
                    mma_f16(S[stt][nt], a0, a1, a2, a3, qB[nt][ks][0], qB[nt][ks][1]);
            }
        }

        // ---- combine hi/lo pieces; logits (log2 units); block max per head
        float L2[4][TPT][2];
        int tokl[4][TPT];
#pragma unroll
        for (int stt = 0; stt < 4; ++stt) {
            float v[TPT][2];
            if constexpr (G == 4) {
                const bool lo_side = t >= 2;
                const float s0 = lo_side ? S[stt][0][0] : S[stt][0][2];
                const float s1 = lo_side ? S[stt][0][1] : S[stt][0][3];
                const float r0 = __shfl_xor_sync(0xffffffffu, s0, 2);
                const float r1 = __shfl_xor_sync(0xffffffffu, s1, 2);
                v[0][0] = (lo_side ? S[stt][0][2] : S[stt][0][0]) + r0;
                v[0][1] = (lo_side ? S[stt][0][3] : S[stt][0][1]) + r1;
                tokl[stt][0] = 16 * stt + g + (lo_side ? 8 : 0);
            } else {
#pragma unroll
                for (int tk = 0; tk < 2; ++tk) {
                    v[tk][0] = S[stt][0][2 * tk] + S[stt][1][2 * tk];
                    v[tk][1] = S[stt][0][2 * tk + 1] + S[stt][1][2 * tk + 1];
                    tokl[stt][tk] = 16 * stt + g + 8 * tk;
                }
            }
#pragma unroll
            for (int tk = 0; tk < TPT; ++tk) {
                const int tl = tokl[stt][tk];
                const bool valid = tok0 + tl < t_end;
                const float2 sz = half2_bits_to_float2(kszw[tl]);
                const float a = sz.x * cs;
                L2[stt][tk][0] = valid ? fmaf(a, v[tk][0], sz.y * wq0) : -INFINITY;
                L2[stt][tk][1] = valid ? fmaf(a, v[tk][1], sz.y * wq1) : -INFINITY;
            }
        }
        float bm[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int stt = 0; stt < 4; ++stt)
#pragma unroll
            for (int tk = 0; tk < TPT; ++tk) {
                bm[0] = fmaxf(bm[0], L2[stt][tk][0]);
                bm[1] = fmaxf(bm[1], L2[stt][tk][1]);
            }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            if constexpr (G == 4)
                bm[hh] = fmaxf(bm[hh], __shfl_xor_sync(0xffffffffu, bm[hh], 2));
            bm[hh] = fmaxf(bm[hh], __shfl_xor_sync(0xffffffffu, bm[hh], 4));
            bm[hh] = fmaxf(bm[hh], __shfl_xor_sync(0xffffffffu, bm[hh], 8));
            bm[hh] = fmaxf(bm[hh], __shfl_xor_sync(0xffffffffu, bm[hh], 16));
            if (bm[hh] > m_run[hh] + kLazy) {
                const float alpha = ex2(m_run[hh] - bm[hh]);
                l_run[hh] *= alpha;
                lz_run[hh] *= alpha;
#pragma unroll
                for (int m = 0; m < C::MT; ++m)
#pragma unroll
                    for (int nt = 0; nt < C::NT; ++nt) {
                        O[m][nt][hh] *= alpha;
                        O[m][nt][2 + hh] *= alpha;
                    }
                m_run[hh] = bm[hh];
            }
        }

        // ---- probabilities, value-scale products P' = p * s^v split into f16 hi/lo,
        //      written transposed (column = head piece, slot pairs (j, j+8))
#pragma unroll
        for (int stt = 0; stt < 4; ++stt) {
            __half ph[TPT][2][2];               // [token][head][hi/lo]
#pragma unroll
            for (int tk = 0; tk < TPT; ++tk) {
                const int tl = tokl[stt][tk];
                const bool valid = tok0 + tl < t_end;
                const float2 vz = half2_bits_to_float2(vszw[tl]);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float p = ex2(L2[stt][tk][hh] - m_run[hh]);
                    l_run[hh] += p;
                    lz_run[hh] = valid ? fmaf(p, vz.y, lz_run[hh]) : lz_run[hh];
                    const float pp = valid ? p * vz.x : 0.f;
                    const __half hi = __float2half_rn(pp);
                    const __half lo = __float2half_rn(pp - __half2float(hi));
                    ph[tk][hh][0] = hi;
                    ph[tk][hh][1] = lo;
                }
            }
            if constexpr (G == 4) {
                const int slot = 16 * stt + 2 * g + (t >= 2 ? 1 : 0);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    pbuf[(hp + hh) * C::PSTRIDE + slot] = ph[0][hh][0];
                    pbuf[(G + hp + hh) * C::PSTRIDE + slot] = ph[0][hh][1];
                }
            } else {
                const int slot = 16 * stt + 2 * g;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int pc = 0; pc < 2; ++pc) {
                        __half2 w2 = __halves2half2(ph[0][hh][pc], ph[1][hh][pc]);
                        *reinterpret_cast<__half2 *>(&pbuf[(pc * G + hp + hh) * C::PSTRIDE + slot]) = w2;
                    }
            }
        }
        __syncwarp();

        // ---- O^T += Vcodes^T . P'^T
#pragma unroll
        for (int stt = 0; stt < 4; ++stt) {
            uint32_t vw[2 * C::WV];
            lds_words<2 * C::WV>(vw, st + C::KC_BYTES + C::SZ_BYTES + stt * C::VTILE + lane * C::VCH);
            uint32_t pb[C::NT][2];
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt) {
                const __half *pc = pbuf + (8 * nt + g) * C::PSTRIDE + 16 * stt + 2 * t;
                pb[nt][0] = *reinterpret_cast<const uint32_t *>(pc);
                pb[nt][1] = *reinterpret_cast<const uint32_t *>(pc + 8);
            }
#pragma unroll
            for (int m = 0; m < C::MT; ++m) {
                const uint32_t a0 = ext_v<BV, C::CPBV, C::EV, C::WV>(vw, 0, 2 * m);
                const uint32_t a1 = ext_v<BV, C::CPBV, C::EV, C::WV>(vw, 0, 2 * m + 1);
                const uint32_t a2 = ext_v<BV, C::CPBV, C::EV, C::WV>(vw, 1, 2 * m);
                const uint32_t a3 = ext_v<BV, C::CPBV, C::EV, C::WV>(vw, 1, 2 * m + 1);
#pragma unroll
                for (int nt = 0; nt < C::NT; ++nt)
                    mma_f16(O[m][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
        }
        __syncwarp();
        if (lane == 0 && jj + kDecodeStages < my_nblk) {
            fence_proxy_async_smem();
            issue(jj + kDecodeStages, s);
        }
    }
    if (timed_out && lane == 0)
        flag(P.dev_err, KVQ_DEVERR_WAIT_TIMEOUT);

    // ---- per-warp reduction across threads sharing heads
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        if constexpr (G == 4) {
            l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 2);
            lz_run[hh] += __shfl_xor_sync(0xffffffffu, lz_run[hh], 2);
        }
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], off);
            lz_run[hh] += __shfl_xor_sync(0xffffffffu, lz_run[hh], off);
        }
    }
    float Osum[C::MT][4];
#pragma unroll
    for (int m = 0; m < C::MT; ++m)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (G == 4)
                Osum[m][i] = O[m][0][i] + __shfl_xor_sync(0xffffffffu, O[m][0][i], 2);
            else
                Osum[m][i] = O[m][0][i] + O[m][1][i];
        }

    __syncthreads();                             // all warps are done with the ring
    for (int s = 0; s < kDecodeStages && lane == 0; ++s)
        mbar_inval(&bars[s]);
    float *mw = reinterpret_cast<float *>(ring);                 // [W][G]
    float *lw = mw + kDecodeWarps * G;                           // [W][G]
    float *ow = lw + kDecodeWarps * G;                           // [W][G][D]
    const bool writer = (G == 4) ? (t < 2) : true;
    if (writer) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int head = hp + hh;
            if (g == 0) {
                mw[warp * G + head] = m_run[hh];
                lw[warp * G + head] = l_run[hh];
            }
#pragma unroll
            for (int m = 0; m < C::MT; ++m) {
                // rows g (n = 2m) and g+8 (n = 2m+1); value-field factor 2^(BV*(n % CPB))
                const int n0 = 2 * m, n1 = 2 * m + 1;
                const float f0 = __int_as_float((127 + 24 - BV * (n0 % C::CPBV)) << 23);
                const float f1 = __int_as_float((127 + 24 - BV * (n1 % C::CPBV)) << 23);
                ow[(warp * G + head) * D + 8 * n0 + g] = fmaf(Osum[m][hh], f0, lz_run[hh]);
                ow[(warp * G + head) * D + 8 * n1 + g] = fmaf(Osum[m][2 + hh], f1, lz_run[hh]);
            }
        }
    }
    __syncthreads();

    // ---- merge warps; either finish the output or store this split's partial
    float *part = P.part + (pair * P.nsplit + sigma) * (size_t)(G * (D + 2));
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
        if (nsplit_b == 1) {
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
    if (nsplit_b == 1)
        return;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        *flag_smem = (atomicAdd(&P.ticket[pair], 1) == nsplit_b - 1);
    __syncthreads();
    if (!*flag_smem)
        return;
    __threadfence();
    const float *pall = P.part + pair * P.nsplit * (size_t)(G * (D + 2));
    for (int idx = threadIdx.x; idx < G * D; idx += kDecodeWarps * 32) {
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
        const size_t oi = ((size_t)b * P.Hq + h * G + head) * D + dim;
        const float r = o / L;
        if (P.out_bf16)
            reinterpret_cast<__nv_bfloat16 *>(P.out)[oi] = __float2bfloat16_rn(r);
        else
            reinterpret_cast<float *>(P.out)[oi] = r;
    }
}

template <int D, int G, int BK, int BV>
cudaError_t launch_decode_t(const DecodeLaunch &L, cudaStream_t st)
{
    using C = Cfg<D, G, BK, BV>;
    // q prologue
    {
        const int bb = L.qprep_bb;
        size_t smem = (size_t)((L.M ? D * (D + 1) : 0) + 2 * bb * G * D + 2 * bb) * 4;
        cudaError_t e = cudaFuncSetAttribute(qprep_kernel<D, G, BK>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        dim3 grid(L.p.Hkv, (L.p.B + bb - 1) / bb);
        qprep_kernel<D, G, BK><<<grid, 256, smem, st>>>(L.q, L.q_bf16, L.M, L.p.B, L.p.Hq,
                                                       L.p.Hkv, bb, const_cast<uint32_t *>(L.p.qfrag),
                                                       const_cast<float *>(L.p.qscale),
                                                       const_cast<float *>(L.p.qw), L.p.ticket);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G, BK, BV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess)
        return e;
    dim3 grid(L.p.nsplit, L.p.Hkv, L.p.B);
    decode_kernel<D, G, BK, BV><<<grid, kDecodeWarps * 32, C::SMEM, st>>>(L.p);
    return cudaGetLastError();
}

}  // namespace

size_t decode_qfrag_words(int d, int G) { return (size_t)((2 * G) / 8) * (d / 16) * 64; }

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
