// Write path for chunks of bfloat16 keys/values on the 5th-generation tensor cores
// ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms", sections 4.2, 4.3 and
// 5.3; "Spend Bits Where Queries Look", "Three requirements", item 3).
//
// CTA = (KV head, one of {K, V}, slice of the 128-token tiles of the flattened
// (sequence, new token) list), one CTA per SM, warps with fixed roles:
//   TMA warp, one lane each 128-token input tile [128 x d] bf16 lands in a 4-stage (d = 64)
//                      or 3-stage (d = 128) shared-memory ring in the 128-byte-swizzled
//                      K-major layout (3-D tensor map over [tokens][Hkv][d], no multicast);
//   MMA warp, one lane tcgen05.mma: X~[128 x d] = X . T_hi^T + X . T_lo^T into one float32
//                      TMEM accumulator (T split into two bfloat16 pieces, 16 significant
//                      bits; X is bfloat16, hence exact), M = 128, N = d, K = 16 per
//                      instruction; one accumulator buffer per epilogue warpgroup so that
//                      the next tiles' MMAs overlap this tile's epilogue;
//   epilogue warps     three (d = 64) or two (d = 128) warpgroups taking the tiles round
//                      robin: thread r owns token r of the tile; tcgen05.ld brings its
//                      transformed values into registers (the whole row at d = 64, 32
//                      columns at a time at d = 128), in two passes: per group the clip
//                      range (order statistics, or the RMS for the QuEST INT quantizer) and
//                      the float16 scale and zero-point, then the codes (the correctly
//                      rounded quotient by a reciprocal and one correction, so the codes are
//                      those of the definition bit for bit) and the fixed-width stores (one
//                      K row, or the token's halves of its 16-token V tile).
// T (the B operand, N = d output dims x K = d input dims, K-major) is converted and
// swizzled into shared memory once per CTA. Every wait is bounded; a wait that gives up
// flags KVQ_DEVERR_WAIT_TIMEOUT, the CTA waits (bounded) for its copies and MMAs in flight,
// frees its TMEM and stops.
// The codes use no conversion unit: rounding by the float addition of 1.5 * 2^23, packing
// by multiply-adds of the resulting bit patterns.
#include "kvq_common.cuh"
#include "kvq_ptx.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace kvq {

namespace {

constexpr int kTcTile = 128;                       // tokens per tile (MMA M)
constexpr int kTcKBlock = 64;                      // bf16 per 128-byte swizzled row

template <int D>
struct TcCfg {
    // epilogue warpgroups, one TMEM accumulator buffer each: at d = 64 three, so that one
    // CTA per SM keeps 12 epilogue warps with the register budget to hold a whole row
    static constexpr int EPI = D == 64 ? 3 : 2;
    static constexpr int EPI_WARPS = 4 * EPI;
    static constexpr int THREADS = (EPI_WARPS + 2) * 32;      // + TMA warp + MMA warp
    static constexpr int STAGES = D == 64 ? 4 : 3;            // input tile ring
    static constexpr int KB = D / kTcKBlock;                  // 128-byte K blocks
    static constexpr int A_BLOCK = kTcTile * kTcKBlock * 2;   // 16 KB: one K block of a tile
    static constexpr int A_BYTES = KB * A_BLOCK;              // one input stage
    static constexpr int B_BLOCK = D * kTcKBlock * 2;         // one K block of T_hi or T_lo
    static constexpr int B_BYTES = KB * B_BLOCK;
    static constexpr int OFF_B_HI = STAGES * A_BYTES;
    static constexpr int OFF_B_LO = OFF_B_HI + B_BYTES;
    static constexpr int OFF_BAR = OFF_B_LO + B_BYTES;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;         // barriers + alignment slack
    static constexpr int TMEM_COLS = 256;                     // EPI accumulators of D columns
    static constexpr int PER_SM = 1;
    // registers per thread: each of the SM's 4 schedulers holds 16K registers for its
    // ceil(warps / 4) warps, in whole 8-register steps (d = 64: 14 warps, 128 registers;
    // d = 128: 10 warps, 168)
    static constexpr int WARPS_PER_SMSP = (THREADS / 32 + 3) / 4;
    static constexpr int MAXREG_RAW = (16384 / (32 * WARPS_PER_SMSP)) / 8 * 8;
    static constexpr int MAXREG = MAXREG_RAW > 255 ? 248 : MAXREG_RAW;
    static_assert(EPI * D <= TMEM_COLS, "TMEM accumulators");
    static_assert((2 * STAGES + 2 * EPI) * 8 + 8 <= 256, "barrier area");
    static_assert(PER_SM * (SMEM + 1024) <= 228 * 1024, "shared memory oversubscribed");
};

struct TcParams {
    const float *Tk, *Tv;
    int B, n, Hkv, T_cap, bits_k, bits_v;
    int clip;                   // order-statistic index kappa, or kQuestClip
    uint8_t *k_codes;
    uint32_t *k_sz;
    uint8_t *v_codes;
    uint32_t *v_sz;
    const int32_t *pos;
    int32_t *dev_err;
    PageMap pm;
};

// An arrive that orders nothing but itself: the epilogue's release of an accumulator
// buffer. Its TMEM loads are complete (tcgen05.wait::ld) and fenced before the arrive;
// its global stores need no ordering with the next MMA, and a releasing arrive would
// hold the warp until they drain.
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// Codes of a group: c = clamp(rint(f32(f32(x - z) / s)), 0, qmax) for float16 (s, z).
// The quotient is the correctly rounded one (div_rn: a reciprocal and one correction), so
// the codes are those of the definition bit for bit with no tie test; the clamp comes first
// (the same result: rint and the clamp are both monotone and the clamp bounds are
// integers) and the rounding to nearest even is the float addition of 1.5 * 2^23, whose
// bit pattern is then 0x4B400000 + c. A zero or non-finite scale (rc = 0) gives code 0.
constexpr float kRoundMagic = 12582912.0f;        // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

// Two codes at a time on the paired float32 instructions of sm_100 (add/mul/fma .f32x2;
// each lane of a pair is an ordinary IEEE float32 operation): the bits 0x4B400000 + c of
// the code of xa with the parameters (za, sa, ra = RN(1/sa)) and of xb with (zb, sb, rb),
// given as pairs nz = (-za, -zb), nsb2 = (-sa, -sb), rc2 = (ra, rb): x - z and the
// quotient by div_rn's steps (RN(a y), the exact residual, one correction) on pairs, then
// per value the clamp and the magic addition. The first element of a pair is its low 32
// bits; callers pair adjacent registers (no moves to build the pairs).
__device__ __forceinline__ uint64_t f2pack(uint32_t a, uint32_t b)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ void f2unpack(uint64_t v, uint32_t &a, uint32_t &b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
}

__device__ __forceinline__ void code_rn2(uint32_t xa, uint32_t xb, uint64_t nz, uint64_t nsb2,
                                         uint64_t rc2, float qmax, uint32_t &ca, uint32_t &cb)
{
    uint64_t a, q0, r, q;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(a) : "l"(f2pack(xa, xb)), "l"(nz));      // x - z
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q0) : "l"(a), "l"(rc2));                 // RN(a y)
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(q0), "l"(nsb2), "l"(a));    // a - q0 s
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(r), "l"(rc2), "l"(q0));     // q0 + r y
    uint32_t qa, qb;
    f2unpack(q, qa, qb);
    const float ya = fminf(fmaxf(__uint_as_float(qa), 0.f), qmax);
    const float yb = fminf(fmaxf(__uint_as_float(qb), 0.f), qmax);
    ca = __float_as_uint(__fadd_rn(ya, kRoundMagic));
    cb = __float_as_uint(__fadd_rn(yb, kRoundMagic));
}

// sum over e < N of 0x4B400000 * 2^(B*e), modulo 2^32: what packing N magic-rounded codes
// with multiply-adds leaves above the codes themselves
__host__ __device__ constexpr uint32_t magic_sum(int B, int N)
{
    uint32_t s = 0;
    for (int e = 0; e < N; ++e)
        s += kRoundMagicBits << (B * e);
    return s;
}

__device__ __forceinline__ float fmin3(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 32 TMEM columns of this thread's lane into registers; the load completes at the next
// tmem_wait (the hardware holds readers of the registers until then).
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// Per-group quantities selected by a group index known only at run time, without a
// local-memory array (NG <= 4 compile-time slots).
template <int NG>
__device__ __forceinline__ float pick(const float (&a)[NG], int gr)
{
    float v = a[0];
#pragma unroll
    for (int i = 1; i < NG; ++i)
        v = gr == i ? a[i] : v;
    return v;
}


// (a, a) as a float32 pair
__device__ __forceinline__ uint64_t f2dup(float a)
{
    return ((uint64_t)__float_as_uint(a) << 32) | __float_as_uint(a);
}

// The 32 codes (magic bit patterns) of chunk c (dims 32c .. 32c + 31) of a row, two
// adjacent values at a time, with the parameters of the chunk's group.
template <int GS, int NG>
__device__ __forceinline__ void chunk_codes(const uint32_t (&cur)[32], int c,
                                            const float (&zf)[NG], const float (&sf)[NG],
                                            const float (&rc)[NG], float qmax, uint32_t (&cc)[32])
{
    const int gr = (32 * c) / GS;
    const uint64_t nz2 = f2dup(-pick(zf, gr)), ns2 = f2dup(-pick(sf, gr)), rc2 = f2dup(pick(rc, gr));
#pragma unroll
    for (int e = 0; e < 32; e += 2)
        code_rn2(cur[e], cur[e + 1], nz2, ns2, rc2, qmax, cc[e], cc[e + 1]);
}

// Value-tile halves from one chunk's codes: the chunk's dims are 32c + 8 n8 + gq (n8 < 4,
// gq < 8), and half (gq, rr) holds dims 8(E rr + s) + gq at bits BITS*s, E = 16/BITS, so
// the chunk gives fields base .. base + 3 of half gq (base = 4 (c & 1) for 2-bit codes,
// 0 for 4-bit codes).
template <int BITS>
__device__ __forceinline__ void v_fields(const uint32_t (&cc)[32], int base, uint32_t (&hv)[8])
{
#pragma unroll
    for (int gq = 0; gq < 8; ++gq) {
        uint32_t acc = 0u - (magic_sum(BITS, 4) << (BITS * base));
#pragma unroll
        for (int n8 = 0; n8 < 4; ++n8)
            acc += cc[8 * n8 + gq] << (BITS * (base + n8));
        hv[gq] = acc;
    }
}

// One token's codes from its TMEM row, two 32-column chunks per TMEM round trip, stored as
// the K row (little-endian bit stream, dim j at bit BITS*j) or as the token's halves of
// its 16-token V tile (with 2-bit codes the chunk pair fills whole halves). row < 0: codes
// not stored (the warp still takes part in the TMEM loads).
template <int D, int GS, int NG, int BITS, bool V>
__device__ __forceinline__ void store_codes(const TcParams &P, long long row, uint32_t taddr,
                                            const float (&zf)[NG], const float (&sf)[NG],
                                            const float (&rc)[NG], float qmax)
{
    constexpr int NCH = D / 32;
    static_assert(NCH % 2 == 0, "chunk pairs");
    unsigned char *vbase = nullptr;
    int tok = 0;
    if (V && row >= 0) {
        vbase = P.v_codes + (size_t)(row / kTileTokens) * (kTileTokens * D * BITS / 8);
        tok = (int)(row % kTileTokens);
    }
#pragma unroll 1
    for (int c = 0; c < NCH; c += 2) {
        uint32_t xa[32], xb[32];
        tmem_ld32_async(taddr + 32 * c, xa);
        tmem_ld32_async(taddr + 32 * (c + 1), xb);
        tmem_ld_wait();
        uint32_t ca[32], cb[32];
        chunk_codes<GS, NG>(xa, c, zf, sf, rc, qmax, ca);
        chunk_codes<GS, NG>(xb, c + 1, zf, sf, rc, qmax, cb);
        if (!V) {
            // word q of chunk c: dims 32c + (32/BITS) q + e at BITS*e
            constexpr int PER = 32 / BITS;
            uint32_t w[2 * BITS];
#pragma unroll
            for (int q = 0; q < 2 * BITS; ++q) {
                uint32_t acc = 0u - magic_sum(BITS, PER);
#pragma unroll
                for (int e = 0; e < PER; ++e)
                    acc += (q < BITS ? ca[PER * q + e] : cb[PER * (q - BITS) + e]) << (BITS * e);
                w[q] = acc;
            }
            if (row >= 0) {
                uint4 *dst = reinterpret_cast<uint4 *>(
                    reinterpret_cast<uint32_t *>(P.k_codes + row * (D * BITS / 8)) + BITS * c);
                if constexpr (BITS == 2) {
                    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                } else {
                    dst[0] = make_uint4(w[0], w[1 % (2 * BITS)], w[2 % (2 * BITS)], w[3 % (2 * BITS)]);
                    dst[1] = make_uint4(w[4 % (2 * BITS)], w[5 % (2 * BITS)], w[6 % (2 * BITS)],
                                        w[7 % (2 * BITS)]);
                }
            }
        } else {
            uint32_t ha[8], hb[8];
            v_fields<BITS>(ca, BITS == 2 ? 0 : 0, ha);
            v_fields<BITS>(cb, BITS == 2 ? 4 : 0, hb);
            if (row >= 0) {
#pragma unroll
                for (int gq = 0; gq < 8; ++gq) {
                    if constexpr (BITS == 4) {
                        *reinterpret_cast<uint16_t *>(vbase + v_half_offset(D, 4, tok, gq, c)) =
                            (uint16_t)ha[gq];
                        *reinterpret_cast<uint16_t *>(vbase + v_half_offset(D, 4, tok, gq, c + 1)) =
                            (uint16_t)hb[gq];
                    } else {
                        // chunks c (fields 0-3) and c + 1 (fields 4-7) of half rr = c / 2
                        *reinterpret_cast<uint16_t *>(vbase + v_half_offset(D, 2, tok, gq, c >> 1)) =
                            (uint16_t)(ha[gq] + hb[gq]);
                    }
                }
            }
        }
    }
}

// d = 64: the token's whole row x0 (dims 0-31), x1 (dims 32-63) is in registers. Codes
// with the group parameters of each half (index 0: dims 0-31, 1: dims 32-63), stored as
// the K row (one or two 16-byte stores) or as the token's halves of its V tile (whole
// 16-bit halves: half (gq, rr) holds dims 8(E rr + s) + gq at BITS*s, E = 16/BITS).
// row < 0: nothing stored.
template <int BITS>
__device__ __forceinline__ void store_row64(const TcParams &P, int which, long long row,
                                            const uint32_t (&x0)[32], const uint32_t (&x1)[32],
                                            const float (&z)[2], const float (&sc)[2],
                                            const float (&rc)[2], float qmax)
{
    auto pair = [](float a, float b) {
        return ((uint64_t)__float_as_uint(b) << 32) | __float_as_uint(a);
    };
    // the 64 codes (magic bit patterns), two adjacent values at a time, half 0 then half 1
    uint32_t c0[32], c1[32];
    {
        const uint64_t nz0 = pair(-z[0], -z[0]), ns0 = pair(-sc[0], -sc[0]),
                       r0 = pair(rc[0], rc[0]);
        const uint64_t nz1 = pair(-z[1], -z[1]), ns1 = pair(-sc[1], -sc[1]),
                       r1 = pair(rc[1], rc[1]);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            code_rn2(x0[e], x0[e + 1], nz0, ns0, r0, qmax, c0[e], c0[e + 1]);
            code_rn2(x1[e], x1[e + 1], nz1, ns1, r1, qmax, c1[e], c1[e + 1]);
        }
    }
    if (!which) {
        // word q of a 32-dim half: dims (32/BITS) q + e at BITS*e
        constexpr int PER = 32 / BITS;
        uint32_t w[2][BITS];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int q = 0; q < BITS; ++q) {
                uint32_t acc = 0u - magic_sum(BITS, PER);
#pragma unroll
                for (int e = 0; e < PER; ++e)
                    acc += (hf ? c1[PER * q + e] : c0[PER * q + e]) << (BITS * e);
                w[hf][q] = acc;
            }
        if (row >= 0) {
            uint4 *dst = reinterpret_cast<uint4 *>(P.k_codes + row * (64 * BITS / 8));
            if constexpr (BITS == 2) {
                dst[0] = make_uint4(w[0][0], w[0][1 % BITS], w[1][0], w[1][1 % BITS]);
            } else {
                dst[0] = make_uint4(w[0][0], w[0][1 % BITS], w[0][2 % BITS], w[0][3 % BITS]);
                dst[1] = make_uint4(w[1][0], w[1][1 % BITS], w[1][2 % BITS], w[1][3 % BITS]);
            }
        }
    } else {
        unsigned char *vbase = nullptr;
        int tok = 0;
        if (row >= 0) {
            vbase = P.v_codes + (size_t)(row / kTileTokens) * (kTileTokens * 64 * BITS / 8);
            tok = (int)(row % kTileTokens);
        }
#pragma unroll
        for (int gq = 0; gq < 8; ++gq) {
            if constexpr (BITS == 2) {
                // one half per gq: s < 4 from half 0 (dim gq + 8 s), s >= 4 from half 1
                uint32_t acc = 0u - magic_sum(2, 8);
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2)
                    acc += (c0[8 * s2 + gq] << (2 * s2)) + (c1[8 * s2 + gq] << (2 * (4 + s2)));
                if (row >= 0)
                    *reinterpret_cast<uint16_t *>(vbase + v_half_offset(64, 2, tok, gq, 0)) =
                        (uint16_t)acc;
            } else {
                // halves rr = 0 (half 0) and rr = 1 (half 1), s < 4: dim gq + 8 (4 rr + s)
                uint32_t a0 = 0u - magic_sum(4, 4), a1 = a0;
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    a0 += c0[8 * s2 + gq] << (4 * s2);
                    a1 += c1[8 * s2 + gq] << (4 * s2);
                }
                if (row >= 0) {
                    *reinterpret_cast<uint16_t *>(vbase + v_half_offset(64, 4, tok, gq, 0)) =
                        (uint16_t)a0;
                    *reinterpret_cast<uint16_t *>(vbase + v_half_offset(64, 4, tok, gq, 1)) =
                        (uint16_t)a1;
                }
            }
        }
    }
}

// Running clip statistics of one group of a row: kappa = 0 (min, max), kappa = 1 (second
// smallest and largest), kappa <= 8 (the 9 smallest and largest by insertion), or the
// QuEST INT sum of squares (float64, each square exact).
struct ClipStats {
    float lo, hi, m1, m2, M1, M2, sm9[9], lg9[9];
    double ss;

    __device__ __forceinline__ void reset(int clip)
    {
        lo = m1 = m2 = INFINITY;
        hi = M1 = M2 = -INFINITY;
        ss = 0.0;
        if (clip > 1) {
#pragma unroll
            for (int e = 0; e < 9; ++e) {
                sm9[e] = INFINITY;
                lg9[e] = -INFINITY;
            }
        }
    }

    __device__ __forceinline__ void add32(const uint32_t (&cur)[32], int clip, bool quest)
    {
        if (quest) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const double v = (double)__uint_as_float(cur[j]);
                ss = fma(v, v, ss);
            }
        } else if (clip == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                lo = fmin3(lo, __uint_as_float(cur[j]), __uint_as_float(cur[j + 1]));
                hi = fmax3(hi, __uint_as_float(cur[j]), __uint_as_float(cur[j + 1]));
            }
        } else if (clip == 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float v = __uint_as_float(cur[j]);
                m2 = fminf(m2, fmaxf(m1, v));
                m1 = fminf(m1, v);
                M2 = fmaxf(M2, fminf(M1, v));
                M1 = fmaxf(M1, v);
            }
        } else {
#pragma unroll 4
            for (int j = 0; j < 32; ++j) {
                float av = __uint_as_float(cur[j]), bv = av;
#pragma unroll
                for (int e = 0; e < 9; ++e) {
                    const float s0 = fminf(sm9[e], av), s1 = fmaxf(sm9[e], av);
                    sm9[e] = s0;
                    av = s1;
                    const float l0 = fmaxf(lg9[e], bv), l1 = fminf(lg9[e], bv);
                    lg9[e] = l0;
                    bv = l1;
                }
            }
        }
    }

    // the clip range [x_(kappa), x_(g-1-kappa)] of the values added
    __device__ __forceinline__ void range(int clip, float &glo, float &ghi) const
    {
        glo = lo;
        ghi = hi;
        if (clip == 1) {
            glo = m2;
            ghi = M2;
        } else if (clip > 1) {
            glo = sm9[0];
            ghi = lg9[0];
#pragma unroll
            for (int e = 1; e < 9; ++e)
                if (e == clip) {
                    glo = sm9[e];
                    ghi = lg9[e];
                }
        }
    }
};

template <int D, int GS>
__global__ void __launch_bounds__(TcCfg<D>::THREADS) __maxnreg__(TcCfg<D>::MAXREG)
append_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 TcParams P)
{
    using C = TcCfg<D>;
    constexpr int NG = D / GS;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *empty = full + C::STAGES;
    uint64_t *accf = empty + C::STAGES;
    uint64_t *acce = accf + C::EPI;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acce + C::EPI);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int h = blockIdx.y, which = blockIdx.z;
    const CUtensorMap *tmap = which ? &tm_v : &tm_k;
    const float *T = which ? P.Tv : P.Tk;
    const int bits = which ? P.bits_v : P.bits_k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long total = (long)P.B * P.n;
    const long ntiles = (total + kTcTile - 1) / kTcTile;
    const int my_tiles =
        blockIdx.x < ntiles ? (int)((ntiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::EPI; ++a) {
            mbar_init(&accf[a], 1);
            mbar_init(&acce[a], 128);                  // one epilogue warpgroup
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0)
        tmem_alloc(tmem_slot, C::TMEM_COLS);

    // ---- T_h -> bf16 (hi, lo) in the K-major 128-byte-swizzled layout: row i (output dim)
    //      of K block kb at kb*B_BLOCK + (i/8)*1024 + (i%8)*128, 16-byte chunk c of the row
    //      at position c ^ (i % 8)
    for (int c = threadIdx.x; c < D * D / 8; c += C::THREADS) {
        const int i = c / (D / 8), j0 = 8 * (c % (D / 8));
        const float4 *src = reinterpret_cast<const float4 *>(T + ((size_t)h * D + i) * D + j0);
        const float4 f0 = src[0], f1 = src[1];
        const float v[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * e]);
            const __nv_bfloat16 h1 = __float2bfloat16_rn(v[2 * e + 1]);
            const __nv_bfloat16 l0 = __float2bfloat16_rn(v[2 * e] - __bfloat162float(h0));
            const __nv_bfloat16 l1 = __float2bfloat16_rn(v[2 * e + 1] - __bfloat162float(h1));
            hw[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
            lw[e] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
        }
        const int kb = j0 / kTcKBlock, chunk = (j0 % kTcKBlock) / 8;
        const int off = kb * C::B_BLOCK + (i / 8) * 1024 + (i % 8) * 128 + ((chunk ^ (i % 8)) * 16);
        *reinterpret_cast<uint4 *>(smem + C::OFF_B_HI + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4 *>(smem + C::OFF_B_LO + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    fence_proxy_async_smem();           // generic stores -> operands of the tensor core
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    int issued = 0, consumed = 0;       // TMA lane: tiles loaded; MMA lane: tiles multiplied
    if (warp == C::EPI_WARPS) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(tmap);
            for (int k = 0; k < my_tiles && !*abort_flag; ++k) {
                const int s = k % C::STAGES;
                if (!mbar_wait_bounded(&empty[s], ((k / C::STAGES) & 1) ^ 1)) {
                    *abort_flag = 1;
                    break;
                }
                const long tile = blockIdx.x + (long)k * gridDim.x;
                mbar_arrive_expect_tx(&full[s], C::A_BYTES);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(smem + s * C::A_BYTES + kb * C::A_BLOCK, tmap, kb * kTcKBlock, h,
                                (int)(tile * kTcTile), &full[s]);
                issued = k + 1;
            }
        }
    } else if (warp == C::EPI_WARPS + 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32(kTcTile, D);
            for (int k = 0; k < my_tiles && !*abort_flag; ++k) {
                const int s = k % C::STAGES, a = k % C::EPI;
                if (!mbar_wait_bounded(&acce[a], ((k / C::EPI) & 1) ^ 1) ||
                    !mbar_wait_bounded(&full[s], (k / C::STAGES) & 1)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + (uint32_t)(a * D);
                const unsigned char *As = smem + s * C::A_BYTES;
#pragma unroll
                for (int piece = 0; piece < 2; ++piece)
#pragma unroll
                    for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
                        for (int kk = 0; kk < kTcKBlock / 16; ++kk) {
                            const uint64_t ad = umma_desc_sw128_kmajor(As + kb * C::A_BLOCK + kk * 32);
                            const uint64_t bd = umma_desc_sw128_kmajor(
                                smem + (piece ? C::OFF_B_LO : C::OFF_B_HI) + kb * C::B_BLOCK + kk * 32);
                            umma_bf16(d_tmem, ad, bd, idesc, (piece | kb | kk) != 0);
                        }
                umma_commit(&empty[s]);     // the stage may be refilled once these are done
                umma_commit(&accf[a]);      // the accumulator is complete
                consumed = k + 1;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Warpgroup wg takes the tiles k = wg, wg + EPI, ... (accumulator buffer wg); thread
        // r of warp quarter q owns TMEM lane (token row) 32 q + r. Two passes over the row:
        // the clip parameters of every group, then the codes (d = 64: the whole row held in
        // registers; d = 128: 32 columns at a time from TMEM). The buffer is released after
        // the row is done.
        const int wg = warp / 4, quarter = warp % 4;
        const int r = quarter * 32 + lane;
        const float qmax = (float)((1u << bits) - 1u);
        const float rqmax = __frcp_rn(qmax);
        const bool quest = P.clip == kQuestClip;
        for (int k = wg; k < my_tiles; k += C::EPI) {
            const int a = k % C::EPI;
            // the token's cache row first: its position load overlaps the wait below
            const long tile = blockIdx.x + (long)k * gridDim.x;
            const long u = tile * kTcTile + r;
            long long row = -1;
            if (u < total) {
                const unsigned uu = (unsigned)u;            // the launcher keeps B * n < 2^31
                const int b = (int)(uu / (unsigned)P.n), i = (int)(uu - (unsigned)b * (unsigned)P.n);
                const int p0 = P.pos[b];
                if (p0 < 0 || (long)p0 + P.n > P.T_cap) {
                    if (i == 0)
                        flag(P.dev_err, KVQ_DEVERR_POS_RANGE);
                } else {
                    row = cache_row(P.pm, b, h, P.Hkv, P.T_cap, p0 + i);
                    if (row < 0)
                        flag(P.dev_err, KVQ_DEVERR_PAGE_RANGE);
                }
            }
            if (*abort_flag || !mbar_wait_bounded(&accf[a], (k / C::EPI) & 1)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t taddr =
                tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * D);
            // ---- pass 1: clip parameters per group (every lane takes part in the loads)
            float zf[NG], sf[NG], rc[NG];
#pragma unroll
            for (int gg = 0; gg < NG; ++gg)
                zf[gg] = sf[gg] = rc[gg] = 0.f;
            ClipStats cs;
            cs.reset(P.clip);
            // group gr is complete: its scale and zero-point, stored with the row
            auto finish = [&](int gr) {
                __half sh, zh;
                bool finite;
                if (quest) {
                    const float rms = __double2float_rn(sqrt(cs.ss / (double)GS));
                    const float sv = __fmul_rn(rms, quest_delta(bits));
                    sh = __float2half_rn(sv);
                    zh = __float2half_rn(__fmul_rn(-0.5f * qmax, __half2float(sh)));
                    finite = isfinite(sv);
                } else {
                    float glo, ghi;
                    cs.range(P.clip, glo, ghi);
                    const float range = __fsub_rn(ghi, glo);
                    // range / qmax correctly rounded (div_rn; tiny or non-finite ranges,
                    // outside its conditions, by IEEE division)
                    const float sv = (range >= 0x1p-100f && range <= 0x1p+100f)
                                         ? div_rn(range, qmax, rqmax)
                                         : __fdiv_rn(range, qmax);
                    sh = __float2half_rn(sv);
                    zh = __float2half_rn(glo);
                    finite = isfinite(range) && isfinite(sv);
                }
                const float sfv = __half2float(sh), zfv = __half2float(zh);
                const bool zr = !finite || sfv == 0.f;
                const float rcv = zr ? 0.f : __frcp_rn(sfv);
#pragma unroll
                for (int gg = 0; gg < NG; ++gg)
                    if (gg == gr) {
                        sf[gg] = sfv;
                        zf[gg] = zfv;
                        rc[gg] = rcv;
                    }
                if (row >= 0) {
                    if (!finite)
                        flag(P.dev_err, KVQ_DEVERR_NONFINITE);
                    (which ? P.v_sz : P.k_sz)[row * NG + gr] =
                        (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);
                }
                cs.reset(P.clip);                           // the next group starts fresh
            };
            if constexpr (D == 64) {
                // the whole row in registers: one TMEM round trip for both passes
                uint32_t x0[32], x1[32];
                tmem_ld32_async(taddr, x0);
                tmem_ld32_async(taddr + 32, x1);
                tmem_ld_wait();
                cs.add32(x0, P.clip, quest);
                if (GS == 32)
                    finish(0);
                cs.add32(x1, P.clip, quest);
                finish(NG - 1);
                const float z2[2] = {zf[0], zf[NG - 1]}, s2[2] = {sf[0], sf[NG - 1]};
                const float r2[2] = {rc[0], rc[NG - 1]};
                if (bits == 2)
                    store_row64<2>(P, which, row, x0, x1, z2, s2, r2, qmax);
                else
                    store_row64<4>(P, which, row, x0, x1, z2, s2, r2, qmax);
            } else {
                // pass 1 over chunk pairs: two 32-column loads per TMEM round trip
#pragma unroll 1
                for (int c = 0; c < D / 32; c += 2) {
                    uint32_t xa[32], xb[32];
                    tmem_ld32_async(taddr + 32 * c, xa);
                    tmem_ld32_async(taddr + 32 * (c + 1), xb);
                    tmem_ld_wait();
                    cs.add32(xa, P.clip, quest);
                    if ((32 * c + 32) % GS == 0)          // the group ends with chunk c
                        finish((32 * c) / GS);
                    cs.add32(xb, P.clip, quest);
                    if ((32 * c + 64) % GS == 0)          // ... or with chunk c + 1
                        finish((32 * c + 32) / GS);
                }
                // ---- pass 2: codes
                if (!which) {
                    if (bits == 2)
                        store_codes<D, GS, NG, 2, false>(P, row, taddr, zf, sf, rc, qmax);
                    else
                        store_codes<D, GS, NG, 4, false>(P, row, taddr, zf, sf, rc, qmax);
                } else {
                    if (bits == 2)
                        store_codes<D, GS, NG, 2, true>(P, row, taddr, zf, sf, rc, qmax);
                    else
                        store_codes<D, GS, NG, 4, true>(P, row, taddr, zf, sf, rc, qmax);
                }
            }
            tc_fence_before_sync();
            mbar_arrive_relaxed(&acce[a]);                  // the MMA warp may reuse it
        }
    }

    // ---- teardown: on a timeout, wait (bounded) for what this CTA still has in flight
    __syncthreads();
    if (*abort_flag) {
        if (threadIdx.x == 0)
            flag(P.dev_err, KVQ_DEVERR_WAIT_TIMEOUT);
        if (warp == C::EPI_WARPS && lane == 0)             // copies never consumed
            for (int k = consumed; k < issued; ++k)
                mbar_wait_bounded(&full[k % C::STAGES], (k / C::STAGES) & 1);
        if (warp == C::EPI_WARPS + 1 && lane == 0 && consumed > 0)   // the last MMAs
            mbar_wait_bounded(&accf[(consumed - 1) % C::EPI], ((consumed - 1) / C::EPI) & 1);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Tensor map over in[tokens][Hkv][D] bf16: dims (D, Hkv, tokens), box (64, 1, 128) with the
// 128-byte swizzle; rows past the last token read as zeros.
bool make_input_map(CUtensorMap *m, const void *base, int D, int Hkv, long tokens)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
    cuuint32_t box[3] = {kTcKBlock, 1, kTcTile};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int GS>
cudaError_t launch_tc_t(const void *k, const void *v, const float *Tk, const float *Tv, int B, int n,
                        const kvq_cache *c, int clip, const int32_t *pos, int32_t *dev_err,
                        cudaStream_t st)
{
    using Cf = TcCfg<D>;
    static unsigned long long attr_done = 0;
    cudaError_t e = ensure_dynamic_smem(append_tc_kernel<D, GS>, Cf::SMEM, attr_done);
    if (e != cudaSuccess)
        return e;
    const long tokens = (long)B * n;
    CUtensorMap mk, mv;
    if (!make_input_map(&mk, k, D, c->Hkv, tokens) || !make_input_map(&mv, v, D, c->Hkv, tokens))
        return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long ntiles = (tokens + kTcTile - 1) / kTcTile;
    long gx = ((long)sms * Cf::PER_SM) / (2L * c->Hkv);
    if (gx < 1)
        gx = 1;
    if (gx > ntiles)
        gx = ntiles;
    TcParams P;
    P.Tk = Tk;
    P.Tv = Tv;
    P.B = B;
    P.n = n;
    P.Hkv = c->Hkv;
    P.T_cap = c->T_cap;
    P.bits_k = c->qp.bits_k;
    P.bits_v = c->qp.bits_v;
    P.clip = clip;
    P.k_codes = (uint8_t *)c->k_codes;
    P.k_sz = (uint32_t *)c->k_sz;
    P.v_codes = (uint8_t *)c->v_codes;
    P.v_sz = (uint32_t *)c->v_sz;
    P.pos = pos;
    P.dev_err = dev_err;
    P.pm = PageMap{c->block_table, c->page_tokens, c->num_pages};
    append_tc_kernel<D, GS><<<dim3((unsigned)gx, (unsigned)c->Hkv, 2), Cf::THREADS, Cf::SMEM, st>>>(
        mk, mv, P);
    return cudaGetLastError();
}

}  // namespace

// bf16 chunks with both transforms: X . T^T on tcgen05 tensor cores. Needs the inputs
// 16-byte aligned (tensor-map base) and B * n < 2^31 tokens.
cudaError_t append_tc(const void *k, const void *v, const float *Tk, const float *Tv, int B, int n,
                      const kvq_cache *c, int clip, const int32_t *pos, int32_t *dev_err,
                      cudaStream_t st)
{
    const int d = c->d, g = c->qp.group;
    if (d == 64 && g == 64)
        return launch_tc_t<64, 64>(k, v, Tk, Tv, B, n, c, clip, pos, dev_err, st);
    if (d == 64 && g == 32)
        return launch_tc_t<64, 32>(k, v, Tk, Tv, B, n, c, clip, pos, dev_err, st);
    if (d == 128 && g == 128)
        return launch_tc_t<128, 128>(k, v, Tk, Tv, B, n, c, clip, pos, dev_err, st);
    if (d == 128 && g == 64)
        return launch_tc_t<128, 64>(k, v, Tk, Tv, B, n, c, clip, pos, dev_err, st);
    if (d == 128 && g == 32)
        return launch_tc_t<128, 32>(k, v, Tk, Tv, B, n, c, clip, pos, dev_err, st);
    return cudaErrorInvalidValue;
}

}  // namespace kvq
