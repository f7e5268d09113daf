// Shared device/host helpers of the kvq CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kTileTokens = 16;      // V codes are stored in 16-token tiles
constexpr int kQuestClip = -1;       // clip parameter of the append kernels: QuEST INT

// QuEST INT step in units of the group RMS: the uniform step of least mean squared
// error for a unit Gaussian with 2^bits levels (4 levels: 0.9957, 16 levels: 0.3352).
__host__ __device__ inline float quest_delta(int bits)
{
    return bits == 2 ? 0.9957f : 0.3352f;
}
constexpr int kCapAlign = 64;        // T_cap granularity (whole decode blocks)

// Correctly rounded a / b from y = RN(1/b) by Markstein's correction (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990): q0 = RN(a y) is within an ulp of a/b, the residual r = a - q0 b is
// exact in one fused multiply-add, and RN(q0 + r y) is RN(a / b) when nothing overflows or
// underflows -- here b is a positive float16 scale (a normal float32 number) and |a / b|
// stays far inside the float32 range. No branch and no call, so it can run for every
// value of a row; the quantizers then need no tie test (tests/test_division_method.py
// carries out these steps in exact arithmetic against the correctly rounded quotient, on
// random and near-tie operands; the append parity tests compare every code with the
// oracle's).
__device__ __forceinline__ float div_rn(float a, float b, float y)
{
    const float q0 = __fmul_rn(a, y);
    const float r = __fmaf_rn(-q0, b, a);
    return __fmaf_rn(r, y, q0);
}

// Bits of the device error word (see kvq.h).
__device__ __forceinline__ void flag(int32_t *dev_err, int32_t bit)
{
    if (dev_err)
        atomicOr(dev_err, bit);
}

__device__ __forceinline__ float load_in(const void *p, int bf16, size_t i)
{
    if (bf16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

// Byte offset, inside a 16-token V tile, of the 16-bit half that holds token `tok`
// (0..15) at the dims {8*(E*r + s) + gq : s < E}. Lane chunk 4*gq + tq holds tokens
// {tq, tq+4, tq+8, tq+12}; word p*W + r holds token tq+4p (low half) and tq+4p+8 (high).
__host__ __device__ __forceinline__ int v_half_offset(int d, int bits, int tok, int gq, int r)
{
    const int E = 16 / bits;
    const int W = d / (8 * E);
    const int chunk = d * bits / 16;
    const int tq = tok & 3, p = (tok >> 2) & 1, hi = tok >> 3;
    const int lane = 4 * gq + tq;
    return lane * chunk + (p * W + r) * 4 + 2 * hi;
}

// Quantized middle length of a sequence of L positions with a full-precision window
// (WUSH-KV section 4.4): the flush runs after every append and quantizes the oldest
// S_flush eligible positions while at least S_flush are eligible, so the middle
// [S_sink, S_sink + Q) holds Q = S_flush * floor(max(0, L - S_sink - S_keep) / S_flush).
__host__ __device__ inline int window_quantized(int L, int S_sink, int S_keep, int S_flush)
{
    const int e = L - S_sink - S_keep;
    return e > 0 ? (e / S_flush) * S_flush : 0;
}

// Where the positions of a (sequence, KV head) live: contiguous planes [B][Hkv][T_cap]
// (table == nullptr) or pages [page][Hkv][page_tokens] through a block table
// [B][T_cap / page_tokens].
struct PageMap {
    const int32_t *table;
    int page_tokens;
    int num_pages;
};

// Token slot (row of the K-code and scale/zero planes; value tiles hold slots
// 16i..16i+15) of position t of sequence b, KV head h. -1 if the block table holds a page
// outside [0, num_pages).
__device__ __forceinline__ long long cache_row(const PageMap &pm, int b, int h, int Hkv, int T_cap,
                                               int t)
{
    if (!pm.table)
        return ((long long)b * Hkv + h) * T_cap + t;
    const int page = pm.table[(size_t)b * (T_cap / pm.page_tokens) + t / pm.page_tokens];
    if ((unsigned)page >= (unsigned)pm.num_pages)
        return -1;
    return ((long long)page * Hkv + h) * pm.page_tokens + t % pm.page_tokens;
}

// Host-side: thread-local last error text.
void set_error(const char *fmt, ...);

// Host-side: cudaFuncSetAttribute(MaxDynamicSharedMemorySize) applies to the current
// device; `done_mask` remembers per device (ordinal mod 64) that it has been set, so the
// driver call happens once per kernel and device, before any stream capture.
template <typename F>
cudaError_t ensure_dynamic_smem(F *func, int bytes, unsigned long long &done_mask)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (done_mask & bit)
        return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        done_mask |= bit;
    return e;
}

}  // namespace kvq

#define KVQ_FAIL(code, ...)                 \
    do {                                    \
        ::kvq::set_error(__VA_ARGS__);      \
        return code;                        \
    } while (0)
