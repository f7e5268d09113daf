// Write side of the full-precision window ("WUSH-KV: KV Cache Quantization with
// Data-Adaptive Transforms", section 4.4): new tokens of a decode step go to the sink
// (positions below S_sink) or to the recent ring (slot t mod (S_keep + S_flush)). The read
// side is the window split of the decode grid (window_attn.cuh).
#include "kvq_common.cuh"
#include "decode_shapes.h"

namespace kvq {

namespace {

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

}  // namespace kvq
