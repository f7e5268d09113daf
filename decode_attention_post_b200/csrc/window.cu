// Full-precision window of the read path ("WUSH-KV: KV Cache Quantization with
// Data-Adaptive Transforms", section 4.4): attention over the positions a sequence keeps
// in full precision -- the first S_sink positions and those after the quantized middle --
// as one more partial (running max, sum of weights, weighted sum of values) next to the
// splits of the quantized middle, merged by the decode kernel's last split.
//
// One CTA per (KV head, sequence), 128 threads, for the G query heads of the KV head:
//   logit_t = log2(e)/sqrt(d) * q . k_t  (the query as given: q . k = (T_k^{-T} q) . (T_k k)),
//   m = max_t logit_t, p_t = 2^(logit_t - m), l = sum_t p_t, o = T_v sum_t p_t v_t,
// in float32 on CUDA cores (the window is a few hundred positions at most), T_v applied
// so that o is in the value-transform domain like the quantized values. The logits are in
// log2 units, as the decode kernel's partials. When nothing of the sequence is quantized
// the partial is the whole attention and o / l is written as the output.
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

constexpr int kWinThreads = 128;
constexpr float kWinLog2e = 1.4426950408889634f;

template <int D, int G>
__global__ void __launch_bounds__(kWinThreads) window_kernel(WindowParams W)
{
    extern __shared__ __align__(16) float wsm[];
    const int h = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int R = W.S_keep + W.S_flush;                 // recent ring slots
    const int WMAX = W.S_sink + R;                      // window positions at most
    float *qf = wsm;                                    // [G][D]
    float *of = qf + G * D;                             // [G][D]
    float *stat = of + G * D;                           // [G][2]: m, l
    float *lg = stat + 2 * G;                           // [G][WMAX]: logits, then weights

    int L = W.seqlens[b];
    L = L < 0 ? 0 : (L > W.max_seqlen ? W.max_seqlen : L);
    if (L == 0)
        return;                                         // the q prologue wrote zeros
    const int Q = window_quantized(L, W.S_sink, W.S_keep, W.S_flush);
    const int nsink = min(W.S_sink, L);
    const int rec0 = W.S_sink + Q;                      // first recent position
    const int nrec = L > rec0 ? L - rec0 : 0;
    const int nw = nsink + nrec;
    const size_t pair = (size_t)b * W.Hkv + h;
    const float sc = kWinLog2e * rsqrtf((float)D);

    // row of window position w (w < nsink: sink, else recent ring slot)
    auto k_row = [&](int w) -> const __nv_bfloat16 * {
        if (w < nsink)
            return reinterpret_cast<const __nv_bfloat16 *>(W.k_sink) +
                   (pair * W.S_sink + w) * D;
        const int t = rec0 + (w - nsink);
        return reinterpret_cast<const __nv_bfloat16 *>(W.k_recent) + (pair * R + t % R) * D;
    };
    auto v_row = [&](int w) -> const __nv_bfloat16 * {
        if (w < nsink)
            return reinterpret_cast<const __nv_bfloat16 *>(W.v_sink) +
                   (pair * W.S_sink + w) * D;
        const int t = rec0 + (w - nsink);
        return reinterpret_cast<const __nv_bfloat16 *>(W.v_recent) + (pair * R + t % R) * D;
    };

    for (int idx = tid; idx < G * D; idx += kWinThreads)
        qf[idx] = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(
            W.q)[((size_t)b * W.Hq + h * G + idx / D) * D + idx % D]);
    __syncthreads();
    // ---- logits: thread per (head, position)
    for (int idx = tid; idx < G * nw; idx += kWinThreads) {
        const int head = idx / nw, w = idx % nw;
        const __nv_bfloat16 *kr = k_row(w);
        const float *qh = qf + head * D;
        float acc = 0.f;
#pragma unroll 8
        for (int j = 0; j < D; ++j)
            acc = fmaf(qh[j], __bfloat162float(kr[j]), acc);
        lg[head * WMAX + w] = sc * acc;
    }
    __syncthreads();
    // ---- per head: max, weights 2^(logit - m), their sum
    for (int head = warp; head < G; head += kWinThreads / 32) {
        float m = -INFINITY;
        for (int w = lane; w < nw; w += 32)
            m = fmaxf(m, lg[head * WMAX + w]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float l = 0.f;
        for (int w = lane; w < nw; w += 32) {
            const float p = ex2(lg[head * WMAX + w] - m);
            lg[head * WMAX + w] = p;
            l += p;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            l += __shfl_xor_sync(0xffffffffu, l, off);
        if (lane == 0) {
            stat[2 * head] = m;
            stat[2 * head + 1] = l;
        }
    }
    __syncthreads();
    // ---- sum_t p_t v_t (untransformed values): thread per (head, dim)
    for (int idx = tid; idx < G * D; idx += kWinThreads) {
        const int head = idx / D, j = idx % D;
        float acc = 0.f;
        for (int w = 0; w < nw; ++w)
            acc = fmaf(lg[head * WMAX + w], __bfloat162float(v_row(w)[j]), acc);
        of[idx] = acc;
    }
    __syncthreads();
    // ---- o = T_v (sum p v), then the partial (or the output)
    const float *Tv = W.T_v ? W.T_v + (size_t)h * D * D : nullptr;
    float *part = W.part + (pair * W.part_slots + W.slot) * (size_t)(G * (D + 2));
    for (int idx = tid; idx < G * D; idx += kWinThreads) {
        const int head = idx / D, i = idx % D;
        float o = of[idx];
        if (Tv) {
            const float *row = Tv + (size_t)i * D;
            const float *oh = of + head * D;
            float acc = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; ++j)
                acc = fmaf(row[j], oh[j], acc);
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
        if (tid == 0) {
            __threadfence();
            atomicAdd(&W.ticket[pair], 1);
        }
    }
}

constexpr int kWinMaxPositions = 2048;       // S_sink + S_keep + S_flush limit (host-checked)

template <int D, int G>
constexpr size_t window_smem_bytes(int positions)
{
    return (size_t)(2 * G * D + 2 * G + G * positions) * sizeof(float);
}

template <int D, int G>
cudaError_t launch_window_t(const WindowParams &W, cudaStream_t st)
{
    const int WMAX = W.S_sink + W.S_keep + W.S_flush;
    // the attribute is set once per device for the largest window, so every call fits
    static unsigned long long attr_done = 0;
    cudaError_t e = ensure_dynamic_smem(window_kernel<D, G>,
                                        (int)window_smem_bytes<D, G>(kWinMaxPositions), attr_done);
    if (e != cudaSuccess)
        return e;
    window_kernel<D, G><<<dim3(W.Hkv, W.B), kWinThreads, window_smem_bytes<D, G>(WMAX), st>>>(W);
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
