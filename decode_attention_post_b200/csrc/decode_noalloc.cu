// Allocation-free variant of kvq_decode_attention.
//
// Some callers cannot hand the library a workspace: an inference engine that reserves
// nearly all device memory for its own KV pool at start-up (a further cudaMalloc fails
// or fragments that pool), or a latency-critical serving loop that forbids cudaMalloc
// because it synchronises the device. For them this entry point takes its scratch
// (split partials, query fragments, merge tickets) from a fixed array that the library
// itself declares in device memory, and allocates nothing.
//
// Costs and limits:
//  - every GPU that loads the library holds KVQ_NOALLOC_SCRATCH_BYTES (8 MiB) for this
//    array until the process exits;
//  - a call whose scratch need (kvq_decode_workspace_bytes) exceeds that size is
//    rejected with KVQ_ERR_WORKSPACE before anything is launched;
//  - all calls on one device share the array and it keeps the previous call's contents:
//    the query prologue rewrites every ticket to zero and every other section is written
//    before it is read, so stale contents are harmless; but two calls whose kernels
//    overlap on the GPU (different streams, no ordering between them) race on it;
//  - the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress, once per device, with that device current); make that first
//    call before any stream capture.
#include "kvq_common.cuh"

#include <mutex>

namespace kvq {
namespace {

constexpr size_t kNoallocScratchBytes = KVQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kMaxDevices];

// Device address of the scratch array for the current device (set-up on first use).
kvq_status noalloc_scratch(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        KVQ_FAIL(KVQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        KVQ_FAIL(KVQ_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            KVQ_FAIL(KVQ_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return KVQ_OK;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" KVQ_API kvq_status kvq_decode_attention_noalloc(
    const void *q, kvq_dtype q_dtype, int Hq, const float *Tk_invT, const kvq_cache *cache,
    const int32_t *seqlens, int max_seqlen, void *out, kvq_dtype out_dtype, int32_t *dev_err,
    kvq_stream_t stream)
{
    const size_t need = kvq_decode_workspace_bytes(cache, Hq, max_seqlen);
    if (need > kNoallocScratchBytes)
        KVQ_FAIL(KVQ_ERR_WORKSPACE,
                 "this decode needs %zu bytes of scratch; the allocation-free entry point "
                 "holds %zu (use kvq_decode_attention with a caller workspace)",
                 need, kNoallocScratchBytes);
    void *scratch = nullptr;
    kvq_status s = noalloc_scratch(&scratch);
    if (s != KVQ_OK)
        return s;
    // need == 0 means invalid arguments: the regular entry point reports which one.
    return kvq_decode_attention(q, q_dtype, Hq, Tk_invT, cache, seqlens, max_seqlen, out,
                                out_dtype, scratch, kNoallocScratchBytes, dev_err, stream);
}
