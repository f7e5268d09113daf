// Launch-time shapes shared by the decode kernels and the host-side C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kvq {

constexpr int kDecodeWarps = 4;     // warps per decode CTA
constexpr int kDecodeStages = 2;    // bulk-copy ring depth per warp
constexpr int kDecodeMinBlocks = 4; // resident CTAs per SM the register budget targets
constexpr int kDecodeBlock = 64;    // tokens per ring stage

struct DecodeParams {
    const uint8_t *k_codes;
    const uint32_t *k_sz;
    const uint8_t *v_codes;
    const uint32_t *v_sz;
    const int32_t *seqlens;
    int B, Hkv, Hq, T_cap, max_seqlen;
    int nsplit;          // CTAs per (sequence, KV head) along the tokens
    int split_tokens;    // tokens per split, a multiple of kDecodeBlock
    const uint32_t *qfrag;
    const float *qscale;
    const float *qw;
    float *part;
    int *ticket;
    void *out;
    int out_bf16;
    int32_t *dev_err;
    const int32_t *block_table; // paged cache: [B][T_cap/page_tokens]; nullptr = contiguous
    int page_tokens;
    int num_pages;
    int part_slots;             // partial slots per (sequence, KV head): split slots
                                // (>= nsplit) + 1, the last one for the window's partial
    // full-precision window (win_flush = 0: none): the cache holds the quantized middle,
    // seqlens are whole lengths; one more CTA per pair (grid slice z = 0) attends over the
    // window and its partial goes to the last slot
    int win_sink, win_keep, win_flush;
    const void *win_q;                                  // bfloat16 [B][Hq][d], as given
    const void *k_sink, *v_sink, *k_recent, *v_recent;  // bfloat16 window rows
    const float *win_Tv;                                // [Hkv][d][d] or nullptr
    // > 0: failure-path test hook, each warp first waits this long on a barrier that
    // nothing arrives at, then takes the timeout path (KVQ_TEST_STALL_NS in kvq.h)
    long long stall_test_ns;
};

struct DecodeLaunch {
    DecodeParams p;
    const void *q;
    int q_bf16;
    const float *M;
    int d, G, bits_k, bits_v;
};

// Byte offsets of the decode workspace sections (each 256-byte aligned).
struct DecodeWorkspace {
    size_t qfrag, qscale, qw, part, ticket, qt, total;
};

size_t decode_qfrag_words(int d, int G);
int decode_resident_ctas(int d, int G, int bk, int bv);
cudaError_t launch_decode(const DecodeLaunch &L, cudaStream_t st);
cudaError_t launch_qprep_qt(const DecodeLaunch &L, float *qt_out, cudaStream_t st);

// Vector-quantized decode: the query prologue (writing q~ to qt) and the VQ decode grid
// over the same split layout, partials, tickets and output as DecodeLaunch describes.
struct VqLaunch {
    DecodeLaunch L;
    float *qt;
    const uint8_t *k_idx, *v_idx;
    const uint16_t *k_gain, *v_gain;
    const uint16_t *cb_k, *cb_v;
};
cudaError_t launch_vq_decode(const VqLaunch &V, cudaStream_t st);


}  // namespace kvq
