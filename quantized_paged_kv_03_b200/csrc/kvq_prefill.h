// kvq_prefill.h -- parameter block and launcher of the chunked-prefill
// attention kernel (kvq_prefill.cu), used by the C-ABI layer.
#pragma once

#include "kvq_common.cuh"

namespace kvq {

constexpr int kPrefillRows = 128;    // query rows (token, head) per CTA: 8 warps x 16
constexpr int kPrefillThreads = 256;

// Bytes of the first shared-memory region of a CTA at head_dim D and key tile
// T: q (128 rows) and the key and value tiles (T rows each) during the key
// loop, 16-bit elements with rows padded by 8; the per-warp fp32 output rows
// (padded by 4) in the epilogue.  Rounded up to 128 bytes.
KVQ_HD constexpr int64_t prefill_region0(int D, int T) {
    const int64_t qkv = (int64_t)(kPrefillRows + 2 * T) * (D + 8) * 2;
    const int64_t osm = (int64_t)(kPrefillThreads / 32) * 16 * (D + 4) * 4;
    return ((qkv > osm ? qkv : osm) + 127) & ~int64_t(127);
}

struct PrefillParams {
    Layout L;
    const uint8_t* slabs;        // first slab of the layer
    const uint16_t* q;           // bf16 [Tq][Hq][D]
    const int32_t* cu_q_lens;    // [B + 1] query-row offsets of each sequence
    const int32_t* block_table;  // [B][max_pages]
    int max_pages;
    const int32_t* seq_lens;     // [B] cached tokens, the chunk included
    int B, Hq, G;
    int slots;                   // CTAs per (sequence, kv-head); each takes every slots-th query block
    void* out;                   // [Tq][Hq][D], fp32 or bf16
    int out_fp32;
    float q_mult;                // softmax_scale * log2(e) * K tensor scale
    float o_mult;                // V tensor scale (1 otherwise)
    bool rot_k, rot_v;
    uint32_t* status;
    // set by the launch from the plan
    int T;                       // key tile: tokens per stage (divides the page size)
    int st_ks, st_vc, st_vs, st_bytes;   // a stage's K-scale / V-code / V-scale offsets, size
    int stages;
};

struct PrefillPlan {
    int T, stages;
    int st_ks, st_vc, st_vs, st_bytes;
    size_t smem;
};

bool prefill_supported(int fmt, int D);
cudaError_t plan_prefill(const Layout& L, PrefillPlan* plan);
cudaError_t launch_prefill(const PrefillParams& p, const PrefillPlan& plan, int64_t grid, cudaStream_t s);

}  // namespace kvq
