// kvq_prefill.h -- parameter block and launcher of the chunked-prefill
// attention kernel (kvq_prefill.cu), used by the C-ABI layer.
#pragma once

#include "kvq_common.cuh"

namespace kvq {

constexpr int kPrefillRows = 128;    // query rows (token, head) per CTA: 8 warps x 16
constexpr int kPrefillThreads = 256;

// Bytes of the first shared-memory region of a CTA at head_dim D and key tile
// T: during the key loop the 16-bit operand tiles of the tensor core -- q
// (128 x D), keys and values (T x D each) and the probabilities P (128 x T);
// in the epilogue the fp32 output rows (128 x (D + 4)).  Rounded up to 1 KB.
KVQ_HD constexpr int64_t prefill_region0(int D, int T) {
    const int64_t ops = ((int64_t)kPrefillRows * D + 2 * (int64_t)T * D + (int64_t)kPrefillRows * T) * 2;
    const int64_t osm = (int64_t)kPrefillRows * (D + 4) * 4;
    return ((ops > osm ? ops : osm) + 1023) & ~int64_t(1023);
}
// Bytes after the stage ring: the ring's mbarriers, the S and O completion
// mbarriers, the row exchange buffer (2 x 128 floats), the rows' q multipliers
// (128 floats), the tensor-memory address and the abort flag.
KVQ_HD constexpr int64_t prefill_tail_bytes(int stages) { return 8 * (stages + 2) + 3 * kPrefillRows * 4 + 16; }

// The warp-specialised kernel's shared memory: q (128 x D), double-buffered
// key and value tiles (T x D each) and P (128 x T), all 16-bit -- or, if larger,
// the fp32 output rows (128 x (D + 4)) of the epilogue -- rounded up to 1 KB;
// then 16 mbarriers, the rows' q multipliers (128 floats), a 32-word exchange
// buffer, the tensor-memory address and the abort flag.
KVQ_HD constexpr int64_t prefill_ws_region(int D, int T) {
    const int64_t ops = ((int64_t)kPrefillRows * D + 4 * (int64_t)T * D + 2 * (int64_t)kPrefillRows * T) * 2;
    const int64_t osm = (int64_t)kPrefillRows * (D + 4) * 4;
    return ((ops > osm ? ops : osm) + 1023) & ~int64_t(1023);
}
KVQ_HD constexpr int64_t prefill_ws_smem(int D, int T) { return prefill_ws_region(D, T) + 16 * 8 + kPrefillRows * 4 + 32 * 4 + 16; }

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
    long wait_polls;             // polls of a pipeline wait before it gives up
    uint32_t* status;
    // set by the launch from the plan
    int T;                       // key tile: tokens per stage (divides the page size)
    int st_ks, st_vc, st_vs, st_bytes;   // a stage's K-scale / V-code / V-scale offsets, size
    int stages;
};

struct PrefillPlan {
    int kernel;                  // 1: warp-specialised (prefill_ws_kernel), 0: every warp in every phase
    int T, stages;
    int st_ks, st_vc, st_vs, st_bytes;
    size_t smem;
};

bool prefill_supported(int fmt, int D);
cudaError_t plan_prefill(const Layout& L, PrefillPlan* plan);
cudaError_t launch_prefill(const PrefillParams& p, const PrefillPlan& plan, int64_t grid, cudaStream_t s);

}  // namespace kvq
