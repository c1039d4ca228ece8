// kvq_internal.h -- kernel parameter blocks and launchers used by the C-ABI layer.
#pragma once

#include "kvq_common.cuh"

namespace kvq {

struct AppendParams {
    Layout L;
    uint8_t* slabs;              // first slab of the layer
    const uint16_t* k;           // bf16 [n_tokens][H][D]
    const uint16_t* v;
    const int64_t* slots;
    int n_tokens;
    bool rot_k, rot_v;
    float k_scale, v_scale;      // per-tensor scales (FP8_TENSOR)
    uint32_t* status;
    bool cap32;                  // set by the launch: pool slots fit 31 bits
};

struct ReadParams {
    Layout L;
    const uint8_t* slabs;
    const int64_t* slots;
    int n;
    uint8_t *k_codes, *k_scales, *v_codes, *v_scales;
};

struct DequantParams {
    Layout L;
    const uint8_t* slabs;
    const int64_t* slots;
    int n;
    float k_scale, v_scale;
    float *k_out, *v_out;
};

// The unit a decode stage holds: a whole page (one copy of the page slab), or,
// for 128- and 256-token pages too large for the stage ring, 64 tokens of it
// (four copies: those rows of K codes, K scales, V codes, V scales).  A unit's
// stage layout is the page layout for its row count.
struct SpanLayout {
    int lg_up, sp;                       // log2(units per page), tokens per unit
    int off_ks, off_vc, off_vs, bytes;   // the unit's arrays in its stage
};
inline SpanLayout make_span(const Layout& L, int lg_up) {
    SpanLayout u;
    u.lg_up = lg_up;
    u.sp = L.P >> u.lg_up;
    u.off_ks = (int)align16((int64_t)u.sp * L.kc);
    u.off_vc = u.off_ks + (int)align16((int64_t)u.sp * L.ks);
    u.off_vs = u.off_vc + (int)align16((int64_t)u.sp * L.vc);
    u.bytes = u.off_vs + (int)align16((int64_t)u.sp * L.vs);
    return u;
}

struct DecodeParams {
    Layout L;
    SpanLayout U;                // set by the launch from L
    int seg_cost;                // set by the launch: a segment's fixed cost in units
    uint8_t* slabs;              // first slab of the layer (written only by the fused append)
    const uint16_t* q;           // bf16 [B][Hq][D]
    int Hq, G, HB;               // query heads, GQA group, 8-head blocks per kv-head
    const int32_t* block_table;
    int max_pages;
    const int32_t* seq_lens;
    int B;
    void* out;
    int out_fp32;
    float q_mult;                // softmax_scale * log2(e)
    float k_tmult;               // K tensor scale (FP8_TENSOR; 1 otherwise), applied to fp32 scores
    float o_mult;                // V tensor scale (1 otherwise)
    bool rot_k, rot_v;
    long wait_polls;             // polls of a pipeline wait before it gives up
    float* partials;             // [gridDim.x][2][16 + 8 * D]: (max, sum, output) of cut segments
    float* group_partials;       // [gridDim.x][16 + 8 * D]: merge of the group of parts ending in each CTA
    unsigned* grp_count;         // [gridDim.x] parts counted in of the group ending in each CTA (zero between calls)
    unsigned* seg_groups;        // [gridDim.x] groups counted in of the segment ending in each CTA (zero between calls)
    uint32_t* status;
    int stages;                  // pipeline depth (page slabs in shared memory)
    int pid_cap;                 // page ids of a CTA's range preloaded into shared memory
    const uint16_t* k_new;       // fused append: bf16 [B][H][D] rows of each sequence's newest
    const uint16_t* v_new;       //   token (position seq_len - 1), or null for decode only
    float k_scale, v_scale;      // per-tensor scales of the append (FP8_TENSOR)
    int max_seq_len;             // host-side: sizes the plan
};

// Polls a pipeline wait makes before it gives up (the default unless a test
// changed it with kvq_debug_set_wait_polls).
long wait_polls();

cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
cudaError_t launch_read_rows(const ReadParams& p, cudaStream_t s);
cudaError_t launch_dequant(const DequantParams& p, cudaStream_t s);
cudaError_t launch_encode(int code, const float* x, int64_t n, uint8_t* out, cudaStream_t s);

// Decode: grid / smem plan for a layout (host side), then the launch.
struct DecodePlan {
    int grid, stages, threads, pid_cap;
    int lg_up;                   // log2(stage units per page)
    size_t smem;
};
cudaError_t plan_decode(const Layout& L, int B, int HB, int max_seq_len, DecodePlan* plan);
size_t decode_workspace_bytes(const Layout& L, int B, int HB, int grid);
// Byte range of a decode workspace that must hold zeros when a call starts.
void decode_workspace_zero_region(const Layout& L, int B, int HB, int grid, size_t* offset, size_t* bytes);
cudaError_t launch_decode(const DecodeParams& p, const DecodePlan& plan, cudaStream_t s);
bool decode_supported(int fmt, int D);

}  // namespace kvq

struct kvq_cache;

namespace kvq {
// The C-ABI layer's decode path in steps (kvq_api.cu), shared by every decode
// entry point: validate on the host (kvq_status codes; *batch0 set when batch
// is 0 and there is nothing to launch), plan for the current device, launch
// on a workspace.
int decode_setup(kvq_cache* cache, int32_t layer, const void* k_new, const void* v_new, const void* q,
                 int32_t n_q_heads, const int32_t* block_table, int32_t max_pages_per_seq, const int32_t* seq_lens,
                 int32_t batch, int32_t max_seq_len, void* out, int32_t out_fp32, float softmax_scale,
                 DecodeParams* p, bool* batch0);
int decode_plan(DecodeParams* p, DecodePlan* plan);
int decode_launch(DecodeParams* p, const DecodePlan& plan, void* workspace, cudaStream_t stream);
}  // namespace kvq

// Page layout of a cache handle (defined with the handle in kvq_api.cu).
const kvq::Layout* kvq_cache_layout(const kvq_cache* cache);
