// kvq_api.cu -- the extern "C" boundary of libkvq (declared in include/kvq.h):
// argument validation on the host, page-layout bookkeeping, kernel launches.
// Nothing here allocates device memory.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "../../include/kvq.h"
#include "kvq_internal.h"
#include "kvq_prefill.h"

using namespace kvq;

struct kvq_cache {
    Layout L;
    uint8_t* pool;
    size_t pool_bytes;
    uint32_t flags;
    float* tensor_scales;   // host [num_layers][2]
};

const Layout* kvq_cache_layout(const kvq_cache* cache) { return cache ? &cache->L : nullptr; }

static int desc_layout(const kvq_cache_desc* d, Layout* out) {
    if (!d) return KVQ_ERR_ARG;
    if (d->format < 0 || d->format >= F_COUNT) return KVQ_ERR_FORMAT;
    const int D = d->head_dim;
    const int kk = kind_of(d->format, 0), vk = kind_of(d->format, 1);
    if (!kind_valid_for(kk, D) || !kind_valid_for(vk, D)) return KVQ_ERR_FORMAT;
    const bool rot = !(d->flags & KVQ_FLAG_NO_ROTATE) && (rotated(d->format, 0) || rotated(d->format, 1));
    if (rot && D != 256) return KVQ_ERR_FORMAT;
    if (d->n_kv_heads < 1 || d->num_layers < 1 || d->num_pages < 1) return KVQ_ERR_SHAPE;
    if (d->page_size < 16 || d->page_size > 256 || d->page_size % 16) return KVQ_ERR_SHAPE;
    if ((int64_t)d->num_pages * d->page_size > ((int64_t)1 << 40)) return KVQ_ERR_SHAPE;
    *out = make_layout(d->format, D, d->n_kv_heads, d->page_size, d->num_pages, d->num_layers);
    return KVQ_OK;
}

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

// Polls of a kernel's bounded pipeline waits (stage arrivals, MMA completion):
// about a second at the default; a test lowers it to make a wait give up.
static constexpr long long kDefaultWaitPolls = 1ll << 22;
static std::atomic<long long> g_wait_polls{kDefaultWaitPolls};
long kvq::wait_polls() { return (long)g_wait_polls.load(std::memory_order_relaxed); }

static uint8_t* layer_slabs(const kvq_cache* c, int layer) {
    const Layout& L = c->L;
    return c->pool + kHeaderBytes + (int64_t)layer * L.num_pages * L.H * L.slab;
}

extern "C" {

size_t kvq_token_bytes(int32_t format, int32_t head_dim) {
    if (format < 0 || format >= F_COUNT) return 0;
    const int kk = kind_of(format, 0), vk = kind_of(format, 1);
    if (!kind_valid_for(kk, head_dim) || !kind_valid_for(vk, head_dim)) return 0;
    return (size_t)row_code_bytes(kk, head_dim) + row_scale_bytes(kk, head_dim) + row_code_bytes(vk, head_dim) +
           row_scale_bytes(vk, head_dim);
}

int kvq_row_bytes(int32_t format, int32_t head_dim, int32_t is_v, int32_t* code_bytes, int32_t* scale_bytes) {
    if (format < 0 || format >= F_COUNT) return KVQ_ERR_FORMAT;
    const int k = kind_of(format, is_v ? 1 : 0);
    if (!kind_valid_for(k, head_dim)) return KVQ_ERR_FORMAT;
    if (code_bytes) *code_bytes = row_code_bytes(k, head_dim);
    if (scale_bytes) *scale_bytes = row_scale_bytes(k, head_dim);
    return KVQ_OK;
}

size_t kvq_cache_bytes(const kvq_cache_desc* desc) {
    Layout L;
    if (desc_layout(desc, &L) != KVQ_OK) return 0;
    return (size_t)kHeaderBytes + (size_t)L.num_layers * L.num_pages * L.H * (size_t)L.slab;
}

int kvq_cache_create(const kvq_cache_desc* desc, void* pool, size_t pool_bytes, kvq_cache** out) {
    if (!desc || !pool || !out) return KVQ_ERR_ARG;
    *out = nullptr;
    Layout L;
    int st = desc_layout(desc, &L);
    if (st != KVQ_OK) return st;
    if (((uintptr_t)pool & 255) != 0) return KVQ_ERR_ARG;
    if (pool_bytes < kvq_cache_bytes(desc)) return KVQ_ERR_WORKSPACE;
    kvq_cache* c = (kvq_cache*)calloc(1, sizeof(kvq_cache));
    if (!c) return KVQ_ERR_ARG;
    c->L = L;
    c->pool = (uint8_t*)pool;
    c->pool_bytes = pool_bytes;
    c->flags = desc->flags;
    c->tensor_scales = (float*)malloc(sizeof(float) * 2 * L.num_layers);
    if (!c->tensor_scales) {
        free(c);
        return KVQ_ERR_ARG;
    }
    for (int l = 0; l < L.num_layers; l++) {
        float ks = 1.f, vs = 1.f;
        if (desc->format == F_FP8_TENSOR && desc->tensor_scales) {
            ks = desc->tensor_scales[2 * l];
            vs = desc->tensor_scales[2 * l + 1];
            if (!(ks > 0.f) || !(vs > 0.f) || !isfinite(ks) || !isfinite(vs)) {
                free(c->tensor_scales);
                free(c);
                return KVQ_ERR_ARG;
            }
        }
        c->tensor_scales[2 * l] = ks;
        c->tensor_scales[2 * l + 1] = vs;
    }
    *out = c;
    return KVQ_OK;
}

int kvq_cache_destroy(kvq_cache* cache) {
    if (!cache) return KVQ_ERR_ARG;
    free(cache->tensor_scales);
    free(cache);
    return KVQ_OK;
}

static bool rot_of(const kvq_cache* c, int is_v) {
    return !(c->flags & KVQ_FLAG_NO_ROTATE) && rotated(c->L.fmt, is_v);
}

int kvq_append(kvq_cache* cache, int32_t layer, const void* k, const void* v, const int64_t* slot_mapping,
               int32_t n_tokens, void* stream) {
    if (!cache || n_tokens < 0 || layer < 0 || layer >= cache->L.num_layers) return KVQ_ERR_ARG;
    if (n_tokens == 0) return KVQ_OK;
    if (!k || !v || !slot_mapping) return KVQ_ERR_ARG;
    if (((uintptr_t)k & 15) || ((uintptr_t)v & 15) || ((uintptr_t)slot_mapping & 7)) return KVQ_ERR_ARG;
    AppendParams p;
    p.L = cache->L;
    p.slabs = layer_slabs(cache, layer);
    p.k = (const uint16_t*)k;
    p.v = (const uint16_t*)v;
    p.slots = slot_mapping;
    p.n_tokens = n_tokens;
    p.rot_k = rot_of(cache, 0);
    p.rot_v = rot_of(cache, 1);
    p.k_scale = cache->tensor_scales[2 * layer];
    p.v_scale = cache->tensor_scales[2 * layer + 1];
    p.status = (uint32_t*)cache->pool;
    return cuda_status(launch_append(p, (cudaStream_t)stream));
}

static int decode_shape(const kvq_cache* c, int32_t batch, int32_t n_q_heads, int32_t max_seq_len, int* G, int* HB) {
    if (!c || batch < 0 || n_q_heads < 1 || max_seq_len < 0) return KVQ_ERR_ARG;
    if (n_q_heads % c->L.H) return KVQ_ERR_SHAPE;
    if (!decode_supported(c->L.fmt, c->L.D)) return KVQ_ERR_FORMAT;
    if (batch > 4096) return KVQ_ERR_SHAPE;
    *G = n_q_heads / c->L.H;
    *HB = (*G + 7) / 8;
    return KVQ_OK;
}

size_t kvq_decode_workspace_bytes(const kvq_cache* cache, int32_t batch, int32_t n_q_heads, int32_t max_seq_len) {
    int G, HB;
    if (decode_shape(cache, batch, n_q_heads, max_seq_len, &G, &HB) != KVQ_OK) return 0;
    DecodePlan plan;
    if (plan_decode(cache->L, batch, HB, max_seq_len, &plan) != cudaSuccess) return 0;
    return decode_workspace_bytes(cache->L, batch, HB, plan.grid);
}

static int decode_common(kvq_cache* cache, int32_t layer, const void* k_new, const void* v_new, const void* q,
                         int32_t n_q_heads, const int32_t* block_table, int32_t max_pages_per_seq,
                         const int32_t* seq_lens, int32_t batch, int32_t max_seq_len, void* out, int32_t out_fp32,
                         float softmax_scale, void* workspace, size_t workspace_bytes, void* stream);

int kvq_decode_attention(kvq_cache* cache, int32_t layer, const void* q, int32_t n_q_heads, const int32_t* block_table,
                         int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch, int32_t max_seq_len,
                         void* out, int32_t out_fp32, float softmax_scale, void* workspace, size_t workspace_bytes,
                         void* stream) {
    return decode_common(cache, layer, nullptr, nullptr, q, n_q_heads, block_table, max_pages_per_seq, seq_lens,
                         batch, max_seq_len, out, out_fp32, softmax_scale, workspace, workspace_bytes, stream);
}

int kvq_append_decode(kvq_cache* cache, int32_t layer, const void* k_new, const void* v_new, const void* q,
                      int32_t n_q_heads, const int32_t* block_table, int32_t max_pages_per_seq,
                      const int32_t* seq_lens, int32_t batch, int32_t max_seq_len, void* out, int32_t out_fp32,
                      float softmax_scale, void* workspace, size_t workspace_bytes, void* stream) {
    if (batch > 0 && (!k_new || !v_new || ((uintptr_t)k_new & 15) || ((uintptr_t)v_new & 15))) return KVQ_ERR_ARG;
    return decode_common(cache, layer, k_new, v_new, q, n_q_heads, block_table, max_pages_per_seq, seq_lens, batch,
                         max_seq_len, out, out_fp32, softmax_scale, workspace, workspace_bytes, stream);
}

}  // extern "C"

// Validates a decode call on the host (every check that needs neither the
// device nor a workspace) and fills its kernel parameters.  *batch0 is set when there is nothing to
// launch (batch 0).  Shared by kvq_decode_attention, kvq_append_decode and the
// allocation-free entry point, so all three accept and reject the same calls.
int kvq::decode_setup(kvq_cache* cache, int32_t layer, const void* k_new, const void* v_new, const void* q,
                      int32_t n_q_heads, const int32_t* block_table, int32_t max_pages_per_seq,
                      const int32_t* seq_lens, int32_t batch, int32_t max_seq_len, void* out, int32_t out_fp32,
                      float softmax_scale, DecodeParams* pp, bool* batch0) {
    int G, HB;
    *batch0 = false;
    int st = decode_shape(cache, batch, n_q_heads, max_seq_len, &G, &HB);
    if (st != KVQ_OK) return st;
    if (layer < 0 || layer >= cache->L.num_layers) return KVQ_ERR_ARG;
    if (batch == 0) {
        *batch0 = true;
        return KVQ_OK;
    }
    if (!q || !block_table || !seq_lens || !out || max_pages_per_seq < 1) return KVQ_ERR_ARG;
    if ((int64_t)max_pages_per_seq * cache->L.P < max_seq_len) return KVQ_ERR_SHAPE;
    if (((uintptr_t)q & 15) || ((uintptr_t)out & 15)) return KVQ_ERR_ARG;
    if (!(softmax_scale >= 0.f) || !isfinite(softmax_scale)) return KVQ_ERR_ARG;
    // the kernel names a page slab by a 30-bit index (page * n_kv_heads + kv-head)
    if ((int64_t)cache->L.num_pages * cache->L.H >= ((int64_t)1 << 30)) return KVQ_ERR_SHAPE;
    DecodeParams& p = *pp;
    p.L = cache->L;
    p.slabs = layer_slabs(cache, layer);
    p.q = (const uint16_t*)q;
    p.Hq = n_q_heads;
    p.G = G;
    p.HB = HB;
    p.block_table = block_table;
    p.max_pages = max_pages_per_seq;
    p.seq_lens = seq_lens;
    p.B = batch;
    p.out = out;
    p.out_fp32 = out_fp32 ? 1 : 0;
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)cache->L.D);
    p.q_mult = scale * 1.4426950408889634f;
    p.k_tmult = cache->tensor_scales[2 * layer];
    p.o_mult = cache->tensor_scales[2 * layer + 1];
    p.rot_k = rot_of(cache, 0);
    p.rot_v = rot_of(cache, 1);
    p.wait_polls = kvq::wait_polls();
    p.partials = nullptr;
    p.group_partials = nullptr;
    p.grp_count = nullptr;
    p.seg_groups = nullptr;
    p.status = (uint32_t*)cache->pool;
    p.k_new = (const uint16_t*)k_new;
    p.v_new = (const uint16_t*)v_new;
    p.k_scale = cache->tensor_scales[2 * layer];
    p.v_scale = cache->tensor_scales[2 * layer + 1];
    p.max_seq_len = max_seq_len;
    return KVQ_OK;
}

// The launch plan of a set-up decode (queries the current device).
int kvq::decode_plan(DecodeParams* p, DecodePlan* plan) {
    if (plan_decode(p->L, p->B, p->HB, p->max_seq_len, plan) != cudaSuccess) return KVQ_ERR_CUDA;
    p->stages = plan->stages;
    p->pid_cap = plan->pid_cap;
    return KVQ_OK;
}

// Points a set-up decode at its workspace (which must be large enough) and launches it.
int kvq::decode_launch(DecodeParams* p, const DecodePlan& plan, void* workspace, cudaStream_t stream) {
    size_t zoff = 0, zbytes = 0;
    decode_workspace_zero_region(p->L, p->B, p->HB, plan.grid, &zoff, &zbytes);
    p->partials = (float*)workspace;
    p->group_partials = p->partials + (size_t)plan.grid * 2 * (16 + 8 * (size_t)p->L.D);
    p->grp_count = (unsigned*)((uint8_t*)workspace + zoff);
    p->seg_groups = p->grp_count + plan.grid;
    return cuda_status(launch_decode(*p, plan, stream));
}

extern "C" {

static int decode_common(kvq_cache* cache, int32_t layer, const void* k_new, const void* v_new, const void* q,
                         int32_t n_q_heads, const int32_t* block_table, int32_t max_pages_per_seq,
                         const int32_t* seq_lens, int32_t batch, int32_t max_seq_len, void* out, int32_t out_fp32,
                         float softmax_scale, void* workspace, size_t workspace_bytes, void* stream) {
    DecodeParams p;
    DecodePlan plan;
    bool none = false;
    int st = decode_setup(cache, layer, k_new, v_new, q, n_q_heads, block_table, max_pages_per_seq, seq_lens, batch,
                          max_seq_len, out, out_fp32, softmax_scale, &p, &none);
    if (st != KVQ_OK || none) return st;
    if (!workspace || ((uintptr_t)workspace & 15)) return KVQ_ERR_ARG;
    if ((st = decode_plan(&p, &plan)) != KVQ_OK) return st;
    if (workspace_bytes < decode_workspace_bytes(cache->L, batch, p.HB, plan.grid)) return KVQ_ERR_WORKSPACE;
    return decode_launch(&p, plan, workspace, (cudaStream_t)stream);
}

int kvq_prefill_attention(kvq_cache* cache, int32_t layer, const void* q, int32_t n_q_heads,
                          const int32_t* cu_q_lens, int32_t max_q_len, const int32_t* block_table,
                          int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch, void* out,
                          int32_t out_fp32, float softmax_scale, void* stream) {
    if (!cache || layer < 0 || layer >= cache->L.num_layers) return KVQ_ERR_ARG;
    if (batch < 0 || n_q_heads < 1 || max_q_len < 0) return KVQ_ERR_ARG;
    if (n_q_heads % cache->L.H) return KVQ_ERR_SHAPE;
    if (!prefill_supported(cache->L.fmt, cache->L.D)) return KVQ_ERR_FORMAT;
    if (batch == 0 || max_q_len == 0) return KVQ_OK;
    if (!q || !cu_q_lens || !block_table || !seq_lens || !out || max_pages_per_seq < 1) return KVQ_ERR_ARG;
    if (((uintptr_t)q & 15) || ((uintptr_t)out & 15)) return KVQ_ERR_ARG;
    if (!(softmax_scale >= 0.f) || !isfinite(softmax_scale)) return KVQ_ERR_ARG;
    PrefillPlan plan;
    if (plan_prefill(cache->L, &plan) != cudaSuccess) return KVQ_ERR_SHAPE;
    const int G = n_q_heads / cache->L.H;
    const int64_t slots = ((int64_t)max_q_len * G + kPrefillRows - 1) / kPrefillRows;
    const int64_t grid = (int64_t)batch * cache->L.H * slots;
    if (grid > 0x7FFFFFFF) return KVQ_ERR_SHAPE;
    PrefillParams p;
    memset(&p, 0, sizeof(p));
    p.L = cache->L;
    p.slabs = layer_slabs(cache, layer);
    p.q = (const uint16_t*)q;
    p.cu_q_lens = cu_q_lens;
    p.block_table = block_table;
    p.max_pages = max_pages_per_seq;
    p.seq_lens = seq_lens;
    p.B = batch;
    p.Hq = n_q_heads;
    p.G = G;
    p.slots = (int)slots;
    p.out = out;
    p.out_fp32 = out_fp32 ? 1 : 0;
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)cache->L.D);
    p.q_mult = scale * 1.4426950408889634f * cache->tensor_scales[2 * layer];
    p.o_mult = cache->tensor_scales[2 * layer + 1];
    p.rot_k = rot_of(cache, 0);
    p.rot_v = rot_of(cache, 1);
    p.wait_polls = kvq::wait_polls();
    p.status = (uint32_t*)cache->pool;
    return cuda_status(launch_prefill(p, plan, grid, (cudaStream_t)stream));
}

int kvq_dequant(kvq_cache* cache, int32_t layer, const int64_t* slots, int32_t n, float* k_out, float* v_out,
                void* stream) {
    if (!cache || n < 0 || layer < 0 || layer >= cache->L.num_layers) return KVQ_ERR_ARG;
    if (n == 0) return KVQ_OK;
    if (!slots || !k_out || !v_out) return KVQ_ERR_ARG;
    DequantParams p;
    p.L = cache->L;
    p.slabs = layer_slabs(cache, layer);
    p.slots = slots;
    p.n = n;
    p.k_scale = cache->tensor_scales[2 * layer];
    p.v_scale = cache->tensor_scales[2 * layer + 1];
    p.k_out = k_out;
    p.v_out = v_out;
    return cuda_status(launch_dequant(p, (cudaStream_t)stream));
}

int kvq_read_rows(kvq_cache* cache, int32_t layer, const int64_t* slots, int32_t n, uint8_t* k_codes,
                  uint8_t* k_scales, uint8_t* v_codes, uint8_t* v_scales, void* stream) {
    if (!cache || n < 0 || layer < 0 || layer >= cache->L.num_layers) return KVQ_ERR_ARG;
    if (n == 0) return KVQ_OK;
    if (!slots || !k_codes || !v_codes) return KVQ_ERR_ARG;
    if ((cache->L.ks && !k_scales) || (cache->L.vs && !v_scales)) return KVQ_ERR_ARG;
    ReadParams p;
    p.L = cache->L;
    p.slabs = layer_slabs(cache, layer);
    p.slots = slots;
    p.n = n;
    p.k_codes = k_codes;
    p.k_scales = k_scales;
    p.v_codes = v_codes;
    p.v_scales = v_scales;
    return cuda_status(launch_read_rows(p, (cudaStream_t)stream));
}

int kvq_encode(int32_t code, const float* x, int64_t n, uint8_t* out, void* stream) {
    if (code < KVQ_CODE_E4M3 || code > KVQ_CODE_UE4M3 || n < 0) return KVQ_ERR_ARG;
    if (n == 0) return KVQ_OK;
    if (!x || !out) return KVQ_ERR_ARG;
    return cuda_status(launch_encode(code, x, n, out, (cudaStream_t)stream));
}

int kvq_read_device_status(kvq_cache* cache, int32_t clear, uint32_t* status, void* stream) {
    if (!cache || !status) return KVQ_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(status, cache->pool, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && clear) {
        e = cudaMemsetAsync(cache->pool, 0, sizeof(uint32_t), s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    }
    return cuda_status(e);
}

const char* kvq_status_string(int status) {
    switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_ARG: return "invalid argument";
    case KVQ_ERR_FORMAT: return "format not supported for this head_dim";
    case KVQ_ERR_SHAPE: return "inconsistent or unsupported sizes";
    case KVQ_ERR_WORKSPACE: return "pool or workspace too small";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    case KVQ_ERR_DEVICE_BOUNDS: return "a kernel recorded an out-of-range index or a wait that gave up";
    default: return "unknown status";
    }
}

int64_t kvq_debug_set_wait_polls(int64_t polls) {
    return (int64_t)g_wait_polls.exchange(polls < 0 ? kDefaultWaitPolls : (long long)polls);
}

int kvq_version(void) { return KVQ_VERSION; }

}  // extern "C"
