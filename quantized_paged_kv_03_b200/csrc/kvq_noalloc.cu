// kvq_noalloc.cu -- decode attention for callers that cannot allocate device
// memory.
//
// kvq_decode_attention needs a caller-provided device workspace for its split
// partials and its merge counters.  Some callers have no way to provide one: a
// plugin handed only its input and output buffers by a host engine, a process
// running under a fixed device-memory budget that forbids new allocations
// after start-up, or a real-time loop where cudaMalloc/cudaFree (which may
// synchronise the device) are not allowed.  This entry point runs the same
// decode kernel with its scratch placed in a fixed array that is part of the
// library's device image, so the call itself allocates nothing.
#include <mutex>

#include "../../include/kvq.h"
#include "kvq_internal.h"

namespace {

// The scratch array.  Every GPU that loads this library holds these bytes
// until the process exits.  In host code `g_decode_scratch` is only a stand-in
// for the symbol, not a device address: its device address is looked up once
// per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on the
// first call for that device, with that device current).
int scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || !p) return KVQ_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KVQ_OK;
}

}  // namespace

extern "C" int kvq_decode_attention_noalloc(kvq_cache* cache, int32_t layer, const void* q, int32_t n_q_heads,
                                            const int32_t* block_table, int32_t max_pages_per_seq,
                                            const int32_t* seq_lens, int32_t batch, int32_t max_seq_len,
                                            void* out, int32_t out_fp32, float softmax_scale, void* stream) {
    // the same validation as kvq_decode_attention (same status codes), then the
    // scratch size limit, then -- only for a call that will launch -- the memset
    kvq::DecodeParams p;
    kvq::DecodePlan plan;
    bool none = false;
    int st = kvq::decode_setup(cache, layer, nullptr, nullptr, q, n_q_heads, block_table, max_pages_per_seq,
                               seq_lens, batch, max_seq_len, out, out_fp32, softmax_scale, &p, &none);
    if (st != KVQ_OK || none) return st;
    if ((st = kvq::decode_plan(&p, &plan)) != KVQ_OK) return st;
    const size_t need = kvq::decode_workspace_bytes(p.L, batch, p.HB, plan.grid);
    if (need > (size_t)KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_WORKSPACE;
    void* scratch = nullptr;
    st = scratch_for_current_device(&scratch);
    if (st != KVQ_OK) return st;
    // The array keeps whatever the previous call left there: clear the part
    // the kernel expects to start at zero.
    size_t zoff = 0, zbytes = 0;
    kvq::decode_workspace_zero_region(p.L, batch, p.HB, plan.grid, &zoff, &zbytes);
    if (cudaMemsetAsync((unsigned char*)scratch + zoff, 0, zbytes, (cudaStream_t)stream) != cudaSuccess)
        return KVQ_ERR_CUDA;
    return kvq::decode_launch(&p, plan, scratch, (cudaStream_t)stream);
}
