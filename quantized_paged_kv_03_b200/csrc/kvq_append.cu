// kvq_append.cu -- append kernel (quantise new K/V rows into their page slots)
// and the test-surface kernels (element encoder, logical row read-back,
// dequantisation).
//
// Append follows the per-format recipe of "NInfer KV Cache 量化指南：BF16、INT8、FP8、
// NVFP4 与 K8V4 五种格式怎么选" (format paragraphs) plus "TokenSpeed量化实战" (mxfp8
// row of the --kv-cache-dtype table) and "FP8 KV Cache如何提速 ... 长上下文推理"
// (per-tensor symmetric fp8):
//   bf16 row -> [Hadamard-256] -> group amax -> scale rounded to its own format
//   -> codes = round-nearest-even(value / decoded scale), saturating -> 16-byte
//   aligned stores into the slot's page slab.
// One warp owns kAppendRows consecutive (token, kv-head, K|V) rows, loading
// all of them before quantising each (quantize_loaded in kvq_quant.cuh).
#include "kvq_quant.cuh"

namespace kvq {

// -------------------------------------------------------------- append

constexpr int kAppendRows = 2;   // rows per warp, their loads in flight together

// Row and slot arithmetic in 32 bits (64-bit division is a long software
// sequence): the launch guarantees rows < 2^31; a slot below the pool capacity
// fits 32 bits whenever the capacity does (`p.cap32`), else 64-bit division.
template <int KK, int KV, int D>
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
    const int lane = threadIdx.x & 31;
    const uint32_t H = (uint32_t)p.L.H;
    const uint32_t nrows = (uint32_t)p.n_tokens * 2u * H;   // row = (token*2 + kv)*H + h
    const uint32_t row0 = ((uint32_t)blockIdx.x * 8u + (threadIdx.x >> 5)) * kAppendRows;
    RowBits raw[kAppendRows];
    int64_t slot[kAppendRows];
#pragma unroll
    for (int r = 0; r < kAppendRows; r++) {
        const uint32_t row = row0 + r;
        slot[r] = -1;
        if (row < nrows) {
            const uint32_t hk = row / H;                 // token*2 + kv
            const uint32_t h = row - hk * H, tok = hk >> 1;
            slot[r] = p.slots[tok];
            raw[r] = load_row<D>(((hk & 1) ? p.v : p.k) + ((int64_t)tok * H + h) * D, lane);
        }
    }
    const int64_t cap = (int64_t)p.L.num_pages * p.L.P;
#pragma unroll
    for (int r = 0; r < kAppendRows; r++) {
        const uint32_t row = row0 + r;
        if (slot[r] < 0) continue;   // past the end, or skipped by the caller
        if (slot[r] >= cap) {
            if (lane == 0) atomicOr(p.status, kStatusBadSlot);
            continue;
        }
        const uint32_t hk = row / H;
        const int h = (int)(row - hk * H), kv = (int)(hk & 1);
        int64_t page;
        int t;
        if (p.cap32) {
            const uint32_t sl = (uint32_t)slot[r], pg = sl / (uint32_t)p.L.P;
            page = pg;
            t = (int)(sl - pg * (uint32_t)p.L.P);
        } else {
            page = slot[r] / p.L.P;
            t = (int)(slot[r] % p.L.P);
        }
        uint8_t* slab = p.slabs + (page * p.L.H + h) * p.L.slab;
        if (kv == 0) {
            quantize_loaded<KK, D>(raw[r], p.rot_k, p.k_scale, slab + (int64_t)t * p.L.kc,
                                   slab + p.L.off_ks + (int64_t)t * p.L.ks, t, lane);
        } else {
            quantize_loaded<KV, D>(raw[r], p.rot_v, p.v_scale, slab + p.L.off_vc + (int64_t)t * p.L.vc,
                                   slab + p.L.off_vs + (int64_t)t * p.L.vs, t, lane);
        }
    }
}

// -------------------------------------------------------------- read rows

// Copy a stored row back in logical byte order (undo the chunk permutation).
__global__ void read_rows_kernel(ReadParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);   // (i*2 + kv)*H + h
    if (row >= (int64_t)p.n * 2 * p.L.H) return;
    const int h = (int)(row % p.L.H);
    const int kv = (int)((row / p.L.H) & 1);
    const int64_t i = row / (2 * p.L.H);
    const int64_t slot = p.slots[i];
    const int64_t cap = (int64_t)p.L.num_pages * p.L.P;
    if (slot < 0 || slot >= cap) return;
    const int64_t page = slot / p.L.P;
    const int t = (int)(slot % p.L.P);
    const uint8_t* slab = p.slabs + (page * p.L.H + h) * p.L.slab;
    const int kind = kv ? p.L.vk : p.L.kk;
    const int cb = kv ? p.L.vc : p.L.kc, sb = kv ? p.L.vs : p.L.ks;
    const uint8_t* crow = slab + (kv ? p.L.off_vc : 0) + (int64_t)t * cb;
    const uint8_t* srow = slab + (kv ? p.L.off_vs : p.L.off_ks) + (int64_t)t * sb;
    uint8_t* cdst = (kv ? p.v_codes : p.k_codes) + (i * p.L.H + h) * cb;
    uint8_t* sdst = (kv ? p.v_scales : p.k_scales);
    const int swz = row_swizzle(kind, p.L.D, t);
    for (int b = lane; b < cb; b += 32) cdst[b] = crow[phys_byte(b, swz)];
    if (sdst && sb)
        for (int b = lane; b < sb; b += 32) sdst[(i * p.L.H + h) * sb + b] = srow[b];
}

// -------------------------------------------------------------- dequant

__device__ __forceinline__ float dequant_elem(int kind, int D, const uint8_t* crow, const uint8_t* srow, int t,
                                              int d, float tscale) {
    const int swz = row_swizzle(kind, D, t);
    switch (kind) {
    case RK_BF16RAW: {
        int b = phys_byte(2 * d, swz);
        return bf16_bits_to_f32(crow[b] | (crow[b + 1] << 8));
    }
    case RK_FP16: {
        int b = phys_byte(2 * d, swz);
        return f16_bits_to_f32(crow[b] | (crow[b + 1] << 8));
    }
    case RK_E4M3_ROW256:
    case RK_INT8_G64: {
        int G = kind_group(kind), g = d / G;
        float s = f16_bits_to_f32(srow[2 * g] | (srow[2 * g + 1] << 8));
        uint32_t c = crow[phys_byte(d, swz)];
        float v = (kind == RK_INT8_G64) ? (float)(int8_t)c : e4m3_to_f32(c);
        return v * s;
    }
    case RK_E2M1_G16: {
        uint32_t c = (crow[phys_byte(d >> 1, swz)] >> ((d & 1) * 4)) & 0xF;
        return e2m1_to_f32(c) * e4m3_to_f32(srow[d / 16]);
    }
    case RK_E4M3_MX32:
        return e4m3_to_f32(crow[phys_byte(d, swz)]) * ue8m0_to_f32(srow[d / 32]);
    case RK_E4M3_TENSOR:
        return e4m3_to_f32(crow[phys_byte(d, swz)]) * tscale;
    default:
        return 0.f;
    }
}

__global__ void dequant_kernel(DequantParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= (int64_t)p.n * 2 * p.L.H) return;
    const int h = (int)(row % p.L.H);
    const int kv = (int)((row / p.L.H) & 1);
    const int64_t i = row / (2 * p.L.H);
    const int64_t slot = p.slots[i];
    const int64_t cap = (int64_t)p.L.num_pages * p.L.P;
    float* dst = (kv ? p.v_out : p.k_out) + (i * p.L.H + h) * p.L.D;
    if (slot < 0 || slot >= cap) {
        for (int d = lane; d < p.L.D; d += 32) dst[d] = 0.f;
        return;
    }
    const int64_t page = slot / p.L.P;
    const int t = (int)(slot % p.L.P);
    const uint8_t* slab = p.slabs + (page * p.L.H + h) * p.L.slab;
    const int kind = kv ? p.L.vk : p.L.kk;
    const uint8_t* crow = slab + (kv ? p.L.off_vc : 0) + (int64_t)t * (kv ? p.L.vc : p.L.kc);
    const uint8_t* srow = slab + (kv ? p.L.off_vs : p.L.off_ks) + (int64_t)t * (kv ? p.L.vs : p.L.ks);
    const float ts = kv ? p.v_scale : p.k_scale;
    for (int d = lane; d < p.L.D; d += 32) dst[d] = dequant_elem(kind, p.L.D, crow, srow, t, d, ts);
}

// -------------------------------------------------------------- encode

__global__ void encode_kernel(int code, const float* __restrict__ x, int64_t n, uint8_t* __restrict__ out) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float v = x[i];
    switch (code) {
    case 0: out[i] = (uint8_t)enc_e4m3x2(v, 0.f); break;
    case 1: out[i] = (uint8_t)(enc_e2m1x2(v, 0.f) & 0xF); break;
    case 2: out[i] = (uint8_t)(enc_int8(v) & 0xFF); break;
    case 3: reinterpret_cast<uint16_t*>(out)[i] = (uint16_t)(enc_f16x2_sat(v, 0.f) & 0xFFFFu); break;
    case 4: out[i] = (uint8_t)(enc_e4m3x2(v, 0.f) & 0x7F); break;
    default: break;
    }
}

// -------------------------------------------------------------- launchers

template <int KK, int KV>
static cudaError_t launch_append_kv(const AppendParams& p0, cudaStream_t s) {
    // launches of at most 2^30 rows (the kernel's row arithmetic is 32-bit)
    AppendParams p = p0;
    p.cap32 = (int64_t)p.L.num_pages * p.L.P < ((int64_t)1 << 31);
    const int64_t per = ((int64_t)1 << 30) / (2 * p.L.H);
    for (int64_t t0 = 0; t0 < p0.n_tokens; t0 += per) {
        p.n_tokens = (int)(p0.n_tokens - t0 < per ? p0.n_tokens - t0 : per);
        p.k = p0.k + t0 * p.L.H * p.L.D;
        p.v = p0.v + t0 * p.L.H * p.L.D;
        p.slots = p0.slots + t0;
        const int64_t rows = (int64_t)p.n_tokens * 2 * p.L.H;
        dim3 grid((unsigned)((rows + 8 * kAppendRows - 1) / (8 * kAppendRows)));
        if (p.L.D == 256) append_kernel<KK, KV, 256><<<grid, 256, 0, s>>>(p);
        else append_kernel<KK, KV, 128><<<grid, 256, 0, s>>>(p);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
    if (p.n_tokens <= 0) return cudaSuccess;
    switch (p.L.fmt) {
    case F_BF16: return launch_append_kv<RK_BF16RAW, RK_FP16>(p, s);
    case F_FP8_ROW256: return launch_append_kv<RK_E4M3_ROW256, RK_E4M3_ROW256>(p, s);
    case F_INT8_G64: return launch_append_kv<RK_INT8_G64, RK_INT8_G64>(p, s);
    case F_NVFP4_G16: return launch_append_kv<RK_E2M1_G16, RK_E2M1_G16>(p, s);
    case F_K8V4: return launch_append_kv<RK_E4M3_ROW256, RK_E2M1_G16>(p, s);
    case F_MXFP8_G32: return launch_append_kv<RK_E4M3_MX32, RK_E4M3_MX32>(p, s);
    case F_FP8_TENSOR: return launch_append_kv<RK_E4M3_TENSOR, RK_E4M3_TENSOR>(p, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_read_rows(const ReadParams& p, cudaStream_t s) {
    if (p.n <= 0) return cudaSuccess;
    int64_t rows = (int64_t)p.n * 2 * p.L.H;
    read_rows_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const DequantParams& p, cudaStream_t s) {
    if (p.n <= 0) return cudaSuccess;
    int64_t rows = (int64_t)p.n * 2 * p.L.H;
    dequant_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_encode(int code, const float* x, int64_t n, uint8_t* out, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    encode_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(code, x, n, out);
    return cudaGetLastError();
}

}  // namespace kvq
