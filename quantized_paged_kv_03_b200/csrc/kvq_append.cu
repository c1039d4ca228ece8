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
// One warp owns one (token, kv-head, K|V) row: D/32 values per lane, a
// shuffle-based Hadamard, shuffle reductions for the group amax.
#include "kvq_internal.h"

namespace kvq {

// -------------------------------------------------------------- append

template <int KIND, int D>
__device__ __forceinline__ void quantize_row(const uint16_t* __restrict__ src, bool rot, float tscale,
                                             uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                             int t, int lane) {
    constexpr int EPL = D / 32;                 // values per lane
    constexpr int BITS = kind_bits(KIND);
    constexpr int BPL = EPL * BITS / 8;         // code bytes per lane
    float x[8];
    uint32_t raw[4];
    // load EPL bf16 values (16 B for D=256, 8 B for D=128)
    if constexpr (EPL == 8) {
        uint4 v = *reinterpret_cast<const uint4*>(src + lane * 8);
        raw[0] = v.x; raw[1] = v.y; raw[2] = v.z; raw[3] = v.w;
    } else {
        uint2 v = *reinterpret_cast<const uint2*>(src + lane * 4);
        raw[0] = v.x; raw[1] = v.y; raw[2] = 0; raw[3] = 0;
    }
#pragma unroll
    for (int e = 0; e < EPL; e++) x[e] = bf16_bits_to_f32((raw[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
    if constexpr (EPL == 8) {
        if (rot) fwht256_warp(x, lane);
    }

    const int swz = row_swizzle(KIND, D, t);
    uint8_t* dst = codes + phys_byte(lane * BPL, swz);
    uint32_t out[4] = {0, 0, 0, 0};

    if constexpr (KIND == RK_BF16RAW) {
#pragma unroll
        for (int i = 0; i < EPL / 2; i++) out[i] = raw[i];
    } else if constexpr (KIND == RK_FP16) {
#pragma unroll
        for (int i = 0; i < EPL / 2; i++) out[i] = enc_f16_sat(x[2 * i]) | ((uint32_t)enc_f16_sat(x[2 * i + 1]) << 16);
    } else if constexpr (KIND == RK_E4M3_TENSOR) {
        // [FP8-KV]: one symmetric scale for the whole tensor; [TokenSpeed] unit scale = 1
#pragma unroll
        for (int i = 0; i < EPL / 2; i++) {
            uint32_t c = enc_e4m3x2(__fdiv_rn(x[2 * i], tscale), __fdiv_rn(x[2 * i + 1], tscale));
            out[i >> 1] |= c << ((i & 1) * 16);
        }
    } else {
        constexpr int GROUP = kind_group(KIND);
        constexpr int LPG = GROUP / EPL;          // lanes per group (power of two)
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; e++) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
        for (int m = 1; m < LPG; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
        const int g = (lane * EPL) / GROUP;       // this lane's group
        const bool leader = (lane % LPG) == 0;
        if constexpr (KIND == RK_E4M3_ROW256 || KIND == RK_INT8_G64) {
            const float qmax = (KIND == RK_E4M3_ROW256) ? 448.f : 127.f;
            uint16_t sb = enc_f16_sat(__fdiv_rn(amax, qmax));
            float s = f16_bits_to_f32(sb);
            if (leader) *reinterpret_cast<uint16_t*>(scales + 2 * g) = sb;
            if constexpr (KIND == RK_E4M3_ROW256) {
#pragma unroll
                for (int i = 0; i < EPL / 2; i++) {
                    uint32_t c = (s != 0.f) ? enc_e4m3x2(__fdiv_rn(x[2 * i], s), __fdiv_rn(x[2 * i + 1], s)) : 0u;
                    out[i >> 1] |= c << ((i & 1) * 16);
                }
            } else {
#pragma unroll
                for (int e = 0; e < EPL; e++) {
                    uint32_t c = (s != 0.f) ? (uint32_t)(enc_int8(__fdiv_rn(x[e], s)) & 0xFF) : 0u;
                    out[e >> 2] |= c << ((e & 3) * 8);
                }
            }
        } else if constexpr (KIND == RK_E2M1_G16) {
            uint32_t sb = enc_e4m3x2(__fdiv_rn(amax, 6.f), 0.f) & 0x7Fu;    // UE4M3
            float s = e4m3_to_f32(sb);
            if (leader) scales[g] = (uint8_t)sb;
#pragma unroll
            for (int i = 0; i < EPL / 2; i++) {
                uint32_t c = (s != 0.f) ? enc_e2m1x2(__fdiv_rn(x[2 * i], s), __fdiv_rn(x[2 * i + 1], s)) : 0u;
                out[i >> 2] |= c << ((i & 3) * 8);
            }
        } else if constexpr (KIND == RK_E4M3_MX32) {
            // shared exponent E = floor(log2 amax) - 8 (448 = 1.75 * 2^8), codes of value * 2^-E
            int e2;
            (void)frexpf(amax, &e2);
            int E = min(127, max(-127, e2 - 1 - 8));
            float inv = (-E == -127) ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(127 - E) << 23);
            bool nz = amax > 0.f;
            if (leader) scales[g] = nz ? (uint8_t)(E + 127) : (uint8_t)0;
#pragma unroll
            for (int i = 0; i < EPL / 2; i++) {
                uint32_t c = nz ? enc_e4m3x2(__fmul_rn(x[2 * i], inv), __fmul_rn(x[2 * i + 1], inv)) : 0u;
                out[i >> 1] |= c << ((i & 1) * 16);
            }
        }
    }
    // store this lane's code bytes (a whole lane slice never straddles a 16-byte chunk)
    if constexpr (BPL == 16) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
    } else if constexpr (BPL == 8) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(out[0], out[1]);
    } else if constexpr (BPL == 4) {
        *reinterpret_cast<uint32_t*>(dst) = out[0];
    } else {
        *reinterpret_cast<uint16_t*>(dst) = (uint16_t)out[0];
    }
}

template <int KK, int KV, int D>
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);   // ((token*2 + kv)*H + h)
    if (row >= (int64_t)p.n_tokens * 2 * p.L.H) return;
    const int h = (int)(row % p.L.H);
    const int kv = (int)((row / p.L.H) & 1);
    const int64_t tok = row / (2 * p.L.H);
    const int64_t slot = p.slots[tok];
    if (slot < 0) return;
    const int64_t cap = (int64_t)p.L.num_pages * p.L.P;
    if (slot >= cap) {
        if (lane == 0) atomicOr(p.status, kStatusBadSlot);
        return;
    }
    const int64_t page = slot / p.L.P;
    const int t = (int)(slot % p.L.P);
    uint8_t* slab = p.slabs + (page * p.L.H + h) * p.L.slab;
    const uint16_t* src = (kv ? p.v : p.k) + (tok * p.L.H + h) * D;
    if (kv == 0) {
        quantize_row<KK, D>(src, p.rot_k, p.k_scale, slab + (int64_t)t * p.L.kc, slab + p.L.off_ks + (int64_t)t * p.L.ks,
                            t, lane);
    } else {
        quantize_row<KV, D>(src, p.rot_v, p.v_scale, slab + p.L.off_vc + (int64_t)t * p.L.vc,
                            slab + p.L.off_vs + (int64_t)t * p.L.vs, t, lane);
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
    case 3: reinterpret_cast<uint16_t*>(out)[i] = enc_f16_sat(v); break;
    case 4: out[i] = (uint8_t)(enc_e4m3x2(v, 0.f) & 0x7F); break;
    default: break;
    }
}

// -------------------------------------------------------------- launchers

template <int KK, int KV>
static cudaError_t launch_append_kv(const AppendParams& p, cudaStream_t s) {
    int64_t rows = (int64_t)p.n_tokens * 2 * p.L.H;
    dim3 grid((unsigned)((rows + 7) / 8));
    if (p.L.D == 256) append_kernel<KK, KV, 256><<<grid, 256, 0, s>>>(p);
    else append_kernel<KK, KV, 128><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
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
