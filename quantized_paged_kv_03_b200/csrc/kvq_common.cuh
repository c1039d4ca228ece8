// kvq_common.cuh -- formats, page layout and element codecs shared by the
// libkvq kernels (device) and the C-ABI layer (host).
//
// Formats ([NInfer] = "NInfer KV Cache 量化指南：BF16、INT8、FP8、NVFP4 与 K8V4 五种格式怎么选",
// format paragraphs and per-token byte table; [TokenSpeed] = "TokenSpeed量化实战：
// fp8、NVFP4与KV缓存压缩如何省下50%显存", --kv-cache-dtype table; [FP8-KV] =
// "FP8 KV Cache如何提速 ... 长上下文推理的加速秘密", kv_cache_scheme):
//   each stored row (one token, one kv-head, K or V) has a "row kind" that fixes
//   its code type, group size and scale type.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define KVQ_HD __host__ __device__ __forceinline__

namespace kvq {

constexpr int kHeaderBytes = 256;   // pool header: device status word(s)

enum RowKind : int {
    RK_BF16RAW = 0,      // bf16 bit pattern ([NInfer] BF16 paragraph: K kept bit for bit)
    RK_FP16 = 1,         // fp16, nearest-even, saturating ([NInfer] BF16 paragraph: V written as fp16)
    RK_E4M3_ROW256 = 2,  // E4M3 codes + fp16 scale per 256 values ([NInfer] FP8 row-256)
    RK_INT8_G64 = 3,     // int8 codes + fp16 scale per 64 values ([NInfer] INT8-G64)
    RK_E2M1_G16 = 4,     // E2M1 codes + UE4M3 scale per 16 values ([NInfer] NVFP4-G16)
    RK_E4M3_MX32 = 5,    // E4M3 codes + UE8M0 scale per 32 values ([TokenSpeed] mxfp8)
    RK_E4M3_TENSOR = 6   // E4M3 codes, one fp32 scale per tensor ([FP8-KV], [TokenSpeed] fp8_e4m3)
};

enum Format : int { F_BF16 = 0, F_FP8_ROW256 = 1, F_INT8_G64 = 2, F_NVFP4_G16 = 3, F_K8V4 = 4,
                    F_MXFP8_G32 = 5, F_FP8_TENSOR = 6, F_COUNT = 7 };

KVQ_HD constexpr int kind_of(int fmt, int is_v) {
    switch (fmt) {
    case F_BF16: return is_v ? RK_FP16 : RK_BF16RAW;
    case F_FP8_ROW256: return RK_E4M3_ROW256;
    case F_INT8_G64: return RK_INT8_G64;
    case F_NVFP4_G16: return RK_E2M1_G16;
    case F_K8V4: return is_v ? RK_E2M1_G16 : RK_E4M3_ROW256;
    case F_MXFP8_G32: return RK_E4M3_MX32;
    case F_FP8_TENSOR: return RK_E4M3_TENSOR;
    default: return -1;
    }
}

// [NInfer] format paragraphs: INT8 applies the 256-point Hadamard to K before
// it is written; NVFP4 applies it to both K and V; K8V4's V is NVFP4 and is
// rotated likewise.
KVQ_HD constexpr bool rotated(int fmt, int is_v) {
    switch (fmt) {
    case F_INT8_G64: return !is_v;
    case F_NVFP4_G16: return true;
    case F_K8V4: return is_v != 0;
    default: return false;
    }
}

KVQ_HD constexpr int kind_bits(int k) { return (k == RK_BF16RAW || k == RK_FP16) ? 16 : (k == RK_E2M1_G16 ? 4 : 8); }

// values per scale (0 = no per-row scale)
KVQ_HD constexpr int kind_group(int k) {
    switch (k) {
    case RK_E4M3_ROW256: return 256;
    case RK_INT8_G64: return 64;
    case RK_E2M1_G16: return 16;
    case RK_E4M3_MX32: return 32;
    default: return 0;
    }
}

KVQ_HD constexpr int kind_scale_bytes(int k) {   // bytes of one scale
    return (k == RK_E4M3_ROW256 || k == RK_INT8_G64) ? 2 : ((k == RK_E2M1_G16 || k == RK_E4M3_MX32) ? 1 : 0);
}

KVQ_HD constexpr int row_code_bytes(int k, int D) { return D * kind_bits(k) / 8; }
KVQ_HD constexpr int row_scale_bytes(int k, int D) { return kind_group(k) ? (D / kind_group(k)) * kind_scale_bytes(k) : 0; }

KVQ_HD constexpr bool kind_valid_for(int k, int D) {
    if (!(D == 128 || D == 256)) return false;
    int g = kind_group(k);
    return g == 0 || D % g == 0;
}

KVQ_HD constexpr int64_t align16(int64_t x) { return (x + 15) & ~int64_t(15); }

// Page slab of one (layer, page, kv-head): [K codes P x kc][K scales P x ks]
// [V codes P x vc][V scales P x vs], each region 16-byte aligned.  Within a
// code row the 16-byte chunks are permuted (chunk' = chunk ^ row_swizzle) so
// that the decode kernel's shared-memory reads of consecutive token rows hit
// distinct banks; scale rows are stored plainly.
struct Layout {
    int fmt, D, H, P, num_pages, num_layers;
    int kk, vk;                  // row kinds
    int kc, ks, vc, vs;          // row bytes
    int64_t off_ks, off_vc, off_vs, slab;
};

KVQ_HD Layout make_layout(int fmt, int D, int H, int P, int num_pages, int num_layers) {
    Layout L;
    L.fmt = fmt; L.D = D; L.H = H; L.P = P; L.num_pages = num_pages; L.num_layers = num_layers;
    L.kk = kind_of(fmt, 0); L.vk = kind_of(fmt, 1);
    L.kc = row_code_bytes(L.kk, D); L.ks = row_scale_bytes(L.kk, D);
    L.vc = row_code_bytes(L.vk, D); L.vs = row_scale_bytes(L.vk, D);
    L.off_ks = align16((int64_t)P * L.kc);
    L.off_vc = L.off_ks + align16((int64_t)P * L.ks);
    L.off_vs = L.off_vc + align16((int64_t)P * L.vc);
    L.slab = L.off_vs + align16((int64_t)P * L.vs);
    return L;
}

// 16-byte chunk permutation of code row t (see Layout).  Matches the decode
// kernel's read pattern: 16 B per lane over two rows per phase (8-bit rows),
// 8 B per lane over four rows per phase (E2M1 rows, MX rows), 32 B per lane
// over two rows (16-bit rows).
KVQ_HD constexpr int row_swizzle(int kind, int D, int t) {
    int bits = kind_bits(kind);
    int W = D * bits / 8;
    if (bits == 16) return t & 1;
    if (W < 128) return 0;
    if (bits == 4 || kind == RK_E4M3_MX32) return (t & 3) << 1;
    return (t & 1) << 2;
}

KVQ_HD constexpr int phys_byte(int logical, int swz) { return (((logical >> 4) ^ swz) << 4) | (logical & 15); }

// Device status word bits (pool header).
constexpr uint32_t kStatusBadSlot = 1u;
constexpr uint32_t kStatusBadPage = 2u;
constexpr uint32_t kStatusWaitTimeout = 4u;

#ifdef __CUDACC__

// ------------------------------------------------------------ encoders
// All encoders round to nearest-even and saturate at the format's largest
// finite value; the sign of zero is kept.

__device__ __forceinline__ uint16_t enc_f16_sat(float x) {
    uint16_t b = __half_as_ushort(__float2half_rn(x));
    if ((b & 0x7FFFu) == 0x7C00u) b = (uint16_t)((b & 0x8000u) | 0x7BFFu);   // +-inf -> +-65504
    return b;
}

// two fp16 codes (RNE, saturating to +-65504), `lo` in bits 0..15: one
// instruction for the pair; same results as enc_f16_sat on each value
__device__ __forceinline__ uint32_t enc_f16x2_sat(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// two E4M3 codes, `lo` in bits 0..7
__device__ __forceinline__ uint32_t enc_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// two E2M1 codes in one byte, `lo` in bits 0..3
__device__ __forceinline__ uint32_t enc_e2m1x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ int enc_int8(float x) {
    int v = __float2int_rn(x);
    return max(-127, min(127, v));
}

// ------------------------------------------------------------ decoders

// two E4M3 codes (bits 0..15) -> f16x2 (code in bits 0..7 -> low half); exact
__device__ __forceinline__ uint32_t dec_e4m3x2_f16x2(uint32_t v) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((uint16_t)v));
    return r;
}

// two E2M1 codes (byte: bits 0..3 -> low half) -> f16x2; exact
__device__ __forceinline__ uint32_t dec_e2m1x2_f16x2(uint32_t v) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "r"(v));
    return r;
}

// four int8 codes -> two f16x2 (exact): bias to unsigned, place under the
// exponent of 1024 (fp16 0x6400 + u has value 1024 + u), subtract 1152.
__device__ __forceinline__ void dec_int8x4_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    uint32_t u = w ^ 0x80808080u;
    uint32_t a, b;
    asm("prmt.b32 %0, %1, %2, 0x4140;" : "=r"(a) : "r"(u), "r"(0x64646464u));
    asm("prmt.b32 %0, %1, %2, 0x4342;" : "=r"(b) : "r"(u), "r"(0x64646464u));
    const uint32_t k1152 = 0x64806480u;   // (1152, 1152) in f16x2
    asm("sub.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(a), "r"(k1152));
    asm("sub.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(b), "r"(k1152));
}

__device__ __forceinline__ float f16_bits_to_f32(uint32_t h) { return __half2float(__ushort_as_half((uint16_t)h)); }
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
    return f16_bits_to_f32(dec_e4m3x2_f16x2(c & 0xFFu) & 0xFFFFu);
}
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
    return f16_bits_to_f32(dec_e2m1x2_f16x2(c & 0xFu) & 0xFFFFu);
}
// UE8M0 byte -> 2^(b-127) as fp32 (b = 0 -> 2^-127, a subnormal)
__device__ __forceinline__ float ue8m0_to_f32(uint32_t b) {
    return __uint_as_float(b ? (b << 23) : 0x00400000u);
}

// 2^e as fp32, exact, built from the exponent field: subnormal below 2^-126,
// 0 below 2^-149, +inf above 2^127.
__device__ __forceinline__ float pow2i(int e) {
    if (e > 127) return __uint_as_float(0x7F800000u);
    if (e >= -126) return __uint_as_float((uint32_t)(e + 127) << 23);
    if (e >= -149) return __uint_as_float(1u << (e + 149));
    return 0.f;
}
// floor(log2 x) of a positive finite fp32 value (-127 for every subnormal).
__device__ __forceinline__ int exp2_floor(float x) { return (int)(__float_as_uint(x) >> 23) - 127; }

// ------------------------------------------------------------ Hadamard-256
// Normalised Sylvester Hadamard of a 256-vector held 8 per lane (lane l holds
// elements 8l..8l+7).  Ascending butterfly stages h = 1..128, each pair giving
// (a + b, a - b) in fp32, then x 1/16: the evaluation order that fixes the bits
// of the stored codes.
__device__ __forceinline__ void fwht256_warp(float (&x)[8], int lane) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int e = 0; e < 8; e++) {
            if (!(e & h)) {
                float a = x[e], b = x[e + h];
                x[e] = __fadd_rn(a, b);
                x[e + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        bool upper = (lane & m) != 0;
#pragma unroll
        for (int e = 0; e < 8; e++) {
            float o = __shfl_xor_sync(0xffffffffu, x[e], m);
            x[e] = upper ? __fsub_rn(o, x[e]) : __fadd_rn(x[e], o);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; e++) x[e] = __fmul_rn(x[e], 0.0625f);
}

#endif  // __CUDACC__

}  // namespace kvq
