// kvq_quant.cuh -- quantisation of one K or V row by one warp (append step),
// shared by the append kernel and the fused append + decode kernel.
//
// Recipe per format ("NInfer KV Cache 量化指南：BF16、INT8、FP8、NVFP4 与 K8V4 五种格式怎么选",
// format paragraphs; "TokenSpeed量化实战", mxfp8 row of the --kv-cache-dtype
// table; "FP8 KV Cache如何提速 ... 长上下文推理", per-tensor symmetric fp8):
//   bf16 row -> [Hadamard-256] -> group amax -> scale rounded to its own format
//   -> codes = round-nearest-even(value / decoded scale), saturating.
// D/32 values per lane, a shuffle-based Hadamard, shuffle reductions for the
// group amax, one store per lane through the row's chunk permutation -- into
// one row, or into two (the fused decode writes the same row into its stage
// and into the cache; their row indices differ by a multiple of 64, so the
// chunk permutation is the same).
#pragma once

#include "kvq_internal.h"

namespace kvq {

// A lane's D/32 bf16 values of one row (16 B for D=256, 8 B for D=128).
struct RowBits {
    uint32_t w[4];
};
template <int D>
__device__ __forceinline__ RowBits load_row(const uint16_t* __restrict__ src, int lane) {
    RowBits r;
    if constexpr (D / 32 == 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + lane * 8);
        r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
    } else {
        const uint2 v = *reinterpret_cast<const uint2*>(src + lane * 4);
        r.w[0] = v.x; r.w[1] = v.y; r.w[2] = 0; r.w[3] = 0;
    }
    return r;
}

template <int KIND, int D>
__device__ __forceinline__ void quantize_loaded(const RowBits& rb, bool rot, float tscale, uint8_t* codes,
                                                uint8_t* scales, int t, int lane, uint8_t* codes2 = nullptr,
                                                uint8_t* scales2 = nullptr) {
    constexpr int EPL = D / 32;                 // values per lane
    constexpr int BITS = kind_bits(KIND);
    constexpr int BPL = EPL * BITS / 8;         // code bytes per lane
    float x[8];
    const uint32_t* raw = rb.w;
#pragma unroll
    for (int e = 0; e < EPL; e++) x[e] = bf16_bits_to_f32((raw[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
    if constexpr (EPL == 8) {
        if (rot) fwht256_warp(x, lane);
    }

    const int swz = row_swizzle(KIND, D, t);
    const int lane_off = phys_byte(lane * BPL, swz);
    uint32_t out[4] = {0, 0, 0, 0};

    if constexpr (KIND == RK_BF16RAW) {
#pragma unroll
        for (int i = 0; i < EPL / 2; i++) out[i] = raw[i];
    } else if constexpr (KIND == RK_FP16) {
#pragma unroll
        for (int i = 0; i < EPL / 2; i++) out[i] = enc_f16x2_sat(x[2 * i], x[2 * i + 1]);
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
            if (leader) {
                *reinterpret_cast<uint16_t*>(scales + 2 * g) = sb;
                if (scales2) *reinterpret_cast<uint16_t*>(scales2 + 2 * g) = sb;
            }
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
            if (leader) {
                scales[g] = (uint8_t)sb;
                if (scales2) scales2[g] = (uint8_t)sb;
            }
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
            if (leader) {
                scales[g] = nz ? (uint8_t)(E + 127) : (uint8_t)0;
                if (scales2) scales2[g] = scales[g];
            }
#pragma unroll
            for (int i = 0; i < EPL / 2; i++) {
                uint32_t c = nz ? enc_e4m3x2(__fmul_rn(x[2 * i], inv), __fmul_rn(x[2 * i + 1], inv)) : 0u;
                out[i >> 1] |= c << ((i & 1) * 16);
            }
        }
    }
    // store this lane's code bytes (a whole lane slice never straddles a 16-byte chunk)
    auto store = [&](uint8_t* dst) {
        if constexpr (BPL == 16) {
            *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
        } else if constexpr (BPL == 8) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(out[0], out[1]);
        } else if constexpr (BPL == 4) {
            *reinterpret_cast<uint32_t*>(dst) = out[0];
        } else {
            *reinterpret_cast<uint16_t*>(dst) = (uint16_t)out[0];
        }
    };
    store(codes + lane_off);
    if (codes2) store(codes2 + lane_off);
}

template <int KIND, int D>
__device__ __forceinline__ void quantize_row(const uint16_t* __restrict__ src, bool rot, float tscale,
                                             uint8_t* codes, uint8_t* scales, int t, int lane,
                                             uint8_t* codes2 = nullptr, uint8_t* scales2 = nullptr) {
    quantize_loaded<KIND, D>(load_row<D>(src, lane), rot, tscale, codes, scales, t, lane, codes2, scales2);
}

}  // namespace kvq
