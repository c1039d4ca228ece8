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
// A row is spread over D/32 lanes, 32 values each (quantize_lane32 below); the
// fused append + decode uses the warp-per-row form in kvq_quant.cuh, with the
// same arithmetic per value.
#include "kvq_quant.cuh"

namespace kvq {

// -------------------------------------------------------------- append
//
// A row (token, kv-head, K|V) is held by D/32 lanes, 32 consecutive values
// each, so that five of the Hadamard-256's eight butterfly stages and every
// group maximum but the row-256 one stay inside a lane; a warp takes 32/(D/32)
// rows (kAppendPasses times, all loads issued first).  Shuffles name only the
// row's own lanes, so rows of different kinds (K and V rows side by side when
// H is small) and rows past the end may diverge.  Every value goes through the
// same fp32 operations in the same order as in the warp-per-row quantiser of
// the fused decode, so both write the same codes.  (Measured on B200: one pass
// at four CTAs per SM beat two passes, three CTAs per SM, and a persistent
// grid with cp.async double buffering.)

constexpr int kAppendPasses = 1;

// Hadamard-256 of a row held 32 per lane by 8 lanes (lane li of the row holds
// elements 32 li .. 32 li + 31), without its final 1/16: ascending butterfly
// stages h = 1..128, each pair giving (a + b, a - b) in fp32.  Stages 1..16
// are in the lane; 32, 64, 128 pair lane li with li ^ 1, 2, 4, the upper
// element's a - b computed as fma(b, -1, a) (the same single rounding).  The
// 1/16 is exact (no value here is small enough to lose bits to it), so the
// callers fold it into their divisors: (x / 16) / s and x / (16 s) round alike.
__device__ __forceinline__ void fwht256_lanes8_unscaled(float (&x)[32], int li, unsigned gmask) {
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int e = 0; e < 32; e++) {
            if (!(e & h)) {
                const float a = x[e], b = x[e + h];
                x[e] = __fadd_rn(a, b);
                x[e + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) {
        const float sgn = (li & m) ? -1.f : 1.f;
#pragma unroll
        for (int e = 0; e < 32; e++) {
            const float o = __shfl_xor_sync(gmask, x[e], m);
            x[e] = __fmaf_rn(x[e], sgn, o);
        }
    }
}

// The 32 quotients x / d (correctly rounded) of a lane, as an encoder sees
// them.  qa = x * rs, rs = 1/d rounded and normal, lies within 2^-23 |q| of
// the quotient q, i.e. within a few units in the last place of the rounded
// quotient.  For a grid whose rounding boundaries all have at most MBITS bits
// after the leading one (E2M1: 2; E4M3: 4, its subnormal range included; the
// half-integers below 128: 7), unless qa is within 16 units of a value whose
// low 23 - MBITS mantissa bits are zero -- every boundary is one -- qa and the
// rounded quotient round to the same grid value, and qa is used.  If any of
// the lane's 32 is near one, all 32 are divided (rare: the branch is uniform
// in practice and the division code appears once).
template <int MBITS, int NG>
__device__ __forceinline__ void lane_quotients(const float (&x)[32], const float (&d)[NG], float (&q)[32]) {
    constexpr uint32_t kMask = (1u << (23 - MBITS)) - 1u, kNear = 16u;
    constexpr int GS = 32 / NG;   // values per divisor
    float rs[NG];
    bool near = false;
#pragma unroll
    for (int g = 0; g < NG; g++) {
        rs[g] = __frcp_rn(d[g]);
        near |= !(rs[g] >= 0x1p-126f && rs[g] <= 0x1p126f);
    }
#pragma unroll
    for (int e = 0; e < 32; e++) {
        q[e] = __fmul_rn(x[e], rs[e / GS]);
        near |= ((__float_as_uint(q[e]) + kNear) & kMask) < 2u * kNear;
    }
    if (near) {
#pragma unroll
        for (int e = 0; e < 32; e++) q[e] = __fdiv_rn(x[e], d[e / GS]);
    }
}

// Quantise one row's 32 values of this lane and store its codes (and, for the
// lane that leads a scale group, the group's scale) into the row's slots.
template <int KIND, int D>
__device__ __forceinline__ void quantize_lane32(const uint4 (&raw)[4], int li, unsigned gmask, bool rot, float tscale,
                                                uint8_t* codes, uint8_t* scales, int t) {
    constexpr int BITS = kind_bits(KIND);
    constexpr int BPL = 32 * BITS / 8;            // code bytes of the lane
    const uint32_t rw[16] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w, raw[1].x, raw[1].y, raw[1].z, raw[1].w,
                             raw[2].x, raw[2].y, raw[2].z, raw[2].w, raw[3].x, raw[3].y, raw[3].z, raw[3].w};
    uint32_t out[BPL / 4];
#pragma unroll
    for (int i = 0; i < BPL / 4; i++) out[i] = 0u;
    if constexpr (KIND == RK_BF16RAW) {
#pragma unroll
        for (int i = 0; i < 16; i++) out[i] = rw[i];
    } else {
        float x[32];
#pragma unroll
        for (int e = 0; e < 32; e++) x[e] = bf16_bits_to_f32((rw[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
        // f: the Hadamard's 1/16 still to divide by (1 without rotation)
        float f = 1.f;
        if constexpr (D == 256) {
            if (rot) {
                fwht256_lanes8_unscaled(x, li, gmask);
                f = 16.f;
            }
        }
        if constexpr (KIND == RK_FP16 || KIND == RK_E4M3_MX32) {
            // (no format rotates these kinds; kept exact if one did)
            if (f != 1.f) {
#pragma unroll
                for (int e = 0; e < 32; e++) x[e] = __fmul_rn(x[e], 0.0625f);
            }
        }
        if constexpr (KIND == RK_FP16) {
#pragma unroll
            for (int i = 0; i < 16; i++) out[i] = enc_f16x2_sat(x[2 * i], x[2 * i + 1]);
        } else if constexpr (KIND == RK_E4M3_TENSOR) {
            const float dd[1] = {f * tscale};
            float q[32];
            lane_quotients<4, 1>(x, dd, q);
#pragma unroll
            for (int i = 0; i < 16; i++) out[i >> 1] |= enc_e4m3x2(q[2 * i], q[2 * i + 1]) << ((i & 1) * 16);
        } else if constexpr (KIND == RK_E2M1_G16) {
            // two groups of 16 in the lane: UE4M3 scale amax / 6 each
            float d[2];
            uint32_t sb[2];
#pragma unroll
            for (int gg = 0; gg < 2; gg++) {
                float amax = 0.f;
#pragma unroll
                for (int e = 0; e < 16; e++) amax = fmaxf(amax, fabsf(x[16 * gg + e]));
                sb[gg] = enc_e4m3x2(__fdiv_rn(amax, f * 6.f), 0.f) & 0x7Fu;
                d[gg] = f * e4m3_to_f32(sb[gg]);
            }
            *reinterpret_cast<uint16_t*>(scales + 2 * li) = (uint16_t)(sb[0] | (sb[1] << 8));
            // (a zero scale gives zero codes; 1 keeps the quotients finite)
            const float dd[2] = {d[0] != 0.f ? d[0] : 1.f, d[1] != 0.f ? d[1] : 1.f};
            float q[32];
            lane_quotients<2, 2>(x, dd, q);
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const int gg = i >> 3;
                const uint32_t c = (sb[gg] != 0u) ? enc_e2m1x2(q[2 * i], q[2 * i + 1]) : 0u;
                out[i >> 2] |= c << ((i & 3) * 8);
            }
        } else if constexpr (KIND == RK_E4M3_MX32) {
            // one group of 32 in the lane: E = floor(log2 amax) - 8, codes of value x 2^-E
            float amax = 0.f;
#pragma unroll
            for (int e = 0; e < 32; e++) amax = fmaxf(amax, fabsf(x[e]));
            int e2;
            (void)frexpf(amax, &e2);
            const int E = min(127, max(-127, e2 - 1 - 8));
            const float inv = (-E == -127) ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(127 - E) << 23);
            const bool nz = amax > 0.f;
            scales[li] = nz ? (uint8_t)(E + 127) : (uint8_t)0;
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const uint32_t c = nz ? enc_e4m3x2(__fmul_rn(x[2 * i], inv), __fmul_rn(x[2 * i + 1], inv)) : 0u;
                out[i >> 1] |= c << ((i & 1) * 16);
            }
        } else {
            // INT8 (groups of 64: two lanes) and E4M3 row-256 (one group: eight lanes),
            // fp16 scale amax / qmax
            constexpr int LPG = kind_group(KIND) / 32 < D / 32 ? kind_group(KIND) / 32 : D / 32;
            float amax = 0.f;
#pragma unroll
            for (int e = 0; e < 32; e++) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
            for (int m = 1; m < LPG; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, m));
            const float qmax = (KIND == RK_E4M3_ROW256) ? 448.f : 127.f;
            const uint16_t sb = enc_f16_sat(__fdiv_rn(amax, f * qmax));
            const float sc = f16_bits_to_f32(sb);
            if (li % LPG == 0) *reinterpret_cast<uint16_t*>(scales + 2 * (li / LPG)) = sb;
            // a zero scale (all-zero group) gives zero codes; 1 keeps the quotients finite
            const float dd[1] = {sc != 0.f ? f * sc : 1.f};
            float q[32];
            lane_quotients<(KIND == RK_E4M3_ROW256) ? 4 : 7, 1>(x, dd, q);
            if constexpr (KIND == RK_E4M3_ROW256) {
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const uint32_t c = (sc != 0.f) ? enc_e4m3x2(q[2 * i], q[2 * i + 1]) : 0u;
                    out[i >> 1] |= c << ((i & 1) * 16);
                }
            } else {
                // past 128 both the rounded quotient and qa clamp to +-127
#pragma unroll
                for (int e = 0; e < 32; e++) {
                    const uint32_t c = (sc != 0.f) ? (uint32_t)(enc_int8(q[e]) & 0xFF) : 0u;
                    out[e >> 2] |= c << ((e & 3) * 8);
                }
            }
        }
    }
    // the lane's BPL / 16 chunks, each to its place under the row's chunk permutation
    const int swz = row_swizzle(KIND, D, t);
#pragma unroll
    for (int c = 0; c < BPL / 16; c++)
        *reinterpret_cast<uint4*>(codes + phys_byte(li * BPL + 16 * c, swz)) =
            make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
}

// Row and slot arithmetic in 32 bits (64-bit division is a long software
// sequence): the launch guarantees rows < 2^31; a slot below the pool capacity
// fits 32 bits whenever the capacity does (`p.cap32`), else 64-bit division.
template <int KK, int KV, int D>
__global__ void __launch_bounds__(256, 4) append_kernel(AppendParams p) {
    constexpr int LPR = D / 32, RPW = 32 / LPR;   // lanes per row, rows per warp and pass
    const int lane = threadIdx.x & 31, li = lane % LPR, sub = lane / LPR;
    const unsigned gmask = (LPR == 32) ? 0xffffffffu : (((1u << LPR) - 1u) << (sub * LPR));
    const uint32_t H = (uint32_t)p.L.H;
    const uint32_t nrows = (uint32_t)p.n_tokens * 2u * H;   // row = (token*2 + kv)*H + h
    const uint32_t row0 = ((uint32_t)blockIdx.x * 8u + (threadIdx.x >> 5)) * (uint32_t)(RPW * kAppendPasses) + sub;
    uint4 raw[kAppendPasses][4];
    int64_t slot[kAppendPasses];
#pragma unroll
    for (int r = 0; r < kAppendPasses; r++) {
        const uint32_t row = row0 + r * RPW;
        slot[r] = -1;
        if (row < nrows) {
            const uint32_t hk = row / H;                 // token*2 + kv
            const uint32_t h = row - hk * H, tok = hk >> 1;
            slot[r] = p.slots[tok];
            const uint4* src =
                reinterpret_cast<const uint4*>(((hk & 1) ? p.v : p.k) + ((int64_t)tok * H + h) * D + li * 32);
#pragma unroll
            for (int k = 0; k < 4; k++) raw[r][k] = __ldcs(src + k);
        }
    }
    const int64_t cap = (int64_t)p.L.num_pages * p.L.P;
#pragma unroll
    for (int r = 0; r < kAppendPasses; r++) {
        const uint32_t row = row0 + r * RPW;
        if (slot[r] < 0) continue;   // past the end, or skipped by the caller (the row's lanes alike)
        if (slot[r] >= cap) {
            if (li == 0) atomicOr(p.status, kStatusBadSlot);
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
            quantize_lane32<KK, D>(raw[r], li, gmask, p.rot_k, p.k_scale, slab + (int64_t)t * p.L.kc,
                                   slab + p.L.off_ks + (int64_t)t * p.L.ks, t);
        } else {
            quantize_lane32<KV, D>(raw[r], li, gmask, p.rot_v, p.v_scale, slab + p.L.off_vc + (int64_t)t * p.L.vc,
                                   slab + p.L.off_vs + (int64_t)t * p.L.vs, t);
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
        const int64_t per_cta = 8 * (32 / (p.L.D / 32)) * kAppendPasses;   // 8 warps
        dim3 grid((unsigned)((rows + per_cta - 1) / per_cta));
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
