// kvq_prefill.cu -- chunked-prefill causal attention over the quantized pages.
//
// What it computes: sequence b holds seq_len cached tokens, of which the last
// n_b are a chunk of new query tokens (their K/V already appended).  Query
// token i of the chunk sits at position pos = seq_len - n_b + i; query head h
// (kv-head h / G) gets softmax(scale * q K[0..pos]^T) V[0..pos] -- causal, the
// token itself included -- with K and V read from the cache as code x scale.
// This is the multi-token form of the decode attention: the attention over the
// quantized cache that "NInfer KV Cache 量化指南" files under its causal_cache
// path (K8V4 paragraph), for a prompt processed in chunks.  A row whose
// position would be negative (a chunk longer than the sequence) has no keys
// and is written as zeros.
//
// Design (B200, sm_100a):
//  * One CTA per (sequence, kv-head, block of 128 query rows); a row is a
//    (query token, head of the GQA group) pair, so the G heads that share a
//    kv-head share every key tile, and the 128 rows are the M of the tensor
//    core's MMA.  A (sequence, kv-head)'s heaviest block (its last rows, which
//    see the most keys) starts first.
//  * Unlike decode, every key feeds many query rows: 4 x head_dim FLOPs per
//    (row, key), a dense contraction for the tensor cores.  A key tile (64
//    tokens, or fewer when the page size or shared memory asks) arrives by
//    cp.async.bulk into a two-stage ring; all 8 warps dequantise it once into
//    fp16 operand tiles in shared memory (scales folded in; BF16 keys stay
//    bf16, the format's own bits).
//  * S = Q K^T and O += P V run on tcgen05.mma (M = 128, N = the tile or
//    head_dim), issued by one thread, operands read from shared memory by the
//    tensor core, accumulators in tensor memory (O in columns [0, D), S in
//    [D, D + 64)).  Per tile: keys dequantised -> S issued -> values
//    dequantised while S runs (after the previous P V has released them) ->
//    every thread loads half of its row of S, the two halves exchange their
//    maxima, P = 2^(s - m) goes to shared memory -> P V issued; the next
//    tile's keys are dequantised while it runs.
//  * Online softmax in the log2 domain with a lazy reference maximum: O in
//    tensor memory is rescaled (load, multiply, store) only when a row's
//    maximum grows by more than 2^8, so weights stay below 256.  The causal
//    mask is applied on tiles that cross a lane group's first position.
//  * Rotated K: q is rotated by the Hadamard-256 when staged (orthonormal, so
//    q.k is unchanged); rotated V: each output row is rotated back in the
//    epilogue (the matrix is symmetric and its own inverse).
//
// Precision: q and the key/value tiles are fp16 (bf16 for BF16 keys).  Codes
// of every format are exact in fp16.  For INT8, E4M3 row-256 and MX, whose
// scales span more than fp16's range, values enter as code x scale x 2^-e, e
// the exponent of the sequence's largest K (or V) scale, found by one pass
// over the scale rows when the CTA starts; the 2^e goes back in fp32 (keys:
// into the score multiplier, values: into the output's normalisation).  So no
// value saturates, and the largest ones keep full fp16 precision whatever
// their magnitude; values far below the sequence's largest (by 2^14 or more)
// lose precision to fp16 subnormals, an absolute error below 2^-25 of the
// largest, negligible against the tolerance, which scales with max|V|.  What
// remains is one nearest-even rounding (relative 2^-11) of code x scale for
// INT8 and E4M3 row-256, whose fp16 scales carry 11 bits.  E2M1 x UE4M3 and
// per-tensor E4M3 (tensor scales applied in fp32) are exact.  q is normalised
// per row by a power of two (returned in fp32), so its magnitude is free too.
#include "kvq_prefill.h"
#include "kvq_tc.cuh"

namespace kvq {
namespace {

constexpr long kPrefillWaitPolls = 1l << 22;
constexpr int kMaxT = 64;   // largest key tile (tokens): S holds 64 tensor-memory columns

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(phase)
        : "memory");
    return ok != 0;
}
// Bounded wait: gives up after kPrefillWaitPolls polls, or at once when another
// thread already gave up (`abort` set), so a copy that never lands cannot hang
// the CTA; the caller records the timeout in the status word.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase, volatile int* abort,
                                          long polls = kPrefillWaitPolls) {
    for (long i = 0; i < polls; i++) {
        if (mbar_try_wait(bar, phase)) return true;
        if (*abort) return false;
    }
    *abort = 1;
    return false;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ uint32_t f16x2_of(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t bf16x2_of(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t mul_f16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ float2 f16x2_to_f32(uint32_t h) {
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}
// 2^x (softmax weights, x <= 8 here); -inf gives 0.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t splat16(uint32_t h) { return (h & 0xFFFFu) * 0x10001u; }

// ------------------------------------------------------------ tiles
//
// The operand tiles, 16-bit elements in 8 x 8 core matrices (kvq_tc.cuh):
//  * q, 128 rows x D, the K-major A of S: core (r/8, d/8) at ((r/8)(D/8) + d/8) x 128
//    (LBO 128, SBO 16 D);
//  * keys and values, T rows x D: each 8-column block holds the T rows' 16-byte
//    chunks in row order, core (t/8, d/8) at (d/8)(16 T) + (t/8) 128.  Keys are
//    the K-major B of S (LBO 16 T along head_dim, SBO 128 along the tokens),
//    values the MN-major B of P V (LBO 128 along the tokens, SBO 16 T along
//    head_dim);
//  * P, 128 rows x T, the K-major A of P V: core (r/8, t/8) at (t/8) 2048 + (r/8) 128
//    (LBO 2048, SBO 128).
// Rows of one 8-column block are consecutive 16-byte chunks, so threads that
// write consecutive rows of a block write one contiguous run (no bank conflict).

__device__ __forceinline__ uint32_t kv_off(int t, int d, int T) { return (uint32_t)((d >> 3) * (T << 4) + (t << 4)); }
__device__ __forceinline__ uint32_t p_off(int r, int c) { return (uint32_t)((c >> 3) * (kPrefillRows * 16) + (r << 4)); }

// Dequantise one 16-byte code chunk (chunk j of row t, logical order) into the
// tile, with the row's scales applied: 8, 16 or 32 elements by the code width.
// `smul` = 2^-e, e the sequence's scale exponent (sequence_scale_exps): INT8,
// E4M3 row-256 and MX scales enter as scale x 2^-e, so every dequantised value
// lies below 2 x the largest code, inside fp16's range.
template <int KIND>
__device__ __forceinline__ uint32_t chunk_scale_bits(const uint8_t* srow, int j) {
    if constexpr (kind_bits(KIND) == 4) {
        return (uint32_t)srow[2 * j] | ((uint32_t)srow[2 * j + 1] << 8);   // the chunk's two UE4M3 scales
    } else if constexpr (KIND == RK_INT8_G64 || KIND == RK_E4M3_ROW256) {
        const int g = j * 16 / kind_group(KIND);
        return (uint32_t)srow[2 * g] | ((uint32_t)srow[2 * g + 1] << 8);   // fp16 scale of the chunk's group
    } else if constexpr (KIND == RK_E4M3_MX32) {
        return srow[j * 16 / 32];                                          // UE8M0 scale of the chunk's group
    } else {
        return 0u;
    }
}

template <int KIND, int D>
__device__ __forceinline__ void dequant_chunk(const uint4 w, uint32_t sbits, int j, uint8_t* tile, int t, int T,
                                              float smul) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    if constexpr (kind_bits(KIND) == 16) {
        *reinterpret_cast<uint4*>(tile + kv_off(t, j * 8, T)) = w;   // bf16 keys / fp16 values: the stored bits
    } else if constexpr (kind_bits(KIND) == 4) {
        // 32 E2M1 codes (two groups of 16, UE4M3 scales): code x scale is exact in fp16
        const uint32_t sc = dec_e4m3x2_f16x2(sbits);
        const uint32_t s0 = splat16(sc), s1 = splat16(sc >> 16);
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 16; i++) h[i] = mul_f16x2(dec_e2m1x2_f16x2((ws[i >> 2] >> (8 * (i & 3))) & 0xFFu),
                                                      i < 8 ? s0 : s1);
#pragma unroll
        for (int i = 0; i < 4; i++)
            *reinterpret_cast<uint4*>(tile + kv_off(t, j * 32 + 8 * i, T)) =
                make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
    } else {
        // 16 eight-bit codes, all in one scale group
        uint32_t h[8];
        if constexpr (KIND == RK_INT8_G64) {
#pragma unroll
            for (int i = 0; i < 4; i++) dec_int8x4_f16x2(ws[i], h[2 * i], h[2 * i + 1]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) h[i] = dec_e4m3x2_f16x2(ws[i >> 1] >> (16 * (i & 1)));
        }
        if constexpr (KIND == RK_INT8_G64 || KIND == RK_E4M3_ROW256) {
            // fp16 scale: one nearest-even rounding of code x scale
            const float sf = f16_bits_to_f32(sbits) * smul;
            const uint32_t sc = splat16(__half_as_ushort(__float2half_rn(sf)));
#pragma unroll
            for (int i = 0; i < 8; i++) h[i] = mul_f16x2(h[i], sc);
        } else if constexpr (KIND == RK_E4M3_MX32) {
            // UE8M0 scale 2^(e-127): applied in fp32 (exact), then to fp16
            const float sc = ue8m0_to_f32(sbits) * smul;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float2 f = f16x2_to_f32(h[i]);
                h[i] = enc_f16x2_sat(f.x * sc, f.y * sc);
            }
        }
        *reinterpret_cast<uint4*>(tile + kv_off(t, j * 16, T)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(tile + kv_off(t, j * 16 + 8, T)) = make_uint4(h[4], h[5], h[6], h[7]);
    }
}

// Dequantise rows [0, T) of one array of a stage (codes: row stride
// row_code_bytes, chunk-permuted as stored; scales: plain rows) into a tile.
// Thread c takes row t = c % T and chunk (c / T + t) % (chunks per row): the
// 8 threads of a shared-memory phase read 8 different chunk columns and write
// 8 consecutive rows.  A thread loads all its chunks before converting any, so
// their shared-memory latencies overlap.  Rows at or past `valid` lie beyond
// the sequence's last token and hold no data: they are written as zeros, so
// that a masked key's weight 0 never meets a non-finite value.
template <int KIND, int D>
__device__ __forceinline__ void dequant_tile(const uint8_t* codes, const uint8_t* scales, uint8_t* tile, int T,
                                             int lgT, int valid, int tid, float smul) {
    constexpr int CB = row_code_bytes(KIND, D), SB = row_scale_bytes(KIND, D);
    constexpr int CPR = CB / 16;                       // chunks per row (a power of two)
    constexpr int EPC = 128 / kind_bits(KIND);         // elements per chunk
    constexpr int NPT = (kMaxT * CPR + kPrefillThreads - 1) / kPrefillThreads;   // chunks per thread, at most
    const int total = T * CPR;
    uint4 w[NPT];
#pragma unroll
    for (int i = 0; i < NPT; i++) {
        const int c = tid + i * kPrefillThreads;
        const int t = c & (T - 1), j = ((c >> lgT) + t) & (CPR - 1);
        w[i] = make_uint4(0, 0, 0, 0);
        if (c < total && t < valid)
            w[i] = *reinterpret_cast<const uint4*>(codes + t * CB + ((j ^ row_swizzle(KIND, D, t)) << 4));
    }
#pragma unroll
    for (int i = 0; i < NPT; i++) {
        const int c = tid + i * kPrefillThreads;
        const int t = c & (T - 1), j = ((c >> lgT) + t) & (CPR - 1);
        if (c >= total) continue;
        if (t >= valid) {
#pragma unroll
            for (int e = 0; e < EPC / 8; e++)
                *reinterpret_cast<uint4*>(tile + kv_off(t, j * EPC + 8 * e, T)) = make_uint4(0, 0, 0, 0);
        } else {
            dequant_chunk<KIND, D>(w[i], chunk_scale_bits<KIND>(scales + t * SB, j), j, tile, t, T, smul);
        }
    }
}

// Kinds whose dequantised values are normalised per tile (fp16 or UE8M0
// scales, whose range exceeds fp16's); E2M1 x UE4M3, per-tensor E4M3 and the
// 16-bit kinds are exact in fp16 as they are.
__host__ __device__ constexpr bool scale_normalised(int k) {
    return k == RK_INT8_G64 || k == RK_E4M3_ROW256 || k == RK_E4M3_MX32;
}

// Largest scale magnitude (as comparable bits: the fp16 pattern without its
// sign, or the UE8M0 byte) among `nb` bytes of scale rows at `src`, which
// is 16-byte aligned; bytes past nb are ignored.  Pieces of 16 bytes, lane l
// taking pieces l, l + 32, ...
template <int KIND>
__device__ __forceinline__ uint32_t scale_bits_max(const uint8_t* src, int nb, int lane) {
    uint32_t mx = 0;
    for (int i = lane; 16 * i < nb; i += 32) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const int rem = nb - 16 * i - 4 * k;   // bytes of this word that hold scales
            const uint32_t x = rem >= 4 ? w[k] : (rem > 0 ? w[k] & ((1u << (8 * rem)) - 1u) : 0u);
            if constexpr (KIND == RK_E4M3_MX32)
                mx = max(mx, max(max(x & 0xFFu, (x >> 8) & 0xFFu), max((x >> 16) & 0xFFu, x >> 24)));
            else
                mx = max(mx, max(x & 0x7FFFu, (x >> 16) & 0x7FFFu));
        }
    }
    return mx;
}

// floor(log2) of a scale given as scale_bits_max bits (0 for 0).
template <int KIND>
__device__ __forceinline__ int scale_exp_of_bits(uint32_t mx) {
    if (mx == 0) return 0;
    if constexpr (KIND == RK_E4M3_MX32) return (int)mx - 127;
    else return (int)max(mx >> 10, 1u) - 15;   // fp16 exponent field (subnormals: 2^-14)
}

// The scale exponents of a (sequence, kv-head): floor(log2) of its largest K
// and V scale over the cached tokens [0, Ls), the same in every thread of the
// CTA.  Every tile of the sequence is dequantised as code x scale x 2^-e, so
// every value lies below 2 x the largest code, and the 2^e goes back in fp32.
// One pass over the scale rows (16 bytes per token for INT8 at head_dim 256),
// once per CTA, while the ring's first copies are in flight.
template <int KK, int KV, int D, int NT = kPrefillThreads>
__device__ void sequence_scale_exps(const PrefillParams& p, int b, int hh, int Ls, uint32_t* red, int* ek, int* ev) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int NW = NT / 32;   // red holds 2 NW words
    uint32_t mk = 0, mv = 0;
    const int np = (Ls + p.L.P - 1) / p.L.P;
    // warp w takes 32 pages at a time (pages w*32 + 8*32*k + q), their ids loaded
    // by the lanes at once; each page id then comes from a shuffle, so the
    // scale loads of several pages are in flight together
    for (int pg0 = warp * 32; pg0 < np; pg0 += NW * 32) {
        int pid = -1;
        if (pg0 + lane < np && pg0 + lane < p.max_pages) pid = p.block_table[(int64_t)b * p.max_pages + pg0 + lane];
        if (pid < 0 || pid >= p.L.num_pages) pid = 0;   // recorded by the ring's copies
        const int cnt = min(32, np - pg0);
#pragma unroll 4
        for (int q = 0; q < cnt; q++) {
            const int id = __shfl_sync(0xffffffffu, pid, q);
            const uint8_t* slab = p.slabs + ((int64_t)id * p.L.H + hh) * p.L.slab;
            const int rows = min(p.L.P, Ls - (pg0 + q) * p.L.P);
            if constexpr (scale_normalised(KK)) mk = max(mk, scale_bits_max<KK>(slab + p.L.off_ks, rows * p.L.ks, lane));
            if constexpr (scale_normalised(KV)) mv = max(mv, scale_bits_max<KV>(slab + p.L.off_vs, rows * p.L.vs, lane));
        }
    }
    mk = __reduce_max_sync(0xffffffffu, mk);
    mv = __reduce_max_sync(0xffffffffu, mv);
    __syncthreads();   // `red` may still be read by the previous block's epilogue
    if (lane == 0) {
        red[warp] = mk;
        red[NW + warp] = mv;
    }
    __syncthreads();
    for (int w = 0; w < NW; w++) {
        mk = max(mk, red[w]);
        mv = max(mv, red[NW + w]);
    }
    *ek = scale_exp_of_bits<KK>(mk);
    *ev = scale_exp_of_bits<KV>(mv);
}

// Stage the block's 128 query rows into sQ: row r is global row R0 + r of the
// (sequence, kv-head), i.e. query token (R0 + r) / G, head (R0 + r) % G.  fp16
// (rotated by the Hadamard-256 first when K is rotated), or the bf16 bits
// themselves for BF16 keys; rows past the chunk are zeros.  One warp per row.
template <int D, bool QBF16, int NT = kPrefillThreads>
__device__ __forceinline__ void stage_q(const PrefillParams& p, uint8_t* sQ, float* qrm, int64_t qrow0, int hh,
                                        int64_t R0, int64_t rows_total, int warp, int lane) {
    constexpr int EPL = D / 32;
    for (int r = warp; r < kPrefillRows; r += NT / 32) {
        const int64_t gr = R0 + r;
        uint32_t bits[EPL / 2];
#pragma unroll
        for (int i = 0; i < EPL / 2; i++) bits[i] = 0;
        if (gr < rows_total) {
            const int64_t i = gr / p.G, g = gr % p.G;
            const uint16_t* src = p.q + ((qrow0 + i) * p.Hq + (int64_t)hh * p.G + g) * D + lane * EPL;
            if constexpr (EPL == 8) {
                const uint4 v = *reinterpret_cast<const uint4*>(src);
                bits[0] = v.x; bits[1] = v.y; bits[2] = v.z; bits[3] = v.w;
            } else {
                const uint2 v = *reinterpret_cast<const uint2*>(src);
                bits[0] = v.x; bits[1] = v.y;
            }
        }
        uint32_t h[EPL / 2];
        float rm = 1.f;   // the row's power of two, returned to its scores in fp32
        if constexpr (QBF16) {
#pragma unroll
            for (int i = 0; i < EPL / 2; i++) h[i] = bits[i];
        } else {
            float x[EPL];
#pragma unroll
            for (int i = 0; i < EPL / 2; i++) {
                x[2 * i] = bf16_bits_to_f32(bits[i] & 0xFFFFu);
                x[2 * i + 1] = bf16_bits_to_f32(bits[i] >> 16);
            }
            if constexpr (D == 256) {
                if (p.rot_k) fwht256_warp(x, lane);
            }
            // normalised so that the row's largest element lies in [1, 2): fp16
            // keeps full precision whatever q's magnitude
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < EPL; i++) amax = fmaxf(amax, fabsf(x[i]));
            amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
            const int eq = amax > 0.f ? exp2_floor(amax) : 0;
            const float nq = pow2i(-eq);
            rm = pow2i(eq);
#pragma unroll
            for (int i = 0; i < EPL / 2; i++) h[i] = enc_f16x2_sat(x[2 * i] * nq, x[2 * i + 1] * nq);
        }
        if (lane == 0) qrm[r] = rm;
        if constexpr (EPL == 8) {
            *reinterpret_cast<uint4*>(sQ + tc::blk(r, lane * 8, D)) = make_uint4(h[0], h[1], h[2], h[3]);
        } else {
            *reinterpret_cast<uint2*>(sQ + tc::blk(r, (lane * 4) & ~7, D) + (lane & 1) * 8) = make_uint2(h[0], h[1]);
        }
    }
}

// ------------------------------------------------------------ kernel

template <int KK, int KV, int D>
__global__ void __launch_bounds__(kPrefillThreads, 1) prefill_kernel(const PrefillParams p) {
    constexpr bool KBF = (KK == RK_BF16RAW);   // bf16 keys: S on bf16 operands
    constexpr int EPL = D / 32;                // output values per lane in the epilogue
    constexpr int OST = D + 4;                 // fp32 row stride of the output staging
    constexpr uint32_t kCols = D == 256 ? 512 : 256;   // tensor memory: O in [0, D), S in [D, D + 64)
    extern __shared__ __align__(1024) uint8_t smem[];
    const int T = p.T, lgT = 31 - __clz(T);
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + kPrefillRows * D * 2;
    uint8_t* sV = sK + T * D * 2;
    uint8_t* sP = sV + T * D * 2;
    float* sO = reinterpret_cast<float*>(smem);
    uint8_t* ring = smem + prefill_region0(D, T);
    uint64_t* bars = reinterpret_cast<uint64_t*>(ring + (size_t)p.stages * p.st_bytes);
    float* red = reinterpret_cast<float*>(bars + p.stages + 2);   // [2][128]: per-half row values
    float* qrm = red + 2 * kPrefillRows;                          // [128]: each row's q power of two
    uint32_t* tslot = reinterpret_cast<uint32_t*>(qrm + kPrefillRows);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int64_t idx = blockIdx.x;
    const int slot = (int)(idx % p.slots);
    idx /= p.slots;
    const int hh = (int)(idx % p.L.H);
    const int b = (int)(idx / p.L.H);
    const int64_t qrow0 = p.cu_q_lens[b];
    const int n = max(0, p.cu_q_lens[b + 1] - (int)qrow0);
    const int Ls = p.seq_lens[b];
    const int64_t rows_total = (int64_t)n * p.G;
    const int64_t nblk = (rows_total + kPrefillRows - 1) / kPrefillRows;
    if (slot >= nblk) return;

    const uint32_t barS = smem_addr(&bars[p.stages]), barO = smem_addr(&bars[p.stages + 1]);
    if (tid == 0) {
        for (int s = 0; s < p.stages + 2; s++) mbar_init(smem_addr(&bars[s]), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tc::alloc(smem_addr(tslot), kCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t tO = tmem, tS = tmem + D;

    // this thread's TMEM lane (= row of the block) and column half
    const int g4 = warp & 3, h = warp >> 2;
    const int r = g4 * 32 + lane;
    const uint32_t lane_bits = (uint32_t)(g4 * 32) << 16;
    const uint32_t idS = tc::idesc_f16(KBF, false, T), idO = tc::idesc_f16(false, true, D);
    const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV), aP = smem_addr(sP);

    // key tile k of this sequence into stage s: the whole page slab in one copy
    // when the tile is the page, else the tile's rows of the slab's four arrays
    // thread 0's counts of what it handed to the copy engine and the tensor
    // core: copies issued (ring positions 0 .. n_issued - 1), S and O commits
    uint32_t n_issued = 0, n_s = 0, n_o = 0;
    auto issue = [&](uint32_t seq, int k) {
        if (*abort_flag) return;   // after a wait gave up nothing new is started
        n_issued = seq + 1;
        const int s = (int)(seq % (uint32_t)p.stages);
        const int t0 = k * T;
        const int page = t0 / p.L.P;   // past the block table's width: a sequence longer than it holds
        int pid = page < p.max_pages ? p.block_table[(int64_t)b * p.max_pages + page] : -1;
        if (pid < 0 || pid >= p.L.num_pages) {
            atomicOr(p.status, kStatusBadPage);
            pid = 0;
        }
        const uint8_t* src = p.slabs + ((int64_t)pid * p.L.H + hh) * p.L.slab;
        const int64_t r0 = t0 % p.L.P;
        const uint32_t bar = smem_addr(&bars[s]);
        const uint32_t dst = smem_addr(ring + (size_t)s * p.st_bytes);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (T == p.L.P) {
            mbar_expect_tx(bar, (uint32_t)p.L.slab);
            bulk_g2s(dst, src, (uint32_t)p.L.slab, bar);
        } else {
            const uint32_t nk = T * p.L.kc, nks = T * p.L.ks, nv = T * p.L.vc, nvs = T * p.L.vs;
            mbar_expect_tx(bar, nk + nks + nv + nvs);
            bulk_g2s(dst, src + r0 * p.L.kc, nk, bar);
            if (nks) bulk_g2s(dst + (uint32_t)p.st_ks, src + p.L.off_ks + r0 * p.L.ks, nks, bar);
            bulk_g2s(dst + (uint32_t)p.st_vc, src + p.L.off_vc + r0 * p.L.vc, nv, bar);
            if (nvs) bulk_g2s(dst + (uint32_t)p.st_vs, src + p.L.off_vs + r0 * p.L.vs, nvs, bar);
        }
    };
    auto wait_or_flag = [&](uint32_t bar, uint32_t phase) {
        if (!mbar_wait(bar, phase, abort_flag, p.wait_polls) && lane == 0) atomicOr(p.status, kStatusWaitTimeout);
    };

    // key tiles of query block jb: those up to its largest position
    auto block_tiles = [&](int64_t jb) {
        const int64_t R0 = (nblk - 1 - jb) * kPrefillRows;   // the heaviest block first
        const int64_t r_last = min(R0 + kPrefillRows, rows_total) - 1;
        const int pos_hi = Ls - n + (int)(r_last / p.G);        // largest position in the block
        return pos_hi >= 0 ? pos_hi / T + 1 : 0;
    };
    // the first block's ring starts filling before the scale scan below
    if (tid == 0)
        for (int k = 0; k < p.stages && k < block_tiles(slot); k++) issue(k, k);

    // the sequence's scale exponents (INT8, E4M3 row-256, MX)
    int ek_seq = 0, ev_seq = 0;
    if constexpr (scale_normalised(KK) || scale_normalised(KV))
        sequence_scale_exps<KK, KV, D>(p, b, hh, Ls, reinterpret_cast<uint32_t*>(red), &ek_seq, &ev_seq);
    const float kmul = pow2i(-ek_seq), vmul = pow2i(-ev_seq);

    uint32_t seq = 0;   // key tiles consumed by this CTA: ring stage seq % stages, phase seq / stages
    uint32_t rnd = 0;   // MMA rounds (one S and one O per tile): phase of barS and barO
    for (int64_t jb = slot; jb < nblk; jb += p.slots) {
        const int64_t R0 = (nblk - 1 - jb) * kPrefillRows;
        const int ntiles = block_tiles(jb);
        if (tid == 0 && jb != slot)
            for (int k = 0; k < p.stages && k < ntiles; k++) issue(seq + k, k);
        stage_q<D, KBF>(p, sQ, qrm, qrow0, hh, R0, rows_total, warp, lane);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");

        // this thread's row position (-1: past the chunk, no keys) and the
        // smallest position among the 32 rows of its lane group
        const int64_t gr = R0 + r;
        const int pos = gr < rows_total ? Ls - n + (int)(gr / p.G) : -1;
        const int64_t gfirst = R0 + g4 * 32;
        const int gpos_min = gfirst + 31 < rows_total ? Ls - n + (int)(gfirst / p.G) : -1;
        float m_ref = -INFINITY, l_part = 0.f;
        __syncthreads();   // q staged
        const float qm = p.q_mult * pow2i(ek_seq) * qrm[r];   // this row's score multiplier

        for (int k = 0; k < ntiles; k++, seq++, rnd++) {
            const int s = (int)(seq % (uint32_t)p.stages);
            const uint8_t* st = ring + (size_t)s * p.st_bytes;
            wait_or_flag(smem_addr(&bars[s]), (seq / (uint32_t)p.stages) & 1u);
            const int t0 = k * T;
            const int valid = min(T, Ls - t0);
            // keys first: S of this tile can start while the values are dequantised
            dequant_tile<KK, D>(st, st + p.st_ks, sK, T, lgT, valid, tid, kmul);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncthreads();
            if (tid == 0 && !*abort_flag) {
                tc::fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++)
                    tc::mma_f16(tS, tc::sdesc(aQ + 256 * kk, 128, 16 * D), tc::sdesc(aK + kk * 32 * T, 16 * T, 128),
                                idS, kk > 0);
                tc::commit(barS);
                n_s++;
            }
            if (k > 0) {   // the previous P V still reads the value and P tiles
                wait_or_flag(barO, (rnd - 1) & 1u);
                tc::fence_after();
            }
            dequant_tile<KV, D>(st + p.st_vc, st + p.st_vs, sV, T, lgT, valid, tid, vmul);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");

            // ---- scores of this thread's row, columns [32 h, 32 h + 32) of the tile
            wait_or_flag(barS, rnd & 1u);
            tc::fence_after();
            const int c0 = h * 32;
            const bool active = c0 < T;   // with tiles of 32 or 16 keys the second half has none
            float sv[32];
            float mx = -INFINITY;
            if (active) {
                uint32_t v[32];
                tc::ld32(tS + lane_bits + c0, v);
                tc::wait_ld();
                const bool mask = t0 + T - 1 > gpos_min;
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    float x = __uint_as_float(v[i]) * qm;
                    if (c0 + i >= T || (mask && t0 + c0 + i > pos)) x = -INFINITY;
                    sv[i] = x;
                    mx = fmaxf(mx, x);
                }
            }
            red[h * kPrefillRows + r] = mx;
            tc::fence_before();
            __syncthreads();   // row maxima exchanged; the stage and the S columns are free
            if (tid == 0 && k + p.stages < ntiles) issue(seq + p.stages, k + p.stages);
            // lazy rescale: keep the reference max unless the tile's max exceeds it by
            // more than 2^8 (weights up to 256 are safe in fp16 and fp32)
            const float mt = fmaxf(red[r], red[kPrefillRows + r]);
            float corr = 1.f;
            const bool resc = mt > m_ref + 8.f;
            if (resc) {
                corr = ex2(m_ref - mt);
                m_ref = mt;
            }
            const float base = m_ref == -INFINITY ? 0.f : m_ref;
            float rs = 0.f;
            if (active) {
#pragma unroll
                for (int q8 = 0; q8 < 4; q8++) {
                    uint32_t hw[4];
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const float pa = ex2(sv[8 * q8 + 2 * i] - base), pb = ex2(sv[8 * q8 + 2 * i + 1] - base);
                        rs += pa + pb;
                        hw[i] = f16x2_of(pa, pb);
                    }
                    if (c0 + 8 * q8 < T)
                        *reinterpret_cast<uint4*>(sP + p_off(r, c0 + 8 * q8)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                }
            }
            l_part = l_part * corr + rs;
            if (k > 0 && __any_sync(0xffffffffu, resc)) {
                // O of this thread's row, columns [h D/2, h D/2 + D/2), times corr
#pragma unroll 1
                for (int cc = 0; cc < D / 2; cc += 32) {
                    uint32_t v[32];
                    const uint32_t ta = tO + lane_bits + h * (D / 2) + cc;
                    tc::ld32(ta, v);
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i++) v[i] = __float_as_uint(__uint_as_float(v[i]) * corr);
                    tc::st32(ta, v);
                }
                tc::wait_st();
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc::fence_before();
            __syncthreads();   // P and the value tile written, O rescaled
            if (tid == 0 && !*abort_flag) {
                tc::fence_after();
#pragma unroll
                for (int kk = 0; kk < kMaxT / 16; kk++)
                    if (kk < T / 16)
                        tc::mma_f16(tO, tc::sdesc(aP + kk * 2 * (kPrefillRows * 16), kPrefillRows * 16, 128),
                                    tc::sdesc(aV + 256 * kk, 128, 16 * T), idO, k > 0 || kk > 0);
                tc::commit(barO);
                n_o++;
            }
        }

        // ---- epilogue: normalise, stage the rows, rotate V back, store
        if (ntiles > 0) {
            wait_or_flag(barO, (rnd - 1) & 1u);
            tc::fence_after();
        }
        red[h * kPrefillRows + r] = l_part;
        __syncthreads();
        const float l = red[r] + red[kPrefillRows + r];
        const float inv = l > 0.f ? p.o_mult / l * pow2i(ev_seq) : 0.f;   // O is in units of 2^ev_seq
        float* so = sO + r * OST + h * (D / 2);
#pragma unroll 1
        for (int cc = 0; cc < D / 2; cc += 32) {
            uint32_t v[32];
            if (ntiles > 0) {
                tc::ld32(tO + lane_bits + h * (D / 2) + cc, v);
                tc::wait_ld();
            }
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(so + cc + i) =
                    ntiles > 0 ? make_float4(__uint_as_float(v[i]) * inv, __uint_as_float(v[i + 1]) * inv,
                                             __uint_as_float(v[i + 2]) * inv, __uint_as_float(v[i + 3]) * inv)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        tc::fence_before();
        __syncthreads();   // output rows staged; tensor memory reads done
        for (int rr = warp; rr < kPrefillRows; rr += kPrefillThreads / 32) {
            const int64_t grr = R0 + rr;
            if (grr >= rows_total) break;
            float x[EPL];
#pragma unroll
            for (int i = 0; i < EPL; i += 4) {
                const float4 v = *reinterpret_cast<const float4*>(sO + rr * OST + lane * EPL + i);
                x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
            }
            if constexpr (D == 256) {
                if (p.rot_v) fwht256_warp(x, lane);
            }
            const int64_t i_tok = grr / p.G, g = grr % p.G;
            const int64_t o = ((qrow0 + i_tok) * p.Hq + (int64_t)hh * p.G + g) * D + lane * EPL;
            if (p.out_fp32) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o);
#pragma unroll
                for (int i = 0; i < EPL / 4; i++) dst[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
            } else {
                uint32_t hb[EPL / 2];
#pragma unroll
                for (int i = 0; i < EPL / 2; i++) hb[i] = bf16x2_of(x[2 * i], x[2 * i + 1]);
                uint16_t* dst = static_cast<uint16_t*>(p.out) + o;
                if constexpr (EPL == 8) {
                    *reinterpret_cast<uint4*>(dst) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
                } else {
                    *reinterpret_cast<uint2*>(dst) = make_uint2(hb[0], hb[1]);
                }
            }
        }
        __syncthreads();   // the shared region is free for the next block
    }
    if (tid == 0 && *abort_flag) {
        // a wait gave up: before the tensor memory is freed and the CTA exits,
        // wait (with the default bound) for what was already handed out -- the
        // last copy into each ring stage, and the last S and O products (each
        // is issued only after the previous one of its kind was waited for)
        int ignore = 0;
        for (uint32_t j = n_issued > (uint32_t)p.stages ? n_issued - p.stages : 0; j < n_issued; j++)
            (void)mbar_wait(smem_addr(&bars[j % p.stages]), (j / p.stages) & 1u, &ignore);
        if (n_s) (void)mbar_wait(barS, (n_s - 1) & 1u, &ignore);
        if (n_o) (void)mbar_wait(barO, (n_o - 1) & 1u, &ignore);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(tmem, kCols);
}


// ------------------------------------------------------------ warp-specialised kernel
//
// Same computation, same tiles, same arithmetic per value, with the work split
// by role so that the tensor core, the softmax and the dequantisation overlap:
//  * warp 0 (one thread) issues the products.  Tile order S(0), S(1), PV(0),
//    S(2), PV(1), ...: S(k + 1) runs while the softmax of tile k does.
//  * warps 4..7 run the softmax, one query row per thread (its tensor-memory
//    lane): a thread loads its whole row of S, so no row maximum is exchanged.
//    O in tensor memory is rescaled (lazily, as above) by its row's thread,
//    after the previous P V is done and before the next is issued.
//  * warps 1..3 and 8..15 dequantise key and value tiles straight from the page slabs
//    in global memory (the next tile's codes are loaded while this tile's are
//    converted) into double-buffered fp16 operand tiles.
//  * all warps stage q and store the output between query blocks.
// Key, value, S and P buffers are double-buffered; the hand-offs go through
// mbarriers -- kfull/vfull (dequant -> MMA, 11 arrivals), kfree/sfull/pvdone
// (tcgen05.commit), sfree/pfull (softmax -> MMA, 4 arrivals) -- whose phase
// parities follow the CTA's running tile count g: buffer g & 1, phase
// (g >> 1) & 1.  Every wait is bounded; a wait that gives up sets the abort
// flag, after which every role leaves its loop.

constexpr int kWsThreads = 512;
constexpr int kDqWarps = 11;      // dequantising warps: 1..3 and 8..15
constexpr int kWsBars = 15;       // kfull[2] vfull[2] kfree[2] sfull[2] sfree[2] pfull[2] pvdone[2] drain

// 32 bytes from global memory (one 256-bit load; the address is 32-byte aligned)
__device__ __forceinline__ void ldg256(const void* src, uint4& lo, uint4& hi) {
    asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
                 : "l"(src));
}

// A dequantising thread's share of one key or value tile, read from the page
// slab in global memory.  A lane takes two adjacent 16-byte chunks of a row
// (one 32-byte load; the row's chunk permutation XORs chunk indices with an
// even value, or swaps the two of a pair for 16-bit codes, so a pair stays a
// pair) and their scale bits (one load: the pair shares its INT8, E4M3-row or
// MX group; E2M1's four scales are contiguous).  A warp's step covers RB rows
// x 2 LR chunks, lane l holding row l % RB and the pair l / RB: each 8-lane
// phase of its 16-byte shared-memory stores writes one chunk column of 8
// consecutive rows -- consecutive 16-byte slots of the operand tile, free of
// bank conflicts.  Rows at or past `valid` load as zero codes with zero
// scales, which dequantise to zeros.
template <int KIND, int D>
struct DqShare {
    static constexpr int CB = row_code_bytes(KIND, D), SB = row_scale_bytes(KIND, D);
    static constexpr int CPR = CB / 16;                     // chunks per row: 4 .. 32
    static constexpr int LR = CPR / 2 < 4 ? CPR / 2 : 4;    // lanes per row in a step
    static constexpr int RB = 32 / LR;                      // rows of a step: 8 or 16
    static constexpr int NW = kDqWarps;
    static constexpr int NPT = ((kMaxT / RB) * (CPR / (2 * LR)) + NW - 1) / NW;   // steps per warp at T = 64
    uint4 w[NPT][2];
    uint32_t sb[NPT];

    // lgR = log2(T / RB): the tile's row blocks
    __device__ __forceinline__ static void pair_of(int i, int lgR, int dw, int l, int& t, int& j, bool& in) {
        const int id = dw + i * NW;                    // step id
        in = id < ((CPR / (2 * LR)) << lgR);
        t = (id & ((1 << lgR) - 1)) * RB + (l % RB);
        j = (id >> lgR) * (2 * LR) + 2 * (l / RB);     // the pair's first chunk (even)
    }
    __device__ __forceinline__ void fetch(const uint8_t* codes, const uint8_t* scales, int r0, int lgR, int valid,
                                          int dw, int l) {
#pragma unroll
        for (int i = 0; i < NPT; i++) {
            int t, j;
            bool in;
            pair_of(i, lgR, dw, l, t, j, in);
            w[i][0] = w[i][1] = make_uint4(0, 0, 0, 0);
            sb[i] = 0;
            if (in && t < valid) {
                const int row = r0 + t;
                const int pj = j ^ row_swizzle(KIND, D, row);   // physical chunk of j; j + 1 at pj ^ 1
                uint4 lo, hi;
                ldg256(codes + (int64_t)row * CB + ((pj & ~1) << 4), lo, hi);
                w[i][0] = (pj & 1) ? hi : lo;
                w[i][1] = (pj & 1) ? lo : hi;
                if constexpr (SB > 0) {
                    const uint8_t* srow = scales + (int64_t)row * SB;
                    if constexpr (kind_bits(KIND) == 4) {
                        sb[i] = __ldg(reinterpret_cast<const uint32_t*>(srow + 2 * j));   // 2 chunks x 2 scales
                    } else if constexpr (kind_scale_bytes(KIND) == 2) {
                        sb[i] = __ldg(reinterpret_cast<const uint16_t*>(srow + 2 * (j * 16 / kind_group(KIND))));
                    } else {
                        sb[i] = __ldg(srow + j * 16 / kind_group(KIND));
                    }
                }
            }
        }
    }
    __device__ __forceinline__ void store(uint8_t* tile, int T, int lgR, int dw, int l, float smul) const {
#pragma unroll
        for (int i = 0; i < NPT; i++) {
            int t, j;
            bool in;
            pair_of(i, lgR, dw, l, t, j, in);
            if (in) {
                const uint32_t s1 = kind_bits(KIND) == 4 ? sb[i] >> 16 : sb[i];   // the second chunk's scale bits
                dequant_chunk<KIND, D>(w[i][0], sb[i] & (kind_bits(KIND) == 4 ? 0xFFFFu : 0xFFFFFFFFu), j, tile, t, T,
                                       smul);
                dequant_chunk<KIND, D>(w[i][1], s1, j + 1, tile, t, T, smul);
            }
        }
    }
};

template <int KK, int KV, int D>
__global__ void __launch_bounds__(kWsThreads, 1) prefill_ws_kernel(const PrefillParams p) {
    constexpr bool KBF = (KK == RK_BF16RAW);
    constexpr int EPL = D / 32;
    constexpr int OST = D + 4;
    constexpr uint32_t kCols = D == 256 ? 512 : 256;   // O in [0, D), S(b) in [D + 64 b, D + 64 b + 64)
    extern __shared__ __align__(1024) uint8_t smem[];
    const int T = p.T, lgT = 31 - __clz(T);
    uint8_t* sQ = smem;
    uint8_t* sK0 = sQ + kPrefillRows * D * 2;     // sK(b) = sK0 + b T D 2
    uint8_t* sV0 = sK0 + 2 * T * D * 2;
    uint8_t* sP0 = sV0 + 2 * T * D * 2;           // sP(b) = sP0 + b 128 T 2
    float* sO = reinterpret_cast<float*>(smem);   // epilogue staging, over the operand tiles
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + prefill_ws_region(D, T));
    float* qrm = reinterpret_cast<float*>(bars + kWsBars + 1);
    uint32_t* red = reinterpret_cast<uint32_t*>(qrm + kPrefillRows);   // [32]
    uint32_t* tslot = red + 32;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
    enum { KFULL = 0, VFULL = 2, KFREE = 4, SFULL = 6, SFREE = 8, PFULL = 10, PVDONE = 12, DRAIN = 14 };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int64_t idx = blockIdx.x;
    const int slot = (int)(idx % p.slots);
    idx /= p.slots;
    const int hh = (int)(idx % p.L.H);
    const int b = (int)(idx / p.L.H);
    const int64_t qrow0 = p.cu_q_lens[b];
    const int n = max(0, p.cu_q_lens[b + 1] - (int)qrow0);
    const int Ls = p.seq_lens[b];
    const int64_t rows_total = (int64_t)n * p.G;
    const int64_t nblk = (rows_total + kPrefillRows - 1) / kPrefillRows;
    if (slot >= nblk) return;

    auto bar = [&](int i) { return smem_addr(&bars[i]); };
    if (tid == 0) {
        for (int i = 0; i < kWsBars; i++)
            mbar_init(bar(i), i < KFREE ? (uint32_t)kDqWarps : (i >= SFREE && i < PVDONE) ? 4u : 1u);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tc::alloc(smem_addr(tslot), kCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t tO = tmem;
    auto tS = [&](uint32_t bb) { return tmem + D + 64 * bb; };
    auto sK = [&](uint32_t bb) { return sK0 + bb * T * D * 2; };
    auto sV = [&](uint32_t bb) { return sV0 + bb * T * D * 2; };
    auto sP = [&](uint32_t bb) { return sP0 + bb * kPrefillRows * T * 2; };
    // a bounded wait taken by every lane of the warp alike
    auto wait_warp = [&](int i, uint32_t phase) {
        bool ok = mbar_wait(bar(i), phase, abort_flag, p.wait_polls);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0) atomicOr(p.status, kStatusWaitTimeout);
        return ok;
    };

    auto block_tiles = [&](int64_t jb) {
        const int64_t R0 = (nblk - 1 - jb) * kPrefillRows;   // the heaviest block first
        const int64_t r_last = min(R0 + kPrefillRows, rows_total) - 1;
        const int pos_hi = Ls - n + (int)(r_last / p.G);
        return pos_hi >= 0 ? pos_hi / T + 1 : 0;
    };

    int ek_seq = 0, ev_seq = 0;
    if constexpr (scale_normalised(KK) || scale_normalised(KV))
        sequence_scale_exps<KK, KV, D, kWsThreads>(p, b, hh, Ls, red, &ek_seq, &ev_seq);
    const float kmul = pow2i(-ek_seq), vmul = pow2i(-ev_seq);

    // where key tile k of the sequence lives: the block-table entry of its page
    // (-1 past the table's width), then its page slab and first row there
    auto tile_pid = [&](int k) -> int {
        const int page = k * T / p.L.P;
        return page < p.max_pages ? p.block_table[(int64_t)b * p.max_pages + page] : -1;
    };
    auto tile_slab = [&](int pid, int k, int& r0) -> const uint8_t* {
        const int t0 = k * T;
        r0 = t0 % p.L.P;
        if (pid < 0 || pid >= p.L.num_pages) {
            if ((threadIdx.x & 31) == 0) atomicOr(p.status, kStatusBadPage);
            pid = 0;
        }
        return p.slabs + ((int64_t)pid * p.L.H + hh) * p.L.slab;
    };

    const uint32_t idS = tc::idesc_f16(KBF, false, T), idO = tc::idesc_f16(false, true, D);
    uint32_t gk = 0;      // key tiles of earlier query blocks (every role counts alike)
    float l_row = 0.f;    // softmax threads: the row's sum of weights
    for (int64_t jb = slot; jb < nblk; jb += p.slots) {
        const int64_t R0 = (nblk - 1 - jb) * kPrefillRows;
        const int ntiles = block_tiles(jb);
        stage_q<D, KBF, kWsThreads>(p, sQ, qrm, qrow0, hh, R0, rows_total, warp, lane);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();   // q staged

        if (warp == 0) {
            // ---- the products, issued by one thread
            if (lane == 0 && ntiles > 0) {
                const uint32_t aQ = smem_addr(sQ);
                auto wait1 = [&](int i, uint32_t phase) {
                    const bool ok = mbar_wait(bar(i), phase, abort_flag, p.wait_polls);
                    if (!ok) atomicOr(p.status, kStatusWaitTimeout);
                    return ok;
                };
                for (int k = 0; k <= ntiles; k++) {
                    if (k < ntiles) {
                        const uint32_t g = gk + k, bb = g & 1u, ph = (g >> 1) & 1u;
                        if (!wait1(KFULL + bb, ph)) break;
                        if (k >= 2 && !wait1(SFREE + bb, ph ^ 1u)) break;   // softmax of tile g - 2 done
                        tc::fence_after();
                        const uint32_t aK = smem_addr(sK(bb));
#pragma unroll
                        for (int kk = 0; kk < D / 16; kk++)
                            tc::mma_f16(tS(bb), tc::sdesc(aQ + 256 * kk, 128, 16 * D),
                                        tc::sdesc(aK + kk * 32 * T, 16 * T, 128), idS, kk > 0);
                        tc::commit(bar(SFULL + bb));
                        tc::commit(bar(KFREE + bb));
                    }
                    if (k >= 1) {
                        const uint32_t g = gk + k - 1, bb = g & 1u, ph = (g >> 1) & 1u;
                        if (!wait1(PFULL + bb, ph) || !wait1(VFULL + bb, ph)) break;
                        tc::fence_after();
                        const uint32_t aP = smem_addr(sP(bb)), aV = smem_addr(sV(bb));
#pragma unroll
                        for (int kk = 0; kk < kMaxT / 16; kk++)
                            if (kk < T / 16)
                                tc::mma_f16(tO, tc::sdesc(aP + kk * 2 * (kPrefillRows * 16), kPrefillRows * 16, 128),
                                            tc::sdesc(aV + 256 * kk, 128, 16 * T), idO, k > 1 || kk > 0);
                        tc::commit(bar(PVDONE + bb));
                    }
                }
            }
        } else if (warp >= 4 && warp < 8) {
            // ---- softmax: thread = row r, tensor-memory lane r
            const int g4 = warp & 3, r = g4 * 32 + lane;
            const uint32_t lane_bits = (uint32_t)(g4 * 32) << 16;
            const int64_t gr = R0 + r;
            const int pos = gr < rows_total ? Ls - n + (int)(gr / p.G) : -1;
            const int64_t gfirst = R0 + g4 * 32;
            const int gpos_min = gfirst + 31 < rows_total ? Ls - n + (int)(gfirst / p.G) : -1;
            // this row's score multiplier, kept positive (masked scores are -inf
            // and go through fma(s, qm, -base))
            const float qm = fmaxf(p.q_mult * pow2i(ek_seq) * qrm[r], 1.17549435e-38f);
            float m_ref = -INFINITY;
            l_row = 0.f;
            bool ok = true;
            for (int k = 0; k < ntiles && ok; k++) {
                const uint32_t g = gk + k, bb = g & 1u, ph = (g >> 1) & 1u;
                if (!(ok = wait_warp(SFULL + bb, ph))) break;
                tc::fence_after();
                uint32_t v[64];
                tc::ld32(tS(bb) + lane_bits, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                if (T > 32) {
                    tc::ld32(tS(bb) + lane_bits + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                } else {
#pragma unroll
                    for (int i = 32; i < 64; i++) v[i] = 0u;
                }
                tc::wait_ld();
                tc::fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(SFREE + bb));   // S(b) may be overwritten
                // raw scores: the row's multiplier qm > 0 goes into the exponent
                // (fma(s, qm, -base)), so the maximum is taken over the raw values
                const int t0 = k * T;
                if (t0 + T - 1 > gpos_min || T < 64) {   // keys past the tile or past a row's position
#pragma unroll
                    for (int i = 0; i < 64; i++)
                        if (i >= T || t0 + i > pos) v[i] = __float_as_uint(-INFINITY);
                }
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four chains for latency
#pragma unroll
                for (int i = 0; i < 64; i++) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(v[i]));
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * qm;
                float corr = 1.f;
                const bool resc = mx > m_ref + 8.f;
                if (resc) {
                    corr = ex2(m_ref - mx);
                    m_ref = mx;
                }
                const float base = m_ref == -INFINITY ? 0.f : m_ref;
                float rs4[4] = {0.f, 0.f, 0.f, 0.f};
                uint8_t* pt = sP(bb);
#pragma unroll
                for (int q8 = 0; q8 < 8; q8++) {
                    uint32_t hw[4];
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const float pa = ex2(fmaf(__uint_as_float(v[8 * q8 + 2 * i]), qm, -base));
                        const float pb = ex2(fmaf(__uint_as_float(v[8 * q8 + 2 * i + 1]), qm, -base));
                        rs4[i] += pa + pb;
                        hw[i] = f16x2_of(pa, pb);
                    }
                    if (8 * q8 < T) *reinterpret_cast<uint4*>(pt + p_off(r, 8 * q8)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                }
                l_row = l_row * corr + ((rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
                if (k > 0 && __any_sync(0xffffffffu, resc)) {
                    // O of this row times corr, once the previous P V has landed in it
                    const uint32_t gp = g - 1;
                    if (!(ok = wait_warp(PVDONE + (gp & 1u), (gp >> 1) & 1u))) break;
                    tc::fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < D; cc += 32) {
                        uint32_t o[32];
                        tc::ld32(tO + lane_bits + cc, o);
                        tc::wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
                        tc::st32(tO + lane_bits + cc, o);
                    }
                    tc::wait_st();
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                tc::fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(PFULL + bb));
            }
            if (ok && ntiles > 0) {   // the block's last P V
                const uint32_t gl = gk + ntiles - 1;
                if (wait_warp(PVDONE + (gl & 1u), (gl >> 1) & 1u)) tc::fence_after();
            }
        } else {
            // ---- dequantisation of key and value tiles, straight from the slabs
            const int dw = warp < 4 ? warp - 1 : warp - 5;   // dequantising warp 0..10
            DqShare<KK, D> rk;
            DqShare<KV, D> rv;
            // log2(T / RB) of each array's steps (T >= RB: tiles of 16 tokens or more)
            const int lgRk = lgT - (DqShare<KK, D>::RB == 16 ? 4 : 3), lgRv = lgT - (DqShare<KV, D>::RB == 16 ? 4 : 3);
            // tile k + 1's codes are loaded while tile k is converted, and tile
            // k + 2's block-table entry with them, so no load waits on another
            int r0 = 0;
            const uint8_t* slab = ntiles > 0 ? tile_slab(tile_pid(0), 0, r0) : p.slabs;
            int pid_next = ntiles > 1 ? tile_pid(1) : 0;
            int valid = min(T, Ls);
            if (ntiles > 0) {
                rk.fetch(slab, slab + p.L.off_ks, r0, lgRk, valid, dw, lane);
                rv.fetch(slab + p.L.off_vc, slab + p.L.off_vs, r0, lgRv, valid, dw, lane);
            }
            for (int k = 0; k < ntiles; k++) {
                const uint32_t g = gk + k, bb = g & 1u, ph = (g >> 1) & 1u;
                if (k >= 2 && !wait_warp(KFREE + bb, ph ^ 1u)) break;   // S of tile g - 2 done with sK(b)
                rk.store(sK(bb), T, lgRk, dw, lane, kmul);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(KFULL + bb));
                int r1 = 0;
                const uint8_t* slab1 = slab;
                if (k + 1 < ntiles) {
                    slab1 = tile_slab(pid_next, k + 1, r1);
                    valid = min(T, Ls - (k + 1) * T);
                    rk.fetch(slab1, slab1 + p.L.off_ks, r1, lgRk, valid, dw, lane);
                    pid_next = k + 2 < ntiles ? tile_pid(k + 2) : 0;
                }
                if (k >= 2 && !wait_warp(PVDONE + bb, ph ^ 1u)) break;   // P V of tile g - 2 done with sV(b)
                rv.store(sV(bb), T, lgRv, dw, lane, vmul);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(VFULL + bb));
                if (k + 1 < ntiles) rv.fetch(slab1 + p.L.off_vc, slab1 + p.L.off_vs, r1, lgRv, valid, dw, lane);
            }
        }
        gk += (uint32_t)ntiles;

        // ---- epilogue: normalise, stage the rows, rotate V back, store
        tc::fence_before();
        __syncthreads();   // every product of the block done; the operand tiles are free
        tc::fence_after();
        if (warp >= 4 && warp < 8) {
            const int g4 = warp & 3, r = g4 * 32 + lane;
            const uint32_t lane_bits = (uint32_t)(g4 * 32) << 16;
            const float inv = l_row > 0.f ? p.o_mult / l_row * pow2i(ev_seq) : 0.f;   // O is in units of 2^ev_seq
            float* so = sO + r * OST;
            const bool have = __all_sync(0xffffffffu, ntiles > 0 && !*abort_flag);
#pragma unroll 1
            for (int cc = 0; cc < D; cc += 32) {
                uint32_t v[32];
                if (have) {
                    tc::ld32(tO + lane_bits + cc, v);
                    tc::wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i++) v[i] = 0u;
                }
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4*>(so + cc + i) =
                        make_float4(__uint_as_float(v[i]) * inv, __uint_as_float(v[i + 1]) * inv,
                                    __uint_as_float(v[i + 2]) * inv, __uint_as_float(v[i + 3]) * inv);
            }
        }
        tc::fence_before();
        __syncthreads();   // output rows staged; tensor memory reads done
        for (int rr = warp; rr < kPrefillRows; rr += kWsThreads / 32) {
            const int64_t grr = R0 + rr;
            if (grr >= rows_total) break;
            float x[EPL];
#pragma unroll
            for (int i = 0; i < EPL; i += 4) {
                const float4 v = *reinterpret_cast<const float4*>(sO + rr * OST + lane * EPL + i);
                x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
            }
            if constexpr (D == 256) {
                if (p.rot_v) fwht256_warp(x, lane);
            }
            const int64_t i_tok = grr / p.G, gq = grr % p.G;
            const int64_t o = ((qrow0 + i_tok) * p.Hq + (int64_t)hh * p.G + gq) * D + lane * EPL;
            if (p.out_fp32) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o);
#pragma unroll
                for (int i = 0; i < EPL / 4; i++) dst[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
            } else {
                uint32_t hb[EPL / 2];
#pragma unroll
                for (int i = 0; i < EPL / 2; i++) hb[i] = bf16x2_of(x[2 * i], x[2 * i + 1]);
                uint16_t* dst = static_cast<uint16_t*>(p.out) + o;
                if constexpr (EPL == 8) {
                    *reinterpret_cast<uint4*>(dst) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
                } else {
                    *reinterpret_cast<uint2*>(dst) = make_uint2(hb[0], hb[1]);
                }
            }
        }
        __syncthreads();   // the shared region is free for the next block
    }
    // every product issued has completed before the tensor memory is freed
    // (on a normal exit they have; after a wait gave up, wait -- bounded -- here)
    if (tid == 0) {
        tc::commit(bar(DRAIN));
        int ignore = 0;
        (void)mbar_wait(bar(DRAIN), 0, &ignore);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(tmem, kCols);
}

}  // namespace

// ------------------------------------------------------------ host side

bool prefill_supported(int fmt, int D) {
    if (fmt == F_FP8_ROW256 || fmt == F_K8V4) return D == 256;
    return fmt >= 0 && fmt < F_COUNT && (D == 128 || D == 256);
}

static constexpr size_t kSmemLimit = 227 * 1024;   // opt-in shared memory per CTA on sm_100

cudaError_t plan_prefill(const Layout& L, PrefillPlan* plan) {
    int T = 64;
    while (L.P % T) T >>= 1;   // the largest of 64, 32, 16 that divides the page
    // the warp-specialised kernel, whenever its tiles fit and the slab's rows
    // and regions allow its 32-byte loads (true of every layout today)
    const bool a32 = L.kc % 32 == 0 && L.vc % 32 == 0 && L.off_ks % 32 == 0 && L.off_vc % 32 == 0 &&
                     L.off_vs % 32 == 0 && L.slab % 32 == 0;
    if (a32) {
        PrefillPlan q;
        memset(&q, 0, sizeof(q));
        q.T = T;
        q.kernel = 1;
        q.smem = (size_t)prefill_ws_smem(L.D, T);
        if (q.smem <= kSmemLimit) {
            *plan = q;
            return cudaSuccess;
        }
    }
    const int stages = 2;
    for (;;) {
        PrefillPlan q;
        memset(&q, 0, sizeof(q));
        q.T = T;
        q.kernel = 0;
        q.stages = stages;
        q.st_ks = (int)align16((int64_t)T * L.kc);
        q.st_vc = q.st_ks + (int)align16((int64_t)T * L.ks);
        q.st_vs = q.st_vc + (int)align16((int64_t)T * L.vc);
        q.st_bytes = q.st_vs + (int)align16((int64_t)T * L.vs);
        q.smem = (size_t)prefill_region0(L.D, T) + (size_t)stages * q.st_bytes + (size_t)prefill_tail_bytes(stages);
        if (q.smem <= kSmemLimit) {
            *plan = q;
            return cudaSuccess;
        }
        if (T == 16) return cudaErrorInvalidValue;
        T >>= 1;
    }
}

template <int KK, int KV, int D>
static cudaError_t launch_t(const PrefillParams& p, const PrefillPlan& plan, int64_t grid, cudaStream_t s) {
    auto kern = plan.kernel == 1 ? prefill_ws_kernel<KK, KV, D> : prefill_kernel<KK, KV, D>;
    const int threads = plan.kernel == 1 ? kWsThreads : kPrefillThreads;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)grid, threads, plan.smem, s>>>(p);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_d(const PrefillParams& p, const PrefillPlan& plan, int64_t grid, cudaStream_t s) {
    switch (p.L.fmt) {
    case F_BF16: return launch_t<RK_BF16RAW, RK_FP16, D>(p, plan, grid, s);
    case F_INT8_G64: return launch_t<RK_INT8_G64, RK_INT8_G64, D>(p, plan, grid, s);
    case F_NVFP4_G16: return launch_t<RK_E2M1_G16, RK_E2M1_G16, D>(p, plan, grid, s);
    case F_MXFP8_G32: return launch_t<RK_E4M3_MX32, RK_E4M3_MX32, D>(p, plan, grid, s);
    case F_FP8_TENSOR: return launch_t<RK_E4M3_TENSOR, RK_E4M3_TENSOR, D>(p, plan, grid, s);
    default: break;
    }
    if constexpr (D == 256) {
        if (p.L.fmt == F_FP8_ROW256) return launch_t<RK_E4M3_ROW256, RK_E4M3_ROW256, 256>(p, plan, grid, s);
        if (p.L.fmt == F_K8V4) return launch_t<RK_E4M3_ROW256, RK_E2M1_G16, 256>(p, plan, grid, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_prefill(const PrefillParams& p0, const PrefillPlan& plan, int64_t grid, cudaStream_t s) {
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
    PrefillParams p = p0;
    p.T = plan.T;
    p.stages = plan.stages;
    p.st_ks = plan.st_ks;
    p.st_vc = plan.st_vc;
    p.st_vs = plan.st_vs;
    p.st_bytes = plan.st_bytes;
    return p.L.D == 256 ? launch_d<256>(p, plan, grid, s) : launch_d<128>(p, plan, grid, s);
}

}  // namespace kvq
