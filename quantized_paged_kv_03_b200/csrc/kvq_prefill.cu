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
//    kv-head share every key tile.  8 warps, 16 rows each, the whole head_dim
//    per warp.  A (sequence, kv-head)'s heaviest block (its last rows, which
//    see the most keys) starts first.
//  * Unlike decode, every key feeds many query rows: 4 x head_dim FLOPs per
//    (row, key), a dense contraction for the tensor cores.  A key tile (64
//    tokens, or fewer when the page size asks) arrives by cp.async.bulk into a
//    two-stage ring; all threads then dequantise it once into fp16 tiles in
//    shared memory, scales folded in (BF16 keys stay bf16, the format's own
//    bits), and every warp reads its MMA operands from them with ldmatrix.
//  * S = Q K^T and O += P V with mma.sync m16n8k16 and fp32 accumulators in
//    registers; online softmax in the log2 domain; the causal mask is applied
//    only on tiles that cross a warp's first position, and tiles past a warp's
//    last position are skipped.
//  * Rotated K: q is rotated by the Hadamard-256 when staged (orthonormal, so
//    q.k is unchanged); rotated V: each output row is rotated back in the
//    epilogue (the matrix is symmetric and its own inverse).
//
// Precision: q and the key/value tiles are fp16 (bf16 for BF16 keys).  Codes
// of every format are exact in fp16; a dequantised value code x scale is exact
// for E2M1 x UE4M3, E4M3 per tensor (the tensor scale is applied in fp32) and
// MX E4M3 x 2^k in fp16's normal range, and rounded once (nearest-even,
// relative 2^-11) for INT8 and E4M3 row-256 with their fp16 scales.  Stored
// values beyond fp16's range (|x| > 65504) saturate; the decode kernel, which
// applies scales in fp32, has no such limit.
#include "kvq_prefill.h"

namespace kvq {
namespace {

constexpr long kPrefillWaitPolls = 1l << 22;
constexpr int kMaxT = 64;   // largest key tile (tokens)

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
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase, volatile int* abort) {
    for (long i = 0; i < kPrefillWaitPolls; i++) {
        if (mbar_try_wait(bar, phase)) return true;
        if (*abort) return false;
    }
    *abort = 1;
    return false;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

template <bool BF16>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (BF16) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
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
// 2^x for x <= 0 (softmax weights); -inf gives 0.
__device__ __forceinline__ float exp2_neg(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t splat16(uint32_t h) { return (h & 0xFFFFu) * 0x10001u; }

// ------------------------------------------------------------ tiles

// Row stride (16-bit elements) of q and of the key/value tiles in shared
// memory: 8 elements of padding put the 8 rows that one ldmatrix phase reads
// in 8 distinct 16-byte bank groups.
template <int D>
constexpr int kTileStride = D + 8;

// Dequantise one 16-byte code chunk (chunk j of a row, logical order) into
// 16-bit elements at `d` (8, 16 or 32 of them, by the code width), with the
// row's scales applied.
template <int KIND, int D>
__device__ __forceinline__ void dequant_chunk(const uint4 w, const uint8_t* srow, int j, uint16_t* d) {
    constexpr int SB = kind_scale_bytes(KIND);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    if constexpr (kind_bits(KIND) == 16) {
        *reinterpret_cast<uint4*>(d + j * 8) = w;           // bf16 keys / fp16 values: the stored bits
    } else if constexpr (kind_bits(KIND) == 4) {
        // 32 E2M1 codes (two groups of 16, UE4M3 scales): code x scale is exact in fp16
        const uint32_t sc = dec_e4m3x2_f16x2((uint32_t)srow[2 * j] | ((uint32_t)srow[2 * j + 1] << 8));
        const uint32_t s0 = splat16(sc), s1 = splat16(sc >> 16);
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 16; i++) h[i] = mul_f16x2(dec_e2m1x2_f16x2((ws[i >> 2] >> (8 * (i & 3))) & 0xFFu),
                                                      i < 8 ? s0 : s1);
        uint4* o = reinterpret_cast<uint4*>(d + j * 32);
#pragma unroll
        for (int i = 0; i < 4; i++) o[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
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
            const int g = j * 16 / kind_group(KIND);
            const uint32_t sc = splat16((uint32_t)srow[SB * g] | ((uint32_t)srow[SB * g + 1] << 8));
#pragma unroll
            for (int i = 0; i < 8; i++) h[i] = mul_f16x2(h[i], sc);
        } else if constexpr (KIND == RK_E4M3_MX32) {
            // UE8M0 scale 2^(e-127): applied in fp32 (exact), then to fp16
            const float sc = ue8m0_to_f32(srow[j * 16 / 32]);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float2 f = f16x2_to_f32(h[i]);
                h[i] = enc_f16x2_sat(f.x * sc, f.y * sc);
            }
        }
        uint4* o = reinterpret_cast<uint4*>(d + j * 16);
        o[0] = make_uint4(h[0], h[1], h[2], h[3]);
        o[1] = make_uint4(h[4], h[5], h[6], h[7]);
    }
}

// Dequantise rows [0, T) of one array of a stage (codes: row stride
// row_code_bytes, chunk-permuted as stored; scales: plain rows) into a tile.
// Rows at or past `valid` lie beyond the sequence's last token and hold no
// data: they are written as zeros, so that a masked key's weight 0 never meets
// a non-finite value.
template <int KIND, int D>
__device__ __forceinline__ void dequant_tile(const uint8_t* codes, const uint8_t* scales, uint16_t* tile, int T,
                                             int valid, int tid) {
    constexpr int CB = row_code_bytes(KIND, D), SB = row_scale_bytes(KIND, D);
    constexpr int CPR = CB / 16;                       // chunks per row (a power of two)
    constexpr int EPC = 128 / kind_bits(KIND);         // elements per chunk
    for (int c = tid; c < T * CPR; c += kPrefillThreads) {
        const int t = c / CPR, j = c % CPR;
        uint16_t* d = tile + t * kTileStride<D>;
        if (t >= valid) {
            uint4* o = reinterpret_cast<uint4*>(d + j * EPC);
#pragma unroll
            for (int i = 0; i < EPC / 8; i++) o[i] = make_uint4(0, 0, 0, 0);
            continue;
        }
        const uint4 w = *reinterpret_cast<const uint4*>(codes + t * CB + ((j ^ row_swizzle(KIND, D, t)) << 4));
        dequant_chunk<KIND, D>(w, scales + t * SB, j, d);
    }
}

// Stage the block's 128 query rows into sQ: row r is global row R0 + r of the
// (sequence, kv-head), i.e. query token (R0 + r) / G, head (R0 + r) % G.  fp16
// (rotated by the Hadamard-256 first when K is rotated), or the bf16 bits
// themselves for BF16 keys; rows past the chunk are zeros.  One warp per row.
template <int D, bool QBF16>
__device__ __forceinline__ void stage_q(const PrefillParams& p, uint16_t* sQ, int64_t qrow0, int hh, int64_t R0,
                                        int64_t rows_total, int warp, int lane) {
    constexpr int EPL = D / 32;
    for (int r = warp; r < kPrefillRows; r += kPrefillThreads / 32) {
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
#pragma unroll
            for (int i = 0; i < EPL / 2; i++) h[i] = enc_f16x2_sat(x[2 * i], x[2 * i + 1]);
        }
        uint16_t* d = sQ + r * kTileStride<D> + lane * EPL;
        if constexpr (EPL == 8) {
            *reinterpret_cast<uint4*>(d) = make_uint4(h[0], h[1], h[2], h[3]);
        } else {
            *reinterpret_cast<uint2*>(d) = make_uint2(h[0], h[1]);
        }
    }
}

// ------------------------------------------------------------ kernel

template <int KK, int KV, int D>
__global__ void __launch_bounds__(kPrefillThreads, 1) prefill_kernel(const PrefillParams p) {
    constexpr bool KBF = (KK == RK_BF16RAW);   // bf16 keys: S on the bf16 MMA
    constexpr int TS = kTileStride<D>;
    constexpr int NO = D / 8;                  // output n-tiles (8 dims each)
    constexpr int NS = kMaxT / 8;              // score n-tiles of the largest key tile
    constexpr int EPL = D / 32;                // output values per lane in the epilogue
    constexpr int OST = D + 4;                 // fp32 row stride of the output staging
    extern __shared__ __align__(128) uint8_t smem[];
    const int T = p.T, nts = T / 8;
    uint16_t* sQ = reinterpret_cast<uint16_t*>(smem);
    uint16_t* sK = sQ + kPrefillRows * TS;
    uint16_t* sV = sK + T * TS;
    float* sO = reinterpret_cast<float*>(smem);
    uint8_t* ring = smem + prefill_region0(D, T);
    uint64_t* bars = reinterpret_cast<uint64_t*>(ring + (size_t)p.stages * p.st_bytes);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + p.stages);

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

    if (tid == 0) {
        for (int s = 0; s < p.stages; s++) mbar_init(smem_addr(&bars[s]), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // key tile k of this sequence into stage s: the whole page slab in one copy
    // when the tile is the page, else the tile's rows of the slab's four arrays
    auto issue = [&](uint32_t seq, int k) {
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

    // ldmatrix lane addresses: q rows (A operand), key rows (B of S), value
    // rows (B of O, transposed on load)
    const uint32_t qa_addr = smem_addr(sQ + (warp * 16 + (lane & 15)) * TS + (lane >> 4) * 8);
    const uint32_t kb_addr = smem_addr(sK + (lane & 7) * TS + (lane >> 3) * 8);
    const uint32_t vb_addr = smem_addr(sV + ((lane & 7) + ((lane >> 3) & 1) * 8) * TS + (lane >> 4) * 8);

    uint32_t seq = 0;   // key tiles consumed by this CTA: stage = seq % stages, phase = seq / stages
    for (int64_t jb = slot; jb < nblk; jb += p.slots) {
        const int64_t R0 = (nblk - 1 - jb) * kPrefillRows;   // the heaviest block first
        const int64_t r_last = min(R0 + kPrefillRows, rows_total) - 1;
        const int pos_hi = Ls - n + (int)(r_last / p.G);        // largest position in the block
        const int ntiles = pos_hi >= 0 ? pos_hi / T + 1 : 0;
        if (tid == 0)
            for (int k = 0; k < p.stages && k < ntiles; k++) issue(seq + k, k);
        stage_q<D, KBF>(p, sQ, qrow0, hh, R0, rows_total, warp, lane);

        // this thread's two rows (lane/4 and lane/4 + 8 of the warp's 16) and the
        // warp's position range; rows past the chunk get position -1 (no keys)
        const int64_t ra = R0 + warp * 16 + (lane >> 2), rb = ra + 8;
        const int pos_a = ra < rows_total ? Ls - n + (int)(ra / p.G) : -1;
        const int pos_b = rb < rows_total ? Ls - n + (int)(rb / p.G) : -1;
        const int64_t w0 = R0 + warp * 16;
        const int wpos_min = w0 + 15 < rows_total ? Ls - n + (int)(w0 / p.G) : -1;
        const int wpos_max = w0 < rows_total ? Ls - n + (int)((min(w0 + 15, rows_total - 1)) / p.G) : -1;

        float O[NO][4];
#pragma unroll
        for (int i = 0; i < NO; i++) O[i][0] = O[i][1] = O[i][2] = O[i][3] = 0.f;
        float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
        __syncthreads();   // q staged

        for (int k = 0; k < ntiles; k++, seq++) {
            const int s = (int)(seq % (uint32_t)p.stages);
            const uint8_t* st = ring + (size_t)s * p.st_bytes;
            if (!mbar_wait(smem_addr(&bars[s]), (seq / (uint32_t)p.stages) & 1u, abort_flag) && lane == 0)
                atomicOr(p.status, kStatusWaitTimeout);
            const int t0 = k * T;
            const int valid = min(T, Ls - t0);
            dequant_tile<KK, D>(st, st + p.st_ks, sK, T, valid, tid);
            dequant_tile<KV, D>(st + p.st_vc, st + p.st_vs, sV, T, valid, tid);
            __syncthreads();   // tiles ready; the stage is free again
            if (tid == 0 && k + p.stages < ntiles) issue(seq + p.stages, k + p.stages);

            if (t0 <= wpos_max) {
                // ---- S = Q K^T: 16 rows x T keys, head_dim in steps of 32
                float S[NS][4];
#pragma unroll
                for (int i = 0; i < NS; i++) S[i][0] = S[i][1] = S[i][2] = S[i][3] = 0.f;
#pragma unroll
                for (int kp = 0; kp < D / 32; kp++) {
                    uint32_t qa0[4], qa1[4];
                    ldsm_x4(qa0, qa_addr + kp * 64);
                    ldsm_x4(qa1, qa_addr + kp * 64 + 32);
#pragma unroll
                    for (int nt = 0; nt < NS; nt++) {
                        if (nt < nts) {
                            uint32_t kb[4];
                            ldsm_x4(kb, kb_addr + nt * 8 * TS * 2 + kp * 64);
                            mma16816<KBF>(S[nt], qa0, kb[0], kb[1]);
                            mma16816<KBF>(S[nt], qa1, kb[2], kb[3]);
                        }
                    }
                }
                // ---- online softmax (log2 domain), causal mask where the tile
                // crosses a row's position
                const bool mask = t0 + T - 1 > wpos_min;
                float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < NS; nt++) {
                    if (nt < nts) {
                        const int key = t0 + nt * 8 + (lane & 3) * 2;
                        float s0 = S[nt][0] * p.q_mult, s1 = S[nt][1] * p.q_mult;
                        float s2 = S[nt][2] * p.q_mult, s3 = S[nt][3] * p.q_mult;
                        if (mask) {
                            if (key > pos_a) s0 = -INFINITY;
                            if (key + 1 > pos_a) s1 = -INFINITY;
                            if (key > pos_b) s2 = -INFINITY;
                            if (key + 1 > pos_b) s3 = -INFINITY;
                        }
                        S[nt][0] = s0; S[nt][1] = s1; S[nt][2] = s2; S[nt][3] = s3;
                        mx_a = fmaxf(mx_a, fmaxf(s0, s1));
                        mx_b = fmaxf(mx_b, fmaxf(s2, s3));
                    }
                }
                mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
                mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
                mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
                mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
                const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
                const float base_a = mn_a == -INFINITY ? 0.f : mn_a;
                const float base_b = mn_b == -INFINITY ? 0.f : mn_b;
                const float corr_a = exp2_neg(m_a - base_a), corr_b = exp2_neg(m_b - base_b);
                m_a = mn_a;
                m_b = mn_b;
                float rs_a = 0.f, rs_b = 0.f;
                uint32_t pa[NS / 2][4];
#pragma unroll
                for (int kt = 0; kt < NS / 2; kt++) {
                    if (2 * kt < nts) {
                        const float p00 = exp2_neg(S[2 * kt][0] - base_a), p01 = exp2_neg(S[2 * kt][1] - base_a);
                        const float p02 = exp2_neg(S[2 * kt][2] - base_b), p03 = exp2_neg(S[2 * kt][3] - base_b);
                        const float p10 = exp2_neg(S[2 * kt + 1][0] - base_a), p11 = exp2_neg(S[2 * kt + 1][1] - base_a);
                        const float p12 = exp2_neg(S[2 * kt + 1][2] - base_b), p13 = exp2_neg(S[2 * kt + 1][3] - base_b);
                        rs_a += (p00 + p01) + (p10 + p11);
                        rs_b += (p02 + p03) + (p12 + p13);
                        pa[kt][0] = f16x2_of(p00, p01);
                        pa[kt][1] = f16x2_of(p02, p03);
                        pa[kt][2] = f16x2_of(p10, p11);
                        pa[kt][3] = f16x2_of(p12, p13);
                    }
                }
                l_a = l_a * corr_a + rs_a;
                l_b = l_b * corr_b + rs_b;
                if (__any_sync(0xffffffffu, corr_a != 1.f || corr_b != 1.f)) {
#pragma unroll
                    for (int i = 0; i < NO; i++) {
                        O[i][0] *= corr_a; O[i][1] *= corr_a;
                        O[i][2] *= corr_b; O[i][3] *= corr_b;
                    }
                }
                // ---- O += P V: 16 keys per k-step, 16 output dims per load
#pragma unroll
                for (int kt = 0; kt < NS / 2; kt++) {
                    if (2 * kt < nts) {
#pragma unroll
                        for (int dp = 0; dp < D / 16; dp++) {
                            uint32_t vb[4];
                            ldsm_x4_t(vb, vb_addr + (kt * 16 * TS + dp * 16) * 2);
                            mma16816<false>(O[2 * dp], pa[kt], vb[0], vb[1]);
                            mma16816<false>(O[2 * dp + 1], pa[kt], vb[2], vb[3]);
                        }
                    }
                }
            }
            __syncthreads();   // tiles consumed
        }

        // ---- epilogue: normalise, stage the warp's rows, rotate V back, store
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
        const float inv_a = l_a > 0.f ? p.o_mult / l_a : 0.f;
        const float inv_b = l_b > 0.f ? p.o_mult / l_b : 0.f;
        float* so = sO + warp * 16 * OST;
#pragma unroll
        for (int i = 0; i < NO; i++) {
            const int col = i * 8 + (lane & 3) * 2;
            *reinterpret_cast<float2*>(so + (lane >> 2) * OST + col) = make_float2(O[i][0] * inv_a, O[i][1] * inv_a);
            *reinterpret_cast<float2*>(so + ((lane >> 2) + 8) * OST + col) =
                make_float2(O[i][2] * inv_b, O[i][3] * inv_b);
        }
        __syncwarp();
        for (int r = 0; r < 16; r++) {
            const int64_t gr = w0 + r;
            if (gr >= rows_total) break;
            float x[EPL];
#pragma unroll
            for (int i = 0; i < EPL; i += 4) {
                const float4 v = *reinterpret_cast<const float4*>(so + r * OST + lane * EPL + i);
                x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
            }
            if constexpr (D == 256) {
                if (p.rot_v) fwht256_warp(x, lane);
            }
            const int64_t i_tok = gr / p.G, g = gr % p.G;
            const int64_t o = ((qrow0 + i_tok) * p.Hq + (int64_t)hh * p.G + g) * D + lane * EPL;
            if (p.out_fp32) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o);
#pragma unroll
                for (int i = 0; i < EPL / 4; i++) dst[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
            } else {
                uint32_t h[EPL / 2];
#pragma unroll
                for (int i = 0; i < EPL / 2; i++) h[i] = bf16x2_of(x[2 * i], x[2 * i + 1]);
                uint16_t* dst = static_cast<uint16_t*>(p.out) + o;
                if constexpr (EPL == 8) {
                    *reinterpret_cast<uint4*>(dst) = make_uint4(h[0], h[1], h[2], h[3]);
                } else {
                    *reinterpret_cast<uint2*>(dst) = make_uint2(h[0], h[1]);
                }
            }
        }
        __syncthreads();   // the shared region is free for the next block
    }
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
    const int stages = 2;
    for (;;) {
        PrefillPlan q;
        q.T = T;
        q.stages = stages;
        q.st_ks = (int)align16((int64_t)T * L.kc);
        q.st_vc = q.st_ks + (int)align16((int64_t)T * L.ks);
        q.st_vs = q.st_vc + (int)align16((int64_t)T * L.vc);
        q.st_bytes = q.st_vs + (int)align16((int64_t)T * L.vs);
        q.smem = (size_t)prefill_region0(L.D, T) + (size_t)stages * q.st_bytes + 8 * stages + 16;
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
    auto kern = prefill_kernel<KK, KV, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)grid, kPrefillThreads, plan.smem, s>>>(p);
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
