// kvq_decode.cu -- split-K paged GQA decode attention over the quantized cache.
//
// What it computes (one query token per sequence, query head h reading kv-head
// h / G): out = softmax(scale * q K^T) V over the sequence's tokens, with K and
// V taken from the cache as code x scale.  "NInfer KV Cache 量化指南" (why quantise:
// every decoded token re-reads the whole KV, so stored bytes set decode speed)
// and "FP8 KV Cache如何提速 ... 长上下文推理" (the bottleneck is memory bandwidth,
// not arithmetic) make this a streaming kernel: its roofline is HBM bandwidth.
//
// Design (B200, sm_100a):
//  * Persistent grid of two 8-warp CTAs per SM.  The work units of the whole
//    batch -- a page of one kv-head, or a 64-token span of a larger page --
//    ordered (sequence, kv-head, 8-head block, unit), are cut into gridDim.x
//    contiguous ranges of equal cost, where a unit costs 1 and every segment a
//    range touches adds the fixed price of its start, end and merge; ragged
//    batches balance to within about one unit.
//  * A whole-page unit (K codes, K scales, V codes, V scales of one kv-head:
//    one contiguous range in HBM) arrives with ONE cp.async.bulk into a
//    shared-memory stage; a span of a larger page with one copy per part.
//    Completion is tracked by an mbarrier.  Warps release a stage with a
//    shared counter; the last warp to release it issues the next copy into it,
//    so warps never wait for each other unit by unit.
//  * A warp owns a 16-token tile over all of head_dim.  Codes become fp16
//    (exact for every format) in registers straight from shared memory and
//    feed mma.sync m16n8k16 with the GQA group (<= 8 query heads) as N:
//    S^T = K q^T (tokens as M), then O^T += V^T P^T (head_dim as M; movmatrix
//    transposes the V and P fragments).  Group scales are folded into fp32
//    scores (K) or into P (V, against a power-of-two reference); NVFP4 scales
//    go into the operand, where code x scale is exact in fp16.
//  * Online softmax in the log2 domain; the warps merge in shared memory at
//    the end of each (sequence, kv-head) segment.  A segment cut by a range
//    boundary leaves a partial (max, sum, unnormalised output), merged by
//    whichever CTA counts in last (in groups of kFewParts parts, then the
//    groups), so no CTA ever waits on another.
//  * Rotated K: q is rotated by the same normalised Hadamard-256 (orthonormal,
//    so q.k is unchanged).  Rotated V: the output is rotated back (the matrix
//    is symmetric and its own inverse).
#include <type_traits>

#include "kvq_quant.cuh"

namespace kvq {

constexpr int kDecThreads = 256;   // 8 warps, each a 16-token tile over all of head_dim
// Row stride (floats) of the output-combine buffer: 4 floats of padding per head
// row spread the heads a warp writes over different banks.
template <int D>
constexpr int kOsmStride = D + 4;
constexpr int kMaxStages = 8;
// A segment's fused append is quantised at the segment start when the range
// holds at most this many of its units (its last unit then comes within about
// the ring's first fill), else when its last unit's data have arrived.  Only
// for INT8-G64 (fused_early): there it shortened the step by 6 %, while on the
// other formats the extra path cost the unit loop 1-2 % whether it ran or not.
constexpr int kFusedEarly = 16;
__host__ __device__ constexpr bool fused_early(int kk, int kv) { return kk == RK_INT8_G64 && kv == RK_INT8_G64; }
constexpr int kMaxBatch = 4096;
// Parts of a cut segment merged together by the CTA that completes them: a
// segment of more parts is merged in groups of this many, then the groups.
constexpr int kFewParts = 16;
constexpr long kWaitPolls = 1l << 22;

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

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
// Bounded wait for a stage.  Gives up after `polls` polls, or at once when
// another warp has already given up (`abort` set), so a failed copy never hangs
// the CTA: every warp then runs through its remaining work without waiting.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase, volatile int* abort, long polls = kWaitPolls) {
    for (long i = 0; i < polls; i++) {
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

__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
    uint32_t r;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t f16_splat(uint32_t h16) { return (h16 & 0xFFFFu) * 0x10001u; }
// 2^x for x <= 0 (softmax weights): one MUFU instruction; results below 2^-126 flush to 0.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Eight E2M1 codes (one word, element 2i in the low nibble of byte i) -> four
// f16x2, byte i giving (element 2i, element 2i+1).  Exact.
__device__ __forceinline__ void dec_e2m1x8(uint32_t w, uint32_t (&o)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
        : "r"(w));
}
// Four E4M3 codes (one word) -> two f16x2: (e0, e1), (e2, e3).  Exact.
__device__ __forceinline__ void dec_e4m3x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 h0, h1;\n\tmov.b32 {h0, h1}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, h0;\n\tcvt.rn.f16x2.e4m3x2 %1, h1;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

template <int NB>
struct Bytes { uint32_t w[NB / 4]; };   // NB bytes of one row, as words

// Load NB (8/16/32) bytes of a code row at byte offset `off` from `base`
// (base 32-byte aligned, off 8- or 16-byte aligned).  A 32-byte slice is two
// 16-byte chunks c, c+1 with c even; the row permutation of 16-bit rows flips
// bit 0 of the chunk index, so the second chunk sits at off ^ 16.
template <int NB>
__device__ __forceinline__ Bytes<NB> lds_bytes(const uint8_t* base, uint32_t off) {
    Bytes<NB> b;
    if constexpr (NB == 8) {
        uint2 v = *reinterpret_cast<const uint2*>(base + off);
        b.w[0] = v.x; b.w[1] = v.y;
    } else if constexpr (NB == 16) {
        uint4 v = *reinterpret_cast<const uint4*>(base + off);
        b.w[0] = v.x; b.w[1] = v.y; b.w[2] = v.z; b.w[3] = v.w;
    } else {
        uint4 v0 = *reinterpret_cast<const uint4*>(base + off);
        uint4 v1 = *reinterpret_cast<const uint4*>(base + (off ^ 16u));
        b.w[0] = v0.x; b.w[1] = v0.y; b.w[2] = v0.z; b.w[3] = v0.w;
        b.w[4] = v1.x; b.w[5] = v1.y; b.w[6] = v1.z; b.w[7] = v1.w;
    }
    return b;
}

// All codes of a lane's slice of one row -> f16x2 pairs: x[2*step] = elements
// (4 step, 4 step + 1), x[2*step + 1] = (4 step + 2, 4 step + 3).  No scale.
template <int KIND, int NB, int STEPS>
__device__ __forceinline__ void slice_f16(const Bytes<NB>& b, uint32_t (&x)[2 * STEPS]) {
    if constexpr (kind_bits(KIND) == 16) {
#pragma unroll
        for (int i = 0; i < 2 * STEPS; i++) x[i] = b.w[i];
    } else if constexpr (kind_bits(KIND) == 4) {
#pragma unroll
        for (int i = 0; i < STEPS / 2; i++) {
            uint32_t o[4];
            dec_e2m1x8(b.w[i], o);
            x[4 * i] = o[0]; x[4 * i + 1] = o[1]; x[4 * i + 2] = o[2]; x[4 * i + 3] = o[3];
        }
    } else if constexpr (KIND == RK_INT8_G64) {
#pragma unroll
        for (int i = 0; i < STEPS; i++) dec_int8x4_f16x2(b.w[i], x[2 * i], x[2 * i + 1]);
    } else {
#pragma unroll
        for (int i = 0; i < STEPS; i++) dec_e4m3x4(b.w[i], x[2 * i], x[2 * i + 1]);
    }
}

template <int KK, int KV, int D>
struct DecTraits {
    static constexpr int KBITS = kind_bits(KK), VBITS = kind_bits(KV);
    static constexpr int KCH = (KK == RK_E4M3_MX32) ? 2 : 4;   // k-steps per K load
    static constexpr int VCH = (KV == RK_E4M3_MX32) ? 2 : 4;   // d-tiles per V load
    static constexpr int KSTEPS = D / 16, DTILES = D / 16;
    static constexpr int KCW = 16 * KCH, VCW = 16 * VCH;       // chunk widths in head_dim
    static constexpr int KNB = 4 * KCH * KBITS / 8;            // bytes per lane per K row load
    static constexpr int VNB = 4 * VCH * VBITS / 8;
    static constexpr int KCHUNKS = KSTEPS / KCH, VCHUNKS = DTILES / VCH;
    static constexpr int QS = (KK == RK_BF16RAW) ? 2 : 1;      // q split into hi (+ lo)
    static constexpr int KC = row_code_bytes(KK, D), KS = row_scale_bytes(KK, D);   // row bytes
    static constexpr int VC = row_code_bytes(KV, D), VS = row_scale_bytes(KV, D);
    static constexpr int EPL = D / 32;
};

// Cursor over this CTA's page-heads: (sequence b, head pair hh = h*HB + hb, page).
struct Cursor {
    int b, hh, h, hb, span, nspans;   // hh = h * HB + hb; span = 64-token unit (or page)
};

__device__ __forceinline__ void cursor_next(Cursor& c, const int* pref, int B, int HH, int HB) {
    if (++c.span < c.nspans) return;
    c.span = 0;
    if (++c.hh < HH) {
        if (++c.hb == HB) {
            c.hb = 0;
            c.h++;
        }
        return;
    }
    c.hh = c.h = c.hb = 0;
    do {
        c.b++;
    } while (c.b < B && pref[c.b + 1] == pref[c.b]);
    c.nspans = (c.b < B) ? pref[c.b + 1] - pref[c.b] : 0;
}

__device__ __forceinline__ void cursor_locate(Cursor& c, int64_t w, const int* pref, int B, int HH, int HB) {
    int lo = 0, hi = B - 1;   // largest b with pref[b]*HH <= w
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((int64_t)pref[mid] * HH <= w) lo = mid;
        else hi = mid - 1;
    }
    while (lo < B - 1 && pref[lo + 1] == pref[lo]) lo++;   // skip empty sequences
    c.b = lo;
    c.nspans = pref[lo + 1] - pref[lo];
    int64_t idx = w - (int64_t)pref[lo] * HH;
    c.hh = (int)(idx / c.nspans);
    c.span = (int)(idx % c.nspans);
    c.h = c.hh / HB;
    c.hb = c.hh % HB;
}

// How the units are cut between the G CTAs: into ranges of equal cost, where
// a unit costs 1 and every segment (sequence, kv-head, head block) adds `c` at
// its start -- the fixed work of starting and finishing a segment, so that CTAs
// whose range touches many short segments get fewer units.  Cost positions:
// sequence b starts at pref[b] * HH + c * HH * b (empty sequences keep their
// segment costs; they only shift positions), segment hh of b occupies
// c + n_b positions, its unit u sits at position c + u of them.
struct Partition {
    const int* pref;
    int B, HH, c, G;
    int64_t W, C;   // units, total cost

    __device__ int64_t seq_cost(int b) const { return (int64_t)pref[b] * HH + (int64_t)c * HH * b; }
    // first unit at or after cost position X
    __device__ int64_t unit_at(int64_t X) const {
        if (X >= C) return W;
        int lo = 0, hi = B - 1;   // largest b with seq_cost(b) <= X
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (seq_cost(mid) <= X) lo = mid;
            else hi = mid - 1;
        }
        const int nb = pref[lo + 1] - pref[lo];
        const int64_t local = X - seq_cost(lo), len = (int64_t)nb + c;
        const int64_t hh = local / len, r = local - hh * len;
        return (int64_t)pref[lo] * HH + hh * nb + (r > c ? r - c : 0);
    }
    __device__ int64_t start(int i) const { return unit_at((int64_t)i * C / G); }
    // CTA whose range holds unit w = (b, hh, u)
    __device__ int owner(int b, int hh, int u) const {
        const int64_t x = seq_cost(b) + (int64_t)hh * (pref[b + 1] - pref[b] + c) + c + u;
        return (int)(((x + 1) * G + C - 1) / C) - 1;
    }
};

// The Hadamard-256 of one row held 8 values per lane, out of line: the segment
// start (rotating q) and the segment end (rotating the output back) share one
// copy of the code, which keeps those rarely run paths short to fetch.
struct Row8 {
    float v[8];
};
__device__ __noinline__ Row8 fwht256_row(Row8 x, int lane) {
    fwht256_warp(x.v, lane);
    return x;
}

// Store EPL consecutive output values (fp32 or bf16) at element offset `ob`.
template <int EPL>
__device__ __forceinline__ void store_out(void* out, int out_fp32, int64_t ob, const float* x) {
    if (out_fp32) {
        float* dst = reinterpret_cast<float*>(out) + ob;
#pragma unroll
        for (int e = 0; e < EPL; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
    } else {
        uint16_t* dst = reinterpret_cast<uint16_t*>(out) + ob;
#pragma unroll
        for (int e = 0; e < EPL; e += 4)
            *reinterpret_cast<uint2*>(dst + e) = make_uint2(pack_bf16(x[e], x[e + 1]), pack_bf16(x[e + 2], x[e + 3]));
    }
}


// Merge P parts of one cut segment -- part k's (max[8], sum[8], unnormalised
// output [8][D]) at part_ptr(k) -- in the order k = 0, 1, ... (so the result
// does not depend on which CTA merges, or when).  One pass: each output float4
// (head g, d4) is folded by tpo threads, each taking every tpo-th part with a
// running (max, sum, output) -- the log-sum-exp merge, loads of kMergeBatch
// parts in flight together -- and the threads' folds are combined by
// shuffles.  The result goes to the output rows (normalised), or, when `dst`
// is given, to dst as one more part (unnormalised, with its max and sum).
constexpr int kMergeBatch = 8;   // parts whose loads are in flight together

// Part k lies at first (k = 0), last (k = P - 1), else base + k * stride
// floats.  Out of line: it runs once or twice per CTA, after the main loop.
template <int D>
__device__ __noinline__ void merge_parts(const float* first, const float* last, const float* base, int64_t stride,
                                         int P, float* dst, void* out, int out_fp32, float o_mult, int Hq, int Gq,
                                         int b, int h, int hb) {
    const int tid = threadIdx.x;
    auto part_ptr = [&](int k) { return k == 0 ? first : k == P - 1 ? last : base + k * stride; };
    const int gv = min(8, Gq - hb * 8);
    const int no = gv * (D / 4);   // float4 outputs
    int tpo = 1;                   // threads per output, splitting the parts
    while (tpo < 32 && tpo * 2 * no <= kDecThreads) tpo *= 2;
    const int per_pass = kDecThreads / tpo;
    for (int ob = 0; ob < no; ob += per_pass) {
        const int o = ob + tid / tpo, pl = tid % tpo;
        const bool valid = o < no;
        const int g = valid ? o / (D / 4) : 0, d4 = valid ? o % (D / 4) : 0;
        float M = -INFINITY, L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) {
            for (int k0 = pl; k0 < P; k0 += kMergeBatch * tpo) {
                float mk[kMergeBatch], lk[kMergeBatch];
                float4 v[kMergeBatch];
#pragma unroll
                for (int q = 0; q < kMergeBatch; q++) {
                    const int k = k0 + q * tpo;
                    mk[q] = -INFINITY;
                    if (k < P) {
                        const float* pk = part_ptr(k);
                        mk[q] = __ldcg(pk + g);
                        lk[q] = __ldcg(pk + 8 + g);
                        v[q] = __ldcg(reinterpret_cast<const float4*>(pk + 16 + g * D) + d4);
                    }
                }
#pragma unroll
                for (int q = 0; q < kMergeBatch; q++) {
                    if (mk[q] == -INFINITY) continue;
                    const float Mn = fmaxf(M, mk[q]);
                    const float a = (M == -INFINITY) ? 0.f : exp2f(M - Mn), w = exp2f(mk[q] - Mn);
                    acc.x = fmaf(w, v[q].x, acc.x * a); acc.y = fmaf(w, v[q].y, acc.y * a);
                    acc.z = fmaf(w, v[q].z, acc.z * a); acc.w = fmaf(w, v[q].w, acc.w * a);
                    L = fmaf(w, lk[q], L * a);
                    M = Mn;
                }
            }
        }
        for (int m = 1; m < tpo; m <<= 1) {
            const float M2 = __shfl_xor_sync(0xffffffffu, M, m), L2 = __shfl_xor_sync(0xffffffffu, L, m);
            const float x2 = __shfl_xor_sync(0xffffffffu, acc.x, m), y2 = __shfl_xor_sync(0xffffffffu, acc.y, m);
            const float z2 = __shfl_xor_sync(0xffffffffu, acc.z, m), w2 = __shfl_xor_sync(0xffffffffu, acc.w, m);
            const float Mn = fmaxf(M, M2);
            const float a = (M == -INFINITY) ? 0.f : exp2f(M - Mn), c = (M2 == -INFINITY) ? 0.f : exp2f(M2 - Mn);
            acc.x = acc.x * a + x2 * c; acc.y = acc.y * a + y2 * c;
            acc.z = acc.z * a + z2 * c; acc.w = acc.w * a + w2 * c;
            L = L * a + L2 * c;
            M = Mn;
        }
        if (valid && pl == 0) {
            if (dst) {
                *reinterpret_cast<float4*>(dst + 16 + g * D + 4 * d4) = acc;
                if (d4 == 0) {
                    dst[g] = M;
                    dst[8 + g] = L;
                }
            } else {
                const float inv = (L > 0.f) ? o_mult / L : 0.f;
                const float x[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
                const int64_t oo = ((int64_t)b * Hq + h * Gq + hb * 8 + g) * D + 4 * d4;
                store_out<4>(out, out_fp32, oo, x);
            }
        }
    }
}

// CTAs per SM a decode kernel is compiled for: two (16 warps, up to 128
// registers per thread), which every format's full-head_dim accumulators need.
__host__ __device__ constexpr int decode_ctas(int kk, int vk, int D) {
    (void)kk;
    (void)vk;
    (void)D;
    return 2;
}

// The fused append (kvq_append_decode) of one sequence's newest token: role 0
// quantises its K row, role 1 its V row, role 2 both, into the stage (row t of
// the unit) and, when g is set, into the cache slab (row tp of the page).  Out
// of line: it runs once per sequence, and keeping it out of the decode loop
// keeps the loop's code compact.
template <int KK, int KV, int D>
__device__ __noinline__ void fused_append_rows(int role, int lane, const uint16_t* k_src, const uint16_t* v_src,
                                               bool rot_k, bool rot_v, float k_scale, float v_scale, uint8_t* st,
                                               uint8_t* g, int t, int tp, int u_ks, int u_vc, int u_vs, int c_ks,
                                               int c_vc, int c_vs) {
    using T = DecTraits<KK, KV, D>;
    if (role != 1) {
        quantize_row<KK, D>(k_src, rot_k, k_scale, st + t * T::KC, st + u_ks + t * T::KS, t, lane,
                            g ? g + tp * T::KC : nullptr, g ? g + c_ks + tp * T::KS : nullptr);
    }
    if (role != 0) {
        quantize_row<KV, D>(v_src, rot_v, v_scale, st + u_vc + t * T::VC, st + u_vs + t * T::VS, t, lane,
                            g ? g + c_vc + tp * T::VC : nullptr, g ? g + c_vs + tp * T::VS : nullptr);
    }
}

// The same rows quantised ahead of their unit (which == 0: K, 1: V) into a
// row buffer -- K codes at 0, K scales at KC, V codes at KC + 16, V scales at
// KC + 16 + VC (FusedRow) -- in row t's chunk permutation, and, when g is set,
// into the cache slab.
template <int KK, int KV, int D>
struct FusedRow {
    using T = DecTraits<KK, KV, D>;
    static constexpr int ks = T::KC, vc = T::KC + 16, vs = T::KC + 16 + T::VC;
    static_assert(T::KS <= 16 && T::VS <= 16 && T::KC % 16 == 0 && T::VC % 16 == 0, "row buffer layout");
    static_assert(T::KC <= 512 && T::VC <= 512, "one 16-byte piece per lane");
};
template <int KK, int KV, int D>
__device__ __noinline__ void fused_append_buf(int which, int lane, const uint16_t* src, bool rot, float tscale,
                                              uint8_t* buf, uint8_t* g, int t, int tp, int c_ks, int c_vc,
                                              int c_vs) {
    using T = DecTraits<KK, KV, D>;
    using R = FusedRow<KK, KV, D>;
    if (which == 0) {
        quantize_row<KK, D>(src, rot, tscale, buf, buf + R::ks, t, lane, g ? g + tp * T::KC : nullptr,
                            g ? g + c_ks + tp * T::KS : nullptr);
    } else {
        quantize_row<KV, D>(src, rot, tscale, buf + R::vc, buf + R::vs, t, lane,
                            g ? g + c_vc + tp * T::VC : nullptr, g ? g + c_vs + tp * T::VS : nullptr);
    }
}

template <int KK, int KV, int D, bool FUSED>
__global__ void __launch_bounds__(kDecThreads, decode_ctas(KK, KV, D)) decode_kernel(const DecodeParams p) {
    using T = DecTraits<KK, KV, D>;
    constexpr bool VFOLD = (KV == RK_E4M3_ROW256 || KV == RK_INT8_G64 || KV == RK_E4M3_MX32);
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = lane >> 2, j = lane & 3;
    const int H = p.L.H, P = p.L.P, HB = p.HB, HH = H * HB, B = p.B;
    const int64_t slab = p.L.slab;            // page slab stride in HBM
    const SpanLayout& U = p.U;                // what one stage holds
    const int NS = p.stages;

    // shared memory carve-up
    size_t off = ((size_t)NS * U.bytes + 127) & ~(size_t)127;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + off);   // full[stage]
    off += 8 * kMaxStages;
    int* rel = reinterpret_cast<int*>(smem + off);               // release count[stage]
    off += 4 * kMaxStages;
    volatile int* tagv = reinterpret_cast<volatile int*>(smem + off);   // unit last issued into [stage]
    off += 4 * kMaxStages;
    int* iss = reinterpret_cast<int*>(smem + off);               // copies issued into [stage]
    off += 4 * kMaxStages;
    float* osm = reinterpret_cast<float*>(smem + off);   // [8][D]: output combine
    off += 8 * kOsmStride<D> * 4;
    uint8_t* qst = smem + off;                           // q fragments of the segment (fp16 / bf16 hi, lo)
    off += 8 * (size_t)D * 2 * T::QS;
    float* wml = reinterpret_cast<float*>(smem + off);   // [8 warps][m 8, l 8]
    off += 8 * 16 * 4;
    float* fin = reinterpret_cast<float*>(smem + off);   // [m 8][l 8] of the merged segment
    off += 16 * 4;
    float* qhm = reinterpret_cast<float*>(smem + off);   // [8] score multiplier of each head of the block
    off += 8 * 4;
    int* flags = reinterpret_cast<int*>(smem + off);     // [0] abort, [1] this CTA merges
    off += 16;
    int* pref = reinterpret_cast<int*>(smem + off);      // [B + 1] page prefix
    off += 4 * (size_t)(B + 1);
    int* pids = reinterpret_cast<int*>(smem + off);      // [pid_cap] page ids of this CTA's range
    volatile int* abort_flag = flags;
    // units of a sequence of L tokens (at most max_pages pages of it)
    auto n_units = [&](int L) {
        const int u = L > 0 ? (L + U.sp - 1) / U.sp : 0;
        return min(u, p.max_pages << U.lg_up);
    };

    // ---- unit prefix over the batch (block scan): units of sequence b are
    // pref[b] .. pref[b + 1] - 1
    {
        const int per = (B + kDecThreads - 1) / kDecThreads;
        const int b0 = tid * per, b1 = min(B, b0 + per);
        int local = 0;
        for (int b = b0; b < b1; b++) {
            const int L = p.seq_lens[b];
            if (L > 0 && (L + P - 1) / P > p.max_pages) atomicOr(p.status, kStatusBadPage);
            local += n_units(L);
        }
        int incl = local;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, incl, m);
            if (lane >= m) incl += v;
        }
        if (lane == 31) wml[warp] = __int_as_float(incl);
        if (tid == 0) flags[0] = flags[1] = flags[2] = flags[3] = 0;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < warp; w++) base += __float_as_int(wml[w]);
        int run = base + incl - local;
        for (int b = b0; b < b1; b++) {
            pref[b] = run;
            run += n_units(p.seq_lens[b]);
        }
        if (tid == kDecThreads - 1) pref[B] = run;
        if (B == 0 && tid == 0) pref[0] = 0;
        __syncthreads();
    }

    // zero rows for empty sequences (one CTA per sequence)
    for (int b = blockIdx.x; b < B; b += gridDim.x) {
        if (pref[b + 1] == pref[b]) {
            for (int i = tid; i < p.Hq * D; i += kDecThreads) {
                int64_t o = (int64_t)b * p.Hq * D + i;
                if (p.out_fp32) reinterpret_cast<float*>(p.out)[o] = 0.f;
                else reinterpret_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(0.f);
            }
        }
    }

    const int64_t W = (int64_t)pref[B] * HH;
    if (W == 0) return;
    const int G = (int)(((int64_t)gridDim.x < W) ? (int64_t)gridDim.x : W);
    if ((int)blockIdx.x >= G) return;
    Partition part;
    part.pref = pref;
    part.B = B;
    part.HH = HH;
    part.c = p.seg_cost;
    part.G = G;
    part.W = W;
    part.C = part.seq_cost(B);
    const int64_t w0 = part.start(blockIdx.x), w1 = part.start(blockIdx.x + 1);
    const int n = (int)(w1 - w0);

    // ---- page ids of this CTA's range, loaded in parallel up front so that a
    // refill never waits on a block-table read
    auto checked = [&](int pid) {
        if (pid < 0 || pid >= p.L.num_pages) {
            atomicOr(p.status, kStatusBadPage);
            pid = 0;
        }
        return pid;
    };
    auto pid_at = [&](const Cursor& c) {
        return checked(p.block_table[(int64_t)c.b * p.max_pages + (c.span >> U.lg_up)]);
    };
    // Where unit w (of the whole batch) comes from: (slab index << 2) | the
    // unit's 64-token span within its page (for pages staged in spans).
    const uint32_t span_mask = (1u << U.lg_up) - 1u;
    auto unit_word = [&](const Cursor& c) {
        return ((uint32_t)(pid_at(c) * H + c.h) << 2) | ((uint32_t)c.span & span_mask);
    };
    auto unit_src = [&](int k) {   // unit k of this CTA's range
        if (k < p.pid_cap) return (uint32_t)pids[k];
        Cursor c;
        cursor_locate(c, w0 + k, pref, B, HH, HB);
        return unit_word(c);
    };

    // ---- producer: unit k of the range into stage k % NS (one copy of a whole
    // page slab, or the unit's rows of each of the slab's four arrays).  The
    // warp groups release their units independently, so units are refilled
    // out of order; tagv[s] records the unit a stage was last issued for, and a
    // consumer waits on the stage's mbarrier only once the tag names its unit
    // (the mbarrier's phase parity cannot tell a pending copy from a phase
    // completed two uses ago).
    auto issue = [&](int k, int s) {   // s == k % NS
        const uint32_t us = unit_src(k);
        const uint8_t* src = p.slabs + (int64_t)(us >> 2) * slab;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        const uint32_t bar = smem_u32(&bars[s]);
        const uint32_t dst = smem_u32(smem + (size_t)s * U.bytes);
        if (U.lg_up == 0) {
            mbar_expect_tx(bar, (uint32_t)slab);
            bulk_g2s(dst, src, (uint32_t)slab, bar);
        } else {
            const int64_t r0 = (int64_t)(us & 3u) * U.sp;
            const uint32_t nk = U.sp * p.L.kc, nks = U.sp * p.L.ks, nv = U.sp * p.L.vc, nvs = U.sp * p.L.vs;
            mbar_expect_tx(bar, nk + nks + nv + nvs);
            bulk_g2s(dst, src + r0 * p.L.kc, nk, bar);
            if (nks) bulk_g2s(dst + (uint32_t)U.off_ks, src + p.L.off_ks + r0 * p.L.ks, nks, bar);
            bulk_g2s(dst + (uint32_t)U.off_vc, src + p.L.off_vc + r0 * p.L.vc, nv, bar);
            if (nvs) bulk_g2s(dst + (uint32_t)U.off_vs, src + p.L.off_vs + r0 * p.L.vs, nvs, bar);
        }
        iss[s]++;
        __threadfence_block();
        tagv[s] = k;
    };
    // warp 0 starts the ring, lane s with stage s: its own cursor, block-table
    // read and copy, so that the first stages' latencies overlap, while the
    // other warps preload the range's unit sources
    if (warp == 0) {
        if (lane < NS) {
            mbar_init(smem_u32(&bars[lane]), 1);
            rel[lane] = 0;
            iss[lane] = 0;
            tagv[lane] = -1;
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        __syncwarp();
        if (lane < NS && lane < n) {
            Cursor c;
            cursor_locate(c, w0 + lane, pref, B, HH, HB);
            pids[lane] = (int)unit_word(c);
            issue(lane, lane);
        }
    }
    {
        // the q rows of the range's first segments, towards L2 ahead of their
        // segment starts (rows of one 8-head block are contiguous)
        Cursor c;
        cursor_locate(c, w0, pref, B, HH, HB);
        int64_t w = w0;
        for (int k = 0; k < 8 && w < w1; k++) {
            const int gq0 = c.hb * 8, rows = min(8, p.G - gq0);
            const uint16_t* q0 = p.q + ((int64_t)c.b * p.Hq + (int64_t)c.h * p.G + gq0) * D;
            if (tid < rows * D * 2 / 128)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(q0 + tid * 64));
            w += c.nspans - c.span;
            c.span = c.nspans - 1;
            cursor_next(c, pref, B, HH, HB);
        }
    }
    for (int k = NS + tid; k < n && k < p.pid_cap; k += kDecThreads) {
        Cursor c;
        cursor_locate(c, w0 + k, pref, B, HH, HB);
        pids[k] = (int)unit_word(c);
    }
    __syncthreads();

    // ---- consumer layout.  A warp owns a 16-token tile over all of head_dim.
    // A unit's tiles go to a group of wpu warps; the CTA's ngrp groups take a
    // segment's units in turn (unit i + g, i + g + ngrp, ... to group g), so
    // several units are in flight and every warp's state covers the whole
    // segment.
    const int tiles = U.sp >> 4;                  // 16-token tiles per unit
    const int wpu = tiles < 8 ? tiles : 8;        // warps per unit
    const int ngrp = (kDecThreads / 32) / wpu;    // units in flight
    const int grp = warp / wpu, tile = warp - grp * wpu;
    int seq_len = 0;
    float o[T::DTILES][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float hm0 = 1.f, hm1 = 1.f;   // score multipliers of heads 2j, 2j + 1 (q's power of two, K tensor scale)
    // V scales folded into P' (FP8 row-256, INT8, MX V): P' = P * (scale * 2^-ve),
    // ve a warp-uniform power-of-two reference raised (with the accumulators
    // rescaled) when a scale exceeds 2^(ve + 4); o is in units of 2^ve.  This
    // keeps P' inside fp16's normal range whatever the magnitude of V.
    int ve = 0;
    float vmul = 1.f, vthr = 0.f;   // 2^-ve; 2^(ve + 4), 0 before the segment's first nonzero scale

    // Per-lane byte offsets inside a stage: lane (r, j) reads token rows r and
    // r + 8 of a tile (same chunk permutation, since the permutation depends on
    // the row modulo 4), chunk cl at 4 * KCH * j within it.
    const int swk = row_swizzle(KK, D, r), swv = row_swizzle(KV, D, r);
    auto koff = [&](int cl) { return (uint32_t)(r * T::KC + phys_byte((T::KCW * cl + 4 * T::KCH * j) * T::KBITS / 8, swk)); };
    auto voff = [&](int cl) { return (uint32_t)(r * T::VC + phys_byte((T::VCW * cl + 4 * T::VCH * j) * T::VBITS / 8, swv)); };
    auto ksoff = [&](int cl) {
        if constexpr (KK == RK_E2M1_G16) return (uint32_t)(r * T::KS + (T::KCW * cl + 16 * j) / 16);
        else if constexpr (KK == RK_INT8_G64) return (uint32_t)(r * T::KS + 2 * cl);
        else if constexpr (KK == RK_E4M3_MX32) return (uint32_t)(r * T::KS + cl);
        else return (uint32_t)(r * T::KS);
    };
    auto vsoff = [&](int cl) {
        if constexpr (KV == RK_E2M1_G16) return (uint32_t)(r * T::VS + (T::VCW * cl + 16 * j) / 16);
        else if constexpr (KV == RK_INT8_G64) return (uint32_t)(r * T::VS + 2 * cl);
        else if constexpr (KV == RK_E4M3_MX32) return (uint32_t)(r * T::VS + cl);
        else return (uint32_t)(r * T::VS);
    };
    const uint32_t off_ks = (uint32_t)U.off_ks, off_vc = (uint32_t)U.off_vc, off_vs = (uint32_t)U.off_vs;

    Cursor cc;
    cursor_locate(cc, w0, pref, B, HH, HB);
    for (int i = 0; i < n;) {
        const int b = cc.b, h = cc.h, hb = cc.hb;
        const int span0 = cc.span, nspans = cc.nspans;
        const int seg_n = min(nspans - span0, n - i);   // this segment's units in the range
        const bool seg_first = (i == 0);
        seq_len = p.seq_lens[b];
        {
            // ---- segment start: q rows of this 8-head block, rotated and scaled.
            // Warp w stages head w, already in the MMA fragment order: for
            // k-step st, lane group j, head n, the 4 values of that lane's slice
            // as fp16 pairs (hi, and lo for a bf16 split).
            const int gq = hb * 8 + warp;
            float x[8];
            if (gq < p.G) {
                const uint16_t* qrow = p.q + ((int64_t)b * p.Hq + h * p.G + gq) * D + lane * T::EPL;
                uint32_t raw[4];
                if constexpr (T::EPL == 8) {
                    const uint4 v = *reinterpret_cast<const uint4*>(qrow);
                    raw[0] = v.x; raw[1] = v.y; raw[2] = v.z; raw[3] = v.w;
                } else {
                    const uint2 v = *reinterpret_cast<const uint2*>(qrow);
                    raw[0] = v.x; raw[1] = v.y; raw[2] = raw[3] = 0;
                }
#pragma unroll
                for (int e = 0; e < T::EPL; e++) x[e] = bf16_bits_to_f32((raw[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
                if constexpr (D == 256) {
                    if (p.rot_k) {
                        Row8 y;
#pragma unroll
                        for (int e = 0; e < 8; e++) y.v[e] = x[e];
                        y = fwht256_row(y, lane);
#pragma unroll
                        for (int e = 0; e < 8; e++) x[e] = y.v[e];
                    }
                }
                // q x softmax scale x log2(e), normalised by a power of two so
                // that its largest element lies in [1, 2): fp16 keeps full
                // precision whatever q's magnitude; the 2^e returns in the
                // fp32 scores (with the K tensor scale, for FP8 per tensor)
                float amax = 0.f;
#pragma unroll
                for (int e = 0; e < T::EPL; e++) {
                    x[e] *= p.q_mult;
                    amax = fmaxf(amax, fabsf(x[e]));
                }
                amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
                const int eq = amax > 0.f ? exp2_floor(amax) : 0;
                const float nq = pow2i(-eq);
#pragma unroll
                for (int e = 0; e < T::EPL; e++) x[e] *= nq;
                if (lane == 0) qhm[warp] = pow2i(eq) * p.k_tmult;
            } else {
#pragma unroll
                for (int e = 0; e < T::EPL; e++) x[e] = 0.f;
                if (lane == 0) qhm[warp] = 0.f;
            }
#pragma unroll
            for (int g4 = 0; g4 < T::EPL / 4; g4++) {
                const int d0 = lane * T::EPL + 4 * g4;
                const int c = d0 / T::KCW, rem = d0 % T::KCW;
                const int jj = rem / (4 * T::KCH), ks = (rem % (4 * T::KCH)) / 4;
                const int st = c * T::KCH + ks;
                const float* v = x + 4 * g4;
                const int slot = (st * 4 + jj) * 8 + warp;
                if constexpr (T::QS == 2) {
                    float lo[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) lo[e] = v[e] - __bfloat162float(__float2bfloat16_rn(v[e]));
                    reinterpret_cast<uint4*>(qst)[slot] = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                                     pack_bf16(lo[0], lo[1]), pack_bf16(lo[2], lo[3]));
                } else {
                    reinterpret_cast<uint2*>(qst)[slot] = make_uint2(pack_f16(v[0], v[1]), pack_f16(v[2], v[3]));
                }
            }
            if (FUSED && fused_early(KK, KV) && warp >= 6 && span0 + seg_n == nspans && seg_n <= kFusedEarly) {
                // fused append ahead of its unit: the range reaches the segment's
                // last unit soon, so its copies are in flight now.  Warp 6
                // quantises the newest token's K row, warp 7 its V row, into the
                // row buffer in the output-combine area (untouched until the
                // segment's units are done) and, for head block 0, into the cache.
                const int span = nspans - 1;
                const int t = (seq_len - 1) - span * U.sp;
                if (t < U.sp) {
                    const int tp = t + (span & ((1 << U.lg_up) - 1)) * U.sp;
                    uint8_t* g = (hb == 0) ? p.slabs + (int64_t)(unit_src(i + seg_n - 1) >> 2) * slab : nullptr;
                    const int64_t row = ((int64_t)b * H + h) * D;
                    const int which = warp - 6;
                    fused_append_buf<KK, KV, D>(which, lane, (which ? p.v_new : p.k_new) + row,
                                                which ? p.rot_v : p.rot_k, which ? p.v_scale : p.k_scale,
                                                reinterpret_cast<uint8_t*>(osm), g, t, tp, (int)p.L.off_ks,
                                                (int)p.L.off_vc, (int)p.L.off_vs);
                }
            }
        }
        __syncthreads();
        hm0 = qhm[2 * j];
        hm1 = qhm[2 * j + 1];
#pragma unroll
        for (int u = 0; u < T::DTILES; u++) o[u][0] = o[u][1] = o[u][2] = o[u][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
        ve = 0;
        vmul = 1.f;
        vthr = 0.f;

        // ---- this group's units of the segment
        // the group's first unit of the segment: its stage and mbarrier phase
        // (one division per segment; per unit they advance by ngrp)
        int s = (i + grp) % NS;
        uint32_t ph = (uint32_t)((i + grp) / NS) & 1u;
        for (int u = i + grp; u < i + seg_n; u += ngrp) {
            const int span = span0 + (u - i);
            {
                // wait until the stage was issued for this unit, then for its data
                long it = 0;
                while (tagv[s] != u && !*abort_flag) {
                    if (++it > p.wait_polls) {
                        *abort_flag = 1;
                        break;
                    }
                }
                (void)mbar_wait(smem_u32(&bars[s]), ph, abort_flag, p.wait_polls);
            }
            const uint32_t stg = (uint32_t)s * (uint32_t)U.bytes;   // byte offset of the stage

            if (FUSED && span == nspans - 1) {
                // fused append: the sequence's newest token (position seq_len - 1) lies
                // in its last unit.  Quantise it into this stage (row t of the unit),
                // over whatever the copy brought, and into the cache (row tp of the
                // page; one head block writes the cache).  t and tp differ by a
                // multiple of 64, so the row's chunk permutation is the same.
                // A sequence longer than its block table (flagged by the unit
                // prefix) has no row to append: t would fall outside the unit.
                // With few of the segment's units in the range the row was
                // quantised at the segment start; the warp that owns row t's tile
                // (the only one that reads it) copies it from the row buffer.
                const int t = (seq_len - 1) - span * U.sp;
                const int tp = t + (span & ((1 << U.lg_up) - 1)) * U.sp;
                // 0: K row, 1: V row, 2: both (a group of one warp), 3: neither
                const int role = t >= U.sp                                 ? 3
                                 : fused_early(KK, KV) && seg_n <= kFusedEarly ? 4
                                 : wpu >= 2                                    ? (tile < 2 ? tile : 3)
                                                                               : 2;
                if (role == 4 && tile == (t >> 4) % wpu) {
                    using R = FusedRow<KK, KV, D>;
                    const uint8_t* fb = reinterpret_cast<const uint8_t*>(osm);
                    uint8_t* st = smem + stg;
                    if (lane < T::KC / 16)
                        reinterpret_cast<uint4*>(st + t * T::KC)[lane] = reinterpret_cast<const uint4*>(fb)[lane];
                    if (lane < T::VC / 16)
                        reinterpret_cast<uint4*>(st + off_vc + t * T::VC)[lane] =
                            reinterpret_cast<const uint4*>(fb + R::vc)[lane];
                    if (lane < T::KS) st[off_ks + t * T::KS + lane] = fb[R::ks + lane];
                    if (lane < T::VS) st[off_vs + t * T::VS + lane] = fb[R::vs + lane];
                }
                if (role <= 2) {
                    uint8_t* g = (hb == 0) ? p.slabs + (int64_t)(unit_src(u) >> 2) * slab : nullptr;
                    const int64_t row = (int64_t)b * H + h;
                    fused_append_rows<KK, KV, D>(role, lane, p.k_new + row * D, p.v_new + row * D, p.rot_k, p.rot_v,
                                                 p.k_scale, p.v_scale, smem + stg, g, t, tp, (int)off_ks, (int)off_vc,
                                                 (int)off_vs, (int)p.L.off_ks, (int)p.L.off_vc, (int)p.L.off_vs);
                }
                if (wpu > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(wpu * 32) : "memory");
                else __syncwarp();
            }

            for (int mt = tile; mt < tiles; mt += wpu) {
                const int valid = seq_len - (span * U.sp + mt * 16);
                if (valid <= 0) break;
                const uint32_t kt = stg + mt * 16 * T::KC, kst = stg + off_ks + mt * 16 * T::KS;
                const uint32_t vt = stg + off_vc + mt * 16 * T::VC, vst = stg + off_vs + mt * 16 * T::VS;
                // ---------- S^T = K q^T over all of head_dim (tokens as M, heads as N)
                float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int cl = 0; cl < T::KCHUNKS; cl++) {
                    uint32_t xa[2 * T::KCH], xb[2 * T::KCH];
                    slice_f16<KK, T::KNB, T::KCH>(lds_bytes<T::KNB>(smem + kt, koff(cl)), xa);
                    slice_f16<KK, T::KNB, T::KCH>(lds_bytes<T::KNB>(smem + kt, koff(cl) + 8 * T::KC), xb);
                    if constexpr (KK == RK_E2M1_G16) {
                        const uint32_t sa = f16_splat(dec_e4m3x2_f16x2(smem[kst + ksoff(cl)]));
                        const uint32_t sb = f16_splat(dec_e4m3x2_f16x2(smem[kst + ksoff(cl) + 8 * T::KS]));
#pragma unroll
                        for (int e = 0; e < 2 * T::KCH; e++) {
                            xa[e] = hmul2(xa[e], sa);
                            xb[e] = hmul2(xb[e], sb);
                        }
                    }
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < T::KCH; ks++) {
                        const int sl = cl * T::KCH + ks;
                        const uint32_t a[4] = {xa[2 * ks], xb[2 * ks], xa[2 * ks + 1], xb[2 * ks + 1]};
                        if constexpr (T::QS == 2) {
                            const uint4 qv = reinterpret_cast<const uint4*>(qst)[(sl * 4 + j) * 8 + r];
                            mma_bf16(acc, a, qv.x, qv.y);
                            mma_bf16(acc, a, qv.z, qv.w);
                        } else {
                            const uint2 qv = reinterpret_cast<const uint2*>(qst)[(sl * 4 + j) * 8 + r];
                            mma_f16(acc, a, qv.x, qv.y);
                        }
                    }
                    if constexpr (KK == RK_INT8_G64 || KK == RK_E4M3_MX32) {
                        float fa, fb;
                        if constexpr (KK == RK_INT8_G64) {
                            fa = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(smem + kst + ksoff(cl)));
                            fb = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(smem + kst + ksoff(cl) + 8 * T::KS));
                        } else {
                            fa = ue8m0_to_f32(smem[kst + ksoff(cl)]);
                            fb = ue8m0_to_f32(smem[kst + ksoff(cl) + 8 * T::KS]);
                        }
                        sc[0] = fmaf(acc[0], fa, sc[0]);
                        sc[1] = fmaf(acc[1], fa, sc[1]);
                        sc[2] = fmaf(acc[2], fb, sc[2]);
                        sc[3] = fmaf(acc[3], fb, sc[3]);
                    } else {
                        sc[0] += acc[0]; sc[1] += acc[1]; sc[2] += acc[2]; sc[3] += acc[3];
                    }
                }
                if constexpr (KK == RK_E4M3_ROW256) {
                    const float fa = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(smem + kst + ksoff(0)));
                    const float fb = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(smem + kst + ksoff(0) + 8 * T::KS));
                    sc[0] *= fa; sc[1] *= fa; sc[2] *= fb; sc[3] *= fb;
                }
                // q's power of two (and the K tensor scale) back into the fp32 scores
                sc[0] *= hm0; sc[1] *= hm1; sc[2] *= hm0; sc[3] *= hm1;
                const bool oka = r < valid, okb = r + 8 < valid;
                if (!oka) sc[0] = sc[1] = -INFINITY;
                if (!okb) sc[2] = sc[3] = -INFINITY;

                // ---------- online softmax (log2 domain), heads 2j and 2j+1.  The
                // running max is raised (with a warp-wide reduction and a rescale of
                // the accumulators) only when a score exceeds it by more than 2^3;
                // otherwise weights up to 8 are kept as they are.
                {
                    const float x0 = fmaxf(sc[0], sc[2]), x1 = fmaxf(sc[1], sc[3]);
                    if (__any_sync(0xffffffffu, (x0 > m0 + 3.f) || (x1 > m1 + 3.f))) {
                        float y0 = x0, y1 = x1;
#pragma unroll
                        for (int m = 4; m < 32; m <<= 1) {
                            y0 = fmaxf(y0, __shfl_xor_sync(0xffffffffu, y0, m));
                            y1 = fmaxf(y1, __shfl_xor_sync(0xffffffffu, y1, m));
                        }
                        const float n0 = fmaxf(m0, y0), n1 = fmaxf(m1, y1);
                        const float a0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - n0);
                        const float a1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - n1);
#pragma unroll
                        for (int u2 = 0; u2 < T::DTILES; u2++) {
                            o[u2][0] *= a0; o[u2][1] *= a1; o[u2][2] *= a0; o[u2][3] *= a1;
                        }
                        l0 *= a0;
                        l1 *= a1;
                        m0 = n0;
                        m1 = n1;
                    }
                }
                const float r0 = (m0 == -INFINITY) ? 0.f : m0, r1 = (m1 == -INFINITY) ? 0.f : m1;
                const float p0 = fast_exp2(sc[0] - r0), p1 = fast_exp2(sc[1] - r1);
                const float p2 = fast_exp2(sc[2] - r0), p3 = fast_exp2(sc[3] - r1);
                l0 += p0 + p2;
                l1 += p1 + p3;

                // ---------- O^T += V^T P^T over all of head_dim
                // rows past seq_len hold bytes never written: keep them out of the
                // product entirely (their P is 0, but 0 x NaN would still be NaN)
                const bool partial = valid < 16;
                uint32_t pb0 = 0, pb1 = 0;   // P'^T fragment (B operand)
                // V scales folded into P': this lane's rows r and r + 8, one per
                // chunk (INT8, MX) or one per row (FP8 row-256), rows past seq_len 0
                constexpr int NVS = VFOLD ? (KV == RK_E4M3_ROW256 ? 1 : T::VCHUNKS) : 1;
                float vfa[NVS], vfb[NVS];
                if constexpr (VFOLD) {
                    float smax = 0.f;
#pragma unroll
                    for (int c = 0; c < NVS; c++) {
                        if constexpr (KV == RK_E4M3_MX32) {
                            vfa[c] = ue8m0_to_f32(smem[vst + vsoff(c)]);
                            vfb[c] = ue8m0_to_f32(smem[vst + vsoff(c) + 8 * T::VS]);
                        } else {
                            vfa[c] = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(smem + vst + vsoff(c)));
                            vfb[c] = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(smem + vst + vsoff(c) + 8 * T::VS));
                        }
                        vfa[c] = oka ? vfa[c] : 0.f;
                        vfb[c] = okb ? vfb[c] : 0.f;
                        smax = fmaxf(smax, fmaxf(vfa[c], vfb[c]));
                    }
                    if (__any_sync(0xffffffffu, smax > vthr)) {
                        // raise the reference to the warp's largest scale (an exact power of two)
                        const int en =
                            exp2_floor(__uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(smax))));
                        const float f = vthr > 0.f ? pow2i(ve - en) : 1.f;
#pragma unroll
                        for (int u2 = 0; u2 < T::DTILES; u2++) {
                            o[u2][0] *= f; o[u2][1] *= f; o[u2][2] *= f; o[u2][3] *= f;
                        }
                        ve = en;
                        vmul = pow2i(-en);
                        vthr = pow2i(en + 4);
                    }
#pragma unroll
                    for (int c = 0; c < NVS; c++) {
                        vfa[c] *= vmul;
                        vfb[c] *= vmul;
                    }
                }
                if constexpr (KV == RK_E4M3_ROW256) {
                    pb0 = movtrans(pack_f16(p0 * vfa[0], p1 * vfa[0]));
                    pb1 = movtrans(pack_f16(p2 * vfb[0], p3 * vfb[0]));
                } else if constexpr (!VFOLD) {
                    pb0 = movtrans(pack_f16(p0, p1));
                    pb1 = movtrans(pack_f16(p2, p3));
                }
#pragma unroll
                for (int cl = 0; cl < T::VCHUNKS; cl++) {
                    if constexpr (KV == RK_INT8_G64 || KV == RK_E4M3_MX32) {
                        pb0 = movtrans(pack_f16(p0 * vfa[cl], p1 * vfa[cl]));
                        pb1 = movtrans(pack_f16(p2 * vfb[cl], p3 * vfb[cl]));
                    }
                    uint32_t xa[2 * T::VCH], xb[2 * T::VCH];
                    slice_f16<KV, T::VNB, T::VCH>(lds_bytes<T::VNB>(smem + vt, voff(cl)), xa);
                    slice_f16<KV, T::VNB, T::VCH>(lds_bytes<T::VNB>(smem + vt, voff(cl) + 8 * T::VC), xb);
                    if constexpr (KV == RK_E2M1_G16) {
                        const uint32_t sa = f16_splat(dec_e4m3x2_f16x2(smem[vst + vsoff(cl)]));
                        const uint32_t sb = f16_splat(dec_e4m3x2_f16x2(smem[vst + vsoff(cl) + 8 * T::VS]));
#pragma unroll
                        for (int e = 0; e < 2 * T::VCH; e++) {
                            xa[e] = hmul2(xa[e], sa);
                            xb[e] = hmul2(xb[e], sb);
                        }
                    }
                    if (partial) {
#pragma unroll
                        for (int e = 0; e < 2 * T::VCH; e++) {
                            xa[e] = oka ? xa[e] : 0u;
                            xb[e] = okb ? xb[e] : 0u;
                        }
                    }
#pragma unroll
                    for (int u2 = 0; u2 < T::VCH; u2++) {
                        const uint32_t a[4] = {movtrans(xa[2 * u2]), movtrans(xa[2 * u2 + 1]), movtrans(xb[2 * u2]),
                                               movtrans(xb[2 * u2 + 1])};
                        mma_f16(o[cl * T::VCH + u2], a, pb0, pb1);
                    }
                }
            }

            // ---- release stage s; the last warp of the group to release it refills
            // it.  The warp's reads of the stage have all returned (their values
            // fed the MMAs above), so the count needs no fence before it.
            __syncwarp();
            if (lane == 0) {
                const int old = atomicAdd(&rel[s], 1);
                if (old == wpu - 1) {
                    rel[s] = 0;
                    __threadfence_block();
                    if (u + NS < n && !*abort_flag) issue(u + NS, s);
                }
            }
            s += ngrp;
            while (s >= NS) {
                s -= NS;
                ph ^= 1u;
            }
        }

        // ---- segment end: merge the warps -- max, rescaled sums, rescaled
        // outputs.  Every warp holds a state for the segment (a warp that saw no
        // token of it has m = -inf, l = 0, o = 0).
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, m);
            l1 += __shfl_xor_sync(0xffffffffu, l1, m);
        }
        if (r == 0) {
            wml[warp * 16 + 2 * j] = m0;
            wml[warp * 16 + 2 * j + 1] = m1;
            wml[warp * 16 + 8 + 2 * j] = l0;
            wml[warp * 16 + 8 + 2 * j + 1] = l1;
        }
        __syncthreads();   // every warp's units of the segment done; osm free
        {
            float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
            for (int w = 0; w < 8; w++) {
                M0 = fmaxf(M0, wml[w * 16 + 2 * j]);
                M1 = fmaxf(M1, wml[w * 16 + 2 * j + 1]);
            }
            // this warp's outputs back in real units: o is held in units of 2^ve
            const float vu = VFOLD ? pow2i(ve) : 1.f;
            const float f0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - M0) * vu;
            const float f1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M1) * vu;
            if (tid < 8) {
                float M = -INFINITY, Ls = 0.f;
                for (int w = 0; w < 8; w++) M = fmaxf(M, wml[w * 16 + tid]);
                for (int w = 0; w < 8; w++) {
                    const float mw = wml[w * 16 + tid];
                    if (mw != -INFINITY) Ls += exp2f(mw - M) * wml[w * 16 + 8 + tid];
                }
                fin[tid] = M;
                fin[8 + tid] = Ls;
            }
            // eight rounds: in round q warp w adds d-tile chunk (w + q) % 8 of its
            // output into the combine buffer (round 0 stores), so all warps work in
            // every round on disjoint chunks; the order of the sum is fixed.  A
            // lane's values: heads 2j, 2j+1; dims VCW*(u/VCH) + 4*(u%VCH) + [0 | 2]
            // + its row part (u the d-tile).  The chunk is picked by a switch so
            // that o is indexed statically and stays in registers.
            float* pa = osm + (2 * j) * kOsmStride<D> + 4 * T::VCH * (r >> 1) + (r & 1);
            float* pb = pa + kOsmStride<D>;
            constexpr int DT8 = T::DTILES / 8;
            // d-tiles u of chunk ch (a static index into o for each case)
            auto add_chunk = [&](auto chc, bool first) {
                constexpr int ch = decltype(chc)::value;
#pragma unroll
                for (int z = 0; z < DT8; z++) {
                    const int u2 = ch * DT8 + z;
                    const int d = T::VCW * (u2 / T::VCH) + 4 * (u2 % T::VCH);
                    if (first) {
                        pa[d] = o[u2][0] * f0; pb[d] = o[u2][1] * f1;
                        pa[d + 2] = o[u2][2] * f0; pb[d + 2] = o[u2][3] * f1;
                    } else {
                        pa[d] += o[u2][0] * f0; pb[d] += o[u2][1] * f1;
                        pa[d + 2] += o[u2][2] * f0; pb[d + 2] += o[u2][3] * f1;
                    }
                }
            };
#pragma unroll 1
            for (int q = 0; q < 8; q++) {
                const bool first = q == 0;
                switch ((warp + q) & 7) {
                case 0: add_chunk(std::integral_constant<int, 0>{}, first); break;
                case 1: add_chunk(std::integral_constant<int, 1>{}, first); break;
                case 2: add_chunk(std::integral_constant<int, 2>{}, first); break;
                case 3: add_chunk(std::integral_constant<int, 3>{}, first); break;
                case 4: add_chunk(std::integral_constant<int, 4>{}, first); break;
                case 5: add_chunk(std::integral_constant<int, 5>{}, first); break;
                case 6: add_chunk(std::integral_constant<int, 6>{}, first); break;
                default: add_chunk(std::integral_constant<int, 7>{}, first); break;
                }
                __syncthreads();
            }
        }

        // ---- a whole segment is normalised and stored here; a segment cut by
        // a range boundary leaves its unnormalised output as this CTA's partial
        // (rotated back already: the Hadamard is linear, so merging commutes
        // with it) for the merge after the loop.
        {
            const int64_t seg_w0 = (int64_t)pref[b] * HH + (int64_t)cc.hh * nspans;
            const bool whole = (seg_w0 >= w0) && (seg_w0 + nspans <= w1);
            float* part = p.partials + ((int64_t)blockIdx.x * 2 + (seg_first ? 0 : 1)) * (16 + 8 * D);
            if (!whole && tid < 16) part[tid] = fin[tid];
            const int nh = warp;   // warp w finishes head w of the block
            const int gq = hb * 8 + nh;
            if (gq < p.G) {
                const float Ls = fin[8 + nh];
                const float inv = whole ? ((Ls > 0.f) ? p.o_mult / Ls : 0.f) : 1.f;
                float x[8];
#pragma unroll
                for (int e = 0; e < T::EPL; e++) x[e] = osm[nh * kOsmStride<D> + lane * T::EPL + e] * inv;
                if constexpr (D == 256) {
                    if (p.rot_v) {
                        Row8 y;
#pragma unroll
                        for (int e = 0; e < 8; e++) y.v[e] = x[e];
                        y = fwht256_row(y, lane);
#pragma unroll
                        for (int e = 0; e < 8; e++) x[e] = y.v[e];
                    }
                }
                if (!whole) {
                    float* dst = part + 16 + nh * D + lane * T::EPL;
#pragma unroll
                    for (int e = 0; e < T::EPL; e += 4)
                        *reinterpret_cast<float4*>(dst + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
                } else {
                    const int64_t ob = ((int64_t)b * p.Hq + h * p.G + gq) * D + lane * T::EPL;
                    store_out<T::EPL>(p.out, p.out_fp32, ob, x);
                }
            }
        }
        __syncthreads();   // osm, fin and qst are free again

        i += seg_n;
        if (i < n) {   // to the next segment's first unit
            cc.span = nspans - 1;
            cursor_next(cc, pref, B, HH, HB);
        }
    }

    __syncthreads();
    if (*abort_flag) {
        if (tid == 0) {
            atomicOr(p.status, kStatusWaitTimeout);
            // wait (bounded) for the copies still in flight: the last one issued into each stage
            int dummy = 0;
            for (int s2 = 0; s2 < NS; s2++)
                if (iss[s2] > 0) (void)mbar_wait(smem_u32(&bars[s2]), (uint32_t)((iss[s2] - 1) & 1), &dummy);
        }
        __syncthreads();
    }

    // ---- merge the cut segments, with no CTA waiting on another.  A cut
    // segment's parts (CTAs i_first..i_last) fall in groups of kFewParts
    // consecutive CTAs; every part counts itself in on its group's counter,
    // and the last to arrive merges the group.  A segment of one group is
    // then done; otherwise the group's merge is one more part, counted in on
    // the segment's counter, and the last group merged merges the groups.
    // Counters are indexed by the CTA holding the group's (or segment's)
    // last part -- a CTA ends at most one group of one cut segment -- and
    // are left zero for the next call.
    if (G > 1 && n > 0) {
        Cursor c0, c1;
        cursor_locate(c0, w0, pref, B, HH, HB);
        cursor_locate(c1, w1 - 1, pref, B, HH, HB);
        const int64_t PSZ = 16 + 8 * (int64_t)D;   // floats of one part
        for (int k = 0; k < 2; k++) {
            const Cursor& c = k == 0 ? c0 : c1;
            if (k == 1 && c1.b == c0.b && c1.hh == c0.hh) break;
            const int64_t seg_w0 = (int64_t)pref[c.b] * HH + (int64_t)c.hh * c.nspans;
            if (seg_w0 >= w0 && seg_w0 + c.nspans <= w1) continue;     // whole: already stored
            const int i_first = part.owner(c.b, c.hh, 0);
            const int i_last = part.owner(c.b, c.hh, c.nspans - 1);
            const int P = i_last - i_first + 1, Q = (P + kFewParts - 1) / kFewParts;
            const int g_first = i_first + ((int)blockIdx.x - i_first) / kFewParts * kFewParts;
            const int g_last = min(i_last, g_first + kFewParts - 1);
            __syncthreads();   // this CTA's partial is written
            if (tid == 0) {
                __threadfence();
                const unsigned old = atomicAdd(&p.grp_count[g_last], 1u);
                flags[1] = (old == (unsigned)(g_last - g_first));
                if (flags[1]) {
                    p.grp_count[g_last] = 0u;
                    __threadfence();
                }
            }
            __syncthreads();
            if (!flags[1]) continue;
            // parts: slot 1 of the segment's first CTA if the segment is its
            // range's last, else slot 0 (the segment is every other part's first)
            const int slot0 = part.start(i_first) >= seg_w0 ? 0 : 1;
            const float* pbase = p.partials + (int64_t)g_first * 2 * PSZ;     // part kk at pbase + 2 kk PSZ
            const float* pfirst = pbase + (g_first == i_first ? slot0 : 0) * PSZ;
            const float* plast = p.partials + (int64_t)g_last * 2 * PSZ;
            if (Q == 1) {
                merge_parts<D>(pfirst, plast, pbase, 2 * PSZ, P, nullptr, p.out, p.out_fp32, p.o_mult, p.Hq, p.G,
                               c.b, c.h, c.hb);
                continue;
            }
            merge_parts<D>(pfirst, plast, pbase, 2 * PSZ, g_last - g_first + 1, p.group_partials + (int64_t)g_last * PSZ,
                           p.out, p.out_fp32, p.o_mult, p.Hq, p.G, c.b, c.h, c.hb);
            __syncthreads();   // the group's merge is written
            if (tid == 0) {
                __threadfence();
                const unsigned old = atomicAdd(&p.seg_groups[i_last], 1u);
                flags[1] = (old == (unsigned)(Q - 1));
                if (flags[1]) {
                    p.seg_groups[i_last] = 0u;
                    __threadfence();
                }
            }
            __syncthreads();
            if (!flags[1]) continue;
            // group qq's merge sits at the CTA of its last part: i_first + 16 qq + 15, the last at i_last
            const float* gbase = p.group_partials + (int64_t)(i_first + kFewParts - 1) * PSZ;
            merge_parts<D>(gbase, p.group_partials + (int64_t)i_last * PSZ, gbase, kFewParts * PSZ, Q, nullptr, p.out,
                           p.out_fp32, p.o_mult, p.Hq, p.G, c.b, c.h, c.hb);
        }
    }
}

// ------------------------------------------------------------ host side

template <int KK, int KV, int D>
static const void* kernel_ptr(bool fused) {
    return fused ? reinterpret_cast<const void*>(&decode_kernel<KK, KV, D, true>)
                 : reinterpret_cast<const void*>(&decode_kernel<KK, KV, D, false>);
}

static const void* decode_kernel_for(int fmt, int D, bool fused) {
    const int kk = kind_of(fmt, 0), vk = kind_of(fmt, 1);
#define KVQ_CASE(KK, KV)                                        \
    if (kk == KK && vk == KV) {                                 \
        if (D == 256) return kernel_ptr<KK, KV, 256>(fused);    \
        if (D == 128) return kernel_ptr<KK, KV, 128>(fused);    \
    }
    KVQ_CASE(RK_BF16RAW, RK_FP16)
    KVQ_CASE(RK_E4M3_ROW256, RK_E4M3_ROW256)
    KVQ_CASE(RK_INT8_G64, RK_INT8_G64)
    KVQ_CASE(RK_E2M1_G16, RK_E2M1_G16)
    KVQ_CASE(RK_E4M3_ROW256, RK_E2M1_G16)
    KVQ_CASE(RK_E4M3_MX32, RK_E4M3_MX32)
    KVQ_CASE(RK_E4M3_TENSOR, RK_E4M3_TENSOR)
#undef KVQ_CASE
    return nullptr;
}

bool decode_supported(int fmt, int D) {
    if (fmt == F_FP8_ROW256 || fmt == F_K8V4) return D == 256;
    return D == 128 || D == 256;
}

static size_t fixed_smem(int D, int B, int pid_cap, int qs) {
    const size_t ostr = (size_t)D + 4;   // kOsmStride
    const size_t osm = 8 * ostr * 4;
    const size_t qst = 8 * (size_t)D * 2 * qs;
    return 8 * kMaxStages + 3 * 4 * kMaxStages + osm + qst + 8 * 16 * 4 + 16 * 4 + 8 * 4 + 16 + 4 * (size_t)(B + 1) +
           4 * (size_t)pid_cap + 128;
}

cudaError_t plan_decode(const Layout& L, int B, int HB, int max_seq_len, DecodePlan* plan) {
    if (B > kMaxBatch) return cudaErrorInvalidValue;
    int dev = 0, sms = 0, smem_sm = 0, smem_blk = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&smem_blk, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
    // decode-only and fused kernels share the plan (and so the workspace size)
    const void* kerns[2] = {decode_kernel_for(L.fmt, L.D, false), decode_kernel_for(L.fmt, L.D, true)};
    if (!kerns[0] || !kerns[1]) return cudaErrorInvalidValue;
    // The most CTAs per SM the kernel allows, each with at least three stages
    // (one CTA: two).  A stage holds a whole page if that fits, else (128- and
    // 256-token pages) a 64-token unit.  The shared memory left over holds the
    // preloaded page ids.
    constexpr int kMinPids = 64;
    const int lg_unit = L.P == 128 ? 1 : L.P == 256 ? 2 : 0;
    for (int ctas = decode_ctas(L.kk, L.vk, L.D); ctas >= 1; ctas--) {
        const size_t fixed = fixed_smem(L.D, B, kMinPids, L.kk == RK_BF16RAW ? 2 : 1);
        const int64_t budget = ctas >= 2 ? (int64_t)smem_sm / ctas - 1024 : (int64_t)smem_blk;
        for (int lg_up = 0; lg_up <= lg_unit; lg_up += (lg_unit ? lg_unit : 1)) {
            const SpanLayout U = make_span(L, lg_up);
            const int64_t units = (max_seq_len + U.sp - 1) / U.sp;
            const int64_t work = (int64_t)B * units * L.H * HB > 0 ? (int64_t)B * units * L.H * HB : 1;
            const int64_t grid = (int64_t)sms * ctas < work ? (int64_t)sms * ctas : work;
            int64_t stages = (budget - (int64_t)fixed) / U.bytes;
            if (stages > 6) stages = 6;
            if (stages < (ctas >= 2 ? 3 : 2)) continue;
            const int64_t stage_bytes = ((int64_t)stages * U.bytes + 127) & ~(int64_t)127;
            int64_t cap = (work + grid - 1) / grid + 1;                  // units of the largest range
            if (cap < stages) cap = stages;   // the first stages' page ids go there too
            const int64_t room = kMinPids + (budget - (int64_t)fixed - stage_bytes) / 4;
            if (cap > room) cap = room;
            if (cap > 4096) cap = 4096;
            const size_t smem = (size_t)stage_bytes + (fixed - 4 * (size_t)kMinPids) + 4 * (size_t)cap;
            int fits = 1;
            for (const void* kern : kerns) {
                if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
                    cudaSuccess)
                    return e;
                int resident = 0;
                if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kern, kDecThreads, smem)) !=
                    cudaSuccess)
                    return e;
                if (resident < ctas) fits = 0;
            }
            if (!fits) continue;
            plan->stages = (int)stages;
            plan->threads = kDecThreads;
            plan->pid_cap = (int)cap;
            plan->smem = smem;
            plan->grid = (int)grid;
            plan->lg_up = lg_up;
            return cudaSuccess;
        }
    }
    return cudaErrorInvalidConfiguration;
}

// Partials: two per CTA (its range's first and last segment), then one group
// merge per CTA (the group of parts ending in it), each 16 + 8 D floats.
static size_t partial_bytes(const Layout& L, int grid) {
    return (((size_t)grid * 3 * (16 + 8 * (size_t)L.D) * sizeof(float)) + 255) & ~(size_t)255;
}

// Zeroed region: two counters per CTA -- the parts counted in of the group
// ending in it, the groups counted in of the segment ending in it.
static size_t zero_bytes(int grid) { return (8 * (size_t)grid + 255) & ~(size_t)255; }

size_t decode_workspace_bytes(const Layout& L, int B, int HB, int grid) {
    (void)B;
    (void)HB;
    return partial_bytes(L, grid) + zero_bytes(grid);
}

void decode_workspace_zero_region(const Layout& L, int B, int HB, int grid, size_t* offset, size_t* bytes) {
    (void)B;
    (void)HB;
    *offset = partial_bytes(L, grid);
    *bytes = zero_bytes(grid);
}

cudaError_t launch_decode(const DecodeParams& p, const DecodePlan& plan, cudaStream_t s) {
    const void* k = decode_kernel_for(p.L.fmt, p.L.D, p.k_new != nullptr);
    if (!k) return cudaErrorInvalidValue;
    DecodeParams q = p;
    q.U = make_span(p.L, plan.lg_up);
    // cost of a segment's start, end and merge in units: about 512 tokens of
    // streaming (measured on B200 over the five decode workloads; 256 and 768
    // were both slower)
    q.seg_cost = q.U.sp >= 256 ? 2 : 512 / q.U.sp;
    void* args[] = {&q};
    // no CTA waits on another (the merges go to whoever finishes last), so a
    // plain launch: one resident wave by the plan's sizing, not by requirement
    return cudaLaunchKernel(k, dim3(plan.grid), dim3(plan.threads), args, plan.smem, s);
}

}  // namespace kvq
