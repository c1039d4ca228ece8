/*
 * kvq_oracle.c -- plain, slow CPU oracle for the quantized paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only tests/, __graft_entry__.smoke() and the cpu_baseline
 * leg of bench.py use it.  It shares no source with the CUDA library
 * (quantized_paged_kv_03_b200/csrc); the two are written independently from
 * the same page text so that agreement between them means something.
 *
 * Sources (pages, cited by title and section):
 *   [NInfer]     "NInfer KV Cache 量化指南：BF16、INT8、FP8、NVFP4 与 K8V4 五种格式怎么选"
 *                -- per-token byte table ("五种格式的每个 token ... 物理开销对比") and
 *                   the format paragraphs ("五种格式逐个认识").
 *   [TokenSpeed] "TokenSpeed量化实战：fp8、NVFP4与KV缓存压缩如何省下50%显存"
 *                -- table under "KV缓存压缩 --kv-cache-dtype" (fp8_e4m3 unit scale,
 *                   mxfp8 = one UE8M0 scale per 32 head_dim elements).
 *   [FP8-KV]     "FP8 KV Cache如何提速 ... 长上下文推理的加速秘密"
 *                -- kv_cache_scheme {8-bit float, strategy tensor, symmetric}.
 *
 * Readings where the pages are silent (each repeated where it is used):
 *   R1  Hadamard-256 = Sylvester order, no random signs, normalised by 1/16,
 *       evaluated in fp32 as ascending butterfly stages h = 1,2,...,128 with
 *       (a+b, a-b) per pair, then x16^-1.  The butterfly order fixes the bits.
 *   R2  Scales are rounded to nearest-even in their own format and the codes
 *       are computed by dividing by the DECODED scale (IEEE fp32 division).
 *   R3  A group whose decoded scale is 0 stores all codes +0.
 *   R4  fp16 and e4m3/e2m1 encoders saturate at their largest finite value;
 *       the sign of zero is kept.
 *   R5  int8 is symmetric: round-to-nearest-even, clamp to [-127, 127].
 *   R6  NVFP4 carries no second-level (per-tensor) scale: 288 B/token leaves
 *       no room for one (2 x (128 + 16) = 288).
 *   R7  Two E2M1 codes per byte, the lower element index in the low nibble.
 *   R8  MXFP8 scale = 2^(floor(log2 amax) - 8), exponent clamped to
 *       [-127, 127], byte = exponent + 127; amax = 0 gives byte 0 and +0 codes.
 *   R9  K8V4: K is FP8-E4M3 row-256 (not rotated), V is NVFP4-G16 rotated.
 *  R10  BF16 format: K is the bf16 bit pattern, V is fp16 (RNE, saturating).
 *  R11  MLA latent cache (or_mla_attend): one row of DC + DR values per token
 *       (DeepSeek-V2 report: DC = 512 latent, DR = 64 rotary key), shared by
 *       every query head, attended in the absorbed form; the value is the
 *       latent part of the same row.  FP8 storage is the per-tensor format of
 *       [TokenSpeed]'s fp8 switch applied to the whole row (576 B per token
 *       against 1152 B in BF16: the table's 0.5x).
 *
 * Parity unpinned: every function below is pinned by value (tests/
 * test_oracle_pins.py: closed forms, brute force over the format grids,
 * library routines), but the bit-level choices of R1 (butterfly order), R2
 * (rounding direction of a scale), R3 (zero scale) and R7 (nibble order) are
 * readings no page fixes; the CUDA path agrees with them because it follows
 * the same readings, not because the pages confirm them.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* Format ids: the same numbering as the public header, restated here. */
enum { OR_BF16 = 0, OR_FP8_ROW256 = 1, OR_INT8_G64 = 2, OR_NVFP4_G16 = 3,
       OR_K8V4 = 4, OR_MXFP8_G32 = 5, OR_FP8_TENSOR = 6 };
enum { OR_FLAG_NO_ROTATE = 1u };

/* Element codecs, used by or_encode(). */
enum { OR_CODE_E4M3 = 0, OR_CODE_E2M1 = 1, OR_CODE_INT8 = 2, OR_CODE_FP16 = 3,
       OR_CODE_UE4M3 = 4 };

/* Per-tensor "kinds" of a stored row. */
enum { KIND_BF16RAW, KIND_FP16, KIND_E4M3_ROW256, KIND_INT8_G64, KIND_E2M1_G16,
       KIND_E4M3_MX32, KIND_E4M3_TENSOR };

static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* ---------------------------------------------------------------- floats */

/* Nearest value (ties to an even significand) on the grid of a binary float
 * format with `mbits` stored significand bits and minimum normal exponent
 * `emin`; subnormals below 2^emin.  `a` is a non-negative finite double that
 * came from an fp32, so every step below is exact in double. */
static double round_grid(double a, int mbits, int emin)
{
    if (a == 0.0) return 0.0;
    int e;
    (void)frexp(a, &e);          /* a = f * 2^e, f in [0.5, 1) */
    int E = e - 1;               /* floor(log2 a) */
    if (E < emin) E = emin;      /* subnormal range shares the quantum of 2^emin */
    double quantum = ldexp(1.0, E - mbits);
    double n = rint(a / quantum); /* default rounding mode: to nearest, ties to even */
    return n * quantum;
}

/* Bits of a representable magnitude `m` in a format with `mbits`, `emin`, `bias`. */
static uint32_t grid_bits(double m, int mbits, int emin, int bias)
{
    if (m == 0.0) return 0;
    int e;
    (void)frexp(m, &e);
    int E = e - 1;
    if (E < emin) {              /* subnormal: exponent field 0 */
        return (uint32_t)(m / ldexp(1.0, emin - mbits));
    }
    uint32_t mant = (uint32_t)(m / ldexp(1.0, E - mbits)) - (1u << mbits);
    return ((uint32_t)(E + bias) << mbits) | mant;
}

/* IEEE binary16, round to nearest even, saturating at 65504 (R4). */
uint16_t or_f32_to_f16(float x)
{
    uint32_t s = f2u(x) >> 31;
    double a = fabs((double)x);
    double m = isinf(a) ? 65504.0 : round_grid(a, 10, -14);
    if (m > 65504.0) m = 65504.0;
    return (uint16_t)((s << 15) | grid_bits(m, 10, -14, 15));
}

double or_f16_to_f64(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double v = (e == 0) ? ldexp((double)f, -24) : ldexp(1024.0 + f, e - 25);
    return s ? -v : v;
}

/* OCP FP8 E4M3 ("fn": no infinities, 0x7F/0xFF are NaN), max 448, RNE,
 * saturating (R4).  [NInfer] FP8 paragraph; [TokenSpeed] fp8_e4m3. */
uint8_t or_f32_to_e4m3(float x)
{
    uint32_t s = f2u(x) >> 31;
    double a = fabs((double)x);
    double m = isinf(a) ? 448.0 : round_grid(a, 3, -6);
    if (m > 448.0) m = 448.0;
    return (uint8_t)((s << 7) | grid_bits(m, 3, -6, 7));
}

double or_e4m3_to_f64(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, f = c & 7;
    double v = (e == 0) ? ldexp((double)f, -9) : ldexp(8.0 + f, e - 10);
    return s ? -v : v;
}

/* FP4 E2M1: magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, RNE on the code's last
 * bit, saturating at 6 (R4).  Returns a nibble.  [NInfer] NVFP4 paragraph. */
uint8_t or_f32_to_e2m1(float x)
{
    uint32_t s = f2u(x) >> 31;
    double a = fabs((double)x);
    double m = isinf(a) ? 6.0 : round_grid(a, 1, 0);
    if (m > 6.0) m = 6.0;
    return (uint8_t)((s << 3) | grid_bits(m, 1, 0, 1));
}

double or_e2m1_to_f64(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, f = c & 1;
    double v = (e == 0) ? 0.5 * f : ldexp(2.0 + f, e - 2);
    return s ? -v : v;
}

/* UE4M3: E4M3 restricted to non-negative inputs (the NVFP4 scale byte). */
uint8_t or_f32_to_ue4m3(float x)
{
    return (uint8_t)(or_f32_to_e4m3(x) & 0x7F);
}

/* Symmetric int8 (R5). */
int8_t or_f32_to_int8(float x)
{
    double r = rint((double)x);
    if (r > 127.0) r = 127.0;
    if (r < -127.0) r = -127.0;
    return (int8_t)r;
}

/* MX shared exponent of a group (R8). */
int or_mx_exponent(float amax)
{
    if (!(amax > 0.0f)) return -127;
    int e;
    (void)frexp((double)amax, &e);
    int E = (e - 1) - 8;          /* 8 = exponent of E4M3's largest normal, 448 = 1.75 * 2^8 */
    if (E < -127) E = -127;
    if (E > 127) E = 127;
    return E;
}

/* Element-wise encoder used by the exhaustive tests: codes of x[i]. */
void or_encode(int code, const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++) {
        float v = x[i];
        switch (code) {
        case OR_CODE_E4M3: out[i] = or_f32_to_e4m3(v); break;
        case OR_CODE_E2M1: out[i] = or_f32_to_e2m1(v); break;
        case OR_CODE_INT8: out[i] = (uint8_t)or_f32_to_int8(v); break;
        case OR_CODE_UE4M3: out[i] = or_f32_to_ue4m3(v); break;
        case OR_CODE_FP16: {
            uint16_t h = or_f32_to_f16(v);
            out[2 * i] = (uint8_t)(h & 0xFF);
            out[2 * i + 1] = (uint8_t)(h >> 8);
        } break;
        default: break;
        }
    }
}

/* The same encoders over consecutive fp32 bit patterns [start, start+n). */
void or_encode_bits(int code, uint32_t start, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++) {
        float v = u2f(start + (uint32_t)i);
        or_encode(code, &v, 1, code == OR_CODE_FP16 ? out + 2 * i : out + i);
    }
}

/* --------------------------------------------------------------- Hadamard */

/* Normalised Hadamard-256 in fp32, R1.  [NInfer] INT8 / NVFP4 paragraphs:
 * a normalised 256-dimensional Hadamard as preprocessing before quantising. */
void or_fwht256(float* x)
{
    for (int h = 1; h < 256; h <<= 1)
        for (int i = 0; i < 256; i++)
            if (!(i & h)) {
                float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
    for (int i = 0; i < 256; i++) x[i] *= 0.0625f;
}

/* Entry (i, j) of the normalised Sylvester Hadamard matrix of order n (a power
 * of two): (-1)^popcount(i & j) / sqrt(n).  Used in fp64 by or_attend(). */
double or_hadamard_entry(int n, int i, int j)
{
    int p = 0;
    for (unsigned v = (unsigned)(i & j); v; v &= v - 1) p++;
    return ((p & 1) ? -1.0 : 1.0) / sqrt((double)n);
}

/* --------------------------------------------------------- stored rows */

/* What one row (one token, one kv-head, K or V) of each format stores. */
static int row_kind(int fmt, int is_v)
{
    switch (fmt) {
    case OR_BF16: return is_v ? KIND_FP16 : KIND_BF16RAW;            /* R10 */
    case OR_FP8_ROW256: return KIND_E4M3_ROW256;
    case OR_INT8_G64: return KIND_INT8_G64;
    case OR_NVFP4_G16: return KIND_E2M1_G16;
    case OR_K8V4: return is_v ? KIND_E2M1_G16 : KIND_E4M3_ROW256;     /* R9 */
    case OR_MXFP8_G32: return KIND_E4M3_MX32;
    case OR_FP8_TENSOR: return KIND_E4M3_TENSOR;
    default: return -1;
    }
}

/* Which tensors are rotated before quantising.  [NInfer]: INT8 rotates K,
 * NVFP4 rotates K and V; K8V4's V is NVFP4 and rotated (R9). */
int or_is_rotated(int fmt, int is_v, unsigned flags)
{
    if (flags & OR_FLAG_NO_ROTATE) return 0;
    switch (fmt) {
    case OR_INT8_G64: return !is_v;
    case OR_NVFP4_G16: return 1;
    case OR_K8V4: return is_v;
    default: return 0;
    }
}

/* Bytes per stored row: codes and scales.  Returns -1 for an invalid pair.
 * [NInfer] table at D=256: BF16 512+512, INT8-G64 264+264, FP8 258+258,
 * NVFP4 144+144, K8V4 258+144. */
int or_row_bytes(int fmt, int is_v, int D, int* code_bytes, int* scale_bytes)
{
    int k = row_kind(fmt, is_v);
    int cb = -1, sb = -1;
    switch (k) {
    case KIND_BF16RAW: case KIND_FP16: cb = 2 * D; sb = 0; break;
    case KIND_E4M3_ROW256: if (D % 256 == 0) { cb = D; sb = 2 * (D / 256); } break;
    case KIND_INT8_G64: if (D % 64 == 0) { cb = D; sb = 2 * (D / 64); } break;
    case KIND_E2M1_G16: if (D % 16 == 0) { cb = D / 2; sb = D / 16; } break;
    case KIND_E4M3_MX32: if (D % 32 == 0) { cb = D; sb = D / 32; } break;
    case KIND_E4M3_TENSOR: cb = D; sb = 0; break;
    default: break;
    }
    if (cb < 0) return -1;
    if (code_bytes) *code_bytes = cb;
    if (scale_bytes) *scale_bytes = sb;
    return 0;
}

static float amax_of(const float* y, int n)
{
    float m = 0.0f;
    for (int i = 0; i < n; i++) {
        float a = fabsf(y[i]);
        if (a > m) m = a;
    }
    return m;
}

/* Quantise one bf16 row of length D (append steps A2..A5).  Writes the row's
 * codes and scales in logical order: element i of the row at code index i,
 * group g's scale at scale index g (little-endian for 2-byte scales). */
int or_quantize_row(int fmt, int is_v, unsigned flags, float tensor_scale, int D,
                    const uint16_t* x_bf16, uint8_t* codes, uint8_t* scales)
{
    int k = row_kind(fmt, is_v);
    if (k < 0 || or_row_bytes(fmt, is_v, D, 0, 0) < 0) return -1;
    float y[4096];
    if (D > 4096) return -1;
    for (int i = 0; i < D; i++) y[i] = u2f((uint32_t)x_bf16[i] << 16);   /* bf16 -> fp32 is exact */
    if (or_is_rotated(fmt, is_v, flags)) {
        if (D != 256) return -1;
        or_fwht256(y);
    }
    switch (k) {
    case KIND_BF16RAW:
        for (int i = 0; i < D; i++) { codes[2 * i] = (uint8_t)x_bf16[i]; codes[2 * i + 1] = (uint8_t)(x_bf16[i] >> 8); }
        break;
    case KIND_FP16:
        for (int i = 0; i < D; i++) {
            uint16_t h = or_f32_to_f16(y[i]);
            codes[2 * i] = (uint8_t)h; codes[2 * i + 1] = (uint8_t)(h >> 8);
        }
        break;
    case KIND_E4M3_ROW256: case KIND_INT8_G64: {
        int G = (k == KIND_E4M3_ROW256) ? 256 : 64;
        float qmax = (k == KIND_E4M3_ROW256) ? 448.0f : 127.0f;
        for (int g = 0; g < D / G; g++) {
            const float* yg = y + g * G;
            uint16_t sbits = or_f32_to_f16(amax_of(yg, G) / qmax);   /* R2 */
            float s = (float)or_f16_to_f64(sbits);
            scales[2 * g] = (uint8_t)sbits; scales[2 * g + 1] = (uint8_t)(sbits >> 8);
            for (int i = 0; i < G; i++) {
                uint8_t c = 0;                                        /* R3 */
                if (s != 0.0f) {
                    float t = yg[i] / s;
                    c = (k == KIND_E4M3_ROW256) ? or_f32_to_e4m3(t) : (uint8_t)or_f32_to_int8(t);
                }
                codes[g * G + i] = c;
            }
        }
    } break;
    case KIND_E2M1_G16:
        memset(codes, 0, (size_t)D / 2);
        for (int g = 0; g < D / 16; g++) {
            const float* yg = y + g * 16;
            uint8_t sb = or_f32_to_ue4m3(amax_of(yg, 16) / 6.0f);   /* R2, R6 */
            float s = (float)or_e4m3_to_f64(sb);
            scales[g] = sb;
            for (int i = 0; i < 16; i++) {
                uint8_t c = (s != 0.0f) ? or_f32_to_e2m1(yg[i] / s) : 0;
                int idx = g * 16 + i;
                codes[idx / 2] |= (uint8_t)(c << ((idx & 1) ? 4 : 0));  /* R7 */
            }
        }
        break;
    case KIND_E4M3_MX32:
        for (int g = 0; g < D / 32; g++) {
            const float* yg = y + g * 32;
            float amax = amax_of(yg, 32);
            int E = or_mx_exponent(amax);                                /* R8 */
            scales[g] = (amax > 0.0f) ? (uint8_t)(E + 127) : 0;
            float inv = (float)ldexp(1.0, -E);
            for (int i = 0; i < 32; i++)
                codes[g * 32 + i] = (amax > 0.0f) ? or_f32_to_e4m3(yg[i] * inv) : 0;
        }
        break;
    case KIND_E4M3_TENSOR:
        /* [FP8-KV]: one symmetric scale for the whole tensor; [TokenSpeed]
         * fp8_e4m3 is the special case scale = 1. */
        for (int i = 0; i < D; i++) codes[i] = or_f32_to_e4m3(y[i] / tensor_scale);
        break;
    default: return -1;
    }
    return 0;
}

/* Decode one stored row to fp64 values in the stored (rotated) domain:
 * code x decoded scale (exact). */
int or_dequant_row(int fmt, int is_v, float tensor_scale, int D,
                   const uint8_t* codes, const uint8_t* scales, double* out)
{
    int k = row_kind(fmt, is_v);
    if (k < 0 || or_row_bytes(fmt, is_v, D, 0, 0) < 0) return -1;
    switch (k) {
    case KIND_BF16RAW:
        for (int i = 0; i < D; i++)
            out[i] = (double)u2f(((uint32_t)codes[2 * i] | ((uint32_t)codes[2 * i + 1] << 8)) << 16);
        break;
    case KIND_FP16:
        for (int i = 0; i < D; i++)
            out[i] = or_f16_to_f64((uint16_t)(codes[2 * i] | (codes[2 * i + 1] << 8)));
        break;
    case KIND_E4M3_ROW256: case KIND_INT8_G64: {
        int G = (k == KIND_E4M3_ROW256) ? 256 : 64;
        for (int i = 0; i < D; i++) {
            int g = i / G;
            double s = or_f16_to_f64((uint16_t)(scales[2 * g] | (scales[2 * g + 1] << 8)));
            double c = (k == KIND_E4M3_ROW256) ? or_e4m3_to_f64(codes[i]) : (double)(int8_t)codes[i];
            out[i] = c * s;
        }
    } break;
    case KIND_E2M1_G16:
        for (int i = 0; i < D; i++) {
            uint8_t c = (uint8_t)((codes[i / 2] >> ((i & 1) ? 4 : 0)) & 0xF);
            out[i] = or_e2m1_to_f64(c) * or_e4m3_to_f64(scales[i / 16]);
        }
        break;
    case KIND_E4M3_MX32:
        for (int i = 0; i < D; i++) {
            int b = scales[i / 32];
            out[i] = or_e4m3_to_f64(codes[i]) * ldexp(1.0, b - 127);
        }
        break;
    case KIND_E4M3_TENSOR:
        for (int i = 0; i < D; i++) out[i] = or_e4m3_to_f64(codes[i]) * (double)tensor_scale;
        break;
    default: return -1;
    }
    return 0;
}

/* Many rows at once (rows are independent). */
int or_quantize_rows(int fmt, int is_v, unsigned flags, float tensor_scale, int D, int64_t n,
                     const uint16_t* x, uint8_t* codes, uint8_t* scales)
{
    int cb, sb;
    if (or_row_bytes(fmt, is_v, D, &cb, &sb) < 0) return -1;
    for (int64_t r = 0; r < n; r++)
        if (or_quantize_row(fmt, is_v, flags, tensor_scale, D, x + r * D, codes + r * cb,
                            sb ? scales + r * sb : scales) < 0)
            return -1;
    return 0;
}

int or_dequant_rows(int fmt, int is_v, float tensor_scale, int D, int64_t n,
                    const uint8_t* codes, const uint8_t* scales, double* out)
{
    int cb, sb;
    if (or_row_bytes(fmt, is_v, D, &cb, &sb) < 0) return -1;
    for (int64_t r = 0; r < n; r++)
        if (or_dequant_row(fmt, is_v, tensor_scale, D, codes + r * cb, sb ? scales + r * sb : scales,
                           out + r * D) < 0)
            return -1;
    return 0;
}

/* --------------------------------------------------------------- attention */

/* Decode attention for G query heads that share one kv-head, in fp64, over L
 * dequantised cache rows (stored domain).  Plain definition:
 *   q' = H q if K was rotated (H orthonormal, so q.k = (Hq).(Hk));
 *   s_t = scale * q' . k_t;  p = softmax(s);  o = sum_t p_t v_t;
 *   o <- H o if V was rotated (H is symmetric and its own inverse).
 * q: [G][D] values; k, v: [L][D]; out: [G][D].  Returns -1 on bad sizes. */
int or_attend(int D, int64_t L, int G, const double* q, int k_rot, int v_rot,
              const double* k, const double* v, double scale, double* out)
{
    if (L <= 0 || D <= 0 || D > 4096 || G <= 0) return -1;
    if ((k_rot || v_rot) && D != 256) return -1;
    double qr[4096], acc[4096];
    for (int g = 0; g < G; g++) {
        const double* qg = q + (int64_t)g * D;
        for (int i = 0; i < D; i++) {
            if (k_rot) {
                double t = 0.0;
                for (int j = 0; j < D; j++) t += or_hadamard_entry(D, i, j) * qg[j];
                qr[i] = t;
            } else {
                qr[i] = qg[i];
            }
        }
        double m = -INFINITY;
        /* two passes over the rows: max, then sum of exponentials */
        for (int64_t t = 0; t < L; t++) {
            double d = 0.0;
            for (int i = 0; i < D; i++) d += qr[i] * k[t * D + i];
            d *= scale;
            if (d > m) m = d;
        }
        double l = 0.0;
        for (int i = 0; i < D; i++) acc[i] = 0.0;
        for (int64_t t = 0; t < L; t++) {
            double d = 0.0;
            for (int i = 0; i < D; i++) d += qr[i] * k[t * D + i];
            double p = exp(d * scale - m);
            l += p;
            for (int i = 0; i < D; i++) acc[i] += p * v[t * D + i];
        }
        double* og = out + (int64_t)g * D;
        for (int i = 0; i < D; i++) acc[i] /= l;
        for (int i = 0; i < D; i++) {
            if (v_rot) {
                double t = 0.0;
                for (int j = 0; j < D; j++) t += or_hadamard_entry(D, i, j) * acc[j];
                og[i] = t;
            } else {
                og[i] = acc[i];
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------ MLA latent decode */

/* Decode attention over a multi-head latent attention (MLA) cache, in fp64,
 * absorbed form.  [TokenSpeed] recipe section (Kimi K2.5 served with
 * --attention-backend trtllm_mla and --kv-cache-dtype fp8) and the GLM 8xB200
 * deployment page (DSA+MLA) name the method; its shape comes from the
 * DeepSeek-V2 report, section "Multi-Head Latent Attention" (R11).
 * One cached row per token serves every query head: DC latent values c_t
 * (the compressed key-value, which is also the value) followed by DR values
 * r_t (the decoupled rotary key, shared by the heads).  A head's query row is
 * (q_lat, q_rope), q_lat = W_UK^T q_nope already carrying the key
 * up-projection, so that q_lat . c_t = q_nope . (W_UK c_t):
 *   s_t = scale * (q_lat . c_t + q_rope . r_t);  p = softmax(s);
 *   o = sum_t p_t c_t   (the latent output; W_UV is applied after attention).
 * q: [G][DC + DR]; kv: [L][DC + DR]; out: [G][DC].  Returns -1 on bad sizes. */
int or_mla_attend(int DC, int DR, int64_t L, int G, const double* q, const double* kv,
                  double scale, double* out)
{
    if (L <= 0 || DC <= 0 || DR < 0 || DC + DR > 4096 || G <= 0) return -1;
    const int W = DC + DR;
    double acc[4096];
    for (int g = 0; g < G; g++) {
        const double* qg = q + (int64_t)g * W;
        double m = -INFINITY;
        for (int64_t t = 0; t < L; t++) {
            const double* row = kv + t * W;
            double lat = 0.0, rope = 0.0;
            for (int i = 0; i < DC; i++) lat += qg[i] * row[i];
            for (int i = 0; i < DR; i++) rope += qg[DC + i] * row[DC + i];
            double s = scale * (lat + rope);
            if (s > m) m = s;
        }
        double l = 0.0;
        for (int i = 0; i < DC; i++) acc[i] = 0.0;
        for (int64_t t = 0; t < L; t++) {
            const double* row = kv + t * W;
            double lat = 0.0, rope = 0.0;
            for (int i = 0; i < DC; i++) lat += qg[i] * row[i];
            for (int i = 0; i < DR; i++) rope += qg[DC + i] * row[DC + i];
            double p = exp(scale * (lat + rope) - m);
            l += p;
            for (int i = 0; i < DC; i++) acc[i] += p * row[i];
        }
        double* og = out + (int64_t)g * DC;
        for (int i = 0; i < DC; i++) og[i] = acc[i] / l;
    }
    return 0;
}
