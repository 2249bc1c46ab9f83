/*
 * Plain CPU oracle for blockwise codebook quantization.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the library path may include, link or
 * call this file. Only the tests, __graft_entry__.smoke() and the cpu_baseline
 * leg of bench.py use it. It shares no code, header, table or helper with the
 * CUDA library; the two agree only because both follow the same written rules.
 *
 * Built with: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * so every float operation below is one IEEE-754 binary32 operation rounded to
 * nearest-even, with no fused multiply-add and no flush of subnormals.
 *
 * Sources (the pages this follows):
 *  [P1] bitsandbytes k-bit patch series ("Add k-bit quantization kernels
 *       (K=2-5, blocksize=32)" and follow-ups):
 *         - tests/test_kbit_quantization.py quantize_kbit_ref, dequantize_kbit_ref,
 *           pack_kbit_ref, unpack_kbit_ref (the pure-PyTorch reference);
 *         - csrc/ops.cu kQuantizeBlockwise_kbit / kDequantizeBlockwise_kbit.
 *  [P2] pull request "Fuse nested 4-bit scale reconstruction on SM103",
 *       sections Summary and Implementation.
 *
 * Readings taken where the pages leave a step open:
 *  - Nearest entry: the first index i that minimises fabsf(xn - c[i]); the scan
 *    starts from +infinity (the reference's argmin), so ties go to the lowest i.
 *  - Padding of the last k-bit block: padded lanes hold 0.0f and are quantized
 *    like any other value; their bits are part of the stored words.
 *  - Nested 4-bit codes: element 2j sits in the high nibble (bits 7..4) of byte
 *    j and element 2j+1 in the low nibble.
 *  - NaN results of the float->half/bfloat16 conversions are returned as a
 *    quiet NaN with the input's sign; only the NaN class is meaningful.
 *  - E4M4 encode: floor(log2 a) is the exact floor; an infinite absmax encodes
 *    as 0xFF; at and above 32 the exponent field clamps to 15 while the
 *    mantissa is rounded in a's own binade, as the pages' steps do.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

/* dtype codes used by this oracle's own interface */
enum { ORC_F16 = 0, ORC_BF16 = 1, ORC_F32 = 2 };

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, sizeof f); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, sizeof u); return u; }

/* ------------------------------------------------------------------ */
/* Exact widening conversions                                          */
/* ------------------------------------------------------------------ */

/* IEEE binary16 -> binary32 (exact). */
float orc_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h >> 15) << 31;
    uint32_t e = (h >> 10) & 0x1f;
    uint32_t m = h & 0x3ff;
    if (e == 0x1f)                       /* inf / NaN */
        return bits_to_f32(sign | 0x7f800000u | (m << 13));
    if (e == 0) {                        /* zero / subnormal: m * 2^-24, exact */
        float mag = (float)m * 5.9604644775390625e-08f;
        return sign ? -mag : mag;
    }
    return bits_to_f32(sign | ((e - 15 + 127) << 23) | (m << 13));
}

/* bfloat16 -> binary32 (exact: the upper half of the binary32 pattern). */
float orc_bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* ------------------------------------------------------------------ */
/* Narrowing conversions, round to nearest, ties to even                */
/* ------------------------------------------------------------------ */

/* m / 2^s rounded to nearest, ties to even (s may be <= 0). */
static uint64_t rne_shift(uint64_t m, int s)
{
    if (s <= 0) return m << (-s);
    if (s >= 64) return 0;
    uint64_t q = m >> s;
    uint64_t r = m & ((1ull << s) - 1);
    uint64_t half = 1ull << (s - 1);
    if (r > half || (r == half && (q & 1))) q++;
    return q;
}

/*
 * Generic narrowing of a binary32 value to a format with `mbits` stored
 * mantissa bits, exponent bias `bias` and all-ones exponent `emax_field`.
 * The value v = man * 2^E is rounded to a multiple of the quantum 2^Q, where
 * Q = max(floor(log2|v|), 1 - bias) - mbits; the rounded multiple N gives the
 * encoding ((Q + mbits + bias - 1) << mbits) + N directly (N reaching 2^(mbits+1)
 * carries into the exponent field, and an overflow lands on infinity).
 */
static uint16_t narrow(float f, int mbits, int bias, uint32_t emax_field, uint16_t qnan)
{
    uint32_t u = f32_to_bits(f);
    uint16_t sign = (uint16_t)((u >> 31) << 15);
    uint32_t a = u & 0x7fffffffu;
    uint16_t inf = (uint16_t)(emax_field << mbits);
    if (a > 0x7f800000u) return sign | qnan;
    if (a == 0x7f800000u) return sign | inf;
    if (a == 0) return sign;
    int exp = (int)(a >> 23);
    uint64_t man = a & 0x7fffff;
    int E;                                /* v = man * 2^E */
    int e;                                /* floor(log2 v) */
    if (exp) { man |= 0x800000; E = exp - 150; e = exp - 127; }
    else {                               /* binary32 subnormal */
        E = -149;
        e = -150;
        for (uint64_t t = man; t; t >>= 1) e++;
    }
    int emin = 1 - bias;
    int Q = (e > emin ? e : emin) - mbits;
    uint64_t N = rne_shift(man, Q - E);
    uint64_t enc = ((uint64_t)(Q + mbits + bias - 1) << mbits) + N;
    if (enc >= inf) return sign | inf;
    return sign | (uint16_t)enc;
}

uint16_t orc_f32_to_f16(float f) { return narrow(f, 10, 15, 0x1f, 0x7e00); }
uint16_t orc_f32_to_bf16(float f) { return narrow(f, 7, 127, 0xff, 0x7fc0); }

void orc_f32_to_f16_array(const float* x, int64_t n, uint16_t* out)
{ for (int64_t i = 0; i < n; i++) out[i] = orc_f32_to_f16(x[i]); }
void orc_f32_to_bf16_array(const float* x, int64_t n, uint16_t* out)
{ for (int64_t i = 0; i < n; i++) out[i] = orc_f32_to_bf16(x[i]); }
void orc_f16_to_f32_array(const uint16_t* x, int64_t n, float* out)
{ for (int64_t i = 0; i < n; i++) out[i] = orc_f16_to_f32(x[i]); }

static float load_elem(const void* A, int dtype, int64_t m)
{
    if (dtype == ORC_F32) return ((const float*)A)[m];
    uint16_t h = ((const uint16_t*)A)[m];
    return dtype == ORC_F16 ? orc_f16_to_f32(h) : orc_bf16_to_f32(h);
}

static void store_elem(void* out, int dtype, int64_t m, float v)
{
    if (dtype == ORC_F32) ((float*)out)[m] = v;
    else if (dtype == ORC_F16) ((uint16_t*)out)[m] = orc_f32_to_f16(v);
    else ((uint16_t*)out)[m] = orc_f32_to_bf16(v);
}

/* ------------------------------------------------------------------ */
/* k-bit blockwise codec, blocksize 32 [P1]                             */
/* ------------------------------------------------------------------ */

#define ORC_KBIT_BS 32

/* Nearest codebook entry: first i minimising |xn - c[i]| (fp32 subtract, then abs). */
int orc_nearest_entry(float xn, const float* cb, int nentries)
{
    float best = INFINITY;
    int idx = 0;
    for (int i = 0; i < nentries; i++) {
        float dist = fabsf(xn - cb[i]);
        if (dist < best) { best = dist; idx = i; }
    }
    return idx;
}

/* Bit-plane packing: word j of a block holds bit j of element i's index at bit i. */
void orc_kbit_pack(const uint8_t* idx, int64_t n, int K, uint32_t* packed)
{
    int64_t nb = (n + ORC_KBIT_BS - 1) / ORC_KBIT_BS;
    for (int64_t b = 0; b < nb; b++)
        for (int j = 0; j < K; j++) {
            uint32_t w = 0;
            for (int i = 0; i < ORC_KBIT_BS; i++) {
                int64_t m = b * ORC_KBIT_BS + i;
                uint32_t v = m < n ? idx[m] : 0;
                w |= ((v >> j) & 1u) << i;
            }
            packed[b * K + j] = w;
        }
}

/* Inverse of orc_kbit_pack for the first n elements. */
void orc_kbit_unpack(const uint32_t* packed, int64_t n, int K, uint8_t* idx)
{
    for (int64_t m = 0; m < n; m++) {
        int64_t b = m / ORC_KBIT_BS;
        int i = (int)(m % ORC_KBIT_BS);
        uint32_t v = 0;
        for (int j = 0; j < K; j++)
            v |= ((packed[b * K + j] >> i) & 1u) << j;
        idx[m] = (uint8_t)v;
    }
}

/*
 * Quantize n elements of A (dtype) with a 2^K-entry codebook.
 * absmax[nb] receives each block's raw max |x| (padding counts as 0.0f);
 * packed[nb*K] receives the bit-plane words; idx_out (optional, nb*32 bytes)
 * receives the index chosen for every lane including the padding lanes.
 */
int orc_kbit_quantize(const void* A, int dtype, int64_t n, int K, const float* cb,
                      float* absmax, uint32_t* packed, uint8_t* idx_out)
{
    if (K < 1 || K > 8 || n <= 0) return 1;
    int nent = 1 << K;
    int64_t nb = (n + ORC_KBIT_BS - 1) / ORC_KBIT_BS;
    for (int64_t b = 0; b < nb; b++) {
        float x[ORC_KBIT_BS];
        uint8_t q[ORC_KBIT_BS];
        for (int i = 0; i < ORC_KBIT_BS; i++) {
            int64_t m = b * ORC_KBIT_BS + i;
            x[i] = m < n ? load_elem(A, dtype, m) : 0.0f;
        }
        /* block absmax with fmaxf semantics (a NaN is ignored unless all are NaN) */
        float amax = fabsf(x[0]);
        for (int i = 1; i < ORC_KBIT_BS; i++) amax = fmaxf(amax, fabsf(x[i]));
        absmax[b] = amax;
        float d = fmaxf(amax, 1e-8f);            /* divisor; the stored absmax stays raw */
        for (int i = 0; i < ORC_KBIT_BS; i++) {
            float xn = x[i] / d;                  /* IEEE division, round to nearest */
            q[i] = (uint8_t)orc_nearest_entry(xn, cb, nent);
        }
        for (int j = 0; j < K; j++) {
            uint32_t w = 0;
            for (int i = 0; i < ORC_KBIT_BS; i++) w |= ((uint32_t)(q[i] >> j) & 1u) << i;
            packed[b * K + j] = w;
        }
        if (idx_out) memcpy(idx_out + b * ORC_KBIT_BS, q, ORC_KBIT_BS);
    }
    return 0;
}

/* out[m] = T(codebook[idx_m] * absmax[m / 32]) for m < n: one fp32 multiply, one rounding to T. */
int orc_kbit_dequantize(const uint32_t* packed, const float* absmax, const float* cb,
                        int K, int64_t n, int dtype, void* out)
{
    if (K < 1 || K > 8 || n <= 0) return 1;
    for (int64_t m = 0; m < n; m++) {
        int64_t b = m / ORC_KBIT_BS;
        int i = (int)(m % ORC_KBIT_BS);
        uint32_t v = 0;
        for (int j = 0; j < K; j++) v |= ((packed[b * K + j] >> i) & 1u) << j;
        float y = cb[v] * absmax[b];
        store_elem(out, dtype, m, y);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* E4M4 uint8 absmax [P1 PATCH 005 "Add vectorized dequant kernel and   */
/* E4M4 uint8 absmax support": encode_absmax_e4m4, decode_absmax_e4m4,  */
/* decode_e4m4_absmax]                                                  */
/* ------------------------------------------------------------------ */

#define ORC_E4M4_BIAS 11

/*
 * Decode: e = code >> 4, m = code & 15. e > 0: 2^(e - bias) * (1 + m/16);
 * e == 0: 2^(1 - bias) * (m/16) (IEEE-style subnormals, code 0 is 0.0).
 * Every such value is exact in binary32 (computed here as an integer times a
 * power of two in double, then narrowed without rounding).
 */
float orc_e4m4_decode(uint8_t code)
{
    int e = code >> 4, m = code & 15;
    if (e == 0) return (float)ldexp((double)m, 1 - ORC_E4M4_BIAS - 4);
    return (float)ldexp((double)(16 + m), e - ORC_E4M4_BIAS - 4);
}

/*
 * Encode, following the pages' steps in order:
 *   values that are not > 0 encode as 0 (this covers 0, negatives and NaN);
 *   e_unb = floor(log2(a));  e_biased = clamp(e_unb + bias, 0, 15);
 *   if e_unb + bias <= 0 (subnormal): e_biased = 0, m = round(a / 2^(1-bias) * 16);
 *   else m = round((a / 2^e_unb - 1) * 16) with the unclamped e_unb;
 *   m is clamped to [0, 15]; code = e_biased << 4 | m.
 * round() is round-half-to-even (torch.round). Readings: floor(log2 a) is the
 * exact floor (frexp), not a rounded fp32 logarithm; an infinite absmax
 * encodes as the largest code 0xFF. All arithmetic below is exact in double.
 */
uint8_t orc_e4m4_encode(float a)
{
    if (!(a > 0.0f)) return 0;
    if (isinf(a)) return 0xFF;
    int ex;
    (void)frexp((double)a, &ex);          /* a = f * 2^ex, f in [0.5, 1) */
    int e_unb = ex - 1;                   /* floor(log2 a) */
    int e_biased = e_unb + ORC_E4M4_BIAS;
    double m_real;
    if (e_biased <= 0) {
        e_biased = 0;
        m_real = ldexp((double)a, -(1 - ORC_E4M4_BIAS)) * 16.0;
    } else {
        if (e_biased > 15) e_biased = 15;
        m_real = (ldexp((double)a, -e_unb) - 1.0) * 16.0;
    }
    double m = nearbyint(m_real);         /* default rounding mode: to nearest, ties to even */
    if (m < 0.0) m = 0.0;
    if (m > 15.0) m = 15.0;
    return (uint8_t)((e_biased << 4) | (int)m);
}

void orc_e4m4_encode_array(const float* a, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_e4m4_encode(a[i]);
}

void orc_e4m4_decode_array(const uint8_t* c, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_e4m4_decode(c[i]);
}

/* ------------------------------------------------------------------ */
/* Nested 4-bit dequantization [P2]                                     */
/* ------------------------------------------------------------------ */

/* Outer-block scale: General8 code times the inner absmax, then plus the offset, each rounded. */
float orc_nested_scale(float code2_val, float absmax2_val, float offset)
{
    float prod = code2_val * absmax2_val;
    float s = prod + offset;
    return s;
}

/*
 * out[m] = T(code4[nib_m] * scale_{m / bs}) with
 * scale_b = (code2[absmax_q[b]] * absmax2[b / bs2]) + offset.
 */
int orc_nested_dequantize(const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                          const float* absmax2, float offset, const float* code4,
                          int64_t n, int64_t bs, int64_t bs2, int dtype, void* out)
{
    if (n <= 0 || bs <= 0 || bs2 <= 0) return 1;
    for (int64_t m = 0; m < n; m++) {
        uint8_t byte = codes[m / 2];
        unsigned nib = (m % 2 == 0) ? (unsigned)(byte >> 4) : (unsigned)(byte & 0x0f);
        int64_t b = m / bs;
        float s = orc_nested_scale(code2[absmax_q[b]], absmax2[b / bs2], offset);
        float y = code4[nib] * s;
        store_elem(out, dtype, m, y);
    }
    return 0;
}

/* Plain 4-bit dequantization with an fp32 absmax per block [P2, the last launch of the
 * unfused path]: out[m] = T(code4[nib_m] * absmax[m / bs]); same nibble order. */
int orc_dequantize_4bit(const uint8_t* codes, const float* absmax, const float* code4,
                        int64_t n, int64_t bs, int dtype, void* out)
{
    if (n <= 0 || bs <= 0) return 1;
    for (int64_t m = 0; m < n; m++) {
        uint8_t byte = codes[m / 2];
        unsigned nib = (m % 2 == 0) ? (unsigned)(byte >> 4) : (unsigned)(byte & 0x0f);
        float y = code4[nib] * absmax[m / bs];
        store_elem(out, dtype, m, y);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* 4-bit quantize and nested absmax compression: the inverse of the     */
/* nested dequant. [P2] gives only the decode and leaves the stored     */
/* formats as they were, so every step below is a reading: the k-bit    */
/* rule of [P1] applied per outer block, the offset as a mean of the    */
/* outer absmax, General8 codes of the centred absmax per group of      */
/* blocksize2 outer blocks.                                             */
/* ------------------------------------------------------------------ */

/*
 * Per outer block b of bs elements: absmax[b] = max |x| (raw, an fmaxf fold from
 * the first element, so NaN only when every element is NaN); d = fmaxf(absmax,
 * 1e-8f); code of element m = first i minimising fabsf(x_m / d - code4[i]) (IEEE
 * fp32 division, as the k-bit codec). Codes are packed two per byte, element 2j
 * in the high nibble of codes[j]; for odd n the last low nibble is 0.
 */
int orc_quantize_4bit(const void* A, int dtype, int64_t n, int64_t bs, const float* code4,
                      float* absmax, uint8_t* codes)
{
    if (n <= 0 || bs <= 0) return 1;
    memset(codes, 0, (size_t)((n + 1) / 2));
    int64_t nbo = (n + bs - 1) / bs;
    for (int64_t b = 0; b < nbo; b++) {
        int64_t lo = b * bs, hi = lo + bs < n ? lo + bs : n;
        float amax = fabsf(load_elem(A, dtype, lo));
        for (int64_t m = lo + 1; m < hi; m++) amax = fmaxf(amax, fabsf(load_elem(A, dtype, m)));
        absmax[b] = amax;
        float d = fmaxf(amax, 1e-8f);
        for (int64_t m = lo; m < hi; m++) {
            unsigned idx = (unsigned)orc_nearest_entry(load_elem(A, dtype, m) / d, code4, 16);
            codes[m / 2] |= (uint8_t)((m % 2 == 0) ? idx << 4 : idx);
        }
    }
    return 0;
}

/* Pairwise binary64 sum of a[lo .. lo+len) (len a power of two), entries at or beyond n
 * counting as 0.0: the sum of the lower half plus the sum of the upper half. */
static double orc_tree_sum(const float* a, int64_t n, int64_t lo, int64_t len)
{
    if (lo >= n) return 0.0;
    if (len == 1) return (double)a[lo];
    int64_t h = len / 2;
    return orc_tree_sum(a, n, lo, h) + orc_tree_sum(a, n, lo + h, h);
}

/*
 * The nested offset: the mean of the nbo outer absmax values, summed in binary64 by a
 * fixed binary tree (the values zero-padded to the next power of two, each node the sum
 * of its two halves), divided by nbo in binary64 and rounded once to binary32.
 */
float orc_absmax_offset(const float* absmax, int64_t nbo)
{
    int64_t p = 1;
    while (p < nbo) p <<= 1;
    return (float)(orc_tree_sum(absmax, nbo, 0, p) / (double)nbo);
}

/*
 * General8 compression of the outer absmax, per group g of bs2 outer blocks:
 * c_b = fl(absmax[b] - offset); absmax2[g] = max |c_b| over the group (fmaxf fold);
 * absmax_q[b] = first i minimising fabsf(c_b / fmaxf(absmax2[g], 1e-8f) - code2[i])
 * over the 256 entries. The nested dequant rebuilds fl(fl(code2[q] * absmax2) + offset).
 */
int orc_quantize_absmax_nested(const float* absmax, int64_t nbo, float offset, const float* code2,
                               int64_t bs2, uint8_t* absmax_q, float* absmax2)
{
    if (nbo <= 0 || bs2 <= 0) return 1;
    int64_t nbi = (nbo + bs2 - 1) / bs2;
    for (int64_t g = 0; g < nbi; g++) {
        int64_t lo = g * bs2, hi = lo + bs2 < nbo ? lo + bs2 : nbo;
        float m = fabsf(absmax[lo] - offset);
        for (int64_t b = lo + 1; b < hi; b++) m = fmaxf(m, fabsf(absmax[b] - offset));
        absmax2[g] = m;
        float d = fmaxf(m, 1e-8f);
        for (int64_t b = lo; b < hi; b++)
            absmax_q[b] = (uint8_t)orc_nearest_entry((absmax[b] - offset) / d, code2, 256);
    }
    return 0;
}
