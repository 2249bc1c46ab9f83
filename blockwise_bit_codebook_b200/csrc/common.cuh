// Device helpers shared by the library's kernels (sm_100a only).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace bbc {

enum DType : int { F16 = 0, BF16 = 1, F32 = 2 };

__host__ __device__ constexpr int dtype_size(int dt) { return dt == F32 ? 4 : 2; }

// ---- programmatic dependent launch (a no-op for a kernel launched without the attribute) ----

// Waits until the grid this one follows in the stream has completed and its writes are visible.
// Kernels call it before their first global access. They do not trigger their dependents early:
// the trigger is implicit when each CTA exits (an early trigger let the next launches' CTAs sit
// waiting on SMs that short launches left free, and slowed them: c1 dequant 1.7 -> 2.9 us).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---- 128/256-bit streaming global accesses -------------------------------

// Read-only, not kept in L1: every input byte is used exactly once.
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

struct u32x8 { uint32_t v[8]; };

// 256-bit read of data used once (the quantize kernels' input): not kept in L1, and marked first
// for eviction in L2, so that the small tables read by every CTA (codebooks) and the lines
// written by the kernel stay there (c2 fp32 quantize: 66 -> 77-82 % of HBM; 16-bit +1-3 points).
__device__ __forceinline__ u32x8 ldg_stream_v8(const void* p) {
    u32x8 r;
    asm volatile("{ .reg .b64 pol;\n"
                 "createpolicy.fractional.L2::evict_first.b64 pol, 1.0;\n"
                 "ld.global.nc.L1::no_allocate.L2::cache_hint.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], pol; }"
                 : "=r"(r.v[0]), "=r"(r.v[1]), "=r"(r.v[2]), "=r"(r.v[3]),
                   "=r"(r.v[4]), "=r"(r.v[5]), "=r"(r.v[6]), "=r"(r.v[7])
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint2 ldg_stream_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ void stg_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" :: "l"(p), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__device__ __forceinline__ void stg_v8(void* p, const uint32_t* v) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :: "l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]),
                    "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]) : "memory");
}

// ---- conversions ----------------------------------------------------------

// Two fp32 -> packed pair, round to nearest even; `lo` lands at the lower address.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ uint16_t f32_to_f16_bits(float x) {
    uint16_t r;
    asm("cvt.rn.f16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h16) { return __uint_as_float(h16 << 16); }
__device__ __forceinline__ float f16_bits_to_f32(uint32_t h16) {
    float f;
    asm("{ .reg .f16 h; mov.b16 h, %1; cvt.f32.f16 %0, h; }" : "=f"(f) : "h"((uint16_t)h16));
    return f;
}

// Store an fp32 value as element m of a typed array (one rounding to the type).
template <int DT>
__device__ __forceinline__ void store_from_f32(void* out, int64_t m, float v) {
    if constexpr (DT == F32) reinterpret_cast<float*>(out)[m] = v;
    else if constexpr (DT == BF16) reinterpret_cast<uint16_t*>(out)[m] = f32_to_bf16_bits(v);
    else reinterpret_cast<uint16_t*>(out)[m] = f32_to_f16_bits(v);
}

// Pack 8 fp32 values (memory order) of type DT into out_words (4 words for 16-bit, 8 for fp32).
template <int DT>
__device__ __forceinline__ void pack8(const float* y, uint32_t* w) {
    if constexpr (DT == F32) {
#pragma unroll
        for (int i = 0; i < 8; i++) w[i] = __float_as_uint(y[i]);
    } else {
#pragma unroll
        for (int i = 0; i < 4; i++)
            w[i] = DT == BF16 ? pack_bf16x2(y[2 * i], y[2 * i + 1]) : pack_f16x2(y[2 * i], y[2 * i + 1]);
    }
}

// Three-input NaN-propagating max of absolute values (sm_100 three-input form).
__device__ __forceinline__ float max3_abs_nan(float a, float b, float c) {
    float r;
    asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float max_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// Ordered 32-bit key of an fp32 value: unsigned comparison of keys is the numeric order of
// the non-NaN values (-0 just below +0), and consecutive keys are adjacent fp32 values.
__device__ __forceinline__ uint32_t okey(float f) {
    const uint32_t b = __float_as_uint(f);
    return b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
}
__device__ __forceinline__ float okey_f32(uint32_t k) {
    return __uint_as_float(k ^ ((uint32_t)((int32_t)~k >> 31) | 0x80000000u));
}

// Byte permute.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// ---- E4M4 uint8 absmax (4-bit exponent, bias 11, 4-bit mantissa, subnormals) ----

// Exact value of a code: e > 0: 2^(e - 11) * (1 + m/16); e == 0: m * 2^-14.
// t = bits (c + 1856) << 19 places e + 116 in the fp32 exponent and m in its top mantissa
// bits, the value for e > 0. For e == 0 it is 2^-11 + m * 2^-15, and 2t - 2^-10 = m * 2^-14
// (exact); that is below t exactly when t < 2^-10, i.e. for the 16 subnormal codes.
__device__ __forceinline__ float e4m4_decode(uint32_t code) {
    const float t = __uint_as_float((code << 19) + (1856u << 19));
    return fminf(t, __fmaf_rn(t, 2.0f, -0x1p-10f));
}

// Code of an absmax: exponent floor(log2 a) + 11 clamped to [0, 15] (subnormal at <= 0), the
// mantissa rounded half-to-even in a's own binade and clamped to 15; values that are not > 0
// (zero, NaN) give 0, +infinity gives 0xFF.
__device__ __forceinline__ uint32_t e4m4_encode(float a) {
    const uint32_t u = __float_as_uint(a);
    if (!(a > 0.0f)) return 0u;
    if (u == 0x7f800000u) return 0xffu;
    const int eb = (int)(u >> 23) - 127 + 11;        // fp32 subnormals land far below 0
    if (eb <= 0) return (uint32_t)min(__float2int_rn(a * 16384.0f), 15);   // a * 2^14 is exact
    const uint32_t f = u & 0x7fffffu;
    const uint32_t m = min((f + 0x3ffffu + ((f >> 19) & 1u)) >> 19, 15u);    // RNE of f / 2^19
    return ((uint32_t)min(eb, 15) << 4) | m;
}

// Per-block absmax in either storage format.
__device__ __forceinline__ void store_absmax(float* p, int64_t b, float a) { p[b] = a; }
__device__ __forceinline__ void store_absmax(uint8_t* p, int64_t b, float a) { p[b] = (uint8_t)e4m4_encode(a); }
__device__ __forceinline__ float load_absmax(const float* p, int64_t b) { return __ldg(p + b); }
__device__ __forceinline__ float load_absmax(const uint8_t* p, int64_t b) { return e4m4_decode(__ldg(p + b)); }

// ---- bit-plane gather (k-bit decode) ----

// Byte offset (idx * 4) of element e (0..7) of a plane group B (byte j = plane j for
// elements 0..7; B3 = B << 3). For e >= 3 bits 8j+e are moved to bits 34+j of the 64-bit
// product (multiplier sum_j 2^(34-7j-e)); every cross term lands outside bits 34..37 on
// distinct positions, so no carry reaches the field. For e < 3 the same gather runs on B3.
template <int E>
__device__ __forceinline__ uint32_t plane_offset4(uint32_t B, uint32_t B3) {
    constexpr int e = E < 3 ? E + 3 : E;
    constexpr uint32_t mask = 0x01010101u << e;
    constexpr uint32_t mult = (1u << (34 - e)) | (1u << (27 - e)) | (1u << (20 - e)) | (1u << (13 - e));
    const uint32_t src = E < 3 ? B3 : B;
    return __umulhi(src & mask, mult) & 0x3Cu;
}


// ---- k-bit weights of a 32-element block: plane groups and per-element decode ----

// Element 8q + E of a block as fp32 (codebook entry times absmax, one rounding), from plane group
// Bq (byte j = plane j of elements 8q .. 8q+7, Bqs = Bq << 3) and, for K = 5, p4q (bit i = plane
// 4 of element 8q + i); cbb is the codebook in shared memory (byte address).
template <int KB, int DT, int E>
__device__ __forceinline__ float kbit_elem(uint32_t Bq, uint32_t Bqs, uint32_t p4q, float am, const char* cbb) {
    uint32_t off = plane_offset4<E>(Bq, Bqs);
    if constexpr (KB == 5) off |= (E <= 6 ? (p4q << (6 - E)) : (p4q >> (E - 6))) & 0x40u;
    return __fmul_rn(*reinterpret_cast<const float*>(cbb + off), am);
}
// The plane groups of a lane's run: all four for a 32-element run; for a 16-element run, the
// two groups of half h of the block.
template <int KB, int R>
__device__ __forceinline__ void kbit_groups(const uint32_t (&w)[KB], int h, uint32_t (&G)[R / 8], uint32_t& p4) {
    const uint32_t w0 = w[0], w1 = w[1 % KB], w2 = KB > 2 ? w[2 % KB] : 0u, w3 = KB > 3 ? w[3 % KB] : 0u;
    p4 = KB == 5 ? w[4 % KB] : 0u;
    if constexpr (R == 32) {
        const uint32_t t0 = prmt(w0, w1, 0x5140u), t1 = prmt(w0, w1, 0x7362u);
        const uint32_t t2 = prmt(w2, w3, 0x5140u), t3 = prmt(w2, w3, 0x7362u);
        G[0] = prmt(t0, t2, 0x5410u);
        G[1] = prmt(t0, t2, 0x7632u);
        G[2] = prmt(t1, t3, 0x5410u);
        G[3] = prmt(t1, t3, 0x7632u);
    } else {
        const uint32_t sel = h ? 0x7362u : 0x5140u;            // bytes 2h, 2h + 1 of two words
        const uint32_t tl = prmt(w0, w1, sel), th = prmt(w2, w3, sel);
        G[0] = prmt(tl, th, 0x5410u);
        G[1] = prmt(tl, th, 0x7632u);
        p4 >>= 16 * h;
    }
}

// ---- debug builds (-DBBC_DEBUG): bounds guards -------------------------------
//
// In a debug build every global access whose address a kernel computes is checked against the
// extent the launch's arguments give that buffer; a failed check sets its bit in this
// translation unit's status word and skips the access (no trap: the context stays usable), and
// bbc_debug_status reads the words. In a release build a guard is the constant true.
enum GuardBit : unsigned {
    kGuardQuantIn = 1u << 0,      // quantize input loads (k-bit and 4-bit), L2 prefetches
    kGuardQuantOut = 1u << 1,     // quantize stores: plane words, codes, absmax
    kGuardDequantIn = 1u << 2,    // k-bit dequant loads: plane words, absmax
    kGuardDequantOut = 1u << 3,   // k-bit dequant output stores
    kGuardNestedIn = 1u << 4,     // nested dequant loads (fused and three-launch)
    kGuardNestedOut = 1u << 5,    // nested dequant stores (output, scale workspace)
    kGuardTree = 1u << 6,         // offset tree loads and node stores
    kGuardCompress = 1u << 7,     // General8 compression loads and stores
    kGuardLinear = 1u << 8,       // fused linear weight loads (both linear kernels)
};
#ifdef BBC_DEBUG
static __device__ unsigned int g_bbc_guard;      // one status word per translation unit
#define BBC_GUARD(cond, bit) ((cond) || (atomicOr(&::bbc::g_bbc_guard, (unsigned)(bit)), false))
#define BBC_GUARD_ACCESSOR(name)                                                              \
    cudaError_t name(unsigned int* v, bool reset) {                                           \
        cudaError_t e = cudaMemcpyFromSymbol(v, g_bbc_guard, sizeof(unsigned int));           \
        if (e != cudaSuccess || !reset) return e;                                             \
        const unsigned int zero = 0;                                                          \
        return cudaMemcpyToSymbol(g_bbc_guard, &zero, sizeof(unsigned int));                  \
    }
#else
#define BBC_GUARD(cond, bit) (true)
#define BBC_GUARD_ACCESSOR(name)                                                              \
    cudaError_t name(unsigned int* v, bool) {                                                 \
        *v = 0;                                                                               \
        return cudaSuccess;                                                                   \
    }
#endif

}  // namespace bbc
