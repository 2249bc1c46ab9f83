// k-bit blockwise codebook quantization (K = 2..5, blocksize 32), bit-exact.
//
// Operation (bitsandbytes k-bit patch series, PATCH 001 "Add k-bit quantization
// kernels (K=2-5, blocksize=32)": quantize_kbit_ref and kQuantizeBlockwise_kbit):
// per block of 32, absmax = max|x| (stored raw), d = max(absmax, 1e-8f),
// xn = x / d in IEEE fp32, idx = first i minimising fabsf(xn - c[i]), and the K
// bit planes of the 32 indices are stored as K uint32 words.
//
// B200 design (not the pages' warp-per-block brute-force loop):
//
// 1. Exact decision thresholds. For a codebook that is finite, strictly
//    ascending and spaced at least 2^-19 * (1 + max|c|) apart, a fp32 distance
//    fl(xn - c_i) can never tie with a farther entry on the same side, so the
//    index is a non-decreasing step function of xn:
//        idx(xn) = #{ j >= 1 : xn >= T_j },
//    where T_j is the smallest fp32 value at which entry j beats entry j-1
//    under the exact rule fl(c_j - v) < fl(v - c_{j-1}). Each CTA finds the
//    T_j by bisection over the ordered fp32 bit patterns (<= 32 steps), using
//    the same IEEE subtractions as the rule itself. Any other codebook takes
//    the brute-force search, which is the rule verbatim.
//
// 2. One table lookup per element instead of 2^K distance tests. The quotient
//    is estimated as q = x * RN(1/d) (one multiply; |q - RN(x/d)| < 1.5*2^-23 |x/d|).
//    A 256-cell table indexed by round(8192*q)/128 (cells 1/64 wide, found
//    with one fused multiply-add and a mask) holds, per cell, the only
//    threshold that can matter there, widened to a guard band
//    [T - g, T + g), g = 2^-19 |T| + 2^-100, and the byte-spread bit patterns
//    of the two possible indices. Outside the band the estimate decides
//    exactly; inside it (about 2^-16 of elements for the normal-float
//    codebooks) the thread redoes its 8 elements with IEEE division and the
//    brute-force rule. Cells with two candidate thresholds are all-guard.
//    The table is replicated 8 times so the 8 lanes of each quarter-warp
//    phase of a 128-bit shared load always hit distinct banks.
//
// 3. Bit-plane packing without ballots. A thread owns 8 consecutive elements
//    (one quarter of a block); adding spread(idx_e) << e, where spread puts
//    bit k of idx at bit 8k, builds byte k = bits of plane k for its 8
//    elements in one register. A 4x4 byte transpose across the block's four
//    lanes (two xor-shuffles, two byte permutes) leaves word j in lane j.
//    K = 5 keeps plane 4 in a second register (bit 4 of idx is xn >= T_16).
//
// Blocks whose NaN-propagating absmax is NaN, infinite or above 2^125 (where
// 1/d would be subnormal) take the exact path for all their elements.
#include <cfloat>

#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kThreads = 256;
constexpr int kCells = 256;
constexpr int kReplicas = 8;

__device__ __forceinline__ int64_t f32_key(float f) {
    const int32_t b = __float_as_int(f);
    return b >= 0 ? (int64_t)b : -(int64_t)(b & 0x7fffffff) - 1;
}
__device__ __forceinline__ float key_f32(int64_t k) {
    const uint32_t b = k >= 0 ? (uint32_t)k : ((uint32_t)(-(k + 1)) | 0x80000000u);
    return __uint_as_float(b);
}

// Smallest fp32 v in [lo, hi] where entry `hi` beats entry `lo` under the exact
// rule; the predicate is false at lo and true at hi and monotone in v.
__device__ float bisect_threshold(float lo_c, float hi_c) {
    int64_t lo = f32_key(lo_c), hi = f32_key(hi_c);
    for (int it = 0; it < 40 && hi - lo > 1; it++) {
        const int64_t mid = lo + ((hi - lo) >> 1);
        const float v = key_f32(mid);
        if (__fsub_rn(hi_c, v) < __fsub_rn(v, lo_c)) hi = mid;
        else lo = mid;
    }
    return key_f32(hi);
}

// Bits 0..3 of v moved to bits 0, 8, 16, 24.
__device__ __forceinline__ uint32_t spread4(uint32_t v) { return ((v & 15u) * 0x00204081u) & 0x01010101u; }

// Brute-force nearest entry: first index with the smallest fp32 distance.
template <int NE>
__device__ __forceinline__ uint32_t nearest_entry(float xn, const float* cb) {
    float best = __int_as_float(0x7f800000);
    uint32_t idx = 0;
#pragma unroll
    for (int i = 0; i < NE; i++) {
        const float dist = fabsf(__fsub_rn(xn, cb[i]));
        if (dist < best) { best = dist; idx = i; }
    }
    return idx;
}

template <int DT, bool VEC>
__device__ __forceinline__ void load8(const void* A, int64_t n, int64_t Q, bool active, float* x) {
    const int64_t m0 = Q * 8;
    if (VEC && active && m0 + 8 <= n) {
        if constexpr (DT == F32) {
            const char* p = reinterpret_cast<const char*>(A) + m0 * 4;
            const uint4 a = ldg_stream_v4(p), b = ldg_stream_v4(p + 16);
            x[0] = __uint_as_float(a.x); x[1] = __uint_as_float(a.y);
            x[2] = __uint_as_float(a.z); x[3] = __uint_as_float(a.w);
            x[4] = __uint_as_float(b.x); x[5] = __uint_as_float(b.y);
            x[6] = __uint_as_float(b.z); x[7] = __uint_as_float(b.w);
        } else {
            const uint4 v = ldg_stream_v4(reinterpret_cast<const char*>(A) + m0 * 2);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                if constexpr (DT == BF16) {
                    x[2 * i] = __uint_as_float(w[i] << 16);
                    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
                } else {
                    x[2 * i] = f16_bits_to_f32(w[i] & 0xffffu);
                    x[2 * i + 1] = f16_bits_to_f32(w[i] >> 16);
                }
            }
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; e++)
            x[e] = (active && m0 + e < n) ? load_as_f32<DT>(A, m0 + e) : 0.0f;
    }
}

template <int K, int DT, bool VEC>
__global__ void __launch_bounds__(kThreads)
kbit_quant_kernel(const void* __restrict__ A, int64_t n, const float* __restrict__ codebook,
                  float* __restrict__ absmax, uint32_t* __restrict__ packed) {
    constexpr int NE = 1 << K;
    __shared__ __align__(16) float4 lut[kCells * kReplicas];    // 32 KB
    __shared__ float cb[32];
    __shared__ float thr[33];
    __shared__ int fast_ok;

    const int tid = threadIdx.x;
    const int lane = tid & 31;

    // ---- per-CTA set-up: codebook check, thresholds, lookup table ----
    if (tid < 32) {
        const float c = tid < NE ? codebook[tid] : 0.0f;
        cb[tid] = c;
        float mag = tid < NE ? fabsf(c) : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mag = max_nan(mag, __shfl_xor_sync(0xffffffffu, mag, o));
        const float D = __fadd_rn(1.0f, mag);
        const float prev = __shfl_up_sync(0xffffffffu, c, 1);
        bool ok = true;
        if (tid < NE) {
            ok = fabsf(c) <= FLT_MAX;                                  // finite (false for NaN)
            if (tid > 0) ok = ok && (__fsub_rn(c, prev) >= __fmul_rn(D, 0x1p-19f));
        }
        ok = ok && (D <= FLT_MAX);
        const bool fast = __all_sync(0xffffffffu, ok);
        if (tid == 0) fast_ok = fast ? 1 : 0;
        if (fast && tid >= 1 && tid < NE) thr[tid] = bisect_threshold(prev, c);
    }
    __syncthreads();
    const bool fast_cb = fast_ok != 0;
    if (fast_cb) {
        for (int cell = tid; cell < kCells; cell += kThreads) {
            const int cs = cell < 128 ? cell : cell - 256;
            const float wlo = __fsub_rn((float)cs * 0.015625f, 0x1p-13f + 0x1p-12f);
            const float whi = __fadd_rn((float)(cs + 1) * 0.015625f, 0x1p-13f + 0x1p-12f);
            int below = 0, rel = 0, relj = 0;
            for (int j = 1; j < NE; j++) {
                const float T = thr[j];
                if (T < wlo) below++;
                else if (T <= whi) { rel++; relj = j; }
            }
            float tlo = __int_as_float(0x7f800000), thi = tlo;               // +inf: never crossed
            if (rel == 1) {
                const float T = thr[relj];
                const float g = __fadd_ru(__fmul_ru(fabsf(T), 0x1p-19f), 0x1p-100f);
                tlo = __fsub_rd(T, g);
                thi = __fadd_ru(T, g);
            } else if (rel > 1) {
                tlo = __int_as_float(0xff800000);                              // -inf: always guard
            }
            const float4 ent = make_float4(tlo, thi, __uint_as_float(spread4((uint32_t)below)),
                                           __uint_as_float(spread4((uint32_t)below + 1)));
#pragma unroll
            for (int r = 0; r < kReplicas; r++) lut[cell * kReplicas + r] = ent;
        }
    }
    __syncthreads();

    const char* lutb = reinterpret_cast<const char*>(lut);
    const uint32_t lutoff = (uint32_t)(lane & 7) << 4;
    const uint32_t part = lane & 3;
    const uint32_t sel_a = (part & 1) ? 0x3715u : 0x6240u;
    const uint32_t sel_b = (part & 2) ? 0x3276u : 0x5410u;
    const uint32_t grp_mask = 0xFu << (lane & ~3);
    const float t16 = (K == 5 && fast_cb) ? thr[16] : 0.0f;

    const int64_t nq = ((n + 31) >> 5) * 4;                      // quarter blocks
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t wbase = (int64_t)blockIdx.x * kThreads + (tid & ~31); wbase < nq; wbase += stride) {
        const int64_t Q = wbase + lane;
        const bool active = Q < nq;                               // the 4 lanes of a block agree
        float x[8];
        load8<DT, VEC>(A, n, Q, active, x);

        // NaN-propagating block max decides between the fast and the exact path
        float m = max3_abs_nan(x[0], x[1], x[2]);
        m = max3_abs_nan(m, x[3], x[4]);
        m = max3_abs_nan(m, x[5], x[6]);
        m = max_nan(m, fabsf(x[7]));
        m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, 2));
        const bool special = !(m <= 0x1p125f);
        float amax = m;
        if (special) {   // the stored absmax ignores NaN unless the whole block is NaN
            float a = fabsf(x[0]);
#pragma unroll
            for (int e = 1; e < 8; e++) a = fmaxf(a, fabsf(x[e]));
            a = fmaxf(a, __shfl_xor_sync(grp_mask, a, 1));
            a = fmaxf(a, __shfl_xor_sync(grp_mask, a, 2));
            amax = a;
        }
        const float d = fmaxf(amax, 1e-8f);

        uint32_t acc = 0, acc4 = 0;
        bool exact = special || !fast_cb;
        if (!exact) {
            const float r = __frcp_rn(d);
            bool guard = false;
#pragma unroll
            for (int e = 0; e < 8; e++) {
                const float q = __fmul_rn(x[e], r);
                const float f = __fmaf_rn(q, 8192.0f, 12582912.0f);
                const float4 ent = *reinterpret_cast<const float4*>(
                    lutb + ((__float_as_uint(f) & 0x7f80u) | lutoff));
                const bool a = q >= ent.x;
                const bool b = q >= ent.y;
                guard |= (a != b);
                acc += (b ? __float_as_uint(ent.w) : __float_as_uint(ent.z)) << e;
                if constexpr (K == 5) acc4 |= set_ge(q, t16) & (1u << e);
            }
            exact = guard;
        }
        if (exact) {
            acc = 0;
            acc4 = 0;
#pragma unroll
            for (int e = 0; e < 8; e++) {
                const uint32_t idx = nearest_entry<NE>(__fdiv_rn(x[e], d), cb);
                acc |= spread4(idx) << e;
                if constexpr (K == 5) acc4 |= ((idx >> 4) & 1u) << e;
            }
        }

        // 4x4 byte transpose across the block's lanes: lane j ends with plane word j
        acc = prmt(acc, __shfl_xor_sync(0xffffffffu, acc, 1), sel_a);
        acc = prmt(acc, __shfl_xor_sync(0xffffffffu, acc, 2), sel_b);
        if constexpr (K == 5) {
            acc4 = prmt(acc4, __shfl_xor_sync(0xffffffffu, acc4, 1), sel_a);
            acc4 = prmt(acc4, __shfl_xor_sync(0xffffffffu, acc4, 2), sel_b);
        }
        if (active) {
            const int64_t b = Q >> 2;
            if (part < (uint32_t)(K < 4 ? K : 4)) packed[b * K + part] = acc;
            if (part == 0) {
                if constexpr (K == 5) packed[b * 5 + 4] = acc4;
                absmax[b] = amax;
            }
        }
    }
}

template <int K, int DT>
cudaError_t launch_t(const void* A, int64_t n, const float* codebook, float* absmax,
                     uint32_t* packed, bool vec, cudaStream_t s) {
    const int64_t nq = ((n + 31) >> 5) * 4;
    if (vec) {
        auto k = kbit_quant_kernel<K, DT, true>;
        int grid = persistent_grid(k, kThreads, 0, nq, kThreads);
        k<<<grid, kThreads, 0, s>>>(A, n, codebook, absmax, packed);
    } else {
        auto k = kbit_quant_kernel<K, DT, false>;
        int grid = persistent_grid(k, kThreads, 0, nq, kThreads);
        k<<<grid, kThreads, 0, s>>>(A, n, codebook, absmax, packed);
    }
    return cudaGetLastError();
}

template <int K>
cudaError_t launch_k(const void* A, int dt, int64_t n, const float* codebook, float* absmax,
                     uint32_t* packed, bool vec, cudaStream_t s) {
    switch (dt) {
        case F16: return launch_t<K, F16>(A, n, codebook, absmax, packed, vec, s);
        case BF16: return launch_t<K, BF16>(A, n, codebook, absmax, packed, vec, s);
        default: return launch_t<K, F32>(A, n, codebook, absmax, packed, vec, s);
    }
}

}  // namespace

cudaError_t launch_kbit_quantize(const void* A, int dtype, int64_t n, int K, const float* codebook,
                                 float* absmax, uint32_t* packed, bool vec, cudaStream_t s) {
    switch (K) {
        case 2: return launch_k<2>(A, dtype, n, codebook, absmax, packed, vec, s);
        case 3: return launch_k<3>(A, dtype, n, codebook, absmax, packed, vec, s);
        case 4: return launch_k<4>(A, dtype, n, codebook, absmax, packed, vec, s);
        default: return launch_k<5>(A, dtype, n, codebook, absmax, packed, vec, s);
    }
}

}  // namespace bbc
