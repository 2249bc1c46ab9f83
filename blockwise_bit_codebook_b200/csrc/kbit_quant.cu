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
//    fl(xn - c_i) never ties with a farther entry on the same side, so the index
//    is a non-decreasing step function of xn:  idx(xn) = #{ j >= 1 : xn >= T_j },
//    where T_j is the smallest fp32 value at which entry j beats entry j-1 under
//    the exact rule fl(c_j - v) < fl(v - c_{j-1}). Each CTA finds the T_j by
//    bisection over the ordered fp32 bit patterns, using the same IEEE
//    subtractions as the rule. Any other codebook takes the brute-force search,
//    which is the rule verbatim.
//
// 2. An exact test against one threshold without dividing. With h_T half the
//    gap from T down to the next fp32 value, RN(x/d) >= T  <=>  x/d > T - h_T
//    (x/d is never exactly an fp32 midpoint: its numerator would need more
//    than 24 significant bits), i.e. x - T*d + h_T*d > 0, and the sign of that
//    sum is computed exactly by v = fma(h_T, d, fma(-T, d, x)): when |x - T*d|
//    is below ulp(T)*d the inner fma is exact, otherwise its rounding cannot
//    change the sign of the sum. Two paired f32x2 FMAs per element pair.
//
// 3. One table lookup finds the threshold. A 256-cell table indexed by the cell
//    c = round(64 x/d) (cells 1/64 wide, centred on multiples of 1/64; one paired fma
//    with a magic constant, stored at slot c + 128) holds, per cell, the only threshold
//    that can matter there and the byte-spread bit pattern of the index below it. The
//    entry's shared address is one multiply-add of the fma's bits (bits * 128 plus a
//    per-lane constant that absorbs the magic constant, the table base and the lane's
//    replica). A codebook whose thresholds are closer than a cell takes the brute-force
//    search. Half-block threads (fp32, unaligned input) read 16-byte entries (-T, h_T,
//    spread(L), spread(L + 1)), 8 replicas so that the 8 lanes of each 128-bit
//    shared-load phase always hit distinct banks.
//
//    Whole-block threads (32-byte-aligned 16-bit input) use an 8-byte entry instead
//    (16 replicas): {-A, spread(L)} with A = prev(T) for T > 0 and A = T for T < 0, so
//    that the decision midpoint is always A + copysign(ulp(|A|) / 2, A); that half-ulp H
//    is 2^-24 times the sign and exponent bits of A, so -H * d is (the masked bits of
//    -A) * (d * 2^-24), both exact (one mask per element, one multiply per block); the
//    test becomes v = fma(-H, d, fma(-A, d, x)) with the same exactness argument, and
//    instead of selecting spread(L) or spread(L + 1) the sign bits of v are collected
//    (one funnel shift per element) and added to the K plane words of the block at the
//    end as a bit-sliced increment. Half the shared-memory bytes per element, one
//    select fewer. The thresholds must lie at least 2^-100 from zero (they do for any
//    codebook the fast path accepts; the set-up checks it).
//
// 4. Bit-plane packing without ballots. Adding spread(idx) << e (bit k of idx at
//    bit 8k) builds, per 8 elements, one register whose byte k holds plane k
//    (K = 5 accumulates 4 elements per register with plane 4 in bits 4..7). For
//    32-byte-aligned 16-bit input a thread owns a whole block (two 32-byte loads,
//    the next block prefetched into registers; two CTAs per SM leave room for
//    that) and eight byte permutes turn its four registers into the K plane
//    words. Otherwise (fp32, unaligned input, the ragged end) a thread owns half a
//    block and one xor-shuffle plus four byte permutes between the two lanes of
//    a block leave words 2h, 2h+1 in lane h.
//
// Blocks whose NaN-propagating absmax is NaN, infinite or above 2^125 take the
// brute-force path (IEEE division and the rule verbatim) for all their elements.
#include <cfloat>

#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kThreads = 256;
constexpr int kCells = 256;
constexpr int kReplicas = 8;
constexpr int kReplicas8 = 16;           // the 8-byte table: 16 lanes per shared-load phase
// Resident CTAs per SM the register budget targets: the vector paths (the whole-block 16-bit
// path and the fp32 half-block path) trade occupancy for per-thread parallelism (at three CTAs
// the fp32 path spilled and ran 2-10 % slower); the unaligned path keeps three.
template <int DT, bool VEC> constexpr int kMinCtas = VEC ? 2 : 3;

// The largest fp32 value below v (v finite and above -FLT_MAX).
__device__ __forceinline__ float prev_f32(float v) { return okey_f32(okey(v) - 1u); }

// The exact rule at v for two entries a < b: entry b is strictly nearer than entry a.
__device__ __forceinline__ bool beats(float a, float b, float v) { return __fsub_rn(b, v) < __fsub_rn(v, a); }

// Smallest fp32 v in (a, b] where entry b beats entry a under the exact rule, found by the 8
// lanes of a lane group (r = lane & 7; lanes 8g .. 8g+7 of the warp; every lane of the warp
// calls this together). The rule is false at a, true at b and monotone in between (fl(b - v)
// does not increase and fl(v - a) does not decrease with v).
//
// 1. Where it can be. For v below the midpoint m = (a + b) / 2, fl(b - v) >= fl(v - a); above
//    m + ulp(b - a) / 2 the two distances differ by more than their rounding can hide. So the
//    threshold lies in (m, m + ulp(b - a) / 2].
// 2. Candidates. There the rule can change only where b - v or v - a crosses a rounding boundary
//    of fp32 near (b - a) / 2 (the midpoint beta of two neighbouring fp32 values): at v = b - beta
//    or v = a + beta. Each lane takes one boundary (8 neighbouring ones cover the interval) and
//    tests the smallest fp32 at or above each of its two breakpoints and the next value; the
//    group keeps the smallest candidate where the rule holds.
// 3. Check. It is the threshold if the rule holds there and fails one fp32 value below (the rule
//    being monotone), however the candidates were formed. Every lane checks it (no vote needed).
// 4. Otherwise (never seen for codebooks the fast path accepts) a search over the ordered keys
//    from the bracket of step 1 (checked at both ends first): 8 keys per step split it into 9
//    parts (at most 11 steps for 2^32 keys).
// `ok` is false when even the search did not converge.
__device__ __forceinline__ float group_threshold(float a, float b, bool live, bool& ok) {
    const int lane = threadIdx.x & 31, r = lane & 7, gs = lane & 24;
    uint32_t lo = okey(a), hi = okey(b);
    const float w = __fsub_ru(b, a);
    const double uh = (double)__uint_as_float(__float_as_uint(w) & 0x7f800000u) * 0x1p-24;   // ulp(w) / 2
    // 2. candidates from this lane's rounding boundary of the distances
    const double h = 0.5 * ((double)b - (double)a);
    const uint32_t k0 = okey(__double2float_rd(h - uh)) - 1u + (uint32_t)r;
    const double beta = 0.5 * ((double)okey_f32(k0) + (double)okey_f32(k0 + 1u));
    const uint32_t c1 = okey(__double2float_ru((double)b - beta));
    const uint32_t c2 = okey(__double2float_ru((double)a + beta));
    uint32_t best = hi;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t c = (i & 2 ? c2 : c1) + (uint32_t)(i & 1);
        if (c > lo && c < best && beats(a, b, okey_f32(c))) best = c;
    }
    best = min(best, __shfl_xor_sync(0xffffffffu, best, 1));
    best = min(best, __shfl_xor_sync(0xffffffffu, best, 2));
    best = min(best, __shfl_xor_sync(0xffffffffu, best, 4));
    // 3. the check, in every lane of the group
    const bool done = best > lo && !beats(a, b, okey_f32(best - 1u)) && beats(a, b, okey_f32(best));
    if (done) {
        lo = best - 1u;
        hi = best;
    }
    // 4. fallback search
    if (__any_sync(0xffffffffu, live && !done)) {
        const double m = 0.5 * (double)a + 0.5 * (double)b;
        uint32_t lo1 = okey(__double2float_rd(m)) - 1u, hi1 = okey(__double2float_ru(m + uh)) + 1u;
        lo1 = max(lo1, lo);
        hi1 = min(hi1, hi);
        // lane 0 checks that the rule is false at lo1, lane 1 that it is true at hi1
        const bool p = beats(a, b, okey_f32(r == 0 ? lo1 : hi1));
        const uint32_t g = (__ballot_sync(0xffffffffu, p) >> gs) & 0xffu;
        if (!done && (g & 3u) == 2u && lo1 < hi1) { lo = lo1; hi = hi1; }
        constexpr uint32_t kNinth = 477218588u;                  // floor(2^32 / 9)
        for (int it = 0; it < 12; it++) {
            const uint32_t range = hi - lo;
            if (!__any_sync(0xffffffffu, live && range > 1u)) break;
            // key lo + floor(range (r + 1) / 9) (rounded down; non-decreasing in r, below hi)
            const uint32_t pt = lo + __umulhi(range, (uint32_t)(r + 1) * kNinth);
            const bool q = beats(a, b, okey_f32(pt));
            const uint32_t gq = (__ballot_sync(0xffffffffu, q) >> gs) & 0xffu;
            const uint32_t below = 8u - (uint32_t)__popc(gq);    // points where the rule is still false
            const uint32_t nlo = lo + __umulhi(range, below * kNinth);
            const uint32_t nhi = below == 8u ? hi : lo + __umulhi(range, (below + 1u) * kNinth);
            if (range > 1u) { lo = nlo; hi = nhi; }
        }
    }
    ok = hi - lo <= 1u;
    return okey_f32(hi);
}

// Bits 0..3 of v at bits 0, 8, 16, 24; for K = 5 also bit 4 of v at bit 4.
template <int K>
__device__ __forceinline__ uint32_t spread(uint32_t v) {
    uint32_t s = ((v & 15u) * 0x00204081u) & 0x01010101u;
    if constexpr (K == 5) s |= (v & 16u);
    return s;
}

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

// Number of thresholds thr[1 .. NE-1] below x (LESS) or at most x (!LESS): a branch-free binary
// search over the ascending thresholds (thr[NE .. 32] hold +inf).
template <int NE, bool LESS>
__device__ __forceinline__ int count_thresholds(const float* thr, float x) {
    int k = 0;
#pragma unroll
    for (int step = NE / 2; step >= 1; step >>= 1) {
        const float T = thr[k + step];
        if (LESS ? (T < x) : (T <= x)) k += step;
    }
    return k;
}

// Per-CTA set-up of the exact threshold method for a 2^K-entry codebook (every thread of the
// CTA calls it; the result is CTA-uniform): loads the codebook into cb[], decides whether the
// fast path applies (finite, strictly ascending, spaced >= 2^-19 (1 + max|c|), at most one
// threshold per table cell), finds the thresholds (one 8-lane group each, all warps at once)
// and fills the 256-cell table (8 replicas) whose entries are {-T, h_T, pattern(L),
// pattern(L + 1)}: the bit-plane spread of the index for the k-bit codec, the index itself for
// nibble codes. With `lut8` it fills the 8-byte table {-A, pattern(L)} (16 replicas) instead
// (see step 3 of the header).
// The codebook entry a thread of warp 0 loads for the set-up (lanes >= 2^K hold 0). The load
// goes to L2 (the coherence point), never to L1: the set-up may read the codebook before
// griddepcontrol.wait, and the check after it (codebook_changed) must not see a stale L1 copy.
__device__ __forceinline__ float ldg_f32_l2(const float* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

template <int K>
__device__ __forceinline__ float load_codebook_entry(const float* __restrict__ codebook) {
    return threadIdx.x < (1u << K) ? ldg_f32_l2(codebook + threadIdx.x) : 0.0f;
}

template <int K, bool NIBBLE>
__device__ __forceinline__ bool setup_exact_table(float c, float* cb, float* thr,
                                                  int* fast_ok, uint4* lut, uint2* lut8 = nullptr) {
    constexpr int NE = 1 << K;
    static_assert((NE - 1) * 8 <= kThreads, "one 8-lane group per threshold");
    const int tid = threadIdx.x;
    // thresholds: group j - 1 (threads 8(j-1) .. 8j-1) finds the one between entries j-1 and j
    const int j = (tid >> 3) + 1;
    const bool live = j < NE;
    if (tid < 32) {
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
        if (tid == 0) *fast_ok = fast ? 1 : 0;
        if (tid >= NE) thr[tid] = __int_as_float(0x7f800000);        // +inf past the last threshold
        if (tid == 0) thr[32] = __int_as_float(0x7f800000);
    }
    __syncthreads();
    const float ca = live ? cb[j - 1] : 0.0f, cbv = live ? cb[j] : 1.0f;
    bool conv = true;
    const float T = group_threshold(ca, cbv, live, conv);
    if (live && (tid & 7) == 0) thr[j] = T;
    const int unconverged = __syncthreads_or(live && !conv);
    int multi = 0;
    if (*fast_ok && !unconverged) {
        for (int cell = tid; cell < kCells; cell += kThreads) {
            // cell cs = round(64 xn) at slot cs + 128: it holds every xn within half a cell
            const int cs = cell - 128;
            const float lo_edge = ((float)cs - 0.5f) * 0.015625f;
            const float hi_edge = ((float)cs + 0.5f) * 0.015625f;
            const float wlo = __fsub_rn(lo_edge, 0x1p-13f + 0x1p-12f);
            const float whi = __fadd_rn(hi_edge, 0x1p-13f + 0x1p-12f);
            const int below = count_thresholds<NE, true>(thr, wlo);
            const int rel = count_thresholds<NE, false>(thr, whi) - below;
            float negT = __int_as_float(0xff800000), half = 0.0f;     // -inf, 0: never crossed
            const float Tr = thr[below + 1];                          // the one relevant threshold
            if (rel == 1) {
                negT = -Tr;
                half = __fmul_rn(__fsub_rn(Tr, prev_f32(Tr)), 0.5f);
            }
            multi |= rel > 1;
            const uint32_t p0 = NIBBLE ? (uint32_t)below : spread<K>((uint32_t)below);
            const uint32_t p1 = NIBBLE ? (uint32_t)below + 1 : spread<K>((uint32_t)below + 1);
            if (!lut8) {
                const uint4 ent = make_uint4(__float_as_uint(negT), __float_as_uint(half), p0, p1);
                // the 8 lanes of a store phase write 8 different replicas: distinct banks
#pragma unroll
                for (int r = 0; r < kReplicas; r++) lut[cell * kReplicas + ((r + tid) & (kReplicas - 1))] = ent;
            } else {
                float nA = __int_as_float(0xff800000);               // -inf: never crossed
                if (rel == 1) {
                    const float Av = Tr > 0.0f ? prev_f32(Tr) : Tr;
                    nA = -Av;
                    multi |= !(fabsf(Av) >= 0x1p-100f);              // keep the rebuilt half-ulp normal
                }
                const uint32_t e = __float_as_uint(nA);
                // replicas 2q, 2q + 1 in one 16-byte store; the 8 lanes of a store phase write 8
                // different replica pairs: distinct banks
                uint4* row = reinterpret_cast<uint4*>(lut8 + cell * kReplicas8);
#pragma unroll
                for (int q = 0; q < kReplicas8 / 2; q++) row[(q + tid) & (kReplicas8 / 2 - 1)] = make_uint4(e, p0, e, p0);
            }
        }
    }
    return (*fast_ok != 0) && !unconverged && !__syncthreads_or(multi);
}

// After griddepcontrol.wait: true (CTA-uniform) if the codebook differs, bit for bit, from the
// values the set-up used (read before the wait, while the previous kernel of the stream may still
// have been writing them). The table is a function of those values alone, so when they are equal
// it is the table that stream order defines; otherwise the caller runs the set-up again.
template <int K>
__device__ __forceinline__ bool codebook_changed(const float* __restrict__ codebook, const float* cb) {
    bool diff = false;
    if (threadIdx.x < (1u << K))
        diff = __float_as_uint(ldg_f32_l2(codebook + threadIdx.x)) != __float_as_uint(cb[threadIdx.x]);
    return __syncthreads_or(diff) != 0;
}

// Programmatic dependent launch, early form: lets the next kernel of the stream be scheduled once
// every CTA of this grid has executed it. Used only by a grid that fills the GPU (every SM at this
// kernel's occupancy), so that the next launch's CTAs take SMs only as this grid's CTAs retire
// and run their set-up during this grid's tail.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Prefetch of `bytes` (a multiple of 16, 16-byte aligned) into L2. Safe before griddepcontrol.wait:
// nothing reaches the SM, and L2 is coherent, so the loads after the wait see current data.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(bytes) : "memory");
}

// Raw input words of one half block (16 elements): 8 words for 16-bit types, 16 for fp32.
template <int DT>
struct Raw { uint32_t w[DT == F32 ? 16 : 8]; };

template <int DT, bool VEC>
__device__ __forceinline__ Raw<DT> load_raw(const void* A, int64_t n, int64_t H, bool active) {
    Raw<DT> r;
    const int64_t m0 = H * 16;
    if (VEC && active && m0 + 16 <= n) {
        const char* p = reinterpret_cast<const char*>(A) + m0 * dtype_size(DT);
        const u32x8 a = ldg_stream_v8(p);
#pragma unroll
        for (int i = 0; i < 8; i++) r.w[i] = a.v[i];
        if constexpr (DT == F32) {
            const u32x8 b = ldg_stream_v8(p + 32);
#pragma unroll
            for (int i = 0; i < 8; i++) r.w[8 + i] = b.v[i];
        }
    } else {
        // ragged tail or unaligned input: element-wise raw loads, zeros beyond n
        if constexpr (DT == F32) {
            const float* a = reinterpret_cast<const float*>(A);
#pragma unroll
            for (int e = 0; e < 16; e++) r.w[e] = (active && m0 + e < n) ? __float_as_uint(a[m0 + e]) : 0u;
        } else {
            const uint16_t* a = reinterpret_cast<const uint16_t*>(A);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const uint32_t lo = (active && m0 + 2 * i < n) ? (uint32_t)a[m0 + 2 * i] : 0u;
                const uint32_t hi = (active && m0 + 2 * i + 1 < n) ? (uint32_t)a[m0 + 2 * i + 1] : 0u;
                r.w[i] = lo | (hi << 16);
            }
        }
    }
    return r;
}

// Exact fp32 values of the two 16-bit elements packed in w (element 2i in the low half).
// Raw words of a half block that lies entirely inside the input (vector loads only).
template <int DT>
__device__ __forceinline__ Raw<DT> load_full(const void* A, int64_t H, bool active, int64_t n) {
    Raw<DT> r;
    if (active && BBC_GUARD(H >= 0 && (H + 1) * 16 <= n, kGuardQuantIn)) {
        const char* p = reinterpret_cast<const char*>(A) + H * 16 * dtype_size(DT);
        const u32x8 a = ldg_stream_v8(p);
#pragma unroll
        for (int i = 0; i < 8; i++) r.w[i] = a.v[i];
        if constexpr (DT == F32) {
            const u32x8 b = ldg_stream_v8(p + 32);
#pragma unroll
            for (int i = 0; i < 8; i++) r.w[8 + i] = b.v[i];
        }
    } else {
#pragma unroll
        for (int i = 0; i < (DT == F32 ? 16 : 8); i++) r.w[i] = 0u;
    }
    return r;
}

template <int DT>
__device__ __forceinline__ void widen_pair(uint32_t w, float& lo, float& hi) {
    if constexpr (DT == BF16) {
        lo = __uint_as_float(w << 16);
        hi = __uint_as_float(w & 0xffff0000u);
    } else {
        lo = f16_bits_to_f32(w & 0xffffu);
        hi = f16_bits_to_f32(w >> 16);
    }
}

// Per-half NaN-propagating max of absolute values of two packed pairs (the sign bit of the
// result is not meaningful; callers take the absolute value).
template <int DT>
__device__ __forceinline__ uint32_t pair_absmax(uint32_t a, uint32_t b) {
    uint32_t r;
    if constexpr (DT == BF16) asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    else asm("max.NaN.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

template <int DT>
__device__ __forceinline__ void widen(const Raw<DT>& r, float* x) {
    if constexpr (DT == F32) {
#pragma unroll
        for (int e = 0; e < 16; e++) x[e] = __uint_as_float(r.w[e]);
    } else if constexpr (DT == BF16) {
#pragma unroll
        for (int i = 0; i < 8; i++) {
            x[2 * i] = __uint_as_float(r.w[i] << 16);
            x[2 * i + 1] = __uint_as_float(r.w[i] & 0xffff0000u);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) {
            x[2 * i] = f16_bits_to_f32(r.w[i] & 0xffffu);
            x[2 * i + 1] = f16_bits_to_f32(r.w[i] >> 16);
        }
    }
}

__device__ __forceinline__ float rcp_approx(float d) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}

// Per-thread constants of the main loop.
struct LoopCtx {
    uint32_t lut_c;         // address of slot 0 of this lane's replica (16-byte table) minus the
                            // magic constant's bits * 128
    uint32_t lut8_s;        // shared address of the 8-byte table (whole-block path)
    uint32_t lane8;         // this lane's replica offset in it
    uint32_t lut8_c;        // address of slot 0 of this lane's replica minus the magic constant's bits * 128
    uint32_t h;             // which half of the block this lane owns
    uint32_t sel_send, sel_keep, sel_wa, sel_wb, pair_mask;
    bool fast_cb;
    bool packed_v2;
    bool packed_v4;
    uint32_t* stage;        // this warp's 32 * 5 words (whole-block path, K = 5)
    int lane;
    int64_t nb;             // blocks of the input (bounds guards of debug builds)
};

// The table entry of the cell whose index sits in bits 7..14 of `fbits`.
__device__ __forceinline__ uint4 lut_entry(const LoopCtx& c, uint32_t fbits) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(fbits * 128u + c.lut_c));
    return v;
}

// The 8-byte table entry {-A, spread(L)} of the cell in bits 7..14 of `fbits` (128 bytes per
// cell, as the 16-byte table: the same cell offset).
__device__ __forceinline__ uint2 lut8_entry(const LoopCtx& c, uint32_t fbits) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(fbits * 128u + c.lut8_c));
    return v;
}

// Fast path for one half block: thresholds via the table, exact two-FMA test per element.
template <int K, int DT>
__device__ __forceinline__ void fast_codes(const Raw<DT>& raw, float d, const LoopCtx& c, uint32_t* acc) {
    constexpr int EPA = K == 5 ? 4 : 8;           // 4 elements per accumulator for K = 5, else 8
    const float rs = __fmul_rn(rcp_approx(d), 64.0f);
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
        float x0, x1;
        if constexpr (DT == F32) {
            x0 = __uint_as_float(raw.w[e]);
            x1 = __uint_as_float(raw.w[e + 1]);
        } else {
            widen_pair<DT>(raw.w[e / 2], x0, x1);
        }
        const float2 f = __ffma2_rn(make_float2(x0, x1), make_float2(rs, rs),
                                    make_float2(12582912.0f, 12582912.0f));
        const uint4 t0 = lut_entry(c, __float_as_uint(f.x));
        const uint4 t1 = lut_entry(c, __float_as_uint(f.y));
        const float v0 = __fmaf_rn(__uint_as_float(t0.y), d, __fmaf_rn(__uint_as_float(t0.x), d, x0));
        const float v1 = __fmaf_rn(__uint_as_float(t1.y), d, __fmaf_rn(__uint_as_float(t1.x), d, x1));
        acc[e / EPA] += (v0 > 0.0f ? t0.w : t0.z) << (e % EPA);
        acc[(e + 1) / EPA] += (v1 > 0.0f ? t1.w : t1.z) << ((e + 1) % EPA);
    }
}

// Brute-force path for one half block: IEEE division and the nearest-entry rule verbatim.
template <int K, int DT>
__device__ __forceinline__ void exact_codes(const Raw<DT>& raw, float d, const float* cb, uint32_t* acc) {
    constexpr int EPA = K == 5 ? 4 : 8;
    float x[16];
    widen<DT>(raw, x);
#pragma unroll
    for (int e = 0; e < 16; e++) {
        const uint32_t idx = nearest_entry<1 << K>(__fdiv_rn(x[e], d), cb);
        acc[e / EPA] += spread<K>(idx) << (e % EPA);
    }
}

// Quantize the half block H held in `raw` (16 elements) and store its share of the block's
// words. Every lane of the warp must call this together (it exchanges data with its pair
// lane); `active` lanes store.
template <int K, int DT, typename AT>
__device__ __forceinline__ void quantize_half(const Raw<DT>& raw, int64_t H, bool active, const LoopCtx& c,
                                              const float* cb, AT* __restrict__ absmax,
                                              uint32_t* __restrict__ packed) {
    constexpr int NACC = K == 5 ? 4 : 2;
    // NaN-propagating block max decides between the fast and the exact path. For 16-bit
    // inputs it runs on the packed pairs (exact: the max of values of the type is one of them).
    float m;
    if constexpr (DT == F32) {
        const float* xf = reinterpret_cast<const float*>(raw.w);
        m = max3_abs_nan(xf[0], xf[1], xf[2]);
        m = max3_abs_nan(m, xf[3], xf[4]);
        m = max3_abs_nan(m, xf[5], xf[6]);
        m = max3_abs_nan(m, xf[7], xf[8]);
        m = max3_abs_nan(m, xf[9], xf[10]);
        m = max3_abs_nan(m, xf[11], xf[12]);
        m = max3_abs_nan(m, xf[13], xf[14]);
        m = max_nan(m, fabsf(xf[15]));
    } else {
        uint32_t p = pair_absmax<DT>(raw.w[0], raw.w[1]);
#pragma unroll
        for (int i = 2; i < 8; i++) p = pair_absmax<DT>(p, raw.w[i]);
        float lo, hi;
        widen_pair<DT>(p, lo, hi);
        m = max_nan(fabsf(lo), fabsf(hi));
    }
    m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, 1));
    const bool special = !(m <= 0x1p125f);          // NaN, infinite or too large for 1/d
    float amax = m;
    if (special) {   // rare: the stored absmax ignores NaN unless the whole block is NaN
        float x[16];
        widen<DT>(raw, x);
        float a = fabsf(x[0]);
#pragma unroll
        for (int e = 1; e < 16; e++) a = fmaxf(a, fabsf(x[e]));
        amax = fmaxf(a, __shfl_xor_sync(c.pair_mask, a, 1));   // both lanes of the block are here
    }
    const float d = fmaxf(amax, 1e-8f);

    uint32_t acc[NACC];
#pragma unroll
    for (int g = 0; g < NACC; g++) acc[g] = 0;
    if (!special && c.fast_cb) fast_codes<K, DT>(raw, d, c, acc);
    else exact_codes<K, DT>(raw, d, cb, acc);

    // planes 0..3 of elements 0..7 (B0) and 8..15 (B1): byte j = plane j
    uint32_t B0, B1, p4 = 0;
    if constexpr (K == 5) {
        B0 = (acc[0] & 0x0f0f0f0fu) | ((acc[1] & 0x0f0f0f0fu) << 4);
        B1 = (acc[2] & 0x0f0f0f0fu) | ((acc[3] & 0x0f0f0f0fu) << 4);
        p4 = ((acc[0] >> 4) & 0xfu) | (acc[1] & 0xf0u) | (((acc[2] >> 4) & 0xfu) << 8) | ((acc[3] & 0xf0u) << 8);
    } else {
        B0 = acc[0];
        B1 = acc[1];
    }
    // lane h holds bytes 2h, 2h+1 of every word; swap halves so it ends with words 2h, 2h+1
    const uint32_t send = prmt(B0, B1, c.sel_send);
    const uint32_t keep = prmt(B0, B1, c.sel_keep);
    const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 1);
    const uint32_t wa = prmt(keep, recv, c.sel_wa);
    const uint32_t wb = prmt(keep, recv, c.sel_wb);
    uint32_t w4 = 0;
    if constexpr (K == 5) w4 = p4 | (__shfl_xor_sync(0xffffffffu, p4, 1) << 16);

    const int64_t b = H >> 1;
    uint32_t* out = packed + b * K;
    const bool st = active && BBC_GUARD(b >= 0 && b < c.nb, kGuardQuantOut);
    if (K == 4 && c.packed_v2) {
        if (st) asm volatile("st.global.v2.u32 [%0], {%1,%2};" :: "l"(out + 2 * c.h), "r"(wa), "r"(wb) : "memory");
    } else {
        if (st && 2 * c.h < K) out[2 * c.h] = wa;
        if (st && 2 * c.h + 1 < K) out[2 * c.h + 1] = wb;
        if constexpr (K == 5) { if (st && c.h == 0) out[4] = w4; }
    }
    if (st && c.h == 0) store_absmax(absmax, b, amax);
}

// ---- one whole block (32 elements of a 16-bit type) per thread ----

// Raw words of one block of a 16-bit type (element 2i in the low half of word i).
template <int DT>
struct Raw32 { uint32_t w[16]; };

template <int DT>
__device__ __forceinline__ Raw32<DT> load_block(const void* A, int64_t b, int64_t n) {
    Raw32<DT> r;
    if (!BBC_GUARD(b >= 0 && (b + 1) * 32 <= n, kGuardQuantIn)) {
#pragma unroll
        for (int i = 0; i < 16; i++) r.w[i] = 0u;
        return r;
    }
    const char* p = reinterpret_cast<const char*>(A) + b * 64;
    const u32x8 a = ldg_stream_v8(p);
    const u32x8 q = ldg_stream_v8(p + 32);
#pragma unroll
    for (int i = 0; i < 8; i++) { r.w[i] = a.v[i]; r.w[8 + i] = q.v[i]; }
    return r;
}

// Quantize block b held in `raw` and store its K plane words and absmax (no exchange
// between lanes; the block lies entirely inside the input).
template <int K, int DT, typename AT>
__device__ __forceinline__ void quantize_block(const Raw32<DT>& raw, int64_t b, const LoopCtx& c,
                                               const float* cb, AT* __restrict__ absmax,
                                               uint32_t* __restrict__ packed) {
    constexpr int EPA = K == 5 ? 4 : 8;
    uint32_t p = pair_absmax<DT>(raw.w[0], raw.w[1]);
#pragma unroll
    for (int i = 2; i < 16; i++) p = pair_absmax<DT>(p, raw.w[i]);
    float lo, hi;
    widen_pair<DT>(p, lo, hi);
    const float m = max_nan(fabsf(lo), fabsf(hi));
    const bool special = !(m <= 0x1p125f);
    float amax = m;
    if (special) {
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; i++) {
            float x0, x1;
            widen_pair<DT>(raw.w[i], x0, x1);
            a = i == 0 ? fabsf(x0) : fmaxf(a, fabsf(x0));
            a = fmaxf(a, fabsf(x1));
        }
        amax = a;
    }
    const float d = fmaxf(amax, 1e-8f);
    // B_q: byte j = plane j of elements 8q .. 8q+7; w4: plane 4 (K = 5)
    uint32_t B[4], w4 = 0;
    const float rs = __fmul_rn(rcp_approx(d), 64.0f);
    const float d24 = __fmul_rn(d, 0x1p-24f);                  // exact: d >= 1e-8 stays normal
    const bool fast = !special && c.fast_cb;
    uint32_t sv = 0;                     // fast path: sign of v per element, element 0 shifted in first
    // K = 5 accumulates 4 elements per register: two passes of 16 keep 4 registers live
    constexpr int NPASS = K == 5 ? 2 : 1;
    constexpr int PE = 32 / NPASS;
#pragma unroll
    for (int pass = 0; pass < NPASS; pass++) {
        uint32_t acc[4] = {0u, 0u, 0u, 0u};
        if (fast) {
#pragma unroll
            for (int e = 0; e < PE; e += 2) {
                float x0, x1;
                widen_pair<DT>(raw.w[(pass * PE + e) / 2], x0, x1);
                const float2 f = __ffma2_rn(make_float2(x0, x1), make_float2(rs, rs),
                                            make_float2(12582912.0f, 12582912.0f));
                const uint2 t0 = lut8_entry(c, __float_as_uint(f.x));
                const uint2 t1 = lut8_entry(c, __float_as_uint(f.y));
                // -H * d = (sign and exponent bits of -A) * (d * 2^-24), both factors exact
                const float h0 = __uint_as_float(t0.x & 0xff800000u);
                const float h1 = __uint_as_float(t1.x & 0xff800000u);
                // (scalar FMAs: pairing them as f32x2 operations measured 2-7 points slower)
                const float v0 = __fmaf_rn(h0, d24, __fmaf_rn(__uint_as_float(t0.x), d, x0));
                const float v1 = __fmaf_rn(h1, d24, __fmaf_rn(__uint_as_float(t1.x), d, x1));
                sv = __funnelshift_l(__float_as_uint(v0), sv, 1);                         // sign bits
                sv = __funnelshift_l(__float_as_uint(v1), sv, 1);
                acc[e / EPA] += t0.y << (e % EPA);
                acc[(e + 1) / EPA] += t1.y << ((e + 1) % EPA);
            }
        } else {
#pragma unroll
            for (int e = 0; e < PE; e += 2) {
                float x0, x1;
                widen_pair<DT>(raw.w[(pass * PE + e) / 2], x0, x1);
                acc[e / EPA] += spread<K>(nearest_entry<1 << K>(__fdiv_rn(x0, d), cb)) << (e % EPA);
                acc[(e + 1) / EPA] += spread<K>(nearest_entry<1 << K>(__fdiv_rn(x1, d), cb)) << ((e + 1) % EPA);
            }
        }
        if constexpr (K == 5) {
#pragma unroll
            for (int q = 0; q < 2; q++) {
                B[2 * pass + q] = (acc[2 * q] & 0x0f0f0f0fu) | ((acc[2 * q + 1] & 0x0f0f0f0fu) << 4);
                w4 |= (((acc[2 * q] >> 4) & 0xfu) | (acc[2 * q + 1] & 0xf0u)) << (8 * (2 * pass + q));
            }
        } else {
#pragma unroll
            for (int q = 0; q < 4; q++) B[q] = acc[q];
        }
    }
    const uint32_t lo01 = prmt(B[0], B[1], 0x5140u), lo23 = prmt(B[2], B[3], 0x5140u);
    const uint32_t hi01 = prmt(B[0], B[1], 0x7362u), hi23 = prmt(B[2], B[3], 0x7362u);
    uint32_t w[5] = {prmt(lo01, lo23, 0x5410u), prmt(lo01, lo23, 0x7632u), prmt(hi01, hi23, 0x5410u),
                     prmt(hi01, hi23, 0x7632u), w4};
    if (fast) {
        // planes of L + 1 where v > 0: a bit-sliced increment (the bit-reversed signs put
        // element i at bit i; L + 1 never exceeds 2^K - 1)
        uint32_t cy = ~__brev(sv);
#pragma unroll
        for (int j = 0; j < K; j++) {
            const uint32_t carry = w[j] & cy;
            w[j] ^= cy;
            cy = carry;
        }
    }
    uint32_t* out = packed + b * K;
    // the K = 5 transpose stores the warp's 32 consecutive blocks b - lane .. b - lane + 31
    const bool st = BBC_GUARD(b >= 0 && b < c.nb && (K != 5 || (b - c.lane >= 0 && b - c.lane + 32 <= c.nb)),
                              kGuardQuantOut);
    if constexpr (K == 2) {
        if (!st) {
        } else if (c.packed_v2) asm volatile("st.global.v2.u32 [%0], {%1,%2};" :: "l"(out), "r"(w[0]), "r"(w[1]) : "memory");
        else { out[0] = w[0]; out[1] = w[1]; }
    } else if constexpr (K == 4) {
        if (!st) {
        } else if (c.packed_v4) stg_v4(out, w[0], w[1], w[2], w[3]);
        else { out[0] = w[0]; out[1] = w[1]; out[2] = w[2]; out[3] = w[3]; }
    } else if constexpr (K == 5) {
        // the warp's 32 consecutive blocks are 160 contiguous words: transposed through shared
        // memory so that each store instruction writes 128 contiguous bytes (five 4-byte stores
        // at a 20-byte lane stride left the K = 5 kernel 2-3 points slower)
        uint32_t* stg = c.stage;
#pragma unroll
        for (int j = 0; j < K; j++) stg[c.lane * K + j] = w[j];
        __syncwarp();
        uint32_t* outw = packed + (b - c.lane) * K;
#ifdef BBC_DEBUG
        const bool st_warp = __all_sync(0xffffffffu, st);
#else
        const bool st_warp = true;
#endif
        if (st_warp) {
#pragma unroll
            for (int j = 0; j < K; j++) outw[j * 32 + c.lane] = stg[j * 32 + c.lane];
        }
        __syncwarp();
    } else {
#pragma unroll
        for (int j = 0; j < K; j++)
            if (st) out[j] = w[j];
    }
    if (st) store_absmax(absmax, b, amax);
}

template <int K, int DT, bool VEC, typename AT>
__global__ void __launch_bounds__(kThreads, (kMinCtas<DT, VEC>))
kbit_quant_kernel(const void* __restrict__ A, int64_t n, const float* __restrict__ codebook,
                  AT* __restrict__ absmax, uint32_t* __restrict__ packed, int early_trigger) {
    constexpr bool WHOLE = VEC && DT != F32;                   // whole blocks per thread: 8-byte table
    __shared__ __align__(16) uint4 lut[WHOLE ? 1 : kCells * kReplicas];     // 32 KB
    __shared__ __align__(16) uint2 lut8[WHOLE ? kCells * kReplicas8 : 1];   // 32 KB
    __shared__ float cb[32];
    __shared__ float thr[33];
    __shared__ int fast_ok;
    __shared__ uint32_t stage[WHOLE && K == 5 ? kThreads * K : 1];   // per-warp store staging

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    if (early_trigger) pdl_launch_dependents();

    // Persistent grid-stride loop over whole blocks (16-bit input, 32-byte aligned) or half blocks
    // of whole blocks (no bounds checks), unrolled by two with ping-pong prefetch; then the
    // ragged last block, if any.
    const int64_t nh_full = VEC ? (n >> 5) * 2 : 0;
    const int64_t nh = ((n + 31) >> 5) * 2;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    int64_t wbase = (int64_t)blockIdx.x * kThreads + (tid & ~31);
    const int64_t bend = (n >> 5) & ~(int64_t)31;     // whole-block path: blocks of whole warp iterations

    // ---- per-CTA set-up, before griddepcontrol.wait so that it overlaps the previous kernel of
    // the stream: codebook check, thresholds, lookup table; meanwhile this warp's first two
    // iterations of input stream into L2 ----
    const float cbe = load_codebook_entry<K>(codebook);
    if (VEC && lane == 0) {
        constexpr int64_t unit = 64;                    // bytes of a block (16-bit) or half block (fp32)
        const int64_t end = WHOLE ? bend : nh_full;
        for (int i = 0; i < 2; i++) {
            const int64_t u0 = wbase + i * stride;
            if (u0 < end && BBC_GUARD((u0 + min(end - u0, (int64_t)32)) * unit <= n * dtype_size(DT), kGuardQuantIn))
                prefetch_l2(static_cast<const char*>(A) + u0 * unit, (uint32_t)(min(end - u0, (int64_t)32) * unit));
        }
    }
    bool fast_cb = setup_exact_table<K, false>(cbe, cb, thr, &fast_ok, lut, WHOLE ? lut8 : nullptr);
    pdl_wait();               // writes of the previous kernel in the stream are visible from here
    Raw32<DT> first_b;
    Raw<DT> first_h;
    if constexpr (WHOLE) {
        if (wbase < bend) first_b = load_block<DT>(A, wbase + lane, n);
    } else {
        if (wbase < nh_full) first_h = load_full<DT>(A, wbase + lane, wbase + lane < nh_full, n);
    }
    if (codebook_changed<K>(codebook, cb))                  // rare: the codebook was being written
        fast_cb = setup_exact_table<K, false>(load_codebook_entry<K>(codebook), cb, thr, &fast_ok, lut,
                                              WHOLE ? lut8 : nullptr);
    LoopCtx c;
    c.stage = stage + (WHOLE && K == 5 ? (tid & ~31) * K : 0);
    c.lane = lane;
    c.fast_cb = fast_cb;
    c.lut_c = (uint32_t)__cvta_generic_to_shared(lut) + ((uint32_t)(lane & 7) << 4) + 128u * 128u -
              0x4B400000u * 128u;                                 // mod 2^32
    c.lut8_s = (uint32_t)__cvta_generic_to_shared(lut8);
    c.lane8 = (uint32_t)(lane & (kReplicas8 - 1)) << 3;
    c.lut8_c = c.lut8_s + c.lane8 + 128u * 128u - 0x4B400000u * 128u;     // mod 2^32
    c.packed_v2 = (reinterpret_cast<uintptr_t>(packed) & 7u) == 0;
    c.packed_v4 = (reinterpret_cast<uintptr_t>(packed) & 15u) == 0;
    c.h = lane & 1;
    c.sel_send = c.h ? 0x5140u : 0x7362u;
    c.sel_keep = c.h ? 0x7362u : 0x5140u;
    c.sel_wa = c.h ? 0x1054u : 0x5410u;
    c.sel_wb = c.h ? 0x3276u : 0x7632u;
    c.pair_mask = 3u << (lane & ~1);
    c.nb = (n + 31) >> 5;

    if constexpr (WHOLE) {
        // whole warp iterations of 32 blocks, one block per thread, the next one prefetched;
        // what is left (at most the last partial iteration and a ragged block) goes by halves
        int64_t wb = wbase;                                 // in blocks
        if (K == 5 && wb < bend) {
            // K = 5: one copy of the block code in the loop and a register copy of the prefetched
            // block (two unrolled copies of its larger body stalled on instruction fetch)
            Raw32<DT> ra = first_b;
            while (true) {
                const int64_t wn = wb + stride;
                const bool more = wn < bend;
                Raw32<DT> rb;
                if (more) rb = load_block<DT>(A, wn + lane, n);
                quantize_block<K, DT, AT>(ra, wb + lane, c, cb, absmax, packed);
                wb = wn;
                if (!more) break;
                ra = rb;
            }
        } else if (wb < bend) {
            Raw32<DT> ra = first_b;
            Raw32<DT> rb;
            while (true) {
                int64_t wn = wb + stride;
                bool more = wn < bend;
                if (more) rb = load_block<DT>(A, wn + lane, n);
                quantize_block<K, DT, AT>(ra, wb + lane, c, cb, absmax, packed);
                wb = wn;
                if (!more) break;
                wn = wb + stride;
                more = wn < bend;
                if (more) ra = load_block<DT>(A, wn + lane, n);
                quantize_block<K, DT, AT>(rb, wb + lane, c, cb, absmax, packed);
                wb = wn;
                if (!more) break;
            }
        }
        c.fast_cb = false;                  // the ragged end (under one warp iteration): the rule verbatim
        for (int64_t t = 2 * bend + (int64_t)blockIdx.x * kThreads + (tid & ~31); t < nh; t += stride) {
            const Raw<DT> r = load_raw<DT, VEC>(A, n, t + lane, t + lane < nh);
            quantize_half<K, DT, AT>(r, t + lane, t + lane < nh, c, cb, absmax, packed);
        }
        return;
    }
    if (wbase < nh_full) {
        Raw<DT> ra = first_h;
        Raw<DT> rb;
        while (true) {
            rb = load_full<DT>(A, wbase + stride + lane, wbase + stride + lane < nh_full, n);
            quantize_half<K, DT, AT>(ra, wbase + lane, wbase + lane < nh_full, c, cb, absmax, packed);
            wbase += stride;
            if (wbase >= nh_full) break;
            ra = load_full<DT>(A, wbase + stride + lane, wbase + stride + lane < nh_full, n);
            quantize_half<K, DT, AT>(rb, wbase + lane, wbase + lane < nh_full, c, cb, absmax, packed);
            wbase += stride;
            if (wbase >= nh_full) break;
        }
    }
    // remaining half blocks (the ragged last block, or everything when the input is unaligned)
    for (int64_t t = nh_full + (int64_t)blockIdx.x * kThreads + (tid & ~31); t < nh; t += stride) {
        const Raw<DT> r = load_raw<DT, false>(A, n, t + lane, t + lane < nh);
        quantize_half<K, DT, AT>(r, t + lane, t + lane < nh, c, cb, absmax, packed);
    }
}

// ---- 4-bit codes with nibble packing (the inverse of the plain / nested 4-bit decode) ----
//
// A thread owns 64 bytes of input: 32 elements of a 16-bit type or 16 of fp32 (EPT), so an
// outer block of bs elements spans bs / EPT threads, and a CTA iteration covers 256 * EPT
// elements (at least one block of 4096). Per thread: two 32-byte loads (the next slice
// prefetched into registers), the NaN-propagating and the NaN-ignoring max of |x| reduced over
// the block's lanes (xor-shuffles, then shared memory for blocks wider than a warp), the exact
// threshold search per element, and EPT / 2 bytes of codes stored at once.

template <int DT> constexpr int kEpt = DT == F32 ? 16 : 32;    // elements per thread (64 bytes)

struct Raw16w { uint32_t w[16]; };

// The 64-byte slice U of A: vector loads when it lies inside the input, else element-wise
// loads with zeros past n.
template <int DT, bool VEC>
__device__ __forceinline__ Raw16w load_slice(const void* A, int64_t n, int64_t U, bool active) {
    Raw16w r;
    constexpr int E = kEpt<DT>;
    const int64_t m0 = U * E;
    if (VEC && active && m0 + E <= n) {
        const char* p = reinterpret_cast<const char*>(A) + U * 64;
        const u32x8 a = ldg_stream_v8(p), b = ldg_stream_v8(p + 32);
#pragma unroll
        for (int i = 0; i < 8; i++) { r.w[i] = a.v[i]; r.w[8 + i] = b.v[i]; }
    } else if constexpr (DT == F32) {
        const float* a = reinterpret_cast<const float*>(A);
#pragma unroll
        for (int e = 0; e < 16; e++) r.w[e] = (active && m0 + e < n) ? __float_as_uint(a[m0 + e]) : 0u;
    } else {
        const uint16_t* a = reinterpret_cast<const uint16_t*>(A);
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const uint32_t lo = (active && m0 + 2 * i < n) ? (uint32_t)a[m0 + 2 * i] : 0u;
            const uint32_t hi = (active && m0 + 2 * i + 1 < n) ? (uint32_t)a[m0 + 2 * i + 1] : 0u;
            r.w[i] = lo | (hi << 16);
        }
    }
    return r;
}

// Element e of the slice as fp32 (exact widening).
template <int DT>
__device__ __forceinline__ float slice_elem(const Raw16w& r, int e) {
    if constexpr (DT == F32) return __uint_as_float(r.w[e]);
    else {
        float lo, hi;
        widen_pair<DT>(r.w[e >> 1], lo, hi);
        return (e & 1) ? hi : lo;
    }
}

// NaN-propagating and NaN-ignoring max of |x| over the slice.
template <int DT>
__device__ __forceinline__ void slice_absmax2(const Raw16w& r, float& mnan, float& mnum) {
    if constexpr (DT == F32) {
        const float* xf = reinterpret_cast<const float*>(r.w);
        float a = fabsf(xf[0]), b = fabsf(xf[0]);
#pragma unroll
        for (int e = 1; e < 16; e++) { a = max_nan(a, fabsf(xf[e])); b = fmaxf(b, fabsf(xf[e])); }
        mnan = a; mnum = b;
    } else {
        uint32_t p = pair_absmax<DT>(r.w[0], r.w[1]), q;
        // NaN-ignoring packed max (maxNum: a NaN operand yields the other one)
        if constexpr (DT == BF16) asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(r.w[0]), "r"(r.w[1]));
        else asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(q) : "r"(r.w[0]), "r"(r.w[1]));
#pragma unroll
        for (int i = 2; i < 16; i++) {
            p = pair_absmax<DT>(p, r.w[i]);
            if constexpr (DT == BF16) asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(q), "r"(r.w[i]));
            else asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(q) : "r"(q), "r"(r.w[i]));
        }
        float lo, hi;
        widen_pair<DT>(p, lo, hi);
        mnan = max_nan(fabsf(lo), fabsf(hi));
        widen_pair<DT>(q, lo, hi);
        mnum = fmaxf(fabsf(lo), fabsf(hi));
    }
}

// Bit position of element e's nibble within its 32-bit word of codes (little-endian bytes,
// element 2j in the high nibble of byte j).
__host__ __device__ constexpr int nib_shift(int e) { return 8 * ((e & 7) >> 1) + ((e & 1) ? 0 : 4); }

template <int DT, bool VEC>
__global__ void __launch_bounds__(kThreads, 2)
quant4_kernel(const void* __restrict__ A, int64_t n, int log2_bs, const float* __restrict__ code4,
              float* __restrict__ absmax, uint8_t* __restrict__ codes, int early_trigger) {
    constexpr int E = kEpt<DT>;
    constexpr int NW = E / 8;                                   // code words per thread
    __shared__ __align__(16) uint2 lut8[kCells * kReplicas8];  // 32 KB: {-A, L}
    __shared__ uint32_t nib_spread[256];                         // bit i of a byte -> nibble i's low bit
    __shared__ float cb[32];
    __shared__ float thr[33];
    __shared__ int fast_ok;
    __shared__ float2 red[2][kThreads / 32];                    // per-warp maxima, two buffers

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    {
        uint32_t v = 0;
#pragma unroll
        for (int i = 0; i < 8; i++) v |= ((uint32_t)(tid >> i) & 1u) << nib_shift(i);
        nib_spread[tid] = v;                                     // kThreads == 256
    }
    if (early_trigger) pdl_launch_dependents();
    const int tpb_log2 = log2_bs - (DT == F32 ? 4 : 5);        // threads per outer block
    const int tpb = 1 << tpb_log2;
    const int64_t nu = (n + E - 1) / E;                         // 64-byte slices
    const int64_t nbytes = (n + 1) >> 1;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    int buf = 0;
    int64_t base = (int64_t)blockIdx.x * kThreads;
    // set-up before griddepcontrol.wait (checked after it), as in the k-bit kernel; this warp's
    // first two slices of input stream into L2 meanwhile
    const float cbe = load_codebook_entry<4>(code4);
    if (VEC && lane == 0) {
        const int64_t nfull = n / E;                            // slices entirely inside the input
        for (int i = 0; i < 2; i++) {
            const int64_t u0 = base + (tid & ~31) + i * stride;
            if (u0 < nfull && BBC_GUARD((u0 + min(nfull - u0, (int64_t)32)) * 64 <= n * dtype_size(DT), kGuardQuantIn))
                prefetch_l2(static_cast<const char*>(A) + u0 * 64, (uint32_t)(min(nfull - u0, (int64_t)32) * 64));
        }
    }
    LoopCtx c;
    c.fast_cb = setup_exact_table<4, true>(cbe, cb, thr, &fast_ok, nullptr, lut8);
    pdl_wait();               // writes of the previous kernel in the stream are visible from here
    Raw16w cur = load_slice<DT, VEC>(A, n, base + tid, base + tid < nu);
    if (codebook_changed<4>(code4, cb))                     // rare: the table was being written
        c.fast_cb = setup_exact_table<4, true>(load_codebook_entry<4>(code4), cb, thr, &fast_ok, nullptr, lut8);
    c.lut8_s = (uint32_t)__cvta_generic_to_shared(lut8);
    c.lane8 = (uint32_t)(lane & (kReplicas8 - 1)) << 3;
    c.lut8_c = c.lut8_s + c.lane8 + 128u * 128u - 0x4B400000u * 128u;     // mod 2^32

    for (; base < nu; base += stride) {                         // CTA-uniform
        const int64_t U = base + tid;
        const bool active = U < nu;
        const int64_t m0 = U * E;
        const int64_t Un = U + stride;
        const Raw16w nxt = load_slice<DT, VEC>(A, n, Un, Un < nu);
        float mnan, mnum;
        slice_absmax2<DT>(cur, mnan, mnum);
        for (int o = 1; o < tpb && o < 32; o <<= 1) {
            mnan = max_nan(mnan, __shfl_xor_sync(0xffffffffu, mnan, o));
            mnum = fmaxf(mnum, __shfl_xor_sync(0xffffffffu, mnum, o));
        }
        if (tpb > 32) {                                          // blocks wider than a warp
            if (lane == 0) red[buf][warp] = make_float2(mnan, mnum);
            __syncthreads();
            const int w0 = warp & ~((tpb >> 5) - 1);
            mnan = red[buf][w0].x; mnum = red[buf][w0].y;
            for (int w = 1; w < (tpb >> 5); w++) {
                mnan = max_nan(mnan, red[buf][w0 + w].x);
                mnum = fmaxf(mnum, red[buf][w0 + w].y);
            }
            buf ^= 1;
        }
        const bool special = !(mnan <= 0x1p125f);
        const float amax = mnum;
        const float d = fmaxf(amax, 1e-8f);

        uint32_t acc[NW];
#pragma unroll
        for (int g = 0; g < NW; g++) acc[g] = 0u;
        if (!special && c.fast_cb) {
            const float rs = __fmul_rn(rcp_approx(d), 64.0f);
            const float d24 = __fmul_rn(d, 0x1p-24f);           // exact: d >= 1e-8 stays normal
            uint32_t sv = 0;                                     // signs of v, element 0 shifted in first
#pragma unroll
            for (int e = 0; e < E; e += 2) {
                const float x0 = slice_elem<DT>(cur, e), x1 = slice_elem<DT>(cur, e + 1);
                const float2 f = __ffma2_rn(make_float2(x0, x1), make_float2(rs, rs),
                                            make_float2(12582912.0f, 12582912.0f));
                const uint2 t0 = lut8_entry(c, __float_as_uint(f.x));
                const uint2 t1 = lut8_entry(c, __float_as_uint(f.y));
                // -H * d = (sign and exponent bits of -A) * (d * 2^-24), both factors exact
                const float h0 = __uint_as_float(t0.x & 0xff800000u);
                const float h1 = __uint_as_float(t1.x & 0xff800000u);
                // (scalar FMAs: the paired f32x2 form spills here and was slower in the k-bit kernel)
                const float v0 = __fmaf_rn(h0, d24, __fmaf_rn(__uint_as_float(t0.x), d, x0));
                const float v1 = __fmaf_rn(h1, d24, __fmaf_rn(__uint_as_float(t1.x), d, x1));
                sv = __funnelshift_l(__float_as_uint(v0), sv, 1);
                sv = __funnelshift_l(__float_as_uint(v1), sv, 1);
                acc[e / 8] += t0.y << nib_shift(e);
                acc[(e + 1) / 8] += t1.y << nib_shift(e + 1);
            }
            // L + 1 where v > 0 (never beyond 15): element i's increment at bit i of ~brev(sv)
            const uint32_t inc = ~__brev(sv) >> (32 - E);
#pragma unroll
            for (int g = 0; g < NW; g++) acc[g] += nib_spread[(inc >> (8 * g)) & 0xffu];
        } else {
#pragma unroll
            for (int e = 0; e < E; e++)
                acc[e / 8] += nearest_entry<16>(__fdiv_rn(slice_elem<DT>(cur, e), d), cb) << nib_shift(e);
        }
        if (active) {
            uint8_t* cp = codes + U * (E / 2);
            if (VEC && m0 + E <= n) {
                if constexpr (NW == 4) stg_v4(cp, acc[0], acc[1], acc[2], acc[3]);
                else asm volatile("st.global.v2.u32 [%0], {%1,%2};" :: "l"(cp), "r"(acc[0]), "r"(acc[NW - 1]) : "memory");
            } else {
                // ragged end (or unaligned codes): nibbles of elements >= n are 0, bytes >= nbytes unwritten
#pragma unroll
                for (int e = 0; e < E; e++)
                    if (m0 + e >= n) acc[e / 8] &= ~(15u << nib_shift(e));
#pragma unroll
                for (int j = 0; j < E / 2; j++)
                    if (U * (E / 2) + j < nbytes) cp[j] = (uint8_t)(acc[j / 4] >> (8 * (j & 3)));
            }
            if ((tid & (tpb - 1)) == 0 &&
                BBC_GUARD((U >> tpb_log2) < ((n + (int64_t(1) << log2_bs) - 1) >> log2_bs), kGuardQuantOut))
                absmax[U >> tpb_log2] = amax;
        }
        cur = nxt;
    }
}

template <int K, int DT, typename AT>
cudaError_t launch_t(const void* A, int64_t n, const float* codebook, AT* absmax,
                     uint32_t* packed, bool vec, cudaStream_t s) {
    const int64_t nh = ((n + 31) >> 5) * 2;
    auto k = vec ? kbit_quant_kernel<K, DT, true, AT> : kbit_quant_kernel<K, DT, false, AT>;
    static std::atomic<uint64_t> carveout_set[2];
    const cudaError_t e = set_attr_once(k, carveout_set[vec], cudaFuncAttributePreferredSharedMemoryCarveout,
                                        cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int cap = resident_ctas(reinterpret_cast<const void*>(k), kThreads, 0);
    const int grid = persistent_grid(k, kThreads, 0, nh, kThreads);
    return launch_pdl(k, grid, kThreads, 0, s, A, n, codebook, absmax, packed, grid >= cap ? 1 : 0);
}

template <int K, typename AT>
cudaError_t launch_k(const void* A, int dt, int64_t n, const float* codebook, AT* absmax,
                     uint32_t* packed, bool vec, cudaStream_t s) {
    switch (dt) {
        case F16: return launch_t<K, F16>(A, n, codebook, absmax, packed, vec, s);
        case BF16: return launch_t<K, BF16>(A, n, codebook, absmax, packed, vec, s);
        default: return launch_t<K, F32>(A, n, codebook, absmax, packed, vec, s);
    }
}

template <typename AT>
cudaError_t launch_any(const void* A, int dtype, int64_t n, int K, const float* codebook, AT* absmax,
                       uint32_t* packed, bool vec, cudaStream_t s) {
    switch (K) {
        case 2: return launch_k<2>(A, dtype, n, codebook, absmax, packed, vec, s);
        case 3: return launch_k<3>(A, dtype, n, codebook, absmax, packed, vec, s);
        case 4: return launch_k<4>(A, dtype, n, codebook, absmax, packed, vec, s);
        default: return launch_k<5>(A, dtype, n, codebook, absmax, packed, vec, s);
    }
}

}  // namespace

BBC_GUARD_ACCESSOR(guard_status_kbit_quant)

cudaError_t launch_kbit_quantize(const void* A, int dtype, int64_t n, int K, const float* codebook,
                                 float* absmax, uint32_t* packed, bool vec, cudaStream_t s) {
    return launch_any(A, dtype, n, K, codebook, absmax, packed, vec, s);
}

cudaError_t launch_quantize_4bit(const void* A, int dtype, int64_t n, int log2_bs, const float* code4,
                                 float* absmax, uint8_t* codes, bool vec, cudaStream_t s) {
    auto pick = [&](auto kv, auto kn) { return vec ? kv : kn; };
    void (*k)(const void*, int64_t, int, const float*, float*, uint8_t*, int);
    switch (dtype) {
        case F16: k = pick(quant4_kernel<F16, true>, quant4_kernel<F16, false>); break;
        case BF16: k = pick(quant4_kernel<BF16, true>, quant4_kernel<BF16, false>); break;
        default: k = pick(quant4_kernel<F32, true>, quant4_kernel<F32, false>); break;
    }
    const int64_t nu = (n + 15) >> 4;                           // upper bound on 64-byte slices
    const int cap = resident_ctas(reinterpret_cast<const void*>(k), kThreads, 0);
    const int grid = persistent_grid(k, kThreads, 0, nu, kThreads);
    return launch_pdl(k, grid, kThreads, 0, s, A, n, log2_bs, code4, absmax, codes, grid >= cap ? 1 : 0);
}

cudaError_t launch_kbit_quantize_e4m4(const void* A, int dtype, int64_t n, int K, const float* codebook,
                                      uint8_t* absmax, uint32_t* packed, bool vec, cudaStream_t s) {
    return launch_any(A, dtype, n, K, codebook, absmax, packed, vec, s);
}

}  // namespace bbc
