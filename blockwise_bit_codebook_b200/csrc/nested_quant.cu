// Nested 4-bit quantize: the inverse of the nested dequant.
//
// The nested-dequant pull request ("Fuse nested 4-bit scale reconstruction on SM103") defines
// the decode: scale_b = fl(fl(code2[absmax_q[b]] * absmax2[b / 256]) + offset). Producing that
// state takes three steps here (each a stated reading of the pages):
//   1. 4-bit codes and the fp32 absmax of every outer block (quant4_kernel, kbit_quant.cu):
//      the k-bit rule of the bitsandbytes k-bit series per outer block.
//   2. offset = the mean of the outer absmax: a pairwise binary64 sum over the values
//      zero-padded to a power of two (each tree node the sum of its two halves), divided by
//      the block count, rounded once to fp32 (tree_sum_kernel). IEEE addition is commutative
//      and adding +0.0 is exact, so a CTA that sums 8 leaves per thread as a tree, combines
//      lanes by xor-shuffles and warps in shared memory computes exactly the nodes of that
//      tree; each level of 2048 nodes is one launch.
//   3. per group of 256 outer blocks, c_b = fl(absmax_b - offset): absmax2 = max |c_b| and
//      absmax_q_b = the first nearest General8 entry to fl(c_b / fmaxf(absmax2, 1e-8f)) (the
//      quotient correctly rounded from one reciprocal per group and Markstein's correction)
//      (absmax_compress_kernel). For a strictly ascending table whose neighbouring gaps are
//      within a factor 2^20 of each other (the fast form; the General8 stand-in and tables built
//      by decades are) the first nearest entry is the number of switch points D_i <= xn, D_i the
//      smallest fp32 at which t_i beats t_{i-1} in fp32 distances, found per CTA by bisection
//      over ordered keys; a bucket table (64 buckets per binade of |xn| from 2^-24 up to 1)
//      holds per bucket the switch points below it and the first one inside it, so a value
//      costs one table read and one comparison. Other ascending tables take an exact search:
//      p = the last index with t_p <= xn: fl(|xn - t_i|) does not increase up to t_p and does
//      not decrease after it, so the minimum is at t_p or t_{p+1} and the first index holding
//      it is found by walking down a plateau of equal distances; p comes from the same buckets
//      holding the entries and a forward scan (comparisons t_p <= xn are exact). Any other table
//      takes the rule verbatim over all 256 entries.
#include <algorithm>
#include <cfloat>
#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kTree = 2048;            // tree leaves per CTA (256 threads x 8)
constexpr int kGroup = 256;            // outer blocks per inner absmax

// Leaves [base, base + 8) of a node (zeros past count) summed as a tree, with vector loads when
// all eight lie inside (base is a multiple of 8 and the values 16-byte aligned).
__device__ __forceinline__ double leaf8(const float* __restrict__ in, int64_t count, int64_t base) {
    double v[8];
    if (base + 8 <= count) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(in + base));
        const float4 b = __ldg(reinterpret_cast<const float4*>(in + base + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
        for (int j = 0; j < 8; j++) v[j] = base + j < count ? (double)in[base + j] : 0.0;
    }
    return __dadd_rn(__dadd_rn(__dadd_rn(v[0], v[1]), __dadd_rn(v[2], v[3])),
                     __dadd_rn(__dadd_rn(v[4], v[5]), __dadd_rn(v[6], v[7])));
}

__device__ __forceinline__ double leaf8(const double* __restrict__ in, int64_t count, int64_t base) {
    double v[8];
    if (base + 8 <= count) {
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const double2 a = __ldg(reinterpret_cast<const double2*>(in + base + j));
            v[j] = a.x; v[j + 1] = a.y;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; j++) v[j] = base + j < count ? in[base + j] : 0.0;
    }
    return __dadd_rn(__dadd_rn(__dadd_rn(v[0], v[1]), __dadd_rn(v[2], v[3])),
                     __dadd_rn(__dadd_rn(v[4], v[5]), __dadd_rn(v[6], v[7])));
}

// Node `blk` of one level of the pairwise sum: in[2048 blk .. 2048 blk + 2048) (zeros past
// count) summed as a binary tree by the whole CTA (8 leaves per thread as a tree, lanes by
// xor-shuffles, warps in shared memory); the result is returned to every thread.
template <typename T>
__device__ __forceinline__ double tree_node(const T* __restrict__ in, int64_t count, int64_t blk, double* ws) {
    double s = leaf8(in, count, blk * kTree + threadIdx.x * 8);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
    __syncthreads();                                            // ws may hold a previous use
    if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = s;
    __syncthreads();
    return __dadd_rn(__dadd_rn(__dadd_rn(ws[0], ws[1]), __dadd_rn(ws[2], ws[3])),
                     __dadd_rn(__dadd_rn(ws[4], ws[5]), __dadd_rn(ws[6], ws[7])));
}

// One level of the pairwise sum below the root: node b = the tree of in[2048 b .. 2048 b + 2048),
// kNodesPerCta consecutive nodes per CTA (their loads all in flight together), each summed
// exactly as tree_node does.
constexpr int kNodesPerCta = 4;

template <typename T>
__global__ void __launch_bounds__(256)
tree_sum_kernel(const T* __restrict__ in, int64_t count, int64_t nnodes, double* __restrict__ nodes) {
    __shared__ double ws[kNodesPerCta][8];
    // (no early trigger: letting the compression's CTAs in beside these ones to run their table
    // set-up measured 2-4 us slower at 4.2 M outer blocks)
    pdl_wait();               // the values come from the launch just before this one
    double s[kNodesPerCta];
#pragma unroll
    for (int k = 0; k < kNodesPerCta; k++)
        s[k] = leaf8(in, count, ((int64_t)blockIdx.x * kNodesPerCta + k) * kTree + threadIdx.x * 8);
#pragma unroll
    for (int k = 0; k < kNodesPerCta; k++) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) s[k] = __dadd_rn(s[k], __shfl_xor_sync(0xffffffffu, s[k], o));
        if ((threadIdx.x & 31) == 0) ws[k][threadIdx.x >> 5] = s[k];
    }
    __syncthreads();
    const int k = threadIdx.x;
    const int64_t blk = (int64_t)blockIdx.x * kNodesPerCta + k;
    if (k < kNodesPerCta && blk < nnodes)
        nodes[blk] = __dadd_rn(__dadd_rn(__dadd_rn(ws[k][0], ws[k][1]), __dadd_rn(ws[k][2], ws[k][3])),
                               __dadd_rn(__dadd_rn(ws[k][4], ws[k][5]), __dadd_rn(ws[k][6], ws[k][7])));
}

// The General8 table in shared memory as 32 lane-interleaved replicas (entry i of replica r at
// i * 32 + r): each lane reads its own replica, so the data-dependent probes of a binary search
// never conflict. `t` below is a lane's replica base; entry i is t[i * kRep].
constexpr int kRep = 32;

// Buckets of the scaled value xn (|xn| <= 1 or NaN): 64 per binade of |xn| from 2^-24
// (M(k) = the float with bits (k + kLutE0) << 17 is the lower edge of magnitude bucket k; all
// smaller magnitudes fall in bucket 0), negative values first in ascending order of value:
// bucket 1536 - k holds the negatives of magnitude in [M(k), M(k + 1)) and its lower point is
// -M(k + 1); bucket 1537 + k holds the positives in [M(k), M(k + 1)) and its lower point is
// M(k) (0 for k = 0). lut[j] = base | cnt << 9: base = #{i : t_i <= lower point of bucket j}
// (0..256) and cnt = min(#{i : t_i above it and at or below the next bucket's}, 127), which
// bounds the forward scan from base - 1 for any xn in the bucket.
constexpr int kLutShift = 17;
constexpr int kLutE0 = (127 - 24) << (23 - kLutShift);
constexpr int kLutHalf = 24 << (23 - kLutShift);                // magnitude buckets 0..1536
constexpr int kLutN = 2 * kLutHalf + 2;                         // 3074 buckets

// Bucket of a value with |xn| <= 1 (NaN lands anywhere; the caller overrides it).
__device__ __forceinline__ int lut_bucket(float xn) {
    const uint32_t b = __float_as_uint(xn);
    const int k = min(max((int)((b << 1) >> (kLutShift + 1)) - kLutE0, 0), kLutHalf);
    // kLutHalf - k for a set sign bit (k ^ -1 = -k - 1), kLutHalf + 1 + k otherwise
    return kLutHalf + 1 + (k ^ ((int)b >> 31));
}

// First bucket whose lower point is >= x (kLutN if none), for any float x.
__device__ __forceinline__ int lut_first_at_or_above(float x) {
    const uint32_t b = __float_as_uint(x);
    const int k = (int)((b & 0x7fffffffu) >> kLutShift) - kLutE0;   // M(k) <= |x| < M(k + 1) if k >= 0
    if (x != x) return kLutN;
    if (b >> 31) return max(kLutHalf + 1 - max(k, 0), 0);     // -M(mb + 1) >= x  <=>  mb + 1 <= k
    if (b == 0) return kLutHalf + 1;
    const bool edge = (b & ((1u << kLutShift) - 1)) == 0 && k >= 1;    // x == M(k)
    return min(kLutHalf + 1 + max(edge ? k : k + 1, 1), kLutN);         // least M(mb) >= x
}

// First index minimising fl(|xn - t_i|) over an ascending 256-entry table (see the header).
// The common path has no branch, so the eight values a lane handles overlap their table reads.
__device__ __forceinline__ uint32_t nearest_ascending(float xn, const float* t, const uint16_t* lut) {
    const uint32_t e = lut[lut_bucket(xn)];
    // p = the last index with t_p <= xn: the bucket's base less one, then a forward scan over
    // the at most e >> 9 entries inside the bucket (one step unconditionally, more rarely)
    int p = xn != xn ? -1 : (int)(e & 511u) - 1;
    p += (p < 255 && t[min(p + 1, 255) * kRep] <= xn) ? 1 : 0;
    if ((e >> 9) > 1)
        while (p < 255 && t[(p + 1) * kRep] <= xn) p++;
    // The first nearest entry is t[p] or t[p + 1]. With p clamped to 0 the same selects give 0
    // when no entry is <= xn (t[1] is never strictly closer than t[0] below t[0]) and for a NaN
    // xn (no comparison holds); at p = 255 the clamped neighbour is t[255] itself.
    const int q = max(p, 0), r = min(q + 1, 255);
    const float dq = fabsf(__fsub_rn(xn, t[q * kRep]));
    const float dr = fabsf(__fsub_rn(xn, t[r * kRep]));
    // walk down a plateau of equal distances below q (equal entries, or distances that round
    // alike: rare)
    int i = q;
    if (q > 0 && fabsf(__fsub_rn(xn, t[max(q - 1, 0) * kRep])) == dq) {
        i--;
        while (i > 0 && fabsf(__fsub_rn(xn, t[(i - 1) * kRep])) == dq) i--;
    }
    return (uint32_t)(dr < dq ? r : i);
}

__device__ __forceinline__ uint32_t nearest_any(float xn, const float* t) {
    float best = __int_as_float(0x7f800000);
    uint32_t idx = 0;
    for (int i = 0; i < 256; i++) {
        const float dist = fabsf(__fsub_rn(xn, t[i * kRep]));
        if (dist < best) { best = dist; idx = (uint32_t)i; }
    }
    return idx;
}

// Switch point of the exact rule between neighbouring entries a < b of a strictly ascending
// table: the smallest fp32 xn in (a, b] at which b is strictly nearer, fl(b - xn) < fl(xn - a).
// Both rounded distances are monotone in xn, so the comparison is false at a, true at b and
// changes once in between; a bisection over the ordered keys finds the change (at most 32 steps,
// from a checked bracket 4).
__device__ __forceinline__ float switch_point(float a, float b) {
    uint32_t lo = okey(a), hi = okey(b);
    // The change usually lies within a few ulps of the midpoint: a bracket of 16 keys around it,
    // taken only if the comparison is false at its low end and true at its high end, leaves four
    // steps (near zero, or across binades, the whole interval is searched).
    const uint32_t c = okey(__double2float_rn(0.5 * ((double)a + (double)b)));   // finite: no wrap below
    const uint32_t l2 = max(lo, c - 8u), h2 = min(hi, c + 8u);
    const float vl = okey_f32(l2), vh = okey_f32(h2);
    if (l2 < h2 && !(__fsub_rn(b, vl) < __fsub_rn(vl, a)) && __fsub_rn(b, vh) < __fsub_rn(vh, a)) {
        lo = l2;
        hi = h2;
    }
    while (hi - lo > 1u) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        const float v = okey_f32(mid);
        if (__fsub_rn(b, v) < __fsub_rn(v, a)) hi = mid; else lo = mid;
    }
    return okey_f32(hi);
}

// First nearest entry from the switch-point table (the fast form): the index is the number of
// switch points at or below xn; ent[bucket] = {the first switch point above the bucket's lower
// point (+inf if none), base | min(cnt, 127) << 9} with base the switch points at or below that
// point and cnt those up to the next bucket's; dsw[1..255] the switch points. A NaN xn takes 0
// (no comparison of the verbatim rule holds, so its first entry stays).
__device__ __forceinline__ uint32_t nearest_fast(float xn, const uint2* ent, const float* dsw) {
    const uint2 e = ent[lut_bucket(xn)];
    uint32_t idx = (e.y & 511u) + (xn >= __uint_as_float(e.x) ? 1u : 0u);
    if (e.y >= (2u << 9))                                       // two or more in the bucket: rare
        while (idx < 255u && xn >= dsw[idx + 1]) idx++;
    return xn == xn ? idx : 0u;
}

// One warp per group of 256 outer blocks (8 consecutive ones per lane), persistent over the
// groups; every CTA first forms the offset from the last level of the tree.
//
// Table forms (CTA-uniform, decided from the General8 table alone):
//  * fast: finite, strictly ascending, every two neighbouring gaps within a factor 2^20 of each
//    other, and, when the last entry is below 1, a last gap of at least 2^-20 (1 + |t_254|).
//    For xn in [t_{i-1}, t_i] the rounded distance to any other entry then exceeds the smaller
//    of the two neighbours' (a gap g beyond a distance below g' >= 2^-20 g exceeds an ulp of
//    their sum), so the verbatim rule picks i - 1 or i, by the switch point D_i; below t_0 it
//    picks 0 (ties go to the first index) and above t_255 (up to xn = 1) entry 255. Hence
//    index = #{i : D_i <= xn}.
//  * ascending otherwise: nearest_ascending over 32 replicas of the table and the 16-bit bucket
//    table of the entries.
//  * anything else: the verbatim rule over all 256 entries.
template <typename T>
__global__ void __launch_bounds__(256)
absmax_compress_kernel(const float* __restrict__ absmax, int64_t nbo, const T* __restrict__ root_in,
                       int64_t root_count, float* __restrict__ offset_p,
                       const float* __restrict__ code2, uint8_t* __restrict__ absmax_q,
                       float* __restrict__ absmax2) {
    // 32 KB: the 32 replicas of the table, or (fast form) the bucket entries and switch points
    __shared__ __align__(16) float tr[256 * kRep];
    static_assert(2 * kLutN + 257 <= 256 * kRep, "bucket entries and switch points fit");
    __shared__ uint32_t hist[kLutN + 1];                        // then the 16-bit bucket table
    __shared__ uint32_t warp_sum[8];
    uint2* const ent = reinterpret_cast<uint2*>(tr);            // 8-byte aligned: tr is 16-byte aligned
    float* const dsw = tr + 2 * kLutN;                          // D_i at dsw[i], i = 1 .. 255
    uint16_t* const lut = reinterpret_cast<uint16_t*>(hist);
    const int tid = threadIdx.x;
    const float v = code2[tid];
    const float prev = tid > 0 ? code2[tid - 1] : v;
    const float next = tid < 255 ? code2[tid + 1] : v;
    const bool ascending = __syncthreads_and(v <= next);        // false if any entry is NaN
    bool ok = fabsf(v) <= FLT_MAX && (tid == 255 || v < next);
    if (tid > 0 && tid < 255) {
        // fp64 gaps: exact to 2^-53 relative, far inside the factor-4 margin of the bound used
        const double g0 = (double)v - (double)prev, g1 = (double)next - (double)v;
        ok = ok && g0 >= 0x1p-20 * g1 && g1 >= 0x1p-20 * g0;
    }
    if (tid == 255 && v < 1.0f) ok = ok && (double)v - (double)prev >= 0x1p-20 * (1.0 + fabs((double)prev));
    const bool fast = __syncthreads_and(ok) != 0;
    // the value this thread enters into the bucket histogram: its switch point, or its entry
    float key = v;
    if (fast) {
        if (tid > 0) {
            key = switch_point(prev, v);
            dsw[tid] = key;
        }
    } else {
        // entry i's 32 replicas are 128 contiguous bytes: 8 rotated 16-byte stores per thread (the
        // 8 threads of a store phase write 8 different 16-byte columns, so no bank is hit twice)
        static_assert(kRep == 32, "one entry is 8 float4 columns");
        const float4 v4 = make_float4(v, v, v, v);
#pragma unroll
        for (int k = 0; k < 8; k++)
            reinterpret_cast<float4*>(tr)[tid * 8 + ((k + tid) & 7)] = v4;
    }
    // Bucket table from a histogram: h[J] = #{keys whose first bucket at or above them is J}
    // (J = kLutN: above every bucket); with S its inclusive prefix sum, bucket j's base is S(j)
    // (the keys at or below its lower point) and h[j + 1] = S(j + 1) - S(j) the keys inside it.
    // Thread k owns slots [13k, 13k + 13) of the prefix sum. Meaningful only for an ascending
    // table (the keys then ascend too).
    constexpr int kSlots = 13;
    static_assert(kSlots * 256 >= kLutN + 1, "every slot has an owner");
    {
        const int s0 = tid * kSlots;
#pragma unroll
        for (int k = 0; k < kSlots; k++)
            if (s0 + k <= kLutN) hist[s0 + k] = 0;
        __syncthreads();                                        // also: the switch points are visible
        if (!fast || tid > 0) atomicAdd(&hist[lut_first_at_or_above(key)], 1u);
        __syncthreads();
        uint32_t h[kSlots + 1];
#pragma unroll
        for (int k = 0; k <= kSlots; k++) h[k] = s0 + k <= kLutN ? hist[s0 + k] : 0u;
        uint32_t run = 0;                                        // total over own slots
#pragma unroll
        for (int k = 0; k < kSlots; k++) run += h[k];
        uint32_t x = run;                                        // inclusive scan of thread totals
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if ((tid & 31) >= o) x += y;
        }
        if ((tid & 31) == 31) warp_sum[tid >> 5] = x;
        __syncthreads();                                         // also: every read of hist is done
        uint32_t sum = x - run;
        for (int w = 0; w < (tid >> 5); w++) sum += warp_sum[w];
#pragma unroll
        for (int k = 0; k < kSlots; k++) {
            sum += h[k];
            if (s0 + k < kLutN) {
                const uint32_t e = sum | min(h[k + 1], 127u) << 9;
                if (fast)        // a bucket with keys inside holds the first of them (sum + 1 <= 255)
                    ent[s0 + k] = make_uint2(h[k + 1] ? __float_as_uint(dsw[sum + 1]) : 0x7f800000u, e);
                else
                    lut[s0 + k] = (uint16_t)e;
            }
        }
    }
    __syncthreads();                                            // the tables are complete
    // Everything above reads only the General8 table, an input written before the quantize's
    // first launch; the outer absmax and the tree nodes below come from the launches just before
    // this one (programmatic dependent launch: this set-up overlaps their end).
    pdl_wait();
    const float* t = tr + (tid & (kRep - 1));
    const int lane = tid & 31;
    const int64_t ngroups = (nbo + kGroup - 1) / kGroup;
    const int64_t nfull = nbo / kGroup;
    const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t g0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (tid >> 5);
    const bool q_vec = (reinterpret_cast<uintptr_t>(absmax_q) & 7u) == 0;
    // A full group's 8 absmax values of this lane: two 16-byte loads (absmax is 256-byte aligned).
    auto load_full = [&](int64_t g, float4& x0, float4& x1) {
        if (!BBC_GUARD(g >= 0 && (g + 1) * kGroup <= nbo, kGuardCompress)) return;
        const float* p = absmax + g * kGroup + lane * 8;
        x0 = __ldg(reinterpret_cast<const float4*>(p));
        x1 = __ldg(reinterpret_cast<const float4*>(p + 4));
    };
    // the first full group's values go out before the root is formed, so the loads overlap
    const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float4 n0 = z, n1 = z;
    if (g0 < nfull) load_full(g0, n0, n1);
    // the offset: the root of the pairwise tree over the last level (<= 2048 values), the
    // same in every CTA; CTA 0 stores it
    __shared__ double ws[8];
    const float off = __double2float_rn(__ddiv_rn(tree_node(root_in, root_count, 0, ws), (double)nbo));
    if (blockIdx.x == 0 && tid == 0) *offset_p = off;
    // one group: FULL groups (all 256 blocks inside nbo) need no bounds checks and take their
    // values from x0, x1; FORM is the table form (0 fast, 1 ascending, 2 any), uniform over the
    // kernel
    auto group = [&](int64_t g, auto full, auto form, float4 x0, float4 x1) {
        constexpr bool FULL = decltype(full)::value;
        constexpr int FORM = decltype(form)::value;
        const int64_t b0 = g * kGroup + lane * 8;
        float cv[8];
        if constexpr (FULL) {
            const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
            for (int j = 0; j < 8; j++) cv[j] = __fsub_rn(xs[j], off);
        } else {
#pragma unroll
            for (int j = 0; j < 8; j++)
                cv[j] = b0 + j < nbo ? __fsub_rn(__ldg(absmax + b0 + j), off) : __int_as_float(0x7fc00000);
        }
        float m = __int_as_float(0x7fc00000);                   // NaN: ignored by fmaxf
#pragma unroll
        for (int j = 0; j < 8; j++) m = fmaxf(m, fabsf(cv[j]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0 && BBC_GUARD(g >= 0 && g < ngroups, kGuardCompress)) absmax2[g] = m;
        const float d = fmaxf(m, 1e-8f);
        // xn = RN(c / d) from the correctly rounded reciprocal y: q0 = RN(c y), r = c - d q0 (exact
        // by the fma), xn = RN(q0 + r y) is the correctly rounded quotient by Markstein's theorem
        // (y within half an ulp of 1/d, q0 within one ulp of c / d, no underflow); zero, tiny and
        // NaN quotients take the IEEE division instead
        // (the rare cases are collected per warp and handled behind one vote, off the common path)
        const float y = __frcp_rn(d);
        float xn[8];
        bool rare = false;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const float q0 = __fmul_rn(cv[j], y);
            xn[j] = __fmaf_rn(__fmaf_rn(-d, q0, cv[j]), y, q0);
            rare |= !(fabsf(q0) >= 0x1p-100f);
        }
        if (__any_sync(0xffffffffu, rare)) {
#pragma unroll
            for (int j = 0; j < 8; j++)
                if (!(fabsf(__fmul_rn(cv[j], y)) >= 0x1p-100f)) xn[j] = __fdiv_rn(cv[j], d);
        }
        uint32_t q[8];
        if constexpr (FORM == 0) {
            // one table read and one comparison per value; buckets holding two or more switch
            // points and NaN quotients redo the value through nearest_fast
            bool redo = false;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const uint2 e = ent[lut_bucket(xn[j])];
                q[j] = (e.y & 511u) + (xn[j] >= __uint_as_float(e.x) ? 1u : 0u);
                redo |= e.y >= (2u << 9) || xn[j] != xn[j];
            }
            if (__any_sync(0xffffffffu, redo)) {
#pragma unroll
                for (int j = 0; j < 8; j++) q[j] = nearest_fast(xn[j], ent, dsw);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; j++) q[j] = FORM == 1 ? nearest_ascending(xn[j], t, lut) : nearest_any(xn[j], t);
        }
        if (FULL && q_vec) {
            const uint32_t w0 = q[0] | q[1] << 8 | q[2] << 16 | q[3] << 24;
            const uint32_t w1 = q[4] | q[5] << 8 | q[6] << 16 | q[7] << 24;
            if (BBC_GUARD(b0 + 8 <= nbo, kGuardCompress))
                asm volatile("st.global.v2.u32 [%0], {%1,%2};" :: "l"(absmax_q + b0), "r"(w0), "r"(w1) : "memory");
        } else {
#pragma unroll
            for (int j = 0; j < 8; j++)
                if ((FULL && BBC_GUARD(b0 + j < nbo, kGuardCompress)) || b0 + j < nbo) absmax_q[b0 + j] = (uint8_t)q[j];
        }
    };
    using Fast = std::integral_constant<int, 0>;
    using Asc = std::integral_constant<int, 1>;
    using Any = std::integral_constant<int, 2>;
    int64_t g = g0;
    // full groups with the next group's values in flight, then the partial last group
    auto run = [&](auto form) {
        for (; g < nfull; g += wstride) {
            const float4 c0 = n0, c1 = n1;
            if (g + wstride < nfull) load_full(g + wstride, n0, n1);
            group(g, std::true_type{}, form, c0, c1);
        }
        for (; g < ngroups; g += wstride) group(g, std::false_type{}, form, z, z);
    };
    if (fast) run(Fast{});
    else if (ascending) run(Asc{});
    else for (; g < ngroups; g += wstride) group(g, std::false_type{}, Any{}, z, z);
}

}  // namespace

BBC_GUARD_ACCESSOR(guard_status_nested_quant)

namespace {
int64_t tree_nodes(int64_t count) { return (count + kTree - 1) / kTree; }
int64_t absmax_bytes(int64_t nbo) { return ((nbo * 4 + 255) / 256) * 256; }
int64_t even(int64_t x) { return x + (x & 1); }                // keeps the second node buffer 16-byte aligned
}  // namespace

size_t nested_quant_workspace_bytes(int64_t n, int log2_bs) {
    const int64_t nbo = (n + (1ll << log2_bs) - 1) >> log2_bs;
    const int64_t s1 = tree_nodes(nbo), s2 = tree_nodes(s1);
    return (size_t)(absmax_bytes(nbo) + (even(s1) + s2) * 8);
}

cudaError_t launch_quantize_4bit_nested(const void* A, int dtype, int64_t n, int log2_bs, const float* code4,
                                        const float* code2, uint8_t* codes, uint8_t* absmax_q, float* absmax2,
                                        float* offset, void* workspace, bool vec, cudaStream_t s) {
    const int64_t nbo = (n + (1ll << log2_bs) - 1) >> log2_bs;
    float* absmax = static_cast<float*>(workspace);
    double* buf_a = reinterpret_cast<double*>(static_cast<char*>(workspace) + absmax_bytes(nbo));
    double* buf_b = buf_a + even(tree_nodes(nbo));
    cudaError_t e = launch_quantize_4bit(A, dtype, n, log2_bs, code4, absmax, codes, vec, s);
    if (e != cudaSuccess) return e;
    // the pairwise sum: one launch per level while more than 2048 values remain; the root (at
    // most 2048 values) is formed by every CTA of the compression kernel
    const int64_t ngroups = (nbo + kGroup - 1) / kGroup;
    if (nbo <= kTree) {
        const int grid = std::min(persistent_grid(absmax_compress_kernel<float>, 256, 0, ngroups, 32), 2 * sm_count());
        return launch_pdl(absmax_compress_kernel<float>, grid, 256, 0, s, absmax, nbo, absmax, nbo, offset, code2,
                          absmax_q, absmax2);
    }
    int64_t count = tree_nodes(nbo);
    e = launch_pdl(tree_sum_kernel<float>, (unsigned)((count + kNodesPerCta - 1) / kNodesPerCta), 256, 0, s, absmax,
                   nbo, count, buf_a);
    if (e != cudaSuccess) return e;
    const double* in = buf_a;
    double* out = buf_b;
    while (count > kTree) {
        const int64_t next = tree_nodes(count);
        e = launch_pdl(tree_sum_kernel<double>, (unsigned)((next + kNodesPerCta - 1) / kNodesPerCta), 256, 0, s, in,
                       count, next, out);
        if (e != cudaSuccess) return e;
        in = out;
        out = out == buf_b ? buf_a : buf_b;        // a level never outgrows the one before it
        count = next;
    }
    // at least 32 groups per CTA (4 per warp) amortise the per-CTA table set-up; persistent
    // above that, two CTAs per SM (every SM the same share; more CTAs only repeat the set-up)
    const int grid = std::min(persistent_grid(absmax_compress_kernel<double>, 256, 0, ngroups, 32), 2 * sm_count());
    return launch_pdl(absmax_compress_kernel<double>, grid, 256, 0, s, absmax, nbo, in, count, offset, code2, absmax_q,
                      absmax2);
}

}  // namespace bbc
