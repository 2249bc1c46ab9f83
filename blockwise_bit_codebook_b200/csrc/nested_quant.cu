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
//      (absmax_compress_kernel). For an ascending table the nearest entry is found exactly from
//      p = the last index with t_p <= xn: fl(|xn - t_i|) does not increase up to t_p and does
//      not decrease after it, so the minimum is at t_p or t_{p+1} and the first index holding
//      it is found by walking down a plateau of equal distances. p itself comes from a table of
//      its values at the lower ends of 64 buckets per binade of |xn| (from 2^-24 up to 1) and a
//      forward scan inside the bucket; comparisons t_p <= xn are exact, so this is the same p a
//      search over all entries gives. Any other table takes the rule verbatim over all 256
//      entries.
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
    const int k = min(max((int)((b & 0x7fffffffu) >> kLutShift) - kLutE0, 0), kLutHalf);
    return (b >> 31) ? kLutHalf - k : kLutHalf + 1 + k;
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

// One warp per group of 256 outer blocks (8 per lane), persistent over the groups; every CTA
// first forms the offset from the last level of the tree.
template <typename T>
__global__ void __launch_bounds__(256)
absmax_compress_kernel(const float* __restrict__ absmax, int64_t nbo, const T* __restrict__ root_in,
                       int64_t root_count, float* __restrict__ offset_p,
                       const float* __restrict__ code2, uint8_t* __restrict__ absmax_q,
                       float* __restrict__ absmax2) {
    __shared__ __align__(16) float tr[256 * kRep];              // 32 KB
    const float v = code2[threadIdx.x];
    const float next = threadIdx.x < 255 ? code2[threadIdx.x + 1] : v;
    // entry i's 32 replicas are 128 contiguous bytes: 8 rotated 16-byte stores per thread (the 8
    // threads of a store phase write 8 different 16-byte columns, so no bank is hit twice)
    static_assert(kRep == 32, "one entry is 8 float4 columns");
    const float4 v4 = make_float4(v, v, v, v);
#pragma unroll
    for (int k = 0; k < 8; k++)
        reinterpret_cast<float4*>(tr)[threadIdx.x * 8 + ((k + threadIdx.x) & 7)] = v4;
    // bucket table from a histogram: h[J] = #{i : first bucket at or above t_i is J} (J = kLutN:
    // above every bucket); with S its inclusive prefix sum, bucket j's base is S(j) (the entries
    // at or below its lower point) and h[j + 1] = S(j + 1) - S(j) the entries inside it. Thread k
    // owns slots [13k, 13k + 13) of the prefix sum. Meaningful only for an ascending table.
    constexpr int kSlots = 13;
    static_assert(kSlots * 256 >= kLutN + 1, "every slot has an owner");
    __shared__ uint32_t hist[kLutN + 1];                        // then the table, as 16-bit entries
    __shared__ uint32_t warp_sum[8];
    uint16_t* const lut = reinterpret_cast<uint16_t*>(hist);
    {
        const int s0 = threadIdx.x * kSlots;
#pragma unroll
        for (int k = 0; k < kSlots; k++)
            if (s0 + k <= kLutN) hist[s0 + k] = 0;
        __syncthreads();
        atomicAdd(&hist[lut_first_at_or_above(v)], 1u);
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
            if ((threadIdx.x & 31) >= o) x += y;
        }
        if ((threadIdx.x & 31) == 31) warp_sum[threadIdx.x >> 5] = x;
        __syncthreads();                                         // also: every read of hist is done
        uint32_t sum = x - run;
        for (int w = 0; w < (int)(threadIdx.x >> 5); w++) sum += warp_sum[w];
#pragma unroll
        for (int k = 0; k < kSlots; k++) {
            sum += h[k];
            if (s0 + k < kLutN) lut[s0 + k] = (uint16_t)(sum | min(h[k + 1], 127u) << 9);
        }
    }
    // the barrier also makes the replicas and the bucket table visible
    const bool ascending = __syncthreads_and(v <= next);        // false if any entry is NaN
    // Everything above reads only the General8 table, an input written before the quantize's
    // first launch; the outer absmax and the tree nodes below come from the launches just before
    // this one (programmatic dependent launch: this set-up overlaps their end).
    pdl_wait();
    const float* t = tr + (threadIdx.x & (kRep - 1));
    // the offset: the root of the pairwise tree over the last level (<= 2048 values), the
    // same in every CTA; CTA 0 stores it
    __shared__ double ws[8];
    const float off = __double2float_rn(__ddiv_rn(tree_node(root_in, root_count, 0, ws), (double)nbo));
    if (blockIdx.x == 0 && threadIdx.x == 0) *offset_p = off;
    const int lane = threadIdx.x & 31;
    const int64_t ngroups = (nbo + kGroup - 1) / kGroup;
    const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
    // one group: FULL groups (all 256 blocks inside nbo) need no bounds checks; ASC selects the
    // search (uniform over the kernel)
    auto group = [&](int64_t g, auto full, auto asc) {
        constexpr bool FULL = decltype(full)::value;
        constexpr bool ASC = decltype(asc)::value;
        float cv[8];
        float m = __int_as_float(0x7fc00000);                   // NaN: ignored by fmaxf
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int64_t b = g * kGroup + lane + 32 * j;
            cv[j] = (FULL || b < nbo) ? __fsub_rn(__ldg(absmax + b), off) : __int_as_float(0x7fc00000);
            m = fmaxf(m, fabsf(cv[j]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) absmax2[g] = m;
        const float d = fmaxf(m, 1e-8f);
        // xn = RN(c / d) from the correctly rounded reciprocal y: q0 = RN(c y), r = c - d q0 (exact
        // by the fma), xn = RN(q0 + r y) is the correctly rounded quotient by Markstein's theorem
        // (y within half an ulp of 1/d, q0 within one ulp of c / d, no underflow); zero, tiny and
        // NaN quotients take the IEEE division instead
        const float y = __frcp_rn(d);
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int64_t b = g * kGroup + lane + 32 * j;
            if (FULL || b < nbo) {
                const float q0 = __fmul_rn(cv[j], y);
                float xn = __fmaf_rn(__fmaf_rn(-d, q0, cv[j]), y, q0);
                if (!(fabsf(q0) >= 0x1p-100f)) xn = __fdiv_rn(cv[j], d);
                absmax_q[b] = (uint8_t)(ASC ? nearest_ascending(xn, t, lut) : nearest_any(xn, t));
            }
        }
    };
    const int64_t nfull = nbo / kGroup;
    const int64_t g0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (ascending) {
        for (int64_t g = g0; g < ngroups; g += wstride) {
            if (g < nfull) group(g, std::true_type{}, std::true_type{});
            else group(g, std::false_type{}, std::true_type{});
        }
    } else {
        for (int64_t g = g0; g < ngroups; g += wstride) group(g, std::false_type{}, std::false_type{});
    }
}

}  // namespace

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
        const int grid = persistent_grid(absmax_compress_kernel<float>, 256, 0, ngroups, 32);
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
    // 32 groups per CTA (4 per warp) amortise the 32 KB table set-up; persistent above that
    const int grid = persistent_grid(absmax_compress_kernel<double>, 256, 0, ngroups, 32);
    return launch_pdl(absmax_compress_kernel<double>, grid, 256, 0, s, absmax, nbo, in, count, offset, code2, absmax_q,
                      absmax2);
}

}  // namespace bbc
