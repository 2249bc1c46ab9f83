// Dequant fused into its linear consumer for larger activation batches (M > 32), on the
// fifth-generation tensor cores: Y[M, N] = X[M, K] @ W[N, K]^T with W the nested 4-bit weight
// ("Fuse nested 4-bit scale reconstruction on SM103", Summary: scale of outer block b =
// fl(fl(code2[absmax_q[b]] * absmax2[b / 256]) + offset), w = T(fl(code4[nibble] * scale))) or the
// k-bit weight of the k-bit patch series (dequantize_kbit: w = T(fl(codebook[idx] * absmax))),
// exactly the values the unfused dequantize-then-linear path materialises; here W never exists
// in global memory.
//
// Tiling (weight rows on the MMA's M side): a CTA owns 128 rows of W and NT (16, 32, 64, 128 or
// 256) activation rows; its accumulator D[128 x NT] (fp32) lives in tensor memory. K advances in
// 64-wide stages:
//   * warp 0, one thread: TMA loads of the X tiles (NT rows x 64 k, 128-byte swizzle) into a ring
//     of 6-8 shared-memory stages;
//   * warps 2..17 (512 threads): decode the W tile (thread = one weight row and a quarter of the
//     64 k: 8 code bytes or half a k-bit block, loaded 4 stages ahead into registers) and write it
//     straight into tensor memory (tcgen05.st: the row is the thread's lane), a ring of 8 A tiles;
//     no shared memory and no proxy fence sits between a decoder's loads and the MMA;
//   * warp 1, one thread: four tcgen05.mma (kind::f16, K = 16 each, A from tensor memory, B from
//     the swizzled X tile) per stage, then commits that free the X and W slots when the MMAs have
//     read them.
// Full and empty slots are tracked with mbarriers; every wait is bounded (on expiry it counts a
// timeout, see bbc_wait_timeouts, and the kernel winds down instead of hanging).
//
// Split K over a thread-block cluster: with few output tiles the S CTAs of a cluster (S <= 8)
// take K / S each; after the main loop each CTA sends the accumulator columns another CTA owns
// to that CTA's shared memory (distributed shared memory, st.shared::cluster) and every CTA sums
// its own columns over the S partials in rank order (a fixed order: results do not depend on
// timing) before rounding to T once and storing Y. No global workspace is used.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace bbc {

// Bounded waits that gave up, per device (read and reset by bbc_wait_timeouts).
__device__ unsigned int g_wait_timeouts;

namespace {

constexpr int kTcRows = 128;              // weight rows per CTA (the MMA's M)
constexpr int kTcBK = 64;                 // k per stage: one 128-byte swizzle row of 16-bit values
constexpr int kTcDecoders = 512;          // warps 2..17
constexpr int kTcThreads = 64 + kTcDecoders;
constexpr uint32_t kWaitRoundNs = 100000;          // suspend-time hint of one try_wait round (100 us)
constexpr uint32_t kWaitLimit = 1u << 13;          // rounds before a wait gives up
constexpr int kPrefetch = 4;                       // stages of decoder inputs loaded ahead

// ---- mbarriers ----

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}
// One round of waiting: the thread is suspended until the phase completes or kWaitRoundNs pass
// (it does not spin, so waiting roles take no issue slots from the decoders).
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(bar), "r"(parity), "r"(kWaitRoundNs) : "memory");
    return ok != 0;
}
// Waits for the phase of `bar` with the given parity; false (and one timeout counted) if it did
// not complete within kWaitLimit rounds (about a second).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitLimit; i++)
        if (mbar_try_wait(bar, parity)) return true;
    atomicAdd(&g_wait_timeouts, 1u);
    return false;
}

// ---- TMA and the tensor-core instructions ----

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}

// Shared-memory matrix descriptor of a K-major tile in the 128-byte swizzle layout (rows of 128
// bytes, 8-row atoms of 1024 bytes): start address / 16, leading offset 1 (unused by this
// layout), stride between 8-row groups 1024 bytes, descriptor version 1, layout 2 (128B swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, A and B of type DT (fp16 0, bf16 1),
// both K-major, N = nt, M = 128.
__host__ __device__ constexpr uint32_t mma_idesc(int dt_is_bf16, int nt) {
    return (1u << 4) | ((uint32_t)dt_is_bf16 << 7) | ((uint32_t)dt_is_bf16 << 10) | ((uint32_t)(nt >> 3) << 17) |
           ((uint32_t)(kTcRows >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }"
                 :: "r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
// The same with A in tensor memory (lane = row of A, 32-bit column c = elements 2c, 2c + 1 of the
// row's K slice, element 2c in the low half).
__device__ __forceinline__ void mma_f16_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }"
                 :: "r"(tmem_d), "r"(tmem_a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
// Eight consecutive 32-bit columns of this thread's tensor-memory lane, from registers
// (asynchronous: tmem_wait_st waits for this thread's stores to complete).
__device__ __forceinline__ void tmem_st8(uint32_t addr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :: "r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Arrives on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

// 16 consecutive fp32 accumulator columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld16(uint32_t addr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(addr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}

// ---- clusters ----

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The shared::cluster address of `addr` (a shared::cta address) in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// ---- decoding a weight tile into the tensor cores' operand layout ----

// The nested 4-bit weight (flattened element m = n * K + k).
struct NestedW {
    const uint8_t* codes;         // two codes per byte, element 2j in the high nibble of byte j
    const uint8_t* absmax_q;      // General8 code of each outer block
    const float* code2;           // 256-entry General8 table
    const float* absmax2;         // one inner absmax per 256 outer blocks
    const float* code4;           // 16-entry value table
    float offset;
    int log2_bs;
};
// The k-bit weight: K plane words and one fp32 absmax per block of 32 elements.
struct KbitW {
    const uint32_t* packed;
    const float* absmax;
    const float* codebook;
};

template <int DT>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    return DT == BF16 ? pack_bf16x2(lo, hi) : pack_f16x2(lo, hi);
}

// The inputs of the 16 weights m0 .. m0 + 15 of a nested 4-bit row (m0 a multiple of 16, so they
// share one outer block b): 8 code bytes, the General8 code of b and the inner absmax of b.
// Loaded several stages ahead of their use (the decoder's prefetch ring).
struct NestedIn {
    uint2 c;
    uint32_t q;
    float a2;
};
__device__ __forceinline__ NestedIn load_nested16(const NestedW& w, int64_t m0) {
    NestedIn r;
    r.c = __ldg(reinterpret_cast<const uint2*>(w.codes + (m0 >> 1)));
    const int64_t b = m0 >> w.log2_bs;
    r.q = __ldg(w.absmax_q + b);
    r.a2 = __ldg(w.absmax2 + (b >> 8));
    return r;
}

// The decode table: entry (byte, r) = (code4[byte >> 4], code4[byte & 15]) at byte offset
// byte * 128 + r * 8, 16 interleaved replicas: the 16 lanes of an 8-byte shared-load phase read
// replica lane & 15, so they never conflict.
constexpr int kPairBytes = 256 * 16 * 8;           // 32 KB

// Those 16 weights as 8 packed pairs of T: the scale fl(fl(code2[q] * absmax2) + offset), then per
// code byte one table read of (code4[hi], code4[lo]) (its address: the byte moved to bits 7..14 or-ed
// with the lane's replica), times the scale (one paired multiply), one paired conversion.
template <int DT>
__device__ __forceinline__ void decode_nested16(const NestedIn& in, float offset, const float* c2s,
                                                const unsigned char* pairs, uint32_t lane_off, uint32_t (&out)[8]) {
    const float s = __fadd_rn(__fmul_rn(c2s[in.q], in.a2), offset);
    const float2 s2 = make_float2(s, s);
    const uint32_t words[2] = {in.c.x, in.c.y};
#pragma unroll
    for (int i = 0; i < 2; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t sel = (j == 0 ? (words[i] << 7) : (words[i] >> (8 * j - 7))) & 0x7f80u;
            const float2 p = __fmul2_rn(*reinterpret_cast<const float2*>(pairs + (sel | lane_off)), s2);
            out[4 * i + j] = pack2<DT>(p.x, p.y);
        }
}

// The inputs of the 32 weights of k-bit block b: its K plane words and its absmax.
template <int KB>
struct KbitIn {
    uint32_t w[KB];
    float am;
};
template <int KB>
__device__ __forceinline__ KbitIn<KB> load_kbit32(const KbitW& w, int64_t b) {
    KbitIn<KB> r;
    const uint32_t* p = w.packed + b * KB;
    if constexpr (KB == 4) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        r.w[0] = v.x; r.w[1 % KB] = v.y; r.w[2 % KB] = v.z; r.w[3 % KB] = v.w;
    } else if constexpr (KB == 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        r.w[0] = v.x; r.w[1 % KB] = v.y;
    } else {
#pragma unroll
        for (int j = 0; j < KB; j++) r.w[j] = __ldg(p + j);
    }
    r.am = __ldg(w.absmax + b);
    return r;
}

// Half hb of those 32 weights (elements 16 hb .. 16 hb + 15) as 8 packed pairs of T (elements 2i,
// 2i + 1 in word i): the K plane words transposed into the half's two plane groups, each index
// gathered by one multiply-high (plane_offset4), the codebook entry (cbb, shared) times the absmax.
template <int DT, int KB>
__device__ __forceinline__ void decode_kbit16(const KbitIn<KB>& in, int hb, const char* cbb, uint32_t (&out)[8]) {
    uint32_t G[2], p4;
    kbit_groups<KB, 16>(in.w, hb, G, p4);
    const float am = in.am;
#pragma unroll
    for (int q = 0; q < 2; q++) {
        const uint32_t B = G[q], Bs = B << 3, P = p4 >> (8 * q);
        out[4 * q + 0] = pack2<DT>(kbit_elem<KB, DT, 0>(B, Bs, P, am, cbb), kbit_elem<KB, DT, 1>(B, Bs, P, am, cbb));
        out[4 * q + 1] = pack2<DT>(kbit_elem<KB, DT, 2>(B, Bs, P, am, cbb), kbit_elem<KB, DT, 3>(B, Bs, P, am, cbb));
        out[4 * q + 2] = pack2<DT>(kbit_elem<KB, DT, 4>(B, Bs, P, am, cbb), kbit_elem<KB, DT, 5>(B, Bs, P, am, cbb));
        out[4 * q + 3] = pack2<DT>(kbit_elem<KB, DT, 6>(B, Bs, P, am, cbb), kbit_elem<KB, DT, 7>(B, Bs, P, am, cbb));
    }
}

// All lanes of the warp wait for the phase of `bar` with the given parity (the loop ends for all
// of them at once); false, with one timeout counted, if it did not complete within kWaitLimit.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitLimit; i++)
        if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if ((threadIdx.x & 31) == 0) atomicAdd(&g_wait_timeouts, 1u);
    return false;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" :: "r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(addr), "f"(v) : "memory");
}

// Tensor memory of a CTA (512 columns): the accumulator D[128 x NT] in columns 0 .. NT-1, and a ring
// of kTcWStages = 8 decoded weight tiles (A operands: 128 rows x 64 k of 16-bit values = 32 columns
// each) in columns 256 .. 511.
constexpr int kTmemCols = 512;
constexpr int kTmemA = 256;
constexpr int kTcWStages = 8;

// Shared memory of a CTA (dynamic, rounded up to a 1024-byte boundary for the swizzle atoms): a
// ring of kXStages X tiles (NT rows x 128 bytes), the nested decode table, then the mbarriers, the
// tensor-memory address and the other tables. After the main loop the X area holds the split-K receive buffer.
template <int NT>
struct TcSmem {
    static constexpr int kXTile = NT * 128;                       // a multiple of 1024 for NT >= 8
    static constexpr int kXStages = NT >= 256 ? 6 : 8;
    static constexpr int kPairs = kXStages * kXTile;             // the 32 KB decode table (nested weights)
    static constexpr int kBars = kPairs + kPairBytes;            // x_full, x_empty, w_full, w_empty, acc_full
    static constexpr int kNumBars = 2 * kXStages + 2 * kTcWStages + 1;   // at most 33
    static constexpr int kTmemSlot = kBars + 272;
    static constexpr int kTables = kBars + 288;                  // code2 (256 floats), code4 / codebook (32)
    static_assert(kNumBars * 8 <= 272, "barriers before the tensor-memory slot");
    static constexpr int kBytes = kTables + (256 + 32) * 4;
    static constexpr int kAlloc = kBytes + 1024;                  // with the alignment slack
    static_assert(kXTile % 1024 == 0, "X tiles start on swizzle-atom boundaries");
    // the split-K receive buffer, S x 128 rows x (NT / S + 4) floats at most (S <= 8)
    static constexpr int kRecvMax = kTcRows * 4 * (NT + 4 * 8);
    // (below NT = 64 the bound is loose: W < 16 needs no padding, so S x 128 x W x 4 = 512 NT bytes)
    static_assert(kRecvMax <= kXStages * kXTile || NT * kTcRows * 4 <= kXStages * kXTile, "receive buffer fits");
    static_assert(kTables % 16 == 0, "tables aligned");
};

template <int DT, int NT, bool NESTED, int KB>
__global__ void __launch_bounds__(kTcThreads, 1)
linear_tc_kernel(const __grid_constant__ CUtensorMap tmx, int M, int64_t N, int64_t K, NestedW nw, KbitW kw,
                 uint16_t* __restrict__ Y) {
    pdl_wait();               // writes of the previous kernel in the stream are visible from here
    using L = TcSmem<NT>;
    constexpr int XS = L::kXStages, WS = kTcWStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = (uint32_t)__cvta_generic_to_shared(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_p = smem_raw + (base - raw);
    auto x_full = [&](int s) { return base + L::kBars + 8u * s; };
    auto x_empty = [&](int s) { return base + L::kBars + 8u * (XS + s); };
    auto w_full = [&](int s) { return base + L::kBars + 8u * (2 * XS + s); };
    auto w_empty = [&](int s) { return base + L::kBars + 8u * (2 * XS + WS + s); };
    const uint32_t acc_full = base + L::kBars + 8u * (2 * XS + 2 * WS);
    float* const c2s = reinterpret_cast<float*>(base_p + L::kTables);
    float* const c4s = c2s + 256;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)blockIdx.y * kTcRows;
    const int m_tile0 = blockIdx.z * NT;
    const uint32_t S = gridDim.x;
    const uint32_t rank = S > 1 ? cluster_rank() : 0u;
    const int64_t C = K / kTcBK;
    const int64_t c_lo = C * rank / S;
    const int nchunks = (int)(C * (rank + 1) / S - c_lo);

    // Decoder thread (warps 2..): one weight row (its tensor-memory lane) and one quarter (16 k) of a
    // stage's 64 k. Its first kPrefetch stages of inputs are loaded before the set-up below, so that
    // their latency overlaps the tables, the barriers and the tensor-memory allocation.
    const int64_t d_mrow = (n0 + 32 * (warp & 3) + lane) * K + c_lo * kTcBK + 16 * ((warp - 2) >> 2);
    using In = std::conditional_t<NESTED, NestedIn, KbitIn<KB>>;
    auto load_in = [&](int i) -> In {
        const int64_t m0 = d_mrow + (int64_t)i * kTcBK;
        if (!BBC_GUARD(m0 >= 0 && m0 + 16 <= N * K, kGuardLinear)) return In{};
        if constexpr (NESTED) return load_nested16(nw, m0);
        else return load_kbit32<KB>(kw, m0 >> 5);
    };
    In pre[kPrefetch];
    if (warp >= 2) {
#pragma unroll
        for (int j = 0; j < kPrefetch; j++)
            if (j < nchunks) pre[j] = load_in(j);
    }

    // ---- set-up: tables, barriers, tensor memory ----
    unsigned char* const pairs = base_p + L::kPairs;
    if (NESTED) {
        for (int i = threadIdx.x; i < 256; i += kTcThreads) c2s[i] = nw.code2[i];
        if (threadIdx.x < 256) {
            // thread i writes the 16 replicas of entry i as 8 rotated 16-byte stores
            const int byte = threadIdx.x;
            const float hi = nw.code4[byte >> 4], lo = nw.code4[byte & 15];
            const float4 v = make_float4(hi, lo, hi, lo);
#pragma unroll
            for (int r = 0; r < 8; r++) *reinterpret_cast<float4*>(pairs + byte * 128 + ((r + byte) & 7) * 16) = v;
        }
    }
    if (threadIdx.x < 32)
        c4s[threadIdx.x] = NESTED ? (threadIdx.x < 16 ? nw.code4[threadIdx.x] : 0.0f)
                                  : (threadIdx.x < (1 << KB) ? kw.codebook[threadIdx.x] : 0.0f);
    if (threadIdx.x == 0) {
        for (int s = 0; s < XS; s++) {
            mbar_init(x_full(s), 1);                        // the TMA thread's arrive (+ the bytes)
            mbar_init(x_empty(s), 1);                       // the MMA thread's commit
        }
        for (int s = 0; s < WS; s++) {
            mbar_init(w_full(s), kTcDecoders / 32);         // one arrive per decoder warp
            mbar_init(w_empty(s), 1);                       // the MMA thread's commit
        }
        mbar_init(acc_full, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(base + (uint32_t)L::kTmemSlot), "r"((uint32_t)kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_p + L::kTmemSlot);

    if (warp == 0) {
        // ---- X tiles by TMA ----
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tmx)) : "memory");
            int issued = 0;
            for (int i = 0; i < nchunks; i++) {
                const int s = i % XS, r = i / XS;
                if (r > 0 && !mbar_wait(x_empty(s), (r & 1) ^ 1)) break;
                mbar_arrive_expect_tx(x_full(s), L::kXTile);
                tma_load_2d(base + s * L::kXTile, &tmx, (int)((c_lo + i) * kTcBK), m_tile0, x_full(s));
                issued = i + 1;
            }
            // the last loads in flight have landed before the CTA moves on (bounded)
            for (int i = issued > XS ? issued - XS : 0; i < issued; i++) mbar_wait(x_full(i % XS), (i / XS) & 1);
        }
    } else if (warp == 1) {
        // ---- the MMAs: D[128 x NT] += W[128 x 64] X[NT x 64]^T per stage, W from tensor memory ----
        if (lane == 0) {
            constexpr uint32_t idesc = mma_idesc(DT == BF16 ? 1 : 0, NT);
            for (int i = 0; i < nchunks; i++) {
                const int sx = i % XS, rx = i / XS, sw = i % WS, rw = i / WS;
                if (!mbar_wait(x_full(sx), rx & 1) || !mbar_wait(w_full(sw), rw & 1)) break;
                tc_fence_after();
                const uint32_t xa = base + sx * L::kXTile, wa = tmem + kTmemA + 32u * sw;
#pragma unroll
                for (int kk = 0; kk < kTcBK / 16; kk++)
                    mma_f16_ta(tmem, wa + 8u * kk, smem_desc_sw128(xa + 32 * kk), idesc, (i > 0 || kk > 0) ? 1u : 0u);
                mma_commit(x_empty(sx));
                mma_commit(w_empty(sw));
            }
            mma_commit(acc_full);          // once every MMA issued above has completed
        }
    } else {
        // ---- W tiles decoded into tensor memory ----
        // 8 of a stage's 32 A columns per thread (see d_mrow above). Its inputs are loaded kPrefetch
        // stages ahead of their decode (a register ring); no shared memory and no proxy fence is
        // involved.
        const int qk = (warp - 2) >> 2;                           // which 16 of a stage's 64 k
        const uint32_t lane_a = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + kTmemA + 8u * qk;
        const uint32_t lane_off = (uint32_t)(lane & 15) * 8u;
        bool live = true;
        int done_to = 0;                                          // stages whose stores were issued
        for (int i0 = 0; i0 < nchunks && live; i0 += kPrefetch) {
#pragma unroll
            for (int j = 0; j < kPrefetch; j++) {
                const int i = i0 + j;
                if (i >= nchunks) break;
                const int s = i % WS, r = i / WS;
                if (r > 0 && !warp_wait(w_empty(s), (r & 1) ^ 1)) {
                    live = false;
                    break;
                }
                uint32_t v[8];
                if constexpr (NESTED) decode_nested16<DT>(pre[j], nw.offset, c2s, pairs, lane_off, v);
                else decode_kbit16<DT, KB>(pre[j], qk & 1, reinterpret_cast<const char*>(c4s), v);
                if (i + kPrefetch < nchunks) pre[j] = load_in(i + kPrefetch);
                // the previous stage's tensor-memory stores completed while this one was decoded:
                // signal it now, then start this stage's stores
                if (i > 0) {
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(w_full((i - 1) % WS));
                }
                tmem_st8(lane_a + 32u * s, v);
                done_to = i + 1;
            }
        }
        if (done_to > 0) {
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(w_full((done_to - 1) % WS));
        }
    }

    // ---- epilogue (decoder warps): accumulator -> Y, summed over the cluster for split K ----
    const bool epi = warp >= 2;
    const int row = 32 * (warp & 3) + lane;
    const int g = (warp - 2) >> 2;                                // which of four column groups
    const int64_t n = n0 + row;
    const uint32_t lane_tmem = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    auto store = [&](int col, float v) {
        const int m = m_tile0 + col;
        if (m < M) Y[(int64_t)m * N + n] = DT == BF16 ? f32_to_bf16_bits(v) : f32_to_f16_bits(v);
    };
    if (epi) {
        warp_wait(acc_full, 0);
        tc_fence_after();
    }
    if (S == 1) {
        if (epi)
            for (int c = 16 * g; c < NT; c += 64) {                // 16-column chunks, rotating groups
                float v[16];
                tmem_ld16(lane_tmem + c, v);
#pragma unroll
                for (int i = 0; i < 16; i++) store(c + i, v[i]);
            }
    } else {
        // CTA `rank` owns columns [rank W, rank W + W) (W = NT / S >= 2); its receive buffer holds the
        // partial of rank s for owned column c at [s][row][c - rank W], rows WP floats apart (WP = W + 4
        // when W >= 16: 16-byte accesses of 8 consecutive rows then hit different banks)
        const int W = NT / (int)S, own0 = (int)rank * W, WP = W >= 16 ? W + 4 : W;
        cluster_sync();                                           // every CTA is past its main loop
        if (epi)
            for (int c = 16 * g; c < NT; c += 64) {
                if (c >= own0 && c + 16 <= own0 + W) continue;    // all of this chunk stays here
                float v[16];
                tmem_ld16(lane_tmem + c, v);
                if (W >= 16) {                                    // the chunk has one owner: 16-byte stores
                    const int owner = c / W;
                    const uint32_t dst = map_to_rank(base, (uint32_t)owner) +
                                         (uint32_t)((((int)rank * kTcRows + row) * WP + (c - owner * W)) * 4);
#pragma unroll
                    for (int i = 0; i < 16; i += 4) st_cluster_v4(dst + 4u * i, v[i], v[i + 1], v[i + 2], v[i + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        const int owner = (c + i) / W;
                        if (owner == (int)rank) continue;
                        const uint32_t dst = map_to_rank(base, (uint32_t)owner);
                        st_cluster_f32(dst + (uint32_t)((((int)rank * kTcRows + row) * WP + (c + i - owner * W)) * 4),
                                       v[i]);
                    }
                }
            }
        cluster_sync();                                           // every partial has arrived
        if (epi) {
            const float* recv = reinterpret_cast<const float*>(base_p);
            for (int c = (own0 & ~15) + 16 * g; c < own0 + W; c += 64) {
                float v[16];
                tmem_ld16(lane_tmem + c, v);
                if (W >= 16) {
                    // the chunk lies inside the owned columns (both 16-aligned): the partials are read
                    // four columns at a time, 16-byte loads whose 8-row phases hit different banks
                    // (WP = W + 4); the sum keeps rank order
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        const int cl = c + i - own0;
                        float4 acc = rank == 0 ? make_float4(v[i], v[i + 1], v[i + 2], v[i + 3])
                                               : *reinterpret_cast<const float4*>(recv + row * WP + cl);
                        for (uint32_t s = 1; s < S; s++) {
                            const float4 p = s == rank ? make_float4(v[i], v[i + 1], v[i + 2], v[i + 3])
                                                       : *reinterpret_cast<const float4*>(
                                                             recv + ((int)s * kTcRows + row) * WP + cl);
                            acc = make_float4(__fadd_rn(acc.x, p.x), __fadd_rn(acc.y, p.y), __fadd_rn(acc.z, p.z),
                                              __fadd_rn(acc.w, p.w));
                        }
                        store(c + i, acc.x);
                        store(c + i + 1, acc.y);
                        store(c + i + 2, acc.z);
                        store(c + i + 3, acc.w);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        const int cl = c + i - own0;
                        if (cl < 0 || cl >= W) continue;
                        float acc = rank == 0 ? v[i] : recv[row * WP + cl];
                        for (uint32_t s = 1; s < S; s++)
                            acc = __fadd_rn(acc, s == rank ? v[i] : recv[((int)s * kTcRows + row) * WP + cl]);
                        store(c + i, acc);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"((uint32_t)kTmemCols)
                     : "memory");
}

// ---- host side ----

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
EncodeTiled tensor_map_encoder(cudaError_t* err) {
    static std::once_flag once;
    static EncodeTiled fn = nullptr;
    static cudaError_t status = cudaSuccess;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        status = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (status == cudaSuccess && (q != cudaDriverEntryPointSuccess || !p)) status = cudaErrorNotSupported;
        fn = reinterpret_cast<EncodeTiled>(p);
    });
    *err = status;
    return fn;
}

// Split factor S (a cluster of S CTAs shares an output tile along K): the S in {1, 2, 4, 8}, with at
// least two K stages per CTA, of the least estimated time, in units of one 64-wide K stage (~0.6 us
// per CTA, measured with in-kernel timestamps): per wave of `cap` resident CTAs, a CTA's set-up (~5
// stages), its K stages, and its epilogue — a direct store (~NT/128 + 1) or, for S > 1, the
// exchange of partial sums through distributed shared memory and the wait for the cluster's
// slowest CTA (~NT/16: 9 us at NT = 256). A larger S must be 5 % better. (Counting only how well
// the CTAs fill the waves picked S = 8 for 86 row tiles of N = 11008 at M = 256: five waves of
// short CTAs dominated by set-up and epilogue, 158 us against ~45 us with S = 1.)
int pick_split(int64_t tiles, int cap, int64_t stages_k, int nt) {
    int best = 1;
    double best_t = 0.0;
    for (int S = 1; S <= 8; S *= 2) {
        if (S > 1 && stages_k < 2 * S) break;
        const int64_t waves = (tiles * S + cap - 1) / cap;
        const double per_cta = 5.0 + (double)stages_k / S + (S == 1 ? nt / 128.0 + 1.0 : nt / 16.0);
        const double t = (double)waves * per_cta;
        if (S == 1 || t < best_t * 0.95) {
            best = S;
            best_t = t;
        }
    }
    return best;
}

template <int DT, int NT, bool NESTED, int KB>
cudaError_t launch_tc(const uint16_t* X, int M, int64_t N, int64_t K, const NestedW& nw, const KbitW& kw,
                      uint16_t* Y, cudaStream_t s) {
    using L = TcSmem<NT>;
    auto k = linear_tc_kernel<DT, NT, NESTED, KB>;
    static std::atomic<uint64_t> attr{0};
    cudaError_t e = set_attr_once(k, attr, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    EncodeTiled encode = tensor_map_encoder(&e);
    if (e != cudaSuccess) return e;
    // X [M, K] row-major: inner dimension K; tiles of 64 k x NT rows, 128-byte swizzle; rows past M
    // read as zeros
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kTcBK, (cuuint32_t)NT};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(&map, DT == BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                              2, const_cast<uint16_t*>(X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int64_t mtiles = (M + NT - 1) / NT, ntiles = N / kTcRows;
    const int cap = resident_ctas(reinterpret_cast<const void*>(k), kTcThreads, L::kAlloc);
    if (cap < 1) return cudaErrorInvalidConfiguration;
    const int S = pick_split(ntiles * mtiles, cap, K / kTcBK, NT);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, (unsigned)ntiles, (unsigned)mtiles);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = s;
    // programmatic stream serialisation (the kernel's first act is griddepcontrol.wait), and the
    // cluster of the K split when there is one
    cudaLaunchAttribute attr_c[2];
    attr_c[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr_c[0].val.programmaticStreamSerializationAllowed = 1;
    attr_c[1].id = cudaLaunchAttributeClusterDimension;
    attr_c[1].val.clusterDim.x = (unsigned)S;
    attr_c[1].val.clusterDim.y = 1;
    attr_c[1].val.clusterDim.z = 1;
    cfg.attrs = attr_c;
    cfg.numAttrs = S > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, k, map, M, N, K, nw, kw, Y);
}

template <int DT, bool NESTED, int KB>
cudaError_t launch_tc_nt(const uint16_t* X, int M, int64_t N, int64_t K, const NestedW& nw, const KbitW& kw,
                         uint16_t* Y, cudaStream_t s) {
    if (M <= 16) return launch_tc<DT, 16, NESTED, KB>(X, M, N, K, nw, kw, Y, s);
    if (M <= 32) return launch_tc<DT, 32, NESTED, KB>(X, M, N, K, nw, kw, Y, s);
    if (M <= 64) return launch_tc<DT, 64, NESTED, KB>(X, M, N, K, nw, kw, Y, s);
    if (M <= 128) return launch_tc<DT, 128, NESTED, KB>(X, M, N, K, nw, kw, Y, s);
    return launch_tc<DT, 256, NESTED, KB>(X, M, N, K, nw, kw, Y, s);
}

template <bool NESTED, int KB>
cudaError_t launch_tc_dt(const void* X, int dtype, int M, int64_t N, int64_t K, const NestedW& nw, const KbitW& kw,
                         void* Y, cudaStream_t s) {
    const uint16_t* x = static_cast<const uint16_t*>(X);
    uint16_t* y = static_cast<uint16_t*>(Y);
    if (dtype == BF16) return launch_tc_nt<BF16, NESTED, KB>(x, M, N, K, nw, kw, y, s);
    return launch_tc_nt<F16, NESTED, KB>(x, M, N, K, nw, kw, y, s);
}

}  // namespace

cudaError_t launch_linear_4bit_nested_tc(const void* X, int dtype, int M, int64_t N, int64_t K, const uint8_t* codes,
                                         const uint8_t* absmax_q, const float* code2, const float* absmax2,
                                         float offset, const float* code4, int log2_bs, void* Y, cudaStream_t s) {
    const NestedW nw{codes, absmax_q, code2, absmax2, code4, offset, log2_bs};
    return launch_tc_dt<true, 4>(X, dtype, M, N, K, nw, KbitW{}, Y, s);
}

cudaError_t launch_linear_kbit_tc(const void* X, int dtype, int M, int64_t N, int64_t K, const uint32_t* packed,
                                  const float* absmax, const float* codebook, int KB, void* Y, cudaStream_t s) {
    const KbitW kw{packed, absmax, codebook};
    switch (KB) {
        case 2: return launch_tc_dt<false, 2>(X, dtype, M, N, K, NestedW{}, kw, Y, s);
        case 3: return launch_tc_dt<false, 3>(X, dtype, M, N, K, NestedW{}, kw, Y, s);
        case 4: return launch_tc_dt<false, 4>(X, dtype, M, N, K, NestedW{}, kw, Y, s);
        default: return launch_tc_dt<false, 5>(X, dtype, M, N, K, NestedW{}, kw, Y, s);
    }
}

// Bounded waits that gave up on the current device since the last call (and reset the count).
cudaError_t wait_timeouts(unsigned int* count) {
    cudaError_t e = cudaMemcpyFromSymbol(count, g_wait_timeouts, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_wait_timeouts, &zero, sizeof(unsigned int));
}

BBC_GUARD_ACCESSOR(guard_status_linear_tc)

}  // namespace bbc
