// Dequant fused into its linear consumer for larger activation batches (M > 32), on the
// fifth-generation tensor cores: Y[M, N] = X[M, K] @ W[N, K]^T with W the nested 4-bit weight
// ("Fuse nested 4-bit scale reconstruction on SM103", Summary: scale of outer block b =
// fl(fl(code2[absmax_q[b]] * absmax2[b / 256]) + offset), w = T(fl(code4[nibble] * scale))) or the
// k-bit weight of the k-bit patch series (dequantize_kbit: w = T(fl(codebook[idx] * absmax))),
// exactly the values the unfused dequantize-then-linear path materialises; here W never exists
// in global memory.
//
// Tiling (weight rows on the MMA's M side): a CTA owns 128 rows of W and NT (64, 128 or 256)
// activation rows; its accumulator D[128 x NT] (fp32) lives in tensor memory. K advances in
// 64-wide stages through a 4-deep shared-memory ring:
//   * warp 0, one thread: TMA load of the X tile (NT rows x 64 k, 128-byte swizzle);
//   * warps 2..9 (256 threads): decode the W tile (thread = one weight row and one half of the
//     64 k: 16 code bytes or one k-bit block) straight into the same swizzled K-major layout;
//   * warp 1, one thread: four tcgen05.mma (kind::f16, K = 16 each) per stage, then a commit that
//     frees the stage when the MMAs have read it.
// Full and empty stages are tracked with mbarriers; every wait is bounded (on expiry it counts a
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

#include "common.cuh"
#include "launch.h"

namespace bbc {

// Bounded waits that gave up, per device (read and reset by bbc_wait_timeouts).
__device__ unsigned int g_wait_timeouts;

namespace {

constexpr int kTcRows = 128;              // weight rows per CTA (the MMA's M)
constexpr int kTcBK = 64;                 // k per stage: one 128-byte swizzle row of 16-bit values
constexpr int kTcStages = 4;
constexpr int kTcDecoders = 256;          // warps 2..9
constexpr int kTcThreads = 64 + kTcDecoders;
constexpr int kTcWTile = kTcRows * kTcBK * 2;      // 16 KB
constexpr uint32_t kWaitLimit = 1u << 20;          // try_wait rounds before a wait gives up

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
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// Waits for the phase of `bar` with the given parity; false (and one timeout counted) if it did
// not complete within kWaitLimit rounds.
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
// Arrives on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
// Generic-proxy writes to shared memory made visible to the tensor cores (async proxy).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

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

// Byte address, in a K-major 128-byte-swizzled tile (rows of 128 bytes, 8-row atoms of 1024
// bytes), of 16-byte chunk c (k 8c .. 8c + 7) of row r: chunk c of row r sits at position
// c ^ (r mod 8) of its row. The 8 rows of a 16-byte store phase (consecutive r, same c) hit 8
// different chunk positions: no bank conflicts.
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t tile, int r, int c) {
    return tile + (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" :: "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

template <int DT>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    return DT == BF16 ? pack_bf16x2(lo, hi) : pack_f16x2(lo, hi);
}

// The 32 weights m0 .. m0 + 31 of a nested 4-bit row (m0 a multiple of 32, so they share one
// outer block) as 16 packed pairs of T: one 16-byte code load, one scale
// fl(fl(code2[q] * absmax2) + offset), then per code byte the pair (code4[hi], code4[lo]) times the
// scale (one paired multiply) and one paired conversion. c4s holds code4 in shared memory (16
// entries in 16 banks: lanes never conflict).
template <int DT>
__device__ __forceinline__ void decode_nested32(const NestedW& w, int64_t m0, const float* c2s, const float* c4s,
                                                uint32_t (&out)[16]) {
    const uint4 c = __ldg(reinterpret_cast<const uint4*>(w.codes + (m0 >> 1)));
    const int64_t b = m0 >> w.log2_bs;
    const float s = __fadd_rn(__fmul_rn(c2s[__ldg(w.absmax_q + b)], __ldg(w.absmax2 + (b >> 8))), w.offset);
    const float2 s2 = make_float2(s, s);
    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t hi = (words[i] >> (8 * j + 4)) & 15u, lo = (words[i] >> (8 * j)) & 15u;
            const float2 p = __fmul2_rn(make_float2(c4s[hi], c4s[lo]), s2);
            out[4 * i + j] = pack2<DT>(p.x, p.y);
        }
}

// The 32 weights of k-bit block b as 16 packed pairs of T (elements 2i, 2i + 1 in word i): the
// block's K plane words transposed into four plane groups, each index gathered by one
// multiply-high (plane_offset4), the codebook entry (cbb, shared) times the absmax.
template <int DT, int KB>
__device__ __forceinline__ void decode_kbit32(const KbitW& w, int64_t b, const char* cbb, uint32_t (&out)[16]) {
    uint32_t wd[KB];
    const uint32_t* p = w.packed + b * KB;
    if constexpr (KB == 4) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        wd[0] = v.x; wd[1 % KB] = v.y; wd[2 % KB] = v.z; wd[3 % KB] = v.w;
    } else if constexpr (KB == 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        wd[0] = v.x; wd[1 % KB] = v.y;
    } else {
#pragma unroll
        for (int j = 0; j < KB; j++) wd[j] = __ldg(p + j);
    }
    const float am = __ldg(w.absmax + b);
    uint32_t G[4], p4;
    kbit_groups<KB, 32>(wd, 0, G, p4);
#pragma unroll
    for (int q = 0; q < 4; q++) {
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

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(addr), "f"(v) : "memory");
}

// Shared memory of a CTA (dynamic, rounded up to a 1024-byte boundary for the swizzle atoms):
// kTcStages stages of {W tile 16 KB, X tile NT x 128 bytes}, then the mbarriers, the tensor-memory
// address and the tables. After the main loop the stage area holds the split-K receive buffer.
template <int NT>
struct TcSmem {
    static constexpr int kXTile = NT * 128;
    static constexpr int kStage = kTcWTile + kXTile;              // a multiple of 1024
    static constexpr int kBars = kTcStages * kStage;             // x_full[4], w_full[4], empty[4], acc_full
    static constexpr int kTmemSlot = kBars + 13 * 8;
    static constexpr int kTables = kBars + 128;                  // code2 (256 floats), code4 / codebook (32)
    static constexpr int kBytes = kTables + (256 + 32) * 4;
    static constexpr int kAlloc = kBytes + 1024;                  // with the alignment slack
    static_assert(kStage % 1024 == 0, "stages start on swizzle-atom boundaries");
    static_assert(NT * kTcRows * 4 <= kTcStages * kStage, "the receive buffer fits in the stage area");
};

template <int DT, int NT, bool NESTED, int KB>
__global__ void __launch_bounds__(kTcThreads, 1)
linear_tc_kernel(const __grid_constant__ CUtensorMap tmx, int M, int64_t N, int64_t K, NestedW nw, KbitW kw,
                 uint16_t* __restrict__ Y) {
    using L = TcSmem<NT>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = (uint32_t)__cvta_generic_to_shared(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_p = smem_raw + (base - raw);
    auto x_full = [&](int s) { return base + L::kBars + 8u * s; };
    auto w_full = [&](int s) { return base + L::kBars + 32u + 8u * s; };
    auto empty = [&](int s) { return base + L::kBars + 64u + 8u * s; };
    const uint32_t acc_full = base + L::kBars + 96u;
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

    // ---- set-up: tables, barriers, tensor memory ----
    if (NESTED)
        for (int i = threadIdx.x; i < 256; i += kTcThreads) c2s[i] = nw.code2[i];
    if (threadIdx.x < 32)
        c4s[threadIdx.x] = NESTED ? (threadIdx.x < 16 ? nw.code4[threadIdx.x] : 0.0f)
                                  : (threadIdx.x < (1 << KB) ? kw.codebook[threadIdx.x] : 0.0f);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; s++) {
            mbar_init(x_full(s), 1);                        // the TMA thread's arrive (+ the bytes)
            mbar_init(w_full(s), kTcDecoders / 32);         // one arrive per decoder warp
            mbar_init(empty(s), 1);                         // the MMA thread's commit
        }
        mbar_init(acc_full, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(base + (uint32_t)L::kTmemSlot), "r"((uint32_t)NT) : "memory");
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
                const int s = i % kTcStages, r = i / kTcStages;
                if (r > 0 && !mbar_wait(empty(s), (r & 1) ^ 1)) break;
                mbar_arrive_expect_tx(x_full(s), L::kXTile);
                tma_load_2d(base + s * L::kStage + kTcWTile, &tmx, (int)((c_lo + i) * kTcBK), m_tile0, x_full(s));
                issued = i + 1;
            }
            // the last loads in flight have landed before the CTA moves on (bounded)
            for (int i = issued > kTcStages ? issued - kTcStages : 0; i < issued; i++)
                mbar_wait(x_full(i % kTcStages), (i / kTcStages) & 1);
        }
    } else if (warp == 1) {
        // ---- the MMAs: D[128 x NT] += W[128 x 64] X[NT x 64]^T per stage ----
        if (lane == 0) {
            constexpr uint32_t idesc = mma_idesc(DT == BF16 ? 1 : 0, NT);
            for (int i = 0; i < nchunks; i++) {
                const int s = i % kTcStages, r = i / kTcStages;
                if (!mbar_wait(x_full(s), r & 1) || !mbar_wait(w_full(s), r & 1)) break;
                tc_fence_after();
                const uint32_t wa = base + s * L::kStage, xa = wa + kTcWTile;
#pragma unroll
                for (int kk = 0; kk < kTcBK / 16; kk++)
                    mma_f16(tmem, smem_desc_sw128(wa + 32 * kk), smem_desc_sw128(xa + 32 * kk), idesc,
                            (i > 0 || kk > 0) ? 1u : 0u);
                mma_commit(empty(s));
            }
            mma_commit(acc_full);          // once every MMA issued above has completed
        }
    } else {
        // ---- W tiles decoded into shared memory ----
        const int row = 32 * (warp & 3) + lane;                   // also this warp's tensor-memory lane
        const int h = (warp - 2) >> 2;                            // which 32 of a stage's 64 k
        const int64_t n = n0 + row;
        for (int i = 0; i < nchunks; i++) {
            const int s = i % kTcStages, r = i / kTcStages;
            if (r > 0 && !warp_wait(empty(s), (r & 1) ^ 1)) break;
            const int64_t m0 = n * K + (c_lo + i) * kTcBK + 32 * h;
            uint32_t v[16];
            if constexpr (NESTED) decode_nested32<DT>(nw, m0, c2s, c4s, v);
            else decode_kbit32<DT, KB>(kw, m0 >> 5, reinterpret_cast<const char*>(c4s), v);
            const uint32_t tile = base + s * L::kStage;
#pragma unroll
            for (int c = 0; c < 4; c++)
                sts128(sw128_chunk(tile, row, 4 * h + c), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(w_full(s));
        }
    }

    // ---- epilogue (decoder warps): accumulator -> Y, summed over the cluster for split K ----
    const bool epi = warp >= 2;
    const int row = 32 * (warp & 3) + lane;
    const int g = (warp - 2) >> 2;                                // which half of the columns
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
            for (int c = g * (NT / 2); c < (g + 1) * (NT / 2); c += 16) {
                float v[16];
                tmem_ld16(lane_tmem + c, v);
#pragma unroll
                for (int i = 0; i < 16; i++) store(c + i, v[i]);
            }
    } else {
        // receive buffer of this CTA: [S][W][128] floats, partial of rank s for owned column c at
        // [s][c - rank * W][row]
        const int W = NT / (int)S;
        cluster_sync();                                           // every CTA is past its main loop
        if (epi)
            for (int c = g * (NT / 2); c < (g + 1) * (NT / 2); c += 16) {
                const uint32_t owner = (uint32_t)(c / W);
                if (owner == rank) continue;
                float v[16];
                tmem_ld16(lane_tmem + c, v);
                const uint32_t dst = map_to_rank(base, owner);
#pragma unroll
                for (int i = 0; i < 16; i++)
                    st_cluster_f32(dst + (uint32_t)(((rank * W + (c - (int)owner * W) + i) * kTcRows + row) * 4), v[i]);
            }
        cluster_sync();                                           // every partial has arrived
        if (epi) {
            const float* recv = reinterpret_cast<const float*>(base_p);
            for (int c = (int)rank * W + g * (W / 2); c < (int)rank * W + (g + 1) * (W / 2); c += 16) {
                float v[16];
                tmem_ld16(lane_tmem + c, v);
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const int cl = c - (int)rank * W + i;
                    float acc = rank == 0 ? v[i] : recv[(0 * W + cl) * kTcRows + row];
                    for (uint32_t s = 1; s < S; s++)
                        acc = __fadd_rn(acc, s == rank ? v[i] : recv[((int)s * W + cl) * kTcRows + row]);
                    store(c + i, acc);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"((uint32_t)NT) : "memory");
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

// Split factor S (a cluster of S CTAs shares an output tile along K): the S in {1, 2, 4, 8} that
// fills the machine best (output tiles x S CTAs over waves of `cap` resident CTAs), with at least
// 32 accumulator columns and two K stages per CTA; a larger S only when it is 5 % better.
int pick_split(int64_t tiles, int cap, int nt, int64_t stages_k) {
    int best = 1;
    double best_eff = 0.0;
    for (int S = 1; S <= 8; S *= 2) {
        if (S > nt / 32 || stages_k < 2 * S) break;
        const int64_t ctas = tiles * S;
        const int64_t waves = (ctas + cap - 1) / cap;
        const double eff = (double)ctas / (double)(waves * cap);
        if (eff > best_eff * 1.05) {
            best = S;
            best_eff = eff;
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
    const int S = pick_split(ntiles * mtiles, cap, NT, K / kTcBK);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, (unsigned)ntiles, (unsigned)mtiles);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = s;
    cudaLaunchAttribute attr_c[1];
    attr_c[0].id = cudaLaunchAttributeClusterDimension;
    attr_c[0].val.clusterDim.x = (unsigned)S;
    attr_c[0].val.clusterDim.y = 1;
    attr_c[0].val.clusterDim.z = 1;
    cfg.attrs = attr_c;
    cfg.numAttrs = S > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k, map, M, N, K, nw, kw, Y);
}

template <int DT, bool NESTED, int KB>
cudaError_t launch_tc_nt(const uint16_t* X, int M, int64_t N, int64_t K, const NestedW& nw, const KbitW& kw,
                         uint16_t* Y, cudaStream_t s) {
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

}  // namespace bbc
