// Nested 4-bit dequant fused into its linear consumer: Y[M, N] = X[M, K] @ W[N, K]^T.
//
// W is the nested 4-bit weight of "Fuse nested 4-bit scale reconstruction on SM103" (flattened
// element m = n*K + k; scale of outer block b = fl(fl(code2[absmax_q[b]] * absmax2[b / 256]) +
// offset); w = T(fl(code4[nibble] * scale)) in the activation type T, exactly what the unfused
// dequantize-then-linear path materialises). The page's public-path controls time that
// dequantize-plus-linear sequence at M = 1, 8 and 32; here the weight never exists in memory:
// it is decoded in registers straight into tensor-core operand fragments.
//
// Layout of the work: a CTA owns a tile of 16 rows of W (16 outputs per activation row) and
// its 8 warps split K; partial sums meet in shared memory and are added in warp order. Each
// warp walks 64-wide windows of K with mma.sync m16n8k16 (T inputs, fp32 accumulators), one
// n-tile per 8 activation rows (M <= 32). Both operands use the same permutation of the 16
// k-slots of each mma step s (slot of lane-quad t -> k = 16 t + 4 s + 0..3), so a lane needs
// 16 consecutive k of a window: 8 contiguous code bytes per W row and 32 contiguous bytes of
// each activation row. Each code byte is decoded through a 256-entry shared table of the pair
// (code4[hi], code4[lo]), multiplied by the block scale (paired fp32 multiply) and rounded to T.
// The loads of the next window (code bytes, scale codes, activation fragments) are issued
// before the current window is decoded and multiplied.
#include <atomic>

#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kLinThreads = 256;          // two CTAs per SM: one wave for N <= 4736

template <int DT>
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    if constexpr (DT == BF16)
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
                     "{%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    else
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
                     "{%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The decode table: entry (byte, r) = (code4[byte >> 4], code4[byte & 15]) at index byte * 16 + r,
// 16 interleaved replicas: the 16 lanes of an 8-byte shared-load phase read replica lane & 15,
// so they always hit 16 different bank pairs.
constexpr int kPairReplicas = 16;

// 16 weights of one W row from 8 code bytes (element 2j in the high nibble of byte j), as 8
// packed pairs of T: word j = (w[2j], w[2j+1]) with w[2j] in the low half.
template <int DT>
__device__ __forceinline__ void decode16(uint2 cw, float scale, const float2* pairs_r, uint32_t* w) {
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const uint32_t byte = ((j < 4 ? cw.x : cw.y) >> (8 * (j & 3))) & 0xffu;
        const float2 v = pairs_r[byte * kPairReplicas];             // (code4[hi], code4[lo])
        const float2 p = __fmul2_rn(v, make_float2(scale, scale));
        w[j] = DT == BF16 ? pack_bf16x2(p.x, p.y) : pack_f16x2(p.x, p.y);
    }
}

// Code bytes and scale inputs of one window for this lane's two W rows.
struct WinCodes {
    uint2 ca, cb;                 // 8 code bytes of W rows g and g + 8
    uint32_t qa, qb;              // their outer blocks' General8 codes
    float a2a, a2b;               // and inner absmax
};

__device__ __forceinline__ WinCodes load_codes(int64_t K, const uint8_t* codes, const uint8_t* absmax_q,
                                               const float* absmax2, int log2_bs, int64_t ra, int64_t rb,
                                               int64_t win, int t) {
    WinCodes r;
    const int64_t k0 = win * 64 + 16 * t;                           // this lane's 16 k
    const int64_t ea = ra * K + k0, eb = rb * K + k0;               // flattened element indices
    r.ca = __ldg(reinterpret_cast<const uint2*>(codes + (ea >> 1)));
    r.cb = __ldg(reinterpret_cast<const uint2*>(codes + (eb >> 1)));
    const int64_t ba = ea >> log2_bs, bb = eb >> log2_bs;           // outer blocks (16 k inside one)
    r.qa = __ldg(absmax_q + ba);
    r.qb = __ldg(absmax_q + bb);
    r.a2a = __ldg(absmax2 + (ba >> 8));
    r.a2b = __ldg(absmax2 + (bb >> 8));
    return r;
}

// 16 consecutive k of activation row m (zeros past M), from global memory or shared staging.
template <bool SMEM>
__device__ __forceinline__ void load_x(const uint16_t* X, const uint16_t* xs, int64_t xs_stride, int M,
                                       int64_t K, int m, int64_t k0, uint32_t* xb) {
    if (m < M) {
        const uint4* xp = SMEM ? reinterpret_cast<const uint4*>(xs + (int64_t)m * xs_stride + k0)
                               : reinterpret_cast<const uint4*>(X + (int64_t)m * K + k0);
        const uint4 x0 = SMEM ? xp[0] : __ldg(xp), x1 = SMEM ? xp[1] : __ldg(xp + 1);
        xb[0] = x0.x; xb[1] = x0.y; xb[2] = x0.z; xb[3] = x0.w;
        xb[4] = x1.x; xb[5] = x1.y; xb[6] = x1.z; xb[7] = x1.w;
    } else {
#pragma unroll
        for (int j = 0; j < 8; j++) xb[j] = 0u;
    }
}

// Windows whose code loads are issued together (registers allow fewer as M grows).
template <int NT> constexpr int kBatch = NT == 1 ? 4 : 2;
constexpr size_t kMaxXs = 72 * 1024;        // largest shared staging of X (two CTAs per SM)

// With XS (M <= 8 and X small enough) X is staged in shared memory (rows padded by 8 elements:
// conflict-free fragment reads); otherwise it is read from global memory (it stays in L2).
template <int DT, int NT, bool XS>
__global__ void __launch_bounds__(kLinThreads, 2)
linear4_nested_kernel(const uint16_t* __restrict__ X, int M, int64_t N, int64_t K,
                      const uint8_t* __restrict__ codes, const uint8_t* __restrict__ absmax_q,
                      const float* __restrict__ code2, const float* __restrict__ absmax2, float offset,
                      const float* __restrict__ code4, int log2_bs, uint16_t* __restrict__ Y) {
    constexpr int NWARP = kLinThreads / 32;
    constexpr int B = kBatch<NT>;
    __shared__ float c2[256];
    __shared__ float red[NWARP][32][4 * NT];
    extern __shared__ __align__(16) unsigned char dsm[];       // decode table (32 KB), then X
    float2* pairs = reinterpret_cast<float2*>(dsm);
    uint16_t* xs = reinterpret_cast<uint16_t*>(dsm + 256 * kPairReplicas * sizeof(float2));   // [M][K + 8]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t r0 = (int64_t)blockIdx.x * 16;
    const int64_t ra = r0 + g, rb = r0 + g + 8;
    const int64_t nwin = K >> 6;
    const int64_t w_lo = nwin * warp / NWARP, w_hi = nwin * (warp + 1) / NWARP;
    const int64_t xs_stride = K + 8;

    // the first batch of code loads goes out before the tables and X are staged
    WinCodes wc[B];
#pragma unroll
    for (int i = 0; i < B; i++)
        if (w_lo + i < w_hi) wc[i] = load_codes(K, codes, absmax_q, absmax2, log2_bs, ra, rb, w_lo + i, t);
    {
        // code4 held once per warp (lane l: entry l & 15); table entries built by shuffles
        const float c4 = __ldg(code4 + (lane & 15));
        if (threadIdx.x < 256) c2[threadIdx.x] = __ldg(code2 + threadIdx.x);
#pragma unroll 4
        for (int i = threadIdx.x; i < 256 * kPairReplicas; i += kLinThreads) {
            const int byte = i / kPairReplicas;
            const float hi = __shfl_sync(0xffffffffu, c4, byte >> 4);
            const float lo = __shfl_sync(0xffffffffu, c4, byte & 15);
            pairs[i] = make_float2(hi, lo);
        }
    }
    const float2* pairs_r = pairs + (lane & (kPairReplicas - 1));
    if (XS) {
        // asynchronous 16-byte copies (L2 -> shared), all in flight at once
        const int64_t chunks = (int64_t)M * (K / 8);               // 16-byte chunks of X
        const uint32_t xs_s = (uint32_t)__cvta_generic_to_shared(xs);
        for (int64_t c = threadIdx.x; c < chunks; c += kLinThreads) {
            const int64_t m = c / (K / 8), kk = (c % (K / 8)) * 8;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                         :: "r"(xs_s + (uint32_t)((m * xs_stride + kk) * 2)), "l"(X + m * K + kk) : "memory");
        }
        asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();

    float acc[NT][4];
#pragma unroll
    for (int q = 0; q < NT; q++) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;

    for (int64_t wb0 = w_lo; wb0 < w_hi; wb0 += B) {
#pragma unroll
        for (int i = 0; i < B; i++) {
            const int64_t win = wb0 + i;
            if (win >= w_hi) break;
            const int64_t k0 = win * 64 + 16 * t;
            uint32_t xb[NT][8];
#pragma unroll
            for (int q = 0; q < NT; q++) load_x<XS>(X, xs, xs_stride, M, K, q * 8 + g, k0, xb[q]);
            const float sa = __fadd_rn(__fmul_rn(c2[wc[i].qa], wc[i].a2a), offset);
            const float sb = __fadd_rn(__fmul_rn(c2[wc[i].qb], wc[i].a2b), offset);
            uint32_t wa[8], wbv[8];
            decode16<DT>(wc[i].ca, sa, pairs_r, wa);
            decode16<DT>(wc[i].cb, sb, pairs_r, wbv);
            // the same slot of the next batch can be refilled as soon as this one is decoded
            if (win + B < w_hi) wc[i] = load_codes(K, codes, absmax_q, absmax2, log2_bs, ra, rb, win + B, t);
#pragma unroll
            for (int q = 0; q < NT; q++)
#pragma unroll
                for (int s = 0; s < 4; s++) {
                    const uint32_t a[4] = {wa[2 * s], wbv[2 * s], wa[2 * s + 1], wbv[2 * s + 1]};
                    mma16816<DT>(acc[q], a, xb[q][2 * s], xb[q][2 * s + 1]);
                }
        }
    }

    // split-K partials: warp w's fragment in red[w], summed in warp order by warp 0
#pragma unroll
    for (int q = 0; q < NT; q++)
#pragma unroll
        for (int i = 0; i < 4; i++) red[warp][lane][4 * q + i] = acc[q][i];
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int q = 0; q < NT; q++) {
        float y[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            float s = red[0][lane][4 * q + i];
            for (int w = 1; w < NWARP; w++) s = __fadd_rn(s, red[w][lane][4 * q + i]);
            y[i] = s;
        }
        // c0, c1: W row g, activation rows 2t, 2t+1; c2, c3: W row g + 8
        const int m0 = q * 8 + 2 * t;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int m = m0 + (i & 1);
            const int64_t nn = (i < 2) ? ra : rb;
            if (m < M) {
                const uint16_t h = DT == BF16 ? f32_to_bf16_bits(y[i]) : f32_to_f16_bits(y[i]);
                Y[(int64_t)m * N + nn] = h;
            }
        }
    }
}

template <int DT, int NT, bool XS>
cudaError_t launch_nt(const uint16_t* X, int M, int64_t N, int64_t K, const uint8_t* codes,
                      const uint8_t* absmax_q, const float* code2, const float* absmax2, float offset,
                      const float* code4, int log2_bs, uint16_t* Y, cudaStream_t s) {
    auto k = linear4_nested_kernel<DT, NT, XS>;
    constexpr size_t kTable = 256 * kPairReplicas * sizeof(float2);
    const size_t dyn = kTable + (XS ? (size_t)M * (size_t)(K + 8) * 2 : 0);
    {
        // the dynamic shared-memory limit is set once per device (function attributes are per device)
        static std::atomic<uint64_t> attr_set{0};
        int dev = 0;
        cudaGetDevice(&dev);
        const uint64_t bit = 1ull << (dev & 63);
        if (!(attr_set.load() & bit)) {
            const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)(kTable + (XS ? kMaxXs : 0)));
            if (e != cudaSuccess) return e;
            attr_set.fetch_or(bit);
        }
    }
    k<<<(unsigned)(N / 16), kLinThreads, dyn, s>>>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4,
                                                   log2_bs, Y);
    return cudaGetLastError();
}

template <int DT>
cudaError_t launch_dt(const uint16_t* X, int M, int64_t N, int64_t K, const uint8_t* codes,
                      const uint8_t* absmax_q, const float* code2, const float* absmax2, float offset,
                      const float* code4, int log2_bs, uint16_t* Y, cudaStream_t s) {
    switch ((M + 7) / 8) {
        case 1:
            if ((size_t)M * (size_t)(K + 8) * 2 <= kMaxXs)
                return launch_nt<DT, 1, true>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
            return launch_nt<DT, 1, false>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
        case 2: return launch_nt<DT, 2, false>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
        case 3: return launch_nt<DT, 3, false>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
        default: return launch_nt<DT, 4, false>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
    }
}

}  // namespace

cudaError_t launch_linear_4bit_nested(const void* X, int dtype, int M, int64_t N, int64_t K,
                                      const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                                      const float* absmax2, float offset, const float* code4, int log2_bs,
                                      void* Y, cudaStream_t s) {
    const uint16_t* x = static_cast<const uint16_t*>(X);
    uint16_t* y = static_cast<uint16_t*>(Y);
    if (dtype == BF16) return launch_dt<BF16>(x, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, y, s);
    return launch_dt<F16>(x, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, y, s);
}

}  // namespace bbc
