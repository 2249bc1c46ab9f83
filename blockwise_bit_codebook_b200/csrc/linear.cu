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
// warp walks windows of K (a 64-wide window ends the row when 128-wide windows leave 64) with
// mma.sync m16n8k16 (T inputs, fp32 accumulators), one n-tile per 8 activation rows (M <= 32).
// Both operands use the same permutation of the 16 k-slots of each mma step s: the slots of
// lane-quad t are k = (W/4) t + 4 s + 0..3 for a window of width W, so a lane needs W/4
// consecutive k of a window: one 16-byte (8-byte) load of code bytes per W row, all inside one
// outer block (blocksize >= 32), so one scale per row per window, and W/2 contiguous bytes of
// each activation row. Windows are 128 wide when the activations are staged in shared memory
// (M <= 8) and 64 wide when they are read from global memory (the quad's loads of a row then
// stay within one 128-byte line). Each code byte is decoded through a 256-entry shared table of
// the pair (code4[hi], code4[lo]) (one shift and one logic operation form the table address),
// multiplied by the block scale (paired fp32 multiply) and rounded to T. The code loads of the
// next windows are in flight while the current one is decoded and multiplied.
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kLinThreads = 256;          // two CTAs per SM: one wave for N <= 4736
constexpr int kNWarp = kLinThreads / 32;

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

// The decode table: entry (byte, r) = (code4[byte >> 4], code4[byte & 15]) at byte offset
// byte * 128 + r * 8, 16 interleaved replicas: the 16 lanes of an 8-byte shared-load phase read
// replica lane & 15, so they always hit 16 different bank pairs.
constexpr int kPairReplicas = 16;
constexpr int kPairBytes = 256 * kPairReplicas * 8;      // 32 KB
static_assert(kPairReplicas * 8 == 128, "one table entry spans bits 7..14 of the byte offset");

// Two weights (w[2j], w[2j+1] of this lane's run, w[2j] in the low half) from byte J of `word`:
// the byte moved to bits 7..14 is the entry's offset, the lane's replica is or-ed in.
template <int DT, int J>
__device__ __forceinline__ uint32_t decode_byte(uint32_t word, uint32_t lane_off, float2 scale,
                                                const unsigned char* table) {
    const uint32_t sel = (J == 0 ? (word << 7) : (word >> (8 * J - 7))) & 0x7f80u;
    const float2 v = *reinterpret_cast<const float2*>(table + (sel | lane_off));
    const float2 p = __fmul2_rn(v, scale);
    return DT == BF16 ? pack_bf16x2(p.x, p.y) : pack_f16x2(p.x, p.y);
}

// Code bytes and scale inputs of one window for this lane's two W rows (g and g + 8). Lane t of
// a row quad takes the W/4 consecutive k from (W/4) t: one 16-byte (8-byte) code load per row,
// all inside one outer block (blocksize >= 32 >= W/4, and the run starts at a multiple of W/4),
// so one scale per row per window.
template <int W>
struct Win {
    uint32_t ca[W / 32], cb[W / 32];      // code word c: the lane's k 8c .. 8c + 7 of the window
    uint32_t qa, qb;                      // the General8 code of each row's outer block
    float a2a, a2b;                       // and its inner absmax
};

// ea, eb: flattened index of the window's first weight in rows g and g + 8.
template <int W>
__device__ __forceinline__ void load_win(Win<W>& r, const uint8_t* codes, const uint8_t* absmax_q,
                                         const float* absmax2, int log2_bs, int64_t ea, int64_t eb, int t,
                                         int64_t nw) {
    const int64_t la = ea + (W / 4) * t, lb = eb + (W / 4) * t;
    if (!BBC_GUARD(la >= 0 && lb >= 0 && la + W / 4 <= nw && lb + W / 4 <= nw, kGuardLinear)) {
        r = Win<W>{};
        return;
    }
    if constexpr (W == 128) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(codes + (la >> 1)));
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(codes + (lb >> 1)));
        r.ca[0] = a.x; r.ca[1] = a.y; r.ca[2] = a.z; r.ca[3] = a.w;
        r.cb[0] = b.x; r.cb[1] = b.y; r.cb[2] = b.z; r.cb[3] = b.w;
    } else {
        const uint2 a = __ldg(reinterpret_cast<const uint2*>(codes + (la >> 1)));
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(codes + (lb >> 1)));
        r.ca[0] = a.x; r.ca[1] = a.y;
        r.cb[0] = b.x; r.cb[1] = b.y;
    }
    const int64_t ba = la >> log2_bs, bb = lb >> log2_bs;
    r.qa = __ldg(absmax_q + ba);
    r.qb = __ldg(absmax_q + bb);
    r.a2a = __ldg(absmax2 + (ba >> 8));
    r.a2b = __ldg(absmax2 + (bb >> 8));
}

// Code words W0 .. W1-1 of a window of width W for this lane: the activation words xw (word 4c + i:
// the lane's k 8c + 2i, 8c + 2i + 1) and the rows' scales; decodes both rows' codes and runs their
// mma steps (two per word).
template <int DT, int NT, int W, int W0, int W1>
__device__ __forceinline__ void mma_win(float (&acc)[NT][4], const Win<W>& wc, float2 sa2, float2 sb2,
                                        const uint32_t (&xw)[NT][W / 8], const unsigned char* table,
                                        uint32_t lane_off) {
#pragma unroll
    for (int w = W0; w < W1; w++) {
        // code word w holds the bytes of mma steps 2w and 2w + 1
        const uint32_t wa = wc.ca[w], wb = wc.cb[w];
        uint32_t a[2][4];
        a[0][0] = decode_byte<DT, 0>(wa, lane_off, sa2, table);
        a[0][1] = decode_byte<DT, 0>(wb, lane_off, sb2, table);
        a[0][2] = decode_byte<DT, 1>(wa, lane_off, sa2, table);
        a[0][3] = decode_byte<DT, 1>(wb, lane_off, sb2, table);
        a[1][0] = decode_byte<DT, 2>(wa, lane_off, sa2, table);
        a[1][1] = decode_byte<DT, 2>(wb, lane_off, sb2, table);
        a[1][2] = decode_byte<DT, 3>(wa, lane_off, sa2, table);
        a[1][3] = decode_byte<DT, 3>(wb, lane_off, sb2, table);
#pragma unroll
        for (int q = 0; q < NT; q++) {
            mma16816<DT>(acc[q], a[0], xw[q][4 * w], xw[q][4 * w + 1]);
            mma16816<DT>(acc[q], a[1], xw[q][4 * w + 2], xw[q][4 * w + 3]);
        }
    }
}

// One window: xr[q] is the lane's activation row of n-tile q (rows past M repeat row M - 1:
// their outputs are never stored), in shared or global memory; kw is the window's first k.
template <int DT, int NT, int W>
__device__ __forceinline__ void run_win(float (&acc)[NT][4], const Win<W>& wc, const float* c2s, float offset,
                                        const unsigned char* table, uint32_t lane_off,
                                        const uint16_t* const (&xr)[NT], int64_t kw, int t) {
    // activation words of chunks C0 .. C1-1 (chunk c: the lane's k 8c .. 8c + 7)
    uint32_t xw[NT][W / 8];
    auto load_x = [&](auto c0, auto c1) {
#pragma unroll
        for (int q = 0; q < NT; q++)
#pragma unroll
            for (int c = decltype(c0)::value; c < decltype(c1)::value; c++) {
                const uint4 x = *reinterpret_cast<const uint4*>(xr[q] + kw + (W / 4) * t + 8 * c);
                xw[q][4 * c + 0] = x.x; xw[q][4 * c + 1] = x.y; xw[q][4 * c + 2] = x.z; xw[q][4 * c + 3] = x.w;
            }
    };
    // with three or four n-tiles the second half of a 128-wide window is fetched after the first
    // half's mma steps (registers)
    constexpr int CH = (NT >= 3 && W == 128) ? 2 : W / 32;
    load_x(std::integral_constant<int, 0>{}, std::integral_constant<int, CH>{});
    const float sa = __fadd_rn(__fmul_rn(c2s[wc.qa], wc.a2a), offset);
    const float sb = __fadd_rn(__fmul_rn(c2s[wc.qb], wc.a2b), offset);
    const float2 sa2 = make_float2(sa, sa), sb2 = make_float2(sb, sb);
    mma_win<DT, NT, W, 0, CH>(acc, wc, sa2, sb2, xw, table, lane_off);
    if constexpr (CH < W / 32) {
        load_x(std::integral_constant<int, CH>{}, std::integral_constant<int, W / 32>{});
        mma_win<DT, NT, W, CH, W / 32>(acc, wc, sa2, sb2, xw, table, lane_off);
    }
}

// Windows whose code loads are issued together: 512, 256 or 128 k of codes in flight per lane
// (registers allow fewer as M grows).
template <int NT, int W> constexpr int kBatch = (NT == 1 ? 512 : NT == 2 ? 256 : 128) / W;
constexpr size_t kMaxXs = 72 * 1024;        // largest shared staging of X (two CTAs per SM)

// X[M][K] into shared memory rows of K + 8 elements with asynchronous 16-byte copies (L2 ->
// shared), all in flight at once; the caller's barrier publishes them.
__device__ __forceinline__ void stage_x(const uint16_t* X, uint16_t* xs, int M, int64_t K) {
    const int64_t chunks = (int64_t)M * (K / 8);
    const int64_t xs_stride = K + 8;
    const uint32_t xs_s = (uint32_t)__cvta_generic_to_shared(xs);
    for (int64_t c = threadIdx.x; c < chunks; c += kLinThreads) {
        const int64_t m = c / (K / 8), kk = (c % (K / 8)) * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                     :: "r"(xs_s + (uint32_t)((m * xs_stride + kk) * 2)), "l"(X + m * K + kk) : "memory");
    }
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

// Split-K partials: warp w's fragment in red[w], summed in warp order by warp 0, which rounds
// each sum once to T and stores it (c0, c1: W row g, activation rows 2t, 2t + 1; c2, c3: row
// g + 8). Called by every thread of the CTA after the last read of whatever `red` overlays.
template <int DT, int NT>
__device__ __forceinline__ void reduce_store(float (*red)[32][4 * NT], const float (&acc)[NT][4], int M,
                                             int64_t N, int64_t ra, int64_t rb, uint16_t* Y) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, t = lane & 3;
    __syncthreads();
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
            for (int w = 1; w < kNWarp; w++) s = __fadd_rn(s, red[w][lane][4 * q + i]);
            y[i] = s;
        }
        const int m0 = q * 8 + 2 * t;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int m = m0 + (i & 1);
            const int64_t nn = (i < 2) ? ra : rb;
            if (m < M) Y[(int64_t)m * N + nn] = DT == BF16 ? f32_to_bf16_bits(y[i]) : f32_to_f16_bits(y[i]);
        }
    }
}

// With XS (M <= 8 and X small enough) X is staged in shared memory (rows padded by 8 elements);
// otherwise it is read from global memory (it stays in L2).
template <int DT, int NT, bool XS>
__global__ void __launch_bounds__(kLinThreads, 2)
linear4_nested_kernel(const uint16_t* __restrict__ X, int M, int64_t N, int64_t K,
                      const uint8_t* __restrict__ codes, const uint8_t* __restrict__ absmax_q,
                      const float* __restrict__ code2, const float* __restrict__ absmax2, float offset,
                      const float* __restrict__ code4, int log2_bs, uint16_t* __restrict__ Y) {
    static_assert(kLinThreads == 256, "the table build gives one thread to each of the 256 code bytes");
    // windows of 128 k with X in shared memory; of 64 k with X in global memory, where a lane's
    // 32-byte run keeps the quad's activation loads of a row within one 128-byte line
    constexpr int WM = XS ? 128 : 64;
    constexpr int B = kBatch<NT, WM>;
    __shared__ __align__(16) unsigned char table[kPairBytes];   // decode table; then the split-K partials
    __shared__ float c2s[256];
    extern __shared__ __align__(16) uint16_t xs[];              // [M][K + 8] staged X (XS only)

    pdl_wait();               // writes of the previous kernel in the stream are visible from here
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t r0 = (int64_t)blockIdx.x * 16;
    const int64_t ra = r0 + g, rb = r0 + g + 8;
    const int64_t nwin = K / WM;                                 // full-width windows
    const int64_t w_lo = nwin * warp / kNWarp, w_hi = nwin * (warp + 1) / kNWarp;
    const int64_t ea0 = ra * K, eb0 = rb * K;                    // first weight of rows g, g + 8

    // the first batch of code loads goes out before the tables and X are staged
    Win<WM> wc[B];
#pragma unroll
    for (int i = 0; i < B; i++)
        if (w_lo + i < w_hi)
            load_win<WM>(wc[i], codes, absmax_q, absmax2, log2_bs, ea0 + (w_lo + i) * WM,
                         eb0 + (w_lo + i) * WM, t, N * K);
    {
        // thread i writes the 16 replicas of entry i as 8 rotated 16-byte stores (each store
        // phase of 8 threads covers all 32 banks)
        const int byte = threadIdx.x;
        const float hi = __ldg(code4 + (byte >> 4)), lo = __ldg(code4 + (byte & 15));
        const float4 v = make_float4(hi, lo, hi, lo);
#pragma unroll
        for (int r = 0; r < kPairReplicas / 2; r++)
            *reinterpret_cast<float4*>(table + byte * 128 + ((r + byte) & 7) * 16) = v;
        c2s[byte] = __ldg(code2 + byte);
    }
    if (XS) stage_x(X, xs, M, K);
    __syncthreads();

    const uint32_t lane_off = (uint32_t)(lane & (kPairReplicas - 1)) * 8u;
    const uint16_t* xr[NT];
#pragma unroll
    for (int q = 0; q < NT; q++) {
        const int m = min(q * 8 + g, M - 1);
        xr[q] = XS ? xs + m * (K + 8) : X + (int64_t)m * K;
    }
    float acc[NT][4];
#pragma unroll
    for (int q = 0; q < NT; q++) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;

    for (int64_t wb0 = w_lo; wb0 < w_hi; wb0 += B) {
#pragma unroll
        for (int i = 0; i < B; i++) {
            const int64_t win = wb0 + i;
            if (win >= w_hi) break;
            run_win<DT, NT, WM>(acc, wc[i], c2s, offset, table, lane_off, xr, win * WM, t);
            // the slot is refilled with the window B ahead once this one is decoded
            if (win + B < w_hi)
                load_win<WM>(wc[i], codes, absmax_q, absmax2, log2_bs, ea0 + (win + B) * WM,
                             eb0 + (win + B) * WM, t, N * K);
        }
    }
    if (WM == 128 && (K & 64) && warp == kNWarp - 1) {
        // the last 64 k of every row
        Win<64> tw;
        load_win<64>(tw, codes, absmax_q, absmax2, log2_bs, ea0 + K - 64, eb0 + K - 64, t, N * K);
        run_win<DT, NT, 64>(acc, tw, c2s, offset, table, lane_off, xr, K - 64, t);
    }
    // the partials overlay the decode table, which no warp reads any more after the barrier
    static_assert(kNWarp * 32 * 4 * 4 * sizeof(float) <= kPairBytes, "partials fit over the table");
    reduce_store<DT, NT>(reinterpret_cast<float (*)[32][4 * NT]>(table), acc, M, N, ra, rb, Y);
}

// ---- k-bit weights (K = 2..5, blocksize 32, bit-plane packed, fp32 absmax) ----
//
// The weight of the k-bit patch series' dequantize_kbit: w[n][k] = T(fl(codebook[idx] *
// absmax[b])) for flattened element m = n*K + k in block b = m / 32, idx gathered from the K
// plane words of block b. With K % 64 == 0 blocks never straddle rows, and the lane's run of a
// window (32 k for 128-wide windows, 16 for 64-wide) lies in one block: one absmax and the
// block's K words per row per window. Each element's index is gathered from the byte-transposed
// plane groups with one multiply-high (as in the dequant kernel), looked up in a 32-float shared
// codebook (every entry its own bank), multiplied by the absmax and rounded to T in pairs.

template <int KB>
struct KWin {
    uint32_t wa[KB], wb[KB];              // plane words of the block holding the lane's run, rows g, g + 8
    float ama, amb;                       // and the blocks' absmax
};

// ea, eb: flattened index of the window's first weight in rows g and g + 8. `packed` is 16-byte
// aligned, so block b's words start on a 16-byte (K = 4) or 8-byte (K = 2) boundary.
template <int KB, int W>
__device__ __forceinline__ void load_kwin(KWin<KB>& r, const uint32_t* packed, const float* absmax, int64_t ea,
                                          int64_t eb, int t, int64_t nw) {
    const int64_t ba = (ea + (W / 4) * t) >> 5, bb = (eb + (W / 4) * t) >> 5;
    if (!BBC_GUARD(ba >= 0 && bb >= 0 && (ba + 1) * 32 <= nw && (bb + 1) * 32 <= nw, kGuardLinear)) {
        r = KWin<KB>{};
        return;
    }
    const uint32_t* pa = packed + ba * KB;
    const uint32_t* pb = packed + bb * KB;
    if constexpr (KB == 4) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(pa)), b = __ldg(reinterpret_cast<const uint4*>(pb));
        r.wa[0] = a.x; r.wa[1] = a.y; r.wa[2 % KB] = a.z; r.wa[3 % KB] = a.w;
        r.wb[0] = b.x; r.wb[1] = b.y; r.wb[2 % KB] = b.z; r.wb[3 % KB] = b.w;
    } else if constexpr (KB == 2) {
        const uint2 a = __ldg(reinterpret_cast<const uint2*>(pa)), b = __ldg(reinterpret_cast<const uint2*>(pb));
        r.wa[0] = a.x; r.wa[1 % KB] = a.y;
        r.wb[0] = b.x; r.wb[1 % KB] = b.y;
    } else {
#pragma unroll
        for (int j = 0; j < KB; j++) { r.wa[j] = ldg_u32(pa + j); r.wb[j] = ldg_u32(pb + j); }
    }
    r.ama = __ldg(absmax + ba);
    r.amb = __ldg(absmax + bb);
}

template <int KB, int DT>
__device__ __forceinline__ void kbit_group(uint32_t Bq, uint32_t p4q, float am, const char* cbb, uint32_t (&pr)[4]) {
    const uint32_t Bqs = Bq << 3;
    const float y0 = kbit_elem<KB, DT, 0>(Bq, Bqs, p4q, am, cbb), y1 = kbit_elem<KB, DT, 1>(Bq, Bqs, p4q, am, cbb);
    const float y2 = kbit_elem<KB, DT, 2>(Bq, Bqs, p4q, am, cbb), y3 = kbit_elem<KB, DT, 3>(Bq, Bqs, p4q, am, cbb);
    const float y4 = kbit_elem<KB, DT, 4>(Bq, Bqs, p4q, am, cbb), y5 = kbit_elem<KB, DT, 5>(Bq, Bqs, p4q, am, cbb);
    const float y6 = kbit_elem<KB, DT, 6>(Bq, Bqs, p4q, am, cbb), y7 = kbit_elem<KB, DT, 7>(Bq, Bqs, p4q, am, cbb);
    pr[0] = DT == BF16 ? pack_bf16x2(y0, y1) : pack_f16x2(y0, y1);
    pr[1] = DT == BF16 ? pack_bf16x2(y2, y3) : pack_f16x2(y2, y3);
    pr[2] = DT == BF16 ? pack_bf16x2(y4, y5) : pack_f16x2(y4, y5);
    pr[3] = DT == BF16 ? pack_bf16x2(y6, y7) : pack_f16x2(y6, y7);
}

// K <= 4: the same eight weights through a table of (codebook[a], codebook[b]) pairs. The 8 plane
// bits of elements 2i, 2i + 1 (bits 8j + 2i + s of Bq) are gathered by one wide multiply into an
// 8-bit index: multiplier 2^30 + 2^20 + 2^10 + 1 moves bit 8j + 2i + s to bit 24 + 2i + 2(3 - j) + s;
// every cross term lands outside those 8 bits on a position of its own, so no carry reaches them
// (checked over all 256 bit patterns at each i). Entry i of the table is (codebook[a], codebook[b])
// with a = sum_j bit(i, 6 - 2j) 2^j, b = sum_j bit(i, 7 - 2j) 2^j, 16 lane-interleaved replicas.
template <int DT>
__device__ __forceinline__ void kbit_group_pairs(uint32_t Bq, float am, uint32_t lane_off, const unsigned char* table,
                                                 uint32_t (&pr)[4]) {
    const float2 sc = make_float2(am, am);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint64_t prod = (uint64_t)(Bq & (0x03030303u << (2 * i))) * 0x40100401u;
        const uint32_t sel = (uint32_t)(prod >> (17 + 2 * i)) & 0x7f80u;          // index * 128
        const float2 v = *reinterpret_cast<const float2*>(table + (sel | lane_off));
        const float2 p = __fmul2_rn(v, sc);
        pr[i] = DT == BF16 ? pack_bf16x2(p.x, p.y) : pack_f16x2(p.x, p.y);
    }
}

// One window of width W: the lane's run of W/4 weights in rows g and g + 8, decoded group by
// group (8 weights = one code word's worth of mma steps) into the same fragments as the nested
// kernel's.
template <int DT, int NT, int KB, int W>
__device__ __forceinline__ void run_kwin(float (&acc)[NT][4], const KWin<KB>& wc, const char* cbb,
                                         const unsigned char* table, uint32_t lane_off,
                                         const uint16_t* const (&xr)[NT], int64_t kw, int t) {
    constexpr int R = W / 4;
    uint32_t xw[NT][W / 8];
#pragma unroll
    for (int q = 0; q < NT; q++)
#pragma unroll
        for (int c = 0; c < R / 8; c++) {
            const uint4 x = *reinterpret_cast<const uint4*>(xr[q] + kw + R * t + 8 * c);
            xw[q][4 * c + 0] = x.x; xw[q][4 * c + 1] = x.y; xw[q][4 * c + 2] = x.z; xw[q][4 * c + 3] = x.w;
        }
    uint32_t Ga[R / 8], Gb[R / 8], p4a, p4b;
    kbit_groups<KB, R>(wc.wa, t & 1, Ga, p4a);
    kbit_groups<KB, R>(wc.wb, t & 1, Gb, p4b);
#pragma unroll
    for (int w = 0; w < R / 8; w++) {
        uint32_t pa[4], pb[4];
        if constexpr (KB <= 4) {
            kbit_group_pairs<DT>(Ga[w], wc.ama, lane_off, table, pa);
            kbit_group_pairs<DT>(Gb[w], wc.amb, lane_off, table, pb);
        } else {
            kbit_group<KB, DT>(Ga[w], p4a >> (8 * w), wc.ama, cbb, pa);
            kbit_group<KB, DT>(Gb[w], p4b >> (8 * w), wc.amb, cbb, pb);
        }
        const uint32_t a0[4] = {pa[0], pb[0], pa[1], pb[1]};
        const uint32_t a1[4] = {pa[2], pb[2], pa[3], pb[3]};
#pragma unroll
        for (int q = 0; q < NT; q++) {
            mma16816<DT>(acc[q], a0, xw[q][4 * w], xw[q][4 * w + 1]);
            mma16816<DT>(acc[q], a1, xw[q][4 * w + 2], xw[q][4 * w + 3]);
        }
    }
}

template <int DT, int NT, bool XS, int KB>
__global__ void __launch_bounds__(kLinThreads, 2)
linear_kbit_kernel(const uint16_t* __restrict__ X, int M, int64_t N, int64_t K,
                   const uint32_t* __restrict__ packed, const float* __restrict__ absmax,
                   const float* __restrict__ codebook, uint16_t* __restrict__ Y) {
    constexpr int WM = XS ? 128 : 64;
    constexpr int B = kBatch<NT, WM> < 4 ? kBatch<NT, WM> : 4;   // a window holds 2 (K + 1) registers
    constexpr bool PAIRS = KB <= 4;                              // pair table (else per-weight codebook)
    __shared__ float cbs[32];
    __shared__ __align__(16) unsigned char table[PAIRS ? kPairBytes : 16];     // then the split-K partials
    __shared__ __align__(16) float red5[PAIRS ? 1 : kNWarp * 32 * 4 * NT];     // split-K partials (K = 5)
    extern __shared__ __align__(16) uint16_t xs[];              // [M][K + 8] staged X (XS only)

    pdl_wait();               // writes of the previous kernel in the stream are visible from here
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t r0 = (int64_t)blockIdx.x * 16;
    const int64_t ra = r0 + g, rb = r0 + g + 8;
    const int64_t nwin = K / WM;
    const int64_t w_lo = nwin * warp / kNWarp, w_hi = nwin * (warp + 1) / kNWarp;
    const int64_t ea0 = ra * K, eb0 = rb * K;

    KWin<KB> wc[B];
#pragma unroll
    for (int i = 0; i < B; i++)
        if (w_lo + i < w_hi) load_kwin<KB, WM>(wc[i], packed, absmax, ea0 + (w_lo + i) * WM, eb0 + (w_lo + i) * WM, t, N * K);
    if (threadIdx.x < 32) cbs[threadIdx.x] = threadIdx.x < (1 << KB) ? __ldg(codebook + threadIdx.x) : 0.0f;
    if constexpr (PAIRS) {
        // thread i writes the 16 replicas of entry i (rotated 16-byte stores, as the nested table)
        const int i = threadIdx.x;
        int a = 0, b = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            a |= ((i >> (6 - 2 * j)) & 1) << j;
            b |= ((i >> (7 - 2 * j)) & 1) << j;
        }
        const float ca = __ldg(codebook + (a & ((1 << KB) - 1))), cbv = __ldg(codebook + (b & ((1 << KB) - 1)));
        const float4 v = make_float4(ca, cbv, ca, cbv);
#pragma unroll
        for (int r = 0; r < kPairReplicas / 2; r++)
            *reinterpret_cast<float4*>(table + i * 128 + ((r + i) & 7) * 16) = v;
    }
    if (XS) stage_x(X, xs, M, K);
    __syncthreads();

    const char* cbb = reinterpret_cast<const char*>(cbs);
    const uint32_t lane_off = (uint32_t)(lane & (kPairReplicas - 1)) * 8u;
    const uint16_t* xr[NT];
#pragma unroll
    for (int q = 0; q < NT; q++) {
        const int m = min(q * 8 + g, M - 1);
        xr[q] = XS ? xs + m * (K + 8) : X + (int64_t)m * K;
    }
    float acc[NT][4];
#pragma unroll
    for (int q = 0; q < NT; q++) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;

    for (int64_t wb0 = w_lo; wb0 < w_hi; wb0 += B) {
#pragma unroll
        for (int i = 0; i < B; i++) {
            const int64_t win = wb0 + i;
            if (win >= w_hi) break;
            run_kwin<DT, NT, KB, WM>(acc, wc[i], cbb, table, lane_off, xr, win * WM, t);
            if (win + B < w_hi)
                load_kwin<KB, WM>(wc[i], packed, absmax, ea0 + (win + B) * WM, eb0 + (win + B) * WM, t, N * K);
        }
    }
    if (WM == 128 && (K & 64) && warp == kNWarp - 1) {
        KWin<KB> tw;
        load_kwin<KB, 64>(tw, packed, absmax, ea0 + K - 64, eb0 + K - 64, t, N * K);
        run_kwin<DT, NT, KB, 64>(acc, tw, cbb, table, lane_off, xr, K - 64, t);
    }
    // with the pair table the partials overlay it (no warp reads it after the barrier)
    reduce_store<DT, NT>(reinterpret_cast<float (*)[32][4 * NT]>(PAIRS ? static_cast<void*>(table)
                                                                       : static_cast<void*>(red5)),
                         acc, M, N, ra, rb, Y);
}

// The dynamic shared-memory limit of kernel `k` raised to `bytes`, once per device (function
// attributes are per device); one flag word per kernel instantiation.
template <typename Kernel>
cudaError_t allow_dyn_smem(Kernel k, std::atomic<uint64_t>& done, size_t bytes) {
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load() & bit) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done.fetch_or(bit);
    return e;
}

bool stage_in_smem(int M, int64_t K) { return M <= 8 && (size_t)M * (size_t)(K + 8) * 2 <= kMaxXs; }

template <int DT, int NT, bool XS>
cudaError_t launch_nt(const uint16_t* X, int M, int64_t N, int64_t K, const uint8_t* codes,
                      const uint8_t* absmax_q, const float* code2, const float* absmax2, float offset,
                      const float* code4, int log2_bs, uint16_t* Y, cudaStream_t s) {
    auto k = linear4_nested_kernel<DT, NT, XS>;
    static std::atomic<uint64_t> attr{0};
    const cudaError_t e = allow_dyn_smem(k, attr, XS ? kMaxXs : 0);
    if (e != cudaSuccess) return e;
    const size_t dyn = XS ? (size_t)M * (size_t)(K + 8) * 2 : 0;
    return launch_pdl(k, (unsigned)(N / 16), kLinThreads, dyn, s, X, M, N, K, codes, absmax_q, code2, absmax2, offset,
                      code4, log2_bs, Y);
}

template <int DT>
cudaError_t launch_dt(const uint16_t* X, int M, int64_t N, int64_t K, const uint8_t* codes,
                      const uint8_t* absmax_q, const float* code2, const float* absmax2, float offset,
                      const float* code4, int log2_bs, uint16_t* Y, cudaStream_t s) {
    switch ((M + 7) / 8) {
        case 1:
            if (stage_in_smem(M, K))
                return launch_nt<DT, 1, true>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
            return launch_nt<DT, 1, false>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
        case 2: return launch_nt<DT, 2, false>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
        case 3: return launch_nt<DT, 3, false>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
        default: return launch_nt<DT, 4, false>(X, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, Y, s);
    }
}

template <int DT, int NT, bool XS, int KB>
cudaError_t launch_kbit_nt(const uint16_t* X, int M, int64_t N, int64_t K, const uint32_t* packed,
                           const float* absmax, const float* codebook, uint16_t* Y, cudaStream_t s) {
    auto k = linear_kbit_kernel<DT, NT, XS, KB>;
    static std::atomic<uint64_t> attr{0};
    const cudaError_t e = allow_dyn_smem(k, attr, XS ? kMaxXs : 0);
    if (e != cudaSuccess) return e;
    const size_t dyn = XS ? (size_t)M * (size_t)(K + 8) * 2 : 0;
    return launch_pdl(k, (unsigned)(N / 16), kLinThreads, dyn, s, X, M, N, K, packed, absmax, codebook, Y);
}

template <int DT, int KB>
cudaError_t launch_kbit_k(const uint16_t* X, int M, int64_t N, int64_t K, const uint32_t* packed,
                          const float* absmax, const float* codebook, uint16_t* Y, cudaStream_t s) {
    switch ((M + 7) / 8) {
        case 1:
            if (stage_in_smem(M, K)) return launch_kbit_nt<DT, 1, true, KB>(X, M, N, K, packed, absmax, codebook, Y, s);
            return launch_kbit_nt<DT, 1, false, KB>(X, M, N, K, packed, absmax, codebook, Y, s);
        case 2: return launch_kbit_nt<DT, 2, false, KB>(X, M, N, K, packed, absmax, codebook, Y, s);
        case 3: return launch_kbit_nt<DT, 3, false, KB>(X, M, N, K, packed, absmax, codebook, Y, s);
        default: return launch_kbit_nt<DT, 4, false, KB>(X, M, N, K, packed, absmax, codebook, Y, s);
    }
}

template <int DT>
cudaError_t launch_kbit_dt(const uint16_t* X, int M, int64_t N, int64_t K, const uint32_t* packed,
                           const float* absmax, const float* codebook, int KB, uint16_t* Y, cudaStream_t s) {
    switch (KB) {
        case 2: return launch_kbit_k<DT, 2>(X, M, N, K, packed, absmax, codebook, Y, s);
        case 3: return launch_kbit_k<DT, 3>(X, M, N, K, packed, absmax, codebook, Y, s);
        case 4: return launch_kbit_k<DT, 4>(X, M, N, K, packed, absmax, codebook, Y, s);
        default: return launch_kbit_k<DT, 5>(X, M, N, K, packed, absmax, codebook, Y, s);
    }
}

}  // namespace

cudaError_t launch_linear_4bit_nested(const void* X, int dtype, int M, int64_t N, int64_t K,
                                      const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                                      const float* absmax2, float offset, const float* code4, int log2_bs,
                                      void* Y, cudaStream_t s) {
    if (M > 32)
        return launch_linear_4bit_nested_tc(X, dtype, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs,
                                            Y, s);
    const uint16_t* x = static_cast<const uint16_t*>(X);
    uint16_t* y = static_cast<uint16_t*>(Y);
    if (dtype == BF16) return launch_dt<BF16>(x, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, y, s);
    return launch_dt<F16>(x, M, N, K, codes, absmax_q, code2, absmax2, offset, code4, log2_bs, y, s);
}

cudaError_t launch_linear_kbit(const void* X, int dtype, int M, int64_t N, int64_t K, const uint32_t* packed,
                               const float* absmax, const float* codebook, int KB, void* Y, cudaStream_t s) {
    if (M > 32) return launch_linear_kbit_tc(X, dtype, M, N, K, packed, absmax, codebook, KB, Y, s);
    const uint16_t* x = static_cast<const uint16_t*>(X);
    uint16_t* y = static_cast<uint16_t*>(Y);
    if (dtype == BF16) return launch_kbit_dt<BF16>(x, M, N, K, packed, absmax, codebook, KB, y, s);
    return launch_kbit_dt<F16>(x, M, N, K, packed, absmax, codebook, KB, y, s);
}

BBC_GUARD_ACCESSOR(guard_status_linear)

}  // namespace bbc
