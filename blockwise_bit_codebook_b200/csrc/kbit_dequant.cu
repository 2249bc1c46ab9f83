// k-bit blockwise dequantization (K = 2..5, blocksize 32).
//
// Operation (bitsandbytes k-bit patch series, dequantize_kbit_ref and
// kDequantizeBlockwise_kbit): out[m] = T(codebook[idx_m] * absmax[m / 32]),
// where idx_m is gathered from the K bit-plane words of block m / 32.
//
// B200 layout, two forms chosen per launch on the host. Whole blocks (16-bit outputs, 32-byte
// aligned, at K = 5, for the E4M4 K = 3 case and below 2^26 elements): a thread owns a
// block, reads its absmax and K words once (one vector load when the packed array
// allows), byte-transposes them with eight permutes into four plane groups (byte j
// of group q = plane j of elements 8q..8q+7), decodes each 4-bit index with one
// multiply-high bit gather, and writes 16 outputs per 32-byte store, so every lane
// writes whole sectors; the next block's words are loaded before the current one is
// decoded. Half blocks (otherwise: long 16-bit streams and all fp32 outputs;
// always for the ragged last block and unaligned outputs): 16 elements per thread, the
// two lanes of a block read the same words and keep bytes 2h, 2h+1. The codebook lives in
// shared memory: 32 consecutive floats occupy the 32 banks once, so the per-element lookup
// never conflicts.
// Persistent grid-stride loops.
#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kThreads = 256;

template <int K>
struct BlockIn {
    float am;
    uint32_t w[K];
};

template <int K, typename AT>
__device__ __forceinline__ BlockIn<K> load_block(const uint32_t* packed, const AT* absmax,
                                                 int64_t b, bool active, int64_t nb) {
    BlockIn<K> r;
    if (active && BBC_GUARD(b >= 0 && b < nb, kGuardDequantIn)) {
        r.am = load_absmax(absmax, b);          // fp32 as stored, or the exact E4M4 value
        const uint32_t* wp = packed + b * K;
#pragma unroll
        for (int j = 0; j < K; j++) r.w[j] = ldg_u32(wp + j);
    } else {
        r.am = 0.0f;
#pragma unroll
        for (int j = 0; j < K; j++) r.w[j] = 0u;
    }
    return r;
}

// One whole block's absmax and K words (block b lies inside the input); one vector load of the
// words when `packed` allows it (K = 2: 8-byte, K = 4: 16-byte alignment of the array).
template <int K, typename AT>
__device__ __forceinline__ BlockIn<K> load_whole(const uint32_t* packed, const AT* absmax, int64_t b,
                                                 bool vec_words, int64_t n) {
    BlockIn<K> r;
    if (!BBC_GUARD(b >= 0 && (b + 1) * 32 <= n, kGuardDequantIn)) {
        r.am = 0.0f;
#pragma unroll
        for (int j = 0; j < K; j++) r.w[j] = 0u;
        return r;
    }
    r.am = load_absmax(absmax, b);
    const uint32_t* wp = packed + b * K;
    if (K == 4 && vec_words) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(wp));
        r.w[0] = v.x; r.w[1] = v.y; r.w[2 % K] = v.z; r.w[3 % K] = v.w;
    } else if (K == 2 && vec_words) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(wp));
        r.w[0] = v.x; r.w[1 % K] = v.y;
    } else {
#pragma unroll
        for (int j = 0; j < K; j++) r.w[j] = ldg_u32(wp + j);
    }
    return r;
}

// Decode a whole block (32 elements) and store it: byte-transpose the K words into four
// plane groups (byte j of group q = plane j of elements 8q .. 8q+7), gather each index with one
// multiply-high and write 64 bytes (128 for fp32) as whole 32-byte sectors.
template <int K, int DT>
__device__ __forceinline__ void decode_whole(const BlockIn<K>& in, const char* cbb, char* dst) {
    const uint32_t w0 = in.w[0], w1 = in.w[1 % K];
    const uint32_t w2 = K > 2 ? in.w[2 % K] : 0u, w3 = K > 3 ? in.w[3 % K] : 0u;
    const uint32_t t0 = prmt(w0, w1, 0x5140u), t1 = prmt(w0, w1, 0x7362u);
    const uint32_t t2 = prmt(w2, w3, 0x5140u), t3 = prmt(w2, w3, 0x7362u);
    const uint32_t B[4] = {prmt(t0, t2, 0x5410u), prmt(t0, t2, 0x7632u), prmt(t1, t3, 0x5410u),
                           prmt(t1, t3, 0x7632u)};
    const uint32_t p4 = K == 5 ? in.w[4 % K] : 0u;             // plane 4: bit i is element i
    const float am = in.am;
    // 16 elements per 32-byte store (a whole sector per lane); fp32 needs two per 16
#pragma unroll
    for (int g = 0; g < 2; g++) {
        uint32_t wv[DT == F32 ? 16 : 8];
#pragma unroll
        for (int qq = 0; qq < 2; qq++) {
            const int q = 2 * g + qq;
            const uint32_t Bq = B[q], Bqs = B[q] << 3;
            const uint32_t p4q = p4 >> (8 * q);
            float y[8];
#define BBC_DQW_ELEM(E)                                                                       \
            {                                                                                 \
                uint32_t off = plane_offset4<(E)>(Bq, Bqs);                                  \
                if constexpr (K == 5) off |= ((E) <= 6 ? (p4q << (6 - (E))) : (p4q >> ((E) - 6))) & 0x40u; \
                y[E] = __fmul_rn(*reinterpret_cast<const float*>(cbb + off), am);             \
            }
            BBC_DQW_ELEM(0) BBC_DQW_ELEM(1) BBC_DQW_ELEM(2) BBC_DQW_ELEM(3)
            BBC_DQW_ELEM(4) BBC_DQW_ELEM(5) BBC_DQW_ELEM(6) BBC_DQW_ELEM(7)
#undef BBC_DQW_ELEM
            pack8<DT>(y, wv + qq * (DT == F32 ? 8 : 4));
        }
        char* d = dst + g * 16 * dtype_size(DT);
        stg_v8(d, wv);
        if constexpr (DT == F32) stg_v8(d + 32, wv + 8);
    }
}

// VEC: 32-byte-aligned output, vector stores. WHOLE (with VEC): a thread owns whole blocks;
// otherwise half blocks (16 outputs per thread, the two lanes of a block read the same words).
template <int K, int DT, bool VEC, bool WHOLE, typename AT>
__global__ void __launch_bounds__(kThreads)
kbit_dequant_kernel(const uint32_t* __restrict__ packed, const AT* __restrict__ absmax,
                    const float* __restrict__ codebook, int64_t n, void* __restrict__ out) {
    __shared__ float cb[32];
    pdl_wait();               // writes of the previous kernel in the stream are visible from here
    // the codebook is published to shared memory after the first block's loads are issued
    const float cbv = threadIdx.x < (1u << K) ? codebook[threadIdx.x] : 0.0f;
    auto publish_codebook = [&]() {
        if (threadIdx.x < 32) cb[threadIdx.x] = cbv;
        __syncthreads();
    };
    const char* cbb = reinterpret_cast<const char*>(cb);

    const int64_t nh = ((n + 31) >> 5) * 2;                       // half blocks
    const uint32_t h = threadIdx.x & 1;
    // bytes 2h and 2h+1 of two words a, b -> [a.2h, b.2h, a.2h+1, b.2h+1]
    const uint32_t sel = (2 * h) | ((4 + 2 * h) << 4) | ((2 * h + 1) << 8) | ((5 + 2 * h) << 12);
    const int64_t stride = (int64_t)gridDim.x * kThreads;

    int64_t H0 = 0;                                                // first half block left
    if constexpr (VEC && WHOLE) {
        // whole blocks, one per thread, the next one's words prefetched
        const int64_t nbf = n >> 5;                                 // blocks entirely inside n
        const bool vec_words = (reinterpret_cast<uintptr_t>(packed) & (K == 4 ? 15u : 7u)) == 0;
        int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x;
        BlockIn<K> cb0;
        if (b < nbf) cb0 = load_whole<K, AT>(packed, absmax, b, vec_words, n);
        publish_codebook();
        if (b < nbf) {
            while (true) {
                const int64_t bn = b + stride;
                BlockIn<K> cb1;
                if (bn < nbf) cb1 = load_whole<K, AT>(packed, absmax, bn, vec_words, n);
                if (BBC_GUARD((b + 1) * 32 <= n, kGuardDequantOut))
                    decode_whole<K, DT>(cb0, cbb, reinterpret_cast<char*>(out) + b * 32 * dtype_size(DT));
                b = bn;
                if (b >= nbf) break;
                cb0 = cb1;
            }
        }
        H0 = 2 * nbf;
    }
    int64_t H = H0 + (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t nb = nh >> 1;
    BlockIn<K> cur = load_block<K, AT>(packed, absmax, H >> 1, H < nh, nb);
    if constexpr (!(VEC && WHOLE)) publish_codebook();
    for (; H < nh; H += stride) {
        const int64_t Hn = H + stride;
        const BlockIn<K> nxt = load_block<K, AT>(packed, absmax, Hn >> 1, Hn < nh, nb);

        uint32_t B0, B1;
        if constexpr (K == 2) {
            const uint32_t t = prmt(cur.w[0], cur.w[1], sel);
            B0 = prmt(t, 0u, 0x4410u);
            B1 = prmt(t, 0u, 0x4432u);
        } else {
            const uint32_t t01 = prmt(cur.w[0], cur.w[1], sel);
            const uint32_t t23 = K == 3 ? prmt(cur.w[2], 0u, (2 * h) | (4u << 4) | ((2 * h + 1) << 8) | (4u << 12))
                                        : prmt(cur.w[2], cur.w[K > 3 ? 3 : 2], sel);
            B0 = prmt(t01, t23, 0x5410u);
            B1 = prmt(t01, t23, 0x7632u);
        }
        uint32_t p4 = 0;
        if constexpr (K == 5) p4 = cur.w[4] >> (16 * h);           // plane 4: bit e is element e
        const uint32_t B0s = B0 << 3, B1s = B1 << 3;
        const float am = cur.am;

        float y[16];
#define BBC_DQ_ELEM(E)                                                                        \
        {                                                                                     \
            uint32_t off = (E) < 8 ? plane_offset4<(E) & 7>(B0, B0s) : plane_offset4<(E) & 7>(B1, B1s); \
            if constexpr (K == 5)                                                             \
                off |= ((E) <= 6 ? (p4 << (6 - (E))) : (p4 >> ((E) - 6))) & 0x40u;           \
            y[E] = __fmul_rn(*reinterpret_cast<const float*>(cbb + off), am);                 \
        }
        BBC_DQ_ELEM(0) BBC_DQ_ELEM(1) BBC_DQ_ELEM(2) BBC_DQ_ELEM(3)
        BBC_DQ_ELEM(4) BBC_DQ_ELEM(5) BBC_DQ_ELEM(6) BBC_DQ_ELEM(7)
        BBC_DQ_ELEM(8) BBC_DQ_ELEM(9) BBC_DQ_ELEM(10) BBC_DQ_ELEM(11)
        BBC_DQ_ELEM(12) BBC_DQ_ELEM(13) BBC_DQ_ELEM(14) BBC_DQ_ELEM(15)
#undef BBC_DQ_ELEM

        const int64_t m0 = H * 16;
        if (VEC && m0 + 16 <= n) {
            uint32_t wv[16];
            pack8<DT>(y, wv);
            pack8<DT>(y + 8, wv + (DT == F32 ? 8 : 4));
            char* dst = reinterpret_cast<char*>(out) + m0 * dtype_size(DT);
            stg_v8(dst, wv);
            if constexpr (DT == F32) stg_v8(dst + 32, wv + 8);
        } else {
#pragma unroll
            for (int e = 0; e < 16; e++)
                if (m0 + e < n) store_from_f32<DT>(out, m0 + e, y[e]);
        }
        cur = nxt;
    }
}

template <int K, int DT, typename AT>
cudaError_t launch_t(const uint32_t* packed, const AT* absmax, const float* codebook, int64_t n,
                     void* out, bool vec, cudaStream_t s) {
    const int64_t nh = ((n + 31) >> 5) * 2;
    // Whole blocks per thread or half blocks (measured, c5 = 268 M bf16 outputs / c2 = 16.8 M):
    // half blocks write 32 contiguous bytes per lane and were faster on long streams (c5, K = 2..4:
    // +1 to +7 points) and for every fp32 output (c2: 20 % faster at K = 2..4, 22 % at K = 5, where
    // a whole block's 128 output bytes per lane spread one store instruction over 4 KB), whole
    // blocks for 16-bit outputs on short streams (c2: 6-20 % faster), at K = 5 (five words
    // re-read by both lanes of a block) and for the E4M4 absmax at K = 3.
    const bool whole = DT != F32 && (K == 5 || (sizeof(AT) == 1 && K == 3) || n < (int64_t(1) << 26));
    auto k = !vec ? kbit_dequant_kernel<K, DT, false, false, AT>
                  : whole ? kbit_dequant_kernel<K, DT, true, true, AT> : kbit_dequant_kernel<K, DT, true, false, AT>;
    const int grid = persistent_grid(k, kThreads, 0, nh, kThreads);
    return launch_pdl(k, grid, kThreads, 0, s, packed, absmax, codebook, n, out);
}

template <int K, typename AT>
cudaError_t launch_k(const uint32_t* packed, const AT* absmax, const float* codebook, int64_t n,
                     int dt, void* out, bool vec, cudaStream_t s) {
    switch (dt) {
        case F16: return launch_t<K, F16>(packed, absmax, codebook, n, out, vec, s);
        case BF16: return launch_t<K, BF16>(packed, absmax, codebook, n, out, vec, s);
        default: return launch_t<K, F32>(packed, absmax, codebook, n, out, vec, s);
    }
}

template <typename AT>
cudaError_t launch_any(const uint32_t* packed, const AT* absmax, const float* codebook, int K, int64_t n,
                       int out_dtype, void* out, bool vec, cudaStream_t s) {
    switch (K) {
        case 2: return launch_k<2>(packed, absmax, codebook, n, out_dtype, out, vec, s);
        case 3: return launch_k<3>(packed, absmax, codebook, n, out_dtype, out, vec, s);
        case 4: return launch_k<4>(packed, absmax, codebook, n, out_dtype, out, vec, s);
        default: return launch_k<5>(packed, absmax, codebook, n, out_dtype, out, vec, s);
    }
}

}  // namespace

BBC_GUARD_ACCESSOR(guard_status_kbit_dequant)

cudaError_t launch_kbit_dequantize(const uint32_t* packed, const float* absmax,
                                   const float* codebook, int K, int64_t n, int out_dtype,
                                   void* out, bool vec, cudaStream_t s) {
    return launch_any(packed, absmax, codebook, K, n, out_dtype, out, vec, s);
}

cudaError_t launch_kbit_dequantize_e4m4(const uint32_t* packed, const uint8_t* absmax,
                                        const float* codebook, int K, int64_t n, int out_dtype,
                                        void* out, bool vec, cudaStream_t s) {
    return launch_any(packed, absmax, codebook, K, n, out_dtype, out, vec, s);
}

}  // namespace bbc
