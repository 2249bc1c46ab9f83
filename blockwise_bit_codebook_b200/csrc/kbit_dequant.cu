// k-bit blockwise dequantization (K = 2..5, blocksize 32).
//
// Operation (bitsandbytes k-bit patch series, dequantize_kbit_ref and
// kDequantizeBlockwise_kbit): out[m] = T(codebook[idx_m] * absmax[m / 32]),
// where idx_m is gathered from the K bit-plane words of block m / 32.
//
// B200 layout: a thread owns half a block (16 consecutive elements), so the two
// threads of a block sit in adjacent lanes and a warp covers 16 blocks (512
// elements). Each thread reads the block's absmax and K words (the two lanes
// of a block hit the same addresses), keeps bytes 2h and 2h+1 of every word
// (one byte permute per word pair), decodes each 4-bit index with one
// multiply-high bit gather and writes its 16 outputs with one 32-byte store
// (two for fp32). The loads of the next half block are issued before the
// current one is decoded, so each thread keeps two round trips in flight. The
// codebook lives in shared memory: 32 consecutive floats occupy the 32 banks
// once, so the per-element lookup never conflicts. Persistent grid-stride loop.
#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kThreads = 256;

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

template <int K>
struct BlockIn {
    float am;
    uint32_t w[K];
};

template <int K, typename AT>
__device__ __forceinline__ BlockIn<K> load_block(const uint32_t* packed, const AT* absmax,
                                                 int64_t b, bool active) {
    BlockIn<K> r;
    if (active) {
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

template <int K, int DT, bool VEC, typename AT>
__global__ void __launch_bounds__(kThreads)
kbit_dequant_kernel(const uint32_t* __restrict__ packed, const AT* __restrict__ absmax,
                    const float* __restrict__ codebook, int64_t n, void* __restrict__ out) {
    __shared__ float cb[32];
    if (threadIdx.x < 32) cb[threadIdx.x] = threadIdx.x < (1u << K) ? codebook[threadIdx.x] : 0.0f;
    __syncthreads();
    const char* cbb = reinterpret_cast<const char*>(cb);

    const int64_t nh = ((n + 31) >> 5) * 2;                       // half blocks
    const uint32_t h = threadIdx.x & 1;
    // bytes 2h and 2h+1 of two words a, b -> [a.2h, b.2h, a.2h+1, b.2h+1]
    const uint32_t sel = (2 * h) | ((4 + 2 * h) << 4) | ((2 * h + 1) << 8) | ((5 + 2 * h) << 12);
    const int64_t stride = (int64_t)gridDim.x * kThreads;

    int64_t H = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    BlockIn<K> cur = load_block<K, AT>(packed, absmax, H >> 1, H < nh);
    for (; H < nh; H += stride) {
        const int64_t Hn = H + stride;
        const BlockIn<K> nxt = load_block<K, AT>(packed, absmax, Hn >> 1, Hn < nh);

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
    auto k = vec ? kbit_dequant_kernel<K, DT, true, AT> : kbit_dequant_kernel<K, DT, false, AT>;
    const int grid = persistent_grid(k, kThreads, 0, nh, kThreads);
    k<<<grid, kThreads, 0, s>>>(packed, absmax, codebook, n, out);
    return cudaGetLastError();
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
