// k-bit blockwise dequantization (K = 2..5, blocksize 32).
//
// Operation (bitsandbytes k-bit patch series, dequantize_kbit_ref and
// kDequantizeBlockwise_kbit): out[m] = T(codebook[idx_m] * absmax[m / 32]),
// where idx_m is gathered from the K bit-plane words of block m / 32.
//
// B200 layout: a thread owns one quarter block (8 consecutive elements), so
// the four threads of a block sit in adjacent lanes and a warp covers 8 blocks
// (256 elements): the output is written with one 16-byte store per thread per
// 16-bit element type (two for fp32), fully coalesced. Each thread reads the K
// words of its block (the 4 lanes of a block hit the same addresses), keeps
// byte `part` of each, and decodes its 8 indices with one multiply-high bit
// gather per element. The codebook lives in shared memory: 32 consecutive
// floats occupy the 32 banks once, so the per-element lookup never conflicts.
// The grid is persistent (SMs x resident CTAs) with a grid-stride loop.
#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kThreads = 256;

// Byte offset (idx * 4) of element e of a quarter block from the gathered planes.
// B holds byte `part` of plane word j in its byte j (j < 4); B3 = B << 3.
// For e >= 3 the bits j*8+e are moved to bits 34+j of the 64-bit product
// (multiplier sum_j 2^(34-7j-e)); every cross term lands outside bits 34..37,
// on distinct positions, so no carry reaches the field. For e < 3 the same
// gather runs on B3 with e+3.
template <int E>
__device__ __forceinline__ uint32_t plane_offset4(uint32_t B, uint32_t B3) {
    constexpr int e = E < 3 ? E + 3 : E;
    constexpr uint32_t mask = 0x01010101u << e;
    constexpr uint32_t mult = (1u << (34 - e)) | (1u << (27 - e)) | (1u << (20 - e)) | (1u << (13 - e));
    const uint32_t src = E < 3 ? B3 : B;
    return __umulhi(src & mask, mult) & 0x3Cu;
}

template <int K, int DT, bool VEC>
__global__ void __launch_bounds__(kThreads)
kbit_dequant_kernel(const uint32_t* __restrict__ packed, const float* __restrict__ absmax,
                    const float* __restrict__ codebook, int64_t n, void* __restrict__ out) {
    __shared__ float cb[32];
    if (threadIdx.x < 32) cb[threadIdx.x] = threadIdx.x < (1u << K) ? codebook[threadIdx.x] : 0.0f;
    __syncthreads();
    const char* cbb = reinterpret_cast<const char*>(cb);

    const int64_t nq = ((n + 31) >> 5) * 4;                       // quarter blocks
    const uint32_t part = threadIdx.x & 3;
    const uint32_t sel01 = part | ((4 + part) << 4);              // byte `part` of a, then of b
    const int64_t stride = (int64_t)gridDim.x * kThreads;

    for (int64_t Q = (int64_t)blockIdx.x * kThreads + threadIdx.x; Q < nq; Q += stride) {
        const int64_t b = Q >> 2;
        const float am = __ldg(absmax + b);
        const uint32_t* wp = packed + b * K;
        uint32_t w[K];
#pragma unroll
        for (int j = 0; j < K; j++) w[j] = ldg_u32(wp + j);

        uint32_t B;
        if constexpr (K == 2) {
            B = prmt(w[0], w[1], sel01) & 0xFFFFu;
        } else if constexpr (K == 3) {
            B = prmt(prmt(w[0], w[1], sel01), prmt(w[2], 0u, part | 0x4440u), 0x5410u);
        } else {
            B = prmt(prmt(w[0], w[1], sel01), prmt(w[2], w[3], sel01), 0x5410u);
        }
        const uint32_t B3 = B << 3;
        uint32_t hi4 = 0;
        if constexpr (K == 5) hi4 = w[4] >> (8 * part);           // plane 4: bit e is element e

        float y[8];
#define BBC_DQ_ELEM(E)                                                              \
        {                                                                           \
            uint32_t off = plane_offset4<E>(B, B3);                                 \
            if constexpr (K == 5)                                                   \
                off |= (E <= 6 ? (hi4 << (6 - E)) : (hi4 >> 1)) & 0x40u;           \
            y[E] = __fmul_rn(*reinterpret_cast<const float*>(cbb + off), am);       \
        }
        BBC_DQ_ELEM(0) BBC_DQ_ELEM(1) BBC_DQ_ELEM(2) BBC_DQ_ELEM(3)
        BBC_DQ_ELEM(4) BBC_DQ_ELEM(5) BBC_DQ_ELEM(6) BBC_DQ_ELEM(7)
#undef BBC_DQ_ELEM

        const int64_t m0 = Q * 8;
        if (VEC && m0 + 8 <= n) {
            uint32_t wv[8];
            pack8<DT>(y, wv);
            char* dst = reinterpret_cast<char*>(out) + m0 * dtype_size(DT);
            if constexpr (DT == F32) {
                stg_v4(dst, wv[0], wv[1], wv[2], wv[3]);
                stg_v4(dst + 16, wv[4], wv[5], wv[6], wv[7]);
            } else {
                stg_v4(dst, wv[0], wv[1], wv[2], wv[3]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; e++)
                if (m0 + e < n) store_from_f32<DT>(out, m0 + e, y[e]);
        }
    }
}

template <int K, int DT>
cudaError_t launch_t(const uint32_t* packed, const float* absmax, const float* codebook, int64_t n,
                     void* out, bool vec, cudaStream_t s) {
    const int64_t nq = ((n + 31) >> 5) * 4;
    if (vec) {
        auto k = kbit_dequant_kernel<K, DT, true>;
        int grid = persistent_grid(k, kThreads, 0, nq, kThreads);
        k<<<grid, kThreads, 0, s>>>(packed, absmax, codebook, n, out);
    } else {
        auto k = kbit_dequant_kernel<K, DT, false>;
        int grid = persistent_grid(k, kThreads, 0, nq, kThreads);
        k<<<grid, kThreads, 0, s>>>(packed, absmax, codebook, n, out);
    }
    return cudaGetLastError();
}

template <int K>
cudaError_t launch_k(const uint32_t* packed, const float* absmax, const float* codebook, int64_t n,
                     int dt, void* out, bool vec, cudaStream_t s) {
    switch (dt) {
        case F16: return launch_t<K, F16>(packed, absmax, codebook, n, out, vec, s);
        case BF16: return launch_t<K, BF16>(packed, absmax, codebook, n, out, vec, s);
        default: return launch_t<K, F32>(packed, absmax, codebook, n, out, vec, s);
    }
}

}  // namespace

cudaError_t launch_kbit_dequantize(const uint32_t* packed, const float* absmax,
                                   const float* codebook, int K, int64_t n, int out_dtype,
                                   void* out, bool vec, cudaStream_t s) {
    switch (K) {
        case 2: return launch_k<2>(packed, absmax, codebook, n, out_dtype, out, vec, s);
        case 3: return launch_k<3>(packed, absmax, codebook, n, out_dtype, out, vec, s);
        case 4: return launch_k<4>(packed, absmax, codebook, n, out_dtype, out, vec, s);
        default: return launch_k<5>(packed, absmax, codebook, n, out_dtype, out, vec, s);
    }
}

}  // namespace bbc
