// Nested NF4/FP4 dequantization with the outer scale rebuilt in the decode.
//
// Operation (pull request "Fuse nested 4-bit scale reconstruction on SM103",
// Summary and Implementation): for outer block b,
//     scale_b = fl(fl(code2[absmax_q[b]] * absmax2[b / 256]) + offset)
// (a separately rounded fp32 multiply then add, never a fused multiply-add),
// and each 4-bit code v of the block decodes to T(fl(code4[v] * scale_b)).
// No scale tensor is written: the scale is formed in registers next to the
// values it multiplies, in the one kernel that reads the codes.
//
// B200 layout: a thread owns 16 consecutive outputs (8 code bytes, one 8-byte
// load); outer blocks are >= 32 elements, so the 16 share one scale. A warp
// covers 512 outputs with coalesced 8-byte loads and 16-byte stores. Both code
// tables sit in shared memory; the 16-entry value table lives in 16 distinct
// banks, so the per-element lookup never conflicts. Persistent grid-stride loop.
#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 16;

// Byte offset (code * 4) of element 2i (high nibble of byte i) and 2i+1 (low nibble)
// of the little-endian word W holding bytes 4k..4k+3.
template <int I>
__device__ __forceinline__ uint32_t hi_off(uint32_t W) { return (W >> (8 * I + 2)) & 0x3Cu; }
template <int I>
__device__ __forceinline__ uint32_t lo_off(uint32_t W) {
    if constexpr (I == 0) return (W << 2) & 0x3Cu;
    else return (W >> (8 * I - 2)) & 0x3Cu;
}

template <int DT, bool VEC>
__global__ void __launch_bounds__(kThreads)
nested_dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ absmax_q,
                      const float* __restrict__ code2, const float* __restrict__ absmax2,
                      float offset, const float* __restrict__ code4, int64_t n, int log2_bs,
                      void* __restrict__ out) {
    __shared__ float c2[256];
    __shared__ float c4[16];
    c2[threadIdx.x] = code2[threadIdx.x];
    if (threadIdx.x < 16) c4[threadIdx.x] = code4[threadIdx.x];
    __syncthreads();
    const char* c4b = reinterpret_cast<const char*>(c4);

    const int64_t nbytes = (n + 1) >> 1;
    const int64_t nu = (n + kPerThread - 1) / kPerThread;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < nu; u += stride) {
        const int64_t m0 = u * kPerThread;
        const bool full = m0 + kPerThread <= n;
        uint32_t w0, w1;
        if (VEC && full) {
            const uint2 v = ldg_stream_v2(codes + u * 8);
            w0 = v.x;
            w1 = v.y;
        } else {
            uint32_t wb[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int64_t bi = u * 8 + i;
                const uint32_t byte = bi < nbytes ? (uint32_t)codes[bi] : 0u;
                wb[i >> 2] |= byte << (8 * (i & 3));
            }
            w0 = wb[0];
            w1 = wb[1];
        }

        const int64_t b = m0 >> log2_bs;
        const float s = __fadd_rn(__fmul_rn(c2[__ldg(absmax_q + b)], __ldg(absmax2 + (b >> 8))), offset);

        float y[16];
#define BBC_ND_BYTE(I, W, BASE)                                                           \
        y[BASE + 2 * (I)] = __fmul_rn(*reinterpret_cast<const float*>(c4b + hi_off<I>(W)), s); \
        y[BASE + 2 * (I) + 1] = __fmul_rn(*reinterpret_cast<const float*>(c4b + lo_off<I>(W)), s);
        BBC_ND_BYTE(0, w0, 0) BBC_ND_BYTE(1, w0, 0) BBC_ND_BYTE(2, w0, 0) BBC_ND_BYTE(3, w0, 0)
        BBC_ND_BYTE(0, w1, 8) BBC_ND_BYTE(1, w1, 8) BBC_ND_BYTE(2, w1, 8) BBC_ND_BYTE(3, w1, 8)
#undef BBC_ND_BYTE

        if (VEC && full) {
            uint32_t wv[16];
            pack8<DT>(y, wv);
            pack8<DT>(y + 8, wv + (DT == F32 ? 8 : 4));
            char* dst = reinterpret_cast<char*>(out) + m0 * dtype_size(DT);
            if constexpr (DT == F32) {
#pragma unroll
                for (int i = 0; i < 4; i++) stg_v4(dst + 16 * i, wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
            } else {
                stg_v4(dst, wv[0], wv[1], wv[2], wv[3]);
                stg_v4(dst + 16, wv[4], wv[5], wv[6], wv[7]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < kPerThread; e++)
                if (m0 + e < n) store_from_f32<DT>(out, m0 + e, y[e]);
        }
    }
}

template <int DT>
cudaError_t launch_t(const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                     const float* absmax2, float offset, const float* code4, int64_t n,
                     int log2_bs, void* out, bool vec, cudaStream_t s) {
    const int64_t nu = (n + kPerThread - 1) / kPerThread;
    if (vec) {
        auto k = nested_dequant_kernel<DT, true>;
        int grid = persistent_grid(k, kThreads, 0, nu, kThreads);
        k<<<grid, kThreads, 0, s>>>(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out);
    } else {
        auto k = nested_dequant_kernel<DT, false>;
        int grid = persistent_grid(k, kThreads, 0, nu, kThreads);
        k<<<grid, kThreads, 0, s>>>(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_nested_dequantize(const uint8_t* codes, const uint8_t* absmax_q,
                                     const float* code2, const float* absmax2, float offset,
                                     const float* code4, int64_t n, int log2_bs, int out_dtype,
                                     void* out, bool vec, cudaStream_t s) {
    switch (out_dtype) {
        case F16: return launch_t<F16>(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out, vec, s);
        case BF16: return launch_t<BF16>(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out, vec, s);
        default: return launch_t<F32>(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out, vec, s);
    }
}

}  // namespace bbc
