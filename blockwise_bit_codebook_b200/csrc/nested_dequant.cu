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
// load; 32 per thread measured slower on B200 because of the lower residency);
// outer blocks are >= 32 elements and aligned, so the 16 share one scale. A
// warp covers 512 outputs with coalesced loads and 32-byte stores, and the
// codes, General8 code and inner absmax of the next group are loaded before
// the current group is decoded. Both code tables sit in shared
// memory; the 16-entry value table lives in 16 distinct banks, so the
// per-element lookup never conflicts. Persistent grid-stride loop.
#include <mutex>

#include "bbc.h"
#include "common.cuh"
#include "launch.h"

namespace bbc {

namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 16;                        // outputs per thread (16 or 32 supported)
static_assert(kPerThread == 16 || kPerThread == 32, "16 or 32 outputs per thread");
constexpr int kCodeBytes = kPerThread / 2;

// Byte offset (code * 4) of element 2i (high nibble of byte i) and 2i+1 (low nibble)
// of the little-endian word W holding bytes 4k..4k+3.
template <int I>
__device__ __forceinline__ uint32_t hi_off(uint32_t W) { return (W >> (8 * I + 2)) & 0x3Cu; }
template <int I>
__device__ __forceinline__ uint32_t lo_off(uint32_t W) {
    if constexpr (I == 0) return (W << 2) & 0x3Cu;
    else return (W >> (8 * I - 2)) & 0x3Cu;
}

struct GroupIn {
    uint4 c;          // code bytes (8 or 16) of the group
    uint32_t q;       // General8 code of the outer block
    float a2;         // inner absmax
};

// NESTED: the group's scale inputs are a General8 code (absmax_q) and an inner absmax
// (absmax2, one per 256 outer blocks). Otherwise `absmax2` is a plain fp32 absmax per outer
// block (the last launch of the three-launch chain, or a non-nested 4-bit state).
template <bool VEC, bool NESTED>
__device__ __forceinline__ GroupIn load_group(const uint8_t* codes, const uint8_t* absmax_q,
                                              const float* absmax2, int64_t n, int64_t u,
                                              int log2_bs, bool active) {
    GroupIn g;
    g.c = make_uint4(0u, 0u, 0u, 0u);
    g.q = 0u;
    g.a2 = 0.0f;
    if (!active) return g;
    const int64_t m0 = u * kPerThread;
    if (VEC && m0 + kPerThread <= n) {
        if constexpr (kCodeBytes == 16) {
            g.c = ldg_stream_v4(codes + u * 16);
        } else {
            const uint2 v = ldg_stream_v2(codes + u * 8);
            g.c = make_uint4(v.x, v.y, 0u, 0u);
        }
    } else {
        const int64_t nbytes = (n + 1) >> 1;
        uint32_t wb[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < kCodeBytes; i++) {
            const int64_t bi = u * kCodeBytes + i;
            const uint32_t byte = bi < nbytes ? (uint32_t)codes[bi] : 0u;
            wb[i >> 2] |= byte << (8 * (i & 3));
        }
        g.c = make_uint4(wb[0], wb[1], wb[2], wb[3]);
    }
    const int64_t b = m0 >> log2_bs;
    if (!BBC_GUARD(m0 < n && b < ((n + (int64_t(1) << log2_bs) - 1) >> log2_bs), kGuardNestedIn)) return g;
    if constexpr (NESTED) {
        g.q = __ldg(absmax_q + b);
        g.a2 = __ldg(absmax2 + (b >> 8));
    } else {
        g.a2 = __ldg(absmax2 + b);
    }
    return g;
}

template <int DT, bool VEC, bool NESTED>
__global__ void __launch_bounds__(kThreads)
nested_dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ absmax_q,
                      const float* __restrict__ code2, const float* __restrict__ absmax2,
                      float offset, const float* __restrict__ code4, int64_t n, int log2_bs,
                      void* __restrict__ out) {
    __shared__ float c2[256];
    __shared__ float c4[16];
    pdl_wait();               // writes of the previous kernel in the stream are visible from here
    const float c2v = NESTED ? code2[threadIdx.x] : 0.0f;
    const float c4v = threadIdx.x < 16 ? code4[threadIdx.x] : 0.0f;
    const char* c4b = reinterpret_cast<const char*>(c4);

    const int64_t nu = (n + kPerThread - 1) / kPerThread;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    GroupIn cur = load_group<VEC, NESTED>(codes, absmax_q, absmax2, n, u, log2_bs, u < nu);
    // the tables are published after the first group's loads are issued
    if (NESTED) c2[threadIdx.x] = c2v;
    if (threadIdx.x < 16) c4[threadIdx.x] = c4v;
    __syncthreads();
    for (; u < nu; u += stride) {
        const int64_t un = u + stride;
        const GroupIn nxt = load_group<VEC, NESTED>(codes, absmax_q, absmax2, n, un, log2_bs, un < nu);

        // outer scale: General8 code times inner absmax, then plus offset, each rounded
        const float s = NESTED ? __fadd_rn(__fmul_rn(c2[cur.q], cur.a2), offset) : cur.a2;
        const uint32_t W[4] = {cur.c.x, cur.c.y, cur.c.z, cur.c.w};
        const int64_t m0 = u * kPerThread;
#pragma unroll
        for (int half = 0; half < kPerThread / 16; half++) {
            float y[16];
#pragma unroll
            for (int k = 0; k < 2; k++) {
                const uint32_t w = W[2 * half + k];
#define BBC_ND_BYTE(I)                                                                       \
                y[8 * k + 2 * (I)] = __fmul_rn(*reinterpret_cast<const float*>(c4b + hi_off<I>(w)), s); \
                y[8 * k + 2 * (I) + 1] = __fmul_rn(*reinterpret_cast<const float*>(c4b + lo_off<I>(w)), s);
                BBC_ND_BYTE(0) BBC_ND_BYTE(1) BBC_ND_BYTE(2) BBC_ND_BYTE(3)
#undef BBC_ND_BYTE
            }
            const int64_t mh = m0 + 16 * half;
            if (VEC && m0 + kPerThread <= n) {
                uint32_t wv[16];
                pack8<DT>(y, wv);
                pack8<DT>(y + 8, wv + (DT == F32 ? 8 : 4));
                char* dst = reinterpret_cast<char*>(out) + mh * dtype_size(DT);
                stg_v8(dst, wv);
                if constexpr (DT == F32) stg_v8(dst + 32, wv + 8);
            } else {
#pragma unroll
                for (int e = 0; e < 16; e++)
                    if (mh + e < n) store_from_f32<DT>(out, mh + e, y[e]);
            }
        }
        cur = nxt;
    }
}

template <int DT, bool NESTED>
cudaError_t launch_t(const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                     const float* absmax2, float offset, const float* code4, int64_t n,
                     int log2_bs, void* out, bool vec, cudaStream_t s) {
    const int64_t nu = (n + kPerThread - 1) / kPerThread;
    auto k = vec ? nested_dequant_kernel<DT, true, NESTED> : nested_dequant_kernel<DT, false, NESTED>;
    const int grid = persistent_grid(k, kThreads, 0, nu, kThreads);
    return launch_pdl(k, grid, kThreads, 0, s, codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out);
}

template <bool NESTED>
cudaError_t launch_dt(const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                      const float* absmax2, float offset, const float* code4, int64_t n, int log2_bs,
                      int out_dtype, void* out, bool vec, cudaStream_t s) {
    switch (out_dtype) {
        case F16: return launch_t<F16, NESTED>(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out, vec, s);
        case BF16: return launch_t<BF16, NESTED>(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out, vec, s);
        default: return launch_t<F32, NESTED>(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out, vec, s);
    }
}

// ---- the legacy three-launch chain: General8 scale, offset add, then plain 4-bit decode ----

// scale[b] = fl(code2[absmax_q[b]] * absmax2[b / 256])
__global__ void __launch_bounds__(kThreads)
general8_scale_kernel(const uint8_t* __restrict__ absmax_q, const float* __restrict__ code2,
                      const float* __restrict__ absmax2, int64_t nbo, float* __restrict__ scale) {
    __shared__ float c2[256];
    c2[threadIdx.x] = code2[threadIdx.x];
    __syncthreads();
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nbo; b += (int64_t)gridDim.x * kThreads)
        scale[b] = __fmul_rn(c2[__ldg(absmax_q + b)], __ldg(absmax2 + (b >> 8)));
}

// scale[b] = fl(scale[b] + offset)
__global__ void __launch_bounds__(kThreads)
add_offset_kernel(float* __restrict__ scale, int64_t nbo, float offset) {
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nbo; b += (int64_t)gridDim.x * kThreads)
        scale[b] = __fadd_rn(scale[b], offset);
}

// Fixed scratch for the scale tensor of the allocation-free chain: one copy per device, kept
// for the life of the process. Host code must not use this name as a device address; it
// asks the runtime for the address on each device (scratch_address below).
static __device__ __align__(256) float g_chain_scale_scratch[BBC_NOALLOC_SCRATCH_FLOATS];

}  // namespace

BBC_GUARD_ACCESSOR(guard_status_nested_dequant)

// Device address of this device's copy of the scratch array, looked up with that device current;
// nullptr if the lookup failed (the error is returned in *err). A call made while `s` is not being
// captured looks the address up again (cheap once the module is loaded), so that after the
// device's context has been torn down and the module reloaded (cudaDeviceReset) the new address
// is used; a call during capture takes the one the last such call found.
static float* scratch_address(cudaStream_t s, cudaError_t* err) {
    static std::mutex mu;
    static float* addr[64] = {};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    *err = cudaStreamIsCapturing(s, &cap);
    if (*err != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || cap == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_chain_scale_scratch);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = static_cast<float*>(p);
    }
    return addr[dev];
}

cudaError_t launch_nested_dequantize_chain_noalloc(const uint8_t* codes, const uint8_t* absmax_q,
                                                   const float* code2, const float* absmax2, float offset,
                                                   const float* code4, int64_t n, int log2_bs,
                                                   int out_dtype, void* out, bool vec, cudaStream_t s) {
    cudaError_t err = cudaSuccess;
    float* scale = scratch_address(s, &err);
    if (!scale) return err;
    return launch_nested_dequantize_chain(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs,
                                          out_dtype, out, scale, vec, s);
}

cudaError_t launch_nested_dequantize(const uint8_t* codes, const uint8_t* absmax_q,
                                     const float* code2, const float* absmax2, float offset,
                                     const float* code4, int64_t n, int log2_bs, int out_dtype,
                                     void* out, bool vec, cudaStream_t s) {
    return launch_dt<true>(codes, absmax_q, code2, absmax2, offset, code4, n, log2_bs, out_dtype, out, vec, s);
}

cudaError_t launch_dequantize_4bit(const uint8_t* codes, const float* absmax, const float* code4,
                                   int64_t n, int log2_bs, int out_dtype, void* out, bool vec,
                                   cudaStream_t s) {
    return launch_dt<false>(codes, nullptr, nullptr, absmax, 0.0f, code4, n, log2_bs, out_dtype, out, vec, s);
}

cudaError_t launch_nested_dequantize_chain(const uint8_t* codes, const uint8_t* absmax_q,
                                           const float* code2, const float* absmax2, float offset,
                                           const float* code4, int64_t n, int log2_bs, int out_dtype,
                                           void* out, float* scale, bool vec, cudaStream_t s) {
    const int64_t nbo = ((n - 1) >> log2_bs) + 1;
    const int grid_s = persistent_grid(general8_scale_kernel, kThreads, 0, nbo, kThreads);
    general8_scale_kernel<<<grid_s, kThreads, 0, s>>>(absmax_q, code2, absmax2, nbo, scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int grid_o = persistent_grid(add_offset_kernel, kThreads, 0, nbo, kThreads);
    add_offset_kernel<<<grid_o, kThreads, 0, s>>>(scale, nbo, offset);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_dequantize_4bit(codes, scale, code4, n, log2_bs, out_dtype, out, vec, s);
}

}  // namespace bbc
