// Host-side launchers of the library's kernels (called by abi.cpp after validation).
#pragma once
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

namespace bbc {

// Launch with programmatic stream serialisation allowed: the kernel's CTAs may be scheduled as the
// previous kernel of the stream finishes (once all of that kernel's CTAs have exited, before its
// completion is signalled), so the launch latency overlaps its tail; the kernel's
// griddepcontrol.wait (pdl_wait in common.cuh), executed before any global access, holds it until
// that kernel has completed and its writes are visible, so stream order is kept.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t dyn_smem,
                              cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = dyn_smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Sets a function attribute of `kernel` on the current device once per device (function
// attributes are per device): `done` holds one bit per device index below 64 (others set it on
// every call). Concurrent first calls may both set it; the value is the same.
template <typename Kernel>
inline cudaError_t set_attr_once(Kernel kernel, std::atomic<uint64_t>& done, cudaFuncAttribute attr, int value) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load() & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, attr, value);
    if (e == cudaSuccess && bit) done.fetch_or(bit);
    return e;
}

// Persistent grid: enough CTAs to fill every SM at the kernel's occupancy, never more than
// the work needs. The occupancy query runs once per (kernel, device, block, smem) and is
// cached (grid.cpp); if it fails both return 0 (an empty grid, whose launch then fails).
int resident_ctas(const void* kernel, int block, size_t dyn_smem);
int sm_count();

template <typename Kernel>
inline int persistent_grid(Kernel kernel, int block, size_t dyn_smem, int64_t work_items,
                           int items_per_cta) {
    const int64_t cap = resident_ctas(reinterpret_cast<const void*>(kernel), block, dyn_smem);
    if (cap < 1) return 0;
    int64_t need = (work_items + items_per_cta - 1) / items_per_cta;
    if (need < 1) need = 1;
    return (int)(need < cap ? need : cap);
}

cudaError_t launch_kbit_quantize(const void* A, int dtype, int64_t n, int K, const float* codebook,
                                 float* absmax, uint32_t* packed, bool vec, cudaStream_t s);

cudaError_t launch_kbit_dequantize(const uint32_t* packed, const float* absmax,
                                   const float* codebook, int K, int64_t n, int out_dtype,
                                   void* out, bool vec, cudaStream_t s);

// 4-bit codes (two per byte, element 2j in the high nibble) and fp32 absmax per outer block of
// 2^log2_bs elements (32 .. 4096).
cudaError_t launch_quantize_4bit(const void* A, int dtype, int64_t n, int log2_bs, const float* code4,
                                 float* absmax, uint8_t* codes, bool vec, cudaStream_t s);

// The nested 4-bit state of A: codes, General8 codes of the centred outer absmax, inner absmax
// per 256 outer blocks and the offset (device scalar). `workspace` holds
// nested_quant_workspace_bytes(n, log2_bs) bytes (the fp32 outer absmax and binary64 partials).
size_t nested_quant_workspace_bytes(int64_t n, int log2_bs);
cudaError_t launch_quantize_4bit_nested(const void* A, int dtype, int64_t n, int log2_bs, const float* code4,
                                        const float* code2, uint8_t* codes, uint8_t* absmax_q, float* absmax2,
                                        float* offset, void* workspace, bool vec, cudaStream_t s);

// Y[M, N] = X[M, K] @ W^T with W the nested 4-bit weight decoded in registers (M <= 32,
// N % 16 == 0, K % 64 == 0; X 16-byte and codes 8-byte aligned; dtype F16 or BF16).
cudaError_t launch_linear_4bit_nested(const void* X, int dtype, int M, int64_t N, int64_t K,
                                      const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                                      const float* absmax2, float offset, const float* code4, int log2_bs,
                                      void* Y, cudaStream_t s);

cudaError_t launch_linear_kbit(const void* X, int dtype, int M, int64_t N, int64_t K, const uint32_t* packed,
                               const float* absmax, const float* codebook, int KB, void* Y, cudaStream_t s);

// The same two layers for M > 32 on the tensor cores (tcgen05; N % 128 == 0, K % 64 == 0, X 16-byte
// aligned): linear_tc.cu.
cudaError_t launch_linear_4bit_nested_tc(const void* X, int dtype, int M, int64_t N, int64_t K, const uint8_t* codes,
                                         const uint8_t* absmax_q, const float* code2, const float* absmax2,
                                         float offset, const float* code4, int log2_bs, void* Y, cudaStream_t s);
cudaError_t launch_linear_kbit_tc(const void* X, int dtype, int M, int64_t N, int64_t K, const uint32_t* packed,
                                  const float* absmax, const float* codebook, int KB, void* Y, cudaStream_t s);

// Bounded waits (mbarrier waits of the tensor-core kernels) that gave up on the current device
// since the last call; reads and resets the device's count (synchronous).
cudaError_t wait_timeouts(unsigned int* count);

// The same two operations with the per-block absmax stored as one E4M4 byte.
cudaError_t launch_kbit_quantize_e4m4(const void* A, int dtype, int64_t n, int K, const float* codebook,
                                      uint8_t* absmax, uint32_t* packed, bool vec, cudaStream_t s);

cudaError_t launch_kbit_dequantize_e4m4(const uint32_t* packed, const uint8_t* absmax,
                                        const float* codebook, int K, int64_t n, int out_dtype,
                                        void* out, bool vec, cudaStream_t s);

cudaError_t launch_nested_dequantize(const uint8_t* codes, const uint8_t* absmax_q,
                                     const float* code2, const float* absmax2, float offset,
                                     const float* code4, int64_t n, int log2_bs, int out_dtype,
                                     void* out, bool vec, cudaStream_t s);

cudaError_t launch_dequantize_4bit(const uint8_t* codes, const float* absmax, const float* code4,
                                   int64_t n, int log2_bs, int out_dtype, void* out, bool vec,
                                   cudaStream_t s);

cudaError_t launch_nested_dequantize_chain(const uint8_t* codes, const uint8_t* absmax_q,
                                           const float* code2, const float* absmax2, float offset,
                                           const float* code4, int64_t n, int log2_bs, int out_dtype,
                                           void* out, float* scale, bool vec, cudaStream_t s);

// The chain with its scale tensor in the library's static scratch (no allocation).
cudaError_t launch_nested_dequantize_chain_noalloc(const uint8_t* codes, const uint8_t* absmax_q,
                                                   const float* code2, const float* absmax2, float offset,
                                                   const float* code4, int64_t n, int log2_bs,
                                                   int out_dtype, void* out, bool vec, cudaStream_t s);

// Debug builds: each translation unit's guard status word (0 in a release build), read and
// optionally cleared on the current device; abi.cpp ors them for bbc_debug_status.
cudaError_t guard_status_kbit_quant(unsigned int* v, bool reset);
cudaError_t guard_status_kbit_dequant(unsigned int* v, bool reset);
cudaError_t guard_status_nested_dequant(unsigned int* v, bool reset);
cudaError_t guard_status_nested_quant(unsigned int* v, bool reset);
cudaError_t guard_status_linear(unsigned int* v, bool reset);
cudaError_t guard_status_linear_tc(unsigned int* v, bool reset);

}  // namespace bbc
