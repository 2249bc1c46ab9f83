// extern "C" entry points declared in include/bbc.h: host-side validation, then one launch.
#include "bbc.h"

#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <initializer_list>
#include <string>

#include "launch.h"

namespace {

thread_local std::string g_last_error;

int fail(int status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

int ok() {
    g_last_error.clear();
    return BBC_OK;
}

int cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return ok();
    return fail(BBC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_dtype(int dt) { return dt == BBC_F16 || dt == BBC_BF16 || dt == BBC_F32; }

int elem_size(int dt) { return dt == BBC_F32 ? 4 : 2; }

// A buffer of a call: its address, its extent in bytes and its name for messages.
struct Buf {
    const void* p;
    size_t bytes;
    const char* name;
};

bool overlap(const Buf& x, const Buf& y) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(x.p), b = reinterpret_cast<uintptr_t>(y.p);
    return x.bytes && y.bytes && a < b + y.bytes && b < a + x.bytes;
}

// The checks of a call's buffers, after its scalar arguments passed and before anything is
// launched: no output overlaps an input or another output (host arithmetic only), then every
// buffer is memory of the current device (a device allocation on it, or a managed allocation),
// as cudaPointerGetAttributes reports: host memory, pinned or not, memory of another device or an
// address the CUDA runtime does not know is refused with BBC_ERR_INVALID rather than handed to a
// kernel. (The extent of an allocation is not known to the runtime; only its start is checked.)
int check_buffers(const char* fn, std::initializer_list<Buf> in, std::initializer_list<Buf> out) {
    for (auto o = out.begin(); o != out.end(); ++o) {
        for (const Buf& i : in)
            if (overlap(*o, i)) return fail(BBC_ERR_INVALID, "%s: output %s overlaps input %s", fn, o->name, i.name);
        for (auto o2 = o + 1; o2 != out.end(); ++o2)
            if (overlap(*o, *o2))
                return fail(BBC_ERR_INVALID, "%s: outputs %s and %s overlap", fn, o->name, o2->name);
    }
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(BBC_ERR_INVALID, "%s: the buffers cannot be checked as device memory: %s", fn,
                    cudaGetErrorString(e));
    }
    for (const auto* list : {&in, &out})
        for (const Buf& b : *list) {
            cudaPointerAttributes a{};
            e = cudaPointerGetAttributes(&a, b.p);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return fail(BBC_ERR_INVALID, "%s: %s is not memory the CUDA runtime knows: %s", fn, b.name,
                            cudaGetErrorString(e));
            }
            if (a.type == cudaMemoryTypeManaged) continue;
            if (a.type != cudaMemoryTypeDevice)
                return fail(BBC_ERR_INVALID, "%s: %s is host memory; device memory is required", fn, b.name);
            if (a.device != dev)
                return fail(BBC_ERR_INVALID, "%s: %s is memory of device %d, the current device is %d", fn, b.name,
                            a.device, dev);
        }
    return BBC_OK;
}

size_t cdiv(int64_t a, int64_t b) { return (size_t)((a + b - 1) / b); }

// log2 of a 4-bit outer blocksize (a power of two in [32, 4096]), or -1.
int log2_blocksize(int blocksize) {
    for (int l = 5; l <= 12; l++)
        if (blocksize == (1 << l)) return l;
    return -1;
}

}  // namespace

extern "C" {

// Shared validation of the k-bit entry points; `absmax` is fp32 or E4M4 bytes (`am_size`).
static int check_kbit(const char* fn, const void* data, const void* absmax, size_t am_size, const float* codebook,
               const uint32_t* packed, int64_t n, int K, int dtype, int blocksize, const void* typed,
               int typed_dtype) {
    if (!data || !absmax || !codebook || !packed)
        return fail(BBC_ERR_INVALID, "%s: null pointer argument", fn);
    if (n <= 0) return fail(BBC_ERR_INVALID, "%s: n must be >= 1 (got %lld)", fn, (long long)n);
    if (K < 2 || K > 5) return fail(BBC_ERR_INVALID, "%s: K must be 2..5 (got %d)", fn, K);
    if (!valid_dtype(dtype)) return fail(BBC_ERR_INVALID, "%s: bad dtype %d", fn, dtype);
    if (blocksize != 32)
        return fail(BBC_ERR_UNSUPPORTED, "%s: blocksize must be 32 (got %d)", fn, blocksize);
    if (!aligned(typed, elem_size(typed_dtype)) || !aligned(codebook, 4) || !aligned(absmax, am_size) ||
        !aligned(packed, 4))
        return fail(BBC_ERR_INVALID, "%s: pointer not aligned to its element size", fn);
    return BBC_OK;
}

int kbit_quantize(const void* A, int dtype, int64_t n, int K, int blocksize,
                  const float* codebook, float* absmax, uint32_t* packed, void* stream) {
    const int st = check_kbit("kbit_quantize", A, absmax, 4, codebook, packed, n, K, dtype, blocksize, A, dtype);
    if (st != BBC_OK) return st;
    const size_t nb = cdiv(n, 32);
    const int sb = check_buffers("kbit_quantize", {{A, (size_t)n * elem_size(dtype), "A"}, {codebook, 4u << K, "codebook"}},
                                 {{absmax, nb * 4, "absmax"}, {packed, nb * K * 4, "packed"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(A, 32);     // 256-bit loads of 16-element groups
    return cuda_status(bbc::launch_kbit_quantize(A, dtype, n, K, codebook, absmax, packed, vec,
                                                 static_cast<cudaStream_t>(stream)),
                       "kbit_quantize launch");
}

int kbit_dequantize(const uint32_t* packed, const float* absmax, const float* codebook,
                    int K, int blocksize, int64_t n, int out_dtype, void* out, void* stream) {
    const int st = check_kbit("kbit_dequantize", out, absmax, 4, codebook, packed, n, K, out_dtype, blocksize,
                              out, out_dtype);
    if (st != BBC_OK) return st;
    const size_t nb = cdiv(n, 32);
    const int sb = check_buffers("kbit_dequantize", {{packed, nb * K * 4, "packed"}, {absmax, nb * 4, "absmax"},
                                                     {codebook, 4u << K, "codebook"}},
                                 {{out, (size_t)n * elem_size(out_dtype), "out"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(out, 32);     // 32-byte stores of 16-element groups
    return cuda_status(bbc::launch_kbit_dequantize(packed, absmax, codebook, K, n, out_dtype, out, vec,
                                                   static_cast<cudaStream_t>(stream)),
                       "kbit_dequantize launch");
}

int kbit_quantize_e4m4(const void* A, int dtype, int64_t n, int K, int blocksize, const float* codebook,
                       uint8_t* absmax_e4m4, uint32_t* packed, void* stream) {
    const int st = check_kbit("kbit_quantize_e4m4", A, absmax_e4m4, 1, codebook, packed, n, K, dtype, blocksize,
                              A, dtype);
    if (st != BBC_OK) return st;
    const size_t nb = cdiv(n, 32);
    const int sb = check_buffers("kbit_quantize_e4m4", {{A, (size_t)n * elem_size(dtype), "A"}, {codebook, 4u << K, "codebook"}},
                                 {{absmax_e4m4, nb, "absmax_e4m4"}, {packed, nb * K * 4, "packed"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(A, 32);
    return cuda_status(bbc::launch_kbit_quantize_e4m4(A, dtype, n, K, codebook, absmax_e4m4, packed, vec,
                                                      static_cast<cudaStream_t>(stream)),
                       "kbit_quantize_e4m4 launch");
}

int kbit_dequantize_e4m4(const uint32_t* packed, const uint8_t* absmax_e4m4, const float* codebook, int K,
                         int blocksize, int64_t n, int out_dtype, void* out, void* stream) {
    const int st = check_kbit("kbit_dequantize_e4m4", out, absmax_e4m4, 1, codebook, packed, n, K, out_dtype,
                              blocksize, out, out_dtype);
    if (st != BBC_OK) return st;
    const size_t nb = cdiv(n, 32);
    const int sb = check_buffers("kbit_dequantize_e4m4", {{packed, nb * K * 4, "packed"}, {absmax_e4m4, nb, "absmax_e4m4"},
                                                          {codebook, 4u << K, "codebook"}},
                                 {{out, (size_t)n * elem_size(out_dtype), "out"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(out, 32);
    return cuda_status(bbc::launch_kbit_dequantize_e4m4(packed, absmax_e4m4, codebook, K, n, out_dtype, out, vec,
                                                        static_cast<cudaStream_t>(stream)),
                       "kbit_dequantize_e4m4 launch");
}

int dequantize_4bit_nested(const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                           const float* absmax2, float offset, const float* code4,
                           int64_t n, int blocksize, int blocksize2, int out_dtype, void* out,
                           void* stream) {
    if (!codes || !absmax_q || !code2 || !absmax2 || !code4 || !out)
        return fail(BBC_ERR_INVALID, "dequantize_4bit_nested: null pointer argument");
    if (n <= 0)
        return fail(BBC_ERR_INVALID, "dequantize_4bit_nested: n must be >= 1 (got %lld)", (long long)n);
    if (!valid_dtype(out_dtype))
        return fail(BBC_ERR_INVALID, "dequantize_4bit_nested: bad dtype %d", out_dtype);
    const int log2_bs = log2_blocksize(blocksize);
    if (log2_bs < 0)
        return fail(BBC_ERR_INVALID,
                    "dequantize_4bit_nested: blocksize must be a power of two in [32, 4096] (got %d)",
                    blocksize);
    if (blocksize2 != 256)
        return fail(BBC_ERR_UNSUPPORTED, "dequantize_4bit_nested: blocksize2 must be 256 (got %d)",
                    blocksize2);
    if (!aligned(out, elem_size(out_dtype)) || !aligned(code2, 4) || !aligned(absmax2, 4) || !aligned(code4, 4))
        return fail(BBC_ERR_INVALID, "dequantize_4bit_nested: pointer not aligned to its element size");
    const size_t nbo = cdiv(n, blocksize);
    const int sb = check_buffers("dequantize_4bit_nested",
                                 {{codes, cdiv(n, 2), "codes"}, {absmax_q, nbo, "absmax_q"}, {code2, 1024, "code2"},
                                  {absmax2, cdiv((int64_t)nbo, 256) * 4, "absmax2"}, {code4, 64, "code4"}},
                                 {{out, (size_t)n * elem_size(out_dtype), "out"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(out, 32) && aligned(codes, 16);   // 8/16-byte loads, 32-byte stores
    return cuda_status(bbc::launch_nested_dequantize(codes, absmax_q, code2, absmax2, offset, code4, n,
                                                     log2_bs, out_dtype, out, vec,
                                                     static_cast<cudaStream_t>(stream)),
                       "dequantize_4bit_nested launch");
}

int dequantize_4bit(const uint8_t* codes, const float* absmax, const float* code4, int64_t n,
                    int blocksize, int out_dtype, void* out, void* stream) {
    if (!codes || !absmax || !code4 || !out)
        return fail(BBC_ERR_INVALID, "dequantize_4bit: null pointer argument");
    if (n <= 0) return fail(BBC_ERR_INVALID, "dequantize_4bit: n must be >= 1 (got %lld)", (long long)n);
    if (!valid_dtype(out_dtype)) return fail(BBC_ERR_INVALID, "dequantize_4bit: bad dtype %d", out_dtype);
    const int log2_bs = log2_blocksize(blocksize);
    if (log2_bs < 0)
        return fail(BBC_ERR_INVALID, "dequantize_4bit: blocksize must be a power of two in [32, 4096] (got %d)",
                    blocksize);
    if (!aligned(out, elem_size(out_dtype)) || !aligned(absmax, 4) || !aligned(code4, 4))
        return fail(BBC_ERR_INVALID, "dequantize_4bit: pointer not aligned to its element size");
    const int sb = check_buffers("dequantize_4bit",
                                 {{codes, cdiv(n, 2), "codes"}, {absmax, cdiv(n, blocksize) * 4, "absmax"}, {code4, 64, "code4"}},
                                 {{out, (size_t)n * elem_size(out_dtype), "out"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(out, 32) && aligned(codes, 16);
    return cuda_status(bbc::launch_dequantize_4bit(codes, absmax, code4, n, log2_bs, out_dtype, out, vec,
                                                   static_cast<cudaStream_t>(stream)),
                       "dequantize_4bit launch");
}

int quantize_4bit(const void* A, int dtype, int64_t n, int blocksize, const float* code4, float* absmax,
                  uint8_t* codes, void* stream) {
    const char* fn = "quantize_4bit";
    if (!A || !code4 || !absmax || !codes) return fail(BBC_ERR_INVALID, "%s: null pointer argument", fn);
    if (n <= 0) return fail(BBC_ERR_INVALID, "%s: n must be >= 1 (got %lld)", fn, (long long)n);
    if (!valid_dtype(dtype)) return fail(BBC_ERR_INVALID, "%s: bad dtype %d", fn, dtype);
    const int log2_bs = log2_blocksize(blocksize);
    if (log2_bs < 0)
        return fail(BBC_ERR_INVALID, "%s: blocksize must be a power of two in [32, 4096] (got %d)", fn, blocksize);
    if (!aligned(A, elem_size(dtype)) || !aligned(absmax, 4) || !aligned(code4, 4))
        return fail(BBC_ERR_INVALID, "%s: pointer not aligned to its element size", fn);
    const int sb = check_buffers(fn, {{A, (size_t)n * elem_size(dtype), "A"}, {code4, 64, "code4"}},
                                 {{absmax, cdiv(n, blocksize) * 4, "absmax"}, {codes, cdiv(n, 2), "codes"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(A, 32) && aligned(codes, 16);     // 256-bit loads, 8/16-byte code stores
    return cuda_status(bbc::launch_quantize_4bit(A, dtype, n, log2_bs, code4, absmax, codes, vec,
                                                 static_cast<cudaStream_t>(stream)),
                       "quantize_4bit launch");
}

size_t quantize_4bit_nested_workspace_bytes(int64_t n, int blocksize) {
    const int log2_bs = log2_blocksize(blocksize);
    if (n <= 0 || log2_bs < 0) return 0;
    return bbc::nested_quant_workspace_bytes(n, log2_bs);
}

int quantize_4bit_nested(const void* A, int dtype, int64_t n, int blocksize, const float* code4,
                         const float* code2, int blocksize2, uint8_t* codes, uint8_t* absmax_q, float* absmax2,
                         float* offset, void* workspace, size_t workspace_bytes, void* stream) {
    const char* fn = "quantize_4bit_nested";
    if (!A || !code4 || !code2 || !codes || !absmax_q || !absmax2 || !offset || !workspace)
        return fail(BBC_ERR_INVALID, "%s: null pointer argument", fn);
    if (n <= 0) return fail(BBC_ERR_INVALID, "%s: n must be >= 1 (got %lld)", fn, (long long)n);
    if (!valid_dtype(dtype)) return fail(BBC_ERR_INVALID, "%s: bad dtype %d", fn, dtype);
    const int log2_bs = log2_blocksize(blocksize);
    if (log2_bs < 0)
        return fail(BBC_ERR_INVALID, "%s: blocksize must be a power of two in [32, 4096] (got %d)", fn, blocksize);
    if (blocksize2 != 256)
        return fail(BBC_ERR_UNSUPPORTED, "%s: blocksize2 must be 256 (got %d)", fn, blocksize2);
    const size_t need = bbc::nested_quant_workspace_bytes(n, log2_bs);
    if (workspace_bytes < need)
        return fail(BBC_ERR_INVALID, "%s: workspace holds %zu bytes, %zu needed", fn, workspace_bytes, need);
    if (!aligned(A, elem_size(dtype)) || !aligned(code4, 4) || !aligned(code2, 4) || !aligned(absmax2, 4) ||
        !aligned(offset, 4) || !aligned(workspace, 256))
        return fail(BBC_ERR_INVALID, "%s: pointer not aligned (elements; workspace to 256 bytes)", fn);
    const size_t nbo = cdiv(n, blocksize);
    const int sb = check_buffers(fn, {{A, (size_t)n * elem_size(dtype), "A"}, {code4, 64, "code4"}, {code2, 1024, "code2"}},
                                 {{codes, cdiv(n, 2), "codes"}, {absmax_q, nbo, "absmax_q"},
                                  {absmax2, cdiv((int64_t)nbo, 256) * 4, "absmax2"}, {offset, 4, "offset"},
                                  {workspace, need, "workspace"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(A, 32) && aligned(codes, 16);
    return cuda_status(bbc::launch_quantize_4bit_nested(A, dtype, n, log2_bs, code4, code2, codes, absmax_q,
                                                        absmax2, offset, workspace, vec,
                                                        static_cast<cudaStream_t>(stream)),
                       "quantize_4bit_nested launch");
}

int linear_4bit_nested(const void* X, int dtype, int64_t M, int64_t N, int64_t K, const uint8_t* codes,
                       const uint8_t* absmax_q, const float* code2, const float* absmax2, float offset,
                       const float* code4, int blocksize, int blocksize2, void* Y, void* stream) {
    const char* fn = "linear_4bit_nested";
    if (!X || !codes || !absmax_q || !code2 || !absmax2 || !code4 || !Y)
        return fail(BBC_ERR_INVALID, "%s: null pointer argument", fn);
    if (M <= 0 || N <= 0 || K <= 0)
        return fail(BBC_ERR_INVALID, "%s: M, N, K must be >= 1 (got %lld, %lld, %lld)", fn, (long long)M,
                    (long long)N, (long long)K);
    if (dtype != BBC_F16 && dtype != BBC_BF16)
        return fail(BBC_ERR_UNSUPPORTED, "%s: activations must be fp16 or bf16 (got dtype %d)", fn, dtype);
    if (N % 16 != 0 || K % 64 != 0 || (M > 32 && N % 128 != 0) || M > INT32_MAX || K > INT32_MAX)
        return fail(BBC_ERR_UNSUPPORTED,
                    "%s: needs K %% 64 == 0 and N %% 16 == 0 (N %% 128 == 0 when M > 32) (got M=%lld, N=%lld, K=%lld)",
                    fn, (long long)M, (long long)N, (long long)K);
    const int log2_bs = log2_blocksize(blocksize);
    if (log2_bs < 0)
        return fail(BBC_ERR_INVALID, "%s: blocksize must be a power of two in [32, 4096] (got %d)", fn, blocksize);
    if (blocksize2 != 256)
        return fail(BBC_ERR_UNSUPPORTED, "%s: blocksize2 must be 256 (got %d)", fn, blocksize2);
    if (!aligned(X, 16) || !aligned(codes, 16) || !aligned(Y, 2) || !aligned(code2, 4) || !aligned(absmax2, 4) ||
        !aligned(code4, 4))
        return fail(BBC_ERR_INVALID, "%s: X and codes must be 16-byte aligned (others: element size)", fn);
    const int sb = check_buffers(fn, {{X, (size_t)(M * K) * 2, "X"}, {codes, (size_t)(N * K / 2), "codes"},
                                      {absmax_q, cdiv(N * K, blocksize), "absmax_q"}, {code2, 1024, "code2"},
                                      {absmax2, cdiv((int64_t)cdiv(N * K, blocksize), 256) * 4, "absmax2"},
                                      {code4, 64, "code4"}},
                                 {{Y, (size_t)(M * N) * 2, "Y"}});
    if (sb != BBC_OK) return sb;
    return cuda_status(bbc::launch_linear_4bit_nested(X, dtype, (int)M, N, K, codes, absmax_q, code2, absmax2,
                                                      offset, code4, log2_bs, Y, static_cast<cudaStream_t>(stream)),
                       "linear_4bit_nested launch");
}

int linear_kbit(const void* X, int dtype, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                const float* absmax, const float* codebook, int bits, int blocksize, void* Y, void* stream) {
    const char* fn = "linear_kbit";
    if (!X || !packed || !absmax || !codebook || !Y) return fail(BBC_ERR_INVALID, "%s: null pointer argument", fn);
    if (M <= 0 || N <= 0 || K <= 0)
        return fail(BBC_ERR_INVALID, "%s: M, N, K must be >= 1 (got %lld, %lld, %lld)", fn, (long long)M,
                    (long long)N, (long long)K);
    if (bits < 2 || bits > 5) return fail(BBC_ERR_INVALID, "%s: bits must be 2..5 (got %d)", fn, bits);
    if (blocksize != 32) return fail(BBC_ERR_UNSUPPORTED, "%s: blocksize must be 32 (got %d)", fn, blocksize);
    if (dtype != BBC_F16 && dtype != BBC_BF16)
        return fail(BBC_ERR_UNSUPPORTED, "%s: activations must be fp16 or bf16 (got dtype %d)", fn, dtype);
    if (N % 16 != 0 || K % 64 != 0 || (M > 32 && N % 128 != 0) || M > INT32_MAX || K > INT32_MAX)
        return fail(BBC_ERR_UNSUPPORTED,
                    "%s: needs K %% 64 == 0 and N %% 16 == 0 (N %% 128 == 0 when M > 32) (got M=%lld, N=%lld, K=%lld)",
                    fn, (long long)M, (long long)N, (long long)K);
    if (!aligned(X, 16) || !aligned(packed, 16) || !aligned(Y, 2) || !aligned(absmax, 4) || !aligned(codebook, 4))
        return fail(BBC_ERR_INVALID, "%s: X and packed must be 16-byte aligned (others: element size)", fn);
    const int sb = check_buffers(fn, {{X, (size_t)(M * K) * 2, "X"}, {packed, (size_t)(N * K / 32) * bits * 4, "packed"},
                                      {absmax, (size_t)(N * K / 32) * 4, "absmax"}, {codebook, 4u << bits, "codebook"}},
                                 {{Y, (size_t)(M * N) * 2, "Y"}});
    if (sb != BBC_OK) return sb;
    return cuda_status(bbc::launch_linear_kbit(X, dtype, (int)M, N, K, packed, absmax, codebook, bits, Y,
                                               static_cast<cudaStream_t>(stream)),
                       "linear_kbit launch");
}

int dequantize_4bit_nested_chain(const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                                 const float* absmax2, float offset, const float* code4,
                                 int64_t n, int blocksize, int blocksize2, int out_dtype, void* out,
                                 float* scale_workspace, void* stream) {
    if (!codes || !absmax_q || !code2 || !absmax2 || !code4 || !out || !scale_workspace)
        return fail(BBC_ERR_INVALID, "dequantize_4bit_nested_chain: null pointer argument");
    if (n <= 0)
        return fail(BBC_ERR_INVALID, "dequantize_4bit_nested_chain: n must be >= 1 (got %lld)", (long long)n);
    if (!valid_dtype(out_dtype))
        return fail(BBC_ERR_INVALID, "dequantize_4bit_nested_chain: bad dtype %d", out_dtype);
    const int log2_bs = log2_blocksize(blocksize);
    if (log2_bs < 0)
        return fail(BBC_ERR_INVALID,
                    "dequantize_4bit_nested_chain: blocksize must be a power of two in [32, 4096] (got %d)",
                    blocksize);
    if (blocksize2 != 256)
        return fail(BBC_ERR_UNSUPPORTED, "dequantize_4bit_nested_chain: blocksize2 must be 256 (got %d)",
                    blocksize2);
    if (!aligned(out, elem_size(out_dtype)) || !aligned(code2, 4) || !aligned(absmax2, 4) ||
        !aligned(code4, 4) || !aligned(scale_workspace, 4))
        return fail(BBC_ERR_INVALID, "dequantize_4bit_nested_chain: pointer not aligned to its element size");
    const size_t nbo = cdiv(n, blocksize);
    const int sb = check_buffers("dequantize_4bit_nested_chain",
                                 {{codes, cdiv(n, 2), "codes"}, {absmax_q, nbo, "absmax_q"}, {code2, 1024, "code2"},
                                  {absmax2, cdiv((int64_t)nbo, 256) * 4, "absmax2"}, {code4, 64, "code4"}},
                                 {{out, (size_t)n * elem_size(out_dtype), "out"}, {scale_workspace, nbo * 4, "scale_workspace"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(out, 32) && aligned(codes, 16);
    return cuda_status(bbc::launch_nested_dequantize_chain(codes, absmax_q, code2, absmax2, offset, code4, n,
                                                           log2_bs, out_dtype, out, scale_workspace, vec,
                                                           static_cast<cudaStream_t>(stream)),
                       "dequantize_4bit_nested_chain launch");
}

int dequantize_4bit_nested_chain_noalloc(const uint8_t* codes, const uint8_t* absmax_q,
                                         const float* code2, const float* absmax2, float offset,
                                         const float* code4, int64_t n, int blocksize, int blocksize2,
                                         int out_dtype, void* out, void* stream) {
    const char* fn = "dequantize_4bit_nested_chain_noalloc";
    if (!codes || !absmax_q || !code2 || !absmax2 || !code4 || !out)
        return fail(BBC_ERR_INVALID, "%s: null pointer argument", fn);
    if (n <= 0) return fail(BBC_ERR_INVALID, "%s: n must be >= 1 (got %lld)", fn, (long long)n);
    if (!valid_dtype(out_dtype)) return fail(BBC_ERR_INVALID, "%s: bad dtype %d", fn, out_dtype);
    const int log2_bs = log2_blocksize(blocksize);
    if (log2_bs < 0)
        return fail(BBC_ERR_INVALID, "%s: blocksize must be a power of two in [32, 4096] (got %d)", fn,
                    blocksize);
    if (blocksize2 != 256)
        return fail(BBC_ERR_UNSUPPORTED, "%s: blocksize2 must be 256 (got %d)", fn, blocksize2);
    const int64_t nbo = (n + blocksize - 1) / blocksize;
    if (nbo > BBC_NOALLOC_SCRATCH_FLOATS)
        return fail(BBC_ERR_UNSUPPORTED,
                    "%s: needs %lld scale slots (n=%lld, blocksize=%d) but the static scratch holds %d; "
                    "use dequantize_4bit_nested_chain with a workspace or dequantize_4bit_nested",
                    fn, (long long)nbo, (long long)n, blocksize, BBC_NOALLOC_SCRATCH_FLOATS);
    if (!aligned(out, elem_size(out_dtype)) || !aligned(code2, 4) || !aligned(absmax2, 4) || !aligned(code4, 4))
        return fail(BBC_ERR_INVALID, "%s: pointer not aligned to its element size", fn);
    const int sb = check_buffers(fn, {{codes, cdiv(n, 2), "codes"}, {absmax_q, (size_t)nbo, "absmax_q"}, {code2, 1024, "code2"},
                                      {absmax2, cdiv(nbo, 256) * 4, "absmax2"}, {code4, 64, "code4"}},
                                 {{out, (size_t)n * elem_size(out_dtype), "out"}});
    if (sb != BBC_OK) return sb;
    const bool vec = aligned(out, 32) && aligned(codes, 16);
    return cuda_status(bbc::launch_nested_dequantize_chain_noalloc(codes, absmax_q, code2, absmax2, offset,
                                                                   code4, n, log2_bs, out_dtype, out, vec,
                                                                   static_cast<cudaStream_t>(stream)),
                       fn);
}

int bbc_wait_timeouts(unsigned int* count) {
    if (!count) return fail(BBC_ERR_INVALID, "bbc_wait_timeouts: null pointer argument");
    return cuda_status(bbc::wait_timeouts(count), "bbc_wait_timeouts");
}

int bbc_debug_status(unsigned int* status, int reset) {
    if (!status) return fail(BBC_ERR_INVALID, "bbc_debug_status: null pointer argument");
    cudaError_t (*const words[])(unsigned int*, bool) = {
        bbc::guard_status_kbit_quant, bbc::guard_status_kbit_dequant, bbc::guard_status_nested_dequant,
        bbc::guard_status_nested_quant, bbc::guard_status_linear, bbc::guard_status_linear_tc};
    unsigned int all = 0;
    for (auto word : words) {
        unsigned int v = 0;
        const cudaError_t e = word(&v, reset != 0);
        if (e != cudaSuccess) return cuda_status(e, "bbc_debug_status");
        all |= v;
    }
    *status = all;
    return BBC_OK;
}

int bbc_is_debug_build(void) {
#ifdef BBC_DEBUG
    return 1;
#else
    return 0;
#endif
}

const char* bbc_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
