/*
 * bbc.h - C ABI of the blockwise bit-codebook library (NVIDIA B200, sm_100a).
 *
 * Operations on weight tensors, defined by the pages this library follows
 * (cited per entry point below):
 *   1. k-bit blockwise codebook quantization (K = 2..5, blocksize 32) and its
 *      inverse, with bit-plane packing of the codes, with an fp32 or an E4M4
 *      byte absmax per block;
 *   2. nested NF4/FP4 dequantization, where each outer block's fp32 scale is
 *      rebuilt from a General8-coded absmax inside the value-decode kernel,
 *      its unfused three-launch form, and the plain 4-bit decode;
 *   3. the inverse of 2: 4-bit quantization and the nested absmax state
 *      (readings: the pages give only the decode);
 *   4. the nested 4-bit and the k-bit decode fused into their linear consumer
 *      (Y = X W^T with the weight decoded in registers, never written to memory).
 *
 * Conventions for every entry point:
 *   - Buffer pointers are DEVICE pointers (memory of the current CUDA device)
 *     unless a comment says host. The caller allocates and owns every buffer;
 *     the library never allocates, frees or keeps a pointer after returning.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Calls are asynchronous on that stream and never synchronize.
 *   - Inputs are read-only. Outputs must not overlap any input.
 *   - Arguments are validated on the host before any launch; on failure the
 *     call returns a non-zero bbc_status, launches nothing and writes nothing.
 *     bbc_last_error() then returns a message (per calling thread).
 *   - A launch failure returns BBC_ERR_CUDA (message from cudaGetErrorString).
 *   - dtype values: BBC_F16 (IEEE binary16), BBC_BF16 (bfloat16), BBC_F32.
 *   - Conversions to fp16/bf16 round to nearest, ties to even; subnormals are
 *     kept (no flush to zero) in every step.
 *   - Device pointers need only the natural alignment of their element type.
 *     Well-aligned buffers take the vectorised path (32 bytes for the input of
 *     the quantizers and for the outputs of the dequantizers, 16 bytes for the
 *     4-bit codes), others a scalar path with identical results.
 */
#ifndef BBC_H
#define BBC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bbc_dtype { BBC_F16 = 0, BBC_BF16 = 1, BBC_F32 = 2 } bbc_dtype;

typedef enum bbc_status {
    BBC_OK = 0,
    BBC_ERR_INVALID = 1,      /* bad argument: null pointer, n <= 0, K out of range, bad dtype */
    BBC_ERR_UNSUPPORTED = 2,  /* valid in principle but not built: blocksize != 32, bs2 != 256 */
    BBC_ERR_CUDA = 3          /* a CUDA runtime call or launch failed */
} bbc_status;

/*
 * kbit_quantize - k-bit blockwise codebook quantization.
 *
 * Defined by: bitsandbytes k-bit patch series, PATCH 001 "Add k-bit
 * quantization kernels (K=2-5, blocksize=32)": quantize_kbit_ref in
 * tests/test_kbit_quantization.py and kQuantizeBlockwise_kbit in csrc/ops.cu.
 *
 * For each block b of 32 consecutive elements of A (the last block padded
 * with 0.0):
 *   absmax[b] = max_i |x_i|                       (raw, unclamped)
 *   d         = max(absmax[b], 1e-8f)
 *   xn_i      = x_i / d                           (IEEE fp32 division)
 *   idx_i     = first i minimising fabsf(xn_i - codebook[i])
 *   packed[b*K + j] bit i = bit j of idx_i        (bit-plane layout)
 * Padding lanes of the last block are quantized like 0.0 and their bits are
 * stored.
 *
 *   A          [n] elements of `dtype` (fp16, bf16 or fp32).
 *   n          element count, >= 1.
 *   K          bits per code, 2..5.
 *   blocksize  must be 32 (BBC_ERR_UNSUPPORTED otherwise).
 *   codebook   [2^K] fp32 device values. Any values give the exact result;
 *              finite, strictly ascending entries spaced at least
 *              2^-19 * (1 + max|c|) apart take the fast threshold search,
 *              others a brute-force search.
 *   absmax     [ceil(n/32)] fp32 output.
 *   packed     [ceil(n/32) * K] uint32 output.
 * NaN or infinite inputs give the same result as the rule above (a NaN is
 * ignored by the max unless the whole block is NaN; NaN distances never win).
 */
int kbit_quantize(const void* A, int dtype, int64_t n, int K, int blocksize,
                  const float* codebook, float* absmax, uint32_t* packed, void* stream);

/*
 * kbit_dequantize - inverse of kbit_quantize.
 *
 * Defined by: the same patch series, dequantize_kbit_ref and
 * kDequantizeBlockwise_kbit: out[m] = T(codebook[idx_m] * absmax[m / 32]),
 * one fp32 multiply then one rounding to the output type, for m < n only.
 *
 *   packed     [ceil(n/32) * K] uint32, layout as written by kbit_quantize.
 *   absmax     [ceil(n/32)] fp32.
 *   codebook   [2^K] fp32.
 *   K          2..5.   blocksize must be 32.
 *   n          element count, >= 1.
 *   out_dtype  BBC_F16, BBC_BF16 or BBC_F32.
 *   out        [n] elements of out_dtype (nothing beyond n is written).
 */
int kbit_dequantize(const uint32_t* packed, const float* absmax, const float* codebook,
                    int K, int blocksize, int64_t n, int out_dtype, void* out, void* stream);

/*
 * kbit_quantize_e4m4 / kbit_dequantize_e4m4 - the k-bit codec with each block's
 * absmax stored as one E4M4 byte instead of an fp32 word (K=4: 4.25 instead of
 * 5 bits per element).
 *
 * Defined by: bitsandbytes k-bit patch series, PATCH 005 "Add vectorized
 * dequant kernel and E4M4 uint8 absmax support" (encode_absmax_e4m4,
 * decode_absmax_e4m4, decode_e4m4_absmax, quantize_kbit absmax_format "e4m4").
 * Code c: e = c >> 4, m = c & 15; value 2^(e-11) * (1 + m/16) for e > 0 and
 * m * 2^-14 for e == 0 (0.0 at c == 0; range 2^-14 .. 31.0).
 * Encode of an absmax a: a not > 0 (zero, NaN) -> 0; +inf -> 0xFF (a reading);
 * otherwise exponent field floor(log2 a) + 11 clamped to [0, 15] (subnormal
 * when <= 0: m = round(a * 2^14)), mantissa round((a / 2^floor(log2 a) - 1) * 16)
 * half-to-even, clamped to [0, 15]. At and above 32 the exponent field clamps
 * while the mantissa stays that of a's own binade, as the page's steps compute.
 *
 * kbit_quantize_e4m4: as kbit_quantize; the packed words are identical to its
 *   (indices use the exact fp32 absmax), absmax_e4m4 [ceil(n/32)] receives the
 *   codes. Alignment: any uint8 pointer.
 * kbit_dequantize_e4m4: as kbit_dequantize with each block's scale the exact
 *   value of its code: out[m] = T(codebook[idx_m] * value(absmax_e4m4[m / 32])).
 * Errors as kbit_quantize / kbit_dequantize.
 */
int kbit_quantize_e4m4(const void* A, int dtype, int64_t n, int K, int blocksize, const float* codebook,
                       uint8_t* absmax_e4m4, uint32_t* packed, void* stream);
int kbit_dequantize_e4m4(const uint32_t* packed, const uint8_t* absmax_e4m4, const float* codebook, int K,
                         int blocksize, int64_t n, int out_dtype, void* out, void* stream);

/*
 * dequantize_4bit_nested - NF4/FP4 dequantization with the nested
 * ("compressed statistics") scale rebuilt inside the decode.
 *
 * Defined by: pull request "Fuse nested 4-bit scale reconstruction on SM103",
 * Summary and Implementation: the outer-block fp32 scale is the General8 code
 * of the quantized absmax times the inner absmax, then plus the offset, as a
 * separately rounded fp32 multiply and add (no fused multiply-add), applied
 * while the 4-bit values are decoded, with no intermediate scale tensor:
 *   b        = m / blocksize
 *   scale_b  = fl(fl(code2[absmax_q[b]] * absmax2[b / blocksize2]) + offset)
 *   out[m]   = T(fl(code4[nibble_m] * scale_b))
 * Nibble order (a reading; the page does not print it): element 2j is the
 * high nibble (bits 7..4) of codes[j], element 2j+1 the low nibble.
 *
 *   codes       [ceil(n/2)] uint8, two 4-bit codes per byte.
 *   absmax_q    [ceil(n/blocksize)] uint8 General8 codes of the outer absmax.
 *   code2       [256] fp32 General8 code table.
 *   absmax2     [ceil(ceil(n/blocksize)/blocksize2)] fp32 inner absmax.
 *   offset      fp32 scalar added to every outer scale.
 *   code4       [16] fp32 value table (NF4 or FP4).
 *   n           element count, >= 1.
 *   blocksize   outer block size: a power of two in [32, 4096].
 *   blocksize2  inner block size: must be 256 (BBC_ERR_UNSUPPORTED otherwise).
 *   out_dtype   BBC_F16, BBC_BF16 or BBC_F32;   out [n] elements.
 */
int dequantize_4bit_nested(const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                           const float* absmax2, float offset, const float* code4,
                           int64_t n, int blocksize, int blocksize2, int out_dtype, void* out,
                           void* stream);

/*
 * dequantize_4bit - plain NF4/FP4 dequantization with an fp32 absmax per block.
 *
 * Defined by: pull request "Fuse nested 4-bit scale reconstruction on SM103",
 * Summary: the NF4/FP4 value dequantization that is the last of the three
 * launches of the unfused path, out[m] = T(fl(code4[nibble_m] * absmax[m / blocksize])).
 * Nibble order as in dequantize_4bit_nested.
 *
 *   codes      [ceil(n/2)] uint8.   absmax [ceil(n/blocksize)] fp32.
 *   code4      [16] fp32.           n >= 1.   blocksize: power of two in [32, 4096].
 *   out_dtype  BBC_F16, BBC_BF16 or BBC_F32;   out [n] elements.
 */
int dequantize_4bit(const uint8_t* codes, const float* absmax, const float* code4, int64_t n,
                    int blocksize, int out_dtype, void* out, void* stream);

/*
 * quantize_4bit - 4-bit codes and fp32 absmax per outer block: the inverse of
 * dequantize_4bit.
 *
 * Defined by: the pages give only the decode (pull request "Fuse nested 4-bit
 * scale reconstruction on SM103"); the encode is the k-bit rule of the
 * bitsandbytes k-bit series (PATCH 001 quantize_kbit_ref) applied per outer
 * block of `blocksize` elements, a reading:
 *   absmax[b] = max |x| over the block (raw; NaN only if every element is NaN)
 *   d         = fmaxf(absmax[b], 1e-8f)
 *   code_m    = first i minimising fabsf(fl(x_m / d) - code4[i])
 * packed two per byte, element 2j in the high nibble of codes[j] (the unused
 * low nibble of an odd n is 0).
 *
 *   A        [n] elements of dtype.   n >= 1.   blocksize: power of two in [32, 4096].
 *   code4    [16] fp32 (NF4, FP4 or any table; ascending well-spaced tables take the
 *            fast exact path, others the rule verbatim).
 *   absmax   [ceil(n/blocksize)] fp32 out.   codes [ceil(n/2)] uint8 out.
 * Fast paths need A 32-byte and codes 16-byte aligned; other alignments give the
 * same results more slowly.
 */
int quantize_4bit(const void* A, int dtype, int64_t n, int blocksize, const float* code4, float* absmax,
                  uint8_t* codes, void* stream);

/*
 * quantize_4bit_nested - the nested ("compressed statistics") 4-bit state of A,
 * the inverse of dequantize_4bit_nested.
 *
 * Defined by: the same decode; the encode steps are readings (no page gives them):
 *   1. codes and fp32 absmax per outer block as quantize_4bit;
 *   2. offset = mean of the outer absmax, summed in binary64 by a fixed pairwise
 *      tree (the values zero-padded to the next power of two, each node the sum of
 *      its two halves), divided by the block count, rounded once to fp32;
 *   3. per group of blocksize2 = 256 outer blocks, c_b = fl(absmax_b - offset):
 *      absmax2[g] = max |c_b|,  absmax_q[b] = first i minimising
 *      fabsf(fl(c_b / fmaxf(absmax2[g], 1e-8f)) - code2[i]).
 * dequantize_4bit_nested then rebuilds each scale as fl(fl(code2[q] * absmax2) + offset).
 *
 *   code2      [256] fp32 General8 table.   blocksize2: must be 256.
 *   codes      [ceil(n/2)] uint8 out.   absmax_q [ceil(n/blocksize)] uint8 out.
 *   absmax2    [ceil(ceil(n/blocksize)/256)] fp32 out.
 *   offset     one fp32 out, a DEVICE pointer (read it back before dequantizing).
 *   workspace  DEVICE scratch of quantize_4bit_nested_workspace_bytes(n, blocksize)
 *              bytes, 256-byte aligned, caller-owned, not overlapping any argument.
 * Two launches on `stream` (codes, then the absmax compression, which also forms the
 * offset) plus one per level of the offset tree above 2048 outer blocks (three at 4M
 * outer blocks). Errors as quantize_4bit; a workspace that is too small
 * is BBC_ERR_INVALID, blocksize2 != 256 BBC_ERR_UNSUPPORTED.
 */
size_t quantize_4bit_nested_workspace_bytes(int64_t n, int blocksize);
int quantize_4bit_nested(const void* A, int dtype, int64_t n, int blocksize, const float* code4,
                         const float* code2, int blocksize2, uint8_t* codes, uint8_t* absmax_q, float* absmax2,
                         float* offset, void* workspace, size_t workspace_bytes, void* stream);

/*
 * dequantize_4bit_nested_chain - the unfused three-launch form of
 * dequantize_4bit_nested, kept as an in-library comparator.
 *
 * Defined by: the same pull request, Summary: General8 scale dequantization
 * (scale_b = fl(code2[absmax_q[b]] * absmax2[b / blocksize2]) into an fp32
 * tensor), an offset add (scale_b = fl(scale_b + offset)), then NF4/FP4 value
 * dequantization reading that tensor. Results are identical to
 * dequantize_4bit_nested; the cost is the extra launches and the round trip
 * of the scale tensor through memory.
 *
 * Arguments as dequantize_4bit_nested, plus:
 *   scale_workspace  DEVICE buffer of ceil(n/blocksize) floats, caller-owned; it
 *                    receives the scales and must not overlap any other argument.
 */
int dequantize_4bit_nested_chain(const uint8_t* codes, const uint8_t* absmax_q, const float* code2,
                                 const float* absmax2, float offset, const float* code4,
                                 int64_t n, int blocksize, int blocksize2, int out_dtype, void* out,
                                 float* scale_workspace, void* stream);

/*
 * Capacity, in floats, of the library's static scale scratch used by
 * dequantize_4bit_nested_chain_noalloc (4 MiB; every GPU that loads the
 * library keeps it until the process exits).
 */
#define BBC_NOALLOC_SCRATCH_FLOATS 1048576

/*
 * dequantize_4bit_nested_chain_noalloc - dequantize_4bit_nested_chain without a
 * caller-supplied workspace and without any allocation.
 *
 * The pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory -- for example code hosted inside another
 * framework that hands it only input and output buffers and owns every other
 * byte of the GPU, or a latency-sensitive loop that must not call cudaMalloc
 * once it is running, because allocation can block on the device. The
 * intermediate scale tensor lives in one fixed array inside the library, so
 * the call only needs its inputs and its output.
 *
 * Arguments, results and errors are those of dequantize_4bit_nested_chain
 * without scale_workspace. In addition:
 *   - ceil(n / blocksize) must not exceed BBC_NOALLOC_SCRATCH_FLOATS; larger
 *     requests return BBC_ERR_UNSUPPORTED and launch nothing.
 *   - Each call made while `stream` is not being captured looks up the
 *     current device's copy of the array (so that it stays right after
 *     cudaDeviceReset reloads the library's module); a call during stream
 *     capture uses the address the last such call found, so make the first call
 *     on each device before capturing any stream. Neither allocates anything.
 *   - All calls share the one array per device and it keeps whatever the last
 *     call left there. Each call writes every scale it later reads, so nothing
 *     needs clearing, but calls whose work can overlap on the GPU (different
 *     streams, or host threads that do not order their launches) race on it:
 *     keep such calls on one stream or otherwise ordered.
 */
int dequantize_4bit_nested_chain_noalloc(const uint8_t* codes, const uint8_t* absmax_q,
                                         const float* code2, const float* absmax2, float offset,
                                         const float* code4, int64_t n, int blocksize, int blocksize2,
                                         int out_dtype, void* out, void* stream);

/*
 * linear_4bit_nested - Y = X W^T, with W the nested 4-bit weight of
 * dequantize_4bit_nested decoded on the fly (W is never written to memory).
 *
 * Defined by: "Fuse nested 4-bit scale reconstruction on SM103", Summary and
 * its timing of the public dequantize-plus-linear paths (the "recurrent grad_A"
 * and "fallback forward" controls at M = 1, 8 and 32 activation rows). Each
 * weight is exactly the element dequantize_4bit_nested would write in the
 * activation type T: w[n][k] = T(fl(code4[nibble(n*K + k)] * scale_b)),
 * scale_b = fl(fl(code2[absmax_q[b]] * absmax2[b / 256]) + offset),
 * b = (n*K + k) / blocksize (the weight is the flattened N x K row-major tensor).
 * The products x*w are exact in fp32 and are summed in fp32 (tensor-core
 * accumulation, a fixed order: the same inputs give the same bits); each Y
 * element is rounded once to T. Not bit-exact against a float64 sum: the error
 * is at most 2*K*2^-24*sum_k |x w| plus half an ulp of T.
 * M <= 32 runs warp-level MMAs on weights decoded in registers; M > 32 runs the
 * fifth-generation tensor cores (tcgen05, accumulators in tensor memory) on
 * 128-row weight tiles decoded into shared memory, with activation tiles loaded
 * by TMA and, when there are few output tiles, K split over a thread-block
 * cluster whose partial sums are added in a fixed order in distributed shared
 * memory (no workspace). Its mbarrier waits are bounded: see bbc_wait_timeouts.
 *
 *   X        [M][K] activations, row-major, dtype BBC_F16 or BBC_BF16 (T),
 *            16-byte aligned.
 *   M        >= 1.   N: a multiple of 16 (of 128 when M > 32).
 *   K        a multiple of 64.
 *   codes    [N*K/2] uint8 (element 2j in the high nibble of byte j),
 *            16-byte aligned.
 *   absmax_q [ceil(N*K/blocksize)] uint8.   code2 [256] fp32.
 *   absmax2  [ceil(ceil(N*K/blocksize)/256)] fp32.   offset: fp32 by value.
 *   code4    [16] fp32 value table (NF4 or FP4).
 *   blocksize  power of two in [32, 4096].   blocksize2: must be 256.
 *   Y        [M][N] out, row-major, dtype T.
 * One launch on `stream`. Errors: null pointers, M/N/K < 1, a bad blocksize or
 * misaligned X/codes -> BBC_ERR_INVALID; another dtype, N % 16 != 0 (N % 128
 * != 0 when M > 32), K % 64 != 0 or blocksize2 != 256 -> BBC_ERR_UNSUPPORTED.
 */
int linear_4bit_nested(const void* X, int dtype, int64_t M, int64_t N, int64_t K, const uint8_t* codes,
                       const uint8_t* absmax_q, const float* code2, const float* absmax2, float offset,
                       const float* code4, int blocksize, int blocksize2, void* Y, void* stream);

/*
 * linear_kbit - Y = X W^T, with W the k-bit weight of kbit_quantize decoded on
 * the fly (W is never written to memory).
 *
 * Defined by: the k-bit patch series, dequantize_kbit (the decode) followed by
 * a linear layer, the consumer the nested-dequant pull request times on its
 * public paths ("Fuse nested 4-bit scale reconstruction on SM103", Summary).
 * Each weight is exactly the element kbit_dequantize would write in the
 * activation type T: w[n][k] = T(fl(codebook[idx(m)] * absmax[m / 32])) for the
 * flattened element m = n*K + k of the N x K row-major weight. Accumulation,
 * error bound and the two paths (M <= 32, M > 32) as linear_4bit_nested (fp32
 * tensor-core sums in a fixed order, at most 2*K*2^-24*sum_k |x w| plus half an
 * ulp of T from the float64 result).
 *
 *   X        [M][K] activations, row-major, dtype BBC_F16 or BBC_BF16 (T),
 *            16-byte aligned.
 *   M        >= 1.   N: a multiple of 16 (of 128 when M > 32).
 *   K        a multiple of 64.
 *   packed   [N*K/32 * bits] uint32 bit-plane words (kbit_quantize layout),
 *            16-byte aligned.
 *   absmax   [N*K/32] fp32.   codebook: [2^bits] fp32.
 *   bits     2..5 (the K of kbit_quantize).   blocksize: must be 32.
 *   Y        [M][N] out, row-major, dtype T.
 * One launch on `stream`. Errors: null pointers, M/N/K < 1, bits outside 2..5
 * or misaligned X/packed -> BBC_ERR_INVALID; another dtype, N % 16 != 0 (N % 128
 * != 0 when M > 32), K % 64 != 0 or blocksize != 32 -> BBC_ERR_UNSUPPORTED.
 */
int linear_kbit(const void* X, int dtype, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                const float* absmax, const float* codebook, int bits, int blocksize, void* Y, void* stream);

/*
 * bbc_nf_codebook - the 2^K-entry normal-float codebook, on the HOST.
 *
 * Defined by: the k-bit patch series, create_normal_float_codebook: standard
 * normal quantiles at the bin midpoints (2i+1)/(2^(K+1)), computed in double,
 * rounded to fp32, then divided (in fp32) by the largest magnitude. Sorted
 * ascending, largest magnitude exactly 1.
 *
 *   K            1..8.
 *   codebook_out HOST buffer of 2^K floats, written by the call.
 * Host-only: no CUDA call is made.
 */
int bbc_nf_codebook(int K, float* codebook_out);

/*
 * bbc_wait_timeouts - failure detection for the kernels that wait on one
 * another's progress inside a CTA (the tensor-core linear layers: mbarrier
 * waits between the TMA, decode, MMA and epilogue roles). Every such wait gives
 * up after a bounded number of polls instead of hanging, counts itself in a
 * per-device counter and lets the kernel wind down (its results are then not
 * meaningful). No counterpart on the pages.
 *
 *   count  HOST pointer: receives the number of waits that gave up on the
 *          current device since the previous call; the counter is reset.
 * Synchronous (a device-to-host copy on the legacy stream). Errors: a null
 * pointer -> BBC_ERR_INVALID; a failed copy -> BBC_ERR_CUDA.
 */
int bbc_wait_timeouts(unsigned int* count);

/*
 * bbc_debug_status - the bounds guards of a debug build (the library compiled
 * with -DBBC_DEBUG, libbbc_debug.so next to libbbc.so). In that build every
 * global load and store whose address a kernel computes is checked against the
 * extent its launch's arguments give that buffer; a failed check skips the
 * access (no trap: the context stays usable) and sets a bit in a per-device
 * status word: 1 quantize input loads and prefetches, 2 quantize stores, 4 k-bit
 * dequant loads, 8 k-bit dequant stores, 16 nested dequant loads, 32 nested
 * dequant stores, 64 offset tree, 128 General8 compression, 256 fused linear
 * weight loads. Outputs of a launch that set a bit are not meaningful. A release
 * build has no guards and always reports 0. No counterpart on the pages.
 *
 *   status HOST pointer: receives the OR of the bits set on the current device
 *          since the last reset.
 *   reset  nonzero: clear the bits after reading them.
 * Synchronous (device-to-host copies on the legacy stream). Errors: a null
 * pointer -> BBC_ERR_INVALID; a failed copy -> BBC_ERR_CUDA.
 */
int bbc_debug_status(unsigned int* status, int reset);

/* 1 in a debug build (bounds guards compiled in, see bbc_debug_status), else 0. */
int bbc_is_debug_build(void);

/* Message for the last non-OK status returned on the calling thread ("" if none). */
const char* bbc_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BBC_H */
