/*
 * int4.h - C ABI of the B200 (sm_100a) INT4 weight-only quantization library.
 *
 * Symmetric group-wise INT4 quantization with two's-complement nibble packing
 * and the weight-only dequantizing matmul, as stated by the web page
 * "Implement INT4 group quantization, nibble packing and a dequantizing
 * matmul" (inferenceinterviews.com drill), problem statement: three functions
 * quantize_int4(w, group) -> (packed, scales, K), unpack_int4(packed, K) and
 * int4_matmul(x, packed, scales, K, group).  The entry points below keep that
 * argument order: inputs in the page's order, then derived shapes, then the
 * outputs, then the CUDA stream.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument is a DEVICE pointer owned by the caller.  The
 *   library allocates no device or host memory and keeps no reference to the
 *   buffers after the call returns.
 * - All tensors are dense and row-major with no padding between rows:
 *     w       [N, K]         fp32, bf16 or fp16 (w_dtype)
 *     packed  [N, ceil(K/2)] uint8; row stride ceil(K/2) bytes
 *     scales  [N, G]         fp16 bit patterns, G = ceil(K / group)
 *     unpack  [N, K]         int8
 *     x       [M, K]         fp32, bf16 or fp16 (x_dtype)
 *     y       [M, N]         fp32
 * - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL means
 *   the legacy default stream), like a kernel launch.  A zero return means
 *   the work was launched, not that it has finished.
 * - Buffers must not overlap, except that nothing is written to an input.
 * - Return value: INT4_OK (0) or one of the INT4_ERR_* codes.  Arguments are
 *   validated on the host before anything is launched; on a non-zero return
 *   nothing was launched and no output was touched, except INT4_ERR_CUDA,
 *   which reports a launch failure (its message is in int4_last_error()).
 * - Thread safety: entry points may be called from several host threads; the
 *   last-error message is kept per host thread.
 * - Sizes: N, M >= 1, K >= 1, group >= 1.  (N or M == 0, an empty problem,
 *   returns INT4_OK and launches nothing.)  N * K, M * K and M * N must each
 *   be below 2^62.
 */
#ifndef INT4_B200_H
#define INT4_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define INT4_OK             0
#define INT4_ERR_ARG        1  /* null pointer, negative size, group < 1, size overflow */
#define INT4_ERR_DTYPE      2  /* unknown dtype code */
#define INT4_ERR_ALIGN      3  /* a pointer not aligned to its element size */
#define INT4_ERR_CUDA       4  /* a CUDA launch or runtime call failed */
#define INT4_ERR_TIMEOUT    5  /* a bounded device-side wait gave up (see int4_device_status) */
#define INT4_ERR_UNSUPPORTED 6 /* a forced kernel path cannot run this shape */

/* Element type codes for w_dtype and x_dtype. */
#define INT4_DTYPE_F32   0
#define INT4_DTYPE_BF16  1
#define INT4_DTYPE_F16   2

/*
 * int4_quantize - group absmax, fp16 scale, INT4 codes and nibble packing.
 *
 * Page: the drill's quantize_int4 ("scale = absmax of the group / 7", "q =
 * round(w / scale) clipped to [-8, 7], as a two's-complement nibble; element
 * 2j in the low nibble of byte j (an odd K pads one zero nibble; a group of
 * zeros gets scale 0)"), with the per-row blocks along K of the page
 * "Building a pure-Python INT4 transformer weight quantizer with block-wise
 * per-channel scaling", sections 3 and 4.
 *
 * For row n and group g (columns [g*group, min((g+1)*group, K))):
 *   m      = max |w[n, k]| over the group's real columns (exact)
 *   s      = fp16_RNE( fp32(m) / 7 )   (IEEE fp32 division, then RNE to fp16)
 *   q[n,k] = clamp( rint_half_even( fp32(w[n,k]) / fp32(s) ), -8, 7 )
 *            (IEEE fp32 division), and q = 0 for the whole group when s == 0
 *   packed[n, j] = (q[n,2j] & 0xF) | ((q[n,2j+1] & 0xF) << 4), q[n,K] := 0
 *   scales[n, g] = bit pattern of s
 * The outputs are bit-exact functions of w under this convention.
 * Precondition: w is finite (NaN/Inf input gives unspecified codes).
 *
 * w       [N, K] device buffer of w_dtype; alignment: its element size.
 * w_dtype INT4_DTYPE_F32 / _BF16 / _F16.
 * packed  [N, ceil(K/2)] device output; any alignment.
 * scales  [N, ceil(K/group)] device output (fp16 bits); 2-byte aligned.
 */
int int4_quantize(const void* w, int32_t w_dtype, int64_t N, int64_t K, int32_t group,
                  uint8_t* packed, uint16_t* scales, void* stream);

/*
 * int4_unpack - nibbles to sign-extended int8.
 *
 * Page: the drill's unpack_int4(packed, K) -> int8 [N, K], sign-extended
 * (its hidden suite names "sign extension of -8").  out[n, k] is the low
 * nibble of packed[n, k/2] for even k and the high nibble for odd k, read as
 * a 4-bit two's-complement value in [-8, 7].  The pad nibble of an odd K is
 * not read.  Bit-exact.
 *
 * packed [N, ceil(K/2)] device input; any alignment.
 * out    [N, K] int8 device output; any alignment.
 */
int int4_unpack(const uint8_t* packed, int64_t K, int64_t N, int8_t* out, void* stream);

/*
 * int4_dequantize - the dequantized weights w_hat = q * s, as a dense matrix.
 *
 * Pages: "Building a pure-Python INT4 transformer weight quantizer with
 * block-wise per-channel scaling", section 5 (w_hat = q * s per block), and
 * the drill, whose hidden suite checks the matmul "against a full
 * dequantization"; "Quantizing a Language Model From Scratch" runs its model
 * on such fake-quantized weights.  out[n, k] = RNE_out( q[n, k] * s[n, k /
 * group] ): the product is exact in fp32 and rounded once, to nearest even,
 * to out_dtype (fp32 output is exact; fp16 output overflows to +-inf where
 * |q s| > 65504).  Bit-exact.  It is the first half of the unfused
 * dequantize-then-GEMM design the fused int4_matmul replaces; it is not used
 * by int4_matmul.
 *
 * packed    [N, ceil(K/2)] device input; any alignment.
 * scales    [N, ceil(K/group)] fp16 bits; 2-byte aligned.
 * out       [N, K] device output of out_dtype; alignment: its element size.
 * out_dtype INT4_DTYPE_F32 / _BF16 / _F16.
 */
int int4_dequantize(const uint8_t* packed, const uint16_t* scales, int64_t K, int32_t group,
                    int64_t N, void* out, int32_t out_dtype, void* stream);

/*
 * int4_matmul - weight-only dequantizing matmul y = x @ dequantize(W)^T.
 *
 * Page: the drill's int4_matmul(x, packed, scales, K, group) -> float32
 * [M, N]: "computed one group at a time: multiply x by the group's integer
 * weights first, then apply the group's scale to each output column".
 *   y[m, n] = sum_g s[n, g] * ( sum_{k in g} x[m, k] * q[n, k] )
 * Integer weights enter the arithmetic exactly (-8..7 is exact in bf16, fp16
 * and fp32); group partial sums are accumulated in fp32 (fp64 across groups
 * for fp32 x); the group's scale is applied to each partial before it joins
 * the running sum.  The decode kernel for groups that are a multiple of 128
 * forms each 128-k block's sum x.q exactly in integers wherever x is an
 * integer multiple of 2^-29 times the block's largest power of two (every
 * bf16 x within 2^22 of the block's largest |x|, fp16 within 2^19); a block
 * of a batch row where that does not hold (a wider span, values below about
 * 2^-93, NaN or infinity) is computed with bf16/fp16 products and fp32 sums
 * instead, so x is never rounded.
 * Accuracy, for every finite input: |y - y_exact| <= c * sum_k |x[m,k]| |w_hat[n,k]|
 * with c = 1e-5 for fp32 x and c = 4e-3 for bf16 / fp16 x.  NaN or infinity
 * in x propagates as in IEEE arithmetic.  Summation order differs between
 * kernels; results are deterministic for a given shape, dtype, schedule
 * (with or without a workspace) and device.
 *
 * x       [M, K] device input of x_dtype; alignment: its element size.
 * packed  [N, ceil(K/2)] device input; any alignment.
 * scales  [N, ceil(K/group)] fp16 bits; 2-byte aligned.
 * y       [M, N] fp32 device output; 4-byte aligned.
 *
 * Kernel choice (automatic): bf16/fp16 x with M <= 16 takes the streaming
 * decode kernel; bf16/fp16 x with larger M takes the tcgen05 tensor-core
 * kernel; fp32 x, and shapes the fast kernels do not cover (K or group not a
 * multiple of 32, unaligned rows), take the general CUDA-core kernel.
 *
 * int4_matmul needs no workspace.  Its decode schedule gives each CTA whole
 * row tiles, and batches of 3..16 rows take the bf16/fp16 decode kernel; with
 * a workspace (int4_matmul_ws) the decode splits tiles evenly over one wave
 * of CTAs and runs the integer kernel at every M, which is faster when the
 * row tiles do not fill the GPU evenly.
 *
 * Stream ordering: the decode kernels (M <= 16, bf16/fp16 x) launch with
 * programmatic stream serialization and wait for the preceding work on
 * `stream` before touching memory, so ordinary stream order holds.
 * They also signal dependents early: a kernel that the caller launches after
 * them with programmatic stream serialization must execute
 * griddepcontrol.wait (cudaGridDependencySynchronize) before it reads y.
 */
int int4_matmul(const void* x, int32_t x_dtype, const uint8_t* packed, const uint16_t* scales,
                int64_t K, int32_t group, int64_t M, int64_t N, float* y, void* stream);

/*
 * int4_matmul_workspace_size - bytes of device workspace int4_matmul_ws
 * needs for this problem on the current device (written to *bytes; 0 when
 * the chosen kernel needs none).  Host-only; launches nothing.  The size
 * depends on the device (its SM count), so query it on the device that runs
 * the call.
 */
int int4_matmul_workspace_size(int32_t x_dtype, int64_t K, int32_t group, int64_t M, int64_t N,
                               size_t* bytes);

/*
 * int4_matmul_ws - int4_matmul with a caller-owned device workspace.
 *
 * Same contract and result bounds as int4_matmul.  The library allocates
 * nothing: `workspace` holds the decode kernels' scratch (arrival counters,
 * partial tiles of the split, and the integer digits of x at M > 2), or the
 * tensor-core kernel's partial sums of a split K.
 *   - workspace_bytes must be at least int4_matmul_workspace_size(...) for
 *     this problem, else INT4_ERR_ARG (nothing launched).  workspace == NULL
 *     with workspace_bytes == 0 selects the schedule of int4_matmul.  On the
 *     tensor-core path (M > 16) the workspace is optional: when the last
 *     wave of the matrix's tiles (128 weight rows x 128 or 256 batch rows)
 *     leaves SMs idle, a workspace of the queried size lets the call split
 *     the K of that wave's tiles into pieces whose fp32 sums a second kernel
 *     adds in piece order; a smaller or NULL one runs every tile whole.
 *   - workspace must be 256-byte aligned (INT4_ERR_ALIGN) and zero-filled
 *     before its first use; every call leaves its counters zero again, so a
 *     workspace can serve any number of calls, of any shape, that are
 *     ordered on one stream.  Calls that may overlap in time (different
 *     streams) need different workspaces.
 *   - After int4_device_status reports INT4_ERR_TIMEOUT, zero-fill the
 *     workspaces that were in use before reusing them.
 */
int int4_matmul_ws(const void* x, int32_t x_dtype, const uint8_t* packed, const uint16_t* scales,
                   int64_t K, int32_t group, int64_t M, int64_t N, float* y, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Kernel selectors for int4_matmul_path. */
#define INT4_PATH_AUTO     0
#define INT4_PATH_SIMT     1  /* general CUDA-core kernel (any shape, any dtype) */
#define INT4_PATH_DECODE   2  /* skinny decode kernel (bf16/fp16 x, M <= 16) */
#define INT4_PATH_PREFILL  3  /* tcgen05 tensor-core kernel (bf16/fp16 x) */

/*
 * int4_matmul_path - int4_matmul_ws with the kernel chosen by the caller.
 *
 * Same contract as int4_matmul_ws (workspace == NULL with workspace_bytes ==
 * 0: no workspace); `path` is one of INT4_PATH_*.  A forced path that cannot
 * run the given shape or dtype returns INT4_ERR_UNSUPPORTED and launches
 * nothing.  Used to test every kernel on every shape it accepts.
 */
int int4_matmul_path(const void* x, int32_t x_dtype, const uint8_t* packed, const uint16_t* scales,
                     int64_t K, int32_t group, int64_t M, int64_t N, float* y, int32_t path,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * int4_quantize_affine - the asymmetric variant: per-group scale and zero
 * point, unsigned codes.
 *
 * Page: "Build a Blockwise INT4 Inference Engine", step 2 (blockwise
 * quantization with per-group scales and zero-points); "Quantizing a
 * Language Model From Scratch" (affine quantization, x' = S (x_q - Z)).  For
 * row n and group g (the real columns of [g*group, (g+1)*group)):
 *   mn, mx = min and max of w over the group (exact)
 *   s      = fp16_RNE( fp32( fp32(mx - mn) / 15 ) )      (IEEE fp32 ops)
 *   z      = clamp( rint_half_even( fp32(-mn / fp32(s)) ), 0, 15 )
 *   q[n,k] = clamp( rint_half_even( fp32( fp32(w / fp32(s)) + z ) ), 0, 15 )
 *   s == 0 (a constant group, or a range that underflows fp16): q = 0, z = 0
 *   packed[n, j] = q[n,2j] | (q[n,2j+1] << 4) (unsigned nibbles, element 2j
 *   in the low nibble as in int4_quantize; an odd K pads a zero nibble)
 * Bit-exact under this convention.  w_hat = (q - z) s; a zero weight in a
 * group whose range spans 0 is coded exactly.  Precondition: w finite with
 * (mx - mn) / 15 below 65520 in every group.
 *
 * w [N, K] (w_dtype, aligned to its element size); packed [N, ceil(K/2)];
 * scales [N, G] fp16 bits (2-byte aligned); zeros [N, G] uint8.
 */
int int4_quantize_affine(const void* w, int32_t w_dtype, int64_t N, int64_t K, int32_t group,
                         uint8_t* packed, uint16_t* scales, uint8_t* zeros, void* stream);

/*
 * int4_dequantize_affine - w_hat = (q - z) * s rounded once, to nearest even,
 * to out_dtype (int4_dequantize for the asymmetric variant; the same
 * arguments plus the zero points [N, G] uint8).
 */
int int4_dequantize_affine(const uint8_t* packed, const uint16_t* scales, const uint8_t* zeros,
                           int64_t K, int32_t group, int64_t N, void* out, int32_t out_dtype,
                           void* stream);

/* Epilogue flags of int4_matmul_ex. */
#define INT4_EPI_RELU 1  /* y = max(y, 0) after the bias (NaN stays NaN) */

/*
 * int4_matmul_ex - int4_matmul_path with the asymmetric scheme and a fused
 * epilogue.
 *
 * Pages: "Build a Blockwise INT4 Inference Engine", step 3 (the fused kernel
 * computes D = relu(A @ dequantize(Q)) with dequantize = (q - zp) * scale)
 * and step 4 (the layer computes x @ W_dq^T + bias, then ReLU).
 *   y[m, n] = epilogue( sum_g s[n, g] * sum_{k in g} x[m, k] * (q[n, k] - z[n, g]) )
 *   epilogue(v) = v + bias[n] (if bias), then max(., 0) (if INT4_EPI_RELU)
 * zeros   NULL: the symmetric scheme of int4_matmul (two's-complement codes,
 *         z = 0); else [N, ceil(K/group)] uint8 zero points and unsigned
 *         codes from int4_quantize_affine.  Every kernel subtracts z from the
 *         codes before the products, so each group's sum stays exact where
 *         int4_matmul's does, and the accuracy bound of int4_matmul holds with
 *         w_hat = (q - z) s.
 * bias    NULL or [N] fp32, 4-byte aligned; added in fp32 (one rounding).
 * flags   0 or INT4_EPI_RELU.
 * The other arguments, the kernel choice, the workspace rules and the
 * stream ordering are those of int4_matmul_path.
 */
int int4_matmul_ex(const void* x, int32_t x_dtype, const uint8_t* packed, const uint16_t* scales,
                   const uint8_t* zeros, int64_t K, int32_t group, int64_t M, int64_t N,
                   const float* bias, int32_t flags, float* y, int32_t path, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Allocation-free decode matmul.  The pages have no counterpart: this entry
 * exists for callers that must not allocate device memory during the call,
 * such as a serving loop that runs inside a fixed memory budget, or a
 * latency-critical path that must not enter an allocator (whose calls can
 * block, synchronize or fail under memory pressure).
 *
 * Computes what int4_matmul_ws computes on its decode path (same kernels, same
 * split, same result bits), with the partial tiles of the split (4 MiB: one wave of up to
 * 512 CTAs), their arrival counters (2 KiB) and the integer digits of x
 * (4 MiB: K up to 64384 at M = 16, 246528 at M <= 4; not used at M <= 2) kept
 * in a fixed library-owned device array instead of per-stream scratch.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.  The array's arrival counters must start at zero: they
 * are zero when the library loads and every call leaves them zero (after a
 * device-side wait gave up, int4_device_status zeroes them again).
 *
 * Arguments and layouts are those of int4_matmul.  Returns
 * INT4_ERR_UNSUPPORTED when the decode kernel cannot run the shape (x must be
 * bf16 or fp16, M <= 16, K % 32 == 0, group 32, 64 or a multiple of 128, x and
 * packed 16-byte aligned), and INT4_ERR_ARG with a message naming both sizes
 * when the call needs more scratch than the array holds.
 *
 * The first call on each device resolves the array's address with
 * cudaGetSymbolAddress (that device current); make that first call before any
 * stream capture.  The array is shared by all calls on a device: calls that
 * can overlap in time (different streams, or host threads) race on it and
 * must be serialized by the caller. */
int int4_matmul_decode_noalloc(const void* x, int32_t x_dtype, const uint8_t* packed,
                               const uint16_t* scales, int64_t K, int32_t group, int64_t M,
                               int64_t N, float* y, void* stream);

/*
 * int4_matmul_select - the path int4_matmul would take for this problem
 * (one of INT4_PATH_SIMT / _DECODE / _PREFILL), or a negative status if the
 * arguments are invalid.  Host-only; launches nothing.
 */
int int4_matmul_select(int32_t x_dtype, int64_t K, int32_t group, int64_t M, int64_t N);

/*
 * int4_device_status - synchronize `stream`, then read and clear the
 * library's device-side status word of the current device.  Returns INT4_OK,
 * or INT4_ERR_TIMEOUT if a kernel's bounded wait on an mbarrier gave up since
 * the last call (that kernel wrote no output and returned), or INT4_ERR_CUDA.
 */
int int4_device_status(void* stream);

/*
 * int4_selftest_wait_timeout - launch one small kernel whose mbarrier wait is
 * never satisfied, with an iteration limit of `spins`, so that the bounded
 * wait gives up and sets the device status word; used by the tests of the
 * failure path.  No other kernel state is touched.  Returns INT4_OK if the
 * launch succeeded (call int4_device_status to read the outcome).
 */
int int4_selftest_wait_timeout(uint32_t spins, void* stream);

/* Message for the last non-zero status returned on this host thread. */
const char* int4_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int int4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* INT4_B200_H */
