/*
 * aq.h — C ABI of a B200 (sm_100a) library for group-wise affine weight-only
 * quantization and the quantized matmul that consumes it.
 *
 * The method (sources: metalworking "MLX Quantization", section "Mechanics";
 * "Quantizing a Model for MLX", section "What MLX quantization stores"; anllm
 * "Tutorial 10: Quantization", sections 2-5):
 *   W[N,K] is cut along K into groups of G = 32, 64 or 128 consecutive values
 *   of one row.  Each group stores one fp16 scale, one fp16 bias and 2/3/4/8-bit
 *   unsigned codes, so that  w ~= code * scale + bias.
 *     scale = fp16((max - min) / (2^bits - 1))   (fp32 arithmetic, RNE)
 *     bias  = fp16(min)
 *     code  = clamp(rint_even(fp32(fp32(w - bias) / scale)), 0, 2^bits - 1)
 *             computed from the stored fp16 scale and bias; code 0 when scale == 0.
 *   Codes of one row form an LSB-first bitstream: code k occupies bits
 *   [k*bits, k*bits + bits) of the row, and word j holds bits [32j, 32j + 32).
 *   For bits = 2/4/8 this is "(word >> bits*j) & mask" (Tutorial 10, section 3);
 *   for bits = 3 a code may straddle two words (32 codes per 3 words).
 *
 * Types: fp16 and bf16 values travel as their 16-bit patterns (uint16_t).
 * Layouts: every array is row-major and contiguous.
 *   w        fp32      [N, K]
 *   packed   uint32    [N, K*bits/32]
 *   scales   fp16 bits [N, K/G]
 *   biases   fp16 bits [N, K/G]
 *   x        bf16 bits [M, K]
 *   y        bf16 bits [M, N]       y = x @ dequant(W)^T
 * Ownership: every pointer argument is DEVICE memory, allocated, owned and freed
 * by the caller.  Only the tensor-core matmul path (large M) needs temporary
 * device memory (a workspace: the activations converted to fp16 and, for a
 * product of few 256 x 256 tiles, the fp32 partial sums of its K split);
 * aq_matmul and
 * aq_matmul_with take it, stream-ordered on `stream`, from a memory pool the
 * library creates per device and keeps (it holds the largest workspace in use
 * at once until the process exits), aq_matmul_ws takes it from the caller, and
 * aq_matmul_with(AQ_KERNEL_QMM_NOWS) and aq_matmul_qmm_static need none from
 * anybody at call time.
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 * stream); outputs are valid once the stream reaches the call.  The one
 * exception is aq_gather_matmul_grouped with more than 256 experts (or K*bits
 * not a multiple of 128), which reads per-expert counts on the host and so
 * synchronizes its stream.
 *
 * Entry points beyond quantize / dequantize / matmul, each documented below:
 *   aq_quantize_mse           range-search quantizer (same format)
 *   aq_embedding              dequantized rows of a packed table by id
 *   aq_gather_matmul(_grouped) MoE: each token times its routed expert
 *   aq_mxfp4_* / aq_nvfp4_* / aq_mxfp8_*  the block-scaled float modes
 *                              (their own packed layouts, no biases)
 * Errors: arguments are validated synchronously, before anything is launched;
 * a rejected call launches nothing and returns a non-zero status.  Nothing is
 * thrown across the ABI and no kernel traps.
 */
#ifndef AQ_H_
#define AQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *aq_stream_t;

typedef enum {
  AQ_OK = 0,
  AQ_ERR_INVALID_ARG = 1, /* null pointer, N/M/K <= 0, K % G != 0, size overflow */
  AQ_ERR_UNSUPPORTED = 2, /* bits not in {2,3,4,8}, G not in {32,64,128}, shape outside a forced kernel's range,
                             or a device that is not sm_100 */
  AQ_ERR_ALIGNMENT = 3,   /* a pointer not 16-byte aligned */
  AQ_ERR_CUDA = 4,        /* a CUDA runtime error at launch (see aq_last_cuda_error) */
  AQ_ERR_DEVICE_FAULT = 5 /* a kernel recorded a bounded-wait timeout (see aq_device_fault) */
} aq_status;

/* Kernel choice for aq_matmul_with (aq_matmul always uses AQ_KERNEL_AUTO). */
typedef enum {
  AQ_KERNEL_AUTO = 0, /* host-side per-shape dispatch (see aq_dispatch) */
  AQ_KERNEL_QMV = 1,  /* decode kernel, M <= 8 (warp-level integer MMAs; CUDA cores for 3-bit codes) */
  AQ_KERNEL_QMM = 2,  /* tcgen05 / TMEM tensor-core kernel, any M; fp16 activations in a workspace */
  AQ_KERNEL_QMV_TCGEN05 = 3, /* decode kernel, M <= 8, 2/4/8-bit codes, on tcgen05 integer MMAs (codes
                                unpacked into tensor memory); K a multiple of 256 (128 at G = 32); other
                                shapes run AQ_KERNEL_QMV */
  AQ_KERNEL_QMM_NOWS = 4 /* tcgen05 tensor-core kernel, any M, without workspace: activations converted to
                            fp16 on chip (slower than AQ_KERNEL_QMM; for callers that cannot allocate) */
} aq_kernel;

/* Words of the packed code array: N*K*bits/32 (0 if the arguments are invalid). */
size_t aq_packed_words(int64_t N, int64_t K, int bits);

/* Bytes of codes + scales + biases: N*K*bits/8 + 4*N*K/G (0 if invalid).
 * At bits=4, G=64 this is 4.5 bits per weight ("Quantizing a Model for MLX",
 * section "What MLX quantization stores"). */
size_t aq_packed_bytes(int64_t N, int64_t K, int G, int bits);

/* Quantize fp32 W[N,K] into packed codes, fp16 scales and fp16 biases.
 * Source: metalworking "MLX Quantization", section "Mechanics" (mx.quantize);
 * "Quantizing a Model for MLX", section "What MLX quantization stores".
 * Results are bit-exact with the definition in this header. */
aq_status aq_quantize(const float *w, int64_t N, int64_t K, int G, int bits,
                      uint32_t *packed, uint16_t *scales, uint16_t *biases, aq_stream_t stream);

/* Range-search quantize: the same outputs, format and arguments as aq_quantize,
 * with each group's grid chosen by a search over shrunk ranges.
 * Source: "mlx-gptq" page, section "How it works" (--mse: a group's min-max
 * range is shrunk when clipping its extremes costs less error than the coarser
 * step costs the rest of the group; the pages give no grid, so these readings):
 *  - candidates p = k/32, k = 32 down to 1; candidate p spans
 *    [lo, hi] = [fp32(p*min), fp32(p*max)] (a zero bound is +0.0) and gets the
 *    plain grid of that range: scale16 = fp16(fp32(hi - lo)/(2^bits - 1)),
 *    bias16 = fp16(lo), codes clamp(rint_even((w - bias16)/scale16)), so values
 *    outside [lo, hi] are clipped to the end codes; p = 1 is aq_quantize's grid;
 *  - a candidate's error is the fp32 sum of e*e, e = fp32(w - fp32(q*scale16 +
 *    bias16)), summed from zero in element order within each run of 32
 *    elements, the runs' sums then added pairwise ((r0+r1)+(r2+r3) for G=128);
 *  - the least error wins; equal errors keep the larger p.
 * The result is bit-exact with that definition.  The squared error of the
 * chosen grid is never above aq_quantize's (up to fp32 summation rounding).
 * Cost: 32 candidate grids per group, ALU-bound (one-off, offline). */
aq_status aq_quantize_mse(const float *w, int64_t N, int64_t K, int G, int bits,
                          uint32_t *packed, uint16_t *scales, uint16_t *biases, aq_stream_t stream);

/* Dequantize to bf16: w_out[n,k] = bf16_rn(fp32_rn(code*scale + bias)) (a single
 * fp32 rounding of the exact value, then RNE to bf16).
 * Source: anllm "Tutorial 10: Quantization", sections 3 and 7 (dequantize, then
 * astype(bfloat16)). */
aq_status aq_dequantize(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                        int64_t N, int64_t K, int G, int bits, uint16_t *w_out_bf16, aq_stream_t stream);

/* Same as aq_dequantize with fp32 output fp32_rn(code*scale + bias). */
aq_status aq_dequantize_f32(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                            int64_t N, int64_t K, int G, int bits, float *w_out, aq_stream_t stream);

/* Quantized matmul y[M,N] = x[M,K] @ dequant(W)^T, bf16 (RNE) output, without
 * materialising dequant(W) in global memory.
 * Source: anllm "Tutorial 10: Quantization", section 5, approach 2
 * (mx.quantized_matmul(..., transpose=True)); metalworking "MLX Quantization",
 * section "Mechanics" (QMV for decode, QMM for prefill, host-side per-shape
 * dispatch).  Accuracy: |y - y_ref| <= 8e-3 * (|y_ref| + rms(y_ref)) against the
 * exact product.  Kernels:
 *  - QMV for M <= 8.  2/4/8-bit codes with K a multiple of 8*G: integer tensor
 *    cores on the exact codes; each group's activations enter as 16-bit fixed
 *    point, rint(x * 2^e) with 2^e the power of two that puts the group's
 *    largest |x| in [2^13, 2^14) (error <= 2^-14 of that largest |x| per
 *    element); group dot products exact in int32, then
 *    y += scale * 2^-e * dot + bias * sum(x) in fp32.  Where the staged
 *    activations of all M tokens would take more than 120 KB of shared memory
 *    ((2K + 64) bytes per token: M > 4 at K = 14336), the tokens run as
 *    balanced chunks, one launch each, in stream order.  Other shapes and 3-bit
 *    codes: CUDA cores, fp32 arithmetic on the exact codes.
 *  - QMM otherwise: tcgen05 tensor cores on fp16 operands, weights
 *    fp16_rn(fp32_rn(code*scale + bias)), activations scaled per row by an
 *    exact power of two into fp16, fp32 accumulation. */
aq_status aq_matmul(const uint16_t *x_bf16, int64_t M, int64_t K,
                    const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                    int64_t N, int G, int bits, uint16_t *y_bf16, aq_stream_t stream);

/* Flags of aq_matmul_ex. */
enum {
  /* Launch the decode kernel as a programmatic dependent of the kernel before it
   * in `stream`, so its start overlaps that kernel's tail: it reads x only after
   * the previous kernel has completed (its writes visible), but it reads the
   * packed codes, scales and biases before.  The caller guarantees that no kernel
   * still running in the stream writes those three arrays.  Honoured by the
   * tensor-core QMV; other kernels launch as usual. */
  AQ_MATMUL_OVERLAP_PREVIOUS = 1u
};

/* aq_matmul with flags (a bitwise OR of the AQ_MATMUL_* values; unknown bits ->
 * AQ_ERR_INVALID_ARG).  Same results as aq_matmul, bit for bit. */
aq_status aq_matmul_ex(const uint16_t *x_bf16, int64_t M, int64_t K,
                       const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                       int64_t N, int G, int bits, uint16_t *y_bf16, uint32_t flags, aq_stream_t stream);

/* One matmul of aq_matmul_sequence: y [M, N] = x [M, K] . dequant(W)^T with W
 * given as packed [N, K*bits/32], scales and biases [N, K/G] (the layouts of
 * aq_matmul).  Device pointers, 16-byte aligned. */
typedef struct {
  const uint16_t *x_bf16;
  const uint32_t *packed;
  const uint16_t *scales;
  const uint16_t *biases;
  uint16_t *y_bf16;
  int64_t N;
  int64_t K;
} aq_matmul_desc;

/* Decode matmuls of one step in a single launch ("MLX Quantization",
 * "Mechanics": QMV streams each weight once per decode step; several linears
 * run back to back).  Computes calls[j] for j = 0 .. n-1 (1 <= n <= 4) in
 * order, all with the same M (1..8), G and bits (2, 4 or 8), each with its own
 * N and K, with the accuracy of aq_matmul's tensor-core QMV (each K chunk's
 * sums are one work unit here, where aq_matmul may split a chunk in two, so
 * the two may differ in the last bit of y).
 * Ordering: matmul j reads its x only after every element of matmul j-1's y is
 * written, so calls[j].x_bf16 may be calls[j-1].y_bf16 (a chain of linears);
 * the weights of matmul j stream while matmul j-1 finishes.  No other
 * overlap between one call's y and any call's inputs is allowed.
 * The launch places one CTA on each SM and synchronises them between the
 * matmuls; it needs every one of its CTAs resident at once, so it must not
 * share the GPU with kernels that hold SMs for long (a barrier wait that runs
 * out sets a bit of aq_device_fault and the results are undefined).
 * flags: 0 or AQ_MATMUL_OVERLAP_PREVIOUS (the first matmul's weights may be
 * read before the previous kernel in the stream completes).
 * Errors: n outside 1..4, a null pointer, unknown flags -> AQ_ERR_INVALID_ARG;
 * M > 8, bits not 2/4/8, G not 32/64/128, or a shape the decode kernel does not
 * take (K a multiple of 8*G, N >= 16) -> AQ_ERR_UNSUPPORTED; unaligned
 * pointers -> AQ_ERR_ALIGNMENT.  Asynchronous on `stream`; allocates nothing. */
aq_status aq_matmul_sequence(const aq_matmul_desc *calls, int n, int64_t M, int G, int bits, uint32_t flags,
                             aq_stream_t stream);

/* Bytes of workspace aq_matmul_ws needs for this shape (0 when the dispatched
 * kernel needs none, or when the arguments would be rejected).  Host only.
 * For AQ_KERNEL_QMM: the fp16 activations (2*M*K bytes) and their row scales
 * (4*M), each rounded up to 256.  When M > 128 and N % 8 == 0 the product runs
 * in T = ceil(M/256)*ceil(N/256) tiles on up to 74 CTA pairs; when T <= 37,
 * each tile's K range is cut into ks = min(74 / T, 4, KB / 32) parts (KB: K
 * blocks of 64, or 128 for 3-bit codes; split when ks >= 2), which adds T*24
 * uint32 arrival counters (rounded up to 256) and ks*T*2*128*256 fp32 partial
 * sums.  The parts are added in a fixed order, so results repeat bit for bit. */
size_t aq_matmul_workspace_bytes(int64_t M, int64_t N, int64_t K, int G, int bits);

/* aq_matmul with caller-provided workspace: `workspace` is device memory of at
 * least aq_matmul_workspace_bytes(M, N, K, G, bits) bytes, 16-byte aligned,
 * not used by any other call in flight (NULL is allowed when that size is 0).
 * Too small or NULL when needed -> AQ_ERR_INVALID_ARG. */
aq_status aq_matmul_ws(const uint16_t *x_bf16, int64_t M, int64_t K,
                       const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                       int64_t N, int G, int bits, uint16_t *y_bf16, void *workspace, size_t workspace_bytes,
                       aq_stream_t stream);

/* Size of the fixed device workspace behind aq_matmul_qmm_static: 80 MiB.  A
 * call needs 2*M*K + 4*M bytes (each term rounded up to 256; the fp16
 * activations and their row scales), so for example M = 8192 with K = 4096, or
 * M = 2048 with K = 14336, fit.  A shape with a K split (aq_matmul_workspace_bytes)
 * runs it when the whole of that workspace fits, and unsplit otherwise (same
 * results within the tolerance). */
#define AQ_QMM_STATIC_WORKSPACE_BYTES (80u * 1024u * 1024u)

/* The tensor-core matmul (AQ_KERNEL_QMM) without any allocation: its workspace
 * is a fixed device array compiled into this library (every GPU that loads the
 * library holds AQ_QMM_STATIC_WORKSPACE_BYTES of it until the process exits)
 * instead of cudaMallocAsync or caller memory.  No counterpart on the pages: it
 * exists for callers that cannot allocate device memory at call time, e.g. work
 * captured into graphs whose launch path rejects memory-allocation nodes, or
 * runtimes that reserve the whole device up front and forbid later cudaMalloc.
 * Same arguments, layouts and result as aq_matmul_with(AQ_KERNEL_QMM, ...).
 * Errors: shapes whose activations' workspace (2*M*K + 4*M bytes, as above)
 * exceeds AQ_QMM_STATIC_WORKSPACE_BYTES -> AQ_ERR_UNSUPPORTED, checked before
 * anything is launched; otherwise as aq_matmul_with.
 * The first call on each device looks up the array's device address (which may
 * load the module), and so does the first call after that device's context has
 * been recreated (cudaDeviceReset): make such a call before any stream capture.
 * Every call shares the one array per device, so calls that can overlap on the
 * GPU (different streams, or graphs replayed concurrently) race on it; serialize
 * them.  The array keeps the last call's contents; nothing in it needs to start
 * at zero (each call writes all of it that it reads). */
aq_status aq_matmul_qmm_static(const uint16_t *x_bf16, int64_t M, int64_t K,
                               const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                               int64_t N, int G, int bits, uint16_t *y_bf16, aq_stream_t stream);

/* aq_matmul with an explicit kernel.  AQ_KERNEL_QMV and AQ_KERNEL_QMV_TCGEN05
 * return AQ_ERR_UNSUPPORTED when M > 8 or the shared-memory staging of x does
 * not fit, even in token chunks; AQ_KERNEL_QMM and AQ_KERNEL_QMM_NOWS return AQ_ERR_UNSUPPORTED when
 * K*bits is not a multiple of 128.  AQ_KERNEL_QMM takes its workspace from
 * the library's stream-ordered pool (see Ownership above); AQ_KERNEL_QMM_NOWS
 * allocates nothing (each token row's power-of-two scale is kept, until the
 * epilogue overwrites it, in bytes of y's own output tile). */
aq_status aq_matmul_with(aq_kernel kernel, const uint16_t *x_bf16, int64_t M, int64_t K,
                         const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                         int64_t N, int G, int bits, uint16_t *y_bf16, aq_stream_t stream);

/* The kernel aq_matmul would run for this shape (host logic only; no GPU needed),
 * or -1 if the arguments would be rejected. */
int aq_dispatch(int64_t M, int64_t N, int64_t K, int G, int bits);

/* Human-readable name of a status code (static storage). */
const char *aq_status_string(aq_status status);

/* The last CUDA error code seen by this library on the calling thread (0 if none). */
int aq_last_cuda_error(void);

/* Quantized embedding lookup: out[t, :] = bf16_rn(fp32_rn(code*scale + bias))
 * of row ids[t] of the packed table [V, D] (the row aq_dequantize would give).
 * ids: device int32 [T] (4-byte aligned); packed/scales/biases as produced by
 * aq_quantize on a [V, D] table and out, device bf16 [T, D], 16-byte aligned.
 * D % G == 0.  T, V, D <= 0 or a null pointer -> AQ_ERR_INVALID_ARG.  An id
 * outside [0, V) gives a zero row and sets bit 5 (AQ_FAULT_BAD_INDEX) of the
 * device fault word.
 * Source: anllm "Tutorial 10: Quantization", section 6 "Quantized
 * Embeddings"; ExecuTorch "MLX backend — Quantization" (quantized embedding
 * layers, G = 32 or 128). */
aq_status aq_embedding(const int32_t *ids, int64_t T, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t V, int64_t D, int G, int bits, uint16_t *out_bf16,
                       aq_stream_t stream);

/* Gather matmul for mixture-of-experts layers: for each token t,
 * y[t, :] = x[t, :] @ dequant(W[experts[t]])^T, where W holds E experts of
 * shape [N, K] stacked along the rows (packed [E, N, K*bits/32], scales and
 * biases [E, N, K/G], each expert as aq_quantize produces it).  experts is a
 * device int32 [T] (4-byte aligned); x bf16 [T, K] and y bf16 [T, N] on the
 * device.  Each token streams its expert's weights (tokens sharing an expert
 * read it again).  Shapes: bits in {2, 4, 8}, K a multiple of 8*G, N >= 16
 * (others -> AQ_ERR_UNSUPPORTED); E*N < 2^31.  An expert id outside [0, E)
 * gives a zero output row and sets AQ_FAULT_BAD_INDEX in the device fault word.
 * Accuracy as aq_matmul.  Source: metalworking "MLX Quantization", the kernel
 * family list ("gather variants for MoE experts"). */
aq_status aq_gather_matmul(const uint16_t *x_bf16, int64_t T, int64_t K, const uint32_t *packed,
                           const uint16_t *scales, const uint16_t *biases, int64_t E, int64_t N, int G, int bits,
                           const int32_t *experts, uint16_t *y_bf16, aq_stream_t stream);

/* Prefill form of aq_gather_matmul: the same result (y[t, :] = x[t, :] @
 * dequant(W[experts[t]])^T, a zero row and AQ_FAULT_BAD_INDEX for an id outside
 * [0, E)), computed by grouping the tokens by expert so that each expert's
 * weights are multiplied once against all of its tokens: a routing kernel
 * orders the tokens by expert, x rows are gathered into that order, and the
 * rows are scattered back after the matmul.  With E <= 256 and K*bits a
 * multiple of 128 the matmul is ONE tensor-core launch over every expert's
 * segment, whose tile count the kernel reads from the device-side segment
 * offsets (on CTA pairs with 256-token tiles when the segments average more
 * than 192 rows, else on single CTAs): the call is asynchronous and can be
 * captured in a CUDA graph.
 * Otherwise each expert's rows go through aq_matmul's per-shape kernels; the
 * host then reads the E per-expert counts once, so the call synchronizes its
 * stream (and cannot be captured).  Workspace (offsets, positions, x and y in expert order, the QMM
 * workspace) comes from the library's stream-ordered pool.  Shapes: as aq_matmul for
 * every segment size, N a multiple of 8, each expert's packed/scale/bias block a
 * multiple of 16 bytes, E <= 16384 (others -> AQ_ERR_UNSUPPORTED or
 * AQ_ERR_INVALID_ARG).  Accuracy as aq_matmul.  Source: metalworking "MLX
 * Quantization", the kernel family list ("gather variants for MoE experts"). */
aq_status aq_gather_matmul_grouped(const uint16_t *x_bf16, int64_t T, int64_t K, const uint32_t *packed,
                                   const uint16_t *scales, const uint16_t *biases, int64_t E, int64_t N, int G,
                                   int bits, const int32_t *experts, uint16_t *y_bf16, aq_stream_t stream);

/* ---- mxfp4: block-scaled fp4 ------------------------------------------------
 * Source: metalworking "MLX Quantization" (the newer block-scaled float modes:
 * mxfp4 with groups of 32) and "Quantizing a Model for MLX", section "Modes,
 * bits and mixed recipes" (mxfp4: 4 bits, groups of 32, an exponent per group
 * rather than a scale and a bias).  The pages leave the encodings open; these
 * follow the OCP Microscaling v1.0 formats:
 *  - packed: uint32 [N, K/8], E2M1 code k of a row at bits 4k..4k+3 (LSB
 *    first); code bit 3 = sign, bits 2..1 = exponent, bit 0 = mantissa, so codes
 *    0..7 are the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
 *  - scales: uint8 [N, K/32], E8M0: byte s means X = 2^(s - 127) (255 = NaN);
 *  - w ~= X * e2m1(code), no bias.
 * Quantize, per 32 consecutive weights of a row: shared exponent
 * floor(log2 max|w|) - 2, clamped to [-127, 127], s = shared + 127 (an all-zero
 * group: s = 0); each code is the E2M1 magnitude nearest to |w| / X, ties to the
 * even code, saturating at 6, with the sign bit only on a non-zero magnitude.
 * Results are bit-exact with that definition.  Dequantized values are exact in
 * fp32 and bf16.  K must be a multiple of 32 (else AQ_ERR_INVALID_ARG); every
 * pointer 16-byte aligned (AQ_ERR_ALIGNMENT).  Inputs must be finite. */

/* Bytes of codes + scales: N*K/2 + N*K/32 (4.25 bits per weight); 0 if invalid. */
size_t aq_mxfp4_packed_bytes(int64_t N, int64_t K);

/* Quantize fp32 W[N, K] (device) into packed codes and E8M0 scales (device,
 * caller-allocated). */
aq_status aq_mxfp4_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                            aq_stream_t stream);

/* Dequantize to bf16 [N, K] (exact). */
aq_status aq_mxfp4_dequantize(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K,
                              uint16_t *w_out_bf16, aq_stream_t stream);

/* Dequantize to fp32 [N, K] (exact). */
aq_status aq_mxfp4_dequantize_f32(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K,
                                  float *w_out, aq_stream_t stream);

/* y[M, N] = x[M, K] @ dequant(W)^T (bf16 in and out, device).  Decode,
 * M <= 8, on the integer tensor cores: each code becomes the signed byte
 * 2 * e2m1(code), the activations enter as 16-bit fixed point per group (as in
 * aq_matmul's decode kernel) and the fold applies X / 2.  Supported shapes:
 * M <= 8, N >= 16, K a multiple of 512 (others -> AQ_ERR_UNSUPPORTED).  flags:
 * 0 or AQ_MATMUL_OVERLAP_PREVIOUS, as for aq_matmul_ex.  Accuracy as aq_matmul,
 * provided X / 2 times the activations' per-group power of two stays within
 * the fp32 range (true unless both the weights' scale and the activations are
 * within a few octaves of the fp32 limits).
 * Prefill, M > 8: the tensor-core matmul of aq_matmul (tcgen05, fp16
 * operands, fp32 accumulation): the codes are dequantized to fp16 on chip,
 * each W row scaled by a power of two 2^-B chosen from its largest block scale
 * so that every value of a group within 2^22 of that scale is exact (the
 * epilogue multiplies by 2^B); smaller groups round as fp16 subnormals, below
 * the matmul tolerance.  The activations' fp16 workspace comes from the
 * library's pool; flags are then ignored. */
aq_status aq_mxfp4_matmul(const uint16_t *x_bf16, int64_t M, int64_t K, const uint32_t *packed,
                          const uint8_t *scales, int64_t N, uint16_t *y_bf16, uint32_t flags, aq_stream_t stream);

/* ---- mxfp8: block-scaled fp8 ------------------------------------------------
 * Source: metalworking "MLX Quantization" (the newer modes: mxfp8 with groups of
 * 32) and "Quantizing a Model for MLX", section "Modes, bits and mixed recipes"
 * (mxfp8: 8 bits, groups of 32, an exponent per group).  Encodings as read from
 * the OCP Microscaling v1.0 MXFP8 (E4M3) format:
 *  - packed: uint32 [N, K/4], code k of a row in byte k (LSB first); code = sign
 *    bit 7 + E4M3 magnitude (exponent bits 6..3 with bias 7, mantissa bits
 *    2..0, subnormals m * 2^-9, largest 448);
 *  - scales: uint8 [N, K/32], E8M0 as for mxfp4 (X = 2^(s - 127)).
 * Quantize: shared exponent floor(log2 max|w|) - 8, clamped to [-127, 127] (an
 * all-zero group: s = 0); element = E4M3 magnitude nearest to |w| / X, ties to
 * even, saturating at 448; sign only on a non-zero magnitude.  Bit-exact with
 * that definition.  Dequantized value: X * e4m3(code) rounded once to fp32 (then
 * bf16 RNE).  K a multiple of 32; pointers 16-byte aligned. */

/* Bytes of codes + scales: N*K + N*K/32; 0 if invalid. */
size_t aq_mxfp8_packed_bytes(int64_t N, int64_t K);

aq_status aq_mxfp8_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                            aq_stream_t stream);
aq_status aq_mxfp8_dequantize(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K,
                              uint16_t *w_out_bf16, aq_stream_t stream);
aq_status aq_mxfp8_dequantize_f32(const uint32_t *packed, const uint8_t *scales, int64_t N, int64_t K,
                                  float *w_out, aq_stream_t stream);

/* y[M, N] = x[M, K] @ dequant(W)^T (bf16, device).  Decode, M <= 8: E4M3
 * codes do not fit the integer MMA: each pair is widened to fp16x2 (exact) and
 * multiplied on the tensor cores (mma.sync m16n8k16, fp32 accumulate) against
 * the activations staged as fp16 x * 2^e per group (exact for |x| above 2^-14
 * of the group's largest); the fold applies X * 2^-e.  Supported: M <= 8,
 * N >= 16, K a multiple of 512 (others -> AQ_ERR_UNSUPPORTED).  flags: 0 or
 * AQ_MATMUL_OVERLAP_PREVIOUS.  Accuracy as aq_matmul.
 * Prefill, M > 8: the tensor-core matmul of aq_matmul (tcgen05, fp16
 * operands, fp32 accumulation): the codes are dequantized to fp16 on chip,
 * each W row scaled by a power of two 2^-B chosen from its largest block scale
 * so that every value of a group within 2^22 of that scale is exact (the
 * epilogue multiplies by 2^B); smaller groups round as fp16 subnormals, below
 * the matmul tolerance.  The activations' fp16 workspace comes from the
 * library's pool; flags are then ignored. */
aq_status aq_mxfp8_matmul(const uint16_t *x_bf16, int64_t M, int64_t K, const uint32_t *packed,
                          const uint8_t *scales, int64_t N, uint16_t *y_bf16, uint32_t flags, aq_stream_t stream);

/* ---- nvfp4: fp4 with E4M3 block scales and a tensor scale ------------------
 * Source: ExecuTorch "MLX backend — Quantization" (the NVFP4 weight-only
 * config, group size 16) and "Quantizing a Model for MLX", section "Modes, bits
 * and mixed recipes" (nvfp4: groups of 16, 4 bits).  The pages leave the
 * encodings open; these follow NVIDIA's NVFP4 format:
 *  - packed: uint32 [N, K/8], E2M1 codes as for mxfp4;
 *  - scales: uint8 [N, K/16], E4M3 (sign 0, exponent bits 6..3 with bias 7,
 *    mantissa bits 2..0, subnormals m * 2^-9, largest 448);
 *  - tensor_scale: one device fp32 g;
 *  - w ~= e2m1(code) * scale * g.
 * Quantize: g = fp32(max|w| / 2688) over the whole tensor (1 if it is all
 * zero); block byte = E4M3 nearest to fp32(amax_block / fp32(6 * g)), ties to
 * even, saturating at 448; element = E2M1 nearest to fp32(|w| / fp32(scale *
 * g)), ties to the even code, sign only on a non-zero magnitude; a zero block
 * scale gives code 0.  Bit-exact with that definition.  Dequantized value:
 * fp32(fp32(e2m1 * scale) * g).  K must be a multiple of 32; packed, scales and
 * outputs 16-byte aligned, tensor_scale 4-byte aligned.  Inputs must be finite. */

/* Bytes of codes + scales + tensor scale: N*K/2 + N*K/16 + 4; 0 if invalid. */
size_t aq_nvfp4_packed_bytes(int64_t N, int64_t K);

/* Quantize fp32 W[N, K] (device); writes packed, scales and *tensor_scale (device). */
aq_status aq_nvfp4_quantize(const float *w, int64_t N, int64_t K, uint32_t *packed, uint8_t *scales,
                            float *tensor_scale, aq_stream_t stream);

/* Dequantize to bf16 (RNE of the fp32 value) or fp32 [N, K]. */
aq_status aq_nvfp4_dequantize(const uint32_t *packed, const uint8_t *scales, const float *tensor_scale, int64_t N,
                              int64_t K, uint16_t *w_out_bf16, aq_stream_t stream);
aq_status aq_nvfp4_dequantize_f32(const uint32_t *packed, const uint8_t *scales, const float *tensor_scale,
                                  int64_t N, int64_t K, float *w_out, aq_stream_t stream);

/* y[M, N] = x[M, K] @ dequant(W)^T (bf16, device).  Decode, M <= 8, on the
 * integer tensor cores: one MMA K step spans two 16-weight groups, whose halves
 * feed two accumulator columns; each column is folded with its E4M3 scale and
 * the output multiplied by g.  One launch holds up to 4 tokens; M = 5..8 runs as
 * two launches (rows 0..3, then the rest), reading the weights twice.
 * Supported: M <= 8, N >= 16, K a multiple of 256 (others ->
 * AQ_ERR_UNSUPPORTED).  flags: 0 or AQ_MATMUL_OVERLAP_PREVIOUS (both launches).
 * Accuracy as aq_matmul.
 * Prefill, M > 8: the tensor-core matmul of aq_matmul (tcgen05, fp16
 * operands, fp32 accumulation): the codes are dequantized to fp16 on chip,
 * each W row scaled by a power of two 2^-B chosen from its largest block scale
 * so that every value of a group within 2^22 of that scale is exact (the
 * epilogue multiplies by 2^B); smaller groups round as fp16 subnormals, below
 * the matmul tolerance.  The activations' fp16 workspace comes from the
 * library's pool; flags are then ignored.  The tensor scale g multiplies every output. */
aq_status aq_nvfp4_matmul(const uint16_t *x_bf16, int64_t M, int64_t K, const uint32_t *packed,
                          const uint8_t *scales, const float *tensor_scale, int64_t N, uint16_t *y_bf16,
                          uint32_t flags, aq_stream_t stream);

/* Bits of the device fault word. */
enum {
  AQ_FAULT_WAIT_MASK = 0x1Fu, /* bits 0-4: a kernel gave up a bounded wait and returned early */
  AQ_FAULT_BAD_INDEX = 0x20u  /* an embedding id or an expert id was out of range */
};

/* Limit, in SM clock cycles, of every bounded wait of the decode kernel (the
 * tensor-core QMV behind aq_matmul for M <= 8, the gather matmul and the
 * block-scaled decode matmuls) in launches made after this call, from any
 * thread; cycles <= 0 restores the default of 2e9 cycles (about one second).
 * No counterpart on the pages: it exists to test the timeout path.  A wait that
 * runs out sets a bit of AQ_FAULT_WAIT_MASK in the device fault word, the
 * kernel stops issuing work, waits for its own copies in flight and returns;
 * that call's output is then invalid.  A limit far below the time a copy from
 * HBM takes (a few thousand cycles) makes the waits run out on purpose. */
void aq_set_wait_limit(int64_t cycles);

/* on != 0: every decode-kernel launch made afterwards (from any thread) also
 * waits, after staging its activations, on a barrier that nothing completes,
 * so that this bounded wait runs out (after aq_set_wait_limit's limit): the
 * launch sets its fault bit, issues no more work, waits for its own copies in
 * flight and returns, its output invalid.  on = 0 restores normal launches.
 * No counterpart on the pages: it exists to test the timeout path. */
void aq_set_wait_stall(int on);

/* Reads and clears the device-side fault word of the current device: non-zero
 * when a kernel gave up a bounded wait (an mbarrier that never completed) and
 * returned early, its output then invalid (bits 0-4), or when an embedding id
 * or an expert id was out of range (bit 5).  Synchronizes the device. */
aq_status aq_device_fault(uint32_t *fault_word);

#ifdef __cplusplus
}
#endif

#endif /* AQ_H_ */
