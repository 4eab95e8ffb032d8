/*
 * mx.h -- C ABI of libmx.so: microscaling quantization (MXFP8 E4M3/E5M2, MXFP6
 * E3M2, MXFP4, NVFP4) and the block-scaled matrix multiply that consumes it, on
 * one NVIDIA B200 (sm_100a).
 *
 * Sources for what each call computes (page title, section):
 *   [MX]    "Microscaling MXFP4/NVFP4 on Blackwell for reasoning LLMs"
 *           (produtoramaxvision.com.br), sections "Fundamentos matemáticos do
 *           formato MXFP4 e E8M0" (E2M1 values, E8M0 = 2^(E-127), x = S * x_elem,
 *           4.25 bits/element, E4M3 range [-448, 448], the format table's
 *           MXFP6 = E3M2 with an E8M0 scale per 32, 6.25 bits), "Arquitetura Blackwell
 *           SM100 e aceleração nativa de NVFP4" (the tensor core applies the
 *           block scales during FP32 accumulation) and the FAQ entry on how E8M0
 *           picks the block exponent (E = ceil(log2(max|x| / max_elem)) + 127).
 *   [NEWS]  "NVIDIA's FP4 format delivers 1.68x speedup" (zubnet.ai): NVFP4 is
 *           E2M1 in 16-element blocks; MXFP8 is E4M3/E5M2 in 32-element blocks.
 *   [IMPL]  "Implementação da quantização NVFP4 e MXFP8" (matsubara.tec.br):
 *           Linear layers with both operands quantized, the quantize kernel as a
 *           bottleneck for small tensors, CUDA Graphs for batch-1 launches.
 *   [OAS]   "Unveiling the Potential of Quantization with MXFP4: Strategies for
 *           Quantization Error Reduction" (gist.science), section 2.A
 *           (overflow-aware scaling) and sections 3-4 (QSNR as the fidelity
 *           measure).
 *
 * Conventions for every call:
 *   - Device pointers are plain CUDA device addresses; the caller allocates and
 *     owns every buffer.  The library allocates nothing.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Nothing blocks the host except mx_check_device_error.
 *   - Errors are returned as mx_status; nothing throws across the ABI.
 *     Argument errors are detected on the host before any launch.  Faults the
 *     GPU detects (a bounded wait that ran out, a bounds check) are recorded in
 *     a per-process device error word read by mx_check_device_error.
 *   - All device pointers must be 16-byte aligned (TMA and vector accesses).
 *   - Matrices are row-major; the reduction dimension K is contiguous.
 */
#ifndef MX_H_
#define MX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element formats.  Block size 32 with an E8M0 scale for the four MX formats;
 * block size 16 with an E4M3 scale plus one FP32 per-tensor scale for NVFP4;
 * MXFP4_MBS ([OAS] section B, macro block scaling): E2M1 in blocks of 16 with
 * E8M0 scales, plus one byte m per 128 elements (a factor 1 + m/256 on the
 * whole macro block), m from the block maximum (mx_quantize, the static
 * variant) or by error search (mx_quantize_mbs_dynamic).  mx_gemm multiplies
 * two MXFP4_MBS operands: the tensor core sums each macro block's products
 * with the base-block scales, and the macro factors are applied to that
 * partial sum on the CUDA cores.
 * E3M2 ([MX] format table, MXFP6): sign, 3 exponent bits with bias 3, 2
 * mantissa bits, no infinities or NaN, largest magnitude 28. */
typedef enum {
    MX_MXFP8_E4M3 = 0,
    MX_MXFP8_E5M2 = 1,
    MX_MXFP4 = 2,
    MX_NVFP4 = 3,
    MX_MXFP6_E3M2 = 4,
    MX_MXFP4_MBS = 5
} mx_format;

typedef enum {
    MX_OK = 0,
    MX_ERR_INVALID_ARG = 1,       /* NULL pointer, bad enum, negative size, ... */
    MX_ERR_UNSUPPORTED_SHAPE = 2, /* K not a multiple of what the call needs    */
    MX_ERR_MISALIGNED = 3,        /* pointer or leading dimension not 16-B aligned */
    MX_ERR_CUDA = 4,              /* a CUDA runtime call failed (launch, ...)   */
    MX_ERR_TIMEOUT = 5,           /* a bounded device-side wait ran out         */
    MX_ERR_DEVICE = 6             /* a device-side bounds/consistency check hit */
} mx_status;

/* A quantized [rows x cols] matrix (cols = K, the blocked dimension).
 *   codes : device, mx_codes_bytes(fmt, rows, cols) bytes.  FP8: one code per
 *           byte, row-major.  FP4: two codes per byte, byte j of a row holds
 *           code 2j in its low nibble and code 2j+1 in its high nibble.  FP6:
 *           code k of a row occupies bits 6k .. 6k+5 of the row read as a
 *           little-endian bit string (16 codes in 12 bytes; a row is 3K/4
 *           bytes).
 *   scales: device, mx_scales_bytes(fmt, rows, cols) bytes.  One scale byte per
 *           block (E8M0 for MX, E4M3 for NVFP4), laid out in 512-byte tiles of
 *           128 rows x 4 scale columns: scale (r, c) of a matrix with C scale
 *           columns is at ((r/128)*ceil(C/4) + c/4)*512 + (r%32)*16
 *           + ((r%128)/32)*4 + c%4 -- the layout the sm_100 tensor core reads.
 *           Padding bytes (rows >= rows, columns >= C) are 0.  MXFP4_MBS
 *           appends its macro bytes, [rows][cols/128] row-major, zero-padded to
 *           a multiple of 16 bytes, after the tiles.
 *   gscale: device, one float (NVFP4 only; NULL otherwise): the per-tensor
 *           decode multiplier g.  Real value = g * scale * element.           */
typedef struct {
    int32_t fmt;
    int32_t reserved;
    int64_t rows;
    int64_t cols;
    void *codes;
    uint8_t *scales;
    float *gscale;
} mx_tensor;

/* Sizes in bytes of the two buffers of an mx_tensor.  0 for a bad format. */
size_t mx_codes_bytes(int fmt, int64_t rows, int64_t cols);
size_t mx_scales_bytes(int fmt, int64_t rows, int64_t cols);
/* Elements per scale block: 32 (MX formats) or 16 (NVFP4); 0 for a bad format. */
int mx_block_size(int fmt);

/* Quantize a bf16 matrix src [M x K] (row pitch ld_src elements, ld_src >= K,
 * ld_src % 8 == 0) into dst ([MX] "Fundamentos" and FAQ; [NEWS]; [OAS] B).
 *   MX formats: per block, E = ceil(log2(max|x| / max_elem)) + 127 clamped to
 *     [0, 254] (0 for an all-zero block), elements = RNE(x / 2^(E-127))
 *     saturating to the element format (max_elem = 448 / 57344 / 6 / 28 for
 *     E4M3 / E5M2 / E2M1 / E3M2).
 *   NVFP4: g = the FP32 value *gscale_in if gscale_in != NULL, else
 *     amax(|src|) / 2688 rounded up to FP32 (1.0 for an all-zero tensor),
 *     computed on the device (an extra read of src: a pre-pass, or, for
 *     M*K <= 16384, inside every CTA of the quantize kernel).  g is written to
 *     *dst->gscale.  Block scale s = smallest positive finite E4M3 with
 *     max|x| <= 6*g*s (0 for an all-zero block); element = RNE of the exact
 *     quotient x / (g*s) onto E2M1, saturating at 6.
 *   MXFP4_MBS: per 128 elements, with alpha = max|x| and e = floor(log2(alpha
 *     / 6)), m = the smallest byte with alpha <= 6 (256 + m) 2^(e-8) (0 for a
 *     zero block); per 16 elements E = the smallest exponent with max|x| <=
 *     6 (1 + m/256) 2^(E-127); elements = RNE of the exact quotient
 *     x / ((1 + m/256) 2^(E-127)) onto E2M1, saturating at 6.  K % 128 == 0.
 * Rounding is to nearest, ties to even; a value that rounds to zero keeps its
 * sign.  K must be a multiple of the block size (32, or 16 for NVFP4).
 * dst->rows/cols must equal M/K and dst->fmt must equal fmt.  Non-finite
 * inputs are outside the contract (their block's codes are unspecified). */
mx_status mx_quantize(int fmt, const void *src_bf16, int64_t M, int64_t K, int64_t ld_src,
                      mx_tensor *dst, const float *gscale_in, void *stream);

/* Dequantize: dst[r][k] = RNE_bf16(g * scale * element), computed exactly
 * before the single rounding ([MX] "Fundamentos": x_real = S * x_elem).
 * ld_dst >= cols, ld_dst % 8 == 0. */
mx_status mx_dequantize(const mx_tensor *src, void *dst_bf16, int64_t ld_dst, void *stream);

/* MXFP4 with overflow-aware scaling ([OAS] section 2.A): as mx_quantize(MX_MXFP4, ...) except that each block's scale
 * maps its max |x| into (3.5, 7] instead of (3, 6]:
 *   E = ceil(log2(max|x| / 7)) + 127 clamped to [0, 254],
 * elements = RNE(x / 2^(E-127)) saturating at 6 (so the block maximum may
 * clip to 6 while the rest of the block gets a step half as large).  dst is an
 * ordinary MXFP4 tensor (dst->fmt == MX_MXFP4): mx_dequantize and mx_gemm
 * consume it unchanged.  Same requirements as mx_quantize. */
mx_status mx_quantize_oas(const void *src_bf16, int64_t M, int64_t K, int64_t ld_src, mx_tensor *dst,
                          void *stream);

/* MXFP4 with dynamic macro-block scaling ([OAS] section 2.B, the variant whose
 * macro factor minimises the quantization error): as mx_quantize(MX_MXFP4_MBS,
 * ...) except that each 128-element macro block's mantissa byte m is the one
 * in [0, 255] whose quantization of the block (base-block exponents and
 * elements exactly as for the static variant, given m) has the smallest sum
 * of squared errors sum (x - xhat)^2, the terms added in element order in
 * fp64 (round to nearest); ties go to the smallest m.  dst is an ordinary
 * MXFP4_MBS tensor (dst->fmt == MX_MXFP4_MBS): mx_dequantize, mx_qsnr and
 * mx_gemm consume it unchanged.  K % 128 == 0, M <= 65535; otherwise as
 * mx_quantize.  An exhaustive search: 256 candidates per macro block, a few
 * hundred times the work of the static variant. */
mx_status mx_quantize_mbs_dynamic(const void *src_bf16, int64_t M, int64_t K, int64_t ld_src, mx_tensor *dst,
                                  void *stream);

/* Walsh-Hadamard rotation fused with quantization ([MX] section "Técnicas de
 * preservação de acurácia": Hadamard rotations spread a block's outlier
 * energy over its 32 elements before 4-bit quantization).  Every 32-element
 * block x_b along K is replaced by
 *   y_b = c * (H32 x_b),  H32 the Sylvester-ordered Hadamard matrix
 *   (H1 = [1], H2n = [[Hn, Hn], [Hn, -Hn]]),  c = RN_fp32(1 / sqrt(32)),
 * computed in fp32 as butterflies of half-width 1, 2, 4, 8, 16 in that order
 * (each (a, b) -> (a + b, a - b), rounded), then one product with c; y is then
 * quantized exactly as mx_quantize quantizes its input (NVFP4: g from
 * gscale_in, else RU(max|y| / 2688) from an extra pass over src).  Rotating
 * both GEMM operands this way leaves A * B^T unchanged up to rounding
 * (H32 H32^T = 32 I).  K % 32 == 0; otherwise as mx_quantize.  A block
 * whose butterfly sums overflow fp32 (possible only when its inputs come
 * within a factor 32 of the bf16 maximum) is outside the contract, like a
 * non-finite input. */
mx_status mx_quantize_rht(int fmt, const void *src_bf16, int64_t M, int64_t K, int64_t ld_src, mx_tensor *dst,
                          const float *gscale_in, void *stream);

/* Quantization SNR inputs ([OAS] sections 3-4 report fidelity as QSNR):
 * sums[0] = sum x^2 and sums[1] = sum (x - xhat)^2 over the bf16 source
 * src [rows x cols] (pitch ld_src, ld_src % 8 == 0) and xhat = the
 * dequantized value of q, accumulated in fp64 on the device; QSNR in dB is
 * 10 log10(sums[0] / sums[1]).  sums: device pointer to 2 doubles (8-byte
 * aligned), zeroed and then written by the call on `stream`; the summation
 * order is unspecified (results agree with an fp64 reference to ~1e-12
 * relative). */
mx_status mx_qsnr(const mx_tensor *q, const void *src_bf16, int64_t ld_src, double *sums, void *stream);

/* Block-scaled GEMM on the tensor cores ([MX] "Arquitetura Blackwell SM100"):
 *   C[i][j] = RNE_bf16( sum_k A_dq[i][k] * B_dq[j][k] ),  A [M x K], B [N x K],
 * A_dq / B_dq the dequantized operands (the scales are applied inside the
 * tensor core during FP32 accumulation; NVFP4 also multiplies by gA * gB in
 * the epilogue).  A->cols == B->cols == K, K % 128 == 0.  Formats: A->fmt ==
 * B->fmt, or any two of the four MX formats (E4M3, E5M2, E3M2, MXFP4 E2M1;
 * all with E8M0 scales on 32-element blocks), which run on kind::mxf8f6f4 at
 * the FP8 rate (MXFP6 x MXFP6 included); such a call needs the codes of an
 * FP6 or FP4 operand 32-byte aligned (else MX_ERR_MISALIGNED).  NVFP4 pairs
 * only with NVFP4.  C is bf16 [M x N] with row pitch ldc (ldc >= N).  Accuracy contract:
 *   |C - C_ref| <= 2^-8 |C_ref| + 1e-4 (|A_dq| |B_dq|^T)  elementwise.       */
mx_status mx_gemm(const mx_tensor *A, const mx_tensor *B, void *C_bf16, int64_t ldc, void *stream);

/* Epilogues of the fused call. */
typedef enum { MX_EPI_NONE = 0, MX_EPI_GELU = 1 } mx_epilogue;

/* Fused activation-quantize + GEMM ([IMPL] section "Implementação da
 * quantização NVFP4 e MXFP8": a Linear layer with both its activations and its
 * weights quantized, and section "Desafios e soluções na implementação": the
 * activation quantize as the bottleneck on small tensors; [MX] FAQ entry on
 * applying microscaling to activations as well as weights).
 * X is bf16 [M x K] (row pitch ldx), W a
 * pre-quantized [N x K] mx_tensor; X is quantized to format fmt, and W's format
 * is fmt or, as in mx_gemm, any MX format that pairs with it (e.g. MXFP8
 * activations with MXFP4 or MXFP6 weights).  X is quantized exactly as
 * mx_quantize would (same codes and scales, bit for bit) once, into the
 * caller's `workspace`, 128-row band by band, and the GEMM's TMA producers
 * load A from a band as soon as its count in the workspace says it is written
 * (by default the quantize kernel writes X while the GEMM kernel, launched to
 * overlap it, starts on the bands already done; MX_DEBUG_FUSED_MODE selects
 * the quantize inside the GEMM kernel instead).  The result is C = X_dq *
 * W_dq^T as in mx_gemm.  X's quantized form is not an output of this call.
 * Launches: a one-thread-block kernel that clears the workspace's counters,
 * the quantize kernel and the GEMM kernel (NVFP4 without x_gscale or x_amax:
 * also the amax pre-pass, except for M*K <= 16384, where the quantize kernel
 * computes amax(|X|) itself).
 *   workspace: device buffer of at least mx_fused_workspace_bytes(fmt, M, K)
 *              bytes, 256-byte aligned; its contents are scratch, and calls
 *              that overlap on the GPU must not share one.  With at least
 *              mx_fused_split_workspace_bytes(fmt, M, K) bytes and no
 *              epilogue function, the GEMM may also split its last wave of
 *              output tiles along K so that every SM has work: when the tile
 *              count leaves more than 15% of the SMs (CTA pairs) without a
 *              tile in the last wave, those tiles' K stages are shared evenly
 *              over all of them, each piece's fp32 partial sum goes to the
 *              workspace, and the worker holding a tile's last stages adds the
 *              others' partial sums to its own, in a fixed order, before the
 *              epilogue.  Results then differ from mx_gemm's only in the fp32
 *              summation order (within the same accuracy contract); they are
 *              the same from call to call for one shape, device and workspace
 *              size.
 *   epilogue : MX_EPI_NONE, or MX_EPI_GELU: the exact-erf form x Phi(x) =
 *              0.5 x erfc(-x / sqrt 2), applied in FP32 before the bf16
 *              rounding, with erfc(z) = t exp(-z^2 + P(t)), t = 1/(1 + z/2),
 *              P a degree-5 polynomial fitted to it (erfc's relative error
 *              below 7.7e-6), and the hardware's approximate reciprocal and
 *              base-2 exponential: within one bf16 ulp of the correctly
 *              rounded GELU.
 *   amax_out : NULL, or a device float that receives max |C| over the bf16
 *              outputs (it is zeroed by this call first).  Feeding it to the
 *              next call's x_amax chains two NVFP4 GEMMs without a host sync.
 *   NVFP4 only, how g of X is found (first non-NULL wins):
 *     x_gscale : device float holding g itself;
 *     x_amax   : device float holding amax(|X|); g = RU_fp32(amax / 2688);
 *     neither  : amax(|X|) is computed on the device: by a pre-pass over X,
 *                or, for M*K <= 16384, by every CTA of the quantize kernel.
 * K % 128 == 0, ldx % 8 == 0. */
mx_status mx_gemm_fused_act(int fmt, const void *X_bf16, int64_t M, int64_t K, int64_t ldx,
                            const mx_tensor *W, void *C_bf16, int64_t ldc, int epilogue,
                            float *amax_out, const float *x_gscale, const float *x_amax,
                            void *workspace, size_t workspace_bytes, void *stream);
/* Workspace bytes mx_gemm_fused_act needs for an [M x K] activation of format
 * fmt (a header of 64 bytes, 4 per 128-row band and 4 per partial-sum slot,
 * rounded up to 256, then X's codes and scales); 0 for a bad format or size. */
size_t mx_fused_workspace_bytes(int fmt, int64_t M, int64_t K);
/* Workspace bytes with which mx_gemm_fused_act may also split its last wave
 * along K: mx_fused_workspace_bytes plus 148 partial-sum slots of 32 KB per
 * 32 rows of min(M, 128) (fp32 sums of 256 columns; 19.4 MB for M > 96); 0
 * for a bad format or size. */
size_t mx_fused_split_workspace_bytes(int fmt, int64_t M, int64_t K);

/* mx_gemm_fused_act without a workspace argument, for callers that cannot
 * allocate device memory: code inside an inference engine's enqueue or plugin
 * callback, where the engine owns all memory and forbids allocation;
 * latency-critical paths that must not pay for cudaMalloc's implicit device
 * synchronization; and runtimes that run under a fixed memory budget.  The
 * pages have no counterpart to this call; it exists for those callers only.
 *   Scratch: a fixed array of MX_NOALLOC_SCRATCH_BYTES inside libmx.so itself,
 *   one per GPU that loads the library, kept until the process exits.  The
 *   call allocates nothing (no cudaMalloc, cudaFree or allocating library
 *   routine).  Shapes whose mx_fused_workspace_bytes(fmt, M, K) exceeds the
 *   array are rejected with MX_ERR_UNSUPPORTED_SHAPE before any launch.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, once per device, with that device current); make
 *   that first call before any stream capture.
 *   The array is smaller than any workspace with room for the K split (the
 *   partial-sum slots alone take 148 x 32 KB), so this call never splits its
 *   tiles along K: a workspace call with a workspace of
 *   MX_NOALLOC_SCRATCH_BYTES bytes gives the same results bit for bit.
 *   Every call uses the same array and leaves its contents behind (whatever
 *   must start at zero is cleared by the call).  Calls that overlap on the GPU
 *   -- on different streams, or from several host threads -- race on it and
 *   must be serialized by the caller.
 * All other arguments, results and errors are those of mx_gemm_fused_act. */
#define MX_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
mx_status mx_gemm_fused_act_noalloc(int fmt, const void *X_bf16, int64_t M, int64_t K, int64_t ldx,
                                    const mx_tensor *W, void *C_bf16, int64_t ldc, int epilogue,
                                    float *amax_out, const float *x_gscale, const float *x_amax,
                                    void *stream);

/* Synchronize `stream`, then read and clear the device error word.  Returns
 * MX_OK, MX_ERR_TIMEOUT (a bounded wait inside a kernel gave up: the kernel
 * returned early and its outputs are unspecified) or MX_ERR_DEVICE.  If info is
 * non-NULL it receives {flags, first site id, first block id, count}. */
mx_status mx_check_device_error(void *stream, uint32_t info[4]);

/* Human-readable name of a status. */
const char *mx_status_string(mx_status s);

/* Library version (major*10000 + minor*100 + patch). */
int mx_version(void);

/* Test hooks (host-side settings read at each launch):
 *   MX_DEBUG_WAIT_LIMIT_NS : limit of every device-side wait (default 1e9 ns).
 *   MX_DEBUG_SKIP_PRODUCER : 1 = GEMM producers skip their loads, so the
 *                            consumers' bounded waits run out (fault test);
 *                            never set in normal use.
 *   MX_DEBUG_PAIR_GEMM     : 1 (default) = GEMMs with M > 128 and N > 128 run
 *                            on CTA pairs (256 x 256 tiles); 0 = single-CTA
 *                            128 x 256 tiles for every shape.
 *   MX_DEBUG_OVERLAP_LAUNCH: 1 (default) = quantize and GEMM kernels are
 *                            launched with programmatic stream serialization:
 *                            their setup (barriers, TMEM, descriptors) overlaps
 *                            the tail of the previous kernel in the stream, and
 *                            they read no input before that kernel completes.
 *                            0 = ordinary stream order.
 *   MX_DEBUG_MAX_GEMM_CTAS : n > 0 = GEMM grids of at most n CTAs (CTA-pair
 *                            grids: at most ceil(n / 2) pairs), so that each
 *                            CTA walks several tiles even on small shapes;
 *                            0 (default) = one CTA per SM.  The result does
 *                            not depend on it (each tile is summed in the
 *                            same order wherever it runs), except where the
 *                            fused call splits tiles along K (the split
 *                            follows the grid).
 *   MX_DEBUG_FUSED_MODE    : how mx_gemm_fused_act runs (same results bit for
 *                            bit in every mode):
 *                            MX_FUSED_PIPELINED (default): the quantize kernel
 *                            counts each 128-row band of X as written, and the
 *                            GEMM kernel, launched to overlap it, loads a band
 *                            of A as soon as its count is complete (an X of at
 *                            most 128 rows, one band, runs as
 *                            MX_FUSED_TWO_KERNELS);
 *                            MX_FUSED_IN_KERNEL: one GEMM kernel whose epilogue
 *                            warps (idle until the first accumulator) quantize
 *                            X band by band before their first tile;
 *                            MX_FUSED_TWO_KERNELS: the quantize kernel, then the
 *                            GEMM kernel after it has completed.
 *   MX_DEBUG_K_SPLIT       : when the fused call splits its last wave along K
 *                            (given the workspace room): MX_K_SPLIT_AUTO
 *                            (default, when the last wave would leave more than
 *                            15% of the workers idle), MX_K_SPLIT_NEVER, or
 *                            MX_K_SPLIT_ALWAYS (whenever the tile count is not
 *                            a multiple of the workers and each worker gets at
 *                            least two K stages).
 * Returns MX_ERR_INVALID_ARG for an unknown key or value. */
typedef enum {
    MX_DEBUG_WAIT_LIMIT_NS = 1,
    MX_DEBUG_SKIP_PRODUCER = 2,
    MX_DEBUG_PAIR_GEMM = 3,
    MX_DEBUG_OVERLAP_LAUNCH = 4,
    MX_DEBUG_MAX_GEMM_CTAS = 5,
    MX_DEBUG_FUSED_MODE = 6,
    MX_DEBUG_K_SPLIT = 7
} mx_debug_key;
/* Values of MX_DEBUG_FUSED_MODE. */
typedef enum {
    MX_FUSED_PIPELINED = 0,
    MX_FUSED_IN_KERNEL = 1,
    MX_FUSED_TWO_KERNELS = 2
} mx_fused_mode;
/* Values of MX_DEBUG_K_SPLIT. */
typedef enum {
    MX_K_SPLIT_AUTO = 0,
    MX_K_SPLIT_NEVER = 1,
    MX_K_SPLIT_ALWAYS = 2
} mx_k_split_mode;
mx_status mx_debug_set(int key, uint64_t value);

/* The GEMM kernels' work schedule, for tests (host only, no GPU needed): the
 * plan for `tiles` output tiles of `kt` K stages each on at most `workers`
 * workers (CTAs, or CTA pairs) under split mode `mode` (mx_k_split_mode, with
 * room for the partial sums), and the work units of worker `worker` in the
 * order it runs them: out[5u .. 5u + 4] = {tile, first K stage, end K stage,
 * kind (0 whole tile, 1 partial piece, 2 finishing piece), the first worker
 * holding a partial sum of the tile (kind 2)}, for up to max_units units.
 * *n_workers (if non-NULL) receives the grid's worker count.  Returns the
 * worker's number of units, or -1 for invalid arguments. */
int mx_debug_split_units(int64_t tiles, int workers, int kt, int mode, int worker, int32_t *out, int max_units,
                         int *n_workers);

#ifdef __cplusplus
}
#endif
#endif /* MX_H_ */
