/*
 * awq_w4a16.h -- C ABI of a W4A16 group-quantized linear layer (AWQ) for NVIDIA B200 (sm_100a).
 *
 * The layer computes  y = x' . dequant(W)^T  where W is an N x K (out x in) weight quantized to unsigned
 * 4-bit codes with one fp16 scale and one 4-bit zero point per group of g = 64, 128 or 256 consecutive input
 * channels (128 is the pages' setting),
 * dequantized as (q - z) * scale, and x' is the fp16 activation with the AWQ per-input-channel scale
 * divided out.  Sources (web pages on AWQ; each cited by title and section):
 *   [AWQ/GPTQ]   "AWQ and GPTQ algorithms" (jsqmd.com), section 2.1 (2) importance E[|X_j|],
 *                section 2.1 (3) channel scaling: multiply salient weight channels by s, divide the
 *                activations by s at inference, mathematically equivalent before rounding;
 *                section 1.1: W4A16 = 4-bit weights, fp16 activations.
 *   [LLM-AWQ]    "LLM-AWQ academic impact" (blog.csdn.net mirror), section "quantization flow":
 *                --w_bit 4 --q_group_size 128, two stages (scale search, then real quantization).
 *   [AutoAWQ]    "LLM quantization speed-up" (bjdmk.com.cn), section "quantization parameters":
 *                group size 128, zero-point quantization, GEMV mode (single batch) vs GEMM mode;
 *                section "fused modules": several steps merged into one operation.
 * The group size is a parameter of the pages' command line (--q_group_size); g = 64 and 256 are offered
 * beside 128 with the same grid and layout.
 * Where the pages leave a step open, the library takes the plain reading stated at each entry point.
 *
 * Conventions (all entry points):
 *   - Pointers named d_* are DEVICE pointers (global memory of the current CUDA device).  The caller
 *     allocates and frees every buffer; the library never allocates device memory and never
 *     synchronizes, except awq_last_device_status().
 *   - fp16 values are passed as uint16_t bit patterns (IEEE binary16).
 *   - Every call enqueues its kernels on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *     returns at once.  Arguments are checked on the host first; on failure the call returns the
 *     status code and launches nothing.  A launch failure returns AWQ_ERR_CUDA.
 *   - Device pointers must be 16-byte aligned (AWQ_ERR_MISALIGNED otherwise).
 *   - NaN or Inf anywhere in W, s, xcal or x is undefined behaviour (not checked).
 *   - Kernels launched by this library call griddepcontrol.wait before they read any activation or
 *     write any output, so they may be launched with programmatic dependent launch; they read only
 *     packed weights before that point.  Hence the packed weights a linear call reads must not be written
 *     by work still in flight on the stream, unless that work signals its dependents only when it has
 *     completed.  awq_pack's kernel never signals early (its dependents start when it has finished), so
 *     awq_pack followed by a linear call on the same stream, with no synchronisation, is safe.  A caller's
 *     own kernel that writes packed weights must not trigger programmatic completion before its last write
 *     to them, or must be separated from the linear call by an event or a host synchronisation.
 *
 * ---------------------------------------------------------------------------------------------------
 * PACKED WEIGHT LAYOUT (this library's own; the producer is awq_pack)
 *
 *   N_pad = N rounded up to a multiple of 32.   G = K / g (g = 64, 128 or 256).   Row n, input channel k.
 *
 *   qweight  uint32_t[N_pad * K / 8].  The rows are cut into row blocks of 32 rows (rb = n / 32,
 *            r = n % 32) and K into chunks of 32 channels (kc = k / 32).  Each (rb, kc) tile is 512
 *            contiguous bytes: 32 rows x 4 words, row r's 4 words at word offset 4*r.  Tiles are stored
 *            row-block major:  tile (rb, kc) begins at word  (rb * (K/32) + kc) * 128.
 *            Word j (0..3) of row r in tile (rb, kc) holds the 8 codes of channels
 *            k = 32*kc + 8*j + e, e = 0..7, in nibbles (bits 4p..4p+3, p = 0..7) ordered so that
 *              nibble p = e/2      holds the code of even e,
 *              nibble p = 4 + e/2  holds the code of odd e;
 *            i.e. nibble order e = [0, 2, 4, 6, 1, 3, 5, 7].  (Masking the word with 0x000F000F puts
 *            channels e=0,1 in the two 16-bit halves; 0x00F000F0 gives e=2,3; the word shifted right by
 *            8 gives e=4,5 and e=6,7 the same way.)
 *            Consequence: the 32 rows x g channels of one (row block, group) -- a "unit",
 *            u = rb * G + gi -- are 16 * g contiguous bytes starting at byte u * 16 * g (2048 at g = 128).
 *   scales   uint16_t (fp16)[G * N_pad], unit major: the scale of row n, group gi is
 *            scales[(rb * G + gi) * 32 + r]  (rb = n / 32, r = n % 32): 64 contiguous bytes per unit.
 *   qzeros   uint32_t[G * N_pad / 8], unit major: the zero of row n, group gi is nibble (r % 8)
 *            (bits 4*(r%8) .. +3) of word qzeros[(rb * G + gi) * 4 + r / 8]: 16 bytes per unit.
 *   So consecutive units are consecutive in all three arrays, and a range of units is one contiguous
 *   stretch of each array.
 *   Padding rows n = N .. N_pad-1 hold code 0, scale 0 and zero 0 in every array.
 *   Bytes per weight (N a multiple of 32): 0.5 + 2.5/g = 0.51953 at g = 128 (0.53906 at 64, 0.50977 at 256).
 *
 * 3-BIT LAYOUT (awq_pack3; read by w3a16_gemv): the same row blocks, 32-channel chunks, units, scales and
 * zeros as above, with 12 bytes per row per chunk instead of 16:
 *   qweight  uint32_t[N_pad * K / 32 * 3].  Tile (rb, kc) is 384 contiguous bytes, 32 rows x 3 words, row r's
 *            words at word offset (rb * (K/32) + kc) * 96 + 3 r.  For channel c = 8j + 2p + h of the chunk
 *            (j = 0..3 the 8-channel group, p = 0..3 the pair, h = 0..1 the half) with 3-bit code q:
 *              word j / 2 holds q & 3 at bits 8 (j % 2) + 2p + 16h .. +1   (the low 2-bit plane),
 *              word 2 holds q >> 2 at bit 4j + p + 16h                     (the high-bit plane).
 *            So for group j and pair p, ((word_{j/2} >> (8 (j%2) + 2p)) & 0x00030003) | ((word_2 >> (4j + p))
 *            & 0x00010001) << 2 puts the codes of channels 8j + 2p and 8j + 2p + 1 in the two 16-bit halves.
 *            A unit (32 rows x g channels) is 12 g contiguous bytes.  Bytes per weight: 0.375 + 2.5/g
 *            (0.39453 at g = 128, 24 % less than the 4-bit layout).
 *
 * QUANTIZATION GRID (what awq_pack computes; plain reading of [AutoAWQ] zero point + [LLM-AWQ] w_bit 4,
 * q_group_size g as asymmetric min/max round-to-nearest), per row n and group gi, all in IEEE fp32
 * with correctly rounded operations and no fused multiply-add:
 *   w'_k  = W_nk * s_k                                   (exact: an fp16 x fp16 product fits fp32)
 *   mn    = min_k w'_k,  mx = max_k w'_k                 (over the g channels of the group)
 *   sc32  = max((mx - mn) / 15, 1e-5f);   sc = fp16_rne(sc32);   S = float(sc)
 *   z     = clamp(rint(-mn / S), 0, 15)                  (rint = round half to even)
 *   q_k   = clamp(rint(w'_k / S) + z, 0, 15)
 * Dequantized weight: (q_k - z) * S.
 * ---------------------------------------------------------------------------------------------------
 */
#ifndef AWQ_W4A16_H
#define AWQ_W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum awq_status {
  AWQ_OK = 0,
  AWQ_ERR_INVALID_ARG = 1,     /* a size or pointer argument is out of range or NULL */
  AWQ_ERR_UNSUPPORTED = 2,     /* a valid request this library does not implement (e.g. g = 32) */
  AWQ_ERR_MISALIGNED = 3,      /* a device pointer is not 16-byte aligned */
  AWQ_ERR_CUDA = 4,            /* a CUDA runtime call or kernel launch failed */
  AWQ_ERR_DEVICE_TIMEOUT = 5,  /* a kernel gave up on a bounded wait (read via awq_last_device_status) */
  AWQ_ERR_WORKSPACE = 6,       /* the workspace is NULL or smaller than w4a16_workspace_bytes() */
  AWQ_ERR_NUMERIC = 7          /* a factorisation met a non-positive pivot (read via awq_last_device_status) */
} awq_status;

/* Opaque stream handle, ABI-compatible with cudaStream_t. */
typedef struct CUstream_st* awq_stream_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* awq_status_string(awq_status st);

/* Library version, e.g. 100 for 0.1.0. */
int awq_version(void);

/*
 * awq_packed_sizes -- byte sizes of the three packed arrays for an N x K weight at group size g
 * (layout above; [LLM-AWQ] "quantization flow" fixes w_bit 4 and q_group_size 128, [AWQ/GPTQ] section
 * 2.3 the saving these sizes realise: 0.51953 B per weight, 74 % below fp16).  Host only; launches nothing.
 * Errors: AWQ_ERR_INVALID_ARG if N < 1, K < 1, K % g != 0 or an output pointer is NULL;
 *         AWQ_ERR_UNSUPPORTED if g is not 64, 128 or 256.
 */
awq_status awq_packed_sizes(int N, int K, int g, size_t* qweight_bytes, size_t* scales_bytes,
                            size_t* qzeros_bytes);

/*
 * awq_act_scale -- per-input-channel AWQ scale from calibration activations.
 * [AWQ/GPTQ] section 2.1 (2): the statistic is the mean absolute activation E[|X_j|] over the
 * calibration rows; the scale is that statistic raised to the exponent alpha = 0.5 (this library's fixed
 * exponent; the scale search over alpha is not part of this entry point):
 *     s_j = fp16_rne( sqrt( (sum_r |xcal_rj|) / R ) ),   sum, division and sqrt in IEEE fp64.
 * (The fp64 sum of up to 8192 fp16 magnitudes is exact, so the result does not depend on order.)
 *   d_xcal  [R][K] fp16, row major, device.        d_s  [K] fp16, device, written.
 * Errors: AWQ_ERR_INVALID_ARG if R < 1, R > 8192, K < 1, or a pointer is NULL.
 */
awq_status awq_act_scale(const uint16_t* d_xcal, int R, int K, uint16_t* d_s, awq_stream_t stream);

/*
 * awq_apply_inv_scale -- divide the activations by the AWQ scale ([AWQ/GPTQ] section 2.1 (3): at
 * inference the activations carry the inverse of the factor folded into the weights, so that
 * x' . (W diag(s))^T = x . W^T before rounding):
 *     x'_mk = fp16_rne( x_mk / s_k ),   the division in IEEE fp64.
 *   d_x [M][K] fp16, d_s [K] fp16, d_xp [M][K] fp16 written (may alias d_x).  Device pointers.
 * Errors: AWQ_ERR_INVALID_ARG if M < 1, K < 1, or a pointer is NULL.
 */
awq_status awq_apply_inv_scale(const uint16_t* d_x, const uint16_t* d_s, int M, int K, uint16_t* d_xp,
                               awq_stream_t stream);

/*
 * awq_pack -- fold the AWQ scale into W, quantize with the grid above and write the packed layout.
 * Bit-exact: the three arrays depend only on W, s, N, K.
 *   d_W       [N][K] fp16, row major, device.
 *   d_s       [K] fp16 per-input-channel scale, device; NULL means s = 1 (plain round-to-nearest).
 *   d_qweight, d_scales, d_qzeros: outputs of awq_packed_sizes() bytes each (padding rows written).
 * Errors: AWQ_ERR_INVALID_ARG (N < 1, K < g, K % g != 0, NULL output), AWQ_ERR_UNSUPPORTED (g not 64, 128
 *         or 256), AWQ_ERR_MISALIGNED, AWQ_ERR_CUDA.
 */
awq_status awq_pack(const uint16_t* d_W, const uint16_t* d_s, int N, int K, int g, uint32_t* d_qweight,
                    uint16_t* d_scales, uint32_t* d_qzeros, awq_stream_t stream);

/*
 * awq_pack_bits -- awq_pack with the bit width of the grid as a parameter: w_bit = 4 is awq_pack; w_bit = 3 is
 * the 3-bit grid ([LLM-AWQ] "choose 4-bit or 3-bit quantization by hardware resources"; [INT4-VLM] introduction:
 * AWQ at INT3): the same asymmetric grid with qmax = 7 (sc32 = max((mx - mn)/7, 1e-5), z and q clamped to
 * 0..7).  The codes are stored in the same 4-bit layout, so every linear entry point runs the result unchanged;
 * the 3-bit grid gives its accuracy, not a smaller weight (0.52 bytes per weight as at 4 bits).
 * Errors: as awq_pack; AWQ_ERR_UNSUPPORTED for w_bit other than 3 or 4.
 */
awq_status awq_pack_bits(const uint16_t* d_W, const uint16_t* d_s, int N, int K, int g, int w_bit, uint32_t* d_qweight,
                         uint16_t* d_scales, uint32_t* d_qzeros, awq_stream_t stream);

/* awq_packed3_sizes -- byte sizes of the three arrays of the 3-bit layout (above) for an N x K weight at g. */
awq_status awq_packed3_sizes(int N, int K, int g, size_t* qweight_bytes, size_t* scales_bytes, size_t* qzeros_bytes);

/*
 * awq_pack3 -- awq_pack on the 3-bit grid (qmax = 7; awq_pack_bits with w_bit = 3) written in the packed 3-bit
 * layout ([LLM-AWQ] "choose 4-bit or 3-bit quantization by hardware resources"; [INT4-VLM] introduction, AWQ at
 * INT3): 0.39 bytes per weight.  Arguments and errors as awq_pack; outputs sized by awq_packed3_sizes.
 */
awq_status awq_pack3(const uint16_t* d_W, const uint16_t* d_s, int N, int K, int g, uint32_t* d_qweight,
                     uint16_t* d_scales, uint32_t* d_qzeros, awq_stream_t stream);

/*
 * w3a16_gemv -- the decode kernel of w4a16_gemv on a weight from awq_pack3: the same plans, warp roles, tensor-core
 * contraction (exact q - z products, fp32 sums) and epilogue, with each unit's codes read from the 3-bit layout.
 * Any M (passes of up to 16 rows).  Arguments, workspace (w4a16_workspace_bytes(AWQ_MODE_GEMV, ...)) and errors
 * as w4a16_gemv.  There is no 3-bit GEMM: prefill-sized M runs here, in passes.
 */
awq_status w3a16_gemv(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                      const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g, void* d_workspace,
                      size_t workspace_bytes, awq_stream_t stream);

/*
 * awq_pack_gate_up -- packs the gate and up projections of a gated MLP (both [NI][K], the same input x)
 * as ONE packed weight of N = 2 * NI rows for w4a16_gate_up_silu ([AutoAWQ] "fused modules": one weight
 * stream and one read of x for both projections).  Row 32j + i of the packed weight is gate row 16j + i
 * for i < 16 and up row 16j + i - 16 for i >= 16; each row is quantized exactly as awq_pack quantizes it
 * (same grid, same s), so the packed arrays equal awq_pack of that interleaved [2 NI][K] matrix.
 *   d_Wgate, d_Wup  [NI][K] fp16, row major, device.   NI >= 16 with NI % 16 == 0.
 *   d_s, g, outputs (sized by awq_packed_sizes(2 * NI, K, g, ...)), stream: as awq_pack.
 * Errors: as awq_pack; AWQ_ERR_INVALID_ARG also when NI % 16 != 0.
 */
awq_status awq_pack_gate_up(const uint16_t* d_Wgate, const uint16_t* d_Wup, const uint16_t* d_s, int NI, int K, int g,
                            uint32_t* d_qweight, uint16_t* d_scales, uint32_t* d_qzeros, awq_stream_t stream);

/*
 * The three linear-layer entry points share one argument list:
 *   d_x       [M][K] fp16 activations (already divided by s), row major, device.
 *   d_qweight, d_scales, d_qzeros: packed weight from awq_pack for the same N, K, g.
 *   d_y       [M][N] fp16 output, row major, device; y_mn = fp16_rne(sum_k x'_mk (q_nk - z) S),
 *             accumulated in fp32 (summation order is implementation defined).
 *   M >= 1, N >= 1 with N % 8 == 0, g in {64, 128, 256}, K >= g with K % g == 0.
 *   d_workspace / workspace_bytes: device scratch of at least w4a16_workspace_bytes(mode, M, N, K, g)
 *             bytes (may be NULL when that is 0).  The workspace must be zero-filled once before its
 *             first use (cudaMemsetAsync); every call leaves it ready for the next call.  Calls that
 *             share a workspace must not run concurrently on the GPU.
 * Errors: AWQ_ERR_INVALID_ARG, AWQ_ERR_UNSUPPORTED, AWQ_ERR_MISALIGNED, AWQ_ERR_WORKSPACE, AWQ_ERR_CUDA.
 */

/* w4a16_gemv -- decode path ([AutoAWQ] "GEMV mode", single batch): streams the packed weights once per
 * pass of up to 16 rows of x' (M <= 8: one pass of 8; larger M: passes of 16) through per-warp shared-memory
 * rings filled by TMA bulk copies, turns each code into the exact fp16 integer q - z in registers and
 * contracts it with x' on the tensor cores (mma.sync m16n8k16, exact products, fp32 accumulation); each
 * group's fp32 sum is multiplied by its scale in fp32.  Units of the weight are spread over the SMs; a row
 * block split between CTAs is combined in the workspace in a fixed order (results are deterministic). */
awq_status w4a16_gemv(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                      const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g,
                      void* d_workspace, size_t workspace_bytes, awq_stream_t stream);

/*
 * w4a16_gemv_s -- w4a16_gemv with the AWQ activation scaling fused in: d_x holds the RAW activations x and
 * d_s the per-channel AWQ scale s ([K] fp16, device, 16-byte aligned); the kernel uses
 * x'_mk = fp16_rne(x_mk / s_k), bit-identical to awq_apply_inv_scale (the correctly rounded fp32 quotient
 * of two fp16 values rounds to the same fp16 as the exact quotient), so y equals
 * w4a16_gemv(awq_apply_inv_scale(x, s)) bit for bit.  [AWQ/GPTQ] section 2.1 (3) (activations divided
 * by s at inference); [AutoAWQ] "fused modules" (the separate scaling pass disappears).  x is staged in
 * shared memory, which bounds M x K per pass: AWQ_ERR_UNSUPPORTED when it does not fit (every M = 1
 * shape with K <= 32768 fits).  Other arguments, workspace and errors: as w4a16_gemv; d_s NULL gives
 * AWQ_ERR_INVALID_ARG.
 */
awq_status w4a16_gemv_s(const uint16_t* d_x, const uint16_t* d_s, const uint32_t* d_qweight,
                        const uint16_t* d_scales, const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g,
                        void* d_workspace, size_t workspace_bytes, awq_stream_t stream);

/* w4a16_gemm -- prefill path ([AutoAWQ] "GEMM mode", long context): packed tiles staged by the TMA,
 * dequantized to fp16 in shared memory and contracted on the 5th-generation tensor cores (tcgen05,
 * fp32 accumulators in tensor memory). */
awq_status w4a16_gemm(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                      const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g,
                      void* d_workspace, size_t workspace_bytes, awq_stream_t stream);

/* w4a16_gemv_noalloc -- the same computation as w4a16_gemv for callers that cannot allocate device
 * memory (e.g. a plug-in whose host framework owns every allocation, or a serving loop whose memory
 * budget is fixed at start-up).  The pages have no counterpart: this is a deployment convenience.
 * The split scratch is a library-owned static device array of 512 KiB per device (held by every GPU
 * that loads the library until exit); sizes whose scratch would exceed it return AWQ_ERR_WORKSPACE.  Most
 * shapes need no scratch at all (w4a16_workspace_bytes(AWQ_MODE_GEMV, ...) == 0); the array serves the
 * shapes whose row blocks are split between CTAs.
 * Nothing is allocated: the call clears the array's counters with cudaMemsetAsync and launches the
 * GEMV.  The first call on a device looks up the array's address (cudaGetSymbolAddress); make it
 * before any stream capture.  All calls share the array: calls that overlap on the GPU race. */
awq_status w4a16_gemv_noalloc(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                              const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g,
                              awq_stream_t stream);

/* w4a16_linear -- the mode choice of [AutoAWQ] "quantization parameters" (GEMV mode for a single batch,
 * GEMM mode for long contexts): picks GEMV when M <= w4a16_gemv_max_m(N, K), GEMM otherwise, and calls it. */
awq_status w4a16_linear(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                        const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g,
                        void* d_workspace, size_t workspace_bytes, awq_stream_t stream);

/*
 * w4a16_linear_pf -- w4a16_linear with a prefetch hint; the pages have no counterpart (a scheduling
 * aid for a caller that knows which weight it will use next, e.g. the next linear of a decode step).
 * In GEMV mode, while the kernel runs, its CTAs also ask for the next_bytes at d_next to be brought
 * into L2 (cp.async.bulk.prefetch.L2; weights only, issued before the kernel's dependency wait, so
 * d_next must not be written by earlier work still in flight).  The outputs are exactly those of
 * w4a16_linear.  In GEMM mode, or with d_next NULL or next_bytes 0, the hint is ignored.
 *   d_next      device pointer, 16-byte aligned (AWQ_ERR_MISALIGNED otherwise); typically the next
 *               linear's d_qweight.      next_bytes  a multiple of 16 (AWQ_ERR_INVALID_ARG otherwise).
 * Other arguments, layout and errors: as w4a16_linear.
 */
awq_status w4a16_linear_pf(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                           const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g, void* d_workspace,
                           size_t workspace_bytes, const void* d_next, size_t next_bytes, awq_stream_t stream);

/*
 * w4a16_gate_up_silu -- the gate and up projections of a gated MLP with the activation fused into the
 * epilogue ([AutoAWQ] "fused modules"; the SiLU gate of the Llama-style MLP whose shapes the decode
 * workloads use):  h_mj = fp16_rne(silu(a_mj) * b_mj),  a = x' . dequant(W_gate)^T and b = x' . dequant(W_up)^T
 * accumulated in fp32 and never rounded to fp16 on the way, silu(a) = a / (1 + e^-a) in fp32.
 *   d_x       [M][K] fp16 (x' as for the linear calls), device.
 *   d_qweight, d_scales, d_qzeros: from awq_pack_gate_up for the same NI, K, g.
 *   d_h       [M][NI] fp16 output, row major, device.   NI >= 16 with NI % 16 == 0.
 *   Mode: GEMV when M <= w4a16_gemv_max_m(2 NI, K), else GEMM; workspace of
 *   w4a16_workspace_bytes(AWQ_MODE_LINEAR, M, 2 * NI, K, g) bytes, under the same rules as the linear calls.
 * Errors: as w4a16_linear; AWQ_ERR_INVALID_ARG also when NI % 16 != 0.
 */
awq_status w4a16_gate_up_silu(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                              const uint32_t* d_qzeros, uint16_t* d_h, int M, int NI, int K, int g, void* d_workspace,
                              size_t workspace_bytes, awq_stream_t stream);

/*
 * awq_search_scale -- the AWQ scale search ([AWQ/GPTQ] section 2.1 (3): choose the per-channel scale that
 * minimises the layer's output error after quantization over calibration data; [LLM-AWQ] "quantization
 * flow": the search stage, whose result the real-quantization stage, awq_pack, then uses).  Reading taken:
 * the scales s(alpha)_j = fp16_rne((mean_r |xcal_rj|)^alpha) on the grid alpha_i = i / n_grid,
 * i = 0 .. n_grid (the mean and the power in fp64; alpha = 0 gives s = 1, i.e. plain round-to-nearest,
 * alpha = 0.5 the scale of awq_act_scale); for each, the layer as deployed -- awq_pack(W, s), x' =
 * awq_apply_inv_scale(xcal, s), the fp16 output of w4a16_linear (GEMV or GEMM by R) -- and the loss
 *   L_i = sum_{r < R, n < N} (y'_rn - y_rn)^2  (fp64),  y = xcal . W^T unquantized (fp32 sums of exact products);
 * the winner is the first i of least L_i.  Everything runs on `stream` with no host synchronisation.
 *   d_W        [N][K] fp16 weight, device.        d_xcal   [R][K] fp16 calibration activations, device.
 *   N % 8 == 0; g in {64, 128, 256}, K % g == 0; 1 <= R <= 8192; 1 <= n_grid <= 1000.
 *   d_losses   [n_grid + 1] double, written: L_0 .. L_n_grid.
 *   d_s        [K] fp16, written: s of the winning alpha (pass it to awq_pack and awq_apply_inv_scale).
 *   d_best     one int32, written: the winning index i (alpha = i / n_grid).
 *   d_workspace / workspace_bytes: at least awq_search_workspace_bytes(N, K, R, g, n_grid) bytes (no
 *             zero-fill needed; the call clears what it needs).  Searches sharing a workspace must not
 *             run concurrently.
 * A channel whose calibration activations are all zero gives s = 0 for alpha > 0 (undefined behaviour, like
 * NaN input).  Errors: AWQ_ERR_INVALID_ARG, AWQ_ERR_UNSUPPORTED (g), AWQ_ERR_MISALIGNED, AWQ_ERR_WORKSPACE,
 * AWQ_ERR_CUDA.
 */
awq_status awq_search_scale(const uint16_t* d_W, const uint16_t* d_xcal, int N, int K, int R, int g, int n_grid,
                            double* d_losses, uint16_t* d_s, int32_t* d_best, void* d_workspace,
                            size_t workspace_bytes, awq_stream_t stream);

/* Workspace bytes awq_search_scale needs (SIZE_MAX for invalid sizes). */
size_t awq_search_workspace_bytes(int N, int K, int R, int g, int n_grid);

/*
 * gptq_quantize -- GPTQ ([AWQ/GPTQ] section 3.1: minimise ||W X - W_hat X||_F^2 over calibration activations X,
 * Hessian H = X^T X, columns quantized in blocks of 128 with each column's error compensated in the columns
 * not yet quantized through the inverse Hessian, obtained via Cholesky, and lazy batch updates of the
 * columns after each block; section 3.3: a small diagonal term, 1e-6 on the page, against a singular H),
 * writing the SAME packed layout as awq_pack, so every linear entry point runs the result unchanged.
 * Reading taken: H = X^T X + damp I in fp64; U upper triangular with H^-1 = U^T U; the columns in order, each
 * group's grid (awq_pack's fp32 min/max grid with s = 1) computed at the group's first column from the
 * group's current (error-compensated) weights rounded to fp32; code q = clamp(rint(w / S) + z, 0, 15) of the
 * current weight; its error (w - (q - z) S) / U_ii subtracted, times U_ij, from every later column j (at once
 * inside the 128-column block, after the block for the rest).  All but the grid is fp64.
 *   d_W       [N][K] fp16 weight, device.       d_xcal  [R][K] fp16 calibration activations, device.
 *   N % 8 == 0; K % 128 == 0 and K % g == 0 (g in {64, 128, 256}), K <= 65536; R >= 1; damp >= 0
 *   (1e-6 as on the page; a larger damp, e.g. 1% of the mean diagonal, steadies a rank-deficient H).
 *   d_qweight, d_scales, d_qzeros: outputs sized by awq_packed_sizes(N, K, g) (padding rows written).
 *   d_workspace: at least gptq_workspace_bytes(N, K, R, g) bytes (two K x K and one N x K fp64 arrays), no
 *   zero-fill needed.  Asynchronous on `stream`.  A non-positive pivot (H not positive definite in fp64) sets
 *   the device status word: awq_last_device_status then returns AWQ_ERR_NUMERIC.
 * Errors: AWQ_ERR_INVALID_ARG, AWQ_ERR_UNSUPPORTED (g), AWQ_ERR_MISALIGNED, AWQ_ERR_WORKSPACE, AWQ_ERR_CUDA.
 */
awq_status gptq_quantize(const uint16_t* d_W, const uint16_t* d_xcal, int N, int K, int R, int g, double damp,
                         uint32_t* d_qweight, uint16_t* d_scales, uint32_t* d_qzeros, void* d_workspace,
                         size_t workspace_bytes, awq_stream_t stream);

/* Workspace bytes gptq_quantize needs (SIZE_MAX for invalid sizes). */
size_t gptq_workspace_bytes(int N, int K, int R, int g);

/* Mode selector used by w4a16_linear: the largest M for which GEMV mode is chosen (32: the crossover
 * measured on B200 for the 70B-class shapes). */
int w4a16_gemv_max_m(int N, int K);

/* Modes for w4a16_workspace_bytes. */
#define AWQ_MODE_GEMV 1
#define AWQ_MODE_GEMM 2
#define AWQ_MODE_LINEAR 3

/* Workspace bytes a call needs on the current device (0 if none); SIZE_MAX for invalid sizes. */
size_t w4a16_workspace_bytes(int mode, int M, int N, int K, int g);

/*
 * awq_last_device_status -- synchronizes `stream`, then reads and clears the device status word that
 * kernels set when a bounded wait runs out (AWQ_ERR_DEVICE_TIMEOUT) or a factorisation met a non-positive
 * pivot (AWQ_ERR_NUMERIC).  Returns AWQ_OK, one of those two, or AWQ_ERR_CUDA.
 */
awq_status awq_last_device_status(awq_stream_t stream);

/*
 * awq_selftest_wait_timeout -- check of the timeout path above; the pages have no counterpart.
 * Launches one kernel of one thread that waits on a shared-memory mbarrier phase nothing completes,
 * with the bounded wait helper of the GEMM (backoff = 0: polling) or of the GEMV (backoff != 0:
 * polling with nanosleep).  After about 2 s the wait gives up, the device status word is set (so the
 * next awq_last_device_status returns AWQ_ERR_DEVICE_TIMEOUT) and the kernel writes 1 to *d_returned
 * (2 would mean the wait completed).  The CUDA context stays usable.  Device memory: d_returned, one
 * uint32_t, written.  Errors: AWQ_ERR_INVALID_ARG if d_returned is NULL, AWQ_ERR_CUDA on a launch failure.
 */
awq_status awq_selftest_wait_timeout(int backoff, uint32_t* d_returned, awq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_W4A16_H */
