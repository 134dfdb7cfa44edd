/*
 * libqlora -- the NF4 QLoRA linear layer on one NVIDIA B200 (sm_100a).
 *
 * C ABI. Every pointer argument is either a host pointer (marked "host") or a
 * device pointer in the current CUDA device's memory (marked "device"). The
 * library never allocates, frees or synchronises: the caller owns every
 * buffer, passes scratch space explicitly ("workspace") and reads results
 * after synchronising the stream itself. Calls are asynchronous on `stream`
 * (NULL = the legacy default stream). Argument errors are detected on the host
 * and returned synchronously before anything is launched; errors that only the
 * GPU can see (non-finite weights, a bounded wait that ran out) are written to
 * an optional device status word. No C++ exception crosses this boundary.
 *
 * Layouts: every matrix is row-major and contiguous; bf16 values are passed as
 * their 16-bit patterns (uint16_t). Device pointers must be 16-byte aligned.
 *
 * Notation: W is the frozen weight [N, K] (N = out features, K = in features),
 * X the activations [M, K] (M tokens), A the LoRA down matrix [r, K], B the
 * LoRA up matrix [N, r], s = alpha / r. The layer computes
 *     Y = X W'^T + s (X A^T) B^T
 * where W' is the NF4 weight dequantised to bf16 ("QLoRA, in depth", section
 * "The mechanism in brief": each forward dequantises W to the compute dtype
 * and adds (alpha / r) B A x; backward gives gradients for A, B and the
 * activations, never for W).
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,        /* null pointer, bad size, bad scalar */
  QLORA_ERR_UNSUPPORTED_SHAPE = 2,  /* a shape the kernels do not cover */
  QLORA_ERR_MISALIGNED = 3,         /* a device pointer not 16-byte aligned */
  QLORA_ERR_WORKSPACE = 4,          /* workspace missing or too small */
  QLORA_ERR_NONFINITE = 5,          /* device status: NaN or inf in a weight */
  QLORA_ERR_TIMEOUT = 6,            /* device status: a bounded wait ran out */
  QLORA_ERR_CUDA = 7                /* a CUDA runtime call failed */
} qlora_status_t;

/* Same type as cudaStream_t; spelled out so this header needs no CUDA header. */
typedef struct CUstream_st *qlora_stream_t;

/*
 * An NF4 matrix: a non-owning view of three device buffers.
 * Format ("QLoRA, in depth", "The mechanism in brief"; "What is QLoRA ...",
 * "The three QLoRA ideas"): W[rows, cols] is cut into blocks of 64
 * consecutive row-major elements (cols % 64 == 0, so a block lies inside one
 * row); each weight is a 4-bit code into the 16-level NF4 codebook; each block
 * has an 8-bit scale; each group of 256 consecutive blocks has one fp32
 * second-level scale.
 *   codes : rows*cols/2 bytes; byte j = (code[2j] << 4) | code[2j+1]
 *           (the first element of a pair in the high nibble).
 *   scale8: nb = rows*cols/64 bytes; block b's constant is scale8[b] * scale2[b/256].
 *   scale2: ng = ceil(nb/256) floats, scale2[g] = RN32(max c1 in group g / 255).
 * Dequantised weight: w' = bf16_rn(fp32_rn(level[code] * fp32_rn(scale8[b] * scale2[b/256]))).
 */
typedef struct {
  int64_t rows;
  int64_t cols;
  uint8_t *codes;
  uint8_t *scale8;
  float *scale2;
} qlora_nf4_t;

/* Byte sizes of the three buffers of a [rows, cols] NF4 matrix (host).
 * Source: "QLoRA, in depth", "The mechanism in brief" (about 4.127 bits per
 * weight). Errors: INVALID_ARG on null outputs or rows/cols <= 0,
 * UNSUPPORTED_SHAPE when cols % 64 != 0. */
qlora_status_t qlora_nf4_sizes(int64_t rows, int64_t cols, size_t *codes_bytes,
                               size_t *scale8_bytes, size_t *scale2_bytes);

/* Copies the 16 NF4 levels (float32, ascending, level[0] = -1, level[7] = 0,
 * level[15] = 1) into out (host, 16 floats). The levels are normal quantiles
 * ("QLoRA and Fine-Tuning on One Consumer GPU", "NF4 and double
 * quantisation"). */
qlora_status_t qlora_nf4_codebook(float *out);

/* Quantise W (device, float32 [q->rows, q->cols]) into q's buffers (device).
 * Per block: c1 = max|w|; code = nearest level to fp32_rn(w / c1), ties to the
 * lower level, all-zero block -> code 7; per group: c2 = max c1,
 * scale8 = round-half-even(255 c1 / c2), scale2 = fp32_rn(c2 / 255).
 * Source: "QLoRA, in depth", "The mechanism in brief"; "What is QLoRA ...",
 * "The three QLoRA ideas".
 * dev_status (device int32, may be NULL): set to 0 by this call, then to
 * QLORA_ERR_NONFINITE if any weight is NaN or inf (the outputs are then
 * written but meaningless). Errors returned: INVALID_ARG, UNSUPPORTED_SHAPE,
 * MISALIGNED, CUDA. */
qlora_status_t qlora_nf4_quantize(const float *W, const qlora_nf4_t *q,
                                  int32_t *dev_status, qlora_stream_t stream);

/* Dequantise q (device buffers) into out (device, bf16 [rows, cols]),
 * bit-exactly by the formula in the qlora_nf4_t comment. Source: "QLoRA, in
 * depth", "The mechanism in brief" (W is dequantised to the compute dtype,
 * usually bf16). Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, CUDA. */
qlora_status_t qlora_nf4_dequantize(const qlora_nf4_t *q, uint16_t *out,
                                    qlora_stream_t stream);

/* Comparison codec. The same stored format (packed 4-bit codes, 8-bit block
 * constants, fp32 second-level scales) with another 16-level codebook, so
 * that the error NF4 saves can be measured ("What is QLoRA ...",
 * "Follow-up questions to expect": evenly spaced int4 levels waste levels on
 * rare large values, NF4 follows the bell-shaped weights and errs less).
 * QLORA_CODEBOOK_NF4 is the codebook of qlora_nf4_quantize/dequantize;
 * QLORA_CODEBOOK_INT4 has the levels (k - 8) / 7, k = 0..15 (fp32), zero at
 * code 8. Encoding rules, ties and the double quantisation are those of NF4. */
typedef enum { QLORA_CODEBOOK_NF4 = 0, QLORA_CODEBOOK_INT4 = 1 } qlora_codebook_t;

/* The 16 fp32 levels of a codebook (host). Errors: INVALID_ARG. */
qlora_status_t qlora_codec_levels(int32_t codebook, float *out);

/* As qlora_nf4_quantize / qlora_nf4_dequantize with the given codebook.
 * Errors: as those calls, and INVALID_ARG for an unknown codebook. */
qlora_status_t qlora_codec_quantize(const float *W, const qlora_nf4_t *q, int32_t codebook, int32_t *dev_status,
                                    qlora_stream_t stream);
qlora_status_t qlora_codec_dequantize(const qlora_nf4_t *q, int32_t codebook, uint16_t *out, qlora_stream_t stream);

/* Comparison second level. NF4 codes and first-level blocks as above, with
 * the block constants stored the way the paper the pages cite does it
 * ("QLoRA and Fine-Tuning on One Consumer GPU", "NF4 and double
 * quantisation": double quantisation quantises the absmax constants and saves
 * about 0.37 bits per parameter; "What is QLoRA ...", "The three QLoRA ideas":
 * 8 bits in blocks of 256): per group of 256 blocks the constants are centred
 * on their mean and kept as 8-bit floats.
 *   mu_g = RN32(RN64(S / n)), S the float64 sum of the group's c1_b in block
 *          order, n its blocks; cen_b = RN32(c1_b - mu_g); a_g = max |cen_b|;
 *   d_g = RN32(a_g / 448); scale8[b] = E4M3 code of RN32(cen_b / d_g)
 *          (round to nearest even, saturating to +-448; 0 when d_g = 0);
 *   scale2[2g] = d_g, scale2[2g + 1] = mu_g (2 * ng floats, 8-byte aligned);
 *   block scale s_b = RN32(RN32(e4m3(scale8[b]) * d_g) + mu_g) and
 *   w' = RN_bf16(RN32(level[code] * s_b)).
 * 4 + 8/64 + 64/16384 = 4.1289 bits per weight. Only the codec runs on this
 * format (the GEMMs read the linear one); it exists to measure the error of
 * the two second levels on the same weights.
 * qlora_dqfp8_sizes: as qlora_nf4_sizes with s2_b = 8 * ng. Errors: INVALID_ARG.
 * qlora_dqfp8_quantize / qlora_dqfp8_dequantize: as qlora_nf4_quantize /
 * qlora_nf4_dequantize. Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED,
 * CUDA; NONFINITE in dev_status. */
qlora_status_t qlora_dqfp8_sizes(int64_t rows, int64_t cols, size_t *codes_b, size_t *s8_b, size_t *s2_b);
qlora_status_t qlora_dqfp8_quantize(const float *W, const qlora_nf4_t *q, int32_t *dev_status,
                                    qlora_stream_t stream);
qlora_status_t qlora_dqfp8_dequantize(const qlora_nf4_t *q, uint16_t *out, qlora_stream_t stream);

/* Workspace bytes that qlora_linear_fwd and qlora_linear_bwd need for M
 * tokens through an [N, K] layer of rank r (host). Interface only: no passage
 * of the pages defines it; it exists because this library never allocates, so
 * the caller sizes and owns the scratch memory the kernels use. It takes
 * (M, N, K, r) rather than the weight itself so that a caller can size the
 * workspace before any weight is quantised. The workspace starts with a
 * 256-byte counter page that must be zero before the workspace is first used
 * (e.g. one cudaMemsetAsync of the whole buffer); every call that completes
 * without a device error leaves the page zero, and the rest of the workspace
 * needs no initialisation. The same workspace may be reused by consecutive
 * calls on one stream; calls that run concurrently need separate workspaces.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE. */
qlora_status_t qlora_linear_workspace(int64_t M, int64_t N, int64_t K, int32_t r,
                                      size_t *bytes);

/* Forward of the QLoRA linear: Y = X W'^T + s (X A^T) B^T.
 * W: NF4 weight [N, K] (struct on the host, buffers on the device).
 * X [M, K], A [r, K], B [N, r]: device bf16. Y [M, N]: device bf16, written.
 * sU_out [M, r]: device bf16 or NULL; if given, receives bf16_rn(s X A^T), the
 *   value the backward can reuse instead of recomputing it. For M <= 16 the
 *   forward is the single launch of qlora_linear_fwd_group for this one
 *   linear: it forms sU itself (its fp32 sum runs in a different order than
 *   qlora_lora_xa's, so a backward that recomputes sU may see it differ by
 *   bf16 rounding) and applies each block constant to the block's partial
 *   sum (Y then equals the definition up to the bf16 rounding of the levels,
 *   within the same tolerance).
 * ws / ws_bytes: device workspace of at least qlora_linear_workspace() bytes
 *   (its first 256 bytes zero before first use, see there).
 * dev_status: device int32 or NULL; set to QLORA_ERR_TIMEOUT if a bounded wait
 *   inside a kernel ran out (results are then incomplete). It is not cleared.
 * Supported: M >= 1, N % 16 == 0, K % 64 == 0, r % 8 == 0 with 8 <= r <= 64,
 * s finite. fp32 accumulation; W' is dequantised tile by tile in shared memory
 * and never written to global memory ("QLoRA and Fine-Tuning on One Consumer
 * GPU", "The idea in one line": each weight tile is dequantised to bf16 only
 * for the moment it is used in a matmul).
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, CUDA. */
qlora_status_t qlora_linear_fwd(const qlora_nf4_t *W, const uint16_t *X, int64_t M,
                                const uint16_t *A, const uint16_t *B, int32_t r, float s,
                                uint16_t *Y, uint16_t *sU_out, void *ws, size_t ws_bytes,
                                int32_t *dev_status, qlora_stream_t stream);

/* Backward of the QLoRA linear with W frozen (no dW is ever formed):
 *   T  = dY B                  (kept as bf16_rn(s T) in the workspace)
 *   dX = dY W' + s T A         [M, K] bf16   (skipped when dX == NULL)
 *   dA = s T^T X               [r, K] fp32   (overwritten)
 *   dB = s dY^T (X A^T)        [N, r] fp32   (overwritten)
 * dY [M, N] device bf16. sU (device bf16 [M, r]) is the forward's sU_out; if
 * NULL it is recomputed from X and A. Other arguments as in qlora_linear_fwd.
 * Source: "QLoRA, in depth", "The mechanism in brief".
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, CUDA. */
qlora_status_t qlora_linear_bwd(const qlora_nf4_t *W, const uint16_t *X, int64_t M,
                                const uint16_t *A, const uint16_t *B, int32_t r, float s,
                                const uint16_t *dY, const uint16_t *sU, uint16_t *dX,
                                float *dA, float *dB, void *ws, size_t ws_bytes,
                                int32_t *dev_status, qlora_stream_t stream);

/*
 * Forward of several linears over the same few tokens in one launch, e.g. the
 * query, key and value projections of one attention layer, or the gate and up
 * projections of one MLP ("QLoRA and Fine-Tuning on One Consumer GPU", section
 * "Where 24 GB goes": adapters on the attention and MLP projections; section
 * "The idea in one line": each weight tile is dequantised to bf16 only for the
 * moment it is used in a matmul).
 * Each problem is one QLoRA linear with the arguments of qlora_linear_fwd:
 *   Y = X W'^T + sU B^T,  sU = bf16_rn(s X A^T)  (written to sU_out if given).
 * All problems of a call share the token count M, 1 <= M <= 16; X may be the
 * same buffer for several problems. A few-token forward reads each packed
 * weight once and does 2M flops per weight, so it is bound by memory and by
 * the expansion of the codes, and one launch over the whole group keeps every
 * SM streaming. The launch splits the (linear, 128-row tile, 64-weight block)
 * work evenly over the SMs; the levels enter the tensor cores as
 * bf16(1.43675 * level) with the block constant divided by 1.43675 applied to
 * each block's fp32 partial sum, so Y equals the composite forward up to the
 * bf16 rounding of the weights (within the GEMM tolerance of this library),
 * and the result does not depend on timing.
 * flags: 0, or QLORA_FWD_OVERLAP_PREVIOUS: the NF4 weights (codes, scale8,
 *   scale2) are not written by the work queued before this call on the
 *   stream, so the launch may begin streaming them before that work has
 *   finished (programmatic dependent launch); X, A, B and the workspace are
 *   still read only after it has finished.
 * ws / ws_bytes: device workspace of at least qlora_linear_fwd_group_workspace()
 *   bytes, 16-byte aligned, zero-filled before its first use. Every call leaves
 *   it as it found it (a launch resets each counter and flag it sets, so a
 *   captured call can be replayed); one call at a time may use it. After a
 *   QLORA_ERR_TIMEOUT in dev_status the workspace must be zero-filled (or
 *   replaced) before it is used again.
 * More than 16 problems run as consecutive launches of 16 on `stream`.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (M > 16, or a shape qlora_linear_fwd
 * rejects), MISALIGNED, WORKSPACE, CUDA; TIMEOUT in dev_status.
 */
typedef struct {
  qlora_nf4_t W;           /* [N, K] NF4 weight (buffers on the device) */
  const uint16_t *X;       /* [M, K] device bf16 */
  const uint16_t *A;       /* [r, K] device bf16 */
  const uint16_t *B;       /* [N, r] device bf16 */
  int32_t r;               /* 8 <= r <= 64, r % 8 == 0 */
  float s;                 /* alpha / r, finite */
  uint16_t *Y;             /* [M, N] device bf16, written */
  uint16_t *sU_out;        /* [M, r] device bf16 or NULL */
} qlora_linear_problem_t;

#define QLORA_FWD_OVERLAP_PREVIOUS 1

/* Workspace bytes of qlora_linear_fwd_group for these problems on the current
 * device (host; only the shapes, ranks and whether A and sU_out are given are
 * read). Interface only: no passage of the pages defines it.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE. */
qlora_status_t qlora_linear_fwd_group_workspace(const qlora_linear_problem_t *problems, int32_t count,
                                                int64_t M, size_t *bytes);
qlora_status_t qlora_linear_fwd_group(const qlora_linear_problem_t *problems, int32_t count, int64_t M,
                                      int32_t flags, void *ws, size_t ws_bytes, int32_t *dev_status,
                                      qlora_stream_t stream);

/*
 * The five steps of the layer, one entry point each. qlora_linear_fwd runs
 * qlora_lora_xa then qlora_fused_fwd; qlora_linear_bwd runs qlora_lora_dyb,
 * qlora_fused_dx and qlora_lora_grads (and qlora_lora_xa when sU is not
 * given). They are exposed so that a caller can schedule or time the steps
 * separately; arguments, layouts and errors are as in the composite calls.
 * For the skinny products `ws` is a workspace of at least qlora_linear_workspace()
 * bytes for the same (M, N, K, r) (they need none at present; the argument is
 * kept so that a split of their reduction can use it). qlora_fused_workspace()
 * sizes the optional workspace of the two fused GEMMs.
 */

/* sU = bf16_rn(s X A^T), [M, r]. The adapter's down projection, the first
 * half of (alpha / r) B A x ("QLoRA, in depth", "The mechanism in brief").
 * K % 64 == 0. Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, CUDA. */
qlora_status_t qlora_lora_xa(const uint16_t *X, int64_t M, int64_t K, const uint16_t *A, int32_t r,
                             float s, uint16_t *sU, void *ws, size_t ws_bytes, qlora_stream_t stream);

/* Bytes of the optional workspace of qlora_fused_fwd / qlora_fused_dx for M
 * tokens on the current device (it scales with the device's SM count).
 * Errors: INVALID_ARG (M < 1 or bytes NULL), CUDA. */
qlora_status_t qlora_fused_workspace(int64_t M, size_t *bytes);

/* Y = X W'^T + sU B^T with W' dequantised tile by tile in shared memory and
 * fed to the tensor cores; the LoRA term is one extra K-step of the same
 * accumulation ("QLoRA and Fine-Tuning on One Consumer GPU", "The idea in one
 * line").
 * ws / ws_bytes: NULL / 0, or device memory of at least qlora_fused_workspace(M)
 *   bytes, 16-byte aligned. With NULL every CTA takes whole output tiles. With a
 *   workspace and M <= 64 (where whole tiles would leave most SMs idle) the
 *   (tile, K-step) work is split evenly over all SMs and tiles cut between CTAs
 *   are summed through fp32 partials kept there (results equal up to fp32
 *   rounding order); for M <= 16 the forward is the persistent few-token
 *   launch of qlora_linear_fwd_group; larger M keeps whole tiles. The first
 *   256 bytes of the workspace are a counter page that must be zero before
 *   first use and that every call leaves zero; the rest needs no
 *   initialisation and keeps no state the caller sees; one launch at a time
 *   may use a given workspace.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, CUDA. */
qlora_status_t qlora_fused_fwd(const qlora_nf4_t *W, const uint16_t *X, int64_t M, const uint16_t *B,
                               int32_t r, const uint16_t *sU, uint16_t *Y, void *ws, size_t ws_bytes,
                               int32_t *dev_status, qlora_stream_t stream);

/* sT = bf16_rn(s dY B), [M, r]: the gradient reaching the adapter's
 * bottleneck. N % 16 == 0. Errors: as qlora_lora_xa. */
qlora_status_t qlora_lora_dyb(const uint16_t *dY, int64_t M, int64_t N, const uint16_t *B, int32_t r,
                              float s, uint16_t *sT, void *ws, size_t ws_bytes, qlora_stream_t stream);

/* dX = dY W' + sT A, [M, K] bf16, W' dequantised in shared memory as in
 * qlora_fused_fwd (here consumed untransposed); ws as in qlora_fused_fwd.
 * Errors: as qlora_fused_fwd. */
qlora_status_t qlora_fused_dx(const qlora_nf4_t *W, const uint16_t *dY, int64_t M, const uint16_t *A,
                              int32_t r, const uint16_t *sT, uint16_t *dX, void *ws, size_t ws_bytes,
                              int32_t *dev_status, qlora_stream_t stream);

/* dA = sT^T X ([r, K] fp32) and dB = dY^T sU ([N, r] fp32), both overwritten:
 * the adapter gradients ("QLoRA, in depth", "The mechanism in brief").
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, CUDA. */
qlora_status_t qlora_lora_grads(const uint16_t *X, const uint16_t *dY, int64_t M, int64_t N, int64_t K,
                                const uint16_t *sU, const uint16_t *sT, int32_t r, float *dA, float *dB,
                                void *ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * Fused SwiGLU projection of the Llama-style MLP, h = silu(g) * u with
 * g = X Wg'^T + sU_g B_g^T and u = X Wu'^T + sU_u B_u^T ("QLoRA and Fine-Tuning
 * on One Consumer GPU", section "Where 24 GB goes": adapters on the MLP
 * projections, and gradient checkpointing recomputes a layer's MLP
 * intermediates during the backward). The pages do not define this fusion;
 * it is a kernel of this library that computes the same chain as the separate
 * linears with g and u rounded to bf16 before silu, as the unfused chain does.
 *
 * Layout: Wgu is the NF4 quantisation of [Wg; Wu] with rows interleaved in
 * chunks of 64 (rows 128c..128c+63 = gate rows 64c.., rows 128c+64.. = up rows
 * 64c..), [2F, K] with F % 64 == 0 and K % 64 == 0. Bgu [2F, 2r] bf16 is the
 * block-diagonal up-projection in the same row order (qlora_swiglu_pack_b);
 * sUgu [M, 2r] = [sU_g | sU_u], e.g. qlora_lora_xa with A_gu = [A_g; A_u]
 * [2r, K]. r2 = 2r with 8 <= r2 <= 64, r2 % 8 == 0.
 */

/* H [M, F] bf16 = bf16(silu(bf16(g)) * bf16(u)) in one tcgen05 GEMM over Wgu.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, CUDA. */
qlora_status_t qlora_swiglu_fwd(const qlora_nf4_t *Wgu, const uint16_t *X, int64_t M, const uint16_t *Bgu,
                                int32_t r2, const uint16_t *sUgu, uint16_t *H, int32_t *dev_status,
                                qlora_stream_t stream);

/* Backward through silu(g) * u with g and u recomputed inside the GEMM (they
 * are never stored): dGU [M, 2F] bf16 in Wgu's row order, dg = dH u silu'(g)
 * in gate rows and du = dH silu(g) in up rows (g, u as in qlora_swiglu_fwd).
 * dX then follows from qlora_fused_dx over Wgu with A_gu and sT_gu =
 * qlora_lora_dyb(dGU, Bgu); qlora_lora_grads(X, dGU, sUgu, sTgu) gives
 * [dA_g; dA_u] and a [2F, 2r] dB whose diagonal blocks are dB_g, dB_u
 * (qlora_swiglu_unpack_db). dH [M, F] bf16. Errors: as qlora_swiglu_fwd. */
qlora_status_t qlora_swiglu_bwd(const qlora_nf4_t *Wgu, const uint16_t *X, int64_t M, const uint16_t *Bgu,
                                int32_t r2, const uint16_t *sUgu, const uint16_t *dH, uint16_t *dGU,
                                int32_t *dev_status, qlora_stream_t stream);

/* Bgu [2F, 2r] from B_g, B_u [F, r] (device bf16): gate row [B_g row | 0],
 * up row [0 | B_u row], rows interleaved as in Wgu. F % 64 == 0, 4 <= r <= 32,
 * r % 4 == 0. Errors: INVALID_ARG, UNSUPPORTED_SHAPE, CUDA. */
qlora_status_t qlora_swiglu_pack_b(const uint16_t *Bg, const uint16_t *Bu, int64_t F, int32_t r, uint16_t *Bgu,
                                   qlora_stream_t stream);

/* dB_g, dB_u [F, r] fp32 from the diagonal blocks of dBgu [2F, 2r] fp32.
 * Errors: as qlora_swiglu_pack_b. */
qlora_status_t qlora_swiglu_unpack_db(const float *dBgu, int64_t F, int32_t r, float *dBg, float *dBu,
                                      qlora_stream_t stream);

/* Merge the adapter into the base: out = W' + s B A with W' the dequantised
 * NF4 weight [N, K], A [r, K] and B [N, r] device bf16 ("QLoRA"
 * (guide.dupenodi.dev), section "Walking through the tooling": merge
 * W' = W + scaled BA for serving; "QLoRA, in depth", section "Shipping:
 * merge, re-quantize, verify"). Per element fp32(w') + s * sum_j B A (fp32
 * accumulation), written as bf16 (round to nearest even) when out_f32 == 0 or
 * as fp32 otherwise (the input of a re-quantisation with qlora_nf4_quantize).
 * N % 16 == 0, 1 <= r <= 64, out 16-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, CUDA. */
qlora_status_t qlora_nf4_merge(const qlora_nf4_t *W, const uint16_t *A, const uint16_t *B, int32_t r, float s,
                               void *out, int32_t out_f32, qlora_stream_t stream);

/* One AdamW step (decoupled weight decay) of an adapter parameter with 8-bit
 * optimiser states ("QLoRA, in depth", section "A complete run on a 12
 * GB-class GPU": training uses the paged 8-bit AdamW, which keeps its states in
 * 8 bits; paging is not part of this library). p [n] fp32 master weights,
 * updated in place; p_bf16 [n] or NULL receives bf16_rn(p) for the kernels;
 * grad [n] fp32 (e.g. dA or dB from qlora_lora_grads). States in blocks of 256
 * elements: m_q int8 with m = m_q / 127 * m_scale[block], v_q uint8 codes of
 * sqrt(v) with v = (v_q / 255)^2 * v_scale[block] (a nonzero v keeps a code
 * >= 1); zero-initialised states are the usual start.
 * Per element, in fp32 with every operation rounded once:
 *   m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g g;
 *   p -= lr (m / (1 - b1^t) / (sqrt(v / (1 - b2^t)) + eps) + wd p),
 * then per block m_scale = max |m|, v_scale = max v and the codes are
 * rint(127 m / m_scale) and, for v > 0, clamp(rint(255 sqrt(v / v_scale)),
 * 1, 255) (half to even). step t >= 1.
 * Errors: INVALID_ARG, CUDA. */
qlora_status_t qlora_adamw8_step(float *p, uint16_t *p_bf16, const float *grad, int8_t *m_q, uint8_t *v_q,
                                 float *m_scale, float *v_scale, int64_t n, int32_t step, float lr, float beta1,
                                 float beta2, float eps, float weight_decay, qlora_stream_t stream);

/* The adapter gradients of qlora_lora_grads and, in the same launch, one
 * qlora_adamw8_step of both adapters (the update fused into the gradient
 * epilogue: each gradient tile covers whole 256-element state blocks, so no
 * gradient needs to go through memory). The state of each adapter is kept in
 * the order of its gradient tiles, d-major:
 *   A: p[d * r + j] is A[j][d] (the master copy of A^T, [K, r] flattened),
 *      and so are m_q, v_q (blocks of 256 in that order); p_bf16 is A itself,
 *      [r, K] bf16, written transposed;
 *   B: p[n * r + j] is B[n][j] ([N, r], natural order); p_bf16 is B [N, r].
 * The result is bit for bit that of qlora_lora_grads followed by
 * qlora_adamw8_step on dA^T (A) and dB (B) with these layouts. dA and dB are
 * still written when not NULL (fp32, as qlora_lora_grads). The launch reads
 * X, dY, sU and sT only, so A and B may be updated in place while sU, sT
 * computed from them are its inputs.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, CUDA. */
typedef struct {
  float *p;
  uint16_t *p_bf16;   /* may be NULL */
  int8_t *m_q;
  uint8_t *v_q;
  float *m_scale;
  float *v_scale;
} qlora_adamw8_tensor_t;
qlora_status_t qlora_lora_grads_adamw8(const uint16_t *X, const uint16_t *dY, int64_t M, int64_t N, int64_t K,
                                       const uint16_t *sU, const uint16_t *sT, int32_t r, float *dA, float *dB,
                                       const qlora_adamw8_tensor_t *A_state, const qlora_adamw8_tensor_t *B_state,
                                       int32_t step, float lr, float beta1, float beta2, float eps,
                                       float weight_decay, qlora_stream_t stream);

/*
 * Allocation-free forward. The pages have no counterpart to this call: it is an
 * interface convenience of this library for callers that cannot allocate
 * device memory where they run the layer (a plug-in that only receives its
 * inputs and outputs, a server whose device memory is all handed to a fixed
 * pool up front, code that must not call cudaMalloc between launches because
 * that call can synchronise the device).
 * It validates its arguments exactly as qlora_linear_fwd does, before
 * anything is launched, and then runs the same launches with the same
 * schedule, so its results are bit for bit those of qlora_linear_fwd. Its
 * scratch lives in one 8 MiB array compiled into the library, which every GPU
 * that loads the library holds until the process exits; it calls no
 * allocator. The scratch a call needs (it must fit in 8 MiB, else the call
 * returns QLORA_ERR_WORKSPACE before anything is launched):
 * always a 256-byte counter page, and
 *   M <= 16:       the few-token launch's flags, partial tiles (SM count x 128
 *                  rows x 8 or 16 tokens x 4 bytes), pieces of s X A^T and, when
 *                  sU_out is NULL, sU: about 0.6 to 1.3 MB;
 *   16 < M <= 64:  round_up(M*r*2, 256) when sU_out is NULL, plus the fused
 *                  GEMM's workspace (qlora_fused_workspace(M), about 4.9 MB on
 *                  148 SMs);
 *   M > 64:        round_up(M*r*2, 256) when sU_out is NULL, nothing otherwise.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and caches it; make that
 * first call before any stream capture. The cached address belongs to the
 * device's context: after cudaDeviceReset on a device this call must not be
 * used on that device again in the same process. Every call shares the one
 * array and leaves its contents behind; nothing in it needs to start at zero,
 * but calls whose kernels can overlap on the GPU (other streams, other host
 * threads) race on it, so the caller must serialise them.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, CUDA.
 */
qlora_status_t qlora_linear_fwd_noalloc(const qlora_nf4_t *W, const uint16_t *X, int64_t M,
                                        const uint16_t *A, const uint16_t *B, int32_t r, float s,
                                        uint16_t *Y, uint16_t *sU_out, int32_t *dev_status,
                                        qlora_stream_t stream);

/*
 * Tile schedule of the fused GEMM (qlora_fused_fwd, qlora_fused_dx and the
 * composite calls that run them). Every schedule computes the same result up to
 * fp32 summation order; this is a tuning and testing control.
 *   QLORA_SCHEDULE_AUTO   the library's choice (default): CTA pairs for the
 *                         linear forward and dX at 1024 tokens or more when
 *                         their tiles fill the SM pairs about as well as
 *                         single-CTA tiles fill the SMs (fewer dequantisations
 *                         and activation reads per flop: faster once the board
 *                         is at its power cap); otherwise single-CTA tiles of
 *                         128 weight rows, stream-K for short token tiles
 *   QLORA_SCHEDULE_SINGLE single-CTA tiles only
 *   QLORA_SCHEDULE_PAIR   CTA pairs (cta_group::2, 256 weight rows x 512 tokens
 *                         per pair tile) for the linear forward and dX; the
 *                         SwiGLU modes keep single-CTA tiles
 * The setting is process-wide and is read when a call launches its kernel; set
 * it before launching (not while other host threads launch). Errors:
 * INVALID_ARG for an unknown value.
 */
typedef enum { QLORA_SCHEDULE_AUTO = 0, QLORA_SCHEDULE_SINGLE = 1, QLORA_SCHEDULE_PAIR = 2 } qlora_schedule_t;
qlora_status_t qlora_set_gemm_schedule(int32_t schedule);

/* Failure-path self-test. Every wait inside the kernels of this library is
 * bounded: after about one second without progress the waiting thread stops,
 * the kernel writes QLORA_ERR_TIMEOUT to the device status word and returns,
 * and the CUDA context stays usable. This call launches one CTA whose wait can
 * never complete (an mbarrier nothing arrives on), so that the path can be
 * exercised: after the stream is synchronised, *dev_status (device int32,
 * 4-byte aligned) holds QLORA_ERR_TIMEOUT. It takes about one second of GPU
 * time. Errors: INVALID_ARG, MISALIGNED, CUDA. */
qlora_status_t qlora_selftest_bounded_wait(int32_t *dev_status, qlora_stream_t stream);

/* A static, human-readable name for a status code (host). Interface only:
 * no passage of the pages defines it; it turns the codes above into text for
 * error messages. Never NULL; unknown codes give "QLORA_ERR_UNKNOWN". */
const char *qlora_status_string(qlora_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
