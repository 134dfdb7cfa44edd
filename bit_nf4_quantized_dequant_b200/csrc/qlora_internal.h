// Declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace qlora {

constexpr int kBlock = 64;    // weights per first-level block
constexpr int kGroup = 256;   // blocks per second-level group

// Kernel launchers. Each returns the cudaError_t of the launch.
// book: 0 = NF4, 1 = the evenly spaced int4 comparison codebook.
// dq: 0 = linear 8-bit second level (scale2: one float per group), 1 = E4M3
// codes of mean-centred constants (scale2: d, mu per group; NF4 book only).
cudaError_t launch_quantize(const float *W, int64_t rows, int64_t cols, uint8_t *codes,
                            uint8_t *scale8, float *scale2, int32_t *dev_status, cudaStream_t s, int book = 0,
                            int dq = 0);
cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scale8, const float *scale2,
                              int64_t rows, int64_t cols, uint16_t *out, cudaStream_t s, int book = 0, int dq = 0);

// Fused NF4 GEMM (tcgen05). Mode FWD: Y[M,N] = X[M,K] W'^T + sU[M,r] Bl^T.
// Mode DX: dX[M,K] = dY[M,N] W' + sT[M,r] Al.
// SwiGLU modes (W = [Wg; Wu] interleaved in 64-row chunks, N = 2F): the FWD
// product G|U, then 2: out = H[M,F] = bf16(silu(g) u); 3: out = dGU[M,N] with
// dg = dH u silu'(g) in gate rows and du = dH silu(g) in up rows (aux = dH[M,F]).
struct GemmArgs {
  int mode;                 // 0 = FWD, 1 = DX, 2 = SwiGLU FWD, 3 = SwiGLU BWD
  const uint8_t *codes;
  const uint8_t *scale8;
  const float *scale2;
  int64_t N, K, M;
  int r;
  const uint16_t *act;      // X (FWD) or dY (DX), [M, K] or [M, N]
  const uint16_t *lora_w;   // B [N, r] (FWD) or A [r, K] (DX)
  const uint16_t *lora_act; // sU or sT [M, r]
  uint16_t *out;            // Y [M, N] or dX [M, K]
  int32_t *dev_status;
  void *ws;                 // optional stream-K workspace (fused_gemm_ws_bytes(M) bytes), or null
  const uint16_t *aux;      // dH [M, N/2] for mode 3
};
cudaError_t launch_fused_gemm(const GemmArgs &a, cudaStream_t s);
// Workspace of a stream-K launch with M tokens on the current device.
size_t fused_gemm_ws_bytes(int64_t M);

// Forward for M <= 16 tokens: dequantisation into warp-MMA register fragments,
// K split over a thread-block cluster. Same result definition as the FWD mode
// of the fused GEMM (fp32 accumulation, bf16 output).
bool gemv_fwd_supported(int64_t N, int64_t K, int64_t M);
// Exactly one of sU (precomputed bf16(s X A^T)) and Al (the adapter A [r, K],
// with s; the kernel then forms sU itself and writes it to sU_out if given).
cudaError_t launch_nf4_gemv_fwd(const uint8_t *codes, const uint8_t *scale8, const float *scale2, int64_t N,
                                int64_t K, int64_t M, const uint16_t *X, const uint16_t *Bl, const uint16_t *sU,
                                const uint16_t *Al, float s, uint16_t *sU_out, int r, uint16_t *Y,
                                cudaStream_t st);

}  // namespace qlora

#include "qlora.h"

namespace qlora {
// W' + s B A (bf16 or fp32 out), see nf4_merge.cu.
cudaError_t launch_nf4_merge(const uint8_t *codes, const uint8_t *scale8, const float *scale2, int64_t N, int64_t K,
                             const uint16_t *Al, const uint16_t *Bl, int r, float s, void *out, bool f32_out,
                             cudaStream_t st);

// AdamW with 8-bit states (blocks of 256), see adamw8.cu.
cudaError_t launch_adamw8(float *p, uint16_t *p_bf16, const float *grad, int8_t *mq, uint8_t *vq, float *mscale,
                          float *vscale, int64_t n, int step, float lr, float beta1, float beta2, float eps, float wd,
                          cudaStream_t st);

// SwiGLU layout helpers (see swiglu_pack.cu).
cudaError_t launch_swiglu_pack_b(const uint16_t *Bg, const uint16_t *Bu, int64_t F, int r, uint16_t *Bgu,
                                 cudaStream_t st);
cudaError_t launch_swiglu_unpack_db(const float *dBgu, int64_t F, int r, float *dBg, float *dBu, cudaStream_t st);

// The linear forward split into its validation (everything qlora_linear_fwd
// checks before it launches anything), the scratch it needs when sU is or is
// not kept by the caller, and the launches (see api.cu).
qlora_status_t linear_fwd_check(const qlora_nf4_t *W, const uint16_t *X, int64_t M, const uint16_t *A,
                                const uint16_t *B, int32_t r, float s, const uint16_t *Y, const uint16_t *sU_out,
                                const int32_t *dev_status);
size_t linear_fwd_scratch_bytes(int64_t M, int64_t N, int64_t K, int32_t r, bool keep_su);
qlora_status_t linear_fwd_run(const qlora_nf4_t *W, const uint16_t *X, int64_t M, const uint16_t *A,
                              const uint16_t *B, int32_t r, float s, uint16_t *Y, uint16_t *sU_out,
                              void *counters, uint16_t *su_scratch, void *gemm_ws, size_t gemm_ws_bytes,
                              int32_t *dev_status, qlora_stream_t stream);

// Skinny LoRA products (fp32 accumulation).
// out[m, j] = bf16_rn(s * sum_k Z[m, k] * Wl(j, k)); Wl(j, k) = W[j*K + k] if
// w_is_rk else W[k*r + j].
cudaError_t launch_lora_rows(const uint16_t *Z, int64_t M, int64_t K, const uint16_t *W, int r,
                             bool w_is_rk, float s, uint16_t *out, float *ws, size_t ws_floats,
                             cudaStream_t st);
// Adapter gradients in one launch: dA[j, k] = sum_m sT[m, j] X[m, k] and
// dB[n, j] = sum_m dY[m, n] sU[m, j] (fp32, overwritten).
struct AdamFuseArgs;
cudaError_t launch_lora_grads(const uint16_t *X, const uint16_t *dY, int64_t M, int64_t N, int64_t K,
                              const uint16_t *sU, const uint16_t *sT, int r, float *dA, float *dB, cudaStream_t st,
                              const AdamFuseArgs *adam = nullptr);
size_t lora_rows_ws_floats(int64_t M, int64_t K, int r);
size_t lora_cols_ws_floats(int64_t M, int64_t D, int r);

int device_sm_count();

// Token counts up to which the forward streams the weight (nf4_small_m.cu).
constexpr int64_t kSmallM = 16;

// Few-token forward (M <= 16) of one or more linears in one persistent launch
// (see nf4_small_m.cu). Exactly one of A (the kernel then forms
// sU = bf16(s X A^T), written to sU_out when given) and sU_in per linear.
struct SmallProblem {
  const uint8_t *codes;
  const uint8_t *scale8;
  const float *scale2;
  int64_t N, K;
  const uint16_t *X, *A, *B, *sU_in;
  int r;
  float s;
  uint16_t *Y, *sU_out;
};
// Workspace bytes of launch_small_m for these linears (on the current device),
// besides its counter page: kSmallCounterBytes that must be zero before the
// first launch and that every launch leaves zero (nothing else may write them).
constexpr size_t kSmallCounterBytes = 256;
size_t small_m_ws_bytes(const SmallProblem *pr, int count, int64_t M);
// One launch per 16 linears, in order on `st`; with pdl the launch may start
// streaming the weights before the preceding work on the stream has finished.
cudaError_t launch_small_m(const SmallProblem *pr, int count, int64_t M, void *ws, void *counters, bool pdl,
                           int32_t *status, cudaStream_t st);

// One CTA whose bounded mbarrier wait runs out (failure-path self-test).
cudaError_t launch_bounded_wait_selftest(int32_t *status, cudaStream_t st);

// Fused-GEMM tile schedule (qlora_schedule_t values), process-wide.
void set_gemm_schedule(int schedule);
int gemm_schedule();

}  // namespace qlora
