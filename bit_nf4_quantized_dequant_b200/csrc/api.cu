// The C ABI of libqlora (declared in include/qlora.h): argument validation,
// workspace layout, tensor-map encoding and kernel launches. Nothing here
// allocates device memory or synchronises.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "qlora.h"
#include "qlora_device.cuh"
#include "adamw8.cuh"
#include "qlora_internal.h"

namespace qlora {

namespace {
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
std::once_flag g_encode_once;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
}  // namespace

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle) {
  if (!encode_fn()) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D tiled map: dims[0] innermost (contiguous), strides[i] = bytes between
// consecutive indices of dimension i + 1 (any order).
bool encode_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, const uint64_t dims[3],
               const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swizzle) {
  if (!encode_fn()) return false;
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t st[2] = {strides[0], strides[1]};
  cuuint32_t b[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, dtype, 3, const_cast<void *>(base), d, st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Workspace of the few-token forward of one [N, K] linear of rank r that forms
// sU itself and keeps it in the workspace (the largest case).
static size_t small_fwd_ws_bytes(int64_t M, int64_t N, int64_t K, int r) {
  SmallProblem p{};
  p.N = N;
  p.K = K;
  p.r = r;
  p.A = reinterpret_cast<const uint16_t *>(16);   // only "given / not given" matters here
  return small_m_ws_bytes(&p, 1, M);
}
// ... and of the few-token qlora_fused_fwd, which is given sU.
static size_t small_fused_ws_bytes(int64_t M) {
  SmallProblem p{};
  p.N = 16;
  p.K = 64;
  p.r = 8;
  return small_m_ws_bytes(&p, 1, M);
}

// The optional workspace of qlora_fused_fwd / qlora_fused_dx: the few-token
// launch's counter page, then the stream-K partials of the GEMM or, for a few
// tokens, the persistent forward's partials.
static size_t fused_ws_bytes(int64_t M) {
  const size_t g = fused_gemm_ws_bytes(M);
  if (M > kSmallM) return kSmallCounterBytes + g;
  const size_t sm = small_fused_ws_bytes(M);
  return kSmallCounterBytes + (sm > g ? sm : g);
}

// Workspace layout of the linear calls (offsets in bytes, 256-byte aligned):
//   [counter page of the few-token forward (zero between calls)]
//   [sU scratch: M*r bf16][sT: M*r bf16][fp32 partial sums of the skinny products]
//   [stream-K workspace of the fused GEMMs, or the few-token forward's partials]
struct WsLayout {
  size_t cnt, su, st, part, part_floats, gemm, gemm_bytes, total;
};

static WsLayout ws_layout(int64_t M, int64_t N, int64_t K, int r) {
  WsLayout w{};
  const size_t mr = round_up(static_cast<size_t>(M) * r * 2, 256);
  w.cnt = 0;
  w.su = kSmallCounterBytes;
  w.st = w.su + mr;
  w.part = w.st + mr;
  size_t f = lora_rows_ws_floats(M, K, r);
  f = f > lora_rows_ws_floats(M, N, r) ? f : lora_rows_ws_floats(M, N, r);
  f = f > lora_cols_ws_floats(M, K, r) ? f : lora_cols_ws_floats(M, K, r);
  f = f > lora_cols_ws_floats(M, N, r) ? f : lora_cols_ws_floats(M, N, r);
  w.part_floats = f;
  w.gemm = w.part + round_up(f * 4, 256);
  w.gemm_bytes = fused_ws_bytes(M);   // the workspace of qlora_fused_fwd / qlora_fused_dx
  if (M <= kSmallM) {   // the few-token forward uses this region instead (with the page at w.cnt)
    const size_t sm = small_fwd_ws_bytes(M, N, K, r);
    w.gemm_bytes = sm > w.gemm_bytes ? sm : w.gemm_bytes;
  }
  w.total = w.gemm + round_up(w.gemm_bytes, 256);
  return w;
}

static qlora_status_t check_nf4(const qlora_nf4_t *q) {
  if (!q || !q->codes || !q->scale8 || !q->scale2) return QLORA_ERR_INVALID_ARG;
  if (q->rows <= 0 || q->cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (q->cols % kBlock) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q->codes)) return QLORA_ERR_MISALIGNED;
  // scale8 / scale2 are read element-wise by the kernels: natural alignment suffices
  if (reinterpret_cast<uintptr_t>(q->scale2) & 3u) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

static qlora_status_t check_linear(const qlora_nf4_t *W, const uint16_t *X, int64_t M, const uint16_t *A,
                                   const uint16_t *B, int32_t r, float s) {
  qlora_status_t st = check_nf4(W);
  if (st != QLORA_OK) return st;
  if (!X || !A || !B || M <= 0) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(s)) return QLORA_ERR_INVALID_ARG;
  if (r < 8 || r > 64 || (r % 8)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (W->rows % 16) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t(1) << 31) || W->rows > (int64_t(1) << 31) || W->cols > (int64_t(1) << 31))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

static qlora_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

qlora_status_t linear_fwd_check(const qlora_nf4_t *W, const uint16_t *X, int64_t M, const uint16_t *A,
                                const uint16_t *B, int32_t r, float s, const uint16_t *Y, const uint16_t *sU_out,
                                const int32_t *dev_status) {
  qlora_status_t st = check_linear(W, X, M, A, B, r, s);
  if (st != QLORA_OK) return st;
  if (!Y) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(Y) || (sU_out && !aligned16(sU_out))) return QLORA_ERR_MISALIGNED;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

size_t linear_fwd_scratch_bytes(int64_t M, int64_t N, int64_t K, int32_t r, bool keep_su) {
  if (M <= kSmallM) {
    SmallProblem p{};
    p.N = N;
    p.K = K;
    p.r = r;
    p.A = reinterpret_cast<const uint16_t *>(16);
    p.sU_out = keep_su ? reinterpret_cast<uint16_t *>(16) : nullptr;
    return kSmallCounterBytes + small_m_ws_bytes(&p, 1, M);
  }
  size_t b = kSmallCounterBytes + (keep_su ? 0 : round_up(static_cast<size_t>(M) * r * 2, 256));
  if (M <= 64) b += round_up(fused_ws_bytes(M), 256);   // the stream-K schedule of short token tiles
  return b;
}

// The forward after validation. su_scratch: [M, r] bf16 for sU when sU_out is
// NULL and M > kSmallM; gemm_ws: the fused GEMM's workspace (M > kSmallM) or
// the few-token launch's (M <= kSmallM).
qlora_status_t linear_fwd_run(const qlora_nf4_t *W, const uint16_t *X, int64_t M, const uint16_t *A,
                              const uint16_t *B, int32_t r, float s, uint16_t *Y, uint16_t *sU_out,
                              void *counters, uint16_t *su_scratch, void *gemm_ws, size_t gemm_ws_bytes,
                              int32_t *dev_status, qlora_stream_t stream) {
  const int64_t N = W->rows, K = W->cols;
  if (M <= kSmallM) {
    SmallProblem p{};
    p.codes = W->codes;
    p.scale8 = W->scale8;
    p.scale2 = W->scale2;
    p.N = N;
    p.K = K;
    p.X = X;
    p.A = A;
    p.B = B;
    p.r = r;
    p.s = s;
    p.Y = Y;
    p.sU_out = sU_out;
    if (!gemm_ws || gemm_ws_bytes < small_m_ws_bytes(&p, 1, M)) return QLORA_ERR_WORKSPACE;
    return cuda_status(
        launch_small_m(&p, 1, M, gemm_ws, counters, false, dev_status, reinterpret_cast<cudaStream_t>(stream)));
  }
  uint16_t *sU = sU_out ? sU_out : su_scratch;
  qlora_status_t st = qlora_lora_xa(X, M, K, A, r, s, sU, nullptr, 0, stream);
  if (st != QLORA_OK) return st;
  return qlora_fused_fwd(W, X, M, B, r, sU, Y, gemm_ws, gemm_ws_bytes, dev_status, stream);
}

}  // namespace qlora

using namespace qlora;

extern "C" {

qlora_status_t qlora_nf4_sizes(int64_t rows, int64_t cols, size_t *codes_bytes, size_t *scale8_bytes,
                               size_t *scale2_bytes) {
  if (!codes_bytes || !scale8_bytes || !scale2_bytes || rows <= 0 || cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (cols % kBlock) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const size_t n = static_cast<size_t>(rows) * static_cast<size_t>(cols);
  const size_t nb = n / kBlock;
  *codes_bytes = n / 2;
  *scale8_bytes = nb;
  *scale2_bytes = 4 * ((nb + kGroup - 1) / kGroup);
  return QLORA_OK;
}

qlora_status_t qlora_nf4_codebook(float *out) {
  if (!out) return QLORA_ERR_INVALID_ARG;
  static const float levels[16] = QLORA_NF4_LEVELS;
  std::memcpy(out, levels, sizeof(levels));
  return QLORA_OK;
}

qlora_status_t qlora_nf4_quantize(const float *W, const qlora_nf4_t *q, int32_t *dev_status,
                                  qlora_stream_t stream) {
  qlora_status_t st = check_nf4(q);
  if (st != QLORA_OK) return st;
  if (!W) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return QLORA_ERR_MISALIGNED;
  return cuda_status(launch_quantize(W, q->rows, q->cols, q->codes, q->scale8, q->scale2, dev_status,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_nf4_dequantize(const qlora_nf4_t *q, uint16_t *out, qlora_stream_t stream) {
  qlora_status_t st = check_nf4(q);
  if (st != QLORA_OK) return st;
  if (!out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(out)) return QLORA_ERR_MISALIGNED;
  return cuda_status(launch_dequantize(q->codes, q->scale8, q->scale2, q->rows, q->cols, out,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_codec_levels(int32_t codebook, float *out) {
  if (!out) return QLORA_ERR_INVALID_ARG;
  static const float nf4[16] = QLORA_NF4_LEVELS;
  static const float int4[16] = QLORA_INT4_LEVELS;
  if (codebook == QLORA_CODEBOOK_NF4) std::memcpy(out, nf4, sizeof(nf4));
  else if (codebook == QLORA_CODEBOOK_INT4) std::memcpy(out, int4, sizeof(int4));
  else return QLORA_ERR_INVALID_ARG;
  return QLORA_OK;
}

qlora_status_t qlora_codec_quantize(const float *W, const qlora_nf4_t *q, int32_t codebook, int32_t *dev_status,
                                    qlora_stream_t stream) {
  if (codebook != QLORA_CODEBOOK_NF4 && codebook != QLORA_CODEBOOK_INT4) return QLORA_ERR_INVALID_ARG;
  qlora_status_t st = check_nf4(q);
  if (st != QLORA_OK) return st;
  if (!W) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return QLORA_ERR_MISALIGNED;
  return cuda_status(launch_quantize(W, q->rows, q->cols, q->codes, q->scale8, q->scale2, dev_status,
                                     reinterpret_cast<cudaStream_t>(stream), codebook));
}

qlora_status_t qlora_codec_dequantize(const qlora_nf4_t *q, int32_t codebook, uint16_t *out, qlora_stream_t stream) {
  if (codebook != QLORA_CODEBOOK_NF4 && codebook != QLORA_CODEBOOK_INT4) return QLORA_ERR_INVALID_ARG;
  qlora_status_t st = check_nf4(q);
  if (st != QLORA_OK) return st;
  if (!out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(out)) return QLORA_ERR_MISALIGNED;
  return cuda_status(launch_dequantize(q->codes, q->scale8, q->scale2, q->rows, q->cols, out,
                                       reinterpret_cast<cudaStream_t>(stream), codebook));
}

qlora_status_t qlora_dqfp8_sizes(int64_t rows, int64_t cols, size_t *codes_b, size_t *s8_b, size_t *s2_b) {
  qlora_status_t st = qlora_nf4_sizes(rows, cols, codes_b, s8_b, s2_b);
  if (st == QLORA_OK && s2_b) *s2_b *= 2;   // (d, mu) per group
  return st;
}

qlora_status_t qlora_dqfp8_quantize(const float *W, const qlora_nf4_t *q, int32_t *dev_status,
                                    qlora_stream_t stream) {
  qlora_status_t st = check_nf4(q);
  if (st != QLORA_OK) return st;
  if (!W) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(q->scale2) & 7u) return QLORA_ERR_MISALIGNED;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return QLORA_ERR_MISALIGNED;
  return cuda_status(launch_quantize(W, q->rows, q->cols, q->codes, q->scale8, q->scale2, dev_status,
                                     reinterpret_cast<cudaStream_t>(stream), QLORA_CODEBOOK_NF4, 1));
}

qlora_status_t qlora_dqfp8_dequantize(const qlora_nf4_t *q, uint16_t *out, qlora_stream_t stream) {
  qlora_status_t st = check_nf4(q);
  if (st != QLORA_OK) return st;
  if (!out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(out)) return QLORA_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(q->scale2) & 7u) return QLORA_ERR_MISALIGNED;
  return cuda_status(launch_dequantize(q->codes, q->scale8, q->scale2, q->rows, q->cols, out,
                                       reinterpret_cast<cudaStream_t>(stream), QLORA_CODEBOOK_NF4, 1));
}

qlora_status_t qlora_linear_workspace(int64_t M, int64_t N, int64_t K, int32_t r, size_t *bytes) {
  if (!bytes || M <= 0 || N <= 0 || K <= 0) return QLORA_ERR_INVALID_ARG;
  if (K % kBlock || N % 16 || r < 8 || r > 64 || r % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  *bytes = ws_layout(M, N, K, r).total;
  return QLORA_OK;
}

qlora_status_t qlora_lora_xa(const uint16_t *X, int64_t M, int64_t K, const uint16_t *A, int32_t r,
                             float s, uint16_t *sU, void *ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!X || !A || !sU || M <= 0 || K <= 0 || !std::isfinite(s)) return QLORA_ERR_INVALID_ARG;
  if (K % kBlock || r < 8 || r > 64 || r % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(A) || !aligned16(sU) || (ws && !aligned16(ws))) return QLORA_ERR_MISALIGNED;
  const size_t need = lora_rows_ws_floats(M, K, r) * 4;
  if (need > 0 && (!ws || ws_bytes < need)) return QLORA_ERR_WORKSPACE;
  return cuda_status(launch_lora_rows(X, M, K, A, r, /*w_is_rk=*/true, s, sU, static_cast<float *>(ws),
                                      ws_bytes / 4, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_lora_dyb(const uint16_t *dY, int64_t M, int64_t N, const uint16_t *B, int32_t r,
                              float s, uint16_t *sT, void *ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!dY || !B || !sT || M <= 0 || N <= 0 || !std::isfinite(s)) return QLORA_ERR_INVALID_ARG;
  if (N % 16 || r < 8 || r > 64 || r % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(dY) || !aligned16(B) || !aligned16(sT) || (ws && !aligned16(ws))) return QLORA_ERR_MISALIGNED;
  const size_t need = lora_rows_ws_floats(M, N, r) * 4;
  if (need > 0 && (!ws || ws_bytes < need)) return QLORA_ERR_WORKSPACE;
  return cuda_status(launch_lora_rows(dY, M, N, B, r, /*w_is_rk=*/false, s, sT, static_cast<float *>(ws),
                                      ws_bytes / 4, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_fused_workspace(int64_t M, size_t *bytes) {
  if (!bytes || M < 1) return QLORA_ERR_INVALID_ARG;
  *bytes = fused_ws_bytes(M);
  return QLORA_OK;
}

static qlora_status_t fused(int mode, const qlora_nf4_t *W, const uint16_t *act, int64_t M,
                            const uint16_t *lora_w, int32_t r, const uint16_t *lora_act, uint16_t *out,
                            void *ws, size_t ws_bytes, int32_t *dev_status, qlora_stream_t stream) {
  qlora_status_t st = check_linear(W, act, M, lora_w, lora_w, r, 1.0f);
  if (st != QLORA_OK) return st;
  if (!lora_act || !out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(lora_act) || !aligned16(out) || (ws && !aligned16(ws))) return QLORA_ERR_MISALIGNED;
  if (ws && ws_bytes < fused_ws_bytes(M)) return QLORA_ERR_WORKSPACE;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return QLORA_ERR_MISALIGNED;
  GemmArgs g{};
  g.mode = mode;
  g.codes = W->codes;
  g.scale8 = W->scale8;
  g.scale2 = W->scale2;
  g.N = W->rows;
  g.K = W->cols;
  g.M = M;
  g.r = r;
  g.act = act;
  g.lora_w = lora_w;
  g.lora_act = lora_act;
  g.out = out;
  g.dev_status = dev_status;
  g.ws = ws ? static_cast<uint8_t *>(ws) + kSmallCounterBytes : nullptr;
  if (mode == 0 && M <= kSmallM && ws && W->rows <= INT32_MAX && W->cols <= INT32_MAX) {
    // a few tokens with a workspace: the persistent weight-streaming launch
    SmallProblem p{};
    p.codes = W->codes;
    p.scale8 = W->scale8;
    p.scale2 = W->scale2;
    p.N = W->rows;
    p.K = W->cols;
    p.X = act;
    p.B = lora_w;
    p.sU_in = lora_act;
    p.r = r;
    p.Y = out;
    return cuda_status(launch_small_m(&p, 1, M, static_cast<uint8_t *>(ws) + kSmallCounterBytes, ws, false,
                                      dev_status, reinterpret_cast<cudaStream_t>(stream)));
  }
  if (mode == 0 && gemv_fwd_supported(W->rows, W->cols, M))   // a few tokens, no workspace: one cluster launch
    return cuda_status(launch_nf4_gemv_fwd(W->codes, W->scale8, W->scale2, W->rows, W->cols, M, act, lora_w,
                                           lora_act, nullptr, 0.f, nullptr, r, out,
                                           reinterpret_cast<cudaStream_t>(stream)));
  return cuda_status(launch_fused_gemm(g, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_fused_fwd(const qlora_nf4_t *W, const uint16_t *X, int64_t M, const uint16_t *B,
                               int32_t r, const uint16_t *sU, uint16_t *Y, void *ws, size_t ws_bytes,
                               int32_t *dev_status, qlora_stream_t stream) {
  return fused(0, W, X, M, B, r, sU, Y, ws, ws_bytes, dev_status, stream);
}

qlora_status_t qlora_fused_dx(const qlora_nf4_t *W, const uint16_t *dY, int64_t M, const uint16_t *A,
                              int32_t r, const uint16_t *sT, uint16_t *dX, void *ws, size_t ws_bytes,
                              int32_t *dev_status, qlora_stream_t stream) {
  return fused(1, W, dY, M, A, r, sT, dX, ws, ws_bytes, dev_status, stream);
}

qlora_status_t qlora_lora_grads(const uint16_t *X, const uint16_t *dY, int64_t M, int64_t N, int64_t K,
                                const uint16_t *sU, const uint16_t *sT, int32_t r, float *dA, float *dB,
                                void *ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!X || !dY || !sU || !sT || !dA || !dB || M <= 0 || N <= 0 || K <= 0) return QLORA_ERR_INVALID_ARG;
  if (K % kBlock || N % 16 || r < 8 || r > 64 || r % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(sU) || !aligned16(sT) || !aligned16(dA) ||
      !aligned16(dB) || (ws && !aligned16(ws)))
    return QLORA_ERR_MISALIGNED;
  const size_t fa = lora_cols_ws_floats(M, K, r), fb = lora_cols_ws_floats(M, N, r);
  const size_t need = 4 * (fa > fb ? fa : fb);
  if (need > 0 && (!ws || ws_bytes < need)) return QLORA_ERR_WORKSPACE;
  return cuda_status(launch_lora_grads(X, dY, M, N, K, sU, sT, r, dA, dB, reinterpret_cast<cudaStream_t>(stream)));
}

static bool adam_tensor_ok(const qlora_adamw8_tensor_t *t) {
  return t && t->p && t->m_q && t->v_q && t->m_scale && t->v_scale;
}

qlora_status_t qlora_lora_grads_adamw8(const uint16_t *X, const uint16_t *dY, int64_t M, int64_t N, int64_t K,
                                       const uint16_t *sU, const uint16_t *sT, int32_t r, float *dA, float *dB,
                                       const qlora_adamw8_tensor_t *A_state, const qlora_adamw8_tensor_t *B_state,
                                       int32_t step, float lr, float beta1, float beta2, float eps,
                                       float weight_decay, qlora_stream_t stream) {
  if (!X || !dY || !sU || !sT || M <= 0 || N <= 0 || K <= 0) return QLORA_ERR_INVALID_ARG;
  if (!adam_tensor_ok(A_state) || !adam_tensor_ok(B_state)) return QLORA_ERR_INVALID_ARG;
  if (step < 1 || !std::isfinite(lr) || !(eps > 0.f) || !std::isfinite(weight_decay) ||
      !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f))
    return QLORA_ERR_INVALID_ARG;
  if (K % kBlock || N % 16 || r < 8 || r > 64 || r % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(sU) || !aligned16(sT) || (dA && !aligned16(dA)) ||
      (dB && !aligned16(dB)))
    return QLORA_ERR_MISALIGNED;
  qlora::AdamFuseArgs a{};
  a.A = {A_state->p, A_state->m_q, A_state->v_q, A_state->m_scale, A_state->v_scale};
  a.B = {B_state->p, B_state->m_q, B_state->v_q, B_state->m_scale, B_state->v_scale};
  a.A_bf16 = A_state->p_bf16;
  a.B_bf16 = B_state->p_bf16;
  a.step = step;
  a.lr = lr;
  a.beta1 = beta1;
  a.beta2 = beta2;
  a.eps = eps;
  a.wd = weight_decay;
  return cuda_status(launch_lora_grads(X, dY, M, N, K, sU, sT, r, dA, dB, reinterpret_cast<cudaStream_t>(stream), &a));
}

qlora_status_t qlora_linear_fwd(const qlora_nf4_t *W, const uint16_t *X, int64_t M, const uint16_t *A,
                                const uint16_t *B, int32_t r, float s, uint16_t *Y, uint16_t *sU_out,
                                void *ws, size_t ws_bytes, int32_t *dev_status, qlora_stream_t stream) {
  qlora_status_t st = linear_fwd_check(W, X, M, A, B, r, s, Y, sU_out, dev_status);
  if (st != QLORA_OK) return st;
  const int64_t N = W->rows, K = W->cols;
  const WsLayout L = ws_layout(M, N, K, r);
  if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  return linear_fwd_run(W, X, M, A, B, r, s, Y, sU_out, wsb + L.cnt, reinterpret_cast<uint16_t *>(wsb + L.su),
                        wsb + L.gemm, L.gemm_bytes, dev_status, stream);
}

qlora_status_t qlora_linear_fwd_group_workspace(const qlora_linear_problem_t *problems, int32_t count, int64_t M,
                                                size_t *bytes) {
  if (!problems || !bytes || count < 1 || M < 1) return QLORA_ERR_INVALID_ARG;
  if (M > kSmallM) return QLORA_ERR_UNSUPPORTED_SHAPE;
  std::vector<SmallProblem> pr(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    const qlora_linear_problem_t &q = problems[i];
    if (q.W.rows <= 0 || q.W.cols <= 0) return QLORA_ERR_INVALID_ARG;
    if (q.W.cols % kBlock || q.r < 8 || q.r > 64 || q.r % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
    pr[i].N = q.W.rows;
    pr[i].K = q.W.cols;
    pr[i].r = q.r;
    pr[i].A = q.A;
    pr[i].sU_out = q.sU_out;
  }
  *bytes = kSmallCounterBytes + small_m_ws_bytes(pr.data(), count, M);
  return QLORA_OK;
}

qlora_status_t qlora_linear_fwd_group(const qlora_linear_problem_t *problems, int32_t count, int64_t M, int32_t flags,
                                      void *ws, size_t ws_bytes, int32_t *dev_status, qlora_stream_t stream) {
  if (!problems || count < 1 || M < 1) return QLORA_ERR_INVALID_ARG;
  if (M > kSmallM) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (flags & ~QLORA_FWD_OVERLAP_PREVIOUS) return QLORA_ERR_INVALID_ARG;
  std::vector<SmallProblem> pr(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    const qlora_linear_problem_t &q = problems[i];
    qlora_status_t st = linear_fwd_check(&q.W, q.X, M, q.A, q.B, q.r, q.s, q.Y, q.sU_out, dev_status);
    if (st != QLORA_OK) return st;
    if (q.W.rows > INT32_MAX || q.W.cols > INT32_MAX) return QLORA_ERR_UNSUPPORTED_SHAPE;
    SmallProblem &p = pr[i];
    p.codes = q.W.codes;
    p.scale8 = q.W.scale8;
    p.scale2 = q.W.scale2;
    p.N = q.W.rows;
    p.K = q.W.cols;
    p.X = q.X;
    p.A = q.A;
    p.B = q.B;
    p.r = q.r;
    p.s = q.s;
    p.Y = q.Y;
    p.sU_out = q.sU_out;
  }
  if (!ws || ws_bytes < kSmallCounterBytes + small_m_ws_bytes(pr.data(), count, M)) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  return cuda_status(launch_small_m(pr.data(), count, M, static_cast<uint8_t *>(ws) + kSmallCounterBytes, ws,
                                    (flags & QLORA_FWD_OVERLAP_PREVIOUS) != 0, dev_status,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_linear_bwd(const qlora_nf4_t *W, const uint16_t *X, int64_t M, const uint16_t *A,
                                const uint16_t *B, int32_t r, float s, const uint16_t *dY,
                                const uint16_t *sU_in, uint16_t *dX, float *dA, float *dB, void *ws,
                                size_t ws_bytes, int32_t *dev_status, qlora_stream_t stream) {
  qlora_status_t st = check_linear(W, X, M, A, B, r, s);
  if (st != QLORA_OK) return st;
  if (!dY || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(dA) || !aligned16(dB) || (dX && !aligned16(dX)) ||
      (sU_in && !aligned16(sU_in)))
    return QLORA_ERR_MISALIGNED;
  const int64_t N = W->rows, K = W->cols;
  const WsLayout L = ws_layout(M, N, K, r);
  if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  uint16_t *sT = reinterpret_cast<uint16_t *>(wsb + L.st);
  void *part = wsb + L.part;
  const size_t part_bytes = L.part_floats * 4;
  const uint16_t *sU = sU_in;
  if (!sU) {
    uint16_t *su_ws = reinterpret_cast<uint16_t *>(wsb + L.su);
    st = qlora_lora_xa(X, M, K, A, r, s, su_ws, part, part_bytes, stream);
    if (st != QLORA_OK) return st;
    sU = su_ws;
  }
  st = qlora_lora_dyb(dY, M, N, B, r, s, sT, part, part_bytes, stream);
  if (st != QLORA_OK) return st;
  if (dX) {
    st = qlora_fused_dx(W, dY, M, A, r, sT, dX, wsb + L.gemm, L.gemm_bytes, dev_status, stream);
    if (st != QLORA_OK) return st;
  }
  return qlora_lora_grads(X, dY, M, N, K, sU, sT, r, dA, dB, part, part_bytes, stream);
}

static qlora_status_t check_swiglu(const qlora_nf4_t *Wgu, const uint16_t *X, int64_t M, const uint16_t *Bgu,
                                   int32_t r2, const uint16_t *sUgu, const uint16_t *out) {
  qlora_status_t st = check_linear(Wgu, X, M, Bgu, Bgu, r2, 1.0f);
  if (st != QLORA_OK) return st;
  if (!sUgu || !out) return QLORA_ERR_INVALID_ARG;
  if (Wgu->rows % 128 || r2 % 2) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(sUgu) || !aligned16(out)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

static qlora_status_t swiglu_launch(int mode, const qlora_nf4_t *Wgu, const uint16_t *X, int64_t M,
                                   const uint16_t *Bgu, int32_t r2, const uint16_t *sUgu, const uint16_t *dH,
                                   uint16_t *out, int32_t *dev_status, qlora_stream_t stream) {
  GemmArgs g{};
  g.mode = mode;
  g.codes = Wgu->codes;
  g.scale8 = Wgu->scale8;
  g.scale2 = Wgu->scale2;
  g.N = Wgu->rows;
  g.K = Wgu->cols;
  g.M = M;
  g.r = r2;
  g.act = X;
  g.lora_w = Bgu;
  g.lora_act = sUgu;
  g.out = out;
  g.dev_status = dev_status;
  g.aux = dH;
  return cuda_status(launch_fused_gemm(g, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_swiglu_fwd(const qlora_nf4_t *Wgu, const uint16_t *X, int64_t M, const uint16_t *Bgu,
                                int32_t r2, const uint16_t *sUgu, uint16_t *H, int32_t *dev_status,
                                qlora_stream_t stream) {
  qlora_status_t st = check_swiglu(Wgu, X, M, Bgu, r2, sUgu, H);
  if (st != QLORA_OK) return st;
  return swiglu_launch(2, Wgu, X, M, Bgu, r2, sUgu, nullptr, H, dev_status, stream);
}

qlora_status_t qlora_swiglu_bwd(const qlora_nf4_t *Wgu, const uint16_t *X, int64_t M, const uint16_t *Bgu,
                                int32_t r2, const uint16_t *sUgu, const uint16_t *dH, uint16_t *dGU,
                                int32_t *dev_status, qlora_stream_t stream) {
  qlora_status_t st = check_swiglu(Wgu, X, M, Bgu, r2, sUgu, dGU);
  if (st != QLORA_OK) return st;
  if (!dH) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dH)) return QLORA_ERR_MISALIGNED;
  return swiglu_launch(3, Wgu, X, M, Bgu, r2, sUgu, dH, dGU, dev_status, stream);
}

qlora_status_t qlora_swiglu_pack_b(const uint16_t *Bg, const uint16_t *Bu, int64_t F, int32_t r, uint16_t *Bgu,
                                   qlora_stream_t stream) {
  if (!Bg || !Bu || !Bgu || F <= 0) return QLORA_ERR_INVALID_ARG;
  if (F % 64 || r < 4 || r > 32 || r % 4) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return cuda_status(launch_swiglu_pack_b(Bg, Bu, F, r, Bgu, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_swiglu_unpack_db(const float *dBgu, int64_t F, int32_t r, float *dBg, float *dBu,
                                      qlora_stream_t stream) {
  if (!dBgu || !dBg || !dBu || F <= 0) return QLORA_ERR_INVALID_ARG;
  if (F % 64 || r < 4 || r > 32 || r % 4) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return cuda_status(launch_swiglu_unpack_db(dBgu, F, r, dBg, dBu, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_nf4_merge(const qlora_nf4_t *W, const uint16_t *A, const uint16_t *B, int32_t r, float s,
                               void *out, int32_t out_f32, qlora_stream_t stream) {
  qlora_status_t st = check_nf4(W);
  if (st != QLORA_OK) return st;
  if (!A || !B || !out || !std::isfinite(s)) return QLORA_ERR_INVALID_ARG;
  if (W->rows % 16 || r < 1 || r > 64) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(out)) return QLORA_ERR_MISALIGNED;
  return cuda_status(launch_nf4_merge(W->codes, W->scale8, W->scale2, W->rows, W->cols, A, B, r, s, out,
                                      out_f32 != 0, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_adamw8_step(float *p, uint16_t *p_bf16, const float *grad, int8_t *m_q, uint8_t *v_q,
                                 float *m_scale, float *v_scale, int64_t n, int32_t step, float lr, float beta1,
                                 float beta2, float eps, float weight_decay, qlora_stream_t stream) {
  if (!p || !grad || !m_q || !v_q || !m_scale || !v_scale || n <= 0 || step < 1) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(lr) || !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps > 0.f) ||
      !std::isfinite(weight_decay))
    return QLORA_ERR_INVALID_ARG;
  return cuda_status(launch_adamw8(p, p_bf16, grad, m_q, v_q, m_scale, v_scale, n, step, lr, beta1, beta2, eps,
                                   weight_decay, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_selftest_bounded_wait(int32_t *dev_status, qlora_stream_t stream) {
  if (!dev_status) return QLORA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(dev_status) & 3u) return QLORA_ERR_MISALIGNED;
  return cuda_status(qlora::launch_bounded_wait_selftest(dev_status, reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status_t qlora_set_gemm_schedule(int32_t schedule) {
  if (schedule < QLORA_SCHEDULE_AUTO || schedule > QLORA_SCHEDULE_PAIR) return QLORA_ERR_INVALID_ARG;
  qlora::set_gemm_schedule(schedule);
  return QLORA_OK;
}

const char *qlora_status_string(qlora_status_t status) {
  switch (status) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "QLORA_ERR_UNSUPPORTED_SHAPE";
    case QLORA_ERR_MISALIGNED: return "QLORA_ERR_MISALIGNED";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE";
    case QLORA_ERR_NONFINITE: return "QLORA_ERR_NONFINITE";
    case QLORA_ERR_TIMEOUT: return "QLORA_ERR_TIMEOUT";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
  }
  return "QLORA_ERR_UNKNOWN";
}

}  // extern "C"
