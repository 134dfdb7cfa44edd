// Skinny LoRA products of the QLoRA linear ("QLoRA, in depth", section "The
// mechanism in brief": the adapter path (alpha / r) B A x; backward gives the
// gradients of A and B). With rank r <= 64 these are thin, memory-bound
// reductions:
//   rows:  out[m, j]  = bf16_rn(s * sum_k Z[m, k] Wl(j, k))   (sU = s X A^T, sT = s dY B)
//   cols:  out(d, j)  = sum_m Z[m, d] V[m, j]                  (dA = sT^T X, dB = dY^T sU)
// Both split the reduction over CTAs, write fp32 partial sums to the caller's
// workspace and reduce them in a fixed order in a second kernel, so results are
// deterministic.
#include "qlora_device.cuh"

namespace qlora {
namespace {

constexpr int kT = 64;  // tile edge

__device__ __forceinline__ void unpack8(uint4 v, float *dst) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    dst[2 * i] = __uint_as_float(w[i] << 16);
    dst[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// part[split][m][j] = sum over this split's k of Z[m, k] Wl(j, k)
__global__ void __launch_bounds__(256) lora_rows_partial(const uint16_t *__restrict__ Z, int64_t M,
                                                         int64_t K, const uint16_t *__restrict__ W, int r,
                                                         int w_is_rk, int64_t k_per_split,
                                                         float *__restrict__ part) {
  __shared__ float zs[kT][kT + 1];
  __shared__ float ws[kT][kT + 1];
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kT;
  const int64_t kbeg = static_cast<int64_t>(blockIdx.y) * k_per_split;
  const int64_t kend = min(K, kbeg + k_per_split);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int nb = (r + 15) >> 4;
  float acc[4][4] = {};
  for (int64_t k0 = kbeg; k0 < kend; k0 += kT) {
    for (int e = threadIdx.x; e < kT * 8; e += 256) {
      const int row = e >> 3, c8 = (e & 7) * 8;
      float tmp[8];
      const int64_t m = m0 + row, k = k0 + c8;
      if (m < M && k + 8 <= kend) {
        unpack8(__ldg(reinterpret_cast<const uint4 *>(Z + m * K + k)), tmp);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) tmp[q] = (m < M && k + q < kend) ? bf16_to_f(Z[m * K + k + q]) : 0.f;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) zs[row][c8 + q] = tmp[q];
    }
    for (int e = threadIdx.x; e < kT * kT; e += 256) {
      const int j = e >> 6, kk = e & 63;
      float v = 0.f;
      if (j < r && k0 + kk < kend)
        v = bf16_to_f(w_is_rk ? W[static_cast<int64_t>(j) * K + k0 + kk] : W[(k0 + kk) * r + j]);
      ws[j][kk] = v;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kT; ++kk) {
      float zv[4], wv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) zv[a] = zs[ty + 16 * a][kk];
#pragma unroll
      for (int b = 0; b < 4; ++b) wv[b] = ws[tx + 16 * b][kk];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(zv[a], wv[b], acc[a][b]);
    }
    __syncthreads();
  }
  float *dst = part + static_cast<int64_t>(blockIdx.y) * M * r;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int64_t m = m0 + ty + 16 * a;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = tx + 16 * b;
      if (m < M && b < nb && j < r) dst[m * r + j] = acc[a][b];
    }
  }
}

__global__ void lora_rows_finalize(const float *__restrict__ part, int splits, int64_t n, float s,
                                   uint16_t *__restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float acc = 0.f;
  for (int q = 0; q < splits; ++q) acc += part[q * n + i];
  out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(s * acc));
}

// part[split][d][j] = sum over this split's m of Z[m, d] V[m, j]
__global__ void __launch_bounds__(256) lora_cols_partial(const uint16_t *__restrict__ Z, int64_t M,
                                                         int64_t D, const uint16_t *__restrict__ V, int r,
                                                         int64_t m_per_split, float *__restrict__ part) {
  __shared__ float zs[kT][kT + 1];   // [m][d]
  __shared__ float vs[kT][kT + 1];   // [m][j]
  const int64_t d0 = static_cast<int64_t>(blockIdx.x) * kT;
  const int64_t mbeg = static_cast<int64_t>(blockIdx.y) * m_per_split;
  const int64_t mend = min(M, mbeg + m_per_split);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int64_t m0 = mbeg; m0 < mend; m0 += kT) {
    for (int e = threadIdx.x; e < kT * 8; e += 256) {
      const int row = e >> 3, c8 = (e & 7) * 8;
      float tmp[8];
      const int64_t m = m0 + row, d = d0 + c8;
      if (m < mend && d + 8 <= D) {
        unpack8(__ldg(reinterpret_cast<const uint4 *>(Z + m * D + d)), tmp);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) tmp[q] = (m < mend && d + q < D) ? bf16_to_f(Z[m * D + d + q]) : 0.f;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) zs[row][c8 + q] = tmp[q];
    }
    for (int e = threadIdx.x; e < kT * kT; e += 256) {
      const int row = e >> 6, j = e & 63;
      const int64_t m = m0 + row;
      vs[row][j] = (m < mend && j < r) ? bf16_to_f(V[m * r + j]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int mm = 0; mm < kT; ++mm) {
      float zv[4], vv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) zv[a] = zs[mm][tx + 16 * a];
#pragma unroll
      for (int b = 0; b < 4; ++b) vv[b] = vs[mm][ty + 16 * b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(zv[a], vv[b], acc[a][b]);
    }
    __syncthreads();
  }
  float *dst = part + static_cast<int64_t>(blockIdx.y) * D * r;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int64_t d = d0 + tx + 16 * a;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = ty + 16 * b;
      if (d < D && j < r) dst[d * r + j] = acc[a][b];
    }
  }
}

__global__ void lora_cols_finalize(const float *__restrict__ part, int splits, int64_t D, int r,
                                   int transpose_out, float *__restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n = D * r;
  if (i >= n) return;
  float acc = 0.f;
  for (int q = 0; q < splits; ++q) acc += part[q * n + i];
  if (transpose_out) {
    const int64_t d = i / r, j = i % r;
    out[j * D + d] = acc;
  } else {
    out[i] = acc;
  }
}

int rows_splits(int64_t M, int64_t K) {
  const int64_t ctas = (M + kT - 1) / kT;
  const int64_t chunks = (K + kT - 1) / kT;
  int64_t s = (2 * device_sm_count() + ctas - 1) / ctas;
  if (s > chunks) s = chunks;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

int cols_splits(int64_t M, int64_t D) {
  const int64_t ctas = (D + kT - 1) / kT;
  const int64_t chunks = (M + kT - 1) / kT;
  int64_t s = (2 * device_sm_count() + ctas - 1) / ctas;
  if (s > chunks) s = chunks;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

}  // namespace

size_t lora_rows_ws_floats(int64_t M, int64_t K, int r) {
  return static_cast<size_t>(rows_splits(M, K)) * M * r;
}
size_t lora_cols_ws_floats(int64_t M, int64_t D, int r) {
  return static_cast<size_t>(cols_splits(M, D)) * D * r;
}

cudaError_t launch_lora_rows(const uint16_t *Z, int64_t M, int64_t K, const uint16_t *W, int r,
                             bool w_is_rk, float s, uint16_t *out, float *ws, size_t ws_floats,
                             cudaStream_t st) {
  const int splits = rows_splits(M, K);
  if (static_cast<size_t>(splits) * M * r > ws_floats) return cudaErrorInvalidValue;
  const int64_t chunks = (K + kT - 1) / kT;
  const int64_t k_per_split = ((chunks + splits - 1) / splits) * kT;
  const int real_splits = static_cast<int>((K + k_per_split - 1) / k_per_split);
  dim3 grid(static_cast<unsigned>((M + kT - 1) / kT), static_cast<unsigned>(real_splits));
  lora_rows_partial<<<grid, 256, 0, st>>>(Z, M, K, W, r, w_is_rk ? 1 : 0, k_per_split, ws);
  const int64_t n = M * r;
  lora_rows_finalize<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(ws, real_splits, n, s, out);
  return cudaGetLastError();
}

cudaError_t launch_lora_cols(const uint16_t *Z, int64_t M, int64_t D, const uint16_t *V, int r,
                             bool transpose_out, float *out, float *ws, size_t ws_floats,
                             cudaStream_t st) {
  const int splits = cols_splits(M, D);
  if (static_cast<size_t>(splits) * D * r > ws_floats) return cudaErrorInvalidValue;
  const int64_t chunks = (M + kT - 1) / kT;
  const int64_t m_per_split = ((chunks + splits - 1) / splits) * kT;
  const int real_splits = static_cast<int>((M + m_per_split - 1) / m_per_split);
  dim3 grid(static_cast<unsigned>((D + kT - 1) / kT), static_cast<unsigned>(real_splits));
  lora_cols_partial<<<grid, 256, 0, st>>>(Z, M, D, V, r, m_per_split, ws);
  const int64_t n = D * r;
  lora_cols_finalize<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(ws, real_splits, D, r,
                                                                             transpose_out ? 1 : 0, out);
  return cudaGetLastError();
}

}  // namespace qlora
