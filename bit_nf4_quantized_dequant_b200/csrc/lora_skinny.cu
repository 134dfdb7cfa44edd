// Skinny LoRA products of the QLoRA linear ("QLoRA, in depth", section "The
// mechanism in brief": the adapter path (alpha / r) B A x; backward gives the
// gradients of A and B). With rank r <= 64 these are thin, memory-bound
// reductions:
//   rows:  out[m, j]  = bf16_rn(s * sum_k Z[m, k] Wl(j, k))   (sU = s X A^T, sT = s dY B)
//   cols:  out(d, j)  = sum_m Z[m, d] V[m, j]                  (dA = sT^T X, dB = dY^T sU)
// "rows" runs on the warp-level bf16 tensor-core MMA (m16n8k16) with the
// adapter weight staged in shared memory; "cols" accumulates in registers with
// packed fp32x2 FMAs. Both split the reduction over CTAs, write fp32 partial
// sums to the caller's workspace and reduce them in a fixed order in a second
// kernel, so results are deterministic.
#include "qlora_device.cuh"

namespace qlora {
namespace {

// ---------------------------------------------------------------------------
// rows: Z[M, K] (bf16) x Wl(j, k) -> part[split][M][r] (fp32)
// ---------------------------------------------------------------------------
constexpr int kRowsWarps = 4;
constexpr int kRowsTile = 16 * kRowsWarps;   // rows per CTA
constexpr int kKC = 256;                     // k per staged chunk
constexpr int kKCPad = kKC + 8;              // smem row pitch (bf16), conflict-free fragment reads

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ldg_u32(const uint16_t *p) {
  return __ldg(reinterpret_cast<const unsigned int *>(p));
}

template <int NT>  // n-tiles of 8 adapter columns: r_pad = 8 * NT
__global__ void __launch_bounds__(32 * kRowsWarps) lora_rows_mma(const uint16_t *__restrict__ Z, int64_t M,
                                                                  int64_t K, const uint16_t *__restrict__ W,
                                                                  int r, int w_is_rk, int64_t k_per_split,
                                                                  float *__restrict__ part) {
  __shared__ __align__(16) uint16_t ws[NT * 8][kKCPad];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kRowsTile + warp * 16;
  const int64_t kbeg = static_cast<int64_t>(blockIdx.y) * k_per_split;
  const int64_t kend = min(K, kbeg + k_per_split);
  const int64_t ra = m0 + g, rb = m0 + g + 8;
  const bool va = ra < M, vb = rb < M;
  const uint16_t *za = Z + (va ? ra : 0) * K;
  const uint16_t *zb = Z + (vb ? rb : 0) * K;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  for (int64_t k0 = kbeg; k0 < kend; k0 += kKC) {
    const int kc = static_cast<int>(kend - k0 < kKC ? kend - k0 : kKC);
    // stage the adapter weight chunk as [j][k] (bf16), zero beyond r and kend
    for (int e = threadIdx.x; e < NT * 8 * (kKC / 8); e += blockDim.x) {
      const int j = e / (kKC / 8), kk = (e % (kKC / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (j < r && kk < kc) {
        if (w_is_rk) {
          if (kk + 8 <= kc) {
            v = __ldg(reinterpret_cast<const uint4 *>(W + static_cast<int64_t>(j) * K + k0 + kk));
          } else {
            uint16_t t8[8];
            for (int q = 0; q < 8; ++q) t8[q] = (kk + q < kc) ? W[static_cast<int64_t>(j) * K + k0 + kk + q] : 0;
            v = *reinterpret_cast<uint4 *>(t8);
          }
        } else {
          uint16_t t8[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) t8[q] = (kk + q < kc) ? W[(k0 + kk + q) * r + j] : 0;
          v = *reinterpret_cast<uint4 *>(t8);
        }
      }
      *reinterpret_cast<uint4 *>(&ws[j][kk]) = v;
    }
    __syncthreads();
    const int nsteps = (kc + 15) / 16;
    // Loads of eight k-steps are issued before their MMAs so that each lane
    // keeps 32 independent loads in flight.
    for (int s0 = 0; s0 < nsteps; s0 += 8) {
      uint32_t a[8][4];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int kk = (s0 + u) * 16;
        const int64_t kg = k0 + kk;
        if (kk + 16 <= kc) {
          a[u][0] = va ? ldg_u32(za + kg + 2 * c) : 0u;
          a[u][1] = vb ? ldg_u32(zb + kg + 2 * c) : 0u;
          a[u][2] = va ? ldg_u32(za + kg + 2 * c + 8) : 0u;
          a[u][3] = vb ? ldg_u32(zb + kg + 2 * c + 8) : 0u;
        } else if (kk < kc) {
          // ragged tail of the reduction (only when kend is not a multiple of 16)
          auto pick = [&](const uint16_t *zr, bool v, int col) -> uint32_t {
            uint32_t lo = (v && kk + col < kc) ? zr[kg + col] : 0u;
            uint32_t hi = (v && kk + col + 1 < kc) ? zr[kg + col + 1] : 0u;
            return lo | (hi << 16);
          };
          a[u][0] = pick(za, va, 2 * c);
          a[u][1] = pick(zb, vb, 2 * c);
          a[u][2] = pick(za, va, 2 * c + 8);
          a[u][3] = pick(zb, vb, 2 * c + 8);
        } else {
          a[u][0] = a[u][1] = a[u][2] = a[u][3] = 0u;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int kk = (s0 + u) * 16;
        if (kk < kc) {
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const uint32_t b0 = *reinterpret_cast<const uint32_t *>(&ws[t * 8 + g][kk + 2 * c]);
            const uint32_t b1 = *reinterpret_cast<const uint32_t *>(&ws[t * 8 + g][kk + 2 * c + 8]);
            mma_bf16_16816(acc[t], a[u], b0, b1);
          }
        }
      }
    }
    __syncthreads();
  }
  float *dst = part + static_cast<int64_t>(blockIdx.y) * M * r;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int j = t * 8 + 2 * c;
    if (va) {
      if (j < r) dst[ra * r + j] = acc[t][0];
      if (j + 1 < r) dst[ra * r + j + 1] = acc[t][1];
    }
    if (vb) {
      if (j < r) dst[rb * r + j] = acc[t][2];
      if (j + 1 < r) dst[rb * r + j + 1] = acc[t][3];
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

// ---------------------------------------------------------------------------
// cols: sum over m of Z[m, d] V[m, j] -> part[split][D][r] (fp32)
// CTA = 8 warps over 128 columns (4 per lane) and 16 adapter columns (grid.z
// picks the 16-wide slice of r); warps stride over the CTA's rows.
// ---------------------------------------------------------------------------
constexpr int kColsWarps = 8;
constexpr int kColsD = 128;
constexpr int kColsRowsMax = 256;   // rows per CTA (V slice staged in smem)

__global__ void __launch_bounds__(32 * kColsWarps) lora_cols_ffma2(const uint16_t *__restrict__ Z, int64_t M,
                                                                    int64_t D, const uint16_t *__restrict__ V,
                                                                    int r, int64_t m_per_split,
                                                                    float *__restrict__ part) {
  extern __shared__ __align__(16) float smem_cols[];
  float *vs = smem_cols;                          // [kColsRowsMax][16]
  float *red = smem_cols + kColsRowsMax * 16;     // [kColsWarps][32 lanes][64]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t d0 = static_cast<int64_t>(blockIdx.x) * kColsD + lane * 4;
  const int j0 = blockIdx.z * 16;
  const int64_t mbeg = static_cast<int64_t>(blockIdx.y) * m_per_split;
  const int64_t mend = min(M, mbeg + m_per_split);
  const int rows = static_cast<int>(mend - mbeg);

#pragma unroll 4
  for (int e = threadIdx.x; e < rows * 16; e += blockDim.x) {
    const int i = e >> 4, j = e & 15;
    vs[e] = (j0 + j < r) ? __uint_as_float(static_cast<uint32_t>(__ldg(V + (mbeg + i) * r + j0 + j)) << 16) : 0.f;
  }
  __syncthreads();

  float2 acc[4][8];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[q][j] = make_float2(0.f, 0.f);

  const bool dok = d0 < D;   // D % 4 == 0, so a lane's 4 columns are all in or all out
  constexpr int kU = 8;      // rows whose loads are in flight together per warp
  for (int i0 = warp; i0 < rows; i0 += kU * kColsWarps) {
    uint2 zw[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kColsWarps;
      zw[u] = (dok && i < rows) ? __ldg(reinterpret_cast<const uint2 *>(Z + (mbeg + i) * D + d0))
                                : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kColsWarps;
      if (i < rows) {
        const float x[4] = {__uint_as_float(zw[u].x << 16), __uint_as_float(zw[u].x & 0xFFFF0000u),
                            __uint_as_float(zw[u].y << 16), __uint_as_float(zw[u].y & 0xFFFF0000u)};
        const float4 *vr = reinterpret_cast<const float4 *>(vs + i * 16);
        float2 v[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float4 t = vr[h];
          v[2 * h] = make_float2(t.x, t.y);
          v[2 * h + 1] = make_float2(t.z, t.w);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 xx = make_float2(x[q], x[q]);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[q][j] = __ffma2_rn(xx, v[j], acc[q][j]);
        }
      }
    }
  }
  // reduce the 8 warps' accumulators in a fixed order
  float *mine = red + (warp * 32 + lane) * 64;
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      mine[q * 16 + 2 * j] = acc[q][j].x;
      mine[q * 16 + 2 * j + 1] = acc[q][j].y;
    }
  __syncthreads();
  float *dst = part + static_cast<int64_t>(blockIdx.y) * D * r;
  for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
    const int ln = e >> 6, qj = e & 63;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kColsWarps; ++w) sum += red[(w * 32 + ln) * 64 + qj];
    const int64_t d = static_cast<int64_t>(blockIdx.x) * kColsD + ln * 4 + (qj >> 4);
    const int j = j0 + (qj & 15);
    if (d < D && j < r) dst[d * r + j] = sum;
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
  const int64_t ctas = (M + kRowsTile - 1) / kRowsTile;
  const int64_t chunks = (K + kKC - 1) / kKC;
  int64_t s = (2 * device_sm_count() + ctas - 1) / ctas;
  if (s > chunks) s = chunks;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

int cols_splits(int64_t M, int64_t D) {
  const int64_t ctas = (D + kColsD - 1) / kColsD;
  const int64_t chunks = (M + kColsRowsMax - 1) / kColsRowsMax;   // at most kColsRowsMax rows per CTA
  int64_t s = (2 * device_sm_count() + ctas - 1) / ctas;
  if (s < chunks) s = chunks;
  const int64_t max_s = (M + 7) / 8;    // keep at least 8 rows per split
  if (s > max_s) s = max_s;
  if (s < chunks) s = chunks;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

size_t cols_smem_bytes() { return (kColsRowsMax * 16 + kColsWarps * 32 * 64) * sizeof(float); }

template <int NT>
cudaError_t rows_launch(dim3 grid, cudaStream_t st, const uint16_t *Z, int64_t M, int64_t K, const uint16_t *W,
                        int r, bool w_is_rk, int64_t kps, float *ws) {
  lora_rows_mma<NT><<<grid, 32 * kRowsWarps, 0, st>>>(Z, M, K, W, r, w_is_rk ? 1 : 0, kps, ws);
  return cudaGetLastError();
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
  const int64_t chunks = (K + kKC - 1) / kKC;
  const int64_t k_per_split = ((chunks + splits - 1) / splits) * kKC;
  const int real_splits = static_cast<int>((K + k_per_split - 1) / k_per_split);
  dim3 grid(static_cast<unsigned>((M + kRowsTile - 1) / kRowsTile), static_cast<unsigned>(real_splits));
  cudaError_t e;
  switch ((r + 7) / 8) {
    case 1: e = rows_launch<1>(grid, st, Z, M, K, W, r, w_is_rk, k_per_split, ws); break;
    case 2: e = rows_launch<2>(grid, st, Z, M, K, W, r, w_is_rk, k_per_split, ws); break;
    case 3: e = rows_launch<3>(grid, st, Z, M, K, W, r, w_is_rk, k_per_split, ws); break;
    case 4: e = rows_launch<4>(grid, st, Z, M, K, W, r, w_is_rk, k_per_split, ws); break;
    case 5: e = rows_launch<5>(grid, st, Z, M, K, W, r, w_is_rk, k_per_split, ws); break;
    case 6: e = rows_launch<6>(grid, st, Z, M, K, W, r, w_is_rk, k_per_split, ws); break;
    case 7: e = rows_launch<7>(grid, st, Z, M, K, W, r, w_is_rk, k_per_split, ws); break;
    case 8: e = rows_launch<8>(grid, st, Z, M, K, W, r, w_is_rk, k_per_split, ws); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const int64_t n = M * r;
  lora_rows_finalize<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(ws, real_splits, n, s, out);
  return cudaGetLastError();
}

cudaError_t launch_lora_cols(const uint16_t *Z, int64_t M, int64_t D, const uint16_t *V, int r,
                             bool transpose_out, float *out, float *ws, size_t ws_floats,
                             cudaStream_t st) {
  const int splits = cols_splits(M, D);
  if (static_cast<size_t>(splits) * D * r > ws_floats) return cudaErrorInvalidValue;
  const int64_t m_per_split = (M + splits - 1) / splits;
  const int real_splits = static_cast<int>((M + m_per_split - 1) / m_per_split);
  const size_t smem = cols_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(lora_cols_ffma2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((D + kColsD - 1) / kColsD), static_cast<unsigned>(real_splits),
            static_cast<unsigned>((r + 15) / 16));
  lora_cols_ffma2<<<grid, 32 * kColsWarps, smem, st>>>(Z, M, D, V, r, m_per_split, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = D * r;
  lora_cols_finalize<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(ws, real_splits, D, r,
                                                                             transpose_out ? 1 : 0, out);
  return cudaGetLastError();
}

}  // namespace qlora
