// Skinny LoRA products of the QLoRA linear ("QLoRA, in depth", section "The
// mechanism in brief": the adapter path (alpha / r) B A x; backward gives the
// gradients of A and B). With rank r <= 64 these are thin, memory-bound
// reductions over a long dimension:
//   rows:  out[m, j]  = bf16_rn(s * sum_k Z[m, k] Wl(j, k))   (sU = s X A^T, sT = s dY B)
//   cols:  out(d, j)  = sum_m Z[m, d] V[m, j]                  (dA = sT^T X, dB = dY^T sU)
// Both stream Z through a TMA ring (one producer thread keeps several 8-16 KiB
// tiles in flight per CTA), build bf16 tensor-core fragments with ldmatrix and
// accumulate with the warp-level MMA (m16n8k16, fp32). The reduction dimension
// is split over the CTAs of one thread-block cluster; each CTA leaves its fp32
// partial tile in shared memory and the cluster adds the partials through
// distributed shared memory in rank order, so no scratch memory is used and
// the result is deterministic.
#include <cuda.h>

#include "adamw8.cuh"
#include "qlora_device.cuh"

namespace qlora {

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

namespace {

constexpr int kStages = 6;       // rows ring depth
constexpr int kStagesCols = 4;   // cols ring depth (two CTAs fit per SM)
constexpr int kClusterMax = 8;
constexpr uint32_t kSpanZ = 128;   // Z tiles: 64 bf16 per row, SWIZZLE_128B

CUtensorMapSwizzle swizzle_for_span(int span) {
  return span == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                    : (span == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

__device__ __forceinline__ void producer_drain(uint64_t *full, uint32_t mask, uint32_t par) {
  for (int s = 0; s < kStages; ++s) {
    if (!(mask & (1u << s))) continue;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(&full[s], (par >> s) & 1u) && global_timer_ns() - t0 < kWaitLimitNs) {
    }
  }
}

// ---------------------------------------------------------------------------
// rows: 64 rows of Z per CTA (4 consumer warps x 16 rows) + 1 producer warp.
// Stage = Z tile [64 m][64 k] (SW128) + adapter tile for the same 64 k:
//   w_is_rk (W is [r, K]):  [r_pad j][64 k], SW128
//   otherwise (W is [K, r]): [64 k][r_pad j], swizzle span 2 * r_pad
// ---------------------------------------------------------------------------
template <int NT>   // n-tiles of 8 adapter columns: r_pad = 8 * NT (16, 32 or 64)
__global__ void __launch_bounds__(160) lora_rows_kernel(const __grid_constant__ CUtensorMap tm_z,
                                                        const __grid_constant__ CUtensorMap tm_w, int64_t M,
                                                        int64_t K, int r, int w_is_rk, int kb_per_cta, float s,
                                                        uint16_t *__restrict__ out, int32_t *status) {
  constexpr int r_pad = NT * 8;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr uint32_t z_bytes = 64 * 128;
  constexpr uint32_t w_bytes = r_pad * 128;   // 64 k x r_pad j x 2 B
  constexpr uint32_t stage_bytes = z_bytes + ((w_bytes + 1023u) & ~1023u);
  float *red = reinterpret_cast<float *>(base + kStages * stage_bytes);   // [64][r_pad]
  uint64_t *full = reinterpret_cast<uint64_t *>(red + 64 * r_pad);
  uint64_t *empty = full + kStages;
  int *abort_flag_p = reinterpret_cast<int *>(empty + kStages);
  volatile int *abort_flag = abort_flag_p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int csize = static_cast<int>(gridDim.y);
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int kb_begin = static_cast<int>(blockIdx.y) * kb_per_cta;
  const int kb_total = static_cast<int>((K + 63) / 64);
  const int kb_end = kb_begin + kb_per_cta < kb_total ? kb_begin + kb_per_cta : kb_total;
  const int nsteps = kb_end > kb_begin ? kb_end - kb_begin : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    *abort_flag_p = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == 4) {
    if (elect_one()) {
      tma_prefetch_desc(&tm_z);
      tma_prefetch_desc(&tm_w);
      uint32_t mask = 0, par = 0;
      int slot = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nsteps; ++i) {
        if (!mbar_wait(&empty[slot], ph ^ 1u, abort_flag, status)) break;
        uint8_t *st = base + slot * stage_bytes;
        mbar_arrive_expect_tx(&full[slot], z_bytes + w_bytes);
        const int k0 = (kb_begin + i) * 64;
        tma_load_2d(st, &tm_z, &full[slot], k0, static_cast<int32_t>(m0));
        if (w_is_rk) tma_load_2d(st + z_bytes, &tm_w, &full[slot], k0, 0);
        else         tma_load_2d(st + z_bytes, &tm_w, &full[slot], 0, k0);
        mask |= 1u << slot;
        par = (par & ~(1u << slot)) | (ph << slot);
        if (++slot == kStages) { slot = 0; ph ^= 1u; }
      }
      if (*abort_flag) producer_drain(full, mask, par);
    }
  } else {
    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    const uint32_t wspan = w_is_rk ? 128u : static_cast<uint32_t>(2 * r_pad);
    int slot = 0;
    uint32_t ph = 0;
    for (int i = 0; i < nsteps; ++i) {
      if (!mbar_wait(&full[slot], ph, abort_flag, status)) break;
      const uint32_t zs = smem_u32(base + slot * stage_bytes);
      const uint32_t wsm = zs + z_bytes;
#pragma unroll
      for (int kk = 0; kk < 64; kk += 16) {
        uint32_t a[4];
        {
          const uint32_t row = static_cast<uint32_t>(warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8);
          const uint32_t chunk = static_cast<uint32_t>(kk / 8 + (lane >> 4));
          ldmatrix_x4(a, zs + swizzle_off(row * 128u + chunk * 16u, kSpanZ));
        }
#pragma unroll
        for (int t = 0; t < NT; t += 2) {
          uint32_t b[4];
          if (w_is_rk) {
            // tile [j][k]: matrices (j-tile t, k chunk c), (t, c+1), (t+1, c), (t+1, c+1)
            const uint32_t j = static_cast<uint32_t>(8 * (t + (lane >> 4)) + (lane & 7));
            const uint32_t chunk = static_cast<uint32_t>(kk / 8 + ((lane >> 3) & 1));
            ldmatrix_x4(b, wsm + swizzle_off(j * 128u + chunk * 16u, wspan));
          } else {
            // tile [k][j], transposed 8x8 loads: (k rows kk.., j-tile t), (kk+8.., t), (kk.., t+1), (kk+8.., t+1)
            const uint32_t krow = static_cast<uint32_t>(kk + (lane & 7) + ((lane >> 3) & 1) * 8);
            const uint32_t chunk = static_cast<uint32_t>(t + (lane >> 4));
            ldmatrix_x4_trans(b, wsm + swizzle_off(krow * wspan + chunk * 16u, wspan));
          }
          mma_16816(acc[t], a, b[0], b[1]);
          mma_16816(acc[t + 1], a, b[2], b[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (++slot == kStages) { slot = 0; ph ^= 1u; }
    }
    // this CTA's partial sums -> shared memory (row-major [64][r_pad])
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int row = warp * 16 + g, col = t * 8 + 2 * c;
      red[row * r_pad + col] = acc[t][0];
      red[row * r_pad + col + 1] = acc[t][1];
      red[(row + 8) * r_pad + col] = acc[t][2];
      red[(row + 8) * r_pad + col + 1] = acc[t][3];
    }
  }
  // add the cluster's partials in rank order: rank q owns rows [q*64/csize, ..)
  cluster_sync_all();
  const int rows_per = (64 + csize - 1) / csize;
  const int r_lo = static_cast<int>(rank) * rows_per;
  const int r_hi = r_lo + rows_per < 64 ? r_lo + rows_per : 64;
  const uint32_t red_addr = smem_u32(red);
  for (int e = threadIdx.x; e < (r_hi - r_lo) * r; e += blockDim.x) {
    const int row = r_lo + e / r, j = e % r;
    const int64_t m = m0 + row;
    if (m >= M) continue;
    const uint32_t off = static_cast<uint32_t>((row * r_pad + j) * 4);
    float sum = 0.f;
    for (int q = 0; q < csize; ++q) sum += ld_dsmem_f32(mapa_shared(red_addr + off, static_cast<uint32_t>(q)));
    out[m * r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(s * sum));
  }
  cluster_sync_all();
}

// ---------------------------------------------------------------------------
// cols: 128 columns of Z per CTA (8 consumer warps x 16 columns) + 1 producer
// warp. Stage = Z tile [64 m][128 d] as two SW128 boxes of 64 columns, and the
// V tile [64 m][r_pad j] (swizzle span 2 * r_pad). One launch serves two
// products (dA = sT^T X with transposed output, dB = dY^T sU): CTAs with
// blockIdx.x < tiles0 take the first, the rest the second.
// ---------------------------------------------------------------------------
struct ColsProblem {
  int64_t D;
  float *out;          // may be NULL when the gradients feed the fused AdamW step only
  int transpose_out;
};

// The 8-bit AdamW step fused into the epilogue. A CTA's tile holds the
// gradients of 128 consecutive d for every j < r, so in the d-major order
// (element d * r + j) it is r / 2 whole state blocks of 256: product 0's state
// is kept for A^T (A's master copy flattened as [K, r]), product 1's for B
// ([N, r], its natural order). bf16 copies go to A [r, K] and B [N, r], the
// operands the kernels read.
struct AdamFuse {
  Adam8Tensor t[2];
  uint16_t *bf16[2];
  AdamArgs a;
};

template <int NT, bool kAdam>
__global__ void __launch_bounds__(288) lora_cols_kernel(const __grid_constant__ CUtensorMap tm_z0,
                                                        const __grid_constant__ CUtensorMap tm_v0,
                                                        const __grid_constant__ CUtensorMap tm_z1,
                                                        const __grid_constant__ CUtensorMap tm_v1, ColsProblem p0,
                                                        ColsProblem p1, int tiles0, int64_t M, int r,
                                                        int mb_per_cta, int32_t *status, AdamFuse af) {
  constexpr int r_pad = NT * 8;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr uint32_t z_bytes = 2 * 64 * 128;    // two boxes of [64 m][64 d]
  constexpr uint32_t v_bytes = r_pad * 128;     // [64 m][r_pad] bf16
  constexpr uint32_t stage_bytes = z_bytes + ((v_bytes + 1023u) & ~1023u);
  constexpr uint32_t vspan = 2 * r_pad;
  float *red = reinterpret_cast<float *>(base + kStagesCols * stage_bytes);   // [128][r_pad]
  uint64_t *full = reinterpret_cast<uint64_t *>(red + 128 * r_pad);
  uint64_t *empty = full + kStagesCols;
  int *abort_flag_p = reinterpret_cast<int *>(empty + kStagesCols);
  volatile int *abort_flag = abort_flag_p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int csize = static_cast<int>(gridDim.y);
  const bool second = static_cast<int>(blockIdx.x) >= tiles0;
  const CUtensorMap *tm_z = second ? &tm_z1 : &tm_z0;
  const CUtensorMap *tm_v = second ? &tm_v1 : &tm_v0;
  const ColsProblem pr = second ? p1 : p0;
  const int64_t d0 = static_cast<int64_t>(second ? static_cast<int>(blockIdx.x) - tiles0 : static_cast<int>(blockIdx.x)) * 128;
  const int mb_begin = static_cast<int>(blockIdx.y) * mb_per_cta;
  const int mb_total = static_cast<int>((M + 63) / 64);
  const int mb_end = mb_begin + mb_per_cta < mb_total ? mb_begin + mb_per_cta : mb_total;
  const int nsteps = mb_end > mb_begin ? mb_end - mb_begin : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesCols; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 8);
    }
    *abort_flag_p = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == 8) {
    if (elect_one()) {
      tma_prefetch_desc(tm_z);
      tma_prefetch_desc(tm_v);
      uint32_t mask = 0, par = 0;
      int slot = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nsteps; ++i) {
        if (!mbar_wait(&empty[slot], ph ^ 1u, abort_flag, status)) break;
        uint8_t *st = base + slot * stage_bytes;
        mbar_arrive_expect_tx(&full[slot], z_bytes + v_bytes);
        const int mrow = (mb_begin + i) * 64;
        tma_load_2d(st, tm_z, &full[slot], static_cast<int32_t>(d0), mrow);
        tma_load_2d(st + 64 * 128, tm_z, &full[slot], static_cast<int32_t>(d0 + 64), mrow);
        tma_load_2d(st + z_bytes, tm_v, &full[slot], 0, mrow);
        mask |= 1u << slot;
        par = (par & ~(1u << slot)) | (ph << slot);
        if (++slot == kStagesCols) { slot = 0; ph ^= 1u; }
      }
      if (*abort_flag) {
        for (int q = 0; q < kStagesCols; ++q) {
          if (!(mask & (1u << q))) continue;
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(&full[q], (par >> q) & 1u) && global_timer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else {
    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    // warp w: columns 16w..16w+15 = box w/4, 16-column group w%4 inside the box
    const uint32_t box_off = static_cast<uint32_t>((warp >> 2) * 64 * 128);
    const uint32_t dchunk0 = static_cast<uint32_t>((warp & 3) * 2);
    int slot = 0;
    uint32_t ph = 0;
    for (int i = 0; i < nsteps; ++i) {
      if (!mbar_wait(&full[slot], ph, abort_flag, status)) break;
      const uint32_t zs = smem_u32(base + slot * stage_bytes) + box_off;
      const uint32_t vs = smem_u32(base + slot * stage_bytes) + z_bytes;
#pragma unroll
      for (int mm = 0; mm < 64; mm += 16) {
        uint32_t a[4];   // Z^T fragment: rows = 16 columns d, cols = 16 rows m
        {
          const uint32_t mrow = static_cast<uint32_t>(mm + (lane & 7) + ((lane >> 4) & 1) * 8);
          const uint32_t chunk = dchunk0 + static_cast<uint32_t>((lane >> 3) & 1);
          ldmatrix_x4_trans(a, zs + swizzle_off(mrow * 128u + chunk * 16u, kSpanZ));
        }
#pragma unroll
        for (int t = 0; t < NT; t += 2) {
          uint32_t b[4];
          const uint32_t mrow = static_cast<uint32_t>(mm + (lane & 7) + ((lane >> 3) & 1) * 8);
          const uint32_t chunk = static_cast<uint32_t>(t + (lane >> 4));
          ldmatrix_x4_trans(b, vs + swizzle_off(mrow * vspan + chunk * 16u, vspan));
          mma_16816(acc[t], a, b[0], b[1]);
          mma_16816(acc[t + 1], a, b[2], b[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (++slot == kStagesCols) { slot = 0; ph ^= 1u; }
    }
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int row = warp * 16 + g, col = t * 8 + 2 * c;
      red[row * r_pad + col] = acc[t][0];
      red[row * r_pad + col + 1] = acc[t][1];
      red[(row + 8) * r_pad + col] = acc[t][2];
      red[(row + 8) * r_pad + col + 1] = acc[t][3];
    }
  }
  cluster_sync_all();
  const uint32_t red_addr = smem_u32(red);
  if constexpr (kAdam) {
    // whole state blocks, one warp each, spread over the cluster's CTAs; the
    // gradient of each element is summed over the partials in rank order, as below
    const int which = second ? 1 : 0;
    const Adam8Tensor t = af.t[which];
    uint16_t *const pb = af.bf16[which];
    const int64_t n = pr.D * r;
    const int tile_blocks = (128 * r) / kStateBlock;
    const int64_t blk0 = d0 * r / kStateBlock;
    const int nwarps = static_cast<int>(blockDim.x >> 5);
    for (int bk = static_cast<int>(rank) * nwarps + warp; bk < tile_blocks; bk += csize * nwarps) {
      const int64_t blk = blk0 + bk;
      if (blk * kStateBlock >= n) break;
      float g[8], pn[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int il = bk * kStateBlock + e * 32 + lane;
        const int row = il / r, j = il % r;
        const int64_t d = d0 + row;
        g[e] = 0.f;
        if (d < pr.D) {
          const uint32_t off = static_cast<uint32_t>((row * r_pad + j) * 4);
          float sum = 0.f;
          for (int q = 0; q < csize; ++q) sum += ld_dsmem_f32(mapa_shared(red_addr + off, static_cast<uint32_t>(q)));
          g[e] = sum;
          if (pr.out) {
            if (pr.transpose_out) pr.out[static_cast<int64_t>(j) * pr.D + d] = sum;
            else                  pr.out[d * r + j] = sum;
          }
        }
      }
      adamw8_block(t, blk, n, g, af.a, pn);
      if (pb) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int il = bk * kStateBlock + e * 32 + lane;
          const int row = il / r, j = il % r;
          const int64_t d = d0 + row;
          if (d < pr.D) {
            const int64_t o = which == 0 ? static_cast<int64_t>(j) * pr.D + d : d * r + j;
            pb[o] = __bfloat16_as_ushort(__float2bfloat16_rn(pn[e]));
          }
        }
      }
    }
    cluster_sync_all();
    return;
  }
  const int rows_per = (128 + csize - 1) / csize;
  const int r_lo = static_cast<int>(rank) * rows_per;
  const int r_hi = r_lo + rows_per < 128 ? r_lo + rows_per : 128;
  for (int e = threadIdx.x; e < (r_hi - r_lo) * r; e += blockDim.x) {
    const int row = r_lo + e / r, j = e % r;
    const int64_t d = d0 + row;
    if (d >= pr.D) continue;
    const uint32_t off = static_cast<uint32_t>((row * r_pad + j) * 4);
    float sum = 0.f;
    for (int q = 0; q < csize; ++q) sum += ld_dsmem_f32(mapa_shared(red_addr + off, static_cast<uint32_t>(q)));
    if (pr.transpose_out) pr.out[static_cast<int64_t>(j) * pr.D + d] = sum;
    else                  pr.out[d * r + j] = sum;
  }
  cluster_sync_all();
}

int pad_rank(int r) { return r <= 16 ? 16 : (r <= 32 ? 32 : 64); }

size_t rows_smem(int r_pad) {
  const size_t stage = 64 * 128 + ((static_cast<size_t>(r_pad) * 128 + 1023) & ~size_t(1023));
  return 1024 + kStages * stage + 64 * r_pad * 4 + 2 * kStages * 8 + 16;
}
size_t cols_smem(int r_pad) {
  const size_t stage = 2 * 64 * 128 + ((static_cast<size_t>(r_pad) * 128 + 1023) & ~size_t(1023));
  return 1024 + kStagesCols * stage + 128 * r_pad * 4 + 2 * kStagesCols * 8 + 16;
}

// Cluster size for splitting a reduction of `blocks` 64-wide steps when
// `tiles` CTAs already cover the output: as many CTAs as are resident at once
// (`per_sm` per SM, set by shared memory), never a second partial wave.
int cluster_split(int64_t tiles, int64_t blocks, int per_sm) {
  int64_t c = static_cast<int64_t>(per_sm) * device_sm_count() / tiles;
  if (c > kClusterMax) c = kClusterMax;
  if (c > blocks) c = blocks;
  if (c < 1) c = 1;
  return static_cast<int>(c);
}

template <typename Kernel>
cudaError_t launch_cluster(Kernel kernel, dim3 grid, int threads, size_t smem, cudaStream_t st, int csize,
                           void **args) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(csize);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, reinterpret_cast<const void *>(kernel), args);
}

}  // namespace

// The skinny products keep their partial sums in shared memory: no workspace.
size_t lora_rows_ws_floats(int64_t, int64_t, int) { return 0; }
size_t lora_cols_ws_floats(int64_t, int64_t, int) { return 0; }

cudaError_t launch_lora_rows(const uint16_t *Z, int64_t M, int64_t K, const uint16_t *W, int r, bool w_is_rk,
                             float s, uint16_t *out, float *, size_t, cudaStream_t st) {
  const int r_pad = pad_rank(r);
  CUtensorMap tm_z, tm_w;
  bool ok = encode_2d(&tm_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Z, K, M, K * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (w_is_rk) ok &= encode_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, K, r, K * 2, 64, r_pad,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  else         ok &= encode_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, r, K, r * 2, r_pad, 64,
                               swizzle_for_span(2 * r_pad));
  if (!ok) return cudaErrorInvalidValue;
  const int64_t mtiles = (M + 63) / 64;
  const int64_t kblocks = (K + 63) / 64;
  const int csize = cluster_split(mtiles, kblocks, static_cast<int>((228 * 1024) / (rows_smem(r_pad) + 1024)));
  int kb_per_cta = static_cast<int>((kblocks + csize - 1) / csize);
  int w_rk = w_is_rk ? 1 : 0;
  int32_t *status = nullptr;
  int64_t Mv = M, Kv = K;
  int rv = r;
  float sv = s;
  void *args[] = {&tm_z, &tm_w, &Mv, &Kv, &rv, &w_rk, &kb_per_cta, &sv, &out, &status};
  const dim3 grid(static_cast<unsigned>(mtiles), static_cast<unsigned>(csize));
  const size_t smem = rows_smem(r_pad);
  switch (r_pad / 8) {
    case 2: return launch_cluster(lora_rows_kernel<2>, grid, 160, smem, st, csize, args);
    case 4: return launch_cluster(lora_rows_kernel<4>, grid, 160, smem, st, csize, args);
    case 8: return launch_cluster(lora_rows_kernel<8>, grid, 160, smem, st, csize, args);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_lora_grads(const uint16_t *X, const uint16_t *dY, int64_t M, int64_t N, int64_t K,
                              const uint16_t *sU, const uint16_t *sT, int r, float *dA, float *dB, cudaStream_t st,
                              const AdamFuseArgs *adam) {
  const int r_pad = pad_rank(r);
  CUtensorMap tz0, tv0, tz1, tv1;
  // product 0: dA[j, k] = sum_m sT[m, j] X[m, k]  (D = K, transposed output)
  // product 1: dB[n, j] = sum_m dY[m, n] sU[m, j] (D = N)
  bool ok = encode_2d(&tz0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_2d(&tv0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sT, r, M, r * 2, r_pad, 64, swizzle_for_span(2 * r_pad));
  ok &= encode_2d(&tz1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, N, M, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_2d(&tv1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sU, r, M, r * 2, r_pad, 64, swizzle_for_span(2 * r_pad));
  if (!ok) return cudaErrorInvalidValue;
  const int tiles0 = static_cast<int>((K + 127) / 128);
  const int tiles1 = static_cast<int>((N + 127) / 128);
  const int64_t mblocks = (M + 63) / 64;
  const int csize = cluster_split(tiles0 + tiles1, mblocks, static_cast<int>((228 * 1024) / (cols_smem(r_pad) + 1024)));
  int mb_per_cta = static_cast<int>((mblocks + csize - 1) / csize);
  ColsProblem p0{K, dA, 1}, p1{N, dB, 0};
  int t0v = tiles0;
  int64_t Mv = M;
  int rv = r;
  int32_t *status = nullptr;
  AdamFuse af{};
  if (adam) {
    af.t[0] = adam->A;
    af.t[1] = adam->B;
    af.bf16[0] = adam->A_bf16;
    af.bf16[1] = adam->B_bf16;
    af.a = make_adam_args(adam->step, adam->lr, adam->beta1, adam->beta2, adam->eps, adam->wd);
  }
  void *args[] = {&tz0, &tv0, &tz1, &tv1, &p0, &p1, &t0v, &Mv, &rv, &mb_per_cta, &status, &af};
  const dim3 grid(static_cast<unsigned>(tiles0 + tiles1), static_cast<unsigned>(csize));
  const size_t smem = cols_smem(r_pad);
  switch ((r_pad / 8) * 2 + (adam ? 1 : 0)) {
    case 4: return launch_cluster(lora_cols_kernel<2, false>, grid, 288, smem, st, csize, args);
    case 5: return launch_cluster(lora_cols_kernel<2, true>, grid, 288, smem, st, csize, args);
    case 8: return launch_cluster(lora_cols_kernel<4, false>, grid, 288, smem, st, csize, args);
    case 9: return launch_cluster(lora_cols_kernel<4, true>, grid, 288, smem, st, csize, args);
    case 16: return launch_cluster(lora_cols_kernel<8, false>, grid, 288, smem, st, csize, args);
    case 17: return launch_cluster(lora_cols_kernel<8, true>, grid, 288, smem, st, csize, args);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qlora
