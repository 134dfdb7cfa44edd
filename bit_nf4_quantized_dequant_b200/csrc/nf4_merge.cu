// Merging the adapter into the base: W_merged = W' + s B A, where W' is the
// dequantised NF4 weight ("QLoRA" (guide.dupenodi.dev), section "Walking
// through the tooling": at inference the adapter is either merged, W' = W +
// scaled BA, or kept separate; "QLoRA, in depth", section "Shipping: merge,
// re-quantize, verify"). The merged weight
// is written in bf16, or in fp32 for a later re-quantisation.
//
// Per element: w = bf16 W' value, d = sum_j B[n, j] A[j, k] accumulated in
// fp32 by the warp-level MMA (m16n8k16, bf16 in), merged = fp32(w) + s * d
// (one fused multiply-add), then rounded to bf16 or kept in fp32.
//
// The pass is bound by HBM (0.516 B read and 2 or 4 B written per weight), so
// the layout follows the few-token forward: a warp takes 16 weight rows by 4
// NF4 blocks (256 columns); thread (g, c) expands rows g and g + 8 of block c
// into bf16 pairs in registers, which are exactly the pairs its MMA
// accumulator fragment holds once the MMA's 8-column tiles are mapped so that
// tile t covers columns 64 c + 2 t, + 1 of each thread c. A's columns are
// staged in shared memory as (A[2p][k], A[2p+1][k]) pairs, so a B fragment is
// two 32-bit loads; the four blocks' columns are interleaved and the pair
// rows padded so that those loads hit 32 distinct banks. bf16 results go
// through a per-warp shared-memory tile (16-byte chunks XOR-swizzled within
// each block, conflict-free both ways) and leave as whole 512-byte rows.
#include <atomic>

#include "qlora_device.cuh"

namespace qlora {
namespace {

constexpr int kMergeWarps = 8;
constexpr int kCols = 256;   // columns per CTA strip (4 NF4 blocks)
constexpr int kPairStride = kCols + 8;   // words per pair row: 8 mod 32, so the 4 pair rows take distinct banks

// word index of column col (0..255) in a pair row: the 4 blocks interleaved
__device__ __forceinline__ int pair_col(int col) { return 4 * (col & 63) + (col >> 6); }

template <bool kF32Out, int KSTEPS>   // KSTEPS = r_pad / 16
__global__ void __launch_bounds__(kMergeWarps * 32, 2)
    nf4_merge_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scale8,
                     const float *__restrict__ scale2, int64_t N, int64_t K, const uint16_t *__restrict__ Al,
                     const uint16_t *__restrict__ Bl, int r, float s, void *__restrict__ out, int rows_per_cta) {
  // apair[p * kPairStride + pair_col(col)] = (A[2p][col0 + col], A[2p + 1][col0 + col])
  __shared__ uint32_t apair[8 * KSTEPS * kPairStride];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * kCols;
  const int64_t kblocks = K / 64;
  for (int i = threadIdx.x; i < 8 * KSTEPS * kCols; i += blockDim.x) {
    const int p = i / kCols, col = i % kCols;
    const int64_t k = col0 + col;
    uint32_t lo = 0, hi = 0;
    if (k < K) {
      if (2 * p < r) lo = Al[static_cast<int64_t>(2 * p) * K + k];
      if (2 * p + 1 < r) hi = Al[static_cast<int64_t>(2 * p + 1) * K + k];
    }
    apair[p * kPairStride + pair_col(col)] = lo | (hi << 16);
  }
  __syncthreads();

  extern __shared__ __align__(16) uint8_t merge_dyn[];
  uint8_t *wtile = merge_dyn + static_cast<size_t>(warp) * 16 * 512;   // [16 rows][256 cols] bf16
  const int64_t b = col0 / 64 + c;           // this thread's NF4 block along the row
  const bool bvalid = b < kblocks;
  const int64_t row_begin = static_cast<int64_t>(blockIdx.y) * rows_per_cta;
  const int64_t row_end = row_begin + rows_per_cta < N ? row_begin + rows_per_cta : N;

  // The codes, block constants and B rows of a 16-row tile; the next tile's are
  // requested before the current one is expanded, so that one HBM latency is
  // always in flight per warp.
  struct Tile {
    uint4 w0a, w0b, w1a, w1b;
    uint32_t q0, q1;
    float d0, d1;
    uint32_t af[KSTEPS][4];
  };
  auto load_tile = [&](Tile &t, int64_t r0) {
    const int64_t n0 = r0 + g, n1 = n0 + 8;   // N % 16 == 0: both rows exist
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      const int j0 = ks * 16 + 2 * c, j1 = j0 + 8;
      auto pairB = [&](int64_t n, int j) -> uint32_t {
        const uint32_t lo = j < r ? Bl[n * r + j] : 0u;
        const uint32_t hi = j + 1 < r ? Bl[n * r + j + 1] : 0u;
        return lo | (hi << 16);
      };
      t.af[ks][0] = pairB(n0, j0);
      t.af[ks][1] = pairB(n1, j0);
      t.af[ks][2] = pairB(n0, j1);
      t.af[ks][3] = pairB(n1, j1);
    }
    t.w0a = t.w0b = t.w1a = t.w1b = make_uint4(0, 0, 0, 0);
    t.q0 = t.q1 = 0;
    t.d0 = t.d1 = 0.f;
    if (bvalid) {
      const uint8_t *p0 = codes + n0 * (K / 2) + b * 32;
      const uint8_t *p1 = codes + n1 * (K / 2) + b * 32;
      t.w0a = *reinterpret_cast<const uint4 *>(p0);
      t.w0b = *reinterpret_cast<const uint4 *>(p0 + 16);
      t.w1a = *reinterpret_cast<const uint4 *>(p1);
      t.w1b = *reinterpret_cast<const uint4 *>(p1 + 16);
      const int64_t i0 = n0 * kblocks + b, i1 = n1 * kblocks + b;
      t.q0 = __ldg(scale8 + i0);
      t.q1 = __ldg(scale8 + i1);
      t.d0 = __ldg(scale2 + (i0 >> 8));
      t.d1 = __ldg(scale2 + (i1 >> 8));
    }
  };

  Tile cur, nxt;
  int64_t r0 = row_begin + warp * 16;
  if (r0 < row_end) load_tile(cur, r0);
  for (; r0 < row_end; r0 += kMergeWarps * 16) {
    const int64_t rn = r0 + kMergeWarps * 16;
    if (rn < row_end) load_tile(nxt, rn);
    const int64_t n0 = r0 + g, n1 = n0 + 8;
    const Nf4Table t0 = make_table(block_scale(cur.q0, cur.d0)), t1 = make_table(block_scale(cur.q1, cur.d1));
    const uint32_t w0[8] = {cur.w0a.x, cur.w0a.y, cur.w0a.z, cur.w0a.w, cur.w0b.x, cur.w0b.y, cur.w0b.z, cur.w0b.w};
    const uint32_t w1[8] = {cur.w1a.x, cur.w1a.y, cur.w1a.z, cur.w1a.w, cur.w1b.x, cur.w1b.y, cur.w1b.z, cur.w1b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {   // word i: columns 8i .. 8i + 7 of the block, MMA tiles 4i .. 4i + 3
      uint32_t e0[4], e1[4];
      expand8(t0, w0[i], e0);
      expand8(t1, w1[i], e1);
      float m0[8], m1[8];   // merged values of rows n0, n1 at columns 8i .. 8i + 7
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int t = 4 * i + h;
        // B fragment of tile t: column n = g of the tile <-> block (g >> 1), column 2t + (g & 1)
        const int pc = pair_col(64 * (g >> 1) + 2 * t + (g & 1));
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
          mma_16816(d, cur.af[ks], apair[(ks * 8 + c) * kPairStride + pc], apair[(ks * 8 + c + 4) * kPairStride + pc]);
        // d[0..1] = row g, columns 64c + 2t, +1; d[2..3] = row g + 8
        m0[2 * h] = fmaf(s, d[0], __uint_as_float(e0[h] << 16));
        m0[2 * h + 1] = fmaf(s, d[1], __uint_as_float(e0[h] & 0xFFFF0000u));
        m1[2 * h] = fmaf(s, d[2], __uint_as_float(e1[h] << 16));
        m1[2 * h + 1] = fmaf(s, d[3], __uint_as_float(e1[h] & 0xFFFF0000u));
      }
      if (bvalid) {
        const int64_t k = b * 64 + 8 * i;
        if constexpr (kF32Out) {
          float *o = static_cast<float *>(out);
          *reinterpret_cast<float4 *>(o + n0 * K + k) = make_float4(m0[0], m0[1], m0[2], m0[3]);
          *reinterpret_cast<float4 *>(o + n0 * K + k + 4) = make_float4(m0[4], m0[5], m0[6], m0[7]);
          *reinterpret_cast<float4 *>(o + n1 * K + k) = make_float4(m1[0], m1[1], m1[2], m1[3]);
          *reinterpret_cast<float4 *>(o + n1 * K + k + 4) = make_float4(m1[4], m1[5], m1[6], m1[7]);
        }
      }
      if constexpr (!kF32Out) {
        // chunk i of block c of rows g and g + 8, at position i ^ (2c + g) within the block
        const uint32_t pos = static_cast<uint32_t>(8 * c + (i ^ ((2 * c + g) & 7))) * 16u;
        *reinterpret_cast<uint4 *>(wtile + g * 512 + pos) =
            make_uint4(pack_bf16x2(m0[0], m0[1]), pack_bf16x2(m0[2], m0[3]), pack_bf16x2(m0[4], m0[5]),
                       pack_bf16x2(m0[6], m0[7]));
        *reinterpret_cast<uint4 *>(wtile + (g + 8) * 512 + pos) =
            make_uint4(pack_bf16x2(m1[0], m1[1]), pack_bf16x2(m1[2], m1[3]), pack_bf16x2(m1[4], m1[5]),
                       pack_bf16x2(m1[6], m1[7]));
      }
    }
    if constexpr (!kF32Out) {
      __syncwarp();
      // lane L writes bytes 16L .. 16L + 15 of each of the 16 rows: chunk L & 7 of block L >> 3
      const int lc = lane >> 3, li = lane & 7;
      const bool lvalid = col0 / 64 + lc < kblocks;
      uint16_t *o = static_cast<uint16_t *>(out);
#pragma unroll 4
      for (int rho = 0; rho < 16; ++rho) {
        const uint32_t pos = static_cast<uint32_t>(8 * lc + (li ^ ((2 * lc + (rho & 7)) & 7))) * 16u;
        const uint4 v = *reinterpret_cast<const uint4 *>(wtile + rho * 512 + pos);
        if (lvalid) *reinterpret_cast<uint4 *>(o + (r0 + rho) * K + col0 + 8 * lane) = v;
      }
      __syncwarp();
    }
    cur = nxt;
  }
}

// Resident CTAs per SM of one kernel instantiation, found (with its shared
// memory limit raised) on the first launch on each device and kept: the
// query costs microseconds of host time, which a pass over many small
// matrices would otherwise pay per launch.
constexpr int kMergeMaxDevices = 64;

template <typename Kernel>
cudaError_t merge_blocks_per_sm(Kernel kernel, size_t dyn, std::atomic<int> (&cache)[kMergeMaxDevices], int *per_sm) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < kMergeMaxDevices;
  if (cacheable) {
    const int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) {
      *per_sm = v;
      return cudaSuccess;
    }
  }
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn));
  if (e != cudaSuccess) return e;
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kMergeWarps * 32, dyn);
  if (e != cudaSuccess) return e;
  if (n < 1) n = 1;
  if (cacheable) cache[dev].store(n, std::memory_order_relaxed);
  *per_sm = n;
  return cudaSuccess;
}

template <bool kF32Out, int KSTEPS>
std::atomic<int> g_merge_per_sm[kMergeMaxDevices];

template <bool kF32Out>
cudaError_t launch_merge_t(const uint8_t *codes, const uint8_t *scale8, const float *scale2, int64_t N,
                           int64_t K, const uint16_t *Al, const uint16_t *Bl, int r, float s, void *out,
                           cudaStream_t st) {
  const int64_t strips = (K + kCols - 1) / kCols;
  const size_t dyn = kF32Out ? 0 : static_cast<size_t>(kMergeWarps) * 16 * 512;
  auto go = [&](auto kernel, std::atomic<int> (&cache)[kMergeMaxDevices]) -> cudaError_t {
    // one wave: as many (strip, band) CTAs as are resident at once, each a
    // band of rows (a multiple of 16); a second partial wave would leave most
    // SMs idle for its whole length
    int per_sm = 0;
    cudaError_t e = merge_blocks_per_sm(kernel, dyn, cache, &per_sm);
    if (e != cudaSuccess) return e;
    const int64_t resident = static_cast<int64_t>(per_sm) * device_sm_count();
    int64_t bands = resident / strips;
    if (bands > N / 16) bands = N / 16;
    if (bands < 1) bands = 1;
    int64_t rows_per = (N + bands - 1) / bands;
    rows_per = (rows_per + 15) / 16 * 16;
    bands = (N + rows_per - 1) / rows_per;
    const dim3 grid(static_cast<unsigned>(strips), static_cast<unsigned>(bands));
    kernel<<<grid, kMergeWarps * 32, dyn, st>>>(codes, scale8, scale2, N, K, Al, Bl, r, s, out,
                                                static_cast<int>(rows_per));
    return cudaGetLastError();
  };
  switch ((r + 15) / 16) {
    case 1: return go(nf4_merge_kernel<kF32Out, 1>, g_merge_per_sm<kF32Out, 1>);
    case 2: return go(nf4_merge_kernel<kF32Out, 2>, g_merge_per_sm<kF32Out, 2>);
    case 3: return go(nf4_merge_kernel<kF32Out, 3>, g_merge_per_sm<kF32Out, 3>);
    case 4: return go(nf4_merge_kernel<kF32Out, 4>, g_merge_per_sm<kF32Out, 4>);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_nf4_merge(const uint8_t *codes, const uint8_t *scale8, const float *scale2, int64_t N, int64_t K,
                             const uint16_t *Al, const uint16_t *Bl, int r, float s, void *out, bool f32_out,
                             cudaStream_t st) {
  return f32_out ? launch_merge_t<true>(codes, scale8, scale2, N, K, Al, Bl, r, s, out, st)
                 : launch_merge_t<false>(codes, scale8, scale2, N, K, Al, Bl, r, s, out, st);
}

}  // namespace qlora
