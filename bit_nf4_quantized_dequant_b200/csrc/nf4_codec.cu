// NF4 codec kernels: blockwise absmax quantisation with double quantisation of
// the block constants, and standalone dequantisation to bf16.
//
// Format ("QLoRA, in depth", section "The mechanism in brief"; "What is
// QLoRA ...", section "The three QLoRA ideas"): blocks of 64 consecutive
// row-major weights, 4-bit codes into the NF4 levels, one 8-bit constant per
// block, one fp32 second-level scale per group of 256 blocks.
#include "qlora_device.cuh"

namespace qlora {
namespace {

// code = number of midpoints between adjacent levels that n lies strictly
// above: the nearest level, ties to the lower one. The midpoints of two float32
// levels are exact in float64, and so is the comparison.
template <int BOOK>
__device__ __forceinline__ uint32_t nearest_level(float n) {
  constexpr float NF4[16] = QLORA_NF4_LEVELS;
  constexpr float INT4[16] = QLORA_INT4_LEVELS;
  const float *L = BOOK == kBookInt4 ? INT4 : NF4;
  const double x = static_cast<double>(n);
  uint32_t code = 0;
#pragma unroll
  for (int i = 0; i < 15; ++i) {
    const double mid = 0.5 * (static_cast<double>(L[i]) + static_cast<double>(L[i + 1]));
    code += (x > mid) ? 1u : 0u;
  }
  return code;
}

// One CTA per group of 256 blocks; warp w handles blocks w, w+8, ...; lane l
// holds elements 2l and 2l+1 of a block, so the packed byte l of the block is
// written by lane l.
template <int BOOK>
__global__ void __launch_bounds__(256) nf4_quantize_kernel(const float *__restrict__ W, int64_t nb,
                                                           uint8_t *__restrict__ codes,
                                                           uint8_t *__restrict__ scale8,
                                                           float *__restrict__ scale2,
                                                           int32_t *status) {
  __shared__ float c1s[kGroup];
  __shared__ float red[8];
  const int64_t g = blockIdx.x;
  const int64_t b0 = g * kGroup;
  const int nblk = static_cast<int>(nb - b0 < kGroup ? nb - b0 : kGroup);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  bool bad = false;
  for (int i = warp; i < nblk; i += 8) {
    const int64_t b = b0 + i;
    const float2 v = __ldg(reinterpret_cast<const float2 *>(W + b * kBlock) + lane);
    bad |= !isfinite(v.x) || !isfinite(v.y);
    float m = fmaxf(fabsf(v.x), fabsf(v.y));
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    constexpr uint32_t kZero = BOOK == kBookInt4 ? 8u : 7u;   // index of the exact zero level
    uint32_t e0 = kZero, e1 = kZero;
    if (m > 0.f) {
      e0 = nearest_level<BOOK>(__fdiv_rn(v.x, m));
      e1 = nearest_level<BOOK>(__fdiv_rn(v.y, m));
    }
    codes[b * (kBlock / 2) + lane] = static_cast<uint8_t>((e0 << 4) | e1);
    if (lane == 0) c1s[i] = m;
  }
  if (bad) set_status(status, 5 /* QLORA_ERR_NONFINITE */);
  __syncthreads();

  // second level: c2 = max c1 over the group
  const int t = threadIdx.x;
  const float c1 = t < nblk ? c1s[t] : 0.f;
  float m = c1;
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float c2 = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) c2 = fmaxf(c2, red[i]);
  if (t < nblk) {
    uint32_t q = 0;
    if (c2 > 0.f) {
      // 255 c1 is exact in float64 and the float64 quotient is correctly
      // rounded; it cannot reach a half-integer unless the exact ratio is one,
      // so rounding it half-to-even rounds the exact ratio half-to-even.
      q = static_cast<uint32_t>(rint(__ddiv_rn(255.0 * static_cast<double>(c1), static_cast<double>(c2))));
    }
    scale8[b0 + t] = static_cast<uint8_t>(q);
  }
  if (t == 0) scale2[g] = __fdiv_rn(c2, 255.0f);
}

// One thread per half block (32 weights = 16 code bytes -> 64 output bytes).
// Each warp stages its 32 x 64 contiguous output bytes in shared memory and
// writes them with one bulk copy, so global stores are full, contiguous 2 KiB
// runs instead of 64-byte pieces strided across the warp.
template <int BOOK>
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint8_t *__restrict__ codes,
                                                          const uint8_t *__restrict__ scale8,
                                                          const float *__restrict__ scale2,
                                                          int64_t nhalf, uint16_t *__restrict__ out) {
  __shared__ __align__(128) uint4 stage[8][32 * 4];   // per warp: 32 threads x 64 bytes
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t warp_first = (static_cast<int64_t>(blockIdx.x) * blockDim.x) + warp * 32;
  if (warp_first >= nhalf) return;
  const int64_t i = warp_first + lane;
  const int active = static_cast<int>(nhalf - warp_first < 32 ? nhalf - warp_first : 32);
  uint4 *mine = &stage[warp][lane * 4];
  if (i < nhalf) {
    const int64_t b = i >> 1;
    const uint4 c = __ldg(reinterpret_cast<const uint4 *>(codes) + i);
    const float sc = block_scale(__ldg(scale8 + b), __ldg(scale2 + (b >> 8)));
    const Nf4Table t = make_table_book<BOOK>(sc);
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t o[4];
      expand8(t, w[k], o);
      mine[k] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    bulk_store(out + warp_first * 32, &stage[warp][0], static_cast<uint32_t>(active) * 64u);
    bulk_commit_group();
    bulk_wait_group_read<0>();
  }
  __syncwarp();
}

}  // namespace

cudaError_t launch_quantize(const float *W, int64_t rows, int64_t cols, uint8_t *codes,
                            uint8_t *scale8, float *scale2, int32_t *dev_status, cudaStream_t s, int book) {
  const int64_t nb = rows * cols / kBlock;
  const int64_t ng = (nb + kGroup - 1) / kGroup;
  if (dev_status) {
    cudaError_t e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  if (book == kBookInt4)
    nf4_quantize_kernel<kBookInt4><<<static_cast<unsigned>(ng), 256, 0, s>>>(W, nb, codes, scale8, scale2, dev_status);
  else
    nf4_quantize_kernel<kBookNf4><<<static_cast<unsigned>(ng), 256, 0, s>>>(W, nb, codes, scale8, scale2, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scale8, const float *scale2,
                              int64_t rows, int64_t cols, uint16_t *out, cudaStream_t s, int book) {
  const int64_t nhalf = rows * cols / 32;
  const int64_t grid = (nhalf + 255) / 256;
  if (book == kBookInt4)
    nf4_dequant_kernel<kBookInt4><<<static_cast<unsigned>(grid), 256, 0, s>>>(codes, scale8, scale2, nhalf, out);
  else
    nf4_dequant_kernel<kBookNf4><<<static_cast<unsigned>(grid), 256, 0, s>>>(codes, scale8, scale2, nhalf, out);
  return cudaGetLastError();
}

}  // namespace qlora
