// NF4 codec kernels: blockwise absmax quantisation with double quantisation of
// the block constants, and standalone dequantisation to bf16.
//
// Format ("QLoRA, in depth", section "The mechanism in brief"; "What is
// QLoRA ...", section "The three QLoRA ideas"): blocks of 64 consecutive
// row-major weights, 4-bit codes into the NF4 levels, one 8-bit constant per
// block, one fp32 second-level scale per group of 256 blocks.
#include <cuda_fp8.h>

#include <cmath>
#include <limits>

#include "qlora_device.cuh"

namespace qlora {
namespace {

// Second-level formats: kDqLinear = unsigned linear absmax codes, one fp32
// scale per group (the library's format); kDqFp8 = E4M3 codes of the
// group-mean-centred constants, fp32 (d, mu) per group (the comparison
// format of the paper the pages cite: "QLoRA and Fine-Tuning on One Consumer
// GPU", "NF4 and double quantisation"). Decoded constant for kDqFp8:
// s = RN32(RN32(e4m3(q) * d) + mu).
constexpr int kDqLinear = 0;
constexpr int kDqFp8 = 1;
constexpr float kE4m3Max = 448.0f;

__device__ __forceinline__ float e4m3_to_float(uint8_t q) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(q), __NV_E4M3)));
}

template <int DQ>
__device__ __forceinline__ float decoded_scale(const uint8_t *scale8, const float *scale2, int64_t b) {
  if constexpr (DQ == kDqFp8) {
    const float2 dm = __ldg(reinterpret_cast<const float2 *>(scale2) + (b >> 8));
    return __fadd_rn(__fmul_rn(e4m3_to_float(__ldg(scale8 + b)), dm.x), dm.y);
  } else {
    return block_scale(__ldg(scale8 + b), __ldg(scale2 + (b >> 8)));
  }
}

// code = number of midpoints between adjacent levels that n lies strictly
// above: the nearest level, ties to the lower one. The midpoint m of two
// float32 levels is exact in float64; for a float32 n, n > m holds exactly
// when n >= up(m), the smallest float32 above m, so the kernel compares n with
// the fifteen float32 thresholds up(m_i) (computed on the host in float64).
struct Thresholds {
  float t[15];
};

Thresholds thresholds_for(const float (&L)[16]) {
  Thresholds th{};
  for (int i = 0; i < 15; ++i) {
    const double m = 0.5 * (static_cast<double>(L[i]) + static_cast<double>(L[i + 1]));
    float f = static_cast<float>(m);
    if (static_cast<double>(f) <= m) f = std::nextafter(f, std::numeric_limits<float>::infinity());
    th.t[i] = f;
  }
  return th;
}

// The same count with one comparison: [-1, 1] is cut into 129 cells of
// width 1/64, cell j = floor(64 n + 64 + off); cand[j] thresholds lie below
// the cell and at most one, t[j], inside it (+inf if none), so
// code = cand[j] + (n >= t[j]). `off` keeps every threshold at least 1/1000
// of a cell away from the cell edges, so the rounding of 64 n + 64 + off can
// move n to a neighbouring cell only where both cells give the same count.
struct CellTable {
  float t[129];
  int32_t cand[129];
  float off64;   // 64 + off
};

bool cell_table_for(const Thresholds &th, CellTable *ct) {
  static const double offs[] = {0.5, 0.25, 0.75, 0.125, 0.375, 0.625, 0.875, 0.0625, 0.3125, 0.5625, 0.8125};
  for (const double off : offs) {
    bool ok = true;
    for (int i = 0; i < 15 && ok; ++i) {
      const double x = 64.0 * th.t[i] + 64.0 + off, f = x - std::floor(x);
      ok = f > 1e-3 && f < 1.0 - 1e-3;
    }
    for (int j = 0; j <= 128 && ok; ++j) {
      const double lo = (j - 64 - off) / 64.0, hi = lo + 1.0 / 64.0;
      int cand = 0, inside = 0;
      float t = std::numeric_limits<float>::infinity();
      for (int i = 0; i < 15; ++i) {
        if (th.t[i] < lo) ++cand;
        else if (th.t[i] < hi) { ++inside; t = th.t[i]; }
      }
      ok = inside <= 1;
      ct->t[j] = t;
      ct->cand[j] = cand;
    }
    if (ok) {
      ct->off64 = static_cast<float>(64.0 + off);
      return true;
    }
  }
  return false;
}

__device__ __forceinline__ uint32_t cell_code(float n, const float *ts, const int32_t *cs, float off64) {
  // n in [-1, 1] gives j in [0, 128]; the clamp keeps the quotient of a
  // non-finite weight (reported through the status) inside the table
  const int j = min(max(__float2int_rd(fmaf(n, 64.f, off64)), 0), 128);
  return static_cast<uint32_t>(cs[j]) + (n >= ts[j] ? 1u : 0u);
}

// One CTA per group of 256 blocks. A warp load covers two consecutive blocks
// (lanes 0-15 the first, 16-31 the second, four elements each); warp w takes
// block pairs w, w + 8, ..., four pairs at a time (four 512-byte loads in
// flight). Lane l writes the two code bytes of its four elements, so a warp
// writes the 64 code bytes of its pair in one contiguous store.
constexpr int kQuantBatch = 4;

template <int BOOK, int DQ>
__global__ void __launch_bounds__(256) nf4_quantize_kernel(const float *__restrict__ W, int64_t nb,
                                                           uint8_t *__restrict__ codes,
                                                           uint8_t *__restrict__ scale8,
                                                           float *__restrict__ scale2,
                                                           int32_t *status, const CellTable ct) {
  __shared__ float c1s[kGroup];
  __shared__ float cts[129];
  __shared__ int32_t ccs[129];
  for (int i = threadIdx.x; i < 129; i += blockDim.x) {
    cts[i] = ct.t[i];
    ccs[i] = ct.cand[i];
  }
  __syncthreads();
  __shared__ float red[8];
  __shared__ float mu_s;
  const int64_t g = blockIdx.x;
  const int64_t b0 = g * kGroup;
  const int nblk = static_cast<int>(nb - b0 < kGroup ? nb - b0 : kGroup);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  bool bad = false;
  const int half = lane >> 4, hl = lane & 15;
  const int npairs = (nblk + 1) / 2;
  for (int p0 = warp; p0 < npairs; p0 += 8 * kQuantBatch) {
    float4 v[kQuantBatch];
#pragma unroll
    for (int u = 0; u < kQuantBatch; ++u) {   // warp-uniform pair index; the second block may be missing
      const int i = 2 * (p0 + 8 * u) + half;
      v[u] = (p0 + 8 * u < npairs && i < nblk)
                 ? __ldg(reinterpret_cast<const float4 *>(W + (b0 + i) * kBlock) + hl)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kQuantBatch; ++u) {
      if (p0 + 8 * u >= npairs) break;
      const int i = 2 * (p0 + 8 * u) + half;
      bad |= !isfinite(v[u].x) || !isfinite(v[u].y) || !isfinite(v[u].z) || !isfinite(v[u].w);
      float m = fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w)));
#pragma unroll
      for (int o = 8; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));   // within each half
      constexpr uint32_t kZero = BOOK == kBookInt4 ? 8u : 7u;   // index of the exact zero level
      uint32_t e0 = kZero, e1 = kZero, e2 = kZero, e3 = kZero;
      if (m > 0.f) {
        e0 = cell_code(__fdiv_rn(v[u].x, m), cts, ccs, ct.off64);
        e1 = cell_code(__fdiv_rn(v[u].y, m), cts, ccs, ct.off64);
        e2 = cell_code(__fdiv_rn(v[u].z, m), cts, ccs, ct.off64);
        e3 = cell_code(__fdiv_rn(v[u].w, m), cts, ccs, ct.off64);
      }
      if (i < nblk) {
        // bytes 2hl, 2hl+1 of the block: (e0 << 4 | e1), (e2 << 4 | e3)
        const uint16_t two = static_cast<uint16_t>(((e0 << 4) | e1) | (((e2 << 4) | e3) << 8));
        reinterpret_cast<uint16_t *>(codes + (b0 + i) * (kBlock / 2))[hl] = two;
        if (hl == 0) c1s[i] = m;
      }
    }
  }
  if (bad) set_status(status, 5 /* QLORA_ERR_NONFINITE */);
  __syncthreads();

  const int t = threadIdx.x;
  const float c1 = t < nblk ? c1s[t] : 0.f;
  if constexpr (DQ == kDqFp8) {
    // mean of the group's constants: float64 sum in block order, one division
    if (t == 0) {
      double sum = 0.0;
      for (int i = 0; i < nblk; ++i) sum = __dadd_rn(sum, static_cast<double>(c1s[i]));
      mu_s = __double2float_rn(__ddiv_rn(sum, static_cast<double>(nblk)));
    }
    __syncthreads();
    const float mu = mu_s;
    const float cen = t < nblk ? __fsub_rn(c1, mu) : 0.f;
    float a = fabsf(cen);
#pragma unroll
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0) red[warp] = a;
    __syncthreads();
    float amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    const float d = __fdiv_rn(amax, kE4m3Max);
    if (t < nblk)
      scale8[b0 + t] = d > 0.f ? static_cast<uint8_t>(__nv_cvt_float_to_fp8(__fdiv_rn(cen, d), __NV_SATFINITE, __NV_E4M3))
                               : uint8_t{0};
    if (t == 0) {
      scale2[2 * g] = d;
      scale2[2 * g + 1] = mu;
    }
    return;
  }
  // second level: c2 = max c1 over the group
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
template <int BOOK, int DQ>
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
    const float sc = decoded_scale<DQ>(scale8, scale2, b);
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
                            uint8_t *scale8, float *scale2, int32_t *dev_status, cudaStream_t s, int book, int dq) {
  const int64_t nb = rows * cols / kBlock;
  const int64_t ng = (nb + kGroup - 1) / kGroup;
  if (dev_status) {
    cudaError_t e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  const unsigned grid = static_cast<unsigned>(ng);
  static CellTable ct_nf4, ct_int4;
  static const bool ct_ok = [] {
    const float Ln[16] = QLORA_NF4_LEVELS;
    const float Li[16] = QLORA_INT4_LEVELS;
    return cell_table_for(thresholds_for(Ln), &ct_nf4) && cell_table_for(thresholds_for(Li), &ct_int4);
  }();
  if (!ct_ok) return cudaErrorInvalidValue;   // no offset separates the thresholds from the cell edges (never expected)
  if (dq == kDqFp8)
    nf4_quantize_kernel<kBookNf4, kDqFp8><<<grid, 256, 0, s>>>(W, nb, codes, scale8, scale2, dev_status, ct_nf4);
  else if (book == kBookInt4)
    nf4_quantize_kernel<kBookInt4, kDqLinear><<<grid, 256, 0, s>>>(W, nb, codes, scale8, scale2, dev_status, ct_int4);
  else
    nf4_quantize_kernel<kBookNf4, kDqLinear><<<grid, 256, 0, s>>>(W, nb, codes, scale8, scale2, dev_status, ct_nf4);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scale8, const float *scale2,
                              int64_t rows, int64_t cols, uint16_t *out, cudaStream_t s, int book, int dq) {
  const int64_t nhalf = rows * cols / 32;
  const int64_t grid = (nhalf + 255) / 256;
  const unsigned g = static_cast<unsigned>(grid);
  if (dq == kDqFp8)
    nf4_dequant_kernel<kBookNf4, kDqFp8><<<g, 256, 0, s>>>(codes, scale8, scale2, nhalf, out);
  else if (book == kBookInt4)
    nf4_dequant_kernel<kBookInt4, kDqLinear><<<g, 256, 0, s>>>(codes, scale8, scale2, nhalf, out);
  else
    nf4_dequant_kernel<kBookNf4, kDqLinear><<<g, 256, 0, s>>>(codes, scale8, scale2, nhalf, out);
  return cudaGetLastError();
}

}  // namespace qlora
