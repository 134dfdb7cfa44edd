// AdamW step for the adapter parameters with 8-bit optimiser states ("QLoRA,
// in depth", section "A complete run on a 12 GB-class GPU": the run trains
// with the paged 8-bit AdamW, whose states are held in 8 bits; "QLoRA and
// Fine-Tuning on One Consumer GPU", section "Where 24 GB goes": the adapter
// gradients and Adam's m and v). Paging to host memory is not part of this
// library.
//
// State format (the pages give only "8 bits"): the first moment m as int8
// codes with one fp32 absmax per block of 256 elements, m = q / 127 * absmax;
// the second moment v (non-negative) as uint8 codes of sqrt(v) with one fp32
// maximum of v per block, v = (q / 255)^2 * max. A nonzero v never decodes to
// zero (its code is at least 1): a linear 8-bit v would round the small
// second moments of a block to zero and turn their steps into m / eps. One
// warp owns a block (8 elements per lane): it
// decodes the states, applies the decoupled-weight-decay Adam update in fp32
// with every operation rounded once (no contraction into FMAs, so the result
// is reproducible operation by operation), takes the new block absmax / max
// with a warp reduction and re-encodes (round half to even).
#include <cmath>

#include "qlora_device.cuh"

namespace qlora {
namespace {

constexpr int kStateBlock = 256;

struct AdamArgs {
  float lr, beta1, one_minus_beta1, beta2, one_minus_beta2, bc1, bc2, eps, wd;
};

__global__ void __launch_bounds__(256) adamw8_kernel(float *__restrict__ p, uint16_t *__restrict__ p_bf16,
                                                     const float *__restrict__ grad, int8_t *__restrict__ mq,
                                                     uint8_t *__restrict__ vq, float *__restrict__ mscale,
                                                     float *__restrict__ vscale, int64_t n, AdamArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + warp;
  const int64_t base = blk * kStateBlock;
  if (base >= n) return;
  const float ms = mscale[blk], vs = vscale[blk];
  float m[8], v[8];
  float mmax = 0.f, vmax = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int64_t i = base + e * 32 + lane;
    m[e] = v[e] = 0.f;
    if (i < n) {
      const float g = grad[i];
      const float m0 = __fmul_rn(__fdiv_rn(static_cast<float>(mq[i]), 127.f), ms);
      const float tq = __fdiv_rn(static_cast<float>(vq[i]), 255.f);
      const float v0 = __fmul_rn(__fmul_rn(tq, tq), vs);
      m[e] = __fadd_rn(__fmul_rn(a.beta1, m0), __fmul_rn(a.one_minus_beta1, g));
      v[e] = __fadd_rn(__fmul_rn(a.beta2, v0), __fmul_rn(a.one_minus_beta2, __fmul_rn(g, g)));
      const float mh = __fdiv_rn(m[e], a.bc1), vh = __fdiv_rn(v[e], a.bc2);
      const float upd = __fadd_rn(__fdiv_rn(mh, __fadd_rn(__fsqrt_rn(vh), a.eps)), __fmul_rn(a.wd, p[i]));
      const float pn = __fsub_rn(p[i], __fmul_rn(a.lr, upd));
      p[i] = pn;
      if (p_bf16) p_bf16[i] = __bfloat16_as_ushort(__float2bfloat16_rn(pn));
      mmax = fmaxf(mmax, fabsf(m[e]));
      vmax = fmaxf(vmax, v[e]);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int64_t i = base + e * 32 + lane;
    if (i < n) {
      mq[i] = static_cast<int8_t>(mmax > 0.f ? rintf(__fdiv_rn(__fmul_rn(m[e], 127.f), mmax)) : 0.f);
      float qv = 0.f;
      if (v[e] > 0.f) qv = fminf(fmaxf(rintf(__fmul_rn(255.f, __fsqrt_rn(__fdiv_rn(v[e], vmax)))), 1.f), 255.f);
      vq[i] = static_cast<uint8_t>(qv);
    }
  }
  if (lane == 0) {
    mscale[blk] = mmax;
    vscale[blk] = vmax;
  }
}

}  // namespace

cudaError_t launch_adamw8(float *p, uint16_t *p_bf16, const float *grad, int8_t *mq, uint8_t *vq, float *mscale,
                          float *vscale, int64_t n, int step, float lr, float beta1, float beta2, float eps, float wd,
                          cudaStream_t st) {
  AdamArgs a{};
  a.lr = lr;
  a.beta1 = beta1;
  a.one_minus_beta1 = 1.f - beta1;
  a.beta2 = beta2;
  a.one_minus_beta2 = 1.f - beta2;
  // bias corrections 1 - beta^t, computed in float64 and rounded once
  a.bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta1), step));
  a.bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta2), step));
  a.eps = eps;
  a.wd = wd;
  const int64_t blocks = (n + kStateBlock - 1) / kStateBlock;
  const int64_t grid = (blocks + 7) / 8;
  adamw8_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(p, p_bf16, grad, mq, vq, mscale, vscale, n, a);
  return cudaGetLastError();
}

}  // namespace qlora
