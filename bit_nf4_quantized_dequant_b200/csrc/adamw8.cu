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
#include "adamw8.cuh"

namespace qlora {
namespace {

__global__ void __launch_bounds__(256) adamw8_kernel(Adam8Tensor t, uint16_t *__restrict__ p_bf16,
                                                     const float *__restrict__ grad, int64_t n, AdamArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + warp;
  const int64_t base = blk * kStateBlock;
  if (base >= n) return;
  float g[8], pn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int64_t i = base + e * 32 + lane;
    g[e] = i < n ? grad[i] : 0.f;
  }
  adamw8_block(t, blk, n, g, a, pn);
  if (p_bf16) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int64_t i = base + e * 32 + lane;
      if (i < n) p_bf16[i] = __bfloat16_as_ushort(__float2bfloat16_rn(pn[e]));
    }
  }
}

}  // namespace

cudaError_t launch_adamw8(float *p, uint16_t *p_bf16, const float *grad, int8_t *mq, uint8_t *vq, float *mscale,
                          float *vscale, int64_t n, int step, float lr, float beta1, float beta2, float eps, float wd,
                          cudaStream_t st) {
  const AdamArgs a = make_adam_args(step, lr, beta1, beta2, eps, wd);
  const Adam8Tensor t{p, mq, vq, mscale, vscale};
  const int64_t blocks = (n + kStateBlock - 1) / kStateBlock;
  const int64_t grid = (blocks + 7) / 8;
  adamw8_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(t, p_bf16, grad, n, a);
  return cudaGetLastError();
}

}  // namespace qlora
