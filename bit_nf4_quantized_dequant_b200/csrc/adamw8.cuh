// One 256-element block of the 8-bit AdamW step, shared by the standalone
// update (adamw8.cu) and the update fused into the adapter-gradient epilogue
// (lora_skinny.cu). State format and arithmetic are described in adamw8.cu.
#pragma once

#include <cmath>

#include "qlora_device.cuh"

namespace qlora {

constexpr int kStateBlock = 256;

struct AdamArgs {
  float lr, beta1, one_minus_beta1, beta2, one_minus_beta2, bc1, bc2, eps, wd;
};

inline AdamArgs make_adam_args(int step, float lr, float beta1, float beta2, float eps, float wd) {
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
  return a;
}

// The state of one parameter tensor, flattened: element i of p, m_q, v_q; one
// m_scale / v_scale per block of 256.
struct Adam8Tensor {
  float *p;
  int8_t *m_q;
  uint8_t *v_q;
  float *m_scale;
  float *v_scale;
};

// The fused update of both adapters inside the gradient launch (lora_skinny.cu).
struct AdamFuseArgs {
  Adam8Tensor A, B;          // A's state in the d-major order of A^T [K, r]; B's in [N, r]
  uint16_t *A_bf16, *B_bf16; // A [r, K], B [N, r], or NULL
  int step;
  float lr, beta1, beta2, eps, wd;
};

// Block `blk` of a tensor of n elements, one warp: lane l holds elements
// blk * 256 + e * 32 + l (e = 0..7) with gradients g[e] (ignored past n). On
// return pn[e] holds the updated fp32 parameter of each element this lane
// owns (elements past n are left alone).
__device__ __forceinline__ void adamw8_block(const Adam8Tensor &t, int64_t blk, int64_t n, const float (&g)[8],
                                             const AdamArgs &a, float (&pn)[8]) {
  const int lane = threadIdx.x & 31;
  const int64_t base = blk * kStateBlock;
  const float ms = t.m_scale[blk], vs = t.v_scale[blk];
  float m[8], v[8];
  float mmax = 0.f, vmax = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int64_t i = base + e * 32 + lane;
    m[e] = v[e] = pn[e] = 0.f;
    if (i < n) {
      const float m0 = __fmul_rn(__fdiv_rn(static_cast<float>(t.m_q[i]), 127.f), ms);
      const float tq = __fdiv_rn(static_cast<float>(t.v_q[i]), 255.f);
      const float v0 = __fmul_rn(__fmul_rn(tq, tq), vs);
      m[e] = __fadd_rn(__fmul_rn(a.beta1, m0), __fmul_rn(a.one_minus_beta1, g[e]));
      v[e] = __fadd_rn(__fmul_rn(a.beta2, v0), __fmul_rn(a.one_minus_beta2, __fmul_rn(g[e], g[e])));
      const float mh = __fdiv_rn(m[e], a.bc1), vh = __fdiv_rn(v[e], a.bc2);
      const float p0 = t.p[i];
      const float upd = __fadd_rn(__fdiv_rn(mh, __fadd_rn(__fsqrt_rn(vh), a.eps)), __fmul_rn(a.wd, p0));
      pn[e] = __fsub_rn(p0, __fmul_rn(a.lr, upd));
      t.p[i] = pn[e];
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
      t.m_q[i] = static_cast<int8_t>(mmax > 0.f ? rintf(__fdiv_rn(__fmul_rn(m[e], 127.f), mmax)) : 0.f);
      float qv = 0.f;
      if (v[e] > 0.f) qv = fminf(fmaxf(rintf(__fmul_rn(255.f, __fsqrt_rn(__fdiv_rn(v[e], vmax)))), 1.f), 255.f);
      t.v_q[i] = static_cast<uint8_t>(qv);
    }
  }
  if (lane == 0) {
    t.m_scale[blk] = mmax;
    t.v_scale[blk] = vmax;
  }
}

}  // namespace qlora
