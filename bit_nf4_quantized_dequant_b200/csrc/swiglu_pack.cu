// Layout helpers of the fused SwiGLU projection: the Llama-style MLP whose
// gate and up projections feed silu(g) * u ("QLoRA and Fine-Tuning on One
// Consumer GPU", section "Where 24 GB goes": LoRA adapters on the attention
// and MLP projections, and gradient checkpointing recomputes a layer's MLP
// intermediates during the backward).
//
// The fused kernel reads the gate and up weights as one NF4 matrix whose rows
// alternate in chunks of 64 (gate rows 64c..64c+63, then up rows 64c..64c+63),
// so that one 128-row tile holds g and u of the same 64 output columns. The
// adapters keep their own A and B; in the fused product the up-projections B_g
// and B_u become one [2F, 2r] operand in the same row order, block-diagonal:
// a gate row is [B_g row | 0], an up row is [0 | B_u row], and the LoRA term
// uses sU_gu = [sU_g | sU_u]. The adapter gradient of that operand holds dB_g
// and dB_u in its diagonal blocks.
#include "qlora_device.cuh"

namespace qlora {
namespace {

// B_gu[i, :] from B_g, B_u (bf16 bits, [F, r] each); one thread per element of B_gu.
__global__ void swiglu_pack_b_kernel(const uint16_t *__restrict__ Bg, const uint16_t *__restrict__ Bu, int64_t F,
                                     int r, uint16_t *__restrict__ Bgu) {
  const int64_t total = 2 * F * 2 * r;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / (2 * r);
    const int j = static_cast<int>(e % (2 * r));
    const int64_t chunk = i / 128, w = i % 128;
    const bool up = w >= 64;
    const int64_t f = chunk * 64 + (up ? w - 64 : w);
    uint16_t v = 0;
    if (!up && j < r) v = Bg[f * r + j];
    if (up && j >= r) v = Bu[f * r + (j - r)];
    Bgu[e] = v;
  }
}

// dB_g, dB_u (fp32 [F, r]) from the diagonal blocks of dB_gu (fp32 [2F, 2r]).
__global__ void swiglu_unpack_db_kernel(const float *__restrict__ dBgu, int64_t F, int r, float *__restrict__ dBg,
                                        float *__restrict__ dBu) {
  const int64_t total = 2 * F * r;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool up = e >= F * r;
    const int64_t idx = up ? e - F * r : e;
    const int64_t f = idx / r;
    const int j = static_cast<int>(idx % r);
    const int64_t i = (f / 64) * 128 + (up ? 64 : 0) + f % 64;
    const float v = dBgu[i * 2 * r + (up ? r + j : j)];
    if (up) dBu[idx] = v;
    else    dBg[idx] = v;
  }
}

int grid_for(int64_t total) {
  const int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  return static_cast<int>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

cudaError_t launch_swiglu_pack_b(const uint16_t *Bg, const uint16_t *Bu, int64_t F, int r, uint16_t *Bgu,
                                 cudaStream_t st) {
  swiglu_pack_b_kernel<<<grid_for(4 * F * r), 256, 0, st>>>(Bg, Bu, F, r, Bgu);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_unpack_db(const float *dBgu, int64_t F, int r, float *dBg, float *dBu, cudaStream_t st) {
  swiglu_unpack_db_kernel<<<grid_for(2 * F * r), 256, 0, st>>>(dBgu, F, r, dBg, dBu);
  return cudaGetLastError();
}

}  // namespace qlora
