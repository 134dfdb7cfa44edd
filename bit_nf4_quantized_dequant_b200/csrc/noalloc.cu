// Allocation-free variant of the QLoRA linear forward.
//
// qlora_linear_fwd needs a caller-provided workspace for the partial sums of
// s X A^T (and for sU when the caller does not keep it). Some callers have no
// way to provide one at the point where they run the layer: a host that hands
// the library only its inputs and outputs and owns no allocator of its own (a
// plug-in inside someone else's runtime), a serving process that has given all
// device memory to a fixed pool up front, or code that must not call
// cudaMalloc between launches because that call can synchronise the device.
// For them, qlora_linear_fwd_noalloc takes its scratch from one fixed array
// compiled into this library instead of from the caller.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits. Host code
// cannot pass the array's name to a kernel (on the host that name is only a
// stand-in for the device symbol), so the first call on each device looks up
// its device address with cudaGetSymbolAddress, with that device current, and
// caches it; every later call on that device reuses the cached address.
#include <cuda_runtime.h>

#include <mutex>

#include "qlora.h"
#include "qlora_internal.h"

namespace {
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB per device
constexpr int kMaxDevices = 64;
}  // namespace

// The shared scratch. Nothing in it has to start at zero: each call writes
// every byte it later reads (the partial sums and, if used, sU).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

std::mutex g_scratch_mu;
void *g_scratch_dev[kMaxDevices];

// Device address of the scratch array on the current device (looked up once).
qlora_status_t scratch_address(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_dev[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return QLORA_ERR_CUDA;
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return QLORA_OK;
}

size_t round_up_256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" qlora_status_t qlora_linear_fwd_noalloc(const qlora_nf4_t *W, const uint16_t *X, int64_t M,
                                                   const uint16_t *A, const uint16_t *B, int32_t r, float s,
                                                   uint16_t *Y, uint16_t *sU_out, int32_t *dev_status,
                                                   qlora_stream_t stream) {
  if (!W || !X || !A || !B || !Y || M <= 0 || W->rows <= 0 || W->cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (W->cols % qlora::kBlock || r < 8 || r > 64 || r % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (qlora::gemv_fwd_supported(W->rows, W->cols, M))   // a few tokens: one launch, no scratch at all
    return qlora::few_token_forward(W, X, M, A, B, r, s, Y, sU_out, stream);
  // Scratch layout: [sU when the caller does not keep it][fp32 partial sums of s X A^T].
  const size_t su_bytes = sU_out ? 0 : round_up_256(static_cast<size_t>(M) * static_cast<size_t>(r) * 2);
  const size_t part_bytes = qlora::lora_rows_ws_floats(M, W->cols, r) * 4;
  if (su_bytes + part_bytes > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE;   // beyond the fixed maximum
  void *scratch = nullptr;
  qlora_status_t st = scratch_address(&scratch);
  if (st != QLORA_OK) return st;
  unsigned char *base = static_cast<unsigned char *>(scratch);
  uint16_t *sU = sU_out ? sU_out : reinterpret_cast<uint16_t *>(base);
  st = qlora_lora_xa(X, M, W->cols, A, r, s, sU, base + su_bytes, part_bytes, stream);
  if (st != QLORA_OK) return st;
  return qlora_fused_fwd(W, X, M, B, r, sU, Y, nullptr, 0, dev_status, stream);   // whole-tile schedule
}
