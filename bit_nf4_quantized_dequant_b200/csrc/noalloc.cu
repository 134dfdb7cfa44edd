// Allocation-free variant of the QLoRA linear forward.
//
// qlora_linear_fwd needs a caller-provided workspace: for a few tokens the
// partial sums and flags of its persistent launch and the pieces of s X A^T,
// for more tokens sU (when the caller does not keep it) and, up to 64 tokens,
// the fp32 partial tiles of the GEMM's stream-K schedule. Some callers have no
// way to provide one at the point where they run the layer: a host that hands
// the library only its inputs and outputs and owns no allocator of its own (a
// plug-in inside someone else's runtime), a serving process that has given all
// device memory to a fixed pool up front, or code that must not call
// cudaMalloc between launches because that call can synchronise the device.
// For them, qlora_linear_fwd_noalloc takes its scratch from one fixed array
// compiled into this library instead of from the caller, and otherwise runs
// exactly the launches qlora_linear_fwd runs, so the results are the same bits.
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

// The shared scratch. Its first 256 bytes are the few-token launch's counter
// page: zero at load (a __device__ array is zero-initialised) and left zero by
// every call that completes; every other byte a call reads it writes first.
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
  // every argument is checked as qlora_linear_fwd checks it, before anything runs
  qlora_status_t st = qlora::linear_fwd_check(W, X, M, A, B, r, s, Y, sU_out, dev_status);
  if (st != QLORA_OK) return st;
  const int64_t N = W->rows, K = W->cols;
  const size_t need = qlora::linear_fwd_scratch_bytes(M, N, K, r, sU_out != nullptr);
  if (need > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE;   // beyond the fixed maximum
  void *scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != QLORA_OK) return st;
  // [the few-token launch's counter page, zero between calls][the rest]
  unsigned char *cnt = static_cast<unsigned char *>(scratch);
  unsigned char *base = cnt + qlora::kSmallCounterBytes;
  const size_t rest = need - qlora::kSmallCounterBytes;
  if (M <= qlora::kSmallM)   // the few-token launch: its partials and pieces of s X A^T
    return qlora::linear_fwd_run(W, X, M, A, B, r, s, Y, sU_out, cnt, nullptr, base, rest, dev_status, stream);
  // [sU when the caller does not keep it][the GEMM's stream-K partials, up to 64 tokens]
  const size_t su_bytes = sU_out ? 0 : round_up_256(static_cast<size_t>(M) * static_cast<size_t>(r) * 2);
  void *gemm_ws = M <= 64 ? static_cast<void *>(base + su_bytes) : nullptr;
  return qlora::linear_fwd_run(W, X, M, A, B, r, s, Y, sU_out, cnt, reinterpret_cast<uint16_t *>(base), gemm_ws,
                               M <= 64 ? rest - su_bytes : 0, dev_status, stream);
}
