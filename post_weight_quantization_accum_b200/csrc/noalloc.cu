// Allocation-free variant of the GPTQ column loop.
//
// Some callers cannot hand this library a workspace: code that must not call
// cudaMalloc/cudaFree (cudaFree synchronizes the whole device, which a
// latency-sensitive caller cannot afford), plugins that run inside a host
// application which owns every byte of device memory through its own pool,
// and callers that are not allowed to allocate at all.  For them,
// gptq_quantize_layer_noalloc runs the same kernels as gptq_quantize_layer
// with its scratch in a fixed device array compiled into this library.
//
// The array costs every GPU that loads the library kNoAllocScratchBytes of
// device memory until the process exits.  All calls share it: two calls
// whose kernels overlap on the GPU (different streams, or different host
// threads on one device) race on it and give wrong results.  The array keeps
// whatever the last call left in it; the column loop overwrites every byte it
// reads before reading it, so nothing in it needs clearing between calls.
#include <mutex>

#include "common.cuh"

namespace gptq {

size_t quantize_workspace_size(int64_t rows, int n);
gptq_status quantize_layer(const void* W, gptq_dtype wdt, int64_t rows, int n, const float* U, const int32_t* perm,
                           const uint8_t* dead, int bits, int group, int block, uint8_t* codes, float* scales,
                           uint8_t* zeros, int32_t* g_idx, float* Wq_out, float* row_loss, void* ws, size_t ws_bytes,
                           cudaStream_t st);

namespace {

constexpr size_t kNoAllocScratchBytes = GPTQ_NOALLOC_SCRATCH_BYTES;  // 16 MiB
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code `g_noalloc_scratch` only names the
// symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device, with that device current); nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace gptq

extern "C" gptq_status gptq_quantize_layer_noalloc(const void* W, gptq_dtype wdt, int64_t rows, int32_t n,
                                                   const float* U, const int32_t* perm, const uint8_t* dead,
                                                   int32_t bits, int32_t group, int32_t block, uint8_t* codes,
                                                   float* scales, uint8_t* zeros, int32_t* g_idx, float* Wq_out,
                                                   float* row_loss, void* stream) {
  using namespace gptq;
  if (rows < 0 || n < 1 || n > 65535 || !(bits == 2 || bits == 3 || bits == 4 || bits == 8) ||
      !(block >= 32 && block <= 128 && block % 32 == 0) || group < 0 || group > n)
    return GPTQ_ERR_INVALID_ARG;
  if (wdt != GPTQ_F32 && wdt != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if (!(group == 0 || block % group == 0 || group % block == 0)) return GPTQ_ERR_UNSUPPORTED;
  if (rows == 0) return GPTQ_OK;
  if (W == nullptr || U == nullptr || codes == nullptr || scales == nullptr || zeros == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  const size_t need = quantize_workspace_size(rows, n);
  if (need > kNoAllocScratchBytes) return GPTQ_ERR_INVALID_ARG;  // layer too large for the fixed scratch
  void* ws = scratch_on_current_device();
  if (ws == nullptr) return GPTQ_ERR_CUDA;
  return quantize_layer(W, wdt, rows, n, U, perm, dead, bits, group, block, codes, scales, zeros, g_idx, Wq_out,
                        row_loss, ws, kNoAllocScratchBytes, static_cast<cudaStream_t>(stream));
}
