// C ABI of the library: argument validation, per-device state and dispatch to
// the kernels in hessian.cu, hinv.cu, quantize.cu, pack.cu, matvec.cu and round2d.cu.  Nothing here
// allocates device memory; every scratch byte comes from the caller.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <cstdlib>
#include <cxxabi.h>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"

namespace gptq {

size_t hessian_workspace_size(int n, int64_t n_tok);
gptq_status hessian_accum(float* H, double* hdiag, const void* X, int64_t n_tok, int n, int64_t ldx, float alpha,
                          void* ws, size_t ws_bytes, cudaStream_t stream);
size_t prepare_workspace_size(int n);
gptq_status prepare_hinv(const float* H, const double* hdiag, int n, float damp, int act_order, int32_t* perm,
                         uint8_t* dead, float* U, void* ws, size_t ws_bytes, cudaStream_t st);
size_t quantize_workspace_size(int64_t rows, int n);
gptq_status quantize_layer(const void* W, gptq_dtype wdt, int64_t rows, int n, const float* U, const int32_t* perm,
                           const uint8_t* dead, int bits, int group, int block, uint8_t* codes, float* scales,
                           uint8_t* zeros, int32_t* g_idx, float* Wq_out, float* row_loss, void* ws, size_t ws_bytes,
                           cudaStream_t st);
gptq_status quantize_rtn(const void* W, gptq_dtype wdt, int64_t rows, int n, int bits, int group, uint8_t* codes,
                         float* scales, uint8_t* zeros, cudaStream_t st);
gptq_status pack_codes(const uint8_t* codes, int64_t rows, int n, int bits, uint32_t* packed, cudaStream_t st);
size_t matvec_workspace_size(int n, int batch, int xdt_bf16);
gptq_status dequant_matvec(const uint32_t* packed, const float* scales, const uint8_t* zeros, const int32_t* g_idx,
                           int64_t rows, int n, int bits, int group, const void* x, int xdt_bf16, int batch, float* y,
                           void* ws, cudaStream_t st);
size_t round2d_workspace_size(int64_t m, int64_t n);
gptq_status round2d(const void* W, int w_bf16, int64_t m, int64_t n, const float* UL, const float* UR, float scale,
                    int clamp, int qmin, int qmax, int32_t* codes, float* E, void* ws, cudaStream_t st);

// Status words of each device: [0] failures of asynchronous kernels (bounded
// waits), [1] the factorization status of gptq_prepare_hinv.
__device__ int g_status_words[2];

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

std::mutex g_mutex;
DeviceInfo g_info[kMaxDevices];
bool g_have[kMaxDevices] = {};
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};  // read by every launch, set from any thread

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

}  // namespace

const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_have[dev]) {
    DeviceInfo d{};
    d.device = dev;
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_status_words) != cudaSuccess) return nullptr;
    d.status = static_cast<int*>(addr);
    if (cudaMemset(d.status, 0, sizeof(int) * 2) != cudaSuccess) return nullptr;
    g_info[dev] = d;
    g_have[dev] = true;
  }
  return &g_info[dev];
}

bool make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                        uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  std::memset(map, 0, sizeof(*map));
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

static std::atomic<int> g_column_loop{0};  // gptq_set_column_loop
int column_loop_mode() { return g_column_loop.load(std::memory_order_relaxed); }

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// ---------------------------------------------------------------------------
// tracing: per-kernel device time from CUDA events around each launch
// ---------------------------------------------------------------------------

namespace {

struct TraceRec {
  cudaEvent_t begin, end;
  const void* kernel;
  int device;
};

std::atomic<bool> g_trace{false};
std::mutex g_trace_mutex;
std::vector<TraceRec> g_trace_recs;                          // launches not yet read
std::vector<std::pair<int, cudaEvent_t>> g_trace_free;       // (device, event) ready for reuse
thread_local cudaEvent_t t_trace_begin = nullptr;            // this thread's launch in progress

cudaEvent_t trace_event(int dev) {  // caller holds g_trace_mutex
  for (size_t i = 0; i < g_trace_free.size(); ++i)
    if (g_trace_free[i].first == dev) {
      cudaEvent_t e = g_trace_free[i].second;
      g_trace_free[i] = g_trace_free.back();
      g_trace_free.pop_back();
      return e;
    }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// "gptq::(anonymous namespace)::gptq_block_kernel<16>(gptq::...)" -> "gptq_block_kernel<16>"
std::string short_kernel_name(const void* kernel) {
  const char* mangled = nullptr;
  if (cudaFuncGetName(&mangled, kernel) != cudaSuccess || mangled == nullptr) return "unknown";
  int ok = -1;
  char* dem = abi::__cxa_demangle(mangled, nullptr, nullptr, &ok);
  std::string name = (ok == 0 && dem != nullptr) ? dem : mangled;
  std::free(dem);
  int depth = 0;  // drop the parameter list: the first '(' outside template brackets
  for (size_t i = 0; i < name.size(); ++i) {
    if (name[i] == '<') ++depth;
    if (name[i] == '>') --depth;
    if (name[i] == '(' && depth == 0 && i > 0 && name.compare(i, 20, "(anonymous namespace") != 0) {
      name.resize(i);
      break;
    }
  }
  if (name.compare(0, 5, "void ") == 0) name.erase(0, 5);  // template instances carry their return type
  const std::string ns[] = {"gptq::(anonymous namespace)::", "gptq::"};
  for (const std::string& p : ns)
    for (size_t at; (at = name.find(p)) != std::string::npos;) name.erase(at, p.size());
  return name;
}

}  // namespace

bool trace_on() { return g_trace.load(std::memory_order_relaxed); }

void trace_begin(cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  std::lock_guard<std::mutex> lock(g_trace_mutex);
  cudaEvent_t e = trace_event(dev);
  if (e != nullptr && cudaEventRecord(e, st) != cudaSuccess) {
    g_trace_free.emplace_back(dev, e);
    e = nullptr;
  }
  t_trace_begin = e;
}

void trace_end(cudaStream_t st, const void* kernel) {
  cudaEvent_t b = t_trace_begin;
  t_trace_begin = nullptr;
  if (b == nullptr) return;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  std::lock_guard<std::mutex> lock(g_trace_mutex);
  cudaEvent_t e = trace_event(dev);
  if (e == nullptr || cudaEventRecord(e, st) != cudaSuccess) {
    g_trace_free.emplace_back(dev, b);
    if (e != nullptr) g_trace_free.emplace_back(dev, e);
    return;
  }
  g_trace_recs.push_back({b, e, kernel, dev});
}

}  // namespace gptq

using namespace gptq;

namespace {
constexpr int kMaxN = 65535;
bool valid_bits(int32_t b) { return b == 2 || b == 3 || b == 4 || b == 8; }
bool valid_block(int32_t b) { return b >= 32 && b <= 128 && b % 32 == 0; }
bool nests(int32_t group, int32_t block) { return group == 0 || block % group == 0 || group % block == 0; }
}  // namespace

extern "C" {

const char* gptq_status_string(gptq_status s) {
  switch (s) {
    case GPTQ_OK: return "ok";
    case GPTQ_ERR_INVALID_ARG: return "invalid argument";
    case GPTQ_ERR_NOT_PD: return "damped Hessian is not positive definite";
    case GPTQ_ERR_NONFINITE: return "non-finite value in the Hessian";
    case GPTQ_ERR_CUDA: return "CUDA error";
    case GPTQ_ERR_UNSUPPORTED: return "unsupported combination";
    case GPTQ_ERR_TIMEOUT: return "bounded in-kernel wait ran out";
  }
  return "unknown status";
}

int32_t gptq_version(void) { return 100; }

uint64_t gptq_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

void gptq_set_column_loop(int32_t mode) { gptq::g_column_loop.store(mode == 1 ? 1 : 0, std::memory_order_relaxed); }

int32_t gptq_get_column_loop(void) { return gptq::column_loop_mode(); }

void gptq_set_wait_limit_ns(uint64_t ns) {
  g_wait_ns.store(ns == UINT64_MAX ? kDefaultWaitNs : ns, std::memory_order_relaxed);
}

void gptq_trace_enable(int32_t on) { g_trace.store(on != 0, std::memory_order_relaxed); }

int32_t gptq_trace_read(gptq_trace_entry* out, int32_t max_entries) {
  std::lock_guard<std::mutex> lock(g_trace_mutex);
  std::map<const void*, std::pair<uint64_t, double>> sums;
  int err = 0;
  for (const TraceRec& r : g_trace_recs) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.end) != cudaSuccess || cudaEventElapsedTime(&ms, r.begin, r.end) != cudaSuccess)
      err = 1;
    auto& acc = sums[r.kernel];
    acc.first += 1;
    acc.second += ms;
    g_trace_free.emplace_back(r.device, r.begin);
    g_trace_free.emplace_back(r.device, r.end);
  }
  g_trace_recs.clear();
  if (err) return -1;
  std::vector<gptq_trace_entry> entries;
  for (const auto& kv : sums) {
    gptq_trace_entry e{};
    const std::string name = short_kernel_name(kv.first);
    std::strncpy(e.name, name.c_str(), sizeof(e.name) - 1);
    e.launches = kv.second.first;
    e.ms = kv.second.second;
    entries.push_back(e);
  }
  std::sort(entries.begin(), entries.end(), [](const gptq_trace_entry& a, const gptq_trace_entry& b) {
    return a.ms > b.ms;
  });
  const int32_t n = static_cast<int32_t>(std::min<size_t>(entries.size(), max_entries > 0 ? max_entries : 0));
  for (int32_t i = 0; i < n; ++i) out[i] = entries[i];
  return n;
}

gptq_status gptq_get_device_status(void* stream) {
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GPTQ_ERR_CUDA;
  int v = 0;
  cudaStream_t st = as_stream(stream);
  if (cudaMemcpyAsync(&v, info->status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaMemsetAsync(info->status, 0, sizeof(int), st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GPTQ_ERR_CUDA;
  return static_cast<gptq_status>(v);
}

size_t gptq_hessian_workspace_size(int32_t n, int64_t n_tok) {
  if (n < 1 || n > kMaxN || n_tok < 0) return 0;
  return hessian_workspace_size(n, n_tok);
}

gptq_status gptq_hessian_accum(float* H, double* hdiag, const void* X, int64_t n_tok, int32_t n, int64_t ldx,
                               float alpha, void* ws, size_t ws_bytes, void* stream) {
  if (H == nullptr || n < 1 || n > kMaxN || n_tok < 0 || n_tok > (int64_t(1) << 31) - 128 || !std::isfinite(alpha))
    return GPTQ_ERR_INVALID_ARG;
  if (n_tok == 0) return GPTQ_OK;
  if (X == nullptr || ldx < n || ldx % 8 != 0 || !aligned(X, 16) || !aligned(H, 16)) return GPTQ_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < hessian_workspace_size(n, n_tok)) return GPTQ_ERR_INVALID_ARG;
  if (hdiag != nullptr && !aligned(hdiag, 8)) return GPTQ_ERR_INVALID_ARG;
  return hessian_accum(H, hdiag, X, n_tok, n, ldx, alpha, ws, ws_bytes, as_stream(stream));
}

size_t gptq_prepare_workspace_size(int32_t n) {
  if (n < 1 || n > kMaxN) return 0;
  return prepare_workspace_size(n);
}

gptq_status gptq_prepare_hinv(const float* H, const double* hdiag, int32_t n, float damp, int32_t act_order,
                              int32_t* perm, uint8_t* dead, float* U, void* ws, size_t ws_bytes, void* stream) {
  if (H == nullptr || U == nullptr || n < 1 || n > kMaxN || !std::isfinite(damp) || damp < 0.0f)
    return GPTQ_ERR_INVALID_ARG;
  if (act_order && perm == nullptr) return GPTQ_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < prepare_workspace_size(n)) return GPTQ_ERR_INVALID_ARG;
  return prepare_hinv(H, hdiag, n, damp, act_order ? 1 : 0, perm, dead, U, ws, ws_bytes, as_stream(stream));
}

size_t gptq_quantize_workspace_size(int64_t rows, int32_t n, int32_t block) {
  if (rows < 0 || n < 1 || n > kMaxN || !valid_block(block)) return 0;
  return quantize_workspace_size(rows, n);
}

int32_t gptq_num_groups(int32_t n, int32_t group) {
  if (n < 1 || group < 0) return 0;
  return group == 0 ? 1 : static_cast<int32_t>((n + group - 1) / group);
}

gptq_status gptq_quantize_layer(const void* W, gptq_dtype wdt, int64_t rows, int32_t n, const float* U,
                                const int32_t* perm, const uint8_t* dead, int32_t bits, int32_t group, int32_t block,
                                uint8_t* codes, float* scales, uint8_t* zeros, int32_t* g_idx, float* Wq_out,
                                float* row_loss, void* ws, size_t ws_bytes, void* stream) {
  if (rows < 0 || n < 1 || n > kMaxN || !valid_bits(bits) || !valid_block(block) || group < 0 || group > n)
    return GPTQ_ERR_INVALID_ARG;
  if (wdt != GPTQ_F32 && wdt != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if (!nests(group, block)) return GPTQ_ERR_UNSUPPORTED;
  if (rows == 0) return GPTQ_OK;
  if (W == nullptr || U == nullptr || codes == nullptr || scales == nullptr || zeros == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < quantize_workspace_size(rows, n)) return GPTQ_ERR_INVALID_ARG;
  return quantize_layer(W, wdt, rows, n, U, perm, dead, bits, group, block, codes, scales, zeros, g_idx, Wq_out,
                        row_loss, ws, ws_bytes, as_stream(stream));
}

gptq_status gptq_quantize_rtn(const void* W, gptq_dtype wdt, int64_t rows, int32_t n, int32_t bits, int32_t group,
                              uint8_t* codes, float* scales, uint8_t* zeros, void* stream) {
  if (rows < 0 || n < 1 || n > kMaxN || !valid_bits(bits) || group < 0 || group > n) return GPTQ_ERR_INVALID_ARG;
  if (wdt != GPTQ_F32 && wdt != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (W == nullptr || codes == nullptr || scales == nullptr || zeros == nullptr) return GPTQ_ERR_INVALID_ARG;
  return quantize_rtn(W, wdt, rows, n, bits, group, codes, scales, zeros, as_stream(stream));
}

int32_t gptq_packed_words_per_row(int32_t n, int32_t bits) {
  if (n < 0 || !valid_bits(bits)) return 0;
  return bits * ((n + 31) / 32);
}

gptq_status gptq_pack(const uint8_t* codes, int64_t rows, int32_t n, int32_t bits, uint32_t* packed, void* stream) {
  if (rows < 0 || n < 1 || !valid_bits(bits)) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (codes == nullptr || packed == nullptr || !aligned(packed, 4)) return GPTQ_ERR_INVALID_ARG;
  return pack_codes(codes, rows, n, bits, packed, as_stream(stream));
}

size_t gptq_matvec_workspace_size(int32_t n, int32_t batch, gptq_dtype xdt) {
  if (n < 1 || batch < 1) return 0;
  return matvec_workspace_size(n, batch, xdt == GPTQ_BF16 ? 1 : 0);
}

gptq_status gptq_dequant_matvec(const uint32_t* packed, const float* scales, const uint8_t* zeros,
                                const int32_t* g_idx, int64_t rows, int32_t n, int32_t bits, int32_t group,
                                const void* x, gptq_dtype xdt, int32_t batch, float* y, void* ws, size_t ws_bytes,
                                void* stream) {
  if (rows < 0 || n < 1 || n > kMaxN || !valid_bits(bits) || group < 0 || group > n || batch < 1 || batch > 8 ||
      (xdt != GPTQ_F32 && xdt != GPTQ_BF16))
    return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (packed == nullptr || scales == nullptr || zeros == nullptr || x == nullptr || y == nullptr ||
      !aligned(packed, 4) || !aligned(scales, 4) || !aligned(y, 4) || !aligned(x, xdt == GPTQ_BF16 ? 2 : 4) ||
      (g_idx != nullptr && !aligned(g_idx, 4)))
    return GPTQ_ERR_INVALID_ARG;
  const size_t need = matvec_workspace_size(n, batch, xdt == GPTQ_BF16 ? 1 : 0);
  if (need > 0 && (ws == nullptr || !aligned(ws, 256) || ws_bytes < need)) return GPTQ_ERR_INVALID_ARG;
  return dequant_matvec(packed, scales, zeros, g_idx, rows, n, bits, group, x, xdt == GPTQ_BF16 ? 1 : 0, batch, y, ws,
                        as_stream(stream));
}

}  // extern "C"

namespace {
// The push kernel's grid spans max(tiles) - 1 target tiles along y (<= 65535).
constexpr int64_t kMax2dDim = 65536LL * 64;
constexpr int32_t kMax2dCode = 1 << 24;  // codes stay exact in fp32
}  // namespace

extern "C" {

size_t gptq2d_workspace_size(int64_t m, int64_t n) {
  if (m < 0 || n < 0 || m > kMax2dDim || n > kMax2dDim) return 0;
  return round2d_workspace_size(m, n);
}

gptq_status gptq2d_round(const void* W, gptq_dtype wdt, int64_t m, int64_t n, const float* UL, const float* UR,
                         float scale, int32_t clamp, int32_t qmin, int32_t qmax, int32_t* codes, float* E, void* ws,
                         size_t ws_bytes, void* stream) {
  if (m < 0 || n < 0 || m > kMax2dDim || n > kMax2dDim || (wdt != GPTQ_F32 && wdt != GPTQ_BF16) ||
      !(scale > 0.f) || !std::isfinite(scale) || (clamp != 0 && clamp != 1))
    return GPTQ_ERR_INVALID_ARG;
  if (clamp == 1 && (qmin > qmax || qmin < -kMax2dCode || qmax > kMax2dCode)) return GPTQ_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return GPTQ_OK;
  if (W == nullptr || UL == nullptr || UR == nullptr || codes == nullptr || !aligned(W, wdt == GPTQ_BF16 ? 2 : 4) ||
      !aligned(UL, 4) || !aligned(UR, 4) || !aligned(codes, 4) || (E != nullptr && !aligned(E, 4)))
    return GPTQ_ERR_INVALID_ARG;
  const size_t need = round2d_workspace_size(m, n);
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < need) return GPTQ_ERR_INVALID_ARG;
  return round2d(W, wdt == GPTQ_BF16 ? 1 : 0, m, n, UL, UR, scale, clamp, qmin, qmax, codes, E, ws,
                 as_stream(stream));
}

}  // extern "C"
