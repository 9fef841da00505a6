// Inference with the packed weights: y[b, r] = sum_c Q[r, c] x[b, c], with
// Q[r, c] = scales[r, g(c)] * (code[r, c] - zeros[r, g(c)]) read straight from
// the packed rows (GPTQ abstract on the "Daily Papers" page: the packed 3/4-bit
// weights run generative inference faster than FP16; GPTQ knowledge note,
// "Tradeoffs": deployment reads packed weights).
//
// The product streams the packed matrix once, so it is bound by HBM: per
// 4-bit weight half a byte is read, a quarter of a bf16 weight.
//
// Layout of the work: one warp per weight row (grid-stride over rows); lane l
// takes the row's runs of 32 codes l, l + 32, ... (a run is `bits` 32-bit
// words, so a warp reads `bits` * 128 contiguous bytes per step).  x is staged
// in shared memory as xs[b][run][i] = x[b][32 run + i] with a 36-float run
// pitch, so that a lane reads four positions of its run with one 16-byte load
// and eight lanes on consecutive runs hit distinct bank groups.  Codes are turned into floats by
// the 2^23 trick: (0x4B000000 | code) read as a float is 2^23 + code exactly.
//
// Groups: when they are contiguous and a whole number of runs (no g_idx,
// group % 32 == 0 or one group per row) a run lies in one group, and its
// contribution is s * (sum_i code_i x_i - z * sum_i x_i), with the run sums of
// x computed once per CTA.  Otherwise (act-order g_idx, or groups that split
// runs) every code looks up its own scale and zero point.
#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kChunkFloats = 16384;  // x floats staged per pass (64 KB + padding)
constexpr int kRunPitch = 36;        // floats per staged run of 32 (16-byte aligned, bank-spread)

// The BITS words of run q of a packed row; 16- or 8-byte loads when the row
// is aligned for them.
template <int BITS>
__device__ __forceinline__ void load_run(const uint32_t* __restrict__ prow, int q, bool vec, uint32_t (&w)[BITS]) {
  const uint32_t* src = prow + q * BITS;
  if (BITS % 4 == 0 && vec) {
#pragma unroll
    for (int k = 0; k < BITS; k += 4) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + k));
      w[k] = v.x;
      w[k + 1] = v.y;
      w[k + 2] = v.z;
      w[k + 3] = v.w;
    }
  } else if (BITS == 2 && vec) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
    w[0] = v.x;
    w[1] = v.y;
  } else {
#pragma unroll
    for (int k = 0; k < BITS; ++k) w[k] = __ldg(src + k);
  }
}

// code i of a run as a float (the mask and the exponent bits in one step)
template <int BITS>
__device__ __forceinline__ float code_f(const uint32_t (&w)[BITS], int i) {
  const int bit = i * BITS;
  const int k = bit >> 5, s = bit & 31;
  uint32_t v = w[k] >> s;
  if (s + BITS > 32) v |= w[k + 1] << (32 - s);
  return __uint_as_float((v & ((1u << BITS) - 1u)) | 0x4B000000u) - 8388608.0f;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Stages x[:, columns of runs q0 .. q0 + nr) (transposed, see above) and, for
// the contiguous-group path, the runs' sums of x.  A warp takes a run at a
// time: its lanes read the run's 32 consecutive values (coalesced), store them
// as one row of xs and add them with a shuffle reduction.
template <int B, bool kFast, typename T>
__device__ __forceinline__ void stage_x(float* xs, float* xsum, const T* __restrict__ x, int n, int batch, int q0,
                                        int nr, int runs_chunk) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();  // the previous chunk is no longer read
  for (int br = warp; br < B * nr; br += kWarps) {
    const int b = br / nr, run = br - b * nr;
    const int c = 32 * (q0 + run) + lane;
    const float v = (b < batch && c < n) ? to_f32<T>(x[static_cast<int64_t>(b) * n + c]) : 0.0f;
    xs[(b * runs_chunk + run) * kRunPitch + lane] = v;
    if (kFast) {
      float t = v;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) xsum[b * runs_chunk + run] = t;
    }
  }
  __syncthreads();
}

template <int BITS, int B, bool kFast, typename T>
__global__ void __launch_bounds__(kThreads) dequant_matvec_kernel(const uint32_t* __restrict__ packed,
                                                                  const float* __restrict__ scales,
                                                                  const uint8_t* __restrict__ zeros,
                                                                  const int32_t* __restrict__ g_idx, int64_t rows,
                                                                  int n, int G, int n_groups, const T* __restrict__ x,
                                                                  int batch, float* __restrict__ y) {
  extern __shared__ float xs[];  // [B][runs_chunk][kRunPitch], then run sums [B][runs_chunk]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int runs = (n + 31) / 32;
  const int words = BITS * runs;
  const int runs_chunk = (kChunkFloats / B) / 32;
  float* xsum = xs + B * runs_chunk * kRunPitch;
  const int64_t row_stride = static_cast<int64_t>(gridDim.x) * kWarps;
  const bool one_pass = runs <= runs_chunk;  // x staged once for all of the CTA's rows
  if (one_pass) stage_x<B, kFast>(xs, xsum, x, n, batch, 0, runs, runs_chunk);

  for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * kWarps; r0 < rows; r0 += row_stride) {
    const int64_t r = r0 + warp;
    float acc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = 0.0f;
    for (int q0 = 0; q0 < runs; q0 += runs_chunk) {
      const int nr = min(runs_chunk, runs - q0);
      if (!one_pass) stage_x<B, kFast>(xs, xsum, x, n, batch, q0, nr, runs_chunk);
      if (r < rows) {
        const uint32_t* prow = packed + r * words;
        const bool vec = (reinterpret_cast<uintptr_t>(prow) % (BITS == 2 ? 8 : 16)) == 0;
        // runs in groups of kPre per lane: all their words are requested
        // before any is used, so the loads of a row overlap
        constexpr int kPre = 4;
        for (int run0 = lane; run0 < nr; run0 += 32 * kPre) {
          uint32_t w[kPre][BITS];
#pragma unroll
          for (int u = 0; u < kPre; ++u) {
            const int run = run0 + 32 * u;
            if (run < nr) load_run<BITS>(prow, q0 + run, vec, w[u]);
          }
#pragma unroll
          for (int u = 0; u < kPre; ++u) {
            const int run = run0 + 32 * u;
            if (run >= nr) break;
            const int q = q0 + run;
            if (kFast) {
              const int g = (32 * q) / G;
              const float sc = __ldg(scales + r * n_groups + g);
              const float z = static_cast<float>(__ldg(zeros + r * n_groups + g));
              float dot[B];
#pragma unroll
              for (int b = 0; b < B; ++b) dot[b] = 0.0f;
#pragma unroll
              for (int i4 = 0; i4 < 32; i4 += 4) {
                const float c0 = code_f<BITS>(w[u], i4), c1 = code_f<BITS>(w[u], i4 + 1);
                const float c2 = code_f<BITS>(w[u], i4 + 2), c3 = code_f<BITS>(w[u], i4 + 3);
#pragma unroll
                for (int b = 0; b < B; ++b) {
                  const float4 xv = *reinterpret_cast<const float4*>(xs + (b * runs_chunk + run) * kRunPitch + i4);
                  dot[b] = fmaf(c0, xv.x, dot[b]);
                  dot[b] = fmaf(c1, xv.y, dot[b]);
                  dot[b] = fmaf(c2, xv.z, dot[b]);
                  dot[b] = fmaf(c3, xv.w, dot[b]);
                }
              }
#pragma unroll
              for (int b = 0; b < B; ++b) acc[b] = fmaf(sc, fmaf(-z, xsum[b * runs_chunk + run], dot[b]), acc[b]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int c = min(32 * q + i, n - 1);  // codes past n are zero; x there is zero
                const int g = g_idx != nullptr ? __ldg(g_idx + c) : c / G;
                const float sc = __ldg(scales + r * n_groups + g);
                const float z = static_cast<float>(__ldg(zeros + r * n_groups + g));
                const float qv = sc * (code_f<BITS>(w[u], i) - z);
#pragma unroll
                for (int b = 0; b < B; ++b) acc[b] = fmaf(qv, xs[(b * runs_chunk + run) * kRunPitch + i], acc[b]);
              }
            }
          }
        }
      }
    }
    if (r < rows) {
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float v = acc[b];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && b < batch) y[static_cast<int64_t>(b) * rows + r] = v;
      }
    }
  }
}

size_t smem_bytes(int B) {
  const int runs_chunk = (kChunkFloats / B) / 32;
  return (static_cast<size_t>(B) * runs_chunk * kRunPitch + static_cast<size_t>(B) * runs_chunk) * sizeof(float);
}

template <int BITS, int B, bool kFast, typename T>
gptq_status launch_matvec(const uint32_t* packed, const float* scales, const uint8_t* zeros, const int32_t* g_idx,
                          int64_t rows, int n, int G, int n_groups, const T* x, int batch, float* y,
                          cudaStream_t st) {
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GPTQ_ERR_CUDA;
  const size_t smem = smem_bytes(B);
  static std::atomic<bool> attr_set[64] = {};  // per device, shared by host threads
  if (!attr_set[info->device]) {
    if (cudaFuncSetAttribute(dequant_matvec_kernel<BITS, B, kFast, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    attr_set[info->device] = true;
  }
  // as many CTAs as fit at once (x is staged once per CTA), each taking rows
  // in a grid-stride loop
  const int per_sm = std::max(1, std::min(8, static_cast<int>((228 * 1024) / (smem + 1024))));
  const int64_t ctas = std::min<int64_t>(ceil_div(rows, static_cast<int64_t>(kWarps)), int64_t(info->sm_count) * per_sm);
  launch(dequant_matvec_kernel<BITS, B, kFast, T>, static_cast<unsigned>(ctas), kThreads, smem, st, packed, scales, zeros,
         g_idx, rows, n, G, n_groups, x, batch, y);
  return launch_status();
}

template <int BITS, int B, typename T>
gptq_status dispatch_fast(bool fast, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                          const int32_t* g_idx, int64_t rows, int n, int G, int n_groups, const T* x, int batch,
                          float* y, cudaStream_t st) {
  return fast ? launch_matvec<BITS, B, true>(packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st)
              : launch_matvec<BITS, B, false>(packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
}

template <int BITS, typename T>
gptq_status dispatch_batch(bool fast, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                           const int32_t* g_idx, int64_t rows, int n, int G, int n_groups, const T* x, int batch,
                           float* y, cudaStream_t st) {
  if (batch <= 1) return dispatch_fast<BITS, 1>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
  if (batch <= 2) return dispatch_fast<BITS, 2>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
  if (batch <= 4) return dispatch_fast<BITS, 4>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
  return dispatch_fast<BITS, 8>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
}

template <typename T>
gptq_status dispatch_bits(int bits, bool fast, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                          const int32_t* g_idx, int64_t rows, int n, int G, int n_groups, const T* x, int batch,
                          float* y, cudaStream_t st) {
  switch (bits) {
    case 2: return dispatch_batch<2>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
    case 3: return dispatch_batch<3>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
    case 4: return dispatch_batch<4>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
    default: return dispatch_batch<8>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
  }
}

}  // namespace

size_t matvec_workspace_size(int, int, int) { return 0; }

gptq_status dequant_matvec(const uint32_t* packed, const float* scales, const uint8_t* zeros, const int32_t* g_idx,
                           int64_t rows, int n, int bits, int group, const void* x, int xdt_bf16, int batch, float* y,
                           void*, cudaStream_t st) {
  const int G = group > 0 ? group : n;
  const int n_groups = static_cast<int>(ceil_div(n, G));
  const bool fast = g_idx == nullptr && (G % 32 == 0 || G == n);
  if (xdt_bf16)
    return dispatch_bits(bits, fast, packed, scales, zeros, g_idx, rows, n, G, n_groups,
                         static_cast<const __nv_bfloat16*>(x), batch, y, st);
  return dispatch_bits(bits, fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, static_cast<const float*>(x),
                       batch, y, st);
}

}  // namespace gptq
