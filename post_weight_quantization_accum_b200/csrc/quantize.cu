// The GPTQ column loop and the round-to-nearest baseline.
//
// GPTQ knowledge note, "How It Works": all output rows follow one column
// order; after a column is rounded, inverse-Hessian information (a row of the
// upper factor U) moves the columns not yet quantized; 128-column blocks
// accumulate their corrections before one global update of the rest.
// "Daily Papers" GPTQ-2D abstract: fixed order, one entry at a time, errors fed
// forward through a triangular matrix.
//
// Per block [i1, i2) of processing positions:
//   gptq_block_kernel   one warp per weight row; lane l holds columns
//                       l, l+32, l+64, l+96 of the block in registers; the
//                       block's U tile and 1/U_jj sit in shared memory.  Step
//                       j broadcasts w_j with a shuffle, rounds it on the grid,
//                       forms e_j = (w_j - deq_j) / U_jj and updates the
//                       later columns of the block with one FMA per lane and
//                       slot.  Group (scale, zero) are fixed when a group
//                       starts, from the current values (warp min/max).
//   trailing_update_tc (trailing.cu)   W[:, i2:] -= E[:, i1:i2] * U[i1:i2, i2:]
//                       on the tensor cores, fp32-accurate through a 3-term
//                       tf32 split; the block kernel writes E as its tf32
//                       hi / lo halves.
#include <algorithm>

#include "common.cuh"
#include "grid.cuh"

namespace gptq {
namespace {

constexpr int kBMax = 128;       // largest block width
constexpr int kRowsPerCta = 16;  // warps (= rows) per CTA of the block kernel
constexpr size_t kBlockSmem = (kBMax * kBMax + kBMax) * sizeof(float);

template <typename T>
__device__ __forceinline__ float load_w(const T* p);
template <>
__device__ __forceinline__ float load_w<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_w<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Wk[r, p] = dead[perm[p]] ? 0 : W[r, perm[p]]  (processing order, fp32).
template <typename T>
__global__ void gather_weights_kernel(const T* __restrict__ W, const int32_t* __restrict__ perm,
                                      const uint8_t* __restrict__ dead, int64_t rows, int n, float* __restrict__ Wk) {
  const int64_t total = rows * n;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / n;
    const int p = static_cast<int>(e - r * n);
    const int c = perm != nullptr ? perm[p] : p;
    const bool d = dead != nullptr && dead[c];
    Wk[e] = d ? 0.0f : load_w<T>(W + r * n + c);
  }
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

struct BlockArgs {
  float* Wk;             // [rows, n] working weights, processing order
  const float* U;        // [n, n]
  int64_t rows;
  int n;
  int i1, bw;            // block start and width
  int G;                 // group size (n when one group per row)
  int n_groups;
  float maxq;
  float* E_hi;           // [rows, kBMax] scaled errors of the block, tf32 high part
  float* E_lo;           // [rows, kBMax] and the remainder e - hi
  uint8_t* codes;        // [rows, n] processing order
  float* scales;         // [rows, n_groups]
  uint8_t* zeros;        // [rows, n_groups]
  float* row_loss;       // [rows] or nullptr
};

__global__ void __launch_bounds__(kRowsPerCta * 32, 1) gptq_block_kernel(BlockArgs a) {
  extern __shared__ float dyn_smem[];
  float* us = dyn_smem;              // [kBMax][kBMax] U tile of the block
  float* rdiag = dyn_smem + kBMax * kBMax;
  const int bw = a.bw;
  // U tile: each thread issues a batch of loads before storing any of them,
  // 16-byte loads when the rows allow it.
  if (bw == kBMax && a.n % 4 == 0) {
    constexpr int kVec = kBMax * kBMax / 4 / (kRowsPerCta * 32);  // 8 float4 per thread
    float4 v[kVec];
#pragma unroll
    for (int q = 0; q < kVec; ++q) {
      const int e = threadIdx.x + q * kRowsPerCta * 32, j = e / (kBMax / 4), k4 = e % (kBMax / 4);
      v[q] = __ldg(reinterpret_cast<const float4*>(a.U + static_cast<size_t>(a.i1 + j) * a.n + a.i1) + k4);
    }
#pragma unroll
    for (int q = 0; q < kVec; ++q) reinterpret_cast<float4*>(us)[threadIdx.x + q * kRowsPerCta * 32] = v[q];
  } else {
    for (int e0 = 0; e0 < kBMax * kBMax; e0 += 8 * kRowsPerCta * 32) {
      float v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int e = e0 + threadIdx.x + q * kRowsPerCta * 32, j = e / kBMax, k = e % kBMax;
        v[q] = (j < bw && k < bw) ? __ldg(a.U + static_cast<size_t>(a.i1 + j) * a.n + a.i1 + k) : 0.0f;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) us[e0 + threadIdx.x + q * kRowsPerCta * 32] = v[q];
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < bw; j += blockDim.x) rdiag[j] = 1.0f / us[j * kBMax + j];
  __syncthreads();

  const int lane = threadIdx.x % 32;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + threadIdx.x / 32;
  if (r >= a.rows) return;
  float* wrow = a.Wk + r * a.n;

  float w[4], ek[4], qk[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int k = lane + 32 * m;
    w[m] = k < bw ? wrow[a.i1 + k] : 0.0f;
    ek[m] = 0.0f;
    qk[m] = 0.0f;
  }
  // A group that began in an earlier block keeps the (scale, zero) that
  // block fixed; they are read back from the outputs.
  GridParams gp{1.0f, 0.0f};
  if (a.i1 % a.G != 0) {
    const int g = a.i1 / a.G;
    gp.scale = a.scales[r * a.n_groups + g];
    gp.zero = static_cast<float>(a.zeros[r * a.n_groups + g]);
  }
  float loss = 0.0f;

#pragma unroll
  for (int m = 0; m < 4; ++m) {
    if (32 * m >= bw) break;
    for (int jj = 0; jj < 32; ++jj) {
      const int j = 32 * m + jj;
      if (j >= bw) break;
      const int col = a.i1 + j;
      if (col % a.G == 0) {
        // Group start: (scale, zero) from the group's current values.
        const int gend = min(col + a.G, a.n);
        float lo = INFINITY, hi = -INFINITY;
#pragma unroll
        for (int m2 = 0; m2 < 4; ++m2) {
          const int k = lane + 32 * m2;
          if (k >= j && k < bw && a.i1 + k < gend) {
            lo = fminf(lo, w[m2]);
            hi = fmaxf(hi, w[m2]);
          }
        }
        for (int c = a.i1 + bw + lane; c < gend; c += 32) {
          const float v = wrow[c];
          lo = fminf(lo, v);
          hi = fmaxf(hi, v);
        }
        lo = warp_min(lo);
        hi = warp_max(hi);
        gp = grid_params(lo, hi, a.maxq);
        if (lane == 0) {
          const int g = col / a.G;
          a.scales[r * a.n_groups + g] = gp.scale;
          a.zeros[r * a.n_groups + g] = static_cast<uint8_t>(gp.zero);
        }
      }
      const float wj = __shfl_sync(0xffffffffu, w[m], jj);
      const float q = grid_code(wj, gp, a.maxq);
      const float e = __fmul_rn(__fsub_rn(wj, grid_deq(q, gp)), rdiag[j]);
      loss = fmaf(e, e, loss);
      if (lane == jj) {
        ek[m] = e;
        qk[m] = q;
      }
      const float* urow = us + j * kBMax;
#pragma unroll
      for (int m2 = 0; m2 < 4; ++m2) {
        const int k = lane + 32 * m2;
        if (k > j && k < bw) w[m2] = fmaf(-e, urow[k], w[m2]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int k = lane + 32 * m;
    if (k < bw) {
      const float hi = __uint_as_float(__float_as_uint(ek[m]) & 0xffffe000u);
      a.E_hi[r * kBMax + k] = hi;
      a.E_lo[r * kBMax + k] = ek[m] - hi;
      a.codes[r * a.n + a.i1 + k] = static_cast<uint8_t>(qk[m]);
    }
  }
  if (lane == 0 && a.row_loss != nullptr) a.row_loss[r] += loss;
}

// codes[r, perm[p]] = codes_p[r, p]; optional dequantized weights and g_idx.
__global__ void outputs_kernel(const uint8_t* __restrict__ codes_p, const int32_t* __restrict__ perm,
                               const float* __restrict__ scales, const uint8_t* __restrict__ zeros, int64_t rows,
                               int n, int G, int n_groups, uint8_t* __restrict__ codes, float* __restrict__ Wq,
                               int32_t* __restrict__ g_idx) {
  const int64_t total = rows * n;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / n;
    const int p = static_cast<int>(e - r * n);
    const int c = perm != nullptr ? perm[p] : p;
    const uint8_t q = codes_p[e];
    if (codes != codes_p) codes[r * n + c] = q;
    const int g = p / G;
    if (Wq != nullptr) {
      GridParams gp{scales[r * n_groups + g], static_cast<float>(zeros[r * n_groups + g])};
      Wq[r * n + c] = grid_deq(static_cast<float>(q), gp);
    }
    if (r == 0 && g_idx != nullptr) g_idx[c] = g;
  }
}

// Round-to-nearest: one warp per (row, group), groups of G original columns.
template <typename T>
__global__ void rtn_kernel(const T* __restrict__ W, int64_t rows, int n, int G, int n_groups, float maxq,
                           uint8_t* __restrict__ codes, float* __restrict__ scales, uint8_t* __restrict__ zeros) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (wid >= rows * n_groups) return;
  const int64_t r = wid / n_groups;
  const int g = static_cast<int>(wid % n_groups);
  const int c0 = g * G, c1 = min(c0 + G, n);
  const T* wr = W + r * n;
  float lo = INFINITY, hi = -INFINITY;
  for (int c = c0 + lane; c < c1; c += 32) {
    const float v = load_w<T>(wr + c);
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
  lo = warp_min(lo);
  hi = warp_max(hi);
  const GridParams gp = grid_params(lo, hi, maxq);
  for (int c = c0 + lane; c < c1; c += 32) codes[r * n + c] = static_cast<uint8_t>(grid_code(load_w<T>(wr + c), gp, maxq));
  if (lane == 0) {
    scales[r * n_groups + g] = gp.scale;
    zeros[r * n_groups + g] = static_cast<uint8_t>(gp.zero);
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct QuantLayout {
  size_t wk, e_hi, e_lo, codes_p, u_hi, u_lo, total;
  int64_t ldu;
};

QuantLayout quant_layout(int64_t rows, int n) {
  QuantLayout l{};
  l.ldu = (n + 3) / 4 * 4;  // 16-byte row pitch for the tensor-map loads
  size_t off = 0;
  l.wk = off;
  off += align256(static_cast<size_t>(rows) * n * sizeof(float));
  l.e_hi = off;
  off += align256(static_cast<size_t>(rows) * kBMax * sizeof(float));
  l.e_lo = off;
  off += align256(static_cast<size_t>(rows) * kBMax * sizeof(float));
  l.codes_p = off;
  off += align256(static_cast<size_t>(rows) * n);
  l.u_hi = off;
  off += align256(static_cast<size_t>(n) * l.ldu * sizeof(float));
  l.u_lo = off;
  off += align256(static_cast<size_t>(n) * l.ldu * sizeof(float));
  l.total = off;
  return l;
}

}  // namespace

size_t quantize_workspace_size(int64_t rows, int n) { return quant_layout(rows, n).total; }

gptq_status split_u_tf32(const float* U, int n, int64_t ldu, float* U_hi, float* U_lo, cudaStream_t st);
gptq_status trailing_update_tc(float* W, int64_t ldw, int M, int N, int K, int c0, int k0, const float* E_hi,
                               const float* E_lo, int64_t lde, const float* U_hi, const float* U_lo, int64_t ldu,
                               int n_u, cudaStream_t st);

gptq_status quantize_layer(const void* W, gptq_dtype wdt, int64_t rows, int n, const float* U, const int32_t* perm,
                           const uint8_t* dead, int bits, int group, int block, uint8_t* codes, float* scales,
                           uint8_t* zeros, int32_t* g_idx, float* Wq_out, float* row_loss, void* ws, size_t ws_bytes,
                           cudaStream_t st) {
  const QuantLayout l = quant_layout(rows, n);
  if (ws_bytes < l.total) return GPTQ_ERR_INVALID_ARG;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* Wk = reinterpret_cast<float*>(w + l.wk);
  float* E_hi = reinterpret_cast<float*>(w + l.e_hi);
  float* E_lo = reinterpret_cast<float*>(w + l.e_lo);
  float* U_hi = reinterpret_cast<float*>(w + l.u_hi);
  float* U_lo = reinterpret_cast<float*>(w + l.u_lo);
  uint8_t* codes_p = perm != nullptr ? w + l.codes_p : codes;
  const int G = group > 0 ? group : n;
  const int n_groups = static_cast<int>(ceil_div(n, G));

  const unsigned gg = static_cast<unsigned>(std::min<int64_t>(ceil_div(rows * n, 256), 148 * 64));
  if (wdt == GPTQ_BF16)
    launch(gather_weights_kernel<__nv_bfloat16>, gg, 256, 0, st, static_cast<const __nv_bfloat16*>(W), perm, dead, rows,
                                                             n, Wk);
  else
    launch(gather_weights_kernel<float>, gg, 256, 0, st, static_cast<const float*>(W), perm, dead, rows, n, Wk);
  if (row_loss != nullptr && cudaMemsetAsync(row_loss, 0, static_cast<size_t>(rows) * sizeof(float), st) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
  if (split_u_tf32(U, n, l.ldu, U_hi, U_lo, st) != GPTQ_OK) return GPTQ_ERR_CUDA;

  BlockArgs a;
  a.Wk = Wk;
  a.U = U;
  a.rows = rows;
  a.n = n;
  a.G = G;
  a.n_groups = n_groups;
  a.maxq = static_cast<float>((1 << bits) - 1);
  a.E_hi = E_hi;
  a.E_lo = E_lo;
  a.codes = codes_p;
  a.scales = scales;
  a.zeros = zeros;
  a.row_loss = row_loss;
  const unsigned block_ctas = static_cast<unsigned>(ceil_div(rows, kRowsPerCta));
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(gptq_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kBlockSmem)) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    attr_set = true;
  }
  for (int i1 = 0; i1 < n; i1 += block) {
    a.i1 = i1;
    a.bw = std::min(block, n - i1);
    launch(gptq_block_kernel, block_ctas, kRowsPerCta * 32, kBlockSmem, st, a);
    const int i2 = i1 + a.bw;
    if (i2 < n) {
      const gptq_status ts = trailing_update_tc(Wk, n, static_cast<int>(rows), n - i2, a.bw, i2, i1, E_hi, E_lo,
                                                kBMax, U_hi, U_lo, l.ldu, n, st);
      if (ts != GPTQ_OK) return ts;
    }
  }
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
  if (codes_p != codes || Wq_out != nullptr || g_idx != nullptr) {
    launch(outputs_kernel, gg, 256, 0, st, codes_p, perm, scales, zeros, rows, n, G, n_groups, codes, Wq_out, g_idx);
    if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

gptq_status quantize_rtn(const void* W, gptq_dtype wdt, int64_t rows, int n, int bits, int group, uint8_t* codes,
                         float* scales, uint8_t* zeros, cudaStream_t st) {
  const int G = group > 0 ? group : n;
  const int n_groups = static_cast<int>(ceil_div(n, G));
  const int64_t warps = rows * n_groups;
  const unsigned grid = static_cast<unsigned>(ceil_div(warps * 32, 256));
  const float maxq = static_cast<float>((1 << bits) - 1);
  if (wdt == GPTQ_BF16)
    launch(rtn_kernel<__nv_bfloat16>, grid, 256, 0, st, static_cast<const __nv_bfloat16*>(W), rows, n, G, n_groups, maxq,
                                                    codes, scales, zeros);
  else
    launch(rtn_kernel<float>, grid, 256, 0, st, static_cast<const float*>(W), rows, n, G, n_groups, maxq, codes, scales,
                                            zeros);
  return launch_status();
}

}  // namespace gptq
