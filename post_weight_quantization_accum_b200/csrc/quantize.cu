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
//   gptq_block_kernel   one thread per weight row (32 rows per CTA).  The
//                       block's 128 columns are handled as four 32-column
//                       sub-blocks: the current sub-block lives in registers
//                       (fully unrolled, so every index is a constant), the
//                       rest of the block in padded shared memory.  Step j
//                       rounds w_j on the grid, forms e_j = (w_j - deq_j) / U_jj
//                       and updates the later columns of the sub-block; after
//                       a sub-block its 32 errors update the later sub-blocks
//                       from a transposed copy of the U tile.  Group (scale,
//                       zero) come from a thread-local min/max when a group
//                       starts.  Per row and column this costs a few
//                       instructions instead of a warp-wide step.
//   trailing_update_tc (trailing.cu)   W[:, i2:] -= E[:, i1:i2] * U[i1:i2, i2:]
//                       on the tensor cores, fp32-accurate through a 3-term
//                       tf32 split; the block kernel writes E as its tf32
//                       hi / lo halves.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "grid.cuh"

namespace gptq {
namespace {

constexpr int kBMax = 128;        // largest block width
constexpr int kSub = 32;          // columns of a register sub-block
constexpr int kRowsPerCta = 32;   // rows (= threads) per CTA of the block kernel
constexpr int kWPitch = kBMax + 1;  // shared-memory pitch of a row of the block (no bank conflicts)
constexpr size_t kBlockSmem = (3 * kBMax * kBMax + kRowsPerCta * kWPitch + kBMax) * sizeof(float) + 16;

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
  int block;             // nominal block width (the U-tile box is block x block)
  int G;                 // group size (n when one group per row)
  int n_groups;
  float maxq;
  float* E_hi;           // [rows, kBMax] scaled errors of the block, tf32 high part
  float* E_lo;           // [rows, kBMax] and the remainder e - hi
  uint8_t* codes;        // [rows, n] processing order
  float* scales;         // [rows, n_groups]
  uint8_t* zeros;        // [rows, n_groups]
  float* row_loss;       // [rows] or nullptr
  const float2* ext_minmax;  // [rows] (min, max) of a group's columns beyond this block, or nullptr
  int u_tma;                 // 1: the U tile arrives by TMA (u_map), 0: by plain loads
  uint64_t wait_ns;
  int* status;
};

__global__ void __launch_bounds__(kRowsPerCta, 1)
    gptq_block_kernel(const __grid_constant__ CUtensorMap u_map, const __grid_constant__ CUtensorMap uth_map,
                      const __grid_constant__ CUtensorMap utl_map, BlockArgs a) {
  extern __shared__ __align__(128) float dyn_smem[];
  float* us = dyn_smem;                        // [kBMax][kBMax] U tile, us[j][k] = U[i1 + j][i1 + k]
  float* ut = us + kBMax * kBMax;              // [kBMax][kBMax] transposed, ut[k][j] = us[j][k]
  float* tmp = ut + kBMax * kBMax;             // [kBMax][kBMax] landing area of the transposed low half
  float* wsm = tmp + kBMax * kBMax;            // [kRowsPerCta][kWPitch] the rows' block of weights
  float* rdiag = wsm + kRowsPerCta * kWPitch;  // [kBMax] 1 / U_jj
  uint64_t* bar = reinterpret_cast<uint64_t*>(rdiag + kBMax);
  const int bw = a.bw;
  const int tid = threadIdx.x;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kRowsPerCta;
  const int B = a.block;

  // Tiles by TMA (entries past the matrix read as zero): U's block x block
  // tile, and the same tile transposed as the two tf32 halves the trailing
  // update uses (hi + lo == U exactly).  Without 16-byte aligned rows of U the
  // natural tile is rebuilt from the transposed one.
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
    const uint32_t tile = static_cast<uint32_t>(B * B * sizeof(float));
    mbar_arrive_expect_tx(bar, a.u_tma ? 3 * tile : 2 * tile);
    if (a.u_tma) tma_load_2d(us, &u_map, bar, a.i1, a.i1);
    tma_load_2d(ut, &uth_map, bar, a.i1, a.i1);
    tma_load_2d(tmp, &utl_map, bar, a.i1, a.i1);
  }
  __syncthreads();  // the barrier is initialized before anyone waits on it
  // the CTA's rows of the block (row rr of the tile is weight row r0 + rr),
  // one coalesced row per load instruction, 16 rows in flight
  const bool vec_w = (a.n % 4 == 0);
  for (int rr0 = 0; rr0 < kRowsPerCta; rr0 += 16) {
    float4 v[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int64_t r = r0 + rr0 + q;
      const int k = 4 * tid;
      if (r < a.rows && vec_w && k + 3 < bw) {
        v[q] = *reinterpret_cast<const float4*>(a.Wk + r * a.n + a.i1 + k);
      } else {
        const float* src = a.Wk + r * a.n + a.i1 + k;
        v[q].x = (r < a.rows && k + 0 < bw) ? src[0] : 0.0f;
        v[q].y = (r < a.rows && k + 1 < bw) ? src[1] : 0.0f;
        v[q].z = (r < a.rows && k + 2 < bw) ? src[2] : 0.0f;
        v[q].w = (r < a.rows && k + 3 < bw) ? src[3] : 0.0f;
      }
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      float* d = wsm + (rr0 + q) * kWPitch + 4 * tid;
      d[0] = v[q].x;
      d[1] = v[q].y;
      d[2] = v[q].z;
      d[3] = v[q].w;
    }
  }
  if (!mbar_wait(bar, 0u, a.wait_ns)) set_status(a.status, GPTQ_ERR_TIMEOUT);
  __syncthreads();
  // Spread the packed B x B boxes to pitch kBMax (from the last row down, so
  // no entry is overwritten before it is read), zeroing outside the block.
  // Rows past the block are zero already unless B < kBMax; they are written
  // explicitly either way.
  for (int j = kBMax - 1; j >= 0; --j) {
    float h[kBMax / kRowsPerCta], l[kBMax / kRowsPerCta], u[kBMax / kRowsPerCta];
#pragma unroll
    for (int m = 0; m < kBMax / kRowsPerCta; ++m) {  // the whole row is read ...
      const int k = tid + m * kRowsPerCta;
      const bool in = j < bw && k < bw;
      h[m] = in ? ut[j * B + k] : 0.0f;
      l[m] = in ? tmp[j * B + k] : 0.0f;
      u[m] = in && a.u_tma ? us[j * B + k] : 0.0f;
    }
    __syncwarp();
#pragma unroll
    for (int m = 0; m < kBMax / kRowsPerCta; ++m) {  // ... before any of it is written
      const int k = tid + m * kRowsPerCta;
      ut[j * kBMax + k] = h[m] + l[m];
      if (a.u_tma) us[j * kBMax + k] = u[m];
    }
    __syncwarp();
  }
  __syncthreads();
  if (!a.u_tma) {
    for (int e = tid; e < kBMax * kBMax; e += kRowsPerCta) {
      const int j = e / kBMax, k = e % kBMax;
      us[e] = ut[k * kBMax + j];
    }
  }
  for (int j = tid; j < kBMax; j += kRowsPerCta) rdiag[j] = j < bw ? 1.0f / ut[j * kBMax + j] : 0.0f;
  __syncthreads();

  const int64_t r = r0 + tid;
  const bool valid = r < a.rows;
  float* wrow = wsm + tid * kWPitch;
  // A group that began in an earlier block keeps the (scale, zero) that
  // block fixed; they are read back from the outputs.
  GridParams gp{1.0f, 0.0f};
  if (valid && a.i1 % a.G != 0) {
    const int g = a.i1 / a.G;
    gp.scale = a.scales[r * a.n_groups + g];
    gp.zero = static_cast<float>(a.zeros[r * a.n_groups + g]);
  }
  float loss = 0.0f;
  int gpos = a.i1 % a.G;  // position of the current column inside its group

  for (int sb = 0; sb * kSub < bw; ++sb) {
    const int base = sb * kSub;
    float w[kSub], e[kSub];
    uint32_t cw[kSub / 4];
#pragma unroll
    for (int k = 0; k < kSub; ++k) w[k] = wrow[base + k];
#pragma unroll
    for (int k = 0; k < kSub / 4; ++k) cw[k] = 0u;

#pragma unroll
    for (int jj = 0; jj < kSub; ++jj) {
      const int j = base + jj;
      e[jj] = 0.0f;
      if (j < bw) {
        const int col = a.i1 + j;
        const bool group_start = gpos == 0;
        if (++gpos == a.G) gpos = 0;
        if (group_start) {
          // group start: (scale, zero) from the group's current values
          const int gend = min(col + a.G, a.n);
          float lo = INFINITY, hi = -INFINITY;
#pragma unroll
          for (int k = jj; k < kSub; ++k)
            if (base + k < bw && a.i1 + base + k < gend) {
              lo = fminf(lo, w[k]);
              hi = fmaxf(hi, w[k]);
            }
          for (int k = base + kSub; k < bw && a.i1 + k < gend; ++k) {
            lo = fminf(lo, wrow[k]);
            hi = fmaxf(hi, wrow[k]);
          }
          if (valid && a.ext_minmax != nullptr && a.i1 + bw < gend) {
            const float2 mm = a.ext_minmax[r];
            lo = fminf(lo, mm.x);
            hi = fmaxf(hi, mm.y);
          }
          gp = grid_params(lo, hi, a.maxq);
          if (valid) {
            const int g = col / a.G;
            a.scales[r * a.n_groups + g] = gp.scale;
            a.zeros[r * a.n_groups + g] = static_cast<uint8_t>(gp.zero);
          }
        }
        const float wj = w[jj];
        const float q = grid_code(wj, gp, a.maxq);
        const float err = __fmul_rn(__fsub_rn(wj, grid_deq(q, gp)), rdiag[j]);
        e[jj] = err;
        loss = fmaf(err, err, loss);
        cw[jj / 4] |= static_cast<uint32_t>(q) << (8 * (jj % 4));
        // the later columns of this sub-block (U is zero outside the block)
        const float4* urow = reinterpret_cast<const float4*>(us + j * kBMax + base);
#pragma unroll
        for (int k4 = jj / 4; k4 < kSub / 4; ++k4) {
          const float4 u = urow[k4];
          if (4 * k4 + 0 > jj) w[4 * k4 + 0] = fmaf(-err, u.x, w[4 * k4 + 0]);
          if (4 * k4 + 1 > jj) w[4 * k4 + 1] = fmaf(-err, u.y, w[4 * k4 + 1]);
          if (4 * k4 + 2 > jj) w[4 * k4 + 2] = fmaf(-err, u.z, w[4 * k4 + 2]);
          if (4 * k4 + 3 > jj) w[4 * k4 + 3] = fmaf(-err, u.w, w[4 * k4 + 3]);
        }
      }
    }
    // the sub-block's errors update the later sub-blocks of the block, four
    // columns at a time so the FMA chains interleave
    for (int k = base + kSub; k < bw; k += 4) {
      float acc[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] = wrow[k + c];
#pragma unroll
      for (int j4 = 0; j4 < kSub / 4; ++j4) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float4 u = reinterpret_cast<const float4*>(ut + (k + c) * kBMax + base)[j4];
          acc[c] = fmaf(-e[4 * j4 + 0], u.x, acc[c]);
          acc[c] = fmaf(-e[4 * j4 + 1], u.y, acc[c]);
          acc[c] = fmaf(-e[4 * j4 + 2], u.z, acc[c]);
          acc[c] = fmaf(-e[4 * j4 + 3], u.w, acc[c]);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) wrow[k + c] = acc[c];
    }
    if (valid) {
      float* ehi = a.E_hi + r * kBMax + base;
      float* elo = a.E_lo + r * kBMax + base;
#pragma unroll
      for (int k4 = 0; k4 < kSub / 4; ++k4) {
        float4 h, l;
        h.x = __uint_as_float(__float_as_uint(e[4 * k4 + 0]) & 0xffffe000u);
        h.y = __uint_as_float(__float_as_uint(e[4 * k4 + 1]) & 0xffffe000u);
        h.z = __uint_as_float(__float_as_uint(e[4 * k4 + 2]) & 0xffffe000u);
        h.w = __uint_as_float(__float_as_uint(e[4 * k4 + 3]) & 0xffffe000u);
        l.x = e[4 * k4 + 0] - h.x;
        l.y = e[4 * k4 + 1] - h.y;
        l.z = e[4 * k4 + 2] - h.z;
        l.w = e[4 * k4 + 3] - h.w;
        reinterpret_cast<float4*>(ehi)[k4] = h;
        reinterpret_cast<float4*>(elo)[k4] = l;
      }
      uint8_t* crow = a.codes + r * a.n + a.i1 + base;
      const int nvalid = min(kSub, bw - base);
      if (nvalid == kSub && (reinterpret_cast<uintptr_t>(crow) % 16) == 0) {
        reinterpret_cast<uint4*>(crow)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        reinterpret_cast<uint4*>(crow)[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
      } else {
#pragma unroll
        for (int k = 0; k < kSub; ++k)
          if (k < nvalid) crow[k] = static_cast<uint8_t>(cw[k / 4] >> (8 * (k % 4)));
      }
    }
  }
  if (valid && a.row_loss != nullptr) a.row_loss[r] += loss;
}

// Per row, (min, max) of Wk[r, c0 : c1): the part of a group that lies past
// the block it starts in.  One warp per row.
__global__ void group_minmax_kernel(const float* __restrict__ Wk, int64_t rows, int n, int c0, int c1,
                                    float2* __restrict__ out) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (r >= rows) return;
  float lo = INFINITY, hi = -INFINITY;
  for (int c = c0 + lane; c < c1; c += 32) {
    const float v = Wk[r * n + c];
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
  lo = warp_min(lo);
  hi = warp_max(hi);
  if (lane == 0) out[r] = make_float2(lo, hi);
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
  size_t wk, e_hi, e_lo, codes_p, u_hi, u_lo, minmax, total;
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
  l.minmax = off;
  off += align256(static_cast<size_t>(rows) * sizeof(float2));
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
  float2* ext_minmax = reinterpret_cast<float2*>(w + l.minmax);
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GPTQ_ERR_CUDA;
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
  a.block = block;
  a.wait_ns = wait_limit_ns();
  a.status = info->status;
  // the U tile of each block arrives as one TMA box when U's rows are
  // 16-byte aligned
  CUtensorMap u_map;
  std::memset(&u_map, 0, sizeof(u_map));
  a.u_tma = (n % 4 == 0) ? 1 : 0;
  if (a.u_tma && !make_tensor_map_2d(&u_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, U, static_cast<uint64_t>(n),
                                     static_cast<uint64_t>(n), static_cast<uint64_t>(n) * 4, block, block,
                                     CU_TENSOR_MAP_SWIZZLE_NONE))
    return GPTQ_ERR_CUDA;
  CUtensorMap uth_map, utl_map;
  if (!make_tensor_map_2d(&uth_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, U_hi, static_cast<uint64_t>(n),
                          static_cast<uint64_t>(n), static_cast<uint64_t>(l.ldu) * 4, block, block,
                          CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tensor_map_2d(&utl_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, U_lo, static_cast<uint64_t>(n),
                          static_cast<uint64_t>(n), static_cast<uint64_t>(l.ldu) * 4, block, block,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
    return GPTQ_ERR_CUDA;
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
    // a group that starts here and runs past the block: min / max of its
    // columns beyond the block, taken before the block changes anything
    const int gend = std::min(i1 + G, n);
    a.ext_minmax = nullptr;
    if (i1 % G == 0 && i1 + a.bw < gend) {
      launch(group_minmax_kernel, static_cast<unsigned>(ceil_div(rows * 32, 256)), 256, 0, st, Wk, rows, n,
             i1 + a.bw, gend, ext_minmax);
      a.ext_minmax = ext_minmax;
    }
    launch(gptq_block_kernel, block_ctas, kRowsPerCta, kBlockSmem, st, u_map, uth_map, utl_map, a);
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
