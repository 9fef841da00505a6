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
//   gptq_block_kernel   sixteen lanes per weight row (two rows per warp),
//                       lane l owning the block's columns l, l + 16, ...,
//                       l + 112 in registers, the block's U tile in shared
//                       memory (each lane's eight entries of a U row side by
//                       side, two vector loads per step).  Step j broadcasts
//                       w_j from its owner lane (shuffle), every lane rounds
//                       it on the grid and forms e_j = (w_j - deq_j) / U_jj,
//                       then updates its own columns w_k -= e_j U_jk (U is
//                       zero left of the diagonal, so no lane needs a test).
//                       Group (scale, zero) are a shuffle min / max reduction
//                       over the group's current values when the group
//                       starts.  No block-wide synchronisation inside the
//                       loop; one row's chain of dependent steps overlaps the
//                       other warps'.
//   trailing_update_tc (trailing.cu)   W[:, i2:] -= E[:, i1:i2] * U[i1:i2, i2:]
//                       on the tensor cores, fp32-accurate through a 3-term
//                       tf32 split; the block kernel writes E as its tf32
//                       hi / lo halves.
// gptq_superblock_kernel (selected by gptq_set_column_loop(1)) is the fused
// single pass: one launch per super-block in which each CTA takes a slab of
// rows through all of the super-block's blocks (described at the kernel).
#include <algorithm>
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "grid.cuh"

namespace gptq {
namespace {

constexpr int kBMax = 128;        // largest block width
constexpr int kMaxWarpsPerCta = 32;
constexpr int kBlockLanes = 16;  // lanes per weight row in the block kernel

template <typename T>
__device__ __forceinline__ float load_w(const T* p);
template <>
__device__ __forceinline__ float load_w<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_w<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Wk[r, p] = dead[perm[p]] ? 0 : W[r, perm[p]]  (processing order, fp32).
// One thread per column p over a chunk of kGatherRows rows: the column's
// source index and dead flag are read once, and the rows' loads are
// independent of one another, so many are in flight at once.
constexpr int kGatherRows = 16;

template <typename T>
__global__ void gather_weights_kernel(const T* __restrict__ W, const int32_t* __restrict__ perm,
                                      const uint8_t* __restrict__ dead, int64_t rows, int n, float* __restrict__ Wk) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n) return;
  const int c = perm != nullptr ? perm[p] : p;
  const bool d = dead != nullptr && dead[c];
  for (int64_t r0 = static_cast<int64_t>(blockIdx.y) * kGatherRows; r0 < rows;
       r0 += static_cast<int64_t>(gridDim.y) * kGatherRows) {
    const int64_t r1 = r0 + kGatherRows < rows ? r0 + kGatherRows : rows;
#pragma unroll 8
    for (int64_t r = r0; r < r1; ++r) Wk[r * n + p] = d ? 0.0f : load_w<T>(W + r * n + c);
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
  float* E_hi;           // [rows, lde] scaled errors, tf32 high part (this block at column e_off)
  float* E_lo;           // [rows, lde] and the remainder e - hi
  int lde, e_off;
  uint8_t* codes;        // [rows, n] processing order
  float* scales;         // [rows, n_groups]
  uint8_t* zeros;        // [rows, n_groups]
  float* row_loss;       // [rows] or nullptr
  const float2* ext_minmax;  // [rows] (min, max) of a group's columns beyond this block, or nullptr
};

// Lanes per weight row and the shared-memory layout of the U tile: lane li of
// a row owns the block columns li + kLanes m (m < kBMax / kLanes), and row j
// of the tile keeps each lane's entries side by side at a stride of
// kLanes * pitch with a lane pitch whose multiples fall in distinct 16-byte
// bank groups (so the vector loads of eight consecutive lanes do not conflict).
template <int kLanes>
struct BlockShape {
  static constexpr int kCols = kBMax / kLanes;                // columns per lane
  static constexpr int kPitch = kCols == 4 ? 4 : kCols + 4;   // floats per lane slot
  static constexpr int kRowPitch = kLanes * kPitch;           // floats per tile row
  static constexpr size_t kSmem = (static_cast<size_t>(kBMax) * kRowPitch + kBMax) * sizeof(float);
};

// The U tile rows [j0, j0 + nr) x columns [c0, c0 + nc) into the lane-major
// layout by asynchronous 4-byte copies, all in flight at once (coalesced
// along U's rows; zeros outside the tile's extent).  The caller waits.
template <int kLanes>
__device__ __forceinline__ void stage_u_tile(float* us, const float* __restrict__ U, int n, int j0, int c0, int nr,
                                             int nc) {
  using Shape = BlockShape<kLanes>;
  for (int e = threadIdx.x; e < kBMax * kBMax; e += blockDim.x) {
    const int j = e / kBMax, c = e % kBMax;
    const bool in = j < nr && c < nc;
    const float* src = in ? U + static_cast<int64_t>(j0 + j) * n + c0 + c : U;
    cp_async_4(us + j * Shape::kRowPitch + (c % kLanes) * Shape::kPitch + c / kLanes, src, in ? 4u : 0u);
  }
}

// One row's quantize-and-propagate chain over the block [a.i1, a.i1 + a.bw):
// w holds the lane's columns li + kLanes m of the block (fully updated by
// every earlier column), us the block's diagonal U tile and rdiag 1 / U_jj.
// Writes the row's codes, group parameters, scaled errors (tf32 hi / lo) and
// loss; lanes of rows past the matrix (valid false) compute on row rr and
// write nothing.
template <int kLanes>
__device__ __forceinline__ void block_chain(const BlockArgs& a, const float* us, const float* rdiag, int64_t r,
                                            bool valid, int64_t rr, int li, float (&w)[BlockShape<kLanes>::kCols]) {
  using Shape = BlockShape<kLanes>;
  constexpr int C = Shape::kCols;
  const int bw = a.bw;
  // A group that began in an earlier block keeps the (scale, zero) that
  // block fixed; they are read back from the outputs.
  GridParams gp{1.0f, 0.0f};
  if (a.i1 % a.G != 0) {
    const int g = a.i1 / a.G;
    gp.scale = a.scales[rr * a.n_groups + g];
    gp.zero = static_cast<float>(a.zeros[rr * a.n_groups + g]);
  }
  float rcp = __frcp_rn(gp.scale);
  float loss = 0.0f;
  float e_own[C], q_own[C];  // this lane's columns' errors and codes
#pragma unroll
  for (int m = 0; m < C; ++m) e_own[m] = q_own[m] = 0.0f;
  int jg = (a.G - a.i1 % a.G) % a.G;  // block position of the next group start
  const float* ulane = us + li * Shape::kPitch;

#pragma unroll
  for (int mj = 0; mj < C; ++mj) {
    const int jend = min(kLanes, bw - kLanes * mj);
#pragma unroll 1
    for (int jj = 0; jj < jend; ++jj) {
      const int j = kLanes * mj + jj;
      if (j == jg) {
        // group start: (scale, zero) from the group's current values
        jg += a.G;
        const int gend = min(a.i1 + j + a.G, a.n);
        float lo = INFINITY, hi = -INFINITY;
#pragma unroll
        for (int m = 0; m < C; ++m) {
          const int c = li + kLanes * m;
          if (c >= j && c < bw && a.i1 + c < gend) {
            lo = fminf(lo, w[m]);
            hi = fmaxf(hi, w[m]);
          }
        }
#pragma unroll
        for (int o = kLanes / 2; o > 0; o >>= 1) {
          lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
          hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        if (a.ext_minmax != nullptr && a.i1 + bw < gend) {
          const float2 mm = a.ext_minmax[rr];
          lo = fminf(lo, mm.x);
          hi = fmaxf(hi, mm.y);
        }
        gp = grid_params(lo, hi, a.maxq);
        rcp = __frcp_rn(gp.scale);
        if (li == 0 && valid) {
          const int g = (a.i1 + j) / a.G;
          a.scales[r * a.n_groups + g] = gp.scale;
          a.zeros[r * a.n_groups + g] = static_cast<uint8_t>(gp.zero);
        }
      }
      const float wj = __shfl_sync(0xffffffffu, w[mj], jj, kLanes);
      const float q = grid_code_rcp(wj, gp, rcp, a.maxq);
      const float err = __fmul_rn(__fsub_rn(wj, grid_deq(q, gp)), rdiag[j]);
      loss = fmaf(err, err, loss);
      if (li == jj) {
        e_own[mj] = err;
        q_own[mj] = q;
      }
      // w_k -= e_j U_jk for this lane's columns (U_jk = 0 for k < j; the
      // column j itself is not read again)
      const float4* urow = reinterpret_cast<const float4*>(ulane + j * Shape::kRowPitch);
#pragma unroll
      for (int g4 = 0; g4 < C / 4; ++g4) {
        const float4 u = urow[g4];
        w[4 * g4 + 0] = fmaf(-err, u.x, w[4 * g4 + 0]);
        w[4 * g4 + 1] = fmaf(-err, u.y, w[4 * g4 + 1]);
        w[4 * g4 + 2] = fmaf(-err, u.z, w[4 * g4 + 2]);
        w[4 * g4 + 3] = fmaf(-err, u.w, w[4 * g4 + 3]);
      }
    }
  }
  if (!valid) return;
  float* ehi = a.E_hi + r * a.lde + a.e_off;
  float* elo = a.E_lo + r * a.lde + a.e_off;
  uint8_t* crow = a.codes + r * a.n + a.i1;
#pragma unroll
  for (int m = 0; m < C; ++m) {
    const int c = li + kLanes * m;
    if (c < bw) {
      const float h = __uint_as_float(__float_as_uint(e_own[m]) & 0xffffe000u);
      ehi[c] = h;
      elo[c] = e_own[m] - h;
      crow[c] = static_cast<uint8_t>(q_own[m]);
    }
  }
  if (li == 0 && a.row_loss != nullptr) a.row_loss[r] += loss;
}

template <int kLanes>
__global__ void __launch_bounds__(kMaxWarpsPerCta * 32, 1) gptq_block_kernel(BlockArgs a) {
  using Shape = BlockShape<kLanes>;
  constexpr int C = Shape::kCols;
  extern __shared__ __align__(16) float dyn_smem[];
  float* us = dyn_smem;                             // [kBMax][kRowPitch] the U tile, lane-major
  float* rdiag = us + kBMax * Shape::kRowPitch;     // [kBMax] 1 / U_jj
  const int bw = a.bw;
  const int lane = threadIdx.x & 31;
  const int li = lane % kLanes;  // lane within its row group
  const int warps = blockDim.x >> 5;
  // the next kernel of the stream (a trailing update) may start its prologue
  pdl_trigger();
  stage_u_tile<kLanes>(us, a.U, a.n, a.i1, a.i1, bw, bw);
  cp_async_wait_all();
  __syncthreads();
  for (int j = threadIdx.x; j < kBMax; j += blockDim.x)
    rdiag[j] = j < bw ? 1.0f / us[j * Shape::kRowPitch + (j % kLanes) * Shape::kPitch + j / kLanes] : 0.0f;
  __syncthreads();
  // U is fixed for the whole loop; everything below reads or writes what the
  // previous kernels of the stream produce or consume (W, E, codes, groups)
  pdl_wait();

  const int64_t warp_row0 = (static_cast<int64_t>(blockIdx.x) * warps + (threadIdx.x >> 5)) * (32 / kLanes);
  if (warp_row0 >= a.rows) return;  // whole warps leave; no block-wide barrier follows
  const int64_t r = warp_row0 + lane / kLanes;
  const bool valid = r < a.rows;    // a warp's last rows may lie past the matrix
  const int64_t rr = valid ? r : a.rows - 1;  // such lanes compute on a real row and write nothing
  const float* wsrc = a.Wk + rr * a.n + a.i1;
  float w[C];
#pragma unroll
  for (int m = 0; m < C; ++m) {
    const int c = li + kLanes * m;
    w[m] = c < bw ? wsrc[c] : 0.0f;
  }
  block_chain<kLanes>(a, us, rdiag, r, valid, rr, li, w);
}

// One launch per super-block [s1, s2) (fused single pass over a row slab):
// a CTA takes rows_cta = blockDim.x / kLanes rows through every block of the
// super-block.  Block i1 starts from the rows' working weights as the
// previous super-blocks left them and first applies, left-looking, the
// corrections of the super-block's earlier blocks t: w_c -= sum_k E_t[r, k]
// U[t + k, c] over this lane's columns c, fp32 on the CUDA cores, with the
// U tiles (128 x 128) double-buffered in shared memory and the CTA's own
// error rows read back from L2; then the block's chain runs as in
// gptq_block_kernel.  The same sums as the per-block trailing updates in
// another order (every column still receives every earlier column's
// correction before it is quantized).  Requires that no group starting in a
// later block of the super-block reaches past its block (block % G == 0, or
// one group per row): a group's parameters need its columns' current values,
// which the left-looking form has only for the block at hand.  ext_minmax
// belongs to the first block.
constexpr int kSlabMaxRows = 32;  // rows per CTA of the fused kernel (one CTA per SM)

template <int kLanes>
__global__ void __launch_bounds__(kSlabMaxRows * kLanes, 1) gptq_superblock_kernel(BlockArgs a, int s1, int s2,
                                                                                   int block) {
  using Shape = BlockShape<kLanes>;
  constexpr int C = Shape::kCols;
  constexpr int kTile = kBMax * Shape::kRowPitch;
  extern __shared__ __align__(16) float dyn_smem[];
  float* ubuf0 = dyn_smem;             // U tiles, lane-major, two buffers
  float* ubuf1 = dyn_smem + kTile;
  float* rdiag = ubuf1 + kTile;        // [kBMax] 1 / U_jj of the block at hand
  const int lane = threadIdx.x & 31;
  const int li = lane % kLanes;
  const int rows_cta = blockDim.x / kLanes;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * rows_cta + threadIdx.x / kLanes;
  const bool valid = r < a.rows;
  const int64_t rr = valid ? r : a.rows - 1;  // such lanes compute on a real row and write nothing
  for (int i1 = s1; i1 < s2; i1 += block) {
    BlockArgs b = a;
    b.i1 = i1;
    b.bw = min(block, s2 - i1);
    b.e_off = i1 - s1;
    if (i1 != s1) b.ext_minmax = nullptr;
    const int bw = b.bw;
    float w[C];
    const float* wsrc = a.Wk + rr * a.n + i1;
#pragma unroll
    for (int m = 0; m < C; ++m) {
      const int c = li + kLanes * m;
      w[m] = c < bw ? wsrc[c] : 0.0f;
    }
    const int nt = (i1 - s1) / block;  // earlier blocks of the super-block, all `block` wide
    if (nt > 0) {
      // E of block t for this row (written earlier in this launch: plain L2
      // loads, not the read-only path), e = hi + lo exactly: lane li keeps
      // k = 8 li .. 8 li + 7 and hands them to its row's lanes by shuffle;
      // the next tile's values are requested before this tile is used
      auto load_e = [&](int t, float (&e)[8]) {
        const float4* eh = reinterpret_cast<const float4*>(a.E_hi + rr * a.lde + t * block + 8 * li);
        const float4* el = reinterpret_cast<const float4*>(a.E_lo + rr * a.lde + t * block + 8 * li);
        const float4 h0 = __ldcg(eh), h1 = __ldcg(eh + 1), l0 = __ldcg(el), l1 = __ldcg(el + 1);
        e[0] = h0.x + l0.x;
        e[1] = h0.y + l0.y;
        e[2] = h0.z + l0.z;
        e[3] = h0.w + l0.w;
        e[4] = h1.x + l1.x;
        e[5] = h1.y + l1.y;
        e[6] = h1.z + l1.z;
        e[7] = h1.w + l1.w;
      };
      float e_cur[8], e_next[8];
      load_e(0, e_cur);
      stage_u_tile<kLanes>(ubuf0, a.U, a.n, s1, i1, block, bw);
      cp_async_commit();
      for (int t = 0; t < nt; ++t) {
        const float* cur = (t & 1) ? ubuf1 : ubuf0;
        if (t + 1 < nt) {
          load_e(t + 1, e_next);
          stage_u_tile<kLanes>((t & 1) ? ubuf0 : ubuf1, a.U, a.n, s1 + (t + 1) * block, i1, block, bw);
          cp_async_commit();
          cp_async_wait_group<1>();
        } else {
          cp_async_wait_group<0>();
        }
        __syncthreads();
        const float* ulane = cur + li * Shape::kPitch;
#pragma unroll 1
        for (int kb = 0; kb < kBMax / 8; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const float e = __shfl_sync(0xffffffffu, e_cur[kk], kb, kLanes);
            const float4* urow = reinterpret_cast<const float4*>(ulane + (8 * kb + kk) * Shape::kRowPitch);
#pragma unroll
            for (int g4 = 0; g4 < C / 4; ++g4) {
              const float4 u = urow[g4];
              w[4 * g4 + 0] = fmaf(-e, u.x, w[4 * g4 + 0]);
              w[4 * g4 + 1] = fmaf(-e, u.y, w[4 * g4 + 1]);
              w[4 * g4 + 2] = fmaf(-e, u.z, w[4 * g4 + 2]);
              w[4 * g4 + 3] = fmaf(-e, u.w, w[4 * g4 + 3]);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) e_cur[i] = e_next[i];
        __syncthreads();  // the buffer is refilled by a later tile
      }
    }
    stage_u_tile<kLanes>(ubuf0, a.U, a.n, i1, i1, bw, bw);
    cp_async_wait_all();
    __syncthreads();
    for (int j = threadIdx.x; j < kBMax; j += blockDim.x)
      rdiag[j] = j < bw ? 1.0f / ubuf0[j * Shape::kRowPitch + (j % kLanes) * Shape::kPitch + j / kLanes] : 0.0f;
    __syncthreads();
    block_chain<kLanes>(b, ubuf0, rdiag, r, valid, rr, li, w);
    __syncthreads();  // this block's errors are visible to the CTA; the tile buffer is free
  }
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

// codes[r, perm[p]] = codes_p[r, p] and the optional dequantized weights; rows
// along blockIdx.y, so no division per element.
__global__ void outputs_kernel(const uint8_t* __restrict__ codes_p, const int32_t* __restrict__ perm,
                               const float* __restrict__ scales, const uint8_t* __restrict__ zeros, int64_t rows,
                               int n, int G, int n_groups, uint8_t* __restrict__ codes, float* __restrict__ Wq) {
  for (int64_t r = blockIdx.y; r < rows; r += gridDim.y)
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < n; p += gridDim.x * blockDim.x) {
    const int c = perm != nullptr ? perm[p] : p;
    const uint8_t q = codes_p[r * n + p];
    if (codes != codes_p) codes[r * n + c] = q;
    if (Wq != nullptr) {
      const int g = p / G;
      GridParams gp{scales[r * n_groups + g], static_cast<float>(zeros[r * n_groups + g])};
      Wq[r * n + c] = grid_deq(static_cast<float>(q), gp);
    }
  }
}

// g_idx[perm[p]] = p / G: the group of each original column.
__global__ void g_idx_kernel(const int32_t* __restrict__ perm, int n, int G, int32_t* __restrict__ g_idx) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p < n) g_idx[perm != nullptr ? perm[p] : p] = p / G;
}

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

// Two-level lazy blocking: inside a super-block of about kSuper columns each
// block's errors update only the super-block's remaining columns; the rest of
// the matrix gets one update per super-block with K = the super-block width.
// The same sums in another order (every column still receives every earlier
// column's correction before it is quantized), so the outer updates are
// GEMMs of K ~ 1024 instead of a read-modify-write of W per 128 columns.
constexpr int kSuper = 1024;
constexpr int kSuperMinN = 2 * kSuper;  // below this, one level

struct QuantLayout {
  size_t wk, e_hi, e_lo, codes_p, u_hi, u_lo, minmax, total;
  int64_t ldu;
  int lde;  // row pitch of the error buffers: one super-block (or one block)
};

QuantLayout quant_layout(int64_t rows, int n) {
  QuantLayout l{};
  l.ldu = (n + 3) / 4 * 4;  // 16-byte row pitch for the tensor-map loads
  l.lde = n >= kSuperMinN ? kSuper : kBMax;
  size_t off = 0;
  l.wk = off;
  off += align256(static_cast<size_t>(rows) * n * sizeof(float));
  l.e_hi = off;
  off += align256(static_cast<size_t>(rows) * l.lde * sizeof(float));
  l.e_lo = off;
  off += align256(static_cast<size_t>(rows) * l.lde * sizeof(float));
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

// Super-block width: a multiple of the block that fits the error buffers, and
// one level when a group could reach past a super-block (its parameters are
// fixed at its first column from fully updated weights).
int super_width(const QuantLayout& l, int n, int block, int G) {
  if (l.lde < kSuper) return block;
  const int S = block * (kSuper / block);
  return (G == n || S % G == 0) ? S : block;
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

  const dim3 gg(static_cast<unsigned>(ceil_div(n, 256)),
                static_cast<unsigned>(std::min<int64_t>(ceil_div(rows, static_cast<int64_t>(kGatherRows)), 65535)));
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
  a.lde = l.lde;
  a.codes = codes_p;
  a.scales = scales;
  a.zeros = zeros;
  a.row_loss = row_loss;
  // kBlockLanes lanes per row; CTAs of up to 32 warps, sized so that two
  // CTAs per SM cover the rows in one wave
  constexpr int rows_per_warp = 32 / kBlockLanes;
  const size_t block_smem = BlockShape<kBlockLanes>::kSmem;
  const int64_t warps_needed = ceil_div(rows, static_cast<int64_t>(rows_per_warp));
  const int64_t want = ceil_div(warps_needed, static_cast<int64_t>(2 * info->sm_count));
  const int warps_per_cta = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(kMaxWarpsPerCta, want)));
  const unsigned block_ctas = static_cast<unsigned>(ceil_div(warps_needed, static_cast<int64_t>(warps_per_cta)));
  static std::atomic<bool> attr_set[64] = {};  // per device, shared by host threads
  if (!attr_set[info->device]) {
    if (cudaFuncSetAttribute(gptq_block_kernel<kBlockLanes>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(block_smem)) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    attr_set[info->device] = true;
  }
  const int S = super_width(l, n, block, G);
  // Fused single pass (gptq_set_column_loop(1)) where it applies: a
  // two-level loop with 128-wide blocks whose groups stay inside one block
  // (or one group per row), and rows that fit one slab of at most
  // kSlabMaxRows per SM: one launch per super-block.
  const int64_t slab = 2 * ceil_div(rows, 2 * static_cast<int64_t>(info->sm_count));
  const bool fused = column_loop_mode() == 1 && S > block && block == kBMax && (block % G == 0 || G == n) &&
                     slab <= kSlabMaxRows;
  constexpr size_t super_smem =
      (2 * static_cast<size_t>(kBMax) * BlockShape<kBlockLanes>::kRowPitch + kBMax) * sizeof(float);
  const int rows_cta = static_cast<int>(std::max<int64_t>(2, slab));
  if (fused) {
    static std::atomic<bool> super_attr[64] = {};
    if (!super_attr[info->device]) {
      if (cudaFuncSetAttribute(gptq_superblock_kernel<kBlockLanes>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(super_smem)) != cudaSuccess)
        return GPTQ_ERR_CUDA;
      super_attr[info->device] = true;
    }
  }
  for (int s1 = 0; s1 < n; s1 += S) {
    const int s2 = std::min(s1 + S, n);
    if (fused) {
      a.ext_minmax = nullptr;
      const int gend = std::min(s1 + G, n);
      if (s1 % G == 0 && s1 + block < gend) {  // one group per row: its columns past the first block
        launch(group_minmax_kernel, static_cast<unsigned>(ceil_div(rows * 32, 256)), 256, 0, st, Wk, rows, n,
               s1 + block, gend, ext_minmax);
        a.ext_minmax = ext_minmax;
      }
      launch(gptq_superblock_kernel<kBlockLanes>, static_cast<unsigned>(ceil_div(rows, static_cast<int64_t>(rows_cta))),
             rows_cta * kBlockLanes, super_smem, st, a, s1, s2, block);
    }
    for (int i1 = s1; !fused && i1 < s2; i1 += block) {
      a.i1 = i1;
      a.bw = std::min(block, s2 - i1);
      a.e_off = i1 - s1;
      // a group that starts here and runs past the block: min / max of its
      // columns beyond the block, taken before the block changes anything
      const int gend = std::min(i1 + G, n);
      a.ext_minmax = nullptr;
      if (i1 % G == 0 && i1 + a.bw < gend) {
        launch(group_minmax_kernel, static_cast<unsigned>(ceil_div(rows * 32, 256)), 256, 0, st, Wk, rows, n,
               i1 + a.bw, gend, ext_minmax);
        a.ext_minmax = ext_minmax;
      }
      if (launch_pdl(gptq_block_kernel<kBlockLanes>, dim3(block_ctas), dim3(warps_per_cta * 32), block_smem, st, a) !=
          cudaSuccess)
        return GPTQ_ERR_CUDA;
      const int i2 = i1 + a.bw;
      if (i2 < s2) {  // inner update: the rest of the super-block
        const gptq_status ts = trailing_update_tc(Wk, n, static_cast<int>(rows), s2 - i2, a.bw, i2, i1, E_hi + a.e_off,
                                                  E_lo + a.e_off, l.lde, U_hi, U_lo, l.ldu, n, st);
        if (ts != GPTQ_OK) return ts;
      }
    }
    if (s2 < n) {  // outer update: everything after the super-block
      const gptq_status ts = trailing_update_tc(Wk, n, static_cast<int>(rows), n - s2, s2 - s1, s2, s1, E_hi, E_lo,
                                                l.lde, U_hi, U_lo, l.ldu, n, st);
      if (ts != GPTQ_OK) return ts;
    }
  }
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
  if (codes_p != codes || Wq_out != nullptr || g_idx != nullptr) {
    if (codes_p != codes || Wq_out != nullptr) {
      const dim3 og(static_cast<unsigned>(std::min<int64_t>(ceil_div(n, 256), 64)),
                    static_cast<unsigned>(std::min<int64_t>(rows, 65535)));
      launch(outputs_kernel, og, 256, 0, st, codes_p, perm, scales, zeros, rows, n, G, n_groups, codes, Wq_out);
    }
    if (g_idx != nullptr)
      launch(g_idx_kernel, static_cast<unsigned>(ceil_div(n, 256)), 256, 0, st, perm, n, G, g_idx);
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
