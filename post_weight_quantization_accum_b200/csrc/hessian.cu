// Hessian accumulation H += alpha * X^T X on the sm_100a tensor cores.
//
// GPTQ knowledge note, "How It Works": each linear layer's reconstruction loss
// has Hessian H = 2 X X^T built from recorded layer inputs.  X arrives
// token-major (X[t, i], bf16), so the product is X^T X: a symmetric rank-N
// update (SYRK) whose inner dimension is the token count.
//
// Kernel design (persistent CTA pairs, one CTA per SM):
//   * Output tiles of 256 x 256 cover the lower triangle in 256-row blocks.
//     A cluster of two CTAs (one TPC) computes a tile with tcgen05 pair MMAs
//     (cta_group::2, M = 256, N = 256, K = 16): each CTA loads half of the
//     rows' features (A, 128) and half of the columns' features (B, 128) and
//     holds its 128 rows of the fp32 accumulator in its own tensor memory.
//     Per CTA and stage that is 32 KB of operands for 2 * 128 * 256 * 64
//     flops, a third less shared-memory and L2 traffic per flop than a
//     single-CTA 128 x 256 tile.
//   * Both operands are slices of the same X tile stream and are MN-major
//     (features contiguous): TMA loads 64-feature x 64-token boxes with the
//     128-byte swizzle into a 6-stage ring; both CTAs' loads are counted on
//     the even CTA's barrier, whose single thread issues the MMAs; MMA
//     completion is signalled to both CTAs (commit multicast), which frees
//     their stages and hands the accumulators to their epilogue warps.
//   * The accumulator is double-buffered (2 x 256 columns), so the epilogue
//     of one work unit overlaps the next.
//   * The token range is cut into `splits` equal chunks; work unit u covers
//     tile (u % tiles) over chunk (u / tiles) and pairs take units
//     round-robin, so all pairs sweep the tokens in the same order and the
//     X slice they share stays in L2.  Each unit writes its fp32 partial tile
//     to the workspace; a finalize kernel sums the partials in a fixed order,
//     scales by alpha and adds into both triangles of H, so the result is
//     deterministic and exactly symmetric.
//   * Every barrier wait is bounded in time; a wait that runs out records
//     GPTQ_ERR_TIMEOUT and stops the CTA's loops; the CTA then waits (bounded)
//     for the copies and MMAs it is responsible for, meets its peer at a
//     cluster barrier and releases tensor memory before returning.
//
// The fp64 diagonal (act-order key) is accumulated by a separate pair of
// kernels with a fixed summation order.
#include <algorithm>
#include <cstring>
#include <vector>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int kTile = 256;                        // output tile rows = columns (one CTA pair)
constexpr int kHalf = 128;                        // features per CTA for each operand
constexpr int kBK = 64;                           // tokens per pipeline stage
constexpr int kStages = 6;
constexpr int kBoxBytes = 64 * kBK * 2;           // one 64-feature x 64-token bf16 box
constexpr int kHalfBytes = kHalf * kBK * 2;       // 16 KB: one operand half
constexpr int kStageBytes = 2 * kHalfBytes;       // A half + B half = 32 KB per CTA
constexpr int kThreads = 192;                     // producer, MMA, 4 epilogue warps
constexpr uint32_t kTmemCols = 512;               // 2 x 256-column accumulators
constexpr int kBarrierBytes = 256;
constexpr size_t kSmemBytes = 1024 + size_t(kStages) * kStageBytes + kBarrierBytes;
constexpr uint64_t kDrainNs = 2000000000ull;      // bound for draining in-flight work

struct SyrkParams {
  int n;
  int kblocks;   // ceil(n_tok / kBK)
  int splits;    // token chunks
  int tiles;     // lower-triangle tiles
  float* partial;
  int* status;
  uint64_t wait_ns;
};

// Tile t -> (row block, column block) with t = rb (rb + 1) / 2 + cb, cb <= rb.
__host__ __device__ inline void tile_coords(int t, int& rb, int& cb) {
  int r = static_cast<int>((sqrtf(8.0f * static_cast<float>(t) + 1.0f) - 1.0f) * 0.5f);
  while ((r + 1) * (r + 2) / 2 <= t) ++r;
  while (r > 0 && r * (r + 1) / 2 > t) --r;
  rb = r;
  cb = t - r * (r + 1) / 2;
}

inline int tiles_for(int n) {
  const int rbs = static_cast<int>(ceil_div(n, kTile));
  return rbs * (rbs + 1) / 2;
}

__device__ __forceinline__ void unit_range(const SyrkParams& p, int u, int& t, int& kb0, int& kb1) {
  const int s = u / p.tiles;
  t = u - s * p.tiles;
  kb0 = static_cast<int>((static_cast<int64_t>(s) * p.kblocks) / p.splits);
  kb1 = static_cast<int>((static_cast<int64_t>(s + 1) * p.kblocks) / p.splits);
}

__global__ void __launch_bounds__(kThreads, 1)
    syrk_tc_kernel(const __grid_constant__ CUtensorMap xmap, SyrkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(kStages) * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs; 1: its peer
  const int pair = static_cast<int>(blockIdx.x) / 2;
  const int pairs = static_cast<int>(gridDim.x) / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);   // the even CTA's expect-tx arrival (+ both CTAs' bytes)
      mbar_init(empty + s, 1);  // one MMA commit per stage use
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);   // one MMA commit per work unit
      mbar_init(acc_empty + b, 8);  // four epilogue warps of each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&xmap);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_units = p.splits * p.tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;  // per-stage bits for the drain
      for (int u = pair; u < num_units && !*abort_flag; u += pairs) {
        int t, kb0, kb1, rb, cb;
        unit_range(p, u, t, kb0, kb1);
        tile_coords(t, rb, cb);
        const int fa = rb * kTile + static_cast<int>(rank) * kHalf;  // this CTA's A features
        const int fb = cb * kTile + static_cast<int>(rank) * kHalf;  // this CTA's B features
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, p.wait_ns)) {
            set_status(p.status, GPTQ_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
          if (*abort_flag) break;
          uint8_t* a = ring + size_t(stage) * kStageBytes;
          uint8_t* b = a + kHalfBytes;
          const int y = kb * kBK;
          const uint32_t bar = smem_cluster_addr(full + stage, 0);
          if (rank == 0) mbar_arrive_expect_tx(full + stage, 2u * kStageBytes);
          tma_load_2d_pair(a, &xmap, bar, fa, y);
          tma_load_2d_pair(a + kBoxBytes, &xmap, bar, fa + 64, y);
          tma_load_2d_pair(b, &xmap, bar, fb, y);
          tma_load_2d_pair(b + kBoxBytes, &xmap, bar, fb + 64, y);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain (even CTA): every stage it armed has received both CTAs' bytes.
      if (rank == 0) {
        for (int s = 0; s < kStages; ++s) {
          if (issued & (1u << s)) {
            if (!mbar_wait(full + s, (issued_parity >> s) & 1u, kDrainNs)) set_status(p.status, GPTQ_ERR_TIMEOUT);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (even CTA) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      const uint32_t idesc = instr_desc(1u, 1u, 1u, kTile, kTile);
      for (int u = pair; u < num_units && ok; u += pairs, ++local) {
        int t, kb0, kb1;
        unit_range(p, u, t, kb0, kb1);
        const int buf = local & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(local >> 1) & 1u;
        if (!mbar_wait(acc_empty + buf, acc_phase ^ 1u, p.wait_ns) || *abort_flag) {
          set_status(p.status, GPTQ_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kTile);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full + stage, phase, p.wait_ns) || *abort_flag) {
            set_status(p.status, GPTQ_ERR_TIMEOUT);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(ring + size_t(stage) * kStageBytes);
          const uint32_t b_addr = a_addr + kHalfBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(a_addr + kk * 2048, kBoxBytes, 1024);
            const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, kBoxBytes, 1024);
            mma_f16_pair(d_tmem, adesc, bdesc, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair(empty + stage, 0x3);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(acc_full + buf, 0x3);
      }
      // Drain: all pair MMAs issued have completed (they read both CTAs' stages).
      mma_commit_pair(drain, 0x1);
      if (!mbar_wait(drain, 0u, kDrainNs)) set_status(p.status, GPTQ_ERR_TIMEOUT);
    }
  } else {
    // ---------------- epilogue (both CTAs): TMEM -> registers -> workspace ----------------
    const int quad = warp & 3;  // tensor-memory lanes this warp may access
    const int row = static_cast<int>(rank) * kHalf + quad * 32 + lane;
    int local = 0;
    for (int u = pair; u < num_units; u += pairs, ++local) {
      const int buf = local & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(local >> 1) & 1u;
      // lane 0 waits and the warp follows its verdict, so the warp stays
      // converged for the .sync.aligned tensor-memory loads below
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(acc_full + buf, acc_phase, p.wait_ns) && !*abort_flag;
        if (!ok) {
          set_status(p.status, GPTQ_ERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      float* dst = p.partial + (static_cast<size_t>(u) * kTile + row) * kTile;
      for (int c = 0; c < kTile; c += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * kTile + c), r);
        tmem_ld_wait();
        float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          d4[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                              __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(smem_cluster_addr(acc_empty + buf, 0));
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the pair still uses its memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Sums the partial tiles of every token chunk in chunk order, scales by alpha
// and adds the lower triangle into H and its mirror image into the upper one.
// Grid (tiles, 8, 8) x block (32, 8): one 32x32 sub-block per CTA.
__global__ void syrk_finalize_kernel(const float* __restrict__ partial, float* __restrict__ H, int n, int tiles,
                                     int splits, float alpha) {
  int rb, cb;
  tile_coords(blockIdx.x, rb, cb);
  const int sc = blockIdx.y * 32;
  const int sr = blockIdx.z * 32;
  const int r0 = rb * kTile + sr;
  const int cc0 = cb * kTile + sc;
  if (r0 >= n || cc0 >= n || cc0 > r0 + 31) return;
  __shared__ float tr[32][33];
  const int tx = threadIdx.x;
  for (int i = threadIdx.y; i < 32; i += 8) {
    float v = 0.0f;
    for (int s = 0; s < splits; ++s)
      v += partial[(static_cast<size_t>(s * tiles + blockIdx.x) * kTile + sr + i) * kTile + sc + tx];
    v *= alpha;
    tr[tx][i] = v;
    const int r = r0 + i, c = cc0 + tx;
    if (r < n && c < n && c <= r) H[static_cast<size_t>(r) * n + c] += v;
  }
  __syncthreads();
  for (int j = threadIdx.y; j < 32; j += 8) {
    const int c = cc0 + j, r = r0 + tx;
    if (r < n && c < n && c < r) H[static_cast<size_t>(c) * n + r] += tr[j][tx];
  }
}

constexpr int kDiagTokens = 1024;  // tokens per CTA of the fp64 diagonal pass

// Per token chunk and feature pair: sum of squares in fp64, tokens in order.
__global__ void hdiag_partial_kernel(const __nv_bfloat16* __restrict__ X, int64_t n_tok, int n, int64_t ldx,
                                     double* __restrict__ part) {
  const int f = (blockIdx.x * blockDim.x + threadIdx.x) * 2;
  if (f >= n) return;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kDiagTokens;
  const int64_t t1 = min(n_tok, t0 + kDiagTokens);
  double s0 = 0.0, s1 = 0.0;
  for (int64_t t = t0; t < t1; ++t) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(X + t * ldx + f);
    const float a = __bfloat162float(v.x), b = __bfloat162float(v.y);
    s0 += static_cast<double>(a * a);  // exact: a bf16 square fits in fp32
    s1 += static_cast<double>(b * b);
  }
  part[static_cast<size_t>(blockIdx.y) * n + f] = s0;
  if (f + 1 < n) part[static_cast<size_t>(blockIdx.y) * n + f + 1] = s1;
}

__global__ void hdiag_reduce_kernel(const double* __restrict__ part, int chunks, int n, double alpha,
                                    double* __restrict__ hdiag) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= n) return;
  double s = 0.0;
  for (int c = 0; c < chunks; ++c) s += part[static_cast<size_t>(c) * n + f];
  hdiag[f] += alpha * s;
}

// Token chunks for the split-K schedule: the smallest count (<= 16) whose
// round-robin assignment of units to CTA pairs keeps the busiest pair within
// 5% of the average, else the best balance found.  Tiles are equal in cost.
int choose_splits(int n, int64_t n_tok, int pairs) {
  const int tiles = tiles_for(n);
  const int64_t kblocks = ceil_div(n_tok, kBK);
  double best_eff = -1.0;
  int best = 1;
  for (int s = 1; s <= 16 && s <= kblocks; ++s) {
    const int units = s * tiles;
    const int busiest = static_cast<int>(ceil_div(units, pairs));
    const double eff = static_cast<double>(units) / (static_cast<double>(pairs) * busiest);
    if (eff >= 0.95) return s;
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

int pairs_for(const DeviceInfo* info) { return std::max(1, info->sm_count / 2); }

size_t partial_bytes(int n, int splits) {
  return static_cast<size_t>(splits) * tiles_for(n) * kTile * kTile * sizeof(float);
}

size_t diag_bytes(int n, int64_t n_tok) {
  return static_cast<size_t>(ceil_div(n_tok, kDiagTokens)) * n * sizeof(double);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t hessian_workspace_size(int n, int64_t n_tok) {
  const DeviceInfo* info = device_info();
  if (info == nullptr || n <= 0 || n_tok <= 0) return 0;
  const int splits = choose_splits(n, n_tok, pairs_for(info));
  return align256(partial_bytes(n, splits)) + align256(diag_bytes(n, n_tok));
}

gptq_status hessian_accum(float* H, double* hdiag, const void* X, int64_t n_tok, int n, int64_t ldx, float alpha,
                          void* ws, size_t ws_bytes, cudaStream_t stream) {
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GPTQ_ERR_CUDA;
  if (n_tok == 0) return GPTQ_OK;
  const int splits = choose_splits(n, n_tok, pairs_for(info));
  const size_t pbytes = align256(partial_bytes(n, splits));
  if (ws_bytes < pbytes + align256(diag_bytes(n, n_tok))) return GPTQ_ERR_INVALID_ARG;
  float* partial = static_cast<float*>(ws);
  double* dpart = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + pbytes);

  CUtensorMap xmap;
  if (!make_tensor_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(n),
                          static_cast<uint64_t>(n_tok), static_cast<uint64_t>(ldx) * 2, 64, kBK,
                          CU_TENSOR_MAP_SWIZZLE_128B))
    return GPTQ_ERR_CUDA;

  static bool attr_set[64] = {};
  if (!attr_set[info->device]) {
    if (cudaFuncSetAttribute(syrk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    attr_set[info->device] = true;
  }

  SyrkParams p;
  p.n = n;
  p.kblocks = static_cast<int>(ceil_div(n_tok, kBK));
  p.splits = splits;
  p.tiles = tiles_for(n);
  p.partial = partial;
  p.status = info->status;
  p.wait_ns = wait_limit_ns();
  const int units = p.splits * p.tiles;
  const int pairs = std::min(pairs_for(info), units);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const bool traced = trace_on();
  if (traced) trace_begin(stream);
  if (cudaLaunchKernelEx(&cfg, syrk_tc_kernel, xmap, p) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (traced) trace_end(stream, reinterpret_cast<const void*>(syrk_tc_kernel));
  count_launch();
  launch(syrk_finalize_kernel, dim3(p.tiles, kTile / 32, kTile / 32), dim3(32, 8), 0, stream, partial, H, n, p.tiles,
                                                                                        p.splits, alpha);
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;

  if (hdiag != nullptr) {
    const int chunks = static_cast<int>(ceil_div(n_tok, kDiagTokens));
    const int threads = 128;
    dim3 g(static_cast<unsigned>(ceil_div(ceil_div(n, 2), threads)), static_cast<unsigned>(chunks));
    launch(hdiag_partial_kernel, g, threads, 0, stream, static_cast<const __nv_bfloat16*>(X), n_tok, n, ldx, dpart);
    if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
    launch(hdiag_reduce_kernel, static_cast<unsigned>(ceil_div(n, 256)), 256, 0, stream, 
        dpart, chunks, n, static_cast<double>(alpha), hdiag);
    if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

}  // namespace gptq
