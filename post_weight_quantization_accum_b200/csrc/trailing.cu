// The lazy trailing update of the GPTQ column loop on the tensor cores:
//
//   W[:, c0 : c0 + N] -= E[:, 0 : K] * U[k0 : k0 + K, c0 : c0 + N]
//
// (GPTQ knowledge note, "How It Works": blocks of columns accumulate their
// corrections before one global update of the remaining matrix.)
//
// The update must be as accurate as an fp32 product: the corrected weights
// decide integer codes downstream.  Each fp32 operand x is split into
// x_hi = x with its 13 low mantissa bits cleared (exact in tf32) and
// x_lo = x - x_hi (exact in fp32), and the product is formed from three
// tcgen05.mma kind::tf32 passes, E_hi U_hi + E_hi U_lo + E_lo U_hi, accumulated
// in fp32 in tensor memory; the dropped E_lo U_lo term is below 2^-20 of the
// product.
//
// Both operands are K-major (for kind::tf32 an MN-major operand read back as
// zeros in a micro-test), so U's split halves are stored transposed:
// Ut_hi[c][k] = hi(U[k][c]).
//
// Kernel: persistent CTAs over 128 x 256 output tiles (each tile's K range in
// one or more accumulation units, subtracted from W one after another); a TMA
// producer warp
// fills a 2-stage ring (per stage 32 columns of K: E_hi and E_lo as 128 x 32
// boxes, Ut_hi and Ut_lo as 256 x 32 boxes), one thread issues the MMAs into a
// double-buffered 2 x 256-column accumulator, and four epilogue warps read it
// back and apply the read-modify-write to W in fp32.
// Every barrier wait is bounded; on a timeout the CTA drains its own copies
// and MMAs and returns with GPTQ_ERR_TIMEOUT recorded.
#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 32;                                 // fp32 columns of K per stage
constexpr int kStages = 2;
constexpr int kABytes = kBM * kBK * 4;                  // 16 KB per split half
constexpr int kBBytes = kBN * kBK * 4;                  // 32 KB per split half (256 rows of 32 K)
constexpr int kStageBytes = 2 * kABytes + 2 * kBBytes;  // 96 KB
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr size_t kStagingBytes = 4 * 32 * 33 * sizeof(float);  // the epilogue warps' staging buffers
constexpr size_t kSmemBytes = 1024 + size_t(kStages) * kStageBytes + 256 + kStagingBytes;
constexpr uint64_t kDrainNs = 2000000000ull;

struct TrailParams {
  float* W;        // [M, ldw]
  int64_t ldw;
  int M, N, K;     // rows, output columns, contraction length (multiple of 32)
  int unit_chunks; // K chunks (of kBK) accumulated in tensor memory before each subtraction
  int c0, k0;      // first output column of W (and of U), first row of U
  int tiles_m, tiles_n;
  int* status;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(kThreads, 1)
    trailing_tc_kernel(const __grid_constant__ CUtensorMap map_ehi, const __grid_constant__ CUtensorMap map_elo,
                       const __grid_constant__ CUtensorMap map_uhi, const __grid_constant__ CUtensorMap map_ulo,
                       TrailParams p) {
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
  float* staging = reinterpret_cast<float*>(smem + size_t(kStages) * kStageBytes + 256);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_ehi);
    prefetch_tensormap(&map_elo);
    prefetch_tensormap(&map_uhi);
    prefetch_tensormap(&map_ulo);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // the next kernel of the stream (a block kernel) may start its prologue;
  // this one waits for the previous kernels before it reads E or touches W
  pdl_trigger();
  pdl_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = p.tiles_m * p.tiles_n;
  const int kchunks = p.K / kBK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        const int tm = t / p.tiles_n, tn = t - tm * p.tiles_n;
        const int row0 = tm * kBM, col0 = p.c0 + tn * kBN;
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!mbar_wait(empty + stage, phase ^ 1u, p.wait_ns) || *abort_flag) {
            set_status(p.status, GPTQ_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
          uint8_t* s_ahi = ring + size_t(stage) * kStageBytes;
          uint8_t* s_alo = s_ahi + kABytes;
          uint8_t* s_bhi = s_alo + kABytes;
          uint8_t* s_blo = s_bhi + kBBytes;
          mbar_arrive_expect_tx(full + stage, kStageBytes);
          tma_load_2d(s_ahi, &map_ehi, full + stage, kc * kBK, row0);
          tma_load_2d(s_alo, &map_elo, full + stage, kc * kBK, row0);
          tma_load_2d(s_bhi, &map_uhi, full + stage, p.k0 + kc * kBK, col0);
          tma_load_2d(s_blo, &map_ulo, full + stage, p.k0 + kc * kBK, col0);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      for (int s = 0; s < kStages; ++s)
        if (issued & (1u << s))
          if (!mbar_wait(full + s, (issued_parity >> s) & 1u, kDrainNs)) set_status(p.status, GPTQ_ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = instr_desc(2u, 0u, 0u, kBM, kBN);  // tf32, A and B K-major
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        // one accumulation unit per p.unit_chunks chunks of K
        for (int u0 = 0; u0 < kchunks && ok; u0 += p.unit_chunks, ++local) {
          const int u1 = min(u0 + p.unit_chunks, kchunks);
          const int buf = local & 1;
          const uint32_t acc_phase = static_cast<uint32_t>(local >> 1) & 1u;
          if (!mbar_wait(acc_empty + buf, acc_phase ^ 1u, p.wait_ns) || *abort_flag) {
            set_status(p.status, GPTQ_ERR_TIMEOUT);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
          for (int kc = u0; kc < u1; ++kc) {
            if (!mbar_wait(full + stage, phase, p.wait_ns) || *abort_flag) {
              set_status(p.status, GPTQ_ERR_TIMEOUT);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_hi = smem_u32(ring + size_t(stage) * kStageBytes);
            const uint32_t a_lo = a_hi + kABytes;
            const uint32_t b_hi = a_lo + kABytes;
            const uint32_t b_lo = b_hi + kBBytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 8; ++kk) {
              // K-major: the next 8 columns of K are 32 bytes further along
              // each 128-byte row.
              const uint64_t dah = smem_desc_sw128(a_hi + kk * 32, 16, 1024);
              const uint64_t dal = smem_desc_sw128(a_lo + kk * 32, 16, 1024);
              const uint64_t dbh = smem_desc_sw128(b_hi + kk * 32, 16, 1024);
              const uint64_t dbl = smem_desc_sw128(b_lo + kk * 32, 16, 1024);
              const uint32_t acc = (kc > u0 || kk > 0) ? 1u : 0u;
              mma_tf32(d_tmem, dah, dbh, idesc, acc);
              mma_tf32(d_tmem, dah, dbl, idesc, 1u);
              mma_tf32(d_tmem, dal, dbh, idesc, 1u);
            }
            mma_commit(empty + stage);
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          mma_commit(acc_full + buf);
        }
      }
      mma_commit(drain);
      if (!mbar_wait(drain, 0u, kDrainNs)) set_status(p.status, GPTQ_ERR_TIMEOUT);
    }
  } else {
    // ---------------- epilogue: W -= accumulator ----------------
    const int quad = warp & 3;
    const bool vec = (p.ldw % 4 == 0) && (p.c0 % 4 == 0) && (reinterpret_cast<uintptr_t>(p.W) % 16 == 0);
    int local = 0;
    bool live = true;
    for (int t = blockIdx.x; t < num_tiles && live; t += gridDim.x)
    for (int u0 = 0; u0 < kchunks; u0 += p.unit_chunks, ++local) {
      const int tm = t / p.tiles_n, tn = t - tm * p.tiles_n;
      const int col0 = p.c0 + tn * kBN;
      const int ncols = min(kBN, p.c0 + p.N - col0);
      const int buf = local & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(local >> 1) & 1u;
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(acc_full + buf, acc_phase, p.wait_ns) && !*abort_flag;
        if (!ok) {
          set_status(p.status, GPTQ_ERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        live = false;
        break;
      }
      tc_fence_after();
      // W -= acc as L2 reductions (nothing read back into the SM; each element
      // receives one fp32 addition per launch, tiles being disjoint), written
      // through the warp's staging buffer a whole 128-byte line at a time
      float* stg = staging + (warp - 2) * 32 * 33;
      const int row_base = tm * kBM + quad * 32;
      float* wblk = p.W + static_cast<int64_t>(row_base) * p.ldw + col0;
      for (int c = 0; c < kBN; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * kBN + c), v);
        tmem_ld_wait();
        if (c < ncols && row_base < p.M)
          warp_block_out(v, stg, wblk + c, p.ldw, true, p.M - row_base, ncols - c, vec);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + buf);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Ut_hi[c][k] = hi(U[k][c]), Ut_lo[c][k] = U[k][c] - hi, hi = U with its 13
// low mantissa bits cleared; 32 x 32 tiles transposed through shared memory.
__global__ void split_transpose_tf32_kernel(const float* __restrict__ U, int n, float* __restrict__ hi,
                                            float* __restrict__ lo, int64_t ld_dst) {
  __shared__ float t[32][33];
  const int k0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int k = k0 + i, c = c0 + threadIdx.x;
    t[i][threadIdx.x] = (k < n && c < n) ? U[static_cast<int64_t>(k) * n + c] : 0.0f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, k = k0 + threadIdx.x;
    if (c < n && k < n) {
      const float x = t[threadIdx.x][i];
      const float h = __uint_as_float(__float_as_uint(x) & 0xffffe000u);
      hi[static_cast<int64_t>(c) * ld_dst + k] = h;
      lo[static_cast<int64_t>(c) * ld_dst + k] = x - h;
    }
  }
}

bool set_smem_attr(const DeviceInfo* info) {
  static std::atomic<bool> attr_set[64] = {};  // per device, shared by host threads
  if (!attr_set[info->device]) {
    if (cudaFuncSetAttribute(trailing_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
      return false;
    attr_set[info->device] = true;
  }
  return true;
}

}  // namespace

// Splits U [n, n] into transposed tf32 hi / lo halves with row pitch ldu.
gptq_status split_u_tf32(const float* U, int n, int64_t ldu, float* U_hi, float* U_lo, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(ceil_div(n, 32)), static_cast<unsigned>(ceil_div(n, 32)));
  launch(split_transpose_tf32_kernel, grid, dim3(32, 8), 0, st, U, n, U_hi, U_lo, ldu);
  return launch_status();
}

// W[:, c0:c0+N] -= E[:, 0:K] U[k0:k0+K, c0:c0+N]; E given as hi/lo halves
// [M, lde] and U as transposed hi/lo halves Ut[c][k] with pitch ldu; K a
// multiple of 32.
gptq_status trailing_update_tc(float* W, int64_t ldw, int M, int N, int K, int c0, int k0, const float* E_hi,
                               const float* E_lo, int64_t lde, const float* U_hi, const float* U_lo, int64_t ldu,
                               int n_u, cudaStream_t st) {
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GPTQ_ERR_CUDA;
  if (M <= 0 || N <= 0 || K <= 0) return GPTQ_OK;
  if (K % kBK != 0) return GPTQ_ERR_INVALID_ARG;
  CUtensorMap m_ehi, m_elo, m_uhi, m_ulo;
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  // E's maps span exactly the K columns used (the base may sit inside a row)
  if (!make_tensor_map_2d(&m_ehi, f32, E_hi, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                          static_cast<uint64_t>(lde) * 4, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&m_elo, f32, E_lo, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                          static_cast<uint64_t>(lde) * 4, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&m_uhi, f32, U_hi, static_cast<uint64_t>(n_u), static_cast<uint64_t>(n_u),
                          static_cast<uint64_t>(ldu) * 4, kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&m_ulo, f32, U_lo, static_cast<uint64_t>(n_u), static_cast<uint64_t>(n_u),
                          static_cast<uint64_t>(ldu) * 4, kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return GPTQ_ERR_CUDA;
  if (!set_smem_attr(info)) return GPTQ_ERR_CUDA;
  TrailParams p;
  p.W = W;
  p.ldw = ldw;
  p.M = M;
  p.N = N;
  p.K = K;
  p.unit_chunks = K / kBK;  // one unit: the whole contraction
  p.c0 = c0;
  p.k0 = k0;
  p.tiles_m = static_cast<int>(ceil_div(M, kBM));
  p.tiles_n = static_cast<int>(ceil_div(N, kBN));
  p.status = info->status;
  p.wait_ns = wait_limit_ns();
  const int grid = std::min(info->sm_count, p.tiles_m * p.tiles_n);
  if (launch_pdl(trailing_tc_kernel, dim3(grid), dim3(kThreads), kSmemBytes, st, m_ehi, m_elo, m_uhi, m_ulo, p) !=
      cudaSuccess)
    return GPTQ_ERR_CUDA;
  return GPTQ_OK;
}


}  // namespace gptq
