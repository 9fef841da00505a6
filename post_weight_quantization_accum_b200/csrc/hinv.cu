// Damping, act-order and the upper inverse factor U with U^T U = (H + lambda I)^-1.
//
// GPTQ knowledge note, "How It Works": a damped Cholesky formulation supplies
// the correction rows; anthology record SOTA-185: the optional reordering
// trick.  Route taken here (one Cholesky, one triangular inverse, no explicit
// inverse of H):
//
//   A = J P^T (H + lambda I) P J          (J = order reversal, P = act-order)
//   A = L L^T,  X = L^-1                  128-wide panels, see below
//   U = J X J                             (an anti-transpose of Y = X^T)
//
// With H' = P^T (H + lambda I) P, J H' J = L L^T gives H' = (J L J)(J L J)^T
// with J L J upper triangular, so U = (J L J)^-1 = J L^-1 J is upper with
// U^T U = H'^-1: it is the upper Cholesky factor of the inverse.
//
// A is held at a padded order np (a multiple of 128) with the identity in the
// padding, so every tile is a whole 128 x 128 tile; the padding's factor and
// inverse are the identity and never touch the leading n x n block.
#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace gptq {
namespace {

// --------------------------------------------------------------------------
// dead columns, damping and the act-order key
// --------------------------------------------------------------------------

// One CTA: key_i = hdiag_i (or H_ii); dead_i = (key_i == 0); key_i := 1 for a
// dead column; lambda = damp * mean over i of (dead_i ? 1 : H_ii), summed in
// fp64 in a fixed order.
__global__ void diag_prep_kernel(const float* __restrict__ H, const double* __restrict__ hdiag, int n, float damp,
                                 double* __restrict__ key, uint8_t* __restrict__ dead, double* __restrict__ lambda,
                                 int* status) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float hii = H[static_cast<size_t>(i) * n + i];
    double k = hdiag != nullptr ? hdiag[i] : static_cast<double>(hii);
    const bool is_dead = (k == 0.0);
    if (!isfinite(k) || !isfinite(hii)) set_status(status, GPTQ_ERR_NONFINITE);
    key[i] = is_dead ? 1.0 : k;
    dead[i] = is_dead ? 1 : 0;
    s += is_dead ? 1.0 : static_cast<double>(hii);
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *lambda = static_cast<double>(damp) * (red[0] / n);
}

// Stable descending order of the key: column i goes to position
// #{j : key_j > key_i or (key_j == key_i and j < i)}.
__global__ void act_order_rank_kernel(const double* __restrict__ key, int n, int32_t* __restrict__ perm) {
  __shared__ double tile[1024];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const double ki = i < n ? key[i] : 0.0;
  int rank = 0;
  for (int j0 = 0; j0 < n; j0 += blockDim.x) {
    const int j = j0 + threadIdx.x;
    tile[threadIdx.x] = j < n ? key[j] : 0.0;
    __syncthreads();
    const int m = min(static_cast<int>(blockDim.x), n - j0);
    for (int jj = 0; jj < m; ++jj) {
      const double kj = tile[jj];
      rank += (kj > ki) || (kj == ki && j0 + jj < i);
    }
    __syncthreads();
  }
  if (i < n) perm[rank] = i;
}

__global__ void identity_perm_kernel(int32_t* perm, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) perm[i] = i;
}

// A's lower triangle at the padded order np: the damped, permuted and
// reversed Hessian where a, b < n, the identity in the padding.  Dead
// diagonals become 1 + lambda.  (The upper triangle is never read.)
constexpr int kGatherRows = 32;  // rows of A per CTA of gather_reversed_kernel

// One thread per column b of A, over a chunk of kGatherRows rows: its source
// column perm[n-1-b] is read once and the rows' loads are independent of one
// another, so many are in flight at once.
__global__ void gather_reversed_kernel(const float* __restrict__ H, const int32_t* __restrict__ perm,
                                       const uint8_t* __restrict__ dead, const double* __restrict__ lambda, int n,
                                       int64_t np, float* __restrict__ A) {
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= np) return;
  const int pl = b < n ? perm[n - 1 - b] : 0;
  const int64_t a0 = static_cast<int64_t>(blockIdx.y) * kGatherRows;
  const int64_t a1 = a0 + kGatherRows < np ? a0 + kGatherRows : np;
#pragma unroll 8
  for (int64_t a = a0 > b ? a0 : b; a < a1; ++a) {  // the lower triangle: b <= a
    float v;
    if (a < n && b < n) {
      const int ph = perm[n - 1 - a];
      if (a == b) {
        const double base = dead[ph] ? 1.0 : static_cast<double>(H[static_cast<size_t>(ph) * n + ph]);
        v = static_cast<float>(base + *lambda);
      } else {
        v = H[static_cast<size_t>(ph) * n + pl];
      }
    } else {
      v = a == b ? 1.0f : 0.0f;
    }
    A[a * np + b] = v;
  }
}

// U[a][b] = Y[n-1-b][n-1-a] (a, b < n): the anti-transpose of Y = X^T, i.e.
// U = J X J.  32 x 32 tiles through shared memory; tiles strictly below the
// diagonal are zeros and read nothing.
__global__ void anti_transpose_kernel(const float* __restrict__ Y, int64_t ldy, int n, float* __restrict__ U) {
  __shared__ float t[32][33];
  const int a0 = blockIdx.y * 32, b0 = blockIdx.x * 32;
  if (b0 + 31 < a0) {
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
      const int a = a0 + i, b = b0 + threadIdx.x;
      if (a < n && b < n) U[static_cast<int64_t>(a) * n + b] = 0.0f;
    }
    return;
  }
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int b = b0 + i, a = a0 + threadIdx.x;
    t[i][threadIdx.x] = (a < n && b < n) ? Y[static_cast<int64_t>(n - 1 - b) * ldy + (n - 1 - a)] : 0.0f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int a = a0 + i, b = b0 + threadIdx.x;
    if (a < n && b < n) U[static_cast<int64_t>(a) * n + b] = t[threadIdx.x][i];
  }
}

// --------------------------------------------------------------------------
// Cholesky and inverse in one persistent cooperative kernel
// --------------------------------------------------------------------------
//
// A = L L^T is factored in 128-wide panels k = 0 .. nb-1 while X = L^-1 is
// built by a right-looking forward substitution (R = I; block row k of X is
// Linv_kk R_k,<=k, then R_i,<=k -= L_ik X_k,<=k for i > k).  The kernel keeps
// Y = X^T instead of X (and Ry = R^T in Y's places), which makes every tile
// product C = P Q^T with both P and Q read along their rows:
//
//   phase T(k)  trsm      L_ik   = A_ik Linv_kk^T           i > k
//               finalize  Y_jk   = Ry_jk Linv_kk^T          j < k
//   phase U(k)  update    A_ij  -= L_ik L_jk^T              k < j <= i
//               inverse   Ry_ji -= Y_jk L_ik^T              j <= k < i
//               factor    Linv_{k+1,k+1}                     (CTA 0, right
//                         after its own update of that tile; another CTA
//                         writes Y_{k+1,k+1} = its transpose in phase T(k+1))
//
// Every operation is one 128 x 128 x 128 product on the tensor cores
// (tcgen05.mma kind::tf32, fp32 accumulation in tensor memory), fp32-accurate
// through the 3-term split P_hi Q_hi + P_hi Q_lo + P_lo Q_hi (x_hi = x with
// its 13 low mantissa bits cleared, x_lo = x - x_hi; the dropped P_lo Q_lo is
// below 2^-20 of the product).  The tensor cores read an fp32 operand as tf32
// by dropping those 13 bits, so the chunks TMA brings in (128-byte swizzle,
// K-major, a three-stage ring with two chunks in flight ahead) serve as the
// hi halves as they are, and the threads only form the lo halves (a two-stage
// ring in the same layout).  One thread issues the MMAs; the accumulator is
// double-buffered, so one operation's epilogue (tensor memory -> registers ->
// a store, or an L2 vector reduction for the subtracting operations) overlaps
// the next one's products.  Each tile receives at most one result per phase.
// Two time-bounded grid barriers per panel; every wait is bounded, and a CTA
// that gives up lets its own tensor-core work finish and releases its tensor
// memory before returning.

constexpr int kT = 128;                      // panel width and tile order
constexpr int kCk = 32;                      // fp32 columns of K per staged chunk (one 128-byte row)
constexpr int kChunks = kT / kCk;
constexpr int kCholThreads = 256;
constexpr int kBufBytes = kT * kCk * 4;      // one 128 x 32 fp32 operand chunk (16 KB)
constexpr int kPairBytes = 2 * kBufBytes;    // a chunk of both operands: P then Q
constexpr int kRawStages = 3;                // operand chunks as loaded (TMA), 2 in flight ahead
constexpr int kLoStages = 2;                 // their low halves, formed by the threads
constexpr int kSP = 132;                     // row pitch (floats) of the diagonal factor's matrices
constexpr int kSub = 16;                     // sub-panel width of the diagonal factor
constexpr size_t kStageFloats = 8 * 32 * 33;  // the epilogue's per-warp staging buffers
constexpr size_t kRingBytes = static_cast<size_t>(kRawStages + kLoStages) * kPairBytes + kStageFloats * 4;
constexpr size_t kFactorBytes = (2 * static_cast<size_t>(kT) * kSP + static_cast<size_t>(kSub) * kT + kT) * 4;
constexpr size_t kRegionBytes = kFactorBytes > kRingBytes ? kFactorBytes : kRingBytes;
constexpr int kNumBars = 2 * kRawStages + kLoStages + 2 + 1;  // raw full / free, lo free, accumulators, drain
constexpr size_t kCholSmem = 1024 + kRegionBytes + kNumBars * 8 + 16;  // alignment slack, region, barriers, slot
constexpr uint32_t kCholTmemCols = 2 * kT;                         // two 128 x 128 fp32 accumulators
constexpr int kMaxCholCtas = 1024;
constexpr uint64_t kDrainNs = 2000000000ull;

struct CholArgs {
  float* A;         // [np, np] at pitch ld, lower: the damped reversed matrix; panels become L
  float* Y;         // [np, np] at pitch ld, zero on entry: becomes Y = (L^-1)^T (upper)
  float* Linv;      // [2][kT, kT] diagonal block k's inverse (row-major) in slot k % 2
  int64_t ld;       // np, a multiple of kT
  int nb;           // np / kT
  int* fstatus;     // factorization status word
  unsigned* bar;    // grid barrier: [0] arrivals, [1] generation (zeroed on entry)
  int* abort;       // set when a wait runs out (zeroed on entry)
  uint64_t wait_ns;
};

// Grid barrier over the whole (co-resident) grid in two halves: grid_arrive
// (every thread of the CTA; its writes so far become visible first) returns
// the generation that grid_wait then waits to see pass (time-bounded).  A CTA
// may work between the two.
__device__ unsigned grid_arrive(const CholArgs& p) {
  __shared__ unsigned gen_s;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile unsigned* gen_p = p.bar + 1;
    const unsigned gen = *gen_p;
    __threadfence();
    if (atomicAdd(p.bar, 1u) + 1u == gridDim.x) {
      atomicExch(p.bar, 0u);
      __threadfence();
      atomicAdd(p.bar + 1, 1u);
    }
    gen_s = gen;
  }
  __syncthreads();
  return gen_s;
}

__device__ bool grid_wait(const CholArgs& p, unsigned gen) {
  __shared__ int ok_s;
  if (threadIdx.x == 0) {
    int ok = 1;
    volatile unsigned* gen_p = p.bar + 1;
    const uint64_t t0 = global_ns();
    while (*gen_p == gen) {
      if (*reinterpret_cast<volatile int*>(p.abort)) {
        ok = 0;
        break;
      }
      if (global_ns() - t0 > p.wait_ns) {
        set_status(p.fstatus, GPTQ_ERR_TIMEOUT);
        atomicExch(p.abort, 1);
        ok = 0;
        break;
      }
    }
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

__device__ __forceinline__ bool grid_sync(const CholArgs& p) { return grid_wait(p, grid_arrive(p)); }

__device__ __forceinline__ void give_up(const CholArgs& p) {
  if (threadIdx.x == 0) {
    set_status(p.fstatus, GPTQ_ERR_TIMEOUT);
    atomicExch(p.abort, 1);
  }
}

__device__ __forceinline__ float* tile_at(float* base, int64_t ld, int i, int j) {
  return base + static_cast<int64_t>(i) * kT * ld + static_cast<int64_t>(j) * kT;
}

// One tile operation: C = P Q^T (sub == 0) or C -= P Q^T (sub == 1); all
// three are 128 x 128 tiles, rows of P and Q along K.  P and Q are given by
// the tensor map they are loaded through (kMapA, kMapY, kMapL) and the
// coordinates of their first element.
enum { kMapA = 0, kMapY = 1, kMapL = 2 };
struct TileOp {
  int pm, pr, pc;
  int qm, qr, qc;
  float* C;
  int sub;
};

struct Maps {
  const CUtensorMap* m[3];
};

__device__ __forceinline__ float* linv_slot(const CholArgs& p, int k) { return p.Linv + (k & 1) * kT * kT; }

__device__ TileOp op_phase_t(const CholArgs& p, int k, int t) {
  const int ntrsm = p.nb - 1 - k;
  TileOp op;
  op.qm = kMapL;
  op.qr = (k & 1) * kT;  // Linv slot k % 2
  op.qc = 0;
  op.sub = 0;
  const bool trsm = t < ntrsm;
  const int i = trsm ? k + 1 + t : t - ntrsm;
  op.pm = trsm ? kMapA : kMapY;
  op.pr = i * kT;
  op.pc = k * kT;
  op.C = tile_at(trsm ? p.A : p.Y, p.ld, i, k);
  return op;
}

__device__ TileOp op_phase_u(const CholArgs& p, int k, int t) {
  const int m = p.nb - 1 - k;
  const int nupd = m * (m + 1) / 2;
  TileOp op;
  op.sub = 1;
  if (t < nupd) {  // (a, b), b <= a, in row-major order of the lower triangle
    int a = static_cast<int>((sqrtf(8.0f * t + 1.0f) - 1.0f) * 0.5f);
    while ((a + 1) * (a + 2) / 2 <= t) ++a;
    while (a * (a + 1) / 2 > t) --a;
    const int b = t - a * (a + 1) / 2;
    const int i = k + 1 + a, j = k + 1 + b;
    op.pm = kMapA, op.pr = i * kT, op.pc = k * kT;  // L_ik
    op.qm = kMapA, op.qr = j * kT, op.qc = k * kT;  // L_jk
    op.C = tile_at(p.A, p.ld, i, j);
  } else {
    const int tt = t - nupd;
    const int i = k + 1 + tt / (k + 1), j = tt % (k + 1);
    op.pm = kMapY, op.pr = j * kT, op.pc = k * kT;  // Y_jk
    op.qm = kMapA, op.qr = i * kT, op.qc = k * kT;  // L_ik
    op.C = tile_at(p.Y, p.ld, j, i);
  }
  return op;
}

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }

// lo = x - hi(x) for one chunk pair, elementwise (the layout is kept).
__device__ __forceinline__ void form_lo(const uint8_t* raw, uint8_t* lo) {
#pragma unroll
  for (int u = 0; u < kPairBytes / 16 / kCholThreads; ++u) {
    const int off = 16 * (threadIdx.x + u * kCholThreads);
    const float4 x = *reinterpret_cast<const float4*>(raw + off);
    *reinterpret_cast<float4*>(lo + off) =
        make_float4(x.x - tf32_hi(x.x), x.y - tf32_hi(x.y), x.z - tf32_hi(x.z), x.w - tf32_hi(x.w));
  }
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

// The three tf32 products of one chunk (4 K-steps of 8) into d_tmem: the raw
// chunk read as the hi halves, the formed chunk as the lo halves.
__device__ __forceinline__ void issue_chunk(const uint8_t* raw, const uint8_t* lo, uint32_t d_tmem, bool first) {
  const uint32_t idesc = instr_desc(2u, 0u, 0u, kT, kT);  // tf32, both operands K-major, 128 x 128
  const uint32_t ph = smem_u32(raw), qh = ph + kBufBytes, pl = smem_u32(lo), ql = pl + kBufBytes;
#pragma unroll
  for (int kk = 0; kk < kCk / 8; ++kk) {
    // K-major: the next 8 columns of K are 32 bytes further along each row
    const uint64_t dph = smem_desc_sw128(ph + kk * 32, 16, 1024);
    const uint64_t dpl = smem_desc_sw128(pl + kk * 32, 16, 1024);
    const uint64_t dqh = smem_desc_sw128(qh + kk * 32, 16, 1024);
    const uint64_t dql = smem_desc_sw128(ql + kk * 32, 16, 1024);
    mma_tf32(d_tmem, dph, dqh, idesc, (first && kk == 0) ? 0u : 1u);
    mma_tf32(d_tmem, dph, dql, idesc, 1u);
    mma_tf32(d_tmem, dpl, dqh, idesc, 1u);
  }
}

// The accumulator into the output tile: warp w reads lanes 32 (w % 4) .. + 31
// (tile rows) and columns 64 (w / 4) .. + 63, and writes them row by row
// through its staging buffer (whole 128-byte lines per four rows), as stores
// or as L2 reductions (so the old values never travel to the SM).
__device__ __forceinline__ void write_tile(const TileOp& op, int64_t ld, uint32_t acc, float* stage) {
  const int warp = threadIdx.x >> 5;
  const int quad = warp & 3, half = warp >> 2;
  float* stg = stage + warp * 32 * 33;
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int c0 = 64 * half + 32 * x;
    uint32_t v[32];
    tmem_ld_32x32b_x32(acc + (static_cast<uint32_t>(32 * quad) << 16) + static_cast<uint32_t>(c0), v);
    tmem_ld_wait();
    warp_block_out(v, stg, op.C + static_cast<int64_t>(32 * quad) * ld + c0, ld, op.sub != 0, 32, 32, true);
  }
}

// Per-CTA pipeline state (identical in every thread).
struct Pipe {
  uint8_t* raw;          // kRawStages chunk pairs as loaded, 1024-byte aligned
  uint8_t* lo;           // kLoStages chunk pairs of low halves
  float* stage;          // [8 warps][32][33] epilogue staging
  uint64_t* raw_full;    // [kRawStages]: a chunk pair has landed
  uint64_t* raw_free;    // [kRawStages]: the products reading a raw stage are done
  uint64_t* lo_free;     // [kLoStages]: the products reading a lo stage are done
  uint64_t* acc_full;    // [2]: an accumulator's products are done
  uint64_t* drain;
  uint32_t tmem;         // base of the two accumulators
  uint32_t chunks;       // chunk pairs consumed so far (all phases)
  uint32_t ops;          // operations issued so far
};

// Waits for operation number o's products and writes its tile.
__device__ bool finish_op(const CholArgs& p, const Pipe& pp, const TileOp& op, uint32_t o) {
  const bool ok = mbar_wait(pp.acc_full + (o & 1u), (o >> 1) & 1u, p.wait_ns);
  if (!__syncthreads_and(ok)) {
    give_up(p);
    return false;
  }
  tc_fence_after();
  write_tile(op, p.ld, pp.tmem + (o & 1u) * kT, pp.stage);
  tc_fence_before();
  return true;
}

// Thread 0: the TMA loads of chunk c of `op` as chunk pair number q (its raw
// stage must have been released by the products of pair q - kRawStages).
__device__ __forceinline__ bool load_pair(const CholArgs& p, const Maps& mp, const Pipe& pp, const TileOp& op,
                                          int c, uint32_t q) {
  const uint32_t s = q % kRawStages;
  if (q >= kRawStages && !mbar_wait(pp.raw_free + s, ((q - kRawStages) / kRawStages) & 1u, p.wait_ns)) return false;
  uint8_t* dst = pp.raw + s * kPairBytes;
  mbar_arrive_expect_tx(pp.raw_full + s, kPairBytes);
  tma_load_2d(dst, mp.m[op.pm], pp.raw_full + s, op.pc + c * kCk, op.pr);
  tma_load_2d(dst + kBufBytes, mp.m[op.qm], pp.raw_full + s, op.qc + c * kCk, op.qr);
  return true;
}

// On a failure path, thread 0 waits (bounded) for the loads it issued but
// nobody consumed, pairs [from, to) after `base`, so that no copy is still
// landing in shared memory when the CTA returns.
__device__ void drain_loads(const Pipe& pp, uint32_t base, int from, int to) {
  if (threadIdx.x != 0) return;
  for (int l = from; l < to; ++l) {
    const uint32_t q = base + l;
    mbar_wait(pp.raw_full + q % kRawStages, (q / kRawStages) & 1u, kDrainNs);
  }
}

template <bool kPhaseU>
__device__ __forceinline__ TileOp op_at(const CholArgs& p, int k, int t) {
  return kPhaseU ? op_phase_u(p, k, t) : op_phase_t(p, k, t);
}

// Runs operations [lo, hi) of a phase.  Returns false if a wait ran out.
// On return every product this CTA issued is done.
template <bool kPhaseU>
__device__ bool run_ops(const CholArgs& p, const Maps& mp, Pipe& pp, int k, int lo, int hi) {
  if (lo >= hi) return true;
  const int npairs = (hi - lo) * kChunks;
  const uint32_t base = pp.chunks;
  // this CTA's earlier generic writes (the diagonal factor's shared memory,
  // tiles written by its epilogues) before the TMA writes and reads below
  fence_async_all();
  __syncthreads();
  int issued = 0;  // thread 0: pairs of this call whose loads are issued
  bool ok0 = true;
  if (threadIdx.x == 0) {
    while (issued < kRawStages - 1 && issued < npairs && ok0) {
      ok0 = load_pair(p, mp, pp, op_at<kPhaseU>(p, k, lo + issued / kChunks), issued % kChunks, base + issued);
      if (ok0) ++issued;
    }
  }
  TileOp cur = op_at<kPhaseU>(p, k, lo), prev = cur;
#pragma unroll 1
  for (int l = 0; l < npairs; ++l) {
    const int t = lo + l / kChunks, c = l % kChunks;
    if (c == 0 && l > 0) cur = op_at<kPhaseU>(p, k, t);
    const uint32_t q = base + l, s = q % kRawStages, s2 = q % kLoStages;
    bool ok = mbar_wait(pp.raw_full + s, (q / kRawStages) & 1u, p.wait_ns);
    if (ok && q >= kLoStages) ok = mbar_wait(pp.lo_free + s2, ((q - kLoStages) / kLoStages) & 1u, p.wait_ns);
    const uint8_t* raw = pp.raw + s * kPairBytes;
    uint8_t* lop = pp.lo + s2 * kPairBytes;
    if (ok) form_lo(raw, lop);
    fence_async_smem();
    if (!__syncthreads_and(ok && ok0)) {
      give_up(p);
      drain_loads(pp, base, l + (ok ? 1 : 0), issued);
      return false;
    }
    const uint32_t buf = pp.ops & 1u;
    if (threadIdx.x == 0) {
      tc_fence_after();
      issue_chunk(raw, lop, pp.tmem + buf * kT, c == 0);
      mma_commit(pp.raw_free + s);
      mma_commit(pp.lo_free + s2);
      if (c + 1 == kChunks) mma_commit(pp.acc_full + buf);
      if (issued < npairs && ok0) {
        ok0 = load_pair(p, mp, pp, op_at<kPhaseU>(p, k, lo + issued / kChunks), issued % kChunks, base + issued);
        if (ok0) ++issued;
      }
    }
    ++pp.chunks;
    if (c + 1 == kChunks) {
      if (t > lo && !finish_op(p, pp, prev, pp.ops - 1)) {
        drain_loads(pp, base, l + 1, issued);
        return false;
      }
      prev = cur;
      ++pp.ops;
    }
  }
  return finish_op(p, pp, prev, pp.ops - 1);
}

// Right-looking Cholesky of a 16 x 16 block held by one warp: lane l holds
// row l / 2, columns 8 (l % 2) .. + 7 in v (only the lower half is read).
// On return v holds L's lower half and rdiag[j] = 1 / L_jj.  A pivot that is
// not positive or not finite raises a flag and is replaced by 1.
//
// At pivot j every lane subtracts (A_rj / A_jj) A_cj from each of its entries
// right of column j (which of a lane's eight columns lie right of j is fixed
// by j and the lane's half, so no lane branches); entries above the diagonal
// take the same update and are never read.
__device__ __forceinline__ void chol16(float (&v)[8], float* rdiag, bool& nonfinite, bool& notpd) {
  const int lane = threadIdx.x & 31, r = lane >> 1, h = lane & 1;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int jh = j >> 3, jq = j & 7;
    float d = __shfl_sync(0xffffffffu, v[jq], 2 * j + jh);           // A_jj
    const float mine = __shfl_sync(0xffffffffu, v[jq], 2 * r + jh);   // A_rj
    float col[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) col[q] = __shfl_sync(0xffffffffu, v[jq], 16 * h + 2 * q + jh);  // A_cj
    nonfinite |= !isfinite(d);
    notpd |= !(d > 0.0f);
    d = (d > 0.0f && d < INFINITY) ? d : 1.0f;
    const float rs = rsqrtf(d);
    const float m = mine * (rs * rs);  // L_rj / L_jj
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q > j) {
        v[q] = fmaf(-m, col[q], v[q]);  // column q (and 8 + q) right of j in both halves
      } else if (q + 8 > j) {
        const float u = fmaf(-m, col[q], v[q]);  // column 8 + q right of j: the upper half's lanes
        v[q] = h ? u : v[q];
      }
    }
    if (h == jh) v[jq] = r > j ? mine * rs : (r == j ? d * rs : v[jq]);
    if (lane == 0) rdiag[j] = rs;
  }
}

// x <- L_ss^-1 x for the sub-block's factor (lower half of S at (b0, b0))
// and its reciprocal diagonal: the forward substitution both halves of
// phase A below use (for rows of the panel x holds S_i,s, for columns of the
// inverse R_s,j).
__device__ __forceinline__ void solve16(float (&x)[16], const float* S, const float* rd, int b0) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    x[c] *= rd[b0 + c];
#pragma unroll
    for (int c2 = c + 1; c2 < 16; ++c2) x[c2] = fmaf(-x[c], S[(b0 + c2) * kSP + b0 + c], x[c2]);
  }
}

// Factors the diagonal block k (by one CTA): Linv_kk into its Linv slot
// (row-major).
//
// In 16-wide sub-panels s of the block S (its lower half), with R = I beside it:
//   warp 0   Cholesky of the sub-panel's 16 x 16 diagonal block (chol16)
//   phase A  rows i below: L_i,s = S_i,s L_ss^-T, one thread per row, into
//            the panel buffer Pn (transposed); columns j < end of the
//            sub-panel: X_s,j = L_ss^-1 R_s,j, one thread per column, in place
//   phase B  S_ic -= L_i,s L_c,s^T (c <= i below the sub-panel) and
//            R_ij -= L_i,s X_s,j (i below, j < end of the sub-panel) in 4 x 4
//            blocks; warp 0 first updates the next diagonal 16 x 16 block and
//            factors it (the sweep's critical path).
// A pivot that is not positive or not finite sets the status word (a
// non-finite one takes precedence) and is replaced by 1.
__device__ void factor_block(const CholArgs& p, int k, float* fs) {
  float* S = fs;                // [kT][kSP]
  float* XR = S + kT * kSP;     // [kT][kSP]: R, then X = L^-1 (lower)
  float* Pn = XR + kT * kSP;    // [kSub][kT]: the current sub-panel of L, transposed
  float* rd = Pn + kSub * kT;   // [kT]: 1 / L_jj
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const float* Akk = tile_at(p.A, p.ld, k, k);
  {
    constexpr int kPer = kT * (kT / 4) / kCholThreads;  // float4 per thread
    float4 a[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {  // every load in flight before the first store
      const int e = t + u * kCholThreads, r = e >> 5, c = 4 * (e & 31);
      a[u] = __ldcg(reinterpret_cast<const float4*>(Akk + r * p.ld + c));
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = t + u * kCholThreads, r = e >> 5, c = 4 * (e & 31);
      *reinterpret_cast<float4*>(S + r * kSP + c) = a[u];
      *reinterpret_cast<float4*>(XR + r * kSP + c) = make_float4(r == c ? 1.0f : 0.0f, r == c + 1 ? 1.0f : 0.0f,
                                                                 r == c + 2 ? 1.0f : 0.0f, r == c + 3 ? 1.0f : 0.0f);
    }
  }
  __syncthreads();
  bool nonfinite = false, notpd = false;
  if (warp == 0) {
    const int r = lane >> 1, h = lane & 1;
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = S[r * kSP + 8 * h + q];
    chol16(v, rd, nonfinite, notpd);
#pragma unroll
    for (int q = 0; q < 8; ++q) S[r * kSP + 8 * h + q] = v[q];
  }
  __syncthreads();
#pragma unroll 1
  for (int s = 0; s < kT / kSub; ++s) {
    const int b0 = s * kSub, e = b0 + kSub;
    // phase A
    if (t < kT - e) {
      const int i = e + t;
      float x[16];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float4 w = *reinterpret_cast<const float4*>(S + i * kSP + b0 + 4 * g);
        x[4 * g] = w.x;
        x[4 * g + 1] = w.y;
        x[4 * g + 2] = w.z;
        x[4 * g + 3] = w.w;
      }
      solve16(x, S, rd, b0);
#pragma unroll
      for (int c = 0; c < 16; ++c) Pn[c * kT + i] = x[c];
    } else if (t >= kT && t - kT < e) {
      const int j = t - kT;
      float x[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) x[c] = XR[(b0 + c) * kSP + j];
      solve16(x, S, rd, b0);
#pragma unroll
      for (int c = 0; c < 16; ++c) XR[(b0 + c) * kSP + j] = x[c];
    }
    if (e == kT) {
      __syncthreads();
      break;
    }
    // phase B.  Warp 0 needs only the rows it solved itself (the 16 below the
    // sub-panel), so it arrives at barrier 1 without waiting and starts on
    // the next diagonal block; the other warps wait there for all of phase A.
    if (warp == 0) {
      __syncwarp();
      asm volatile("bar.arrive 1, %0;" ::"r"(kCholThreads) : "memory");
      const int r = lane >> 1, h = lane & 1, i = e + r, c0 = e + 8 * h;
      float v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = S[i * kSP + c0 + q];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float li = Pn[q * kT + i];
        const float4 a = *reinterpret_cast<const float4*>(Pn + q * kT + c0);
        const float4 b = *reinterpret_cast<const float4*>(Pn + q * kT + c0 + 4);
        v[0] = fmaf(-li, a.x, v[0]);
        v[1] = fmaf(-li, a.y, v[1]);
        v[2] = fmaf(-li, a.z, v[2]);
        v[3] = fmaf(-li, a.w, v[3]);
        v[4] = fmaf(-li, b.x, v[4]);
        v[5] = fmaf(-li, b.y, v[5]);
        v[6] = fmaf(-li, b.z, v[6]);
        v[7] = fmaf(-li, b.w, v[7]);
      }
      chol16(v, rd + e, nonfinite, notpd);
#pragma unroll
      for (int q = 0; q < 8; ++q) S[i * kSP + c0 + q] = v[q];
    } else {
      asm volatile("bar.sync 1, %0;" ::"r"(kCholThreads) : "memory");
      const int M4 = (kT - e) / 4, E4 = e / 4;
      const int ntr = M4 * (M4 + 1) / 2 - 10;  // lower 4 x 4 blocks outside warp 0's 16 x 16 block
      const int total = ntr + M4 * E4;
      for (int w = t - 32; w < total; w += kCholThreads - 32) {
        float acc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[r][c] = 0.0f;
        float* dst;
        if (w < ntr) {
          const int idx = w + 10;
          int a = static_cast<int>((sqrtf(8.0f * idx + 1.0f) - 1.0f) * 0.5f);
          while ((a + 1) * (a + 2) / 2 <= idx) ++a;
          while (a * (a + 1) / 2 > idx) --a;
          const int bb = idx - a * (a + 1) / 2;
          const int i0 = e + 4 * a, c0 = e + 4 * bb;
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float4 li = *reinterpret_cast<const float4*>(Pn + q * kT + i0);
            const float4 lc = *reinterpret_cast<const float4*>(Pn + q * kT + c0);
            const float lv[4] = {li.x, li.y, li.z, li.w}, cv[4] = {lc.x, lc.y, lc.z, lc.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
              for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(lv[r], cv[c], acc[r][c]);
          }
          dst = S + i0 * kSP + c0;
        } else {
          const int w2 = w - ntr;
          const int i0 = e + 4 * (w2 / E4), j0 = 4 * (w2 % E4);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float4 li = *reinterpret_cast<const float4*>(Pn + q * kT + i0);
            const float4 xq = *reinterpret_cast<const float4*>(XR + (b0 + q) * kSP + j0);
            const float lv[4] = {li.x, li.y, li.z, li.w}, xv[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
              for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(lv[r], xv[c], acc[r][c]);
          }
          dst = XR + i0 * kSP + j0;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          float4 o = *reinterpret_cast<float4*>(dst + r * kSP);
          o.x -= acc[r][0];
          o.y -= acc[r][1];
          o.z -= acc[r][2];
          o.w -= acc[r][3];
          *reinterpret_cast<float4*>(dst + r * kSP) = o;
        }
      }
    }
    __syncthreads();
  }
  if (warp == 0) {
    nonfinite = __any_sync(0xffffffffu, nonfinite);
    notpd = __any_sync(0xffffffffu, notpd);
    if (lane == 0 && (nonfinite || notpd)) set_status(p.fstatus, nonfinite ? GPTQ_ERR_NONFINITE : GPTQ_ERR_NOT_PD);
  }
  // Linv (row-major, zeros above the diagonal); Y_kk = Linv^T is written by
  // another CTA from this slot (write_y_diag), off this CTA's chain
  for (int e = t; e < kT * (kT / 4); e += kCholThreads) {
    const int r = e >> 5, c = 4 * (e & 31);
    float4 x = *reinterpret_cast<const float4*>(XR + r * kSP + c);
    x = make_float4(c <= r ? x.x : 0.0f, c + 1 <= r ? x.y : 0.0f, c + 2 <= r ? x.z : 0.0f, c + 3 <= r ? x.w : 0.0f);
    *reinterpret_cast<float4*>(linv_slot(p, k) + r * kT + c) = x;
  }
  __threadfence();
  __syncthreads();
}

// Y_kk = Linv_kk^T from Linv slot k % 2 (whole tile, zeros below the
// diagonal), transposed through shared memory `T` ([kT][kSP] floats): reads
// with consecutive threads on consecutive rows of Linv (conflict-free
// transposed stores), then whole rows of Y written.
__device__ void write_y_diag(const CholArgs& p, int k, float* T) {
  const int t = threadIdx.x;
  const float* L = linv_slot(p, k);
  __syncthreads();
  for (int e = t; e < kT * (kT / 4); e += kCholThreads) {
    const int rt = e & (kT - 1), ct = 4 * (e >> 7);
    const float4 x = __ldcg(reinterpret_cast<const float4*>(L + rt * kT + ct));
    T[ct * kSP + rt] = x.x;
    T[(ct + 1) * kSP + rt] = x.y;
    T[(ct + 2) * kSP + rt] = x.z;
    T[(ct + 3) * kSP + rt] = x.w;
  }
  __syncthreads();
  float* Ykk = tile_at(p.Y, p.ld, k, k);
  for (int e = t; e < kT * (kT / 4); e += kCholThreads) {
    const int r = e >> 5, c = 4 * (e & 31);
    *reinterpret_cast<float4*>(Ykk + r * p.ld + c) = *reinterpret_cast<const float4*>(T + r * kSP + c);
  }
  __syncthreads();
}

// [lo, hi) of `total` operations for worker w of `workers` (contiguous, equal shares)
__device__ __forceinline__ void share(int total, int w, int workers, int& lo, int& hi) {
  lo = static_cast<int>((static_cast<int64_t>(total) * w) / workers);
  hi = static_cast<int>((static_cast<int64_t>(total) * (w + 1)) / workers);
}

__global__ void __launch_bounds__(kCholThreads, 1)
    chol_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_y,
                   const __grid_constant__ CUtensorMap map_l, CholArgs p) {
  extern __shared__ uint8_t chol_smem_raw[];
  uint8_t* region =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(chol_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(region + kRegionBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  const int warp = threadIdx.x >> 5;
  Maps mp;
  mp.m[kMapA] = &map_a;
  mp.m[kMapY] = &map_y;
  mp.m[kMapL] = &map_l;
  Pipe pp;
  pp.raw = region;
  pp.lo = region + static_cast<size_t>(kRawStages) * kPairBytes;
  pp.stage = reinterpret_cast<float*>(region + static_cast<size_t>(kRawStages + kLoStages) * kPairBytes);
  pp.raw_full = bars;
  pp.raw_free = bars + kRawStages;
  pp.lo_free = bars + 2 * kRawStages;
  pp.acc_full = pp.lo_free + kLoStages;
  pp.drain = pp.acc_full + 2;
  pp.chunks = 0;
  pp.ops = 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bars + i, 1);
    fence_barrier_init();
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_y);
    prefetch_tensormap(&map_l);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kCholTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pp.tmem = *tmem_slot;
  float* fs = reinterpret_cast<float*>(region);  // the diagonal factor's matrices (between products)
  const int G = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x), nb = p.nb;

  if (b == 0) factor_block(p, 0, fs);
  bool live = grid_sync(p);
  for (int k = 0; k < nb && live; ++k) {
    const int m = nb - 1 - k;
    // Y_kk from the Linv slot written by the factor of block k (read from
    // phase U(k) on), by the last CTA before its share of phase T(k)
    if (b == G - 1) write_y_diag(p, k, fs);
    // Phase T(k).  CTA 0 takes the trsm of row block k+1 (operation 0), then
    // arrives, then, while the others finish the panel, updates tile
    // (k+1, k+1) with it (operation 0 of phase U) and factors block k+1 (its
    // inverse goes to the other Linv slot): the diagonal chain overlaps the
    // panel's products.
    if (G == 1) {
      live = run_ops<false>(p, mp, pp, k, 0, nb - 1);
    } else if (b == 0) {
      live = run_ops<false>(p, mp, pp, k, 0, m > 0 ? 1 : 0);
    } else {
      int lo, hi;
      share(nb - 1 - (m > 0 ? 1 : 0), b - 1, G - 1, lo, hi);
      const int off = m > 0 ? 1 : 0;
      live = run_ops<false>(p, mp, pp, k, off + lo, off + hi);
    }
    if (!live) break;
    unsigned gen = grid_arrive(p);
    if (G > 1 && b == 0 && m > 0) {
      live = run_ops<true>(p, mp, pp, k, 0, 1);
      __threadfence();
      __syncthreads();
      if (live) factor_block(p, k + 1, fs);
    }
    if (!live || !grid_wait(p, gen)) {
      live = false;
      break;
    }
    // Phase U(k): every other update and inverse operation, shared by the
    // CTAs other than CTA 0 (all of them when there is only one CTA).
    const int total = m * (m + 1) / 2 + m * (k + 1);
    if (G == 1) {
      live = run_ops<true>(p, mp, pp, k, 0, total);
      if (live && m > 0) factor_block(p, k + 1, fs);
    } else if (b > 0 && total > 1) {
      int lo, hi;
      share(total - 1, b - 1, G - 1, lo, hi);
      live = run_ops<true>(p, mp, pp, k, 1 + lo, 1 + hi);
    }
    if (live) live = grid_sync(p);
  }
  // every exit: this CTA's tensor-core work done, then its tensor memory released
  if (threadIdx.x == 0) {
    mma_commit(pp.drain);
    if (!mbar_wait(pp.drain, 0u, kDrainNs)) set_status(p.fstatus, GPTQ_ERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(pp.tmem, kCholTmemCols);
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline int64_t padded_order(int n) { return ceil_div(n, kT) * kT; }

struct PrepLayout {
  size_t a, y, linv, key, dead, lambda, bar, perm, total;
};

PrepLayout prep_layout(int n) {
  PrepLayout l{};
  const int64_t np = padded_order(n);
  const size_t nn = static_cast<size_t>(np) * static_cast<size_t>(np) * sizeof(float);
  size_t off = 0;
  l.a = off;
  off += align256(nn);
  l.y = off;
  off += align256(nn);
  l.linv = off;
  off += align256(2 * static_cast<size_t>(kT) * kT * sizeof(float));
  l.key = off;
  off += align256(static_cast<size_t>(n) * sizeof(double));
  l.dead = off;
  off += align256(static_cast<size_t>(n));
  l.lambda = off;
  off += 256;
  l.bar = off;  // barrier words and the abort flag
  off += 256;
  l.perm = off;
  off += align256(static_cast<size_t>(n) * sizeof(int32_t));
  l.total = off;
  return l;
}

int chol_grid(const DeviceInfo* info) {
  static std::atomic<int> fits[64] = {};  // per device, shared by host threads: 1 = a CTA fits on an SM
  if (fits[info->device] == 0) {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, chol_tc_kernel, kCholThreads, kCholSmem) != cudaSuccess ||
        b < 1)
      return 0;
    fits[info->device] = 1;
  }
  return std::min(kMaxCholCtas, info->sm_count);  // one CTA per SM (its shared memory and tensor memory)
}

}  // namespace

size_t prepare_workspace_size(int n) { return n > 0 ? prep_layout(n).total : 0; }

gptq_status prepare_hinv(const float* H, const double* hdiag, int n, float damp, int act_order, int32_t* perm_out,
                         uint8_t* dead_out, float* U, void* ws, size_t ws_bytes, cudaStream_t st) {
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GPTQ_ERR_CUDA;
  const PrepLayout l = prep_layout(n);
  if (ws_bytes < l.total) return GPTQ_ERR_INVALID_ARG;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const int64_t np = padded_order(n);
  float* A = reinterpret_cast<float*>(w + l.a);
  float* Y = reinterpret_cast<float*>(w + l.y);
  double* key = reinterpret_cast<double*>(w + l.key);
  uint8_t* dead = w + l.dead;
  double* lambda = reinterpret_cast<double*>(w + l.lambda);
  unsigned* bar = reinterpret_cast<unsigned*>(w + l.bar);
  int32_t* perm = perm_out != nullptr ? perm_out : reinterpret_cast<int32_t*>(w + l.perm);
  int* fstatus = info->status + 1;

  static std::atomic<bool> attr_set[64] = {};  // per device, shared by host threads
  if (!attr_set[info->device]) {
    if (cudaFuncSetAttribute(chol_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kCholSmem)) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    attr_set[info->device] = true;
  }
  const int grid = chol_grid(info);
  if (grid <= 0) return GPTQ_ERR_CUDA;

  if (cudaMemsetAsync(fstatus, 0, sizeof(int), st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaMemsetAsync(bar, 0, 256, st) != cudaSuccess) return GPTQ_ERR_CUDA;
  launch(diag_prep_kernel, 1, 1024, 0, st, H, hdiag, n, damp, key, dead, lambda, fstatus);
  if (act_order)
    launch(act_order_rank_kernel, static_cast<unsigned>(ceil_div(n, 256)), 256, 0, st, key, n, perm);
  else
    launch(identity_perm_kernel, static_cast<unsigned>(ceil_div(n, 256)), 256, 0, st, perm, n);
  if (dead_out != nullptr && cudaMemcpyAsync(dead_out, dead, n, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  launch(gather_reversed_kernel,
         dim3(static_cast<unsigned>(ceil_div(np, 256)), static_cast<unsigned>(ceil_div(np, kGatherRows))), 256, 0, st, H,
         perm, dead, lambda, n, np, A);
  if (cudaMemsetAsync(Y, 0, static_cast<size_t>(np) * static_cast<size_t>(np) * sizeof(float), st) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;

  CholArgs ca;
  ca.A = A;
  ca.Y = Y;
  ca.Linv = reinterpret_cast<float*>(w + l.linv);
  ca.ld = np;
  ca.nb = static_cast<int>(np / kT);
  ca.fstatus = fstatus;
  ca.bar = bar;
  ca.abort = reinterpret_cast<int*>(bar + 2);
  ca.wait_ns = wait_limit_ns();
  CUtensorMap map_a, map_y, map_l;
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (!make_tensor_map_2d(&map_a, f32, A, np, np, np * 4, kCk, kT, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&map_y, f32, Y, np, np, np * 4, kCk, kT, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&map_l, f32, ca.Linv, kT, 2 * kT, kT * 4, kCk, kT, CU_TENSOR_MAP_SWIZZLE_128B))
    return GPTQ_ERR_CUDA;
  void* args[] = {&map_a, &map_y, &map_l, &ca};
  const bool traced = trace_on();
  if (traced) trace_begin(st);
  if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(chol_tc_kernel), dim3(grid), dim3(kCholThreads), args,
                                  kCholSmem, st) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  if (traced) trace_end(st, reinterpret_cast<const void*>(chol_tc_kernel));
  count_launch();
  launch(anti_transpose_kernel, dim3(static_cast<unsigned>(ceil_div(n, 32)), static_cast<unsigned>(ceil_div(n, 32))),
         dim3(32, 8), 0, st, Y, np, n, U);
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;

  int fs = 0;
  if (cudaMemcpyAsync(&fs, fstatus, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GPTQ_ERR_CUDA;
  return static_cast<gptq_status>(fs);
}

}  // namespace gptq
