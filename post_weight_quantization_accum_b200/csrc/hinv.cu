// Damping, act-order and the upper inverse factor U with U^T U = (H + lambda I)^-1.
//
// GPTQ knowledge note, "How It Works": a damped Cholesky formulation supplies
// the correction rows; anthology record SOTA-185: the optional reordering
// trick.  Route taken here (one Cholesky, one triangular inverse, no explicit
// inverse of H):
//
//   A = J P^T (H + lambda I) P J          (J = order reversal, P = act-order)
//   A = L L^T,  X = L^-1                  one persistent cooperative kernel
//   U = J X J                             (X is stored rotated as it is made)
//
// With H' = P^T (H + lambda I) P, J H' J = L L^T gives H' = (J L J)(J L J)^T
// with J L J upper triangular, so U = (J L J)^-1 = J L^-1 J is upper with
// U^T U = H'^-1: it is the upper Cholesky factor of the inverse.
#include <algorithm>

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

// Lower triangle of A = J P^T (H + lambda I) P J; dead diagonals become 1 + lambda.
__global__ void gather_reversed_kernel(const float* __restrict__ H, const int32_t* __restrict__ perm,
                                       const uint8_t* __restrict__ dead, const double* __restrict__ lambda, int n,
                                       float* __restrict__ A) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  const int a = blockIdx.y;
  if (b > a || a >= n) return;
  const int pa = perm[n - 1 - a], pb = perm[n - 1 - b];
  float v;
  if (a == b) {
    const double base = dead[pa] ? 1.0 : static_cast<double>(H[static_cast<size_t>(pa) * n + pa]);
    v = static_cast<float>(base + *lambda);
  } else {
    v = H[static_cast<size_t>(pa) * n + pb];
  }
  A[static_cast<size_t>(a) * n + b] = v;
}

// --------------------------------------------------------------------------
// Cholesky and inverse in one persistent cooperative kernel
// --------------------------------------------------------------------------
//
// A = L L^T is factored in 64-wide panels; X = L^-1 is built alongside it by
// a right-looking forward substitution, R_i = I_i - sum_{m<k} L_im X_m:
//
//   phase T(k)  trsm      L_ik = A_ik Linv_kk^T              for i > k
//               finalize  X_kj = Linv_kk R_kj                for j < k
//   phase U(k)  update    A_ij -= L_ik L_jk^T                for k < j <= i
//               inverse   R_ij -= L_ik X_kj                  for i > k, j <= k
//               factor    L_{k+1,k+1}, Linv_{k+1,k+1}         (by the CTA that
//                         updated that tile first in the phase)
//
// Every step is a 64 x 64 x 64 tile product, and the Cholesky half of a phase
// shrinks as the inverse half grows, so each phase has about the same number
// of tiles.  Two grid barriers per panel (time-bounded).  X is written straight
// into U's rotated position (U = J X J), so no rotation pass is needed;
// R's tiles live in the same places before they are finalized.

constexpr int kT = 64;             // tile width = panel width
constexpr int kPad = 68;           // shared-memory row stride (16-byte aligned rows)
constexpr int kCholThreads = 256;
constexpr size_t kCholSmem = 3 * kT * kPad * sizeof(float);

struct CholArgs {
  float* A;          // [n, n] lower: the damped reversed matrix, becomes L
  float* U;          // [n, n] zeroed on entry; X = L^-1 is written rotated
  int n;
  int nblk;
  int* fstatus;      // factorization status word
  unsigned* bar;     // grid barrier: [0] arrivals, [1] generation (zeroed on entry)
  int* abort;        // set when a barrier wait runs out (zeroed on entry)
  uint64_t wait_ns;
};

typedef float Tile[kPad];

__device__ __forceinline__ float ld_a(const CholArgs& p, int r, int c) {
  return (r < p.n && c < p.n) ? __ldcg(p.A + static_cast<size_t>(r) * p.n + c) : 0.0f;
}
__device__ __forceinline__ float ld_x(const CholArgs& p, int r, int c) {
  return (r < p.n && c < p.n) ? __ldcg(p.U + static_cast<size_t>(p.n - 1 - r) * p.n + (p.n - 1 - c)) : 0.0f;
}
__device__ __forceinline__ float* at_a(const CholArgs& p, int r, int c) { return p.A + static_cast<size_t>(r) * p.n + c; }
__device__ __forceinline__ float* at_x(const CholArgs& p, int r, int c) {
  return p.U + static_cast<size_t>(p.n - 1 - r) * p.n + (p.n - 1 - c);
}

// A thread holds 16 elements of each 64 x 64 tile it stages.
constexpr int kPerThread = kT * kT / kCholThreads;  // 16

// acc[i][j] = sum_k P[k][tr+i] * Q[k][tc+j]  (thread owns a 4x4 block)
__device__ __forceinline__ void tile_product(const Tile* P, const Tile* Q, float (&acc)[4][4]) {
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
#pragma unroll 8
  for (int k = 0; k < kT; ++k) {
    const float4 a = *reinterpret_cast<const float4*>(&P[k][tr]);
    const float4 b = *reinterpret_cast<const float4*>(&Q[k][tc]);
    const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
}

// Lower Cholesky of the 16 x 16 block of `a` at (o, o) by one warp (lanes
// 0..15 own its rows), shuffles only; then the block's inverse, lane c
// solving L x = e_c for column c.  The loops have constant trip counts and
// predicated bodies so that they unroll completely and the row / column stay
// in registers (this kernel runs at its register limit).
__device__ __forceinline__ void warp_chol_inv16(Tile* a, Tile* inv, int o, int* fstatus) {
  const int lane = threadIdx.x & 31;
  const int row = lane & 15;
  float r[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) r[c] = a[o + row][o + c];
#pragma unroll 16
  for (int j = 0; j < 16; ++j) {
    float piv = __shfl_sync(0xffffffffu, r[j], j);
    if (!(piv > 0.0f) || !isfinite(piv)) {
      if (lane == 0) set_status(fstatus, isfinite(piv) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE);
      piv = 1.0f;
    }
    const float d = sqrtf(piv);
    const float rd = 1.0f / d;
    const float l = row > j ? r[j] * rd : (row == j ? d : 0.0f);
    r[j] = l;
#pragma unroll 16
    for (int c = 0; c < 16; ++c) {
      const float lc = __shfl_sync(0xffffffffu, l, c);
      if (c > j && row >= c) r[c] = fmaf(-l, lc, r[c]);
    }
  }
  if (lane < 16) {
#pragma unroll
    for (int c = 0; c < 16; ++c) a[o + row][o + c] = c <= row ? r[c] : 0.0f;
  }
  __syncwarp();
  float x[16];
#pragma unroll 16
  for (int q = 0; q < 16; ++q) {
    float s = q == row ? 1.0f : 0.0f;
#pragma unroll 16
    for (int m = 0; m < 16; ++m)
      if (m < q) s = fmaf(-a[o + q][o + m], x[m], s);
    x[q] = q >= row ? s / a[o + q][o + q] : 0.0f;
  }
  if (lane < 16) {
#pragma unroll
    for (int q = 0; q < 16; ++q) inv[o + q][o + row] = x[q];
  }
}

// Factors the diagonal block k: L_kk into A, Linv_kk into X's diagonal tile.
// One CTA.  Four 16-wide block columns: a warp factors and inverts the 16 x 16
// diagonal piece, the CTA solves the piece below it and updates the trailing
// part; then the inverse's off-diagonal pieces follow by block forward
// substitution, X_ij = -X_ii sum_{m=j}^{i-1} L_im X_mj.
__device__ void factor_diag(const CholArgs& p, int k, Tile* a, Tile* inv, Tile* t) {
  const int k0 = k * kT;
  const int kb = min(kT, p.n - k0);
  {
    float v[kPerThread];
#pragma unroll
    for (int q = 0; q < kPerThread; ++q) {
      const int e = threadIdx.x + q * kCholThreads, r = e / kT, c = e % kT;
      v[q] = (r < kb && c <= r) ? ld_a(p, k0 + r, k0 + c) : (r == c ? 1.0f : 0.0f);
    }
#pragma unroll
    for (int q = 0; q < kPerThread; ++q) {
      const int e = threadIdx.x + q * kCholThreads, r = e / kT, c = e % kT;
      a[r][c] = v[q];
      inv[r][c] = 0.0f;
    }
  }
  __syncthreads();
  const int warp = threadIdx.x / 32;
  for (int kk = 0; kk < 4; ++kk) {
    const int o = 16 * kk;
    if (warp == 0) warp_chol_inv16(a, inv, o, p.fstatus);
    __syncthreads();
    const int below = kT - o - 16;
    if (below > 0) {
      // L_below = A_below * Linv_oo^T  (below x 16), 3 values per thread at most
      float v[3];
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const int e = threadIdx.x + q * kCholThreads;
        float s = 0.0f;
        if (e < below * 16) {
          const int r = o + 16 + e / 16, c = e % 16;
          for (int d = 0; d <= c; ++d) s = fmaf(a[r][o + d], inv[o + c][o + d], s);
        }
        v[q] = s;
      }
      __syncthreads();
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const int e = threadIdx.x + q * kCholThreads;
        if (e < below * 16) a[o + 16 + e / 16][o + e % 16] = v[q];
      }
      __syncthreads();
      // trailing update of the lower part below the block column
      for (int e = threadIdx.x; e < below * below; e += kCholThreads) {
        const int r = o + 16 + e / below, c = o + 16 + e % below;
        if (c <= r) {
          float s = 0.0f;
#pragma unroll
          for (int d = 0; d < 16; ++d) s = fmaf(a[r][o + d], a[c][o + d], s);
          a[r][c] -= s;
        }
      }
      __syncthreads();
    }
  }
  // off-diagonal pieces of the inverse, block row by block row
  for (int bi = 1; bi < 4; ++bi) {
    const int ri = 16 * bi;
    // t[r][c] = sum_{m=j}^{bi-1} L[ri + r][16 m ..] X[16 m .., c], for c < ri
    for (int e = threadIdx.x; e < 16 * ri; e += kCholThreads) {
      const int r = e / ri, c = e % ri;
      const int j = c / 16;
      float s = 0.0f;
      for (int d = 16 * j; d < ri; ++d) s = fmaf(a[ri + r][d], inv[d][c], s);
      t[r][c] = s;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * ri; e += kCholThreads) {
      const int r = e / ri, c = e % ri;
      float s = 0.0f;
#pragma unroll
      for (int d = 0; d < 16; ++d) s = fmaf(inv[ri + r][ri + d], t[d][c], s);
      inv[ri + r][c] = -s;
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < kT * kT; e += kCholThreads) {
    const int r = e / kT, c = e % kT;
    if (r < kb && c < kb) {
      if (c <= r) *at_a(p, k0 + r, k0 + c) = a[r][c];
      *at_x(p, k0 + r, k0 + c) = inv[r][c];
    }
  }
  __syncthreads();
}

// Time-bounded barrier over the whole (co-resident) grid.
__device__ bool grid_sync(const CholArgs& p) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    volatile unsigned* gen_p = p.bar + 1;
    const unsigned gen = *gen_p;
    __threadfence();
    if (atomicAdd(p.bar, 1u) + 1u == gridDim.x) {
      atomicExch(p.bar, 0u);
      __threadfence();
      atomicAdd(p.bar + 1, 1u);
    } else {
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
    }
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// One tile operation of a phase (see the table at the top of this section).
enum { kOpTrsm = 0, kOpFinalize = 1, kOpUpdate = 2, kOpInverse = 3 };
struct TileOp {
  int kind, i0, j0;
};

__device__ __forceinline__ TileOp op_phase_t(int k, int nb, int t) {
  const int ntrsm = nb - k - 1;
  if (t < ntrsm) return {kOpTrsm, (k + 1 + t) * kT, k * kT};
  return {kOpFinalize, k * kT, (t - ntrsm) * kT};
}

__device__ __forceinline__ TileOp op_phase_u(int k, int nb, int t) {
  const int m = nb - k - 1;
  const int nupd = m * (m + 1) / 2;
  if (t < nupd) {
    int a = static_cast<int>((sqrtf(8.0f * t + 1.0f) - 1.0f) * 0.5f);
    while ((a + 1) * (a + 2) / 2 <= t) ++a;
    while (a * (a + 1) / 2 > t) --a;
    const int b = t - a * (a + 1) / 2;
    return {kOpUpdate, (k + 1 + a) * kT, (k + 1 + b) * kT};
  }
  const int tt = t - nupd;
  return {kOpInverse, (k + 1 + tt / (k + 1)) * kT, (tt % (k + 1)) * kT};
}

// Registers holding one tile operation's operands (and, for the subtracting
// operations, the old output values) between its loads and its use.
struct Staged {
  float p[kPerThread], q[kPerThread], o[kPerThread];
};

__device__ __forceinline__ void fetch_op(const CholArgs& p, const TileOp& op, int k0, Staged& st) {
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
#pragma unroll
  for (int q = 0; q < kPerThread; ++q) {
    const int e = threadIdx.x + q * kCholThreads, a = e / kT, b = e % kT;
    switch (op.kind) {
      case kOpTrsm:      // A_ik * Linv_kk^T
        st.p[q] = ld_a(p, op.i0 + a, k0 + b);
        st.q[q] = ld_x(p, k0 + a, k0 + b);
        break;
      case kOpFinalize:  // Linv_kk * R_kj
        st.p[q] = ld_x(p, k0 + a, k0 + b);
        st.q[q] = ld_x(p, k0 + a, op.j0 + b);
        break;
      case kOpUpdate:    // A_ij - L_ik L_jk^T
        st.p[q] = ld_a(p, op.i0 + a, k0 + b);
        st.q[q] = ld_a(p, op.j0 + a, k0 + b);
        break;
      default:           // R_ij - L_ik X_kj
        st.p[q] = ld_a(p, op.i0 + a, k0 + b);
        st.q[q] = ld_x(p, k0 + a, op.j0 + b);
        break;
    }
  }
  if (op.kind == kOpUpdate || op.kind == kOpInverse) {
    const bool to_x = op.kind == kOpInverse;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        st.o[4 * i + j] = to_x ? ld_x(p, op.i0 + tr + i, op.j0 + tc + j) : ld_a(p, op.i0 + tr + i, op.j0 + tc + j);
  }
}

// P is always used as P[r][k]; Q as Q[c][k] (transposed load) for the
// Cholesky operations and as Q[k][c] (natural load) for the inverse ones.
__device__ __forceinline__ void commit_op(const TileOp& op, const Staged& st, Tile* sp, Tile* sq) {
  const bool q_natural = op.kind == kOpFinalize || op.kind == kOpInverse;
#pragma unroll
  for (int q = 0; q < kPerThread; ++q) {
    const int e = threadIdx.x + q * kCholThreads, a = e / kT, b = e % kT;
    sp[b][a] = st.p[q];
    if (q_natural)
      sq[a][b] = st.q[q];
    else
      sq[b][a] = st.q[q];
  }
}

__device__ __forceinline__ void finish_op(const CholArgs& p, const TileOp& op, int k0, const float (&acc)[4][4],
                                          const float* old) {
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
  const bool to_x = op.kind == kOpFinalize || op.kind == kOpInverse;
  const bool subtract = op.kind == kOpUpdate || op.kind == kOpInverse;
  const int r0 = op.kind == kOpFinalize ? k0 : op.i0;
  const int c0 = op.kind == kOpTrsm ? k0 : op.j0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + tr + i;
    if (r >= p.n) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tc + j;
      if (c >= p.n) continue;
      float* dst = to_x ? at_x(p, r, c) : at_a(p, r, c);
      *dst = subtract ? old[4 * i + j] - acc[i][j] : acc[i][j];
    }
  }
}

// Runs the tile operations t0, t0 + step, ... of one phase.  The operands of
// the next operation are loaded into registers while the current one is
// multiplied, so L2 latency overlaps the FMAs.
template <bool kPhaseU>
__device__ void run_phase(const CholArgs& p, int k, int t0, int step, int total, Tile* s0, Tile* s1, Tile* s2) {
  if (t0 >= total) return;
  const int nb = p.nblk, k0 = k * kT;
  Staged st;
  TileOp cur = kPhaseU ? op_phase_u(k, nb, t0) : op_phase_t(k, nb, t0);
  fetch_op(p, cur, k0, st);
  for (int t = t0; t < total; t += step) {
    commit_op(cur, st, s0, s1);
    // the old output values wait in this thread's own slots of s2
    float* old = &s2[0][0] + threadIdx.x * kPerThread;
#pragma unroll
    for (int q = 0; q < kPerThread; ++q) old[q] = st.o[q];
    __syncthreads();
    const int tn = t + step;
    TileOp nxt = cur;
    if (tn < total) {
      nxt = kPhaseU ? op_phase_u(k, nb, tn) : op_phase_t(k, nb, tn);
      fetch_op(p, nxt, k0, st);
    }
    float acc[4][4];
    tile_product(s0, s1, acc);
    finish_op(p, cur, k0, acc, old);
    __syncthreads();
    cur = nxt;
  }
}

__global__ void __launch_bounds__(kCholThreads, 2) chol_inv_kernel(CholArgs p) {
  extern __shared__ __align__(16) float chol_smem[];
  Tile* s0 = reinterpret_cast<Tile*>(chol_smem);
  Tile* s1 = s0 + kT;
  Tile* s2 = s1 + kT;
  const int nb = p.nblk;
  const int G = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
  if (b == 0) factor_diag(p, 0, s0, s1, s2);
  if (!grid_sync(p)) return;
  for (int k = 0; k < nb; ++k) {
    // phase T(k): trsm of panel k and row k of the inverse
    run_phase<false>(p, k, b, G, nb - 1, s0, s1, s2);
    if (!grid_sync(p)) return;
    // phase U(k): CTA 0 updates tile (k+1, k+1) and then factors it; the
    // other CTAs share the remaining updates, so the factorization is the only
    // extra work on the critical path.  The factorization runs outside the
    // pipelined loop, where no prefetched operands are live.
    const int m = nb - k - 1;
    const int total = m * (m + 1) / 2 + m * (k + 1);
    if (G == 1)
      run_phase<true>(p, k, 0, 1, total, s0, s1, s2);
    else if (b == 0)
      run_phase<true>(p, k, 0, total, total, s0, s1, s2);
    else
      run_phase<true>(p, k, b, G - 1, total, s0, s1, s2);
    if (b == 0 && m > 0) factor_diag(p, k + 1, s0, s1, s2);
    if (!grid_sync(p)) return;
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct PrepLayout {
  size_t a, key, dead, lambda, bar, perm, total;
};

PrepLayout prep_layout(int n) {
  PrepLayout l{};
  const size_t nn = static_cast<size_t>(n) * n;
  size_t off = 0;
  l.a = off;
  off += align256(nn * sizeof(float));
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
  static int blocks_per_sm[64] = {};
  if (blocks_per_sm[info->device] == 0) {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, chol_inv_kernel, kCholThreads, kCholSmem) != cudaSuccess ||
        b < 1)
      return 0;
    blocks_per_sm[info->device] = std::min(b, 2);
  }
  return blocks_per_sm[info->device] * info->sm_count;
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
  float* A = reinterpret_cast<float*>(w + l.a);
  double* key = reinterpret_cast<double*>(w + l.key);
  uint8_t* dead = w + l.dead;
  double* lambda = reinterpret_cast<double*>(w + l.lambda);
  unsigned* bar = reinterpret_cast<unsigned*>(w + l.bar);
  int32_t* perm = perm_out != nullptr ? perm_out : reinterpret_cast<int32_t*>(w + l.perm);
  int* fstatus = info->status + 1;

  static bool attr_set[64] = {};
  if (!attr_set[info->device]) {
    if (cudaFuncSetAttribute(chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  launch(gather_reversed_kernel, dim3(static_cast<unsigned>(ceil_div(n, 256)), n), 256, 0, st, H, perm, dead, lambda,
         n, A);
  if (cudaMemsetAsync(U, 0, static_cast<size_t>(n) * n * sizeof(float), st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;

  CholArgs ca;
  ca.A = A;
  ca.U = U;
  ca.n = n;
  ca.nblk = static_cast<int>(ceil_div(n, kT));
  ca.fstatus = fstatus;
  ca.bar = bar;
  ca.abort = reinterpret_cast<int*>(bar + 2);
  ca.wait_ns = wait_limit_ns();
  void* args[] = {&ca};
  if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(chol_inv_kernel), dim3(grid), dim3(kCholThreads),
                                  args, kCholSmem, st) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  count_launch();

  int fs = 0;
  if (cudaMemcpyAsync(&fs, fstatus, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GPTQ_ERR_CUDA;
  return static_cast<gptq_status>(fs);
}

}  // namespace gptq
