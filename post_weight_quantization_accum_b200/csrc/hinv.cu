// Damping, act-order and the upper inverse factor U with U^T U = (H + lambda I)^-1.
//
// GPTQ knowledge note, "How It Works": a damped Cholesky formulation supplies
// the correction rows; anthology record SOTA-185: the optional reordering
// trick.  Route taken here (one Cholesky, one triangular inverse, no explicit
// inverse of H):
//
//   A = J P^T (H + lambda I) P J          (J = order reversal, P = act-order)
//   A = L L^T,  X = L^-1                  blocked, see below
//   U = J X J                             (a reversal of X's storage)
//
// Below n = 8192 one persistent cooperative kernel factors A and builds X in
// 64-wide panels on the CUDA cores.  From there on the same kernel handles
// each 1024 x 1024 diagonal block, and everything between blocks is a
// tensor-core GEMM with the fp32-accurate 3-term tf32 split (trailing.cu):
// for block K (rows and columns [k0, k1)), R the rows of X still being
// formed,
//   X_K,<K  = X_KK R_K,<K                 finalize block row K of X
//   L_>K,K  = A_>K,K X_KK^T               panel (trsm as a product)
//   A_>K,>K -= L_>K,K L_>K,K^T            trailing update (full square, which
//                                         also keeps the diagonal tiles' upper
//                                         halves the factorization reads)
//   R_>K,<=K -= L_>K,K X_K,<=K            inverse update
// so the O(n^3) work runs at tensor-core rate and only the 1024-wide diagonal
// blocks go through the latency-bound panel sweep.
//
// With H' = P^T (H + lambda I) P, J H' J = L L^T gives H' = (J L J)(J L J)^T
// with J L J upper triangular, so U = (J L J)^-1 = J L^-1 J is upper with
// U^T U = H'^-1: it is the upper Cholesky factor of the inverse.
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

constexpr int kT = 64;  // tile width = panel width of the factorization below

// Lower triangle of A = J P^T (H + lambda I) P J; dead diagonals become 1 + lambda.
// Inside the kT x kT diagonal blocks the upper half is written too, as the
// mirror of the lower one (the diagonal factorization reads whole blocks).
__global__ void gather_reversed_kernel(const float* __restrict__ H, const int32_t* __restrict__ perm,
                                       const uint8_t* __restrict__ dead, const double* __restrict__ lambda, int n,
                                       float* __restrict__ A) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  const int a = blockIdx.y;
  if (a >= n || b >= n) return;
  if (b > a && b / kT != a / kT) return;
  const int lo = b > a ? a : b, hi = b > a ? b : a;  // the lower-triangle entry (hi, lo) holds the value
  const int ph = perm[n - 1 - hi], pl = perm[n - 1 - lo];
  float v;
  if (a == b) {
    const double base = dead[ph] ? 1.0 : static_cast<double>(H[static_cast<size_t>(ph) * n + ph]);
    v = static_cast<float>(base + *lambda);
  } else {
    v = H[static_cast<size_t>(ph) * n + pl];
  }
  A[static_cast<size_t>(a) * n + b] = v;
}

// U = J X J for X stored row-major in U's own memory: U[a][b] = X[n-1-a][n-1-b]
// is the reversal of the flat array (element e <-> n*n - 1 - e).
__global__ void reverse_kernel(float* __restrict__ U, int64_t count) {
  const int64_t half = count / 2;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < half;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float a = U[e], b = U[count - 1 - e];
    U[e] = b;
    U[count - 1 - e] = a;
  }
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
// of tiles.  Two grid barriers per panel (time-bounded).  The kernel works on
// one diagonal block of order <= 1024 at any row pitch; R's tiles live in X's
// places before they are finalized.

constexpr int kPad = 68;           // shared-memory row stride (16-byte aligned rows)
constexpr int kCholThreads = 256;
constexpr int kMaxCholCtas = 4096;  // bound on the cooperative grid (SM ids recorded per CTA)
constexpr size_t kCholSmem = 3 * kT * kPad * sizeof(float);

struct CholArgs {
  float* A;          // block [n, n] at row pitch lda, lower: the damped reversed matrix, becomes L
  float* X;          // block [n, n] at row pitch ldx, zero on entry: X = L^-1 is written here
  int64_t lda, ldx;
  int n;             // order of the block
  int nblk;
  int* fstatus;      // factorization status word
  unsigned* bar;     // grid barrier: [0] arrivals, [1] generation (zeroed on entry)
  int* abort;        // set when a barrier wait runs out (zeroed on entry)
  uint64_t wait_ns;
  int vec;           // rows of four along a tile row are 16-byte aligned (lda, ldx, bases)
  unsigned* smids;   // [gridDim.x] SM of each CTA
};

typedef float Tile[kPad];

__device__ __forceinline__ float ld_a(const CholArgs& p, int r, int c) {
  return (r < p.n && c < p.n) ? __ldcg(p.A + r * p.lda + c) : 0.0f;
}
__device__ __forceinline__ float* at_a(const CholArgs& p, int r, int c) { return p.A + r * p.lda + c; }
__device__ __forceinline__ float* at_x(const CholArgs& p, int r, int c) { return p.X + r * p.ldx + c; }

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

// Factors the diagonal block k: L_kk into A, Linv_kk into X's diagonal tile.
//
// A right-looking sweep over the block's 64 pivots by the whole CTA, with the
// inverse built in the same sweep (R = I; at pivot j, X_j = R_j / L_jj and
// R_i -= L_ij X_j for i > j).  Thread t holds row i = t / 4, columns
// 16 (t % 4) .. 16 (t % 4) + 15 of the block in registers: left of the pivot
// those are R's entries, right of it the remaining matrix, upper half
// included.  The upper half makes row j carry, by symmetry, the column under
// the pivot too, so one broadcast per pivot suffices: the four threads of row
// j + 1 store their registers to shared memory (R_{j+1,<j+1}, the next pivot,
// and A_{j+1,>j+1}), one barrier, and every thread reads the pivot, its own
// row's multiplier and its sixteen columns from there.  With s_i = A_ij / d_j
// (d_j the pivot), every update is v -= s_i * row_j[c]: the Schur update
// A_ic -= L_ij L_cj on the right of the pivot and R_ic -= L_ij X_jc on its
// left; the pivot column itself becomes R_ij = -s_i.  X's rows are scaled by
// 1 / L_ii at the end.  A pivot that is not positive or not finite sets the
// status word (a non-finite one takes precedence) and is replaced by 1.
__device__ void factor_diag(const CholArgs& p, int k, Tile* lout, Tile* xout, Tile* bt) {
  const int k0 = k * kT;
  const int kb = min(kT, p.n - k0);
  const int t = threadIdx.x, i = t >> 2, q = t & 3;
  float* bbuf = &bt[0][0];  // two 64-float broadcast rows (pivot parity)
  float v[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int c = 16 * q + m;
    v[m] = (i < kb && c < kb) ? ld_a(p, k0 + i, k0 + c) : (i == c ? 1.0f : 0.0f);
  }
  if (i == 0) {
    float4* d4 = reinterpret_cast<float4*>(bbuf + 16 * q);
#pragma unroll
    for (int g = 0; g < 4; ++g) d4[g] = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
  }
  __syncthreads();
  float myrd = 1.0f;
  bool notpd = false, nonfinite = false;
#pragma unroll 1
  for (int j0 = 0; j0 < kT; j0 += 16) {
    // sixteen pivots per iteration, unrolled so that register indices are constants
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const int j = j0 + jj;
      const float* B = bbuf + (j & 1) * kT;
      float* Bn = bbuf + ((j + 1) & 1) * kT;
      float d = B[j];
      const float bi = B[i];
      float bc[16];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float4 w = *reinterpret_cast<const float4*>(B + 16 * q + 4 * g);
        bc[4 * g] = w.x;
        bc[4 * g + 1] = w.y;
        bc[4 * g + 2] = w.z;
        bc[4 * g + 3] = w.w;
      }
      nonfinite |= !isfinite(d);
      notpd |= !(d > 0.0f);
      d = (d > 0.0f && d < INFINITY) ? d : 1.0f;
      const float rd = rsqrtf(d);
      const float s = bi * rd * rd;
      if (i > j) {
#pragma unroll
        for (int m = 0; m < 16; ++m) v[m] = fmaf(-s, bc[m], v[m]);
        if (q == (j0 >> 4)) v[jj] = -s;
      }
      myrd = i == j ? rd : myrd;
      if (q == 0 && i >= j) lout[i][j] = (i == j ? d : bi) * rd;
      if (i == j + 1) {
        float4* d4 = reinterpret_cast<float4*>(Bn + 16 * q);
#pragma unroll
        for (int g = 0; g < 4; ++g) d4[g] = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
      }
      __syncthreads();
    }
  }
  if (t == 0 && (nonfinite || notpd)) set_status(p.fstatus, nonfinite ? GPTQ_ERR_NONFINITE : GPTQ_ERR_NOT_PD);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int c = 16 * q + m;
    xout[i][c] = c < i ? v[m] * myrd : (c == i ? myrd : 0.0f);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kT * kT; e += kCholThreads) {
    const int r = e / kT, c = e % kT;
    if (r < kb && c < kb) {
      if (c <= r) *at_a(p, k0 + r, k0 + c) = lout[r][c];
      *at_x(p, k0 + r, k0 + c) = xout[r][c];
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

// Four consecutive entries (r, c .. c + 3) of A or of X; c % 4 == 0.  Vector
// loads when p.vec.
__device__ __forceinline__ float4 ld4(const CholArgs& p, bool from_x, int r, int c) {
  if (r >= p.n || c >= p.n) return make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  const float* src = from_x ? at_x(p, r, c) : at_a(p, r, c);
  if (p.vec) return __ldcg(reinterpret_cast<const float4*>(src));
  return make_float4(__ldcg(src), c + 1 < p.n ? __ldcg(src + 1) : 0.0f, c + 2 < p.n ? __ldcg(src + 2) : 0.0f,
                     c + 3 < p.n ? __ldcg(src + 3) : 0.0f);
}
__device__ __forceinline__ float4 ld4_a(const CholArgs& p, int r, int c) { return ld4(p, false, r, c); }
__device__ __forceinline__ float4 ld4_x(const CholArgs& p, int r, int c) { return ld4(p, true, r, c); }

__device__ __forceinline__ void st4(const CholArgs& p, bool to_x, int r, int c, float4 v) {
  if (r >= p.n || c >= p.n) return;
  float* dst = to_x ? at_x(p, r, c) : at_a(p, r, c);
  if (p.vec) {
    *reinterpret_cast<float4*>(dst) = v;
  } else {
    dst[0] = v.x;
    if (c + 1 < p.n) dst[1] = v.y;
    if (c + 2 < p.n) dst[2] = v.z;
    if (c + 3 < p.n) dst[3] = v.w;
  }
}

// Adds v to four consecutive entries (r, c .. c + 3) of A or X in memory (a
// reduction performed in L2: no read into the SM, nothing to wait for).
// Each entry receives one such addition per phase, so the result is that of
// a load, an fp32 addition and a store.
__device__ __forceinline__ void red4(const CholArgs& p, bool to_x, int r, int c, float4 v) {
  if (r >= p.n || c >= p.n) return;
  float* dst = to_x ? at_x(p, r, c) : at_a(p, r, c);
  if (p.vec) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
  } else {
    atomicAdd(dst, v.x);
    if (c + 1 < p.n) atomicAdd(dst + 1, v.y);
    if (c + 2 < p.n) atomicAdd(dst + 2, v.z);
    if (c + 3 < p.n) atomicAdd(dst + 3, v.w);
  }
}

// Which four entries (row a, columns 4 b4 .. 4 b4 + 3) of a 64 x 64 operand
// thread t stages in its slot g.  An operand that shared memory keeps
// transposed uses mapping T: two lanes per row (one 32-byte sector per row and
// instruction), so that the transposed scalar stores of a warp hit 32
// distinct banks.  One kept as loaded uses mapping N: 16 lanes along a row,
// conflict-free vector stores.
__device__ __forceinline__ void slot_t(int g, int& a, int& b4) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  a = (lane >> 1) + 16 * (warp & 3);
  b4 = (lane & 1) + 2 * ((warp >> 2) + 2 * g);
}
__device__ __forceinline__ void slot_n(int g, int& a, int& b4) {
  const int idx = g * kCholThreads + threadIdx.x;
  a = idx >> 4;
  b4 = idx & 15;
}

// Registers holding one tile operation's operands between their loads and
// their use.
struct Staged {
  float4 p[4], q[4];
};

__device__ __forceinline__ bool q_natural(const TileOp& op) { return op.kind == kOpFinalize || op.kind == kOpInverse; }

// The first operand of an operation: A_ik / L_ik (row block i of panel k) for
// trsm, update and inverse, Linv_kk for finalize.  Consecutive operations
// with the same key share it, so it is loaded and staged once.
__device__ __forceinline__ int p_key(const TileOp& op) { return op.kind == kOpFinalize ? -2 : op.i0; }

__device__ __forceinline__ void fetch_op(const CholArgs& p, const TileOp& op, int k0, Staged& st, bool need_p) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    int a, b4, an, bn4;
    slot_t(g, a, b4);
    slot_n(g, an, bn4);
    const int b = 4 * b4;
    if (!need_p) {  // the second operand only (as in the cases below)
      switch (op.kind) {
        case kOpTrsm:
          st.q[g] = ld4_x(p, k0 + a, k0 + b);
          break;
        case kOpUpdate:
          st.q[g] = ld4_a(p, op.j0 + a, k0 + b);
          break;
        default:
          st.q[g] = ld4_x(p, k0 + an, op.j0 + 4 * bn4);
          break;
      }
      continue;
    }
    switch (op.kind) {
      case kOpTrsm:      // A_ik * Linv_kk^T
        st.p[g] = ld4_a(p, op.i0 + a, k0 + b);
        st.q[g] = ld4_x(p, k0 + a, k0 + b);
        break;
      case kOpFinalize:  // Linv_kk * R_kj
        st.p[g] = ld4_x(p, k0 + a, k0 + b);
        st.q[g] = ld4_x(p, k0 + an, op.j0 + 4 * bn4);
        break;
      case kOpUpdate:    // A_ij - L_ik L_jk^T
        st.p[g] = ld4_a(p, op.i0 + a, k0 + b);
        st.q[g] = ld4_a(p, op.j0 + a, k0 + b);
        break;
      default:           // R_ij - L_ik X_kj
        st.p[g] = ld4_a(p, op.i0 + a, k0 + b);
        st.q[g] = ld4_x(p, k0 + an, op.j0 + 4 * bn4);
        break;
    }
  }
}

// P is always used as P[r][k]; Q as Q[c][k] (transposed load) for the
// Cholesky operations and as Q[k][c] (natural load) for the inverse ones.
__device__ __forceinline__ void commit_op(const TileOp& op, const Staged& st, Tile* sp, Tile* sq, bool write_p) {
  const bool qn = q_natural(op);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    int a, b4;
    slot_t(g, a, b4);
    const int b = 4 * b4;
    if (write_p) {
      sp[b + 0][a] = st.p[g].x;
      sp[b + 1][a] = st.p[g].y;
      sp[b + 2][a] = st.p[g].z;
      sp[b + 3][a] = st.p[g].w;
    }
    if (qn) {
      int an, bn4;
      slot_n(g, an, bn4);
      *reinterpret_cast<float4*>(&sq[an][4 * bn4]) = st.q[g];
    } else {
      sq[b + 0][a] = st.q[g].x;
      sq[b + 1][a] = st.q[g].y;
      sq[b + 2][a] = st.q[g].z;
      sq[b + 3][a] = st.q[g].w;
    }
  }
}

// Writes the product (trsm, finalize) or subtracts it in place (update,
// inverse: an L2 reduction, so the old values never travel to the SM).
__device__ __forceinline__ void finish_op(const CholArgs& p, const TileOp& op, int k0, const float (&acc)[4][4]) {
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
  const bool to_x = op.kind == kOpFinalize || op.kind == kOpInverse;
  const bool subtract = op.kind == kOpUpdate || op.kind == kOpInverse;
  const int r0 = op.kind == kOpFinalize ? k0 : op.i0;
  const int c0 = op.kind == kOpTrsm ? k0 : op.j0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (subtract)
      red4(p, to_x, r0 + tr + i, c0 + tc, make_float4(-acc[i][0], -acc[i][1], -acc[i][2], -acc[i][3]));
    else
      st4(p, to_x, r0 + tr + i, c0 + tc, make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]));
  }
}

// Runs the tile operations [lo, hi) of one phase.  Operations are numbered
// row block by row block, so consecutive ones mostly share their first
// operand, which then stays in shared memory.  The operands of the next
// operation are loaded into registers while the current one is multiplied,
// so L2 latency overlaps the FMAs.
template <bool kPhaseU>
__device__ void run_phase(const CholArgs& p, int k, int lo, int hi, Tile* s0, Tile* s1) {
  if (lo >= hi) return;
  const int nb = p.nblk, k0 = k * kT;
  Staged st;
  TileOp cur = kPhaseU ? op_phase_u(k, nb, lo) : op_phase_t(k, nb, lo);
  fetch_op(p, cur, k0, st, true);
  bool write_p = true;
  for (int t = lo; t < hi; ++t) {
    commit_op(cur, st, s0, s1, write_p);
    __syncthreads();
    TileOp nxt = cur;
    bool next_p = false;
    if (t + 1 < hi) {
      nxt = kPhaseU ? op_phase_u(k, nb, t + 1) : op_phase_t(k, nb, t + 1);
      next_p = p_key(nxt) != p_key(cur);
      fetch_op(p, nxt, k0, st, next_p);
    }
    float acc[4][4];
    tile_product(s0, s1, acc);
    finish_op(p, cur, k0, acc);
    __syncthreads();
    cur = nxt;
    write_p = next_p;
  }
  __threadfence();  // this CTA's reductions are performed before its later reads
  __syncthreads();
}

// [lo, hi) of `total` operations for worker w of `workers` (contiguous, equal shares)
__device__ __forceinline__ void share(int total, int w, int workers, int& lo, int& hi) {
  lo = static_cast<int>((static_cast<int64_t>(total) * w) / workers);
  hi = static_cast<int>((static_cast<int64_t>(total) * (w + 1)) / workers);
}

__device__ __forceinline__ unsigned sm_id() {
  unsigned r;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
  return r;
}

__global__ void __launch_bounds__(kCholThreads, 2) chol_inv_kernel(CholArgs p) {
  extern __shared__ __align__(16) float chol_smem[];
  __shared__ int sib_s;
  Tile* s0 = reinterpret_cast<Tile*>(chol_smem);
  Tile* s1 = s0 + kT;
  Tile* s2 = s1 + kT;
  const int nb = p.nblk;
  const int G = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
  // Every CTA records its SM; the CTA that shares CTA 0's SM (if any) takes no
  // tile operations, so the diagonal factorizations (the kernel's critical
  // path, run by CTA 0) have their SM to themselves.
  if (threadIdx.x == 0) p.smids[b] = sm_id();
  if (threadIdx.x == 0) sib_s = -1;
  if (b == 0) factor_diag(p, 0, s0, s1, s2);
  if (!grid_sync(p)) return;
  {
    const unsigned sm0 = __ldcg(p.smids);
    for (int c = 1 + threadIdx.x; c < G; c += blockDim.x)
      if (__ldcg(p.smids + c) == sm0) atomicMax(&sib_s, c);
    __syncthreads();
  }
  const int sib = sib_s;
  const bool idle = (b == sib);
  const int pidx = b - ((sib >= 0 && b > sib) ? 1 : 0);  // index among the CTAs that work
  const int PT = G - (sib >= 0 ? 1 : 0);
  const int W = PT - 1;                                    // workers besides CTA 0
  for (int k = 0; k < nb; ++k) {
    // phase T(k): trsm of panel k and row k of the inverse
    if (!idle) {
      int lo, hi;
      share(nb - 1, pidx, PT, lo, hi);
      run_phase<false>(p, k, lo, hi, s0, s1);
    }
    if (!grid_sync(p)) return;
    // phase U(k): CTA 0 updates tile (k+1, k+1) and then factors it; the
    // other CTAs share the remaining updates, so the factorization is the only
    // extra work on the critical path.  The factorization runs outside the
    // pipelined loop, where no prefetched operands are live.
    const int m = nb - k - 1;
    const int total = m * (m + 1) / 2 + m * (k + 1);
    if (W == 0) {
      if (b == 0) run_phase<true>(p, k, 0, total, s0, s1);
    } else if (b == 0) {
      run_phase<true>(p, k, 0, total > 0 ? 1 : 0, s0, s1);
    } else if (!idle && total > 1) {
      int lo, hi;
      share(total - 1, pidx - 1, W, lo, hi);
      run_phase<true>(p, k, 1 + lo, 1 + hi, s0, s1);
    }
    if (b == 0 && m > 0) factor_diag(p, k + 1, s0, s1, s2);
    if (!grid_sync(p)) return;
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kNB = 1024;  // diagonal block of the blocked factorization
// From this order on, 1024-wide blocks joined by tensor-core GEMMs.  Below it
// the single cooperative kernel is faster (2.9 vs 4.4 ms at 4096: the blocked
// form runs the same 64-wide panel chain plus the GEMM launches) and more
// accurate (U^T U H' v = v to ~7e-7 vs ~4e-6: the tensor-core accumulation
// of each 128-long K chunk rounds like truncation).  At 8192 the two take the
// same time; at 11008 the blocked form is 1.15x faster, and its advantage
// grows with n (its O(n^3) part runs on the tensor cores).
constexpr int kBlockedMinN = 8192;

struct PrepLayout {
  size_t a, key, dead, lambda, bar, perm, ahi, alo, bhi, blo, panel, total;
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
  l.bar = off;  // barrier words and the abort flag, then one SM id per CTA
  off += 256 + align256(kMaxCholCtas * sizeof(unsigned));
  l.perm = off;
  off += align256(static_cast<size_t>(n) * sizeof(int32_t));
  // blocked factorization (n > kNB): tf32 halves of the GEMM operands and the
  // panel L_>K,K, each at most n x kNB
  const size_t blk = n >= kBlockedMinN ? align256(static_cast<size_t>(n) * kNB * sizeof(float)) : 0;
  l.ahi = off;
  off += blk;
  l.alo = off;
  off += blk;
  l.bhi = off;
  off += blk;
  l.blo = off;
  off += blk;
  l.panel = off;
  off += blk;
  l.total = off;
  return l;
}

int chol_grid(const DeviceInfo* info) {
  static std::atomic<int> blocks_per_sm[64] = {};  // per device, shared by host threads
  if (blocks_per_sm[info->device] == 0) {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, chol_inv_kernel, kCholThreads, kCholSmem) != cudaSuccess ||
        b < 1)
      return 0;
    blocks_per_sm[info->device] = std::min(b, 2);
  }
  return std::min(kMaxCholCtas, blocks_per_sm[info->device] * info->sm_count);
}

}  // namespace

size_t prepare_workspace_size(int n) { return n > 0 ? prep_layout(n).total : 0; }

gptq_status split_rows_tf32(const float* src, int64_t lds, int rows, int cols, int kpad, float sign, float* hi,
                            float* lo, cudaStream_t st);
gptq_status split_cols_tf32(const float* src, int64_t lds, int rows, int cols, int kpad, float sign, float* hi,
                            float* lo, cudaStream_t st);
gptq_status gemm_nt_tc(float* C, int64_t ldc, int M, int N, int kpad, const float* A_hi, const float* A_lo,
                       const float* B_hi, const float* B_lo, cudaStream_t st);

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

  static std::atomic<bool> attr_set[64] = {};  // per device, shared by host threads
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

  // The diagonal block [k0, k0 + kb) through the cooperative kernel; X = U
  // (unrotated until the end).
  auto factor_block = [&](int k0, int kb) -> gptq_status {
    if (cudaMemsetAsync(bar, 0, 256, st) != cudaSuccess) return GPTQ_ERR_CUDA;
    CholArgs ca;
    ca.A = A + static_cast<int64_t>(k0) * n + k0;
    ca.X = U + static_cast<int64_t>(k0) * n + k0;
    ca.lda = n;
    ca.ldx = n;
    ca.n = kb;
    ca.nblk = static_cast<int>(ceil_div(kb, kT));
    ca.fstatus = fstatus;
    ca.bar = bar;
    ca.abort = reinterpret_cast<int*>(bar + 2);
    ca.smids = bar + 64;
    ca.wait_ns = wait_limit_ns();
    ca.vec = (n % 4 == 0) ? 1 : 0;
    void* args[] = {&ca};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(chol_inv_kernel), dim3(grid), dim3(kCholThreads),
                                    args, kCholSmem, st) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    count_launch();
    return GPTQ_OK;
  };
  float* Ahi = reinterpret_cast<float*>(w + l.ahi);
  float* Alo = reinterpret_cast<float*>(w + l.alo);
  float* Bhi = reinterpret_cast<float*>(w + l.bhi);
  float* Blo = reinterpret_cast<float*>(w + l.blo);
  float* P = reinterpret_cast<float*>(w + l.panel);
  const int nb_outer = n >= kBlockedMinN ? kNB : n;  // one block: the cooperative kernel alone
  for (int k0 = 0; k0 < n; k0 += nb_outer) {
    const int kb = std::min(nb_outer, n - k0), k1 = k0 + kb, m = n - k1;
    const int kp = static_cast<int>(ceil_div(kb, 32)) * 32;  // padded contraction length
    float* XK = U + static_cast<int64_t>(k0) * n;             // block row K of X (and of R)
    float* XKK = XK + k0;
    gptq_status s = factor_block(k0, kb);
    if (s != GPTQ_OK) return s;
    if (k0 > 0) {
      // finalize: X_K,<K = X_KK R_K,<K  (R_K,<K split, then its place zeroed)
      if ((s = split_cols_tf32(XK, n, kb, k0, kp, 1.0f, Bhi, Blo, st)) != GPTQ_OK) return s;
      if (cudaMemset2DAsync(XK, static_cast<size_t>(n) * 4, 0, static_cast<size_t>(k0) * 4, kb, st) != cudaSuccess)
        return GPTQ_ERR_CUDA;
      if ((s = split_rows_tf32(XKK, n, kb, kb, kp, -1.0f, Ahi, Alo, st)) != GPTQ_OK) return s;
      if ((s = gemm_nt_tc(XK, n, kb, k0, kp, Ahi, Alo, Bhi, Blo, st)) != GPTQ_OK) return s;
    }
    if (m == 0) break;
    // panel: L_>K,K = A_>K,K X_KK^T into P [m, kp]
    float* AIK = A + static_cast<int64_t>(k1) * n + k0;
    if ((s = split_rows_tf32(AIK, n, m, kb, kp, -1.0f, Ahi, Alo, st)) != GPTQ_OK) return s;
    if ((s = split_rows_tf32(XKK, n, kb, kb, kp, 1.0f, Bhi, Blo, st)) != GPTQ_OK) return s;
    if (cudaMemsetAsync(P, 0, static_cast<size_t>(m) * kp * sizeof(float), st) != cudaSuccess) return GPTQ_ERR_CUDA;
    if ((s = gemm_nt_tc(P, kp, m, kb, kp, Ahi, Alo, Bhi, Blo, st)) != GPTQ_OK) return s;
    // trailing update: A_>K,>K -= P P^T
    if ((s = split_rows_tf32(P, kp, m, kb, kp, 1.0f, Ahi, Alo, st)) != GPTQ_OK) return s;
    if ((s = gemm_nt_tc(A + static_cast<int64_t>(k1) * n + k1, n, m, m, kp, Ahi, Alo, Ahi, Alo, st)) != GPTQ_OK)
      return s;
    // inverse update: R_>K,<=K -= P X_K,<=K
    if ((s = split_cols_tf32(XK, n, kb, k1, kp, 1.0f, Bhi, Blo, st)) != GPTQ_OK) return s;
    if ((s = gemm_nt_tc(U + static_cast<int64_t>(k1) * n, n, m, k1, kp, Ahi, Alo, Bhi, Blo, st)) != GPTQ_OK)
      return s;
  }
  {
    const int64_t count = static_cast<int64_t>(n) * n;
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(ceil_div(count / 2, 256), 148 * 16));
    launch(reverse_kernel, static_cast<unsigned>(blocks), 256, 0, st, U, count);
    if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
  }

  int fs = 0;
  if (cudaMemcpyAsync(&fs, fstatus, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GPTQ_ERR_CUDA;
  return static_cast<gptq_status>(fs);
}

}  // namespace gptq
