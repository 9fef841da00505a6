// Damping, act-order and the upper inverse factor U with U^T U = (H + lambda I)^-1.
//
// GPTQ knowledge note, "How It Works": a damped Cholesky formulation supplies
// the correction rows; anthology record SOTA-185: the optional reordering
// trick.  Route taken here (one Cholesky, one triangular inverse, no explicit
// inverse of H):
//
//   A = J P^T (H + lambda I) P J          (J = order reversal, P = act-order)
//   A = L L^T                             blocked right-looking Cholesky, 64-wide
//   B = L^-1                              recursive doubling over diagonal blocks
//   U = J B J                             180-degree rotation of B
//
// With H' = P^T (H + lambda I) P, J H' J = L L^T gives H' = (J L J)(J L J)^T
// with J L J upper triangular, so U = (J L J)^-1 = J L^-1 J is upper with
// U^T U = H'^-1: it is the upper Cholesky factor of the inverse.
#include <algorithm>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int kNB = 64;  // panel / tile width of the factorization kernels

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
// blocked Cholesky of A (lower, in place)
// --------------------------------------------------------------------------

// Factors the kb x kb diagonal block at k0 (kb <= 64) and writes its inverse
// into the same block of Binv.  One CTA of 64 threads; thread i owns row i.
__global__ void __launch_bounds__(kNB) potrf_diag_kernel(float* __restrict__ A, float* __restrict__ Binv, int n,
                                                         int k0, int* fstatus) {
  __shared__ float a[kNB][kNB + 1];
  __shared__ float inv[kNB][kNB + 1];
  __shared__ float col[kNB];
  __shared__ int bad;
  const int kb = min(kNB, n - k0);
  const int i = threadIdx.x;
  if (i == 0) bad = 0;
  for (int r = 0; r < kb; ++r)
    if (i < kb) a[r][i] = (i <= r) ? A[static_cast<size_t>(k0 + r) * n + k0 + i] : 0.0f;
  __syncthreads();
  for (int j = 0; j < kb; ++j) {
    const float piv = a[j][j];
    if (!(piv > 0.0f) || !isfinite(piv)) {
      if (i == 0 && !bad) {
        bad = 1;
        set_status(fstatus, isfinite(piv) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE);
      }
    }
    const float d = sqrtf(fmaxf(piv, 0.0f));
    const float rd = d > 0.0f ? 1.0f / d : 0.0f;
    if (i < kb && i >= j) col[i] = (i == j) ? d : a[i][j] * rd;
    __syncthreads();
    if (i < kb && i >= j) a[i][j] = col[i];
    if (i < kb && i > j) {
      const float lij = col[i];
      for (int k = j + 1; k <= i; ++k) a[i][k] -= lij * col[k];
    }
    __syncthreads();
  }
  for (int r = 0; r < kb; ++r)
    if (i < kb && i <= r) A[static_cast<size_t>(k0 + r) * n + k0 + i] = a[r][i];
  // inverse of the lower factor: thread i solves L x = e_i (forward
  // substitution); x lives in column i of `inv`, which only thread i touches.
  __syncthreads();
  if (i < kb) {
    for (int r = 0; r < kb; ++r) {
      float x = 0.0f;
      if (r >= i) {
        float s = (r == i) ? 1.0f : 0.0f;
        for (int k = i; k < r; ++k) s -= a[r][k] * inv[k][i];
        x = s / a[r][r];
      }
      inv[r][i] = x;
      Binv[static_cast<size_t>(k0 + r) * n + k0 + i] = x;
    }
  }
}

// L21 = A21 * inv(L11)^T for the rows below the diagonal block (64 rows per CTA).
__global__ void __launch_bounds__(256) trsm_panel_kernel(float* __restrict__ A, const float* __restrict__ Binv,
                                                         int n, int k0) {
  __shared__ float a[kNB][kNB + 1];
  __shared__ float li[kNB][kNB + 1];
  const int kb = min(kNB, n - k0);
  const int r0 = k0 + kb + blockIdx.x * kNB;
  const int rows = min(kNB, n - r0);
  for (int e = threadIdx.x; e < kNB * kNB; e += blockDim.x) {
    const int r = e / kNB, c = e % kNB;
    a[r][c] = (r < rows && c < kb) ? A[static_cast<size_t>(r0 + r) * n + k0 + c] : 0.0f;
    li[r][c] = (r < kb && c < kb) ? Binv[static_cast<size_t>(k0 + r) * n + k0 + c] : 0.0f;
  }
  __syncthreads();
  // out[r][c] = sum_{d <= c} a[r][d] * li[c][d]
  for (int e = threadIdx.x; e < kNB * kNB; e += blockDim.x) {
    const int r = e / kNB, c = e % kNB;
    if (r >= rows || c >= kb) continue;
    float s = 0.0f;
    for (int d = 0; d <= c; ++d) s = fmaf(a[r][d], li[c][d], s);
    A[static_cast<size_t>(r0 + r) * n + k0 + c] = s;
  }
}

// Trailing update of the lower triangle: A22 -= L21 L21^T, 64x64 tiles, one
// CTA per lower tile (ti >= tj), 256 threads x (4 x 4) outputs.
__global__ void __launch_bounds__(256) syrk_update_kernel(float* __restrict__ A, int n, int k0) {
  const int kb = min(kNB, n - k0);
  const int base = k0 + kb;
  // blockIdx.x enumerates lower tiles row by row: ti*(ti+1)/2 + tj
  const int t = blockIdx.x;
  int ti = static_cast<int>((sqrtf(8.0f * t + 1.0f) - 1.0f) * 0.5f);
  while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
  while (ti * (ti + 1) / 2 > t) --ti;
  const int tj = t - ti * (ti + 1) / 2;
  const int r0 = base + ti * kNB, c0 = base + tj * kNB;
  __shared__ float li[kNB][kNB + 4];  // L21 rows of the tile row, [k][row]
  __shared__ float lj[kNB][kNB + 4];  // L21 rows of the tile column, [k][col]
  for (int e = threadIdx.x; e < kNB * kNB; e += blockDim.x) {
    const int r = e / kNB, k = e % kNB;
    li[k][r] = (r0 + r < n && k < kb) ? A[static_cast<size_t>(r0 + r) * n + k0 + k] : 0.0f;
    lj[k][r] = (c0 + r < n && k < kb) ? A[static_cast<size_t>(c0 + r) * n + k0 + k] : 0.0f;
  }
  __syncthreads();
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
  float acc[4][4] = {};
  for (int k = 0; k < kb; ++k) {
    float x[4], y[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      x[u] = li[k][tr + u];
      y[u] = lj[k][tc + u];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(x[u], y[v], acc[u][v]);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = r0 + tr + u;
    if (r >= n) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int c = c0 + tc + v;
      if (c < n && c <= r) A[static_cast<size_t>(r) * n + c] -= acc[u][v];
    }
  }
}

// --------------------------------------------------------------------------
// triangular inverse by recursive doubling
// --------------------------------------------------------------------------
//
// With the inverses of the diagonal blocks of size s known (in Binv), the
// inverse of the 2s block [[P, 0], [Q, R]] has lower-left block
// -R^-1 Q P^-1.  Level s computes, for every pair of blocks at once,
//   T = Q * P^-1          (tri_gemm_right_lower)
//   X = -R^-1 * T         (tri_gemm_left_lower)

// T[p] = Q[p] * Pinv[p]; Q[p] = L[b+s : b+s+m, b : b+s], Pinv lower s x s.
// Grid (s/64 col tiles, s/64 row tiles, pairs), 256 threads, 64x64 outputs.
__global__ void __launch_bounds__(256) tri_gemm_right_lower_kernel(const float* __restrict__ L,
                                                                   const float* __restrict__ Binv, int n, int s,
                                                                   float* __restrict__ T) {
  const int p = blockIdx.z;
  const int b = p * 2 * s;
  const int m = min(s, n - b - s);  // rows of Q (the second block may be short)
  if (m <= 0) return;
  const int tr0 = blockIdx.y * kNB, tc0 = blockIdx.x * kNB;
  if (tr0 >= m) return;
  __shared__ float qa[32][kNB + 4];  // [k][row]
  __shared__ float pb[32][kNB + 4];  // [k][col]
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
  float acc[4][4] = {};
  // Pinv[k][c] is zero for k < c: the K range starts at the column tile.
  for (int k0 = tc0; k0 < s; k0 += 32) {
    for (int e = threadIdx.x; e < 32 * kNB; e += blockDim.x) {
      const int r = e / 32, k = e % 32;
      const int gr = b + s + tr0 + r;
      qa[k][r] = (tr0 + r < m) ? L[static_cast<size_t>(gr) * n + b + k0 + k] : 0.0f;
      const int kk = e / kNB, c = e % kNB;
      pb[kk][c] = Binv[static_cast<size_t>(b + k0 + kk) * n + b + tc0 + c];
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      float x[4], y[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        x[u] = qa[k][tr + u];
        y[u] = pb[k][tc + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(x[u], y[v], acc[u][v]);
    }
    __syncthreads();
  }
  float* Tp = T + static_cast<size_t>(p) * s * s;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = tr0 + tr + u;
    if (r >= m) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) Tp[static_cast<size_t>(r) * s + tc0 + tc + v] = acc[u][v];
  }
}

// X = -Rinv * T[p], Rinv = Binv[b+s : b+s+m, b+s : b+s+m] lower; writes X into
// Binv[b+s : b+s+m, b : b+s].
__global__ void __launch_bounds__(256) tri_gemm_left_lower_kernel(float* __restrict__ Binv, const float* __restrict__ T,
                                                                  int n, int s) {
  const int p = blockIdx.z;
  const int b = p * 2 * s;
  const int m = min(s, n - b - s);
  if (m <= 0) return;
  const int tr0 = blockIdx.y * kNB, tc0 = blockIdx.x * kNB;
  if (tr0 >= m) return;
  const float* Tp = T + static_cast<size_t>(p) * s * s;
  __shared__ float ra[32][kNB + 4];  // [k][row]
  __shared__ float tb[32][kNB + 4];  // [k][col]
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
  float acc[4][4] = {};
  const int kend = min(m, tr0 + kNB);  // Rinv[r][k] is zero for k > r
  for (int k0 = 0; k0 < kend; k0 += 32) {
    for (int e = threadIdx.x; e < 32 * kNB; e += blockDim.x) {
      const int r = e / 32, k = e % 32;
      const int gr = tr0 + r, gk = k0 + k;
      ra[k][r] = (gr < m && gk < m) ? Binv[static_cast<size_t>(b + s + gr) * n + b + s + gk] : 0.0f;
      const int kk = e / kNB, c = e % kNB;
      tb[kk][c] = (k0 + kk < m) ? Tp[static_cast<size_t>(k0 + kk) * s + tc0 + c] : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      float x[4], y[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        x[u] = ra[k][tr + u];
        y[u] = tb[k][tc + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(x[u], y[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = tr0 + tr + u;
    if (r >= m) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) Binv[static_cast<size_t>(b + s + r) * n + b + tc0 + tc + v] = -acc[u][v];
  }
}

// U = J B J: swap element e with element n*n - 1 - e.
__global__ void rotate180_kernel(float* __restrict__ U, int64_t nn) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= nn / 2) return;
  const int64_t f = nn - 1 - e;
  const float x = U[e], y = U[f];
  U[e] = y;
  U[f] = x;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct PrepLayout {
  size_t a, t, key, dead, lambda, perm, total;
};

// Scratch of the doubling inverse: the largest level's pairs * s * s floats.
size_t tri_scratch_floats(int n) {
  size_t best = 0;
  for (int s = kNB; s < n; s *= 2) best = std::max(best, static_cast<size_t>(ceil_div(n, 2 * s)) * s * s);
  return best;
}

PrepLayout prep_layout(int n) {
  PrepLayout l{};
  const size_t nn = static_cast<size_t>(n) * n;
  size_t off = 0;
  l.a = off;
  off += align256(nn * sizeof(float));
  l.t = off;
  off += align256(tri_scratch_floats(n) * sizeof(float));
  l.key = off;
  off += align256(static_cast<size_t>(n) * sizeof(double));
  l.dead = off;
  off += align256(static_cast<size_t>(n));
  l.lambda = off;
  off += 256;
  l.perm = off;
  off += align256(static_cast<size_t>(n) * sizeof(int32_t));
  l.total = off;
  return l;
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
  float* T = reinterpret_cast<float*>(w + l.t);
  double* key = reinterpret_cast<double*>(w + l.key);
  uint8_t* dead = w + l.dead;
  double* lambda = reinterpret_cast<double*>(w + l.lambda);
  int32_t* perm = perm_out != nullptr ? perm_out : reinterpret_cast<int32_t*>(w + l.perm);
  int* fstatus = info->status + 1;

  if (cudaMemsetAsync(fstatus, 0, sizeof(int), st) != cudaSuccess) return GPTQ_ERR_CUDA;
  launch(diag_prep_kernel, 1, 1024, 0, st, H, hdiag, n, damp, key, dead, lambda, fstatus);
  if (act_order)
    launch(act_order_rank_kernel, static_cast<unsigned>(ceil_div(n, 256)), 256, 0, st, key, n, perm);
  else
    launch(identity_perm_kernel, static_cast<unsigned>(ceil_div(n, 256)), 256, 0, st, perm, n);
  if (dead_out != nullptr && cudaMemcpyAsync(dead_out, dead, n, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  launch(gather_reversed_kernel, dim3(static_cast<unsigned>(ceil_div(n, 256)), n), 256, 0, st, H, perm, dead, lambda, n,
                                                                                           A);
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;

  // B = L^-1 is built directly in U (zeroed first), then rotated.
  if (cudaMemsetAsync(U, 0, static_cast<size_t>(n) * n * sizeof(float), st) != cudaSuccess) return GPTQ_ERR_CUDA;
  for (int k0 = 0; k0 < n; k0 += kNB) {
    launch(potrf_diag_kernel, 1, kNB, 0, st, A, U, n, k0, fstatus);
    const int below = n - k0 - kNB;
    if (below > 0) {
      const int rt = static_cast<int>(ceil_div(below, kNB));
      launch(trsm_panel_kernel, rt, 256, 0, st, A, U, n, k0);
      launch(syrk_update_kernel, rt * (rt + 1) / 2, 256, 0, st, A, n, k0);
    }
  }
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
  for (int s = kNB; s < n; s *= 2) {
    const int pairs = static_cast<int>(ceil_div(n, 2 * s));
    const dim3 g(static_cast<unsigned>(s / kNB), static_cast<unsigned>(s / kNB), static_cast<unsigned>(pairs));
    launch(tri_gemm_right_lower_kernel, g, 256, 0, st, A, U, n, s, T);
    launch(tri_gemm_left_lower_kernel, g, 256, 0, st, U, T, n, s);
  }
  const int64_t nn = static_cast<int64_t>(n) * n;
  if (nn >= 2) launch(rotate180_kernel, static_cast<unsigned>(ceil_div(nn / 2, 256)), 256, 0, st, U, nn);
  if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;

  int fs = 0;
  if (cudaMemcpyAsync(&fs, fstatus, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GPTQ_ERR_CUDA;
  return static_cast<gptq_status>(fs);
}

}  // namespace gptq
