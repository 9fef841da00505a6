// GPTQ-2D: two-sided adaptive rounding ("Daily Papers" page, GPTQ-2D abstract).
//
// Rounds W [m, n] to scale * integers under ||A (W - Q) B||_F^2, given the upper
// factors UL [m, m] (UL^T UL = (A^T A)^-1) and UR [n, n] (UR^T UR = (B B^T)^-1).
// The one-dimensional algorithm on vec(W) under the Kronecker Gram feeds the
// scaled error e of entry (i', j') into entry (i, j) through UL[i', i] * UR[j', j],
// which vanishes unless i' <= i and j' <= j.  With M = E UR (E the errors found
// so far) the value at which entry (i, j) is rounded is
//     W[i, j] - sum_{i' <= i} UL[i', i] M[i', j],
// and rounding it adds e_ij * UR[j, :] to row i of M (the abstract's cubic-time
// form; entries on one anti-diagonal are independent).
//
// Tiling.  The matrix is cut into 64 x 64 tiles, and tile (I, J) depends only
// on tiles above and to the left of it, so the tiles of one tile anti-diagonal
// D = I + J are independent.  Two buffers carry the feedback between tiles:
//   Wt = W - (contributions of the row blocks above), and
//   M  = E UR restricted to the column tiles already to the left,
// so that when tile (I, J) is reached
//   Wt[I, J] = W[I, J] - sum_{I' < I} UL[I', I]^T M[I', J]   (M[I', J] final)
//   M[I, J]  = sum_{J' < J} E[I, J'] UR[J', J].
// Per wavefront D:
//   round2d_tile_kernel   one CTA per tile: stages Wt[I, J], M[I, J] and the
//                         upper parts of the diagonal blocks UL[I, I], UR[J, J]
//                         in shared memory and runs the tile's local
//                         anti-diagonals with the formula above (M's tile keeps
//                         the left tiles' part, so one formula covers both);
//                         writes the codes, E and the now final M[I, J].
//   push2d_kernel         one CTA per (tile, target tile): right,
//                         M[I, J'] += E[I, J] UR[J, J'] for J' > J; down,
//                         Wt[I', J] -= UL[I, I']^T M[I, J] for I' > I.
// Within one wavefront no two CTAs write the same tile (one tile per row block
// and per column block), and stream order separates the wavefronts.
//
// The work is O(m n (m + n)) fp32 multiply-adds on the CUDA cores, the same as
// the cubic form; the serial chain is about 2 (m + n) local anti-diagonals.
#include <cmath>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int kT = 64;                 // tile edge
constexpr int kRP = kT + 1;            // shared pitch of the round kernel (conflict-free columns)
constexpr int kQP = kT + 4;            // shared pitch of the push kernel (16-byte rows)
constexpr int kRoundThreads = 256;     // 4 threads per entry of a local anti-diagonal
constexpr int kPushThreads = 256;      // 16 x 16 threads, 4 x 4 outputs each
constexpr size_t kRoundSmem = (4 * kT * kRP + kT) * sizeof(float);

struct Round2dArgs {
  const float* UL;
  const float* UR;
  float* Wt;
  float* M;
  float* E;
  int32_t* codes;
  int64_t m, n;
  int mt, nt;  // tiles along the rows and along the columns
  float scale;
  float qmin, qmax;
  int clamp;
};

__device__ __forceinline__ int wave_first(int D, int nt) { return max(0, D - (nt - 1)); }

// Extent of the tile starting at `start` along a dimension of `total` entries.
__device__ __forceinline__ int tile_extent(int64_t total, int64_t start) {
  const int64_t r = total - start;
  return r < kT ? static_cast<int>(r) : kT;
}

__global__ void __launch_bounds__(kRoundThreads) round2d_tile_kernel(Round2dArgs p, int D) {
  extern __shared__ float smem[];
  float* Ws = smem;           // [kT][kRP] current values Wt of the tile
  float* Ms = Ws + kT * kRP;  // [kT][kRP] M of the tile (left tiles' part, then the tile's own)
  float* Ls = Ms + kT * kRP;  // [kT][kRP] Ls[a'][a] = UL[r0 + a', r0 + a] for a' <= a, else 0
  float* Rs = Ls + kT * kRP;  // [kT][kRP] Rs[b][c] = UR[c0 + b, c0 + c] for b <= c, else 0
  float* es = Rs + kT * kRP;  // [kT] scaled errors of the current local anti-diagonal
  const int I = wave_first(D, p.nt) + static_cast<int>(blockIdx.x);
  const int J = D - I;
  const int64_t r0 = static_cast<int64_t>(I) * kT, c0 = static_cast<int64_t>(J) * kT;
  const int rh = tile_extent(p.m, r0);
  const int ch = tile_extent(p.n, c0);
  const int tid = threadIdx.x;

  for (int idx = tid; idx < kT * kT; idx += kRoundThreads) {
    const int a = idx / kT, b = idx % kT;
    float w = 0.f, mv = 0.f, l = 0.f, r = 0.f;
    if (a < rh && b < ch) {
      const int64_t off = (r0 + a) * p.n + c0 + b;
      w = p.Wt[off];
      mv = p.M[off];
    }
    if (a < rh && b < rh && b >= a) l = p.UL[(r0 + a) * p.m + r0 + b];
    if (a < ch && b < ch && b >= a) r = p.UR[(c0 + a) * p.n + c0 + b];
    Ws[a * kRP + b] = w;
    Ms[a * kRP + b] = mv;
    Ls[a * kRP + b] = l;
    Rs[a * kRP + b] = r;
  }
  __syncthreads();

  const int slot = tid >> 2, part = tid & 3;
  for (int d = 0; d <= rh + ch - 2; ++d) {
    const int a_lo = max(0, d - (ch - 1));
    const int cnt = min(d, rh - 1) - a_lo + 1;  // entries (a, d - a), a_lo <= a < a_lo + cnt
    const bool act = slot < cnt;
    const int a = a_lo + slot;
    const int b = d - a;
    float s = 0.f;
    if (act) {
      for (int k = part; k <= a; k += 4) s = fmaf(Ls[k * kRP + a], Ms[k * kRP + b], s);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (act && part == 0) {
      const float v = Ws[a * kRP + b] - s;
      float q = rintf(__fdiv_rn(v, p.scale));
      if (p.clamp) q = fminf(fmaxf(q, p.qmin), p.qmax);
      const float e = (v - p.scale * q) / (Ls[a * kRP + a] * Rs[b * kRP + b]);
      es[slot] = e;
      const int64_t off = (r0 + a) * p.n + c0 + b;
      p.codes[off] = __float2int_rn(q);
      p.E[off] = e;
    }
    __syncthreads();
    // row a of M gains e * UR[b, c] for the tile's columns c >= b
    for (int idx = tid; idx < cnt * kT; idx += kRoundThreads) {
      const int sl = idx / kT, c = idx % kT;
      const int aa = a_lo + sl, bb = d - aa;
      if (c >= bb && c < ch) Ms[aa * kRP + c] = fmaf(es[sl], Rs[bb * kRP + c], Ms[aa * kRP + c]);
    }
    __syncthreads();
  }

  for (int idx = tid; idx < rh * kT; idx += kRoundThreads) {
    const int a = idx / kT, b = idx % kT;
    if (b < ch) p.M[(r0 + a) * p.n + c0 + b] = Ms[a * kRP + b];
  }
}

// out[p, q] += sign * sum_k A(k, p) B(k, q) for one 64 x 64 target tile.
__global__ void __launch_bounds__(kPushThreads) push2d_kernel(Round2dArgs p, int D) {
  __shared__ __align__(16) float As[kT][kQP];
  __shared__ __align__(16) float Bs[kT][kQP];
  const int I = wave_first(D, p.nt) + static_cast<int>(blockIdx.x);
  const int J = D - I;
  const bool right = blockIdx.z == 0;
  const int tgt = (right ? J : I) + 1 + static_cast<int>(blockIdx.y);
  if (tgt >= (right ? p.nt : p.mt)) return;
  const int64_t r0 = static_cast<int64_t>(I) * kT, c0 = static_cast<int64_t>(J) * kT;
  const int64_t t0 = static_cast<int64_t>(tgt) * kT;
  const int rh = tile_extent(p.m, r0);
  const int ch = tile_extent(p.n, c0);

  const float* A;
  int64_t a_sk, a_sp;  // A(k, p) = A[k * a_sk + p * a_sp]
  const float* B;      // B(k, q) = B[k * n + q]
  float* out;          // out[p * n + q]
  int K, P, Q;
  float sign;
  if (right) {  // M[I, tgt] += E[I, J] UR[J, tgt]
    K = ch;
    P = rh;
    Q = tile_extent(p.n, t0);
    A = p.E + r0 * p.n + c0;
    a_sk = 1;
    a_sp = p.n;
    B = p.UR + c0 * p.n + t0;
    out = p.M + r0 * p.n + t0;
    sign = 1.f;
  } else {  // Wt[tgt, J] -= UL[I, tgt]^T M[I, J]
    K = rh;
    P = tile_extent(p.m, t0);
    Q = ch;
    A = p.UL + r0 * p.m + t0;
    a_sk = p.m;
    a_sp = 1;
    B = p.M + r0 * p.n + c0;
    out = p.Wt + t0 * p.n + c0;
    sign = -1.f;
  }

  const int tid = threadIdx.x;
  for (int idx = tid; idx < kT * kT; idx += kPushThreads) {
    // the contiguous index of A's source runs along the threads
    const int k = a_sk == 1 ? idx % kT : idx / kT;
    const int pp = a_sk == 1 ? idx / kT : idx % kT;
    As[k][pp] = (k < K && pp < P) ? A[k * a_sk + pp * a_sp] : 0.f;
    const int kb = idx / kT, qb = idx % kT;
    Bs[kb][qb] = (kb < K && qb < Q) ? B[kb * p.n + qb] : 0.f;
  }
  __syncthreads();

  const int ty = tid / 16, tx = tid % 16;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k = 0; k < K; ++k) {
    const float4 a4 = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
    const float4 b4 = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
    const float av[4] = {a4.x, a4.y, a4.z, a4.w};
    const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int pr = ty * 4 + i;
    if (pr >= P) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int qc = tx * 4 + j;
      if (qc < Q) out[pr * p.n + qc] += sign * acc[i][j];
    }
  }
}

template <typename T>
__global__ void to_f32_kernel(const T* __restrict__ src, float* __restrict__ dst, int64_t count) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = static_cast<float>(src[i]);
}

size_t aligned_bytes(int64_t count) { return static_cast<size_t>((count * 4 + 255) / 256 * 256); }

}  // namespace

size_t round2d_workspace_size(int64_t m, int64_t n) { return 3 * aligned_bytes(m * n); }

gptq_status round2d(const void* W, int w_bf16, int64_t m, int64_t n, const float* UL, const float* UR, float scale,
                    int clamp, int qmin, int qmax, int32_t* codes, float* E, void* ws, cudaStream_t st) {
  if (m == 0 || n == 0) return GPTQ_OK;
  const int64_t count = m * n;
  char* base = static_cast<char*>(ws);
  float* Wt = reinterpret_cast<float*>(base);
  float* M = reinterpret_cast<float*>(base + aligned_bytes(count));
  float* Eb = E != nullptr ? E : reinterpret_cast<float*>(base + 2 * aligned_bytes(count));

  const DeviceInfo* info = device_info();
  if (info == nullptr) return GPTQ_ERR_CUDA;
  const unsigned cgrid = static_cast<unsigned>(std::min<int64_t>(ceil_div(count, 256), 8LL * info->sm_count));
  if (w_bf16)
    launch(to_f32_kernel<__nv_bfloat16>, cgrid, 256, 0, st, static_cast<const __nv_bfloat16*>(W), Wt, count);
  else
    launch(to_f32_kernel<float>, cgrid, 256, 0, st, static_cast<const float*>(W), Wt, count);
  if (cudaMemsetAsync(M, 0, static_cast<size_t>(count) * sizeof(float), st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaFuncSetAttribute(round2d_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kRoundSmem)) != cudaSuccess)
    return GPTQ_ERR_CUDA;

  Round2dArgs p{};
  p.UL = UL;
  p.UR = UR;
  p.Wt = Wt;
  p.M = M;
  p.E = Eb;
  p.codes = codes;
  p.m = m;
  p.n = n;
  p.mt = static_cast<int>(ceil_div(m, kT));
  p.nt = static_cast<int>(ceil_div(n, kT));
  p.scale = scale;
  p.clamp = clamp;
  p.qmin = static_cast<float>(qmin);
  p.qmax = static_cast<float>(qmax);
  const int targets = std::max(p.mt, p.nt) - 1;
  for (int D = 0; D <= p.mt + p.nt - 2; ++D) {
    const int tiles = std::min(D, p.mt - 1) - std::max(0, D - (p.nt - 1)) + 1;
    launch(round2d_tile_kernel, dim3(tiles), dim3(kRoundThreads), kRoundSmem, st, p, D);
    if (targets > 0 && D < p.mt + p.nt - 2)
      launch(push2d_kernel, dim3(tiles, targets, 2), dim3(kPushThreads), 0, st, p, D);
  }
  return launch_status();
}

}  // namespace gptq
