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
// Tiling.  The matrix is cut into 64 x 64 tiles; tile (I, J) depends only on
// the tiles above and to the left of it, so the tiles of one tile
// anti-diagonal D = I + J are independent.  When tile (I, J) is reached its
// feedback is spread over four buffers, each written by one kind of step:
//   Wt[I, J] = W[I, J] - sum_{I' <= I-2} UL[I', I]^T M[I', J]   (far pushes down)
//   Dn[I, J] =           UL[I-1, I]^T M[I-1, J]                 (near push down)
//   Mf[I, J] = sum_{J' <= J-2} E[I, J'] UR[J', J]               (far pushes right)
//   Mn[I, J] = E[I, J-1] UR[J-1, J]                             (near push right)
// and M[I, J] (left part) = Mf + Mn.  Per wavefront D:
//   round2d_tile_kernel  one CTA per tile: runs the tile's local anti-diagonals
//                        in shared memory on Wt - Dn and Mf + Mn, writes the
//                        codes, E and the tile's final M (into Mf), then the two
//                        near pushes (written, not accumulated: one writer each).
//   far_push_kernel      one CTA per (tile, far target): right, Mf[I, J'] +=
//                        E[I, J] UR[J, J'] for J' >= J + 2; down, Wt[I', J] -=
//                        UL[I, I']^T M[I, J] for I' >= I + 2.
// The far pushes of wavefront D only feed wavefronts >= D + 2, so they run on a
// second, low-priority stream while the round kernel of wavefront D + 1 runs on
// a high-priority one; the round kernel of D + 2 waits for them.  No two
// concurrent CTAs write the same element (far pushes write Mf and Wt of tiles
// on wavefronts >= D + 2, the round kernel of D + 1 writes its own tiles and
// Mn, Dn of wavefront D + 2), and every element is summed in a fixed order, so
// the result is deterministic.
//
// The work is O(m n (m + n)) fp32 multiply-adds on the CUDA cores; the serial
// chain is the round kernels, about 2 (m + n) local anti-diagonals.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int kT = 64;                 // tile edge
constexpr int kRP = kT + 1;            // shared pitch of the round kernel (conflict-free columns)
constexpr int kQP = kT + 4;            // shared pitch of the far-push kernel (16-byte rows)
constexpr int kThreads = 256;          // both kernels
constexpr size_t kRoundSmem = (5 * kT * kRP + kT) * sizeof(float);

struct Round2dArgs {
  const float* UL;
  const float* UR;
  float* Wt;
  float* Mf;
  float* Mn;
  float* Dn;
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

__global__ void __launch_bounds__(kThreads) round2d_tile_kernel(Round2dArgs p, int D) {
  extern __shared__ float smem[];
  float* Ws = smem;           // [kT][kRP] values of the tile (Wt - Dn)
  float* Ms = Ws + kT * kRP;  // [kT][kRP] M of the tile (left part, then the tile's own)
  float* Ls = Ms + kT * kRP;  // [kT][kRP] UL[r0 + a', r0 + a] for a' <= a, else 0; later UL[I, I+1]
  float* Rs = Ls + kT * kRP;  // [kT][kRP] UR[c0 + b, c0 + c] for b <= c, else 0; later UR[J, J+1]
  float* Es = Rs + kT * kRP;  // [kT][kRP] the tile's scaled errors
  float* es = Es + kT * kRP;  // [kT] scaled errors of the current local anti-diagonal
  const int I = wave_first(D, p.nt) + static_cast<int>(blockIdx.x);
  const int J = D - I;
  const int64_t r0 = static_cast<int64_t>(I) * kT, c0 = static_cast<int64_t>(J) * kT;
  const int rh = tile_extent(p.m, r0);
  const int ch = tile_extent(p.n, c0);
  const int tid = threadIdx.x;

  for (int idx = tid; idx < kT * kT; idx += kThreads) {
    const int a = idx / kT, b = idx % kT;
    float w = 0.f, mv = 0.f, l = 0.f, r = 0.f;
    if (a < rh && b < ch) {
      const int64_t off = (r0 + a) * p.n + c0 + b;
      w = p.Wt[off] - p.Dn[off];
      mv = p.Mf[off] + p.Mn[off];
    }
    if (a < rh && b < rh && b >= a) l = p.UL[(r0 + a) * p.m + r0 + b];
    if (a < ch && b < ch && b >= a) r = p.UR[(c0 + a) * p.n + c0 + b];
    Ws[a * kRP + b] = w;
    Ms[a * kRP + b] = mv;
    Ls[a * kRP + b] = l;
    Rs[a * kRP + b] = r;
    Es[a * kRP + b] = 0.f;
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
      Es[a * kRP + b] = e;
      const int64_t off = (r0 + a) * p.n + c0 + b;
      p.codes[off] = __float2int_rn(q);
      p.E[off] = e;
    }
    __syncthreads();
    // row a of M gains e * UR[b, c] for the tile's columns c >= b
    for (int idx = tid; idx < cnt * kT; idx += kThreads) {
      const int sl = idx / kT, c = idx % kT;
      const int aa = a_lo + sl, bb = d - aa;
      if (c >= bb && c < ch) Ms[aa * kRP + c] = fmaf(es[sl], Rs[bb * kRP + c], Ms[aa * kRP + c]);
    }
    __syncthreads();
  }

  // the tile's final M (no far push writes this tile any more)
  for (int idx = tid; idx < rh * kT; idx += kThreads) {
    const int a = idx / kT, b = idx % kT;
    if (b < ch) p.Mf[(r0 + a) * p.n + c0 + b] = Ms[a * kRP + b];
  }

  // near pushes: stage UR[J, J+1] into Rs and UL[I, I+1] into Ls (both free now)
  const bool right = J + 1 < p.nt, down = I + 1 < p.mt;
  if (!right && !down) return;
  const int64_t tr = c0 + kT, td = r0 + kT;  // first column of J+1, first row of I+1
  const int Qr = right ? tile_extent(p.n, tr) : 0;
  const int Pd = down ? tile_extent(p.m, td) : 0;
  for (int idx = tid; idx < kT * kT; idx += kThreads) {
    const int k = idx / kT, c = idx % kT;
    Rs[k * kRP + c] = (k < ch && c < Qr) ? p.UR[(c0 + k) * p.n + tr + c] : 0.f;
    Ls[k * kRP + c] = (k < rh && c < Pd) ? p.UL[(r0 + k) * p.m + td + c] : 0.f;
  }
  __syncthreads();
  const int ty = tid / 16, tx = tid % 16;
  if (right) {  // Mn[I, J+1] = E[I, J] UR[J, J+1]
    float acc[4][4] = {};
    for (int k = 0; k < ch; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = Es[(ty * 4 + i) * kRP + k];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Rs[k * kRP + tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int pr = ty * 4 + i;
      if (pr >= rh) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int qc = tx * 4 + j;
        if (qc < Qr) p.Mn[(r0 + pr) * p.n + tr + qc] = acc[i][j];
      }
    }
  }
  if (down) {  // Dn[I+1, J] = UL[I, I+1]^T M[I, J]
    float acc[4][4] = {};
    for (int k = 0; k < rh; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = Ls[k * kRP + ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Ms[k * kRP + tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int pr = ty * 4 + i;
      if (pr >= Pd) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int qc = tx * 4 + j;
        if (qc < ch) p.Dn[(td + pr) * p.n + c0 + qc] = acc[i][j];
      }
    }
  }
}

// Far targets of a tile: right J' in [J + 2, nt), down I' in [I + 2, mt).
__host__ __device__ __forceinline__ int far_right(int J, int nt) { return nt - J - 2 > 0 ? nt - J - 2 : 0; }
__host__ __device__ __forceinline__ int far_down(int I, int mt) { return mt - I - 2 > 0 ? mt - I - 2 : 0; }

// One CTA per (tile of wavefront D, far target); the grid holds exactly the
// wavefront's number of such pairs.  out[p, q] += sign * sum_k A(k, p) B(k, q).
__global__ void __launch_bounds__(kThreads) far_push_kernel(Round2dArgs p, int D) {
  __shared__ __align__(16) float As[kT][kQP];
  __shared__ __align__(16) float Bs[kT][kQP];
  const int first = wave_first(D, p.nt);
  const int last = min(D, p.mt - 1);
  int idx = static_cast<int>(blockIdx.x);
  int I = -1, J = -1, tgt = -1;
  bool right = false;
  for (int t = first; t <= last; ++t) {
    const int jt = D - t;
    const int r = far_right(jt, p.nt), d = far_down(t, p.mt);
    if (idx < r) {
      I = t; J = jt; right = true; tgt = jt + 2 + idx;
      break;
    }
    idx -= r;
    if (idx < d) {
      I = t; J = jt; right = false; tgt = t + 2 + idx;
      break;
    }
    idx -= d;
  }
  if (I < 0) return;  // not reached: the host sizes the grid to the pair count
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
  if (right) {  // Mf[I, tgt] += E[I, J] UR[J, tgt]
    K = ch;
    P = rh;
    Q = tile_extent(p.n, t0);
    A = p.E + r0 * p.n + c0;
    a_sk = 1;
    a_sp = p.n;
    B = p.UR + c0 * p.n + t0;
    out = p.Mf + r0 * p.n + t0;
    sign = 1.f;
  } else {  // Wt[tgt, J] -= UL[I, tgt]^T M[I, J]   (M[I, J] final, held in Mf)
    K = rh;
    P = tile_extent(p.m, t0);
    Q = ch;
    A = p.UL + r0 * p.m + t0;
    a_sk = p.m;
    a_sp = 1;
    B = p.Mf + r0 * p.n + c0;
    out = p.Wt + t0 * p.n + c0;
    sign = -1.f;
  }

  const int tid = threadIdx.x;
  for (int i = tid; i < kT * kT; i += kThreads) {
    // the contiguous index of A's source runs along the threads
    const int k = a_sk == 1 ? i % kT : i / kT;
    const int pp = a_sk == 1 ? i / kT : i % kT;
    As[k][pp] = (k < K && pp < P) ? A[k * a_sk + pp * a_sp] : 0.f;
    const int kb = i / kT, qb = i % kT;
    Bs[kb][qb] = (kb < K && qb < Q) ? B[kb * p.n + qb] : 0.f;
  }
  __syncthreads();

  const int ty = tid / 16, tx = tid % 16;
  float acc[4][4] = {};
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

// Two library streams per device: high priority for the round kernels (the
// serial chain), low priority for the far pushes that fill the other SMs.
struct Streams {
  bool ready = false;
  cudaStream_t hi = nullptr, lo = nullptr;
};
std::mutex g_stream_mutex;
Streams g_streams[64];

const Streams* streams_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_stream_mutex);
  Streams& s = g_streams[dev];
  if (!s.ready) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithPriority(&s.hi, cudaStreamNonBlocking, greatest) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithPriority(&s.lo, cudaStreamNonBlocking, least) != cudaSuccess) return nullptr;
    s.ready = true;
  }
  return &s;
}

}  // namespace

size_t round2d_workspace_size(int64_t m, int64_t n) { return 5 * aligned_bytes(m * n); }

gptq_status round2d(const void* W, int w_bf16, int64_t m, int64_t n, const float* UL, const float* UR, float scale,
                    int clamp, int qmin, int qmax, int32_t* codes, float* E, void* ws, cudaStream_t st) {
  if (m == 0 || n == 0) return GPTQ_OK;
  const int64_t count = m * n;
  const size_t region = aligned_bytes(count);
  char* base = static_cast<char*>(ws);
  float* Wt = reinterpret_cast<float*>(base);
  float* Mf = reinterpret_cast<float*>(base + region);
  float* Mn = reinterpret_cast<float*>(base + 2 * region);
  float* Dn = reinterpret_cast<float*>(base + 3 * region);
  float* Eb = E != nullptr ? E : reinterpret_cast<float*>(base + 4 * region);

  const DeviceInfo* info = device_info();
  const Streams* ss = streams_for_current_device();
  if (info == nullptr || ss == nullptr) return GPTQ_ERR_CUDA;
  const unsigned cgrid = static_cast<unsigned>(std::min<int64_t>(ceil_div(count, 256), 8LL * info->sm_count));
  if (w_bf16)
    launch(to_f32_kernel<__nv_bfloat16>, cgrid, 256, 0, st, static_cast<const __nv_bfloat16*>(W), Wt, count);
  else
    launch(to_f32_kernel<float>, cgrid, 256, 0, st, static_cast<const float*>(W), Wt, count);
  // Mf, Mn and Dn are adjacent: one memset
  if (cudaMemsetAsync(Mf, 0, 3 * region, st) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaFuncSetAttribute(round2d_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kRoundSmem)) != cudaSuccess)
    return GPTQ_ERR_CUDA;

  Round2dArgs p{};
  p.UL = UL;
  p.UR = UR;
  p.Wt = Wt;
  p.Mf = Mf;
  p.Mn = Mn;
  p.Dn = Dn;
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

  // events: fork, the latest round, a ring of two for the far pushes, join
  cudaEvent_t ev_fork, ev_round, ev_far[2], ev_join;
  cudaEvent_t* all[] = {&ev_fork, &ev_round, &ev_far[0], &ev_far[1], &ev_join};
  for (cudaEvent_t* e : all)
    if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return GPTQ_ERR_CUDA;
  bool ok = cudaEventRecord(ev_fork, st) == cudaSuccess && cudaStreamWaitEvent(ss->hi, ev_fork, 0) == cudaSuccess &&
            cudaStreamWaitEvent(ss->lo, ev_fork, 0) == cudaSuccess;
  const int waves = p.mt + p.nt - 1;
  int last_far = -1;  // the far pushes exist for a prefix of the wavefronts
  for (int D = 0; ok && D < waves; ++D) {
    if (D >= 2 && last_far >= 0) {
      const int need = std::min(D - 2, last_far);
      ok = cudaStreamWaitEvent(ss->hi, ev_far[need % 2], 0) == cudaSuccess;
    }
    const int first = std::max(0, D - (p.nt - 1)), lastI = std::min(D, p.mt - 1);
    launch(round2d_tile_kernel, dim3(lastI - first + 1), dim3(kThreads), kRoundSmem, ss->hi, p, D);
    int pairs = 0;
    for (int I = first; I <= lastI; ++I) pairs += far_right(D - I, p.nt) + far_down(I, p.mt);
    if (pairs > 0 && ok) {
      ok = cudaEventRecord(ev_round, ss->hi) == cudaSuccess && cudaStreamWaitEvent(ss->lo, ev_round, 0) == cudaSuccess;
      launch(far_push_kernel, dim3(pairs), dim3(kThreads), 0, ss->lo, p, D);
      ok = ok && cudaEventRecord(ev_far[D % 2], ss->lo) == cudaSuccess;
      last_far = D;
    }
  }
  ok = ok && cudaEventRecord(ev_join, ss->lo) == cudaSuccess && cudaStreamWaitEvent(st, ev_join, 0) == cudaSuccess;
  ok = ok && cudaEventRecord(ev_join, ss->hi) == cudaSuccess && cudaStreamWaitEvent(st, ev_join, 0) == cudaSuccess;
  for (cudaEvent_t* e : all) cudaEventDestroy(*e);
  if (!ok) return GPTQ_ERR_CUDA;
  return launch_status();
}

}  // namespace gptq
