// Inference with the packed weights: y[b, r] = sum_c Q[r, c] x[b, c], with
// Q[r, c] = scales[r, g(c)] * (code[r, c] - zeros[r, g(c)]) read straight from
// the packed rows (GPTQ abstract on the "Daily Papers" page: the packed 3/4-bit
// weights run generative inference faster than FP16; GPTQ knowledge note,
// "Tradeoffs": deployment reads packed weights).
//
// The product streams the packed matrix once, so it is bound by HBM: per
// 4-bit weight half a byte is read, a quarter of a bf16 weight.
//
// Two kernels: 4-bit codes with bf16 x in groups of a multiple of 128 columns
// (or one group per row) go to the tensor cores (matvec_reg4_kernel, further
// below); every other case to the general kernel described here.
//
// Layout of the work (general kernel): one warp per weight row (grid-stride over rows); lane l
// takes the row's runs of 32 codes l, l + 32, ... (a run is `bits` 32-bit
// words, so a warp reads `bits` * 128 contiguous bytes per step).  x is staged
// in shared memory as xs[b][run][i] = x[b][32 run + i] with a 36-float run
// pitch, so that a lane reads four positions of its run with one 16-byte load
// and eight lanes on consecutive runs hit distinct bank groups.  Codes are turned into floats by
// the 2^23 trick: (0x4B000000 | code) read as a float is 2^23 + code exactly.
//
// Groups: when they are contiguous and a whole number of runs (no g_idx,
// group % 32 == 0 or one group per row) a run lies in one group, and its
// contribution is s * (sum_i code_i x_i - z * sum_i x_i), with the run sums of
// x computed once per CTA.  Otherwise (act-order g_idx, or groups that split
// runs) every code looks up its own scale and zero point.
#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kChunkFloats = 16384;  // x floats staged per pass (64 KB + padding)
constexpr int kRunPitch = 36;        // floats per staged run of 32 (16-byte aligned, bank-spread)

// The BITS words of run q of a packed row; 16- or 8-byte loads when the row
// is aligned for them.
template <int BITS>
__device__ __forceinline__ void load_run(const uint32_t* __restrict__ prow, int q, bool vec, uint32_t (&w)[BITS]) {
  const uint32_t* src = prow + q * BITS;
  if (BITS % 4 == 0 && vec) {
#pragma unroll
    for (int k = 0; k < BITS; k += 4) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + k));
      w[k] = v.x;
      w[k + 1] = v.y;
      w[k + 2] = v.z;
      w[k + 3] = v.w;
    }
  } else if (BITS == 2 && vec) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
    w[0] = v.x;
    w[1] = v.y;
  } else {
#pragma unroll
    for (int k = 0; k < BITS; ++k) w[k] = __ldg(src + k);
  }
}

// code i of a run as a float (the mask and the exponent bits in one step)
template <int BITS>
__device__ __forceinline__ float code_f(const uint32_t (&w)[BITS], int i) {
  const int bit = i * BITS;
  const int k = bit >> 5, s = bit & 31;
  uint32_t v = w[k] >> s;
  if (s + BITS > 32) v |= w[k + 1] << (32 - s);
  return __uint_as_float((v & ((1u << BITS) - 1u)) | 0x4B000000u) - 8388608.0f;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Stages x[:, columns of runs q0 .. q0 + nr) (transposed, see above) and, for
// the contiguous-group path, the runs' sums of x.  A warp takes a run at a
// time: its lanes read the run's 32 consecutive values (coalesced), store them
// as one row of xs and add them with a shuffle reduction.
template <int B, bool kFast, typename T>
__device__ __forceinline__ void stage_x(float* xs, float* xsum, const T* __restrict__ x, int n, int batch, int q0,
                                        int nr, int runs_chunk) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();  // the previous chunk is no longer read
  for (int br = warp; br < B * nr; br += kWarps) {
    const int b = br / nr, run = br - b * nr;
    const int c = 32 * (q0 + run) + lane;
    const float v = (b < batch && c < n) ? to_f32<T>(x[static_cast<int64_t>(b) * n + c]) : 0.0f;
    xs[(b * runs_chunk + run) * kRunPitch + lane] = v;
    if (kFast) {
      float t = v;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) xsum[b * runs_chunk + run] = t;
    }
  }
  __syncthreads();
}

template <int BITS, int B, bool kFast, typename T>
__global__ void __launch_bounds__(kThreads) dequant_matvec_kernel(const uint32_t* __restrict__ packed,
                                                                  const float* __restrict__ scales,
                                                                  const uint8_t* __restrict__ zeros,
                                                                  const int32_t* __restrict__ g_idx, int64_t rows,
                                                                  int n, int G, int n_groups, const T* __restrict__ x,
                                                                  int batch, float* __restrict__ y) {
  extern __shared__ float xs[];  // [B][runs_chunk][kRunPitch], then run sums [B][runs_chunk]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int runs = (n + 31) / 32;
  const int words = BITS * runs;
  const int runs_chunk = (kChunkFloats / B) / 32;
  float* xsum = xs + B * runs_chunk * kRunPitch;
  const int64_t row_stride = static_cast<int64_t>(gridDim.x) * kWarps;
  const bool one_pass = runs <= runs_chunk;  // x staged once for all of the CTA's rows
  if (one_pass) stage_x<B, kFast>(xs, xsum, x, n, batch, 0, runs, runs_chunk);

  for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * kWarps; r0 < rows; r0 += row_stride) {
    const int64_t r = r0 + warp;
    float acc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = 0.0f;
    for (int q0 = 0; q0 < runs; q0 += runs_chunk) {
      const int nr = min(runs_chunk, runs - q0);
      if (!one_pass) stage_x<B, kFast>(xs, xsum, x, n, batch, q0, nr, runs_chunk);
      if (r < rows) {
        const uint32_t* prow = packed + r * words;
        const bool vec = (reinterpret_cast<uintptr_t>(prow) % (BITS == 2 ? 8 : 16)) == 0;
        // runs in groups of kPre per lane: all their words are requested
        // before any is used, so the loads of a row overlap
        constexpr int kPre = 4;
        for (int run0 = lane; run0 < nr; run0 += 32 * kPre) {
          uint32_t w[kPre][BITS];
#pragma unroll
          for (int u = 0; u < kPre; ++u) {
            const int run = run0 + 32 * u;
            if (run < nr) load_run<BITS>(prow, q0 + run, vec, w[u]);
          }
#pragma unroll
          for (int u = 0; u < kPre; ++u) {
            const int run = run0 + 32 * u;
            if (run >= nr) break;
            const int q = q0 + run;
            if (kFast) {
              const int g = (32 * q) / G;
              const float sc = __ldg(scales + r * n_groups + g);
              const float z = static_cast<float>(__ldg(zeros + r * n_groups + g));
              float dot[B];
#pragma unroll
              for (int b = 0; b < B; ++b) dot[b] = 0.0f;
#pragma unroll
              for (int i4 = 0; i4 < 32; i4 += 4) {
                const float c0 = code_f<BITS>(w[u], i4), c1 = code_f<BITS>(w[u], i4 + 1);
                const float c2 = code_f<BITS>(w[u], i4 + 2), c3 = code_f<BITS>(w[u], i4 + 3);
#pragma unroll
                for (int b = 0; b < B; ++b) {
                  const float4 xv = *reinterpret_cast<const float4*>(xs + (b * runs_chunk + run) * kRunPitch + i4);
                  dot[b] = fmaf(c0, xv.x, dot[b]);
                  dot[b] = fmaf(c1, xv.y, dot[b]);
                  dot[b] = fmaf(c2, xv.z, dot[b]);
                  dot[b] = fmaf(c3, xv.w, dot[b]);
                }
              }
#pragma unroll
              for (int b = 0; b < B; ++b) acc[b] = fmaf(sc, fmaf(-z, xsum[b * runs_chunk + run], dot[b]), acc[b]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int c = min(32 * q + i, n - 1);  // codes past n are zero; x there is zero
                const int g = g_idx != nullptr ? __ldg(g_idx + c) : c / G;
                const float sc = __ldg(scales + r * n_groups + g);
                const float z = static_cast<float>(__ldg(zeros + r * n_groups + g));
                const float qv = sc * (code_f<BITS>(w[u], i) - z);
#pragma unroll
                for (int b = 0; b < B; ++b) acc[b] = fmaf(qv, xs[(b * runs_chunk + run) * kRunPitch + i], acc[b]);
              }
            }
          }
        }
      }
    }
    if (r < rows) {
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float v = acc[b];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && b < batch) y[static_cast<int64_t>(b) * rows + r] = v;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// 4-bit codes with bf16 x on the tensor cores (mma.sync m16n8k16: bf16
// operands, fp32 accumulation).  A CTA owns 16 weight rows (one m16 tile) and
// multiplies them by up to 8 x vectors, one per column of the B operand.
//
// Memory: the weights go from HBM straight into registers.  The columns come
// in blocks of 128 (16 words per row); in a block, lane (g, t) of a warp
// loads words 4t..4t+3 of rows g and g + 8 (two 16-byte loads), and warp w
// takes blocks w, w + 8, ...  A round of 4 blocks per warp keeps 8 loads per
// lane in flight, all issued at launch when n <= 4096 (the next round is
// requested before the current one is used otherwise), so that HBM sees the
// whole matrix requested at once.  The CTA's scales, zero points and x are
// staged in shared memory while the weights are in flight.  (Staging the
// weights in shared memory through bulk copies, TMA boxes or cp.async rings
// was measured slower at this size: the copies' issue cost and the extra
// shared-memory round trip sat on the critical path.)
//
// Decoding: MMA step m (0..7) of a block takes, in lane (g, t), word
// 4t + m / 2 of each row and its nibble pairs (p, p + 4) for p = 2 (m % 2) and
// p + 1: (word >> 4p) & 0x000F000F | 0x43004300 is the bf16 pair 128 + code
// (exact), 7 ALU operations per 8 codes.  The MMA column order is thereby a
// permutation of the block's codes, and x is staged in the same order: the
// 8 values x[8h..8h + 7] of half-step h = 16 block + 4t + m2 give one 16-byte
// entry (x[8h + p], x[8h + p + 4]), p = 0..3, read by lane 4 b + t for steps
// 2 m2 and 2 m2 + 1.  A block lies in one group (G % 128 == 0, or one group
// per row): the warp adds s * sum (128 + code) x per block, and the offsets
// s (128 + z) X_q of the groups (X_q the group's sum of x) are subtracted once
// per output at the end.  Products of bf16 values are exact; sums are fp32.
constexpr int kRegWarps = 8;
constexpr int kRegThreads = kRegWarps * 32;
constexpr int kRegRound = 4;  // blocks per warp per round
constexpr size_t kRegMaxSmem = 200 * 1024;

struct RegLayout {
  size_t xs, xsum, red, sc, zp, total;  // byte offsets into dynamic shared memory
};

RegLayout reg_layout(int n, int n_groups, int batch) {
  RegLayout l;
  l.xs = 0;
  l.xsum = l.xs + static_cast<size_t>(n) * batch * 2;  // (n / 8) half-steps x batch x 16 bytes
  l.red = l.xsum + static_cast<size_t>(n / 128) * batch * 4;
  l.sc = l.red + static_cast<size_t>(kRegWarps) * 128 * 4;
  l.zp = l.sc + static_cast<size_t>(16) * n_groups * 4;
  l.total = l.zp + static_cast<size_t>(16) * n_groups;
  return l;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int p) { return ((w >> (4 * p)) & 0x000F000Fu) | 0x43004300u; }

// A 16-byte read-only load that the compiler keeps where it is written (a
// volatile asm statement is not moved past the barriers that follow it), so
// that the weight stream starts at launch rather than at first use.
__device__ __forceinline__ uint4 ld_early(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// Requires n % 128 == 0, G % 128 == 0 or one group per row, batch <= 8,
// 16-byte aligned matrix and x.  Shared memory: xs [n / 8 half-steps as
// (block, m2, lane)] uint4, xsum [n / 128][batch], red [kRegWarps][16][8],
// the CTA's scales [16][n_groups] and zero points [16][n_groups].
__global__ void __launch_bounds__(kRegThreads) matvec_reg4_kernel(const uint32_t* __restrict__ packed,
                                                                  const float* __restrict__ scales,
                                                                  const uint8_t* __restrict__ zeros, int64_t rows,
                                                                  int n, int G, int n_groups,
                                                                  const __nv_bfloat16* __restrict__ x, int batch,
                                                                  float* __restrict__ y, uint32_t gmagic,
                                                                  uint32_t xsum_off, uint32_t red_off, uint32_t sc_off,
                                                                  uint32_t zp_off) {
  extern __shared__ __align__(16) uint8_t rg_smem[];
  uint4* xs = reinterpret_cast<uint4*>(rg_smem);
  float* xsum = reinterpret_cast<float*>(rg_smem + xsum_off);
  float* red = reinterpret_cast<float*>(rg_smem + red_off);
  float* ssc = reinterpret_cast<float*>(rg_smem + sc_off);
  uint8_t* szp = rg_smem + zp_off;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 16;
  const int nrows = rows - r0 < 16 ? static_cast<int>(rows - r0) : 16;
  const int64_t words = n / 8;
  const int blocks = n / 128;
  const int my_blocks = blocks > warp ? (blocks - warp + kRegWarps - 1) / kRegWarps : 0;
  const bool va = g < nrows, vb = g + 8 < nrows;
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
  const uint4* pa = reinterpret_cast<const uint4*>(packed + (va ? r0 + g : 0) * words) + t;
  const uint4* pb = reinterpret_cast<const uint4*>(packed + (vb ? r0 + g + 8 : 0) * words) + t;
  uint4 wa[kRegRound], wb[kRegRound];
  auto load_round = [&](int k0) {
#pragma unroll
    for (int i = 0; i < kRegRound; ++i) {
      const bool ok = k0 + i < my_blocks;
      const int blk = warp + (k0 + i) * kRegWarps;
      wa[i] = ok && va ? ld_early(pa + 4 * blk) : zero4;
      wb[i] = ok && vb ? ld_early(pb + 4 * blk) : zero4;
    }
  };

  // Staging: scales and zero points, x in the MMA's column order, and the
  // block sums of x (16 lanes per block, in a shuffle tree).  The first
  // pieces of each are requested before the weights, so that they are not
  // queued behind the weight stream.
  const int pairs = 4 * batch;
  const int nsz = nrows * n_groups;
  const int per_row = n / 8;
  float sv0 = 0.0f;
  uint32_t zv0 = 0u;
  uint4 xv0 = zero4;
  const int e0 = threadIdx.x, h0 = warp * 32 + lane;
  if (e0 < nsz) {
    sv0 = __ldg(scales + r0 * n_groups + e0);
    zv0 = __ldg(zeros + r0 * n_groups + e0);
  }
  if (h0 < per_row) xv0 = __ldg(reinterpret_cast<const uint4*>(x) + h0);
  load_round(0);
  for (int e = e0; e < nsz; e += kRegThreads) {
    ssc[e] = e == e0 ? sv0 : __ldg(scales + r0 * n_groups + e);
    szp[e] = static_cast<uint8_t>(e == e0 ? zv0 : __ldg(zeros + r0 * n_groups + e));
  }
  for (int b = 0; b < batch; ++b) {
    const uint4* xrow = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(b) * n);
    for (int hw = warp * 32; hw < per_row; hw += kRegThreads) {  // warp-uniform bound: all lanes shuffle
      const int h = hw + lane;
      const bool ok = h < per_row;
      const uint4 raw = (b == 0 && hw == warp * 32) ? xv0 : (ok ? __ldg(xrow + h) : zero4);
      float sum = 0.0f;
      if (ok) {
        const int blk = h >> 4, wl = h & 15;  // half-step wl = 4 t' + m2 of block blk
        xs[(blk * 4 + (wl & 3)) * pairs + 4 * b + (wl >> 2)] =
            make_uint4(__byte_perm(raw.x, raw.z, 0x5410), __byte_perm(raw.x, raw.z, 0x7632),
                       __byte_perm(raw.y, raw.w, 0x5410), __byte_perm(raw.y, raw.w, 0x7632));
        const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          sum += __uint_as_float(wv[i] << 16);
          sum += __uint_as_float(wv[i] & 0xFFFF0000u);
        }
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (ok && (lane & 15) == 0) xsum[(h >> 4) * batch + b] = sum;
    }
  }
  __syncthreads();

  float out[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int k0 = 0; k0 < my_blocks; k0 += kRegRound) {
    uint4 ca[kRegRound], cb[kRegRound];
#pragma unroll
    for (int i = 0; i < kRegRound; ++i) {
      ca[i] = wa[i];
      cb[i] = wb[i];
    }
    if (k0 + kRegRound < my_blocks) load_round(k0 + kRegRound);  // next round in flight meanwhile
#pragma unroll
    for (int i = 0; i < kRegRound; ++i) {
      if (k0 + i >= my_blocks) break;
      const int blk = warp + (k0 + i) * kRegWarps;
      const uint4* xb = xs + blk * 4 * pairs + lane;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int m2 = 0; m2 < 4; ++m2) {
        const uint32_t a = word_of(ca[i], m2), bw = word_of(cb[i], m2);
        const uint4 xv = lane < pairs ? xb[m2 * pairs] : zero4;
        mma_bf16_16816(acc, nib_pair(a, 0), nib_pair(bw, 0), nib_pair(a, 1), nib_pair(bw, 1), xv.x, xv.y);
        mma_bf16_16816(acc, nib_pair(a, 2), nib_pair(bw, 2), nib_pair(a, 3), nib_pair(bw, 3), xv.z, xv.w);
      }
      const int q = gmagic == 0u ? blk : static_cast<int>(__umulhi(static_cast<uint32_t>(blk), gmagic));  // blk / (G / 128)
      const float sa = ssc[g * n_groups + q], sb = ssc[(g + 8) * n_groups + q];
      out[0] = fmaf(sa, acc[0], out[0]);
      out[1] = fmaf(sa, acc[1], out[1]);
      out[2] = fmaf(sb, acc[2], out[2]);
      out[3] = fmaf(sb, acc[3], out[3]);
    }
  }

  float* rw = red + warp * 128;
  rw[g * 8 + 2 * t] = out[0];
  rw[g * 8 + 2 * t + 1] = out[1];
  rw[(g + 8) * 8 + 2 * t] = out[2];
  rw[(g + 8) * 8 + 2 * t + 1] = out[3];
  __syncthreads();
  // y[b, r] = sum over warps - sum_q s_rq (128 + z_rq) X_qb: T lanes per
  // output take groups q = sub, sub + T, ... and add in a shuffle tree; X_qb
  // adds the group's block sums in order.
  const int tlog = batch == 1 ? 4 : (batch == 2 ? 3 : (batch <= 4 ? 2 : 1));  // 16 x batch x T <= threads
  const int T = 1 << tlog;
  const int o = threadIdx.x >> tlog, sub = threadIdx.x & (T - 1);  // o = row * batch + b
  const int row = o / batch, b = o - row * batch;
  const bool live = o < 16 * batch && row < nrows;
  const int per_group = n_groups == 1 ? blocks : G / 128;
  float off = 0.0f;
  if (live) {
    for (int q = sub; q < n_groups; q += T) {
      const int k1 = min((q + 1) * per_group, blocks);
      float X = 0.0f;
      for (int k = q * per_group; k < k1; ++k) X += xsum[k * batch + b];
      const int e = row * n_groups + q;
      off = fmaf(ssc[e] * (128.0f + static_cast<float>(szp[e])), X, off);
    }
  }
  for (int w = 1; w < T; w <<= 1) off += __shfl_xor_sync(0xffffffffu, off, w);
  if (live && sub == 0) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kRegWarps; ++w) v += red[w * 128 + row * 8 + b];
    y[static_cast<int64_t>(b) * rows + r0 + row] = v - off;
  }
}

}  // namespace

// ceil(2^32 / d) for d = the blocks of 128 columns per group (all of them with
// one group per row): __umulhi(blk, magic) == blk / d for every block index
// blk < 2^16 (the rounding error blk * (magic * d - 2^32) / 2^32 stays below
// 1 / d there); the largest n the library takes keeps blk below 512.  d = 1
// (groups of 128) would need 2^32: 0 stands for it, and the kernel then takes
// blk itself.
uint32_t group_magic(int n, int G, int n_groups) {
  const uint64_t d = n_groups == 1 ? static_cast<uint64_t>(n / 128) : static_cast<uint64_t>(G / 128);
  return d == 1 ? 0u : static_cast<uint32_t>(((uint64_t(1) << 32) + d - 1) / d);
}

namespace {

gptq_status launch_reg4(const uint32_t* packed, const float* scales, const uint8_t* zeros, int64_t rows, int n, int G,
                        int n_groups, const __nv_bfloat16* x, int batch, float* y, const RegLayout& l,
                        cudaStream_t st) {
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GPTQ_ERR_CUDA;
  static std::atomic<bool> attr_set[64] = {};  // per device, shared by host threads
  if (!attr_set[info->device]) {
    if (cudaFuncSetAttribute(matvec_reg4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kRegMaxSmem)) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    attr_set[info->device] = true;
  }
  launch(matvec_reg4_kernel, static_cast<unsigned>(ceil_div(rows, 16)), kRegThreads, l.total, st, packed, scales,
         zeros, rows, n, G, n_groups, x, batch, y, group_magic(n, G, n_groups), static_cast<uint32_t>(l.xsum),
         static_cast<uint32_t>(l.red), static_cast<uint32_t>(l.sc), static_cast<uint32_t>(l.zp));
  return launch_status();
}

size_t smem_bytes(int B) {
  const int runs_chunk = (kChunkFloats / B) / 32;
  return (static_cast<size_t>(B) * runs_chunk * kRunPitch + static_cast<size_t>(B) * runs_chunk) * sizeof(float);
}

template <int BITS, int B, bool kFast, typename T>
gptq_status launch_matvec(const uint32_t* packed, const float* scales, const uint8_t* zeros, const int32_t* g_idx,
                          int64_t rows, int n, int G, int n_groups, const T* x, int batch, float* y,
                          cudaStream_t st) {
  const DeviceInfo* info = device_info();
  if (info == nullptr) return GPTQ_ERR_CUDA;
  const size_t smem = smem_bytes(B);
  static std::atomic<bool> attr_set[64] = {};  // per device, shared by host threads
  if (!attr_set[info->device]) {
    if (cudaFuncSetAttribute(dequant_matvec_kernel<BITS, B, kFast, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    attr_set[info->device] = true;
  }
  // as many CTAs as fit at once (x is staged once per CTA), each taking rows
  // in a grid-stride loop
  const int per_sm = std::max(1, std::min(8, static_cast<int>((228 * 1024) / (smem + 1024))));
  const int64_t ctas = std::min<int64_t>(ceil_div(rows, static_cast<int64_t>(kWarps)), int64_t(info->sm_count) * per_sm);
  launch(dequant_matvec_kernel<BITS, B, kFast, T>, static_cast<unsigned>(ctas), kThreads, smem, st, packed, scales, zeros,
         g_idx, rows, n, G, n_groups, x, batch, y);
  return launch_status();
}

template <int BITS, int B, typename T>
gptq_status dispatch_fast(bool fast, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                          const int32_t* g_idx, int64_t rows, int n, int G, int n_groups, const T* x, int batch,
                          float* y, cudaStream_t st) {
  return fast ? launch_matvec<BITS, B, true>(packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st)
              : launch_matvec<BITS, B, false>(packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
}

template <int BITS, typename T>
gptq_status dispatch_batch(bool fast, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                           const int32_t* g_idx, int64_t rows, int n, int G, int n_groups, const T* x, int batch,
                           float* y, cudaStream_t st) {
  if (batch <= 1) return dispatch_fast<BITS, 1>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
  if (batch <= 2) return dispatch_fast<BITS, 2>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
  if (batch <= 4) return dispatch_fast<BITS, 4>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
  return dispatch_fast<BITS, 8>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
}

template <typename T>
gptq_status dispatch_bits(int bits, bool fast, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                          const int32_t* g_idx, int64_t rows, int n, int G, int n_groups, const T* x, int batch,
                          float* y, cudaStream_t st) {
  switch (bits) {
    case 2: return dispatch_batch<2>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
    case 3: return dispatch_batch<3>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
    case 4: return dispatch_batch<4>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
    default: return dispatch_batch<8>(fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, x, batch, y, st);
  }
}

}  // namespace

size_t matvec_workspace_size(int, int, int) { return 0; }

gptq_status dequant_matvec(const uint32_t* packed, const float* scales, const uint8_t* zeros, const int32_t* g_idx,
                           int64_t rows, int n, int bits, int group, const void* x, int xdt_bf16, int batch, float* y,
                           void*, cudaStream_t st) {
  const int G = group > 0 ? group : n;
  const int n_groups = static_cast<int>(ceil_div(n, G));
  const bool fast = g_idx == nullptr && (G % 32 == 0 || G == n);
  // 4-bit codes and bf16 x in 128-column blocks that lie in one group: the
  // tensor-core path
  if (bits == 4 && xdt_bf16 && g_idx == nullptr && n % 128 == 0 && (n_groups == 1 || G % 128 == 0) &&
      reinterpret_cast<uintptr_t>(packed) % 16 == 0 && reinterpret_cast<uintptr_t>(x) % 16 == 0) {
    const RegLayout l = reg_layout(n, n_groups, batch);
    if (l.total <= kRegMaxSmem)
      return launch_reg4(packed, scales, zeros, rows, n, G, n_groups, static_cast<const __nv_bfloat16*>(x), batch, y,
                         l, st);
  }
  if (xdt_bf16)
    return dispatch_bits(bits, fast, packed, scales, zeros, g_idx, rows, n, G, n_groups,
                         static_cast<const __nv_bfloat16*>(x), batch, y, st);
  return dispatch_bits(bits, fast, packed, scales, zeros, g_idx, rows, n, G, n_groups, static_cast<const float*>(x),
                       batch, y, st);
}

}  // namespace gptq
