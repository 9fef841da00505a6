// Bit-packing of integer codes (GPTQ knowledge note, "Tradeoffs": deployment
// reads packed weights; encyclopedia "GPTQ", "Performance and Accuracy": 4-bit
// weights take half a byte each).
//
// Format (a reading; the pages give none): each row is a little-endian stream
// of 32-bit words, code j at bits [j*b, (j+1)*b); rows are padded with zero
// codes to a multiple of 32, so one run of 32 codes fills exactly b words.
// One thread packs one run: it reads 32 bytes (two 16-byte loads when the run
// is aligned) and writes b consecutive words, so both sides stay coalesced.
#include "common.cuh"

namespace gptq {
namespace {

template <int BITS>
__global__ void pack_kernel(const uint8_t* __restrict__ codes, int64_t rows, int n, uint32_t* __restrict__ packed,
                            bool vec_ok) {
  const int runs = (n + 31) / 32;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= rows * runs) return;
  const int64_t r = idx / runs;
  const int run = static_cast<int>(idx - r * runs);
  const uint8_t* src = codes + r * n + run * 32;
  const int cnt = min(32, n - run * 32);
  uint8_t c[32];
  if (vec_ok && cnt == 32) {
    const uint4 v0 = reinterpret_cast<const uint4*>(src)[0];
    const uint4 v1 = reinterpret_cast<const uint4*>(src)[1];
    const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int j = 0; j < 32; ++j) c[j] = static_cast<uint8_t>(u[j / 4] >> (8 * (j % 4)));
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) c[j] = j < cnt ? src[j] : 0;
  }
  constexpr uint32_t mask = (1u << BITS) - 1u;
  uint32_t w[BITS];
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] = 0u;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t v = c[j] & mask;
    const int bit = j * BITS;
    const int wi = bit / 32, off = bit % 32;
    w[wi] |= v << off;
    if (off + BITS > 32) w[wi + 1] |= v >> (32 - off);
  }
  uint32_t* dst = packed + r * static_cast<int64_t>(runs) * BITS + static_cast<int64_t>(run) * BITS;
#pragma unroll
  for (int k = 0; k < BITS; ++k) dst[k] = w[k];
}

}  // namespace

gptq_status pack_codes(const uint8_t* codes, int64_t rows, int n, int bits, uint32_t* packed, cudaStream_t st) {
  const int64_t runs = (n + 31) / 32;
  const int64_t total = rows * runs;
  if (total == 0) return GPTQ_OK;
  const unsigned grid = static_cast<unsigned>(ceil_div(total, 256));
  const bool vec_ok = (n % 16 == 0) && (reinterpret_cast<uintptr_t>(codes) % 16 == 0);
  switch (bits) {
    case 2: launch(pack_kernel<2>, grid, 256, 0, st, codes, rows, n, packed, vec_ok); break;
    case 3: launch(pack_kernel<3>, grid, 256, 0, st, codes, rows, n, packed, vec_ok); break;
    case 4: launch(pack_kernel<4>, grid, 256, 0, st, codes, rows, n, packed, vec_ok); break;
    case 8: launch(pack_kernel<8>, grid, 256, 0, st, codes, rows, n, packed, vec_ok); break;
    default: return GPTQ_ERR_INVALID_ARG;
  }
  return launch_status();
}

}  // namespace gptq
