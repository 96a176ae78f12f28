// Device-side fill for the seeded synthetic inputs (same bits as the host
// generator in synth/__init__.py): Philox4x32-10 (Salmon et al., SC'11) maps
// the counter of each 8-element block to four 32-bit words; each 16-bit half
// indexes a 65536-entry bf16 quantile table built on the host.  Integer work
// only, so host and device agree bit for bit.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ void philox_round(uint32_t c[4], uint32_t k0, uint32_t k1) {
  const uint32_t m0 = 0xD2511F53u, m1 = 0xCD9E8D57u;
  uint32_t hi0 = __umulhi(m0, c[0]), lo0 = m0 * c[0];
  uint32_t hi1 = __umulhi(m1, c[2]), lo1 = m1 * c[2];
  uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
  c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
}

__global__ void fill_kernel(uint16_t* __restrict__ dst, unsigned long long count,
                            unsigned long long start, uint32_t key0, uint32_t key1,
                            uint32_t sid, uint32_t attempt,
                            const uint16_t* __restrict__ table) {
  const unsigned long long b_first = start / 8;
  const unsigned long long b_last = (start + count + 7) / 8;
  for (unsigned long long b = b_first + blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x;
       b < b_last; b += (unsigned long long)gridDim.x * blockDim.x) {
    uint32_t c[4] = {(uint32_t)b, (uint32_t)(b >> 32), sid, attempt};
    uint32_t k0 = key0, k1 = key1;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
      if (r) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
      philox_round(c, k0, k1);
    }
    const unsigned long long n0 = b * 8;
    if (n0 >= start && n0 + 8 <= start + count && ((n0 - start) & 7) == 0 &&
        ((reinterpret_cast<uintptr_t>(dst + (n0 - start)) & 15) == 0)) {
      uint4 v;
      v.x = (uint32_t)table[c[0] & 0xFFFF] | ((uint32_t)table[c[0] >> 16] << 16);
      v.y = (uint32_t)table[c[1] & 0xFFFF] | ((uint32_t)table[c[1] >> 16] << 16);
      v.z = (uint32_t)table[c[2] & 0xFFFF] | ((uint32_t)table[c[2] >> 16] << 16);
      v.w = (uint32_t)table[c[3] & 0xFFFF] | ((uint32_t)table[c[3] >> 16] << 16);
      *reinterpret_cast<uint4*>(dst + (n0 - start)) = v;
    } else {
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        unsigned long long n = n0 + h;
        if (n >= start && n < start + count) {
          uint32_t w = c[h >> 1];
          dst[n - start] = table[(h & 1) ? (w >> 16) : (w & 0xFFFF)];
        }
      }
    }
  }
}

}  // namespace

extern "C" int synth_fill_bf16(void* dst, unsigned long long count, unsigned long long start,
                               unsigned long long seed, unsigned int sid, unsigned int attempt,
                               const void* table_dev, void* stream) {
  if (count == 0) return 0;
  if (!dst || !table_dev) return -1;
  const unsigned long long blocks8 = (start + count + 7) / 8 - start / 8;
  unsigned long long grid = (blocks8 + 255) / 256;
  if (grid > 148ull * 16) grid = 148ull * 16;
  fill_kernel<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(
      (uint16_t*)dst, count, start, (uint32_t)seed, (uint32_t)(seed >> 32), sid, attempt,
      (const uint16_t*)table_dev);
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}
