/*
 * Host-side fill for the seeded synthetic inputs: the same generator as the numpy
 * implementation in synth/__init__.py and the device fill in synth_fill.cu, in plain C
 * with OpenMP so that whole expert slabs can be regenerated quickly on the host.
 * Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as
 * 1, 2, 3", SC'11) maps the counter of each 8-element block to four 32-bit words; each
 * 16-bit half indexes a 65536-entry bf16 quantile table built in Python.  Integer work
 * only, so the three implementations agree bit for bit (a CPU test checks it).
 */
#include <stdint.h>

static void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
  const uint32_t m0 = 0xD2511F53u, m1 = 0xCD9E8D57u;
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = (uint64_t)m0 * c[0], p1 = (uint64_t)m1 * c[2];
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c[1] ^ k0, n1 = (uint32_t)p1;
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c[3] ^ k1, n3 = (uint32_t)p0;
    c[0] = n0;
    c[1] = n1;
    c[2] = n2;
    c[3] = n3;
  }
}

/* dst[i] = table[draw(start + i)] for i < count; returns 0, or -1 on a null pointer. */
int synth_host_fill_bf16(uint16_t* dst, unsigned long long count, unsigned long long start,
                         unsigned long long seed, unsigned int sid, unsigned int attempt,
                         const uint16_t* table) {
  if (count == 0) return 0;
  if (!dst || !table) return -1;
  const long long b0 = (long long)(start / 8), b1 = (long long)((start + count + 7) / 8);
  const uint32_t key0 = (uint32_t)seed, key1 = (uint32_t)(seed >> 32);
#pragma omp parallel for schedule(static)
  for (long long b = b0; b < b1; ++b) {
    uint32_t c[4] = {(uint32_t)b, (uint32_t)((unsigned long long)b >> 32), sid, attempt};
    philox4x32_10(c, key0, key1);
    const unsigned long long n0 = (unsigned long long)b * 8;
    for (int h = 0; h < 8; ++h) {
      const unsigned long long n = n0 + h;
      if (n >= start && n < start + count) {
        const uint32_t w = c[h >> 1];
        dst[n - start] = table[(h & 1) ? (w >> 16) : (w & 0xFFFFu)];
      }
    }
  }
  return 0;
}
