// Weight-streaming dot products shared by the streaming kernels: one producer warp moves
// whole weight rows into a shared-memory ring; 15 consumer warps split K, hold their slice
// of the activations in registers as fp32 and accumulate in fp32.
#pragma once
#include "common.cuh"

namespace moe {

namespace {

// 15 consumer warps + the producer = 16 warps, four per SM sub-partition, which leaves 128
// registers per thread (a 17th warp would cut that to 96).  The dot products are latency-
// bound chains of shared-memory loads and FMAs, so warps in flight are what keep the
// consumers ahead of HBM.
constexpr int kCW = 15;              // consumer warps
constexpr int kCT = kCW * 32;        // consumer threads
constexpr int kThreadsS = kCT + 32;  // + one producer warp
constexpr int kCPLf = 3;             // 8-element chunks per lane: K <= 15 warps * 32 lanes * 3 * 8 = 11520

__device__ __forceinline__ void csync() { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }

__device__ __forceinline__ size_t al128(size_t x) { return (x + 127) & ~size_t(127); }

__device__ __forceinline__ void unpack8f(uint4 w, float* f) {
  f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
  f[4] = bf16lo(w.z); f[5] = bf16hi(w.z); f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
}

// Chunk of lane `lane` in warp w's K slice: q = w * qpw + j * 32 + lane, valid if j*32+lane < qpw.
__device__ __forceinline__ bool cvalid(int qpw, int j, int lane) { return j * 32 + lane < qpw; }

// 16 bytes from shared memory at a 32-bit shared-window address.  The row pointers of the dot
// products below all point into the ring in shared memory; addressing them through the shared
// window keeps the per-chunk address arithmetic 32-bit (with generic pointers the same loop
// measured about 15% slower).  volatile: the load stays after the mbarrier wait that made the
// stage's bytes visible, like every other volatile asm around it.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ float4 lds128f(uint32_t addr) {
  const uint4 v = lds128(addr);
  return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
}

// Loads the chunks of R rows (row pointers into shared memory) that lane `lane` covers; rows
// r >= nr and chunks past the warp's slice read as zeros.
template <int R, int CPL>
__device__ __forceinline__ void load_row_chunks(const uint16_t* const (&rp)[R], int nr, int qbase, int qpw, int lane,
                                                uint4 (&w)[R][CPL]) {
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(rp[r]) + (uint32_t)(qbase + lane) * 16u;
#pragma unroll
    for (int j = 0; j < CPL; ++j)
      w[r][j] = (r < nr && cvalid(qpw, j, lane)) ? lds128(base + (uint32_t)j * 512u) : make_uint4(0, 0, 0, 0);
  }
}

// d = a * b + d on a pair of fp32 lanes with one instruction (sm_100 packed FMA; each lane
// rounds exactly like fmaf).
__device__ __forceinline__ void ffma2(float2& d, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rd, {%0, %1};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rd;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d.x), "+f"(d.y)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Per-lane partial dots of R bf16 rows (shared memory only) with NT register slices of the
// activations: out[r * NT + t].  Rows r >= nr contribute zeros.  All chunk loads of all
// rows are issued before the first FMA; the accumulators are independent chains of packed
// FMAs (an even and an odd element per instruction, kA pairs per row and token), so a
// warp's pass over a stage is one short chain instead of R dependent ones.
// CPL: 8-element chunks per lane of the activation slice (deduced from x).
template <int NT, int R, int CPL>
__device__ __forceinline__ void rows_dot(const uint16_t* const (&rp)[R], int nr, const float (&x)[NT][CPL][8],
                                         int qbase, int qpw, int lane, float (&out)[R * NT]) {
  constexpr int kA = (R * NT >= 4) ? 1 : 4 / (R * NT);  // accumulator pairs per (row, token)
  uint4 w[R][CPL];
  load_row_chunks<R, CPL>(rp, nr, qbase, qpw, lane, w);
  float2 acc[R][NT][kA];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int e = 0; e < kA; ++e) acc[r][t][e] = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < CPL; ++j)
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float wf[8];
      unpack8f(w[r][j], wf);
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          ffma2(acc[r][t][e % kA], wf[2 * e], wf[2 * e + 1], x[t][j][2 * e], x[t][j][2 * e + 1]);
    }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float v = 0.f;
#pragma unroll
      for (int e = 0; e < kA; ++e) v += acc[r][t][e].x + acc[r][t][e].y;
      out[r * NT + t] = v;
    }
}

// d = a * b + c for the bf16 in the low (hi = false) or high half of a and of b, in fp32: the
// product of two bf16 values is exact in fp32, so this rounds exactly like fmaf on the
// unpacked values (one instruction instead of two unpacks and an FMA).
template <bool HI>
__device__ __forceinline__ float fma_bf16(uint32_t a, uint32_t b, float c) {
  float d;
  if (HI)
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
  else
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
  return d;
}

// rows_dot for an activation that is itself bf16 (attn_out): x is kept packed, 8 values per
// uint4 chunk, and each product is one mixed-precision FMA.  The accumulators and their order
// are rows_dot's (even elements in .x, odd in .y, kA pairs), so the sums are bit-identical.
template <int NT, int R, int CPL>
__device__ __forceinline__ void rows_dot_bf(const uint16_t* const (&rp)[R], int nr, const uint4 (&x)[NT][CPL],
                                            int qbase, int qpw, int lane, float (&out)[R * NT]) {
  constexpr int kA = (R * NT >= 4) ? 1 : 4 / (R * NT);
  uint4 w[R][CPL];
  load_row_chunks<R, CPL>(rp, nr, qbase, qpw, lane, w);
  float2 acc[R][NT][kA];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int e = 0; e < kA; ++e) acc[r][t][e] = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < CPL; ++j)
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint32_t wv[4] = {w[r][j].x, w[r][j].y, w[r][j].z, w[r][j].w};
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const uint32_t xv[4] = {x[t][j].x, x[t][j].y, x[t][j].z, x[t][j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2& a = acc[r][t][e % kA];
          a.x = fma_bf16<false>(wv[e], xv[e], a.x);
          a.y = fma_bf16<true>(wv[e], xv[e], a.y);
        }
      }
    }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float v = 0.f;
#pragma unroll
      for (int e = 0; e < kA; ++e) v += acc[r][t][e].x + acc[r][t][e].y;
      out[r * NT + t] = v;
    }
}

// rows_dot_bf for a K slice laid out as two full 32-lane chunk rounds per warp at qbase (64
// chunks) plus, in the warps with has_x (warp-uniform), one more round at qx, valid below nch:
// for K above 15 warps x 64 chunks (d_o up to 8192), where an even split over the 15 warps
// would give every warp a third round that is nearly empty (4 of 32 lanes at d_o = 8192), and
// its FMAs on zeros.  x[t][2] holds the extra round's chunk.  Same accumulators as rows_dot_bf;
// the extra round is added last.
template <int NT, int R>
__device__ __forceinline__ void rows_dot_bf_2x(const uint16_t* const (&rp)[R], int nr, const uint4 (&x)[NT][3],
                                               int qbase, int qx, int nch, bool has_x, int lane,
                                               float (&out)[R * NT]) {
  constexpr int kA = (R * NT >= 4) ? 1 : 4 / (R * NT);
  uint4 w[R][3];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(rp[r]);
    w[r][0] = (r < nr) ? lds128(base + (uint32_t)(qbase + lane) * 16u) : make_uint4(0, 0, 0, 0);
    w[r][1] = (r < nr) ? lds128(base + (uint32_t)(qbase + 32 + lane) * 16u) : make_uint4(0, 0, 0, 0);
    w[r][2] = (has_x && r < nr && qx + lane < nch) ? lds128(base + (uint32_t)(qx + lane) * 16u)
                                                   : make_uint4(0, 0, 0, 0);
  }
  float2 acc[R][NT][kA];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int e = 0; e < kA; ++e) acc[r][t][e] = make_float2(0.f, 0.f);
  auto round = [&](int j) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint32_t wv[4] = {w[r][j].x, w[r][j].y, w[r][j].z, w[r][j].w};
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const uint32_t xv[4] = {x[t][j].x, x[t][j].y, x[t][j].z, x[t][j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2& a = acc[r][t][e % kA];
          a.x = fma_bf16<false>(wv[e], xv[e], a.x);
          a.y = fma_bf16<true>(wv[e], xv[e], a.y);
        }
      }
    }
  };
  round(0);
  round(1);
  if (has_x) round(2);
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float v = 0.f;
#pragma unroll
      for (int e = 0; e < kA; ++e) v += acc[r][t][e].x + acc[r][t][e].y;
      out[r * NT + t] = v;
    }
}

// Warp sums of V per-lane values (V a power of two <= 32) with V - 1 + 5 - log2(V) shuffles
// instead of 5 V: each halving step sends one value of every pair across the current lane
// bit and keeps the other.  Every lane returns the total of value multi_index<V>(lane).
template <int V>
__device__ __forceinline__ float warp_reduce_multi(float (&v)[V], int lane) {
  static_assert(V >= 1 && V <= 32 && (V & (V - 1)) == 0, "V must be a power of two <= 32");
#pragma unroll
  for (int o = 16, c = V; c > 1; o >>= 1, c >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < c / 2; ++j) {
      const float send = up ? v[2 * j] : v[2 * j + 1];
      const float keep = up ? v[2 * j + 1] : v[2 * j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float s = v[0];
#pragma unroll
  for (int o = 16 / V; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// Value index held by `lane` after warp_reduce_multi<V>: bit k of the index is lane bit 4 - k.
template <int V>
__device__ __forceinline__ int multi_index(int lane) {
  int idx = 0;
#pragma unroll
  for (int k = 0, c = V; c > 1; ++k, c >>= 1) idx |= ((lane >> (4 - k)) & 1) << k;
  return idx;
}

// One lane per group of 32 / V holds each total.
template <int V>
__device__ __forceinline__ bool multi_writer(int lane) {
  return (lane & (32 / V - 1)) == 0;
}

}  // namespace

}  // namespace moe
