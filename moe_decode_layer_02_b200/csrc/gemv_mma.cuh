// Weight-streaming GEMV on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate).
//
// Decode GEMVs multiply many weight rows by a handful of activation vectors.  Here
// the weight rows are the MMA's N operand (8 rows per instruction) and the tokens are
// its M operand (up to 16 activation rows), so one instruction consumes a 8 x 16
// block of weights with no unpacking: about 5 instructions per 256 weight bytes
// instead of ~2 per weight element on the CUDA cores.  Activations that exist in fp32
// (the RMSNorm output x, the SwiGLU activation a) are split into two bf16 rows,
// hi = bf16(v) and lo = bf16(v - hi), so hi + lo carries v to ~2^-17 relative; the
// products are exact and accumulate in fp32.
//
// Shared-memory layout of a stage: up to 8 weight rows, each a K-chunk of Kc bf16
// copied by its own 1-D bulk copy to a row pitch of Kc*2 + 16 bytes.  With Kc a
// multiple of 64 the pitch is 4 banks past a multiple of 128 bytes, so the eight rows
// of a fragment load start in distinct bank quads and every load is conflict-free.
// Activation rows use the same padding (pitch K*2 + 16).
//
// Fragment ownership (PTX ISA, mma.m16n8k16 with .row.col and 16-bit inputs):
//   lane l, g = l/4, q = l%4
//   A (activations, M x K, row):  a0 = A[g][2q..2q+1], a2 = A[g][2q+8..2q+9]  (rows g < 8;
//                                 a1, a3 are rows g+8, always zero here)
//   B (weights, K x N, col):      b0 = W[row g][2q..2q+1], b1 = W[row g][2q+8..2q+9]
//   D (M x N, fp32):              d0 = D[g][2q], d1 = D[g][2q+1]  (d2, d3: rows g+8, unused)
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kGroupRows = 8;  // weight rows per MMA group

__host__ __device__ __forceinline__ int pitch_bytes(int kc) { return kc * 2 + 16; }

__device__ __forceinline__ void mma_bf16_16816(float* d, uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// One warp's share of a stage: k16-steps [s0, s1) of the chunk [k0, k0 + Kc).
//   stage: weight rows (pitch wp), act: activation rows (pitch ap, M rows valid)
__device__ __forceinline__ void mma_stage(float* d, const unsigned char* stage, int wp, const unsigned char* act,
                                          int ap, int M, int k0, int s0, int s1, int lane) {
  const int g = lane >> 2, q = lane & 3;
  const unsigned char* wrow = stage + g * wp + q * 4;
  const bool has_a = g < M;
  const unsigned char* arow = act + (has_a ? g : 0) * ap + (size_t)k0 * 2 + q * 4;
#pragma unroll 4
  for (int s = s0; s < s1; ++s) {
    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(wrow + s * 32);
    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(wrow + s * 32 + 16);
    uint32_t a0 = 0, a2 = 0;
    if (has_a) {
      a0 = *reinterpret_cast<const uint32_t*>(arow + s * 32);
      a2 = *reinterpret_cast<const uint32_t*>(arow + s * 32 + 16);
    }
    mma_bf16_16816(d, a0, a2, b0, b1);
  }
}

// fp32 -> (hi, lo) bf16 pair with hi + lo ~= v.
__device__ __forceinline__ void split_bf16(float v, uint16_t& hi, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
  hi = *reinterpret_cast<const uint16_t*>(&h);
  lo = *reinterpret_cast<const uint16_t*>(&l);
}

// Writes the 8 warps' partial D (rows m < M of the MMA tile) to red[w][m][n].
__device__ __forceinline__ void mma_store_partial(float* red, const float* d, int M, int warp, int lane) {
  const int g = lane >> 2, q = lane & 3;
  if (g < M) {
    red[(warp * 8 + g) * 8 + 2 * q] = d[0];
    red[(warp * 8 + g) * 8 + 2 * q + 1] = d[1];
  }
}

// Sum over the 8 warps (fixed order) of red[.][m][n].
__device__ __forceinline__ float mma_reduce(const float* red, int m, int n) {
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) s += red[(w * 8 + m) * 8 + n];
  return s;
}

// k16-steps of warp w when S steps are shared by the consumer warps.
__device__ __forceinline__ void warp_steps(int S, int w, int& s0, int& s1) {
  s0 = S * w / kConsumerWarps;
  s1 = S * (w + 1) / kConsumerWarps;
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------------------
// Register-streamed variant: weights go from global memory straight into the B fragments.
//
// One warp covers 8 weight rows x one 64-element k-block per step.  Lane (g, q) loads
// two 16-byte vectors of row g: elements [8q, 8q+8) and [32+8q, 32+8q+8) of the block, so
// each load instruction reads 64 contiguous bytes of every row (no shared memory, no
// unpacking).  The MMA's logical k order is a permutation of the block's 64 elements;
// the same permutation is applied to the activations, so the products and the sum over
// the block are unchanged:
//   step 0: lane q's words 0,1 of the first vector (elements 8q + 0..3)
//   step 1: words 2,3 of the first vector (8q + 4..7)
//   step 2: words 0,1 of the second vector (32 + 8q + 0..3)
//   step 3: words 2,3 of the second vector (32 + 8q + 4..7)
// with a0/b0 the first word of a step and a2/b1 the second.
// ---------------------------------------------------------------------------------------
struct Frag {
  uint4 lo, hi;  // elements [8q, 8q+8) and [32+8q, 32+8q+8) of a 64-element block
};

// 128-bit weight load with an L2 256-byte fetch hint (static weights only).
__device__ __forceinline__ uint4 ld_w128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Weight fragment of k-block starting at `row_kb` (row base + 64*kb elements); zeros if !ok.
__device__ __forceinline__ void load_wfrag(Frag& f, const uint16_t* row_kb, int q, bool ok) {
  if (ok) {
    f.lo = ld_w128(row_kb + 8 * q);
    f.hi = ld_w128(row_kb + 32 + 8 * q);
  } else {
    f.lo = make_uint4(0, 0, 0, 0);
    f.hi = make_uint4(0, 0, 0, 0);
  }
}

// Activation fragment (bf16 row in shared memory, `row_kb` = row + 64*kb elements).
__device__ __forceinline__ void load_afrag(Frag& f, const uint16_t* row_kb, int q, bool ok) {
  if (ok) {
    f.lo = *reinterpret_cast<const uint4*>(row_kb + 8 * q);
    f.hi = *reinterpret_cast<const uint4*>(row_kb + 32 + 8 * q);
  } else {
    f.lo = make_uint4(0, 0, 0, 0);
    f.hi = make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 64-element k-block: activation rows g (ag) and g + 8 (ag8) against weight rows.
__device__ __forceinline__ void mma_kblock(float* d, const Frag& ag, const Frag& ag8, const Frag& w) {
  mma16816(d, ag.lo.x, ag8.lo.x, ag.lo.y, ag8.lo.y, w.lo.x, w.lo.y);
  mma16816(d, ag.lo.z, ag8.lo.z, ag.lo.w, ag8.lo.w, w.lo.z, w.lo.w);
  mma16816(d, ag.hi.x, ag8.hi.x, ag.hi.y, ag8.hi.y, w.hi.x, w.hi.y);
  mma16816(d, ag.hi.z, ag8.hi.z, ag.hi.w, ag8.hi.w, w.hi.z, w.hi.w);
}

// D fragment ownership: lane (g, q): d0 = D[g][2q], d1 = D[g][2q+1], d2 = D[g+8][2q], d3 = D[g+8][2q+1]
// (rows = activation rows, columns = weight rows).  Writes all of it to red[16][8].
__device__ __forceinline__ void store_d(float* red, const float* d, int lane) {
  const int g = lane >> 2, q = lane & 3;
  red[g * 8 + 2 * q] = d[0];
  red[g * 8 + 2 * q + 1] = d[1];
  red[(g + 8) * 8 + 2 * q] = d[2];
  red[(g + 8) * 8 + 2 * q + 1] = d[3];
}

}  // namespace moe
