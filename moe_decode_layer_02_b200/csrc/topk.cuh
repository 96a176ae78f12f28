// Top-k selection, softmax gates and routing tables.
//
// Selection order: larger logit first, equal logits by lower expert index; NaN logits
// rank below every number.  Gates are the softmax over the k selected logits
// (max-subtracted, fp32).  Source: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300
// with agent-assisted kernels", section "How the specialised decode path works"
// (16 of 896 experts per token); the renormalised softmax over the selected experts is
// the layer's stated gate function.
#pragma once
#include <cstddef>
#include <type_traits>
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kCandMax = 128;                              // candidates kept by the threshold pass
constexpr int kCandStride = 2 * kCandMax + 32;             // floats per candidate array
constexpr int kTopkScratch = 64 * 1024;                    // shared memory of the table builder
constexpr int kTopkCandBytes = 2 * 2 * kCandStride * 4;    // two warps' candidate arrays

namespace {

__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Exact top-K (K <= 32, E <= 1024) of one token's logits by one warp; lane j < K receives the
// j-th selection.  Lane l holds the logits of experts 128 i + 4 l + c (float4 loads when E is
// a multiple of 4).  Threshold pass: the K-th largest of the 32 lane maxima, T, is a lower
// bound of the K-th largest logit, so every selected expert is among the logits >= T.  Those
// C candidates are ranked exactly: with C <= 32 one per lane, through shuffles; with
// C <= kCandMax through shared memory; with more (mass ties) the warp falls back to K
// rounds of arg-max.  cand_v / cand_i: kCandStride floats / ints each.
__device__ void warp_topk(const float* logits, int E, int K, float* cand_v, int* cand_i, int lane, float& my_v,
                          int& my_i) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e0 = 128 * i + 4 * lane;
    if ((E & 3) == 0 && e0 + 3 < E) {
      const float4 f = ld_act4(logits + e0);
      v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) v[4 * i + c] = (e0 + c < E) ? ld_act(logits + e0 + c) : -INFINITY;
    }
  }
  float lm = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (v[i] != v[i]) v[i] = -INFINITY;  // NaN never outranks a number
    if (128 * (i >> 2) + 4 * lane + (i & 3) < E) lm = fmaxf(lm, v[i]);
  }
  int rank = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float o = __shfl_sync(0xffffffffu, lm, j);
    rank += (o > lm) || (o == lm && j < lane);
  }
  const unsigned who = __ballot_sync(0xffffffffu, rank == K - 1);
  const float T = __shfl_sync(0xffffffffu, lm, __ffs(who) - 1);
  int cnt = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) cnt += (128 * (i >> 2) + 4 * lane + (i & 3) < E && v[i] >= T);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int C = __shfl_sync(0xffffffffu, incl, 31);
  if (C <= kCandMax) {
    int w = incl - cnt;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = 128 * (i >> 2) + 4 * lane + (i & 3);
      if (e < E && v[i] >= T) {
        cand_v[w] = v[i];
        cand_i[w] = e;
        ++w;
      }
    }
    __syncwarp();
    if (C <= 32) {  // one candidate per lane, ranked through shuffles
      const float x = (lane < C) ? cand_v[lane] : -INFINITY;
      const int xi = (lane < C) ? cand_i[lane] : 0x7FFFFFFF;  // empty lanes rank last
      int r = 0;
#pragma unroll
      for (int o = 0; o < 32; ++o)
        r += better(__shfl_sync(0xffffffffu, x, o), __shfl_sync(0xffffffffu, xi, o), x, xi);
      if (lane < C && r < K) {
        cand_v[2 * kCandMax + r] = x;
        cand_i[2 * kCandMax + r] = xi;
      }
    } else {
      // The rank of a candidate among the candidates is its rank among all experts.
      for (int c = lane; c < C; c += 32) {
        const float cv = cand_v[c];
        const int ci = cand_i[c];
        int r = 0;
        for (int o = 0; o < C; ++o) r += better(cand_v[o], cand_i[o], cv, ci);
        cand_i[kCandMax + c] = r;
      }
      __syncwarp();
      for (int c = lane; c < C; c += 32) {
        const int r = cand_i[kCandMax + c];
        if (r < K) {
          cand_v[2 * kCandMax + r] = cand_v[c];
          cand_i[2 * kCandMax + r] = cand_i[c];
        }
      }
    }
    __syncwarp();
    if (lane < K) {
      my_v = cand_v[2 * kCandMax + lane];
      my_i = cand_i[2 * kCandMax + lane];
    }
    __syncwarp();
    return;
  }
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (128 * (i >> 2) + 4 * lane + (i & 3) >= E) taken |= 1u << i;
  float lbv = -INFINITY;
  int lbi = 0x7fffffff;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = 128 * (i >> 2) + 4 * lane + (i & 3);
    if (!((taken >> i) & 1u) && better(v[i], e, lbv, lbi)) { lbv = v[i]; lbi = e; }
  }
  for (int j = 0; j < K; ++j) {
    float bv = lbv;
    int bi = lbi;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if (lane == j) { my_v = bv; my_i = bi; }
    if (((bi & 127) >> 2) == lane) {  // the winner's lane marks it taken
      const int slot = 4 * (bi >> 7) + (bi & 3);
      taken |= 1u << slot;
      lbv = -INFINITY;
      lbi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int e = 128 * (i >> 2) + 4 * lane + (i & 3);
        if (!((taken >> i) & 1u) && better(v[i], e, lbv, lbi)) { lbv = v[i]; lbi = e; }
      }
    }
  }
}

// Gate of lane j (< K) given the warp's selections; returns the softmax weight.
__device__ __forceinline__ float warp_gate(float my_v, int lane, int K) {
  const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
  const float w = (lane < K) ? expf(my_v - v0) : 0.f;
  const float sum = warp_sum(w);
  return w / sum;
}

// Last-CTA ticket: true in the CTA that arrives last.  All threads call it.
__device__ __forceinline__ bool last_cta_s(unsigned* counter, int* s_flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(counter, 1u);
    *s_flag = (prev == gridDim.x - 1);
  }
  __syncthreads();
  const bool last = *s_flag != 0;
  if (last) __threadfence();
  return last;
}

// Routing tables in global memory for the large-batch expert kernels (every thread of one
// CTA): per-token top-k and gates, the union of selected experts in ascending order, and the
// entries (token, slot) of each union expert in CSR form, tokens ascending.  selected: the
// per-token top-k is already in ws.topk_idx / ws.topk_gate (and the caller's outputs), only
// the tables remain.
__device__ void topk_route(const LayerArgs& a, unsigned char* scratch, bool selected = false) {
  const int B = a.B, E = a.E, K = a.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(scratch);  // [1024] token bitmaps
  int* off_e = reinterpret_cast<int*>(mask + 1024);                         // [1024]
  int* sidx = off_e + 1024;                                                 // [64 * 32]
  int* rsum = sidx + 64 * 32;                                               // [32] per-round entry counts
  int* rnu = rsum + 32;                                                     // [32] per-round union counts
  float* cand = reinterpret_cast<float*>(rnu + 32);                         // [nwarps][2][kCandStride]
  float* cv = cand + warp * 2 * kCandStride;
  int* ci = reinterpret_cast<int*>(cv + kCandStride);

  for (int e = threadIdx.x; e < E; e += blockDim.x) mask[e] = 0ull;
  if (selected) {
    for (int p = threadIdx.x; p < B * K; p += blockDim.x) sidx[p] = ld_act_i(&a.ws.topk_idx[p]);
  }
  for (int t = warp; t < B && !selected; t += nwarps) {
    float my_v = 0.f;
    int my_i = 0;
    warp_topk(a.ws.logits + (size_t)t * E, E, K, cv, ci, lane, my_v, my_i);
    const float gte = warp_gate(my_v, lane, K);
    if (lane < K) {
      const int e = (my_i >= 0 && my_i < E) ? my_i : 0;
      if (e != my_i) atomicOr(a.ws.err, kErrBounds);
      a.ws.topk_idx[t * K + lane] = e;
      a.ws.topk_gate[t * K + lane] = gte;
      if (a.user_idx) a.user_idx[t * K + lane] = e;
      if (a.user_gate) a.user_gate[t * K + lane] = gte;
      sidx[t * K + lane] = e;
    }
  }
  __syncthreads();
  for (int p = threadIdx.x; p < B * K; p += blockDim.x) atomicOr(&mask[sidx[p]], 1ull << (p / K));
  __syncthreads();
  // Scan over experts in rounds of 32 (expert r*32 + lane): round sums, then the rounds'
  // bases, then per-round inclusive scans.  Consecutive experts sit in consecutive words.
  const int R = (E + 31) / 32;
  for (int r = warp; r < R; r += nwarps) {
    const int e = r * 32 + lane;
    const int c = e < E ? __popcll(mask[e]) : 0;
    const int s = __reduce_add_sync(0xffffffffu, c);
    const int f = __reduce_add_sync(0xffffffffu, c > 0 ? 1 : 0);
    if (lane == 0) { rsum[r] = s; rnu[r] = f; }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int bs = 0, bu = 0;
    for (int r = 0; r < R; ++r) {
      const int s = rsum[r], f = rnu[r];
      rsum[r] = bs;
      rnu[r] = bu;
      bs += s;
      bu += f;
    }
    *a.ws.n_union = bu;
    a.ws.union_off[bu] = bs;
  }
  __syncthreads();
  for (int r = warp; r < R; r += nwarps) {
    const int e = r * 32 + lane;
    const int c = e < E ? __popcll(mask[e]) : 0;
    int ic = c, iu = c > 0 ? 1 : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ic, o);
      const int z = __shfl_up_sync(0xffffffffu, iu, o);
      if (lane >= o) { ic += y; iu += z; }
    }
    if (e < E) {
      const int off = rsum[r] + ic - c;
      off_e[e] = off;
      if (c > 0) {
        const int u = rnu[r] + iu - 1;
        a.ws.union_e[u] = e;
        a.ws.union_off[u] = off;
      }
    }
  }
  __syncthreads();
  for (int p = threadIdx.x; p < B * K; p += blockDim.x) {
    const int t = p / K, j = p % K, e = sidx[p];
    const unsigned long long below = (t == 0) ? 0ull : (mask[e] & ((~0ull) >> (64 - t)));
    const int pos = off_e[e] + __popcll(below);
    a.ws.entry_tok[pos] = t;
    a.ws.entry_slot[pos] = j;
  }
}

}  // namespace

// Per-CTA routing of a batch of at most R (2 or kSmallB) tokens with at most 64 entries
// (tokens x top-k), in shared memory only.
constexpr int kSmallB = 4;
template <int R>
struct alignas(16) SmallRouteR {
  int U, n_ent;
  int un_e[64];        // union experts, ascending
  int un_off[65];      // entries of union expert u: [un_off[u], un_off[u + 1])
  int ent_tok[64];     // token of each entry (tokens ascending within an expert)
  float ent_gate[64];  // gate of each entry
  int idx[R][32];      // per-token selection, descending logit
  float gate[R][32];
};

// Threads of the CTA that runs route_small_cta.
constexpr int kRouteThreads = 512;
constexpr int kRouteGroups = kRouteThreads / 8;  // quarter-warp groups

// Scratch of route_small_cta.  Arrays read with 16-byte vector loads are 16-byte aligned.
template <int R>
struct alignas(16) RouteScratchR {
  alignas(16) float cv[R][kCandMax];         // candidate logits
  alignas(16) int ci[R][kCandMax];           // candidate experts
  alignas(16) float gmax[R][kRouteGroups];   // quarter-warp maxima
  float sel_v[R][32];                        // selection in rank order
  int sel_i[R][32];
  unsigned bm[R][32];                        // selected-expert bitmaps (E <= 1024)
  float T[R];                                // candidate bound per token
  int cnt[R];                                // candidates per token
};
// The routing scratch of a kernel holding NT tokens: sized for two tokens up to two (so the
// one- and two-token kernels share a layout), for kSmallB above.
template <int NT>
struct RouteOf {
  static constexpr int R = NT <= 2 ? 2 : kSmallB;
  using Route = SmallRouteR<R>;
  using Scratch = RouteScratchR<R>;
  static constexpr int kFbFloats = R * 2 * kCandStride;  // the mass-tie fallback's candidates
};
// Bytes of a routing scratch for r (2 or kSmallB) tokens: tables, scratch, fallback, alignment.
__host__ __device__ constexpr size_t route_bytes(int r) {
  return r <= 2 ? sizeof(SmallRouteR<2>) + sizeof(RouteScratchR<2>) + (size_t)2 * 2 * kCandStride * 4 + 128
                : sizeof(SmallRouteR<kSmallB>) + sizeof(RouteScratchR<kSmallB>) +
                      (size_t)kSmallB * 2 * kCandStride * 4 + 128;
}
static_assert(offsetof(RouteScratchR<2>, cv) % 16 == 0 && offsetof(RouteScratchR<2>, ci) % 16 == 0 &&
                  offsetof(RouteScratchR<2>, gmax) % 16 == 0 && offsetof(RouteScratchR<kSmallB>, ci) % 16 == 0 &&
                  offsetof(RouteScratchR<kSmallB>, gmax) % 16 == 0,
              "vector-loaded routing arrays must be 16-byte aligned");
static_assert(sizeof(SmallRouteR<2>) % 16 == 0 && sizeof(SmallRouteR<kSmallB>) % 16 == 0,
              "the routing scratch follows the tables");

namespace {

// CTA-wide routing of a batch of B <= NT <= kSmallB tokens, B * K <= 64 (all kRouteThreads
// threads call it; 5 barriers).
//  1. each thread loads its strided share of the logits (E <= 2 * kRouteThreads);
//     quarter-warp maxima go to shared memory;
//  2. T = the k-th largest of a token's group maxima (each group maximum ranked against
//     the others in parallel): k groups hold a logit >= T, so the k-th largest logit is >= T;
//  3. the logits >= T are compacted (one shared atomic per warp);
//  4. warp t ranks token t's candidates exactly (through shuffles when there are at most 32,
//     else through shared memory; with more than kCandMax, e.g. mass ties, it selects by
//     repeated arg-max instead), computes the gates and marks the selection in a bitmap;
//  5. warp 0 scans the bitmaps (word = lane) and places every entry: its union index and
//     its position in the (expert, token)-sorted entry list are a scan value plus a popcount
//     (per-token and union counts packed 8 bits each into one scanned word).
// Inlined: a separate (non-inlined) function measured twice as slow in the fused kernel.
template <int NT>
__device__ __forceinline__ void route_small_cta(const float* logits, int B, int E, int K, int* user_idx,
                                             float* user_gate, uint32_t* err, typename RouteOf<NT>::Route* rt,
                                             typename RouteOf<NT>::Scratch* sc,
                                             float* fallback_cand, bool write_user) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kPer = 2;  // logits per thread per token
  static_assert(NT >= 1 && NT <= kSmallB, "at most kSmallB tokens");
  float v[NT][kPer];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = tid + i * kRouteThreads;
      float x = -INFINITY;
      if (t < B && e < E) {
        x = ld_act(logits + (size_t)t * E + e);
        if (x != x) x = -INFINITY;
      }
      v[t][i] = x;
    }
  if (tid < NT) sc->cnt[tid] = 0;
  if (tid < NT * 32) (&sc->bm[0][0])[tid] = 0u;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float m = fmaxf(v[t][0], v[t][1]);
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((lane & 7) == 0 && t < B) sc->gmax[t][tid >> 3] = m;
  }
  __syncthreads();
  // (2) bound
  if (tid < B * kRouteGroups) {
    const int t = tid / kRouteGroups, gi = tid - t * kRouteGroups;
    const float m = sc->gmax[t][gi];
    int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
#pragma unroll
    for (int o = 0; o < kRouteGroups; o += 4) {
      const float4 x = *reinterpret_cast<const float4*>(&sc->gmax[t][o]);
      r0 += (x.x > m) || (x.x == m && o < gi);
      r1 += (x.y > m) || (x.y == m && o + 1 < gi);
      r2 += (x.z > m) || (x.z == m && o + 2 < gi);
      r3 += (x.w > m) || (x.w == m && o + 3 < gi);
    }
    if ((r0 + r1) + (r2 + r3) == K - 1) sc->T[t] = m;
  }
  __syncthreads();
  // (3) candidates
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    if (t >= B) break;
    const float T = sc->T[t];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = tid + i * kRouteThreads;
      const bool isc = e < E && v[t][i] >= T;
      const unsigned m = __ballot_sync(0xffffffffu, isc);
      int base = 0;
      if (lane == 0 && m) base = atomicAdd(&sc->cnt[t], __popc(m));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (isc) {
        const int slot = base + __popc(m & lt);
        if (slot < kCandMax) {
          sc->cv[t][slot] = v[t][i];
          sc->ci[t][slot] = e;
        }
      }
    }
  }
  __syncthreads();
  // (4) selection and gates, warp t for token t
  if (warp < B) {
    const int t = warp, C = sc->cnt[t];
    if (C <= 32) {
      const float x = (lane < C) ? sc->cv[t][lane] : -INFINITY;
      const int xi = (lane < C) ? sc->ci[t][lane] : 0x7FFFFFFF;  // empty lanes rank last
      int r = 0;
#pragma unroll
      for (int o = 0; o < 32; ++o) r += better(__shfl_sync(0xffffffffu, x, o), __shfl_sync(0xffffffffu, xi, o), x, xi);
      if (lane < C && r < K) {
        sc->sel_v[t][r] = x;
        sc->sel_i[t][r] = xi;
      }
    } else if (C <= kCandMax) {
      for (int c = lane; c < C; c += 32) {
        const float x = sc->cv[t][c];
        const int xi = sc->ci[t][c];
        int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
        for (int o = 0; o < C; o += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(&sc->cv[t][o]);
          const int4 i4 = *reinterpret_cast<const int4*>(&sc->ci[t][o]);
          r0 += better(v4.x, i4.x, x, xi);
          r1 += (o + 1 < C) && better(v4.y, i4.y, x, xi);
          r2 += (o + 2 < C) && better(v4.z, i4.z, x, xi);
          r3 += (o + 3 < C) && better(v4.w, i4.w, x, xi);
        }
        const int r = (r0 + r1) + (r2 + r3);
        if (r < K) {
          sc->sel_v[t][r] = x;
          sc->sel_i[t][r] = xi;
        }
      }
    }
    __syncwarp();
    float my_v = 0.f;
    int my_i = 0;
    if (C > kCandMax) {
      float* cvv = fallback_cand + t * 2 * kCandStride;
      warp_topk(logits + (size_t)t * E, E, K, cvv, reinterpret_cast<int*>(cvv + kCandStride), lane, my_v, my_i);
    } else if (lane < K) {
      my_v = sc->sel_v[t][lane];
      my_i = sc->sel_i[t][lane];
    }
    const float gte = warp_gate(my_v, lane, K);
    if (lane < K) {
      const int e = (my_i >= 0 && my_i < E) ? my_i : 0;
      if (e != my_i) atomicOr(err, kErrBounds);
      rt->idx[t][lane] = e;
      rt->gate[t][lane] = gte;
      atomicOr(&sc->bm[t][e >> 5], 1u << (e & 31));
      if (write_user) {
        if (user_idx) user_idx[t * K + lane] = e;
        if (user_gate) user_gate[t * K + lane] = gte;
      }
    }
  }
  __syncthreads();
  // (5) entries sorted by (expert, token); union experts ascending (warp 0)
  if (warp == 0) {
    using Pack = typename std::conditional<(NT + 1) * 8 <= 32, unsigned, unsigned long long>::type;
    unsigned bw[NT];
    unsigned un = 0;
    Pack own = 0;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      bw[t] = sc->bm[t][lane];
      un |= bw[t];
      own |= (Pack)__popc(bw[t]) << (8 * t);
    }
    own |= (Pack)__popc(un) << (8 * NT);  // every field's total is <= 64
    Pack inc = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const Pack y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const Pack base = inc - own;
    const int n = B * K;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int p = lane + 32 * h;
      const int t = (p < n) ? p / K : 0, j = (p < n) ? p - t * K : 0;
      const int e = rt->idx[t][j], w = e >> 5;
      const unsigned below = (1u << (e & 31)) - 1u;
      const Pack bs = __shfl_sync(0xffffffffu, base, w);
      int pe = 0;
      unsigned wu = 0;
      bool earlier = false;  // a lower token selected e too
#pragma unroll
      for (int tt = 0; tt < NT; ++tt) {
        const unsigned wt = __shfl_sync(0xffffffffu, bw[tt], w);
        wu |= wt;
        pe += (int)((bs >> (8 * tt)) & 0xFFu) + __popc(wt & below);
        if (tt < t && ((wt >> (e & 31)) & 1u)) {
          ++pe;
          earlier = true;
        }
      }
      const int pu = (int)((bs >> (8 * NT)) & 0xFFu) + __popc(wu & below);
      if (p < n) {
        rt->ent_tok[pe] = t;
        rt->ent_gate[pe] = rt->gate[t][j];
        if (!earlier) {  // first entry of expert e
          rt->un_e[pu] = e;
          rt->un_off[pu] = pe;
        }
      }
    }
    if (lane == 31) {
      const int u = (int)((inc >> (8 * NT)) & 0xFFu);
      rt->U = u;
      rt->n_ent = n;
      rt->un_off[u] = n;
    }
  }
  __syncthreads();
}

}  // namespace

}  // namespace moe
