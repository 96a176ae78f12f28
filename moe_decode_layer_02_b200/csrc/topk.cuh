// Top-k selection, softmax gates and routing tables.
//
// Selection order: larger logit first, equal logits by lower expert index; NaN logits
// rank below every number.  Gates are the softmax over the k selected logits
// (max-subtracted, fp32).  Source: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300
// with agent-assisted kernels", section "How the specialised decode path works"
// (16 of 896 experts per token); the renormalised softmax over the selected experts is
// the layer's stated gate function.
#pragma once
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
// j-th selection.  Threshold pass: the K-th largest of the 32 lane maxima, T, is a lower
// bound of the K-th largest logit, so every selected expert is among the logits >= T.  Those
// candidates are ranked exactly; with more than kCandMax of them (mass ties) the warp falls
// back to K rounds of arg-max.  cand_v / cand_i: kCandStride floats / ints each.
__device__ void warp_topk(const float* logits, int E, int K, float* cand_v, int* cand_i, int lane, float& my_v,
                          int& my_i) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = (lane + 32 * i < E) ? ld_act(logits + lane + 32 * i) : -INFINITY;
  float lm = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (v[i] != v[i]) v[i] = -INFINITY;  // NaN never outranks a number
    if (lane + 32 * i < E) lm = fmaxf(lm, v[i]);
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
  for (int i = 0; i < 32; ++i) cnt += (lane + 32 * i < E && v[i] >= T);
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
    for (int i = 0; i < 32; ++i)
      if (lane + 32 * i < E && v[i] >= T) {
        cand_v[w] = v[i];
        cand_i[w] = lane + 32 * i;
        ++w;
      }
    __syncwarp();
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
    if (lane + 32 * i >= E) taken |= 1u << i;
  float lbv = -INFINITY;
  int lbi = 0x7fffffff;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (!((taken >> i) & 1u) && better(v[i], lane + 32 * i, lbv, lbi)) { lbv = v[i]; lbi = lane + 32 * i; }
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
    if ((bi & 31) == lane) {
      taken |= 1u << (bi >> 5);
      lbv = -INFINITY;
      lbi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!((taken >> i) & 1u) && better(v[i], lane + 32 * i, lbv, lbi)) { lbv = v[i]; lbi = lane + 32 * i; }
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
// entries (token, slot) of each union expert in CSR form, tokens ascending.
__device__ void topk_route(const LayerArgs& a, unsigned char* scratch) {
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
  for (int t = warp; t < B; t += nwarps) {
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

// Per-CTA routing of a batch of at most 2 tokens (shared memory only).
struct SmallRoute {
  int U, n_ent;
  int un_e[64];
  int un_off[65];
  int ent_tok[64];
  float ent_gate[64];
  int key[64];
  int idx[2][32];
  float gate[2][32];
};

namespace {

// Every thread of the CTA calls it (two __syncthreads).  Warps 0..B-1 select; warp 0 sorts
// the entries by (expert, token) and marks the union.  write_user: store idx / gates to the
// caller's buffers.
__device__ void route_small(const LayerArgs& a, SmallRoute* rt, float* cand, bool write_user) {
  const int B = a.B, E = a.E, K = a.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < B) {
    float* cv = cand + warp * 2 * kCandStride;
    int* ci = reinterpret_cast<int*>(cv + kCandStride);
    float my_v = 0.f;
    int my_i = 0;
    warp_topk(a.ws.logits + (size_t)warp * E, E, K, cv, ci, lane, my_v, my_i);
    const float gte = warp_gate(my_v, lane, K);
    if (lane < K) {
      const int e = (my_i >= 0 && my_i < E) ? my_i : 0;
      if (e != my_i) atomicOr(a.ws.err, kErrBounds);
      rt->idx[warp][lane] = e;
      rt->gate[warp][lane] = gte;
      if (write_user) {
        if (a.user_idx) a.user_idx[warp * K + lane] = e;
        if (a.user_gate) a.user_gate[warp * K + lane] = gte;
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int n = B * K;  // <= 64, keys unique (a token selects an expert at most once)
    for (int p = lane; p < n; p += 32) {
      const int t = p / K, j = p % K;
      const int key = rt->idx[t][j] * 2 + t;
      int r = 0;
      for (int o = 0; o < n; ++o) r += (rt->idx[o / K][o % K] * 2 + o / K) < key;
      rt->key[r] = key;
      rt->ent_tok[r] = t;
      rt->ent_gate[r] = rt->gate[t][j];
    }
    __syncwarp();
    int base = 0;
    for (int p0 = 0; p0 < n; p0 += 32) {
      const int p = p0 + lane;
      const bool first = p < n && (p == 0 || (rt->key[p - 1] >> 1) != (rt->key[p] >> 1));
      const unsigned m = __ballot_sync(0xffffffffu, first);
      if (first) {
        const int u = base + __popc(m & ((1u << lane) - 1u));
        rt->un_e[u] = rt->key[p] >> 1;
        rt->un_off[u] = p;
      }
      base += __popc(m);
    }
    if (lane == 0) {
      rt->U = base;
      rt->n_ent = n;
      rt->un_off[base] = n;
    }
  }
  __syncthreads();
}

}  // namespace

}  // namespace moe

namespace moe {

// CTA-wide routing of a batch of at most 2 tokens (every thread calls it; 7 barriers).
// Selection with few dependent steps: each thread loads its strided share of the logits;
// quarter-warp maxima (36 per token at 288 threads) give the lower bound T = their K-th
// largest value (K groups hold an element >= T, so the K-th largest logit is >= T); the
// logits >= T are compacted and ranked exactly in parallel.  Entries are then sorted by
// (expert, token) and the union of experts indexed in the same pass.  Falls back to a warp
// arg-max selection when more than kCandMax logits reach the bound.
struct RouteScratch {
  float gmax[2][128];  // quarter-warp maxima (blockDim.x <= 1024)
  float T[2];
  int cnt[2];
  float cv[2][kCandMax];
  int ci[2][kCandMax];
  float sel_v[2][32];
  int sel_i[2][32];
  int key[64];
  unsigned emask[32];  // experts selected by token 0
};

namespace {

__device__ void route_small_cta(const LayerArgs& a, SmallRoute* rt, RouteScratch* sc, float* fallback_cand,
                                bool write_user) {
  const int B = a.B, E = a.E, K = a.k;
  const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kPer = 2;  // logits per thread per token (E <= kPer * nth: 1024 at 512 threads)
  const int ngroups = nth / 8;  // quarter-warp groups
  float v[2][kPer];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = tid + i * nth;
      float x = -INFINITY;
      if (t < B && e < E) {
        x = ld_act(a.ws.logits + (size_t)t * E + e);
        if (x != x) x = -INFINITY;
      }
      v[t][i] = x;
    }
  if (tid < 2) sc->cnt[tid] = 0;
  if (tid < 32) sc->emask[tid] = 0u;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPer; ++i) m = fmaxf(m, v[t][i]);
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((lane & 7) == 0 && t < B) sc->gmax[t][tid >> 3] = m;
  }
  __syncthreads();
  // (2) T[t] = K-th largest group maximum (ties by group index).
  if (tid < B * ngroups) {
    const int t = tid / ngroups, gi = tid - t * ngroups;
    const float m = sc->gmax[t][gi];
    int r = 0;
#pragma unroll 4
    for (int o = 0; o < ngroups; ++o) {
      const float x = sc->gmax[t][o];
      r += (x > m) || (x == m && o < gi);
    }
    if (r == K - 1) sc->T[t] = m;
  }
  __syncthreads();
  // (3) candidates: logits >= T.
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (t >= B) break;
    const float T = sc->T[t];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = tid + i * nth;
      if (e < E && v[t][i] >= T) {
        const int slot = atomicAdd(&sc->cnt[t], 1);
        if (slot < kCandMax) {
          sc->cv[t][slot] = v[t][i];
          sc->ci[t][slot] = e;
        }
      }
    }
  }
  __syncthreads();
  // (4) exact ranks among the candidates (= ranks among all experts).
  for (int z = tid; z < 2 * kCandMax; z += nth) {
    const int t = z / kCandMax, c = z - t * kCandMax;
    if (t < B) {
      const int C = sc->cnt[t];
      if (c < C && C <= kCandMax) {
        const float x = sc->cv[t][c];
        const int xi = sc->ci[t][c];
        int r = 0;
#pragma unroll 4
        for (int o = 0; o < C; ++o) r += better(sc->cv[t][o], sc->ci[t][o], x, xi);
        if (r < K) {
          sc->sel_v[t][r] = x;
          sc->sel_i[t][r] = xi;
        }
      }
    }
  }
  __syncthreads();
  // (5) gates (warp t for token t; overflow tokens take the warp arg-max selection).
  if (warp < B) {
    float my_v = 0.f;
    int my_i = 0;
    if (sc->cnt[warp] > kCandMax) {
      float* cvv = fallback_cand + warp * 2 * kCandStride;
      warp_topk(a.ws.logits + (size_t)warp * E, E, K, cvv, reinterpret_cast<int*>(cvv + kCandStride), lane, my_v,
                my_i);
    } else if (lane < K) {
      my_v = sc->sel_v[warp][lane];
      my_i = sc->sel_i[warp][lane];
    }
    const float gte = warp_gate(my_v, lane, K);
    if (lane < K) {
      const int e = (my_i >= 0 && my_i < E) ? my_i : 0;
      if (e != my_i) atomicOr(a.ws.err, kErrBounds);
      rt->idx[warp][lane] = e;
      rt->gate[warp][lane] = gte;
      sc->key[warp * K + lane] = e * 2 + warp;
      if (warp == 0) atomicOr(&sc->emask[e >> 5], 1u << (e & 31));
      if (write_user) {
        if (a.user_idx) a.user_idx[warp * K + lane] = e;
        if (a.user_gate) a.user_gate[warp * K + lane] = gte;
      }
    }
  }
  __syncthreads();
  // (6) entries sorted by key = expert * 2 + token (unique); an entry opens a union expert
  // when its token is 0 or token 0 did not select that expert.
  const int n = B * K;
  bool opens = false;
  if (tid < n) {
    const int key = sc->key[tid], e = key >> 1, t = key & 1;
    int r = 0, u = 0;
#pragma unroll 4
    for (int o = 0; o < n; ++o) {
      const int k2 = sc->key[o], e2 = k2 >> 1;
      r += k2 < key;
      const bool op2 = (k2 & 1) == 0 || !((sc->emask[e2 >> 5] >> (e2 & 31)) & 1u);
      u += (op2 && e2 < e);
    }
    opens = (t == 0) || !((sc->emask[e >> 5] >> (e & 31)) & 1u);
    rt->key[r] = key;
    rt->ent_tok[r] = t;
    rt->ent_gate[r] = rt->gate[t][tid - t * K];
    if (opens) {
      rt->un_e[u] = e;
      rt->un_off[u] = r;
    }
  }
  const int U = __syncthreads_count(opens);
  if (tid == 0) {
    rt->U = U;
    rt->n_ent = n;
    rt->un_off[U] = n;
  }
  __syncthreads();
}

}  // namespace

}  // namespace moe
