// sm_100a kernels of one MoE decode-layer step.
//
//   K1 k_oproj           h = residual + W_o . attn_out on the tensor cores (weights as the
//                        MMA's N operand) and per-CTA sums of h^2 (no grid-wide step: every
//                        router CTA reduces the partial sums itself, in one fixed order).
//   K2 k_router_topk     rstd from the o_proj partial sums; x = h * rstd * gamma (fp32, split
//                        into bf16 hi + lo for the MMA);
//                        logits = W_r . x; the last CTA selects the top-k per token with
//                        warp shuffles, computes the softmax gates and builds the routing
//                        tables (union of selected experts, per-expert token entries, CSR).
//   K3 k_gateup_small    small-M expert gate/up (batch <= 2): every (union expert, row pair)
//                        streamed once and multiplied with all tokens; a = silu(g) * u.
//      k_gateup_splitk   split-K expert gate/up for larger batches: (expert, K chunk) units
//                        whose partial sums are reduced in chunk order by the last unit of
//                        each expert.
//   K4 k_down_combine    out = bf16(h + sum_j gate_j * W_down[e_j] . a_j): rows of d split over
//                        CTAs, experts streamed in ascending order, fixed reduction order.
//   k_prefetch_l2        side-stream L2 prefetch of the next layer's weights.
//
// Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted
// kernels", section "How the specialised decode path works" (kernels chosen by batch size,
// small-matrix kernels at batch one or two and split-K above; o_proj fused with the
// residual step; next-layer prefetch; 16 of 896 experts per token).
//
// Structure shared by the streaming kernels: one CTA per SM, 8 consumer warps and one
// producer warp.  The producer's lane 0 streams weight rows into a shared-memory ring with
// TMA bulk copies (cp.async.bulk, mbarrier transaction counts, L2 evict-first); the
// consumers multiply and reduce in a fixed order, so every result is bit-reproducible.
#include <algorithm>

#include "common.cuh"
#include "gemv_mma.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kCPL = 4;  // 8-element chunks per lane (CUDA-core split-K kernel): K chunk <= 1024

__device__ __forceinline__ float ld_act_bf16(const uint16_t* p) {
  return bf16f(__ldcg(reinterpret_cast<const unsigned short*>(p)));
}

__device__ __forceinline__ void unpack8(uint4 w, float* f) {
  f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
  f[4] = bf16lo(w.z); f[5] = bf16hi(w.z); f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
}

// Waits for a phase while ignoring the abort flag (used to drain copies in flight).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, uint32_t* err) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) {
      atomicOr(err, kErrTimeout);
      return;
    }
  }
}

// Producer side of the ring: waits until stage `it % S` is free.
__device__ __forceinline__ bool ring_acquire(uint64_t* empty, int it, int S, volatile int* abort_flag,
                                             uint32_t* err) {
  if (it < S) return !*abort_flag;
  return mbar_wait(&empty[it % S], ((it / S) - 1) & 1, abort_flag, err);
}

// Producer epilogue: wait (bounded, ignoring abort) for the last min(S, issued) copies.
__device__ __forceinline__ void ring_drain(uint64_t* full, int issued, int S, uint32_t* err) {
  for (int i = issued - S < 0 ? 0 : issued - S; i < issued; ++i) mbar_drain(&full[i % S], (i / S) & 1, err);
}

// Last-CTA ticket: returns true in the CTA that arrives last.  All threads call it.
__device__ __forceinline__ bool last_cta(unsigned* counter, int* s_flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned prev = atomicAdd(counter, 1u);
    *s_flag = (prev == gridDim.x - 1);
  }
  __syncthreads();
  const bool last = *s_flag != 0;
  if (last) __threadfence();
  return last;
}

__device__ __forceinline__ void init_ring(uint64_t* full, uint64_t* empty, int S) {
  for (int s = 0; s < S; ++s) {
    mbar_init(&full[s], 1);
    if (empty) mbar_init(&empty[s], kConsumerWarps);
  }
}

__device__ __forceinline__ size_t align128(size_t x) { return (x + 127) & ~size_t(127); }

}  // namespace

// =============================================================================
// K1: o_proj + residual + RMSNorm statistics (tensor-core GEMV)
//   CTA c owns rows [r0, r1) of W_o; groups of 8 rows x K chunks stream through the ring;
//   tokens in groups of up to 8 (the MMA's M rows; bf16 attn_out is used as is).
// =============================================================================
__global__ void __launch_bounds__(kThreads, 1) k_oproj(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, d_o = a.d_o, B = a.B;
  const int S = a.k1.stages, kc = a.k1.kc, nch = a.k1.nch, TG = a.k1.tok_group, RM = a.k1.rows_max;
  const int wp = pitch_bytes(kc), ap = pitch_bytes(d_o);
  const size_t SB = align128((size_t)kGroupRows * wp);
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int r0 = (int)lo, r1 = (int)hi, rows = r1 - r0;
  const int ngroups = (rows + kGroupRows - 1) / kGroupRows;
  const int ntg = (B + TG - 1) / TG;

  unsigned char* ring = smem;
  unsigned char* act = ring + (size_t)S * SB;                                   // [TG][ap]
  uint64_t* full = reinterpret_cast<uint64_t*>(act + align128((size_t)TG * ap));
  uint64_t* empty = full + S;
  float* red = reinterpret_cast<float*>(empty + S);                             // [8][8][8]
  float* sq = red + kConsumerWarps * 64;                                        // [RM][TG]
  int* s_misc = reinterpret_cast<int*>(sq + RM * TG);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(full, empty, S);
    s_misc[0] = 0;
    s_misc[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  const uint32_t seg = (uint32_t)kc * 2u;
  if (warp == kConsumerWarps) {
    // Producer: W_o is static, so its rows stream before the dependency resolves.
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      bool ok = true;
      for (int tg = 0; tg < ntg && ok; ++tg)
        for (int g = 0; g < ngroups && ok; ++g) {
          const int rb = r0 + g * kGroupRows, nv = min(kGroupRows, r1 - rb);
          for (int ch = 0; ch < nch; ++ch, ++it) {
            if (!ring_acquire(empty, it, S, abort_flag, a.ws.err)) { ok = false; break; }
            const int s = it % S;
            mbar_arrive_expect_tx(&full[s], nv * seg);
            for (int j = 0; j < nv; ++j)
              bulk_g2s(ring + s * SB + j * wp, a.w_o + (size_t)(rb + j) * d_o + (size_t)ch * kc, seg, &full[s], pol);
          }
        }
      ring_drain(full, it, S, a.ws.err);
    }
  } else {
    pdl_wait();  // attn_out / residual may come from the previous kernel
    const int S_k = kc / 16;
    int s0, s1;
    warp_steps(S_k, warp, s0, s1);
    int it = 0;
    const int cpr = d_o / 8;  // 16-byte chunks per activation row
    for (int tg = 0; tg < ntg; ++tg) {
      const int t0 = tg * TG, nt = min(TG, B - t0);
      for (int z = tid; z < nt * cpr; z += kConsumerThreads) {
        const int t = z / cpr, q = z % cpr;
        *reinterpret_cast<uint4*>(act + (size_t)t * ap + (size_t)q * 16) =
            ld_act_u4(a.attn + (size_t)(t0 + t) * d_o + (size_t)q * 8);
      }
      consumer_sync();
      for (int g = 0; g < ngroups; ++g) {
        const int rb = r0 + g * kGroupRows, nv = min(kGroupRows, r1 - rb);
        float dacc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int ch = 0; ch < nch; ++ch, ++it) {
          const int s = it % S;
          mbar_wait(&full[s], (it / S) & 1, abort_flag, a.ws.err);
          mma_stage(dacc, ring + s * SB, wp, act, ap, nt, ch * kc, s0, s1, lane);
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
        }
        mma_store_partial(red, dacc, nt, warp, lane);
        consumer_sync();
        for (int z = tid; z < nv * nt; z += kConsumerThreads) {
          const int n = z / nt, t = z % nt;
          const size_t o = (size_t)(t0 + t) * d + rb + n;
          const float hv = ld_act_bf16(a.resid + o) + mma_reduce(red, t, n);
          a.ws.h[o] = hv;
          sq[(rb + n - r0) * TG + t] = hv * hv;
        }
        consumer_sync();
      }
      if (tid < nt) {
        float ss = 0.f;
        for (int rr = 0; rr < rows; ++rr) ss += sq[rr * TG + tid];
        a.ws.ss_part[(size_t)c * a.maxB + t0 + tid] = ss;
      }
      consumer_sync();
    }
  }

}

// =============================================================================
// K2: RMSNorm apply + router GEMV + top-k + gates + routing tables
// =============================================================================
namespace {

constexpr int kCandMax = 128;           // candidates kept per token by the threshold pass
constexpr int kTopkScratch = 48 * 1024;  // shared memory used by the last CTA

__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Exact top-K of one token's E logits by one warp: (value desc, index asc).
// Threshold pass: the K-th largest of the 32 lane maxima is a lower bound T of the
// K-th largest logit, so every selected expert has a logit >= T.  Those candidates are
// compacted and ranked exactly; the fallback (more than kCandMax candidates, e.g. mass
// ties) repeats a warp arg-max K times.  Lane j < K returns the j-th selection.
__device__ void warp_topk(const float* logits, int E, int K, float* cand_v, int* cand_i, int lane,
                          float& my_v, int& my_i) {
  float v[32];
  float lm = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    float x = -INFINITY;
    if (e < E) {
      x = ld_act(logits + e);
      if (x != x) x = -INFINITY;  // NaN never outranks a number
    }
    v[i] = x;
    if (e < E) lm = fmaxf(lm, x);
  }
  // Rank of this lane's maximum among the 32 (ties by lane id); T = the (K-1)-ranked one.
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
    // Exact rank of each candidate among the candidates = its rank among all experts.
    for (int cidx = lane; cidx < C; cidx += 32) {
      const float cv = cand_v[cidx];
      const int ci = cand_i[cidx];
      int r = 0;
      for (int o = 0; o < C; ++o) r += better(cand_v[o], cand_i[o], cv, ci);
      cand_v[kCandMax + cidx] = __int_as_float(r);
    }
    __syncwarp();
    for (int cidx = lane; cidx < C; cidx += 32) {
      const int r = __float_as_int(cand_v[kCandMax + cidx]);
      if (r < K) {  // slots [2*kCandMax, 2*kCandMax + 32): selections in rank order
        cand_v[2 * kCandMax + r] = cand_v[cidx];
        cand_i[2 * kCandMax + r] = cand_i[cidx];
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
  // Fallback: K rounds of warp arg-max over the remaining elements.
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

// Executed by every thread of the last router CTA.
__device__ void topk_route(const LayerArgs& a, unsigned char* scratch) {
  const int B = a.B, E = a.E, K = a.k;
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(scratch);  // [1024]
  int* off_e = reinterpret_cast<int*>(mask + 1024);                         // [1024]
  int* sidx = off_e + 1024;                                                 // [64*32]
  float* cand = reinterpret_cast<float*>(sidx + 64 * 32);                   // [nwarps][2*kCandMax+32] x2
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int cstride = 2 * kCandMax + 32;
  float* cv = cand + warp * 2 * cstride;
  int* ci = reinterpret_cast<int*>(cv + cstride);

  for (int e = threadIdx.x; e < E; e += blockDim.x) mask[e] = 0ull;

  for (int t = warp; t < B; t += nwarps) {
    float my_v = 0.f;
    int my_i = 0;
    warp_topk(a.ws.logits + (size_t)t * E, E, K, cv, ci, lane, my_v, my_i);
    const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
    const float w = (lane < K) ? expf(my_v - v0) : 0.f;
    const float sum = warp_sum(w);
    if (lane < K) {
      const float gte = w / sum;
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

  // Union of experts and CSR offsets: warp 0 scans E <= 1024 in 32-expert strips.
  if (warp == 0) {
    int cnt = 0, nu = 0;
    const int e0 = lane * 32;
    for (int e = e0; e < e0 + 32 && e < E; ++e) {
      const int c = __popcll(mask[e]);
      cnt += c;
      nu += (c > 0);
    }
    int icnt = cnt, inu = nu;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, icnt, o);
      const int z = __shfl_up_sync(0xffffffffu, inu, o);
      if (lane >= o) { icnt += y; inu += z; }
    }
    int off = icnt - cnt, u = inu - nu;
    for (int e = e0; e < e0 + 32 && e < E; ++e) {
      const int c = __popcll(mask[e]);
      off_e[e] = off;
      if (c > 0) {
        a.ws.union_e[u] = e;
        a.ws.union_off[u] = off;
        ++u;
      }
      off += c;
    }
    if (lane == 31) {
      *a.ws.n_union = inu;
      a.ws.union_off[inu] = icnt;
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

//   CTA c owns rows [e0, e0 + nrows) of W_r (at most 8): all K chunks stay resident;
//   tokens in groups of 2 (4 MMA rows: hi and lo of each token's x).
__global__ void __launch_bounds__(kThreads, 1) k_router_topk(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, E = a.E, B = a.B;
  const int kc = a.k2.kc, nch = a.k2.nch;
  const int wp = pitch_bytes(kc), ap = pitch_bytes(d);
  const size_t SB = align128((size_t)kGroupRows * wp);
  long long lo, hi;
  split_range(E, G, c, lo, hi);
  const int e0 = (int)lo, nrows = (int)(hi - lo);

  unsigned char* wst = smem;                                          // [nch][8][wp]
  unsigned char* act = wst + (size_t)nch * SB;                        // [4][ap]
  unsigned char* scratch = act + align128((size_t)4 * ap);            // last CTA
  uint64_t* full = reinterpret_cast<uint64_t*>(scratch + kTopkScratch);
  float* red = reinterpret_cast<float*>(full + nch);
  float* rstd_s = red + kConsumerWarps * 64;  // [B]
  int* s_misc = reinterpret_cast<int*>(rstd_s + 64);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(full, nullptr, nch);
    s_misc[0] = 0;
    s_misc[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  const uint32_t seg = (uint32_t)kc * 2u;
  if (warp == kConsumerWarps) {
    // The router slice is static: fetch all of it before the dependency resolves.
    if (lane == 0 && nrows > 0) {
      const uint64_t pol = policy_evict_first();
      for (int ch = 0; ch < nch; ++ch) {
        mbar_arrive_expect_tx(&full[ch], nrows * seg);
        for (int j = 0; j < nrows; ++j)
          bulk_g2s(wst + ch * SB + j * wp, a.w_r + (size_t)(e0 + j) * d + (size_t)ch * kc, seg, &full[ch], pol);
      }
      for (int ch = 0; ch < nch; ++ch) mbar_drain(&full[ch], 0, a.ws.err);
    }
  } else {
    pdl_wait();  // h and the sums of h^2 come from the o_proj kernel
    // rstd[t] = 1/sqrt(sum_c ss_part[c][t] / d + eps): warp t%8 sums the G partials in a
    // fixed order (lane strides, then a butterfly), so every CTA gets the same bits.
    for (int t = warp; t < B; t += kConsumerWarps) {
      float ss = 0.f;
      for (int cc = lane; cc < G; cc += 32) ss += ld_act(&a.ws.ss_part[(size_t)cc * a.maxB + t]);
      ss = warp_sum(ss);
      if (lane == 0) {
        const float r = 1.0f / sqrtf(ss / (float)d + a.eps);
        rstd_s[t] = r;
        if (c == 0) a.ws.rstd[t] = r;
      }
    }
    consumer_sync();
    const int S_k = kc / 16;
    int s0, s1;
    warp_steps(S_k, warp, s0, s1);
    const int cpr = d / 8;
    bool have_w = false;
    for (int t0 = 0; t0 < B; t0 += 2) {
      const int nt = min(2, B - t0);
      for (int t = 0; t < nt; ++t) {
        const float r = rstd_s[t0 + t];
        for (int q = tid; q < cpr; q += kConsumerThreads) {
          const float* hp = a.ws.h + (size_t)(t0 + t) * d + (size_t)q * 8;
          const float4 h0 = ld_act4(hp), h1 = ld_act4(hp + 4);
          float gm[8];
          unpack8(ld_weight_u4(a.gamma + (size_t)q * 8), gm);
          const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
          float xv[8];
          uint16_t xh[8], xl[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            xv[e] = hv[e] * r * gm[e];
            split_bf16(xv[e], xh[e], xl[e]);
          }
          uint4 ph, pl;
          ph.x = xh[0] | ((uint32_t)xh[1] << 16); ph.y = xh[2] | ((uint32_t)xh[3] << 16);
          ph.z = xh[4] | ((uint32_t)xh[5] << 16); ph.w = xh[6] | ((uint32_t)xh[7] << 16);
          pl.x = xl[0] | ((uint32_t)xl[1] << 16); pl.y = xl[2] | ((uint32_t)xl[3] << 16);
          pl.z = xl[4] | ((uint32_t)xl[5] << 16); pl.w = xl[6] | ((uint32_t)xl[7] << 16);
          *reinterpret_cast<uint4*>(act + (size_t)(2 * t) * ap + (size_t)q * 16) = ph;
          *reinterpret_cast<uint4*>(act + (size_t)(2 * t + 1) * ap + (size_t)q * 16) = pl;
          if (q % G == c) {  // each chunk of x is written by exactly one CTA
            float* xp = a.ws.x + (size_t)(t0 + t) * d + (size_t)q * 8;
            *reinterpret_cast<float4*>(xp) = make_float4(xv[0], xv[1], xv[2], xv[3]);
            *reinterpret_cast<float4*>(xp + 4) = make_float4(xv[4], xv[5], xv[6], xv[7]);
          }
        }
      }
      consumer_sync();
      float dacc[4] = {0.f, 0.f, 0.f, 0.f};
      if (nrows > 0) {
        for (int ch = 0; ch < nch; ++ch) {
          if (!have_w) mbar_wait(&full[ch], 0, abort_flag, a.ws.err);
          mma_stage(dacc, wst + ch * SB, wp, act, ap, 2 * nt, ch * kc, s0, s1, lane);
        }
        have_w = true;
      }
      mma_store_partial(red, dacc, 2 * nt, warp, lane);
      consumer_sync();
      for (int z = tid; z < nrows * nt; z += kConsumerThreads) {
        const int n = z / nt, t = z % nt;
        const float v = mma_reduce(red, 2 * t, n) + mma_reduce(red, 2 * t + 1, n);
        a.ws.logits[(size_t)(t0 + t) * E + e0 + n] = v;
      }
      consumer_sync();
    }
  }

  if (last_cta(&a.ws.counters[kCntRouter], &s_misc[1])) {
    topk_route(a, scratch);
    if (tid == 0) a.ws.counters[kCntRouter] = 0;
  }
}

// =============================================================================
// K3 (small-M, batch <= 2): expert gate/up + SiLU*mul on the tensor cores.
//   Units are (union expert u, row pair p) in flattened order; a CTA takes a contiguous
//   range, 4 pairs per MMA group (rows 0..3 gate p.., rows 4..7 up p..), K in chunks.
//   Every token's x is an MMA row pair (hi, lo); a is written only for tokens routed to u.
// =============================================================================
__global__ void __launch_bounds__(kThreads, 1) k_gateup_small(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, I = a.I, E = a.E, B = a.B, K = a.k;
  const int S = a.k3.stages, kc = a.k3.kc, nch = a.k3.nch;
  const int wp = pitch_bytes(kc), ap = pitch_bytes(d);
  const size_t SB = align128((size_t)kGroupRows * wp);
  const int umax = min(E, B * K);

  unsigned char* ring = smem;
  unsigned char* act = ring + (size_t)S * SB;                          // [2B][ap]
  int* un_e = reinterpret_cast<int*>(act + align128((size_t)4 * ap));  // [umax]
  int* un_off = un_e + umax;                                           // [umax+1]
  int* ent_tok = un_off + umax + 1;                                    // [B*K]
  uint64_t* full = reinterpret_cast<uint64_t*>(align128(reinterpret_cast<size_t>(ent_tok + B * K) -
                                                        reinterpret_cast<size_t>(smem)) + smem);
  uint64_t* empty = full + S;
  float* red = reinterpret_cast<float*>(empty + S);
  int* s_misc = reinterpret_cast<int*>(red + kConsumerWarps * 64);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(full, empty, S);
    s_misc[0] = 0;
    fence_barrier_init();
  }
  pdl_wait();  // routing tables and x come from the router kernel
  pdl_trigger();
  int U = ld_act_i(a.ws.n_union);
  if (U < 0 || U > umax) {
    if (tid == 0) atomicOr(a.ws.err, kErrBounds);
    U = 0;
  }
  for (int i = tid; i < U; i += blockDim.x) {
    int e = ld_act_i(&a.ws.union_e[i]);
    if (e < 0 || e >= E) { atomicOr(a.ws.err, kErrBounds); e = 0; }
    un_e[i] = e;
  }
  for (int i = tid; i <= U; i += blockDim.x) un_off[i] = ld_act_i(&a.ws.union_off[i]);
  for (int i = tid; i < B * K; i += blockDim.x) ent_tok[i] = ld_act_i(&a.ws.entry_tok[i]);
  __syncthreads();

  const long long total = (long long)U * I;
  long long q0, q1;
  split_range(total, G, c, q0, q1);
  const uint32_t seg = (uint32_t)kc * 2u;

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      bool ok = true;
      for (long long q = q0; q < q1 && ok; q += 4) {
        const int np = (int)min(4LL, q1 - q);
        for (int ch = 0; ch < nch; ++ch, ++it) {
          if (!ring_acquire(empty, it, S, abort_flag, a.ws.err)) { ok = false; break; }
          const int s = it % S;
          mbar_arrive_expect_tx(&full[s], 2 * np * seg);
          for (int i = 0; i < np; ++i) {
            const int u = (int)((q + i) / I), p = (int)((q + i) % I);
            const uint16_t* base = a.w_gu + ((size_t)un_e[u] * 2 * I + p) * d + (size_t)ch * kc;
            bulk_g2s(ring + s * SB + i * wp, base, seg, &full[s], pol);
            bulk_g2s(ring + s * SB + (4 + i) * wp, base + (size_t)I * d, seg, &full[s], pol);
          }
        }
      }
      ring_drain(full, it, S, a.ws.err);
    }
  } else {
    // x of every token as (hi, lo) bf16 rows.
    const int cpr = d / 8;
    for (int z = tid; z < B * cpr; z += kConsumerThreads) {
      const int t = z / cpr, qq = z % cpr;
      const float* xp = a.ws.x + (size_t)t * d + (size_t)qq * 8;
      const float4 x0 = ld_act4(xp), x1 = ld_act4(xp + 4);
      const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      uint16_t xh[8], xl[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) split_bf16(xv[e], xh[e], xl[e]);
      uint4 ph, pl;
      ph.x = xh[0] | ((uint32_t)xh[1] << 16); ph.y = xh[2] | ((uint32_t)xh[3] << 16);
      ph.z = xh[4] | ((uint32_t)xh[5] << 16); ph.w = xh[6] | ((uint32_t)xh[7] << 16);
      pl.x = xl[0] | ((uint32_t)xl[1] << 16); pl.y = xl[2] | ((uint32_t)xl[3] << 16);
      pl.z = xl[4] | ((uint32_t)xl[5] << 16); pl.w = xl[6] | ((uint32_t)xl[7] << 16);
      *reinterpret_cast<uint4*>(act + (size_t)(2 * t) * ap + (size_t)qq * 16) = ph;
      *reinterpret_cast<uint4*>(act + (size_t)(2 * t + 1) * ap + (size_t)qq * 16) = pl;
    }
    consumer_sync();
    const int S_k = kc / 16;
    int s0, s1;
    warp_steps(S_k, warp, s0, s1);
    int it = 0;
    for (long long q = q0; q < q1; q += 4) {
      const int np = (int)min(4LL, q1 - q);
      float dacc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int ch = 0; ch < nch; ++ch, ++it) {
        const int s = it % S;
        mbar_wait(&full[s], (it / S) & 1, abort_flag, a.ws.err);
        mma_stage(dacc, ring + s * SB, wp, act, ap, 2 * B, ch * kc, s0, s1, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      mma_store_partial(red, dacc, 2 * B, warp, lane);
      consumer_sync();
      for (int z = tid; z < np * B; z += kConsumerThreads) {
        const int i = z / B, t = z % B;
        const int u = (int)((q + i) / I), p = (int)((q + i) % I);
        const float gs = mma_reduce(red, 2 * t, i) + mma_reduce(red, 2 * t + 1, i);
        const float us = mma_reduce(red, 2 * t, 4 + i) + mma_reduce(red, 2 * t + 1, 4 + i);
        for (int en = un_off[u]; en < un_off[u + 1]; ++en)
          if (ent_tok[en] == t) a.ws.a[(size_t)en * I + p] = gs / (1.0f + expf(-gs)) * us;
      }
      consumer_sync();
    }
  }
}
// =============================================================================
// K3 (split-K): expert gate/up for larger batches
//   unit (u, c): rows 0..2I-1 of expert union_e[u] over K chunk c; tokens in groups of NT.
//   Partials go to gu_part[entry][c][2I]; the last unit of each expert (ticket) sums them
//   over c in order and writes a = silu(g) * u.
// =============================================================================
template <int NT>
__global__ void __launch_bounds__(kThreads, 1) k_gateup_splitk(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, cta = blockIdx.x;
  const int d = a.d, I = a.I, E = a.E, NS = a.k3.n_split;
  const int S = a.k3.stages, RS = a.k3.rows_per_stage;
  const int Kc = d / NS;
  const uint32_t seg_bytes = (uint32_t)Kc * 2u;
  const uint32_t stage_bytes = (uint32_t)RS * seg_bytes;

  unsigned char* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  uint64_t* empty = full + S;
  int* s_misc = reinterpret_cast<int*>(empty + S);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    s_misc[0] = 0;
    s_misc[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  const int U = ld_act_i(a.ws.n_union);
  const long long units = (long long)U * NS;
  long long v0, v1;
  split_range(units, G, cta, v0, v1);
  const int R2 = 2 * I;

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      bool ok = true;
      for (long long v = v0; v < v1 && ok; ++v) {
        const int u = (int)(v / NS), ck = (int)(v % NS);
        int e = ld_act_i(&a.ws.union_e[u]);
        if (e < 0 || e >= E) { atomicOr(a.ws.err, kErrBounds); e = 0; }
        for (int r = 0; r < R2; r += RS, ++it) {
          const int n = min(RS, R2 - r);
          if (!ring_acquire(empty, it, S, abort_flag, a.ws.err)) { ok = false; break; }
          const int s = it % S;
          mbar_arrive_expect_tx(&full[s], n * seg_bytes);
          for (int j = 0; j < n; ++j)
            bulk_g2s(ring + (size_t)s * stage_bytes + (size_t)j * seg_bytes,
                     a.w_gu + ((size_t)e * R2 + r + j) * d + (size_t)ck * Kc, seg_bytes, &full[s], pol);
        }
      }
      ring_drain(full, it, S, a.ws.err);
    }
  } else {
    // Lane mapping inside a K chunk: 8-element chunks qq = i*32 + lane, qq < Kc/8.
    // Stages outer, token groups inner, so each stage is released after its last group.
    const int cq = Kc / 8;  // 8-element chunks in the K chunk (at most kCPL * 32)
    int it = 0;
    float xr[NT][kCPL][8];
    long long cur_v = -1;
    int cur_g = -1;
    for (long long v = v0; v < v1; ++v) {
      const int u = (int)(v / NS), ck = (int)(v % NS);
      const int off = ld_act_i(&a.ws.union_off[u]);
      const int m = ld_act_i(&a.ws.union_off[u + 1]) - off;
      for (int r = 0; r < R2; r += RS, ++it) {
        const int n = min(RS, R2 - r), s = it % S;
        mbar_wait(&full[s], (it / S) & 1, abort_flag, a.ws.err);
        const unsigned char* st = ring + (size_t)s * stage_bytes;
        for (int g0 = 0; g0 < m; g0 += NT) {
          const int nt = min(NT, m - g0);
          if (v != cur_v || g0 != cur_g) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              int tok = (t < nt) ? ld_act_i(&a.ws.entry_tok[off + g0 + t]) : -1;
              if (tok >= a.B) { atomicOr(a.ws.err, kErrBounds); tok = -1; }
#pragma unroll
              for (int i = 0; i < kCPL; ++i) {
                if (tok >= 0 && i * 32 + lane < cq) {
                  const float* xp = a.ws.x + (size_t)tok * d + (size_t)ck * Kc + (size_t)(i * 32 + lane) * 8;
                  const float4 x0 = ld_act4(xp), x1 = ld_act4(xp + 4);
                  xr[t][i][0] = x0.x; xr[t][i][1] = x0.y; xr[t][i][2] = x0.z; xr[t][i][3] = x0.w;
                  xr[t][i][4] = x1.x; xr[t][i][5] = x1.y; xr[t][i][6] = x1.z; xr[t][i][7] = x1.w;
                } else {
#pragma unroll
                  for (int e = 0; e < 8; ++e) xr[t][i][e] = 0.f;
                }
              }
            }
            cur_v = v;
            cur_g = g0;
          }
          for (int j = warp; j < n; j += kConsumerWarps) {
            float acc[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[t] = 0.f;
#pragma unroll
            for (int i = 0; i < kCPL; ++i) {
              if (i * 32 + lane >= cq) continue;
              const uint4 w = *reinterpret_cast<const uint4*>(st + (size_t)j * seg_bytes + (size_t)(i * 32 + lane) * 16);
#pragma unroll
              for (int t = 0; t < NT; ++t) acc[t] = dot8(w, xr[t][i], acc[t]);
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              const float vv = warp_sum(acc[t]);
              if (lane == 0 && t < nt)
                a.ws.gu_part[((size_t)(off + g0 + t) * NS + ck) * R2 + r + j] = vv;
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // Publish this unit; the last of the expert's NS units reduces in chunk order.
      __threadfence();
      consumer_sync();
      if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(&a.ws.gu_tick[u], 1u);
        s_misc[1] = (prev == (unsigned)NS - 1);
      }
      consumer_sync();
      if (s_misc[1]) {
        __threadfence();
        for (int z = threadIdx.x; z < m * I; z += kConsumerThreads) {
          const int t = z / I, r = z % I;
          const float* pp = a.ws.gu_part + (size_t)(off + t) * NS * R2;
          float gs = 0.f, us = 0.f;
          for (int cc = 0; cc < NS; ++cc) {
            gs += ld_act(pp + (size_t)cc * R2 + r);
            us += ld_act(pp + (size_t)cc * R2 + I + r);
          }
          a.ws.a[(size_t)(off + t) * I + r] = gs / (1.0f + expf(-gs)) * us;
        }
        if (threadIdx.x == 0) a.ws.gu_tick[u] = 0;
      }
      consumer_sync();
    }
  }
}

// =============================================================================
// K4: expert down projection + gate-weighted combine into the residual
//   CTA c owns output rows [i0, i1); one stage = those rows of one union expert (contiguous
//   in W_down).  Routing tables, gates and (when they fit) all activations a are staged in
//   shared memory first.  NT > 0 (batch <= 2): each lane accumulates its slice of every row
//   over all experts in registers; one warp reduction per (row, token) at the end.
//   NT == 0 (any batch): one warp reduction per (expert, token, row) into shared memory.
//   Both add the experts in ascending order, so the result is deterministic.
// =============================================================================
template <int NT>
__global__ void __launch_bounds__(kThreads, 1) k_down_combine(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kRPW = 7;  // rows per warp in the NT path (rows_max <= 56)
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, I = a.I, E = a.E, B = a.B, K = a.k;
  const int S = a.k4.stages, RM = a.k4.rows_max;
  const bool a_smem = a.k4.a_in_smem != 0;
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int i0 = (int)lo, nrows = (int)(hi - lo);
  const uint32_t row_bytes = (uint32_t)I * 2u;
  const size_t SB = align128((size_t)RM * row_bytes);
  const int umax = min(E, B * K), nent = B * K;

  unsigned char* ring = smem;
  float* a_s = reinterpret_cast<float*>(ring + (size_t)S * SB);                  // [nent][I] if staged
  float* acc_s = a_s + (a_smem ? (size_t)nent * I : 0);                         // [RM][B] (NT == 0)
  int* un_e = reinterpret_cast<int*>(acc_s + (NT == 0 ? RM * B : 0));          // [umax]
  int* un_off = un_e + umax;                                                    // [umax+1]
  int* ent_tok = un_off + umax + 1;                                             // [nent]
  float* ent_gate = reinterpret_cast<float*>(ent_tok + nent);                   // [nent]
  uint64_t* full = reinterpret_cast<uint64_t*>(align128(reinterpret_cast<size_t>(ent_gate + nent) -
                                                        reinterpret_cast<size_t>(smem)) + smem);
  uint64_t* empty = full + S;
  int* s_misc = reinterpret_cast<int*>(empty + S);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(full, empty, S);
    s_misc[0] = 0;
    fence_barrier_init();
  }
  // The routing tables were complete before this grid could launch: the gate/up kernel
  // allows its dependents to launch only after its own dependency wait, which returns once
  // the router kernel (the tables' writer) has finished.  So the tables, and the W_down
  // rows they select, may be read now; the activations a are read after pdl_wait.
  int U = ld_act_i(a.ws.n_union);
  if (U < 0 || U > umax) {
    if (tid == 0) atomicOr(a.ws.err, kErrBounds);
    U = 0;
  }
  for (int i = tid; i < U; i += blockDim.x) {
    int e = ld_act_i(&a.ws.union_e[i]);
    if (e < 0 || e >= E) { atomicOr(a.ws.err, kErrBounds); e = 0; }
    un_e[i] = e;
  }
  for (int i = tid; i <= U; i += blockDim.x) un_off[i] = ld_act_i(&a.ws.union_off[i]);
  for (int i = tid; i < B * K; i += blockDim.x) {
    int t = ld_act_i(&a.ws.entry_tok[i]);
    int j = ld_act_i(&a.ws.entry_slot[i]);
    if (t < 0 || t >= B || j < 0 || j >= K) { atomicOr(a.ws.err, kErrBounds); t = 0; j = 0; }
    ent_tok[i] = t;
    ent_gate[i] = ld_act(&a.ws.topk_gate[t * K + j]);
  }
  if (NT == 0)
    for (int z = tid; z < nrows * B; z += blockDim.x) acc_s[z] = 0.f;
  __syncthreads();
  pdl_trigger();

  if (warp == kConsumerWarps) {
    if (lane == 0 && nrows > 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      for (int u = 0; u < U; ++u, ++it) {
        if (!ring_acquire(empty, it, S, abort_flag, a.ws.err)) break;
        const int s = it % S;
        mbar_arrive_expect_tx(&full[s], nrows * row_bytes);
        bulk_g2s(ring + s * SB, a.w_down + ((size_t)un_e[u] * d + i0) * I, nrows * row_bytes, &full[s], pol);
      }
      ring_drain(full, it, S, a.ws.err);
    }
    return;
  }

  pdl_wait();  // the SwiGLU activations come from the gate/up kernel
  if (a_smem) {
    for (int i = tid; i < B * K * I / 4; i += kConsumerThreads)
      reinterpret_cast<float4*>(a_s)[i] = ld_act4(a.ws.a + (size_t)i * 4);
    consumer_sync();
  }

  const int epl = I / 32;  // elements of a row per lane (1..16)
  const bool vec4 = (epl & 3) == 0;
  if constexpr (NT > 0) {
    float acc[kRPW][NT > 0 ? NT : 1];
#pragma unroll
    for (int i = 0; i < kRPW; ++i)
#pragma unroll
      for (int t = 0; t < (NT > 0 ? NT : 1); ++t) acc[i][t] = 0.f;
    for (int u = 0; u < U && nrows > 0; ++u) {
      const int s = u % S;
      mbar_wait(&full[s], (u / S) & 1, abort_flag, a.ws.err);
      const unsigned char* st = ring + s * SB;
      for (int en = un_off[u]; en < un_off[u + 1]; ++en) {
        const int t = ent_tok[en];
        const float g = ent_gate[en];
        float av[16];
        const float* ap_ = a_smem ? a_s + (size_t)en * I : a.ws.a + (size_t)en * I;
#pragma unroll
        for (int x = 0; x < 16; ++x)
          av[x] = (x < epl) ? g * (a_smem ? ap_[lane * epl + x] : ld_act(ap_ + lane * epl + x)) : 0.f;
#pragma unroll
        for (int i = 0; i < kRPW; ++i) {
          const int rl = warp + kConsumerWarps * i;
          if (rl >= nrows) break;
          const uint16_t* wr = reinterpret_cast<const uint16_t*>(st + (size_t)rl * row_bytes) + lane * epl;
          float sdot = 0.f;
          if (vec4) {
#pragma unroll
            for (int x = 0; x < 16; x += 4) {
              if (x >= epl) break;
              const uint2 w4 = *reinterpret_cast<const uint2*>(wr + x);
              sdot = fmaf(bf16lo(w4.x), av[x], sdot);
              sdot = fmaf(bf16hi(w4.x), av[x + 1], sdot);
              sdot = fmaf(bf16lo(w4.y), av[x + 2], sdot);
              sdot = fmaf(bf16hi(w4.y), av[x + 3], sdot);
            }
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x)
              if (x < epl) sdot = fmaf(bf16f(wr[x]), av[x], sdot);
          }
#pragma unroll
          for (int tt = 0; tt < (NT > 0 ? NT : 1); ++tt)
            if (tt == t) acc[i][tt] += sdot;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
#pragma unroll
    for (int i = 0; i < kRPW; ++i) {
      const int rl = warp + kConsumerWarps * i;
#pragma unroll
      for (int t = 0; t < (NT > 0 ? NT : 1); ++t) {
        const float v = warp_sum(acc[i][t]);
        if (lane == 0 && rl < nrows && t < B) {
          const size_t o = (size_t)t * d + i0 + rl;
          const __nv_bfloat16 bv = __float2bfloat16_rn(ld_act(&a.ws.h[o]) + v);
          a.out[o] = *reinterpret_cast<const uint16_t*>(&bv);
        }
      }
    }
  } else {
  // NT == 0: any batch.
  for (int u = 0; u < U && nrows > 0; ++u) {
    const int s = u % S;
    mbar_wait(&full[s], (u / S) & 1, abort_flag, a.ws.err);
    const unsigned char* st = ring + s * SB;
    for (int en = un_off[u]; en < un_off[u + 1]; ++en) {
      const int t = ent_tok[en];
      const float g = ent_gate[en];
      float av[16];
      const float* ap_ = a_smem ? a_s + (size_t)en * I : a.ws.a + (size_t)en * I;
#pragma unroll
      for (int x = 0; x < 16; ++x)
        av[x] = (x < epl) ? (a_smem ? ap_[lane * epl + x] : ld_act(ap_ + lane * epl + x)) : 0.f;
      for (int rl = warp; rl < nrows; rl += kConsumerWarps) {
        const uint16_t* wr = reinterpret_cast<const uint16_t*>(st + (size_t)rl * row_bytes) + lane * epl;
        float sdot = 0.f;
#pragma unroll
        for (int x = 0; x < 16; ++x)
          if (x < epl) sdot = fmaf(bf16f(wr[x]), av[x], sdot);
        sdot = warp_sum(sdot);
        if (lane == 0) acc_s[rl * B + t] += g * sdot;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  consumer_sync();
  for (int z = tid; z < nrows * B; z += kConsumerThreads) {
    const int rl = z / B, t = z % B;
    const size_t o = (size_t)t * d + i0 + rl;
    const __nv_bfloat16 bv = __float2bfloat16_rn(ld_act(&a.ws.h[o]) + acc_s[z]);
    a.out[o] = *reinterpret_cast<const uint16_t*>(&bv);
  }
  }
}

// =============================================================================
// Side-stream L2 prefetch of the next layer's weights (no shared memory, no outputs)
// =============================================================================
__global__ void k_prefetch_l2(const PrefetchArgs p) {
  constexpr unsigned long long kChunk = 32768;
  unsigned long long total = 0;
  for (int i = 0; i < p.n; ++i) total += (p.bytes[i] + kChunk - 1) / kChunk;
  for (unsigned long long q = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; q < total;
       q += (unsigned long long)gridDim.x * blockDim.x) {
    unsigned long long rem = q;
    for (int i = 0; i < p.n; ++i) {
      const unsigned long long nch = (p.bytes[i] + kChunk - 1) / kChunk;
      if (rem < nch) {
        const unsigned long long off = rem * kChunk;
        const unsigned long long len = min(kChunk, p.bytes[i] - off) & ~15ull;
        if (len) bulk_prefetch_l2(static_cast<const unsigned char*>(p.ptr[i]) + off, (uint32_t)len);
        break;
      }
      rem -= nch;
    }
  }
}

// =============================================================================
// Host side: planning and launch
// =============================================================================
namespace {

template <typename Kern>
cudaError_t launch_k(Kern k, int grid, size_t smem, cudaStream_t s, bool pdl, const LayerArgs& a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, a);
}

size_t a128(size_t x) { return (x + 127) & ~size_t(127); }

// Largest multiple of 64 that divides K and keeps an 8-row stage within `stage_cap` bytes.
int pick_kc(int K, size_t stage_cap) {
  int best = 64;
  for (int kc = 64; kc <= K; kc += 64)
    if (K % kc == 0 && (size_t)kGroupRows * (kc * 2 + 16) <= stage_cap) best = kc;
  return best;
}

}  // namespace

bool plan_layer(LayerArgs& a, int G, size_t optin) {
  const size_t budget = optin - 1024 - 256;  // static reservation and alignment slack
  const int maxB = a.B, Kk = a.k;  // shared memory is planned for the batch being launched
  // K1: tensor-core GEMV over W_o, token groups of up to 8.
  {
    KTune& t = a.k1;
    t.rows_max = (a.d + G - 1) / G;
    t.kc = pick_kc(a.d_o, 34 * 1024);
    t.nch = a.d_o / t.kc;
    t.tok_group = std::min(maxB, 8);
    const size_t SB = a128((size_t)kGroupRows * (t.kc * 2 + 16));
    size_t act = a128((size_t)t.tok_group * (a.d_o * 2 + 16));
    size_t extra = 2 * kMaxStages * 8 + kConsumerWarps * 64 * 4 + (size_t)t.rows_max * t.tok_group * 4 + 64;
    while (t.tok_group > 1 && act + extra + 2 * SB > budget) {
      t.tok_group /= 2;
      act = a128((size_t)t.tok_group * (a.d_o * 2 + 16));
      extra = 2 * kMaxStages * 8 + kConsumerWarps * 64 * 4 + (size_t)t.rows_max * t.tok_group * 4 + 64;
    }
    t.stages = (int)std::min<size_t>(kMaxStages, (budget - act - extra) / SB);
    if (t.stages < 2) return false;
    t.smem = (size_t)t.stages * SB + act + extra;
  }
  // K2: the router slice (<= 8 rows) resident in all its K chunks.
  {
    KTune& t = a.k2;
    t.rows_max = (a.E + G - 1) / G;
    if (t.rows_max > kGroupRows) return false;
    t.kc = pick_kc(a.d, 34 * 1024);
    t.nch = a.d / t.kc;
    const size_t SB = a128((size_t)kGroupRows * (t.kc * 2 + 16));
    t.smem = (size_t)t.nch * SB + a128((size_t)4 * (a.d * 2 + 16)) + 48 * 1024 + (size_t)t.nch * 8 +
             kConsumerWarps * 64 * 4 + 64 * 4 + 64;
    if (t.smem > budget) return false;
  }
  // K3: small-M (tensor cores, batch <= 2) or split-K (row segments of one K chunk).
  {
    KTune& t = a.k3;
    if (a.k3.n_split > 0) {
      const int Kc = a.d / a.k3.n_split;
      if (a.d % a.k3.n_split || Kc % 64 || Kc > kCPL * 256) return false;
      const size_t seg = (size_t)Kc * 2;
      t.rows_per_stage = (int)std::max<size_t>(1, 32768 / seg);
      const size_t stage = (size_t)t.rows_per_stage * seg;
      t.stages = (int)std::min<size_t>(kMaxStages, (std::min<size_t>(budget, 200 * 1024) - 64) / stage);
      t.smem = (size_t)t.stages * stage + 2 * t.stages * 8 + 16;
    } else {
      t.kc = pick_kc(a.d, 34 * 1024);
      t.nch = a.d / t.kc;
      const int umax = std::min(a.E, maxB * Kk);
      const size_t SB = a128((size_t)kGroupRows * (t.kc * 2 + 16));
      const size_t act = a128((size_t)4 * (a.d * 2 + 16));
      const size_t extra = a128((size_t)(2 * umax + 1 + maxB * Kk) * 4) + 2 * kMaxStages * 8 +
                           kConsumerWarps * 64 * 4 + 64 + 128;
      t.stages = (int)std::min<size_t>(kMaxStages, (budget - act - extra) / SB);
      t.smem = (size_t)t.stages * SB + act + extra;
    }
    if (t.stages < 2) return false;
  }
  // K4: one expert's block of rows per stage; tables (+ activations when they fit) staged.
  {
    KTune& t = a.k4;
    t.rows_max = (a.d + G - 1) / G;
    if (t.rows_max > 7 * kConsumerWarps) return false;
    const int umax = std::min(a.E, maxB * Kk), nent = maxB * Kk;
    const size_t SB = a128((size_t)t.rows_max * a.I * 2);
    const size_t tables = (size_t)(2 * umax + 1 + 2 * nent) * 4 + 128;
    const size_t accs = (size_t)t.rows_max * maxB * 4;
    const size_t a_bytes = (size_t)nent * a.I * 4;
    const size_t fixed = tables + accs + 2 * kMaxStages * 8 + 64;
    t.a_in_smem = (a_bytes <= 64 * 1024 && fixed + a_bytes + 4 * SB <= budget) ? 1 : 0;
    const size_t rest = budget - fixed - (t.a_in_smem ? a_bytes : 0);
    t.stages = (int)std::min<size_t>(kMaxStages, rest / SB);
    if (t.stages < 2) return false;
    t.smem = (size_t)t.stages * SB + fixed + (t.a_in_smem ? a_bytes : 0);
  }
  return a.k1.smem <= budget && a.k2.smem <= budget && a.k3.smem <= budget && a.k4.smem <= budget;
}

cudaError_t set_kernel_attributes(size_t optin) {
  const int v = (int)optin;
  cudaError_t e = cudaSuccess;
#define SET(k)                                                                              \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, v); \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100)
  SET(k_oproj);
  SET(k_router_topk);
  SET(k_gateup_small);
  SET(k_gateup_splitk<2>);
  SET(k_down_combine<0>);
  SET(k_down_combine<1>);
  SET(k_down_combine<2>);
#undef SET
  return e;
}

cudaError_t launch_oproj(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_k(k_oproj, grid, a.k1.smem, s, pdl, a);
}

cudaError_t launch_router(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_k(k_router_topk, grid, a.k2.smem, s, pdl, a);
}

cudaError_t launch_gateup_small(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  if (a.B > 2) return cudaErrorInvalidValue;  // small-M covers batch 1 and 2
  return launch_k(k_gateup_small, grid, a.k3.smem, s, pdl, a);
}

cudaError_t launch_gateup_splitk(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_k(k_gateup_splitk<2>, grid, a.k3.smem, s, pdl, a);
}

cudaError_t launch_down(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  if (a.B == 1) return launch_k(k_down_combine<1>, grid, a.k4.smem, s, pdl, a);
  if (a.B == 2) return launch_k(k_down_combine<2>, grid, a.k4.smem, s, pdl, a);
  return launch_k(k_down_combine<0>, grid, a.k4.smem, s, pdl, a);
}

cudaError_t launch_prefetch(const PrefetchArgs& p, int grid, cudaStream_t s) {
  k_prefetch_l2<<<grid, 128, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace moe
