// sm_100a kernels of one MoE decode-layer step.
//
//   K1 k_oproj_rms      h = residual + W_o . attn_out; per-CTA sums of h^2; the last CTA
//                       (atomic ticket, no spinning) turns them into rstd.
//   K2 k_router_topk    x = h * rstd * gamma; logits = W_r . x (fp32); the last CTA selects
//                       the top-k per token (warp shuffles), the softmax gates, and builds
//                       the routing tables (union of selected experts, per-expert token
//                       entries in CSR form).
//   K3 k_gateup_small   small-M expert gate/up: each (union expert, row pair) streamed once,
//                       dotted with every token routed to it; a = silu(g) * u.
//      k_gateup_splitk  split-K expert gate/up for larger batches: (expert, K chunk) units,
//                       partial sums reduced in chunk order by the last unit of each expert.
//   K4 k_down_combine   out = bf16(h + sum_j gate_j * W_down[e_j] . a_j), rows of d split
//                       over CTAs, experts streamed in ascending order (deterministic).
//   k_prefetch_l2       side-stream L2 prefetch of the next layer's weights.
//
// Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted
// kernels", section "How the specialised decode path works" (batch-size kernel choice,
// o_proj fused with the residual step, next-layer prefetch, 16 of 896 experts).
//
// Structure shared by the streaming kernels: one CTA per SM, 8 consumer warps and one
// producer warp.  The producer's lane 0 streams weight rows into a shared-memory ring
// with TMA bulk copies (cp.async.bulk, mbarrier transaction counts, L2 evict-first);
// consumers hold their slice of the activations in registers, dot 16-byte weight chunks
// from shared memory, reduce across lanes with shuffles and across warps through shared
// memory in a fixed order, so every result is bit-reproducible.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kCPL = 4;  // 8-element chunks per lane: K <= 8 warps * 32 lanes * 4 * 8 = 8192

__device__ __forceinline__ float ld_act_bf16(const uint16_t* p) {
  return bf16f(__ldcg(reinterpret_cast<const unsigned short*>(p)));
}

// Chunk q of a K-long row handled by (warp cw, lane, i): q = cw*qpw + i*32 + lane,
// valid when i*32 + lane < qpw, where qpw = K/64 chunks per warp.
__device__ __forceinline__ bool chunk_valid(int qpw, int i, int lane) { return i * 32 + lane < qpw; }

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

}  // namespace

// =============================================================================
// K1: o_proj + residual + RMSNorm statistics
// =============================================================================
template <int NT>
__global__ void __launch_bounds__(kThreads, 1) k_oproj_rms(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, d_o = a.d_o, B = a.B;
  const int S = a.k1.stages, RS = a.k1.rows_per_stage, RM = a.k1.rows_max;
  const uint32_t row_bytes = (uint32_t)d_o * 2u;
  const uint32_t stage_bytes = (uint32_t)RS * row_bytes;
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int r0 = (int)lo, r1 = (int)hi, rows = r1 - r0;

  unsigned char* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  uint64_t* empty = full + S;
  float* part = reinterpret_cast<float*>(empty + S);  // [RM][8][NT]
  float* sq = part + RM * kConsumerWarps * NT;         // [RM][NT]
  int* s_misc = reinterpret_cast<int*>(sq + RM * NT);  // [0] abort, [1] last flag
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
  pdl_trigger();

  const int ngroups = (B + NT - 1) / NT;
  if (warp == kConsumerWarps) {
    // ---------------- producer: stream this CTA's rows of W_o (static weights) -----------
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      bool ok = true;
      for (int g = 0; g < ngroups && ok; ++g) {
        for (int r = r0; r < r1; r += RS, ++it) {
          const int n = min(RS, r1 - r);
          if (!ring_acquire(empty, it, S, abort_flag, a.ws.err)) { ok = false; break; }
          const int s = it % S;
          mbar_arrive_expect_tx(&full[s], n * row_bytes);
          bulk_g2s(ring + (size_t)s * stage_bytes, a.w_o + (size_t)r * d_o, n * row_bytes, &full[s], pol);
        }
      }
      ring_drain(full, it, S, a.ws.err);
    }
  } else {
    // ---------------- consumers ----------------------------------------------------------
    pdl_wait();  // activations (attn_out, residual) may come from the previous kernel
    const int cw = warp;
    const int qpw = d_o / 64;
    int it = 0;
    for (int g = 0; g < ngroups; ++g) {
      const int t0 = g * NT, nt = min(NT, B - t0);
      uint4 act[NT][kCPL];
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int i = 0; i < kCPL; ++i) {
          const int q = cw * qpw + i * 32 + lane;
          act[t][i] = (t < nt && chunk_valid(qpw, i, lane))
                          ? ld_act_u4(a.attn + (size_t)(t0 + t) * d_o + (size_t)q * 8)
                          : make_uint4(0, 0, 0, 0);
        }
      for (int r = r0; r < r1; r += RS, ++it) {
        const int n = min(RS, r1 - r), s = it % S;
        mbar_wait(&full[s], (it / S) & 1, abort_flag, a.ws.err);
        const unsigned char* st = ring + (size_t)s * stage_bytes;
        for (int j = 0; j < n; ++j) {
          float acc[NT];
#pragma unroll
          for (int t = 0; t < NT; ++t) acc[t] = 0.f;
#pragma unroll
          for (int i = 0; i < kCPL; ++i) {
            if (!chunk_valid(qpw, i, lane)) continue;
            const int q = cw * qpw + i * 32 + lane;
            const uint4 w = *reinterpret_cast<const uint4*>(st + (size_t)j * row_bytes + (size_t)q * 16);
            float wf[8];
            unpack8(w, wf);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              float af[8];
              unpack8(act[t][i], af);
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[t] = fmaf(wf[e], af[e], acc[t]);
            }
          }
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float v = warp_sum(acc[t]);
            if (lane == 0) part[((r - r0 + j) * kConsumerWarps + cw) * NT + t] = v;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      consumer_sync();
      const int tid = threadIdx.x;
      if (tid < rows) {
        for (int t = 0; t < nt; ++t) {
          float sacc = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) sacc += part[(tid * kConsumerWarps + w) * NT + t];
          const size_t o = (size_t)(t0 + t) * d + r0 + tid;
          const float hv = ld_act_bf16(a.resid + o) + sacc;
          a.ws.h[o] = hv;
          sq[tid * NT + t] = hv * hv;
        }
      }
      consumer_sync();
      if (tid < nt) {
        float ss = 0.f;
        for (int rr = 0; rr < rows; ++rr) ss += sq[rr * NT + tid];
        a.ws.ss_part[(size_t)c * a.maxB + t0 + tid] = ss;
      }
      consumer_sync();
    }
  }

  if (last_cta(&a.ws.counters[kCntOproj], &s_misc[1])) {
    for (int t = threadIdx.x; t < B; t += blockDim.x) {
      float ss = 0.f;
      for (int cc = 0; cc < G; ++cc) ss += ld_act(&a.ws.ss_part[(size_t)cc * a.maxB + t]);
      a.ws.rstd[t] = 1.0f / sqrtf(ss / (float)d + a.eps);
    }
    if (threadIdx.x == 0) a.ws.counters[kCntOproj] = 0;
  }
}

// =============================================================================
// K2: RMSNorm apply + router GEMV + top-k + gates + routing tables
// =============================================================================
namespace {

__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Executed by every thread of the last router CTA.  scratch >= 24 KB.
__device__ void topk_route(const LayerArgs& a, unsigned char* scratch) {
  const int B = a.B, E = a.E, K = a.k;
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(scratch);  // [E]
  int* off_e = reinterpret_cast<int*>(mask + 1024);                         // [E]
  int* uid = off_e + 1024;                                                  // [E]
  int* sidx = uid + 1024;                                                   // [B][K]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;

  for (int e = threadIdx.x; e < E; e += blockDim.x) mask[e] = 0ull;

  // ---- per-token selection: one warp per token -----------------------------------------
  for (int t = warp; t < B; t += nwarps) {
    float v[32];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = lane + 32 * i;
      float x = -INFINITY;
      if (e < E) {
        x = ld_act(&a.ws.logits[(size_t)t * E + e]);
        if (x != x) x = -INFINITY;  // NaN never outranks a number
      } else {
        taken |= 1u << i;
      }
      v[i] = x;
    }
    float lbv = -INFINITY;
    int lbi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (!((taken >> i) & 1u) && better(v[i], lane + 32 * i, lbv, lbi)) { lbv = v[i]; lbi = lane + 32 * i; }
    float my_v = 0.f;
    int my_i = 0;
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

  // ---- union of experts and CSR offsets (warp 0 scans E <= 1024 in 32-expert strips) ---
  if (warp == 0) {
    int cnt = 0, nu = 0;
    const int e0 = lane * 32;
    for (int e = e0; e < e0 + 32 && e < E; ++e) {
      const int c = __popcll(mask[e]);
      cnt += c;
      nu += (c > 0);
    }
    int icnt = cnt, inu = nu;  // inclusive scans across lanes
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
      uid[e] = c > 0 ? u : -1;
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

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) k_router_topk(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, E = a.E, B = a.B;
  const int RM = a.k2.rows_max;
  long long lo, hi;
  split_range(E, G, c, lo, hi);
  const int e0 = (int)lo, nrows = (int)(hi - lo);
  const uint32_t row_bytes = (uint32_t)d * 2u;

  unsigned char* wsl = smem;                                                    // [RM][d] bf16
  unsigned char* scratch = smem + (size_t)RM * row_bytes;                       // 24 KB (last CTA)
  uint64_t* full = reinterpret_cast<uint64_t*>(scratch + 24576);
  float* part = reinterpret_cast<float*>(full + 2);                            // [RM][8][NT]
  int* s_misc = reinterpret_cast<int*>(part + RM * kConsumerWarps * NT);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    s_misc[0] = 0;
    s_misc[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  if (warp == kConsumerWarps) {
    // Router slice is static: fetch it before the dependency resolves.
    if (lane == 0 && nrows > 0) {
      mbar_arrive_expect_tx(&full[0], nrows * row_bytes);
      bulk_g2s(wsl, a.w_r + (size_t)e0 * d, nrows * row_bytes, &full[0], policy_evict_first());
      mbar_drain(&full[0], 0, a.ws.err);
    }
  } else {
    const int cw = warp, qpw = d / 64;
    float gam[kCPL][8];
#pragma unroll
    for (int i = 0; i < kCPL; ++i) {
      const int q = cw * qpw + i * 32 + lane;
      if (chunk_valid(qpw, i, lane)) unpack8(ld_weight_u4(a.gamma + (size_t)q * 8), gam[i]);
      else
#pragma unroll
        for (int e = 0; e < 8; ++e) gam[i][e] = 0.f;
    }
    pdl_wait();
    bool have_w = false;
    for (int t0 = 0; t0 < B; t0 += NT) {
      const int nt = min(NT, B - t0);
      float xr[NT][kCPL][8];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float r = (t < nt) ? ld_act(&a.ws.rstd[t0 + t]) : 0.f;
#pragma unroll
        for (int i = 0; i < kCPL; ++i) {
          const int q = cw * qpw + i * 32 + lane;
          if (t < nt && chunk_valid(qpw, i, lane)) {
            const float* hp = a.ws.h + (size_t)(t0 + t) * d + (size_t)q * 8;
            const float4 h0 = ld_act4(hp), h1 = ld_act4(hp + 4);
            const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) xr[t][i][e] = hv[e] * r * gam[i][e];
            if (q % G == c) {  // each chunk of x is written by exactly one CTA
              float* xp = a.ws.x + (size_t)(t0 + t) * d + (size_t)q * 8;
              *reinterpret_cast<float4*>(xp) = make_float4(xr[t][i][0], xr[t][i][1], xr[t][i][2], xr[t][i][3]);
              *reinterpret_cast<float4*>(xp + 4) = make_float4(xr[t][i][4], xr[t][i][5], xr[t][i][6], xr[t][i][7]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) xr[t][i][e] = 0.f;
          }
        }
      }
      if (nrows > 0) {
        if (!have_w) {
          mbar_wait(&full[0], 0, abort_flag, a.ws.err);
          have_w = true;
        }
        for (int j = 0; j < nrows; ++j) {
          float acc[NT];
#pragma unroll
          for (int t = 0; t < NT; ++t) acc[t] = 0.f;
#pragma unroll
          for (int i = 0; i < kCPL; ++i) {
            if (!chunk_valid(qpw, i, lane)) continue;
            const int q = cw * qpw + i * 32 + lane;
            const uint4 w = *reinterpret_cast<const uint4*>(wsl + (size_t)j * row_bytes + (size_t)q * 16);
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[t] = dot8(w, xr[t][i], acc[t]);
          }
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float v = warp_sum(acc[t]);
            if (lane == 0) part[(j * kConsumerWarps + cw) * NT + t] = v;
          }
        }
      }
      consumer_sync();
      for (int p = threadIdx.x; p < nrows * nt; p += kConsumerThreads) {
        const int j = p / nt, t = p % nt;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) s += part[(j * kConsumerWarps + w) * NT + t];
        a.ws.logits[(size_t)(t0 + t) * E + e0 + j] = s;
      }
      consumer_sync();
    }
  }

  if (last_cta(&a.ws.counters[kCntRouter], &s_misc[1])) {
    topk_route(a, scratch);
    if (threadIdx.x == 0) a.ws.counters[kCntRouter] = 0;
  }
}

// =============================================================================
// K3 (small-M): expert gate/up + SiLU*mul, each (expert, row pair) streamed once
// =============================================================================
template <int NT>
__global__ void __launch_bounds__(kThreads, 1) k_gateup_small(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, I = a.I, E = a.E;
  const int S = a.k3.stages, RS = a.k3.rows_per_stage;
  const uint32_t row_bytes = (uint32_t)d * 2u;
  const uint32_t half_bytes = (uint32_t)RS * row_bytes;  // gate rows, then up rows
  const uint32_t stage_bytes = 2u * half_bytes;

  unsigned char* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  uint64_t* empty = full + S;
  float* part = reinterpret_cast<float*>(empty + S);  // [RS][2][8][NT]
  int* s_misc = reinterpret_cast<int*>(part + RS * 2 * kConsumerWarps * NT);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    s_misc[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // routing tables come from the router kernel
  pdl_trigger();

  const int U = ld_act_i(a.ws.n_union);
  const long long total = (long long)U * I;
  long long q0, q1;
  split_range(total, G, c, q0, q1);

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      for (long long q = q0; q < q1; ++it) {
        const int u = (int)(q / I), p = (int)(q % I);
        const int n = (int)min((long long)min(RS, I - p), q1 - q);
        int e = ld_act_i(&a.ws.union_e[u]);
        if (e < 0 || e >= E) { atomicOr(a.ws.err, kErrBounds); e = 0; }
        if (!ring_acquire(empty, it, S, abort_flag, a.ws.err)) break;
        const int s = it % S;
        const uint16_t* gsrc = a.w_gu + ((size_t)e * 2 * I + p) * d;
        const uint16_t* usrc = a.w_gu + ((size_t)e * 2 * I + I + p) * d;
        mbar_arrive_expect_tx(&full[s], 2u * n * row_bytes);
        bulk_g2s(ring + (size_t)s * stage_bytes, gsrc, n * row_bytes, &full[s], pol);
        bulk_g2s(ring + (size_t)s * stage_bytes + half_bytes, usrc, n * row_bytes, &full[s], pol);
        q += n;
      }
      ring_drain(full, it, S, a.ws.err);
    }
  } else {
    const int cw = warp, qpw = d / 64;
    float xr[NT][kCPL][8];
    int cur_u = -1, cur_g = -1;
    int it = 0;
    for (long long q = q0; q < q1; ++it) {
      const int u = (int)(q / I), p = (int)(q % I);
      const int n = (int)min((long long)min(RS, I - p), q1 - q);
      const int off = ld_act_i(&a.ws.union_off[u]);
      const int m = ld_act_i(&a.ws.union_off[u + 1]) - off;
      const int s = it % S;
      mbar_wait(&full[s], (it / S) & 1, abort_flag, a.ws.err);
      const unsigned char* st = ring + (size_t)s * stage_bytes;
      for (int g0 = 0; g0 < m; g0 += NT) {
        const int nt = min(NT, m - g0);
        if (u != cur_u || g0 != cur_g) {
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            int tok = (t < nt) ? ld_act_i(&a.ws.entry_tok[off + g0 + t]) : -1;
            if (tok >= a.B) { atomicOr(a.ws.err, kErrBounds); tok = -1; }
#pragma unroll
            for (int i = 0; i < kCPL; ++i) {
              const int qq = cw * qpw + i * 32 + lane;
              if (tok >= 0 && chunk_valid(qpw, i, lane)) {
                const float* xp = a.ws.x + (size_t)tok * d + (size_t)qq * 8;
                const float4 x0 = ld_act4(xp), x1 = ld_act4(xp + 4);
                xr[t][i][0] = x0.x; xr[t][i][1] = x0.y; xr[t][i][2] = x0.z; xr[t][i][3] = x0.w;
                xr[t][i][4] = x1.x; xr[t][i][5] = x1.y; xr[t][i][6] = x1.z; xr[t][i][7] = x1.w;
              } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) xr[t][i][e] = 0.f;
              }
            }
          }
          cur_u = u;
          cur_g = g0;
        }
        for (int j = 0; j < 2 * n; ++j) {  // rows: gate 0..n-1, then up 0..n-1
          const unsigned char* row = st + (j < n ? (size_t)j * row_bytes : half_bytes + (size_t)(j - n) * row_bytes);
          float acc[NT];
#pragma unroll
          for (int t = 0; t < NT; ++t) acc[t] = 0.f;
#pragma unroll
          for (int i = 0; i < kCPL; ++i) {
            if (!chunk_valid(qpw, i, lane)) continue;
            const int qq = cw * qpw + i * 32 + lane;
            const uint4 w = *reinterpret_cast<const uint4*>(row + (size_t)qq * 16);
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[t] = dot8(w, xr[t][i], acc[t]);
          }
          const int pr = j < n ? j : j - n, gu = j < n ? 0 : 1;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float v = warp_sum(acc[t]);
            if (lane == 0) part[((pr * 2 + gu) * kConsumerWarps + cw) * NT + t] = v;
          }
        }
        consumer_sync();
        for (int z = threadIdx.x; z < n * nt; z += kConsumerThreads) {
          const int pr = z / nt, t = z % nt;
          float gs = 0.f, us = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            gs += part[((pr * 2 + 0) * kConsumerWarps + w) * NT + t];
            us += part[((pr * 2 + 1) * kConsumerWarps + w) * NT + t];
          }
          const float act = gs / (1.0f + expf(-gs)) * us;
          a.ws.a[(size_t)(off + g0 + t) * I + p + pr] = act;
        }
        consumer_sync();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      q += n;
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
    // Lane mapping inside a K chunk: 8-element chunks qq = i*32 + lane, i < Kc/256.
    // Stages outer, token groups inner, so each stage is released after its last group.
    const int cpl = Kc / 256;  // chunks per lane (Kc is a multiple of 256, at most kCPL*256)
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
                if (tok >= 0 && i < cpl) {
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
              if (i >= cpl) continue;
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
// =============================================================================
__global__ void __launch_bounds__(kThreads, 1) k_down_combine(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, I = a.I, E = a.E, B = a.B, K = a.k;
  const int S = a.k4.stages, RM = a.k4.rows_max;
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int i0 = (int)lo, nrows = (int)(hi - lo);
  const uint32_t row_bytes = (uint32_t)I * 2u;
  const uint32_t stage_bytes = (uint32_t)RM * row_bytes;

  unsigned char* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  uint64_t* empty = full + S;
  float* acc_s = reinterpret_cast<float*>(empty + S);  // [RM][maxB]
  int* s_misc = reinterpret_cast<int*>(acc_s + RM * a.maxB);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    s_misc[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  const int U = ld_act_i(a.ws.n_union);

  if (warp == kConsumerWarps) {
    if (lane == 0 && nrows > 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      for (int u = 0; u < U; ++u, ++it) {
        int e = ld_act_i(&a.ws.union_e[u]);
        if (e < 0 || e >= E) { atomicOr(a.ws.err, kErrBounds); e = 0; }
        if (!ring_acquire(empty, it, S, abort_flag, a.ws.err)) break;
        const int s = it % S;
        mbar_arrive_expect_tx(&full[s], nrows * row_bytes);
        bulk_g2s(ring + (size_t)s * stage_bytes, a.w_down + ((size_t)e * d + i0) * I, nrows * row_bytes,
                 &full[s], pol);
      }
      ring_drain(full, it, S, a.ws.err);
    }
  } else {
    for (int z = threadIdx.x; z < nrows * B; z += kConsumerThreads) acc_s[z] = 0.f;
    consumer_sync();
    const int epl = I / 32;  // elements per lane (1..16)
    if (nrows > 0) {
      for (int u = 0; u < U; ++u) {
        const int s = u % S;
        mbar_wait(&full[s], (u / S) & 1, abort_flag, a.ws.err);
        const unsigned char* st = ring + (size_t)s * stage_bytes;
        const int off = ld_act_i(&a.ws.union_off[u]);
        const int m = ld_act_i(&a.ws.union_off[u + 1]) - off;
        for (int en = 0; en < m; ++en) {
          const int pos = off + en;
          int t = ld_act_i(&a.ws.entry_tok[pos]);
          int j = ld_act_i(&a.ws.entry_slot[pos]);
          if (t < 0 || t >= B || j < 0 || j >= K) { atomicOr(a.ws.err, kErrBounds); continue; }
          const float gte = ld_act(&a.ws.topk_gate[t * K + j]);
          float av[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) av[x] = (x < epl) ? ld_act(&a.ws.a[(size_t)pos * I + lane * epl + x]) : 0.f;
          for (int rl = warp; rl < nrows; rl += kConsumerWarps) {
            const uint16_t* wr = reinterpret_cast<const uint16_t*>(st + (size_t)rl * row_bytes) + lane * epl;
            float dsum = 0.f;
#pragma unroll
            for (int x = 0; x < 16; ++x)
              if (x < epl) dsum = fmaf(bf16f(wr[x]), av[x], dsum);
            dsum = warp_sum(dsum);
            if (lane == 0) acc_s[rl * B + t] += gte * dsum;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
    consumer_sync();
    for (int z = threadIdx.x; z < nrows * B; z += kConsumerThreads) {
      const int rl = z / B, t = z % B;
      const size_t o = (size_t)t * d + i0 + rl;
      const float v = ld_act(&a.ws.h[o]) + acc_s[z];
      const __nv_bfloat16 bv = __float2bfloat16_rn(v);
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

size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

}  // namespace

bool plan_layer(LayerArgs& a, int G, size_t optin) {
  const size_t budget = optin - 1024;  // leave room for the static reservation
  // K1: rows of W_o (d_o*2 bytes each), ~32 KB stages.
  {
    KTune& t = a.k1;
    const size_t row = (size_t)a.d_o * 2;
    t.rows_max = (a.d + G - 1) / G;
    t.rows_per_stage = (int)std::max<size_t>(1, std::min<size_t>(32768 / row, (size_t)t.rows_max));
    const int NT = 4;
    const size_t extra = align16((size_t)t.rows_max * kConsumerWarps * NT * 4 + (size_t)t.rows_max * NT * 4 + 16) +
                         2 * kMaxStages * 8;
    const size_t stage = (size_t)t.rows_per_stage * row;
    t.stages = (int)std::min<size_t>(kMaxStages, (std::min<size_t>(budget, 200 * 1024) - extra) / stage);
    if (t.stages < 2) return false;
    t.smem = (size_t)t.stages * stage + 2 * t.stages * 8 + extra;
    if (t.rows_max > kConsumerThreads) return false;
  }
  // K2: whole router slice resident.
  {
    KTune& t = a.k2;
    t.rows_max = (a.E + G - 1) / G;
    const int NT = 2;
    t.smem = align16((size_t)t.rows_max * a.d * 2) + 24576 + 16 + (size_t)t.rows_max * kConsumerWarps * NT * 4 + 16;
    if (t.smem > budget) return false;
  }
  // K3: small-M (row pairs, full K) or split-K (row segments of one K chunk).
  {
    KTune& t = a.k3;
    const size_t row = (size_t)a.d * 2;
    if (a.k3.n_split > 0) {
      const int Kc = a.d / a.k3.n_split;
      if (a.d % a.k3.n_split || Kc % 256 || Kc > kCPL * 256) return false;
      const size_t seg = (size_t)Kc * 2;
      t.rows_per_stage = (int)std::max<size_t>(1, 32768 / seg);
      const size_t stage = (size_t)t.rows_per_stage * seg;
      t.stages = (int)std::min<size_t>(kMaxStages, (std::min<size_t>(budget, 200 * 1024) - 64) / stage);
      t.smem = (size_t)t.stages * stage + 2 * t.stages * 8 + 16;
    } else {
      t.rows_per_stage = 1;
      const int NT = 2;
      const size_t stage = 2 * (size_t)t.rows_per_stage * row;
      const size_t extra = (size_t)t.rows_per_stage * 2 * kConsumerWarps * NT * 4 + 16;
      t.stages = (int)std::min<size_t>(kMaxStages, (std::min<size_t>(budget, 200 * 1024) - extra) / stage);
      t.smem = (size_t)t.stages * stage + 2 * t.stages * 8 + extra;
    }
    if (t.stages < 2) return false;
  }
  // K4: one expert's block of rows per stage.
  {
    KTune& t = a.k4;
    t.rows_max = (a.d + G - 1) / G;
    const size_t stage = (size_t)t.rows_max * a.I * 2;
    const size_t extra = (size_t)t.rows_max * a.maxB * 4 + 16;
    t.stages = (int)std::min<size_t>(kMaxStages, (std::min<size_t>(budget, 200 * 1024) - extra) / stage);
    if (t.stages < 2) return false;
    t.smem = (size_t)t.stages * stage + 2 * t.stages * 8 + extra;
  }
  return a.k1.smem <= budget && a.k2.smem <= budget && a.k3.smem <= budget && a.k4.smem <= budget;
}

cudaError_t set_kernel_attributes(size_t optin) {
  const int v = (int)optin;
  cudaError_t e = cudaSuccess;
#define SET(k) if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, v)
  SET(k_oproj_rms<1>); SET(k_oproj_rms<2>); SET(k_oproj_rms<4>);
  SET(k_router_topk<1>); SET(k_router_topk<2>);
  SET(k_gateup_small<1>); SET(k_gateup_small<2>);
  SET(k_gateup_splitk<2>);
  SET(k_down_combine);
#undef SET
  return e;
}

cudaError_t launch_oproj(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  if (a.B <= 1) return launch_k(k_oproj_rms<1>, grid, a.k1.smem, s, pdl, a);
  if (a.B <= 2) return launch_k(k_oproj_rms<2>, grid, a.k1.smem, s, pdl, a);
  return launch_k(k_oproj_rms<4>, grid, a.k1.smem, s, pdl, a);
}

cudaError_t launch_router(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  if (a.B <= 1) return launch_k(k_router_topk<1>, grid, a.k2.smem, s, pdl, a);
  return launch_k(k_router_topk<2>, grid, a.k2.smem, s, pdl, a);
}

cudaError_t launch_gateup_small(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  if (a.B <= 1) return launch_k(k_gateup_small<1>, grid, a.k3.smem, s, pdl, a);
  return launch_k(k_gateup_small<2>, grid, a.k3.smem, s, pdl, a);
}

cudaError_t launch_gateup_splitk(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_k(k_gateup_splitk<2>, grid, a.k3.smem, s, pdl, a);
}

cudaError_t launch_down(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_k(k_down_combine, grid, a.k4.smem, s, pdl, a);
}

cudaError_t launch_prefetch(const PrefetchArgs& p, int grid, cudaStream_t s) {
  k_prefetch_l2<<<grid, 128, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace moe
