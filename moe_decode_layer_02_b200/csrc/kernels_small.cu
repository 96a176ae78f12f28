// Small-batch kernels: whole weight rows streamed by TMA, fp32 dot products.
//
// A decode step at batch 1-2 reads 218-306 MB of weights and does about one flop per
// byte, so every kernel here is a weight stream.  What limits it is keeping enough bytes
// in flight with few expensive operations:
//   * the producer warp moves weights with one 1-D bulk copy per stage of whole,
//     contiguous rows (12-56 KB per copy; each bulk copy has a fixed issue cost of the
//     order of a hundred nanoseconds, so many small copies cannot feed an SM);
//   * a ring of up to 8 stages keeps ~100-200 KB in flight per SM;
//   * the 8 consumer warps split K: each holds its slice of the activations in registers
//     as fp32 (exact; x is not rounded for the router), reads 16-byte weight chunks from
//     shared memory (lanes contiguous, conflict-free) and accumulates in fp32;
//   * row partials go to shared memory and are reduced once, in a fixed order, at the end.
// RMSNorm statistics are per-CTA partial sums that every router CTA reduces itself in the
// same order, and the top-k selection and routing are recomputed in every expert CTA.
//
//   k_layer_f    batch 1: the whole layer step as one cooperative launch (the three kernels
//                below as phases, with grid barriers where the kernel boundaries were)
//   k_oproj_f    h = residual + W_o . attn_out, per-CTA sums of h^2         (batch 2 to 4)
//   k_router_f   rstd, x = h * rstd * gamma, logits = W_r . x   (batch 2 to 4; on the
//                large-batch path where k_router_big does not fit, its last CTA also
//                building the global routing tables)
//   k_router_big a router of the large-batch path, h staged by TMA, plus the routing tables
//   k_experts_f  the expert kernel (batch 2 to 4, batch x top-k <= 64): routing once per
//                CTA; gate/up + SiLU*mul
//                for each (selected expert, row pair), each pair streamed once; a grid
//                barrier; then out = bf16(h + sum_j gate_j * W_down[e_j] . a_j), with W_down
//                streaming into the freed ring while the barrier is open
//
// Weights are static, so producers issue their first copies before the programmatic-
// launch dependency wait; activations are read only after it, with L2 loads.
//
// Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted
// kernels", section "How the specialised decode path works" (small-matrix kernels at
// batch one or two; o_proj fused with the residual step; 16 of 896 experts per token).
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "rowdot.cuh"
#include "topk.cuh"

namespace moe {

namespace {

static_assert(kThreadsS == kRouteThreads, "the expert kernel routes with all of its threads");

// Phase B experts per stage for EPL elements per lane (registers bound it).
// Union experts per phase-B stage: the stage's activations of every token are held in
// registers (kEPS * NT * EPL floats per lane), so four tokens take half as many.
__host__ __device__ constexpr int experts_per_stage(int epl, int nt) {
  return epl == 4 ? (nt > 2 ? 2 : 4) : (epl == 8 ? (nt > 2 ? 1 : 2) : 1);
}

// Phase B's gated activations in shared memory.  Up to two tokens: dense, [U][NT][I] with
// zeros where a token did not select the union expert.  Four tokens (where the dense form
// would take up to 128 KB): one row per entry, [B K][I], then the entry of each (union
// expert, token) pair, [min(E, B K)][NT] ints (-1 where the token did not select it).
__host__ __device__ constexpr size_t a_s_floats(int B, int K, int E, int I, int NT) {
  return NT <= 2 ? (size_t)(E < B * K ? E : B * K) * NT * I
                 : (size_t)B * K * I + (((size_t)(E < B * K ? E : B * K) * NT + 3) & ~size_t(3));
}

}  // namespace

// =============================================================================
// K1: o_proj + residual + per-CTA sums of h^2 (batch <= 4)
//   CTA c owns rows [r0, r1) of W_o (contiguous); a stage is RS whole rows (one copy).
// =============================================================================
// CPO 2: d_o <= 7680, the K slice split evenly over the 15 warps in at most two 32-lane chunk
// rounds; CPO 3: two full rounds per warp (64 chunks) and the rest as a third round in the
// first warps only (rows_dot_bf_2x).
template <int NT, int CPO>
__global__ void __launch_bounds__(kThreadsS, 1) k_oproj_f(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, d_o = a.d_o, B = a.B;
  const int S = a.k1.stages, RS = a.k1.rows_per_stage, RM = a.k1.rows_max;
  const uint32_t row_bytes = (uint32_t)d_o * 2u;
  const size_t SB = al128((size_t)RS * row_bytes);
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int r0 = (int)lo, r1 = (int)hi, rows = r1 - r0;

  unsigned char* ring = smem;
  float* part = reinterpret_cast<float*>(ring + (size_t)S * SB);  // [RM][8][NT]
  float* sq = part + RM * kCW * NT;                     // [NT][RM]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + al128((size_t)S * SB + ((size_t)RM * kCW * NT +
                                                                              (size_t)NT * RM) * 4));
  uint64_t* empty = full + S;
  int* s_misc = reinterpret_cast<int*>(empty + S);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(full, empty, S, kCW);
    s_misc[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  if (warp == kCW) {
    if (lane == 0) {  // W_o is static: stream it before the dependency resolves
      const uint64_t pol = policy_evict_first();
      int it = 0;
      for (int r = r0; r < r1; r += RS, ++it) {
        const int n = min(RS, r1 - r);
        if (!ring_acquire(empty, it, S, abort_flag, a.ws.err)) break;
        const int s = it % S;
        mbar_arrive_expect_tx(&full[s], n * row_bytes);
        bulk_g2s(ring + s * SB, a.w_o + (size_t)r * d_o, n * row_bytes, &full[s], pol);
      }
      ring_drain(full, it, S, a.ws.err);
    }
    return;
  }

  pdl_wait();  // attn_out and residual may come from the previous kernel
  constexpr int kRI = 2;  // rows per interleaved pass (a stage is two rows at d_o = 8192)
  const int nch = d_o / 8;
  const int qbase = CPO == 2 ? nch * warp / kCW : 64 * warp;
  const int qpw = CPO == 2 ? nch * (warp + 1) / kCW - qbase : 64;
  const int qx = kCW * 64 + 32 * warp;  // CPO 3: this warp's third round, if any
  const bool has_x = CPO == 3 && qx < nch;
  uint4 xa[NT][CPO];  // attn_out stays packed bf16 (mixed-precision FMAs)
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int j = 0; j < CPO; ++j) {
      uint4 u = make_uint4(0, 0, 0, 0);
      const int q = (j < 2) ? qbase + j * 32 + lane : qx + lane;
      const bool ok = (j < 2) ? cvalid(qpw, j, lane) : (has_x && q < nch);
      if (t < B && ok) u = ld_act_u4(a.attn + (size_t)t * d_o + (size_t)q * 8);
      xa[t][j] = u;
    }
  int it = 0;
  for (int r = r0; r < r1; r += RS, ++it) {
    const int n = min(RS, r1 - r), s = it % S;
    mbar_wait(&full[s], (it / S) & 1, abort_flag, a.ws.err);
    const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + s * SB);
    for (int j0 = 0; j0 < n; j0 += kRI) {
      const uint16_t* rp[kRI];
#pragma unroll
      for (int k = 0; k < kRI; ++k) rp[k] = st + (size_t)min(j0 + k, n - 1) * d_o;
      float v[kRI * NT];
      if constexpr (CPO == 2) rows_dot_bf<NT, kRI>(rp, n - j0, xa, qbase, qpw, lane, v);
      else rows_dot_bf_2x<NT, kRI>(rp, n - j0, xa, qbase, qx, nch, has_x, lane, v);
      const float tot = warp_reduce_multi<kRI * NT>(v, lane);
      const int vi = multi_index<kRI * NT>(lane), j = j0 + vi / NT, t = vi % NT;
      if (multi_writer<kRI * NT>(lane) && j < n) part[((r - r0 + j) * kCW + warp) * NT + t] = tot;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  csync();
  for (int z = tid; z < rows * B; z += kCT) {
    const int rr = z / B, t = z % B;
    float sacc = 0.f;
#pragma unroll
    for (int w = 0; w < kCW; ++w) sacc += part[(rr * kCW + w) * NT + t];
    const size_t o = (size_t)t * d + r0 + rr;
    const float hv = bf16f(__ldcg(reinterpret_cast<const unsigned short*>(a.resid + o))) + sacc;
    a.ws.h[o] = hv;
    sq[t * RM + rr] = hv * hv;
  }
  csync();
  if (warp < B) {  // per-CTA sum of h^2, fixed order
    float ss = 0.f;
    for (int rr = lane; rr < rows; rr += 32) ss += sq[warp * RM + rr];
    ss = warp_sum(ss);
    if (lane == 0) a.ws.ss_part[(size_t)c * a.maxB + warp] = ss;
  }
}

// =============================================================================
// K2: RMSNorm apply + router GEMV (any batch, tokens in groups of NT)
//   CTA c owns rows [e0, e0 + nrows) of W_r: the whole slice is one bulk copy, issued before
//   the dependency wait.  x is exact fp32 in registers.
// =============================================================================
template <int NT, int CPD>
__global__ void __launch_bounds__(kThreadsS, 1) k_router_f(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, E = a.E, B = a.B;
  const int RM = a.k2.rows_max;
  long long lo, hi;
  split_range(E, G, c, lo, hi);
  const int e0 = (int)lo, nrows = (int)(hi - lo);
  const uint32_t row_bytes = (uint32_t)d * 2u;

  uint16_t* wsl = reinterpret_cast<uint16_t*>(smem);                                 // [RM][d]
  float* part = reinterpret_cast<float*>(smem + al128((size_t)RM * row_bytes));    // [RM][8][NT]
  float* rstd_s = part + RM * kCW * NT;                                  // [64]
  uint64_t* full = reinterpret_cast<uint64_t*>(
      smem + al128(static_cast<size_t>(reinterpret_cast<unsigned char*>(rstd_s + 64) - smem)));
  int* s_misc = reinterpret_cast<int*>(full + 1);
  unsigned char* scratch = reinterpret_cast<unsigned char*>(s_misc + 32);          // routing tables
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(full, nullptr, 1);
    s_misc[0] = 0;
    s_misc[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  if (warp == kCW) {
    if (lane == 0 && nrows > 0) {
      mbar_arrive_expect_tx(&full[0], nrows * row_bytes);
      bulk_g2s(wsl, a.w_r + (size_t)e0 * d, nrows * row_bytes, &full[0], policy_evict_first());
    }
    if (lane == 0 && a.pf_w_o) {
      // Next layer: warm L2 while this layer's router, top-k and first expert bytes leave HBM
      // idle.  Each CTA prefetches what the same CTA of the next layer reads first: its router
      // rows and the leading rows of its share of W_o.
      if (nrows > 0) bulk_prefetch_l2(a.pf_w_r + (size_t)e0 * d, nrows * row_bytes);
      if (c == 0) bulk_prefetch_l2(a.pf_gamma, (uint32_t)d * 2u);
      long long o0, o1;
      split_range(d, G, c, o0, o1);
      const size_t orow = (size_t)a.d_o * 2;
      size_t left = (size_t)min((long long)a.pf_w_o_rows, o1 - o0) * orow;
      const unsigned char* src = reinterpret_cast<const unsigned char*>(a.pf_w_o + (size_t)o0 * a.d_o);
      for (size_t off = 0; left > 0;) {
        const uint32_t n = (uint32_t)min(left, (size_t)65536);
        bulk_prefetch_l2(src + off, n);
        off += n;
        left -= n;
      }
    }
    if (lane == 0 && nrows > 0) mbar_drain(&full[0], 0, a.ws.err);
  } else {
    const int qbase = (d / 8) * warp / kCW, qpw = (d / 8) * (warp + 1) / kCW - qbase;
    float gam[CPD][8];
#pragma unroll
    for (int j = 0; j < CPD; ++j) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (cvalid(qpw, j, lane)) u = ld_weight_u4(a.gamma + (size_t)(qbase + j * 32 + lane) * 8);
      unpack8f(u, gam[j]);
    }
    pdl_wait();  // h and the sums of h^2 come from the o_proj kernel
    if (c == 0 && tid == 0) a.ws.counters[kCntGateUp] = 0;  // the expert kernel's grid barrier count
    // h of the first token group, loaded while the sums of h^2 are reduced
    float xr[NT][CPD][8];
    auto load_h = [&](int t0, int nt) {
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int j = 0; j < CPD; ++j) {
          if (t < nt && cvalid(qpw, j, lane)) {
            const float* hp = a.ws.h + (size_t)(t0 + t) * d + (size_t)(qbase + j * 32 + lane) * 8;
            const float4 h0 = ld_act4(hp), h1 = ld_act4(hp + 4);
            xr[t][j][0] = h0.x; xr[t][j][1] = h0.y; xr[t][j][2] = h0.z; xr[t][j][3] = h0.w;
            xr[t][j][4] = h1.x; xr[t][j][5] = h1.y; xr[t][j][6] = h1.z; xr[t][j][7] = h1.w;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) xr[t][j][e] = 0.f;
          }
        }
    };
    load_h(0, min(NT, B));
    for (int t = warp; t < B; t += kCW) {  // fixed order: same bits in every CTA
      float ss = 0.f;
      for (int c0 = 0; c0 < G; c0 += 8 * 32) {  // eight independent loads per lane in flight
        float pv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int cc = c0 + k * 32 + lane;
          pv[k] = cc < G ? ld_act(&a.ws.ss_part[(size_t)cc * a.maxB + t]) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) ss += pv[k];
      }
      ss = warp_sum(ss);
      if (lane == 0) {
        const float r = 1.0f / sqrtf(ss / (float)d + a.eps);
        rstd_s[t] = r;
        if (c == 0) a.ws.rstd[t] = r;
      }
    }
    csync();
    bool have_w = false;
    for (int t0 = 0; t0 < B; t0 += NT) {
      const int nt = min(NT, B - t0);
      if (t0 > 0) load_h(t0, nt);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float r = (t < nt) ? rstd_s[t0 + t] : 0.f;
#pragma unroll
        for (int j = 0; j < CPD; ++j) {
          const int q = qbase + j * 32 + lane;
#pragma unroll
          for (int e = 0; e < 8; ++e) xr[t][j][e] = xr[t][j][e] * r * gam[j][e];
          if (t < nt && cvalid(qpw, j, lane) && q % G == c) {  // each chunk of x is written by one CTA
            float* xp = a.ws.x + (size_t)(t0 + t) * d + (size_t)q * 8;
            *reinterpret_cast<float4*>(xp) = make_float4(xr[t][j][0], xr[t][j][1], xr[t][j][2], xr[t][j][3]);
            *reinterpret_cast<float4*>(xp + 4) = make_float4(xr[t][j][4], xr[t][j][5], xr[t][j][6], xr[t][j][7]);
          }
        }
      }
      if (nrows > 0) {
        if (!have_w) {
          mbar_wait(&full[0], 0, abort_flag, a.ws.err);
          have_w = true;
        }
        constexpr int kRI = NT > 2 ? 2 : 4 / NT;  // rows per interleaved pass (four tokens: CPD 2)
        for (int j0 = 0; j0 < nrows; j0 += kRI) {
          const uint16_t* rp[kRI];
#pragma unroll
          for (int k = 0; k < kRI; ++k) rp[k] = wsl + (size_t)min(j0 + k, nrows - 1) * d;
          float v[kRI * NT];
          rows_dot<NT, kRI>(rp, nrows - j0, xr, qbase, qpw, lane, v);
          const float tot = warp_reduce_multi<kRI * NT>(v, lane);
          const int vi = multi_index<kRI * NT>(lane), j = j0 + vi / NT, t = vi % NT;
          if (multi_writer<kRI * NT>(lane) && j < nrows) part[(j * kCW + warp) * NT + t] = tot;
        }
      }
      csync();
      for (int z = tid; z < nrows * nt; z += kCT) {
        const int j = z / nt, t = z % nt;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kCW; ++w) s += part[(j * kCW + w) * NT + t];
        a.ws.logits[(size_t)(t0 + t) * E + e0 + j] = s;
      }
      csync();
    }
  }
  if (a.route_tables) {  // large-batch expert kernels: the last CTA builds the routing tables
    if (last_cta_s(&a.ws.counters[kCntRouter], &s_misc[1])) {
      topk_route(a, scratch);
      if (tid == 0) a.ws.counters[kCntRouter] = 0;
    }
  }
}

// =============================================================================
// Router of the large-batch path: the same arithmetic as k_router_f, with h staged by TMA.
//   The CTA's W_r slice is one bulk copy issued before the dependency wait (as in
//   k_router_f).  After it, the producer streams h two tokens at a time (one bulk copy of
//   2 x d fp32) into a ring, so the consumers never wait on an L2 round trip per token pair:
//   they turn a stage into x = h * rstd * gamma in registers (releasing the stage at once),
//   write their share of x, and dot it with the staged router rows.  The partial sums of
//   consecutive pairs alternate between two buffers.  The last CTA then builds the routing
//   tables, with the ring as its scratch.
// =============================================================================
__global__ void __launch_bounds__(kThreadsS, 1) k_router_big(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int NT = 2;
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, E = a.E, B = a.B;
  const int RM = a.k2.rows_max, SH = a.k2.stages;
  long long lo, hi;
  split_range(E, G, c, lo, hi);
  const int e0 = (int)lo, nrows = (int)(hi - lo);
  const uint32_t row_bytes = (uint32_t)d * 2u, hrow_bytes = (uint32_t)d * 4u;
  const size_t SHB = al128((size_t)NT * hrow_bytes);  // one stage: two tokens of h
  const size_t region = std::max((size_t)SH * SHB, (size_t)kTopkScratch);

  uint16_t* wsl = reinterpret_cast<uint16_t*>(smem);                                  // [RM][d]
  unsigned char* ring = smem + al128((size_t)RM * row_bytes);                          // h stages
  float* part = reinterpret_cast<float*>(ring + region);                               // [2][RM][kCW][NT]
  float* rstd_s = part + 2 * RM * kCW * NT;                                            // [64]
  uint64_t* fullW = reinterpret_cast<uint64_t*>(
      smem + al128(static_cast<size_t>(reinterpret_cast<unsigned char*>(rstd_s + 64) - smem)));
  uint64_t* fullH = fullW + 1;
  uint64_t* emptyH = fullH + kMaxStages;
  int* s_misc = reinterpret_cast<int*>(emptyH + kMaxStages);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(fullW, nullptr, 1);
    init_ring(fullH, emptyH, SH, kCW);
    s_misc[0] = 0;
    s_misc[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  const int npairs = (B + NT - 1) / NT;
  if (warp == kCW) {
    if (lane == 0) {
      if (nrows > 0) {
        mbar_arrive_expect_tx(&fullW[0], nrows * row_bytes);
        bulk_g2s(wsl, a.w_r + (size_t)e0 * d, nrows * row_bytes, &fullW[0], policy_evict_first());
      }
      if (a.pf_w_o) {  // next layer's first reads into L2, as in k_router_f
        if (nrows > 0) bulk_prefetch_l2(a.pf_w_r + (size_t)e0 * d, nrows * row_bytes);
        if (c == 0) bulk_prefetch_l2(a.pf_gamma, row_bytes);
        long long o0, o1;
        split_range(d, G, c, o0, o1);
        const size_t orow = (size_t)a.d_o * 2;
        size_t left = (size_t)min((long long)a.pf_w_o_rows, o1 - o0) * orow;
        const unsigned char* src = reinterpret_cast<const unsigned char*>(a.pf_w_o + (size_t)o0 * a.d_o);
        for (size_t off = 0; left > 0;) {
          const uint32_t n = (uint32_t)min(left, (size_t)65536);
          bulk_prefetch_l2(src + off, n);
          off += n;
          left -= n;
        }
      }
      pdl_wait();  // h comes from the o_proj kernel
      const uint64_t pol = policy_evict_first();
      int g = 0;
      for (; g < npairs; ++g) {
        const int nt = min(NT, B - g * NT);
        if (!ring_acquire(emptyH, g, SH, abort_flag, a.ws.err)) break;
        const int s = g % SH;
        mbar_arrive_expect_tx(&fullH[s], nt * hrow_bytes);
        bulk_g2s(ring + s * SHB, a.ws.h + (size_t)g * NT * d, nt * hrow_bytes, &fullH[s], pol);
      }
      ring_drain(fullH, g, SH, a.ws.err);
      if (nrows > 0) mbar_drain(&fullW[0], 0, a.ws.err);
    }
  } else {
    const int qbase = (d / 8) * warp / kCW, qpw = (d / 8) * (warp + 1) / kCW - qbase;
    float gam[kCPLf][8];
#pragma unroll
    for (int j = 0; j < kCPLf; ++j) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (cvalid(qpw, j, lane)) u = ld_weight_u4(a.gamma + (size_t)(qbase + j * 32 + lane) * 8);
      unpack8f(u, gam[j]);
    }
    pdl_wait();  // the sums of h^2 come from the o_proj kernel
    if (c == 0 && tid == 0) a.ws.counters[kCntGateUp] = 0;  // the expert kernels' grid barrier count
    for (int t = warp; t < B; t += kCW) {  // fixed order: same bits in every CTA
      float ss = 0.f;
      for (int c0 = 0; c0 < G; c0 += 8 * 32) {
        float pv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int cc = c0 + k * 32 + lane;
          pv[k] = cc < G ? ld_act(&a.ws.ss_part[(size_t)cc * a.maxB + t]) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) ss += pv[k];
      }
      ss = warp_sum(ss);
      if (lane == 0) {
        const float r = 1.0f / sqrtf(ss / (float)d + a.eps);
        rstd_s[t] = r;
        if (c == 0) a.ws.rstd[t] = r;
      }
    }
    csync();
    if (nrows > 0) mbar_wait(&fullW[0], 0, abort_flag, a.ws.err);
    for (int g = 0; g < npairs; ++g) {
      const int t0 = g * NT, nt = min(NT, B - t0), s = g % SH;
      float* pb = part + (size_t)(g & 1) * RM * kCW * NT;
      mbar_wait(&fullH[s], (g / SH) & 1, abort_flag, a.ws.err);
      float xr[NT][kCPLf][8];
      const float* hs = reinterpret_cast<const float*>(ring + s * SHB);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float r = (t < nt) ? rstd_s[t0 + t] : 0.f;
#pragma unroll
        for (int j = 0; j < kCPLf; ++j) {
          const int q = qbase + j * 32 + lane;
          if (t < nt && cvalid(qpw, j, lane)) {
            const float4 h0 = *reinterpret_cast<const float4*>(hs + (size_t)t * d + (size_t)q * 8);
            const float4 h1 = *reinterpret_cast<const float4*>(hs + (size_t)t * d + (size_t)q * 8 + 4);
            xr[t][j][0] = h0.x; xr[t][j][1] = h0.y; xr[t][j][2] = h0.z; xr[t][j][3] = h0.w;
            xr[t][j][4] = h1.x; xr[t][j][5] = h1.y; xr[t][j][6] = h1.z; xr[t][j][7] = h1.w;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) xr[t][j][e] = 0.f;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) xr[t][j][e] = xr[t][j][e] * r * gam[j][e];
          if (t < nt && cvalid(qpw, j, lane) && q % G == c) {  // each chunk of x is written by one CTA
            float* xp = a.ws.x + (size_t)(t0 + t) * d + (size_t)q * 8;
            *reinterpret_cast<float4*>(xp) = make_float4(xr[t][j][0], xr[t][j][1], xr[t][j][2], xr[t][j][3]);
            *reinterpret_cast<float4*>(xp + 4) = make_float4(xr[t][j][4], xr[t][j][5], xr[t][j][6], xr[t][j][7]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&emptyH[s]);  // h of this pair is in registers now
      constexpr int kRI = 4 / NT;
      for (int j0 = 0; j0 < nrows; j0 += kRI) {
        const uint16_t* rp[kRI];
#pragma unroll
        for (int k = 0; k < kRI; ++k) rp[k] = wsl + (size_t)min(j0 + k, nrows - 1) * d;
        float v[kRI * NT];
        rows_dot<NT, kRI>(rp, nrows - j0, xr, qbase, qpw, lane, v);
        const float tot = warp_reduce_multi<kRI * NT>(v, lane);
        const int vi = multi_index<kRI * NT>(lane), j = j0 + vi / NT, t = vi % NT;
        if (multi_writer<kRI * NT>(lane) && j < nrows) pb[(j * kCW + warp) * NT + t] = tot;
      }
      csync();  // this pair's partials are complete (the next pair writes the other buffer)
      for (int z = tid; z < nrows * nt; z += kCT) {
        const int j = z / nt, t = z % nt;
        float sacc = 0.f;
#pragma unroll
        for (int w = 0; w < kCW; ++w) sacc += pb[(j * kCW + w) * NT + t];
        a.ws.logits[(size_t)(t0 + t) * E + e0 + j] = sacc;
      }
    }
  }
  // the last CTA builds the routing tables; the ring (every fill landed and read) is its scratch
  if (last_cta_s(&a.ws.counters[kCntRouter], &s_misc[1])) {
    topk_route(a, ring);
    if (tid == 0) a.ws.counters[kCntRouter] = 0;
  }
}

// =============================================================================
// Grid barrier for the expert kernel (cooperative launch: every CTA is resident).
// Each CTA adds one to a counter with release semantics and waits (acquire loads) until it
// reaches the grid size.  The wait is bounded in time; on expiry the CTA records
// kErrTimeout and carries on (its results are then meaningless, and the error word says
// so).  Called by the consumer warps only.
// =============================================================================
namespace {

// `count` is zero when the kernel starts and only grows during a launch: the n-th barrier
// of a launch opens when it reaches n * gridDim.x (`target`), so the last arrival's add is
// the release (no second round trip).  Who clears it: for the expert kernel, the router
// kernel before its dependents pass their dependency wait; for the fused layer kernel, its
// own last CTA to finish (layer_exit).
__device__ void grid_barrier(unsigned* count, unsigned target, volatile int* abort_flag, uint32_t* err,
                             unsigned long long limit_ns = kWaitLimitNs) {
  // The CTA's writes happen before thread 0's release add: bar.sync orders them before it
  // and the release is cumulative, so no separate fence is needed.
  csync();
  if (threadIdx.x == 0) {
    red_release_add(count, 1u);
    if (ld_acquire_u32(count) < target) {
      const unsigned long long t0 = globaltimer();
      while (ld_acquire_u32(count) < target) {
        if (globaltimer() - t0 > limit_ns) {
          *abort_flag = 1;
          atomicOr(err, kErrTimeout);
          break;
        }
        __nanosleep(32);
      }
    }
  }
  csync();
}

}  // namespace

// Phase B of the batch <= 4 expert kernels (consumer warps): out = bf16(h + sum over the
// union experts of W_down[e] rows [i0, i0 + nrows) . a_s[e]), the W_down blocks arriving in
// the B ring.  A stage holds EPS experts' blocks of this CTA's rows; every load of a stage is
// issued before its FMAs (software-pipelining one expert ahead instead measured slower: fewer
// loads in flight).  Warp w owns rows w, w + 15, ...; lane l holds elements
// [l * epl, (l + 1) * epl) of each row and accumulates over all experts in registers: with
// 4 or 8 elements per lane as one packed fp32x2 accumulator per (row, token) (even elements in
// .x, odd in .y, experts in ascending union order), then .x + .y and one warp reduction.
template <int NT, int EPL>
__device__ __forceinline__ void combine_down(const LayerArgs& a, const unsigned char* ring, size_t SB_B, int SBn,
                                             uint64_t* fullB, uint64_t* emptyB, volatile int* abort_flag,
                                             const float* a_s, const int* ent_of, int U, int i0, int nrows, int warp,
                                             int lane) {
  constexpr int kRPW = 4;  // rows per warp (rows_max <= 60)
  constexpr int kEPS = experts_per_stage(EPL, NT);
  const int d = a.d, I = a.I, B = a.B;
  const int epl = (EPL > 0) ? EPL : I / 32;
  float acc[kRPW][NT];
  float2 acc2[kRPW][NT];
#pragma unroll
  for (int i = 0; i < kRPW; ++i)
#pragma unroll
    for (int t = 0; t < NT; ++t) { acc[i][t] = 0.f; acc2[i][t] = make_float2(0.f, 0.f); }
  // h of the (row, token) this lane writes at the end, loaded now so its latency is hidden
  const int vi_w = multi_index<kRPW * NT>(lane), i_w = vi_w / NT, t_w = vi_w % NT, rl_w = warp + kCW * i_w;
  const bool writer = multi_writer<kRPW * NT>(lane) && rl_w < nrows && t_w < B;
  const size_t o_w = (size_t)t_w * d + i0 + rl_w;
  const float h_w = writer ? ld_act(&a.ws.h[o_w]) : 0.f;
  int g = 0;
  for (int u0 = 0; u0 < U && nrows > 0; u0 += kEPS, ++g) {
    const int s = g % SBn, ne = min(kEPS, U - u0);
    mbar_wait(&fullB[s], (g / SBn) & 1, abort_flag, a.ws.err);
    const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + s * SB_B);
    if constexpr (EPL == 4 || EPL == 8) {
      using WT = typename std::conditional<EPL == 4, uint2, uint4>::type;
      float av[kEPS][NT][EPL];
      WT wv[kEPS][kRPW];
      // 32-bit shared-window addresses (the stage and a_s are both in shared memory)
      const uint32_t st_l = (uint32_t)__cvta_generic_to_shared(st) + (uint32_t)(lane * EPL * 2);
      const uint32_t as_l = (uint32_t)__cvta_generic_to_shared(a_s) + (uint32_t)(lane * EPL * 4);
#pragma unroll
      for (int e = 0; e < kEPS; ++e) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          // dense rows (u, t) up to two tokens; one row per entry, looked up, with four
          const int en = NT <= 2 ? ((e < ne) ? (u0 + e) * NT + t : -1) : ((e < ne) ? ent_of[(u0 + e) * NT + t] : -1);
          const uint32_t ap = as_l + (uint32_t)(max(en, 0) * I) * 4u;
#pragma unroll
          for (int x = 0; x < EPL; x += 4) {
            const float4 f = (en >= 0) ? lds128f(ap + (uint32_t)x * 4u) : make_float4(0.f, 0.f, 0.f, 0.f);
            av[e][t][x] = f.x; av[e][t][x + 1] = f.y; av[e][t][x + 2] = f.z; av[e][t][x + 3] = f.w;
          }
        }
#pragma unroll
        for (int i = 0; i < kRPW; ++i) {
          const int rl = warp + kCW * i;
          WT w{};
          if (e < ne && rl < nrows) {
            const uint32_t wa = st_l + (uint32_t)((e * nrows + rl) * I) * 2u;
            if constexpr (EPL == 4) w = lds64(wa);
            else w = lds128(wa);
          }
          wv[e][i] = w;
        }
      }
#pragma unroll
      for (int e = 0; e < kEPS; ++e)
#pragma unroll
        for (int i = 0; i < kRPW; ++i) {
          float wf[8];
          if constexpr (EPL == 4) {
            wf[0] = bf16lo(wv[e][i].x); wf[1] = bf16hi(wv[e][i].x);
            wf[2] = bf16lo(wv[e][i].y); wf[3] = bf16hi(wv[e][i].y);
          } else {
            unpack8f(reinterpret_cast<const uint4&>(wv[e][i]), wf);
          }
#pragma unroll
          for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int x = 0; x < EPL; x += 2) ffma2(acc2[i][t], wf[x], wf[x + 1], av[e][t][x], av[e][t][x + 1]);
        }
    } else {  // any other I: one expert per stage, epl <= 16 elements per lane
#pragma unroll
      for (int i = 0; i < kRPW; ++i) {
        const int rl = warp + kCW * i;
        if (rl < nrows) {
          const uint16_t* wr = st + (size_t)rl * I + lane * epl;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const int en = NT <= 2 ? u0 * NT + t : ent_of[u0 * NT + t];
            if (en < 0) continue;  // zero contribution, as a zero activation would give
            const float* ap = a_s + (size_t)en * I + lane * epl;
            float sdot = 0.f;
#pragma unroll
            for (int x = 0; x < 16; ++x)
              if (x < epl) sdot = fmaf(bf16f(wr[x]), ap[x], sdot);
            acc[i][t] += sdot;
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&emptyB[s]);
  }
  {
    float v[kRPW * NT];
#pragma unroll
    for (int i = 0; i < kRPW; ++i)
#pragma unroll
      for (int t = 0; t < NT; ++t) v[i * NT + t] = acc[i][t] + (acc2[i][t].x + acc2[i][t].y);
    const float tot = warp_reduce_multi<kRPW * NT>(v, lane);
    if (writer) {
      const __nv_bfloat16 bv = __float2bfloat16_rn(h_w + tot);
      a.out[o_w] = *reinterpret_cast<const uint16_t*>(&bv);
    }
  }
}

// =============================================================================
// K3 (batch <= 4): the expert kernel.  Routing once per CTA, then
//   phase A  gate/up + SiLU*mul: pairs (union expert u, row p) in flattened order, CTA c takes
//            [q0, q1); a stage is up to PS consecutive pairs of one expert (its gate rows and
//            its up rows, two copies).  a goes to global memory.
//   grid barrier (every a is needed by every CTA)
//   phase B  down + combine: CTA c owns output rows [i0, i1); a stage is those rows of one
//            union expert (one copy).  The producer streams phase B's weights into the freed
//            ring while the barrier is still open.  Warp w owns rows w, w + 8, ...; lane l
//            holds elements [l*EPL, (l+1)*EPL) of each row and accumulates over all experts
//            in registers; one warp reduction per (row, token) at the end.
// =============================================================================
template <int NT, int EPL, int CPD>
__global__ void __launch_bounds__(kThreadsS, 1) k_experts_f(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kEPS = experts_per_stage(EPL, NT);
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, I = a.I, B = a.B;
  const int SA = a.k3.stages, PS = a.k3.rows_per_stage, PM = a.k3.rows_max;
  const int SBn = a.k4.stages, RM = a.k4.rows_max;
  const uint32_t row_bytes = (uint32_t)d * 2u, drow_bytes = (uint32_t)I * 2u;
  const size_t SA_B = al128((size_t)2 * PS * row_bytes), SB_B = al128((size_t)kEPS * RM * drow_bytes);
  const size_t region = std::max((size_t)SA * SA_B, (size_t)SBn * SB_B);
  const size_t scratch_f = std::max((size_t)PM * 2 * kCW * NT, a_s_floats(B, a.k, a.E, I, NT));  // floats
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int i0 = (int)lo, nrows = (int)(hi - lo);

  unsigned char* ring = smem;
  float* part = reinterpret_cast<float*>(ring + region);  // phase A partials, then phase B's a
  float* a_s = part;
  using RO = RouteOf<NT>;
  auto* rt = reinterpret_cast<typename RO::Route*>(smem + al128(region + scratch_f * sizeof(float)));
  auto* sc = reinterpret_cast<typename RO::Scratch*>(rt + 1);
  float* fb = reinterpret_cast<float*>(sc + 1);
  uint64_t* fullA = reinterpret_cast<uint64_t*>(
      smem + al128(static_cast<size_t>(reinterpret_cast<unsigned char*>(fb + RO::kFbFloats) - smem)));
  uint64_t* emptyA = fullA + kMaxStages;
  uint64_t* fullB = emptyA + kMaxStages;
  uint64_t* emptyB = fullB + kMaxStages;
  int* s_misc = reinterpret_cast<int*>(emptyB + kMaxStages);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(fullA, emptyA, SA, kCW);
    init_ring(fullB, emptyB, SBn, kCW);
    s_misc[0] = 0;
    fence_barrier_init();
  }
  pdl_wait();  // logits and x come from the router kernel
  pdl_trigger();
  // one half of a 5-to-8-token step: runs only if the router's union says the halves take it
  if (a.split_B && !split_chosen(min(ld_act_i(a.ws.n_union), a.E), a.split_B, a.k)) return;

  // barriers inside also publish the ring init
  route_small_cta<NT>(a.ws.logits, B, a.E, a.k, a.user_idx, a.user_gate, a.ws.err, rt, sc, fb, c == 0);
  // x of every token, in registers (consumers).  Loaded after routing: the loads hit L2 and
  // land before the first weight stage, and holding x across the routing code would spill.
  const int qbase = (d / 8) * warp / kCW, qpw = (d / 8) * (warp + 1) / kCW - qbase;
  float xr[NT][CPD][8];
  if (warp < kCW) {
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < CPD; ++j) {
        if (t < B && cvalid(qpw, j, lane)) {
          const float* xp = a.ws.x + (size_t)t * d + (size_t)(qbase + j * 32 + lane) * 8;
          const float4 x0 = ld_act4(xp), x1 = ld_act4(xp + 4);
          xr[t][j][0] = x0.x; xr[t][j][1] = x0.y; xr[t][j][2] = x0.z; xr[t][j][3] = x0.w;
          xr[t][j][4] = x1.x; xr[t][j][5] = x1.y; xr[t][j][6] = x1.z; xr[t][j][7] = x1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) xr[t][j][e] = 0.f;
        }
      }
  }

  const int U = rt->U;
  long long q0l, q1l;
  split_range((long long)U * I, G, c, q0l, q1l);
  const int q0 = (int)q0l, q1 = (int)q1l;

  if (warp == kCW) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      // This CTA's W_down blocks go to L2 once the ring is primed, so phase B reads them
      // from L2 instead of waiting on HBM after the barrier.
      bool prefetched = false;
      auto prefetch_down = [&]() {
        for (int uu = 0; uu < U && nrows > 0; ++uu)
          bulk_prefetch_l2(a.w_down + ((size_t)rt->un_e[uu] * d + i0) * I, nrows * drow_bytes);
        prefetched = true;
      };
      // phase A: gate/up rows
      int it = 0;
      int u = q0 / I, p = q0 - u * I;
      for (int q = q0; q < q1; ++it) {
        if (it == SA && !prefetched) prefetch_down();
        const int np = min(min(PS, I - p), q1 - q);
        if (!ring_acquire(emptyA, it, SA, abort_flag, a.ws.err)) break;
        const int s = it % SA;
        const uint16_t* base = a.w_gu + ((size_t)rt->un_e[u] * 2 * I + p) * d;
        mbar_arrive_expect_tx(&fullA[s], 2u * np * row_bytes);
        bulk_g2s(ring + s * SA_B, base, np * row_bytes, &fullA[s], pol);
        bulk_g2s(ring + s * SA_B + (size_t)PS * row_bytes, base + (size_t)I * d, np * row_bytes, &fullA[s], pol);
        q += np;
        p += np;
        if (p == I) { p = 0; ++u; }
      }
      if (!prefetched) prefetch_down();
      // The ring is reused by phase B only after every phase-A fill has landed and been read.
      ring_drain(fullA, it, SA, a.ws.err);
      for (int i = it - SA < 0 ? 0 : it - SA; i < it; ++i) mbar_drain(&emptyA[i % SA], (i / SA) & 1, a.ws.err);
      // phase B: this CTA's rows of W_down for every union expert
      if (nrows > 0) {
        const uint32_t blk = (uint32_t)nrows * drow_bytes;  // one expert's rows for this CTA
        int jt = 0;
        for (int u0 = 0; u0 < U; u0 += kEPS, ++jt) {
          const int ne = min(kEPS, U - u0);
          if (!ring_acquire(emptyB, jt, SBn, abort_flag, a.ws.err)) break;
          const int s = jt % SBn;
          mbar_arrive_expect_tx(&fullB[s], ne * blk);
          for (int e = 0; e < ne; ++e)
            bulk_g2s(ring + s * SB_B + (size_t)e * blk, a.w_down + ((size_t)rt->un_e[u0 + e] * d + i0) * I, blk,
                     &fullB[s], pol);
        }
        ring_drain(fullB, jt, SBn, a.ws.err);
      }
    }
    return;
  }

  // ---- phase A (consumers) ------------------------------------------------------------
  // rows per interleaved pass: four values per lane to reduce (two rows of two tokens, four
  // rows of one), or eight with four tokens where their two-chunk slices leave the registers
  // (two rows per pass instead of one: batch 3 / 4 -4.3 / -6.6 us)
  constexpr int kRI = (NT > 2 && CPD == 2) ? 2 : 4 / NT;
  {
    int it = 0;
    int p = q0 - (q0 / I) * I;
    for (int q = q0; q < q1; ++it) {
      const int np = min(min(PS, I - p), q1 - q), s = it % SA;
      mbar_wait(&fullA[s], (it / SA) & 1, abort_flag, a.ws.err);
      const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + s * SA_B);
      const int nrow = 2 * np;  // gate rows 0..np-1, then up rows
      for (int i0 = 0; i0 < nrow; i0 += kRI) {
        const uint16_t* rp[kRI];
#pragma unroll
        for (int k = 0; k < kRI; ++k) {
          const int i = min(i0 + k, nrow - 1), pi = (i < np) ? i : i - np, gu = (i < np) ? 0 : 1;
          rp[k] = st + (size_t)(gu * PS + pi) * d;
        }
        float v[kRI * NT];
        rows_dot<NT, kRI>(rp, nrow - i0, xr, qbase, qpw, lane, v);
        const float tot = warp_reduce_multi<kRI * NT>(v, lane);
        const int vi = multi_index<kRI * NT>(lane), i = i0 + vi / NT, t = vi % NT;
        if (multi_writer<kRI * NT>(lane) && i < nrow) {
          const int pi = (i < np) ? i : i - np, gu = (i < np) ? 0 : 1;
          part[(((q - q0 + pi) * 2 + gu) * kCW + warp) * NT + t] = tot;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&emptyA[s]);
      q += np;
      p += np;
      if (p == I) p = 0;
    }
    csync();
    for (int z = tid; z < (q1 - q0) * B; z += kCT) {
      const int pl = z / B, t = z % B;
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int w = 0; w < kCW; ++w) {
        gs += part[((pl * 2 + 0) * kCW + w) * NT + t];
        us += part[((pl * 2 + 1) * kCW + w) * NT + t];
      }
      const int qq = q0 + pl, u = qq / I, pp = qq - u * I;
      for (int en = rt->un_off[u]; en < rt->un_off[u + 1]; ++en)
        if (rt->ent_tok[en] == t) a.ws.a[(size_t)en * I + pp] = gs / (1.0f + expf(-gs)) * us;
    }
  }

  grid_barrier(&a.ws.counters[kCntGateUp], (unsigned)(a.bar_base + 1) * gridDim.x, abort_flag, a.ws.err);

  // ---- phase B (consumers) ------------------------------------------------------------
  // Up to two tokens a_s[u][t][:] = gate * a of (union expert u, token t), zero where t did
  // not select u; with four, a_s[en][:] = gate * a of entry en and ent_of[u][t] = the entry of
  // (u, t), -1 where t did not select u (phase B then adds nothing for that pair, as a zero
  // activation would).
  int* ent_of = reinterpret_cast<int*>(a_s + (size_t)B * a.k * I);  // four tokens only
  if constexpr (NT <= 2) {
    for (int z = tid; z < U * NT * (I / 4); z += kCT) {
      const int cq = z % (I / 4), ut = z / (I / 4), t = ut % NT, u = ut / NT;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int en = rt->un_off[u]; en < rt->un_off[u + 1]; ++en)
        if (rt->ent_tok[en] == t) {
          const float g = rt->ent_gate[en];
          const float4 x4 = ld_act4(a.ws.a + (size_t)en * I + cq * 4);
          v = make_float4(g * x4.x, g * x4.y, g * x4.z, g * x4.w);
        }
      *reinterpret_cast<float4*>(a_s + ((size_t)u * NT + t) * I + cq * 4) = v;
    }
  } else {
    for (int z = tid; z < rt->n_ent * (I / 4); z += kCT) {
      const int cq = z % (I / 4), en = z / (I / 4);
      const float g = rt->ent_gate[en];
      const float4 x4 = ld_act4(a.ws.a + (size_t)en * I + cq * 4);
      *reinterpret_cast<float4*>(a_s + (size_t)en * I + cq * 4) = make_float4(g * x4.x, g * x4.y, g * x4.z, g * x4.w);
    }
    for (int z = tid; z < U * NT; z += kCT) {
      const int u = z / NT, t = z - u * NT;
      int f = -1;
      for (int en = rt->un_off[u]; en < rt->un_off[u + 1]; ++en)
        if (rt->ent_tok[en] == t) f = en;
      ent_of[z] = f;
    }
  }
  csync();

  combine_down<NT, EPL>(a, ring, SB_B, SBn, fullB, emptyB, abort_flag, a_s, ent_of, U, i0, nrows, warp, lane);
}

// =============================================================================
// The fused layer kernel (batch <= 2): the three kernels above as one cooperative launch,
// with grid barriers where a kernel boundary was:
//   o_proj     h = residual + W_o . attn_out, per-CTA sums of h^2 (as k_oproj_f).  The
//              producer streams this CTA's router rows into the same ring right after its
//              W_o rows, so W_r leaves HBM while the o_proj tail computes.
//   barrier 1  (every h and sum of h^2 written)
//   router     rstd from the 148 partial sums (same order in every CTA), x in registers,
//              logits of this CTA's rows from the ring (as k_router_f)
//   barrier 2  (every logit and x written)
//   routing    recomputed in every CTA, then phase A, barrier 3 and phase B as in k_experts_f.
// Every CTA adds one to the exit ticket after its last barrier; the last one clears the
// barrier count for the next launch.
// =============================================================================
namespace {

// Scratch floats shared by the o_proj, router and phase A partial sums (each phase's use
// ends before the next begins).  Phase B's gated activations live in the ring region, after
// phase B's stages.
__host__ __device__ constexpr size_t oproj_part_floats(int NT, int UC, int RS) {
  return (((size_t)UC * RS * kCW * NT) + 3) & ~size_t(3);  // 16-byte multiple: the residual follows
}
__host__ __device__ constexpr size_t layer_scratch_floats(int NT, int UC, int RS, int RMr, int PM, int d) {
  const size_t o = oproj_part_floats(NT, UC, RS) + (size_t)NT * d / 2 + UC;  // o_proj partials, residual, units
  const size_t r = (size_t)RMr * kCW * NT + 64;                // router partials + rstd
  const size_t pa = (size_t)PM * 2 * kCW * NT;                 // phase A partials
  const size_t m1 = o > r ? o : r;
  return m1 > pa ? m1 : pa;
}

// Most o_proj units (RS rows each) one CTA of G takes: twice an even share, plus one.
__host__ __device__ constexpr int oproj_unit_cap(int d, int RS, int G) {
  return 2 * (((d + RS - 1) / RS + G - 1) / G) + 1;
}

// Called by thread 0 after its CTA's last grid barrier.
__device__ __forceinline__ void layer_exit(unsigned* counters) {
  const unsigned G = gridDim.x;
  if (atomicAdd(&counters[kCntLayerExit], 1u) == G - 1) {  // every CTA is past its last barrier
    counters[kCntLayer] = 0;
    counters[kCntLayerExit] = 0;
    __threadfence();
  }
}

}  // namespace

template <int NT, int EPL, int CPD>
__global__ void __launch_bounds__(kThreadsS, 1) k_layer_f(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kEPS = experts_per_stage(EPL, NT);
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, d_o = a.d_o, I = a.I, B = a.B, E = a.E;
  const int SO = a.k1.stages, RS = a.k1.rows_per_stage, RM = a.k1.rows_max;
  const int RSr = a.k2.rows_per_stage, RMr = a.k2.rows_max;
  const int SA = a.k3.stages, PS = a.k3.rows_per_stage, PM = a.k3.rows_max;
  const int SBn = a.k4.stages;
  const uint32_t orow_bytes = (uint32_t)d_o * 2u, row_bytes = (uint32_t)d * 2u, drow_bytes = (uint32_t)I * 2u;
  const size_t SO_B = std::max(al128((size_t)RS * orow_bytes), al128(row_bytes));  // a W_r row fits a stage
  const size_t SA_B = al128((size_t)2 * PS * row_bytes), SB_B = al128((size_t)kEPS * RM * drow_bytes);
  const size_t a_s_bytes = a_s_floats(B, a.k, E, I, NT) * 4;
  const size_t region =
      std::max(std::max((size_t)SO * SO_B, (size_t)SA * SA_B), (size_t)SBn * SB_B + a_s_bytes);
  const int UC = oproj_unit_cap(d, RS, G);
  const size_t scratch_f = layer_scratch_floats(NT, UC, RS, RMr, PM, d);
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int i0 = (int)lo, nrows = (int)(hi - lo);  // o_proj rows = phase B output rows
  split_range(E, G, c, lo, hi);
  const int e0 = (int)lo, nr = (int)(hi - lo);      // router rows

  unsigned char* ring = smem;
  float* part = reinterpret_cast<float*>(ring + region);
  float* rstd_s = part + RMr * kCW * NT;  // router
  // phase B: after phase B's stages (phase A's fills have all landed and been read by then)
  float* a_s = reinterpret_cast<float*>(ring + (size_t)SBn * SB_B);
  using RO = RouteOf<NT>;
  auto* rt = reinterpret_cast<typename RO::Route*>(smem + al128(region + scratch_f * sizeof(float)));
  auto* sc = reinterpret_cast<typename RO::Scratch*>(rt + 1);
  float* fb = reinterpret_cast<float*>(sc + 1);
  uint64_t* fullO = reinterpret_cast<uint64_t*>(
      smem + al128(static_cast<size_t>(reinterpret_cast<unsigned char*>(fb + RO::kFbFloats) - smem)));
  uint64_t* emptyO = fullO + kMaxStages;
  uint64_t* fullA = emptyO + kMaxStages;
  uint64_t* emptyA = fullA + kMaxStages;
  uint64_t* fullB = emptyA + kMaxStages;
  uint64_t* emptyB = fullB + kMaxStages;
  uint64_t* resbar = emptyB + kMaxStages;  // the residual's copy into shared memory
  int* s_misc = reinterpret_cast<int*>(resbar + 1);
  volatile int* abort_flag = s_misc;
  unsigned* bar_count = &a.ws.counters[kCntLayer];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(fullO, emptyO, SO, kCW);
    init_ring(fullA, emptyA, SA, kCW);
    init_ring(fullB, emptyB, SBn, kCW);
    mbar_init(resbar, 1);
    s_misc[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  const int qbase_o = (d_o / 8) * warp / kCW, qpw_o = (d_o / 8) * (warp + 1) / kCW - qbase_o;
  const int qbase = (d / 8) * warp / kCW, qpw = (d / 8) * (warp + 1) / kCW - qbase;
  // o_proj work units: unit u = W_o rows [u RS, u RS + RS), one ring stage.  Three quarters
  // of the units are split evenly and contiguously over the CTAs (S0 each); the rest are
  // taken one at a time from a global counter, so a CTA whose copies stream faster takes more
  // and the CTAs finish together.  A CTA takes at most UC units (its partial-sum buffers).
  const int n_units = (d + RS - 1) / RS, S0 = (3 * n_units) / (4 * G);
  float* opart = part;                                                         // [UC RS][kCW][NT]
  uint16_t* res_s = reinterpret_cast<uint16_t*>(part + oproj_part_floats(NT, UC, RS));  // [B][d]
  int* ouid = reinterpret_cast<int*>(part + oproj_part_floats(NT, UC, RS) + (size_t)NT * d / 2);  // [UC]
  int* s_unit = s_misc + 8;  // [SO]: unit of each filled stage, -1 = no more units
  int itO = 0;  // O-ring fills (producer) / waits (consumers)
  if (warp == kCW) {
    if (lane == 0) {  // weights are static: the first W_o fills go out before the dependency resolves
      const uint64_t pol = policy_evict_first();
      bulk_prefetch_l2(a.gamma, row_bytes);  // every CTA reads all of gamma after barrier 1
      int held = 0;  // units this CTA has been given (static fills and counter tickets)
      auto fill_unit = [&](int u) -> bool {
        if (!ring_acquire(emptyO, itO, SO, abort_flag, a.ws.err)) return false;
        const int s = itO % SO, r = u * RS, n = min(RS, d - r);
        s_unit[s] = u;
        mbar_arrive_expect_tx(&fullO[s], n * orow_bytes);
        bulk_g2s(ring + s * SO_B, a.w_o + (size_t)r * d_o, n * orow_bytes, &fullO[s], pol);
        ++itO;
        return true;
      };
      bool ok = true;
      int nst = 0;  // static units filled
      for (; nst < S0 && nst < SO && ok; ++nst) ok = fill_unit(c * S0 + nst);
      held = S0;
      // The counter was cleared by the previous launch after its barrier 1; griddepcontrol.wait
      // makes that store visible.  The residual may come from the previous kernel too.
      pdl_wait();
      mbar_arrive_expect_tx(resbar, (uint32_t)B * row_bytes);
      bulk_g2s(res_s, a.resid, (uint32_t)B * row_bytes, resbar, pol);
      unsigned* unit_ctr = &a.ws.counters[kCntOUnit];
      const int base = S0 * G;
      // Two tickets in flight, each in a register of its own (a register array indexed at run
      // time would sit in local memory, and storing a ticket there waits for its atomic).
      int tA = 0, tB = 0;
      bool hA = false, hB = false, more = base < n_units;
      if (more && held < UC) { tA = (int)atomicAdd(unit_ctr, 1u); hA = true; ++held; }
      if (more && held < UC) { tB = (int)atomicAdd(unit_ctr, 1u); hB = true; ++held; }
      for (; nst < S0 && ok; ++nst) ok = fill_unit(c * S0 + nst);  // the tickets' round trips overlap these
      auto use = [&](int& t, bool& h) {  // fill ticket t's unit and take the next ticket in its place
        if (!h) return;
        h = false;
        const int u = base + t;
        if (u < n_units && ok) {
          if (more && held < UC) { t = (int)atomicAdd(unit_ctr, 1u); h = true; ++held; }
          ok = fill_unit(u);
        } else {
          more = false;  // the other ticket is still read
        }
      };
      while (hA || hB) {
        use(tA, hA);
        use(tB, hB);
      }
      if (ok && ring_acquire(emptyO, itO, SO, abort_flag, a.ws.err)) {  // end of the units
        const int s = itO % SO;
        s_unit[s] = -1;
        mbar_arrive(&fullO[s]);
        ++itO;
      }
      for (int j = 0; j < nr && !*abort_flag; j += RSr, ++itO) {
        const int n = min(RSr, nr - j);
        if (!ring_acquire(emptyO, itO, SO, abort_flag, a.ws.err)) break;
        const int s = itO % SO;
        mbar_arrive_expect_tx(&fullO[s], n * row_bytes);
        bulk_g2s(ring + s * SO_B, a.w_r + (size_t)(e0 + j) * d, n * row_bytes, &fullO[s], pol);
      }
      if (a.pf_w_o) {  // next layer: what the same CTA reads first, into L2
        if (nr > 0) bulk_prefetch_l2(a.pf_w_r + (size_t)e0 * d, nr * row_bytes);
        if (c == 0) bulk_prefetch_l2(a.pf_gamma, row_bytes);
        for (int j = 0; j < S0 && (size_t)j * RS < (size_t)a.pf_w_o_rows; ++j) {
          const int u = c * S0 + j;
          bulk_prefetch_l2(a.pf_w_o + (size_t)u * RS * d_o, (uint32_t)min(RS, d - u * RS) * orow_bytes);
        }
      }
      // The O ring's last fills land and are read (the router rows, after barrier 1) while
      // the consumers work towards barrier 2; phase A may then reuse the region at once.
      ring_drain(fullO, itO, SO, a.ws.err);
      for (int i = itO - SO < 0 ? 0 : itO - SO; i < itO; ++i) mbar_drain(&emptyO[i % SO], (i / SO) & 1, a.ws.err);
      mbar_drain(resbar, 0, a.ws.err);
    }
  } else {
    // ---- o_proj (consumers) ----------------------------------------------------------
    pdl_wait();  // attn_out may come from the previous kernel
    int nslot = 0;
    {
      constexpr int kRI = 2;
      // K split of d_o as in k_oproj_f: evenly in at most two chunk rounds up to d_o = 7680,
      // else two full rounds per warp and a third in the first warps only
      const int nch = d_o / 8;
      const bool split2x = nch > 64 * kCW;
      const int qb = split2x ? 64 * warp : qbase_o, qp = split2x ? 64 : qpw_o;
      const int qx = 64 * kCW + 32 * warp;
      const bool has_x = split2x && qx < nch;
      uint4 xa[NT][kCPLf];  // attn_out stays packed bf16 (mixed-precision FMAs)
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int j = 0; j < kCPLf; ++j) {
          uint4 u = make_uint4(0, 0, 0, 0);
          const int q = (j < 2 || !split2x) ? qb + j * 32 + lane : qx + lane;
          const bool ok = (j < 2 || !split2x) ? cvalid(qp, j, lane) : (has_x && q < nch);
          if (t < B && ok) u = ld_act_u4(a.attn + (size_t)t * d_o + (size_t)q * 8);
          xa[t][j] = u;
        }
      while (true) {
        const int s = itO % SO;
        if (!mbar_wait(&fullO[s], (itO / SO) & 1, abort_flag, a.ws.err)) break;
        const int u = s_unit[s];
        if (u < 0 || nslot >= UC) {  // end of the units (the bound only guards the buffers)
          __syncwarp();
          if (lane == 0) mbar_arrive(&emptyO[s]);
          ++itO;
          break;
        }
        const int n = min(RS, d - u * RS);
        if (warp == 0 && lane == 0) ouid[nslot] = u;
        const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + s * SO_B);
        for (int j0 = 0; j0 < n; j0 += kRI) {
          const uint16_t* rp[kRI];
#pragma unroll
          for (int k = 0; k < kRI; ++k) rp[k] = st + (size_t)min(j0 + k, n - 1) * d_o;
          float v[kRI * NT];
          if (split2x) rows_dot_bf_2x<NT, kRI>(rp, n - j0, xa, qb, qx, nch, has_x, lane, v);
          else rows_dot_bf<NT, kRI>(rp, n - j0, xa, qbase_o, qpw_o, lane, v);
          const float tot = warp_reduce_multi<kRI * NT>(v, lane);
          const int vi = multi_index<kRI * NT>(lane), j = j0 + vi / NT, t = vi % NT;
          if (multi_writer<kRI * NT>(lane) && j < n) opart[(((size_t)nslot * RS + j) * kCW + warp) * NT + t] = tot;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&emptyO[s]);
        ++itO;
        ++nslot;
      }
    }
    csync();
    mbar_wait(resbar, 0, abort_flag, a.ws.err);
    for (int z = tid; z < nslot * RS * B; z += kCT) {  // h = residual + sum of the warps' partials
      const int sl = z / (RS * B), rem = z - sl * RS * B, j = rem / B, t = rem - j * B;
      const int row = ouid[sl] * RS + j;
      if (row < d) {
        float sacc = 0.f;
#pragma unroll
        for (int w = 0; w < kCW; ++w) sacc += opart[(((size_t)sl * RS + j) * kCW + w) * NT + t];
        a.ws.h[(size_t)t * d + row] = bf16f(res_s[(size_t)t * d + row]) + sacc;
      }
    }
    grid_barrier(bar_count, (unsigned)G, abort_flag, a.ws.err);
    if (c == 0 && tid == 0) a.ws.counters[kCntOUnit] = 0;  // every CTA has taken its last unit

    // ---- router (consumers) ----------------------------------------------------------
    {
      // h and gamma in one round of loads; the sum of h^2 over d from the same registers
      // (per lane, per warp, then the 15 warps in a fixed order: the same bits in every CTA)
      float xr[NT][CPD][8];
      float gam[CPD][8];
#pragma unroll
      for (int j = 0; j < CPD; ++j) {
        uint4 u = make_uint4(0, 0, 0, 0);
        if (cvalid(qpw, j, lane)) u = ld_weight_u4(a.gamma + (size_t)(qbase + j * 32 + lane) * 8);
        unpack8f(u, gam[j]);
      }
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int j = 0; j < CPD; ++j) {
          if (t < B && cvalid(qpw, j, lane)) {
            const float* hp = a.ws.h + (size_t)t * d + (size_t)(qbase + j * 32 + lane) * 8;
            const float4 h0 = ld_act4(hp), h1 = ld_act4(hp + 4);
            xr[t][j][0] = h0.x; xr[t][j][1] = h0.y; xr[t][j][2] = h0.z; xr[t][j][3] = h0.w;
            xr[t][j][4] = h1.x; xr[t][j][5] = h1.y; xr[t][j][6] = h1.z; xr[t][j][7] = h1.w;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) xr[t][j][e] = 0.f;
          }
        }
      float* wss = rstd_s + 2;  // [kCW][NT]
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float s2 = 0.f;
#pragma unroll
        for (int j = 0; j < CPD; ++j)
#pragma unroll
          for (int e = 0; e < 8; ++e) s2 = fmaf(xr[t][j][e], xr[t][j][e], s2);
        s2 = warp_sum(s2);
        if (lane == 0) wss[warp * NT + t] = s2;
      }
      csync();
      float rv[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float ss = 0.f;
        for (int w = 0; w < kCW; ++w) ss += wss[w * NT + t];
        rv[t] = (t < B) ? 1.0f / sqrtf(ss / (float)d + a.eps) : 0.f;
        if (c == 0 && tid == 0 && t < B) a.ws.rstd[t] = rv[t];
      }
#pragma unroll
      for (int j = 0; j < CPD; ++j) {
        const int q = qbase + j * 32 + lane;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
#pragma unroll
          for (int e = 0; e < 8; ++e) xr[t][j][e] = xr[t][j][e] * rv[t] * gam[j][e];
          if (t < B && cvalid(qpw, j, lane) && q % G == c) {  // each chunk of x is written by one CTA
            float* xp = a.ws.x + (size_t)t * d + (size_t)q * 8;
            *reinterpret_cast<float4*>(xp) = make_float4(xr[t][j][0], xr[t][j][1], xr[t][j][2], xr[t][j][3]);
            *reinterpret_cast<float4*>(xp + 4) = make_float4(xr[t][j][4], xr[t][j][5], xr[t][j][6], xr[t][j][7]);
          }
        }
      }
      // every W_r fill first (they landed during the o_proj tail), then passes of 4 / NT
      // rows across stage boundaries
      const int itR = itO, nfr = (nr + RSr - 1) / RSr;
      for (int f = 0; f < nfr; ++f)
        mbar_wait(&fullO[(itR + f) % SO], ((itR + f) / SO) & 1, abort_flag, a.ws.err);
      constexpr int kRI = 4 / NT;
      for (int j0 = 0; j0 < nr; j0 += kRI) {
        const uint16_t* rp[kRI];
#pragma unroll
        for (int k = 0; k < kRI; ++k) {
          const int j = min(j0 + k, nr - 1), f = j / RSr;
          rp[k] = reinterpret_cast<const uint16_t*>(ring + ((itR + f) % SO) * SO_B) + (size_t)(j - f * RSr) * d;
        }
        float v[kRI * NT];
        rows_dot<NT, kRI>(rp, nr - j0, xr, qbase, qpw, lane, v);
        const float tot = warp_reduce_multi<kRI * NT>(v, lane);
        const int vi = multi_index<kRI * NT>(lane), j = j0 + vi / NT, t = vi % NT;
        if (multi_writer<kRI * NT>(lane) && j < nr) part[(j * kCW + warp) * NT + t] = tot;
      }
      __syncwarp();
      if (lane == 0)
        for (int f = 0; f < nfr; ++f) mbar_arrive(&emptyO[(itR + f) % SO]);
      itO += nfr;
      csync();
      for (int z = tid; z < nr * B; z += kCT) {
        const int j = z / B, t = z % B;
        float sacc = 0.f;
#pragma unroll
        for (int w = 0; w < kCW; ++w) sacc += part[(j * kCW + w) * NT + t];
        a.ws.logits[(size_t)t * E + e0 + j] = sacc;
      }
    }
    grid_barrier(bar_count, 2u * (unsigned)G, abort_flag, a.ws.err);
  }
  __syncthreads();  // the producer warp joins: logits are complete

  route_small_cta<NT>(a.ws.logits, B, E, a.k, a.user_idx, a.user_gate, a.ws.err, rt, sc, fb, c == 0);
  float xr[NT][CPD][8];
  if (warp < kCW) {
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < CPD; ++j) {
        if (t < B && cvalid(qpw, j, lane)) {
          const float* xp = a.ws.x + (size_t)t * d + (size_t)(qbase + j * 32 + lane) * 8;
          const float4 x0 = ld_act4(xp), x1 = ld_act4(xp + 4);
          xr[t][j][0] = x0.x; xr[t][j][1] = x0.y; xr[t][j][2] = x0.z; xr[t][j][3] = x0.w;
          xr[t][j][4] = x1.x; xr[t][j][5] = x1.y; xr[t][j][6] = x1.z; xr[t][j][7] = x1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) xr[t][j][e] = 0.f;
        }
      }
  }

  const int U = rt->U;
  long long q0l, q1l;
  split_range((long long)U * I, G, c, q0l, q1l);
  const int q0 = (int)q0l, q1 = (int)q1l;

  if (warp == kCW) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      // This CTA's W_down blocks go to L2 while phase A streams, so phase B reads them from
      // L2: one expert's block per refill once the ring is primed (the prefetches queue in
      // the same copy engine as the stages, so they are spread out rather than issued at once).
      int npf = 0;
      auto prefetch_down = [&](int upto) {
        for (; npf < upto && npf < U && nrows > 0; ++npf)
          bulk_prefetch_l2(a.w_down + ((size_t)rt->un_e[npf] * d + i0) * I, nrows * drow_bytes);
      };
      int it = 0;
      int u = q0 / I, p = q0 - u * I;
      for (int q = q0; q < q1; ++it) {
        if (it >= SA) prefetch_down(it - SA + 1);
        const int np = min(min(PS, I - p), q1 - q);
        if (!ring_acquire(emptyA, it, SA, abort_flag, a.ws.err)) break;
        const int s = it % SA;
        const uint16_t* base = a.w_gu + ((size_t)rt->un_e[u] * 2 * I + p) * d;
        mbar_arrive_expect_tx(&fullA[s], 2u * np * row_bytes);
        bulk_g2s(ring + s * SA_B, base, np * row_bytes, &fullA[s], pol);
        bulk_g2s(ring + s * SA_B + (size_t)PS * row_bytes, base + (size_t)I * d, np * row_bytes, &fullA[s], pol);
        q += np;
        p += np;
        if (p == I) { p = 0; ++u; }
      }
      prefetch_down(U);
      ring_drain(fullA, it, SA, a.ws.err);
      for (int i = it - SA < 0 ? 0 : it - SA; i < it; ++i) mbar_drain(&emptyA[i % SA], (i / SA) & 1, a.ws.err);
      if (nrows > 0) {
        const uint32_t blk = (uint32_t)nrows * drow_bytes;
        int jt = 0;
        for (int u0 = 0; u0 < U; u0 += kEPS, ++jt) {
          const int ne = min(kEPS, U - u0);
          if (!ring_acquire(emptyB, jt, SBn, abort_flag, a.ws.err)) break;
          const int s = jt % SBn;
          mbar_arrive_expect_tx(&fullB[s], ne * blk);
          for (int e = 0; e < ne; ++e)
            bulk_g2s(ring + s * SB_B + (size_t)e * blk, a.w_down + ((size_t)rt->un_e[u0 + e] * d + i0) * I, blk,
                     &fullB[s], pol);
        }
        ring_drain(fullB, jt, SBn, a.ws.err);
      }
    }
    return;
  }

  // ---- phase A (consumers) ------------------------------------------------------------
  {
    constexpr int kRI = 4 / NT;
    int it = 0;
    int p = q0 - (q0 / I) * I;
    for (int q = q0; q < q1; ++it) {
      const int np = min(min(PS, I - p), q1 - q), s = it % SA;
      mbar_wait(&fullA[s], (it / SA) & 1, abort_flag, a.ws.err);
      const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + s * SA_B);
      const int nrow = 2 * np;
      for (int r0 = 0; r0 < nrow; r0 += kRI) {
        const uint16_t* rp[kRI];
#pragma unroll
        for (int k = 0; k < kRI; ++k) {
          const int i = min(r0 + k, nrow - 1), pi = (i < np) ? i : i - np, gu = (i < np) ? 0 : 1;
          rp[k] = st + (size_t)(gu * PS + pi) * d;
        }
        float v[kRI * NT];
        rows_dot<NT, kRI>(rp, nrow - r0, xr, qbase, qpw, lane, v);
        const float tot = warp_reduce_multi<kRI * NT>(v, lane);
        const int vi = multi_index<kRI * NT>(lane), i = r0 + vi / NT, t = vi % NT;
        if (multi_writer<kRI * NT>(lane) && i < nrow) {
          const int pi = (i < np) ? i : i - np, gu = (i < np) ? 0 : 1;
          part[(((q - q0 + pi) * 2 + gu) * kCW + warp) * NT + t] = tot;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&emptyA[s]);
      q += np;
      p += np;
      if (p == I) p = 0;
    }
    csync();
    for (int z = tid; z < (q1 - q0) * B; z += kCT) {
      const int pl = z / B, t = z % B;
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int w = 0; w < kCW; ++w) {
        gs += part[((pl * 2 + 0) * kCW + w) * NT + t];
        us += part[((pl * 2 + 1) * kCW + w) * NT + t];
      }
      const int qq = q0 + pl, u = qq / I, pp = qq - u * I;
      for (int en = rt->un_off[u]; en < rt->un_off[u + 1]; ++en)
        if (rt->ent_tok[en] == t) a.ws.a[(size_t)en * I + pp] = gs / (1.0f + expf(-gs)) * us;
    }
  }

  grid_barrier(bar_count, 3u * (unsigned)G, abort_flag, a.ws.err);
  if (tid == 0) layer_exit(a.ws.counters);

  // ---- phase B (consumers) ------------------------------------------------------------
  int* ent_of = reinterpret_cast<int*>(a_s + (size_t)B * a.k * I);  // four tokens only
  if constexpr (NT <= 2) {
    for (int z = tid; z < U * NT * (I / 4); z += kCT) {
      const int cq = z % (I / 4), ut = z / (I / 4), t = ut % NT, u = ut / NT;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int en = rt->un_off[u]; en < rt->un_off[u + 1]; ++en)
        if (rt->ent_tok[en] == t) {
          const float g = rt->ent_gate[en];
          const float4 x4 = ld_act4(a.ws.a + (size_t)en * I + cq * 4);
          v = make_float4(g * x4.x, g * x4.y, g * x4.z, g * x4.w);
        }
      *reinterpret_cast<float4*>(a_s + ((size_t)u * NT + t) * I + cq * 4) = v;
    }
  } else {
    for (int z = tid; z < rt->n_ent * (I / 4); z += kCT) {
      const int cq = z % (I / 4), en = z / (I / 4);
      const float g = rt->ent_gate[en];
      const float4 x4 = ld_act4(a.ws.a + (size_t)en * I + cq * 4);
      *reinterpret_cast<float4*>(a_s + (size_t)en * I + cq * 4) = make_float4(g * x4.x, g * x4.y, g * x4.z, g * x4.w);
    }
    for (int z = tid; z < U * NT; z += kCT) {
      const int u = z / NT, t = z - u * NT;
      int f = -1;
      for (int en = rt->un_off[u]; en < rt->un_off[u + 1]; ++en)
        if (rt->ent_tok[en] == t) f = en;
      ent_of[z] = f;
    }
  }
  csync();
  combine_down<NT, EPL>(a, ring, SB_B, SBn, fullB, emptyB, abort_flag, a_s, ent_of, U, i0, nrows, warp, lane);
}

// =============================================================================
// Error-path probe (moe_decode_check_error_path): makes the device error reporting of the
// kernels above run without a fault.
//   what 1: thread 0 waits on an mbarrier that nothing arrives on (mbar_wait), then every
//           CTA waits at a grid barrier whose target is one arrival more than the grid
//           (grid_barrier); both waits run out after limit_ns and record kErrTimeout.  Each
//           CTA then takes its own arrival back, so the counter ends at zero.
//   what 2: an expert index one past the end is met and clamped, recording kErrBounds, the
//           way the routing and the expert kernels treat an out-of-range table entry.
// Nothing is copied asynchronously, so no copy can still be in flight when a CTA exits.
// =============================================================================
__global__ void __launch_bounds__(kThreadsS, 1) k_error_probe(unsigned* count, uint32_t* err, int what,
                                                              unsigned long long limit_ns, int E, int* sink) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (what == 1) {
    if (threadIdx.x == 0) {
      mbar_wait(&bar, 0, &abort_s, err, limit_ns);
      abort_s = 0;  // the grid barrier below must still run out on its own
    }
    __syncthreads();
    if (warp < kCW) grid_barrier(count, gridDim.x + 1u, &abort_s, err, limit_ns);
    if (threadIdx.x == 0) atomicSub(count, 1u);
  } else if (what == 2 && threadIdx.x == 0 && blockIdx.x == 0) {
    const int want = E;  // one past the last expert
    const int e = (want >= 0 && want < E) ? want : 0;
    if (e != want) atomicOr(err, kErrBounds);
    *sink = e;
  }
}

cudaError_t launch_error_probe(unsigned* count, unsigned* err, int what, unsigned long long limit_ns, int E,
                               int* sink, cudaStream_t s) {
  k_error_probe<<<2, kThreadsS, 0, s>>>(count, err, what, limit_ns, E, sink);
  return cudaGetLastError();
}

// =============================================================================
// Host side
// =============================================================================
namespace {

template <typename Kern>
cudaError_t launch_f(Kern k, int grid, size_t smem, cudaStream_t s, bool pdl, const LayerArgs& a,
                     bool cooperative = false) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreadsS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cooperative) {  // the expert kernel's grid barrier needs every CTA resident
    attr[n].id = cudaLaunchAttributeCooperative;
    attr[n].val.cooperative = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, k, a);
}

size_t up128(size_t x) { return (x + 127) & ~size_t(127); }

constexpr size_t kRingCap = 200 * 1024;

}  // namespace

bool plan_small(LayerArgs& a, int G, size_t optin) {
  const size_t budget = optin - 1024 - 256;
  const int NT = a.B <= 2 ? 2 : kSmallB;  // tokens the kernels hold at once (planned at two for B <= 2)
  {  // K1: whole rows of W_o, ~32 KB stages
    KTune& t = a.k1;
    const size_t row = (size_t)a.d_o * 2;
    t.rows_max = (a.d + G - 1) / G;
    t.rows_per_stage = (int)std::max<size_t>(1, std::min<size_t>(32768 / row, (size_t)t.rows_max));
    const size_t SB = up128((size_t)t.rows_per_stage * row);
    const size_t extra = up128(((size_t)t.rows_max * kCW * NT + (size_t)NT * t.rows_max) * 4) +
                         2 * kMaxStages * 8 + 64;
    t.stages = (int)std::min<size_t>(kMaxStages, (std::min(budget, kRingCap) - extra) / SB);
    if (t.stages < 2) return false;
    t.smem = (size_t)t.stages * SB + extra;
  }
  {  // K2: the whole router slice
    KTune& t = a.k2;
    t.rows_max = (a.E + G - 1) / G;
    t.smem = up128((size_t)t.rows_max * a.d * 2) + up128((size_t)t.rows_max * kCW * NT * 4 + 64 * 4) +
             8 + 32 * 4 + (a.route_tables ? kTopkScratch : 0) + 64;
    if (t.smem > budget) return false;
  }
  {  // K3 (phase A): pairs of gate/up rows; K4 fields: phase B of the same kernel
    KTune& t = a.k3;
    KTune& t4 = a.k4;
    const size_t row = (size_t)a.d * 2;
    const long long umax = std::min(a.E, std::max(a.B, 1) * a.k);
    t.rows_max = (int)((umax * a.I + G - 1) / G);  // pairs per CTA
    t4.rows_max = (a.d + G - 1) / G;                // output rows per CTA
    if (t4.rows_max > 4 * kCW) return false;
    const int eps = experts_per_stage(a.I / 32, NT);
    t4.rows_per_stage = eps;
    const size_t scratch_f =
        std::max((size_t)t.rows_max * 2 * kCW * NT, a_s_floats(std::max(a.B, 1), a.k, a.E, a.I, NT));
    const size_t extra = up128(scratch_f * 4) + route_bytes(NT) + 4 * kMaxStages * 8 + 64;
    const size_t SBd = up128((size_t)eps * t4.rows_max * a.I * 2);
    t.stages = 0;
    for (int ps = 2; ps >= 1 && t.stages < 2; --ps) {
      t.rows_per_stage = ps;
      const size_t SB = up128((size_t)2 * ps * row);
      t.stages = extra < budget ? (int)std::min<size_t>(kMaxStages, (budget - extra) / SB) : 0;
    }
    if (t.stages < 2) return false;
    const size_t regionA = (size_t)t.stages * up128((size_t)2 * t.rows_per_stage * row);
    t4.stages = (int)std::min<size_t>(kMaxStages, regionA / SBd);
    if (t4.stages < 2) return false;
    t.smem = std::max(regionA, (size_t)t4.stages * SBd) + extra;
    t4.smem = t.smem;
  }
  return true;
}

bool plan_fused(LayerArgs& a, int G, size_t optin) {
  const size_t budget = optin - 1024 - 256;
  const int NT = 2;
  KTune& o = a.k1;   // o_proj ring (W_r rows follow in the same ring)
  KTune& r = a.k2;   // router rows
  KTune& pa = a.k3;  // phase A
  KTune& pb = a.k4;  // phase B
  const size_t orow = (size_t)a.d_o * 2, row = (size_t)a.d * 2;
  o.rows_max = (a.d + G - 1) / G;
  if (o.rows_max > 4 * kCW) return false;
  r.rows_max = (a.E + G - 1) / G;
  const long long umax = std::min(a.E, std::max(a.B, 1) * a.k);
  pa.rows_max = (int)((umax * a.I + G - 1) / G);
  pb.rows_max = o.rows_max;
  o.rows_per_stage = (int)std::max<size_t>(1, std::min<size_t>(32768 / orow, (size_t)o.rows_max));
  const size_t scratch_f =
      layer_scratch_floats(NT, oproj_unit_cap(a.d, o.rows_per_stage, G), o.rows_per_stage, r.rows_max, pa.rows_max, a.d);
  const size_t a_s_bytes = a_s_floats(std::max(a.B, 1), a.k, a.E, a.I, NT) * 4;
  const size_t extra = up128(scratch_f * 4) + route_bytes(NT) + 6 * kMaxStages * 8 + 8 + 64;
  if (extra >= budget) return false;
  const size_t cap = budget - extra;
  const size_t SO = std::max(up128((size_t)o.rows_per_stage * orow), up128(row));
  o.stages = (int)std::min<size_t>(kMaxStages, cap / SO);
  r.rows_per_stage = (int)(SO / row);
  // the router rows' fills are all resident at once (the consumers wait for every one)
  if ((r.rows_max + r.rows_per_stage - 1) / r.rows_per_stage > o.stages) return false;
  size_t SA = 0;
  pa.stages = 0;
  for (int ps = 2; ps >= 1 && pa.stages < 2; --ps) {
    pa.rows_per_stage = ps;
    SA = up128((size_t)2 * ps * row);
    pa.stages = (int)std::min<size_t>(kMaxStages, cap / SA);
  }
  const int eps = experts_per_stage(a.I / 32, NT);
  pb.rows_per_stage = eps;
  const size_t SBd = up128((size_t)eps * pb.rows_max * a.I * 2);
  pb.stages = cap > a_s_bytes ? (int)std::min<size_t>(kMaxStages, (cap - a_s_bytes) / SBd) : 0;
  if (o.stages < 2 || pa.stages < 2 || pb.stages < 2) return false;
  const size_t region = std::max(std::max((size_t)o.stages * SO, (size_t)pa.stages * SA),
                                 (size_t)pb.stages * SBd + a_s_bytes);
  o.smem = region + extra;
  r.smem = pa.smem = pb.smem = o.smem;
  return o.smem <= budget;
}

// The TMA-staged router of the large-batch path: W_r slice, h ring (>= 2 stages of two tokens; also
// the routing-table builder's scratch), two partial buffers, rstd, barriers.
bool plan_router_big(LayerArgs& a, int G, size_t optin) {
  const size_t budget = optin - 1024 - 256;
  KTune& t = a.k2;
  t.rows_max = (a.E + G - 1) / G;
  const size_t w = up128((size_t)t.rows_max * a.d * 2), SHB = up128((size_t)2 * a.d * 4);
  const size_t tail = up128(((size_t)2 * t.rows_max * kCW * 2 + 64) * 4) + (1 + 2 * kMaxStages) * 8 + 64;
  t.stages = 0;
  for (int sh = kMaxStages; sh >= 2; --sh)
    if (w + std::max((size_t)sh * SHB, (size_t)kTopkScratch) + tail <= budget) {
      t.stages = sh;
      break;
    }
  if (t.stages < 2) return false;
  t.smem = w + std::max((size_t)t.stages * SHB, (size_t)kTopkScratch) + tail;
  return true;
}

bool router_big_ok(const LayerArgs& a0, size_t optin) {
  LayerArgs a = a0;
  return a.B >= 3 && a.B <= 64 && a.d <= 8192 && plan_router_big(a, 148, optin);
}

bool layer_fused_ok(const LayerArgs& a0, size_t optin) {
  LayerArgs a = a0;
  return a.B <= 2 && a.k <= 32 && a.d <= 8192 && a.d_o <= 8192 && a.E <= 2 * kRouteThreads &&
         plan_fused(a, 148, optin);
}

bool small_path_ok(const LayerArgs& a0, size_t optin) {
  LayerArgs a = a0;
  // up to kSmallB tokens with at most 64 (token, expert) entries: the per-CTA routing's tables
  return a.B <= kSmallB && a.B * a.k <= 64 && a.k <= 32 && a.d <= 8192 && a.d_o <= 8192 &&
         plan_small(a, 148, optin);
}

bool oproj_small_ok(const LayerArgs& a, size_t optin) { return small_path_ok(a, optin); }

bool router_ok(const LayerArgs& a0, size_t optin) {
  LayerArgs a = a0;
  const int G = 148;
  KTune& t = a.k2;
  t.rows_max = (a.E + G - 1) / G;
  const int nt = (a.d <= 8 * 32 * 2 * kCW && a.B > 2) ? kSmallB : 2;  // as launch_router_s
  t.smem = up128((size_t)t.rows_max * a.d * 2) + up128((size_t)t.rows_max * kCW * nt * 4 + 64 * 4) + 8 +
           32 * 4 + (a.route_tables ? kTopkScratch : 0) + 64;
  return a.d <= 8192 && t.smem <= optin - 1024 - 256;
}

cudaError_t set_small_attributes(size_t optin) {
  const int v = (int)optin;
  cudaError_t e = cudaSuccess;
#define SETS(k)                                                                                              \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, v); \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100)
  SETS((k_oproj_f<1, 2>));
  SETS((k_oproj_f<2, 2>));
  SETS((k_oproj_f<kSmallB, 2>));
  SETS((k_oproj_f<1, 3>));
  SETS((k_oproj_f<2, 3>));
  SETS((k_oproj_f<kSmallB, 3>));
#define SETS_D(k, ...) \
  SETS((k<__VA_ARGS__, 2>)); \
  SETS((k<__VA_ARGS__, 3>))
  SETS_D(k_router_f, 1);
  SETS_D(k_router_f, 2);
  SETS((k_router_f<kSmallB, 2>));
  SETS_D(k_experts_f, 1, 4);
  SETS_D(k_experts_f, 2, 4);
  SETS_D(k_experts_f, 1, 8);
  SETS_D(k_experts_f, 2, 8);
  SETS_D(k_experts_f, 1, 0);
  SETS_D(k_experts_f, 2, 0);
  SETS_D(k_experts_f, kSmallB, 4);
  SETS_D(k_experts_f, kSmallB, 8);
  SETS_D(k_experts_f, kSmallB, 0);
  SETS(k_router_big);
  SETS_D(k_layer_f, 1, 4);
  SETS_D(k_layer_f, 2, 4);
  SETS_D(k_layer_f, 1, 8);
  SETS_D(k_layer_f, 2, 8);
  SETS_D(k_layer_f, 1, 0);
  SETS_D(k_layer_f, 2, 0);
#undef SETS_D
#undef SETS
  return e;
}

namespace {
LayerArgs planned(const LayerArgs& a0, int grid, size_t optin) {
  LayerArgs a = a0;
  plan_small(a, grid, optin);
  return a;
}

// 8-element chunks per lane of a d-long activation slice over the 15 consumer warps: two cover
// d <= 7680, three the rest of the supported range.  The smaller slice has no chunk slot that
// is always empty (at d = 7168 a lane holds 1.9 chunks), so no loads or FMAs are spent on zeros.
bool two_chunks(int d) { return d <= 8 * 32 * 2 * kCW; }

template <int CPD>
cudaError_t launch_router_d(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  // above two tokens, four at a time where two chunks per lane leave the registers for them
  if (CPD == 2 && a.B > 2) return launch_f(k_router_f<kSmallB, 2>, grid, a.k2.smem, s, pdl, a);
  return a.B == 1 ? launch_f(k_router_f<1, CPD>, grid, a.k2.smem, s, pdl, a)
                  : launch_f(k_router_f<2, CPD>, grid, a.k2.smem, s, pdl, a);
}

template <int CPD>
cudaError_t launch_experts_d(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  const int epl = a.I / 32;
  const size_t sm = a.k3.smem;
  if (a.B > 2) {
    if (epl == 4) return launch_f(k_experts_f<kSmallB, 4, CPD>, grid, sm, s, pdl, a, true);
    if (epl == 8) return launch_f(k_experts_f<kSmallB, 8, CPD>, grid, sm, s, pdl, a, true);
    return launch_f(k_experts_f<kSmallB, 0, CPD>, grid, sm, s, pdl, a, true);
  }
  if (epl == 4)
    return a.B == 1 ? launch_f(k_experts_f<1, 4, CPD>, grid, sm, s, pdl, a, true)
                    : launch_f(k_experts_f<2, 4, CPD>, grid, sm, s, pdl, a, true);
  if (epl == 8)
    return a.B == 1 ? launch_f(k_experts_f<1, 8, CPD>, grid, sm, s, pdl, a, true)
                    : launch_f(k_experts_f<2, 8, CPD>, grid, sm, s, pdl, a, true);
  return a.B == 1 ? launch_f(k_experts_f<1, 0, CPD>, grid, sm, s, pdl, a, true)
                  : launch_f(k_experts_f<2, 0, CPD>, grid, sm, s, pdl, a, true);
}

template <int CPD>
cudaError_t launch_layer_d(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  const int epl = a.I / 32;
  const size_t sm = a.k1.smem;
  if (epl == 4)
    return a.B == 1 ? launch_f(k_layer_f<1, 4, CPD>, grid, sm, s, pdl, a, true)
                    : launch_f(k_layer_f<2, 4, CPD>, grid, sm, s, pdl, a, true);
  if (epl == 8)
    return a.B == 1 ? launch_f(k_layer_f<1, 8, CPD>, grid, sm, s, pdl, a, true)
                    : launch_f(k_layer_f<2, 8, CPD>, grid, sm, s, pdl, a, true);
  return a.B == 1 ? launch_f(k_layer_f<1, 0, CPD>, grid, sm, s, pdl, a, true)
                  : launch_f(k_layer_f<2, 0, CPD>, grid, sm, s, pdl, a, true);
}
}  // namespace

cudaError_t launch_oproj_s(const LayerArgs& a0, int grid, cudaStream_t s, bool pdl, size_t optin) {
  const LayerArgs a = planned(a0, grid, optin);
  if (two_chunks(a.d_o)) {
    if (a.B > 2) return launch_f(k_oproj_f<kSmallB, 2>, grid, a.k1.smem, s, pdl, a);
    return a.B == 1 ? launch_f(k_oproj_f<1, 2>, grid, a.k1.smem, s, pdl, a)
                    : launch_f(k_oproj_f<2, 2>, grid, a.k1.smem, s, pdl, a);
  }
  if (a.B > 2) return launch_f(k_oproj_f<kSmallB, 3>, grid, a.k1.smem, s, pdl, a);
  return a.B == 1 ? launch_f(k_oproj_f<1, 3>, grid, a.k1.smem, s, pdl, a)
                  : launch_f(k_oproj_f<2, 3>, grid, a.k1.smem, s, pdl, a);
}

cudaError_t launch_router_s(const LayerArgs& a0, int grid, cudaStream_t s, bool pdl, size_t optin) {
  LayerArgs a = a0;
  a.k2.rows_max = (a.E + grid - 1) / grid;
  const int nt = (two_chunks(a.d) && a.B > 2) ? kSmallB : 2;  // tokens per pass of the launched kernel
  a.k2.smem = up128((size_t)a.k2.rows_max * a.d * 2) + up128((size_t)a.k2.rows_max * kCW * nt * 4 + 64 * 4) +
              8 + 32 * 4 + (a.route_tables ? kTopkScratch : 0) + 64;
  (void)optin;
  return two_chunks(a.d) ? launch_router_d<2>(a, grid, s, pdl) : launch_router_d<3>(a, grid, s, pdl);
}

cudaError_t launch_experts_s(const LayerArgs& a0, int grid, cudaStream_t s, bool pdl, size_t optin) {
  const LayerArgs a = planned(a0, grid, optin);
  return two_chunks(a.d) ? launch_experts_d<2>(a, grid, s, pdl) : launch_experts_d<3>(a, grid, s, pdl);
}

cudaError_t launch_layer_s(const LayerArgs& a0, int grid, cudaStream_t s, bool pdl, size_t optin) {
  LayerArgs a = a0;
  if (!plan_fused(a, grid, optin)) return cudaErrorInvalidConfiguration;
  return two_chunks(a.d) ? launch_layer_d<2>(a, grid, s, pdl) : launch_layer_d<3>(a, grid, s, pdl);
}

cudaError_t launch_router_big(const LayerArgs& a0, int grid, cudaStream_t s, bool pdl, size_t optin) {
  LayerArgs a = a0;
  if (!plan_router_big(a, grid, optin)) return cudaErrorInvalidConfiguration;
  return launch_f(k_router_big, grid, a.k2.smem, s, pdl, a);
}

}  // namespace moe
