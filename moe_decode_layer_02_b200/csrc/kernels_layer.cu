// The batch <= 2 decode layer as one cooperative kernel per layer (one CTA per SM, a producer
// warp that moves every weight byte with TMA bulk copies, 15 consumer warps).
//
// At batch 1-2 a layer step reads 218-306 MB of weights and does about one flop per byte, so
// the step is a weight stream, and what is not streaming is the serial chain between the
// phases.  The phases and what keeps the chain short:
//
//   o_proj    h = residual + W_o . attn_out for this CTA's rows (whole W_o rows through the
//             ring), per-CTA sums of h^2.  The CTA's router rows follow W_o in the same ring,
//             so they leave HBM during the o_proj tail.
//   barrier 1 (every h and sum of h^2 written)
//   router    the 148 partial sums, this CTA's h slice and (already resident) gamma are read
//             in one round trip; rstd and x = h * rstd * gamma in registers (x stays there
//             for the expert phase); the logits of this CTA's router rows.
//   barrier 2 consumers only arrive.  The producer warp waits for it, selects the top-k of
//             every logit itself (one warp per token), forms the union of the selected
//             experts and issues the first expert copies at once.
//   experts   the union's gate/up rows are cut into chunks of PS row pairs; chunk z goes to
//             CTA z mod G in round z / G, so every round all CTAs work on the same one or two
//             experts and the experts finish in union order.  After each round one warp
//             reduces the chunk's partial dots into a = silu(g) * u, stores it and adds PS to
//             the expert's row counter (release).  Each CTA owns output rows [i0, i1): its
//             block of W_down[e] for every union expert streams through a second ring, and is
//             combined, a few rounds after the expert's last chunk, once the expert's counter
//             shows all I rows published (acquire).  Each lane accumulates its rows over all
//             experts in registers; out = bf16(h + sum) at the end.
// There is no grid barrier between the gate/up and the down projections: the per-expert
// counters order exactly what depends on what, and the down blocks stream while later
// experts' gate/up rows do.  Every wait is bounded; the last CTA to finish clears the
// counters for the next launch.  The producer issues copies in the order the consumers use
// them, so a full ring never blocks an item the consumers are waiting for.
//
// Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted kernels",
// section "How the specialised decode path works" (small-matrix kernels at batch one or two;
// o_proj fused with the residual step; 16 of 896 experts per token; decode is bound by weight
// reads); "vLLM and NVIDIA use coding agents to nearly double Kimi K3 decode speed, then
// rethink how to review it" (fewer kernels per layer).
#include <algorithm>
#include <type_traits>

#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "mma.cuh"
#include "rowdot.cuh"
#include "topk.cuh"

namespace moe {

namespace {

constexpr int kRBox = 224;                // experts per W_r box (one 2-D tensor-map copy)
constexpr int kRBoxBytes = kRBox * 128;   // 64 bf16 columns per expert
constexpr int kPS = 2;       // gate/up row pairs per chunk
constexpr int kDownLag = 2;  // rounds between an expert's last chunk and the use of its down block
constexpr int kDownPrefetch = 2;  // rounds ahead of its copy that a down block is prefetched into L2
constexpr int kRPW = 4;      // output rows per consumer warp (rows per CTA <= 60)

// Routing state of one CTA (shared memory).
struct alignas(16) Route2 {
  float sel_g[2][32];   // gate of each token's j-th selection
  int sel_i[2][32];     // expert of each token's j-th selection (descending logit)
  int un_e[kMaxUnion];  // union experts: token 0's selections, then token 1's new ones
  float un_g[kMaxUnion][2];  // gate of union expert u for each token (0: not selected)
  int U;
  int pad[3];
  float cand[2][2 * kCandStride];  // warp_topk scratch of the two routing warps
  int dry_i[32];                   // outputs of the producer's warm-up pass
  float dry_g[32];
};

// Shared-memory layout (byte offsets), the same on host and device.
struct Smem2 {
  size_t so_b, sp_b, sd_b;  // stage sizes: o_proj/router ring, gate/up ring, down ring
  size_t pring, dring;      // offsets of the gate/up and down rings inside the region
  size_t part, sq, hs, route, bars, misc, total;
};

__host__ __device__ inline size_t up128(size_t x) { return (x + 127) & ~size_t(127); }

__host__ __device__ inline Smem2 smem2(int NT, const LayerArgs& a) {
  Smem2 L;
  const size_t orow = (size_t)a.d_o * 2, row = (size_t)a.d * 2;
  const int RM = a.k1.rows_max;
  // an O-ring stage holds W_o rows or one W_r box (1024-aligned for the 128-byte swizzle)
  L.so_b = up128((size_t)a.k1.rows_per_stage * orow);
  if (L.so_b < (size_t)kRBoxBytes) L.so_b = kRBoxBytes;
  L.so_b = (L.so_b + 1023) & ~size_t(1023);
  L.sp_b = up128((size_t)2 * kPS * row);
  L.sd_b = up128((size_t)RM * a.I * 2);
  L.pring = 0;
  L.dring = (size_t)a.k3.stages * L.sp_b;
  size_t region = (size_t)a.k1.stages * L.so_b;
  if (L.dring + (size_t)a.k4.stages * L.sd_b > region) region = L.dring + (size_t)a.k4.stages * L.sd_b;
  size_t pf = (size_t)RM * kCW * NT;                               // o_proj partials
  if ((size_t)NT * 64 > pf) pf = (size_t)NT * 64;                 // h * gamma of the router columns
  if ((size_t)2 * 2 * kPS * kCW * NT > pf) pf = (size_t)2 * 2 * kPS * kCW * NT;  // chunk partials
  L.part = region;
  L.sq = L.part + up128(pf * 4);
  L.hs = L.sq + up128((size_t)NT * RM * 4);
  L.route = L.hs + up128((size_t)NT * RM * 4);
  L.bars = L.route + up128(sizeof(Route2));
  L.misc = L.bars + (6 * kMaxStages + 2 + kMaxUnion + 4) * 8;
  L.total = L.misc + 64 + 1024;  // + alignment of the dynamic shared memory to 1024
  return L;
}

// Round after which CTA-local consumers use union expert u's down block.
__device__ __forceinline__ int down_round(int u, int cpe, int G) { return ((u + 1) * cpe - 1) / G + kDownLag; }

// Consumers arrive at a grid barrier without waiting (writes before it are released).
__device__ __forceinline__ void grid_arrive(unsigned* count) {
  csync();
  if (threadIdx.x == 0) red_release_add(count, 1u);
}

__device__ __forceinline__ void grid_barrier2(unsigned* count, unsigned target, volatile int* abort_flag,
                                              uint32_t* err) {
  csync();
  if (threadIdx.x == 0) {
    red_release_add(count, 1u);
    if (ld_acquire_u32(count) < target) {
      const unsigned long long t0 = globaltimer();
      while (ld_acquire_u32(count) < target) {
        if (globaltimer() - t0 > kWaitLimitNs) {
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

// Top-k and gates of one token by one warp: lane j < K writes the j-th selection (descending
// logit) and its gate to sel_i / sel_g, and to the caller's outputs when given.  Not inlined,
// so one copy of the code serves every call: the producer warp runs it once on stale data
// during the o_proj tail (its instructions are then resident when the real selection runs
// right after barrier 2, where every SM would otherwise fetch them cold at the same moment).
__device__ __noinline__ void route_token(const float* logits, int E, int K, float* cand, int* sel_i, float* sel_g,
                                         int* user_idx, float* user_gate, uint32_t* err, int lane) {
  float my_v = 0.f;
  int my_i = 0;
  warp_topk(logits, E, K, cand, reinterpret_cast<int*>(cand + kCandStride), lane, my_v, my_i);
  const float g = warp_gate(my_v, lane, K);
  if (lane < K) {
    const int e = (my_i >= 0 && my_i < E) ? my_i : 0;
    if (e != my_i && err) atomicOr(err, kErrBounds);
    sel_i[lane] = e;
    sel_g[lane] = g;
    if (user_idx) user_idx[lane] = e;
    if (user_gate) user_gate[lane] = g;
  }
  __syncwarp();
}

// Bit-exact fp32 RMS statistics: lane partial sums over the per-CTA sums in a fixed order,
// then a butterfly; every warp of every CTA gets the same bits.
__device__ __forceinline__ float rstd_of(const LayerArgs& a, int t, int G, int lane) {
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
  return 1.0f / sqrtf(ss / (float)a.d + a.eps);
}

}  // namespace

template <int NT, int CPLX, int EPL>
__global__ void __launch_bounds__(kThreadsS, 1) k_layer2(const __grid_constant__ CUtensorMap tmR, const LayerArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int CPLO = kCPLf;
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, d_o = a.d_o, I = a.I, B = a.B, E = a.E;
  const int SO = a.k1.stages, RS = a.k1.rows_per_stage, RM = a.k1.rows_max;
  const int SP = a.k3.stages, SD = a.k4.stages;
  const uint32_t orow_bytes = (uint32_t)d_o * 2u, row_bytes = (uint32_t)d * 2u, drow_bytes = (uint32_t)I * 2u;
  const Smem2 L = smem2(NT, a);
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int i0 = (int)lo, nrows = (int)(hi - lo);  // o_proj rows = output rows
  split_range(E, G, c, lo, hi);
  const int e0 = (int)lo, nr = (int)(hi - lo);      // experts whose logits this CTA finishes
  const int x0 = i0 & ~7, nbox = (E + kRBox - 1) / kRBox;  // W_r columns [x0, x0 + 64) in boxes

  unsigned char* ring = smem;
  float* part = reinterpret_cast<float*>(smem + L.part);
  float* sq = reinterpret_cast<float*>(smem + L.sq);  // [NT][RM]
  float* hs = reinterpret_cast<float*>(smem + L.hs);  // [RM][NT]
  Route2* rt = reinterpret_cast<Route2*>(smem + L.route);
  uint64_t* fullO = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* emptyO = fullO + kMaxStages;
  uint64_t* fullP = emptyO + kMaxStages;
  uint64_t* emptyP = fullP + kMaxStages;
  uint64_t* fullD = emptyP + kMaxStages;
  uint64_t* emptyD = fullD + kMaxStages;
  uint64_t* route_ready = emptyD + kMaxStages;
  uint64_t* tok1_ready = route_ready + 1;
  uint64_t* dgate = tok1_ready + 1;  // [kMaxUnion]: expert u's activations are all published
  uint64_t* pfull = dgate + kMaxUnion;  // [2]: every consumer warp wrote its partials of a round
  uint64_t* pfree = pfull + 2;          // [2]: that round's publisher has read them
  int* s_misc = reinterpret_cast<int*>(smem + L.misc);
  volatile int* abort_flag = s_misc;
  unsigned* bar_count = &a.ws.counters[kCntLayer];
  uint32_t* err = a.ws.err;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(fullO, emptyO, SO, kCW);
    init_ring(fullP, emptyP, SP, kCW);
    init_ring(fullD, emptyD, SD, kCW);
    mbar_init(route_ready, 1);
    mbar_init(tok1_ready, 1);
    for (int u = 0; u < kMaxUnion; ++u) mbar_init(&dgate[u], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pfull[b], kCW);
      mbar_init(&pfree[b], 1);
    }
    s_misc[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  const int cpe = I / kPS;  // chunks per expert
  const int qbase_o = (d_o / 8) * warp / kCW, qpw_o = (d_o / 8) * (warp + 1) / kCW - qbase_o;
  const int qbase = (d / 8) * warp / kCW, qpw = (d / 8) * (warp + 1) / kCW - qbase;

  if (warp == kCW) {
    // =========================== producer warp ===========================
    int itO = 0;
    const uint64_t pol = policy_evict_first();
    if (lane == 0) {  // weights are static: W_o, then W_r, before the dependency resolves
      bulk_prefetch_l2(a.gamma, row_bytes);
      for (int r = i0; r < i0 + nrows; r += RS, ++itO) {
        const int n = min(RS, i0 + nrows - r);
        if (!ring_acquire(emptyO, itO, SO, abort_flag, err)) break;
        const int s = itO % SO;
        mbar_arrive_expect_tx(&fullO[s], n * orow_bytes);
        bulk_g2s(ring + s * L.so_b, a.w_o + (size_t)r * d_o, n * orow_bytes, &fullO[s], pol);
      }
      // W_r[:, x0 .. x0 + 64) for every expert, one box of kRBox experts per stage (columns past
      // d and experts past E read as zeros)
      for (int j = 0; j < nbox && !*abort_flag; ++j, ++itO) {
        if (!ring_acquire(emptyO, itO, SO, abort_flag, err)) break;
        const int s = itO % SO;
        mbar_arrive_expect_tx(&fullO[s], (uint32_t)kRBoxBytes);
        tma_load_2d(ring + s * L.so_b, &tmR, x0, j * kRBox, &fullO[s]);
      }
      if (a.pf_w_o) {  // next layer: what the same CTA reads first, into L2
        if (nr > 0) bulk_prefetch_l2(a.pf_w_r + (size_t)e0 * d, nr * row_bytes);
        if (c == 0) bulk_prefetch_l2(a.pf_gamma, row_bytes);
        size_t left = (size_t)min(a.pf_w_o_rows, nrows) * orow_bytes;
        const unsigned char* src = reinterpret_cast<const unsigned char*>(a.pf_w_o + (size_t)i0 * d_o);
        for (size_t off = 0; left > 0;) {
          const uint32_t n = (uint32_t)min(left, (size_t)65536);
          bulk_prefetch_l2(src + off, n);
          off += n;
          left -= n;
        }
      }
    }
    __syncwarp();
    // warm-up pass of the selection code on whatever the logits buffer holds (nothing is
    // written outside this CTA's shared memory)
    route_token(a.ws.logits, E, a.k, rt->cand[0], rt->dry_i, rt->dry_g, nullptr, nullptr, nullptr, lane);
    pdl_wait();  // the previous kernel (counters, logits of an earlier launch) is complete
    if (lane == 0) {
      // every O-ring fill has landed and been read (the W_r boxes, before barrier 1), so the
      // region may take the expert rings
      ring_drain(fullO, itO, SO, err);
      for (int i = itO - SO < 0 ? 0 : itO - SO; i < itO; ++i) mbar_drain(&emptyO[i % SO], (i / SO) & 1, err);
    }
    __syncwarp();
    warp_wait_count(bar_count, 2u * (unsigned)G, abort_flag, err);  // barrier 2: every logit written
    route_token(a.ws.logits, E, a.k, rt->cand[0], rt->sel_i[0], rt->sel_g[0], c == 0 ? a.user_idx : nullptr,
                c == 0 ? a.user_gate : nullptr, err, lane);
    if (B == 2) mbar_wait(tok1_ready, 0, abort_flag, err);  // every lane: token 1's selection
    // union: token 0's selections in rank order, then token 1's experts that token 0 lacks
    const int K = a.k;
    int U = K;
    {
      const int e_0 = (lane < K) ? rt->sel_i[0][lane] : -1;
      if (lane < K) {
        rt->un_e[lane] = e_0;
        rt->un_g[lane][0] = rt->sel_g[0][lane];
        rt->un_g[lane][1] = 0.f;
      }
      if (B == 2) {
        const int e_1 = (lane < K) ? rt->sel_i[1][lane] : -2;
        const float g_1 = (lane < K) ? rt->sel_g[1][lane] : 0.f;
        int pos = -1;
        for (int o = 0; o < K; ++o)
          if (__shfl_sync(0xffffffffu, e_0, o) == e_1) pos = o;
        const unsigned fresh = __ballot_sync(0xffffffffu, lane < K && pos < 0);
        if (lane < K) {
          if (pos >= 0) {
            rt->un_g[pos][1] = g_1;
          } else {
            const int u = K + __popc(fresh & ((1u << lane) - 1u));
            rt->un_e[u] = e_1;
            rt->un_g[u][0] = 0.f;
            rt->un_g[u][1] = g_1;
          }
        }
        U = K + __popc(fresh);
      }
    }
    __syncwarp();
    if (lane == 0) {
      rt->U = U;
      mbar_arrive(route_ready);  // releases the routing state to the consumers
    }
    // ---- expert phase: lane 0 streams the gate/up chunks (and sends down blocks to L2 ahead
    // of their turn), lane 1 streams the down blocks into their own ring, each in the order the
    // consumers use them; the two rings are independent, so neither stream waits on the other.
    const int Z = U * cpe, Mc = (Z > c) ? (Z - c + G - 1) / G : 0;
    const uint32_t blk = (uint32_t)nrows * drow_bytes;
    if (lane == 0) {
      int itP = 0, npf = 0;
      auto prefetch_down = [&](int upto_round) {
        for (; npf < U && nrows > 0 && down_round(npf, cpe, G) <= upto_round; ++npf)
          bulk_prefetch_l2(a.w_down + ((size_t)rt->un_e[npf] * d + i0) * I, blk);
      };
      prefetch_down(kDownPrefetch - 1);
      for (int m = 0; m < Mc; ++m) {
        const int z = c + m * G, u = z / cpe, t0 = (z - u * cpe) * kPS;
        prefetch_down(m + kDownPrefetch);
        if (!ring_acquire(emptyP, itP, SP, abort_flag, err)) break;
        const int s = itP % SP;
        const uint16_t* g_rows = a.w_gu + ((size_t)rt->un_e[u] * 2 * I + t0) * d;
        mbar_arrive_expect_tx(&fullP[s], 2u * kPS * row_bytes);
        bulk_g2s(ring + L.pring + s * L.sp_b, g_rows, kPS * row_bytes, &fullP[s], pol);
        bulk_g2s(ring + L.pring + s * L.sp_b + (size_t)kPS * row_bytes, g_rows + (size_t)I * d, kPS * row_bytes,
                 &fullP[s], pol);
        ++itP;
      }
      prefetch_down(1 << 30);
      ring_drain(fullP, itP, SP, err);
    } else if (lane == 1 && nrows > 0) {
      int itD = 0;
      for (int u = 0; u < U; ++u, ++itD) {
        if (!ring_acquire(emptyD, itD, SD, abort_flag, err)) break;
        const int s = itD % SD;
        mbar_arrive_expect_tx(&fullD[s], blk);
        bulk_g2s(ring + L.dring + s * L.sd_b, a.w_down + ((size_t)rt->un_e[u] * d + i0) * I, blk, &fullD[s], pol);
      }
      ring_drain(fullD, itD, SD, err);
    }
    return;
  }

  // =========================== consumer warps ===========================
  pdl_wait();  // attn_out and residual may come from the previous kernel
  float res_v = 0.f;  // this thread's residual element of the o_proj epilogue (rows x tokens < kCT)
  if (tid < nrows * B) {
    const int rr = tid / B, t = tid % B;
    res_v = bf16f(__ldcg(reinterpret_cast<const unsigned short*>(a.resid + (size_t)t * d + i0 + rr)));
  }
  uint4 gam_raw[CPLX];  // gamma is static: loaded now, used after barrier 1
#pragma unroll
  for (int j = 0; j < CPLX; ++j)
    gam_raw[j] = cvalid(qpw, j, lane) ? ld_weight_u4(a.gamma + (size_t)(qbase + j * 32 + lane) * 8)
                                      : make_uint4(0, 0, 0, 0);
  int itO = 0;
  // ---- o_proj ----
  {
    constexpr int kRI = 2;
    float xa[NT][CPLO][8];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < CPLO; ++j) {
        uint4 u = make_uint4(0, 0, 0, 0);
        if (cvalid(qpw_o, j, lane)) u = ld_act_u4(a.attn + (size_t)t * d_o + (size_t)(qbase_o + j * 32 + lane) * 8);
        unpack8f(u, xa[t][j]);
      }
    for (int r = i0; r < i0 + nrows; r += RS, ++itO) {
      const int n = min(RS, i0 + nrows - r), s = itO % SO;
      mbar_wait(&fullO[s], (itO / SO) & 1, abort_flag, err);
      const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + s * L.so_b);
      for (int j0 = 0; j0 < n; j0 += kRI) {
        const uint16_t* rp[kRI];
#pragma unroll
        for (int k = 0; k < kRI; ++k) rp[k] = st + (size_t)min(j0 + k, n - 1) * d_o;
        float v[kRI * NT];
        rows_dot<NT, kRI>(rp, n - j0, xa, qbase_o, qpw_o, lane, v);
        const float tot = warp_reduce_multi<kRI * NT>(v, lane);
        const int vi = multi_index<kRI * NT>(lane), j = j0 + vi / NT, t = vi % NT;
        if (multi_writer<kRI * NT>(lane) && j < n) part[((r - i0 + j) * kCW + warp) * NT + t] = tot;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&emptyO[s]);
    }
  }
  csync();
  if (tid < nrows * B) {
    const int rr = tid / B, t = tid % B;
    float sacc = 0.f;
#pragma unroll
    for (int w = 0; w < kCW; ++w) sacc += part[(rr * kCW + w) * NT + t];
    const float hv = res_v + sacc;
    a.ws.h[(size_t)t * d + i0 + rr] = hv;
    hs[rr * NT + t] = hv;
    sq[t * RM + rr] = hv * hv;
  }
  csync();
  if (warp < B) {  // per-CTA sum of h^2, fixed order
    float ss = 0.f;
    for (int rr = lane; rr < nrows; rr += 32) ss += sq[warp * RM + rr];
    ss = warp_sum(ss);
    if (lane == 0) a.ws.ss_part[(size_t)c * a.maxB + warp] = ss;
  }
  // Router, split over K: logits[t][e] = rstd[t] * sum_i W_r[e][i] (h[t][i] gamma[i]); this
  // CTA's share is the sum over its own rows i in [i0, i0 + nrows), for every expert, formed
  // here before barrier 1 (it needs no other CTA's h).  h * gamma of columns x0 .. x0 + 63
  // (zero outside the CTA's rows) goes to shared memory (the o_proj partials are spent).
  float* hg = part;  // [NT][64]
  for (int z = tid; z < NT * 64; z += kCT) {
    const int t = z >> 6, k = z & 63, i = x0 + k;
    hg[z] = (t < B && i >= i0 && i < i0 + nrows) ? hs[(i - i0) * NT + t] * bf16f(a.gamma[i]) : 0.f;
  }
  csync();
  {
    for (int j = 0; j < nbox; ++j) mbar_wait(&fullO[(itO + j) % SO], ((itO + j) / SO) & 1, abort_flag, err);
    const int Bp = a.maxB;
    float* P = a.ws.rpart + (size_t)c * E * Bp;  // [E][Bp]: this CTA's partial logits
#pragma unroll 1
    for (int e = tid; e < E; e += kCT) {
      const int j = e / kRBox, r = e - j * kRBox;
      const unsigned char* tile = ring + ((itO + j) % SO) * L.so_b;
      float acc[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t] = 0.f;
#pragma unroll 1
      for (int q = 0; q < 8; ++q) {
        float w[8];
        unpack8f(*reinterpret_cast<const uint4*>(tile + swz(r, q)), w);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float4 g0 = *reinterpret_cast<const float4*>(hg + t * 64 + 8 * q);
          const float4 g1 = *reinterpret_cast<const float4*>(hg + t * 64 + 8 * q + 4);
          acc[t] = fmaf(w[0], g0.x, acc[t]); acc[t] = fmaf(w[1], g0.y, acc[t]);
          acc[t] = fmaf(w[2], g0.z, acc[t]); acc[t] = fmaf(w[3], g0.w, acc[t]);
          acc[t] = fmaf(w[4], g1.x, acc[t]); acc[t] = fmaf(w[5], g1.y, acc[t]);
          acc[t] = fmaf(w[6], g1.z, acc[t]); acc[t] = fmaf(w[7], g1.w, acc[t]);
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) P[(size_t)e * Bp + t] = acc[t];
    }
    __syncwarp();
    if (lane == 0)
      for (int j = 0; j < nbox; ++j) mbar_arrive(&emptyO[(itO + j) % SO]);
  }
  grid_barrier2(bar_count, (unsigned)G, abort_flag, err);

  // ---- after barrier 1: logits of this CTA's experts, then x = h * rstd * gamma ----
  float x[NT][CPLX][8];
  {
    // one warp per (expert, token): lanes sum the CTAs' partials in a fixed lane-strided order,
    // then a butterfly (the loads of all lanes are in flight together)
    const int Bp = a.maxB;
    for (int z = warp; z < nr * NT; z += kCW) {
      const int e = e0 + z / NT, t = z % NT;
      float sacc = 0.f, ss = 0.f;  // the partials and, in the same round trips, the sums of h^2
      for (int c0 = 0; c0 < G; c0 += 8 * 32) {
        float pv[8], qv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int cc = c0 + k * 32 + lane;
          pv[k] = cc < G ? ld_act(a.ws.rpart + ((size_t)cc * E + e) * Bp + t) : 0.f;
          qv[k] = cc < G ? ld_act(&a.ws.ss_part[(size_t)cc * a.maxB + t]) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          sacc += pv[k];
          ss += qv[k];
        }
      }
      sacc = warp_sum(sacc);
      ss = warp_sum(ss);  // the fixed-order sum of rstd_of: the same rstd bits everywhere
      const float r = 1.0f / sqrtf(ss / (float)a.d + a.eps);
      if (lane == 0) a.ws.logits[(size_t)t * E + e] = r * sacc;
    }
  }
  grid_arrive(bar_count);  // barrier 2: the producer warps wait for it
  if (NT == 2 && warp == 1) {  // token 1's selection, in parallel with the producer's token 0
    warp_wait_count(bar_count, 2u * (unsigned)G, abort_flag, err);
    route_token(a.ws.logits + E, E, a.k, rt->cand[1], rt->sel_i[1], rt->sel_g[1],
                c == 0 && a.user_idx ? a.user_idx + a.k : nullptr, c == 0 && a.user_gate ? a.user_gate + a.k : nullptr,
                err, lane);
    if (lane == 0) mbar_arrive(tok1_ready);
  }
  {
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < CPLX; ++j) {
        if (cvalid(qpw, j, lane)) {
          const float* hp = a.ws.h + (size_t)t * d + (size_t)(qbase + j * 32 + lane) * 8;
          const float4 h0 = ld_act4(hp), h1 = ld_act4(hp + 4);
          x[t][j][0] = h0.x; x[t][j][1] = h0.y; x[t][j][2] = h0.z; x[t][j][3] = h0.w;
          x[t][j][4] = h1.x; x[t][j][5] = h1.y; x[t][j][6] = h1.z; x[t][j][7] = h1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) x[t][j][e] = 0.f;
        }
      }
    float rv[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) rv[t] = rstd_of(a, t, G, lane);
    if (c == 0 && warp == 0 && lane < NT) a.ws.rstd[lane] = rv[lane == 0 ? 0 : NT - 1];
#pragma unroll
    for (int j = 0; j < CPLX; ++j) {
      float gam[8];
      unpack8f(gam_raw[j], gam);
      const int q = qbase + j * 32 + lane;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[t][j][e] = x[t][j][e] * rv[t] * gam[e];
        if (cvalid(qpw, j, lane) && q % G == c) {  // each chunk of x is written by one CTA
          float* xp = a.ws.x + (size_t)t * d + (size_t)q * 8;
          *reinterpret_cast<float4*>(xp) = make_float4(x[t][j][0], x[t][j][1], x[t][j][2], x[t][j][3]);
          *reinterpret_cast<float4*>(xp + 4) = make_float4(x[t][j][4], x[t][j][5], x[t][j][6], x[t][j][7]);
        }
      }
    }
  }
  mbar_wait(route_ready, 0, abort_flag, err);
  const int U = rt->U;

  // ---- experts ----
  const int Z = U * cpe, Mc = (Z > c) ? (Z - c + G - 1) / G : 0;
  float acc[kRPW][NT];
#pragma unroll
  for (int i = 0; i < kRPW; ++i)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[i][t] = 0.f;
  int itD = 0;
  auto consume_down = [&](int u) {
    if (nrows == 0) return;
    const int s = itD % SD;
    mbar_wait(&fullD[s], (itD / SD) & 1, abort_flag, err);
    // One load per CTA polls the expert's counter (acquire) and opens a CTA-local gate for the
    // other warps: 148 pollers per expert instead of 148 x 15 on one L2 line.  Warp 0 polls as
    // a whole (lane 0 loads, the result is broadcast), so none of its lanes spins on the gate
    // while the lane that opens it still has to run.
    if (warp == 0) {
      bool done = __shfl_sync(0xffffffffu, lane == 0 ? ld_acquire_u32(&a.ws.ecnt[u]) >= (unsigned)I : false, 0);
      if (!done && !*abort_flag) {
        const unsigned long long t0 = globaltimer();
        while (!done) {
          __nanosleep(64);
          done = __shfl_sync(0xffffffffu, lane == 0 ? ld_acquire_u32(&a.ws.ecnt[u]) >= (unsigned)I : false, 0);
          if (!done && globaltimer() - t0 > kWaitLimitNs) {
            if (lane == 0) {
              *abort_flag = 1;
              atomicOr(err, kErrTimeout);
            }
            break;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&dgate[u]);
    }
    mbar_wait(&dgate[u], 0, abort_flag, err);  // all I activations of expert u published
    const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + L.dring + s * L.sd_b);
    const float* ap = a.ws.a_u + (size_t)u * 2 * I;
    if constexpr (EPL == 4 || EPL == 8) {
      using WT = typename std::conditional<EPL == 4, uint2, uint4>::type;
      float ga[NT][EPL];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float g = rt->un_g[u][t];
#pragma unroll
        for (int x4 = 0; x4 < EPL; x4 += 4) {
          const float4 f = ld_act4(ap + (size_t)t * I + lane * EPL + x4);
          ga[t][x4] = g * f.x; ga[t][x4 + 1] = g * f.y; ga[t][x4 + 2] = g * f.z; ga[t][x4 + 3] = g * f.w;
        }
      }
#pragma unroll
      for (int i = 0; i < kRPW; ++i) {
        const int rl = warp + kCW * i;
        if (rl < nrows) {
          const WT w = *reinterpret_cast<const WT*>(st + (size_t)rl * I + lane * EPL);
          float wf[8];
          if constexpr (EPL == 4) {
            wf[0] = bf16lo(w.x); wf[1] = bf16hi(w.x); wf[2] = bf16lo(w.y); wf[3] = bf16hi(w.y);
          } else {
            unpack8f(reinterpret_cast<const uint4&>(w), wf);
          }
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            float sdot = 0.f;
#pragma unroll
            for (int x1 = 0; x1 < EPL; ++x1) sdot = fmaf(wf[x1], ga[t][x1], sdot);
            acc[i][t] += sdot;
          }
        }
      }
    } else {  // any other I: epl = I / 32 <= 16 elements per lane
      const int epl = I / 32;
#pragma unroll
      for (int i = 0; i < kRPW; ++i) {
        const int rl = warp + kCW * i;
        if (rl < nrows) {
          const uint16_t* wr = st + (size_t)rl * I + lane * epl;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float g = rt->un_g[u][t];
            float sdot = 0.f;
            for (int x1 = 0; x1 < epl; ++x1) sdot = fmaf(bf16f(wr[x1]), g * ld_act(ap + (size_t)t * I + lane * epl + x1), sdot);
            acc[i][t] += sdot;
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&emptyD[s]);
    ++itD;
  };
  int nu = 0;
  for (int m = 0; m < Mc; ++m) {
    const int z = c + m * G, u = z / cpe, t0 = (z - u * cpe) * kPS;
    const int s = m % SP;
    mbar_wait(&fullP[s], (m / SP) & 1, abort_flag, err);
    const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + L.pring + s * L.sp_b);
    constexpr int R = 2 * kPS;  // gate rows, then up rows
    const uint16_t* rp[R];
#pragma unroll
    for (int k = 0; k < R; ++k) rp[k] = st + (size_t)k * d;
    float v[R * NT];
    rows_dot<NT, R>(rp, R, x, qbase, qpw, lane, v);
    float* pb = part + (size_t)(m & 1) * R * kCW * NT;  // [R][kCW][NT]
    // the buffer of round m - 2 must have been read by that round's publisher
    if (m >= 2) mbar_wait(&pfree[m & 1], ((m - 2) >> 1) & 1, abort_flag, err);
    const float tot = warp_reduce_multi<R * NT>(v, lane);
    const int vi = multi_index<R * NT>(lane);
    if (multi_writer<R * NT>(lane)) pb[((vi / NT) * kCW + warp) * NT + vi % NT] = tot;
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&emptyP[s]);
      mbar_arrive(&pfull[m & 1]);
    }
    // The round's publisher (the role rotates, so each warp pays the release below at most
    // once every kCW rounds): a = silu(g) * u of the chunk's rows, then the expert's counter.
    if (warp == m % kCW) {
      mbar_wait(&pfull[m & 1], (m >> 1) & 1, abort_flag, err);
      float* ap = a.ws.a_u + (size_t)u * 2 * I + t0;
#pragma unroll
      for (int p = 0; p < kPS; ++p)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const int w = lane & 15;
          float val = (w < kCW) ? pb[(((lane >> 4) * kPS + p) * kCW + w) * NT + t] : 0.f;
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) val += __shfl_xor_sync(0xffffffffu, val, o);
          const float gs = __shfl_sync(0xffffffffu, val, 0), us = __shfl_sync(0xffffffffu, val, 16);
          if (lane == 0) ap[(size_t)t * I + p] = gs / (1.0f + expf(-gs)) * us;
        }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&pfree[m & 1]);  // the partials are read (the values are in registers)
        red_release_add(&a.ws.ecnt[u], (unsigned)kPS);
      }
    }
    while (nu < U && down_round(nu, cpe, G) <= m) consume_down(nu++);
  }
  while (nu < U) consume_down(nu++);

  // out = bf16(h + sum over the union of gate * W_down . a)
  {
    float v[kRPW * NT];
#pragma unroll
    for (int i = 0; i < kRPW; ++i)
#pragma unroll
      for (int t = 0; t < NT; ++t) v[i * NT + t] = acc[i][t];
    const float tot = warp_reduce_multi<kRPW * NT>(v, lane);
    const int vi = multi_index<kRPW * NT>(lane), i = vi / NT, t = vi % NT, rl = warp + kCW * i;
    if (multi_writer<kRPW * NT>(lane) && rl < nrows && t < B) {
      const __nv_bfloat16 bv = __float2bfloat16_rn(hs[rl * NT + t] + tot);
      a.out[(size_t)t * d + i0 + rl] = *reinterpret_cast<const uint16_t*>(&bv);
    }
  }
  csync();
  if (tid == 0) {  // the last CTA out clears the counters for the next launch
    if (atomicAdd(&a.ws.counters[kCntLayerExit], 1u) == (unsigned)G - 1) {
      for (int u = 0; u < U; ++u) a.ws.ecnt[u] = 0;
      a.ws.counters[kCntLayer] = 0;
      a.ws.counters[kCntLayerExit] = 0;
      __threadfence();
    }
  }
}

// =============================================================================
// Host side
// =============================================================================
bool plan_layer2(LayerArgs& a, int G, size_t optin) {
  if (a.B < 1 || a.B > 2 || a.k > 32 || a.E > 1024 || a.I % 32 || a.I / 32 > 16) return false;
  if ((long long)a.d > 8LL * 32 * kCPLf * kCW || (long long)a.d_o > 8LL * 32 * kCPLf * kCW) return false;
  const int NT = a.B;
  const size_t budget = optin - 256;
  KTune& o = a.k1;
  KTune& p = a.k3;
  KTune& dn = a.k4;
  const size_t orow = (size_t)a.d_o * 2;
  o.rows_max = (a.d + G - 1) / G;
  // rows per CTA: at most kRPW per consumer warp, and inside one 64-column W_r box from x0
  if (o.rows_max > kRPW * kCW || o.rows_max > 57) return false;
  o.rows_per_stage = (int)std::max<size_t>(1, std::min<size_t>(32768 / orow, (size_t)o.rows_max));
  p.rows_per_stage = kPS;
  dn.rows_max = o.rows_max;
  // stage sizes and everything outside the ring region, from a layout with the rings empty
  o.stages = p.stages = dn.stages = 0;
  const Smem2 L0 = smem2(NT, a);
  const size_t fixed = L0.total;  // region 0
  if (fixed >= budget) return false;
  const size_t cap = budget - fixed;
  o.stages = (int)std::min<size_t>(kMaxStages, cap / L0.so_b);
  if (o.stages < 2 || (a.E + kRBox - 1) / kRBox > o.stages) return false;  // every W_r box resident at once
  dn.stages = 3;
  if ((size_t)dn.stages * L0.sd_b >= cap) return false;
  p.stages = (int)std::min<size_t>(kMaxStages, (cap - (size_t)dn.stages * L0.sd_b) / L0.sp_b);
  if (p.stages < 2) return false;
  const Smem2 L = smem2(NT, a);
  o.smem = L.total;
  p.smem = dn.smem = o.smem;
  return o.smem <= budget;
}

bool layer2_ok(const LayerArgs& a0, size_t optin) {
  LayerArgs a = a0;
  CUtensorMap probe;
  return plan_layer2(a, 148, optin) &&
         make_map_2d(&probe, a.w_r ? a.w_r : reinterpret_cast<const uint16_t*>(256), (uint64_t)a.d, (uint64_t)a.E,
                     64, kRBox);
}

namespace {

template <typename Kern>
cudaError_t launch_coop(Kern k, int grid, size_t smem, cudaStream_t s, bool pdl, const CUtensorMap& tmR,
                        const LayerArgs& a) {
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
  attr[n].id = cudaLaunchAttributeCooperative;  // CTAs wait on one another: all must be resident
  attr[n].val.cooperative = 1;
  ++n;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, k, tmR, a);
}

template <int NT, int CPLX>
cudaError_t launch_by_epl(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, const CUtensorMap& tmR) {
  const int epl = a.I / 32;
  if (epl == 4) return launch_coop(k_layer2<NT, CPLX, 4>, grid, a.k1.smem, s, pdl, tmR, a);
  if (epl == 8) return launch_coop(k_layer2<NT, CPLX, 8>, grid, a.k1.smem, s, pdl, tmR, a);
  return launch_coop(k_layer2<NT, CPLX, 0>, grid, a.k1.smem, s, pdl, tmR, a);
}

}  // namespace

cudaError_t launch_layer2(const LayerArgs& a0, int grid, cudaStream_t s, bool pdl, size_t optin) {
  LayerArgs a = a0;
  if (!plan_layer2(a, grid, optin)) return cudaErrorInvalidConfiguration;
  CUtensorMap tmR;  // W_r [E][d]: boxes of 64 columns x kRBox experts
  if (!make_map_2d(&tmR, a.w_r, (uint64_t)a.d, (uint64_t)a.E, 64, kRBox)) return cudaErrorInvalidValue;
  const bool small_x = a.d <= 8 * 32 * 2 * kCW;  // two 8-element chunks per lane cover d
  if (a.B == 1)
    return small_x ? launch_by_epl<1, 2>(a, grid, s, pdl, tmR) : launch_by_epl<1, 3>(a, grid, s, pdl, tmR);
  return small_x ? launch_by_epl<2, 2>(a, grid, s, pdl, tmR) : launch_by_epl<2, 3>(a, grid, s, pdl, tmR);
}

cudaError_t set_layer2_attributes(size_t optin) {
  const int v = (int)optin;
  cudaError_t e = cudaSuccess;
#define SET2(...)                                                                                              \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(__VA_ARGS__, cudaFuncAttributeMaxDynamicSharedMemorySize, v); \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(__VA_ARGS__, cudaFuncAttributePreferredSharedMemoryCarveout, 100)
  SET2(k_layer2<1, 2, 4>);
  SET2(k_layer2<1, 2, 8>);
  SET2(k_layer2<1, 2, 0>);
  SET2(k_layer2<1, 3, 4>);
  SET2(k_layer2<1, 3, 8>);
  SET2(k_layer2<1, 3, 0>);
  SET2(k_layer2<2, 2, 4>);
  SET2(k_layer2<2, 2, 8>);
  SET2(k_layer2<2, 2, 0>);
  SET2(k_layer2<2, 3, 4>);
  SET2(k_layer2<2, 3, 8>);
  SET2(k_layer2<2, 3, 0>);
#undef SET2
  return e;
}

}  // namespace moe
