// sm_100a kernels of one MoE decode-layer step.
//
// Large-batch kernels (the small-batch path and the router are in kernels_small.cu):
//   K1 k_oproj           h = residual + W_o . attn_out on the tensor cores (weights as the
//                        MMA's N operand, staged through a shared-memory ring by TMA bulk
//                        copies), tokens in groups of up to 8, per-CTA sums of h^2.
//   K3 k_gateup_splitk   split-K expert gate/up for batches above two: (expert, K chunk) units
//                        whose partial sums are reduced in chunk order by the last unit of
//                        each expert (atomic ticket per expert, no spinning).
//   K4 k_down_combine    out = bf16(h + sum_j gate_j * W_down[e_j] . a_j): rows of d split over
//                        CTAs, experts streamed in ascending order, fixed reduction order.
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
  // K2 (router, kernels_small.cu): rows of W_r per CTA.
  a.k2.rows_max = (a.E + G - 1) / G;
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
  return a.k1.smem <= budget && a.k3.smem <= budget && a.k4.smem <= budget;
}

cudaError_t set_kernel_attributes(size_t optin) {
  const int v = (int)optin;
  cudaError_t e = cudaSuccess;
#define SET(k)                                                                              \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, v); \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100)
  SET(k_oproj);
  SET(k_gateup_splitk<2>);
  SET(k_down_combine<0>);
#undef SET
  return e;
}

cudaError_t launch_oproj(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_k(k_oproj, grid, a.k1.smem, s, pdl, a);
}

cudaError_t launch_gateup_splitk(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_k(k_gateup_splitk<2>, grid, a.k3.smem, s, pdl, a);
}

cudaError_t launch_down(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_k(k_down_combine<0>, grid, a.k4.smem, s, pdl, a);
}

}  // namespace moe
