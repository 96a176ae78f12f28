// Expert kernels of the large-batch path (above batch 4, or batch x top-k > 64): whole weight
// rows streamed by TMA, tokens grouped per expert.
//
// At those batches the union of selected experts holds 10^4..10^5 independent weight rows
// (224 experts x 512 gate/up rows at batch 16 with I = 256), far more than the 148 SMs
// need, so the rows are not split along K: every row is one contiguous bulk copy and every
// dot product is finished inside one CTA, with no partial sums in global memory.  Each
// expert's tokens (about 1.1-1.7 per expert under uniform routing) are taken up to four at a
// time against the row staged in shared memory (their x held in registers, so an expert with
// at most four tokens loads x once).
//
//   k_gateup_rows  a[entry][p] = silu(W_g[e][p] . x_t) * (W_u[e][p] . x_t) for every entry
//                  (expert e, token t): the (expert, row) pairs of the union are split evenly
//                  over the CTAs; a stage is up to PS gate rows and the matching up rows.
//   k_down_rows    out[t][i] = bf16(h[t][i] + sum_entries gate * W_down[e][i] . a[entry]):
//                  CTA c owns output rows [i0, i1); a stage holds those rows of EPS union
//                  experts; per-(row, token) sums accumulate in shared memory in ascending
//                  expert order.
//
// Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted
// kernels", section "How the specialised decode path works" (separate kernels above batch
// two; 16 of 896 experts per token).
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "rowdot.cuh"

namespace moe {

namespace {

constexpr int kGateUpChunk = 4;  // pairs per gate/up chunk: stages of four whole rows

// Down-kernel experts per stage for EPL elements per lane (registers bound it).
__host__ __device__ constexpr int down_experts_per_stage(int epl) { return epl == 4 ? 4 : (epl == 8 ? 2 : 1); }

__device__ __forceinline__ int clamp_expert(int e, int E, uint32_t* err) {
  if (e < 0 || e >= E) {
    atomicOr(err, kErrBounds);
    return 0;
  }
  return e;
}

}  // namespace

// Routing tables of the union in shared memory: CSR offsets and the token of every entry
// (and, for the down kernel, its gate), loaded once per CTA after the dependency wait.
struct SmemTables {
  int* uoff;    // [U + 1]
  int* etok;    // [n_ent]
  float* egate; // [n_ent] or null
};

__device__ __forceinline__ void load_tables(const LayerArgs& a, int U, int n_ent, SmemTables tb, int tid, int nth) {
  for (int z = tid; z <= U; z += nth) tb.uoff[z] = ld_act_i(&a.ws.union_off[z]);
  for (int z = tid; z < n_ent; z += nth) {
    int t = ld_act_i(&a.ws.entry_tok[z]);
    if (t < 0 || t >= a.B) {
      atomicOr(a.ws.err, kErrBounds);
      t = 0;
    }
    tb.etok[z] = t;
    if (tb.egate) {
      int slot = ld_act_i(&a.ws.entry_slot[z]);
      if (slot < 0 || slot >= a.k) {
        atomicOr(a.ws.err, kErrBounds);
        slot = 0;
      }
      tb.egate[z] = ld_act(&a.ws.topk_gate[t * a.k + slot]);
    }
  }
}

// =============================================================================
// gate/up + SiLU*mul (large-batch path)
//   The CTA's pairs are taken in chunks of up to PC consecutive pairs of one expert; a chunk
//   is two stages, its PC gate rows and then its PC up rows, each one contiguous bulk copy
//   (fewer, larger copies stream faster).  The partial sums of a chunk are reduced once its
//   up stage is done.
// =============================================================================
// CPL: 8-element chunks of x per lane (2 covers d <= 7680: the unused third chunk of a wider
// template would cost a third more unpack and FMA instructions on zeros).
template <int NT, int CPL>
__global__ void __launch_bounds__(kThreadsS, 1) k_gateup_rows(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  static_assert(NT == 2 || NT == 4, "token groups of two or four");
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, I = a.I, E = a.E, B = a.B;
  const int SA = a.k3.stages, PC = a.k3.rows_per_stage;
  const int n_ent = B * a.k;
  const uint32_t row_bytes = (uint32_t)d * 2u;
  const size_t SA_B = al128((size_t)PC * row_bytes);
  const size_t part_f = (size_t)2 * PC * B * kCW;  // floats of one partial buffer

  unsigned char* ring = smem;
  float* part = reinterpret_cast<float*>(ring + (size_t)SA * SA_B);  // [2][2 PC][B][kCW]
  SmemTables tb;
  tb.uoff = reinterpret_cast<int*>(part + 2 * part_f);             // [E + 1]
  tb.etok = tb.uoff + (E + 1);                                      // [n_ent]
  tb.egate = nullptr;
  uint64_t* full = reinterpret_cast<uint64_t*>(
      smem + al128(static_cast<size_t>(reinterpret_cast<unsigned char*>(tb.etok + n_ent) - smem)));
  uint64_t* empty = full + kMaxStages;
  int* s_misc = reinterpret_cast<int*>(empty + kMaxStages);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(full, empty, SA, kCW);
    s_misc[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // the routing tables and x come from the router kernel
  pdl_trigger();

  const int U = min(ld_act_i(a.ws.n_union), E);
  if (a.split_B && split_chosen(U, a.split_B, a.k)) return;  // the four-token kernels take this step
  long long q0l, q1l;
  split_range((long long)U * I, G, c, q0l, q1l);
  const int q0 = (int)q0l, q1 = (int)q1l;

  if (warp == kCW) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0, u = q0 / I, p = q0 - (q0 / I) * I;
      int e = (q0 < q1) ? clamp_expert(ld_act_i(&a.ws.union_e[u]), E, a.ws.err) : 0;
      bool ok = true;
      for (int q = q0; q < q1 && ok;) {
        const int np = min(min(PC, I - p), q1 - q);
        for (int gu = 0; gu < 2; ++gu, ++it) {  // the chunk's gate rows, then its up rows
          if (!ring_acquire(empty, it, SA, abort_flag, a.ws.err)) {
            ok = false;
            break;
          }
          const int s = it % SA;
          mbar_arrive_expect_tx(&full[s], np * row_bytes);
          bulk_g2s(ring + s * SA_B, a.w_gu + ((size_t)e * 2 * I + (size_t)gu * I + p) * d, np * row_bytes,
                   &full[s], pol);
        }
        q += np;
        p += np;
        if (p == I) {
          p = 0;
          ++u;
          if (q < q1) e = clamp_expert(ld_act_i(&a.ws.union_e[u]), E, a.ws.err);
        }
      }
      ring_drain(full, it, SA, a.ws.err);
    }
    return;
  }

  load_tables(a, U, n_ent, tb, tid, kCT);
  csync();

  const int qbase = (d / 8) * warp / kCW, qpw = (d / 8) * (warp + 1) / kCW - qbase;
  float xr[NT][CPL][8];
  int cached_u = -1, cached_g = -1;
  int it = 0, ch = 0, u = q0 / I, p = q0 - (q0 / I) * I;
  for (int q = q0; q < q1; ++ch) {
    const int np = min(min(PC, I - p), q1 - q);
    const int off = tb.uoff[u];
    const int m = min(tb.uoff[u + 1] - off, B);
    float* pb = part + (size_t)(ch & 1) * part_f;
    const int ng = (m + NT - 1) / NT;  // token groups of this expert
    for (int gu = 0; gu < 2; ++gu, ++it) {
      const int s = it % SA;
      bool waited = false;
      // Groups in serpentine order (reversed on every other stage), so each stage starts
      // with the group whose x the previous stage left in registers: ng - 1 reloads per
      // stage instead of ng.
      for (int gi = 0; gi < ng; ++gi) {
        const int g0 = ((it & 1) ? ng - 1 - gi : gi) * NT;
        if (u != cached_u || g0 != cached_g) {  // x of this group's tokens, in registers
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const int tok = (g0 + t < m) ? tb.etok[off + g0 + t] : -1;
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
              if (tok >= 0 && cvalid(qpw, j, lane)) {
                const float* xp = a.ws.x + (size_t)tok * d + (size_t)(qbase + j * 32 + lane) * 8;
                const float4 x0 = ld_act4(xp), x1 = ld_act4(xp + 4);
                xr[t][j][0] = x0.x; xr[t][j][1] = x0.y; xr[t][j][2] = x0.z; xr[t][j][3] = x0.w;
                xr[t][j][4] = x1.x; xr[t][j][5] = x1.y; xr[t][j][6] = x1.z; xr[t][j][7] = x1.w;
              } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) xr[t][j][e] = 0.f;
              }
            }
          }
          cached_u = u;
          cached_g = g0;
        }
        if (!waited) {
          mbar_wait(&full[s], (it / SA) & 1, abort_flag, a.ws.err);
          waited = true;
        }
        const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + s * SA_B);
        const int mg = min(NT, m - g0);  // tokens of this group
        if (mg == 1) {  // a single token: four rows per pass
          const float(&x1)[1][CPL][8] = reinterpret_cast<const float(&)[1][CPL][8]>(xr[0]);
          for (int i0 = 0; i0 < np; i0 += 4) {
            const uint16_t* rp[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) rp[k] = st + (size_t)min(i0 + k, np - 1) * d;
            float v[4];
            rows_dot<1, 4>(rp, np - i0, x1, qbase, qpw, lane, v);
            const float tot = warp_reduce_multi<4>(v, lane);
            const int i = i0 + multi_index<4>(lane);
            if (multi_writer<4>(lane) && i < np) pb[((size_t)(gu * PC + i) * B + g0) * kCW + warp] = tot;
          }
          continue;
        }
        if (NT == 2 || mg == 2) {  // two tokens: two rows per pass
          const float(&x2)[2][CPL][8] = reinterpret_cast<const float(&)[2][CPL][8]>(xr[0]);
          for (int i0 = 0; i0 < np; i0 += 2) {
            const uint16_t* rp[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) rp[k] = st + (size_t)min(i0 + k, np - 1) * d;
            float v[4];
            rows_dot<2, 2>(rp, np - i0, x2, qbase, qpw, lane, v);
            const float tot = warp_reduce_multi<4>(v, lane);
            const int vi = multi_index<4>(lane), i = i0 + vi / 2, t = vi % 2;
            if (multi_writer<4>(lane) && i < np && g0 + t < m)
              pb[((size_t)(gu * PC + i) * B + g0 + t) * kCW + warp] = tot;
          }
          continue;
        }
        if constexpr (NT >= 4) {  // three or four tokens against each row: one unpack per chunk
          for (int i0 = 0; i0 < np; i0 += 2) {
            const uint16_t* rp[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) rp[k] = st + (size_t)min(i0 + k, np - 1) * d;
            float v[2 * NT];
            rows_dot<NT, 2>(rp, np - i0, xr, qbase, qpw, lane, v);
            const float tot = warp_reduce_multi<2 * NT>(v, lane);
            const int vi = multi_index<2 * NT>(lane), i = i0 + vi / NT, t = vi % NT;
            if (multi_writer<2 * NT>(lane) && i < np && g0 + t < m)
              pb[((size_t)(gu * PC + i) * B + g0 + t) * kCW + warp] = tot;
          }
        }
      }
      if (!waited) mbar_wait(&full[s], (it / SA) & 1, abort_flag, a.ws.err);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    csync();  // every warp's partials of this chunk are in pb (the other buffer is the next chunk's)
    // one warp per (pair, token): lanes 0..14 hold the gate partials, 16..30 the up partials
    for (int z = warp; z < np * m; z += kCW) {
      const int pi = z / m, t = z - pi * m, w = lane & 15;
      float v = (w < kCW) ? pb[((size_t)((lane >> 4) * PC + pi) * B + t) * kCW + w] : 0.f;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      const float gs = __shfl_sync(0xffffffffu, v, 0), us = __shfl_sync(0xffffffffu, v, 16);
      if (lane == 0) a.ws.a[(size_t)(off + t) * I + p + pi] = gs / (1.0f + expf(-gs)) * us;
    }
    q += np;
    p += np;
    if (p == I) {
      p = 0;
      ++u;
    }
  }
}

// =============================================================================
// down + gate-weighted combine (large-batch path)
//   A stage holds EPS experts' blocks of this CTA's rows plus the activations a of their
//   entries (one more bulk copy: the entries of consecutive experts are contiguous), up to
//   kAEnt entries; entries past that are read from L2.
// =============================================================================
template <int EPL>
__global__ void __launch_bounds__(kThreadsS, 1) k_down_rows(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kRPW = 4;  // rows per warp (rows_max <= 60)
  constexpr int kEPS = down_experts_per_stage(EPL);
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, I = a.I, E = a.E, B = a.B;
  const int S = a.k4.stages, RM = a.k4.rows_max, AE = a.k4.tok_group;  // a rows per stage
  const int n_ent = B * a.k;
  const uint32_t drow_bytes = (uint32_t)I * 2u;
  const size_t SW = al128((size_t)kEPS * RM * drow_bytes), SB = SW + al128((size_t)AE * I * sizeof(float));
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int i0 = (int)lo, nrows = (int)(hi - lo);

  unsigned char* ring = smem;
  float* acc_s = reinterpret_cast<float*>(ring + (size_t)S * SB);  // [RM][B]
  SmemTables tb;
  tb.uoff = reinterpret_cast<int*>(acc_s + (size_t)RM * B);        // [E + 1]
  tb.etok = tb.uoff + (E + 1);                                      // [n_ent]
  tb.egate = reinterpret_cast<float*>(tb.etok + n_ent);             // [n_ent]
  uint64_t* full = reinterpret_cast<uint64_t*>(
      smem + al128(static_cast<size_t>(reinterpret_cast<unsigned char*>(tb.egate + n_ent) - smem)));
  uint64_t* empty = full + kMaxStages;
  int* s_misc = reinterpret_cast<int*>(empty + kMaxStages);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(full, empty, S, kCW);
    s_misc[0] = 0;
    fence_barrier_init();
  }
  for (int z = tid; z < RM * B; z += blockDim.x) acc_s[z] = 0.f;
  __syncthreads();
  pdl_wait();  // routing tables, gates and a come from earlier kernels
  pdl_trigger();
  const int U = min(ld_act_i(a.ws.n_union), E);
  if (a.split_B && split_chosen(U, a.split_B, a.k)) return;  // the four-token kernels take this step

  if (warp == kCW) {
    if (lane == 0 && nrows > 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t blk = (uint32_t)nrows * drow_bytes;
      int jt = 0;
      for (int u0 = 0; u0 < U; u0 += kEPS, ++jt) {
        const int ne = min(kEPS, U - u0);
        const int en0 = ld_act_i(&a.ws.union_off[u0]), en1 = ld_act_i(&a.ws.union_off[u0 + ne]);
        const int na = max(0, min(en1 - en0, AE));
        if (!ring_acquire(empty, jt, S, abort_flag, a.ws.err)) break;
        const int s = jt % S;
        mbar_arrive_expect_tx(&full[s], ne * blk + (uint32_t)na * I * 4u);
        for (int e = 0; e < ne; ++e) {
          const int ex = clamp_expert(ld_act_i(&a.ws.union_e[u0 + e]), E, a.ws.err);
          bulk_g2s(ring + s * SB + (size_t)e * blk, a.w_down + ((size_t)ex * d + i0) * I, blk, &full[s], pol);
        }
        if (na > 0)
          bulk_g2s(ring + s * SB + SW, a.ws.a + (size_t)en0 * I, (uint32_t)na * I * 4u, &full[s], policy_evict_last());
      }
      ring_drain(full, jt, S, a.ws.err);
    }
    return;
  }

  load_tables(a, U, n_ent, tb, tid, kCT);
  csync();

  const int epl = (EPL > 0) ? EPL : I / 32;
  using WT = typename std::conditional<EPL == 4, uint2, uint4>::type;
  int g = 0;
  for (int u0 = 0; u0 < U && nrows > 0; u0 += kEPS, ++g) {
    const int s = g % S, ne = min(kEPS, U - u0);
    const int en0 = tb.uoff[u0], en1 = tb.uoff[u0 + ne];
    mbar_wait(&full[s], (g / S) & 1, abort_flag, a.ws.err);
    const uint16_t* st = reinterpret_cast<const uint16_t*>(ring + s * SB);
    const float* as = reinterpret_cast<const float*>(ring + s * SB + SW);
    int e_loc = 0;
    for (int en = en0; en < en1; ++en) {
      while (e_loc + 1 < ne && en >= tb.uoff[u0 + e_loc + 1]) ++e_loc;
      const int t = tb.etok[en];
      const float gate = tb.egate[en];
      const bool staged = en - en0 < AE;
      const float* ap = staged ? as + (size_t)(en - en0) * I + lane * epl : a.ws.a + (size_t)en * I + lane * epl;
      float v[kRPW];
      if constexpr (EPL == 4 || EPL == 8) {
        float av[EPL];
#pragma unroll
        for (int x = 0; x < EPL; x += 4) {
          const float4 f = staged ? *reinterpret_cast<const float4*>(ap + x) : ld_act4(ap + x);
          av[x] = f.x; av[x + 1] = f.y; av[x + 2] = f.z; av[x + 3] = f.w;
        }
#pragma unroll
        for (int i = 0; i < kRPW; ++i) {
          const int rl = warp + kCW * i;
          WT w{};
          if (rl < nrows) w = *reinterpret_cast<const WT*>(st + ((size_t)e_loc * nrows + rl) * I + lane * EPL);
          float wf[8];
          if constexpr (EPL == 4) {
            wf[0] = bf16lo(w.x); wf[1] = bf16hi(w.x); wf[2] = bf16lo(w.y); wf[3] = bf16hi(w.y);
          } else {
            unpack8f(reinterpret_cast<const uint4&>(w), wf);
          }
          float sdot = 0.f;
#pragma unroll
          for (int x = 0; x < EPL; ++x) sdot = fmaf(wf[x], av[x], sdot);
          v[i] = sdot;
        }
      } else {
#pragma unroll
        for (int i = 0; i < kRPW; ++i) {
          const int rl = warp + kCW * i;
          float sdot = 0.f;
          if (rl < nrows) {
            const uint16_t* wr = st + ((size_t)e_loc * nrows + rl) * I + lane * epl;
#pragma unroll
            for (int x = 0; x < 16; ++x)
              if (x < epl) sdot = fmaf(bf16f(wr[x]), staged ? ap[x] : ld_act(ap + x), sdot);
          }
          v[i] = sdot;
        }
      }
      const float tot = warp_reduce_multi<kRPW>(v, lane);
      const int i = multi_index<kRPW>(lane), rl = warp + kCW * i;
      if (multi_writer<kRPW>(lane) && rl < nrows) acc_s[rl * B + t] += gate * tot;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  csync();
  for (int z = tid; z < nrows * B; z += kCT) {
    const int r = z / B, t = z - r * B;
    const size_t o = (size_t)t * d + i0 + r;
    const __nv_bfloat16 bv = __float2bfloat16_rn(ld_act(&a.ws.h[o]) + acc_s[r * B + t]);
    a.out[o] = *reinterpret_cast<const uint16_t*>(&bv);
  }
}

// =============================================================================
// Host side
// =============================================================================
namespace {

template <typename Kern>
cudaError_t launch_l(Kern k, int grid, size_t smem, cudaStream_t s, bool pdl, const LayerArgs& a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreadsS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, a);
}

size_t up128h(size_t x) { return (x + 127) & ~size_t(127); }

}  // namespace

bool plan_large(LayerArgs& a, int G, size_t optin) {
  const size_t budget = optin - 1024;
  const size_t bars = 2 * kMaxStages * 8 + 64;
  {  // gate/up: chunks of up to PC pairs, two one-copy stages (gate rows, up rows) per chunk
    KTune& t = a.k3;
    t.rows_per_stage = kGateUpChunk;
    const size_t SA_B = up128h((size_t)t.rows_per_stage * a.d * 2);
    const size_t part = (size_t)2 * 2 * t.rows_per_stage * a.B * kCW * sizeof(float);
    const size_t extra = up128h(part + (size_t)(a.E + 1 + a.B * a.k) * sizeof(int)) + bars;
    t.stages = (budget > extra) ? (int)std::min<size_t>(kMaxStages, (budget - extra) / SA_B) : 0;
    if (t.stages < 2) return false;
    t.smem = (size_t)t.stages * SA_B + extra;
  }
  {  // down: EPS experts' blocks of this CTA's rows per stage
    KTune& t = a.k4;
    t.rows_max = (a.d + G - 1) / G;
    if (t.rows_max > 4 * kCW || a.I / 32 > 16) return false;
    const int eps = down_experts_per_stage(a.I / 32);
    t.rows_per_stage = eps;
    t.tok_group = std::min(a.B * a.k, eps * 8);  // a rows staged per stage
    const size_t SB = up128h((size_t)eps * t.rows_max * a.I * 2) + up128h((size_t)t.tok_group * a.I * sizeof(float));
    const size_t extra = up128h((size_t)t.rows_max * a.B * sizeof(float) + (size_t)(a.E + 1) * sizeof(int) +
                                (size_t)a.B * a.k * (sizeof(int) + sizeof(float))) + bars;
    t.stages = (budget > extra) ? (int)std::min<size_t>(kMaxStages, (budget - extra) / SB) : 0;
    if (t.stages < 2) return false;
    t.smem = (size_t)t.stages * SB + extra;
  }
  return a.d <= 8 * 32 * kCPLf * kCW;
}

cudaError_t set_large_attributes(size_t optin) {
  const int v = (int)optin;
  cudaError_t e = cudaSuccess;
#define SETL(k)                                                                                         \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, v); \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100)
  SETL((k_gateup_rows<4, 2>));
  SETL((k_gateup_rows<2, 3>));
  SETL(k_down_rows<4>);
  SETL(k_down_rows<8>);
  SETL(k_down_rows<0>);
#undef SETL
  return e;
}

cudaError_t launch_gateup_rows(const LayerArgs& a0, int grid, cudaStream_t s, bool pdl, size_t optin) {
  LayerArgs a = a0;
  plan_large(a, grid, optin);
  // x of up to four tokens in registers where two chunks per lane cover d (an expert's tokens
  // rarely exceed four at batch <= 64); pairs of tokens where three chunks are needed
  return a.d <= 8 * 32 * 2 * kCW ? launch_l(k_gateup_rows<4, 2>, grid, a.k3.smem, s, pdl, a)
                                 : launch_l(k_gateup_rows<2, 3>, grid, a.k3.smem, s, pdl, a);
}

cudaError_t launch_down_rows(const LayerArgs& a0, int grid, cudaStream_t s, bool pdl, size_t optin) {
  LayerArgs a = a0;
  plan_large(a, grid, optin);
  const int epl = a.I / 32;
  if (epl == 4) return launch_l(k_down_rows<4>, grid, a.k4.smem, s, pdl, a);
  if (epl == 8) return launch_l(k_down_rows<8>, grid, a.k4.smem, s, pdl, a);
  return launch_l(k_down_rows<0>, grid, a.k4.smem, s, pdl, a);
}

}  // namespace moe
