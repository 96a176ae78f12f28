// The router of the large-batch path with K split over the CTAs (one cooperative launch per layer).
//
// logits[t][e] = sum_i W_r[e][i] x[t][i] with x = h * rstd * gamma, so
// logits[t][e] = rstd[t] * sum_i W_r[e][i] (h[t][i] gamma[i]).  CTA c owns the same d-rows
// [r0, r1) as in o_proj (at most 49) and needs only that slice of h for every token (12 KB
// at batch 64, from L2) and the matching columns of W_r for every expert:
//   1. the producer brings W_r[:, x0 .. x0 + 64) with x0 = r0 rounded down to 8 (a 2-D tensor
//      map, boxes of 224 experts x 64 columns, 128-byte swizzle; columns outside [r0, r1) meet
//      zeros below), issued before the dependency wait since W_r is static;
//   2. consumers stage the o_proj CTAs' sums of h^2 in shared memory (one coalesced pass) and
//      compute rstd of every token from them (the same fixed-order sum as every other kernel),
//      write x for their slice, and place h * gamma of the slice, split into three bf16 terms
//      hi + mid + lo (together within 2^-26 of the fp32 value; two terms leave 2^-18, which
//      over d = 8192 columns moves a logit by ~1e-5), in three swizzled tiles;
//   3. the tensor cores (mma.sync m16n8k16, experts as M, tokens as N; each term's 16-column
//      product in a fresh accumulator, summed in fp32 on the CUDA cores so that the tensor
//      core's own accumulation never carries a long sum) give the CTA's partial logits of
//      every expert and token, stored to a per-CTA slab;
//   4. grid barrier; CTA c sums its 6-7 experts' partials over the CTAs in a fixed order and
//      scales by rstd (the logits);
//   5. grid barrier; CTA t (t < B) selects token t's top-k and gates; the last CTA to finish
//      builds the routing tables (union of experts, CSR entries) for the expert kernels.
// The per-CTA partials cross L2 once (G x E x B floats), instead of every CTA reading every
// token's h as a split over the experts does.
//
// Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted kernels",
// section "How the specialised decode path works" (router over 896 experts, top 16; separate
// kernels above batch two); the router accumulates in fp32 (the layer's stated configuration).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "mma.cuh"
#include "rowdot.cuh"
#include "topk.cuh"

namespace moe {

namespace {

constexpr int kRkBox = 224;                  // experts per TMA box (14 tiles of 16)
constexpr int kRkBoxBytes = kRkBox * 128;    // 64 bf16 columns per expert row
constexpr int kRkTok = 64;                   // token rows of the h tiles (B <= 64)
constexpr int kRkTileBytes = kRkTok * 128;   // one h tile (hi or lo)

__host__ __device__ inline int rk_boxes(int E) { return (E + kRkBox - 1) / kRkBox; }

constexpr int kRkSsStride = kRkTok + 1;  // floats per staged row of h^2 sums (odd: no bank conflicts)
constexpr int kRkItems = (kRkTok * 64 + kCT - 1) / kCT;  // h-tile items per consumer thread

// Shared memory: W_r boxes (also the routing-table scratch of the last CTA), h tiles, the
// staged sums of h^2 of G CTAs, rstd.
__host__ __device__ inline size_t rk_ss_bytes(int G) { return ((size_t)G * kRkSsStride * 4 + 15) & ~size_t(15); }
__host__ __device__ inline size_t rk_smem(int E, int G) {
  size_t w = (size_t)rk_boxes(E) * kRkBoxBytes;
  if (w < (size_t)kTopkScratch) w = kTopkScratch;
  w = (w + 1023) & ~size_t(1023);
  return 1024 + w + 3 * kRkTileBytes + rk_ss_bytes(G) + 64 * 4 + 64;
}

// The o_proj CTAs' sums of h^2 ([G][maxB] in global memory) of the B tokens, copied into
// shared memory rows of kRkSsStride floats by the consumer threads: consecutive threads take
// consecutive tokens of a row, and each thread has eight loads in flight at a time (sixteen
// or 24 were slower).  (Read straight from L2, one token per warp and round, every CTA asked
// for the same 148 lines once per token, and a round took about 2.5 us.)
constexpr int kRkSsRound = 8;
__device__ __forceinline__ void rk_stage_ss(const LayerArgs& a, float* s_ss, int G, int B, int tid) {
  const int n = G * B;
  for (int z0 = tid; z0 < n; z0 += kRkSsRound * kCT) {
    float v[kRkSsRound];
#pragma unroll
    for (int k = 0; k < kRkSsRound; ++k) {
      const int z = z0 + k * kCT;
      v[k] = z < n ? ld_act(&a.ws.ss_part[(size_t)(z / B) * a.maxB + z % B]) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kRkSsRound; ++k) {
      const int z = z0 + k * kCT;
      if (z < n) s_ss[(z / B) * kRkSsStride + z % B] = v[k];
    }
  }
}

// Fixed-order RMS statistics (the same sum as the other router kernels), from the staged sums.
__device__ __forceinline__ float rk_rstd(const LayerArgs& a, const float* s_ss, int t, int G, int lane) {
  float ss = 0.f;
  for (int c0 = 0; c0 < G; c0 += 8 * 32) {
    float pv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int cc = c0 + k * 32 + lane;
      pv[k] = cc < G ? s_ss[cc * kRkSsStride + t] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) ss += pv[k];
  }
  ss = warp_sum(ss);
  return 1.0f / sqrtf(ss / (float)a.d + a.eps);
}

__device__ __forceinline__ void rk_barrier(unsigned* count, unsigned target, volatile int* abort_flag,
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

}  // namespace

__global__ void __launch_bounds__(kThreadsS, 1) k_router_ks(const __grid_constant__ CUtensorMap tmR, const LayerArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, E = a.E, B = a.B, K = a.k;
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int r0 = (int)lo, rows = (int)(hi - lo), x0 = r0 & ~7;
  const int nbox = rk_boxes(E), Bp = (B + 7) & ~7;
  size_t wbytes = (size_t)nbox * kRkBoxBytes;
  if (wbytes < (size_t)kTopkScratch) wbytes = kTopkScratch;
  wbytes = (wbytes + 1023) & ~size_t(1023);
  unsigned char* wr = smem;
  unsigned char* th = smem + wbytes;       // h * gamma, bf16 hi  [64 tokens][64 columns], swizzled
  unsigned char* tm = th + kRkTileBytes;   // bf16 mid
  unsigned char* tl = tm + kRkTileBytes;   // bf16 lo
  float* s_ss = reinterpret_cast<float*>(tl + kRkTileBytes);  // [G][kRkSsStride] sums of h^2
  float* rstd_s = reinterpret_cast<float*>(tl + kRkTileBytes + rk_ss_bytes(G));
  uint64_t* bar = reinterpret_cast<uint64_t*>(rstd_s + 64);
  int* s_misc = reinterpret_cast<int*>(bar + 1);
  volatile int* abort_flag = s_misc;
  unsigned* bar_count = &a.ws.counters[kCntRouterBar];
  uint32_t* err = a.ws.err;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(bar, 1);
    s_misc[0] = 0;
    s_misc[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  if (warp == kCW) {
    if (lane == 0) {  // W_r is static: its column block is requested before the dependency wait
      mbar_arrive_expect_tx(bar, (uint32_t)nbox * kRkBoxBytes);
      for (int j = 0; j < nbox; ++j) tma_load_2d(wr + (size_t)j * kRkBoxBytes, &tmR, x0, j * kRkBox, bar);
      mbar_drain(bar, 0, err);  // no copy may be in flight when this warp moves on
    }
    __syncwarp();
  } else {
    pdl_wait();  // h and the sums of h^2 come from the o_proj kernel
    if (c == 0 && threadIdx.x == 0) a.ws.counters[kCntGateUp] = 0;  // the expert kernels' grid barrier count
    // h of this thread's items of the slice, in flight while the sums of h^2 are staged
    float hv[kRkItems];
#pragma unroll
    for (int n = 0; n < kRkItems; ++n) {
      const int z = tid + n * kCT, t = z >> 6, i = x0 + (z & 63);
      hv[n] = (z < kRkTok * 64 && t < B && i >= r0 && i < r0 + rows) ? ld_act(&a.ws.h[(size_t)t * d + i]) : 0.f;
    }
    rk_stage_ss(a, s_ss, G, B, tid);
    csync();
    for (int t = warp; t < B; t += kCW) {
      const float r = rk_rstd(a, s_ss, t, G, lane);
      if (lane == 0) {
        rstd_s[t] = r;
        if (c == 0) a.ws.rstd[t] = r;
      }
    }
    csync();
    // x of this CTA's slice, and the slice's h * gamma as bf16 hi + lo tiles (zeros outside)
#pragma unroll
    for (int n = 0; n < kRkItems; ++n) {
      const int z = tid + n * kCT;
      if (z >= kRkTok * 64) break;
      const int t = z >> 6, k = z & 63, i = x0 + k;
      float v = 0.f;
      if (t < B && i >= r0 && i < r0 + rows) {
        const float g = bf16f(a.gamma[i]);
        v = hv[n] * g;
        a.ws.x[(size_t)t * d + i] = hv[n] * rstd_s[t] * g;
      }
      const __nv_bfloat16 vh = __float2bfloat16_rn(v);
      const float r1 = v - __bfloat162float(vh);
      const __nv_bfloat16 vm = __float2bfloat16_rn(r1);
      const __nv_bfloat16 vl = __float2bfloat16_rn(r1 - __bfloat162float(vm));
      const uint32_t off = swz(t, k >> 3) + (uint32_t)(k & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(th + off) = vh;
      *reinterpret_cast<__nv_bfloat16*>(tm + off) = vm;
      *reinterpret_cast<__nv_bfloat16*>(tl + off) = vl;
    }
    csync();
    mbar_wait(bar, 0, abort_flag, err);
    // partial logits: experts as M (16-row tiles), tokens as N (pairs of 8-token tiles), K = 64
    {
      const int ai = lane >> 3;
      const int arow = ((ai & 1) << 3) + (lane & 7), achk = ai >> 1;      // A: expert +8 (i & 1), chunk +(i >> 1)
      const int brow0 = ((ai >> 1) << 3) + (lane & 7), bchk = ai & 1;     // B: token tile +(i >> 1), chunk +(i & 1)
      const int g = lane >> 2, q = lane & 3;
      const uint32_t hbase = smem_addr(th), mbase = smem_addr(tm), lbase = smem_addr(tl);
      float* P = a.ws.rpart + (size_t)c * E * Bp;
      const int nmt = (E + 15) / 16, ntp = (B + 15) / 16;
      for (int np = 0; np < ntp; ++np) {
        uint32_t bh[4][4], bm[4][4], bl[4][4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          ldsm4(bh[kk], hbase + swz(16 * np + brow0, 2 * kk + bchk));
          ldsm4(bm[kk], mbase + swz(16 * np + brow0, 2 * kk + bchk));
          ldsm4(bl[kk], lbase + swz(16 * np + brow0, 2 * kk + bchk));
        }
        for (int mt = warp; mt < nmt; mt += kCW) {
          const uint32_t wt = smem_addr(wr + (size_t)(16 * mt / kRkBox) * kRkBoxBytes);
          const int rb = (16 * mt) % kRkBox;
          float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            uint32_t af[4];
            ldsm4(af, wt + swz(rb + arow, 2 * kk + achk));
            // each term's 16-column product in a fresh accumulator, summed in fp32:
            // (hi + (mid + lo)) per k-step, k-steps in order
#pragma unroll
            for (int tile = 0; tile < 2; ++tile) {
              float ph[4] = {0.f, 0.f, 0.f, 0.f}, pm[4] = {0.f, 0.f, 0.f, 0.f}, pl[4] = {0.f, 0.f, 0.f, 0.f};
              mma16816(ph, af, bh[kk][2 * tile], bh[kk][2 * tile + 1]);
              mma16816(pm, af, bm[kk][2 * tile], bm[kk][2 * tile + 1]);
              mma16816(pl, af, bl[kk][2 * tile], bl[kk][2 * tile + 1]);
              float* dd = tile ? d1 : d0;
#pragma unroll
              for (int e = 0; e < 4; ++e) dd[e] += ph[e] + (pm[e] + pl[e]);
            }
          }
          // D: lane (g, q) holds experts 16 mt + g (+8), tokens 2q, 2q + 1 of each token tile
#pragma unroll
          for (int tile = 0; tile < 2; ++tile) {
            const int t = 16 * np + 8 * tile + 2 * q;
            if (t < Bp) {
              const float* dd = tile ? d1 : d0;
              const int e = 16 * mt + g;
              if (e < E) *reinterpret_cast<float2*>(P + (size_t)e * Bp + t) = make_float2(dd[0], dd[1]);
              if (e + 8 < E) *reinterpret_cast<float2*>(P + (size_t)(e + 8) * Bp + t) = make_float2(dd[2], dd[3]);
            }
          }
        }
      }
    }
    rk_barrier(bar_count, (unsigned)G, abort_flag, err);
    // logits of this CTA's experts: the partials summed over the CTAs, times rstd.  gl lanes
    // share an (expert, token) item (as many as the CTA's threads allow), each lane summing
    // every gl-th CTA's partial and the group adding its lanes' sums by shuffles, so that an
    // item's G loads take one or two rounds to L2 instead of G / 8 (a fixed order for a given
    // batch: the same bits on every run)
    {
      split_range(E, G, c, lo, hi);
      const int e0 = (int)lo, ne = (int)(hi - lo), items = ne * B;
      int gl = 32;
      while (gl > 1 && items * gl > kCT) gl >>= 1;
      const int ipw = 32 / gl;  // items per warp and round
      const size_t stride = (size_t)E * Bp;
      for (int base = warp * ipw; base < items; base += kCW * ipw) {
        const int z = base + lane / gl, sub = lane % gl;
        float s = 0.f;
        if (z < items) {
          const float* p = a.ws.rpart + (size_t)(e0 + z / B) * Bp + z % B;
          int cc = sub;
          for (; cc + 7 * gl < G; cc += 8 * gl) {
            float v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = ld_act(p + (size_t)(cc + k * gl) * stride);
#pragma unroll
            for (int k = 0; k < 8; ++k) s += v[k];
          }
          for (; cc < G; cc += gl) s += ld_act(p + (size_t)cc * stride);
        }
        for (int o = gl >> 1; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (z < items && sub == 0) {
          const int e = e0 + z / B, t = z % B;
          a.ws.logits[(size_t)t * E + e] = rstd_s[t] * s;
        }
      }
    }
    rk_barrier(bar_count, 2u * (unsigned)G, abort_flag, err);
    // top-k and gates of token c
    if (c < B && warp == 0) {
      float* cv = reinterpret_cast<float*>(th);  // the h tiles are no longer needed
      float my_v = 0.f;
      int my_i = 0;
      warp_topk(a.ws.logits + (size_t)c * E, E, K, cv, reinterpret_cast<int*>(cv + kCandStride), lane, my_v, my_i);
      const float gte = warp_gate(my_v, lane, K);
      if (lane < K) {
        const int e = (my_i >= 0 && my_i < E) ? my_i : 0;
        if (e != my_i) atomicOr(err, kErrBounds);
        a.ws.topk_idx[c * K + lane] = e;
        a.ws.topk_gate[c * K + lane] = gte;
        if (a.user_idx) a.user_idx[c * K + lane] = e;
        if (a.user_gate) a.user_gate[c * K + lane] = gte;
      }
    }
  }
  // the last CTA to finish builds the routing tables (its W_r boxes are its scratch now) and
  // clears the counters for the next launch
  if (last_cta_s(&a.ws.counters[kCntRouter], &s_misc[1])) {
    topk_route(a, wr, true);
    if (tid == 0) {
      a.ws.counters[kCntRouterBar] = 0;
      a.ws.counters[kCntRouter] = 0;
    }
  }
}

// =============================================================================
// Host side
// =============================================================================
bool router_ks_ok(const LayerArgs& a, int grid, size_t optin) {
  CUtensorMap probe;
  return a.B >= 1 && a.B <= kRkTok && a.E <= 1024 && a.k <= 32 && (a.d + grid - 1) / grid <= 57 &&
         rk_smem(a.E, grid) <= optin - 1024 && a.ws.rpart != nullptr &&
         make_map_2d(&probe, a.w_r ? a.w_r : reinterpret_cast<const uint16_t*>(256), (uint64_t)a.d, (uint64_t)a.E,
                     64, kRkBox);
}

cudaError_t set_router_ks_attributes(size_t optin) {
  cudaError_t e = cudaFuncSetAttribute(k_router_ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)optin);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_router_ks, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  return e;
}

cudaError_t launch_router_ks(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  CUtensorMap tmR;
  if (!make_map_2d(&tmR, a.w_r, (uint64_t)a.d, (uint64_t)a.E, 64, kRkBox)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreadsS);
  cfg.dynamicSmemBytes = rk_smem(a.E, grid);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  attr[n].id = cudaLaunchAttributeCooperative;  // grid barriers: every CTA must be resident
  attr[n].val.cooperative = 1;
  ++n;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, k_router_ks, tmR, a);
}

}  // namespace moe
