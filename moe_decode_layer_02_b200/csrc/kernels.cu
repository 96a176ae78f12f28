// sm_100a kernels of one MoE decode-layer step.
//
// The fallback large-batch o_proj, used on the large-batch path where the TMA tensor maps of
// k_oproj_tc (kernels_tc.cu) cannot be encoded (the small-batch kernels and the router are
// in kernels_small.cu, the large-batch expert kernels in kernels_large.cu):
//   K1 k_oproj           h = residual + W_o . attn_out on the tensor cores (weights as the
//                        MMA's N operand, staged through a shared-memory ring by TMA bulk
//                        copies), tokens in groups of up to 8, per-CTA sums of h^2.
//
// Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted
// kernels", section "How the specialised decode path works" (kernels chosen by batch size;
// o_proj fused with the residual step).
//
// Structure: one CTA per SM, 8 consumer warps and one producer warp.  The producer's lane 0 streams weight rows into a shared-memory ring with
// TMA bulk copies (cp.async.bulk, mbarrier transaction counts, L2 evict-first); the
// consumers multiply and reduce in a fixed order, so every result is bit-reproducible.
#include <algorithm>

#include "common.cuh"
#include "gemv_mma.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

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
  const int maxB = a.B;  // shared memory is planned for the batch being launched
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
  return a.k1.smem <= budget;
}

cudaError_t set_kernel_attributes(size_t optin) {
  const int v = (int)optin;
  cudaError_t e = cudaSuccess;
#define SET(k)                                                                              \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, v); \
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100)
  SET(k_oproj);
#undef SET
  return e;
}

cudaError_t launch_oproj(const LayerArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_k(k_oproj, grid, a.k1.smem, s, pdl, a);
}

}  // namespace moe
