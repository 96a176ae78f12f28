// o_proj of the large-batch path on the tensor cores with TMA tensor tiles.
//
// At batch 16-64, h = residual + attn_out . W_o^T is a skinny GEMM ([B x d_o] x [d_o x d])
// that is still bound by the 117 MB of W_o.  CTA c owns output rows [r0, r1) (49 at most);
// the K dimension (d_o) is streamed 256 at a time: per stage one TMA copy of W_o (56 rows x
// four 64-wide k-blocks) and one of attn_out (B rounded up to 16 tokens x four k-blocks),
// both with the 128-byte swizzle, so W_o is read once and the activations come from L2.  8
// consumer warps run mma.sync m16n8k16 (tokens as M, weight rows as N).  The work of a stage
// is (token tile, half of the weight rows, k-block) items; with fewer than four token tiles
// the four k-blocks are split over the warps as well (each warp then sums its own k-blocks
// and the warps' partial sums are added in a fixed order at the end), so that every warp, and
// so every SM sub-partition's tensor pipe, takes an equal share: with one token tile on two
// warps the two warps' MMAs, issued on one sub-partition, were the bound of the kernel.
// ldmatrix reads both operands through the swizzle.
// The epilogue adds the residual, writes h in fp32 and the CTA's sums of h^2 per token in a
// fixed order.
//
// Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted
// kernels", section "How the specialised decode path works" (o_proj fused with the
// residual step; separate kernels by batch size).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "mma.cuh"

namespace moe {

namespace {

constexpr int kTcBK = 64;        // K of one k-block (128 bytes of bf16: one swizzle span)
constexpr int kTcKB = 4;         // k-blocks per stage: 256 of K per pair of TMA copies
constexpr int kTcRows = 56;      // weight rows per box (a CTA owns at most 49; 56 keeps tiles 1024-aligned)
constexpr int kTcTok = 64;       // most token rows per activation box
constexpr int kTcMaxStages = 8;
constexpr int kTcWTile = kTcRows * kTcBK * 2;          // 7168 bytes per weight k-block tile
constexpr int kTcAOff = kTcKB * kTcWTile;              // 28672: activation tiles follow
constexpr size_t kTcFixed = 1024 + (size_t)kTcTok * kTcRows * 4 + 2 * kTcMaxStages * 8 + 64;

// A stage holds the weight tiles and tokb activation rows per k-block, rounded up to 1 KB for
// the swizzle; as many stages as fit the shared memory keep W_o in flight (5 at 16 tokens,
// 3 at 64).
int tc_stage_bytes(int tokb) { return (kTcAOff + kTcKB * tokb * kTcBK * 2 + 1023) & ~1023; }
int tc_stages(int tokb, size_t optin) {
  const size_t room = optin > kTcFixed ? optin - kTcFixed : 0;
  return std::min<int>(kTcMaxStages, (int)(room / (size_t)tc_stage_bytes(tokb)));
}

}  // namespace

// Tensor maps view W_o [d][d_o] and attn_out [B][d_o] as 3-D {64 (k), rows, d_o / 64
// (k-block)} so one copy brings four 64-wide k-blocks of 56 weight rows (28 KB) or of the
// tokens; tokb = the activation box height (B rounded up to 16); NS stages of sb bytes each.
__global__ void __launch_bounds__(kThreads, 1)
    k_oproj_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA, const LayerArgs a,
               int tokb, int NS, int sb) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, d_o = a.d_o, B = a.B;
  long long lo, hi;
  split_range(d, G, c, lo, hi);
  const int r0 = (int)lo, rows = (int)(hi - lo);
  const int nk = (d_o + kTcKB * kTcBK - 1) / (kTcKB * kTcBK);
  const uint32_t stage_tx = (uint32_t)(kTcAOff + kTcKB * tokb * kTcBK * 2);

  unsigned char* ring = smem;                                          // [NS][sb]
  float* sq = reinterpret_cast<float*>(ring + (size_t)NS * sb);        // [kTcTok][kTcRows]
  uint64_t* full = reinterpret_cast<uint64_t*>(sq + kTcTok * kTcRows);
  uint64_t* empty = full + NS;
  int* s_misc = reinterpret_cast<int*>(empty + NS);
  volatile int* abort_flag = s_misc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (tid == 0) {
    init_ring(full, empty, NS);
    s_misc[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      // W_o is static: the first stages' weight copies go out before the dependency wait; the
      // activation copies (attn_out comes from the previous kernel) only after it.
      const int pre = nk < NS ? nk : NS;
      for (int ks = 0; ks < pre; ++ks) {
        mbar_arrive_expect_tx(&full[ks], stage_tx);
        tma_load_3d(ring + (size_t)ks * sb, &tmW, 0, r0, ks * kTcKB, &full[ks]);
      }
      pdl_wait();
      for (int ks = 0; ks < pre; ++ks)
        tma_load_3d(ring + (size_t)ks * sb + kTcAOff, &tmA, 0, 0, ks * kTcKB, &full[ks]);
      int it = pre;
      for (int ks = pre; ks < nk; ++ks, ++it) {
        if (!ring_acquire(empty, it, NS, abort_flag, a.ws.err)) break;
        const int s = it % NS;
        mbar_arrive_expect_tx(&full[s], stage_tx);
        tma_load_3d(ring + (size_t)s * sb, &tmW, 0, r0, ks * kTcKB, &full[s]);
        tma_load_3d(ring + (size_t)s * sb + kTcAOff, &tmA, 0, 0, ks * kTcKB, &full[s]);
      }
      ring_drain(full, it, NS, a.ws.err);
    }
    return;
  }

  pdl_wait();  // the residual may come from the previous kernel
  // warp -> (token tile mt, row half nh, k-block quarter kq): tokens [16 mt, +16), weight-row
  // tiles 4 nh .. 4 nh + 3, k-blocks [kq kpw, kq kpw + kpw) of every stage
  const int mtiles = tokb / 16, ksplit = mtiles == 1 ? 4 : (mtiles == 2 ? 2 : 1), kpw = kTcKB / ksplit;
  const int combo = warp / ksplit, kq = warp - combo * ksplit;
  const int mt = combo % mtiles, nh = combo / mtiles;
  const bool active = combo < 2 * mtiles && 16 * mt < B;
  float acc[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
  // ldmatrix lane roles: A (16 tokens x 16 k): matrix i = lane / 8 -> token +8 (i & 1), chunk +(i >> 1)
  const int ai = lane >> 3, arow = 16 * mt + ((ai & 1) << 3) + (lane & 7), achk = ai >> 1;
  // B (two 8-row tiles x 16 k): matrix i -> tile +(i >> 1), chunk +(i & 1)
  const int brow0 = 32 * nh + ((ai >> 1) << 3) + (lane & 7), bchk = ai & 1;
  const int ntile2 = (32 * nh + 16 < kTcRows) ? 2 : 1;  // tile pairs inside the 56-row box
  for (int ks = 0; ks < nk; ++ks) {
    const int s = ks % NS;
    mbar_wait(&full[s], (ks / NS) & 1, abort_flag, a.ws.err);
    const uint32_t wbase = smem_addr(ring + (size_t)s * sb);
    const uint32_t abase = wbase + kTcAOff;
    // each 64-wide k-block is summed by the tensor core into fresh registers (4 chained MMAs);
    // the running sums over k-blocks are fp32 adds, which round more tightly than the tensor
    // core's own accumulation of a chain as long as d_o
    auto kblock = [&](int kb) {
      const uint32_t wt = wbase + kb * kTcWTile, at = abase + (uint32_t)(kb * tokb * kTcBK * 2);
      float blk[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) blk[n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < kTcBK / 16; ++kk) {
        uint32_t af[4];
        ldsm4(af, at + swz(arow, 2 * kk + achk));
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          if (np < ntile2) {
            uint32_t bf[4];
            ldsm4(bf, wt + swz(brow0 + 16 * np, 2 * kk + bchk));
            mma16816(blk[2 * np], af, bf[0], bf[1]);
            mma16816(blk[2 * np + 1], af, bf[2], bf[3]);
          }
        }
      }
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] += blk[n][e];
    };
    if (active) {
      if (ksplit == 1) {  // all four k-blocks: unrolled, so their loads and MMAs interleave
#pragma unroll
        for (int kb = 0; kb < kTcKB; ++kb) kblock(kb);
      } else {
#pragma unroll 1
        for (int kb = kq * kpw; kb < kq * kpw + kpw; ++kb) kblock(kb);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (ksplit > 1) {  // the k-block quarters' partial sums, added in a fixed order (ring reused)
    consumer_sync();  // every stage has been read
    float* red = reinterpret_cast<float*>(ring);  // [kConsumerWarps][16][32]
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[(warp * 16 + n * 4 + e) * 32 + lane] = acc[n][e];
    consumer_sync();
    if (kq == 0) {
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = 0.f;
          for (int j = 0; j < ksplit; ++j) v += red[((warp + j) * 16 + n * 4 + e) * 32 + lane];
          acc[n][e] = v;
        }
    }
  }
  // epilogue: D fragment of tile n: lane (g, q) holds tokens 16 mt + g (+8), rows 8 n' + 2q (+1)
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    const int nrow = 32 * nh + 8 * n + 2 * q;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = 16 * mt + g + ((e >> 1) << 3), rr = nrow + (e & 1);
      if (active && kq == 0 && t < B && rr < rows) {
        const size_t o = (size_t)t * d + r0 + rr;
        const float hv = bf16f(__ldcg(reinterpret_cast<const unsigned short*>(a.resid + o))) + acc[n][e];
        a.ws.h[o] = hv;
        sq[t * kTcRows + rr] = hv * hv;
      }
    }
  }
  consumer_sync();
  if (tid < B) {  // per-CTA sum of h^2, rows in order
    float ss = 0.f;
    for (int rr = 0; rr < rows; ++rr) ss += sq[tid * kTcRows + rr];
    a.ws.ss_part[(size_t)c * a.maxB + tid] = ss;
  }
}

// ---- host -------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// bf16 map viewing a row-major [outer][inner] matrix as {64, outer, inner / 64} with boxes
// {64, box_outer, kTcKB} and the 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kTcBK, outer, inner / kTcBK};
  const cuuint64_t strides[2] = {inner * 2, (cuuint64_t)kTcBK * 2};
  const cuuint32_t box[3] = {(cuuint32_t)kTcBK, box_outer, (cuuint32_t)kTcKB};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// bf16 map viewing a row-major [outer][inner] matrix in 2-D with boxes {box_inner, box_outer}
// and the 128-byte swizzle (box_inner * 2 must be 128).
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                 uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool oproj_tc_ok(const LayerArgs& a, int grid, size_t optin) {
  return encode_fn() != nullptr && a.B <= kTcTok && a.d_o % kTcBK == 0 && (a.d + grid - 1) / grid <= 49 &&
         tc_stages(std::min(kTcTok, (a.B + 15) / 16 * 16), optin) >= 3;
}

cudaError_t set_tc_attributes(size_t optin) {
  cudaError_t e = cudaFuncSetAttribute(k_oproj_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)optin);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_oproj_tc, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  return e;
}

cudaError_t launch_oproj_tc(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t optin) {
  CUtensorMap tmW, tmA;
  const int tokb = std::min(kTcTok, (a.B + 15) / 16 * 16);
  if (!make_map(&tmW, a.w_o, (uint64_t)a.d_o, (uint64_t)a.d, kTcRows) ||
      !make_map(&tmA, a.attn, (uint64_t)a.d_o, (uint64_t)a.B, (uint32_t)tokb))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  const int ns = tc_stages(tokb, optin), sb = tc_stage_bytes(tokb);
  cfg.dynamicSmemBytes = kTcFixed + (size_t)ns * sb;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_oproj_tc, tmW, tmA, a, tokb, ns, sb);
}

}  // namespace moe
