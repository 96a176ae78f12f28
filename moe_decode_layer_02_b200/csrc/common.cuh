// Device primitives shared by the sm_100a kernels of the MoE decode layer.
//
// Load rule: weights are static for the life of a handle, so they may be read
// through the non-coherent path (TMA bulk copies, ld.global.nc) and even
// before griddepcontrol.wait.  Activations and routing tables are produced by
// earlier kernels of the same graph, so they are read only after
// griddepcontrol.wait and only with loads that go to L2 (ld.global.cg), never
// with ld.global.nc.  (The pages describe a compiler that hoisted activation
// reads above a synchronisation wait, fixed by restricting that load type to
// static weights: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with
// agent-assisted kernels", section "Why vLLM wants new review rules for
// agent-written kernels".)
//
// Every spin wait is bounded in time: on expiry the kernel records
// kErrTimeout in the error word, marks the CTA aborted, skips the remaining
// waits (but still reaches every barrier), and drains its own copies in
// flight before it exits.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr uint32_t kErrTimeout = 1u;
constexpr uint32_t kErrBounds = 2u;
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;  // + one producer warp
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s
constexpr int kMaxStages = 8;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- programmatic dependent launch --------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- mbarrier -----------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait.  Returns false (and flags the CTA and the error word) when the
// limit expires or the CTA was already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* err, unsigned long long limit_ns = kWaitLimitNs) {
  if (*abort_flag) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort_flag = 1;
      if (err) atomicOr(err, kErrTimeout);
      return false;
    }
  }
}

// Waits for a phase while ignoring the abort flag (used to drain copies in flight).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return;
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) {
      atomicOr(err, kErrTimeout);
      return;
    }
  }
}

// ---- shared-memory ring of S stages (full: TMA completion, empty: consumer warps) ----
__device__ __forceinline__ void init_ring(uint64_t* full, uint64_t* empty, int S, int consumers = kConsumerWarps) {
  for (int s = 0; s < S; ++s) {
    mbar_init(&full[s], 1);
    if (empty) mbar_init(&empty[s], consumers);
  }
}

// Producer: waits until the slot of fill number `it` is free (bounded).
__device__ __forceinline__ bool ring_acquire(uint64_t* empty, int it, int S, volatile int* abort_flag, uint32_t* err) {
  if (it < S) return !*abort_flag;
  return mbar_wait(&empty[it % S], ((it / S) - 1) & 1, abort_flag, err);
}

// Producer epilogue: waits (bounded, ignoring abort) for the last min(S, issued) fills, so
// that no copy is still writing into shared memory when the CTA exits.
__device__ __forceinline__ void ring_drain(uint64_t* full, int issued, int S, uint32_t* err) {
  for (int i = issued - S < 0 ? 0 : issued - S; i < issued; ++i) mbar_drain(&full[i % S], (i / S) & 1, err);
}

// ---- TMA bulk copies (1-D, global -> shared) ---------------------------------------
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// bytes: multiple of 16, src and dst 16-byte aligned, < 2^20 per barrier phase.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes,
                                         uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// L2 prefetch of [src, src + bytes): bytes multiple of 16, src 16-byte aligned.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---- cross-CTA signalling ------------------------------------------------------------
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Every lane of the warp waits (bounded) until *p >= target; each lane's own acquire load
// orders its later reads after the writes released before the count was reached.
__device__ __forceinline__ bool warp_wait_count(const unsigned* p, unsigned target, volatile int* abort_flag,
                                                uint32_t* err) {
  if (__all_sync(0xffffffffu, ld_acquire_u32(p) >= target)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (__all_sync(0xffffffffu, ld_acquire_u32(p) >= target)) return true;
    int expired = (globaltimer() - t0 > kWaitLimitNs) || *abort_flag;
    if (__any_sync(0xffffffffu, expired)) {
      if ((threadIdx.x & 31) == 0) {
        *abort_flag = 1;
        atomicOr(err, kErrTimeout);
      }
      __syncwarp();
      return false;
    }
    __nanosleep(32);
  }
}

// ---- loads --------------------------------------------------------------------------
// Activations / tables written earlier in the same graph: L2-coherent loads.
__device__ __forceinline__ float ld_act(const float* p) { return __ldcg(p); }
__device__ __forceinline__ float4 ld_act4(const float* p) {
  return __ldcg(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ int ld_act_i(const int* p) { return __ldcg(p); }
__device__ __forceinline__ uint4 ld_act_u4(const void* p) {
  return __ldcg(reinterpret_cast<const uint4*>(p));
}
// Static weights: non-coherent read-only path.
__device__ __forceinline__ uint4 ld_weight_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ---- bf16 -------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// 8 bf16 (one uint4) dotted with 8 floats.
__device__ __forceinline__ float dot8(uint4 w, const float* a, float acc) {
  acc = fmaf(bf16lo(w.x), a[0], acc);
  acc = fmaf(bf16hi(w.x), a[1], acc);
  acc = fmaf(bf16lo(w.y), a[2], acc);
  acc = fmaf(bf16hi(w.y), a[3], acc);
  acc = fmaf(bf16lo(w.z), a[4], acc);
  acc = fmaf(bf16hi(w.z), a[5], acc);
  acc = fmaf(bf16lo(w.w), a[6], acc);
  acc = fmaf(bf16hi(w.w), a[7], acc);
  return acc;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}

// Range [lo, hi) of n items for part p of P (balanced, contiguous).
__host__ __device__ __forceinline__ void split_range(long long n, int P, int p, long long& lo,
                                                     long long& hi) {
  lo = n * p / P;
  hi = n * (p + 1) / P;
}

}  // namespace moe
