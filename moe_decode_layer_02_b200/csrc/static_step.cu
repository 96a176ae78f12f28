// moe_decode_step_static: the batch <= 2 layer step with its scratch in a static device array.
//
// Who cannot allocate.  moe_decode_create takes device memory for its workspace (cudaMalloc).
// Some callers are not free to do that when they want a decode step:
//   - a serving engine that reserves nearly all of HBM at start-up for its KV cache and its
//     own caching pool, and counts any allocation made behind the pool's back as a failure
//     (it may not fit, and it fragments memory the pool expects to own);
//   - code that runs under a hard per-process memory cap, where one more allocation can be
//     the one that fails in the middle of serving.
// For them this entry point runs the same kernels as the batch <= 2 path of moe_decode_step
// (one layer kernel: o_proj + residual + RMS statistics, router + top-k, experts; with
// force_variant 1 the o_proj, router and small-M expert kernels), launched directly on
// the caller's stream, with every intermediate in one file-scope device array of
// MOE_STATIC_SCRATCH_BYTES.  Nothing is allocated per call: no
// cudaMalloc/cudaFree and no library routine that allocates.  The array is part of the
// loaded module, so it exists once per device the library runs on.
//
// Setup.  The first call on a device (with that device current) looks up the array's
// device address with cudaGetSymbolAddress and sets the kernels' shared-memory attributes;
// later calls on that device reuse both.  That first call should come before any stream
// capture begins.
//
// Zero start.  The grid barriers and the per-expert counters need their counts at zero and
// the error word must start at zero; every call clears them (one cudaMemsetAsync on the
// caller's stream) before its kernels run.  Nothing else in the array needs a known value.
//
// Sharing.  Every call on a device uses the same array.  Calls whose executions overlap
// (issued on different streams, or from different threads without ordering between them)
// race on it and corrupt one another's results; order them, e.g. on one stream.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/moe_decode.h"
#include "common.cuh"
#include "kernels.cuh"

using namespace moe;

namespace {

__device__ __align__(256) unsigned char g_static_scratch[MOE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct DeviceSetup {
  bool done = false;
  int num_sms = 0;
  size_t smem_optin = 0;
  unsigned char* scratch = nullptr;  // device address of g_static_scratch on this device
};

std::mutex g_setup_mu;
DeviceSetup g_setup[kMaxDevices];

int setup_device(int dev, DeviceSetup* out) {
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED_CONFIG;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  DeviceSetup& s = g_setup[dev];
  if (!s.done) {
    int major = 0, minor = 0, sms = 0, optin = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED_CONFIG;  // sm_100 only
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    if (set_small_attributes((size_t)optin) != cudaSuccess || set_layer2_attributes((size_t)optin) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    s.num_sms = sms;
    s.smem_optin = (size_t)optin;
    s.scratch = static_cast<unsigned char*>(p);
    s.done = true;
  }
  *out = s;
  return MOE_OK;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Scratch layout for B tokens on G CTAs.  Counters and the error word come first so one
// memset clears both.  Returns the bytes used; fills ws when base is non-null.
size_t carve(unsigned char* base, int B, int G, int d, int E, int K, int I, bool layer2, Workspace* ws) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += up256(bytes);
    return base ? base + o : nullptr;
  };
  const size_t entries = (size_t)B * K;
  // grid-barrier counters, the error word and the per-expert counters: cleared by every call
  unsigned char* cnt = take(sizeof(unsigned) * (kNumCounters + 1 + kMaxUnion));
  unsigned char* h = take(sizeof(float) * B * d);
  unsigned char* x = take(sizeof(float) * B * d);
  unsigned char* rstd = take(sizeof(float) * B);
  unsigned char* ss = take(sizeof(float) * G * B);
  unsigned char* lg = take(sizeof(float) * B * E);
  unsigned char* ti = take(sizeof(int) * entries);
  unsigned char* tg = take(sizeof(float) * entries);
  unsigned char* nu = take(sizeof(int));
  unsigned char* ue = take(sizeof(int) * E);
  unsigned char* uo = take(sizeof(int) * (E + 1));
  unsigned char* et = take(sizeof(int) * entries);
  unsigned char* es = take(sizeof(int) * entries);
  unsigned char* act = take(sizeof(float) * entries * I);
  unsigned char* au = take(sizeof(float) * kMaxUnion * 2 * I);
  // the counter-ordered kernel's split-K router partials, [G][E][B]
  unsigned char* rp = layer2 ? take(sizeof(float) * G * E * B) : nullptr;
  if (ws) {
    ws->counters = reinterpret_cast<unsigned*>(cnt);
    ws->err = reinterpret_cast<unsigned*>(cnt) + kNumCounters;
    ws->h = reinterpret_cast<float*>(h);
    ws->x = reinterpret_cast<float*>(x);
    ws->rstd = reinterpret_cast<float*>(rstd);
    ws->ss_part = reinterpret_cast<float*>(ss);
    ws->logits = reinterpret_cast<float*>(lg);
    ws->topk_idx = reinterpret_cast<int*>(ti);
    ws->topk_gate = reinterpret_cast<float*>(tg);
    ws->n_union = reinterpret_cast<int*>(nu);
    ws->union_e = reinterpret_cast<int*>(ue);
    ws->union_off = reinterpret_cast<int*>(uo);
    ws->entry_tok = reinterpret_cast<int*>(et);
    ws->entry_slot = reinterpret_cast<int*>(es);
    ws->a = reinterpret_cast<float*>(act);
    ws->ecnt = reinterpret_cast<unsigned*>(cnt) + kNumCounters + 1;
    ws->a_u = reinterpret_cast<float*>(au);
    ws->rpart = reinterpret_cast<float*>(rp);
  }
  return off;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int moe_decode_step_static(const moe_decode_config* cfg, const moe_decode_layer_weights* w, int batch,
                           const void* attn_out, const void* residual_in, void* out, int32_t* topk_idx,
                           float* topk_gate, uint32_t* err_word, void* stream) {
  if (!cfg || !w || !attn_out || !residual_in || !out) return MOE_ERR_INVALID_ARG;
  const moe_decode_config& c = *cfg;
  const int rc_cfg = check_config(cfg);  // the supported set of moe_decode_create
  if (rc_cfg) return rc_cfg;
  if (c.n_layers != 1 || c.force_variant == 2) return MOE_ERR_UNSUPPORTED_CONFIG;  // one layer, small path
  if (batch < 1 || batch > 2 || batch > c.max_batch) return MOE_ERR_INVALID_ARG;
  if (!w->w_o || !w->gamma || !w->w_router || !w->w_gate_up || !w->w_down) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->w_o) || !aligned16(w->gamma) || !aligned16(w->w_router) || !aligned16(w->w_gate_up) ||
      !aligned16(w->w_down) || !aligned16(attn_out) || !aligned16(residual_in) || !aligned16(out) ||
      (topk_idx && !aligned16(topk_idx)) || (topk_gate && !aligned16(topk_gate)) ||
      (reinterpret_cast<uintptr_t>(err_word) & 3u))
    return MOE_ERR_ALIGNMENT;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  DeviceSetup ds;
  int rc = setup_device(dev, &ds);
  if (rc) return rc;
  const int G = ds.num_sms;
  if ((long long)G * kConsumerThreads < c.d) return MOE_ERR_UNSUPPORTED_CONFIG;

  const bool layer2 = c.force_variant == 3;
  const size_t need = carve(nullptr, batch, G, c.d, c.n_experts, c.top_k, c.inter, layer2, nullptr);
  if (need > (size_t)MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_SCRATCH_LIMIT;

  LayerArgs a{};
  a.B = batch;
  a.maxB = batch;
  a.d = c.d;
  a.d_o = c.d_o;
  a.E = c.n_experts;
  a.k = c.top_k;
  a.I = c.inter;
  a.eps = c.rms_eps;
  a.route_tables = 0;  // the expert kernel routes per CTA
  a.w_o = static_cast<const uint16_t*>(w->w_o);
  a.gamma = static_cast<const uint16_t*>(w->gamma);
  a.w_r = static_cast<const uint16_t*>(w->w_router);
  a.w_gu = static_cast<const uint16_t*>(w->w_gate_up);
  a.w_down = static_cast<const uint16_t*>(w->w_down);
  a.attn = static_cast<const uint16_t*>(attn_out);
  a.resid = static_cast<const uint16_t*>(residual_in);
  a.out = static_cast<uint16_t*>(out);
  a.user_idx = topk_idx;
  a.user_gate = topk_gate;
  carve(ds.scratch, batch, G, c.d, c.n_experts, c.top_k, c.inter, layer2, &a.ws);
  if (!small_path_ok(a, ds.smem_optin) || !router_ok(a, ds.smem_optin)) return MOE_ERR_UNSUPPORTED_CONFIG;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(a.ws.counters, 0, sizeof(unsigned) * (kNumCounters + 1 + kMaxUnion), s);
  // the kernels moe_decode_step picks: one layer kernel (or, where it does not fit, the fused
  // kernel at batch 1), unless force_variant 1 asks for the three small-batch kernels
  const bool by_batch = c.force_variant == 0;
  if (c.force_variant == 3 && layer2_ok(a, ds.smem_optin)) {
    if (e == cudaSuccess) e = launch_layer2(a, G, s, false, ds.smem_optin);
  } else if (by_batch && batch == 1 && layer_fused_ok(a, ds.smem_optin)) {
    if (e == cudaSuccess) e = launch_layer_s(a, G, s, false, ds.smem_optin);
  } else {
    if (e == cudaSuccess) e = launch_oproj_s(a, G, s, false, ds.smem_optin);
    if (e == cudaSuccess) e = launch_router_s(a, G, s, true, ds.smem_optin);
    if (e == cudaSuccess) e = launch_experts_s(a, G, s, true, ds.smem_optin);
  }
  if (e == cudaSuccess && err_word)
    e = cudaMemcpyAsync(err_word, a.ws.err, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // extern "C"
