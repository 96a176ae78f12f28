// C ABI of the MoE decode-layer library: handle life cycle, workspace, CUDA-graph
// capture of the per-layer kernel chain, and the host-buffer variant of the step.
//
// A step of n_layers layers is captured once per (batch, buffer addresses) into one
// CUDA graph.  At batch 1 a layer is one cooperative kernel (o_proj + residual + RMS
// statistics, router, per-CTA routing, gate/up, down + combine, with grid barriers
// between the phases); at batch 2 to 4 (batch x top-k <= 64) it is o_proj -> router -> the
// small-M expert kernel (per-CTA routing, gate/up, down + combine); above it is o_proj -> router +
// routing tables -> gate/up -> down + combine.  Kernels are chained with programmatic dependent launch so
// each one's producer fetches its static weights while the previous kernel drains.  With
// prefetch on, layer l also prefetches into L2 what layer l+1 reads first (its router
// rows, RMSNorm scale and the leading rows of its W_o).
//
// Sources: "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted
// kernels", section "How the specialised decode path works" (kernel choice by batch
// size; next-layer weight prefetch on a side kernel); "vLLM and NVIDIA use coding agents
// to nearly double Kimi K3 decode speed, then rethink how to review it" (fewer kernels
// per layer); "vLLM tests a fast-track review model with Kimi K3's specialized decode
// path", section "Why the review model matters" (reject unsupported configurations at
// startup).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_set>
#include <vector>

#include "../../include/moe_decode.h"
#include "common.cuh"
#include "kernels.cuh"

using namespace moe;

namespace {

struct GraphEntry {
  int batch;
  const void *attn, *resid, *out, *idx, *gate;
  bool host;  // host-buffer step: staging copies in the graph around the layer kernels
  cudaGraphExec_t exec;
  int kernels;
};

// Staging copy of the host-buffer step: n 16-byte words from src to dst, one side pinned host
// memory (through its device address), the other device memory.  The copy-in runs first in the
// graph and lets the first layer kernel launch at once (its producer streams weights while the
// inputs arrive; its consumers wait for this grid); the copy-out waits for the last kernel.
__global__ void k_stage_copy(const uint4* __restrict__ src, uint4* __restrict__ dst, unsigned long long n,
                             int after_previous) {
  if (after_previous) asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
  for (unsigned long long i = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    dst[i] = src[i];
}

cudaError_t launch_stage_copy(const void* src, void* dst, size_t bytes, bool after_previous, cudaStream_t s) {
  const unsigned long long n = (bytes + 15) / 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min<unsigned long long>(148, std::max<unsigned long long>(1, (n + 1023) / 1024)));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_previous ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_stage_copy, static_cast<const uint4*>(src), static_cast<uint4*>(dst), n,
                            after_previous ? 1 : 0);
}

constexpr size_t kPrefetchWoBytes = 16ull << 20;  // bytes of the next W_o prefetched into L2
constexpr int kGraphCacheMax = 16;

}  // namespace

struct moe_decode_handle {
  moe_decode_config cfg;
  std::vector<moe_decode_layer_weights> w;
  int device = 0, num_sms = 0;
  size_t smem_optin = 0;
  Workspace ws{};
  void* ws_base = nullptr;
  uint16_t* resid_pp[2] = {nullptr, nullptr};
  // staging for moe_decode_step_host: device buffers for a step's inputs and outputs, each
  // group contiguous, and pinned host mirrors of them, so a step moves one copy each way
  void *h_in = nullptr, *h_outs = nullptr;      // device: inputs, outputs
  void *pin_in = nullptr, *pin_out = nullptr;   // pinned host mirrors
  void *pin_in_dev = nullptr, *pin_out_dev = nullptr;  // their device addresses
  size_t in_bytes = 0, out_bytes = 0;           // capacities (max_batch)
  LayerArgs plan_base{};
  cudaStream_t cap = nullptr;
  std::vector<GraphEntry> graphs;
  int last_batch = 0;
  bool poisoned = false;
};

namespace {

// Live handles: destroy and step reject pointers that are not (or no longer) handles.
std::mutex g_live_mu;
std::unordered_set<const moe_decode_handle*> g_live;

bool is_live(const moe_decode_handle* h) {
  std::lock_guard<std::mutex> lk(g_live_mu);
  return g_live.count(h) != 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

void release(moe_decode_handle* h) {
  for (auto& g : h->graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  h->graphs.clear();
  if (h->cap) cudaStreamDestroy(h->cap);
  if (h->ws_base) cudaFree(h->ws_base);
  h->cap = nullptr;
  h->ws_base = nullptr;
}

bool use_large(const moe_decode_handle* h, int B) {
  if (B > 4) return true;           // separate large-batch kernels above batch four
  return h->cfg.force_variant == 2;  // small-matrix kernels up to batch four where they fit
}

// Kernel choice of one layer step.
struct Variant {
  bool oproj_small;   // whole-row o_proj (batch <= 4)
  bool experts_small; // small-M gate/up and down with per-CTA routing (batch <= 4)
  bool layer2;        // the batch <= 2 layer kernel with per-expert counters (one launch)
  bool fused;         // the three batch <= 2 kernels as one launch with three grid barriers
  bool split;         // batch 5 to 8: the large-batch o_proj and router, then both expert
                      // paths, of which the kernels run only the one split_chosen() picks on
                      // the device: gate/up and down, or the small-M expert kernel once per
                      // half of the batch (at most four tokens each)
};

// The arguments of the expert kernel for tokens [t0, t0 + nt) of a step (pointers offset to
// them; the routing is recomputed from their logits), its grid barrier the half-th of the step.
LayerArgs half_args(const LayerArgs& a, int t0, int nt, int half) {
  LayerArgs ah = a;
  ah.B = nt;
  ah.ws.logits = a.ws.logits + (size_t)t0 * a.E;
  ah.ws.x = a.ws.x + (size_t)t0 * a.d;
  ah.ws.h = a.ws.h + (size_t)t0 * a.d;
  ah.out = a.out + (size_t)t0 * a.d;
  ah.user_idx = a.user_idx ? a.user_idx + (size_t)t0 * a.k : nullptr;
  ah.user_gate = a.user_gate ? a.user_gate + (size_t)t0 * a.k : nullptr;
  ah.route_tables = 0;
  ah.bar_base = half;
  ah.split_B = a.B;
  return ah;
}

Variant variant_of(const moe_decode_handle* h, const LayerArgs& a) {
  Variant v;
  v.experts_small = !use_large(h, a.B) && small_path_ok(a, h->smem_optin);
  v.oproj_small = v.experts_small && oproj_small_ok(a, h->smem_optin);
  const bool by_batch = !use_large(h, a.B) && h->cfg.force_variant == 0;
  v.layer2 = !use_large(h, a.B) && a.B <= 2 && h->cfg.force_variant == 3 && layer2_ok(a, h->smem_optin);
  // Where the counter-based kernel does not fit: one fused launch at batch 1; at batch 2 the
  // three kernels were measured ahead of that fused launch, so they stay.
  v.fused = !v.layer2 && by_batch && v.oproj_small && a.B == 1 && layer_fused_ok(a, h->smem_optin);
  // Five to eight tokens: both expert paths are launched and the kernels choose on the device
  // (split_chosen): tokens sharing most experts run as two launches of the four-token kernel
  // (each streams its half's experts once), where the large-batch gate/up and down kernels
  // run well below the HBM rate with one or two tokens per expert.
  v.split = false;
  if (!v.experts_small && h->cfg.force_variant == 0 && a.B > 4 && a.B <= 8) {
    LayerArgs ah = a;
    ah.B = 4;
    v.split = small_path_ok(ah, h->smem_optin);
  }
  return v;
}

LayerArgs layer_args(const moe_decode_handle* h, int l, int B, const void* attn, const void* resid,
                     void* out, int32_t* idx, float* gate) {
  const moe_decode_config& c = h->cfg;
  LayerArgs a = h->plan_base;
  a.B = B;
  plan_layer(a, h->num_sms, h->smem_optin);  // validated for every batch size at create
  a.route_tables = variant_of(h, a).experts_small ? 0 : 1;
  a.w_o = static_cast<const uint16_t*>(h->w[l].w_o);
  a.gamma = static_cast<const uint16_t*>(h->w[l].gamma);
  a.w_r = static_cast<const uint16_t*>(h->w[l].w_router);
  a.w_gu = static_cast<const uint16_t*>(h->w[l].w_gate_up);
  a.w_down = static_cast<const uint16_t*>(h->w[l].w_down);
  a.attn = static_cast<const uint16_t*>(attn) + (size_t)l * B * c.d_o;
  a.resid = (l == 0) ? static_cast<const uint16_t*>(resid) : h->resid_pp[(l - 1) & 1];
  a.out = (l == c.n_layers - 1) ? static_cast<uint16_t*>(out) : h->resid_pp[l & 1];
  a.user_idx = idx ? idx + (size_t)l * B * c.top_k : nullptr;
  a.user_gate = gate ? gate + (size_t)l * B * c.top_k : nullptr;
  a.pf_w_o = a.pf_w_r = a.pf_gamma = nullptr;
  a.pf_w_o_rows = 0;
  if (c.enable_prefetch && l + 1 < c.n_layers) {
    const moe_decode_layer_weights& nw = h->w[l + 1];
    a.pf_w_o = static_cast<const uint16_t*>(nw.w_o);
    a.pf_w_r = static_cast<const uint16_t*>(nw.w_router);
    a.pf_gamma = static_cast<const uint16_t*>(nw.gamma);
    const size_t rows = kPrefetchWoBytes / ((size_t)c.d_o * 2) / (size_t)h->num_sms;
    a.pf_w_o_rows = (int)std::max<size_t>(1, rows);
  }
  return a;
}

// Records the whole step on h->cap (which is in capture mode).  Returns kernels launched.
// first_pdl: the first kernel follows another kernel of the same graph (programmatic launch).
int record_step(moe_decode_handle* h, int B, const void* attn, const void* resid, void* out,
                int32_t* idx, float* gate, cudaError_t* err, bool first_pdl = false) {
  const moe_decode_config& c = h->cfg;
  const int G = h->num_sms;
  int kernels = 0;
  cudaError_t e = cudaSuccess;
  for (int l = 0; l < c.n_layers && e == cudaSuccess; ++l) {
    LayerArgs a = layer_args(h, l, B, attn, resid, out, idx, gate);
    const Variant v = variant_of(h, a);
    if (v.layer2 || v.fused) {
      const bool pdl = l > 0 || first_pdl;
      e = v.layer2 ? launch_layer2(a, G, h->cap, pdl, h->smem_optin) : launch_layer_s(a, G, h->cap, pdl, h->smem_optin);
      kernels += 1;
      continue;
    }
    const bool pdl = l > 0 || first_pdl;
    e = v.oproj_small                         ? launch_oproj_s(a, G, h->cap, pdl, h->smem_optin)
        : oproj_tc_ok(a, G, h->smem_optin) ? launch_oproj_tc(a, G, h->cap, pdl, h->smem_optin)
                                            : launch_oproj(a, G, h->cap, pdl);
    if (e == cudaSuccess)
      e = (!v.experts_small && router_ks_ok(a, G, h->smem_optin))    ? launch_router_ks(a, G, h->cap, true)
          : (!v.experts_small && router_big_ok(a, h->smem_optin)) ? launch_router_big(a, G, h->cap, true, h->smem_optin)
                                                                  : launch_router_s(a, G, h->cap, true, h->smem_optin);
    kernels += 2;
    if (v.experts_small) {
      if (e == cudaSuccess) e = launch_experts_s(a, G, h->cap, true, h->smem_optin);
      kernels += 1;
    } else if (v.split) {
      LayerArgs al = a;
      al.split_B = B;
      if (e == cudaSuccess) e = launch_gateup_rows(al, G, h->cap, true, h->smem_optin);
      if (e == cudaSuccess) e = launch_down_rows(al, G, h->cap, true, h->smem_optin);
      kernels += 2;
      for (int t0 = 0, half = 0; t0 < B; t0 += 4, ++half) {
        if (e == cudaSuccess) e = launch_experts_s(half_args(a, t0, std::min(4, B - t0), half), G, h->cap, true, h->smem_optin);
        kernels += 1;
      }
    } else {
      if (e == cudaSuccess) e = launch_gateup_rows(a, G, h->cap, true, h->smem_optin);
      if (e == cudaSuccess) e = launch_down_rows(a, G, h->cap, true, h->smem_optin);
      kernels += 2;
    }
  }
  *err = e;
  return kernels;
}

// host: the step reads its inputs from, and writes its outputs to, the handle's pinned
// staging (in_bytes from pin_in_dev to attn; out_bytes from out to pin_out_dev).
int get_graph(moe_decode_handle* h, int B, const void* attn, const void* resid, void* out,
              int32_t* idx, float* gate, GraphEntry** ge, bool host = false, size_t in_bytes = 0,
              size_t out_bytes = 0) {
  for (auto& g : h->graphs)
    if (g.batch == B && g.attn == attn && g.resid == resid && g.out == out && g.idx == idx && g.gate == gate &&
        g.host == host) {
      *ge = &g;
      return MOE_OK;
    }
  if ((int)h->graphs.size() >= kGraphCacheMax) {
    cudaGraphExecDestroy(h->graphs.front().exec);
    h->graphs.erase(h->graphs.begin());
  }
  cudaGraph_t graph = nullptr;
  if (cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return MOE_ERR_CUDA;
  cudaError_t rec = cudaSuccess;
  int kernels = 0;
  if (host) rec = launch_stage_copy(h->pin_in_dev, const_cast<void*>(attn), in_bytes, false, h->cap);
  if (rec == cudaSuccess) kernels = record_step(h, B, attn, resid, out, idx, gate, &rec, host);
  if (host && rec == cudaSuccess) rec = launch_stage_copy(out, h->pin_out_dev, out_bytes, true, h->cap);
  const cudaError_t end = cudaStreamEndCapture(h->cap, &graph);
  if (rec != cudaSuccess || end != cudaSuccess || !graph) {
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  cudaGraphExec_t exec = nullptr;
  const cudaError_t inst = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (inst != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  h->graphs.push_back(GraphEntry{B, attn, resid, out, idx, gate, host, exec, kernels});
  *ge = &h->graphs.back();
  return MOE_OK;
}

}  // namespace

// Validation shared by moe_decode_create and moe_decode_step_static: the supported set of
// include/moe_decode.h (shapes, batch and layer limits, eps, force_variant).
int moe::check_config(const moe_decode_config* c) {
  if (c->d < 64 || c->d > 8192 || c->d % 64) return MOE_ERR_UNSUPPORTED_CONFIG;
  if (c->d_o < 64 || c->d_o > 8192 || c->d_o % 64) return MOE_ERR_UNSUPPORTED_CONFIG;
  if (c->top_k < 1 || c->top_k > 32) return MOE_ERR_UNSUPPORTED_CONFIG;
  if (c->n_experts < c->top_k || c->n_experts > 1024) return MOE_ERR_UNSUPPORTED_CONFIG;
  if (c->inter < 32 || c->inter > 512 || c->inter % 32) return MOE_ERR_UNSUPPORTED_CONFIG;
  if (c->max_batch < 1 || c->max_batch > 64) return MOE_ERR_UNSUPPORTED_CONFIG;
  if (c->n_layers < 1 || c->n_layers > 64) return MOE_ERR_UNSUPPORTED_CONFIG;
  if (!(c->rms_eps > 0.f)) return MOE_ERR_UNSUPPORTED_CONFIG;
  if (c->force_variant < 0 || c->force_variant > 3) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

extern "C" {

int moe_decode_create(const moe_decode_config* cfg, const moe_decode_layer_weights* weights, void* stream,
                      moe_decode_handle** out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || !weights) return MOE_ERR_INVALID_ARG;
  int rc = check_config(cfg);
  if (rc) return rc;
  for (int l = 0; l < cfg->n_layers; ++l) {
    const moe_decode_layer_weights& w = weights[l];
    if (!w.w_o || !w.gamma || !w.w_router || !w.w_gate_up || !w.w_down) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w.w_o) || !aligned16(w.gamma) || !aligned16(w.w_router) || !aligned16(w.w_gate_up) ||
        !aligned16(w.w_down))
      return MOE_ERR_ALIGNMENT;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED_CONFIG;  // sm_100 only

  moe_decode_handle* h = new (std::nothrow) moe_decode_handle();
  if (!h) return MOE_ERR_OOM;
  h->cfg = *cfg;
  h->w.assign(weights, weights + cfg->n_layers);
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  h->smem_optin = prop.sharedMemPerBlockOptin;
  const int G = h->num_sms, maxB = cfg->max_batch, d = cfg->d, E = cfg->n_experts, K = cfg->top_k,
            I = cfg->inter;
  if ((long long)G * kConsumerThreads < d) {
    delete h;
    return MOE_ERR_UNSUPPORTED_CONFIG;
  }

  // ---- plans: every batch size 1..max_batch must fit ------------------------------------
  LayerArgs base{};
  base.maxB = maxB;
  base.d = d;
  base.d_o = cfg->d_o;
  base.E = E;
  base.k = K;
  base.I = I;
  base.eps = cfg->rms_eps;
  h->plan_base = base;
  bool ok = true;
  for (int B = 1; B <= maxB && ok; ++B) {  // the large-batch kernels must fit at every batch
    LayerArgs t = h->plan_base;
    t.B = B;
    t.route_tables = 1;
    ok = plan_layer(t, G, h->smem_optin) && router_ok(t, h->smem_optin) && plan_large(t, G, h->smem_optin);
  }
  if (!ok) {
    delete h;
    return MOE_ERR_UNSUPPORTED_CONFIG;
  }

  // ---- workspace -----------------------------------------------------------------------
  const size_t entries = (size_t)maxB * K;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += up256(bytes);
    return o;
  };
  const size_t o_h = take(sizeof(float) * maxB * d), o_x = take(sizeof(float) * maxB * d),
               o_rstd = take(sizeof(float) * maxB), o_ss = take(sizeof(float) * G * maxB),
               o_lg = take(sizeof(float) * maxB * E), o_ti = take(sizeof(int) * entries),
               o_tg = take(sizeof(float) * entries), o_nu = take(sizeof(int)), o_ue = take(sizeof(int) * E),
               o_uo = take(sizeof(int) * (E + 1)), o_et = take(sizeof(int) * entries),
               o_es = take(sizeof(int) * entries), o_a = take(sizeof(float) * entries * I),
               o_cnt = take(sizeof(unsigned) * kNumCounters),
               o_err = take(sizeof(unsigned)), o_r0 = take(2ull * maxB * d), o_r1 = take(2ull * maxB * d),
               o_ec = take(sizeof(unsigned) * kMaxUnion), o_au = take(sizeof(float) * kMaxUnion * 2 * I),
               o_rp = take(sizeof(float) * G * E * ((maxB + 7) / 8 * 8));  // the split-K router pads B to 8
  if (cudaMalloc(&h->ws_base, off) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return MOE_ERR_OOM;
  }
  char* b = static_cast<char*>(h->ws_base);
  Workspace& ws = h->ws;
  ws.h = (float*)(b + o_h);
  ws.x = (float*)(b + o_x);
  ws.rstd = (float*)(b + o_rstd);
  ws.ss_part = (float*)(b + o_ss);
  ws.logits = (float*)(b + o_lg);
  ws.topk_idx = (int*)(b + o_ti);
  ws.topk_gate = (float*)(b + o_tg);
  ws.n_union = (int*)(b + o_nu);
  ws.union_e = (int*)(b + o_ue);
  ws.union_off = (int*)(b + o_uo);
  ws.entry_tok = (int*)(b + o_et);
  ws.entry_slot = (int*)(b + o_es);
  ws.a = (float*)(b + o_a);
  ws.counters = (unsigned*)(b + o_cnt);
  ws.err = (unsigned*)(b + o_err);
  ws.ecnt = (unsigned*)(b + o_ec);
  ws.a_u = (float*)(b + o_au);
  ws.rpart = (float*)(b + o_rp);
  h->resid_pp[0] = (uint16_t*)(b + o_r0);
  h->resid_pp[1] = (uint16_t*)(b + o_r1);
  h->plan_base.ws = ws;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(h->ws_base, 0, off, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = set_kernel_attributes(h->smem_optin);
  if (e == cudaSuccess) e = set_small_attributes(h->smem_optin);
  if (e == cudaSuccess) e = set_large_attributes(h->smem_optin);
  if (e == cudaSuccess) e = set_tc_attributes(h->smem_optin);
  if (e == cudaSuccess) e = set_layer2_attributes(h->smem_optin);
  if (e == cudaSuccess) e = set_router_ks_attributes(h->smem_optin);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking);
  if (e != cudaSuccess) {
    cudaGetLastError();
    release(h);
    delete h;
    return MOE_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lk(g_live_mu);
    g_live.insert(h);
  }
  *out = h;
  return MOE_OK;
}

int moe_decode_step(moe_decode_handle* h, int batch, const void* attn_out, const void* residual_in, void* out,
                    int32_t* topk_idx, float* topk_gate, void* stream) {
  if (!h || !is_live(h) || h->poisoned) return MOE_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MOE_ERR_INVALID_ARG;
  if (!attn_out || !residual_in || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(attn_out) || !aligned16(residual_in) || !aligned16(out) || (topk_idx && !aligned16(topk_idx)) ||
      (topk_gate && !aligned16(topk_gate)))
    return MOE_ERR_ALIGNMENT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MOE_ERR_INVALID_ARG;
  GraphEntry* ge = nullptr;
  int rc = get_graph(h, batch, attn_out, residual_in, out, topk_idx, topk_gate, &ge);
  if (rc) return rc;
  if (cudaGraphLaunch(ge->exec, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  h->last_batch = batch;
  return MOE_OK;
}

int moe_decode_step_host(moe_decode_handle* h, int batch, const void* attn_out_host, const void* residual_in_host,
                         void* out_host, int32_t* topk_idx_host, float* topk_gate_host, void* stream) {
  if (!h || !is_live(h) || h->poisoned) return MOE_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MOE_ERR_INVALID_ARG;
  if (!attn_out_host || !residual_in_host || !out_host) return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MOE_ERR_INVALID_ARG;
  const moe_decode_config& c = h->cfg;
  const size_t maxB = c.max_batch;
  // Layout for `batch` tokens: inputs [attn_out | residual_in], outputs [out | idx | gate],
  // each part starting on a 256-byte boundary.
  const size_t n_attn = 2ull * c.n_layers * batch * c.d_o, n_res = 2ull * batch * c.d,
               n_tk = 4ull * c.n_layers * batch * c.top_k;
  const size_t o_res = up256(n_attn), in_used = o_res + n_res;
  const size_t o_idx = up256(n_res), o_gate = o_idx + up256(n_tk);
  const size_t out_used = (topk_gate_host ? o_gate + n_tk : topk_idx_host ? o_idx + n_tk : n_res);
  if (!h->h_in) {
    h->in_bytes = up256(2ull * c.n_layers * maxB * c.d_o) + up256(2ull * maxB * c.d);
    h->out_bytes = up256(2ull * maxB * c.d) + 2 * up256(4ull * c.n_layers * maxB * c.top_k);
    void *di = nullptr, *dout = nullptr, *pi = nullptr, *po = nullptr, *pid = nullptr, *pod = nullptr;
    if (cudaMalloc(&di, h->in_bytes) != cudaSuccess || cudaMalloc(&dout, h->out_bytes) != cudaSuccess ||
        cudaHostAlloc(&pi, h->in_bytes, cudaHostAllocMapped) != cudaSuccess ||
        cudaHostAlloc(&po, h->out_bytes, cudaHostAllocMapped) != cudaSuccess ||
        cudaHostGetDevicePointer(&pid, pi, 0) != cudaSuccess || cudaHostGetDevicePointer(&pod, po, 0) != cudaSuccess) {
      cudaGetLastError();
      if (di) cudaFree(di);
      if (dout) cudaFree(dout);
      if (pi) cudaFreeHost(pi);
      if (po) cudaFreeHost(po);
      return MOE_ERR_OOM;
    }
    h->h_in = di;
    h->h_outs = dout;
    h->pin_in = pi;
    h->pin_out = po;
    h->pin_in_dev = pid;
    h->pin_out_dev = pod;
  }
  char* din = static_cast<char*>(h->h_in);
  char* dout = static_cast<char*>(h->h_outs);
  char* pin = static_cast<char*>(h->pin_in);
  char* pout = static_cast<char*>(h->pin_out);
  // One graph per (batch, outputs wanted): copy-in kernel -> the step's kernels -> copy-out
  // kernel, so a call is one graph launch and one synchronisation.
  GraphEntry* ge = nullptr;
  int rc = get_graph(h, batch, din, din + o_res, dout, topk_idx_host ? (int32_t*)(dout + o_idx) : nullptr,
                     topk_gate_host ? (float*)(dout + o_gate) : nullptr, &ge, true, in_used, out_used);
  if (rc) return rc;
  std::memcpy(pin, attn_out_host, n_attn);
  std::memcpy(pin + o_res, residual_in_host, n_res);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaGraphLaunch(ge->exec, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  h->last_batch = batch;
  std::memcpy(out_host, pout, n_res);
  if (topk_idx_host) std::memcpy(topk_idx_host, pout + o_idx, n_tk);
  if (topk_gate_host) std::memcpy(topk_gate_host, pout + o_gate, n_tk);
  return MOE_OK;
}

int moe_decode_sync_status(moe_decode_handle* h, void* stream) {
  if (!h || !is_live(h)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  unsigned word = 0;
  if (cudaMemcpy(&word, h->ws.err, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (word) {
    // a bounded wait that ran out may leave a grid-barrier or expert count behind
    cudaMemset(h->ws.counters, 0, sizeof(unsigned) * kNumCounters);
    cudaMemset(h->ws.ecnt, 0, sizeof(unsigned) * kMaxUnion);
    cudaMemset(h->ws.err, 0, sizeof word);
    cudaDeviceSynchronize();
    return (word & kErrTimeout) ? MOE_ERR_DEVICE_TIMEOUT : MOE_ERR_DEVICE_BOUNDS;
  }
  return MOE_OK;
}

int moe_decode_check_error_path(moe_decode_handle* h, int what, unsigned long long limit_ns, void* stream) {
  if (!h || !is_live(h) || h->poisoned) return MOE_ERR_INVALID_ARG;
  if ((what != 1 && what != 2) || limit_ns == 0 || limit_ns > 10000000ull) return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MOE_ERR_INVALID_ARG;
  // the probe's sink is n_union, which every step rewrites before anything reads it
  if (launch_error_probe(&h->ws.counters[kCntProbe], h->ws.err, what, limit_ns, h->cfg.n_experts, h->ws.n_union,
                         static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int moe_decode_get_intermediate(moe_decode_handle* h, int which, void* dst, size_t bytes, void* stream) {
  if (!h || !is_live(h) || !dst || h->last_batch < 1) return MOE_ERR_INVALID_ARG;
  const int B = h->last_batch;
  const void* src = nullptr;
  size_t size = 0;
  switch (which) {
    case 0: src = h->ws.h; size = 4ull * B * h->cfg.d; break;
    case 1: src = h->ws.rstd; size = 4ull * B; break;
    case 2: src = h->ws.x; size = 4ull * B * h->cfg.d; break;
    case 3: src = h->ws.logits; size = 4ull * B * h->cfg.n_experts; break;
    default: return MOE_ERR_INVALID_ARG;
  }
  if (cudaMemcpyAsync(dst, src, std::min(bytes, size), cudaMemcpyDeviceToDevice,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int moe_decode_kernels_per_step(moe_decode_handle* h, int batch) {
  if (!h || !is_live(h) || batch < 1 || batch > h->cfg.max_batch) return MOE_ERR_INVALID_ARG;
  const int L = h->cfg.n_layers;
  LayerArgs a = h->plan_base;
  a.B = batch;
  plan_layer(a, h->num_sms, h->smem_optin);
  const Variant v = variant_of(h, a);
  const int per_layer = (v.layer2 || v.fused) ? 1 : v.experts_small ? 3 : v.split ? 4 + (batch + 3) / 4 : 4;
  return per_layer * L;
}

int moe_decode_profile_step(moe_decode_handle* h, int batch, const void* attn_out, const void* residual_in,
                            void* out, int32_t* topk_idx, float* topk_gate, void* stream, float* kernel_ms,
                            int* kernel_id, int max_kernels) {
  if (!h || !is_live(h) || h->poisoned || !kernel_ms || max_kernels < 1) return MOE_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch || !attn_out || !residual_in || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(attn_out) || !aligned16(residual_in) || !aligned16(out) || (topk_idx && !aligned16(topk_idx)) ||
      (topk_gate && !aligned16(topk_gate)))
    return MOE_ERR_ALIGNMENT;
  const moe_decode_config& c = h->cfg;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int G = h->num_sms;
  const int n = std::min(max_kernels, moe_decode_kernels_per_step(h, batch));
  std::vector<cudaEvent_t> ev(2 * n, nullptr);
  cudaError_t e = cudaSuccess;
  for (auto& x : ev)
    if (e == cudaSuccess) e = cudaEventCreate(&x);
  int k = 0;
  auto timed = [&](int id, cudaStream_t st, auto&& fn) {
    if (e != cudaSuccess || k >= n) return;
    e = cudaEventRecord(ev[2 * k], st);
    if (e == cudaSuccess) e = fn(st);
    if (e == cudaSuccess) e = cudaEventRecord(ev[2 * k + 1], st);
    if (kernel_id) kernel_id[k] = id;
    ++k;
  };
  for (int l = 0; l < c.n_layers; ++l) {
    LayerArgs a = layer_args(h, l, batch, attn_out, residual_in, out, topk_idx, topk_gate);
    const Variant v = variant_of(h, a);
    if (v.layer2 || v.fused) {
      timed(6, s, [&](cudaStream_t st) {
        return v.layer2 ? launch_layer2(a, G, st, false, h->smem_optin) : launch_layer_s(a, G, st, false, h->smem_optin);
      });
      continue;
    }
    timed(1, s, [&](cudaStream_t st) {
      return v.oproj_small                         ? launch_oproj_s(a, G, st, false, h->smem_optin)
             : oproj_tc_ok(a, G, h->smem_optin) ? launch_oproj_tc(a, G, st, false, h->smem_optin)
                                                 : launch_oproj(a, G, st, false);
    });
    timed(2, s, [&](cudaStream_t st) {
      return (!v.experts_small && router_ks_ok(a, G, h->smem_optin))    ? launch_router_ks(a, G, st, false)
             : (!v.experts_small && router_big_ok(a, h->smem_optin)) ? launch_router_big(a, G, st, false, h->smem_optin)
                                                                     : launch_router_s(a, G, st, false, h->smem_optin);
    });
    if (v.experts_small) {
      timed(3, s, [&](cudaStream_t st) { return launch_experts_s(a, G, st, false, h->smem_optin); });
    } else if (v.split) {
      LayerArgs al = a;
      al.split_B = batch;
      timed(4, s, [&](cudaStream_t st) { return launch_gateup_rows(al, G, st, false, h->smem_optin); });
      timed(5, s, [&](cudaStream_t st) { return launch_down_rows(al, G, st, false, h->smem_optin); });
      for (int t0 = 0, half = 0; t0 < batch; t0 += 4, ++half)
        timed(3, s, [&](cudaStream_t st) {
          return launch_experts_s(half_args(a, t0, std::min(4, batch - t0), half), G, st, false, h->smem_optin);
        });
    } else {
      timed(4, s, [&](cudaStream_t st) { return launch_gateup_rows(a, G, st, false, h->smem_optin); });
      timed(5, s, [&](cudaStream_t st) { return launch_down_rows(a, G, st, false, h->smem_optin); });
    }
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  for (int i = 0; i < k && e == cudaSuccess; ++i) e = cudaEventElapsedTime(&kernel_ms[i], ev[2 * i], ev[2 * i + 1]);
  for (auto& x : ev)
    if (x) cudaEventDestroy(x);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  h->last_batch = batch;
  return k;
}

int moe_decode_destroy(moe_decode_handle* h) {
  if (!h) return MOE_OK;
  {
    std::lock_guard<std::mutex> lk(g_live_mu);
    if (!g_live.erase(h)) return MOE_ERR_INVALID_ARG;  // not a live handle (e.g. destroyed twice)
  }
  cudaDeviceSynchronize();
  release(h);
  if (h->h_in) cudaFree(h->h_in);
  if (h->h_outs) cudaFree(h->h_outs);
  if (h->pin_in) cudaFreeHost(h->pin_in);
  if (h->pin_out) cudaFreeHost(h->pin_out);
  h->poisoned = true;
  delete h;
  return MOE_OK;
}

const char* moe_decode_strerror(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_CONFIG: return "unsupported configuration";
    case MOE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MOE_ERR_OOM: return "out of device memory";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "device index out of range";
    case MOE_ERR_SCRATCH_LIMIT: return "scratch need exceeds the static array";
    default: return "unknown error";
  }
}

}  // extern "C"
