// Kernel arguments and host launchers of the MoE decode layer (internal).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_decode.h"

namespace moe {

// The supported set of the C ABI (moe_decode.cu): MOE_OK or the MOE_ERR_* code create returns.
int check_config(const moe_decode_config* c);

// Device counters: fused layer kernel's exit ticket, router ticket, expert-kernel grid
// barrier count, fused layer kernel's grid barrier count.  All are zero between launches.
// kCntProbe: the error-path probe's grid-barrier count.
enum Counter {
  kCntLayerExit = 0, kCntRouter = 1, kCntGateUp = 2, kCntLayer = 3, kCntProbe = 4,
  kCntRouterBar = 5,   // the split-K router's grid barriers
  kCntRouterExit = 6,  // its exit ticket (the last CTA out clears 1, 5 and 6)
  kCntOUnit = 7,       // the fused layer kernel's o_proj unit counter (cleared after its barrier 1)
  kNumCounters = 8
};

// Library-owned device workspace (one per handle).
struct Workspace {
  float* h;          // [maxB][d]   residual + o_proj, fp32
  float* x;          // [maxB][d]   RMSNorm output, fp32
  float* rstd;       // [maxB]
  float* ss_part;    // [G][maxB]   per-CTA sums of h^2
  float* logits;     // [maxB][E]   fp32
  int* topk_idx;     // [maxB][k]
  float* topk_gate;  // [maxB][k]
  int* n_union;      // [1]         number of distinct selected experts U
  int* union_e;      // [E]         selected experts, ascending
  int* union_off;    // [E+1]       CSR offsets of each union expert's token entries
  int* entry_tok;    // [maxB*k]    token of each entry (ascending within an expert)
  int* entry_slot;   // [maxB*k]    slot j of that token's top-k list
  float* a;          // [maxB*k][I] SwiGLU activations per entry
  unsigned* counters;  // [kNumCounters]
  unsigned* err;       // error word (kErrTimeout | kErrBounds)
  // batch <= 2 layer kernel: per union expert, rows of its SwiGLU activations published so far
  // (zero between launches), and the activations [kMaxUnion][B][I]
  unsigned* ecnt;      // [kMaxUnion]
  float* a_u;          // [kMaxUnion][2][I]
  float* rpart;        // split-K routers' per-CTA partial logits: [G][E][8 ceil(B / 8)] on the large-batch path,
                       // [G][E][maxB] in the counter-ordered kernel (8 ceil(maxB / 8) per CTA and expert allocated)
};

constexpr int kMaxUnion = 64;  // union experts of a batch <= 2 step (2 tokens x top_k <= 32)

struct KTune {
  int stages = 0;          // ring stages
  int rows_per_stage = 0;  // weight rows (or row pairs) per stage (CUDA-core kernels)
  int rows_max = 0;        // max rows owned by one CTA
  int kc = 0;              // K chunk of one MMA stage (multiple of 64)
  int nch = 0;             // K chunks per row (K = kc * nch)
  int tok_group = 0;       // tokens per pass over the weights (down kernel: entries staged per stage)
  size_t smem = 0;         // dynamic shared memory bytes
};

// Batches of 5 to 8 tokens whose union of experts is under half their (token, expert)
// entries share most experts (draft tokens of one sequence): their expert phase runs as two
// launches of the four-token kernel, each streaming its half's experts once; otherwise the
// large-batch gate/up and down kernels run.  Decided on the device from the router's union,
// the same in every kernel of the step.
__host__ __device__ inline bool split_chosen(int U, int B, int K) { return 2 * U < B * K; }

struct LayerArgs {
  int B, maxB, d, d_o, E, k, I;
  float eps;
  const uint16_t *w_o, *gamma, *w_r, *w_gu, *w_down;  // this layer's weights
  const uint16_t* attn;   // [B][d_o]
  const uint16_t* resid;  // [B][d]
  uint16_t* out;          // [B][d]
  int* user_idx;          // [B][k] or null
  float* user_gate;       // [B][k] or null
  int route_tables;       // the router's last CTA builds the global routing tables
  int bar_base;           // the expert kernel's grid barrier opens at (bar_base + 1) x grid
                          // (1 for the second half of a batch split over two launches)
  int split_B;            // 5 to 8 tokens: the step launches both expert paths and each kernel
                          // runs only if split_chosen() says its path is the one (0: no choice)
  // Next layer's weights for the router kernel's L2 prefetch (null: no prefetch)
  const uint16_t *pf_w_o, *pf_w_r, *pf_gamma;
  int pf_w_o_rows;        // leading rows of each CTA's share of the next W_o to prefetch
  Workspace ws;
  KTune k1, k2, k3, k4;
};

// Host-side planning for a.B tokens (sets the KTune fields, returns false if unsupported).
bool plan_layer(LayerArgs& a, int num_sms, size_t smem_optin);

// Launchers (pdl: launch with programmatic stream serialisation).
cudaError_t launch_oproj(const LayerArgs& a, int grid, cudaStream_t s, bool pdl);

// Small-batch kernels and the router (kernels_small.cu): whole rows streamed by TMA.
bool plan_small(LayerArgs& a, int grid, size_t smem_optin);
bool small_path_ok(const LayerArgs& a, size_t smem_optin);   // o_proj, gate/up, down at batch <= 2
bool oproj_small_ok(const LayerArgs& a, size_t smem_optin);
bool router_ok(const LayerArgs& a, size_t smem_optin);       // router at this batch
cudaError_t set_small_attributes(size_t smem_optin);
cudaError_t launch_oproj_s(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t smem_optin);
cudaError_t launch_router_s(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t smem_optin);
cudaError_t launch_experts_s(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t smem_optin);
// A router of the large-batch path with h staged by TMA (plus the routing tables).
bool plan_router_big(LayerArgs& a, int grid, size_t smem_optin);
bool router_big_ok(const LayerArgs& a, size_t smem_optin);
cudaError_t launch_router_big(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t smem_optin);
// The three small-batch kernels fused into one cooperative launch per layer (batch <= 2).
bool plan_fused(LayerArgs& a, int grid, size_t smem_optin);
bool layer_fused_ok(const LayerArgs& a, size_t smem_optin);
cudaError_t launch_layer_s(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t smem_optin);
cudaError_t set_kernel_attributes(size_t smem_optin);
// The error-path probe (what 1: bounded waits run out; 2: an out-of-range index is clamped).
cudaError_t launch_error_probe(unsigned* count, unsigned* err, int what, unsigned long long limit_ns, int E,
                               int* sink, cudaStream_t s);

// The batch <= 2 layer kernel with per-expert counters instead of a barrier between the
// gate/up and down projections (kernels_layer.cu).
bool plan_layer2(LayerArgs& a, int grid, size_t smem_optin);
bool layer2_ok(const LayerArgs& a, size_t smem_optin);
cudaError_t set_layer2_attributes(size_t smem_optin);
cudaError_t launch_layer2(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t smem_optin);

// The router of the large-batch path with K split over the CTAs, partial logits on the tensor cores,
// and the routing tables (kernels_router.cu).
bool router_ks_ok(const LayerArgs& a, int grid, size_t smem_optin);
cudaError_t set_router_ks_attributes(size_t smem_optin);
cudaError_t launch_router_ks(const LayerArgs& a, int grid, cudaStream_t s, bool pdl);

// o_proj of the large-batch path on the tensor cores with 2-D TMA tiles (kernels_tc.cu).
bool oproj_tc_ok(const LayerArgs& a, int grid, size_t smem_optin);
cudaError_t set_tc_attributes(size_t smem_optin);
cudaError_t launch_oproj_tc(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t smem_optin);

// Expert kernels of the large-batch path (kernels_large.cu): whole rows, tokens grouped per expert.
bool plan_large(LayerArgs& a, int grid, size_t smem_optin);
cudaError_t set_large_attributes(size_t smem_optin);
cudaError_t launch_gateup_rows(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t smem_optin);
cudaError_t launch_down_rows(const LayerArgs& a, int grid, cudaStream_t s, bool pdl, size_t smem_optin);

}  // namespace moe
