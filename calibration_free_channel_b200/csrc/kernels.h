// kernels.h -- argument blocks and launchers of the reader's kernels.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_reader.h"

namespace moe {

// Records the message returned by moe_reader_last_error and returns st.
moe_status set_last_error(moe_status st, const char* msg);
// moe_reader_forward on a given scratch buffer whose combine counters are
// cleared after validation, before any launch (the noalloc entry).
moe_status forward_scratch(const moe_reader_layer* layer, int B, int k, int c, const uint16_t* x,
                           const uint16_t* residual, uint16_t* y, void* scratch, size_t bytes, void* stream);
// Device address of the noalloc entry's scratch array on the current device
// (looked up on the first call on each device); nullptr and *err on failure.
void* noalloc_scratch(cudaError_t* err);

// Workspace carved out of the caller's buffer (see workspace_layout).
struct Workspace {
  uint32_t* err;        // [1] device error word
  int* n_items;         // [1] number of work items this step
  double* logits;       // [B, E]
  int* ids;             // [B, top_e]
  float* wts;           // [B, top_e]
  int8_t* q;            // [B, d] int8 rotated activations
  float* cx;            // [B] dequantisation scale
  int* item_e;          // [max_items]
  int* item_n;          // [max_items]
  int* item_tok;        // [max_items, kMaxGroup]
  int* item_slot;       // [max_items, kMaxGroup]
  float* ye;            // [B, top_e, d] per-expert outputs (fp32)
  unsigned* counters;   // [B, kMaxCluster] arrival counters of the combine
  int max_items;
  // The streamed path (stream.cu).  Pairs (token, slot) are numbered in
  // expert order, tokens ascending within an expert; W = ceil(I / 32).
  int* qsum;            // [B] sum of each token's int8 activations (the code offset)
  int* n_act;           // [1] experts chosen by at least one token this step
  int* act_e;           // [E] those experts, ascending
  int* act_w;           // [E] their weight slots (index into the per-expert arrays)
  int* act_off;         // [E + 1] first pair of each (act_off[n_act] = B * top_e)
  int* pair_tok;        // [P] token of each pair
  int* pair_slot;       // [P] routing slot of each pair
  int* pair_ea;         // [P] active-expert index of each pair
  unsigned* arrive;     // [2, E] arrival counters of the two selection kernels
  float2* sa;           // [P, I] (sigma, ahat) of every channel
  float* zpart;         // [P, ceil(I / 16), r] recovery-input partials of the screen blocks
  uint32_t* candm;      // [P, W] candidate bit masks
  float* apos;          // [P, I] exact a of each pair's candidates (by channel)
  uint32_t* keptm;      // [P, W] kept bit masks
  float* z;             // [P, r] recovery input of each pair
  int* ulist;           // [E, I] candidate union of each active expert, ascending
  int* n_u;             // [E]
  int* dlist;           // [E, I] kept union of each active expert, ascending
  int* n_d;             // [E]
  float* coef;          // [P, I] each pair's coefficient of its expert's kept-union rows
};

// I and r size the streamed path's buffers (pass 0 for none).
size_t workspace_layout(int B, int E, int top_e, int d, int I, int r, void* base, Workspace* ws);
int max_work_items(int B, int E, int top_e, int group);

struct RouteArgs {
  int B, E, d, top_e, cs;
  const uint16_t* x;
  const uint16_t* w_router;
  const float* bias;
  const int8_t* rot_sign;
  Workspace ws;
  int32_t* dbg_ids;
  float* dbg_w;
  bool quantize;  // also rotate + quantize the tokens (sparse path)
  int ep_rank, ep_size;  // expert parallelism: pairs of experts e % ep_size == ep_rank only (ep_size 0/1: all)
  const int32_t* expert_slot;  // [E] weight slot of each expert (< 0: none held), or null (slot = e)
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);

struct ExpertArgs {
  int B, E, top_e, I, d, k, c, r;
  int cs;            // CTAs per cluster (one cluster per work item)
  int force_cs;      // 0: cluster size chosen per launch; else this size
  int nmax;          // max tokens per work item this launch
  int ring_rows;     // copy-ring row slots per warp (sparse) / rows (dense)
  int recovery_input;  // 0: ahat of every skipped channel; 1: exact a of dropped candidates
  unsigned long long wait_ns;  // limit of every bounded copy wait (test hook; kWaitLimitNs normally)
  int withhold_copy;           // test hook: 1 = the one-cluster reader never issues one sketch copy
  int ep_partial;      // 1: write the per-slot outputs only (no combine); expert-parallel steps
  int sk3;             // sketch rows: 0 2-bit codes (d / 4 bytes), 1 base 3 (sk3_row_bytes(d) bytes)
  const uint16_t* x;
  const uint16_t* w_router;  // routing inside the expert kernel (small B)
  const float* bias;
  const int8_t* rot_sign;
  const uint16_t* w_gate;
  const uint16_t* w_up;
  const uint16_t* w_down;
  const uint32_t* sk_gate;
  const uint32_t* sk_up;
  const float* alpha_gate;
  const float* alpha_up;
  const uint16_t* u_sigma;
  const uint16_t* v;
  const uint16_t* residual;
  uint16_t* y;
  Workspace ws;
  // debug outputs (may be null)
  int32_t* dbg_ids;
  float* dbg_w;
  int32_t* dbg_G;
  int32_t* dbg_U;
  float* dbg_sigma;
  int32_t* dbg_cand;
  int32_t* dbg_kept;
  float* dbg_a_kept;
  float* dbg_y_expert;
  unsigned long long* dbg_phase;
};
// Steps of at most this many tokens route inside the expert kernel (one
// launch per step); larger steps use the route and select kernels first.
bool fused_routing(int B);
// The one-cluster reader (reader.cu) runs steps of at most two tokens with
// d <= 2048.
bool reader_supports(int B, int d);
cudaError_t launch_reader(const ExpertArgs& a, cudaStream_t s);
// The streamed reader: screen, top-c, exact candidates, top-k, down rows +
// combine, each one kernel over every pair of the step (after launch_route).
cudaError_t launch_stream(const ExpertArgs& a, cudaStream_t s);
// Expert parallelism: y_partial[b] = sum over the slots of b whose expert this
// rank owns of w * y_e (fp32, slot order); y = bf16(y_sum + residual).
cudaError_t launch_ep_combine(int B, int top_e, int d, int ep_rank, int ep_size, const Workspace& ws,
                              float* y_partial, cudaStream_t s);
cudaError_t launch_ep_finish(int B, int d, const float* y_sum, const uint16_t* residual, uint16_t* y,
                             cudaStream_t s);
cudaError_t launch_dense(const ExpertArgs& a, cudaStream_t s);
cudaError_t query_plan(const ExpertArgs& a, bool dense, int out[4]);

cudaError_t launch_build_sketch(int E, int I, int d, const uint16_t* w_gate, const uint16_t* w_up,
                                uint64_t seed, int8_t* rot_sign, uint32_t* sk_gate, uint32_t* sk_up,
                                float* alpha_gate, float* alpha_up, cudaStream_t s);
// Repacks rows of 2-bit codes ([rows, d / 16] words) as base-3 rows
// ([rows, sk3_row_bytes(d)] bytes).
cudaError_t launch_sketch_to_base3(long rows, int d, const uint32_t* codes, uint8_t* out, cudaStream_t s);
size_t lowrank_ws_bytes(int E, int I, int d, int r);
cudaError_t launch_build_lowrank(int E, int I, int d, int r, const uint16_t* w_down, uint16_t* u_sigma,
                                 uint16_t* v, void* ws, cudaStream_t s);
cudaError_t launch_rmsnorm(int B, int d, float eps, const uint16_t* x, uint16_t* h, cudaStream_t s);
// bytes (a multiple of 16) from src to dst with 16-byte loads and stores on the
// SMs (either side may be device-addressable host memory); chained to the
// previous kernel by programmatic dependent launch.
cudaError_t launch_copy16(const void* src, void* dst, size_t bytes, cudaStream_t s);

}  // namespace moe
