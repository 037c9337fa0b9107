/*
 * moe_reader.h -- C ABI of the calibration-free sparse routed-expert reader
 * for MoE decoding at small batch, on NVIDIA B200 (sm_100a).
 *
 * The method ("Channel Selection for Mixture-of-Experts Decoding Needs No
 * Calibration Data", arXiv:2610.37386, abstract; "KAIST: MoE Decoding Needs
 * No Calibration Data", section "A reader that needs no data at all"): for
 * every (token, routed expert) pair the reader
 *   1. screens the expert's gate/up channels with a resident ternary sketch
 *      of the rotated gate/up weights, built from the weights alone;
 *   2. computes the surviving candidates exactly from the native BF16
 *      gate/up rows;
 *   3. keeps the token's top-k channels by |silu(g) * u| (no calibrated
 *      threshold: abstract, "top-k keeps each token's k highest-scoring
 *      channels");
 *   4. reads only those k rows of the down projection;
 *   5. adds back the skipped channels through a low-rank map of the down
 *      projection.
 *
 * Conventions for every entry point.
 *  - Tensors are dense row-major.  bf16 values are passed as uint16_t bit
 *    patterns.  Every pointer is a DEVICE pointer unless its name ends in
 *    _host, and must be 16-byte aligned.  The caller owns all memory; the
 *    library never allocates or frees device memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls only enqueue work; they never synchronize, except
 *    moe_reader_check_error.
 *  - Arguments are validated on the host before anything is enqueued.  On
 *    MOE_EINVAL / MOE_EUNSUPPORTED nothing was launched.  MOE_ECUDA means a
 *    launch failed.  moe_reader_last_error() describes the last non-OK
 *    status of the calling thread.
 *  - Device-side waits are bounded; a wait that runs out records an error
 *    word in the workspace (read with moe_reader_check_error) instead of
 *    hanging the GPU.
 *
 * Limits of this build: 256 <= d <= 4096 and d a power of two;
 * 16 <= I <= 2048; 1 <= k <= c <= I; r in {0, 8, 16, ..., 128} and r <= I;
 * 1 <= top_e <= min(E, 16); E <= 1024; 1 <= B <= 256.
 */
#ifndef MOE_READER_H
#define MOE_READER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_EINVAL = 1,       /* bad argument (null, misaligned, out of range)      */
  MOE_EUNSUPPORTED = 2, /* valid shape outside this build's compiled limits   */
  MOE_ECUDA = 3,        /* a CUDA launch or query failed                      */
  MOE_ETIMEOUT = 4,     /* a bounded device wait ran out (moe_reader_check_error) */
  MOE_EDEVICE = 5       /* a device-side check failed (moe_reader_check_error)  */
} moe_status;

/* One resident MoE layer: the weights and what the offline builders made
 * from them.  Per expert e, W_gate[e] and W_up[e] are [I, d] (row i =
 * channel i) and W_down[e] is stored channel-major, [I, d] (row i = the
 * output weights of channel i), so "read only the kept rows" reads whole
 * rows. */
typedef struct {
  int32_t E, I, d, top_e, r;
  const uint16_t* w_router;    /* [E, d] bf16                                    */
  const float* router_bias;    /* [E] fp32, or NULL (added to the logits)        */
  const uint16_t* w_gate;      /* [E, I, d] bf16                                 */
  const uint16_t* w_up;        /* [E, I, d] bf16                                 */
  const uint16_t* w_down;      /* [E, I, d] bf16, channel-major                  */
  const int8_t* rot_sign;      /* [d] +-1: the random signs of the rotation      */
  const void* sk_gate;         /* ternary sketch of W_gate, [E, I] rows in the
                                  layout sketch_format names (below)             */
  const void* sk_up;           /* ternary sketch of W_up, same layout             */
  const float* alpha_gate;     /* [E, I] per-row sketch scale                    */
  const float* alpha_up;       /* [E, I]                                         */
  const uint16_t* u_sigma;     /* [E, I, r] bf16 = U_r Sigma_r of W_down, or NULL */
  const uint16_t* v;           /* [E, d, r] bf16 = V_r of W_down, or NULL         */
  /* What the low-rank map recovers from ("A reader that needs no data at
   * all": skipped channels come back through the map).  0: the sketch
   * estimates ahat_i of every skipped channel, z = sum_{i not kept} ahat_i
   * Ubar_i.  1: the exact a_i of the candidates the top-k dropped (the exact
   * stage computed them) and ahat_i only outside the candidate set; it reads
   * no extra weight rows.  Any other value is MOE_EINVAL. */
  int32_t recovery_input;
  /* Which reader runs a sparse step.  Both compute the same routing, dots,
   * scores and candidate sets bit for bit, and outputs within the stated
   * tolerances.
   *   0  automatic: the one-cluster reader when B <= 2 and d <= 2048, the
   *      streamed reader otherwise;
   *   1  the one-cluster reader: one thread-block cluster per routed expert,
   *      every stage in one kernel (B <= 2 and d <= 2048, else
   *      MOE_EUNSUPPORTED);
   *   2  the streamed reader: after routing, five kernels (screen, top-c,
   *      exact candidates, top-k, down rows + combine), each over every
   *      (token, expert) pair of the step on all SMs.
   * Any other value is MOE_EINVAL.  The dense block ignores it. */
  int32_t path;
  /* CTAs per thread-block cluster of the cluster kernels (the one-cluster
   * reader, the dense block): 0 chooses per launch; 2 .. 16 pins the size
   * (MOE_ECUDA "invalid configuration" if that size does not fit the shape
   * on this device).  Other values are MOE_EINVAL. */
  int32_t cluster_size;
  /* Layout of the sketch rows sk_gate / sk_up point to (both readers decode
   * either; the trits, and so every dot, score and set, are the same).
   *   0  2-bit codes: [E, I, d/16] uint32 words as moe_reader_build_sketch
   *      writes them (d/4 bytes per row, 8.3% of the bf16 gate/up bytes);
   *   1  base 3: [E, I, moe_reader_sketch_row_bytes(d, 1)] bytes as
   *      moe_reader_sketch_to_base3 writes them, five trits per byte (416
   *      bytes per row at d = 2048, 6.8%; "A reader that needs no data at
   *      all" puts the resident sketch at about 7% of the BF16 checkpoint).
   * Other values are MOE_EINVAL; the dense block ignores the sketch. */
  int32_t sketch_format;
  /* Which experts' weights the per-expert arrays hold (expert parallelism
   * with a compacted layout): DEVICE [E] int32, expert_slot[e] = the index
   * of expert e in w_gate, w_up, w_down, sk_gate, sk_up, alpha_gate,
   * alpha_up, u_sigma and v, or -1 for an expert whose weights are not held;
   * those arrays then have max(slot) + 1 entries instead of E (the router
   * stays [E, d]).  A rank of an N-way expert-parallel step holding experts
   * e % N == rank passes slot[e] = e / N for those and -1 elsewhere, and
   * holds about E / N of the experts.  NULL: every array holds all E experts
   * (slot = e).  Read by the streamed reader only: with expert_slot set,
   * path 0 runs the streamed reader, path 1 and moe_reader_forward_dense
   * return MOE_EUNSUPPORTED.  A step that routes a token to an expert with
   * slot -1 reads slot 0 in its place and records device error bit 4
   * (moe_reader_check_error: MOE_EDEVICE); under moe_reader_forward_ep only
   * owned experts are read, so -1 is safe for every other expert. */
  const int32_t* expert_slot;
} moe_reader_layer;

/* Optional per-stage outputs of moe_reader_forward (each pointer may be
 * NULL; (b, s) = token b, routing slot s, slot 0 the highest logit). */
typedef struct {
  int32_t* ids;      /* [B, top_e] routed expert ids                             */
  float* weights;    /* [B, top_e] routing weights                               */
  int32_t* dot_gate; /* [B, top_e, I] exact integer sketch dots T^g . q          */
  int32_t* dot_up;   /* [B, top_e, I]                                            */
  float* score;      /* [B, top_e, I] screening score sigma                      */
  int32_t* cand;     /* [B, top_e, c] candidate channels, ascending              */
  int32_t* kept;     /* [B, top_e, k] kept channels, ascending                   */
  float* a_kept;     /* [B, top_e, k] exact silu(g)*u of the kept channels        */
  float* y_expert;   /* [B, top_e, d] fp32 expert output before the combine      */
  uint64_t* phase_ns; /* [B * top_e, 16] device clock (ns) at the stage
                         boundaries of the one-cluster reader, one row per work
                         item (its first CTA): 0 start, 1 tokens rotated,
                         2 router logits done, 3 logits exchanged, 4 item known,
                         5 screen done, 6 first exact rows started, 7 scores
                         exchanged, 8 candidates chosen, 9 exact stage done,
                         10 exact values exchanged, 11 kept chosen, 12 down
                         rows done, 13 partial outputs exchanged, 14 own
                         columns summed, 15 combined; 0 where a stage does not
                         run (the streamed reader writes none)               */
  /* Timing hooks (cudaEvent_t, or NULL): recorded on `stream` right before
   * and right after the expert kernels of this call.  They do not switch on
   * the per-stage outputs above. */
  void* ev_before;
  void* ev_after;
  /* Failure-detection hooks for tests (0 = off).  wait_limit_us: limit of
   * every bounded device wait of this call, in microseconds (default 2 s).
   * withhold_copy = 1: the one-cluster reader sets up, but never issues, one
   * of the sketch copies of each work item, so its bounded wait runs out;
   * the kernel still completes (with unusable outputs) and the error word
   * reads MOE_ETIMEOUT.  Any other value is MOE_EINVAL. */
  uint32_t wait_limit_us;
  int32_t withhold_copy;
} moe_reader_debug;

/* Bytes of device workspace moe_reader_forward / moe_reader_forward_dense
 * need for this shape (16-byte aligned base).  Zero-fill a workspace once
 * before its first use (it holds the device error word); the library keeps
 * the rest consistent from call to call.  A workspace must not be shared by
 * calls that may run concurrently. */
size_t moe_reader_workspace_bytes(int B, int E, int top_e, int I, int d, int k, int c, int r);

/* Offline: the rotated ternary sketch of every gate and up row ("A reader
 * that needs no data at all": a rotated ternary sketch of the gate/up
 * weights, resident on the GPU, built from the weights alone).
 *   rot_sign[j] = +1 if the top bit of output j of SplitMix64(rot_seed) is 0,
 *                 else -1 (Steele, Lea & Flood 2014);
 *   w' = H (rot_sign . w), H the unnormalised Sylvester Walsh-Hadamard
 *        transform (fp32, stages h = 1, 2, 4, ...);
 *   Delta = 0.7 * mean |w'| (fp64, index order); T_j = sign(w'_j) if
 *   |w'_j| > Delta else 0; alpha = mean |w'_j| over T_j != 0 (fp64, index
 *   order; 0 if none), stored fp32 (TWN, Li & Liu 2016).
 * Packing: 16 trits per uint32; word m of a row holds positions
 * 16m..16m+15; position 16m + 4p + b (p, b in 0..3) sits at bits
 * [8b + 2p, 8b + 2p + 1] as the code T + 1 (00 = -1, 01 = 0, 10 = +1).
 * Outputs are bit-identical to the reference definition above. */
moe_status moe_reader_build_sketch(int E, int I, int d, const uint16_t* w_gate, const uint16_t* w_up,
                                   uint64_t rot_seed, int8_t* rot_sign, uint32_t* sk_gate,
                                   uint32_t* sk_up, float* alpha_gate, float* alpha_up, void* stream);

/* Bytes of one sketch row of d trits in a sketch_format (0: d/4; 1: ceil(d/5)
 * rounded up to a multiple of 32); 0 for a d that is not a positive multiple
 * of 16 or an unknown format. */
size_t moe_reader_sketch_row_bytes(int d, int format);

/* Offline: repacks one sketch matrix from the 2-bit codes of
 * moe_reader_build_sketch ([E, I, d/16] words) to base 3 ([E, I,
 * moe_reader_sketch_row_bytes(d, 1)] bytes; sketch_format 1).  Byte g of a
 * row holds trits 5g .. 5g+4 as sum_i (T_{5g+i} + 1) 3^i (at most 242); the
 * last group's positions past d hold zero trits, and the bytes past
 * ceil(d/5) that pad the row to whole 32-byte sectors hold five zero trits
 * (121).  Five trits per byte is 1.6 bits per trit, against 2 for the codes:
 * the sketch's share of the bf16 gate/up bytes drops from 8.3% to 6.8% at
 * d = 2048 ("A reader that needs no data at all": about 7%).  Call it once
 * per matrix (gate, up); the input may be freed afterwards. */
moe_status moe_reader_sketch_to_base3(int E, int I, int d, const uint32_t* sk_codes, uint8_t* sk_base3,
                                      void* stream);

/* Offline: the low-rank map of the down projections ("A reader that needs
 * no data at all": skipped channels are recovered through a low-rank map of
 * the down projections).  Per expert, the rank-r truncated SVD
 * W_down[e] = U S V^T gives u_sigma = U[:, :r] S[:r] ([I, r]) and
 * v = V[:, :r] ([d, r]); in each column the entry of v with the largest
 * magnitude is positive (decided before the bf16 rounding).  Computed by subspace iteration on W W^T with a
 * Rayleigh-Ritz step; factors are rounded to bf16.
 * Needs moe_reader_lowrank_workspace_bytes(E, I, d, r) bytes of workspace. */
size_t moe_reader_lowrank_workspace_bytes(int E, int I, int d, int r);
moe_status moe_reader_build_lowrank(int E, int I, int d, int r, const uint16_t* w_down,
                                    uint16_t* u_sigma, uint16_t* v, void* workspace,
                                    size_t ws_bytes, void* stream);

/* One MoE block step over B tokens x [B, d] (bf16) -> y [B, d] (bf16).
 *   routing: logit_e = W_router[e] . x (+ bias_e), products exact, fp64 sums;
 *     top-`top_e` experts (ties: lower id), weights = softmax over the chosen
 *     logits (the abstract's "routed experts");
 *   per (token, expert): the reader steps 1-5 above with c candidates and
 *     k kept channels; the screening score of channel i is
 *     |silu(ghat_i) uhat_i| with ghat_i = ((float)G_i alpha_i) c_x,
 *     G_i = T_i . q exact, q = int8 quantisation of H (rot_sign . x),
 *     c_x = max|H (rot_sign . x)| / (127 d); candidates and kept sets break
 *     ties toward the lower channel;
 *   recovery (r > 0): + V z with z = sum over skipped channels of
 *     silu(ghat_i) uhat_i u_sigma[i, :];
 *   combine: y_b = sum over slots of w * y_e in fp32, rounded once to bf16;
 *     with `residual` (may be NULL) y_b += residual_b before the rounding.
 * Tokens routed to the same expert share its reads (one sketch read, the
 * union of their candidate and kept rows).  dbg may be NULL. */
moe_status moe_reader_forward(const moe_reader_layer* layer, int B, int k, int c,
                              const uint16_t* x, const uint16_t* residual, uint16_t* y,
                              const moe_reader_debug* dbg, void* workspace, size_t ws_bytes,
                              void* stream);

/* The dense all-channel MoE block on the same layer (same routing and
 * combine; every channel of every routed expert is read): the baseline the
 * reader is measured against. */
moe_status moe_reader_forward_dense(const moe_reader_layer* layer, int B, const uint16_t* x,
                                    const uint16_t* residual, uint16_t* y, void* workspace,
                                    size_t ws_bytes, void* stream);

/* Expert parallelism (one process per GPU, experts split by e % ep_size):
 * the step of rank ep_rank over the experts it owns.  Routing is computed in
 * full on every rank (the router is replicated); only the (token, slot)
 * pairs whose expert this rank owns are read and computed, with the
 * streamed kernels.  Writes y_partial[b] = sum over b's owned slots, in slot
 * order, of w_slot * y_e (DEVICE, [B, d] fp32, 16-byte aligned; no residual,
 * no rounding).  The caller sums y_partial over the ranks (e.g. one NCCL
 * all-reduce) and calls moe_reader_ep_finish.  The per-pair debug outputs
 * are written for owned pairs only.  Needs the layer's own weights for the
 * owned experts at least (other experts' rows are never read): with
 * layer->expert_slot, only the owned experts' weights, compacted.
 * MOE_EINVAL unless 1 <= ep_size <= E and 0 <= ep_rank < ep_size. */
moe_status moe_reader_forward_ep(const moe_reader_layer* layer, int B, int k, int c,
                                 const uint16_t* x, int ep_rank, int ep_size, float* y_partial,
                                 const moe_reader_debug* dbg, void* workspace, size_t ws_bytes,
                                 void* stream);

/* y = bf16(y_sum + residual) (round to nearest even), [B, d]: the last step
 * of an expert-parallel block after the partials are summed.  residual may
 * be NULL; DEVICE pointers. */
moe_status moe_reader_ep_finish(int B, int d, const float* y_sum, const uint16_t* residual,
                                uint16_t* y, void* stream);

/* moe_reader_forward with HOST input and output: copies x_host ([B, d]
 * bf16) into x_dev, runs the step, copies y_dev back into y_host, all
 * enqueued on `stream` after the arguments are validated.  The caller
 * synchronizes.  Page-locked host buffers the device can address (pinned
 * memory under unified addressing, 16-byte aligned) are copied by small
 * kernels on the SMs, chained to the step by programmatic dependent launch:
 * for a few kilobytes that is several microseconds faster than a DMA-engine
 * copy.  Other host memory is copied with cudaMemcpyAsync. */
moe_status moe_reader_forward_host(const moe_reader_layer* layer, int B, int k, int c,
                                   const uint16_t* x_host, uint16_t* x_dev, uint16_t* y_dev,
                                   uint16_t* y_host, void* workspace, size_t ws_bytes, void* stream);

/* moe_reader_forward with no caller-provided workspace, for callers that
 * cannot allocate device memory: serving loops that forbid any allocation
 * after start-up so that their memory footprint stays fixed, and hosts whose
 * device memory is owned by another runtime's allocator, which this library
 * cannot call.  (The paper has no counterpart; this is an interface
 * convenience.)
 *  - The scratch is a fixed 8 MiB __device__ array inside the library; every
 *    GPU that loads the library holds it until the process exits.  Shapes
 *    whose workspace (moe_reader_workspace_bytes) exceeds 8 MiB return
 *    MOE_EINVAL ("workspace has ... bytes, needs ...") and launch nothing.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) once and keeps it for later calls.
 *  - Every call shares the one array per device: calls that may overlap on
 *    the GPU (different streams, no ordering) race and must not be issued.
 *    Each call first clears the array's combine counters (cudaMemsetAsync on
 *    `stream`, after the arguments were validated); nothing is allocated or
 *    freed.
 *  - No debug outputs.  Argument errors as for moe_reader_forward; a bounded
 *    device wait that ran out sets the array's error word, which
 *    moe_reader_check_error(NULL, stream) reads and clears. */
moe_status moe_reader_forward_noalloc(const moe_reader_layer* layer, int B, int k, int c,
                                      const uint16_t* x, const uint16_t* residual, uint16_t* y, void* stream);

/* Between stacked layers: h = bf16(x / sqrt(mean(x^2) + eps)) per token,
 * no learned gain (fp32). */
moe_status moe_reader_rmsnorm(int B, int d, float eps, const uint16_t* x, uint16_t* h, void* stream);

/* The launch the cluster kernel would use for this shape on the current
 * device with an automatic cluster size (dense != 0: the dense block; else
 * the one-cluster reader, B <= 2): out4 = {cluster size, copy-ring rows (dense:
 * per warp; reader: exact-stage row slots per CTA), dynamic shared memory
 * bytes per CTA, co-resident clusters}. */
moe_status moe_reader_launch_plan(int dense, int B, int E, int top_e, int I, int d, int r, int32_t* out4);

/* Synchronizes `stream`, reads and clears the workspace's device error word
 * (workspace NULL: the error word of moe_reader_forward_noalloc's scratch on
 * the current device).  Returns MOE_OK; MOE_ETIMEOUT if a bounded wait ran
 * out since the last check (bit 1); otherwise MOE_EDEVICE for the other
 * device-side checks (bit 2: a work item out of range; bit 4: a routed
 * expert without a weight slot, see moe_reader_layer.expert_slot).  The
 * message names the bits. */
moe_status moe_reader_check_error(void* workspace, void* stream);

/* Message for the last non-OK status returned on this thread. */
const char* moe_reader_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_READER_H */
