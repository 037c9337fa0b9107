// reader.cu -- the sparse routed-expert reader and the dense baseline block.
//
// One thread-block cluster (cs CTAs, 8 <= cs <= 16) runs one work item: an
// expert e and the tokens routed to it (up to NT), so tokens that share an
// expert share its reads.  The reader's steps ("Channel Selection for
// Mixture-of-Experts Decoding Needs No Calibration Data", abstract; "KAIST:
// MoE Decoding Needs No Calibration Data", section "A reader that needs no
// data at all"):
//   R  (B <= 2) routing inside the cluster: every CTA computes the logits of
//      its slice of experts and pushes them to all CTAs; every CTA then takes
//      the same top-e and finds its cluster's work item;
//   S  screen: every CTA reads the ternary sketch rows of its slice of the I
//      channels, forms exact integer dots with the int8 rotated token and the
//      screening score sigma = |silu(ghat) uhat|, and pushes sigma (and the
//      estimate ahat) to every CTA of the cluster;           cluster barrier
//   c  every CTA selects the same top-c candidates per token (ties: lower
//      channel);
//   C  exact: the CTAs split the union of the candidates, read the BF16 gate
//      and up rows, compute a = silu(g) u and push it to every CTA;
//                                                           cluster barrier
//   k  every CTA selects the same top-k per token by |a|: the top-k keep rule,
//      no calibrated threshold;
//   D  down + recovery: every CTA reads its column slice of the kept down
//      rows (with the kept rows of the factor Ubar = U_r S_r) and forms
//      y_e = sum_K a_i W_down[i,:] + V z, z = sum_{i not in K} ahat_i Ubar_i;
//   combine: the last of a token's top_e experts to finish a column slice sums
//      w_s y_e,s in slot order, writes bf16 y and resets the slice's counter.
//
// Large contiguous rows (sketch chunks of 16 channels, BF16 gate/up rows)
// move with 1-D bulk copies (cp.async.bulk) into shared memory, waited on
// through mbarriers with bounded waits.  The many short row slices of the
// down stage are plain 16-byte loads spread over all threads: a bulk copy
// costs the SM's copy engine a fixed issue time per copy, which dominates
// for slices of a few hundred bytes.  Every exchange between the CTAs of a
// cluster is a store into the receivers' shared memory followed by a cluster
// barrier: no CTA reads another CTA's shared memory.
//
// At batch 1 the step is a chain of short dependent stages, so the kernels
// are written for latency: few block barriers per stage, no serial loops over
// warps, the rotation placed under the sketch's DRAM latency, the screen's
// byte-wise dots on pre-masked code words.
//
// Two kernels implement these steps.  reader1_kernel (one-token steps on
// 2-bit sketch rows) follows the stages above as written.  reader_kernel
// (two-token steps, base-3 rows, pinned clusters below 8 CTAs) keeps each
// CTA's channel slice through the whole step: the selections count ranks
// over sorted lists the CTAs exchange, and the exact and down rows of the
// likely channels start before the selections end; it is faster at two
// tokens and slower at one (see the note above reader1_kernel).
#include "common.cuh"
#include "kernels.h"
#include "rotate.cuh"
#include "select.cuh"

namespace moe {

namespace {

constexpr int NTHR = 512;
constexpr int NWARP = NTHR / 32;
constexpr int kMaxCols = 256;  // output columns per CTA
constexpr int kSkBars = 16;    // sketch chunk barriers (a chunk is 16 channels)
constexpr unsigned kFull = 0xffffffffu;

__host__ __device__ inline int rup(int x, int a) { return (x + a - 1) / a * a; }
__host__ __device__ inline int cdiv(int x, int a) { return (x + a - 1) / a; }

// One shared copy of a runtime integer division (kernel code stays small).
__device__ __noinline__ int idiv(int a, int b) { return a / b; }

// ------------------------------------------------------- launch geometry
// Shared-memory offsets and the partitions of a launch, computed on the host.
struct Layout {
  int mbar, misc, hist, x, q, logit, alpha, sig, sa, zred, zparts, z, apos, candm, keptm, ulist, dlist, keys,
      ubar, vown, ring, total;
  int ntok;        // tokens held in smem (fused routing: B; otherwise NT)
  int own_max;     // max channels per CTA
  int cols_max;    // max output columns per CTA
  int words;       // mask words over I
  int ring_bytes;  // per warp
  int d8, d64;     // d / 8, d / 64
  int c_slots;     // candidate row slots (gate + up) per warp
  int skc;         // bytes of 16 sketch rows of one matrix
  int sk_round;    // sketch chunks resident at once
  int ch0[17];     // channel partition over the CTAs of a cluster (multiples of 4)
  int col0[17];    // output-column partition (multiples of 8)
  int ex0[17];     // expert partition (in-kernel routing)
};

__host__ inline Layout make_layout(int NT, int ntok, bool fused, int E, int I, int d, int r, int cs,
                                   int ring_rows, bool dense) {
  Layout L = {};
  L.ntok = ntok;
  for (int o = 0; o <= cs && o < 17; o++) {
    const int c4 = 4 * cdiv(o * cdiv(I, 4), cs);
    L.ch0[o] = c4 < I ? c4 : I;
  }
  L.own_max = 0;
  for (int o = 0; o < cs && o < 16; o++)
    if (L.ch0[o + 1] - L.ch0[o] > L.own_max) L.own_max = L.ch0[o + 1] - L.ch0[o];
  L.cols_max = 8 * cdiv(d / 8, cs);
  L.words = cdiv(I, 32);
  L.ring_bytes = ring_rows * d * 2;
  L.d8 = d / 8;
  L.d64 = d / 64;
  L.c_slots = L.ring_bytes / (4 * d);
  L.skc = 16 * (d / 4);
  for (int o = 0; o <= cs && o < 17; o++) {
    L.col0[o] = 8 * cdiv(o * (d / 8), cs);
    L.ex0[o] = cdiv(o * E, cs);
  }
  const int rr = r > 0 ? r : 1;
  int o = 0;
  auto take = [&](int bytes) {
    int at = o;
    o = rup(o + bytes, 128);
    return at;
  };
  L.mbar = take((NWARP * kMaxSlots + kSkBars + 2) * 8);
  L.misc = take(256 * 4);
  L.hist = take(2 * 2048 * 4);
  L.x = take(ntok * d * 2);
  L.q = dense ? 0 : take(ntok * d);
  L.logit = fused ? take(ntok * E * 8) : 0;
  L.alpha = dense ? 0 : take(2 * L.own_max * 4);
  L.sig = dense ? take(NT * I * 4) : 0;           // dense: h by channel
  L.sa = dense ? 0 : take(rup(I, 4) * NT * 8);    // sparse: (sigma, ahat) by channel, token
  L.zred = dense ? 0 : take(NWARP * NT * rr * 4);
  L.zparts = dense ? 0 : take(cs * NT * rr * 4);
  L.z = dense ? 0 : take(NT * rr * 4);
  L.apos = dense ? 0 : take(NT * I * 4);  // a by union position
  L.candm = dense ? 0 : take(NT * L.words * 4);
  L.keptm = dense ? 0 : take(NT * L.words * 4);
  L.ulist = dense ? 0 : take(I * 4);
  L.dlist = dense ? 0 : take(I * 4);
  L.keys = dense ? 0 : take(I * 4);
  L.ubar = dense ? 0 : take(L.own_max * rr * 2);
  L.vown = dense ? 0 : take(L.cols_max * rr * 2);
  L.ring = take(NWARP * L.ring_bytes);
  L.total = o;
  const int region = NWARP * L.ring_bytes;
  int rounds = (region - 4 * d) / (2 * L.skc);
  if (rounds > kSkBars) rounds = kSkBars;
  if (rounds > cdiv(L.own_max, 16)) rounds = cdiv(L.own_max, 16);
  L.sk_round = dense ? 0 : (rounds > 0 ? rounds : 0);
  return L;
}

// misc ints
enum {
  MI_E = 0, MI_N, MI_NU, MI_ND, MI_DIG, MI_REM, MI_CNT, MI_DONE = 12,
  MI_TOK = 16, MI_SLOT = 32, MI_LAST = 48, MI_TIX = 64, MI_CX = 80, MI_RED = 96, MI_WT = 112,
  MI_RIDS = 128,  // in-kernel routing: ids [B <= 2][top_e <= 16]
  MI_RW = 192,    // in-kernel routing: weights
  MI_FID = 224    // in-kernel routing: first-occurrence ids
};
static_assert(MI_DIG == sel::kSelDig && MI_REM == sel::kSelRem && MI_CNT == sel::kSelCnt && MI_WT == sel::kSelWt,
              "selection scratch positions");
static_assert(NTHR == sel::kSelThreads, "the selections run on whole 512-thread CTAs");
using sel::block_mask_to_list;
using sel::block_select_top;


// ---------------------------------------------------------- cluster helpers
__device__ __forceinline__ int cluster_id() {
  int c;
  asm("mov.u32 %0, %%clusterid.x;" : "=r"(c));
  return c;
}
__device__ __forceinline__ uint32_t cluster_addr(const void* local, int rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
  return ra;
}
__device__ __forceinline__ void st_cluster(const void* local, int rank, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr(local, rank)), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster(const void* local, int rank, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr(local, rank)), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_cluster(const void* local, int rank, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(cluster_addr(local, rank)), "d"(v) : "memory");
}

// -------------------------------------------------------- mixed-precision dot
// 8 bf16 x 8 bf16 accumulated in fp32: fma.rn.f32.bf16 multiplies the bf16
// operands exactly and rounds once into the fp32 accumulator (two chains).
__device__ __forceinline__ void dot8_mixed(uint4 a, uint4 b, float& acc0, float& acc1) {
  asm("{\n\t.reg .b16 a0, a1, a2, a3, a4, a5, a6, a7, b0, b1, b2, b3, b4, b5, b6, b7;\n\t"
      "mov.b32 {a0, a1}, %2;\n\tmov.b32 {a2, a3}, %3;\n\tmov.b32 {a4, a5}, %4;\n\tmov.b32 {a6, a7}, %5;\n\t"
      "mov.b32 {b0, b1}, %6;\n\tmov.b32 {b2, b3}, %7;\n\tmov.b32 {b4, b5}, %8;\n\tmov.b32 {b6, b7}, %9;\n\t"
      "fma.rn.f32.bf16 %0, a0, b0, %0;\n\tfma.rn.f32.bf16 %1, a1, b1, %1;\n\t"
      "fma.rn.f32.bf16 %0, a2, b2, %0;\n\tfma.rn.f32.bf16 %1, a3, b3, %1;\n\t"
      "fma.rn.f32.bf16 %0, a4, b4, %0;\n\tfma.rn.f32.bf16 %1, a5, b5, %1;\n\t"
      "fma.rn.f32.bf16 %0, a6, b6, %0;\n\tfma.rn.f32.bf16 %1, a7, b7, %1;\n\t}"
      : "+f"(acc0), "+f"(acc1)
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w));
}

// --------------------------------------------------------- per-warp rings
// A warp streams `cnt` elements through P slots of its ring.  Lane 0 issues
// element j into slot j % P (issue(j, slot, bar)); all lanes consume it after
// a bounded wait.  `par` holds the parity bit of each slot barrier and
// persists across stages.  Returns false if a wait ran out (the warp then
// stops issuing and drains what is in flight).
template <class Issue, class Consume>
__device__ __forceinline__ bool warp_stream(int cnt, int P, uint64_t* bars, uint32_t& par, uint32_t* err,
                                            Issue issue, Consume consume,
                                            unsigned long long limit_ns = kWaitLimitNs) {
  const int lane = threadIdx.x & 31;
  if (cnt <= 0) return true;
  P = min(P, cnt);
  uint32_t pend = 0;
  if (lane == 0) fence_proxy_async();  // the ring may have been read by generic loads
#pragma unroll 1
  for (int j = 0; j < P; j++) {
    if (lane == 0) issue(j, j, &bars[j]);
    pend |= 1u << j;
  }
  __syncwarp();
  bool ok = true;
  int s = 0;
#pragma unroll 1
  for (int j = 0; j < cnt; j++) {
    ok = mbar_wait_bounded(&bars[s], (par >> s) & 1u, err, limit_ns);
    if (!ok) break;
    par ^= 1u << s;
    pend &= ~(1u << s);
    consume(j, s);
    __syncwarp();
    if (j + P < cnt) {
      if (lane == 0) {
        fence_proxy_async();
        issue(j + P, s, &bars[s]);
      }
      pend |= 1u << s;
      __syncwarp();
    }
    s = s + 1 == P ? 0 : s + 1;
  }
  if (!ok) {
#pragma unroll 1
    for (int q = 0; q < P; q++)
      if ((pend >> q) & 1u)
        if (mbar_wait_bounded(&bars[q], (par >> q) & 1u, err, limit_ns)) par ^= 1u << q;
  }
  return ok;
}

// ------------------------------------------------------- work item set-up
// The item comes from the work table the select kernel wrote (warp 0 reads
// its fields in parallel).
__device__ bool load_item_table(const ExpertArgs& a, int cid, int* misc, int NT) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const bool ok_cid = cid < a.ws.max_items;
    // written by the previous kernel of the step: read through L2
    int v = 0;
    if (lane == 0) v = __ldcg(a.ws.n_items);
    else if (lane == 1 && ok_cid) v = __ldcg(a.ws.item_e + cid);
    else if (lane == 2 && ok_cid) v = __ldcg(a.ws.item_n + cid);
    else if (lane >= 4 && lane < 4 + kMaxGroup && ok_cid) v = __ldcg(a.ws.item_tok + cid * kMaxGroup + lane - 4);
    else if (lane >= 8 && lane < 8 + kMaxGroup && ok_cid) v = __ldcg(a.ws.item_slot + cid * kMaxGroup + lane - 8);
    const int n_items = __shfl_sync(kFull, v, 0);
    int e = __shfl_sync(kFull, v, 1), n = __shfl_sync(kFull, v, 2);
    if (!(cid < n_items && ok_cid)) {
      e = -1;
      n = 0;
    } else if (e < 0 || e >= a.E || n < 1 || n > NT) {
      if (lane == 0) atomicOr(a.ws.err, kErrBadWorkItem);
      e = -1;
      n = 0;
    }
    const int t = lane;
    int tok = __shfl_sync(kFull, v, 4 + (t & 3)), sl = __shfl_sync(kFull, v, 8 + (t & 3));
    if (t < n) {
      if (tok < 0 || tok >= a.B || sl < 0 || sl >= a.top_e) {
        atomicOr(a.ws.err, kErrBadWorkItem);
        tok = 0;
        sl = 0;
      }
      misc[MI_TOK + t] = tok;
      misc[MI_SLOT + t] = sl;
      misc[MI_TIX + t] = t;  // tokens are loaded in item order
      reinterpret_cast<float*>(misc + MI_CX)[t] = __ldcg(a.ws.cx + tok);
    }
    if (lane == 0) {
      misc[MI_E] = e;
      misc[MI_N] = n;
    }
  }
  __syncthreads();
  return misc[MI_E] >= 0;
}

// Loads the item's tokens (misc[MI_TOK + t] -> smem token t): x and, for the
// sparse reader, q.
__device__ void load_tokens(const ExpertArgs& a, const Layout& L, char* smem, const int* misc, int n, bool with_q) {
  uint4* xs = reinterpret_cast<uint4*>(smem + L.x);
  uint4* qs = reinterpret_cast<uint4*>(smem + L.q);
#pragma unroll 1
  for (int t = 0; t < n; t++) {
    const int tok = misc[MI_TOK + t];
    for (int j = threadIdx.x; j < L.d8; j += NTHR)
      xs[t * L.d8 + j] = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)tok * a.d) + j);
    if (with_q)
      for (int j = threadIdx.x; j < L.d8 / 2; j += NTHR)
        qs[t * (L.d8 / 2) + j] = __ldcg(reinterpret_cast<const uint4*>(a.ws.q + (size_t)tok * a.d) + j);
  }
}

// Stage time stamps (globaltimer, ns) of the first CTA of each cluster.
__device__ __forceinline__ void stamp(const ExpertArgs& a, int cid, int rank, int k) {
  if (a.dbg_phase && rank == 0 && threadIdx.x == 0) a.dbg_phase[cid * 16 + k] = global_ns();
}

// 8 consecutive 16-byte vectors per lane (j = j0 + 32u + lane), zero past d8.
__device__ __forceinline__ void load_row8(const uint4* row, int j0, int d8, int lane, uint4 (&w)[8]) {
#pragma unroll
  for (int u = 0; u < 8; u++) {
    const int j = j0 + 32 * u + lane;
    w[u] = j < d8 ? ld_stream(row + j) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// In-kernel routing (B <= NT <= 2): every CTA loads all tokens and computes
// the logits of its slice of experts (one warp per expert; the router row is
// read straight into registers, overlapping the token loads) and pushes them
// to all CTAs; after the cluster barrier every CTA takes the same top-e and
// one warp derives the softmax weights and this cluster's work item (one
// item per routed expert, experts ascending).  `mid()` runs once the tokens
// are in shared memory, while the router rows are still in flight.  Returns
// false if this cluster has no item.
template <int NT, class LT, class Mid>
__device__ bool fused_route(const ExpertArgs& a, const LT& L, char* smem, int* misc, int cs, int rank, int cid,
                            cg::cluster_group& cluster, Mid mid) {
  const int B = a.B, E = a.E, top = a.top_e;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e0 = L.ex0[rank], ne = L.ex0[rank + 1] - e0;
  uint4* xs = reinterpret_cast<uint4*>(smem + L.x);
  // the tokens first (every later step needs them), then the router rows
  uint4 xv[NT][2];
#pragma unroll
  for (int t = 0; t < NT; t++)
#pragma unroll
    for (int k = 0; k < 2; k++) {
      const int j = threadIdx.x + k * NTHR;
      xv[t][k] = t < B && j < L.d8 ? __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d) + j)
                                   : make_uint4(0u, 0u, 0u, 0u);
    }
  uint4 w[8];
  double bias_w = 0.0;
  if (warp < ne) {
    load_row8(reinterpret_cast<const uint4*>(a.w_router + (size_t)(e0 + warp) * a.d), 0, L.d8, lane, w);
    if (a.bias) bias_w = (double)__ldg(a.bias + e0 + warp);
  }
#pragma unroll
  for (int t = 0; t < NT; t++)
#pragma unroll
    for (int k = 0; k < 2; k++) {
      const int j = threadIdx.x + k * NTHR;
      if (t < B && j < L.d8) xs[t * L.d8 + j] = xv[t][k];
    }
  if (threadIdx.x < B) misc[MI_TOK + threadIdx.x] = threadIdx.x;
  __syncthreads();
  mid();
  // logit_e = sum_j W_r[e, j] x_j (+ b_e): bf16 products are exact in fp32
  // (8-bit significands; products below 2^-126 in magnitude excepted) and are
  // summed in fp64
  double* lg = reinterpret_cast<double*>(smem + L.logit);
#pragma unroll 1
  for (int el = warp; el < ne; el += NWARP) {
    const uint4* row = reinterpret_cast<const uint4*>(a.w_router + (size_t)(e0 + el) * a.d);
    double acc0[NT], acc1[NT];
#pragma unroll
    for (int t = 0; t < NT; t++) acc0[t] = acc1[t] = 0.0;
#pragma unroll 1
    for (int j0 = 0; j0 < L.d8; j0 += 256) {
      if (el != warp || j0 != 0) load_row8(row, j0, L.d8, lane, w);
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const int j = j0 + 32 * u + lane;
        if (j < L.d8) {
#pragma unroll
          for (int t = 0; t < NT; t++) {
            const uint4 xv = xs[(t < B ? t : 0) * L.d8 + j];
            acc0[t] += (double)__fmul_rn(bf16lo(w[u].x), bf16lo(xv.x));
            acc1[t] += (double)__fmul_rn(bf16hi(w[u].x), bf16hi(xv.x));
            acc0[t] += (double)__fmul_rn(bf16lo(w[u].y), bf16lo(xv.y));
            acc1[t] += (double)__fmul_rn(bf16hi(w[u].y), bf16hi(xv.y));
            acc0[t] += (double)__fmul_rn(bf16lo(w[u].z), bf16lo(xv.z));
            acc1[t] += (double)__fmul_rn(bf16hi(w[u].z), bf16hi(xv.z));
            acc0[t] += (double)__fmul_rn(bf16lo(w[u].w), bf16lo(xv.w));
            acc1[t] += (double)__fmul_rn(bf16hi(w[u].w), bf16hi(xv.w));
          }
        }
      }
    }
    const int e = e0 + el;
    const double bias = el == warp ? bias_w : a.bias ? (double)a.bias[e] : 0.0;
#pragma unroll
    for (int t = 0; t < NT; t++) {
      const double s = warp_sum(acc0[t] + acc1[t]) + bias;
      if (t < B && lane < cs) st_cluster(&lg[t * E + e], lane, s);
    }
  }
  stamp(a, cid, rank, 2);
  cluster.sync();
  stamp(a, cid, rank, 3);
  // top-e per token by rank: 4 threads per expert count the logits that beat
  // it (larger, or equal with a lower id); rank < top_e is chosen
  int* rids = misc + MI_RIDS;
#pragma unroll 1
  for (int b = 0; b < B; b++) {
    const double* lb = lg + b * E;
    for (int task = threadIdx.x; task < rup(4 * E, 32); task += NTHR) {
      int cnt = 0;
      const int e = task >> 2, qtr = task & 3;
      if (e < E) {
        const double l = lb[e];
        for (int e2 = qtr; e2 < E; e2 += 4) {
          const double l2 = lb[e2];
          cnt += (l2 > l) || (l2 == l && e2 < e);
        }
      }
      cnt += __shfl_xor_sync(kFull, cnt, 1);
      cnt += __shfl_xor_sync(kFull, cnt, 2);
      if (e < E && qtr == 0 && cnt < top) rids[b * top + cnt] = e;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // work table: distinct experts ascending; item cid = the cid-th of them
    const int nent = B * top;  // <= 32
    const bool act = lane < nent;
    const int b = act && lane >= top ? 1 : 0;
    const int id = act ? rids[lane] : 0x7fffffff;
    bool first = act;
    if (B > 1) {
      const unsigned same = __match_any_sync(kFull, id);
      first = act && __ffs(same) - 1 == lane;
    }
    int* fid = misc + MI_FID;
    fid[lane] = first ? id : 0x7fffffff;
    __syncwarp();
    int rk = 0;
#pragma unroll 1
    for (int j4 = 0; j4 < nent; j4 += 4) {
      const int4 f = reinterpret_cast<const int4*>(fid)[j4 >> 2];
      rk += (f.x < id) + (f.y < id) + (f.z < id) + (f.w < id);
    }
    const unsigned mine = __ballot_sync(kFull, first && rk == cid);
    const int e_item = mine ? __shfl_sync(kFull, id, __ffs(mine) - 1) : -1;
    const bool on = act && e_item >= 0 && id == e_item;
    const unsigned bal = __ballot_sync(kFull, on);
    if (on) {
      const int at = __popc(bal & ((1u << lane) - 1u));
      misc[MI_TOK + at] = b;
      misc[MI_SLOT + at] = lane - b * top;
      misc[MI_TIX + at] = b;
    }
    if (lane == 0) {
      misc[MI_E] = e_item;
      misc[MI_N] = __popc(bal);
    }
  }
  __syncthreads();
  return misc[MI_E] >= 0;
}

// Routing weights of the in-kernel router (one warp, off the critical path):
// softmax over the chosen logits, summed in slot order (fp32 exponentials of
// the fp64 logit differences; the weights only scale outputs).
template <class LT>
__device__ void route_weights(const ExpertArgs& a, const LT& L, char* smem, int* misc, int cid, int rank) {
  const int lane = threadIdx.x & 31;
  const int top = a.top_e, nent = a.B * top;
  const double* lg = reinterpret_cast<const double*>(smem + L.logit);
  const bool act = lane < nent;
  const int b = act && lane >= top ? 1 : 0;
  const int id = act ? misc[MI_RIDS + lane] : 0;
  const double l = act ? lg[b * a.E + id] : 0.0;
  const double l0 = __shfl_sync(kFull, l, b * top);
  const double ex = act ? (double)__expf((float)(l - l0)) : 0.0;
  double den = 0.0;
#pragma unroll 1
  for (int s2 = 0; s2 < top; s2++) den += __shfl_sync(kFull, ex, b * top + s2);
  const float wt = act ? (float)(ex / den) : 0.0f;
  if (act) {
    reinterpret_cast<float*>(misc + MI_RW)[lane] = wt;
    if (cid == 0 && rank == 0) {
      a.ws.ids[lane] = id;
      a.ws.wts[lane] = wt;
      if (a.dbg_ids) a.dbg_ids[lane] = id;
      if (a.dbg_w) a.dbg_w[lane] = wt;
    }
  }
}

// Epilogue shared by both kernels: write y_e for this CTA's columns, then the
// last expert of each token to finish this column slice combines and resets
// the slice's counter (so the counters are zero again after every call).
// wts: routing weights [B, top_e] (global or this CTA's shared copy).
__device__ void write_and_combine(const ExpertArgs& a, int rank, int j0, int ncols, int ldy, const float* yfin,
                                  int* misc, const float* wts) {
  const int n = misc[MI_N];
#pragma unroll 1
  for (int t = 0; t < n; t++) {
    const int tok = misc[MI_TOK + t], sl = misc[MI_SLOT + t];
    float* dst = a.ws.ye + ((size_t)tok * a.top_e + sl) * a.d + j0;
    for (int col = threadIdx.x; col < ncols; col += NTHR) {
      dst[col] = yfin[t * ldy + col];
      if (a.dbg_y_expert) a.dbg_y_expert[((size_t)tok * a.top_e + sl) * a.d + j0 + col] = yfin[t * ldy + col];
    }
  }
  // the CTA's stores are ordered before one gpu-scope release by the
  // counting thread (barrier, then fence + atomic)
  __syncthreads();
  if (threadIdx.x < n) {
    const int t = threadIdx.x;
    unsigned old;
    asm volatile("fence.acq_rel.gpu;\n\tatom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                 : "=r"(old)
                 : "l"(&a.ws.counters[misc[MI_TOK + t] * kMaxCluster + rank])
                 : "memory");
    misc[MI_LAST + t] = old == (unsigned)(a.top_e - 1);
  }
  __syncthreads();
#pragma unroll 1
  for (int t = 0; t < n; t++) {
    if (!misc[MI_LAST + t]) continue;
    const int tok = misc[MI_TOK + t];
    for (int col = threadIdx.x; col < ncols; col += NTHR) {
      const int j = j0 + col;
      // slot order; four loads in flight at a time
      float acc = 0.0f;
#pragma unroll 4
      for (int s = 0; s < a.top_e; s++)
        acc = fmaf(wts[tok * a.top_e + s], __ldcg(&a.ws.ye[((size_t)tok * a.top_e + s) * a.d + j]), acc);
      if (a.residual) acc += bf16f(a.residual[(size_t)tok * a.d + j]);
      a.y[(size_t)tok * a.d + j] = f2bf16(acc);
    }
    if (threadIdx.x == 0) a.ws.counters[tok * kMaxCluster + rank] = 0u;
  }
}

// Down rows: thread (g, q) takes 16-byte chunk q of rows g, g + rg, ... (rg
// row groups); chunks q < ncq are 8 W_down columns of this CTA's slice, the
// rest 8 entries of the Ubar row (recovery).  Rows are loaded 8 at a time
// per thread, all in flight together.  coef(m, i, is_w, co[NT]) gives each
// token's coefficient of row m (channel i) and returns whether the chunk is
// needed at all (a chunk whose coefficients are all zero is not read).
// Per-group partial sums land in red[g][t][q * 8 + c]; returns rg.
template <int NT, class Chan, class Coef>
__device__ int down_rows(const ExpertArgs& a, int e, int j0, int ncq, int nr8, int nrows, int rr, Chan chan,
                         Coef coef, float* red) {
  const int nch = ncq + nr8;
  const int g = idiv(threadIdx.x, nch);
  const int q = threadIdx.x - g * nch;
  const int rg = idiv(NTHR, nch);
  float acc[NT][8];
#pragma unroll
  for (int t = 0; t < NT; t++)
#pragma unroll
    for (int c = 0; c < 8; c++) acc[t][c] = 0.0f;
  if (g < rg) {
    const bool is_w = q < ncq;
    const uint16_t* base = is_w ? a.w_down + (size_t)e * a.I * a.d + j0 + 8 * q
                                : a.u_sigma + (size_t)e * a.I * rr + 8 * (q - ncq);
    const size_t stride = is_w ? (size_t)a.d : (size_t)rr;
#pragma unroll 1
    for (int m0 = g; m0 < nrows; m0 += 8 * rg) {
      uint4 w[8];
      float co[8][NT];
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const int m = m0 + u * rg;
        w[u] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int t = 0; t < NT; t++) co[u][t] = 0.0f;
        if (m < nrows) {
          const int i = chan(m);
          if (coef(m, i, is_w, co[u])) w[u] = ld_stream(base + (size_t)i * stride);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const float f[8] = {bf16lo(w[u].x), bf16hi(w[u].x), bf16lo(w[u].y), bf16hi(w[u].y),
                            bf16lo(w[u].z), bf16hi(w[u].z), bf16lo(w[u].w), bf16hi(w[u].w)};
#pragma unroll
        for (int t = 0; t < NT; t++)
#pragma unroll
          for (int c = 0; c < 8; c++) acc[t][c] = fmaf(co[u][t], f[c], acc[t][c]);
      }
    }
#pragma unroll
    for (int t = 0; t < NT; t++) {
      float4* dst = reinterpret_cast<float4*>(red + ((size_t)(g * NT + t) * nch + q) * 8);
      dst[0] = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
      dst[1] = make_float4(acc[t][4], acc[t][5], acc[t][6], acc[t][7]);
    }
  }
  __syncthreads();
  return rg;
}

// Warp totals of one channel's sketch dots: G (gate) and U (up) of each
// token, reduced two values at a time.  On return lanes 0..15 hold (g, u) of
// token (lane >> 3) & 1 when NT = 2, of token 0 when NT = 1.
template <int NT>
__device__ __forceinline__ void reduce_gu(const int (&G)[NT], const int (&U)[NT], int& g, int& u) {
  const int lane = threadIdx.x & 31;
  const bool lo = lane < 16;
  int v;
  if (NT == 1) {
    v = (lo ? G[0] : U[0]) + __shfl_xor_sync(kFull, lo ? U[0] : G[0], 16);
    v += __shfl_xor_sync(kFull, v, 8);
  } else {
    const int k0 = (lo ? G[0] : U[0]) + __shfl_xor_sync(kFull, lo ? U[0] : G[0], 16);
    const int k1 = (lo ? G[NT - 1] : U[NT - 1]) + __shfl_xor_sync(kFull, lo ? U[NT - 1] : G[NT - 1], 16);
    const bool hi8 = lane & 8;
    v = (hi8 ? k1 : k0) + __shfl_xor_sync(kFull, hi8 ? k0 : k1, 8);
  }
  v += __shfl_xor_sync(kFull, v, 4);
  v += __shfl_xor_sync(kFull, v, 2);
  v += __shfl_xor_sync(kFull, v, 1);
  const int o = __shfl_xor_sync(kFull, v, 16);
  g = lo ? v : o;
  u = lo ? o : v;
}


// ================================================================ sparse
// The one-cluster reader for steps of one or two tokens: one cluster of cs
// CTAs per routed expert (work item), every stage in one launch.  CTA `rank`
// owns the channels [ch0[rank], ch0[rank+1]) of the expert for the screen,
// the exact stage and the down rows, and the output columns
// [col0[rank], col0[rank+1]) for the final sum.
//
// Selections without a block-wide histogram.  A channel is a candidate if
// fewer than c channels of the expert beat its screening score (larger, or
// equal with a lower index), and kept if fewer than k candidates beat its
// |a|; that count is all a CTA needs, and only for its own channels.  Each
// CTA sorts its own values (counting ranks among its own channels), pushes
// the sorted list to every other CTA of the cluster, and after the cluster
// barrier adds, for each own channel, how many entries of every other CTA's
// list beat it (a binary search per list).  Four exchanges over distributed
// shared memory, each a push into the receivers' shared memory followed by a
// cluster barrier: the router logits, the sorted score lists, the sorted
// |a| lists of the candidates, and the partial outputs (each CTA sums its
// column slice).  Loads the selections will most likely ask for start before
// the selections are known: after its screen, a CTA starts copying the
// gate/up rows of its own highest-scoring channels; after its exact stage,
// the down rows of all its own candidates.  Rows a selection then leaves out
// are read and not used (measured traffic, not algorithmic bytes).
constexpr int kMaxOwn = 256;        // channels per CTA
constexpr int kRSlots = 4;          // exact-stage row slots per warp (at most)
constexpr int kMaxDSlots = 64;      // down-row slots

struct RLayout {
  int mbar, misc, x, q, logit, alpha, ubar, vown, ahat, aown, vloc, rloc, listc, listk, flags, rows, drows, kslot,
      kco, dcnt, gu, zred, zparts, ztot, ybuf, cntb, q5, ring, total;
  int skrow;    // bytes of one sketch row (2-bit codes: d / 4; base 3: sk3_row_bytes(d))
  int nv3;      // 16-byte chunks of a base-3 row (0 for 2-bit codes)
  int P, Pext;  // exact-stage slots (gate + up rows of one channel, 4d bytes each): P per warp, one more
                // for warps 0 .. Pext - 1
  int W;        // warps that own slots (all when P >= 1)
  int ringb;    // ring bytes
  int ndslot;   // down-row slots (2d bytes each)
  int nskbuf;   // 16-channel sketch chunks resident at once
  int own_max, om4, cols_max, d8, skc, rr, nsteps;
  int ch0[17], col0[17], ex0[17];
};

__host__ inline RLayout make_rlayout(int NT, int B, int E, int I, int d, int r, int cs, int smem_max, bool sk3) {
  RLayout L = {};
  for (int o = 0; o <= cs && o < 17; o++) {
    const int c4 = 4 * cdiv(o * cdiv(I, 4), cs);
    L.ch0[o] = c4 < I ? c4 : I;
    L.col0[o] = 8 * cdiv(o * (d / 8), cs);
    L.ex0[o] = cdiv(o * E, cs);
  }
  for (int o = 0; o < cs && o < 16; o++)
    if (L.ch0[o + 1] - L.ch0[o] > L.own_max) L.own_max = L.ch0[o + 1] - L.ch0[o];
  L.om4 = rup(L.own_max, 4);
  L.nsteps = 0;
  while ((1 << L.nsteps) <= L.om4) L.nsteps++;  // binary-search steps over om4 entries
  L.cols_max = 8 * cdiv(d / 8, cs);
  L.d8 = d / 8;
  L.skc = 16 * (d / 4);
  L.skrow = sk3 ? sk3_row_bytes(d) : d / 4;
  L.nv3 = sk3 ? L.skrow / 16 : 0;
  L.rr = r > 0 ? r : 1;
  int o = 0;
  auto take = [&](int bytes) {
    const int at = o;
    o = rup(o + bytes, 128);
    return at;
  };
  L.mbar = take((kSkBars + 1 + NWARP * kRSlots + kMaxDSlots) * 8);
  L.misc = take(256 * 4);
  L.x = take(B * d * 2);
  L.q = take(B * d);
  L.logit = take(B * E * 8);
  L.alpha = take(2 * L.om4 * 4);
  L.ubar = take(L.om4 * L.rr * 2);
  L.vown = take(L.cols_max * L.rr * 2);
  L.ahat = take(NT * L.om4 * 4);
  L.aown = take(NT * L.om4 * 4);
  L.vloc = take(NT * L.om4 * 8);
  L.rloc = take(NT * L.om4 * 4);
  // the partial outputs arrive (last exchange) long after every CTA is done
  // with the score lists (first exchange): one region serves both
  const int lc_bytes = NT * cs * L.om4 * 8, yb_bytes = cs * NT * L.cols_max * 4;
  L.listc = take(lc_bytes > yb_bytes ? lc_bytes : yb_bytes);
  L.ybuf = L.listc;
  L.listk = take(NT * cs * L.om4 * 8);
  L.flags = take(L.om4);
  L.rows = take(L.om4 * 4);
  L.drows = take(L.om4 * 4);
  L.kslot = take(L.om4 * 4);
  L.kco = take(NT * L.om4 * 4);
  L.dcnt = take(2 * NT * 16 * 4);
  L.gu = take(L.om4 * NT * 2 * 4);
  L.cntb = take(cs * L.om4 * 4);
  L.zred = take(NWARP * NT * L.rr * 4);
  L.zparts = take(cs * NT * L.rr * 4);
  L.ztot = take(NT * L.rr * 4);
  // base-3 sketch: the tokens' activations staged per 16-byte chunk, digit-major
  L.q5 = sk3 ? take(B * L.nv3 * 80) : 0;
  L.ring = o;
  const int avail = smem_max - o;
  const int ring = avail > 0 ? avail / (8 * d) * (8 * d) : 0;
  int ns = ring / (4 * d);
  if (ns > NWARP * kRSlots) ns = NWARP * kRSlots;
  L.P = ns / NWARP;
  L.Pext = ns % NWARP;
  L.W = L.P > 0 ? NWARP : L.Pext;
  L.ndslot = ring / (2 * d) < kMaxDSlots ? ring / (2 * d) : kMaxDSlots;
  // sketch chunks stay clear of the transform's fp32 scratch at the ring's end
  L.nskbuf = (ring - 4 * d) / (8 * d) < kSkBars ? (ring - 4 * d) / (8 * d) : kSkBars;
  L.ringb = ring;
  L.total = o + ring;
  return L;
}

// misc ints of the sparse kernel (beyond the shared positions above)
enum { MI_NCT = 2, MI_NSPEC = 8, MI_NROWS = 9, MI_NDC = 10, MI_NK = 11, MI_SQ = 13 };  // MI_NCT, MI_SQ: B <= 2 ints
static_assert((int)MI_NK < (int)MI_DONE && (int)MI_SQ > (int)MI_DONE && (int)MI_SQ + 2 <= (int)MI_TOK,
              "misc positions");
// flags of an own channel: candidate of token t (bit t), kept by token t
// (bit 2 + t), started before the candidates were known (bit 4)
constexpr unsigned char kFlagSpec = 16;

// Bulk copies of sketch chunk ch (rows i0 + 16 ch .. of both matrices) into
// chunk buffer `slot` of the ring, completing on bars[slot].
__device__ __forceinline__ void issue_sketch(const ExpertArgs& a, const RLayout& L, char* ring, uint64_t* bars, int e,
                                             int i0, int i1, int ch, int slot) {
  const int c0 = i0 + 16 * ch, cnt = min(16, i1 - c0);
  const uint32_t bytes = cnt * L.skrow;
  char* dst = ring + (size_t)slot * 2 * L.skc;
  mbar_expect_tx(&bars[slot], 2 * bytes);
  bulk_g2s(dst, reinterpret_cast<const char*>(a.sk_gate) + ((size_t)e * a.I + c0) * L.skrow, bytes, &bars[slot]);
  // test hook: chunk 0's up rows are expected but never copied, so every
  // wait for that chunk runs out (nothing is left in flight)
  if (a.withhold_copy && ch == 0) return;
  bulk_g2s(dst + L.skc, reinterpret_cast<const char*>(a.sk_up) + ((size_t)e * a.I + c0) * L.skrow, bytes,
           &bars[slot]);
}

// Gate and up rows of channel i into a 4d-byte slot.
__device__ __forceinline__ void issue_gate_up(const ExpertArgs& a, int e, int i, char* dst, uint64_t* bar) {
  const uint32_t rowb = (uint32_t)a.d * 2;
  mbar_expect_tx(bar, 2 * rowb);
  bulk_g2s(dst, a.w_gate + ((size_t)e * a.I + i) * a.d, rowb, bar);
  bulk_g2s(dst + rowb, a.w_up + ((size_t)e * a.I + i) * a.d, rowb, bar);
}

__device__ __forceinline__ void issue_down(const ExpertArgs& a, int e, int i, char* dst, uint64_t* bar) {
  const uint32_t rowb = (uint32_t)a.d * 2;
  mbar_expect_tx(bar, rowb);
  bulk_g2s(dst, a.w_down + ((size_t)e * a.I + i) * a.d, rowb, bar);
}

// Sort key of a channel: its value's bits above, the complement of its index
// below, so that a larger key means a larger value or an equal value at a
// lower channel (the tie rule of both selections); values are non-negative
// floats, so their bit patterns order like the values.
__device__ __forceinline__ uint64_t sort_key(float v, int i) {
  return ((uint64_t)__float_as_uint(v) << 32) | (uint32_t)(0xffffffffu - (uint32_t)i);
}

// rank[li] = #{lj < n : v[lj] > v[li]} for li < n (keys distinct), n <=
// kMaxOwn: thread (li, part) compares against lj = part, part + 4, ...
__device__ void local_ranks(const uint64_t* v, int n, int* rank) {
#pragma unroll 1
  for (int base = 0; base < n; base += NTHR / 4) {
    const int li = base + (threadIdx.x >> 2), part = threadIdx.x & 3;
    const uint64_t vi = li < n ? v[li] : 0ull;
    int cnt = 0;
    if (li < n)
#pragma unroll 4
      for (int lj = part; lj < n; lj += 4) cnt += v[lj] > vi;
    cnt += __shfl_xor_sync(kFull, cnt, 1);
    cnt += __shfl_xor_sync(kFull, cnt, 2);
    if (li < n && part == 0) rank[li] = cnt;
  }
}

// For the n entries of this CTA's sorted list `mine` (descending), how many
// entries of the sorted list of CTA o beat each one: warp o (o < cs, o !=
// self) merges the two lists, lane l taking a run of consecutive own entries
// (one binary search for its first, then steps forward).  cnt[o * om4 + r]
// gets the count for own entry r.  Lists are zero padded to om4 entries;
// zero entries never beat anything.
__device__ __forceinline__ void merge_counts(const uint64_t* lists, const uint64_t* mine, int n, int om4, int nsteps,
                                             int cs, int self, int* cnt) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= cs || warp == self || n <= 0) return;
  const uint64_t* L = lists + (size_t)warp * om4;
  const int run = (n + 31) >> 5, r0 = lane * run, r1 = min(n, r0 + run);
  if (r0 >= r1) return;
  // first own entry of the run: entries of L above it
  const uint64_t v0 = mine[r0];
  int lo = 0, hi = om4;
#pragma unroll 1
  for (int s = 0; s < nsteps && lo < hi; s++) {
    const int mid = (lo + hi) >> 1;
    if (L[mid] > v0) lo = mid + 1;
    else hi = mid;
  }
  cnt[warp * om4 + r0] = lo;
  // the rest of the run: own entries fall, so the count only grows
#pragma unroll 1
  for (int r = r0 + 1; r < r1; r++) {
    const uint64_t v = mine[r];
    while (lo < om4 && L[lo] > v) lo++;
    cnt[warp * om4 + r] = lo;
  }
}

// The sorted list of the nonzero keys among n own keys (local ranks given;
// zero keys, which tie, are left out) into this CTA's slot of a list array,
// whose entries were zeroed at the start.
__device__ __forceinline__ void write_sorted(const uint64_t* v, const int* rank, int n, uint64_t* mine) {
  for (int li = threadIdx.x; li < n; li += NTHR)
    if (v[li]) mine[rank[li]] = v[li];
}

template <int NT, bool DBG, bool SK3>
__global__ void __launch_bounds__(NTHR, 1) reader_kernel(ExpertArgs a, RLayout L) {
  extern __shared__ __align__(128) char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int cid = cluster_id();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t* skbars = reinterpret_cast<uint64_t*>(smem + L.mbar);
  uint64_t* uvbar = skbars + kSkBars;
  const int sbase = warp * L.P + min(warp, L.Pext), Pw = L.P + (warp < L.Pext ? 1 : 0);
  const int W = L.W;  // rows go to warps 0 .. W - 1 (those that own slots)
  uint64_t* wbars = uvbar + 1 + sbase;                // this warp's exact-stage slots
  uint64_t* dbars = uvbar + 1 + NWARP * kRSlots;      // down-row slots
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  unsigned char* flags = reinterpret_cast<unsigned char*>(smem + L.flags);
  if (tid < kSkBars + 1 + NWARP * kRSlots + kMaxDSlots) mbar_init(&skbars[tid], 1);
  for (int i = tid; i < L.om4; i += NTHR) flags[i] = 0;
  {
    // this CTA's slots of both list arrays start zeroed (the peers write only theirs)
    uint64_t* lc = reinterpret_cast<uint64_t*>(smem + L.listc);
    uint64_t* lk = reinterpret_cast<uint64_t*>(smem + L.listk);
    const int rk = (int)cg::this_cluster().block_rank(), ncs = (int)cg::this_cluster().num_blocks();
    for (int i = tid; i < NT * L.om4; i += NTHR) {
      const int t = i / L.om4, j = i - t * L.om4;
      lc[((size_t)t * ncs + rk) * L.om4 + j] = 0ull;
      lk[((size_t)t * ncs + rk) * L.om4 + j] = 0ull;
    }
  }
  if (tid == 0) misc[MI_DONE] = 0;
  fence_mbar_init();
  __syncthreads();
  if (DBG) stamp(a, cid, rank, 0);

  // Programmatic dependent launch: the next kernel in the stream may be
  // scheduled now; nothing in global memory is read before the previous
  // kernel has completed and its writes are visible.
  pdl_trigger();
  pdl_wait();
  const int d = a.d, I = a.I, r = a.r, om = L.om4;
  char* ring = smem + L.ring;
  const uint16_t* xs = reinterpret_cast<const uint16_t*>(smem + L.x);
  int8_t* qs = reinterpret_cast<int8_t*>(smem + L.q);
  float* cxs = reinterpret_cast<float*>(misc + MI_CX);

  char4 sv_pre = make_char4(0, 0, 0, 0);  // rotation signs of elements 4 tid .. 4 tid + 3
  if (tid < d / 4) sv_pre = __ldg(reinterpret_cast<const char4*>(a.rot_sign) + tid);

  // ---------------------------------------------------------- R: routing
  // (every CTA of every cluster takes the same top-e from the exchanged
  // logits; a cluster past the last work item has nothing to do)
  const bool has_item = fused_route<NT>(a, L, smem, misc, cs, rank, cid, cluster, [] {});
  if (!has_item) return;  // uniform per cluster; no exchange follows
  if (DBG) stamp(a, cid, rank, 4);
  const int e = misc[MI_E], n = misc[MI_N];
  const int i0 = L.ch0[rank], i1 = L.ch0[rank + 1], nown = i1 - i0;
  const int j0 = L.col0[rank], ncols = L.col0[rank + 1] - j0;
  uint32_t* err = a.ws.err;
  const int nchunk = cdiv(nown, 16);

  // the sketch chunks (warp w copies chunk w), the sketch scales (on chunk
  // 0's barrier, which every warp waits for first), the factor rows of the
  // own channels and the V rows of the own columns: all in flight at once
  if (lane == 0) {
    if (warp == 0 && I % 4 == 0 && nown > 0) {
      mbar_expect_tx_only(&skbars[0], 2 * nown * 4);
      bulk_g2s(smem + L.alpha, a.alpha_gate + (size_t)e * I + i0, nown * 4, &skbars[0]);
      bulk_g2s(smem + L.alpha + om * 4, a.alpha_up + (size_t)e * I + i0, nown * 4, &skbars[0]);
    }
    if (warp < min(nchunk, L.nskbuf)) issue_sketch(a, L, ring, skbars, e, i0, i1, warp, warp);
    if (warp == NWARP - 1 && r > 0) {
      const uint32_t bu = nown * r * 2, bv = ncols * r * 2;
      mbar_expect_tx(uvbar, bu + bv);
      bulk_g2s(smem + L.ubar, a.u_sigma + ((size_t)e * I + i0) * r, bu, uvbar);
      bulk_g2s(smem + L.vown, a.v + ((size_t)e * d + j0) * r, bv, uvbar);
    }
  }
  float* alg = reinterpret_cast<float*>(smem + L.alpha);
  float* alu = alg + om;
  if (I % 4 != 0) {  // unaligned scale slices: plain loads
    for (int li = tid; li < nown; li += NTHR) {
      alg[li] = __ldg(a.alpha_gate + (size_t)e * I + i0 + li);
      alu[li] = __ldg(a.alpha_up + (size_t)e * I + i0 + li);
    }
  }
  // every token is rotated and quantised while the copies are in flight (the
  // fp32 scratch of the transform sits past the sketch buffers); its block
  // barriers also publish the scale loads above
#pragma unroll 1
  for (int t = 0; t < a.B; t++)
    rotate_quantize(a, xs + (size_t)t * d, qs + (size_t)t * d, reinterpret_cast<float*>(ring + L.ringb - 4 * d),
                    cxs + t, reinterpret_cast<float*>(misc + MI_RED), sv_pre, misc + MI_SQ + t);
  if (SK3) {
    // activations staged per 16-byte chunk of the base-3 rows, digit-major
    // (b3_qpos); zero past d
    for (int o = tid; o < a.B * L.nv3 * 16; o += NTHR) {
      const int t = o / (L.nv3 * 16), g = o - t * (L.nv3 * 16);
      const int8_t* qt = qs + (size_t)t * d;
      char* c5 = smem + L.q5 + ((size_t)t * L.nv3 + (g >> 4)) * 80;
#pragma unroll
      for (int k = 0; k < 5; k++) c5[b3_qpos(g & 15, k)] = 5 * g + k < d ? (char)qt[5 * g + k] : (char)0;
    }
    __syncthreads();
  }
  if (DBG) stamp(a, cid, rank, 1);
  int tix[NT];
#pragma unroll
  for (int t = 0; t < NT; t++) tix[t] = misc[MI_TIX + (t < n ? t : 0)];

  float* ahat = reinterpret_cast<float*>(smem + L.ahat);        // [NT, om] sketch estimates, own channels
  float* aown = reinterpret_cast<float*>(smem + L.aown);        // [NT, om] exact a, own candidates
  uint64_t* vloc = reinterpret_cast<uint64_t*>(smem + L.vloc);  // [NT, om] sort keys, own channels
  int* rloc = reinterpret_cast<int*>(smem + L.rloc);            // [NT, om] local ranks
  uint64_t* listc = reinterpret_cast<uint64_t*>(smem + L.listc);  // [NT, cs, om] sorted score keys
  uint64_t* listk = reinterpret_cast<uint64_t*>(smem + L.listk);  // [NT, cs, om] sorted |a| keys
  float* zparts = reinterpret_cast<float*>(smem + L.zparts);    // [cs, NT, rr]
  int* rows = reinterpret_cast<int*>(smem + L.rows);
  int* drows = reinterpret_cast<int*>(smem + L.drows);
  int* dcnt = reinterpret_cast<int*>(smem + L.dcnt);            // [2, NT, 16] debug list counts
  const uint16_t* ub = reinterpret_cast<const uint16_t*>(smem + L.ubar);

  // ---------------------------------------------------------- S: screen
  // warp w takes channel 16 j + w of every sketch chunk j: per chunk the
  // lanes' partial dots, then the warp reduction of the previous chunk (its
  // shuffles overlap these dots); the sums are parked per channel and one
  // pass over (channel, token) afterwards turns them into scores.
  int* gsum = reinterpret_cast<int*>(smem + L.gu);  // [om, NT, 2] exact G, U (code offset not yet removed)
  {
    const int nv = d >> 6;  // 16-byte sketch vectors per row
    uint4 qr[NT][4];        // activations of sketch vector `lane` (the row's first 32 vectors)
#pragma unroll
    for (int t = 0; t < NT; t++) {
      const uint4* qv = reinterpret_cast<const uint4*>(qs + (size_t)tix[t] * d);
#pragma unroll
      for (int kk = 0; kk < 4; kk++) qr[t][kk] = lane < nv ? qv[4 * lane + kk] : make_uint4(0u, 0u, 0u, 0u);
    }
    int pG[NT], pU[NT];  // the previous chunk's lane partials
#pragma unroll
    for (int t = 0; t < NT; t++) pG[t] = pU[t] = 0;
    auto park = [&](int jc) {  // reduce chunk jc's partials over the warp and park them
      int gs, us;
      reduce_gu<NT>(pG, pU, gs, us);
      const int lc = 16 * jc + warp;
      if (lane < 16 && (lane & 7) == 0 && lc < nown) {
        const int t = NT == 2 ? lane >> 3 : 0;
        gsum[(lc * NT + t) * 2] = gs;
        gsum[(lc * NT + t) * 2 + 1] = us;
      }
    };
    int rb = 0, par = 0;  // first chunk of the resident round, parity of its barriers
#pragma unroll 1
    for (int j = 0; j < nchunk; j++) {
      const int li = 16 * j + warp;
      if (j == rb + L.nskbuf) {
        // the next round of chunks reuses the buffers: every warp is done with them
        __syncthreads();
        rb = j;
        par ^= 1;
        if (tid == 0) {
          const int c1 = min(nchunk, j + L.nskbuf);
          for (int ch = j; ch < c1; ch++) issue_sketch(a, L, ring, skbars, e, i0, i1, ch, ch - j);
        }
      }
      int G[NT], U[NT];
#pragma unroll
      for (int t = 0; t < NT; t++) G[t] = U[t] = 0;
      if (SK3 && li < nown) {
        const int slot = j - rb;
        if (!mbar_wait_bounded(&skbars[slot], par, err, a.wait_ns)) misc[MI_DONE] = 1;
        if (lane < L.nv3) {  // lane = the row's 16-byte chunk (80 trits)
          const uint4 g4 = reinterpret_cast<const uint4*>(ring + (size_t)slot * 2 * L.skc + warp * L.skrow)[lane];
          const uint4 u4 =
              reinterpret_cast<const uint4*>(ring + (size_t)slot * 2 * L.skc + L.skc + warp * L.skrow)[lane];
          uint32_t go[20], uo[20], qd[20];
          b3_decode16(g4, go);
          b3_decode16(u4, uo);
#pragma unroll
          for (int t = 0; t < NT; t++) {
            b3_load_q(smem + L.q5 + ((size_t)tix[t] * L.nv3 + lane) * 80, qd);
            G[t] = b3_dot16(go, qd, 0);
            U[t] = b3_dot16(uo, qd, 0);
          }
        }
      } else if (!SK3 && li < nown) {
        const int slot = j - rb;
        if (!mbar_wait_bounded(&skbars[slot], par, err, a.wait_ns)) misc[MI_DONE] = 1;
        const uint4* gw = reinterpret_cast<const uint4*>(ring + (size_t)slot * 2 * L.skc + warp * (d / 4));
        const uint4* uw = reinterpret_cast<const uint4*>(ring + (size_t)slot * 2 * L.skc + L.skc + warp * (d / 4));
        int ga[NT][4], ua[NT][4];
#pragma unroll
        for (int t = 0; t < NT; t++)
#pragma unroll
          for (int kk = 0; kk < 4; kk++) ga[t][kk] = ua[t][kk] = 0;
#pragma unroll 1
        for (int vv = lane; vv < nv; vv += 32) {
          const uint4 g4 = gw[vv], u4 = uw[vv];
#pragma unroll
          for (int t = 0; t < NT; t++) {
            uint4 q0 = qr[t][0], q1 = qr[t][1], q2 = qr[t][2], q3 = qr[t][3];
            if (vv != lane) {
              const uint4* qv = reinterpret_cast<const uint4*>(qs + (size_t)tix[t] * d) + 4 * vv;
              q0 = qv[0];
              q1 = qv[1];
              q2 = qv[2];
              q3 = qv[3];
            }
            code_dot16(g4.x, q0, ga[t]);
            code_dot16(g4.y, q1, ga[t]);
            code_dot16(g4.z, q2, ga[t]);
            code_dot16(g4.w, q3, ga[t]);
            code_dot16(u4.x, q0, ua[t]);
            code_dot16(u4.y, q1, ua[t]);
            code_dot16(u4.z, q2, ua[t]);
            code_dot16(u4.w, q3, ua[t]);
          }
        }
#pragma unroll
        for (int t = 0; t < NT; t++) {
          G[t] = code_dot_total(ga[t]);
          U[t] = code_dot_total(ua[t]);
        }
      }
      if (j > 0) park(j - 1);
#pragma unroll
      for (int t = 0; t < NT; t++) {
        pG[t] = G[t];
        pU[t] = U[t];
      }
    }
    if (nchunk > 0) park(nchunk - 1);
    if (warp == NWARP - 1) route_weights(a, L, smem, misc, cid, rank);
  }
  __syncthreads();
  // scores of (own channel, token): ghat = ((float)G alpha_g) c_x, uhat
  // likewise, ahat = silu_r(ghat) uhat, sigma = |ahat|; G, U the exact dots
  // less the code offset sum(q)
#pragma unroll 1
  for (int k = tid; k < nown * n; k += NTHR) {
    const int lc = n == 2 ? k >> 1 : k, t = k - lc * n;
    const int g2 = gsum[(lc * NT + t) * 2] - misc[MI_SQ + tix[NT == 2 && t ? NT - 1 : 0]];
    const int u2 = gsum[(lc * NT + t) * 2 + 1] - misc[MI_SQ + tix[NT == 2 && t ? NT - 1 : 0]];
    const float cx = cxs[tix[NT == 2 && t ? NT - 1 : 0]];
    const float gh = __fmul_rn(__fmul_rn((float)g2, alg[lc]), cx);
    const float uh = __fmul_rn(__fmul_rn((float)u2, alu[lc]), cx);
    const float ah = __fmul_rn(silu_r(gh), uh);
    vloc[t * om + lc] = sort_key(fabsf(ah), i0 + lc);
    ahat[t * om + lc] = ah;
    if (DBG) {
      const size_t off = ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * I + i0 + lc;
      if (a.dbg_G) a.dbg_G[off] = g2;
      if (a.dbg_U) a.dbg_U[off] = u2;
      if (a.dbg_sigma) a.dbg_sigma[off] = fabsf(ah);
    }
  }
  __syncthreads();  // sort keys and estimates of the own channels are in place; the sketch buffers are free
  if (DBG) stamp(a, cid, rank, 5);

  // ------------------------------------------- c: candidates (top-c by sigma)
  // own sorted score lists to every CTA, the own channels most likely to be
  // candidates started, then each own channel's rank over the expert
#pragma unroll 1
  for (int t = 0; t < n; t++) local_ranks(vloc + t * om, nown, rloc + t * om);
  __syncthreads();
#pragma unroll 1
  for (int t = 0; t < n; t++) write_sorted(vloc + t * om, rloc + t * om, nown, listc + ((size_t)t * cs + rank) * om);
  __syncthreads();
  {
    const int per = om / 2;  // 16-byte pieces of one list
    const int tot = n * per;
#pragma unroll 1
    for (int w = tid; w < (cs - 1) * tot; w += NTHR) {
      const int pi = idiv(w, tot), j = w - pi * tot;
      const int o = pi + (pi >= rank);
      const int t = j >= per ? 1 : 0, qq = j - t * per;
      const float4* src = reinterpret_cast<const float4*>(listc + ((size_t)t * cs + rank) * om) + qq;
      st_cluster(src, o, *src);
    }
  }
  {
    // started early: each token's highest own scores, as many as the exact
    // stage's slots hold at once
    const int take = (NWARP * L.P + L.Pext) / n;
    if (warp == 0) {
      int base = 0;
      for (int w0 = 0; w0 < nown; w0 += 32) {
        const int li = w0 + lane;
        bool on = false;
#pragma unroll
        for (int t = 0; t < NT; t++) on |= t < n && li < nown && rloc[t * om + li] < take;
        const unsigned bal = __ballot_sync(kFull, on);
        if (on) {
          rows[base + __popc(bal & ((1u << lane) - 1u))] = li;
          flags[li] = kFlagSpec;
        }
        base += __popc(bal);
      }
      if (lane == 0) misc[MI_NSPEC] = base;
    }
    __syncthreads();
    const int nspec = misc[MI_NSPEC];
    if (lane == 0) {
      // the ring held the transform's scratch (generic stores of every
      // thread, ordered by the block barriers since): order them before the
      // copies.  Later copies into the ring only follow generic reads, whose
      // values were consumed before the issuing warp's barrier.
      fence_proxy_async();
      for (int m = 0; m < Pw; m++) {
        const int j = warp + W * m;
        if (j < nspec) issue_gate_up(a, e, i0 + rows[j], ring + (size_t)(sbase + m) * 4 * d, &wbars[m]);
      }
    }
    // the next most likely candidates (own ranks up to 1.15 times the CTA's
    // expected share of c) start moving into L2, so that their copies after
    // the selection hit L2; those the selection leaves out are read unused
    const int pf = min(nown, (int)(1.15f * (float)a.c * (float)nown / (float)I) + 1);
    for (int li = tid; li < nown; li += NTHR) {
      bool on = false;
#pragma unroll
      for (int t = 0; t < NT; t++) on |= t < n && rloc[t * om + li] < pf;
      if (on && flags[li] != kFlagSpec) {
        bulk_prefetch_l2(a.w_gate + ((size_t)e * I + i0 + li) * d, 2 * d);
        bulk_prefetch_l2(a.w_up + ((size_t)e * I + i0 + li) * d, 2 * d);
      }
    }
  }
  if (DBG) stamp(a, cid, rank, 6);
  // the pushes above had the selection's time to land: arrive (release) now
  cluster_arrive();
  cluster_wait();
  if (DBG) stamp(a, cid, rank, 7);
  // candidate of token t: fewer than c channels of the expert beat it
  int* cntb = reinterpret_cast<int*>(smem + L.cntb);  // [cs, om] entries of each peer's list above each own entry
#pragma unroll 1
  for (int t = 0; t < n; t++) {
    merge_counts(listc + (size_t)t * cs * om, listc + ((size_t)t * cs + rank) * om, nown, om, L.nsteps, cs, rank, cntb);
    __syncthreads();
    for (int li = tid; li < nown; li += NTHR) {
      const int r0 = rloc[t * om + li];
      int tot = r0;
#pragma unroll 4
      for (int o = 0; o < cs; o++)
        if (o != rank) tot += cntb[o * om + r0];
      if (tot < a.c) atomicOr(reinterpret_cast<unsigned*>(flags) + (li >> 2), (1u << t) << (8 * (li & 3)));
    }
    __syncthreads();
  }
  if (DBG) stamp(a, cid, rank, 8);
  // the down rows of every own candidate start moving into L2 now (the
  // top-k keeps about k / c of them; their copies follow the exact stage)
  for (int li = tid; li < nown; li += NTHR)
    if (flags[li] & 3u) bulk_prefetch_l2(a.w_down + ((size_t)e * I + i0 + li) * d, 2 * d);
  // rows of the exact stage: the started ones, then the own candidates not
  // started yet; drows: every own candidate, ascending
  const int nspec = misc[MI_NSPEC];
  if (warp == 0) {
    int base = nspec, dbase = 0, nct[NT];
#pragma unroll
    for (int t = 0; t < NT; t++) nct[t] = 0;
    for (int w0 = 0; w0 < nown; w0 += 32) {
      const int li = w0 + lane;
      const unsigned f = li < nown ? flags[li] : 0u;
      const bool cand = (f & 3u) != 0, miss = cand && !(f & kFlagSpec);
      const unsigned bm = __ballot_sync(kFull, miss), bc = __ballot_sync(kFull, cand);
      if (miss) rows[base + __popc(bm & ((1u << lane) - 1u))] = li;
      if (cand) drows[dbase + __popc(bc & ((1u << lane) - 1u))] = li;
      base += __popc(bm);
      dbase += __popc(bc);
#pragma unroll
      for (int t = 0; t < NT; t++) nct[t] += __popc(__ballot_sync(kFull, (f >> t) & 1u));
    }
    if (lane == 0) {
      misc[MI_NROWS] = base;
      misc[MI_NDC] = dbase;
#pragma unroll
      for (int t = 0; t < NT; t++) misc[MI_NCT + t] = nct[t];  // own candidates of each token
    }
  }
  __syncthreads();
  const int nrows = misc[MI_NROWS], ndc = misc[MI_NDC];

  // -------------------------------------------- C: exact candidate stage
  // warp w < W takes rows w, w + W, ...: position m of the warp in its slot m % Pw
  {
    const int nmine = warp < W && nrows > warp ? cdiv(nrows - warp, W) : 0;
    char* wring = ring + (size_t)sbase * 4 * d;
    if (lane == 0) {
      for (int m = 0; m < Pw && m < nmine; m++) {
        const int j = warp + W * m;
        if (j >= nspec) issue_gate_up(a, e, i0 + rows[j], wring + (size_t)m * 4 * d, &wbars[m]);
      }
    }
    __syncwarp();
    const uint4* xv4 = reinterpret_cast<const uint4*>(xs);
    uint32_t par = 0;
#pragma unroll 1
    for (int m = 0; m < nmine; m++) {
      const int s = m % Pw;
      if (!mbar_wait_bounded(&wbars[s], (par >> s) & 1u, err, a.wait_ns)) misc[MI_DONE] = 1;
      par ^= 1u << s;
      const int j = warp + W * m, li = rows[j];
      const unsigned f = flags[li];
      if (f & 3u) {
        const uint4* gr = reinterpret_cast<const uint4*>(wring + (size_t)s * 4 * d);
        const uint4* ur = gr + L.d8;
        float g0[NT], g1[NT], v0[NT], v1[NT];
#pragma unroll
        for (int t = 0; t < NT; t++) g0[t] = g1[t] = v0[t] = v1[t] = 0.0f;
#pragma unroll 2
        for (int vv = lane; vv < L.d8; vv += 32) {
          const uint4 gv = gr[vv], uv = ur[vv];
#pragma unroll
          for (int t = 0; t < NT; t++) {
            const uint4 xq = xv4[tix[t] * L.d8 + vv];
            dot8_mixed(gv, xq, g0[t], g1[t]);
            dot8_mixed(uv, xq, v0[t], v1[t]);
          }
        }
#pragma unroll
        for (int t = 0; t < NT; t++) {
          if (t < n) {
            const float gs = warp_sum(g0[t] + g1[t]), us = warp_sum(v0[t] + v1[t]);
            if (lane == 0 && ((f >> t) & 1u)) aown[t * om + li] = __fmul_rn(silu_r(gs), us);
          }
        }
      }
      __syncwarp();
      if (m + Pw < nmine && lane == 0) {
        issue_gate_up(a, e, i0 + rows[j + W * Pw], wring + (size_t)s * 4 * d, &wbars[s]);
      }
    }
  }
  __syncthreads();  // every issued row was consumed: the ring is free
  if (DBG) stamp(a, cid, rank, 9);
  const bool dspec = ndc <= L.ndslot;

  // ------------------------------------------------ k: kept (top-k by |a|)
  // each token's own candidates: sort keys of |a|, local ranks, sorted lists
  // to every CTA
#pragma unroll 1
  for (int t = 0; t < n; t++)
    for (int m = tid; m < ndc; m += NTHR) {
      const int li = drows[m];
      vloc[t * om + m] = ((flags[li] >> t) & 1u) ? sort_key(fabsf(aown[t * om + li]), i0 + li) : 0ull;
    }
  __syncthreads();
#pragma unroll 1
  for (int t = 0; t < n; t++) local_ranks(vloc + t * om, ndc, rloc + t * om);
  __syncthreads();
#pragma unroll 1
  for (int t = 0; t < n; t++) write_sorted(vloc + t * om, rloc + t * om, ndc, listk + ((size_t)t * cs + rank) * om);
  if (DBG && tid < n) {
    int cnt = 0;
    for (int m = 0; m < ndc; m++) cnt += (flags[drows[m]] >> tid) & 1u;
    dcnt[tid * 16 + rank] = cnt;  // own candidates of token tid (debug list offsets)
  }
  __syncthreads();
  {
    const int per = om / 2;
    const int tot = n * per;
#pragma unroll 1
    for (int w = tid; w < (cs - 1) * tot; w += NTHR) {
      const int pi = idiv(w, tot), j = w - pi * tot;
      const int o = pi + (pi >= rank);
      const int t = j >= per ? 1 : 0, qq = j - t * per;
      const float4* src = reinterpret_cast<const float4*>(listk + ((size_t)t * cs + rank) * om) + qq;
      st_cluster(src, o, *src);
    }
    if (DBG && tid < n)
      for (int o = 0; o < cs; o++)
        if (o != rank) asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr(&dcnt[tid * 16 + rank], o)),
                                    "r"(dcnt[tid * 16 + rank])
                                    : "memory");
  }
  // while the pushes land: the down rows of every own candidate start now
  // (warp m % 16 copies row m; the top-k keeps about k / c of them; if they
  // do not fit, the kept ones follow the selection)
  if (dspec && lane == 0) {
    for (int m = warp; m < ndc; m += NWARP) issue_down(a, e, i0 + drows[m], ring + (size_t)m * 2 * d, &dbars[m]);
  }
  cluster_arrive();
  cluster_wait();
  if (DBG) stamp(a, cid, rank, 10);
#pragma unroll 1
  for (int t = 0; t < n; t++) {
    const int nct = misc[MI_NCT + t];  // own candidates of token t (the nonzero entries of the own list)
    merge_counts(listk + (size_t)t * cs * om, listk + ((size_t)t * cs + rank) * om, nct, om, L.nsteps, cs, rank, cntb);
    __syncthreads();
    for (int m = tid; m < ndc; m += NTHR) {
      const int li = drows[m];
      if (!((flags[li] >> t) & 1u)) continue;
      const int r0 = rloc[t * om + m];
      int tot = r0;
#pragma unroll 4
      for (int o = 0; o < cs; o++)
        if (o != rank) tot += cntb[o * om + r0];
      if (tot < a.k) atomicOr(reinterpret_cast<unsigned*>(flags) + (li >> 2), (4u << t) << (8 * (li & 3)));
    }
    __syncthreads();
  }
  if (DBG && warp < n && (a.dbg_cand || a.dbg_kept || a.dbg_a_kept)) {
    // this CTA's part of the ascending candidate list (offset: the candidates
    // of the lower CTAs); the kept list follows after the last exchange
    const int t = warp;
    int off = 0;
    for (int o = 0; o < rank; o++) off += dcnt[t * 16 + o];
    int* out = a.dbg_cand ? a.dbg_cand + ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * a.c : nullptr;
    int base = off, kc = 0;
    for (int m0 = 0; m0 < ndc; m0 += 32) {
      const int m = m0 + lane;
      const unsigned f = m < ndc ? flags[drows[m]] : 0u;
      const bool on = (f >> t) & 1u;
      const unsigned bal = __ballot_sync(kFull, on);
      if (on && out && base + __popc(bal & ((1u << lane) - 1u)) < a.c)
        out[base + __popc(bal & ((1u << lane) - 1u))] = i0 + drows[m];
      base += __popc(bal);
      kc += __popc(__ballot_sync(kFull, (f >> (2 + t)) & 1u));
    }
    if (lane == 0) dcnt[(NT + t) * 16 + rank] = kc;  // own kept channels of token t
  }
  if (DBG) stamp(a, cid, rank, 11);

  // ------------------------------------------ recovery input z (own part)
  // z_t = sum over the own channels not kept by token t of their recovery
  // input times Ubar_i: the sketch estimate ahat_i, or with the exact input
  // the exact a_i of a dropped candidate.  Warp w takes channels w, w + 16,
  // ..., lane p the entries p, p + 32, ...; the warps' sums meet in shared
  // memory.
  if (r > 0) {
    if (!mbar_wait_bounded(uvbar, 0, err, a.wait_ns)) misc[MI_DONE] = 1;
    const bool rec_exact = a.recovery_input == 1;
    float zacc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
      for (int kk = 0; kk < 4; kk++) zacc[t][kk] = 0.0f;
#pragma unroll 1
    for (int li = warp; li < nown; li += NWARP) {
      const unsigned f = flags[li];
      float co[NT];
#pragma unroll
      for (int t = 0; t < NT; t++) {
        const bool kept = (f >> (2 + t)) & 1u, cand = (f >> t) & 1u;
        co[t] = t >= n || kept ? 0.0f : cand && rec_exact ? aown[t * om + li] : ahat[t * om + li];
      }
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {
        const int p = lane + 32 * kk;
        if (p < r) {
          const float u = bf16f(ub[li * r + p]);
#pragma unroll
          for (int t = 0; t < NT; t++) zacc[t][kk] = fmaf(co[t], u, zacc[t][kk]);
        }
      }
    }
    float* zr = reinterpret_cast<float*>(smem + L.zred);  // [NWARP, NT, r]
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {
        const int p = lane + 32 * kk;
        if (p < r) zr[(warp * NT + t) * r + p] = zacc[t][kk];
      }
  }

  // ---------------------------------------------- D: down rows + recovery
  // kept rows, compacted with each token's coefficient; warp 0 waits for
  // their copies, then thread tid adds columns 4 tid .. 4 tid + 3 of every row
  int* kslot = reinterpret_cast<int*>(smem + L.kslot);
  float* kco = reinterpret_cast<float*>(smem + L.kco);  // [NT, om]
  if (warp == 0) {
    int base = 0;
    for (int m0 = 0; m0 < ndc; m0 += 32) {
      const int m = m0 + lane;
      const int li = m < ndc ? drows[m] : 0;
      const unsigned f = m < ndc ? flags[li] : 0u;
      const bool kept = (f & 12u) != 0;
      const unsigned bal = __ballot_sync(kFull, kept);
      if (kept) {
        const int at = base + __popc(bal & ((1u << lane) - 1u));
        kslot[at] = dspec ? m : li;  // dspec: the slot of the row; else the channel
#pragma unroll
        for (int t = 0; t < NT; t++) kco[t * om + at] = t < n && ((f >> (2 + t)) & 1u) ? aown[t * om + li] : 0.0f;
      }
      base += __popc(bal);
    }
    if (lane == 0) misc[MI_NK] = base;
  }
  __syncthreads();
  const int nk = misc[MI_NK];
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; t++)
#pragma unroll
    for (int c = 0; c < 4; c++) acc[t][c] = 0.0f;
  const bool colt = 4 * tid < d;
  const int rnd = dspec ? (nk > 0 ? nk : 1) : L.ndslot;
#pragma unroll 1
  for (int base = 0; base < nk; base += rnd) {
    const int cnt = min(rnd, nk - base);
    if (!dspec) {
      __syncthreads();  // every thread is done with the previous round's slots
      if (lane == 0) {
        for (int m = warp; m < cnt; m += NWARP)
          issue_down(a, e, i0 + kslot[base + m], ring + (size_t)m * 2 * d, &dbars[m]);
      }
    }
    if (warp == 0) {
      const uint32_t par = dspec ? 0u : (uint32_t)(base / rnd) & 1u;
      for (int m = lane; m < cnt; m += 32) {
        const int s = dspec ? kslot[base + m] : m;
        if (!mbar_wait_bounded(&dbars[s], par, err, a.wait_ns)) misc[MI_DONE] = 1;
      }
    }
    __syncthreads();
    if (colt) {
#pragma unroll 2
      for (int m = 0; m < cnt; m++) {
        const int s = dspec ? kslot[base + m] : m;
        const uint2 w2 = reinterpret_cast<const uint2*>(ring + (size_t)s * 2 * d)[tid];
        const float f0 = bf16lo(w2.x), f1 = bf16hi(w2.x), f2 = bf16lo(w2.y), f3 = bf16hi(w2.y);
#pragma unroll
        for (int t = 0; t < NT; t++) {
          const float co = kco[t * om + base + m];
          acc[t][0] = fmaf(co, f0, acc[t][0]);
          acc[t][1] = fmaf(co, f1, acc[t][1]);
          acc[t][2] = fmaf(co, f2, acc[t][2]);
          acc[t][3] = fmaf(co, f3, acc[t][3]);
        }
      }
    }
  }
  if (dspec && nk < ndc && warp == 1) {
    // copies of rows the top-k left out must land before the CTA ends
    for (int m = lane; m < ndc; m += 32) {
      const unsigned f = flags[drows[m]];
      if (!(f & 12u) && !mbar_wait_bounded(&dbars[m], 0, err, a.wait_ns)) misc[MI_DONE] = 1;
    }
  }
  // the own part of z: the warps' sums (their writes ordered by the block
  // barriers of the down stage)
  if (r > 0) {
    const float* zr = reinterpret_cast<const float*>(smem + L.zred);
    for (int tp = tid; tp < n * r; tp += NTHR) {
      const int t = tp >= r ? 1 : 0, p = tp - t * r;
      float z0 = 0.0f, z1 = 0.0f;
#pragma unroll 4
      for (int w = 0; w < NWARP; w += 2) {
        z0 += zr[(w * NT + t) * r + p];
        z1 += zr[((w + 1) * NT + t) * r + p];
      }
      zparts[(rank * NT + t) * r + p] = z0 + z1;
    }
  }
  __syncthreads();
  if (DBG) stamp(a, cid, rank, 12);
  // push: the partial outputs to the owners of their columns, z to everyone
  float* ybuf = reinterpret_cast<float*>(smem + L.ybuf);  // [cs, NT, cols_max] from every sender
  if (colt) {
    const int c0 = 4 * tid;
    int o = 0;
    while (o + 1 < cs && L.col0[o + 1] <= c0) o++;
#pragma unroll
    for (int t = 0; t < NT; t++)
      if (t < n)
        st_cluster(&ybuf[((size_t)rank * NT + t) * L.cols_max + c0 - L.col0[o]], o,
                   make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]));
  }
  if (r > 0) {
    const int nq = n * r / 4;
    for (int w = tid; w < (cs - 1) * nq; w += NTHR) {
      const int pi = idiv(w, nq), j = w - pi * nq;
      const int o = pi + (pi >= rank);
      const float4* src = reinterpret_cast<const float4*>(zparts + (size_t)rank * NT * r) + j;
      st_cluster(src, o, *src);
    }
  }
  if (DBG && tid < n)
    for (int o = 0; o < cs; o++)
      if (o != rank) asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr(&dcnt[(NT + tid) * 16 + rank], o)),
                                  "r"(dcnt[(NT + tid) * 16 + rank])
                                  : "memory");
  cluster.sync();  // the last exchange: no CTA touches another's shared memory after this
  if (DBG) stamp(a, cid, rank, 13);
  if (DBG && warp < n && (a.dbg_kept || a.dbg_a_kept)) {
    const int t = warp;
    int off = 0;
    for (int o = 0; o < rank; o++) off += dcnt[(NT + t) * 16 + o];
    const size_t obase = ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * a.k;
    int base = off;
    for (int m0 = 0; m0 < ndc; m0 += 32) {
      const int m = m0 + lane;
      const int li = m < ndc ? drows[m] : 0;
      const bool on = m < ndc && ((flags[li] >> (2 + t)) & 1u);
      const unsigned bal = __ballot_sync(kFull, on);
      const int at = base + __popc(bal & ((1u << lane) - 1u));
      if (on && at < a.k) {
        if (a.dbg_kept) a.dbg_kept[obase + at] = i0 + li;
        if (a.dbg_a_kept) a.dbg_a_kept[obase + at] = aown[t * om + li];
      }
      base += __popc(bal);
    }
  }

  // ------------------------------------ the own columns: sum, V z, combine
  float* ztot = reinterpret_cast<float*>(smem + L.ztot);
  if (r > 0)
    for (int tp = tid; tp < n * r; tp += NTHR) {
      const int t = tp / r, p = tp - t * r;
      float zz = 0.0f;
#pragma unroll 1
      for (int o = 0; o < cs; o++) zz += zparts[(o * NT + t) * r + p];
      ztot[t * r + p] = zz;
    }
  __syncthreads();
  float* yfin = reinterpret_cast<float*>(smem + L.x);  // [n, cols_max]; x is no longer needed
  const uint16_t* vo = reinterpret_cast<const uint16_t*>(smem + L.vown);
#pragma unroll 1
  for (int tc = tid; tc < n * ncols; tc += NTHR) {
    const int t = tc >= ncols ? 1 : 0, col = tc - t * ncols;
    float s0 = 0.0f, s1 = 0.0f;
    int o = 0;
#pragma unroll 1
    for (; o + 2 <= cs; o += 2) {
      s0 += ybuf[((size_t)o * NT + t) * L.cols_max + col];
      s1 += ybuf[((size_t)(o + 1) * NT + t) * L.cols_max + col];
    }
    if (o < cs) s0 += ybuf[((size_t)o * NT + t) * L.cols_max + col];
    float rec0 = 0.0f, rec1 = 0.0f;
#pragma unroll 1
    for (int p = 0; p < r; p += 8) {
      const uint4 v8 = *reinterpret_cast<const uint4*>(vo + col * r + p);
      const float4 za = *reinterpret_cast<const float4*>(ztot + t * r + p);
      const float4 zb = *reinterpret_cast<const float4*>(ztot + t * r + p + 4);
      rec0 = fmaf(bf16lo(v8.x), za.x, rec0);
      rec1 = fmaf(bf16hi(v8.x), za.y, rec1);
      rec0 = fmaf(bf16lo(v8.y), za.z, rec0);
      rec1 = fmaf(bf16hi(v8.y), za.w, rec1);
      rec0 = fmaf(bf16lo(v8.z), zb.x, rec0);
      rec1 = fmaf(bf16hi(v8.z), zb.y, rec1);
      rec0 = fmaf(bf16lo(v8.w), zb.z, rec0);
      rec1 = fmaf(bf16hi(v8.w), zb.w, rec1);
    }
    yfin[t * L.cols_max + col] = (s0 + s1) + (rec0 + rec1);
  }
  __syncthreads();
  if (DBG) stamp(a, cid, rank, 14);
  write_and_combine(a, rank, j0, ncols, L.cols_max, yfin, misc, reinterpret_cast<const float*>(misc + MI_RW));
  if (DBG) {
    __syncthreads();
    stamp(a, cid, rank, 15);
  }
}

// ========================================================= batch-1 sparse
// The one-token reader: one cluster per routed expert.  Each CTA screens a
// slice of the expert's channels and pushes its (sigma, ahat) slice and its
// part of the recovery input to every CTA, so that after one exchange every
// CTA holds all I scores and selects the same top-c itself; the candidate
// union is split evenly over the CTAs for the exact stage, whose a values
// are exchanged once more; every CTA then selects the same top-k, reads its
// column slice of the kept down rows (and the recovery rows) and combines.
// Two exchanges in all, and an exact stage balanced over the cluster: at one
// token this is faster than the channel-owning kernel above (30.8 against
// 34.5 us per step on the Qwen layer shape), which wins from two tokens on
// (56.7 against 78.4 us at two).  Prefetching likely rows into L2 ahead of
// the selections, which helps the channel-owning kernel, made this one
// slower (32.4 us) and is left out.
__device__ __forceinline__ void issue_sketch1(const ExpertArgs& a, const Layout& L, char* buf, uint64_t* bars, int e,
                                              int i0, int i1, int ch, int slot) {
  const int c0 = i0 + 16 * ch, cnt = min(16, i1 - c0);
  const uint32_t bytes = cnt * (a.d / 4);
  char* dst = buf + (size_t)slot * 2 * L.skc;
  mbar_expect_tx(&bars[slot], 2 * bytes);
  bulk_g2s(dst, a.sk_gate + ((size_t)e * a.I + c0) * (a.d / 16), bytes, &bars[slot]);
  // test hook: chunk 0's up rows are expected but never copied, so every
  // wait for that chunk runs out (nothing is left in flight)
  if (a.withhold_copy && ch == 0) return;
  bulk_g2s(dst + L.skc, a.sk_up + ((size_t)e * a.I + c0) * (a.d / 16), bytes, &bars[slot]);
}

template <bool DBG>
__global__ void __launch_bounds__(NTHR, 1) reader1_kernel(ExpertArgs a, Layout L) {
  constexpr int NT = 1;         // one token per work item
  constexpr bool FUSED = true;  // routing inside the kernel
  extern __shared__ __align__(128) char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int cid = cluster_id();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.mbar);
  uint64_t* wbars = bars + warp * kMaxSlots;
  uint64_t* skbars = bars + NWARP * kMaxSlots;
  uint64_t* uvbar = skbars + kSkBars;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  int* hist = reinterpret_cast<int*>(smem + L.hist);
  if (tid < NWARP * kMaxSlots + kSkBars + 2) mbar_init(&bars[tid], 1);
  if (tid == 0) misc[MI_DONE] = 0;
  fence_mbar_init();
  __syncthreads();
  if (DBG) stamp(a, cid, rank, 0);

  // Programmatic dependent launch: the next kernel in the stream may be
  // scheduled now (onto free SMs); this one reads nothing in global memory
  // before the previous kernel has completed and its writes are visible.
  pdl_trigger();
  pdl_wait();
  char4 sv_pre = make_char4(0, 0, 0, 0);  // rotation signs of elements 4 tid .. 4 tid + 3 (in-kernel routing)
  if (FUSED) {
    if (tid < a.d / 4) sv_pre = __ldg(reinterpret_cast<const char4*>(a.rot_sign) + tid);
    if (!fused_route<NT>(a, L, smem, misc, cs, rank, cid, cluster, [] {})) return;  // uniform per cluster
  } else {
    if (!load_item_table(a, cid, misc, NT)) return;
  }
  if (DBG) stamp(a, cid, rank, 4);
  const int e = misc[MI_E], n = misc[MI_N];
  const int I = a.I, d = a.d, r = a.r;
  const int i0 = L.ch0[rank], i1 = L.ch0[rank + 1], nown = i1 - i0;
  const int j0 = L.col0[rank], ncols = L.col0[rank + 1] - j0;
  uint32_t* err = a.ws.err;
  char* skbuf = smem + L.ring;
  const int nchunk = cdiv(nown, 16);

  // factor rows of the own channels, V rows of the own columns, and the
  // first round of sketch chunks: all in flight before the token work
  if (tid == 0) {
    if (r > 0) {
      const uint32_t bu = nown * r * 2, bv = ncols * r * 2;
      mbar_expect_tx(uvbar, bu + bv);
      bulk_g2s(smem + L.ubar, a.u_sigma + ((size_t)e * I + i0) * r, bu, uvbar);
      bulk_g2s(smem + L.vown, a.v + ((size_t)e * d + j0) * r, bv, uvbar);
    }
    // the sketch scales of the own channels complete on chunk 0's barrier
    // (every warp waits for chunk 0 before its first channel)
    if (I % 4 == 0 && nown > 0) {
      mbar_expect_tx_only(&skbars[0], 2 * nown * 4);  // chunk 0's copies arrive on it below
      bulk_g2s(smem + L.alpha, a.alpha_gate + (size_t)e * I + i0, nown * 4, &skbars[0]);
      bulk_g2s(smem + L.alpha + L.own_max * 4, a.alpha_up + (size_t)e * I + i0, nown * 4, &skbars[0]);
    }
    const int c1 = min(nchunk, L.sk_round);
    for (int ch = 0; ch < c1; ch++) issue_sketch1(a, L, skbuf, skbars, e, i0, i1, ch, ch);
  }
  float* alg = reinterpret_cast<float*>(smem + L.alpha);
  float* alu = alg + L.own_max;
  if (I % 4 != 0) {  // unaligned scale slices: plain loads, made visible by the barrier below
    for (int li = tid; li < nown; li += NTHR) {
      alg[li] = __ldg(a.alpha_gate + (size_t)e * I + i0 + li);
      alu[li] = __ldg(a.alpha_up + (size_t)e * I + i0 + li);
    }
  }
  int tix[NT];
  if (FUSED) {
    // rotate + quantise every token while the sketch is in flight (the fp32
    // scratch sits past the sketch buffers); its barriers also publish the
    // scales loaded above
    float* scratch = reinterpret_cast<float*>(smem + L.ring + NWARP * L.ring_bytes - d * 4);
#pragma unroll 1
    for (int t = 0; t < a.B; t++)
      rotate_quantize(a, reinterpret_cast<const uint16_t*>(smem + L.x) + (size_t)t * d,
                      reinterpret_cast<int8_t*>(smem + L.q) + (size_t)t * d, scratch,
                      reinterpret_cast<float*>(misc + MI_CX) + t, reinterpret_cast<float*>(misc + MI_RED), sv_pre);
  } else {
    load_tokens(a, L, smem, misc, n, true);
    __syncthreads();
  }
#pragma unroll
  for (int t = 0; t < NT; t++) tix[t] = misc[MI_TIX + (t < n ? t : 0)];
  if (DBG) stamp(a, cid, rank, 1);

  float* sa = reinterpret_cast<float*>(smem + L.sa);          // [I, NT] (sigma, ahat) pairs, slices from the owners
  float* zparts = reinterpret_cast<float*>(smem + L.zparts);  // [cs, NT, r]
  float* z = reinterpret_cast<float*>(smem + L.z);            // [NT, r]
  float* apos = reinterpret_cast<float*>(smem + L.apos);      // [NT, I] by union position
  uint32_t* candm = reinterpret_cast<uint32_t*>(smem + L.candm);
  uint32_t* keptm = reinterpret_cast<uint32_t*>(smem + L.keptm);  // over union positions
  int* ulist = reinterpret_cast<int*>(smem + L.ulist);
  int* dlist = reinterpret_cast<int*>(smem + L.dlist);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.keys);
  const float* cxs = reinterpret_cast<const float*>(misc + MI_CX);

  // ---------------------------------------------------------- S: screen
  {
    const int nv = L.d64;  // 16-byte sketch vectors per row
    int sq[NT];
#pragma unroll
    for (int t = 0; t < NT; t++) {
      const uint4* qv = reinterpret_cast<const uint4*>(smem + L.q + (size_t)tix[t] * d);
      int s = 0;
      for (int j = lane; j < L.d8 / 2; j += 32) {
        const uint4 q4 = qv[j];
        s = __dp4a((int)q4.x, 0x01010101, s);
        s = __dp4a((int)q4.y, 0x01010101, s);
        s = __dp4a((int)q4.z, 0x01010101, s);
        s = __dp4a((int)q4.w, 0x01010101, s);
      }
      sq[t] = warp_sum(s);  // sum of the token's activations: the code offset
    }
    const uint16_t* ub = reinterpret_cast<const uint16_t*>(smem + L.ubar);
    float zacc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
      for (int kk = 0; kk < 4; kk++) zacc[t][kk] = 0.0f;
    bool uv_ready = r == 0;
    // this lane's activations for sketch vector lane (the row's first 32
    // vectors), kept in registers across the channels
    uint4 qr[NT][4];
#pragma unroll
    for (int t = 0; t < NT; t++) {
      const uint4* qv = reinterpret_cast<const uint4*>(smem + L.q + (size_t)tix[t] * d);
#pragma unroll
      for (int kk = 0; kk < 4; kk++) qr[t][kk] = lane < nv ? qv[4 * lane + kk] : make_uint4(0u, 0u, 0u, 0u);
    }
    // warp w takes channel 16 j + w of every sketch chunk j (one channel per
    // warp and chunk).  Each channel's dots are reduced over the warp and
    // parked in the warp's slot of gu; every 4 chunks (and at the end) one
    // pass over the lanes turns the parked sums into sigma and ahat.
    int* gu = hist + warp * 4 * NT * 2;  // [4 channels][NT tokens][g, u]; hist is free during the screen
    int rb = 0, par = 0;  // first chunk of the resident round, parity of its barriers
#pragma unroll 1
    for (int j = 0; j < nchunk; j++) {
      const int li = 16 * j + warp;
      if (j == rb + L.sk_round) {
        // the next round of chunks reuses the buffers: every warp is done with them
        __syncthreads();
        rb = j;
        par ^= 1;
        if (tid == 0) {
          fence_proxy_async();
          const int c1 = min(nchunk, j + L.sk_round);
          for (int ch = j; ch < c1; ch++) issue_sketch1(a, L, skbuf, skbars, e, i0, i1, ch, ch - j);
        }
      }
      int G[NT], U[NT];
#pragma unroll
      for (int t = 0; t < NT; t++) G[t] = U[t] = 0;
      if (li < nown) {
        const int slot = j - rb;
        if (!mbar_wait_bounded(&skbars[slot], par, err, a.wait_ns)) misc[MI_DONE] = 1;
        const uint4* gw = reinterpret_cast<const uint4*>(skbuf + (size_t)slot * 2 * L.skc + warp * (d / 4));
        const uint4* uw = reinterpret_cast<const uint4*>(skbuf + (size_t)slot * 2 * L.skc + L.skc + warp * (d / 4));
        int ga[NT][4], ua[NT][4];
#pragma unroll
        for (int t = 0; t < NT; t++)
#pragma unroll
          for (int kk = 0; kk < 4; kk++) ga[t][kk] = ua[t][kk] = 0;
#pragma unroll 1
        for (int vv = lane; vv < nv; vv += 32) {
          const uint4 g4 = gw[vv], u4 = uw[vv];
#pragma unroll
          for (int t = 0; t < NT; t++) {
            uint4 q0 = qr[t][0], q1 = qr[t][1], q2 = qr[t][2], q3 = qr[t][3];
            if (vv != lane) {
              const uint4* qv = reinterpret_cast<const uint4*>(smem + L.q + (size_t)tix[t] * d) + 4 * vv;
              q0 = qv[0];
              q1 = qv[1];
              q2 = qv[2];
              q3 = qv[3];
            }
            code_dot16(g4.x, q0, ga[t]);
            code_dot16(g4.y, q1, ga[t]);
            code_dot16(g4.z, q2, ga[t]);
            code_dot16(g4.w, q3, ga[t]);
            code_dot16(u4.x, q0, ua[t]);
            code_dot16(u4.y, q1, ua[t]);
            code_dot16(u4.z, q2, ua[t]);
            code_dot16(u4.w, q3, ua[t]);
          }
        }
#pragma unroll
        for (int t = 0; t < NT; t++) {
          G[t] = code_dot_total(ga[t]);
          U[t] = code_dot_total(ua[t]);
        }
      }
      int gs, us;
      reduce_gu<NT>(G, U, gs, us);
      if (lane < 16 && (lane & 7) == 0) {
        const int t = NT == 2 ? lane >> 3 : 0;
        gu[((j & 3) * NT + t) * 2] = gs;
        gu[((j & 3) * NT + t) * 2 + 1] = us;
      }
      if ((j & 3) == 3 || j == nchunk - 1) {
        // the batch's epilogue: lane (channel c, token t), c < 4, t < NT
        __syncwarp();
        const int jb = j & ~3;
        const int c = lane / NT, t = lane - c * NT;
        const int lc = 16 * (jb + c) + warp;
        const bool valid = lane < 4 * NT && jb + c <= j && lc < nown && t < n;
        int g2 = 0, u2 = 0;
        if (lane < 4 * NT) {
          g2 = gu[lane * 2] - (NT == 2 && t ? sq[NT - 1] : sq[0]);
          u2 = gu[lane * 2 + 1] - (NT == 2 && t ? sq[NT - 1] : sq[0]);
        }
        const float cx = cxs[tix[NT == 2 && t ? NT - 1 : 0]];
        const float gh = __fmul_rn(__fmul_rn((float)g2, valid ? alg[lc] : 0.0f), cx);
        const float uh = __fmul_rn(__fmul_rn((float)u2, valid ? alu[lc] : 0.0f), cx);
        const float ah = __fmul_rn(silu_r(gh), uh);
        if (valid) {
          reinterpret_cast<float2*>(sa)[(i0 + lc) * NT + t] = make_float2(fabsf(ah), ah);
          if (DBG) {
            const size_t off = ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * I + i0 + lc;
            if (a.dbg_G) a.dbg_G[off] = g2;
            if (a.dbg_U) a.dbg_U[off] = u2;
            if (a.dbg_sigma) a.dbg_sigma[off] = fabsf(ah);
          }
        }
        // partial recovery input z_w = sum over this warp's channels of ahat_i Ubar_i
        if (r > 0) {
          if (!uv_ready) {
            if (!mbar_wait_bounded(uvbar, 0, err, a.wait_ns)) misc[MI_DONE] = 1;
            uv_ready = true;
          }
#pragma unroll
          for (int cc = 0; cc < 4; cc++) {
            const int lcc = 16 * (jb + cc) + warp;
            if (jb + cc <= j && lcc < nown) {
#pragma unroll
              for (int tt = 0; tt < NT; tt++) {
                const float aht = __shfl_sync(kFull, ah, cc * NT + tt);
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                  const int p = lane + 32 * kk;
                  if (p < r && tt < n) zacc[tt][kk] = fmaf(aht, bf16f(ub[lcc * r + p]), zacc[tt][kk]);
                }
              }
            }
          }
        }
        __syncwarp();
      }
    }
    if (FUSED && warp == NWARP - 1) route_weights(a, L, smem, misc, cid, rank);
    if (DBG) stamp(a, cid, rank, 5);
    // z partials of the CTA, pushed to every CTA: zparts[rank][t]
    if (r > 0) {
      float* zr = reinterpret_cast<float*>(smem + L.zred);  // [NWARP, NT, r]
#pragma unroll
      for (int t = 0; t < NT; t++)
#pragma unroll
        for (int kk = 0; kk < 4; kk++) {
          const int p = lane + 32 * kk;
          if (p < r) zr[(warp * NT + t) * r + p] = zacc[t][kk];
        }
      __syncthreads();
      for (int tp = tid; tp < NT * r; tp += NTHR) {
        float zz = 0.0f;
#pragma unroll
        for (int w = 0; w < NWARP; w++) zz += zr[w * NT * r + tp];
        zparts[rank * NT * r + tp] = zz;
      }
    }
    __syncthreads();
    // push the own (sigma, ahat) slice and z partial to every other CTA: one
    // 16-byte store per thread and peer, all in flight together
    {
      const int nsa4 = cdiv((i1 - i0) * NT * 2, 4), nz4 = r > 0 ? NT * r / 4 : 0, per = nsa4 + nz4;
      const float4* sa4 = reinterpret_cast<const float4*>(sa + i0 * NT * 2);
      const float4* z4 = reinterpret_cast<const float4*>(zparts + rank * NT * r);
#pragma unroll 1
      for (int w = tid; w < (cs - 1) * per; w += NTHR) {
        const int pi = idiv(w, per), j = w - pi * per;
        const int o = pi + (pi >= rank);
        if (j < nsa4) st_cluster(&sa4[j], o, sa4[j]);
        else st_cluster(&z4[j - nsa4], o, z4[j - nsa4]);
      }
    }
  }
  if (DBG) stamp(a, cid, rank, 6);
  cluster.sync();
  if (DBG) stamp(a, cid, rank, 7);

  // ---------------------------------------------------------- c: top-c
#pragma unroll 1
  for (int t = 0; t < n; t++)
    block_select_top(reinterpret_cast<const uint32_t*>(sa) + 2 * t, 2 * NT, I, a.c, hist, misc, candm + t * L.words);
  // union of the candidates, ascending
  block_mask_to_list(candm, n > 1 ? candm + L.words : nullptr, I, ulist, &misc[MI_NU], hist);
  const int nU = misc[MI_NU];
  if (DBG && a.dbg_cand && rank == 0 && warp < n) {
    const int t = warp;
    int base = 0;
    int* out = a.dbg_cand + ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * a.c;
    for (int w0 = 0; w0 < I; w0 += 32) {
      const int p = w0 + lane;
      const bool on = p < I && ((candm[t * L.words + (w0 >> 5)] >> lane) & 1u);
      const unsigned bal = __ballot_sync(kFull, on);
      if (on) out[base + __popc(bal & ((1u << lane) - 1u))] = p;
      base += __popc(bal);
    }
  }
  if (DBG) stamp(a, cid, rank, 8);
  // -------------------------------------------- C: exact candidate stage
  {
    const int u0 = idiv(rank * nU + cs - 1, cs), u1 = idiv((rank + 1) * nU + cs - 1, cs), nsl = u1 - u0;
    const int m0 = (warp * nsl) / NWARP, m1 = ((warp + 1) * nsl) / NWARP;
    const int rowb = d * 2;
    const int P = max(1, min(kMaxSlots, L.c_slots));
    const uint4* xs = reinterpret_cast<const uint4*>(smem + L.x);
    const int vx = L.d8;
    char* ring = smem + L.ring + warp * L.ring_bytes;
    uint32_t par = 0;
    warp_stream(
        m1 - m0, P, wbars, par, err,
        [&](int j, int s, uint64_t* bar) {
          const int i = ulist[u0 + m0 + j];
          char* dst = ring + s * 2 * rowb;
          mbar_expect_tx(bar, 2 * rowb);
          bulk_g2s(dst, a.w_gate + ((size_t)e * I + i) * d, rowb, bar);
          bulk_g2s(dst + rowb, a.w_up + ((size_t)e * I + i) * d, rowb, bar);
          if (j + P < m1 - m0) {
            // the row this slot takes next starts moving into L2 now
            const int i2 = ulist[u0 + m0 + j + P];
            bulk_prefetch_l2(a.w_gate + ((size_t)e * I + i2) * d, rowb);
            bulk_prefetch_l2(a.w_up + ((size_t)e * I + i2) * d, rowb);
          }
        },
        [&](int j, int s) {
          const int u = u0 + m0 + j, i = ulist[u];
          const uint4* gr = reinterpret_cast<const uint4*>(ring + s * 2 * rowb);
          const uint4* ur = gr + vx;
          float g0[NT], g1[NT], v0[NT], v1[NT];
#pragma unroll
          for (int t = 0; t < NT; t++) g0[t] = g1[t] = v0[t] = v1[t] = 0.0f;
#pragma unroll 2
          for (int vv = lane; vv < vx; vv += 32) {
            const uint4 gv = gr[vv], uv = ur[vv];
#pragma unroll
            for (int t = 0; t < NT; t++) {
              const uint4 xv = xs[tix[t] * vx + vv];
              dot8_mixed(gv, xv, g0[t], g1[t]);
              dot8_mixed(uv, xv, v0[t], v1[t]);
            }
          }
#pragma unroll
          for (int t = 0; t < NT; t++) {
            if (t < n) {
              const float gs = warp_sum(g0[t] + g1[t]), us = warp_sum(v0[t] + v1[t]);
              const bool is_c = (candm[t * L.words + (i >> 5)] >> (i & 31)) & 1u;
              const float av = is_c ? __fmul_rn(silu_r(gs), us) : 0.0f;
              if (lane == 0) apos[t * I + u] = av;
            }
          }
        },
        a.wait_ns);
    // push the own a values to every other CTA, one store per thread and peer
    __syncthreads();
    const int per = n * nsl;
#pragma unroll 1
    for (int w = tid; w < (cs - 1) * per; w += NTHR) {
      const int pi = idiv(w, per), j = w - pi * per;
      const int o = pi + (pi >= rank);
      const int t = j >= nsl ? 1 : 0, u = u0 + j - t * nsl;
      st_cluster(&apos[t * I + u], o, apos[t * I + u]);
    }
  }
  if (DBG) stamp(a, cid, rank, 9);
  cluster.sync();  // the last exchange: no CTA touches another's smem after this
  if (DBG) stamp(a, cid, rank, 10);

  // ------------------------------------------------------------ k: top-k
  // over union positions; a token's non-candidates get key 0, its candidates
  // |a| + 1 (same order, ties still to the lower channel)
#pragma unroll 1
  for (int t = 0; t < n; t++) {
    for (int u = tid; u < nU; u += NTHR) {
      const int i = ulist[u];
      const bool c = (candm[t * L.words + (i >> 5)] >> (i & 31)) & 1u;
      keys[u] = c ? __float_as_uint(fabsf(apos[t * I + u])) + 1u : 0u;
    }
    __syncthreads();
    block_select_top(keys, 1, nU, a.k, hist, misc, keptm + t * L.words);
    if (DBG && a.dbg_kept && rank == 0 && warp == 0) {
      const size_t off = ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * a.k;
      int base = 0;
      for (int w0 = 0; w0 < nU; w0 += 32) {
        const int u = w0 + lane;
        const bool on = u < nU && ((keptm[t * L.words + (w0 >> 5)] >> lane) & 1u);
        const unsigned bal = __ballot_sync(kFull, on);
        const int at = base + __popc(bal & ((1u << lane) - 1u));
        if (on && at < a.k) {
          a.dbg_kept[off + at] = ulist[u];
          if (a.dbg_a_kept) a.dbg_a_kept[off + at] = apos[t * I + u];
        }
        base += __popc(bal);
      }
    }
  }
  // rows of the down stage: union positions kept by any token
  block_mask_to_list(keptm, n > 1 ? keptm + L.words : nullptr, nU, dlist, &misc[MI_ND], hist);
  const int nD = misc[MI_ND];
  if (DBG) stamp(a, cid, rank, 11);

  // ---------------------------------------------- D: down rows + recovery
  float* red = reinterpret_cast<float*>(smem + L.ring);
  const int ncq = ncols >> 3, nr8 = r >> 3, nch = ncq + nr8;
  // Rows: the kept union (recovery from the sketch estimates of every skipped
  // channel: the factor rows of the kept channels enter with -ahat), or, with
  // the exact recovery input, the whole candidate union (factor rows of the
  // candidates enter with -(ahat - a) when dropped, -ahat when kept; down
  // rows are read for the kept ones only).
  const bool rec_exact = a.recovery_input == 1;
  const int rg = down_rows<NT>(
      a, e, j0, ncq, nr8, rec_exact ? nU : nD, r, [&](int m) { return ulist[rec_exact ? m : dlist[m]]; },
      [&](int m, int i, bool is_w, float (&co)[NT]) {
        const int u = rec_exact ? m : dlist[m];
        bool need = false;
#pragma unroll
        for (int t = 0; t < NT; t++) {
          const bool kept = t < n && ((keptm[t * L.words + (u >> 5)] >> (u & 31)) & 1u);
          const bool cand = t < n && ((candm[t * L.words + (i >> 5)] >> (i & 31)) & 1u);
          const float ah = sa[(i * NT + t) * 2 + 1];
          if (is_w) co[t] = kept ? apos[t * I + u] : 0.0f;
          else if (kept) co[t] = ah;
          else co[t] = rec_exact && cand ? __fsub_rn(ah, apos[t * I + u]) : 0.0f;
          need |= kept || (!is_w && rec_exact && cand);
        }
        return need;
      },
      red);
  float* yfin = reinterpret_cast<float*>(smem + L.x);  // [n, cols_max]; x is no longer needed
#pragma unroll 1
  for (int o = tid; o < n * nch * 8; o += NTHR) {
    const int t = o >= nch * 8 ? 1 : 0;
    const int oc = o - t * nch * 8;
    const float* rp = red + (size_t)t * nch * 8 + oc;
    const int gstride = NT * nch * 8;
    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
    int gg = 0;
#pragma unroll 1
    for (; gg + 4 <= rg; gg += 4) {
      s0 += rp[(gg + 0) * gstride];
      s1 += rp[(gg + 1) * gstride];
      s2 += rp[(gg + 2) * gstride];
      s3 += rp[(gg + 3) * gstride];
    }
    for (; gg < rg; gg++) s0 += rp[gg * gstride];
    const float s = (s0 + s1) + (s2 + s3);
    if (oc < ncols) {
      yfin[t * L.cols_max + oc] = s;
    } else {
      // z = (sum over the CTAs' partials of all channels) - (the kept part)
      const int p = oc - ncols;
      float z0 = 0.0f, z1 = 0.0f;
      int o = 0;
#pragma unroll 1
      for (; o + 2 <= cs; o += 2) {
        z0 += zparts[(o * NT + t) * r + p];
        z1 += zparts[((o + 1) * NT + t) * r + p];
      }
      if (o < cs) z0 += zparts[(o * NT + t) * r + p];
      z[t * r + p] = (z0 + z1) - s;
    }
  }
  if (r > 0) {
    if (!mbar_wait_bounded(uvbar, 0, err, a.wait_ns)) misc[MI_DONE] = 1;
    __syncthreads();
    const uint16_t* vo = reinterpret_cast<const uint16_t*>(smem + L.vown);
#pragma unroll 1
    for (int t = 0; t < n; t++)
      for (int col = tid; col < ncols; col += NTHR) {
        float rec0 = 0.0f, rec1 = 0.0f;
#pragma unroll 4
        for (int p = 0; p < r; p += 8) {
          const uint4 v8 = *reinterpret_cast<const uint4*>(vo + col * r + p);
          const float4 za = *reinterpret_cast<const float4*>(z + t * r + p);
          const float4 zb = *reinterpret_cast<const float4*>(z + t * r + p + 4);
          rec0 = fmaf(bf16lo(v8.x), za.x, rec0);
          rec1 = fmaf(bf16hi(v8.x), za.y, rec1);
          rec0 = fmaf(bf16lo(v8.y), za.z, rec0);
          rec1 = fmaf(bf16hi(v8.y), za.w, rec1);
          rec0 = fmaf(bf16lo(v8.z), zb.x, rec0);
          rec1 = fmaf(bf16hi(v8.z), zb.y, rec1);
          rec0 = fmaf(bf16lo(v8.w), zb.z, rec0);
          rec1 = fmaf(bf16hi(v8.w), zb.w, rec1);
        }
        yfin[t * L.cols_max + col] += rec0 + rec1;
      }
  }
  __syncthreads();
  if (DBG) stamp(a, cid, rank, 12);
  write_and_combine(a, rank, j0, ncols, L.cols_max, yfin, misc,
                    FUSED ? reinterpret_cast<const float*>(misc + MI_RW) : a.ws.wts);
  if (DBG) {
    __syncthreads();
    stamp(a, cid, rank, 15);
  }
}

// ================================================================= dense
template <int NT, bool FUSED>
__global__ void __launch_bounds__(NTHR, 1) dense_kernel(ExpertArgs a, Layout L) {
  extern __shared__ __align__(128) char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int cid = cluster_id();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.mbar);
  uint64_t* wbars = bars + warp * kMaxSlots;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  if (tid < NWARP * kMaxSlots + kSkBars + 2) mbar_init(&bars[tid], 1);
  if (tid == 0) misc[MI_DONE] = 0;
  fence_mbar_init();
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  if (FUSED) {
    if (!fused_route<NT>(a, L, smem, misc, cs, rank, cid, cluster, [] {})) return;
    if (warp == NWARP - 1) route_weights(a, L, smem, misc, cid, rank);
  } else {
    if (!load_item_table(a, cid, misc, NT)) return;
    load_tokens(a, L, smem, misc, misc[MI_N], false);
    __syncthreads();
  }
  const int e = misc[MI_E], n = misc[MI_N];
  const int I = a.I, d = a.d;
  const int i0 = L.ch0[rank], nown = L.ch0[rank + 1] - i0;
  const int j0 = L.col0[rank], ncols = L.col0[rank + 1] - j0;
  uint32_t* err = a.ws.err;
  uint32_t par = 0;
  char* ring = smem + L.ring + warp * L.ring_bytes;
  int tix[NT];
#pragma unroll
  for (int t = 0; t < NT; t++) tix[t] = misc[MI_TIX + (t < n ? t : 0)];
  float* h = reinterpret_cast<float*>(smem + L.sig);  // [NT, I] pushed by the owners
  {
    const int m0 = (warp * nown) / NWARP, m1 = ((warp + 1) * nown) / NWARP;
    const int rowb = d * 2, vx = L.d8;
    const int P = max(1, min(kMaxSlots, L.c_slots));
    const uint4* xs = reinterpret_cast<const uint4*>(smem + L.x);
    warp_stream(
        m1 - m0, P, wbars, par, err,
        [&](int j, int s, uint64_t* bar) {
          const int i = i0 + m0 + j;
          char* dst = ring + s * 2 * rowb;
          mbar_expect_tx(bar, 2 * rowb);
          bulk_g2s(dst, a.w_gate + ((size_t)e * I + i) * d, rowb, bar);
          bulk_g2s(dst + rowb, a.w_up + ((size_t)e * I + i) * d, rowb, bar);
          if (j + P < m1 - m0) {
            // the row this slot takes next starts moving into L2 now
            bulk_prefetch_l2(a.w_gate + ((size_t)e * I + i + P) * d, rowb);
            bulk_prefetch_l2(a.w_up + ((size_t)e * I + i + P) * d, rowb);
          }
        },
        [&](int j, int s) {
          const int i = i0 + m0 + j;
          const uint4* gr = reinterpret_cast<const uint4*>(ring + s * 2 * rowb);
          const uint4* ur = gr + vx;
          float g0[NT], g1[NT], v0[NT], v1[NT];
#pragma unroll
          for (int t = 0; t < NT; t++) g0[t] = g1[t] = v0[t] = v1[t] = 0.0f;
#pragma unroll 2
          for (int vv = lane; vv < vx; vv += 32) {
            const uint4 gv = gr[vv], uv = ur[vv];
#pragma unroll
            for (int t = 0; t < NT; t++) {
              const uint4 xv = xs[tix[t] * vx + vv];
              dot8_mixed(gv, xv, g0[t], g1[t]);
              dot8_mixed(uv, xv, v0[t], v1[t]);
            }
          }
#pragma unroll
          for (int t = 0; t < NT; t++) {
            if (t < n) {
              const float gs = warp_sum(g0[t] + g1[t]), us = warp_sum(v0[t] + v1[t]);
              if (lane < cs) st_cluster(&h[t * I + i], lane, __fmul_rn(silu_r(gs), us));
            }
          }
        });
  }
  cluster.sync();  // the only exchange: no CTA touches another's smem after this
  float* red = reinterpret_cast<float*>(smem + L.ring);
  const int ncq = ncols >> 3;
  const int rg = down_rows<NT>(
      a, e, j0, ncq, 0, I, 0, [](int m) { return m; },
      [&](int m, int, bool, float (&co)[NT]) {
#pragma unroll
        for (int t = 0; t < NT; t++) co[t] = t < n ? h[t * I + m] : 0.0f;
        return true;
      },
      red);
  float* out = reinterpret_cast<float*>(smem + L.x);
#pragma unroll 1
  for (int o = tid; o < n * ncq * 8; o += NTHR) {
    const int t = o >= ncq * 8 ? 1 : 0;
    const int oc = o - t * ncq * 8;
    const float* rp = red + (size_t)t * ncq * 8 + oc;
    const int gstride = NT * ncq * 8;
    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
    int gg = 0;
#pragma unroll 1
    for (; gg + 4 <= rg; gg += 4) {
      s0 += rp[(gg + 0) * gstride];
      s1 += rp[(gg + 1) * gstride];
      s2 += rp[(gg + 2) * gstride];
      s3 += rp[(gg + 3) * gstride];
    }
    for (; gg < rg; gg++) s0 += rp[gg * gstride];
    out[t * L.cols_max + oc] = (s0 + s1) + (s2 + s3);
  }
  __syncthreads();
  write_and_combine(a, rank, j0, ncols, L.cols_max, out, misc,
                    FUSED ? reinterpret_cast<const float*>(misc + MI_RW) : a.ws.wts);
}

// ---------------------------------------------------------- launch plans
// Cluster size: among the sizes that fit the shape, the one with the least
// estimated time, waves * (1 + 8 / cs) with waves = ceil(items / co-resident
// clusters): a wave costs a fixed latency plus work that shrinks with the
// cluster's width.  `force_cs` (ExpertArgs::force_cs) pins it.

int occupancy_clusters(const void* f, int cs, int smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs);
  cfg.blockDim = dim3(NTHR);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nc = 0;
  if (cudaOccupancyMaxActiveClusters(&nc, f, &cfg) != cudaSuccess) {
    cudaGetLastError();
    nc = 0;
  }
  return nc;
}

// ----- dense block
struct DensePlan {
  int dev, NT, fused, B, E, I, d, items, forced;
  int cs, ring_rows, smem, max_clusters;
  Layout L;
};

template <int NT, bool FUSED>
const void* dense_ptr() {
  return reinterpret_cast<const void*>(&dense_kernel<NT, FUSED>);
}
static_assert(kMaxGroup == 2, "kernels are instantiated for 1 and 2 tokens per item");
const void* pick_dense(int NT, bool fused) {
  if (NT == 1) return fused ? dense_ptr<1, true>() : dense_ptr<1, false>();
  return fused ? dense_ptr<2, true>() : dense_ptr<2, false>();
}

// Ring: the deepest that fits, with room for the down stage's partial sums
// (NT x 16 KB).
cudaError_t plan_dense(const ExpertArgs& a, DensePlan* out) {
  thread_local DensePlan cache[8];
  thread_local int ncache = 0, next = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int NT = a.nmax <= 1 ? 1 : 2;
  const bool fused = fused_routing(a.B);
  const int items = fused ? (a.B * a.top_e < a.E ? a.B * a.top_e : a.E) : a.ws.max_items;
  for (int i = 0; i < ncache; i++) {
    const DensePlan& c = cache[i];
    if (c.dev == dev && c.NT == NT && c.fused == (int)fused && c.B == a.B && c.E == a.E && c.I == a.I &&
        c.d == a.d && c.items == items && c.forced == a.force_cs) {
      *out = c;
      return cudaSuccess;
    }
  }
  int smem_max = 0;
  err = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (err != cudaSuccess) return err;
  const void* f = pick_dense(NT, fused);
  err = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (err != cudaSuccess) return err;
  DensePlan p = {dev, NT, (int)fused, a.B, a.E, a.I, a.d, items, a.force_cs, 0, 0, 0, 0, {}};
  double best = 1e30;
  const int ntok = fused ? a.B : NT;
  for (int cs = 16; cs >= 8; cs--) {
    if (a.force_cs && cs != a.force_cs) continue;
    const int cols_max = 8 * cdiv(a.d / 8, cs);
    if (cols_max > kMaxCols || a.I < cs || (fused && a.E < cs)) continue;
    const int red_need = NT * NTHR * 8 * 4;
    int rr = 0;
    for (int t = 2; t <= 64; t++) {
      const Layout L = make_layout(NT, ntok, fused, a.E, a.I, a.d, 0, cs, t, true);
      if (L.total > smem_max) break;
      if (L.c_slots >= 1 && NWARP * L.ring_bytes >= red_need) rr = t;
    }
    if (rr < 2) continue;
    const Layout L = make_layout(NT, ntok, fused, a.E, a.I, a.d, 0, cs, rr, true);
    err = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (err != cudaSuccess) return err;
    const int nclusters = occupancy_clusters(f, cs, L.total);
    if (nclusters < 1) continue;
    const double cost = (double)cdiv(items, nclusters) * (1.0 + 8.0 / cs);
    if (cost < best - 1e-12) {
      best = cost;
      p.cs = cs;
      p.ring_rows = rr;
      p.smem = L.total;
      p.max_clusters = nclusters;
      p.L = L;
    }
  }
  if (p.cs == 0) return cudaErrorInvalidConfiguration;
  if (ncache < 8) cache[ncache++] = p;
  else cache[next++ % 8] = p;
  *out = p;
  return cudaSuccess;
}

// ----- sparse reader (one or two tokens)
struct ReaderPlan {
  int dev, B, E, I, d, r, top_e, forced, sk3;
  int cs, smem, max_clusters, items;
  RLayout L;
};

template <int NT, bool SK3>
const void* reader_ptr_f(bool dbg) {
  return dbg ? reinterpret_cast<const void*>(&reader_kernel<NT, true, SK3>)
             : reinterpret_cast<const void*>(&reader_kernel<NT, false, SK3>);
}
const void* reader_ptr(int NT, bool sk3, bool dbg) {
  if (NT == 1) return sk3 ? reader_ptr_f<1, true>(dbg) : reader_ptr_f<1, false>(dbg);
  return sk3 ? reader_ptr_f<2, true>(dbg) : reader_ptr_f<2, false>(dbg);
}

cudaError_t plan_reader(const ExpertArgs& a, ReaderPlan* out) {
  thread_local ReaderPlan cache[8];
  thread_local int ncache = 0, next = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (a.B > kMaxGroup) return cudaErrorInvalidConfiguration;
  for (int i = 0; i < ncache; i++) {
    const ReaderPlan& c = cache[i];
    if (c.dev == dev && c.B == a.B && c.E == a.E && c.I == a.I && c.d == a.d && c.r == a.r &&
        c.top_e == a.top_e && c.forced == a.force_cs && c.sk3 == a.sk3) {
      *out = c;
      return cudaSuccess;
    }
  }
  int smem_max = 0;
  err = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (err != cudaSuccess) return err;
  const int NT = a.B;
  const bool sk3 = a.sk3 != 0;
  const void* fns[2] = {reader_ptr(NT, sk3, false), reader_ptr(NT, sk3, true)};
  for (const void* f : fns) {
    err = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
  const int items = a.B * a.top_e < a.E ? a.B * a.top_e : a.E;
  ReaderPlan p = {dev, a.B, a.E, a.I, a.d, a.r, a.top_e, a.force_cs, a.sk3, 0, 0, 0, items, {}};
  double best = 1e30;
  for (int cs = 16; cs >= 2; cs--) {
    if (a.force_cs && cs != a.force_cs) continue;
    if (a.I < 4 * cs || a.E < cs || 8 * cdiv(a.d / 8, cs) > a.d) continue;
    const RLayout L = make_rlayout(NT, a.B, a.E, a.I, a.d, a.r, cs, smem_max, sk3);
    if (L.own_max > kMaxOwn || L.W < 4 || L.nskbuf < 1 || L.ndslot < 1 || L.total > smem_max) continue;
    int nclusters = 1 << 30;
    for (const void* f : fns) {
      err = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
      if (err != cudaSuccess) return err;
      const int nc = occupancy_clusters(f, cs, L.total);
      nclusters = nc < nclusters ? nc : nclusters;
    }
    if (nclusters < 1) continue;
    const double cost = (double)cdiv(items, nclusters) * (1.0 + 8.0 / cs);
    if (cost < best - 1e-12) {
      best = cost;
      p.cs = cs;
      p.smem = L.total;
      p.max_clusters = nclusters;
      p.L = L;
    }
  }
  if (p.cs == 0) return cudaErrorInvalidConfiguration;
  if (ncache < 8) cache[ncache++] = p;
  else cache[next++ % 8] = p;
  *out = p;
  return cudaSuccess;
}

// ----- batch-1 sparse reader (reader1_kernel)
struct Reader1Plan {
  int dev, E, I, d, r, top_e, forced;
  int cs, ring_rows, smem, max_clusters, items;
  Layout L;
};

const void* reader1_ptr(bool dbg) {
  return dbg ? reinterpret_cast<const void*>(&reader1_kernel<true>)
             : reinterpret_cast<const void*>(&reader1_kernel<false>);
}

// Cluster size 8..16 by the same estimate as the dense block; ring: the
// deepest that fits with room for the down stage's partial sums, the
// rotation scratch and at least one sketch chunk.
cudaError_t plan_reader1(const ExpertArgs& a, Reader1Plan* out) {
  thread_local Reader1Plan cache[8];
  thread_local int ncache = 0, next = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  for (int i = 0; i < ncache; i++) {
    const Reader1Plan& c = cache[i];
    if (c.dev == dev && c.E == a.E && c.I == a.I && c.d == a.d && c.r == a.r && c.top_e == a.top_e &&
        c.forced == a.force_cs) {
      *out = c;
      return cudaSuccess;
    }
  }
  int smem_max = 0;
  err = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (err != cudaSuccess) return err;
  const void* fns[2] = {reader1_ptr(false), reader1_ptr(true)};
  for (const void* f : fns) {
    err = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
  const int items = a.top_e < a.E ? a.top_e : a.E;
  Reader1Plan p = {dev, a.E, a.I, a.d, a.r, a.top_e, a.force_cs, 0, 0, 0, 0, items, {}};
  double best = 1e30;
  for (int cs = 16; cs >= 8; cs--) {
    if (a.force_cs && cs != a.force_cs) continue;
    const int cols_max = 8 * cdiv(a.d / 8, cs);
    if (cols_max > kMaxCols || a.I < cs || a.E < cs) continue;
    const int red_need = NTHR * 8 * 4;
    int rr = 0;
    for (int t = 2; t <= 64; t++) {
      const Layout L = make_layout(1, 1, true, a.E, a.I, a.d, a.r, cs, t, false);
      if (L.total > smem_max) break;
      if (L.c_slots >= 1 && NWARP * L.ring_bytes >= red_need && L.sk_round >= 1) rr = t;
    }
    if (rr < 2) continue;
    const Layout L = make_layout(1, 1, true, a.E, a.I, a.d, a.r, cs, rr, false);
    int nclusters = 1 << 30;
    for (const void* f : fns) {
      err = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
      if (err != cudaSuccess) return err;
      const int nc = occupancy_clusters(f, cs, L.total);
      nclusters = nc < nclusters ? nc : nclusters;
    }
    if (nclusters < 1) continue;
    const double cost = (double)cdiv(items, nclusters) * (1.0 + 8.0 / cs);
    if (cost < best - 1e-12) {
      best = cost;
      p.cs = cs;
      p.ring_rows = rr;
      p.smem = L.total;
      p.max_clusters = nclusters;
      p.L = L;
    }
  }
  if (p.cs == 0) return cudaErrorInvalidConfiguration;
  if (ncache < 8) cache[ncache++] = p;
  else cache[next++ % 8] = p;
  *out = p;
  return cudaSuccess;
}

// The batch-1 kernel takes one-token steps on 2-bit sketch rows, with
// clusters of 8 to 16 CTAs (a pinned size below 8 runs the channel-owning
// kernel).
bool use_reader1(const ExpertArgs& a) { return a.B == 1 && a.sk3 == 0 && (a.force_cs == 0 || a.force_cs >= 8); }

cudaLaunchConfig_t cluster_config(int grid, int cs, int smem, cudaStream_t s, cudaLaunchAttribute (&attr)[2]) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NTHR);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;  // programmatic dependent launch: overlaps this launch with the previous kernel's tail
  return cfg;
}

}  // namespace

bool fused_routing(int B) { return B <= kMaxGroup; }

bool reader_supports(int B, int d) { return B <= kMaxGroup && d <= 2048; }

cudaError_t launch_reader(const ExpertArgs& a0, cudaStream_t s) {
  ExpertArgs a = a0;
  const bool dbg = a.dbg_ids || a.dbg_w || a.dbg_G || a.dbg_U || a.dbg_sigma || a.dbg_cand || a.dbg_kept ||
                   a.dbg_a_kept || a.dbg_y_expert || a.dbg_phase;
  if (use_reader1(a)) {
    Reader1Plan p1;
    cudaError_t e1 = plan_reader1(a, &p1);
    if (e1 != cudaSuccess) return e1;
    a.cs = p1.cs;
    a.ring_rows = p1.ring_rows;
    const void* f1 = reader1_ptr(dbg);
    e1 = cudaFuncSetAttribute(f1, cudaFuncAttributeMaxDynamicSharedMemorySize, p1.smem);
    if (e1 != cudaSuccess) return e1;
    cudaLaunchAttribute at1[2];
    cudaLaunchConfig_t c1 = cluster_config(p1.items * a.cs, a.cs, p1.smem, s, at1);
    void* args1[] = {&a, &p1.L};
    return cudaLaunchKernelExC(&c1, f1, args1);
  }
  ReaderPlan plan;
  cudaError_t err = plan_reader(a, &plan);
  if (err != cudaSuccess) return err;
  a.cs = plan.cs;
  const void* fn = reader_ptr(a.B, a.sk3 != 0, dbg);
  err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, plan.smem);
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = cluster_config(plan.items * a.cs, a.cs, plan.smem, s, attr);
  void* args[] = {&a, &plan.L};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

cudaError_t launch_dense(const ExpertArgs& a0, cudaStream_t s) {
  ExpertArgs a = a0;
  DensePlan plan;
  cudaError_t err = plan_dense(a, &plan);
  if (err != cudaSuccess) return err;
  a.cs = plan.cs;
  a.ring_rows = plan.ring_rows;
  const void* fn = pick_dense(plan.NT, plan.fused);
  err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, plan.smem);
  if (err != cudaSuccess) return err;
  const int items = plan.fused ? plan.items : a.ws.max_items;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = cluster_config(items * a.cs, a.cs, plan.smem, s, attr);
  void* args[] = {&a, &plan.L};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

cudaError_t query_plan(const ExpertArgs& a, bool dense, int out[4]) {
  if (dense) {
    DensePlan p;
    cudaError_t e = plan_dense(a, &p);
    if (e != cudaSuccess) return e;
    out[0] = p.cs;
    out[1] = p.ring_rows;
    out[2] = p.smem;
    out[3] = p.max_clusters;
    return cudaSuccess;
  }
  if (use_reader1(a)) {
    Reader1Plan p1;
    cudaError_t e1 = plan_reader1(a, &p1);
    if (e1 != cudaSuccess) return e1;
    out[0] = p1.cs;
    out[1] = p1.ring_rows;
    out[2] = p1.smem;
    out[3] = p1.max_clusters;
    return cudaSuccess;
  }
  ReaderPlan p;
  cudaError_t e = plan_reader(a, &p);
  if (e != cudaSuccess) return e;
  out[0] = p.cs;
  out[1] = p.L.P * NWARP + p.L.Pext;
  out[2] = p.smem;
  out[3] = p.max_clusters;
  return cudaSuccess;
}

}  // namespace moe
