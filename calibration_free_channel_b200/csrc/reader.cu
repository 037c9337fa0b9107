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
#include "common.cuh"
#include "kernels.h"
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
  MI_E = 0, MI_N, MI_NU, MI_ND, MI_DIG, MI_REM, MI_CNT, MI_DONE,
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
                                            Issue issue, Consume consume) {
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
    ok = mbar_wait_bounded(&bars[s], (par >> s) & 1u, err);
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
        if (mbar_wait_bounded(&bars[q], (par >> q) & 1u, err)) par ^= 1u << q;
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
    int v = 0;
    if (lane == 0) v = *a.ws.n_items;
    else if (lane == 1 && ok_cid) v = a.ws.item_e[cid];
    else if (lane == 2 && ok_cid) v = a.ws.item_n[cid];
    else if (lane >= 4 && lane < 4 + kMaxGroup && ok_cid) v = a.ws.item_tok[cid * kMaxGroup + lane - 4];
    else if (lane >= 8 && lane < 8 + kMaxGroup && ok_cid) v = a.ws.item_slot[cid * kMaxGroup + lane - 8];
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
      reinterpret_cast<float*>(misc + MI_CX)[t] = a.ws.cx[tok];
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

// Rotation + int8 quantisation of smem token t: v = FWHT(s . x) in the fp32
// scratch (d floats), q = rint(127 v / amax), c_x = amax / (127 d).  Stages
// h = 1, 2 run in registers (thread c holds elements 4c .. 4c+3) and
// h = 4 .. 64 across the lanes of a warp (a warp holds 128 consecutive
// elements); from h = 128 on, each pass over shared memory applies two stages
// (h and 2h) to four elements held in registers, and a last single stage
// runs alone when the count is odd.  Every element sees the reference
// butterflies (a + b, a - b) of every stage in the reference stage order, so
// the bits equal the reference transform's.  d >= 256.  sv_pre holds the
// signs of elements 4T .. 4T+3, loaded early by the caller.
__device__ void rotate_quantize(const ExpertArgs& a, const Layout& L, char* smem, int t, float* v, float* cx_out,
                                float* red, char4 sv_pre) {
  const int d = a.d;
  const int T = threadIdx.x, lane = T & 31, warp = T >> 5;
  for (int c = T; c < 2 * L.d8; c += NTHR) {  // d / 4 is a multiple of 32: whole warps
    const uint2 xv = reinterpret_cast<const uint2*>(smem + L.x + (size_t)t * d * 2)[c];
    const char4 sv = c == T ? sv_pre : reinterpret_cast<const char4*>(a.rot_sign)[c];
    float r0 = (float)sv.x * bf16lo(xv.x), r1 = (float)sv.y * bf16hi(xv.x);
    float r2 = (float)sv.z * bf16lo(xv.y), r3 = (float)sv.w * bf16hi(xv.y);
    float b0 = __fadd_rn(r0, r1), b1 = __fsub_rn(r0, r1), b2 = __fadd_rn(r2, r3), b3 = __fsub_rn(r2, r3);  // h = 1
    r0 = __fadd_rn(b0, b2);  // h = 2
    r2 = __fsub_rn(b0, b2);
    r1 = __fadd_rn(b1, b3);
    r3 = __fsub_rn(b1, b3);
#pragma unroll 1
    for (int m = 1; m < 32; m <<= 1) {  // h = 4m: partner lane ^ m
      const bool up = lane & m;
      const float p0 = __shfl_xor_sync(kFull, r0, m), p1 = __shfl_xor_sync(kFull, r1, m);
      const float p2 = __shfl_xor_sync(kFull, r2, m), p3 = __shfl_xor_sync(kFull, r3, m);
      r0 = up ? __fsub_rn(p0, r0) : __fadd_rn(r0, p0);
      r1 = up ? __fsub_rn(p1, r1) : __fadd_rn(r1, p1);
      r2 = up ? __fsub_rn(p2, r2) : __fadd_rn(r2, p2);
      r3 = up ? __fsub_rn(p3, r3) : __fadd_rn(r3, p3);
    }
    reinterpret_cast<float4*>(v)[c] = make_float4(r0, r1, r2, r3);
  }
  float m = 0.0f;  // max |v| over this thread's outputs of the last pass
#pragma unroll 1
  for (int h = 128, lh = 7; h < d;) {
    __syncthreads();
    m = 0.0f;
    if (2 * h < d) {
      for (int p = T; p < 2 * L.d8; p += NTHR) {
        const int b = ((p >> lh) << (lh + 2)) | (p & (h - 1));
        const float a0 = v[b], a1 = v[b + h], a2 = v[b + 2 * h], a3 = v[b + 3 * h];
        const float s0 = __fadd_rn(a0, a1), s1 = __fsub_rn(a0, a1);  // stage h
        const float s2 = __fadd_rn(a2, a3), s3 = __fsub_rn(a2, a3);
        const float o0 = __fadd_rn(s0, s2), o2 = __fsub_rn(s0, s2);  // stage 2h
        const float o1 = __fadd_rn(s1, s3), o3 = __fsub_rn(s1, s3);
        v[b] = o0;
        v[b + h] = o1;
        v[b + 2 * h] = o2;
        v[b + 3 * h] = o3;
        m = fmaxf(m, fmaxf(fmaxf(fabsf(o0), fabsf(o1)), fmaxf(fabsf(o2), fabsf(o3))));
      }
      h <<= 2;
      lh += 2;
    } else {  // the last stage, h = d / 2
      for (int p = T; p < 4 * L.d8; p += NTHR) {
        const float x0 = v[p], x1 = v[p + h];
        const float o0 = __fadd_rn(x0, x1), o1 = __fsub_rn(x0, x1);
        v[p] = o0;
        v[p + h] = o1;
        m = fmaxf(m, fmaxf(fabsf(o0), fabsf(o1)));
      }
      h <<= 1;
      lh += 1;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float amax = 0.0f;
#pragma unroll
  for (int w = 0; w < NWARP; w += 4) {
    const float4 r4 = reinterpret_cast<const float4*>(red)[w >> 2];
    amax = fmaxf(amax, fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w)));
  }
  int8_t* q = reinterpret_cast<int8_t*>(smem + L.q) + (size_t)t * d;
  for (int j = T; j < d; j += NTHR) {
    int n = 0;
    if (amax > 0.0f) n = max(-127, min(127, __float2int_rn(__fdiv_rn(__fmul_rn(v[j], 127.0f), amax))));
    q[j] = (int8_t)n;
  }
  if (T == 0) *cx_out = amax > 0.0f ? __fdiv_rn(amax, __fmul_rn(127.0f, (float)d)) : 0.0f;
  __syncthreads();
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
    w[u] = j < d8 ? __ldg(row + j) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// In-kernel routing (B <= NT <= 2): every CTA loads all tokens and computes
// the logits of its slice of experts (one warp per expert; the router row is
// read straight into registers, overlapping the token loads) and pushes them
// to all CTAs; after the cluster barrier every CTA takes the same top-e and
// one warp derives the softmax weights and this cluster's work item (one
// item per routed expert, experts ascending).  Returns false if this cluster
// has no item.
template <int NT>
__device__ bool fused_route(const ExpertArgs& a, const Layout& L, char* smem, int* misc, int cs, int rank,
                            int cid, cg::cluster_group& cluster) {
  const int B = a.B, E = a.E, top = a.top_e;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e0 = L.ex0[rank], ne = L.ex0[rank + 1] - e0;
  uint4* xs = reinterpret_cast<uint4*>(smem + L.x);
  uint4 w[8];
  double bias_w = 0.0;
  if (warp < ne) {
    load_row8(reinterpret_cast<const uint4*>(a.w_router + (size_t)(e0 + warp) * a.d), 0, L.d8, lane, w);
    if (a.bias) bias_w = (double)__ldg(a.bias + e0 + warp);
  }
  for (int t = 0; t < B; t++)
    for (int j = threadIdx.x; j < L.d8; j += NTHR)
      xs[t * L.d8 + j] = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d) + j);
  if (threadIdx.x < B) misc[MI_TOK + threadIdx.x] = threadIdx.x;
  __syncthreads();
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
  stamp(a, cid, rank, 1);
  cluster.sync();
  stamp(a, cid, rank, 2);
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
__device__ void route_weights(const ExpertArgs& a, const Layout& L, char* smem, int* misc, int cid, int rank) {
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
      float v[16];
#pragma unroll
      for (int s = 0; s < 16; s++)
        v[s] = s < a.top_e ? __ldcg(&a.ws.ye[((size_t)tok * a.top_e + s) * a.d + j]) : 0.0f;
      float acc = 0.0f;
#pragma unroll
      for (int s = 0; s < 16; s++)
        if (s < a.top_e) acc = fmaf(wts[tok * a.top_e + s], v[s], acc);
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
          if (coef(m, i, is_w, co[u])) w[u] = __ldg(reinterpret_cast<const uint4*>(base + (size_t)i * stride));
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

// Bulk copies of sketch chunk ch (rows i0 + 16 ch .. of both matrices) into
// buffer slot `slot`, completing on bars[slot].
__device__ __forceinline__ void issue_sketch(const ExpertArgs& a, const Layout& L, char* buf, uint64_t* bars, int e,
                                             int i0, int i1, int ch, int slot) {
  const int c0 = i0 + 16 * ch, cnt = min(16, i1 - c0);
  const uint32_t bytes = cnt * (a.d / 4);
  char* dst = buf + (size_t)slot * 2 * L.skc;
  mbar_expect_tx(&bars[slot], 2 * bytes);
  bulk_g2s(dst, a.sk_gate + ((size_t)e * a.I + c0) * (a.d / 16), bytes, &bars[slot]);
  bulk_g2s(dst + L.skc, a.sk_up + ((size_t)e * a.I + c0) * (a.d / 16), bytes, &bars[slot]);
}

// ================================================================ sparse
template <int NT, bool FUSED, bool DBG>
__global__ void __launch_bounds__(NTHR, 1) reader_kernel(ExpertArgs a, Layout L) {
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
    if (!fused_route<NT>(a, L, smem, misc, cs, rank, cid, cluster)) return;  // uniform per cluster
  } else {
    if (!load_item_table(a, cid, misc, NT)) return;
  }
  if (DBG) stamp(a, cid, rank, 3);
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
    for (int ch = 0; ch < c1; ch++) issue_sketch(a, L, skbuf, skbars, e, i0, i1, ch, ch);
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
      rotate_quantize(a, L, smem, t, scratch, reinterpret_cast<float*>(misc + MI_CX) + t,
                      reinterpret_cast<float*>(misc + MI_RED), sv_pre);
  } else {
    load_tokens(a, L, smem, misc, n, true);
    __syncthreads();
  }
#pragma unroll
  for (int t = 0; t < NT; t++) tix[t] = misc[MI_TIX + (t < n ? t : 0)];
  if (DBG) stamp(a, cid, rank, 4);

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
          for (int ch = j; ch < c1; ch++) issue_sketch(a, L, skbuf, skbars, e, i0, i1, ch, ch - j);
        }
      }
      int G[NT], U[NT];
#pragma unroll
      for (int t = 0; t < NT; t++) G[t] = U[t] = 0;
      if (li < nown) {
        const int slot = j - rb;
        if (!mbar_wait_bounded(&skbars[slot], par, err)) misc[MI_DONE] = 1;
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
            if (!mbar_wait_bounded(uvbar, 0, err)) misc[MI_DONE] = 1;
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
        });
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
    if (!mbar_wait_bounded(uvbar, 0, err)) misc[MI_DONE] = 1;
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
    stamp(a, cid, rank, 13);
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
    if (!fused_route<NT>(a, L, smem, misc, cs, rank, cid, cluster)) return;
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
struct LaunchPlan {
  int dev, dense, NT, fused, B, E, I, d, r, items, forced;
  int cs, ring_rows, smem, max_clusters;
  Layout L;
};

int g_forced_cs = 0;  // 0: automatic

template <int NT, bool FUSED>
const void* kernel_ptr(bool dense, bool dbg) {
  if (dense) return reinterpret_cast<const void*>(&dense_kernel<NT, FUSED>);
  return dbg ? reinterpret_cast<const void*>(&reader_kernel<NT, FUSED, true>)
             : reinterpret_cast<const void*>(&reader_kernel<NT, FUSED, false>);
}
static_assert(kMaxGroup == 2, "kernels are instantiated for 1 and 2 tokens per item");
const void* pick_kernel(bool dense, int NT, bool fused, bool dbg) {
  if (NT == 1) return fused ? kernel_ptr<1, true>(dense, dbg) : kernel_ptr<1, false>(dense, dbg);
  return fused ? kernel_ptr<2, true>(dense, dbg) : kernel_ptr<2, false>(dense, dbg);
}

// Cluster size: among 8..16 (those that fit this shape), the one with the
// least estimated time, waves * (1 + 8 / cs) with waves = ceil(items /
// co-resident clusters): a wave costs a fixed latency plus work that shrinks
// with the cluster's width.  Ring: the deepest that fits, with room for the
// down stage's partial sums (NT x 16 KB), the rotation scratch and at least
// one sketch chunk.
cudaError_t plan_launch(const ExpertArgs& a, bool dense, LaunchPlan* out) {
  thread_local LaunchPlan cache[16];
  thread_local int ncache = 0, next = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int NT = a.nmax <= 1 ? 1 : 2;
  const bool fused = fused_routing(a.B);
  const int items = fused ? (a.B * a.top_e < a.E ? a.B * a.top_e : a.E) : a.ws.max_items;
  for (int i = 0; i < ncache; i++) {
    const LaunchPlan& c = cache[i];
    if (c.dev == dev && c.dense == (int)dense && c.NT == NT && c.fused == (int)fused && c.B == a.B && c.E == a.E &&
        c.I == a.I && c.d == a.d && c.r == a.r && c.items == items && c.forced == g_forced_cs) {
      *out = c;
      return cudaSuccess;
    }
  }
  int smem_max = 0;
  err = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (err != cudaSuccess) return err;
  const void* fns[2] = {pick_kernel(dense, NT, fused, false), pick_kernel(dense, NT, fused, true)};
  for (const void* f : fns) {
    err = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
  LaunchPlan p = {dev, (int)dense, NT, (int)fused, a.B, a.E, a.I, a.d, a.r, items, g_forced_cs, 0, 0, 0, 0, {}};
  double best = 1e30;
  const int ntok = fused ? a.B : NT;
  for (int cs = 16; cs >= 8; cs--) {
    if (g_forced_cs && cs != g_forced_cs) continue;
    const int cols_max = 8 * cdiv(a.d / 8, cs);
    if (cols_max > kMaxCols || a.I < cs || (fused && a.E < cs)) continue;
    const int red_need = NT * NTHR * 8 * 4;
    int rr = 0;
    for (int t = 2; t <= 64; t++) {
      const Layout L = make_layout(NT, ntok, fused, a.E, a.I, a.d, a.r, cs, t, dense);
      if (L.total > smem_max) break;
      const int region = NWARP * L.ring_bytes;
      if (L.c_slots >= 1 && region >= red_need && (dense || L.sk_round >= 1)) rr = t;
    }
    if (rr < 2) continue;
    const Layout L = make_layout(NT, ntok, fused, a.E, a.I, a.d, a.r, cs, rr, dense);
    int nclusters = 1 << 30;
    for (const void* f : fns) {
      err = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
      if (err != cudaSuccess) return err;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cs);
      cfg.blockDim = dim3(NTHR);
      cfg.dynamicSmemBytes = L.total;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int nc = 0;
      err = cudaOccupancyMaxActiveClusters(&nc, f, &cfg);
      if (err != cudaSuccess) {
        cudaGetLastError();
        nc = 0;
      }
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
  if (ncache < 16) cache[ncache++] = p;
  else cache[next++ % 16] = p;
  *out = p;
  return cudaSuccess;
}

cudaError_t launch_expert(const ExpertArgs& a0, cudaStream_t s, bool dense) {
  ExpertArgs a = a0;
  LaunchPlan plan;
  cudaError_t err = plan_launch(a, dense, &plan);
  if (err != cudaSuccess) return err;
  a.cs = plan.cs;
  a.ring_rows = plan.ring_rows;
  const bool dbg = a.dbg_ids || a.dbg_w || a.dbg_G || a.dbg_U || a.dbg_sigma || a.dbg_cand || a.dbg_kept ||
                   a.dbg_a_kept || a.dbg_y_expert || a.dbg_phase;
  const void* fn = pick_kernel(dense, plan.NT, plan.fused, dbg);
  err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, plan.smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.items * a.cs);
  cfg.blockDim = dim3(NTHR);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;  // programmatic dependent launch: overlaps this launch with the previous kernel's tail
  void* args[] = {&a, &plan.L};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace

bool fused_routing(int B) { return B <= kMaxGroup; }
cudaError_t launch_reader(const ExpertArgs& a, cudaStream_t s) { return launch_expert(a, s, false); }
cudaError_t launch_dense(const ExpertArgs& a, cudaStream_t s) { return launch_expert(a, s, true); }
void set_forced_cluster_size(int cs) { g_forced_cs = cs; }
cudaError_t query_plan(const ExpertArgs& a, bool dense, int out[4]) {
  LaunchPlan p;
  cudaError_t e = plan_launch(a, dense, &p);
  if (e != cudaSuccess) return e;
  out[0] = p.cs;
  out[1] = p.ring_rows;
  out[2] = p.smem;
  out[3] = p.max_clusters;
  return cudaSuccess;
}

}  // namespace moe
