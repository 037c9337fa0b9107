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
// Rows move with 1-D bulk copies (cp.async.bulk) into per-warp rings in the
// CTA's own shared memory; every wait on them is bounded.  Every exchange
// between the CTAs of a cluster is a store into the receivers' shared memory
// followed by a cluster barrier: no CTA reads another CTA's shared memory.
//
// At batch 1 the step is a chain of short dependent stages whose code runs
// once per launch, so instruction fetch is a first-order cost: the kernels
// keep their static code small (host-computed geometry instead of runtime
// divisions, short loops kept rolled, one shared copy of the selection).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int NTHR = 512;
constexpr int NWARP = NTHR / 32;
constexpr int kMaxCols = 256;  // output columns per CTA (8 per lane)

__host__ __device__ inline int rup(int x, int a) { return (x + a - 1) / a * a; }
__host__ __device__ inline int cdiv(int x, int a) { return (x + a - 1) / a; }

// One shared copy of a runtime integer division (kernel code stays small).
__device__ __noinline__ int idiv(int a, int b) { return a / b; }

// ------------------------------------------------------- launch geometry
// Shared-memory offsets and the partitions of a launch, computed on the host.
struct Layout {
  int mbar, misc, hist, wtot, pmask, x, q, logit, sig, ahat, zparts, z, apos, candm, keptm, ulist, upos, dlist,
      keys, kidx, ubar, vown, ring, total;
  int ntok;        // tokens held in smem (fused routing: B; otherwise NT)
  int own_max;     // max channels per CTA
  int cols_max;    // max output columns per CTA
  int words;       // mask words over I
  int ring_bytes;  // per warp
  int d8, d16;     // d / 8, d / 16
  int s_per;       // channels per screen slot (half a ring)
  int c_slots;     // candidate-pair slots per warp
  int ch0[17];     // channel partition over the CTAs of a cluster
  int col0[17];    // output-column partition (multiples of 8)
  int ex0[17];     // expert partition (in-kernel routing)
};

__host__ inline Layout make_layout(int NT, int ntok, bool fused, int E, int I, int d, int r, int cs,
                                   int ring_rows, bool dense) {
  Layout L = {};
  L.ntok = ntok;
  L.own_max = cdiv(I, cs);
  L.cols_max = 8 * cdiv(d / 8, cs);
  L.words = cdiv(I, 32);
  L.ring_bytes = ring_rows * d * 2;
  L.d8 = d / 8;
  L.d16 = d / 16;
  L.s_per = (L.ring_bytes / 2) / (2 * (d / 4));
  if (L.s_per > 32) L.s_per = 32;  // one alpha per lane
  L.c_slots = L.ring_bytes / (4 * d);
  for (int o = 0; o <= cs && o < 17; o++) {
    L.ch0[o] = cdiv(o * I, cs);
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
  L.mbar = take((NWARP * kMaxSlots + 4) * 8);
  L.misc = take(256 * 4);
  L.hist = take(2 * 2048 * 4);
  L.wtot = take(64 * 4);
  L.pmask = take(L.words * 4);
  L.x = take(ntok * d * 2);
  L.q = take(ntok * d);
  L.logit = fused ? take(ntok * E * 8) : 0;
  L.sig = take(NT * I * 4);  // sparse: sigma by channel; dense: h by channel
  L.ahat = dense ? 0 : take(NT * I * 4);
  L.zparts = dense ? 0 : take(cs * NT * rr * 4);
  L.z = dense ? 0 : take(NT * rr * 4);
  L.apos = dense ? 0 : take(NT * I * 4);  // a by union position
  L.candm = dense ? 0 : take(NT * L.words * 4);
  L.keptm = dense ? 0 : take(NT * L.words * 4);
  L.ulist = dense ? 0 : take(I * 4);
  L.upos = dense ? 0 : take(I * 4);
  L.dlist = dense ? 0 : take(I * 4);
  L.keys = dense ? 0 : take(I * 4);
  L.kidx = dense ? 0 : take(I * 4);
  L.ubar = dense ? 0 : take(L.own_max * rr * 2);
  L.vown = dense ? 0 : take(L.cols_max * rr * 2);
  L.ring = take(NWARP * L.ring_bytes);
  L.total = o;
  return L;
}

// misc ints
enum {
  MI_E = 0, MI_N, MI_NU, MI_ND, MI_NC, MI_DIG, MI_REM, MI_CNT, MI_DONE,
  MI_TOK = 16, MI_SLOT = 32, MI_LAST = 48, MI_TIX = 64, MI_CX = 80, MI_SCAN = 96,
  MI_RIDS = 128,  // in-kernel routing: ids [B <= 2][top_e <= 16]
  MI_RW = 192     // in-kernel routing: weights
};

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

// Trits of one packed sketch word as four words of signed bytes.  Layout:
// position n (< 8) at bits [4n, 4n+1], position 8+n at bits [4n+2, 4n+3];
// codes 00 = 0, 01 = +1, 11 = -1.  A nibble's code selects a byte of
// kTritLut = {0x00, 0x01, 0x00, 0xff} through byte_perm.
__device__ __forceinline__ uint4 decode_trits(uint32_t w) {
  const uint32_t kTritLut = 0xff000100u;
  const uint32_t lo = w & 0x33333333u;
  const uint32_t hi = (w >> 2) & 0x33333333u;
  return make_uint4(__byte_perm(kTritLut, 0, lo), __byte_perm(kTritLut, 0, lo >> 16),
                    __byte_perm(kTritLut, 0, hi), __byte_perm(kTritLut, 0, hi >> 16));
}
__device__ __forceinline__ int dot16_i8(uint4 t, uint4 q, int acc) {
  acc = __dp4a((int)t.x, (int)q.x, acc);
  acc = __dp4a((int)t.y, (int)q.y, acc);
  acc = __dp4a((int)t.z, (int)q.z, acc);
  acc = __dp4a((int)t.w, (int)q.w, acc);
  return acc;
}

// ----------------------------------------------------------- block helpers
__device__ __noinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  int off = 0, tot = 0;
#pragma unroll 1
  for (int w = 0; w < NWARP; w++) {
    const int s = scratch[w];
    off += w < warp ? s : 0;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return off + inc - v;
}

// Top-n_sel of N keys (uint32, larger first, ties to the lower position):
// radix select with digits of 11, 11 and 10 bits from the top, stopping as
// soon as the boundary bin is taken whole; keys equal to a fully resolved
// threshold are taken in position order.  Sets bit p of out_mask for each
// chosen position p.  hist holds 2 x 2048 ints, wtot 16 ints.
__device__ __noinline__ void block_select_top(const uint32_t* keys, int N, int n_sel, int* hist, int* wtot,
                                              int* misc, uint32_t* out_mask) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (N + 31) >> 5;
  for (int w = tid; w < nw; w += NTHR) out_mask[w] = 0u;
  if (n_sel >= N) {
    __syncthreads();
    for (int p = tid; p < N; p += NTHR) atomicOr(&out_mask[p >> 5], 1u << (p & 31));
    __syncthreads();
    return;
  }
  for (int b = tid; b < 2048; b += NTHR) hist[b] = 0;
  uint32_t prefix = 0u, mask = 0u;
  int rem = n_sel;
  bool done = false;
#pragma unroll 1
  for (int pass = 0; pass < 3 && !done; pass++) {
    const int shift = pass == 0 ? 21 : pass == 1 ? 10 : 0;
    const int lnb = pass == 2 ? 10 : 11;
    const int nb = 1 << lnb;
    int* h = hist + (pass & 1) * 2048;
    int* hn = hist + ((pass + 1) & 1) * 2048;
    __syncthreads();  // h is zero and the previous pass is done with hn
    for (int p = tid; p < N; p += NTHR) {
      const uint32_t k = keys[p];
      if ((k & mask) == prefix) atomicAdd(&h[(k >> shift) & (nb - 1)], 1);
    }
    for (int b = tid; b < 2048; b += NTHR) hn[b] = 0;
    __syncthreads();
    // warp w covers bins [nb - (w+1) bpw, nb - w bpw), top-down; lane l a run
    const int bpl = nb >> 9;                            // bins per lane (4 or 2)
    const int top = nb - (warp * 32 + lane) * bpl;      // bins top-1 .. top-bpl
    int s = 0;
#pragma unroll 1
    for (int j = 1; j <= bpl; j++) s += h[top - j];
    int inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += n;
    }
    if (lane == 31) wtot[warp] = inc;
    __syncthreads();
    int before = inc - s;  // keys in bins above this lane's run
#pragma unroll 1
    for (int w = 0; w < warp; w++) before += wtot[w];
    if (before < rem && before + s >= rem) {
#pragma unroll 1
      for (int j = 1; j <= bpl; j++) {
        const int c = h[top - j];
        if (before + c >= rem) {
          misc[MI_DIG] = top - j;
          misc[MI_REM] = rem - before;
          misc[MI_CNT] = c;
          break;
        }
        before += c;
      }
    }
    __syncthreads();
    prefix |= (uint32_t)misc[MI_DIG] << shift;
    mask |= (uint32_t)(nb - 1) << shift;
    rem = misc[MI_REM];
    done = rem == misc[MI_CNT];
  }
  if (done) {
    // the boundary bin is taken whole: keep every key whose decided bits are
    // at least the boundary prefix
    for (int p = tid; p < N; p += NTHR)
      if ((keys[p] & mask) >= prefix) atomicOr(&out_mask[p >> 5], 1u << (p & 31));
    __syncthreads();
    return;
  }
  // fully resolved threshold T = prefix with more equal keys than needed:
  // keys > T, and the first `rem` keys == T by position
  const int chunk = (N + NTHR - 1) / NTHR;
  const int p0 = min(N, tid * chunk), p1 = min(N, p0 + chunk);
  int eq = 0;
  for (int p = p0; p < p1; p++) eq += keys[p] == prefix;
  int tot;
  int before = block_excl_scan(eq, misc + MI_SCAN, &tot);
  for (int p = p0; p < p1; p++) {
    const uint32_t k = keys[p];
    bool take = k > prefix;
    if (k == prefix) take = before++ < rem;
    if (take) atomicOr(&out_mask[p >> 5], 1u << (p & 31));
  }
  __syncthreads();
}

// Ascending list of the set bits of mask over [0, N), all warps; the count
// lands in *count_out; pos_of (if given) gets each bit's list position or -1.
__device__ __noinline__ void block_mask_to_list(const uint32_t* mask, int N, int* list, int* pos_of,
                                                int* count_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (N + 31) >> 5;
  for (int w = warp; w < nw; w += NWARP) {
    int off = 0;
    for (int v = lane; v < w; v += 32) off += __popc(mask[v]);
    off = warp_sum(off);
    const int p = w * 32 + lane;
    const bool on = p < N && ((mask[w] >> lane) & 1u);
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    const int at = off + __popc(bal & ((1u << lane) - 1u));
    if (on) list[at] = p;
    if (pos_of && p < N) pos_of[p] = on ? at : -1;
    if (w == nw - 1 && lane == 0) *count_out = off + __popc(bal);
  }
  __syncthreads();
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
// The item comes from the work table the select kernel wrote.
__device__ bool load_item_table(const ExpertArgs& a, int cid, int* misc, int NT) {
  if (threadIdx.x == 0) {
    const int n_items = *a.ws.n_items;
    int e = -1, n = 0;
    if (cid < n_items && cid < a.ws.max_items) {
      e = a.ws.item_e[cid];
      n = a.ws.item_n[cid];
      if (e < 0 || e >= a.E || n < 1 || n > NT) {
        atomicOr(a.ws.err, kErrBadWorkItem);
        e = -1;
      }
    }
    misc[MI_E] = e;
    misc[MI_N] = n;
    for (int t = 0; t < n; t++) {
      int tok = a.ws.item_tok[cid * kMaxGroup + t], sl = a.ws.item_slot[cid * kMaxGroup + t];
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
      for (int j = threadIdx.x; j < L.d16; j += NTHR)
        qs[t * L.d16 + j] = __ldcg(reinterpret_cast<const uint4*>(a.ws.q + (size_t)tok * a.d) + j);
  }
}

// Rotation + int8 quantisation of smem token t: v = FWHT(s . x) in the fp32
// scratch (d floats), q = rint(127 v / amax), c_x = amax / (127 d).  Thread T
// (< d/4) holds elements 4T..4T+3: stages h = 1, 2 run in registers, h = 4..64
// across the lanes of a warp (a warp holds 128 consecutive elements), h >= 128
// in shared memory.  Every stage applies the reference butterflies
// (a + b, a - b), lower index first, in the reference stage order, so the
// bits equal the reference transform's.
__device__ void rotate_quantize_smem(const ExpertArgs& a, const Layout& L, char* smem, int t, float* v,
                                     float* cx_out, float* red) {
  const int d = a.d;
  const int T = threadIdx.x, lane = T & 31;
  if (T < 2 * L.d8) {
    const uint2 xv = reinterpret_cast<const uint2*>(smem + L.x + (size_t)t * d * 2)[T];
    const char4 sv = reinterpret_cast<const char4*>(a.rot_sign)[T];
    float r0 = (float)sv.x * bf16lo(xv.x), r1 = (float)sv.y * bf16hi(xv.x);
    float r2 = (float)sv.z * bf16lo(xv.y), r3 = (float)sv.w * bf16hi(xv.y);
    float b0 = __fadd_rn(r0, r1), b1 = __fsub_rn(r0, r1), b2 = __fadd_rn(r2, r3), b3 = __fsub_rn(r2, r3);  // h = 1
    r0 = __fadd_rn(b0, b2);  // h = 2
    r2 = __fsub_rn(b0, b2);
    r1 = __fadd_rn(b1, b3);
    r3 = __fsub_rn(b1, b3);
#pragma unroll 1
    for (int m = 1; m < 32 && 4 * m < d; m <<= 1) {  // h = 4m: partner lane ^ m
      const bool up = lane & m;
      const float p0 = __shfl_xor_sync(0xffffffffu, r0, m), p1 = __shfl_xor_sync(0xffffffffu, r1, m);
      const float p2 = __shfl_xor_sync(0xffffffffu, r2, m), p3 = __shfl_xor_sync(0xffffffffu, r3, m);
      r0 = up ? __fsub_rn(p0, r0) : __fadd_rn(r0, p0);
      r1 = up ? __fsub_rn(p1, r1) : __fadd_rn(r1, p1);
      r2 = up ? __fsub_rn(p2, r2) : __fadd_rn(r2, p2);
      r3 = up ? __fsub_rn(p3, r3) : __fadd_rn(r3, p3);
    }
    reinterpret_cast<float4*>(v)[T] = make_float4(r0, r1, r2, r3);
  }
  __syncthreads();
#pragma unroll 1
  for (int h = 128, lh = 7; h < d; h <<= 1, lh++) {
    for (int p = threadIdx.x; p < 4 * L.d8; p += NTHR) {
      const int j = ((p >> lh) << (lh + 1)) | (p & (h - 1));
      const float x0 = v[j], x1 = v[j + h];
      v[j] = __fadd_rn(x0, x1);
      v[j + h] = __fsub_rn(x0, x1);
    }
    __syncthreads();
  }
  float m = 0.0f;
  for (int j = threadIdx.x; j < d; j += NTHR) m = fmaxf(m, fabsf(v[j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float amax = 0.0f;
#pragma unroll 1
  for (int w = 0; w < NWARP; w++) amax = fmaxf(amax, red[w]);
  int8_t* q = reinterpret_cast<int8_t*>(smem + L.q) + (size_t)t * d;
  for (int j = threadIdx.x; j < d; j += NTHR) {
    int n = 0;
    if (amax > 0.0f) n = max(-127, min(127, __float2int_rn(__fdiv_rn(__fmul_rn(v[j], 127.0f), amax))));
    q[j] = (int8_t)n;
  }
  if (threadIdx.x == 0) *cx_out = amax > 0.0f ? __fdiv_rn(amax, __fmul_rn(127.0f, (float)d)) : 0.0f;
  __syncthreads();
}

// Stage time stamps (globaltimer, ns) of the first CTA of each cluster.
__device__ __forceinline__ void stamp(const ExpertArgs& a, int cid, int rank, int k) {
  if (a.dbg_phase && rank == 0 && threadIdx.x == 0) a.dbg_phase[cid * 16 + k] = global_ns();
}

// In-kernel routing (B <= NT <= 2): every CTA loads all tokens, rotates and
// quantises them, computes the logits of its slice of experts and pushes
// them to all CTAs; after the cluster barrier every CTA takes the same top-e
// and builds the same work table (one item per routed expert, experts
// ascending).  Returns false if this cluster has no item.
template <int NT>
__device__ bool fused_route(const ExpertArgs& a, const Layout& L, char* smem, int* misc, int cs, int rank,
                            int cid, uint64_t* wrbar, cg::cluster_group& cluster) {
  const int B = a.B, E = a.E, d = a.d, top = a.top_e;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e0 = L.ex0[rank], ne = L.ex0[rank + 1] - e0;
  char* wr = smem + L.ring;  // router rows of this CTA's experts
  if (threadIdx.x == 0 && ne > 0) {
    mbar_expect_tx(wrbar, ne * d * 2);
    bulk_g2s(wr, a.w_router + (size_t)e0 * d, ne * d * 2, wrbar);
  }
  if (threadIdx.x < B) {
    misc[MI_TOK + threadIdx.x] = threadIdx.x;
  }
  __syncthreads();
  load_tokens(a, L, smem, misc, B, false);
  __syncthreads();
  // rotate + quantise every token (the ring tail is the fp32 scratch)
  float* scratch = reinterpret_cast<float*>(smem + L.ring + NWARP * L.ring_bytes - d * 4);
  float* cxs = reinterpret_cast<float*>(misc + MI_CX);
#pragma unroll 1
  for (int t = 0; t < B; t++)
    rotate_quantize_smem(a, L, smem, t, scratch, &cxs[t], reinterpret_cast<float*>(misc + MI_SCAN));
  stamp(a, cid, rank, 1);
  // logits of the own experts, one warp per expert, pushed to every CTA
  if (ne > 0 && !mbar_wait_bounded(wrbar, 0, a.ws.err)) misc[MI_DONE] = 1;
  double* lg = reinterpret_cast<double*>(smem + L.logit);
  for (int el = warp; el < ne; el += NWARP) {
    const uint4* wrow = reinterpret_cast<const uint4*>(wr + (size_t)el * d * 2);
    double acc[NT];
#pragma unroll
    for (int t = 0; t < NT; t++) acc[t] = 0.0;
#pragma unroll 1
    for (int j = lane; j < L.d8; j += 32) {
      const uint4 w = wrow[j];
#pragma unroll
      for (int t = 0; t < NT; t++) {
        const uint4 x = reinterpret_cast<const uint4*>(smem + L.x)[(t < B ? t : 0) * L.d8 + j];
        acc[t] = fma((double)bf16lo(w.x), (double)bf16lo(x.x), acc[t]);
        acc[t] = fma((double)bf16hi(w.x), (double)bf16hi(x.x), acc[t]);
        acc[t] = fma((double)bf16lo(w.y), (double)bf16lo(x.y), acc[t]);
        acc[t] = fma((double)bf16hi(w.y), (double)bf16hi(x.y), acc[t]);
        acc[t] = fma((double)bf16lo(w.z), (double)bf16lo(x.z), acc[t]);
        acc[t] = fma((double)bf16hi(w.z), (double)bf16hi(x.z), acc[t]);
        acc[t] = fma((double)bf16lo(w.w), (double)bf16lo(x.w), acc[t]);
        acc[t] = fma((double)bf16hi(w.w), (double)bf16hi(x.w), acc[t]);
      }
    }
    const int e = e0 + el;
    const double bias = a.bias ? (double)a.bias[e] : 0.0;
#pragma unroll
    for (int t = 0; t < NT; t++) {
      const double s = warp_sum(acc[t]) + bias;
      if (t < B && lane < cs) st_cluster(&lg[t * E + e], lane, s);
    }
  }
  stamp(a, cid, rank, 2);
  cluster.sync();
  stamp(a, cid, rank, 3);
  // top-e per token by rank: 4 threads per expert count the logits that beat
  // it (larger, or equal with a lower id); rank < top_e is chosen
  int* rids = misc + MI_RIDS;
  float* rw = reinterpret_cast<float*>(misc + MI_RW);
  double* ex = reinterpret_cast<double*>(smem + L.hist);  // [B, top] scratch
  int* first = reinterpret_cast<int*>(ex + 64);
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
      cnt += __shfl_xor_sync(0xffffffffu, cnt, 1);
      cnt += __shfl_xor_sync(0xffffffffu, cnt, 2);
      if (e < E && qtr == 0 && cnt < top) rids[b * top + cnt] = e;
    }
  }
  __syncthreads();
  // softmax over the chosen logits, summed in slot order (fp32 exponentials
  // of the fp64 logit differences; the weights only scale outputs)
  const int nent = B * top;
  if (threadIdx.x < nent) {
    const int b = threadIdx.x >= top;  // B <= 2
    ex[threadIdx.x] = (double)__expf((float)(lg[b * E + rids[threadIdx.x]] - lg[b * E + rids[b * top]]));
    const int id = rids[threadIdx.x];
    int f = 1;
    for (int j = 0; j < threadIdx.x; j++) f &= rids[j] != id;
    first[threadIdx.x] = f;
  }
  if (threadIdx.x == 0) misc[MI_E] = -1;
  __syncthreads();
  if (threadIdx.x < nent) {
    const int b = threadIdx.x >= top;
    double den = 0.0;
    for (int s2 = 0; s2 < top; s2++) den += ex[b * top + s2];
    const float w = (float)(ex[threadIdx.x] / den);
    rw[threadIdx.x] = w;
    if (cid == 0 && rank == 0) {
      a.ws.ids[threadIdx.x] = rids[threadIdx.x];
      a.ws.wts[threadIdx.x] = w;
      if (a.dbg_ids) a.dbg_ids[threadIdx.x] = rids[threadIdx.x];
      if (a.dbg_w) a.dbg_w[threadIdx.x] = w;
    }
    // work table: distinct experts ascending; item cid = the cid-th of them
    if (first[threadIdx.x]) {
      const int id = rids[threadIdx.x];
      int rk = 0;
      for (int j = 0; j < nent; j++) rk += first[j] && rids[j] < id;
      if (rk == cid) misc[MI_E] = id;
    }
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int e = misc[MI_E];
    const bool on = e >= 0 && lane < nent && rids[lane] == e;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    if (on) {
      const int at = __popc(bal & ((1u << lane) - 1u));
      const int b = lane >= top;
      misc[MI_TOK + at] = b;
      misc[MI_SLOT + at] = lane - b * top;
      misc[MI_TIX + at] = b;
    }
    if (lane == 0) misc[MI_N] = __popc(bal);
  }
  __syncthreads();
  return misc[MI_E] >= 0;
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
  __threadfence();
  __syncthreads();
  if (threadIdx.x < n) {
    const int t = threadIdx.x;
    const unsigned old = atomicAdd(&a.ws.counters[misc[MI_TOK + t] * kMaxCluster + rank], 1u);
    misc[MI_LAST + t] = old == (unsigned)(a.top_e - 1);
  }
  __syncthreads();
#pragma unroll 1
  for (int t = 0; t < n; t++) {
    if (!misc[MI_LAST + t]) continue;
    __threadfence();
    const int tok = misc[MI_TOK + t];
    for (int col = threadIdx.x; col < ncols; col += NTHR) {
      const int j = j0 + col;
      float acc = 0.0f;
#pragma unroll 1
      for (int s = 0; s < a.top_e; s++)
        acc = fmaf(wts[tok * a.top_e + s], __ldcg(&a.ws.ye[((size_t)tok * a.top_e + s) * a.d + j]), acc);
      if (a.residual) acc += bf16f(a.residual[(size_t)tok * a.d + j]);
      a.y[(size_t)tok * a.d + j] = f2bf16(acc);
    }
    if (threadIdx.x == 0) a.ws.counters[tok * kMaxCluster + rank] = 0u;
  }
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
  uint64_t* uvbar = bars + NWARP * kMaxSlots;
  uint64_t* wrbar = uvbar + 1;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  int* hist = reinterpret_cast<int*>(smem + L.hist);
  int* wtot = reinterpret_cast<int*>(smem + L.wtot);
  if (tid < NWARP * kMaxSlots + 2) mbar_init(&bars[tid], 1);
  if (tid == 0) misc[MI_DONE] = 0;
  fence_mbar_init();
  __syncthreads();
  if (DBG) stamp(a, cid, rank, 0);

  if (FUSED) {
    if (!fused_route<NT>(a, L, smem, misc, cs, rank, cid, wrbar, cluster)) return;  // uniform per cluster
  } else {
    pdl_wait();
    if (!load_item_table(a, cid, misc, NT)) return;
  }
  if (DBG) stamp(a, cid, rank, 4);
  const int e = misc[MI_E], n = misc[MI_N];
  const int I = a.I, d = a.d, r = a.r;
  const int i0 = L.ch0[rank], nown = L.ch0[rank + 1] - i0;
  const int j0 = L.col0[rank], ncols = L.col0[rank + 1] - j0;
  uint32_t* err = a.ws.err;
  uint32_t par = 0;
  char* ring = smem + L.ring + warp * L.ring_bytes;
  int tix[NT];
#pragma unroll
  for (int t = 0; t < NT; t++) tix[t] = misc[MI_TIX + (t < n ? t : 0)];

  // factor rows of the own channels and V rows of the own columns
  if (tid == 0 && r > 0) {
    const uint32_t bu = nown * r * 2, bv = ncols * r * 2;
    mbar_expect_tx(uvbar, bu + bv);
    bulk_g2s(smem + L.ubar, a.u_sigma + ((size_t)e * I + i0) * r, bu, uvbar);
    bulk_g2s(smem + L.vown, a.v + ((size_t)e * d + j0) * r, bv, uvbar);
  }
  if (!FUSED) {
    load_tokens(a, L, smem, misc, n, true);
    __syncthreads();
  }

  float* sig = reinterpret_cast<float*>(smem + L.sig);        // [NT, I] pushed by the owners
  float* ahat = reinterpret_cast<float*>(smem + L.ahat);      // [NT, I]
  float* zparts = reinterpret_cast<float*>(smem + L.zparts);  // [cs, NT, r]
  float* z = reinterpret_cast<float*>(smem + L.z);            // [NT, r]
  float* apos = reinterpret_cast<float*>(smem + L.apos);      // [NT, I] by union position
  uint32_t* candm = reinterpret_cast<uint32_t*>(smem + L.candm);
  uint32_t* keptm = reinterpret_cast<uint32_t*>(smem + L.keptm);
  uint32_t* pmask = reinterpret_cast<uint32_t*>(smem + L.pmask);
  int* ulist = reinterpret_cast<int*>(smem + L.ulist);
  int* upos = reinterpret_cast<int*>(smem + L.upos);
  int* dlist = reinterpret_cast<int*>(smem + L.dlist);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.keys);
  int* kidx = reinterpret_cast<int*>(smem + L.kidx);
  const float* cxs = reinterpret_cast<const float*>(misc + MI_CX);

  // ---------------------------------------------------------- S: screen
  {
    const int c0 = i0 + (warp * nown) / NWARP, c1 = i0 + ((warp + 1) * nown) / NWARP;
    const int skrow = 4 * L.d16;  // bytes per sketch row
    const int half = L.ring_bytes / 2;
    const int per = L.s_per;
    const int words = L.d16;
    const uint4* qs = reinterpret_cast<const uint4*>(smem + L.q);
    const float* ag_row = a.alpha_gate + (size_t)e * I;
    const float* au_row = a.alpha_up + (size_t)e * I;
    const int nchunk = c1 > c0 ? idiv(c1 - c0 + per - 1, per) : 0;
    warp_stream(
        nchunk, 2, wbars, par, err,
        [&](int j, int s, uint64_t* bar) {
          const int a0 = c0 + j * per, cnt = min(per, c1 - a0);
          char* dst = ring + s * half;
          mbar_expect_tx(bar, 2 * cnt * skrow);
          bulk_g2s(dst, a.sk_gate + ((size_t)e * I + a0) * words, cnt * skrow, bar);
          bulk_g2s(dst + cnt * skrow, a.sk_up + ((size_t)e * I + a0) * words, cnt * skrow, bar);
        },
        [&](int j, int s) {
          const int a0 = c0 + j * per, cnt = min(per, c1 - a0);
          const uint32_t* gw = reinterpret_cast<const uint32_t*>(ring + s * half);
          const uint32_t* uw = gw + cnt * words;
          // the scales of this chunk, one per lane, loaded ahead of the dots
          const float agl = lane < cnt ? __ldg(ag_row + a0 + lane) : 0.0f;
          const float aul = lane < cnt ? __ldg(au_row + a0 + lane) : 0.0f;
#pragma unroll 1
          for (int ci = 0; ci < cnt; ci++) {
            const int i = a0 + ci;
            int G[NT], U[NT];
#pragma unroll
            for (int t = 0; t < NT; t++) G[t] = U[t] = 0;
#pragma unroll 1
            for (int w = lane; w < words; w += 32) {
              const uint4 tg = decode_trits(gw[ci * words + w]);
              const uint4 tu = decode_trits(uw[ci * words + w]);
#pragma unroll
              for (int t = 0; t < NT; t++) {
                const uint4 qv = qs[tix[t] * words + w];
                G[t] = dot16_i8(tg, qv, G[t]);
                U[t] = dot16_i8(tu, qv, U[t]);
              }
            }
            const float ag = __shfl_sync(0xffffffffu, agl, ci), au = __shfl_sync(0xffffffffu, aul, ci);
#pragma unroll
            for (int t = 0; t < NT; t++) {
              if (t < n) {
                const int gs = warp_sum(G[t]), us = warp_sum(U[t]);
                const float cx = cxs[tix[t]];
                const float gh = __fmul_rn(__fmul_rn((float)gs, ag), cx);
                const float uh = __fmul_rn(__fmul_rn((float)us, au), cx);
                const float ah = __fmul_rn(silu_r(gh), uh);
                if (lane < cs) {
                  st_cluster(&sig[t * I + i], lane, fabsf(ah));
                  st_cluster(&ahat[t * I + i], lane, ah);
                }
                if (DBG && lane == 31) {
                  const size_t off = ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * I + i;
                  if (a.dbg_G) a.dbg_G[off] = gs;
                  if (a.dbg_U) a.dbg_U[off] = us;
                  if (a.dbg_sigma) a.dbg_sigma[off] = fabsf(ah);
                }
              }
            }
          }
        });
    if (DBG) stamp(a, cid, rank, 5);
    // partial recovery input over the own channels, pushed to every CTA:
    // zparts[rank][t] = sum_{own i} ahat_i Ubar_i.  The local ahat of the own
    // channels was written by this CTA's own stores above.
    __syncthreads();
    if (r > 0) {
      if (!mbar_wait_bounded(uvbar, 0, err)) misc[MI_DONE] = 1;
      const uint16_t* ub = reinterpret_cast<const uint16_t*>(smem + L.ubar);
#pragma unroll 1
      for (int t = 0; t < n; t++)
        for (int p = tid; p < r; p += NTHR) {
          float zz = 0.0f;
#pragma unroll 4
          for (int li = 0; li < nown; li++) zz = fmaf(ahat[t * I + i0 + li], bf16f(ub[li * r + p]), zz);
#pragma unroll 1
          for (int o = 0; o < cs; o++) st_cluster(&zparts[(rank * NT + t) * r + p], o, zz);
        }
    }
  }
  if (DBG) stamp(a, cid, rank, 6);
  cluster.sync();
  if (DBG) stamp(a, cid, rank, 7);

  // ---------------------------------------------------------- c: top-c
#pragma unroll 1
  for (int t = 0; t < n; t++)
    block_select_top(reinterpret_cast<const uint32_t*>(sig + t * I), I, a.c, hist, wtot, misc,
                     candm + t * L.words);
  if (DBG) stamp(a, cid, rank, 8);
#pragma unroll 1
  for (int t = 0; t < n; t++)
    for (int p = tid; p < r; p += NTHR) {
      float zz = 0.0f;
#pragma unroll 1
      for (int o = 0; o < cs; o++) zz += zparts[(o * NT + t) * r + p];
      z[t * r + p] = zz;
    }
  // union of the candidates, ascending
  for (int w = tid; w < L.words; w += NTHR) {
    uint32_t m = 0;
#pragma unroll
    for (int t = 0; t < NT; t++) m |= t < n ? candm[t * L.words + w] : 0u;
    pmask[w] = m;
  }
  __syncthreads();
  block_mask_to_list(pmask, I, ulist, upos, &misc[MI_NU]);
  if (DBG && a.dbg_cand && rank == 0 && warp < n) {
    const int t = warp;
    int base = 0;
    int* out = a.dbg_cand + ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * a.c;
    for (int w0 = 0; w0 < I; w0 += 32) {
      const int p = w0 + lane;
      const bool on = p < I && ((candm[t * L.words + (w0 >> 5)] >> lane) & 1u);
      const unsigned bal = __ballot_sync(0xffffffffu, on);
      if (on) out[base + __popc(bal & ((1u << lane) - 1u))] = p;
      base += __popc(bal);
    }
  }
  const int nU = misc[MI_NU];
  if (DBG) stamp(a, cid, rank, 9);

  // -------------------------------------------- C: exact candidate stage
  {
    const int u0 = idiv(rank * nU + cs - 1, cs), u1 = idiv((rank + 1) * nU + cs - 1, cs), nsl = u1 - u0;
    const int m0 = (warp * nsl) / NWARP, m1 = ((warp + 1) * nsl) / NWARP;
    const int rowb = d * 2;
    const int P = max(1, min(kMaxSlots, L.c_slots));
    const uint4* xs = reinterpret_cast<const uint4*>(smem + L.x);
    const int vx = L.d8;
    warp_stream(
        m1 - m0, P, wbars, par, err,
        [&](int j, int s, uint64_t* bar) {
          const int i = ulist[u0 + m0 + j];
          char* dst = ring + s * 2 * rowb;
          mbar_expect_tx(bar, 2 * rowb);
          bulk_g2s(dst, a.w_gate + ((size_t)e * I + i) * d, rowb, bar);
          bulk_g2s(dst + rowb, a.w_up + ((size_t)e * I + i) * d, rowb, bar);
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
              if (lane < cs) st_cluster(&apos[t * I + u], lane, av);
            }
          }
        });
  }
  if (DBG) stamp(a, cid, rank, 10);
  cluster.sync();  // the last exchange: no CTA touches another's smem after this
  if (DBG) stamp(a, cid, rank, 11);

  // ------------------------------------------------------------ k: top-k
#pragma unroll 1
  for (int t = 0; t < n; t++) {
    // the token's candidates in ascending channel order, key |a|
    if (warp == 0) {
      int base = 0;
      for (int w0 = 0; w0 < nU; w0 += 32) {
        const int u = w0 + lane;
        bool on = false;
        int i = 0;
        if (u < nU) {
          i = ulist[u];
          on = (candm[t * L.words + (i >> 5)] >> (i & 31)) & 1u;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, on);
        if (on) {
          const int at = base + __popc(bal & ((1u << lane) - 1u));
          keys[at] = __float_as_uint(fabsf(apos[t * I + u]));
          kidx[at] = i;
        }
        base += __popc(bal);
      }
      if (lane == 0) misc[MI_NC] = base;  // = c
    }
    __syncthreads();
    const int c = misc[MI_NC];
    uint32_t* km = keptm + t * L.words;
    block_select_top(keys, c, a.k, hist, wtot, misc, pmask);  // over compact positions
    for (int w = tid; w < L.words; w += NTHR) km[w] = 0u;
    __syncthreads();
    for (int p = tid; p < c; p += NTHR)
      if ((pmask[p >> 5] >> (p & 31)) & 1u) atomicOr(&km[kidx[p] >> 5], 1u << (kidx[p] & 31));
    __syncthreads();
    if (DBG && a.dbg_kept && rank == 0 && warp == 0) {
      const size_t off = ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * a.k;
      int base = 0;
      for (int w0 = 0; w0 < I; w0 += 32) {
        const int i = w0 + lane;
        const bool on = i < I && ((km[w0 >> 5] >> lane) & 1u);
        const unsigned bal = __ballot_sync(0xffffffffu, on);
        const int at = base + __popc(bal & ((1u << lane) - 1u));
        if (on && at < a.k) {
          a.dbg_kept[off + at] = i;
          if (a.dbg_a_kept) a.dbg_a_kept[off + at] = apos[t * I + upos[i]];
        }
        base += __popc(bal);
      }
    }
  }
  if (DBG) stamp(a, cid, rank, 12);
  // union of the kept channels
  for (int w = tid; w < L.words; w += NTHR) {
    uint32_t m = 0;
#pragma unroll
    for (int t = 0; t < NT; t++) m |= t < n ? keptm[t * L.words + w] : 0u;
    pmask[w] = m;
  }
  __syncthreads();
  block_mask_to_list(pmask, I, dlist, nullptr, &misc[MI_ND]);
  const int nD = misc[MI_ND];
  if (DBG) stamp(a, cid, rank, 13);

  // ---------------------------------------------- D: down rows + recovery
  {
    const int colb = ncols * 2, ubb = r * 2;
    const int eb = rup(colb + ubb, 16);
    const int m0 = (warp * nD) / NWARP, m1 = ((warp + 1) * nD) / NWARP, cnt = m1 - m0;
    const int cap = max(1, idiv(L.ring_bytes, eb));
    int P = min(kMaxSlots, max(1, cnt));
    int per = max(1, min(idiv(cnt + P - 1, P), idiv(cap, P)));
    if (per * P > cap) P = max(1, idiv(cap, per));
    float acc[NT][8];
    float cor[NT][4];
#pragma unroll
    for (int t = 0; t < NT; t++) {
#pragma unroll
      for (int q = 0; q < 8; q++) acc[t][q] = 0.0f;
#pragma unroll
      for (int q = 0; q < 4; q++) cor[t][q] = 0.0f;
    }
    warp_stream(
        cnt > 0 ? idiv(cnt + per - 1, per) : 0, P, wbars, par, err,
        [&](int j, int s, uint64_t* bar) {
          const int g0 = m0 + j * per, gc = min(per, m1 - g0);
          char* dst = ring + s * per * eb;
          mbar_expect_tx(bar, gc * (colb + ubb));
#pragma unroll 1
          for (int q = 0; q < gc; q++) {
            const int i = dlist[g0 + q];
            bulk_g2s(dst + q * eb, a.w_down + ((size_t)e * I + i) * d + j0, colb, bar);
            if (r > 0) bulk_g2s(dst + q * eb + colb, a.u_sigma + ((size_t)e * I + i) * r, ubb, bar);
          }
        },
        [&](int j, int s) {
          const int g0 = m0 + j * per, gc = min(per, m1 - g0);
          const char* src = ring + s * per * eb;
#pragma unroll 1
          for (int q = 0; q < gc; q++) {
            const int i = dlist[g0 + q];
            float co[NT], ch[NT];
#pragma unroll
            for (int t = 0; t < NT; t++) {
              const bool kept = t < n && ((keptm[t * L.words + (i >> 5)] >> (i & 31)) & 1u);
              co[t] = kept ? apos[t * I + upos[i]] : 0.0f;
              ch[t] = kept ? ahat[t * I + i] : 0.0f;
            }
            const uint16_t* wd = reinterpret_cast<const uint16_t*>(src + q * eb);
#pragma unroll
            for (int cg4 = 0; cg4 < 2; cg4++) {
              const int c4 = 4 * lane + 128 * cg4;
              if (c4 < ncols) {
                const uint2 wv = *reinterpret_cast<const uint2*>(wd + c4);
                const float w0 = bf16lo(wv.x), w1 = bf16hi(wv.x), w2 = bf16lo(wv.y), w3 = bf16hi(wv.y);
#pragma unroll
                for (int t = 0; t < NT; t++) {
                  acc[t][4 * cg4 + 0] = fmaf(co[t], w0, acc[t][4 * cg4 + 0]);
                  acc[t][4 * cg4 + 1] = fmaf(co[t], w1, acc[t][4 * cg4 + 1]);
                  acc[t][4 * cg4 + 2] = fmaf(co[t], w2, acc[t][4 * cg4 + 2]);
                  acc[t][4 * cg4 + 3] = fmaf(co[t], w3, acc[t][4 * cg4 + 3]);
                }
              }
            }
            if (r > 0) {
              const uint16_t* ur = reinterpret_cast<const uint16_t*>(src + q * eb + colb);
#pragma unroll
              for (int kk = 0; kk < 4; kk++) {
                const int p = lane + 32 * kk;
                if (p < r) {
                  const float uv = bf16f(ur[p]);
#pragma unroll
                  for (int t = 0; t < NT; t++) cor[t][kk] = fmaf(ch[t], uv, cor[t][kk]);
                }
              }
            }
          }
        });
    __syncwarp();
    float* part = reinterpret_cast<float*>(ring);  // [NT, cols_max] then [NT, r]
    float* cpart = part + NT * L.cols_max;
#pragma unroll
    for (int t = 0; t < NT; t++) {
#pragma unroll
      for (int cg4 = 0; cg4 < 2; cg4++) {
        const int c4 = 4 * lane + 128 * cg4;
        if (c4 < ncols) {
#pragma unroll
          for (int q = 0; q < 4; q++) part[t * L.cols_max + c4 + q] = acc[t][4 * cg4 + q];
        }
      }
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {
        const int p = lane + 32 * kk;
        if (p < r) cpart[t * r + p] = cor[t][kk];
      }
    }
  }
  __syncthreads();
  float* yfin = reinterpret_cast<float*>(smem + L.x);  // [n, cols_max]; x is no longer needed
#pragma unroll 1
  for (int t = 0; t < n; t++)
    for (int p = tid; p < r; p += NTHR) {
      float cc = 0.0f;
#pragma unroll 1
      for (int w = 0; w < NWARP; w++)
        cc += reinterpret_cast<const float*>(smem + L.ring + w * L.ring_bytes)[NT * L.cols_max + t * r + p];
      z[t * r + p] -= cc;
    }
  __syncthreads();
  {
    const uint16_t* vo = reinterpret_cast<const uint16_t*>(smem + L.vown);
#pragma unroll 1
    for (int t = 0; t < n; t++)
      for (int col = tid; col < ncols; col += NTHR) {
        float y = 0.0f;
#pragma unroll 1
        for (int w = 0; w < NWARP; w++)
          y += reinterpret_cast<const float*>(smem + L.ring + w * L.ring_bytes)[t * L.cols_max + col];
        float rec = 0.0f;
#pragma unroll 4
        for (int p = 0; p < r; p++) rec = fmaf(bf16f(vo[col * r + p]), z[t * r + p], rec);
        yfin[t * L.cols_max + col] = y + rec;
      }
  }
  __syncthreads();
  if (DBG) stamp(a, cid, rank, 14);
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
  uint64_t* wrbar = bars + NWARP * kMaxSlots + 1;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  if (tid < NWARP * kMaxSlots + 2) mbar_init(&bars[tid], 1);
  if (tid == 0) misc[MI_DONE] = 0;
  fence_mbar_init();
  __syncthreads();
  if (FUSED) {
    if (!fused_route<NT>(a, L, smem, misc, cs, rank, cid, wrbar, cluster)) return;
  } else {
    pdl_wait();
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
  {
    const int colb = ncols * 2;
    const int eb = rup(colb, 16);
    const int m0 = (warp * I) / NWARP, m1 = ((warp + 1) * I) / NWARP, cnt = m1 - m0;
    const int cap = max(1, idiv(L.ring_bytes, eb));
    int P = min(kMaxSlots, max(1, cnt));
    int per = max(1, min(idiv(cnt + P - 1, P), idiv(cap, P)));
    if (per * P > cap) P = max(1, idiv(cap, per));
    float acc[NT][8];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
      for (int q = 0; q < 8; q++) acc[t][q] = 0.0f;
    warp_stream(
        cnt > 0 ? idiv(cnt + per - 1, per) : 0, P, wbars, par, err,
        [&](int j, int s, uint64_t* bar) {
          const int g0 = m0 + j * per, gc = min(per, m1 - g0);
          char* dst = ring + s * per * eb;
          mbar_expect_tx(bar, gc * colb);
#pragma unroll 1
          for (int q = 0; q < gc; q++)
            bulk_g2s(dst + q * eb, a.w_down + ((size_t)e * I + g0 + q) * d + j0, colb, bar);
        },
        [&](int j, int s) {
          const int g0 = m0 + j * per, gc = min(per, m1 - g0);
          const char* src = ring + s * per * eb;
#pragma unroll 1
          for (int q = 0; q < gc; q++) {
            const int i = g0 + q;
            float co[NT];
#pragma unroll
            for (int t = 0; t < NT; t++) co[t] = t < n ? h[t * I + i] : 0.0f;
            const uint16_t* wd = reinterpret_cast<const uint16_t*>(src + q * eb);
#pragma unroll
            for (int cg4 = 0; cg4 < 2; cg4++) {
              const int c4 = 4 * lane + 128 * cg4;
              if (c4 < ncols) {
                const uint2 wv = *reinterpret_cast<const uint2*>(wd + c4);
                const float w0 = bf16lo(wv.x), w1 = bf16hi(wv.x), w2 = bf16lo(wv.y), w3 = bf16hi(wv.y);
#pragma unroll
                for (int t = 0; t < NT; t++) {
                  acc[t][4 * cg4 + 0] = fmaf(co[t], w0, acc[t][4 * cg4 + 0]);
                  acc[t][4 * cg4 + 1] = fmaf(co[t], w1, acc[t][4 * cg4 + 1]);
                  acc[t][4 * cg4 + 2] = fmaf(co[t], w2, acc[t][4 * cg4 + 2]);
                  acc[t][4 * cg4 + 3] = fmaf(co[t], w3, acc[t][4 * cg4 + 3]);
                }
              }
            }
          }
        });
    __syncwarp();
    float* part = reinterpret_cast<float*>(ring);
#pragma unroll
    for (int t = 0; t < NT; t++) {
#pragma unroll
      for (int cg4 = 0; cg4 < 2; cg4++) {
        const int c4 = 4 * lane + 128 * cg4;
        if (c4 < ncols) {
#pragma unroll
          for (int q = 0; q < 4; q++) part[t * L.cols_max + c4 + q] = acc[t][4 * cg4 + q];
        }
      }
    }
  }
  __syncthreads();
  float* out = reinterpret_cast<float*>(smem + L.x);
#pragma unroll 1
  for (int t = 0; t < n; t++)
    for (int col = tid; col < ncols; col += NTHR) {
      float y = 0.0f;
#pragma unroll 1
      for (int w = 0; w < NWARP; w++)
        y += reinterpret_cast<const float*>(smem + L.ring + w * L.ring_bytes)[t * L.cols_max + col];
      out[t * L.cols_max + col] = y;
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
// per-warp partial sums [NT, cols + r] fp32 of the down stage (and, with the
// in-kernel router, for the CTA's router rows and an fp32 transform scratch).
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
    const int need = NT * (cols_max + a.r) * 4;
    const int wr_need = fused ? cdiv(a.E, cs) * a.d * 2 + a.d * 4 : 0;
    int rr = 0;
    for (int t = 2; t <= 64; t++) {
      const Layout L = make_layout(NT, ntok, fused, a.E, a.I, a.d, a.r, cs, t, dense);
      if (L.total > smem_max) break;
      if (L.ring_bytes >= need && NWARP * L.ring_bytes >= wr_need) rr = t;
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
  cfg.numAttrs = plan.fused ? 1 : 2;  // the in-kernel router makes it the step's first kernel
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
