// reader.cu -- the sparse routed-expert reader and the dense baseline block.
//
// One thread-block cluster (cs CTAs, cs = 16 or 8) runs one work item: an
// expert e and the (up to kMaxGroup) tokens routed to it, so tokens that share
// an expert share its reads.  The steps ("Channel Selection for
// Mixture-of-Experts Decoding Needs No Calibration Data", abstract; "KAIST:
// MoE Decoding Needs No Calibration Data", section "A reader that needs no
// data at all"):
//   S  screen: every CTA reads the ternary sketch rows of its slice of the I
//      channels, computes exact integer dots with the int8 rotated token and
//      the screening score sigma = |silu(ghat) uhat|;          cluster barrier
//   c  every CTA gathers all sigma over distributed shared memory and selects
//      the same top-c candidates per token (ties: lower channel);
//   C  exact: the CTAs split the union of the candidates, read the BF16 gate
//      and up rows and compute a = silu(g) u;                    cluster barrier
//   k  every CTA gathers a and selects the same top-k per token (the
//      top-k keep rule: no calibrated threshold);
//   D  down + recovery: every CTA reads its column slice of the kept down
//      rows (and the kept rows of the low-rank factor U_r S_r) and forms
//      y_e = sum_K a_i W_down[i,:] + V z, z = sum_{i not in K} ahat_i Ubar_i;
//   combine: the last of a token's top_e experts to finish a column slice
//      sums w_s y_e,s in slot order and writes bf16 y.
// All rows move with 1-D bulk copies (cp.async.bulk) into per-warp rings in
// the CTA's own shared memory; every wait on them is bounded.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

__host__ __device__ inline int rup(int x, int a) { return (x + a - 1) / a * a; }
__host__ __device__ inline int cdiv(int x, int a) { return (x + a - 1) / a; }

// Shared-memory carve-up, identical on host and device.
struct Layout {
  int mbar, misc, hist, x, q, sig_own, ahat_own, zpart, ubar, vown, sig_all, ahat_all, z_all, candm,
      keptm, ulist, upos, dlist, keys, kidx, a_own, ring, total;
  int own, cols, words, ring_bytes;  // per CTA: channels, output columns; mask words; ring bytes per warp
};

__host__ __device__ inline Layout make_layout(int nmax, int I, int d, int r, int cs, int ring_rows,
                                              bool dense) {
  Layout L;
  L.own = cdiv(I, cs);
  L.cols = d / cs;
  L.words = cdiv(I, 32);
  L.ring_bytes = ring_rows * d * 2;
  int o = 0;
  auto take = [&](int bytes) {
    int at = o;
    o = rup(o + bytes, 128);
    return at;
  };
  L.mbar = take((kWarps * kMaxSlots + 2) * 8);
  L.misc = take(1024);
  L.hist = take(260 * 4);
  L.x = take(nmax * d * 2);
  L.q = dense ? 0 : take(nmax * d);
  L.sig_own = take(nmax * L.own * 4);  // dense: h of the own channels
  L.ahat_own = dense ? 0 : take(nmax * L.own * 4);
  L.zpart = dense ? 0 : take(nmax * (r > 0 ? r : 1) * 4);
  L.ubar = dense ? 0 : take(L.own * (r > 0 ? r : 1) * 2);
  L.vown = dense ? 0 : take(L.cols * (r > 0 ? r : 1) * 2);
  L.sig_all = take(nmax * I * 4);  // sparse: sigma then a (by U position); dense: h of all channels
  L.ahat_all = dense ? 0 : take(nmax * I * 4);
  L.z_all = dense ? 0 : take(nmax * (r > 0 ? r : 1) * 4);
  L.candm = dense ? 0 : take(nmax * L.words * 4);
  L.keptm = dense ? 0 : take(nmax * L.words * 4);
  L.ulist = dense ? 0 : take(I * 4);
  L.upos = dense ? 0 : take(I * 4);
  L.dlist = dense ? 0 : take(I * 4);
  L.keys = dense ? 0 : take(I * 4);
  L.kidx = dense ? 0 : take(I * 4);
  L.a_own = dense ? 0 : take(nmax * L.own * 4);
  L.ring = take(kWarps * L.ring_bytes);
  L.total = o;
  return L;
}

// misc ints
enum { MI_E = 0, MI_N, MI_NU, MI_ND, MI_ERR, MI_PREFIX, MI_REM, MI_TOK = 8, MI_SLOT = 16, MI_LAST = 24, MI_CX = 32,
       MI_SCAN = 48 };

// ----------------------------------------------------------- block helpers
// Exclusive scan of one int per thread over the CTA; returns the prefix and
// writes the total to *total (every thread).
__device__ int block_excl_scan(int v, int* scratch, int* total) {
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
  for (int w = 0; w < kWarps; w++) {
    if (w < warp) off += scratch[w];
    tot += scratch[w];
  }
  __syncthreads();
  *total = tot;
  return off + inc - v;
}

// Top-n of N keys (uint32, larger = better, ties to the lower position):
// radix select on 8-bit digits, then an ordered pass over the keys equal to
// the threshold.  Sets bit p of out_mask for each chosen position p.
__device__ void block_select_top(const uint32_t* keys, int N, int n_sel, int* hist, int* misc,
                                 uint32_t* out_mask) {
  const int tid = threadIdx.x;
  for (int w = tid; w < cdiv(N, 32); w += kThreads) out_mask[w] = 0u;
  if (n_sel >= N) {
    __syncthreads();
    for (int p = tid; p < N; p += kThreads) atomicOr(&out_mask[p >> 5], 1u << (p & 31));
    __syncthreads();
    return;
  }
  if (tid == 0) {
    misc[MI_PREFIX] = 0;
    misc[MI_REM] = n_sel;
  }
  uint32_t mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += kThreads) hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = (uint32_t)misc[MI_PREFIX];
    for (int p = tid; p < N; p += kThreads) {
      const uint32_t k = keys[p];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // suffix sums over digits 255..0, 8 digits per lane (lane 0 = top digits)
      int loc[8], s = 0;
#pragma unroll
      for (int t = 0; t < 8; t++) {
        loc[t] = hist[255 - (tid * 8 + t)];
        s += loc[t];
      }
      int inc = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (tid >= o) inc += n;
      }
      const int rem = misc[MI_REM];
      int before = inc - s;  // keys with a larger digit than this lane's first
      int found = -1, take_before = 0;
#pragma unroll
      for (int t = 0; t < 8; t++) {
        if (found < 0 && before < rem && before + loc[t] >= rem) {
          found = 255 - (tid * 8 + t);
          take_before = before;
        }
        before += loc[t];
      }
      const unsigned bal = __ballot_sync(0xffffffffu, found >= 0);
      const int src = __ffs(bal) - 1;
      const int dig = __shfl_sync(0xffffffffu, found, src);
      const int tb = __shfl_sync(0xffffffffu, take_before, src);
      if (tid == 0) {
        misc[MI_PREFIX] = (int)(prefix | ((uint32_t)dig << shift));
        misc[MI_REM] = rem - tb;
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = (uint32_t)misc[MI_PREFIX];
  const int rem = misc[MI_REM];  // keys equal to T to take, lowest positions first
  // contiguous chunk per thread for the ordered equal-key pass
  const int chunk = cdiv(N, kThreads);
  const int p0 = min(N, tid * chunk), p1 = min(N, p0 + chunk);
  int eq = 0;
  for (int p = p0; p < p1; p++) eq += keys[p] == T;
  int tot;
  int before = block_excl_scan(eq, misc + MI_SCAN, &tot);
  for (int p = p0; p < p1; p++) {
    const uint32_t k = keys[p];
    bool take = k > T;
    if (k == T) {
      take = before < rem;
      before++;
    }
    if (take) atomicOr(&out_mask[p >> 5], 1u << (p & 31));
  }
  __syncthreads();
}

// Warp 0: ascending list of the set bits of mask over [0, N); returns count
// through misc[slot_idx] (after a __syncthreads by the caller).
__device__ void warp_mask_to_list(const uint32_t* mask, int N, int* list, int* pos_of, int* count_out) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  for (int w0 = 0; w0 < N; w0 += 32) {
    const int p = w0 + lane;
    const bool on = p < N && ((mask[w0 >> 5] >> lane) & 1u);
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    const int at = base + __popc(bal & ((1u << lane) - 1u));
    if (on) list[at] = p;
    if (pos_of && p < N) pos_of[p] = on ? at : -1;
    base += __popc(bal);
  }
  if (lane == 0) *count_out = base;
}

// --------------------------------------------------------- per-warp rings
// A warp streams `cnt` elements through P slots of its ring.  Lane 0 issues
// element j into slot j % P (issue(j, slot, bar)); all lanes consume it after
// a bounded wait.  `par` holds the parity bit of each slot barrier and
// persists across pipelines.  Returns false if a wait ran out (the warp then
// stops issuing and drains what is in flight).
template <class Issue, class Consume>
__device__ bool warp_stream(int cnt, int P, uint64_t* bars, uint32_t& par, uint32_t* err, Issue issue,
                            Consume consume) {
  const int lane = threadIdx.x & 31;
  if (cnt <= 0) return true;
  P = min(P, cnt);
  uint32_t pend = 0;
  // the ring may have been read by generic loads in an earlier stage
  if (lane == 0) fence_proxy_async();
  for (int j = 0; j < P; j++) {
    if (lane == 0) issue(j, j, &bars[j]);
    pend |= 1u << j;
  }
  __syncwarp();
  bool ok = true;
  for (int j = 0; j < cnt && ok; j++) {
    const int s = j % P;
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
  }
  if (!ok) {
    for (int s = 0; s < P; s++)
      if ((pend >> s) & 1u) {
        if (mbar_wait_bounded(&bars[s], (par >> s) & 1u, err)) par ^= 1u << s;
      }
  }
  return ok;
}

// Loads the work item of this cluster; returns false if the cluster is idle.
__device__ bool load_item(const ExpertArgs& a, int cid, int* misc) {
  if (threadIdx.x == 0) {
    const int n_items = *a.ws.n_items;
    int e = -1, n = 0;
    if (cid < n_items && cid < a.ws.max_items) {
      e = a.ws.item_e[cid];
      n = a.ws.item_n[cid];
      if (e < 0 || e >= a.E || n < 1 || n > kMaxGroup || n > a.nmax) {
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
      reinterpret_cast<float*>(misc)[MI_CX + t] = a.ws.cx ? a.ws.cx[tok] : 0.0f;
    }
  }
  __syncthreads();
  return misc[MI_E] >= 0;
}

// Epilogue shared by both kernels: write y_e for this CTA's columns, then the
// last expert of each token to finish this column slice combines.
__device__ void write_and_combine(const ExpertArgs& a, const Layout& L, int rank, const float* yfin,
                                  int* misc) {
  const int n = misc[MI_N];
  const int j0 = rank * L.cols;
  for (int idx = threadIdx.x; idx < n * L.cols; idx += kThreads) {
    const int t = idx / L.cols, col = idx % L.cols;
    const int tok = misc[MI_TOK + t], sl = misc[MI_SLOT + t];
    const size_t off = ((size_t)tok * a.top_e + sl) * a.d + j0 + col;
    a.ws.ye[off] = yfin[idx];
    if (a.dbg_y_expert) a.dbg_y_expert[off] = yfin[idx];
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int t = 0; t < n; t++) {
      const unsigned old = atomicAdd(&a.ws.counters[misc[MI_TOK + t] * kMaxCluster + rank], 1u);
      misc[MI_LAST + t] = old == (unsigned)(a.top_e - 1);
    }
  }
  __syncthreads();
  for (int t = 0; t < n; t++) {
    if (!misc[MI_LAST + t]) continue;
    __threadfence();
    const int tok = misc[MI_TOK + t];
    for (int col = threadIdx.x; col < L.cols; col += kThreads) {
      const int j = j0 + col;
      float acc = 0.0f;
      for (int s = 0; s < a.top_e; s++)
        acc = fmaf(__ldcg(&a.ws.wts[tok * a.top_e + s]), __ldcg(&a.ws.ye[((size_t)tok * a.top_e + s) * a.d + j]),
                   acc);
      if (a.residual) acc += bf16f(a.residual[(size_t)tok * a.d + j]);
      a.y[(size_t)tok * a.d + j] = f2bf16(acc);
    }
  }
}

// Loads x (and q) of the item's tokens into shared memory.
__device__ void load_tokens(const ExpertArgs& a, const Layout& L, char* smem, const int* misc, bool with_q) {
  const int n = misc[MI_N];
  const int vx = a.d / 8, vq = a.d / 16;
  uint4* xs = reinterpret_cast<uint4*>(smem + L.x);
  for (int idx = threadIdx.x; idx < n * vx; idx += kThreads) {
    const int t = idx / vx, j = idx % vx;
    xs[idx] = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)misc[MI_TOK + t] * a.d) + j);
  }
  if (with_q) {
    uint4* qs = reinterpret_cast<uint4*>(smem + L.q);
    for (int idx = threadIdx.x; idx < n * vq; idx += kThreads) {
      const int t = idx / vq, j = idx % vq;
      qs[idx] = __ldcg(reinterpret_cast<const uint4*>(a.ws.q + (size_t)misc[MI_TOK + t] * a.d) + j);
    }
  }
}

// ================================================================ sparse
__global__ void __launch_bounds__(kThreads, 1) reader_kernel(ExpertArgs a) {
  extern __shared__ __align__(128) char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = a.cs;
  const int rank = (int)cluster.block_rank();
  const int cid = blockIdx.x / cs;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Layout L = make_layout(a.nmax, a.I, a.d, a.r, cs, a.ring_rows, false);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.mbar);
  uint64_t* wbars = bars + warp * kMaxSlots;
  uint64_t* uvbar = bars + kWarps * kMaxSlots;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  int* hist = reinterpret_cast<int*>(smem + L.hist);
  if (tid < kWarps * kMaxSlots + 1) mbar_init(&bars[tid], 1);
  fence_mbar_init();
  __syncthreads();

  pdl_wait();
  if (!load_item(a, cid, misc)) return;  // uniform across the cluster
  const int e = misc[MI_E], n = misc[MI_N];
  const int I = a.I, d = a.d, r = a.r;
  const int i0 = cdiv(rank * I, cs), i1 = cdiv((rank + 1) * I, cs), nown = i1 - i0;
  const int j0 = rank * L.cols;
  uint32_t* err = a.ws.err;
  uint32_t par = 0;
  char* ring = smem + L.ring + warp * L.ring_bytes;

  // low-rank factor rows of the own channels and V rows of the own columns
  if (tid == 0 && r > 0) {
    const uint32_t bu = nown * r * 2, bv = L.cols * r * 2;
    mbar_expect_tx(uvbar, bu + bv);
    bulk_g2s(smem + L.ubar, a.u_sigma + ((size_t)e * I + i0) * r, bu, uvbar);
    bulk_g2s(smem + L.vown, a.v + ((size_t)e * d + j0) * r, bv, uvbar);
  }
  load_tokens(a, L, smem, misc, true);
  __syncthreads();

  // ---------------------------------------------------------- S: screen
  {
    float* sig_own = reinterpret_cast<float*>(smem + L.sig_own);
    float* ahat_own = reinterpret_cast<float*>(smem + L.ahat_own);
    const float* cxs = reinterpret_cast<const float*>(misc) + MI_CX;
    const int c0 = i0 + (warp * nown) / kWarps, c1 = i0 + ((warp + 1) * nown) / kWarps;
    const int skrow = d / 4;                           // bytes per sketch row
    const int per = max(1, (L.ring_bytes / 2) / (2 * skrow));  // channels per slot
    const int nch = cdiv(c1 - c0, per);
    const int words = d / 16;
    const uint4* qs = reinterpret_cast<const uint4*>(smem + L.q);
    warp_stream(
        nch, 2, wbars, par, err,
        [&](int j, int s, uint64_t* bar) {
          const int a0 = c0 + j * per, cnt = min(per, c1 - a0);
          char* dst = ring + s * (L.ring_bytes / 2);
          mbar_expect_tx(bar, 2 * cnt * skrow);
          bulk_g2s(dst, a.sk_gate + ((size_t)e * I + a0) * words, cnt * skrow, bar);
          bulk_g2s(dst + cnt * skrow, a.sk_up + ((size_t)e * I + a0) * words, cnt * skrow, bar);
        },
        [&](int j, int s) {
          const int a0 = c0 + j * per, cnt = min(per, c1 - a0);
          const uint32_t* gw = reinterpret_cast<const uint32_t*>(ring + s * (L.ring_bytes / 2));
          const uint32_t* uw = gw + cnt * words;
          for (int ci = 0; ci < cnt; ci++) {
            const int i = a0 + ci;
            int G[kMaxGroup], U[kMaxGroup];
#pragma unroll
            for (int t = 0; t < kMaxGroup; t++) G[t] = U[t] = 0;
            for (int w = lane; w < words; w += 32) {
              const uint32_t g = gw[ci * words + w], u = uw[ci * words + w];
#pragma unroll
              for (int t = 0; t < kMaxGroup; t++) {
                if (t < n) {
                  const uint4 qv = qs[t * words + w];
                  G[t] = trit_dot16(g, qv, G[t]);
                  U[t] = trit_dot16(u, qv, U[t]);
                }
              }
            }
            const float ag = __ldg(&a.alpha_gate[(size_t)e * I + i]);
            const float au = __ldg(&a.alpha_up[(size_t)e * I + i]);
#pragma unroll
            for (int t = 0; t < kMaxGroup; t++) {
              if (t < n) {
                const int gs = warp_sum(G[t]), us = warp_sum(U[t]);
                if (lane == t) {
                  const float gh = __fmul_rn(__fmul_rn((float)gs, ag), cxs[t]);
                  const float uh = __fmul_rn(__fmul_rn((float)us, au), cxs[t]);
                  const float ah = __fmul_rn(silu_r(gh), uh);
                  sig_own[t * L.own + (i - i0)] = fabsf(ah);
                  ahat_own[t * L.own + (i - i0)] = ah;
                  const size_t off = ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * I + i;
                  if (a.dbg_G) a.dbg_G[off] = gs;
                  if (a.dbg_U) a.dbg_U[off] = us;
                  if (a.dbg_sigma) a.dbg_sigma[off] = fabsf(ah);
                }
              }
            }
          }
        });
    __syncthreads();
    // partial recovery input over the own channels: zpart[t] = sum ahat_i Ubar_i
    if (r > 0) {
      if (!mbar_wait_bounded(uvbar, 0, err)) misc[MI_ERR] = 1;
      const uint16_t* ub = reinterpret_cast<const uint16_t*>(smem + L.ubar);
      float* zpart = reinterpret_cast<float*>(smem + L.zpart);
      for (int idx = tid; idx < n * r; idx += kThreads) {
        const int t = idx / r, p = idx % r;
        float z = 0.0f;
        for (int li = 0; li < nown; li++) z = fmaf(ahat_own[t * L.own + li], bf16f(ub[li * r + p]), z);
        zpart[idx] = z;
      }
    }
  }
  cluster.sync();

  // ---------------------------------------------- c: gather sigma, top-c
  float* sig_all = reinterpret_cast<float*>(smem + L.sig_all);  // later: a by U position
  float* ahat_all = reinterpret_cast<float*>(smem + L.ahat_all);
  float* z_all = reinterpret_cast<float*>(smem + L.z_all);
  uint32_t* candm = reinterpret_cast<uint32_t*>(smem + L.candm);
  uint32_t* keptm = reinterpret_cast<uint32_t*>(smem + L.keptm);
  int* ulist = reinterpret_cast<int*>(smem + L.ulist);
  int* upos = reinterpret_cast<int*>(smem + L.upos);
  int* dlist = reinterpret_cast<int*>(smem + L.dlist);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.keys);
  int* kidx = reinterpret_cast<int*>(smem + L.kidx);
  float* a_own = reinterpret_cast<float*>(smem + L.a_own);
  {
    const float* so = reinterpret_cast<const float*>(smem + L.sig_own);
    const float* ao = reinterpret_cast<const float*>(smem + L.ahat_own);
    for (int idx = tid; idx < n * I; idx += kThreads) {
      const int t = idx / I, i = idx % I;
      const int o = (i * cs) / I, li = i - cdiv(o * I, cs);
      sig_all[idx] = cluster.map_shared_rank(so, o)[t * L.own + li];
      ahat_all[idx] = cluster.map_shared_rank(ao, o)[t * L.own + li];
    }
    if (r > 0) {
      const float* zp = reinterpret_cast<const float*>(smem + L.zpart);
      for (int idx = tid; idx < n * r; idx += kThreads) {
        float z = 0.0f;
        for (int o = 0; o < cs; o++) z += cluster.map_shared_rank(zp, o)[idx];
        z_all[idx] = z;
      }
    }
  }
  __syncthreads();
  for (int t = 0; t < n; t++)
    block_select_top(reinterpret_cast<const uint32_t*>(sig_all + t * I), I, a.c, hist, misc,
                     candm + t * L.words);
  // union of the candidates, ascending
  if (warp == 0) {
    uint32_t* um = keys;  // scratch mask
    for (int w = lane; w < L.words; w += 32) {
      uint32_t m = 0;
      for (int t = 0; t < n; t++) m |= candm[t * L.words + w];
      um[w] = m;
    }
    __syncwarp();
    warp_mask_to_list(um, I, ulist, upos, &misc[MI_NU]);
    if (a.dbg_cand && rank == 0) {
      for (int t = 0; t < n; t++) {
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
    }
  }
  __syncthreads();
  const int nU = misc[MI_NU];

  // -------------------------------------------- C: exact candidate stage
  {
    const int u0 = cdiv(rank * nU, cs), u1 = cdiv((rank + 1) * nU, cs), nsl = u1 - u0;
    const int m0 = (warp * nsl) / kWarps, m1 = ((warp + 1) * nsl) / kWarps;
    const int rowb = d * 2;
    const int P = max(1, min(kMaxSlots, L.ring_bytes / (2 * rowb)));
    const uint4* xs = reinterpret_cast<const uint4*>(smem + L.x);
    const int vx = d / 8;
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
          const int m = m0 + j, i = ulist[u0 + m];
          const uint4* gr = reinterpret_cast<const uint4*>(ring + s * 2 * rowb);
          const uint4* ur = gr + vx;
          float g[kMaxGroup], u[kMaxGroup];
#pragma unroll
          for (int t = 0; t < kMaxGroup; t++) g[t] = u[t] = 0.0f;
          for (int v = lane; v < vx; v += 32) {
            const uint4 gv = gr[v], uv = ur[v];
#pragma unroll
            for (int t = 0; t < kMaxGroup; t++)
              if (t < n) {
                const uint4 xv = xs[t * vx + v];
                g[t] = dot8_bf16(gv, xv, g[t]);
                u[t] = dot8_bf16(uv, xv, u[t]);
              }
          }
#pragma unroll
          for (int t = 0; t < kMaxGroup; t++)
            if (t < n) {
              const float gs = warp_sum(g[t]), us = warp_sum(u[t]);
              if (lane == t) {
                const bool is_c = (candm[t * L.words + (i >> 5)] >> (i & 31)) & 1u;
                a_own[t * L.own + m] = is_c ? __fmul_rn(silu_r(gs), us) : 0.0f;
              }
            }
        });
  }
  cluster.sync();

  // ------------------------------------------------ k: gather a, top-k
  float* a_all = sig_all;  // [n, nU] by U position
  for (int idx = tid; idx < n * nU; idx += kThreads) {
    const int t = idx / nU, u = idx % nU;
    const int o = (u * cs) / nU, lu = u - cdiv(o * nU, cs);
    a_all[t * nU + u] = cluster.map_shared_rank(a_own, o)[t * L.own + lu];
  }
  cluster_arrive();  // no remote reads past this point
  __syncthreads();
  for (int t = 0; t < n; t++) {
    // the token's candidates in ascending channel order, key |a|
    if (warp == 0) {
      int base = 0;
      for (int u0 = 0; u0 < nU; u0 += 32) {
        const int u = u0 + lane;
        bool on = false;
        int i = 0;
        if (u < nU) {
          i = ulist[u];
          on = (candm[t * L.words + (i >> 5)] >> (i & 31)) & 1u;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, on);
        if (on) {
          const int at = base + __popc(bal & ((1u << lane) - 1u));
          keys[at] = __float_as_uint(fabsf(a_all[t * nU + u]));
          kidx[at] = i;
        }
        base += __popc(bal);
      }
      if (lane == 0) misc[MI_ND] = base;  // = c
    }
    __syncthreads();
    // select k of the c candidates: a mask over the compact positions,
    // remapped to channel bits below
    block_select_top(keys, misc[MI_ND], a.k, hist, misc, keptm + t * L.words);
    // remap compact positions -> channel bits (in place through a scratch pass)
    if (warp == 0) {
      const int c = misc[MI_ND];
      int* tmp = dlist;  // scratch list of kept channels
      int base = 0;
      for (int p0 = 0; p0 < c; p0 += 32) {
        const int p = p0 + lane;
        const bool on = p < c && ((keptm[t * L.words + (p0 >> 5)] >> lane) & 1u);
        const unsigned bal = __ballot_sync(0xffffffffu, on);
        if (on) tmp[base + __popc(bal & ((1u << lane) - 1u))] = kidx[p];
        base += __popc(bal);
      }
      __syncwarp();
      for (int w = lane; w < L.words; w += 32) keptm[t * L.words + w] = 0u;
      __syncwarp();
      for (int q = lane; q < base; q += 32) atomicOr(&keptm[t * L.words + (tmp[q] >> 5)], 1u << (tmp[q] & 31));
      __syncwarp();
      if (a.dbg_kept && rank == 0) {
        const size_t off = ((size_t)misc[MI_TOK + t] * a.top_e + misc[MI_SLOT + t]) * a.k;
        for (int q = lane; q < base && q < a.k; q += 32) {
          a.dbg_kept[off + q] = tmp[q];
          if (a.dbg_a_kept) a.dbg_a_kept[off + q] = a_all[t * nU + upos[tmp[q]]];
        }
      }
    }
    __syncthreads();
  }
  // union of the kept channels
  if (warp == 0) {
    uint32_t* um = keys;
    for (int w = lane; w < L.words; w += 32) {
      uint32_t m = 0;
      for (int t = 0; t < n; t++) m |= keptm[t * L.words + w];
      um[w] = m;
    }
    __syncwarp();
    warp_mask_to_list(um, I, dlist, nullptr, &misc[MI_ND]);
  }
  __syncthreads();
  const int nD = misc[MI_ND];

  // ---------------------------------------------- D: down rows + recovery
  {
    const int colb = L.cols * 2, ub = r * 2;
    const int eb = rup(colb + ub, 16);
    const int m0 = (warp * nD) / kWarps, m1 = ((warp + 1) * nD) / kWarps, cnt = m1 - m0;
    const int cap = max(1, L.ring_bytes / eb);  // elements resident per warp
    int P = min(kMaxSlots, max(1, cnt));
    int per = max(1, min(cdiv(cnt, P), cap / P));
    if (per * P > cap) P = max(1, cap / per);
    const int ngroups = cdiv(cnt, per);
    const int ncl = cdiv(L.cols, 128);  // column groups of 4 per lane
    float acc[kMaxGroup][8];
    float cor[kMaxGroup][4];
#pragma unroll
    for (int t = 0; t < kMaxGroup; t++) {
#pragma unroll
      for (int q = 0; q < 8; q++) acc[t][q] = 0.0f;
#pragma unroll
      for (int q = 0; q < 4; q++) cor[t][q] = 0.0f;
    }
    warp_stream(
        ngroups, P, wbars, par, err,
        [&](int j, int s, uint64_t* bar) {
          const int g0 = m0 + j * per, gc = min(per, m1 - g0);
          char* dst = ring + s * per * eb;
          mbar_expect_tx(bar, gc * (colb + ub));
          for (int q = 0; q < gc; q++) {
            const int i = dlist[g0 + q];
            bulk_g2s(dst + q * eb, a.w_down + ((size_t)e * I + i) * d + j0, colb, bar);
            if (r > 0) bulk_g2s(dst + q * eb + colb, a.u_sigma + ((size_t)e * I + i) * r, ub, bar);
          }
        },
        [&](int j, int s) {
          const int g0 = m0 + j * per, gc = min(per, m1 - g0);
          const char* src = ring + s * per * eb;
          for (int q = 0; q < gc; q++) {
            const int i = dlist[g0 + q];
            float co[kMaxGroup], ch[kMaxGroup];
#pragma unroll
            for (int t = 0; t < kMaxGroup; t++) {
              co[t] = ch[t] = 0.0f;
              if (t < n && ((keptm[t * L.words + (i >> 5)] >> (i & 31)) & 1u)) {
                co[t] = a_all[t * nU + upos[i]];
                ch[t] = ahat_all[t * I + i];
              }
            }
            const uint16_t* wd = reinterpret_cast<const uint16_t*>(src + q * eb);
#pragma unroll
            for (int cg4 = 0; cg4 < 2; cg4++) {
              const int c4 = 4 * lane + 128 * cg4;
              if (cg4 < ncl && c4 < L.cols) {
                const uint2 wv = *reinterpret_cast<const uint2*>(wd + c4);
                const float w0 = bf16lo(wv.x), w1 = bf16hi(wv.x), w2 = bf16lo(wv.y), w3 = bf16hi(wv.y);
#pragma unroll
                for (int t = 0; t < kMaxGroup; t++)
                  if (t < n) {
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
                  for (int t = 0; t < kMaxGroup; t++)
                    if (t < n) cor[t][kk] = fmaf(ch[t], uv, cor[t][kk]);
                }
              }
            }
          }
        });
    // per-warp partials into the warp's own ring area (its copies are done)
    __syncwarp();
    float* part = reinterpret_cast<float*>(ring);            // [n, cols]
    float* cpart = part + n * L.cols;                        // [n, r]
#pragma unroll
    for (int t = 0; t < kMaxGroup; t++)
      if (t < n) {
#pragma unroll
        for (int cg4 = 0; cg4 < 2; cg4++) {
          const int c4 = 4 * lane + 128 * cg4;
          if (cg4 < ncl && c4 < L.cols) {
#pragma unroll
            for (int q = 0; q < 4; q++) part[t * L.cols + c4 + q] = acc[t][4 * cg4 + q];
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
  float* yfin = reinterpret_cast<float*>(smem + L.x);  // [n, cols]; x is no longer needed
  {
    for (int idx = tid; idx < n * r; idx += kThreads) {
      const int t = idx / r, p = idx % r;
      float c = 0.0f;
      for (int w = 0; w < kWarps; w++) {
        const float* part = reinterpret_cast<const float*>(smem + L.ring + w * L.ring_bytes);
        c += part[n * L.cols + t * r + p];
      }
      z_all[idx] -= c;
    }
    __syncthreads();
    const uint16_t* vo = reinterpret_cast<const uint16_t*>(smem + L.vown);
    for (int idx = tid; idx < n * L.cols; idx += kThreads) {
      const int t = idx / L.cols, col = idx % L.cols;
      float y = 0.0f;
      for (int w = 0; w < kWarps; w++) y += reinterpret_cast<const float*>(smem + L.ring + w * L.ring_bytes)[idx];
      float rec = 0.0f;
      for (int p = 0; p < r; p++) rec = fmaf(bf16f(vo[col * r + p]), z_all[t * r + p], rec);
      yfin[idx] = y + rec;
    }
  }
  __syncthreads();
  write_and_combine(a, L, rank, yfin, misc);
  cluster_wait();
}

// ================================================================= dense
__global__ void __launch_bounds__(kThreads, 1) dense_kernel(ExpertArgs a) {
  extern __shared__ __align__(128) char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = a.cs;
  const int rank = (int)cluster.block_rank();
  const int cid = blockIdx.x / cs;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Layout L = make_layout(a.nmax, a.I, a.d, a.r, cs, a.ring_rows, true);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.mbar);
  uint64_t* wbars = bars + warp * kMaxSlots;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  if (tid < kWarps * kMaxSlots) mbar_init(&bars[tid], 1);
  fence_mbar_init();
  __syncthreads();
  pdl_wait();
  if (!load_item(a, cid, misc)) return;
  const int e = misc[MI_E], n = misc[MI_N];
  const int I = a.I, d = a.d;
  const int i0 = cdiv(rank * I, cs), i1 = cdiv((rank + 1) * I, cs), nown = i1 - i0;
  const int j0 = rank * L.cols;
  uint32_t* err = a.ws.err;
  uint32_t par = 0;
  char* ring = smem + L.ring + warp * L.ring_bytes;
  load_tokens(a, L, smem, misc, false);
  __syncthreads();
  float* h_own = reinterpret_cast<float*>(smem + L.sig_own);
  {
    const int m0 = (warp * nown) / kWarps, m1 = ((warp + 1) * nown) / kWarps;
    const int rowb = d * 2, vx = d / 8;
    const int P = max(1, min(kMaxSlots, L.ring_bytes / (2 * rowb)));
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
          const int m = m0 + j;
          const uint4* gr = reinterpret_cast<const uint4*>(ring + s * 2 * rowb);
          const uint4* ur = gr + vx;
          float g[kMaxGroup], u[kMaxGroup];
#pragma unroll
          for (int t = 0; t < kMaxGroup; t++) g[t] = u[t] = 0.0f;
          for (int v = lane; v < vx; v += 32) {
            const uint4 gv = gr[v], uv = ur[v];
#pragma unroll
            for (int t = 0; t < kMaxGroup; t++)
              if (t < n) {
                const uint4 xv = xs[t * vx + v];
                g[t] = dot8_bf16(gv, xv, g[t]);
                u[t] = dot8_bf16(uv, xv, u[t]);
              }
          }
#pragma unroll
          for (int t = 0; t < kMaxGroup; t++)
            if (t < n) {
              const float gs = warp_sum(g[t]), us = warp_sum(u[t]);
              if (lane == t) h_own[t * L.own + m] = __fmul_rn(silu_r(gs), us);
            }
        });
  }
  cluster.sync();
  float* h_all = reinterpret_cast<float*>(smem + L.sig_all);
  for (int idx = tid; idx < n * I; idx += kThreads) {
    const int t = idx / I, i = idx % I;
    const int o = (i * cs) / I, li = i - cdiv(o * I, cs);
    h_all[idx] = cluster.map_shared_rank(h_own, o)[t * L.own + li];
  }
  cluster_arrive();
  __syncthreads();
  {
    const int colb = L.cols * 2;
    const int eb = rup(colb, 16);
    const int m0 = (warp * I) / kWarps, m1 = ((warp + 1) * I) / kWarps, cnt = m1 - m0;
    const int cap = max(1, L.ring_bytes / eb);
    int P = min(kMaxSlots, max(1, cnt));
    int per = max(1, min(cdiv(cnt, P), cap / P));
    if (per * P > cap) P = max(1, cap / per);
    const int ngroups = cdiv(cnt, per);
    const int ncl = cdiv(L.cols, 128);
    float acc[kMaxGroup][8];
#pragma unroll
    for (int t = 0; t < kMaxGroup; t++)
#pragma unroll
      for (int q = 0; q < 8; q++) acc[t][q] = 0.0f;
    warp_stream(
        ngroups, P, wbars, par, err,
        [&](int j, int s, uint64_t* bar) {
          const int g0 = m0 + j * per, gc = min(per, m1 - g0);
          char* dst = ring + s * per * eb;
          mbar_expect_tx(bar, gc * colb);
          for (int q = 0; q < gc; q++)
            bulk_g2s(dst + q * eb, a.w_down + ((size_t)e * I + g0 + q) * d + j0, colb, bar);
        },
        [&](int j, int s) {
          const int g0 = m0 + j * per, gc = min(per, m1 - g0);
          const char* src = ring + s * per * eb;
          for (int q = 0; q < gc; q++) {
            const int i = g0 + q;
            float co[kMaxGroup];
#pragma unroll
            for (int t = 0; t < kMaxGroup; t++) co[t] = t < n ? h_all[t * I + i] : 0.0f;
            const uint16_t* wd = reinterpret_cast<const uint16_t*>(src + q * eb);
#pragma unroll
            for (int cg4 = 0; cg4 < 2; cg4++) {
              const int c4 = 4 * lane + 128 * cg4;
              if (cg4 < ncl && c4 < L.cols) {
                const uint2 wv = *reinterpret_cast<const uint2*>(wd + c4);
                const float w0 = bf16lo(wv.x), w1 = bf16hi(wv.x), w2 = bf16lo(wv.y), w3 = bf16hi(wv.y);
#pragma unroll
                for (int t = 0; t < kMaxGroup; t++)
                  if (t < n) {
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
    for (int t = 0; t < kMaxGroup; t++)
      if (t < n) {
#pragma unroll
        for (int cg4 = 0; cg4 < 2; cg4++) {
          const int c4 = 4 * lane + 128 * cg4;
          if (cg4 < ncl && c4 < L.cols) {
#pragma unroll
            for (int q = 0; q < 4; q++) part[t * L.cols + c4 + q] = acc[t][4 * cg4 + q];
          }
        }
      }
  }
  __syncthreads();
  float* out = reinterpret_cast<float*>(smem + L.x);  // [n, cols]; x is no longer needed
  for (int idx = tid; idx < n * L.cols; idx += kThreads) {
    float y = 0.0f;
    for (int w = 0; w < kWarps; w++) y += reinterpret_cast<const float*>(smem + L.ring + w * L.ring_bytes)[idx];
    out[idx] = y;
  }
  __syncthreads();
  write_and_combine(a, L, rank, out, misc);
  cluster_wait();
}

// Largest ring that fits; at least two rows per warp, and room for the
// per-warp partial sums [n, cols + r] fp32 that the down stage leaves there.
int pick_ring_rows(const ExpertArgs& a, bool dense, int smem_max) {
  const int need = a.nmax * (a.d / a.cs + a.r) * 4;
  const int min_rows = max(2, cdiv(need, 2 * a.d));
  int best = 0;
  for (int rr = min_rows; rr <= 64; rr++) {
    const Layout L = make_layout(a.nmax, a.I, a.d, a.r, a.cs, rr, dense);
    if (L.total <= smem_max) best = rr;
    else break;
  }
  return best;
}

struct LaunchPlan {
  int dev, dense, nmax, I, d, r, items, forced;
  int cs, ring_rows, smem, max_clusters;
};

int g_forced_cs = 0;  // 0: automatic

// Cluster size: among 16, 8, 4 (those that fit this shape), the one that
// keeps the most SMs busy on this launch, min(items, co-resident clusters)
// * cs, ties to the larger cluster.  Ring depth: the deepest that fits.
// Cached per shape and device.
cudaError_t plan_launch(const ExpertArgs& a, bool dense, LaunchPlan* out) {
  thread_local LaunchPlan cache[16];
  thread_local int ncache = 0, next = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int items = a.ws.max_items;
  for (int i = 0; i < ncache; i++) {
    const LaunchPlan& c = cache[i];
    if (c.dev == dev && c.dense == (int)dense && c.nmax == a.nmax && c.I == a.I && c.d == a.d && c.r == a.r &&
        c.items == items && c.forced == g_forced_cs) {
      *out = c;
      return cudaSuccess;
    }
  }
  int smem_max = 0;
  err = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (err != cudaSuccess) return err;
  auto fn = dense ? dense_kernel : reader_kernel;
  err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (err != cudaSuccess) return err;
  LaunchPlan p = {dev, (int)dense, a.nmax, a.I, a.d, a.r, items, g_forced_cs, 0, 0, 0, 0};
  long best_busy = -1;
  for (int cs = 16; cs >= 4; cs /= 2) {
    if (g_forced_cs && cs != g_forced_cs) continue;
    if (a.d / cs > 256 || a.d / cs < 8 || a.I < cs) continue;
    ExpertArgs t = a;
    t.cs = cs;
    const int rr = pick_ring_rows(t, dense, smem_max);
    if (rr < 2) continue;
    const int smem = make_layout(a.nmax, a.I, a.d, a.r, cs, rr, dense).total;
    err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    err = cudaOccupancyMaxActiveClusters(&nclusters, fn, &cfg);
    if (err != cudaSuccess) {
      cudaGetLastError();
      continue;
    }
    if (nclusters < 1) continue;
    const long busy = (long)(items < nclusters ? items : nclusters) * cs;
    if (busy > best_busy) {
      best_busy = busy;
      p.cs = cs;
      p.ring_rows = rr;
      p.smem = smem;
      p.max_clusters = nclusters;
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
  const Layout L = make_layout(a.nmax, a.I, a.d, a.r, a.cs, a.ring_rows, dense);
  auto fn = dense ? dense_kernel : reader_kernel;
  err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (err != cudaSuccess) return err;
  const int items = a.ws.max_items;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(items * a.cs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, fn, a);
}

}  // namespace

size_t reader_smem_bytes(const ExpertArgs& a, int ring_rows) {
  return make_layout(a.nmax, a.I, a.d, a.r, a.cs, ring_rows, false).total;
}
size_t dense_smem_bytes(const ExpertArgs& a, int ring_rows) {
  return make_layout(a.nmax, a.I, a.d, a.r, a.cs, ring_rows, true).total;
}
cudaError_t launch_reader(const ExpertArgs& a, cudaStream_t s) { return launch_expert(a, s, false); }
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
cudaError_t launch_dense(const ExpertArgs& a, cudaStream_t s) { return launch_expert(a, s, true); }

}  // namespace moe
