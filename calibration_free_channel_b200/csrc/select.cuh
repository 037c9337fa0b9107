// select.cuh -- block-wide exact top-n selection over uint32 keys and the
// bit-mask -> ascending-list conversion, for CTAs of 512 threads.  Used for
// the candidate (top-c by screening score) and kept (top-k by |a|) sets of
// "KAIST: MoE Decoding Needs No Calibration Data", section "Swapping the
// threshold for top-k": a fixed number of channels per (token, expert), ties
// to the lower channel.
#pragma once
#include "common.cuh"

namespace moe {
namespace sel {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr unsigned kSelFull = 0xffffffffu;
// positions in the caller's `misc` ints
constexpr int kSelDig = 4, kSelRem = 5, kSelCnt = 6, kSelWt = 112;

// Top-n_sel of N <= 2048 keys (uint32, larger first, ties to the lower
// position): radix select with digits of 11, 11 and 10 bits from the top.
// A pass counts the keys that share the decided prefix into the bins of the
// next digit (shared-memory atomics), scans the bins from the top (each warp
// a run of bins, warp totals through shared memory) and finds the boundary
// digit.  The selection stops as soon as the boundary bin is taken whole;
// after the last digit the threshold T is fully resolved and the first keys
// equal to T by position fill the rest.  Bit p of out_mask (p < N, words
// [0, ceil(N / 32))) is set for each chosen position p.  Key p sits at
// keys[p * kstride].  hist holds 2 x 2048 ints; misc holds the pass state at
// [kSelDig, kSelCnt] and 16 warp totals from kSelWt.  Every thread of a
// 512-thread CTA calls it (it contains block barriers).
static __device__ __noinline__ void block_select_top(const uint32_t* keys, int kstride, int N, int n_sel,
                                                     int* hist, int* misc, uint32_t* out_mask) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (N + 31) >> 5;
  if (n_sel >= N || n_sel <= 0) {
    for (int w = tid; w < nw; w += kSelThreads) {
      const int left = N - 32 * w;
      out_mask[w] = n_sel <= 0 ? 0u : left >= 32 ? kSelFull : (1u << left) - 1u;
    }
    __syncthreads();
    return;
  }
  reinterpret_cast<int4*>(hist)[tid] = make_int4(0, 0, 0, 0);  // bins 0 .. 2047 (kSelThreads * 4 = 2048)
  int* wt = misc + kSelWt;
  __syncthreads();
  uint32_t prefix = 0u, mask = 0u;
  int rem = n_sel;
  bool done = false;
#pragma unroll 1
  for (int pass = 0; pass < 3; pass++) {
    const int shift = pass == 0 ? 21 : pass == 1 ? 10 : 0;
    const int nb = pass == 2 ? 1024 : 2048;
    int* h = hist + (pass & 1) * 2048;
    // lanes that fall into the same bin add their count once (keys of
    // similar magnitude share the top bits, and same-address shared atomics
    // serialise)
#pragma unroll 1
    for (int base = 0; base < N; base += kSelThreads) {
      const int p = base + tid;
      int bin = -1;
      if (p < N) {
        const uint32_t k = keys[p * kstride];
        if ((k & mask) == prefix) bin = (int)((k >> shift) & (uint32_t)(nb - 1));
      }
      const unsigned grp = __match_any_sync(kSelFull, bin);
      if (bin >= 0 && lane == __ffs(grp) - 1) atomicAdd(&h[bin], __popc(grp));
    }
    // the other half is zeroed for the next pass (its counts were read before the last barrier)
    if (pass < 2) reinterpret_cast<int4*>(hist + ((pass + 1) & 1) * 2048)[tid] = make_int4(0, 0, 0, 0);
    __syncthreads();
    // thread (warp, lane) scans bins top - 1 .. top - bpl, top = nb - (32 warp + lane) bpl
    const int bpl = nb >> 9;
    const int top = nb - (warp * 32 + lane) * bpl;
    int c[4];
    if (bpl == 4) {
      const int4 v = reinterpret_cast<const int4*>(h)[(top >> 2) - 1];
      c[0] = v.w; c[1] = v.z; c[2] = v.y; c[3] = v.x;
    } else {
      const int2 v = reinterpret_cast<const int2*>(h)[(top >> 1) - 1];
      c[0] = v.y; c[1] = v.x; c[2] = 0; c[3] = 0;
    }
    const int s = c[0] + c[1] + c[2] + c[3];
    int inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int nb2 = __shfl_up_sync(kSelFull, inc, o);
      if (lane >= o) inc += nb2;
    }
    if (lane == 31) wt[warp] = inc;
    __syncthreads();
    int before = inc - s;
#pragma unroll
    for (int w4 = 0; w4 < kSelWarps; w4 += 4) {
      const int4 t4 = reinterpret_cast<const int4*>(wt)[w4 >> 2];
      before += (w4 < warp ? t4.x : 0) + (w4 + 1 < warp ? t4.y : 0) + (w4 + 2 < warp ? t4.z : 0) +
                (w4 + 3 < warp ? t4.w : 0);
    }
    if (before < rem && before + s >= rem) {
#pragma unroll
      for (int j = 0; j < 4; j++) {
        if (before + c[j] >= rem) {
          misc[kSelDig] = top - 1 - j;
          misc[kSelRem] = rem - before;
          misc[kSelCnt] = c[j];
          break;
        }
        before += c[j];
      }
    }
    __syncthreads();
    prefix |= (uint32_t)misc[kSelDig] << shift;
    mask |= (uint32_t)(nb - 1) << shift;
    rem = misc[kSelRem];
    done = rem == misc[kSelCnt];
    if (done) break;
  }
  if (done) {
    // the boundary bin is taken whole: every key whose decided bits are at
    // least the boundary prefix
#pragma unroll 1
    for (int base = 0; base < N; base += kSelThreads) {
      const int p = base + tid;
      const unsigned bal = __ballot_sync(kSelFull, p < N && (keys[p * kstride] & mask) >= prefix);
      const int w = (base >> 5) + warp;
      if (lane == 0 && w < nw) out_mask[w] = bal;
    }
    __syncthreads();
    return;
  }
  // fully resolved threshold T = prefix with more equal keys than needed:
  // keys > T, and the first `rem` keys == T by position
  int* wc = hist;  // equal keys per word
#pragma unroll 1
  for (int base = 0; base < N; base += kSelThreads) {
    const int p = base + tid;
    const unsigned bal = __ballot_sync(kSelFull, p < N && keys[p * kstride] == prefix);
    const int w = (base >> 5) + warp;
    if (lane == 0 && w < nw) wc[w] = __popc(bal);
  }
  __syncthreads();
#pragma unroll 1
  for (int base = 0; base < N; base += kSelThreads) {
    const int p = base + tid;
    const int w = (base >> 5) + warp;
    int before = 0;
    for (int v = lane; v < w && v < nw; v += 32) before += wc[v];
    before = warp_sum(before);
    const uint32_t k = p < N ? keys[p * kstride] : 0u;
    const unsigned eq = __ballot_sync(kSelFull, p < N && k == prefix);
    const int rank = before + __popc(eq & ((1u << lane) - 1u));
    const unsigned bal = __ballot_sync(kSelFull, p < N && (k > prefix || (k == prefix && rank < rem)));
    if (lane == 0 && w < nw) out_mask[w] = bal;
  }
  __syncthreads();
}

// Top-n_sel of N <= 2048 keys below 2^31 (non-negative float bit patterns,
// or such patterns plus one), larger first, ties to the lower position: the
// same set as block_select_top, with fewer block barriers in the common case.
// Each pass counts the keys that share the decided prefix into the bins of
// the next digit (bits 30..20, 19..9, 8..0), with warp-aggregated shared
// atomics (lanes that hit one bin add once), then scans the bins from the top
// and finds the boundary bin.  If that bin is taken whole the selection ends;
// if it holds at most 32 keys, one warp ranks them exactly (key, then
// position) and the first `rem` join the selection; otherwise the next digit
// splits the bin.  After the last digit every key left in the boundary bin
// equals the threshold, and the first `rem` of them by position are taken.
// hist: 2048 ints, all zero on entry and zero again on return.  scratch: 96
// ints (64 extra-mask words, 32 collected positions).  misc: pass state at
// kSelDig .. kSelCnt, kSelColl, and 16 warp totals from kSelWt.  Every thread
// of a 512-thread CTA calls it.
constexpr int kSelColl = 7;
static __device__ __noinline__ void block_select_top31(const uint32_t* keys, int kstride, int N, int n_sel,
                                                       int* hist, int* misc, int* scratch, uint32_t* out_mask) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (N + 31) >> 5;
  if (n_sel >= N || n_sel <= 0) {
    for (int w = tid; w < nw; w += kSelThreads) {
      const int left = N - 32 * w;
      out_mask[w] = n_sel <= 0 ? 0u : left >= 32 ? kSelFull : (1u << left) - 1u;
    }
    __syncthreads();
    return;
  }
  uint32_t* extra = reinterpret_cast<uint32_t*>(scratch);
  int* coll = scratch + 64;
  int* wt = misc + kSelWt;
  if (tid < 64) extra[tid] = 0u;
  uint32_t prefix = 0u, pmask = 0u;
  int rem = n_sel;
#pragma unroll 1
  for (int pass = 0; pass < 3; pass++) {
    const int shift = pass == 0 ? 20 : pass == 1 ? 9 : 0;
    const int nb = pass == 2 ? 512 : 2048;
    if (tid == 0) misc[kSelColl] = 0;
#pragma unroll 1
    for (int base = 0; base < N; base += kSelThreads) {
      const int p = base + tid;
      const uint32_t k = p < N ? keys[p * kstride] : 0u;
      const bool on = p < N && (k & pmask) == prefix;
      const int bin = on ? (int)((k >> shift) & (uint32_t)(nb - 1)) : -1;
      const unsigned same = __match_any_sync(kSelFull, bin);
      if (on && __ffs(same) - 1 == lane) atomicAdd(&hist[bin], __popc(same));
    }
    __syncthreads();
    // thread t scans bins top - 1 .. top - 4, top = nb - 4 t (none past nb),
    // and clears them for the next pass / call
    const int top = nb - 4 * tid;
    int c[4] = {0, 0, 0, 0};
    if (top > 0) {
      int4* h4 = reinterpret_cast<int4*>(hist) + (top >> 2) - 1;
      const int4 v = *h4;
      c[0] = v.w; c[1] = v.z; c[2] = v.y; c[3] = v.x;
      *h4 = make_int4(0, 0, 0, 0);
    }
    const int s = c[0] + c[1] + c[2] + c[3];
    int inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int nb2 = __shfl_up_sync(kSelFull, inc, o);
      if (lane >= o) inc += nb2;
    }
    if (lane == 31) wt[warp] = inc;
    __syncthreads();
    int before = inc - s;
#pragma unroll
    for (int w4 = 0; w4 < kSelWarps; w4 += 4) {
      const int4 t4 = reinterpret_cast<const int4*>(wt)[w4 >> 2];
      before += (w4 < warp ? t4.x : 0) + (w4 + 1 < warp ? t4.y : 0) + (w4 + 2 < warp ? t4.z : 0) +
                (w4 + 3 < warp ? t4.w : 0);
    }
    if (top > 0 && before < rem && before + s >= rem) {
#pragma unroll
      for (int j = 0; j < 4; j++) {
        if (before + c[j] >= rem) {
          misc[kSelDig] = top - 1 - j;
          misc[kSelRem] = rem - before;
          misc[kSelCnt] = c[j];
          break;
        }
        before += c[j];
      }
    }
    __syncthreads();
    prefix |= (uint32_t)misc[kSelDig] << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    rem = misc[kSelRem];
    const int cnt = misc[kSelCnt];
    if (rem == cnt) {
      // the boundary bin is taken whole
#pragma unroll 1
      for (int base = 0; base < N; base += kSelThreads) {
        const int p = base + tid;
        const unsigned bal = __ballot_sync(kSelFull, p < N && (keys[p * kstride] & pmask) >= prefix);
        const int w = (base >> 5) + warp;
        if (lane == 0 && w < nw) out_mask[w] = bal;
      }
      __syncthreads();
      return;
    }
    if (cnt <= 32 || pass == 2) break;
  }
  const int cnt = misc[kSelCnt];
  if (cnt <= 32) {
    // collect the boundary bin's positions; one warp ranks them exactly
#pragma unroll 1
    for (int base = 0; base < N; base += kSelThreads) {
      const int p = base + tid;
      const bool on = p < N && (keys[p * kstride] & pmask) == prefix;
      const unsigned bal = __ballot_sync(kSelFull, on);
      int at = 0;
      if (lane == 0 && bal) at = atomicAdd(&misc[kSelColl], __popc(bal));
      at = __shfl_sync(kSelFull, at, 0);
      if (on) coll[at + __popc(bal & ((1u << lane) - 1u))] = p;
    }
    __syncthreads();
    if (warp == 0) {
      const bool has = lane < cnt;
      const int p = has ? coll[lane] : 0;
      const uint32_t k = has ? keys[p * kstride] : 0u;
      int rank = 0;
#pragma unroll 1
      for (int m = 0; m < cnt; m++) {
        const uint32_t km = __shfl_sync(kSelFull, k, m);
        const int pm = __shfl_sync(kSelFull, p, m);
        rank += (km > k) || (km == k && pm < p);
      }
      if (has && rank < rem) atomicOr(&extra[p >> 5], 1u << (p & 31));
    }
  } else if (warp == 0) {
    // every key left equals the threshold: the first `rem` by position
    int left = rem;
#pragma unroll 1
    for (int w = 0; w < nw && left > 0; w++) {
      const int p = 32 * w + lane;
      const unsigned eq = __ballot_sync(kSelFull, p < N && keys[p * kstride] == prefix);
      const int n_eq = __popc(eq);
      uint32_t take = eq;
      if (n_eq > left) {
        // the lowest `left` set bits of eq
        const bool mine = ((eq >> lane) & 1u) && __popc(eq & ((1u << lane) - 1u)) < left;
        take = __ballot_sync(kSelFull, mine);
      }
      if (lane == 0) extra[w] = take;
      left -= __popc(take);
    }
  }
  __syncthreads();
#pragma unroll 1
  for (int base = 0; base < N; base += kSelThreads) {
    const int p = base + tid;
    const unsigned bal = __ballot_sync(kSelFull, p < N && (keys[p * kstride] & pmask) > prefix);
    const int w = (base >> 5) + warp;
    if (lane == 0 && w < nw) out_mask[w] = bal | extra[w];
  }
  __syncthreads();
}

// Ascending list of the set bits of (m0 | m1) over [0, N), N <= 2048 (m1
// may be null); the count lands in *count_out.  Warp 0 forms the union words
// and their exclusive prefix counts (scratch, 64 ints each), then every warp
// writes the positions of its words.
static __device__ __noinline__ void block_mask_to_list(const uint32_t* m0, const uint32_t* m1, int N, int* list,
                                                       int* count_out, int* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (N + 31) >> 5;
  uint32_t* uw = reinterpret_cast<uint32_t*>(scratch + 64);
  if (warp == 0) {
    uint32_t a0 = 0u, a1 = 0u;
    if (lane < nw) a0 = m0[lane] | (m1 ? m1[lane] : 0u);
    if (lane + 32 < nw) a1 = m0[lane + 32] | (m1 ? m1[lane + 32] : 0u);
    const int c0 = __popc(a0), c1 = __popc(a1);
    int i0 = c0, i1 = c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n0 = __shfl_up_sync(kSelFull, i0, o), n1 = __shfl_up_sync(kSelFull, i1, o);
      if (lane >= o) {
        i0 += n0;
        i1 += n1;
      }
    }
    const int t0 = __shfl_sync(kSelFull, i0, 31), t1 = __shfl_sync(kSelFull, i1, 31);
    scratch[lane] = i0 - c0;
    scratch[lane + 32] = t0 + i1 - c1;
    uw[lane] = a0;
    uw[lane + 32] = a1;
    if (lane == 0) *count_out = t0 + t1;
  }
  __syncthreads();
  for (int w = warp; w < nw; w += kSelWarps) {
    const uint32_t m = uw[w];
    if ((m >> lane) & 1u) list[scratch[w] + __popc(m & ((1u << lane) - 1u))] = 32 * w + lane;
  }
  __syncthreads();
}

}  // namespace sel
}  // namespace moe
