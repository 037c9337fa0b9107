// route.cu -- router logits, rotation + int8 quantisation, top-e selection
// and the per-step tables: work items of up to two tokens (one-cluster and
// dense kernels) and the active experts with their (token, slot) pairs in
// expert order (streamed kernels; under expert parallelism only the experts
// e % ep_size == ep_rank).
//
// Routing follows the pages' "routed experts" (abstract of "Channel Selection
// for Mixture-of-Experts Decoding Needs No Calibration Data"): softmax routing
// to the top-e experts, renormalised over the chosen ones.  Logits are exact
// bf16*bf16 products summed in fp64.  The rotation H (s . x) is the rotated
// domain of the "rotated ternary sketch" ("KAIST: MoE Decoding Needs No
// Calibration Data", section "A reader that needs no data at all").
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kRouteExpertsPerCta = 2;  // four warps per expert row
constexpr int kRouteTokensPerCta = 8;

__device__ __forceinline__ void dfma8(uint4 w, uint4 x, double& acc) {
  acc = fma((double)bf16lo(w.x), (double)bf16lo(x.x), acc);
  acc = fma((double)bf16hi(w.x), (double)bf16hi(x.x), acc);
  acc = fma((double)bf16lo(w.y), (double)bf16lo(x.y), acc);
  acc = fma((double)bf16hi(w.y), (double)bf16hi(x.y), acc);
  acc = fma((double)bf16lo(w.z), (double)bf16lo(x.z), acc);
  acc = fma((double)bf16hi(w.z), (double)bf16hi(x.z), acc);
  acc = fma((double)bf16lo(w.w), (double)bf16lo(x.w), acc);
  acc = fma((double)bf16hi(w.w), (double)bf16hi(x.w), acc);
}

// Blocks [0, n_logit_blocks) compute logits; the next B blocks (sparse path)
// rotate and quantise one token each.  A logits block takes 2 experts and up
// to 8 tokens: 4 warps per expert, each a quarter of d (two 16-byte chunks
// per lane at a time, the chunks of every token in flight together); the
// quarters' fp64 sums meet in shared memory.
__global__ void __launch_bounds__(256) route_kernel(RouteArgs a, int n_logit_blocks, int n_eblk) {
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if ((int)blockIdx.x < n_logit_blocks) {
    __shared__ double part[kRouteExpertsPerCta][4][kRouteTokensPerCta];
    const int el = warp >> 2, wq = warp & 3;
    const int e = (blockIdx.x % n_eblk) * kRouteExpertsPerCta + el;
    const int t0 = (blockIdx.x / n_eblk) * kRouteTokensPerCta;
    const int nt = min(kRouteTokensPerCta, a.B - t0);
    double acc[kRouteTokensPerCta];
#pragma unroll
    for (int t = 0; t < kRouteTokensPerCta; t++) acc[t] = 0.0;
    const int d8 = a.d / 8;
    if (e < a.E) {
      const uint4* wrow = reinterpret_cast<const uint4*>(a.w_router + (size_t)e * a.d);
      // chunk j = 32 wq + lane + 128 u of the row
#pragma unroll 1
      for (int u0 = 0; 128 * u0 < d8; u0 += 2) {
        uint4 w[2], xv[kRouteTokensPerCta][2];
#pragma unroll
        for (int u = 0; u < 2; u++) {
          const int j = 32 * wq + lane + 128 * (u0 + u);
          w[u] = j < d8 ? __ldg(wrow + j) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int t = 0; t < kRouteTokensPerCta; t++)
            xv[t][u] = j < d8 && t < nt ? __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)(t0 + t) * a.d) + j)
                                        : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int t = 0; t < kRouteTokensPerCta; t++) {
          dfma8(w[0], xv[t][0], acc[t]);
          dfma8(w[1], xv[t][1], acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kRouteTokensPerCta; t++) {
      const double s = warp_sum(acc[t]);
      if (lane == 0) part[el][wq][t] = s;
    }
    __syncthreads();
    if (threadIdx.x < kRouteExpertsPerCta * kRouteTokensPerCta) {
      const int ee = threadIdx.x / kRouteTokensPerCta, t = threadIdx.x % kRouteTokensPerCta;
      const int eg = (blockIdx.x % n_eblk) * kRouteExpertsPerCta + ee;
      if (eg < a.E && t < nt) {
        const double s = (part[ee][0][t] + part[ee][1][t]) + (part[ee][2][t] + part[ee][3][t]);
        a.ws.logits[(size_t)(t0 + t) * a.E + eg] = s + (a.bias ? (double)a.bias[eg] : 0.0);
      }
    }
    return;
  }
  // ---- rotate + quantise token b: v = FWHT(s . x), q = rint(127 v / amax)
  extern __shared__ float v[];
  __shared__ float red[kWarps];
  const int b = blockIdx.x - n_logit_blocks;
  const int d = a.d;
  for (int j = threadIdx.x; j < d; j += blockDim.x)
    v[j] = (float)a.rot_sign[j] * bf16f(a.x[(size_t)b * d + j]);
  __syncthreads();
  // Sylvester order, stages h = 1, 2, 4, ...: the same butterflies as the
  // reference transform, so the same bits.
  for (int h = 1, lh = 0; h < d; h <<= 1, lh++) {
    for (int p = threadIdx.x; p < d / 2; p += blockDim.x) {
      const int j = ((p >> lh) << (lh + 1)) | (p & (h - 1));
      const float x0 = v[j], x1 = v[j + h];
      v[j] = __fadd_rn(x0, x1);
      v[j + h] = __fsub_rn(x0, x1);
    }
    __syncthreads();
  }
  float m = 0.0f;
  for (int j = threadIdx.x; j < d; j += blockDim.x) m = fmaxf(m, fabsf(v[j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float amax = 0.0f;
  for (int w = 0; w < (int)(blockDim.x >> 5); w++) amax = fmaxf(amax, red[w]);
  int8_t* q = a.ws.q + (size_t)b * d;
  int qs = 0;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    int n = 0;
    if (amax > 0.0f) {
      n = __float2int_rn(__fdiv_rn(__fmul_rn(v[j], 127.0f), amax));
      n = max(-127, min(127, n));
    }
    q[j] = (int8_t)n;
    qs += n;
  }
  // the sum of the activations: the sketch dots' code offset (codes are T + 1)
  __shared__ int redq[kWarps];
  qs = warp_sum(qs);
  if (lane == 0) redq[warp] = qs;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); w++) tot += redq[w];
    a.ws.qsum[b] = tot;
    a.ws.cx[b] = amax > 0.0f ? __fdiv_rn(amax, __fmul_rn(127.0f, (float)d)) : 0.0f;
  }
}


// One CTA: top-e per token (ties to the lower id) and softmax weights, one
// warp per token; then, one warp per expert, the token-ordered tables of the
// step from ballots over the tokens: the work items of up to kMaxGroup tokens
// (one-cluster and dense kernels), the active experts and the pairs in expert
// order (streamed kernels).  Also zeroes the step's counters.
__global__ void __launch_bounds__(512) select_kernel(RouteArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sm[];
  const int E = a.E, top = a.top_e, B = a.B;
  int* sids = sm;              // [B * top] chosen experts
  int* cnt = sids + B * top;   // [E] tokens per expert
  int* pbase = cnt + E;        // [E] first pair of each expert
  int* ibase = pbase + E;      // [E] first work item of each expert
  int* aidx = ibase + E;       // [E] active index (experts with tokens)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  for (int b = warp; b < B; b += nwarp) {
    const double* L = a.ws.logits + (size_t)b * E;
    uint32_t taken = 0;
    // this lane's logits (E <= 1024), read once; the unrolled loops stop at
    // the first m past E (m < ceil(E / 32))
    const int nm = (E + 31) >> 5;
    double lv[32];
#pragma unroll
    for (int m = 0; m < 32; m++) {
      if (m >= nm) break;
      lv[m] = lane + 32 * m < E ? L[lane + 32 * m] : -INFINITY;
    }
    double l0 = 0.0, my_l = 0.0;
    int my_id = 0;
    for (int s = 0; s < top; s++) {
      double bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int m = 0; m < 32; m++) {
        if (m >= nm) break;
        const int e = lane + 32 * m;
        if (e >= E || (taken & (1u << m))) continue;
        if (bi == 0x7fffffff || lv[m] > bv) {
          bv = lv[m];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
          bv = ov;
          bi = oi;
        }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (s == 0) l0 = bv;
      if (lane == s) {
        my_l = bv;
        my_id = bi;
      }
    }
    // softmax over the chosen logits: fp32 exponentials of the fp64
    // differences to the largest (the weights only scale outputs)
    const float ex = lane < top ? __expf((float)(my_l - l0)) : 0.0f;
    double den = (double)ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane < top) {
      const float w = (float)((double)ex / den);
      a.ws.ids[b * top + lane] = my_id;
      a.ws.wts[b * top + lane] = w;
      sids[b * top + lane] = my_id;
      if (a.dbg_ids) a.dbg_ids[b * top + lane] = my_id;
      if (a.dbg_w) a.dbg_w[b * top + lane] = w;
    }
  }
  for (int i = threadIdx.x; i < B * kMaxCluster; i += blockDim.x) a.ws.counters[i] = 0u;
  for (int i = threadIdx.x; i < 2 * E; i += blockDim.x) a.ws.arrive[i] = 0u;
  // tokens per expert, and each expert's token set as a bit mask (emask[e]
  // holds nwb words): one pass over the (token, slot) entries
  const int nwb = (B + 31) >> 5;
  uint32_t* emask = reinterpret_cast<uint32_t*>(aidx + E);  // [E, nwb]
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  for (int i = threadIdx.x; i < E * nwb; i += blockDim.x) emask[i] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < B * top; i += blockDim.x) {
    const int e = sids[i], t = i / top;
    atomicAdd(&cnt[e], 1);
    atomicOr(&emask[e * nwb + (t >> 5)], 1u << (t & 31));
  }
  __syncthreads();
  // experts this rank owns (expert parallelism); the pair table holds only theirs
  auto owned = [&](int e) { return a.ep_size <= 1 || e % a.ep_size == a.ep_rank; };
  // exclusive prefixes over the experts: pairs, work items, active experts
  if (warp == 0) {
    int rp = 0, ri = 0, ra = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int ca = e < E ? cnt[e] : 0, it = (ca + kMaxGroup - 1) / kMaxGroup;
      const int c = e < E && owned(e) ? ca : 0, ac = c > 0;
      int ip = c, ii = it, ia = ac;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int vp = __shfl_up_sync(0xffffffffu, ip, o), vi = __shfl_up_sync(0xffffffffu, ii, o),
                  va = __shfl_up_sync(0xffffffffu, ia, o);
        if (lane >= o) {
          ip += vp;
          ii += vi;
          ia += va;
        }
      }
      if (e < E) {
        pbase[e] = rp + ip - c;
        ibase[e] = ri + ii - it;
        aidx[e] = ra + ia - ac;
        if (ac) {
          a.ws.act_e[ra + ia - 1] = e;
          int w = a.expert_slot ? __ldg(a.expert_slot + e) : e;
          if (w < 0) {  // routed to an expert whose weights this caller does not hold
            atomicOr(a.ws.err, kErrNoWeights);
            w = 0;
          }
          a.ws.act_w[ra + ia - 1] = w;
          a.ws.act_off[ra + ia - 1] = rp + ip - c;
        }
      }
      rp += __shfl_sync(0xffffffffu, ip, 31);
      ri += __shfl_sync(0xffffffffu, ii, 31);
      ra += __shfl_sync(0xffffffffu, ia, 31);
    }
    if (lane == 0) {
      *a.ws.n_items = ri;
      *a.ws.n_act = ra;
      a.ws.act_off[ra] = rp;
    }
  }
  __syncthreads();
  // each expert's pairs and work items, tokens ascending: entry (t, s) of
  // expert e sits at the count of e's tokens below t
  for (int i = threadIdx.x; i < B * top; i += blockDim.x) {
    const int e = sids[i], t = i / top, slot = i - t * top;
    const uint32_t* em = emask + e * nwb;
    int pos = __popc(em[t >> 5] & ((1u << (t & 31)) - 1u));
    for (int w = 0; w < (t >> 5); w++) pos += __popc(em[w]);
    if (owned(e)) {
      const int pr = pbase[e] + pos;
      a.ws.pair_tok[pr] = t;
      a.ws.pair_slot[pr] = slot;
      a.ws.pair_ea[pr] = aidx[e];
    }
    const int item = ibase[e] + pos / kMaxGroup, g = pos % kMaxGroup;
    if (item < a.ws.max_items) {
      a.ws.item_tok[item * kMaxGroup + g] = t;
      a.ws.item_slot[item * kMaxGroup + g] = slot;
      if (g == 0) {
        a.ws.item_e[item] = e;
        a.ws.item_n[item] = min(kMaxGroup, cnt[e] - pos);
      }
    }
  }
}

}  // namespace

int max_work_items(int B, int E, int top_e, int group) {
  const long T = (long)B * top_e;
  const long m = T < E ? T : E;
  return (int)((T + m * (group - 1)) / group);
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t workspace_layout(int B, int E, int top_e, int d, int I, int r, void* base, Workspace* ws) {
  const int mi = max_work_items(B, E, top_e, kMaxGroup);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  // error word and combine counters sit at fixed offsets for every shape, so
  // a workspace stays valid when it is reused for a different batch size
  const size_t o_err = take(16), o_ct = take(sizeof(unsigned) * kMaxTokens * kMaxCluster), o_ni = take(16);
  const size_t o_log = take(sizeof(double) * B * E);
  const size_t o_ids = take(sizeof(int) * B * top_e), o_w = take(sizeof(float) * B * top_e);
  const size_t o_q = take((size_t)B * d), o_cx = take(sizeof(float) * B);
  const size_t o_ie = take(sizeof(int) * mi), o_in = take(sizeof(int) * mi);
  const size_t o_it = take(sizeof(int) * mi * kMaxGroup), o_is = take(sizeof(int) * mi * kMaxGroup);
  const size_t o_ye = take(sizeof(float) * B * top_e * (size_t)d);
  // the streamed path
  const size_t P = (size_t)B * top_e, W = (size_t)(I + 31) / 32, nbs = (size_t)(I + 15) / 16;
  const bool st = I > 0;
  const size_t o_qs = take(sizeof(int) * B), o_na = take(16), o_ae = take(sizeof(int) * E), o_aw = take(sizeof(int) * E),
               o_ao = take(sizeof(int) * (E + 1)), o_pt = take(sizeof(int) * P), o_ps = take(sizeof(int) * P),
               o_pe = take(sizeof(int) * P), o_ar = take(sizeof(unsigned) * 2 * E);
  const size_t o_sa = st ? take(sizeof(float2) * P * I) : 0, o_zp = st ? take(sizeof(float) * P * nbs * r) : 0,
               o_cm = st ? take(sizeof(uint32_t) * P * W) : 0, o_ap = st ? take(sizeof(float) * P * I) : 0,
               o_km = st ? take(sizeof(uint32_t) * P * W) : 0, o_z = st ? take(sizeof(float) * P * r) : 0,
               o_ul = st ? take(sizeof(int) * E * (size_t)I) : 0, o_nu = st ? take(sizeof(int) * E) : 0,
               o_dl = st ? take(sizeof(int) * E * (size_t)I) : 0, o_nd = st ? take(sizeof(int) * E) : 0,
               o_co = st ? take(sizeof(float) * P * I) : 0;
  if (ws && base) {
    char* p = static_cast<char*>(base);
    ws->err = reinterpret_cast<uint32_t*>(p + o_err);
    ws->n_items = reinterpret_cast<int*>(p + o_ni);
    ws->logits = reinterpret_cast<double*>(p + o_log);
    ws->ids = reinterpret_cast<int*>(p + o_ids);
    ws->wts = reinterpret_cast<float*>(p + o_w);
    ws->q = reinterpret_cast<int8_t*>(p + o_q);
    ws->cx = reinterpret_cast<float*>(p + o_cx);
    ws->item_e = reinterpret_cast<int*>(p + o_ie);
    ws->item_n = reinterpret_cast<int*>(p + o_in);
    ws->item_tok = reinterpret_cast<int*>(p + o_it);
    ws->item_slot = reinterpret_cast<int*>(p + o_is);
    ws->ye = reinterpret_cast<float*>(p + o_ye);
    ws->counters = reinterpret_cast<unsigned*>(p + o_ct);
    ws->max_items = mi;
    ws->qsum = reinterpret_cast<int*>(p + o_qs);
    ws->n_act = reinterpret_cast<int*>(p + o_na);
    ws->act_e = reinterpret_cast<int*>(p + o_ae);
    ws->act_w = reinterpret_cast<int*>(p + o_aw);
    ws->act_off = reinterpret_cast<int*>(p + o_ao);
    ws->pair_tok = reinterpret_cast<int*>(p + o_pt);
    ws->pair_slot = reinterpret_cast<int*>(p + o_ps);
    ws->pair_ea = reinterpret_cast<int*>(p + o_pe);
    ws->arrive = reinterpret_cast<unsigned*>(p + o_ar);
    ws->sa = st ? reinterpret_cast<float2*>(p + o_sa) : nullptr;
    ws->zpart = st ? reinterpret_cast<float*>(p + o_zp) : nullptr;
    ws->candm = st ? reinterpret_cast<uint32_t*>(p + o_cm) : nullptr;
    ws->apos = st ? reinterpret_cast<float*>(p + o_ap) : nullptr;
    ws->keptm = st ? reinterpret_cast<uint32_t*>(p + o_km) : nullptr;
    ws->z = st ? reinterpret_cast<float*>(p + o_z) : nullptr;
    ws->ulist = st ? reinterpret_cast<int*>(p + o_ul) : nullptr;
    ws->n_u = st ? reinterpret_cast<int*>(p + o_nu) : nullptr;
    ws->dlist = st ? reinterpret_cast<int*>(p + o_dl) : nullptr;
    ws->n_d = st ? reinterpret_cast<int*>(p + o_nd) : nullptr;
    ws->coef = st ? reinterpret_cast<float*>(p + o_co) : nullptr;
  }
  return off;
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  const int n_eblk = (a.E + kRouteExpertsPerCta - 1) / kRouteExpertsPerCta;
  const int n_tblk = (a.B + kRouteTokensPerCta - 1) / kRouteTokensPerCta;
  const int nlog = n_eblk * n_tblk;
  const int grid = nlog + (a.quantize ? a.B : 0);
  const size_t smem = a.quantize ? sizeof(float) * a.d : 0;
  route_kernel<<<grid, 256, smem, s>>>(a, nlog, n_eblk);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(512);
  cfg.dynamicSmemBytes = sizeof(int) * (4 * a.E + a.B * a.top_e + a.E * ((a.B + 31) / 32));
  if (cfg.dynamicSmemBytes > 48 * 1024) {
    err = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cfg.dynamicSmemBytes);
    if (err != cudaSuccess) return err;
  }
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_kernel, a);
}

}  // namespace moe
