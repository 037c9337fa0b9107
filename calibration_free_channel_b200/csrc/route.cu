// route.cu -- router logits, rotation + int8 quantisation, top-e selection
// and the per-step work table.
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

constexpr int kRouteExpertsPerCta = 8;  // one warp per expert row
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
// rotate and quantise one token each.
__global__ void __launch_bounds__(256) route_kernel(RouteArgs a, int n_logit_blocks, int n_eblk) {
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if ((int)blockIdx.x < n_logit_blocks) {
    const int e = (blockIdx.x % n_eblk) * kRouteExpertsPerCta + warp;
    const int t0 = (blockIdx.x / n_eblk) * kRouteTokensPerCta;
    const int nt = min(kRouteTokensPerCta, a.B - t0);
    if (e >= a.E) return;
    double acc[kRouteTokensPerCta];
#pragma unroll
    for (int t = 0; t < kRouteTokensPerCta; t++) acc[t] = 0.0;
    const uint4* wrow = reinterpret_cast<const uint4*>(a.w_router + (size_t)e * a.d);
    for (int j = lane; j < a.d / 8; j += 32) {
      const uint4 w = __ldg(wrow + j);
#pragma unroll
      for (int t = 0; t < kRouteTokensPerCta; t++)
        if (t < nt) dfma8(w, __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)(t0 + t) * a.d) + j), acc[t]);
    }
#pragma unroll
    for (int t = 0; t < kRouteTokensPerCta; t++) {
      if (t < nt) {
        const double s = warp_sum(acc[t]);
        if (lane == 0) a.ws.logits[(size_t)(t0 + t) * a.E + e] = s + (a.bias ? (double)a.bias[e] : 0.0);
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
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    int n = 0;
    if (amax > 0.0f) {
      n = __float2int_rn(__fdiv_rn(__fmul_rn(v[j], 127.0f), amax));
      n = max(-127, min(127, n));
    }
    q[j] = (int8_t)n;
  }
  if (threadIdx.x == 0) a.ws.cx[b] = amax > 0.0f ? __fdiv_rn(amax, __fmul_rn(127.0f, (float)d)) : 0.0f;
}

// One CTA: top-e per token (ties to the lower id), softmax weights, the work
// table (one item per (expert, group of <= kMaxGroup tokens)), and the
// combine counters reset.
__global__ void __launch_bounds__(512) select_kernel(RouteArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sm[];
  int* cnt = sm;             // [E]
  int* base = sm + a.E;      // [E]
  int* cursor = base + a.E;  // [E]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const int E = a.E, top = a.top_e;
  for (int b = warp; b < a.B; b += nwarp) {
    const double* L = a.ws.logits + (size_t)b * E;
    uint32_t taken = 0;
    double chosen[16];
    int chosen_id[16];
    double lv[32];  // this lane's logits (E <= 1024), read once
#pragma unroll
    for (int m = 0; m < 32; m++) lv[m] = lane + 32 * m < E ? L[lane + 32 * m] : -INFINITY;
    for (int s = 0; s < top; s++) {
      double bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int m = 0; m < 32; m++) {
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
      chosen[s] = bv;
      chosen_id[s] = bi;
    }
    if (lane == 0) {
      double den = 0.0;
      for (int s = 0; s < top; s++) den += exp(chosen[s] - chosen[0]);
      for (int s = 0; s < top; s++) {
        const float w = (float)(exp(chosen[s] - chosen[0]) / den);
        a.ws.ids[b * top + s] = chosen_id[s];
        a.ws.wts[b * top + s] = w;
        if (a.dbg_ids) a.dbg_ids[b * top + s] = chosen_id[s];
        if (a.dbg_w) a.dbg_w[b * top + s] = w;
      }
    }
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    cnt[e] = 0;
    cursor[e] = 0;
  }
  for (int i = threadIdx.x; i < a.B * kMaxCluster; i += blockDim.x) a.ws.counters[i] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < a.B * top; i += blockDim.x) atomicAdd(&cnt[a.ws.ids[i]], 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; e++) {
      base[e] = run;
      run += (cnt[e] + kMaxGroup - 1) / kMaxGroup;
    }
    *a.ws.n_items = run;
  }
  __syncthreads();
  // Tokens enter their expert's items in increasing token order.
  for (int t = 0; t < a.B; t++) {
    if (threadIdx.x < top) {
      const int e = a.ws.ids[t * top + threadIdx.x];
      const int pos = cursor[e]++;
      const int item = base[e] + pos / kMaxGroup, g = pos % kMaxGroup;
      if (item < a.ws.max_items) {
        a.ws.item_tok[item * kMaxGroup + g] = t;
        a.ws.item_slot[item * kMaxGroup + g] = threadIdx.x;
        if (g == 0) {
          a.ws.item_e[item] = e;
          a.ws.item_n[item] = min(kMaxGroup, cnt[e] - pos);
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace

int max_work_items(int B, int E, int top_e, int group) {
  const long T = (long)B * top_e;
  const long m = T < E ? T : E;
  return (int)((T + m * (group - 1)) / group);
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t workspace_layout(int B, int E, int top_e, int d, void* base, Workspace* ws) {
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
  cfg.dynamicSmemBytes = sizeof(int) * 3 * a.E;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_kernel, a);
}

}  // namespace moe
