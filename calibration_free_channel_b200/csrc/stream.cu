// stream.cu -- the streamed reader: the steps of the sparse reader of
// "KAIST: MoE Decoding Needs No Calibration Data" (section "A reader that
// needs no data at all": screen with the rotated ternary sketch, top-c
// candidates, exact BF16 gate/up of the candidates, top-k by |a|, the kept
// down rows plus the low-rank recovery of the skipped ones), each one kernel
// over every (token, expert) pair of the step, on all SMs.
//
// Stage kernels, after the route and select kernels (route.cu):
//   screen_kernel     sketch dots of every (pair, channel): sigma, ahat, and
//                     the recovery-input partial of each 32-channel block
//   select_c_kernel   one pair per CTA: top-c by sigma; the expert's last pair
//                     forms the candidate union (rows of the next stage)
//   exact_kernel      16 union rows of one expert per unit: g, u of every
//                     token of the expert on the tensor cores (mma.sync bf16),
//                     a = silu(g) u for its candidates
//   select_k_kernel   one pair per CTA: top-k by |a| over its candidates, the
//                     recovery input z; the expert's last pair forms the kept
//                     union and the per-pair row coefficients
//   down_kernel       one (expert, column slice) per unit: kept down rows,
//                     V z, and the combine over the top-e slots by the last
//                     arriving slot of each (token, slice)
// Expert-parallel steps (one rank's experts) skip that combine; then
// ep_combine_kernel sums the rank's slots per token into an fp32 partial and,
// after the caller's all-reduce, ep_finish_kernel adds the residual and rounds.
// Each kernel is launched with programmatic dependent launch and waits on
// its predecessor before reading its outputs; weights are read with
// non-allocating loads, data written by earlier kernels of the chain through
// L2 (ld.global.cg).  Sets and rounding points are those of the one-cluster
// reader (reader.cu), so both paths give the same candidate and kept sets.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace moe {

namespace {

constexpr unsigned kFullMask = 0xffffffffu;

constexpr int kSThreads = 128;  // screen: 4 warps, 8 / NVL channels per warp
constexpr int kSTG = 2;         // screen: tokens per register group
constexpr int kSelT = sel::kSelThreads;
constexpr int kDThreads = 256;  // down rows
constexpr int kDTG = 4;         // down: tokens per register group
constexpr int kDRows = 256;     // down: kept-union rows staged per chunk
constexpr int kMaxI = 2048;
constexpr int kMaxAct = 1024;   // active experts (E <= 1024)

// 16-byte load of weights that are read once per step: no L1 allocation.
__device__ __forceinline__ uint4 ld_cg4(const void* p) { return __ldcg(reinterpret_cast<const uint4*>(p)); }

// Counts one arrival at ctr (release of everything this thread ordered
// before, acquire of the earlier arrivals); true for the last of `total`.
__device__ __forceinline__ bool arrive_last(unsigned* ctr, unsigned total) {
  unsigned old;
  asm volatile("fence.acq_rel.gpu;\n\tatom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
               : "=r"(old)
               : "l"(ctr)
               : "memory");
  return old == total - 1u;
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 w, float (&f)[8]) {
  f[0] = bf16lo(w.x);
  f[1] = bf16hi(w.x);
  f[2] = bf16lo(w.y);
  f[3] = bf16hi(w.y);
  f[4] = bf16lo(w.z);
  f[5] = bf16hi(w.z);
  f[6] = bf16lo(w.w);
  f[7] = bf16hi(w.w);
}

// Screen-block geometry for NVL = 1 (d <= 2048) and NVL = 2 (d = 4096): a
// warp takes kPerWarp channels, each split over kParts lanes (parts of d);
// a block's sketch rows are 16 KB per matrix either way.
template <int NVL>
struct ScreenGeom {
  static constexpr int kPerWarp = 8 / NVL;
  static constexpr int kParts = 32 / kPerWarp;
  static constexpr int kChannels = 4 * kPerWarp;  // 4 warps
};
constexpr int kSkBytes = 16384;                      // sketch rows of one block, per matrix
constexpr int kSStageBytes = 2 * kSkBytes + 8192 + 256;  // + the block's Ubar rows (<= 32 x 128 bf16), alpha_g, alpha_u
constexpr int kQChunk = 80;                          // staged activations: 64 bytes per chunk, padded

// ------------------------------------------------------------------ screen
// Unit = (active expert, block of ScreenGeom::kChannels channels).  The
// block's gate and up sketch rows (and its Ubar rows) are contiguous: one
// thread copies them into shared memory with bulk copies, the next unit's
// copies in flight while this one is computed (two stages).  Lane (c, p) of a
// warp takes channel c and part p of d: it walks its 64-trit chunks of both
// rows (in an order rotated by lane, so the eight lanes of a shared-memory
// wavefront read distinct banks) against the tokens' activations, staged kSTG
// tokens at a time; two shuffles sum the parts, and lane p = t of the channel
// finishes token t.  Scores follow the one-cluster reader: ghat =
// ((float)G alpha_g) c_x, uhat likewise, ahat = silu_r(ghat) uhat,
// sigma = |ahat|, with G, U the exact integer dots less the code offset sum(q).
template <int NVL, bool SK3>
__device__ __forceinline__ void screen_issue(const ExpertArgs& a, int u, int nblk, char* dst, uint64_t* bar) {
  using Geo = ScreenGeom<NVL>;
  const int ea = u / nblk, blk = u - ea * nblk;
  const int e = __ldcg(a.ws.act_w + ea);  // weight slot of the active expert
  const int i0 = blk * Geo::kChannels, ncw = min(Geo::kChannels, a.I - i0);
  const size_t row = SK3 ? (size_t)sk3_row_bytes(a.d) : (size_t)a.d / 4;  // bytes of one sketch row
  const uint32_t bytes = (uint32_t)(ncw * row), ubytes = (uint32_t)(ncw * a.r * 2);
  const bool acopy = a.I % 4 == 0;  // the scales' slices are 16-byte aligned (else plain loads)
  mbar_expect_tx(bar, 2 * bytes + ubytes + (acopy ? 8 * ncw : 0));
  bulk_g2s(dst, reinterpret_cast<const char*>(a.sk_gate) + ((size_t)e * a.I + i0) * row, bytes, bar);
  bulk_g2s(dst + kSkBytes, reinterpret_cast<const char*>(a.sk_up) + ((size_t)e * a.I + i0) * row, bytes, bar);
  if (ubytes) bulk_g2s(dst + 2 * kSkBytes, a.u_sigma + ((size_t)e * a.I + i0) * a.r, ubytes, bar);
  if (acopy) {
    bulk_g2s(dst + 2 * kSkBytes + 8192, a.alpha_gate + (size_t)e * a.I + i0, 4 * ncw, bar);
    bulk_g2s(dst + 2 * kSkBytes + 8192 + 128, a.alpha_up + (size_t)e * a.I + i0, 4 * ncw, bar);
  }
}

template <int NVL, bool SK3>
__global__ void __launch_bounds__(kSThreads) screen_kernel(ExpertArgs a) {
  pdl_trigger();
  pdl_wait();
  using Geo = ScreenGeom<NVL>;
  extern __shared__ __align__(128) char sk_stage[];  // [2][gate 16 KB | up 16 KB | Ubar 8 KB]
  __shared__ __align__(16) char qst[kSTG * 64 * kQChunk];  // staged activations (d <= 4096)
  __shared__ float sah[kSTG][Geo::kChannels];
  __shared__ float salg[Geo::kChannels], salu[Geo::kChannels];
  __shared__ int stok[kSTG], sqs[kSTG];
  __shared__ float scx[kSTG];
  __shared__ __align__(8) uint64_t bars[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int I = a.I, d = a.d, r = a.r;
  const int nv = d >> 6;                     // 64-trit chunks (16 bytes) per row
  const int nch = nv / Geo::kParts;          // chunks per lane
  const int c = lane / Geo::kParts, part = lane - c * Geo::kParts;
  const int lc = warp * Geo::kPerWarp + c;   // the lane's channel in the block
  const int rot = lane & 7;
  const int nblk = (I + Geo::kChannels - 1) / Geo::kChannels;
  const int zstride = (I + 15) / 16;         // zpart blocks per pair (the finest geometry)
  const int n_act = __ldcg(a.ws.n_act);
  const int units = n_act * nblk;
  uint32_t* err = a.ws.err;
  // base 3: rows of skrow bytes, nv3 16-byte chunks (80 trits each); lane
  // part p takes chunks p, p + kParts, ...
  const int skrow = SK3 ? sk3_row_bytes(d) : d / 4, nv3 = skrow / 16;
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // units are dealt round-robin: the CTAs in flight together read one
  // contiguous stretch of the sketch arrays, which spreads the reads evenly
  // over the DRAM channels (contiguous ranges per CTA measured slower)
  const bool acopy = I % 4 == 0;  // the scales arrive with the stage's bulk copies
  if (tid == 0 && (int)blockIdx.x < units) screen_issue<NVL, SK3>(a, blockIdx.x, nblk, sk_stage, &bars[0]);
  int it = 0, staged_p0 = -1, staged_tg = -1;
#pragma unroll 1
  for (int u = blockIdx.x; u < units; u += gridDim.x, it++) {
    const int st = it & 1;
    if (tid == 0 && u + (int)gridDim.x < units)
      screen_issue<NVL, SK3>(a, u + gridDim.x, nblk, sk_stage + (st ^ 1) * kSStageBytes, &bars[st ^ 1]);
    const int ea = u / nblk, blk = u - ea * nblk;
    const int e = __ldcg(a.ws.act_w + ea), p0 = __ldcg(a.ws.act_off + ea);  // e: weight slot
    const int m = __ldcg(a.ws.act_off + ea + 1) - p0;
    const int i0 = blk * Geo::kChannels, ncw = min(Geo::kChannels, I - i0);
    const bool ok = lc < ncw;
    const char* stage = sk_stage + st * kSStageBytes;
    if (!acopy && tid < ncw) {
      salg[tid] = __ldg(a.alpha_gate + (size_t)e * I + i0 + tid);
      salu[tid] = __ldg(a.alpha_up + (size_t)e * I + i0 + tid);
    }
    const float* alg = acopy ? reinterpret_cast<const float*>(stage + 2 * kSkBytes + 8192) : salg;
    const float* alu = acopy ? reinterpret_cast<const float*>(stage + 2 * kSkBytes + 8192 + 128) : salu;
    const uint4* grow = reinterpret_cast<const uint4*>(stage) + (size_t)lc * nv + part * nch;
    const uint4* urow = reinterpret_cast<const uint4*>(stage + kSkBytes) + (size_t)lc * nv + part * nch;
    const uint16_t* ubs = reinterpret_cast<const uint16_t*>(stage + 2 * kSkBytes);
    // a stage whose copy did not land in time is not read (the error word
    // records it; the unit's scores stay zero)
    const bool landed = mbar_wait_bounded(&bars[st], (it >> 1) & 1, err, a.wait_ns);
#pragma unroll 1
    for (int tg = 0; tg < m; tg += kSTG) {
      const int ng = min(kSTG, m - tg);
      __syncthreads();  // the previous group is done with qst (and the alpha stores are visible)
      if (p0 != staged_p0 || tg != staged_tg) {
        if (tid < kSTG) {
          const int tk = __ldcg(a.ws.pair_tok + p0 + tg + min(tid, ng - 1));
          stok[tid] = tk;
          sqs[tid] = __ldcg(a.ws.qsum + tk);
          scx[tid] = __ldcg(a.ws.cx + tk);
        }
        if (SK3) {
          // per 16-byte chunk of a base-3 row (16 groups of 5 trits), digit-major (b3_qpos)
          for (int o = tid; o < ng * nv3 * 16; o += kSThreads) {
            const int t = o / (nv3 * 16), g = o - t * nv3 * 16;
            const int tk = __ldcg(a.ws.pair_tok + p0 + tg + t);
            const signed char* qt = reinterpret_cast<const signed char*>(a.ws.q) + (size_t)tk * d;
            char* c5 = qst + (t * nv3 + (g >> 4)) * kQChunk;
#pragma unroll
            for (int k = 0; k < 5; k++) c5[b3_qpos(g & 15, k)] = 5 * g + k < d ? (char)__ldcg(qt + 5 * g + k) : (char)0;
          }
        } else {
          for (int o = tid; o < ng * nv * 4; o += kSThreads) {
            const int t = o / (nv * 4), w = o - t * nv * 4;
            const int tk = __ldcg(a.ws.pair_tok + p0 + tg + t);
            *reinterpret_cast<uint4*>(qst + (t * nv + (w >> 2)) * kQChunk + (w & 3) * 16) =
                ld_cg4(reinterpret_cast<const uint4*>(a.ws.q + (size_t)tk * d) + w);
          }
        }
        staged_p0 = p0;
        staged_tg = tg;
        __syncthreads();
      }
      int ga[kSTG][4], ua[kSTG][4];
#pragma unroll
      for (int t = 0; t < kSTG; t++)
#pragma unroll
        for (int w = 0; w < 4; w++) ga[t][w] = ua[t][w] = 0;
      if (SK3 && ok && landed) {
        const uint4* g3 = reinterpret_cast<const uint4*>(stage + (size_t)lc * skrow);
        const uint4* u3 = reinterpret_cast<const uint4*>(stage + kSkBytes + (size_t)lc * skrow);
#pragma unroll 1
        for (int j = part; j < nv3; j += Geo::kParts) {
          uint32_t go[20], uo[20];
          b3_decode16(g3[j], go);
          b3_decode16(u3[j], uo);
#pragma unroll
          for (int t = 0; t < kSTG; t++) {
            if (t >= ng) break;
            uint32_t qd[20];
            b3_load_q(qst + (t * nv3 + j) * kQChunk, qd);
            ga[t][0] = b3_dot16(go, qd, ga[t][0]);
            ua[t][0] = b3_dot16(uo, qd, ua[t][0]);
          }
        }
      } else if (!SK3 && ok && landed) {
#pragma unroll 2
        for (int j = 0; j < nch; j++) {
          const int jr = (j + rot) & (nch - 1);
          const uint4 g4 = grow[jr], u4 = urow[jr];
          const char* qc = qst + (part * nch + jr) * kQChunk;
#pragma unroll
          for (int t = 0; t < kSTG; t++) {
            if (t >= ng) break;
            const uint4* qv = reinterpret_cast<const uint4*>(qc + t * nv * kQChunk);
            const uint4 q0 = qv[0], q1 = qv[1], q2 = qv[2], q3 = qv[3];
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
      }
      // sum over the channel's parts (adjacent lanes)
      int G[kSTG], U[kSTG];
#pragma unroll
      for (int t = 0; t < kSTG; t++) {
        G[t] = SK3 ? ga[t][0] : code_dot_total(ga[t]);
        U[t] = SK3 ? ua[t][0] : code_dot_total(ua[t]);
#pragma unroll
        for (int o = 1; o < Geo::kParts; o <<= 1) {
          G[t] += __shfl_xor_sync(kFullMask, G[t], o);
          U[t] += __shfl_xor_sync(kFullMask, U[t], o);
        }
      }
      if (ok && part < ng) {
        const int t = part;
        int g = G[0], uu = U[0];
#pragma unroll
        for (int tt = 1; tt < kSTG; tt++)
          if (t == tt) {
            g = G[tt];
            uu = U[tt];
          }
        const int i = i0 + lc, pr = p0 + tg + t;
        const int g2 = g - sqs[t], u2 = uu - sqs[t];
        const float gh = __fmul_rn(__fmul_rn((float)g2, alg[lc]), scx[t]);
        const float uh = __fmul_rn(__fmul_rn((float)u2, alu[lc]), scx[t]);
        const float ah = __fmul_rn(silu_r(gh), uh);
        a.ws.sa[(size_t)pr * I + i] = make_float2(fabsf(ah), ah);
        sah[t][lc] = ah;
        if (a.dbg_G || a.dbg_U || a.dbg_sigma) {
          const size_t off = ((size_t)stok[t] * a.top_e + __ldcg(a.ws.pair_slot + pr)) * I + i;
          if (a.dbg_G) a.dbg_G[off] = g2;
          if (a.dbg_U) a.dbg_U[off] = u2;
          if (a.dbg_sigma) a.dbg_sigma[off] = fabsf(ah);
        }
      }
      // recovery-input partial of the block: sum over its channels of
      // ahat_i Ubar_i; four adjacent lanes split the channels of one
      // (token, column) and meet in two shuffles
      if (r > 0) {
        __syncthreads();
        const int nq = ng * r * 4, per = Geo::kChannels / 4;
        for (int o0 = 0; o0 < nq; o0 += kSThreads) {
          const int o = o0 + tid, tp = o >> 2, q4 = o & 3;
          const int t = tp / r, p = tp - t * r;
          float z = 0.0f;
          if (o < nq && landed) {
            const int l1 = min(ncw, q4 * per + per);
            for (int l = q4 * per; l < l1; l++) z = fmaf(sah[t][l], bf16f(ubs[(size_t)l * r + p]), z);
          }
          z += __shfl_xor_sync(kFullMask, z, 1);
          z += __shfl_xor_sync(kFullMask, z, 2);
          if (o < nq && q4 == 0) a.ws.zpart[((size_t)(p0 + tg + t) * zstride + blk) * r + p] = z;
        }
      }
    }
    // every warp is done with this stage before the copy two units on reuses it
    __syncthreads();
    if (tid == 0) fence_proxy_async();
  }
}

// Shared memory of the selection kernels (one pair per CTA, 512 threads).
struct SelSmem {
  __align__(16) int hist[2 * 2048];
  __align__(16) uint32_t keys[kMaxI];
  __align__(16) int list[kMaxI];
  __align__(16) int misc[128];
  __align__(16) int scratch[128];
  __align__(16) uint32_t mk[64];
  __align__(16) uint32_t kw[64];
};

// -------------------------------------------------------------- top-c
// One pair per CTA: the c channels with the largest sigma (ties to the lower
// channel).  The last pair of an expert to finish ORs its expert's candidate
// masks into the union list the exact stage reads.
__global__ void __launch_bounds__(kSelT) select_c_kernel(ExpertArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ SelSmem sm;
  const int tid = threadIdx.x;
  const int I = a.I, W = (I + 31) >> 5;
  const int P = __ldcg(a.ws.act_off + __ldcg(a.ws.n_act));  // pairs of this step (this rank's, under EP)
#pragma unroll 1
  for (int p = blockIdx.x; p < P; p += gridDim.x) {
    const float* sp = reinterpret_cast<const float*>(a.ws.sa + (size_t)p * I);
    for (int i = tid; i < I; i += kSelT) sm.keys[i] = __float_as_uint(__ldcg(sp + 2 * i));  // sigma >= 0
    __syncthreads();
    sel::block_select_top(sm.keys, 1, I, a.c, sm.hist, sm.misc, sm.mk);
    for (int w = tid; w < W; w += kSelT) a.ws.candm[(size_t)p * W + w] = sm.mk[w];
    if (a.dbg_cand) {
      const int tok = __ldcg(a.ws.pair_tok + p), slot = __ldcg(a.ws.pair_slot + p);
      sel::block_mask_to_list(sm.mk, nullptr, I, a.dbg_cand + ((size_t)tok * a.top_e + slot) * a.c, &sm.misc[1],
                              sm.scratch);
    }
    const int ea = __ldcg(a.ws.pair_ea + p);
    const int p0 = __ldcg(a.ws.act_off + ea), m = __ldcg(a.ws.act_off + ea + 1) - p0;
    __syncthreads();  // the CTA's mask stores precede the release below
    if (tid == 0) sm.misc[0] = arrive_last(a.ws.arrive + ea, (unsigned)m);
    __syncthreads();
    if (sm.misc[0]) {
      for (int w = tid; w < W; w += kSelT) {
        uint32_t o = 0u;
        for (int q = 0; q < m; q++) o |= __ldcg(a.ws.candm + (size_t)(p0 + q) * W + w);
        sm.mk[w] = o;
      }
      __syncthreads();
      sel::block_mask_to_list(sm.mk, nullptr, I, a.ws.ulist + (size_t)ea * I, a.ws.n_u + ea, sm.scratch);
    }
    __syncthreads();
  }
}

// -------------------------------------------------------------- top-k
// One pair per CTA: the k candidates with the largest |a| (ties to the lower
// channel), then the recovery input z = sum over the block partials of
// ahat Ubar minus the part of the channels the down rows cover: -ahat_i Ubar_i
// for kept channels and, with the exact recovery input, -(ahat_i - a_i) Ubar_i
// for dropped candidates.  The last pair of an expert forms the kept union
// and the coefficient of every pair on each of its rows.
__global__ void __launch_bounds__(kSelT) select_k_kernel(ExpertArgs a, int nblk) {
  pdl_trigger();
  pdl_wait();
  __shared__ SelSmem sm;
  const int tid = threadIdx.x;
  const int I = a.I, W = (I + 31) >> 5, r = a.r;
  const int P = __ldcg(a.ws.act_off + __ldcg(a.ws.n_act));  // pairs of this step (this rank's, under EP)
  const int zstride = (I + 15) / 16;
  const bool rec_exact = a.recovery_input == 1;
#pragma unroll 1
  for (int p = blockIdx.x; p < P; p += gridDim.x) {
    const int ea = __ldcg(a.ws.pair_ea + p);
    const int e = __ldcg(a.ws.act_w + ea);  // weight slot of the pair's expert
    // the expert's Ubar block starts moving into L2 for the gather below
    if (tid == 0 && r > 0) bulk_prefetch_l2(a.u_sigma + (size_t)e * I * r, (uint32_t)(I * r * 2));
    for (int w = tid; w < W; w += kSelT) {
      sm.mk[w] = __ldcg(a.ws.candm + (size_t)p * W + w);
      sm.kw[w] = 0u;
    }
    __syncthreads();
    // candidate channels, ascending, and their keys |a|
    sel::block_mask_to_list(sm.mk, nullptr, I, sm.list, &sm.misc[1], sm.scratch);
    const int nc = sm.misc[1];
    const float* ap = a.ws.apos + (size_t)p * I;
    for (int j = tid; j < nc; j += kSelT) sm.keys[j] = __float_as_uint(fabsf(__ldcg(ap + sm.list[j])));
    __syncthreads();
    sel::block_select_top(sm.keys, 1, nc, a.k, sm.hist, sm.misc, sm.mk);  // mk: kept positions
    for (int j = tid; j < nc; j += kSelT)
      if ((sm.mk[j >> 5] >> (j & 31)) & 1u) atomicOr(&sm.kw[sm.list[j] >> 5], 1u << (sm.list[j] & 31));
    __syncthreads();
    for (int w = tid; w < W; w += kSelT) a.ws.keptm[(size_t)p * W + w] = sm.kw[w];
    if (a.dbg_kept) {
      // kept channels ascending: the kept positions in order
      int* klist = reinterpret_cast<int*>(sm.keys);
      sel::block_mask_to_list(sm.mk, nullptr, nc, klist, &sm.misc[2], sm.scratch);
      const int tok = __ldcg(a.ws.pair_tok + p), slot = __ldcg(a.ws.pair_slot + p);
      const size_t off = ((size_t)tok * a.top_e + slot) * a.k;
      for (int t = tid; t < a.k && t < sm.misc[2]; t += kSelT) {
        const int i = sm.list[klist[t]];
        a.dbg_kept[off + t] = i;
        if (a.dbg_a_kept) a.dbg_a_kept[off + t] = __ldcg(ap + i);
      }
      __syncthreads();
    }
    if (r > 0) {
      // coefficient of each candidate position (0 where its Ubar row does not
      // enter), then thread (jl, c) sums coefficient x Ubar chunk c (8 entries)
      // over positions jl, jl + nj, ...; the partials meet in the (free)
      // selection histogram in a fixed order
      float* co = reinterpret_cast<float*>(sm.keys);
      const float* sap = reinterpret_cast<const float*>(a.ws.sa + (size_t)p * I);
      for (int j = tid; j < nc; j += kSelT) {
        const bool kept = (sm.mk[j >> 5] >> (j & 31)) & 1u;
        const int i = sm.list[j];
        float v = 0.0f;
        if (kept || rec_exact) {
          const float ah = __ldcg(sap + 2 * i + 1);
          v = kept ? ah : __fsub_rn(ah, __ldcg(ap + i));
        }
        co[j] = v;
      }
      __syncthreads();
      const int nchk = r / 8, nj = kSelT / nchk;
      const int c = tid % nchk, jl = tid / nchk;
      float acc[8];
#pragma unroll
      for (int h = 0; h < 8; h++) acc[h] = 0.0f;
      if (jl < nj) {
        const uint16_t* ub = a.u_sigma + (size_t)e * I * r + 8 * c;
#pragma unroll 4
        for (int j = jl; j < nc; j += nj) {
          const float cj = co[j];
          if (cj == 0.0f) continue;
          float f[8];
          bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(ub + (size_t)sm.list[j] * r)), f);
#pragma unroll
          for (int h = 0; h < 8; h++) acc[h] = fmaf(cj, f[h], acc[h]);
        }
      }
      float* zs = reinterpret_cast<float*>(sm.hist);  // [nj][r]
      if (jl < nj)
#pragma unroll
        for (int h = 0; h < 8; h++) zs[jl * r + 8 * c + h] = acc[h];
      __syncthreads();
      if (tid < r) {
        float s0 = 0.0f, s1 = 0.0f;
        for (int q = 0; q < nj; q++) s0 += zs[q * r + tid];
        // the screen blocks' partials: independent loads, eight in flight
        const float* zp = a.ws.zpart + (size_t)p * zstride * r + tid;
        float zb[8];
#pragma unroll
        for (int h = 0; h < 8; h++) zb[h] = 0.0f;
        int b = 0;
        for (; b + 8 <= nblk; b += 8)
#pragma unroll
          for (int h = 0; h < 8; h++) zb[h] += __ldcg(zp + (size_t)(b + h) * r);
        for (; b < nblk; b++) zb[0] += __ldcg(zp + (size_t)b * r);
        s1 = ((zb[0] + zb[1]) + (zb[2] + zb[3])) + ((zb[4] + zb[5]) + (zb[6] + zb[7]));
        a.ws.z[(size_t)p * r + tid] = s1 - s0;
      }
    }
    // the expert's last pair: kept union and row coefficients
    const int p0 = __ldcg(a.ws.act_off + ea), m = __ldcg(a.ws.act_off + ea + 1) - p0;
    __syncthreads();
    if (tid == 0) sm.misc[0] = arrive_last(a.ws.arrive + a.E + ea, (unsigned)m);
    __syncthreads();
    if (sm.misc[0]) {
      for (int w = tid; w < W; w += kSelT) {
        uint32_t o = 0u;
        for (int q = 0; q < m; q++) o |= __ldcg(a.ws.keptm + (size_t)(p0 + q) * W + w);
        sm.kw[w] = o;
      }
      __syncthreads();
      int* dl = a.ws.dlist + (size_t)ea * I;
      sel::block_mask_to_list(sm.kw, nullptr, I, sm.list, &sm.misc[3], sm.scratch);
      const int nd = sm.misc[3];
      for (int u = tid; u < nd; u += kSelT) dl[u] = sm.list[u];
      if (tid == 0) a.ws.n_d[ea] = nd;
      for (int o = tid; o < m * nd; o += kSelT) {
        const int q = o / nd, u = o - q * nd, i = sm.list[u];
        const bool kept = (__ldcg(a.ws.keptm + (size_t)(p0 + q) * W + (i >> 5)) >> (i & 31)) & 1u;
        a.ws.coef[(size_t)(p0 + q) * I + u] = kept ? __ldcg(a.ws.apos + (size_t)(p0 + q) * I + i) : 0.0f;
      }
    }
    __syncthreads();
  }
}

// bf16 m16n8k16 tensor-core product, fp32 accumulate: c += A B.
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Expert of unit u: cu holds the exclusive prefix of units per active expert.
__device__ __forceinline__ int unit_expert(const int* cu, int n_act, int u) {
  int lo = 0, hi = n_act;  // cu[lo] <= u < cu[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= u) lo = mid;
    else hi = mid;
  }
  return lo;
}

// ------------------------------------------------------- exact candidates
// g = W_gate[e] x and u = W_up[e] x for kXRows rows of the expert's
// candidate union and up to 16 of its tokens per pass, on the tensor cores:
// D[token][row] += X[token][k] W[row][k] with tokens as M (16, zero-padded),
// rows as N (one 8-row tile per warp) and d as K, bf16 products summed in
// fp32.  The order of the K sum is free, so each thread loads 16 contiguous
// bytes of its row (and of its token from shared memory) and uses them as the
// fragments of two k-steps (both operands permuted alike).  Warp w takes tile
// w % 2 and the K slice w / 2 (one eighth of d); the slices' partial sums meet
// in shared memory.  Each CTA takes a contiguous range of units and prefetches
// the next unit's rows into L2 while it computes.
constexpr int kXThreads = 512, kXWarps = kXThreads / 32, kXRows = 16, kXTok = 16;

__global__ void __launch_bounds__(kXThreads, 1) exact_kernel(ExpertArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) char xsm[];  // [kXTok][2 d + 64] bf16 tokens (padded rows)
  __shared__ int cu[kMaxAct + 1];
  __shared__ int tw[kMaxAct], toff[kMaxAct + 1], tnu[kMaxAct];
  __shared__ int srow3[3][kXRows];
  __shared__ __align__(16) float red[2][kXWarps / 2][32][8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int tile = warp & 1, kq = warp >> 1;
  const int gid = lane >> 2, tig = lane & 3;
  const int I = a.I, d = a.d, W = (I + 31) >> 5;
  const int xstride = 2 * d + 64;                // bytes; rows land 16 banks apart
  const int kslice = d / 8, nkb = kslice / 32;   // elements and 32-element blocks per warp
  const int n_act = __ldcg(a.ws.n_act);
  if (warp == 0) {
    int run = 0;
    for (int b0 = 0; b0 < n_act; b0 += 32) {
      const int ea = b0 + lane;
      const int c = ea < n_act ? (__ldcg(a.ws.n_u + ea) + kXRows - 1) / kXRows : 0;
      int inc = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFullMask, inc, o);
        if (lane >= o) inc += v;
      }
      if (ea < n_act) cu[ea] = run + inc - c;
      run += __shfl_sync(kFullMask, inc, 31);
    }
    if (lane == 0) cu[n_act] = run;
  }
  // per active expert, read once: weight slot, first pair, candidate-union size
  for (int ea = tid; ea < n_act; ea += kXThreads) {
    tw[ea] = __ldcg(a.ws.act_w + ea);
    toff[ea] = __ldcg(a.ws.act_off + ea);
    tnu[ea] = __ldcg(a.ws.n_u + ea);
  }
  if (tid == 0) toff[n_act] = __ldcg(a.ws.act_off + n_act);
  __syncthreads();
  const int total = cu[n_act];
  const int ub = (int)((long long)total * blockIdx.x / gridDim.x);
  const int ue = (int)((long long)total * (blockIdx.x + 1) / gridDim.x);
  // row `lane16` of unit un (-1 past the expert's union) and its L2 prefetch
  auto unit_row = [&](int un, int l16) {
    const int ean = unit_expert(cu, n_act, un);
    const int jn = (un - cu[ean]) * kXRows + l16;
    return jn < tnu[ean] ? __ldcg(a.ws.ulist + (size_t)ean * I + jn) : -1;
  };
  auto prefetch_row = [&](int un, int row) {
    if (row < 0) return;
    const size_t g = (size_t)tw[unit_expert(cu, n_act, un)] * I + row;
    bulk_prefetch_l2(a.w_gate + g * d, 2 * d);
    bulk_prefetch_l2(a.w_up + g * d, 2 * d);
  };
  // the rows of units u .. u + 2 sit in a ring of three; the first two now
  if (tid < kXRows)
    for (int un = ub; un < ub + 2 && un < ue; un++) {
      const int rw = unit_row(un, tid);
      srow3[un % 3][tid] = rw;
      prefetch_row(un, rw);
    }
  int staged_ea = -1, staged_mt = -1;
#pragma unroll 1
  for (int u = ub; u < ue; u++) {
    const int ea = unit_expert(cu, n_act, u);
    const int e = tw[ea], p0 = toff[ea];  // e: weight slot
    const int m = toff[ea + 1] - p0;
    const int j0 = (u - cu[ea]) * kXRows;
    const int nrows = min(kXRows, tnu[ea] - j0);
    const int* srow = srow3[u % 3];
    // the rows of the unit two on: loaded while this one is computed, then
    // stored into the ring and started into L2
    int row2 = -1;
    if (tid < kXRows && u + 2 < ue) row2 = unit_row(u + 2, tid);
    __syncthreads();  // the previous unit is done with xsm and red (and the ring slots are written)
#pragma unroll 1
    for (int mt = 0; mt < m; mt += kXTok) {
      const int nt = min(kXTok, m - mt);
      if (mt > 0) __syncthreads();  // the previous pass's epilogue is done with red
      if (ea != staged_ea || mt != staged_mt) {
        const int d8 = d >> 3;
        for (int o = tid; o < nt * d8; o += kXThreads) {
          const int t = o / d8, j8 = o - t * d8;
          const int tok = __ldcg(a.ws.pair_tok + p0 + mt + t);
          *reinterpret_cast<uint4*>(xsm + (size_t)t * xstride + 16 * j8) =
              __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)tok * d) + j8);
        }
        staged_ea = ea;
        staged_mt = mt;
      }
      __syncthreads();
      // the epilogue's candidate-mask words, in flight during the products
      uint32_t cmw[4] = {0u, 0u, 0u, 0u};
      if (kq == 0)
#pragma unroll
        for (int h = 0; h < 4; h++) {
          const int tl = gid + (h >= 2 ? 8 : 0), rl = tile * 8 + tig * 2 + (h & 1);
          if (tl < nt && rl < nrows)
            cmw[h] = __ldcg(a.ws.candm + (size_t)(p0 + mt + tl) * W + (srow[rl] >> 5));
        }
      const int rowi = srow[tile * 8 + gid];
      const uint4* gr = reinterpret_cast<const uint4*>(a.w_gate + ((size_t)e * I + max(rowi, 0)) * d);
      const uint4* ur = reinterpret_cast<const uint4*>(a.w_up + ((size_t)e * I + max(rowi, 0)) * d);
      const char* xa_p = xsm + (size_t)gid * xstride;
      const char* xb_p = xsm + (size_t)(gid + 8) * xstride;
      float cg[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
      for (int kb0 = 0; kb0 < nkb; kb0 += 8) {
        uint4 wg[8], wu[8];
#pragma unroll
        for (int j = 0; j < 8; j++) {
          const int kel = kq * kslice + (kb0 + j) * 32 + tig * 8;
          const bool ok = kb0 + j < nkb && rowi >= 0;
          wg[j] = ok ? ld_stream(gr + kel / 8) : make_uint4(0u, 0u, 0u, 0u);
          wu[j] = ok ? ld_stream(ur + kel / 8) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < 8; j++) {
          if (kb0 + j >= nkb) break;
          const int kel = kq * kslice + (kb0 + j) * 32 + tig * 8;
          const uint4 xa = gid < nt ? *reinterpret_cast<const uint4*>(xa_p + 2 * kel) : make_uint4(0u, 0u, 0u, 0u);
          const uint4 xb =
              gid + 8 < nt ? *reinterpret_cast<const uint4*>(xb_p + 2 * kel) : make_uint4(0u, 0u, 0u, 0u);
          mma16816(cg, xa.x, xb.x, xa.y, xb.y, wg[j].x, wg[j].y);
          mma16816(cv, xa.x, xb.x, xa.y, xb.y, wu[j].x, wu[j].y);
          mma16816(cg, xa.z, xb.z, xa.w, xb.w, wg[j].z, wg[j].w);
          mma16816(cv, xa.z, xb.z, xa.w, xb.w, wu[j].z, wu[j].w);
        }
      }
      float4* rp = reinterpret_cast<float4*>(&red[tile][kq][lane][0]);
      rp[0] = make_float4(cg[0], cg[1], cg[2], cg[3]);
      rp[1] = make_float4(cv[0], cv[1], cv[2], cv[3]);
      __syncthreads();
      if (kq == 0) {
        float sg[4] = {0.0f, 0.0f, 0.0f, 0.0f}, su[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int q = 0; q < kXWarps / 2; q++) {
          const float4 pg = *reinterpret_cast<const float4*>(&red[tile][q][lane][0]);
          const float4 pu = *reinterpret_cast<const float4*>(&red[tile][q][lane][4]);
          sg[0] += pg.x;
          sg[1] += pg.y;
          sg[2] += pg.z;
          sg[3] += pg.w;
          su[0] += pu.x;
          su[1] += pu.y;
          su[2] += pu.z;
          su[3] += pu.w;
        }
        // element h: token gid (+ 8 for h >= 2), tile row tig * 2 + (h & 1)
#pragma unroll
        for (int h = 0; h < 4; h++) {
          const int tl = gid + (h >= 2 ? 8 : 0), rl = tile * 8 + tig * 2 + (h & 1);
          if (tl < nt && rl < nrows) {
            const int i = srow[rl], pr = p0 + mt + tl;
            if ((cmw[h] >> (i & 31)) & 1u) a.ws.apos[(size_t)pr * I + i] = __fmul_rn(silu_r(sg[h]), su[h]);
          }
        }
      }
    }
    if (tid < kXRows && u + 2 < ue) {
      srow3[(u + 2) % 3][tid] = row2;
      prefetch_row(u + 2, row2);
    }
  }
}

// ------------------------------------------------ down rows + combine
// Unit = (active expert, column slice of SW columns).  Thread (g, q) takes
// the 16-byte chunk q of the slice in kept-union rows g, g + G, ...; each
// row enters every token of the expert with its coefficient (a if the token
// kept the channel, else 0).  Then y_e = (row sum) + V z per (token, column),
// written to the step's per-slot outputs; the last of a token's top-e slots
// to arrive for a slice combines them in slot order (fp32 FMAs, plus the
// residual) into bf16.
template <int SW>
__global__ void __launch_bounds__(kDThreads) down_kernel(ExpertArgs a) {
  pdl_trigger();
  pdl_wait();
  constexpr int QW = SW / 8, G = kDThreads / QW, CR = 16 * G;  // CR: rows staged per chunk (16 per thread)
  static_assert(CR <= kDRows, "row chunk exceeds the staging arrays");
  __shared__ __align__(16) float red[G][kDTG][SW];
  __shared__ int sidx[kDRows];
  __shared__ float scoef[kDTG][kDRows];
  __shared__ int lastf[kDTG];
  const int tid = threadIdx.x;
  const int I = a.I, d = a.d, r = a.r, ns = d / SW, d8 = d >> 3;
  const int g = tid / QW, q = tid - g * QW;
  const int n_act = __ldcg(a.ws.n_act);
  const int units = n_act * ns;
  // units are dealt round-robin: the column slices of one expert's rows are
  // read by different CTAs at about the same time, whole rows at once (one
  // CTA taking a contiguous range of slices measured slower)
  int staged_ea = -1, staged_tg = -1, staged_r0 = -1, cur_ea = -1;
  __shared__ int se[4];  // the current expert: weight slot, first pair, last pair + 1, kept-union size
#pragma unroll 1
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int ea = u / ns, sl = u - ea * ns, j0 = sl * SW;
    if (ea != cur_ea) {
      __syncthreads();  // every thread is done with the previous expert's scalars
      if (tid == 0) {
        const int w = __ldcg(a.ws.act_w + ea), o0 = __ldcg(a.ws.act_off + ea), o1 = __ldcg(a.ws.act_off + ea + 1),
                  n = __ldcg(a.ws.n_d + ea);
        se[0] = w;
        se[1] = o0;
        se[2] = o1;
        se[3] = n;
      }
      __syncthreads();
      cur_ea = ea;
    }
    const int e = se[0], p0 = se[1];  // e: weight slot
    const int m = se[2] - p0, nd = se[3];
    const int* dl = a.ws.dlist + (size_t)ea * I;
    // this slice's V rows start moving into L2 for the epilogue below
    if (tid == 0 && r > 0) bulk_prefetch_l2(a.v + ((size_t)e * d + j0) * r, (uint32_t)(SW * r * 2));
    const uint4* wd = reinterpret_cast<const uint4*>(a.w_down + (size_t)e * I * d + j0) + q;
#pragma unroll 1
    for (int tg = 0; tg < m; tg += kDTG) {
      const int ng = min(kDTG, m - tg);
      float acc[kDTG][8];
#pragma unroll
      for (int t = 0; t < kDTG; t++)
#pragma unroll
        for (int c = 0; c < 8; c++) acc[t][c] = 0.0f;
      const float* cf = a.ws.coef + (size_t)(p0 + tg) * I;
#pragma unroll 1
      for (int r0 = 0; r0 < nd; r0 += CR) {
        // the chunk's row indices and coefficients, staged once for all threads
        const int nr = min(CR, nd - r0);
        if (ea != staged_ea || tg != staged_tg || r0 != staged_r0) {
          __syncthreads();
          for (int o = tid; o < nr; o += kDThreads) sidx[o] = __ldcg(dl + r0 + o);
          for (int o = tid; o < kDTG * nr; o += kDThreads) {
            const int t = o / nr, rr = o - t * nr;
            scoef[t][rr] = t < ng ? __ldcg(cf + (size_t)t * I + r0 + rr) : 0.0f;
          }
          staged_ea = ea;
          staged_tg = tg;
          staged_r0 = r0;
          __syncthreads();
        }
        // every row of the chunk this thread takes, all loads in flight together
        uint4 w[16];
#pragma unroll
        for (int k = 0; k < 16; k++) {
          const int mr = g + k * G;
          w[k] = mr < nr ? ld_stream(wd + (size_t)sidx[mr] * d8) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < 16; k++) {
          const int mr = g + k * G;
          if (mr >= nr) break;
          float f[8];
          bf16x8_to_f32(w[k], f);
#pragma unroll
          for (int t = 0; t < kDTG; t++) {
            const float co = scoef[t][mr];
#pragma unroll
            for (int c = 0; c < 8; c++) acc[t][c] = fmaf(co, f[c], acc[t][c]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kDTG; t++) {
        float4* dst = reinterpret_cast<float4*>(&red[g][t][8 * q]);
        dst[0] = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
        dst[1] = make_float4(acc[t][4], acc[t][5], acc[t][6], acc[t][7]);
      }
      __syncthreads();
      for (int o = tid; o < ng * SW; o += kDThreads) {
        const int t = o / SW, col = o - t * SW;
        float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
        for (int gg = 0; gg < G; gg += 2) {
          s0 += red[gg][t][col];
          s1 += red[gg + 1][t][col];
        }
        float y = s0 + s1;
        const int pr = p0 + tg + t;
        if (r > 0) {
          const uint16_t* vr = a.v + ((size_t)e * d + j0 + col) * r;
          const float* zp = a.ws.z + (size_t)pr * r;
          float r0 = 0.0f, r1 = 0.0f;
#pragma unroll 4
          for (int k = 0; k < r; k += 8) {
            const uint4 v8 = __ldg(reinterpret_cast<const uint4*>(vr + k));
            const float4 za = __ldcg(reinterpret_cast<const float4*>(zp + k));
            const float4 zb = __ldcg(reinterpret_cast<const float4*>(zp + k + 4));
            r0 = fmaf(bf16lo(v8.x), za.x, r0);
            r1 = fmaf(bf16hi(v8.x), za.y, r1);
            r0 = fmaf(bf16lo(v8.y), za.z, r0);
            r1 = fmaf(bf16hi(v8.y), za.w, r1);
            r0 = fmaf(bf16lo(v8.z), zb.x, r0);
            r1 = fmaf(bf16hi(v8.z), zb.y, r1);
            r0 = fmaf(bf16lo(v8.w), zb.z, r0);
            r1 = fmaf(bf16hi(v8.w), zb.w, r1);
          }
          y += r0 + r1;
        }
        const int tok = __ldcg(a.ws.pair_tok + pr), slot = __ldcg(a.ws.pair_slot + pr);
        const size_t off = ((size_t)tok * a.top_e + slot) * d + j0 + col;
        a.ws.ye[off] = y;
        if (a.dbg_y_expert) a.dbg_y_expert[off] = y;
      }
      __syncthreads();  // the CTA's outputs precede the releases below
      if (a.ep_partial) continue;  // expert-parallel step: the per-slot outputs are the result
      if (tid < ng) {
        const int tok = __ldcg(a.ws.pair_tok + p0 + tg + tid);
        lastf[tid] = arrive_last(a.ws.counters + tok * kMaxCluster + sl, (unsigned)a.top_e);
      }
      __syncthreads();
#pragma unroll 1
      for (int t = 0; t < ng; t++) {
        if (!lastf[t]) continue;
        const int tok = __ldcg(a.ws.pair_tok + p0 + tg + t);
        for (int col = tid; col < SW; col += kDThreads) {
          const int j = j0 + col;
          float acc2 = 0.0f;
          for (int s = 0; s < a.top_e; s++)
            acc2 = fmaf(__ldcg(a.ws.wts + tok * a.top_e + s), __ldcg(a.ws.ye + ((size_t)tok * a.top_e + s) * d + j),
                        acc2);
          if (a.residual) acc2 += bf16f(a.residual[(size_t)tok * d + j]);
          a.y[(size_t)tok * d + j] = f2bf16(acc2);
        }
        if (tid == 0) a.ws.counters[tok * kMaxCluster + sl] = 0u;
      }
      __syncthreads();
    }
  }
}

// Resident CTAs per SM of each kernel, per device (queried once).
struct Occupancy {
  int dev = -1, sms = 0;
  int screen1 = 0, screen2 = 0, screen1b3 = 0, screen2b3 = 0, selc = 0, selk = 0, exact = 0, down128 = 0,
      down256 = 0;
};
thread_local Occupancy g_occ;  // per calling thread: occupancies on its current device

// Also raises the kernel's dynamic shared-memory limit to `smem`.
template <class K>
int occ(K kernel, int threads, size_t smem) {
  int n = 0;
  if (smem > 48 * 1024) cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess) n = 1;
  return n > 0 ? n : 1;
}

template <class K, class... Args>
cudaError_t launch_pdl(K kernel, int grid, int threads, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid > 0 ? grid : 1);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

size_t exact_smem(int d) { return (size_t)kXTok * (2 * d + 64); }

// ------------------------------------------------- expert parallelism
// y_partial[b][j] = sum over b's slots s whose expert this rank owns of
// w[b][s] y_e[b][s][j], fp32 FMAs in slot order.
__global__ void __launch_bounds__(256) ep_combine_kernel(int B, int top_e, int d, int ep_rank, int ep_size,
                                                         Workspace ws, float* y_partial) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.y, j = blockIdx.x * 256 + threadIdx.x;
  if (j >= d) return;
  float acc = 0.0f;
  for (int s = 0; s < top_e; s++) {
    const int e = __ldcg(ws.ids + b * top_e + s);
    if (e % ep_size != ep_rank) continue;
    acc = fmaf(__ldcg(ws.wts + b * top_e + s), __ldcg(ws.ye + ((size_t)b * top_e + s) * d + j), acc);
  }
  y_partial[(size_t)b * d + j] = acc;
}

// y = bf16(y_sum + residual) after the ranks' partials are summed.
__global__ void __launch_bounds__(256) ep_finish_kernel(int B, int d, const float* y_sum, const uint16_t* residual,
                                                        uint16_t* y) {
  const size_t o = (size_t)blockIdx.x * 256 + threadIdx.x;
  if (o >= (size_t)B * d) return;
  float v = y_sum[o];
  if (residual) v += bf16f(residual[o]);
  y[o] = f2bf16(v);
}

}  // namespace

cudaError_t launch_ep_combine(int B, int top_e, int d, int ep_rank, int ep_size, const Workspace& ws,
                              float* y_partial, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((d + 255) / 256, B);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, ep_combine_kernel, B, top_e, d, ep_rank, ep_size, ws, y_partial);
}

cudaError_t launch_ep_finish(int B, int d, const float* y_sum, const uint16_t* residual, uint16_t* y,
                             cudaStream_t s) {
  const size_t n = (size_t)B * d;
  ep_finish_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(B, d, y_sum, residual, y);
  return cudaGetLastError();
}


cudaError_t launch_stream(const ExpertArgs& a, cudaStream_t s) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (g_occ.dev != dev) {
    Occupancy o;
    o.dev = dev;
    err = cudaDeviceGetAttribute(&o.sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    o.exact = occ(exact_kernel, kXThreads, exact_smem(4096));  // the largest staging; sets the limit
    o.screen1 = occ(screen_kernel<1, false>, kSThreads, 2 * kSStageBytes);
    o.screen2 = occ(screen_kernel<2, false>, kSThreads, 2 * kSStageBytes);
    o.screen1b3 = occ(screen_kernel<1, true>, kSThreads, 2 * kSStageBytes);
    o.screen2b3 = occ(screen_kernel<2, true>, kSThreads, 2 * kSStageBytes);
    o.selc = occ(select_c_kernel, kSelT, 0);
    o.selk = occ(select_k_kernel, kSelT, 0);
    o.down128 = occ(down_kernel<128>, kDThreads, 0);
    o.down256 = occ(down_kernel<256>, kDThreads, 0);
    g_occ = o;
  }
  const int P = a.B * a.top_e, nact = a.E < P ? a.E : P;
  const int sms = g_occ.sms;
  // screen
  const int nvl = a.d <= 2048 ? 1 : 2;
  const int chans = nvl == 1 ? ScreenGeom<1>::kChannels : ScreenGeom<2>::kChannels;
  const int nblk = (a.I + chans - 1) / chans;
  const int socc = a.sk3 ? (nvl == 1 ? g_occ.screen1b3 : g_occ.screen2b3) : (nvl == 1 ? g_occ.screen1 : g_occ.screen2);
  const int gs = nact * nblk < sms * socc ? nact * nblk : sms * socc;
  if (a.sk3)
    err = nvl == 1 ? launch_pdl(screen_kernel<1, true>, gs, kSThreads, 2 * kSStageBytes, s, a)
                   : launch_pdl(screen_kernel<2, true>, gs, kSThreads, 2 * kSStageBytes, s, a);
  else
    err = nvl == 1 ? launch_pdl(screen_kernel<1, false>, gs, kSThreads, 2 * kSStageBytes, s, a)
                   : launch_pdl(screen_kernel<2, false>, gs, kSThreads, 2 * kSStageBytes, s, a);
  if (err != cudaSuccess) return err;
  // top-c
  err = launch_pdl(select_c_kernel, P < sms * g_occ.selc ? P : sms * g_occ.selc, kSelT, 0, s, a);
  if (err != cudaSuccess) return err;
  // exact candidates
  err = launch_pdl(exact_kernel, sms * g_occ.exact, kXThreads, exact_smem(a.d), s, a);
  if (err != cudaSuccess) return err;
  // top-k
  err = launch_pdl(select_k_kernel, P < sms * g_occ.selk ? P : sms * g_occ.selk, kSelT, 0, s, a, nblk);
  if (err != cudaSuccess) return err;
  // down rows + combine
  if (a.d <= 2048) {
    const int ns = a.d / 128, gd = nact * ns < sms * g_occ.down128 ? nact * ns : sms * g_occ.down128;
    return launch_pdl(down_kernel<128>, gd, kDThreads, 0, s, a);
  }
  const int ns = a.d / 256, gd = nact * ns < sms * g_occ.down256 ? nact * ns : sms * g_occ.down256;
  return launch_pdl(down_kernel<256>, gd, kDThreads, 0, s, a);
}

}  // namespace moe
