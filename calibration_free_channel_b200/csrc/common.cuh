// common.cuh -- device helpers shared by the reader's kernels (sm_100a).
#pragma once
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;          // threads per CTA of the route kernel
constexpr int kWarps = kThreads / 32;
constexpr int kMaxSlots = 16;          // row slots per warp in the copy rings
constexpr int kMaxGroup = 2;           // tokens per work item (tokens sharing an expert)
constexpr int kMaxCluster = 16;
constexpr int kMaxTokens = 256;        // tokens per step (B)

// Error word bits (workspace), set by bounded waits that ran out.
constexpr uint32_t kErrCopyTimeout = 1u;
constexpr uint32_t kErrBadWorkItem = 2u;
constexpr uint32_t kErrNoWeights = 4u;     // an active expert has no weight slot (expert_slot[e] < 0)
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// ------------------------------------------------------------------ bf16
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
// fp32 -> bf16, round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f2bf16(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)((u >> 16) | ((u & 0xffff) ? 0x40 : 0));
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// ------------------------------------------------------------ exp / SiLU
// exp_r: Cody & Waite reduction t = n ln2 + r (ln 2 split into a
// 16-significant-bit head and an fp32 tail), degree-7 Taylor polynomial of
// exp(r) in Horner form with correctly rounded FMAs, exact scale by 2^n.
// Input clamped to [-87, 88] so the result is a normal float.  Every step is
// a single correctly rounded operation, so the host reference computes the
// same bits.
__device__ __forceinline__ float exp_r(float t) {
  const float kLog2e = 0x1.715476p+0f;
  const float kLn2Hi = 0x1.62e4p-1f;
  const float kLn2Lo = 0x1.7f7d1cp-20f;
  t = fminf(fmaxf(t, -87.0f), 88.0f);
  const float n = rintf(__fmul_rn(t, kLog2e));
  float r = __fmaf_rn(-n, kLn2Hi, t);
  r = __fmaf_rn(-n, kLn2Lo, r);
  float p = 0x1.a01a02p-13f;             // 1/7!
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);  // 1/6!
  p = __fmaf_rn(p, r, 0x1.111112p-7f);   // 1/5!
  p = __fmaf_rn(p, r, 0x1.555556p-5f);   // 1/4!
  p = __fmaf_rn(p, r, 0x1.555556p-3f);   // 1/3!
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const float two_n = __uint_as_float((uint32_t)((int)n + 127) << 23);
  return __fmul_rn(p, two_n);
}

__device__ __forceinline__ float silu_r(float t) {
  return __fdiv_rn(t, __fadd_rn(1.0f, exp_r(-t)));
}

// ------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// try_wait with a suspend-time hint: the warp sleeps until the phase
// completes (or the hint elapses) instead of spinning.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}
// Non-blocking test of an mbarrier phase (a few tens of cycles; try_wait costs
// about four times as much even on a completed phase).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on an mbarrier phase.  Returns false (and sets *err) if the
// phase did not complete within limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t* err,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_test_wait(bar, parity)) return true;
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) {
      atomicOr(err, kErrCopyTimeout);
      return false;
    }
  }
}
// Raises the transaction count of the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx_only(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// L2 policy of the streamed weights: evict first.  A decode step reads each
// weight byte once, and far more of them than the L2 holds; marking them
// first to go keeps the lines that are reused from launch to launch (the
// kernels' code, the per-step tables) resident instead.
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// 16-byte load of streamed weights: read-only, not kept in L1, evict-first
// in L2.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p), "l"(evict_first_policy()));
  return v;
}
// Bulk prefetch of [src, src + bytes) into L2 (16-byte aligned, multiple of 16).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;" ::"l"(src), "r"(bytes),
               "l"(evict_first_policy())
               : "memory");
}
// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`
// (weights: evict-first in L2).  dst, src 16-byte aligned; bytes a multiple
// of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(evict_first_policy())
      : "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- reductions
template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Ternary-sketch dot of one packed row word with 16 int8 activations.
// Word layout: position 4p + b (p, b in 0..3) at bits [8b + 2p, 8b + 2p + 1]
// as the code T + 1 (0, 1 or 2).  Masking the word with 0x03030303 << 2p
// leaves the codes of positions 4p .. 4p+3 in four bytes, scaled by 4^p;
// dp4a multiplies them with the activation bytes exactly.  The four partial
// sums are kept apart (acc[p] is a multiple of 4^p) and combined by
// code_dot_total; the row's code offset is removed by subtracting the sum of
// the activations once per row.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ void code_dot16(uint32_t w, uint4 q, int (&acc)[4]) {
  acc[0] = dp4a_us(w & 0x03030303u, q.x, acc[0]);
  acc[1] = dp4a_us(w & 0x0c0c0c0cu, q.y, acc[1]);
  acc[2] = dp4a_us(w & 0x30303030u, q.z, acc[2]);
  acc[3] = dp4a_us(w & 0xc0c0c0c0u, q.w, acc[3]);
}
__device__ __forceinline__ int code_dot_total(const int (&acc)[4]) {
  return acc[0] + (acc[1] >> 2) + (acc[2] >> 4) + (acc[3] >> 6);
}

// ------------------------------------------------- base-3 sketch rows
// Five trits per byte: byte g of a row holds trits 5g .. 5g+4 as
// sum_i (t_{5g+i} + 1) 3^i (at most 242).  A row of d trits takes
// ceil(d / 5) bytes; it is padded to whole 32-byte sectors with bytes of
// five zero trits (121), so rows stay 16-byte aligned for bulk copies.
//
// Decoding is plain integer arithmetic on four bytes at once: the bytes sit
// in two registers as 16-bit lanes (bytes 0 and 2, bytes 1 and 3), and
// floor(b / 3^k) comes from one multiply and shift per lane pair
// (b * 171 >> 9, b * 57 >> 9, b * 19 >> 9, b * 203 >> 14 are exact for
// b <= 242 and stay inside 16 bits), so digit k = floor(b / 3^k) -
// 3 floor(b / 3^(k+1)).  The digits come out digit-major: word k holds
// digit k (the code t + 1 of trit 5g + k) of the four bytes, one per byte,
// ready for dp4a against the activations staged the same way:
// qd[5w + k] = (q[5(4w + b) + k], b = 0..3) for the bytes 4w .. 4w+3 of a
// 16-byte chunk (w = 0..3; 80 bytes per chunk).
__host__ __device__ inline int sk3_row_bytes(int d) { return ((d + 4) / 5 + 31) / 32 * 32; }
__device__ __forceinline__ void b3_digits2(uint32_t R, uint32_t (&dg)[5]) {
  const uint32_t f1 = ((R * 171u) >> 9) & 0x007f007fu;   // floor(b / 3)
  const uint32_t f2 = ((R * 57u) >> 9) & 0x001f001fu;    // floor(b / 9)
  const uint32_t f3 = ((R * 19u) >> 9) & 0x000f000fu;    // floor(b / 27)
  const uint32_t f4 = ((R * 203u) >> 14) & 0x00030003u;  // floor(b / 81)
  dg[0] = R - 3u * f1;
  dg[1] = f1 - 3u * f2;
  dg[2] = f2 - 3u * f3;
  dg[3] = f3 - 3u * f4;
  dg[4] = f4;
}
// The codes of one 16-byte chunk (80 trits), digit-major: o[5w + k].
__device__ __forceinline__ void b3_decode16(uint4 s, uint32_t (&o)[20]) {
  const uint32_t sw[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
  for (int w = 0; w < 4; w++) {
    uint32_t dx[5], dy[5];
    b3_digits2(sw[w] & 0x00ff00ffu, dx);
    b3_digits2((sw[w] >> 8) & 0x00ff00ffu, dy);
#pragma unroll
    for (int k = 0; k < 5; k++) o[5 * w + k] = dx[k] | (dy[k] << 8);
  }
}
__device__ __forceinline__ int b3_dot16(const uint32_t (&o)[20], const uint32_t* qd, int acc) {
#pragma unroll
  for (int i = 0; i < 20; i++) acc = dp4a_us(o[i], qd[i], acc);
  return acc;
}
// The 20 staged activation words of one chunk (16-byte aligned).
__device__ __forceinline__ void b3_load_q(const void* p, uint32_t (&qd)[20]) {
  const uint4* q4 = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int v = 0; v < 5; v++) {
    const uint4 w4 = q4[v];
    qd[4 * v] = w4.x;
    qd[4 * v + 1] = w4.y;
    qd[4 * v + 2] = w4.z;
    qd[4 * v + 3] = w4.w;
  }
}
// Staging position (byte offset in an 80-byte chunk) of activation q[5g + k]
// for group g of the chunk (0..15).
__host__ __device__ inline int b3_qpos(int g, int k) { return 4 * (5 * (g >> 2) + k) + (g & 3); }

}  // namespace moe
