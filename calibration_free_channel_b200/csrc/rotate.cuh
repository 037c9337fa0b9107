// rotate.cuh -- the rotation and int8 quantisation of a token, shared by the
// reader kernels: q = rint(127 v / amax) of v = H (s . x), H the unnormalised
// Sylvester Walsh-Hadamard transform in fp32 with the stages in the fixed
// order h = 1, 2, 4, ... ("KAIST: MoE Decoding Needs No Calibration Data",
// section "A reader that needs no data at all": the sketch screens in the
// rotated domain).
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kRotThreads = 512;  // the rotation runs on whole 512-thread blocks

// Rotation + int8 quantisation of one token: v = FWHT(s . x) in the fp32
// scratch (d floats), q = rint(127 v / amax), c_x = amax / (127 d).  Stages
// h = 1, 2 run in registers (thread c holds elements 4c .. 4c+3) and
// h = 4 .. 64 across the lanes of a warp (a warp holds 128 consecutive
// elements); from h = 128 on, each pass over shared memory applies two stages
// (h and 2h) to four elements held in registers, and a last single stage
// runs alone when the count is odd.  Every element sees the reference
// butterflies (a + b, a - b) of every stage in the reference stage order, so
// the bits equal the reference transform's.  d >= 256.  sv_pre holds the
// signs of elements 4T .. 4T+3, loaded early by the caller.  xt: the token
// (bf16, shared memory), qt: its int8 codes.  qsum_out (may be null): the sum
// of the codes (the offset of the sketch's code dots).  Every thread of a
// 512-thread block calls it.
template <class Args>
__device__ void rotate_quantize(const Args& a, const uint16_t* xt, int8_t* qt, float* v, float* cx_out,
                                float* red, char4 sv_pre, int* qsum_out = nullptr) {
  const int d = a.d, d8 = d >> 3;
  const int T = threadIdx.x, lane = T & 31, warp = T >> 5;
  if (T == 0 && qsum_out) *qsum_out = 0;  // published by the block barriers below
  for (int c = T; c < 2 * d8; c += kRotThreads) {  // d / 4 is a multiple of 32: whole warps
    const uint2 xv = reinterpret_cast<const uint2*>(xt)[c];
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
      const float p0 = __shfl_xor_sync(0xffffffffu, r0, m), p1 = __shfl_xor_sync(0xffffffffu, r1, m);
      const float p2 = __shfl_xor_sync(0xffffffffu, r2, m), p3 = __shfl_xor_sync(0xffffffffu, r3, m);
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
      for (int p = T; p < 2 * d8; p += kRotThreads) {
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
      for (int p = T; p < 4 * d8; p += kRotThreads) {
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
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float amax = 0.0f;
#pragma unroll
  for (int w = 0; w < (kRotThreads / 32); w += 4) {
    const float4 r4 = reinterpret_cast<const float4*>(red)[w >> 2];
    amax = fmaxf(amax, fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w)));
  }
  int8_t* q = qt;
  int qs = 0;
  for (int j = T; j < d; j += kRotThreads) {
    int n = 0;
    if (amax > 0.0f) n = max(-127, min(127, __float2int_rn(__fdiv_rn(__fmul_rn(v[j], 127.0f), amax))));
    q[j] = (int8_t)n;
    qs += n;
  }
  if (qsum_out) {
    qs = warp_sum(qs);
    if (lane == 0) atomicAdd(qsum_out, qs);
  }
  if (T == 0) *cx_out = amax > 0.0f ? __fdiv_rn(amax, __fmul_rn(127.0f, (float)d)) : 0.0f;
  __syncthreads();
}

}  // namespace moe
