// build_sketch.cu -- offline: the rotated ternary sketch of every gate/up row.
//
// "KAIST: MoE Decoding Needs No Calibration Data", section "A reader that
// needs no data at all": each expert keeps a rotated ternary sketch of its
// gate and up weights, resident on the GPU, made from the weights alone.
// Per row: w' = H (s . w) (unnormalised Sylvester Walsh-Hadamard, fp32, stages
// h = 1, 2, 4, ...); Delta = 0.7 mean|w'| and alpha = mean |w'| over the kept
// entries, both fp64 in index order (TWN, Li & Liu 2016); 2-bit codes T + 1,
// position 4p + b of a 16-position word at bits 8b + 2p.  The
// index-order sums are done by one thread per row so the result equals the
// serial definition bit for bit.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kRowsPerCta = 8;

// s_j = +1 if the top bit of SplitMix64 output j is 0, else -1 (Steele, Lea &
// Flood 2014: output j = mix(seed + (j+1) * 0x9E3779B97F4A7C15)).
__global__ void rot_sign_kernel(int d, uint64_t seed, int8_t* s) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  uint64_t z = seed + (uint64_t)(j + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  s[j] = (z >> 63) ? (int8_t)-1 : (int8_t)1;
}

__global__ void __launch_bounds__(256) sketch_kernel(int E, int I, int d, const uint16_t* __restrict__ wg,
                                                     const uint16_t* __restrict__ wu,
                                                     const int8_t* __restrict__ sign, uint32_t* skg,
                                                     uint32_t* sku, float* ag, float* au) {
  extern __shared__ float v[];  // [kRowsPerCta][d]
  __shared__ double delta[kRowsPerCta];
  const long rows_per_mat = (long)E * I;
  const long row0 = (long)blockIdx.x * kRowsPerCta;
  const int nr = (int)min((long)kRowsPerCta, 2 * rows_per_mat - row0);
  for (int idx = threadIdx.x; idx < nr * d; idx += blockDim.x) {
    const int rr = idx / d, j = idx % d;
    const long g = row0 + rr;
    const uint16_t* w = g < rows_per_mat ? wg + g * d : wu + (g - rows_per_mat) * d;
    v[rr * d + j] = (float)sign[j] * bf16f(w[j]);
  }
  __syncthreads();
  for (int h = 1, lh = 0; h < d; h <<= 1, lh++) {
    for (int p = threadIdx.x; p < nr * (d / 2); p += blockDim.x) {
      const int rr = p / (d / 2), pp = p % (d / 2);
      const int j = ((pp >> lh) << (lh + 1)) | (pp & (h - 1));
      float* x = v + rr * d;
      const float x0 = x[j], x1 = x[j + h];
      x[j] = __fadd_rn(x0, x1);
      x[j + h] = __fsub_rn(x0, x1);
    }
    __syncthreads();
  }
  if (threadIdx.x < nr) {
    const int rr = threadIdx.x;
    const float* x = v + rr * d;
    double sabs = 0.0;
    for (int j = 0; j < d; j++) sabs += fabs((double)x[j]);
    const double dl = 0.7 * (sabs / (double)d);
    double snz = 0.0;
    int nnz = 0;
    for (int j = 0; j < d; j++) {
      const double a = fabs((double)x[j]);
      if (a > dl) {
        snz += a;
        nnz++;
      }
    }
    delta[rr] = dl;
    const long g = row0 + rr;
    const float alpha = nnz ? (float)(snz / (double)nnz) : 0.0f;
    if (g < rows_per_mat) ag[g] = alpha;
    else au[g - rows_per_mat] = alpha;
  }
  __syncthreads();
  const int words = d / 16;
  for (int idx = threadIdx.x; idx < nr * words; idx += blockDim.x) {
    const int rr = idx / words, m = idx % words;
    const float* x = v + rr * d + 16 * m;
    const double dl = delta[rr];
    uint32_t word = 0;
#pragma unroll
    for (int p = 0; p < 16; p++) {
      const float xv = x[p];
      uint32_t code = 1u;  // T + 1
      if (fabs((double)xv) > dl) code = xv > 0.0f ? 2u : 0u;
      word |= code << (8 * (p & 3) + 2 * (p >> 2));
    }
    const long g = row0 + rr;
    if (g < rows_per_mat) skg[g * words + m] = word;
    else sku[(g - rows_per_mat) * words + m] = word;
  }
}

// Base-3 repacking: output byte g of a row = sum_i code(5g + i) 3^i with
// code = t + 1 read from the 2-bit words (code 1, a zero trit, past d); the
// bytes past ceil(d / 5) that pad the row to whole sectors hold five zero
// trits (121).
__global__ void sketch_base3_kernel(long rows, int d, const uint32_t* __restrict__ codes, uint8_t* __restrict__ out) {
  const int rb = sk3_row_bytes(d), words = d / 16;
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * rb) return;
  const long row = idx / rb;
  const int g = (int)(idx - row * rb);
  const uint32_t* w = codes + row * words;
  uint32_t v = 0, pw = 1;
  for (int i = 0; i < 5; i++) {
    const int j = 5 * g + i;
    uint32_t code = 1u;
    if (j < d) {
      const int p = j & 15;
      code = (w[j >> 4] >> (8 * (p & 3) + 2 * (p >> 2))) & 3u;
    }
    v += code * pw;
    pw *= 3u;
  }
  out[idx] = (uint8_t)v;
}

__global__ void rmsnorm_kernel(int d, float eps, const uint16_t* __restrict__ x, uint16_t* __restrict__ h) {
  __shared__ float red[32];
  const uint16_t* xb = x + (size_t)blockIdx.x * d;
  float ss = 0.0f;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    const float t = bf16f(xb[j]);
    ss = fmaf(t, t, ss);
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.0f;
  for (int w = 0; w < (int)(blockDim.x >> 5); w++) tot += red[w];
  const float inv = 1.0f / sqrtf(tot / (float)d + eps);
  for (int j = threadIdx.x; j < d; j += blockDim.x) h[(size_t)blockIdx.x * d + j] = f2bf16(bf16f(xb[j]) * inv);
}

}  // namespace

cudaError_t launch_build_sketch(int E, int I, int d, const uint16_t* w_gate, const uint16_t* w_up,
                                uint64_t seed, int8_t* rot_sign, uint32_t* sk_gate, uint32_t* sk_up,
                                float* alpha_gate, float* alpha_up, cudaStream_t s) {
  rot_sign_kernel<<<(d + 255) / 256, 256, 0, s>>>(d, seed, rot_sign);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t smem = sizeof(float) * kRowsPerCta * d;
  err = cudaFuncSetAttribute(sketch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const long rows = 2L * E * I;
  const long grid = (rows + kRowsPerCta - 1) / kRowsPerCta;
  sketch_kernel<<<(unsigned)grid, 256, smem, s>>>(E, I, d, w_gate, w_up, rot_sign, sk_gate, sk_up, alpha_gate,
                                                   alpha_up);
  return cudaGetLastError();
}

cudaError_t launch_sketch_to_base3(long rows, int d, const uint32_t* codes, uint8_t* out, cudaStream_t s) {
  const long n = rows * sk3_row_bytes(d);
  if (n == 0) return cudaSuccess;
  sketch_base3_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(rows, d, codes, out);
  return cudaGetLastError();
}

namespace {
__global__ void __launch_bounds__(256) copy16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                     size_t n16) {
  pdl_trigger();
  pdl_wait();  // the previous kernel's writes (and reads of dst) are complete
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}
}  // namespace

cudaError_t launch_copy16(const void* src, void* dst, size_t bytes, cudaStream_t s) {
  const size_t n16 = bytes / 16;
  if (n16 == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  const size_t blocks = (n16 + 255) / 256;
  cfg.gridDim = dim3((unsigned)(blocks < 148 ? blocks : 148));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, copy16_kernel, reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst),
                            n16);
}

cudaError_t launch_rmsnorm(int B, int d, float eps, const uint16_t* x, uint16_t* h, cudaStream_t s) {
  rmsnorm_kernel<<<B, 256, 0, s>>>(d, eps, x, h);
  return cudaGetLastError();
}

}  // namespace moe
