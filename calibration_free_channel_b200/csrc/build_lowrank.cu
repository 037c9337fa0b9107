// build_lowrank.cu -- offline: the low-rank map of the down projections.
//
// "KAIST: MoE Decoding Needs No Calibration Data", section "A reader that
// needs no data at all": skipped channels are recovered through a low-rank
// map of the down projections, made from the weights alone.  The map here is
// the rank-r truncated SVD W_down[e] = U S V^T: u_sigma = U_r S_r [I, r],
// v = V_r [d, r], and in each column the entry of v with the largest magnitude
// is positive (ties: lower index).
//
// Per expert: M = W W^T (fp32 Gram); subspace iteration Y <- orth(M Y) on p =
// r + 32 columns (Cholesky-QR in fp64); Rayleigh-Ritz H = Y^T M Y solved by
// cyclic Jacobi rotations (fp64); U_r = Y S_r, sigma = sqrt(lambda);
// V_r = W^T U_r / sigma.  Subspace iteration with Rayleigh-Ritz converges for
// the top r pairs at the rate lambda_{p+1} / lambda_j per step.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kIters = 40;
constexpr int kOversample = 32;
constexpr int kMaxP = 96;
constexpr int kChunk = 16;

__host__ __device__ inline int lr_p(int I, int r) { return I < r + kOversample ? I : r + kOversample; }

struct LrWs {
  float *M, *Y, *Z, *Ur, *V;
  double* sigma;
};

__host__ __device__ inline size_t lr_layout(int E, int I, int d, int r, char* base, LrWs* w) {
  const int p = lr_p(I, r);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = (off + bytes + 255) & ~(size_t)255;
    return o;
  };
  const size_t oM = take(sizeof(float) * (size_t)E * I * I);
  const size_t oY = take(sizeof(float) * (size_t)E * I * p);
  const size_t oZ = take(sizeof(float) * (size_t)E * I * p);
  const size_t oU = take(sizeof(float) * (size_t)E * I * r);
  const size_t oV = take(sizeof(float) * (size_t)E * d * r);
  const size_t oS = take(sizeof(double) * (size_t)E * r);
  if (w && base) {
    w->M = reinterpret_cast<float*>(base + oM);
    w->Y = reinterpret_cast<float*>(base + oY);
    w->Z = reinterpret_cast<float*>(base + oZ);
    w->Ur = reinterpret_cast<float*>(base + oU);
    w->V = reinterpret_cast<float*>(base + oV);
    w->sigma = reinterpret_cast<double*>(base + oS);
  }
  return off;
}

// M[e] = W[e] W[e]^T, 64x64 tiles, fp32 accumulation of exact bf16 products.
__global__ void __launch_bounds__(256) gram_kernel(int I, int d, const uint16_t* __restrict__ W, float* M) {
  __shared__ float As[32][65], Bs[32][65];
  const int e = blockIdx.z;
  const int bi = blockIdx.y * 64, bj = blockIdx.x * 64;
  const uint16_t* We = W + (size_t)e * I * d;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += 32) {
    for (int idx = threadIdx.x; idx < 64 * 32; idx += 256) {
      const int rr = idx / 32, kk = idx % 32;
      As[kk][rr] = (bi + rr < I) ? bf16f(We[(size_t)(bi + rr) * d + k0 + kk]) : 0.0f;
      Bs[kk][rr] = (bj + rr < I) ? bf16f(We[(size_t)(bj + rr) * d + k0 + kk]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; kk++) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        a[q] = As[kk][ty * 4 + q];
        b[q] = Bs[kk][tx * 4 + q];
      }
#pragma unroll
      for (int u = 0; u < 4; u++)
#pragma unroll
        for (int v = 0; v < 4; v++) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
  for (int u = 0; u < 4; u++)
    for (int v = 0; v < 4; v++) {
      const int i = bi + ty * 4 + u, j = bj + tx * 4 + v;
      if (i < I && j < I) M[((size_t)e * I + i) * I + j] = acc[u][v];
    }
}

// Z = M Y for one expert (M symmetric, so M[k][i] is read coalesced).
__device__ void mul_MY(int I, int p, const float* M, const float* Y, float* Z, float* ys) {
  for (int c0 = 0; c0 < p; c0 += kChunk) {
    const int cw = min(kChunk, p - c0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < I * kChunk; idx += blockDim.x) {
      const int k = idx / kChunk, c = idx % kChunk;
      ys[idx] = c < cw ? Y[(size_t)k * p + c0 + c] : 0.0f;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < I; i += blockDim.x) {
      float acc[kChunk];
#pragma unroll
      for (int c = 0; c < kChunk; c++) acc[c] = 0.0f;
      for (int k = 0; k < I; k++) {
        const float m = M[(size_t)k * I + i];
#pragma unroll
        for (int c = 0; c < kChunk; c++) acc[c] = fmaf(m, ys[k * kChunk + c], acc[c]);
      }
      for (int c = 0; c < cw; c++) Z[(size_t)i * p + c0 + c] = acc[c];
    }
  }
  __syncthreads();
}

// Y = Z R^{-1} with Z^T Z = R^T R (Cholesky, fp64): an orthonormal basis of
// span(Z).  L (lower, = R^T) is p x p in shared memory.
__device__ void chol_qr(int I, int p, const float* Z, float* Y, double* L) {
  const int np = p * (p + 1) / 2;
  for (int idx = threadIdx.x; idx < np; idx += blockDim.x) {
    // unrank (a, b) with a <= b
    int a = 0, rem = idx;
    while (rem >= p - a) {
      rem -= p - a;
      a++;
    }
    const int b = a + rem;
    double s = 0.0;
    for (int i = 0; i < I; i++) s = fma((double)Z[(size_t)i * p + a], (double)Z[(size_t)i * p + b], s);
    L[a * p + b] = s;
    L[b * p + a] = s;
  }
  __syncthreads();
  // right-looking Cholesky; L[j][j..] upper part left as scratch
  for (int j = 0; j < p; j++) {
    if (threadIdx.x == 0) {
      double dj = L[j * p + j];
      L[j * p + j] = dj > 1e-300 ? sqrt(dj) : 1e-150;
    }
    __syncthreads();
    const double djj = L[j * p + j];
    for (int i = j + 1 + threadIdx.x; i < p; i += blockDim.x) L[i * p + j] /= djj;
    __syncthreads();
    const int rest = p - j - 1;
    for (int idx = threadIdx.x; idx < rest * rest; idx += blockDim.x) {
      const int i = j + 1 + idx / rest, k = j + 1 + idx % rest;
      if (k <= i) L[i * p + k] -= L[i * p + j] * L[k * p + j];
    }
    __syncthreads();
  }
  // rows of Y: y R = z with R[a][c] = L[c][a]
  for (int i = threadIdx.x; i < I; i += blockDim.x) {
    for (int c = 0; c < p; c++) {
      double s = (double)Z[(size_t)i * p + c];
      for (int a = 0; a < c; a++) s -= (double)Y[(size_t)i * p + a] * L[c * p + a];
      Y[(size_t)i * p + c] = (float)(s / L[c * p + c]);
    }
  }
  __syncthreads();
}

// Cyclic Jacobi on the symmetric p x p matrix A (fp64, shared); S <- S J.
__device__ void jacobi_eig(int p, double* A, double* S, double* rot) {
  for (int idx = threadIdx.x; idx < p * p; idx += blockDim.x) S[idx] = (idx / p == idx % p) ? 1.0 : 0.0;
  __syncthreads();
  for (int sweep = 0; sweep < 30; sweep++) {
    // off-diagonal norm
    __shared__ double off_s, diag_s;
    if (threadIdx.x == 0) {
      double off = 0.0, dg = 0.0;
      for (int a = 0; a < p; a++)
        for (int b = 0; b < p; b++) {
          if (a != b) off += A[a * p + b] * A[a * p + b];
          else dg += A[a * p + b] * A[a * p + b];
        }
      off_s = off;
      diag_s = dg;
    }
    __syncthreads();
    if (off_s <= 1e-30 * diag_s) break;
    for (int pp = 0; pp < p - 1; pp++)
      for (int qq = pp + 1; qq < p; qq++) {
        if (threadIdx.x == 0) {
          const double apq = A[pp * p + qq];
          double c = 1.0, s = 0.0, t = 0.0;
          if (fabs(apq) > 1e-300) {
            const double theta = (A[qq * p + qq] - A[pp * p + pp]) / (2.0 * apq);
            t = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
            c = 1.0 / sqrt(t * t + 1.0);
            s = t * c;
          }
          rot[0] = c;
          rot[1] = s;
          rot[2] = t;
          rot[3] = apq;
        }
        __syncthreads();
        const double c = rot[0], s = rot[1], t = rot[2], apq = rot[3];
        if (s != 0.0) {
          for (int k = threadIdx.x; k < p; k += blockDim.x) {
            if (k != pp && k != qq) {
              const double akp = A[k * p + pp], akq = A[k * p + qq];
              const double np_ = c * akp - s * akq, nq = s * akp + c * akq;
              A[k * p + pp] = np_;
              A[pp * p + k] = np_;
              A[k * p + qq] = nq;
              A[qq * p + k] = nq;
            }
            const double vkp = S[k * p + pp], vkq = S[k * p + qq];
            S[k * p + pp] = c * vkp - s * vkq;
            S[k * p + qq] = s * vkp + c * vkq;
          }
          __syncthreads();
          if (threadIdx.x == 0) {
            A[pp * p + pp] -= t * apq;
            A[qq * p + qq] += t * apq;
            A[pp * p + qq] = 0.0;
            A[qq * p + pp] = 0.0;
          }
        }
        __syncthreads();
      }
  }
}

__global__ void __launch_bounds__(256) subspace_kernel(int I, int r, LrWs w) {
  extern __shared__ __align__(16) char sm[];
  const int e = blockIdx.x;
  const int p = lr_p(I, r);
  float* ys = reinterpret_cast<float*>(sm);                                   // [I, kChunk]
  double* L = reinterpret_cast<double*>(sm + sizeof(float) * I * kChunk);     // [p, p]
  double* S = L + p * p;                                                      // [p, p]
  __shared__ double rot[4];
  __shared__ int order[kMaxP];
  const float* M = w.M + (size_t)e * I * I;
  float* Y = w.Y + (size_t)e * I * p;
  float* Z = w.Z + (size_t)e * I * p;
  // deterministic start: entries in [-1, 1) from SplitMix64 of the index
  for (int idx = threadIdx.x; idx < I * p; idx += blockDim.x) {
    uint64_t z = (uint64_t)(idx + 1) * 0x9E3779B97F4A7C15ull + 12345;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    Z[idx] = (float)((double)(z >> 11) * 0x1.0p-52 - 1.0);
  }
  __syncthreads();
  chol_qr(I, p, Z, Y, L);
  for (int it = 0; it < kIters; it++) {
    mul_MY(I, p, M, Y, Z, ys);
    chol_qr(I, p, Z, Y, L);
  }
  chol_qr(I, p, Y, Z, L);  // re-orthonormalise: Z = orth(Y)
  // Rayleigh-Ritz: H = Z^T M Z
  mul_MY(I, p, M, Z, Y, ys);  // Y = M Z
  for (int idx = threadIdx.x; idx < p * p; idx += blockDim.x) {
    const int a = idx / p, b = idx % p;
    double s = 0.0;
    for (int i = 0; i < I; i++) s = fma((double)Z[(size_t)i * p + a], (double)Y[(size_t)i * p + b], s);
    L[idx] = s;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < p * p; idx += blockDim.x) {
    const int a = idx / p, b = idx % p;
    if (a < b) {
      const double m = 0.5 * (L[a * p + b] + L[b * p + a]);
      L[a * p + b] = m;
      L[b * p + a] = m;
    }
  }
  __syncthreads();
  jacobi_eig(p, L, S, rot);
  if (threadIdx.x == 0) {
    for (int a = 0; a < p; a++) order[a] = a;
    for (int a = 0; a < r; a++) {
      int best = a;
      for (int b = a + 1; b < p; b++)
        if (L[order[b] * p + order[b]] > L[order[best] * p + order[best]]) best = b;
      const int tmp = order[a];
      order[a] = order[best];
      order[best] = tmp;
    }
    for (int a = 0; a < r; a++) {
      const double lam = L[order[a] * p + order[a]];
      w.sigma[(size_t)e * r + a] = lam > 0 ? sqrt(lam) : 0.0;
    }
  }
  __syncthreads();
  float* Ur = w.Ur + (size_t)e * I * r;
  for (int idx = threadIdx.x; idx < I * r; idx += blockDim.x) {
    const int i = idx / r, rho = idx % r;
    double s = 0.0;
    for (int a = 0; a < p; a++) s = fma((double)Z[(size_t)i * p + a], S[a * p + order[rho]], s);
    Ur[idx] = (float)s;
  }
}

// V[e][j][rho] = sum_i W[e][i][j] Ur[i][rho] / sigma_rho
__global__ void __launch_bounds__(128) v_kernel(int I, int d, int r, const uint16_t* __restrict__ W, LrWs w) {
  extern __shared__ float us[];  // [I, r]
  const int e = blockIdx.y;
  for (int idx = threadIdx.x; idx < I * r; idx += blockDim.x) us[idx] = w.Ur[(size_t)e * I * r + idx];
  __syncthreads();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  float acc[64];
#pragma unroll
  for (int q = 0; q < 64; q++) acc[q] = 0.0f;
  const uint16_t* We = W + (size_t)e * I * d;
  for (int i = 0; i < I; i++) {
    const float wv = bf16f(We[(size_t)i * d + j]);
#pragma unroll
    for (int q = 0; q < 64; q++)
      if (q < r) acc[q] = fmaf(wv, us[i * r + q], acc[q]);
  }
  for (int q = 0; q < r; q++) {
    const double sg = w.sigma[(size_t)e * r + q];
    w.V[((size_t)e * d + j) * r + q] = sg > 0 ? (float)(acc[q] / sg) : 0.0f;
  }
}

// Sign rule and bf16 output.
__global__ void __launch_bounds__(256) finalize_kernel(int I, int d, int r, LrWs w, uint16_t* u_sigma, uint16_t* v) {
  __shared__ float sgn[128];
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* V = w.V + (size_t)e * d * r;
  for (int rho = warp; rho < r; rho += blockDim.x / 32) {
    float best = -1.0f, val = 0.0f;
    int bj = 0x7fffffff;
    for (int j = lane; j < d; j += 32) {
      const float x = V[(size_t)j * r + rho];
      if (fabsf(x) > best) {
        best = fabsf(x);
        bj = j;
        val = x;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      const float ov = __shfl_xor_sync(0xffffffffu, val, o);
      if (ob > best || (ob == best && oj < bj)) {
        best = ob;
        bj = oj;
        val = ov;
      }
    }
    if (lane == 0) sgn[rho] = val < 0 ? -1.0f : 1.0f;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < I * r; idx += blockDim.x) {
    const int rho = idx % r;
    const float s = (float)w.sigma[(size_t)e * r + rho];
    u_sigma[(size_t)e * I * r + idx] = f2bf16(w.Ur[(size_t)e * I * r + idx] * s * sgn[rho]);
  }
  for (int idx = threadIdx.x; idx < d * r; idx += blockDim.x)
    v[(size_t)e * d * r + idx] = f2bf16(V[idx] * sgn[idx % r]);
}

}  // namespace

size_t lowrank_ws_bytes(int E, int I, int d, int r) { return lr_layout(E, I, d, r, nullptr, nullptr); }

cudaError_t launch_build_lowrank(int E, int I, int d, int r, const uint16_t* w_down, uint16_t* u_sigma,
                                 uint16_t* v, void* ws, cudaStream_t s) {
  LrWs w;
  lr_layout(E, I, d, r, static_cast<char*>(ws), &w);
  const int p = lr_p(I, r);
  dim3 g((I + 63) / 64, (I + 63) / 64, E);
  gram_kernel<<<g, 256, 0, s>>>(I, d, w_down, w.M);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t sm = sizeof(float) * I * kChunk + 2 * sizeof(double) * p * p;
  err = cudaFuncSetAttribute(subspace_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (err != cudaSuccess) return err;
  subspace_kernel<<<E, 256, sm, s>>>(I, r, w);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t smv = sizeof(float) * I * r;
  err = cudaFuncSetAttribute(v_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smv);
  if (err != cudaSuccess) return err;
  v_kernel<<<dim3((d + 127) / 128, E), 128, smv, s>>>(I, d, r, w_down, w);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  finalize_kernel<<<E, 256, 0, s>>>(I, d, r, w, u_sigma, v);
  return cudaGetLastError();
}

}  // namespace moe
