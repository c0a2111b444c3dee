// factor_kernels.cuh — S4: U = upper Cholesky factor of H^-1.
//
// ("模型量化实战…" §3.2 prepare: damped Hessian -> Cholesky -> inverse -> upper Cholesky.)
// Here the same U is reached in two steps instead of three: a reverse-ordered Cholesky
// A = V V^T with V upper-triangular, then U = V^-1 (upper), since then
// A^-1 = V^-T V^-1 = U^T U and the upper Cholesky factor with positive diagonal is unique.
//
// The host drives a recursion over diagonal blocks (bottom-right block first):
//   [V22,U22] = f(A22);  V12 = A12 U22^T;  A11 -= V12 V12^T;  [V11,U11] = f(A11);
//   U12 = -U11 (V12 U22)
// whose leaves are NB x NB diagonal blocks handled by chol_inv_base_kernel below, and whose
// other steps are GEMMs.
#pragma once

#include "sm100_ptx.cuh"

namespace gptq {

constexpr int FB_NB = 64;          // leaf block
constexpr int FB_THREADS = 256;

// Leaf: V_kk (A_kk = V_kk V_kk^T, V_kk upper) and U_kk = V_kk^-1 for the diagonal block at
// offset o.  Reads the upper triangle of A's block; writes full NB x NB blocks of V and U
// (zeros below the diagonal).  A non-positive or non-finite pivot sets ST_NOT_PD (the pivot
// is replaced by 1 so the kernel still terminates with finite work).
__global__ void __launch_bounds__(FB_THREADS)
    chol_inv_base_kernel(const float* __restrict__ A, float* __restrict__ V, float* __restrict__ U, int n, int o,
                         int* __restrict__ status) {
  constexpr int NB = FB_NB;
  __shared__ float S[NB][NB + 1];
  __shared__ float X[NB][NB + 1];
  __shared__ float col[NB];
  __shared__ int bad;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  for (int idx = tid; idx < NB * NB; idx += FB_THREADS) {
    const int i = idx / NB, j = idx % NB;
    S[i][j] = (i <= j) ? A[static_cast<size_t>(o + i) * n + o + j] : 0.0f;
    X[i][j] = 0.0f;
  }
  __syncthreads();

  // reverse (bottom-right first) right-looking Cholesky on the upper triangle
  for (int c = NB - 1; c >= 0; --c) {
    float d = S[c][c];
    if (!(d > 0.0f) || !isfinite(d)) {
      if (tid == 0) bad = 1;
      d = 1.0f;
    }
    const float sd = sqrtf(d);
    const float rsd = 1.0f / sd;
    if (tid <= c) col[tid] = (tid == c) ? sd : S[tid][c] * rsd;
    __syncthreads();
    // S[i][j] -= col[i] col[j] for i <= j < c ; column c of V replaces S[:, c]
    const int pairs = c * (c + 1) / 2;
    for (int p = tid; p < pairs; p += FB_THREADS) {
      // p -> (i, j) with 0 <= i <= j < c, enumerated by j
      int j = static_cast<int>((sqrtf(8.0f * p + 1.0f) - 1.0f) * 0.5f);
      while (j * (j + 1) / 2 > p) --j;
      while ((j + 1) * (j + 2) / 2 <= p) ++j;
      const int i = p - j * (j + 1) / 2;
      S[i][j] = fmaf(-col[i], col[j], S[i][j]);
    }
    if (tid <= c) S[tid][c] = col[tid];
    __syncthreads();
  }

  // X = V^-1 (upper), one column per thread by back substitution
  if (tid < NB) {
    const int c = tid;
    X[c][c] = 1.0f / S[c][c];
    for (int r = c - 1; r >= 0; --r) {
      float s = 0.0f;
      for (int l = r + 1; l <= c; ++l) s = fmaf(S[r][l], X[l][c], s);
      X[r][c] = -s / S[r][r];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < NB * NB; idx += FB_THREADS) {
    const int i = idx / NB, j = idx % NB;
    const size_t g = static_cast<size_t>(o + i) * n + o + j;
    V[g] = (i <= j) ? S[i][j] : 0.0f;
    U[g] = (i <= j) ? X[i][j] : 0.0f;
  }
  if (tid == 0 && bad) atomicOr(status, ST_NOT_PD);
}

}  // namespace gptq
