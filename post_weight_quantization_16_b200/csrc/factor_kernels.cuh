// factor_kernels.cuh — S4: U = upper Cholesky factor of H^-1.
//
// ("模型量化实战…" §3.2 prepare: damped Hessian -> Cholesky -> inverse -> upper Cholesky.)
// Here the same U is reached in two steps instead of three: a reverse-ordered Cholesky
// A = V V^T with V upper-triangular, then U = V^-1 (upper), since then
// A^-1 = V^-T V^-1 = U^T U and the upper Cholesky factor with positive diagonal is unique.
//
// The host drives a recursion over diagonal blocks (bottom-right block first):
//   [U22] = f(A22);  V12 = A12 U22^T;  A11 -= V12 V12^T;  T = V12 U22;  [U11] = f(A11);
//   U12 = -U11 T
// whose products run on the tensor cores (gemm_tc.cuh) and whose leaves are the 128 x 128
// diagonal blocks handled by leaf_chol_inv_kernel below.  Matrices live as tf32 hi/lo
// pairs (X = hi + lo to about 2^-23) so that they can feed the three-product GEMM.
#pragma once

#include "sm100_ptx.cuh"

namespace gptq {

constexpr int LF_NB = 128;     // leaf block
constexpr int LF_P = 32;       // panel width (one warp)
constexpr int LF_THREADS = 256;
constexpr int LF_LD = LF_NB + 1;
constexpr int LF_SMEM = 3 * LF_NB * LF_LD * 4 + 16;

__device__ __forceinline__ float tf32_round(float x) {
  uint32_t u = __float_as_uint(x);
  u += 0xFFFu + ((u >> 13) & 1u);
  return __uint_as_float(u & 0xFFFFE000u);
}

// Warp 0: UL Cholesky of the 32 x 32 block S[P0.., P0..] (upper triangle) into V, and its
// inverse into X.  Lane i holds row i in registers; columns are broadcast with shuffles.
__device__ __forceinline__ void leaf_diag_factor(float (*S)[LF_LD], float (*V)[LF_LD], float (*X)[LF_LD], int P0,
                                                 int lane, int* bad) {
  float d[LF_P];
#pragma unroll
  for (int j = 0; j < LF_P; ++j) d[j] = S[P0 + lane][P0 + j];
#pragma unroll
  for (int c = LF_P - 1; c >= 0; --c) {
    float piv = __shfl_sync(0xffffffffu, d[c], c);
    if (!(piv > 0.0f) || !isfinite(piv)) {
      if (lane == 0) *bad = 1;
      piv = 1.0f;
    }
    const float s = sqrtf(piv);
    const float rs = 1.0f / s;
    const float col = (lane < c) ? d[c] * rs : (lane == c ? s : 0.0f);
    d[c] = col;
#pragma unroll
    for (int j = 0; j < c; ++j) {
      const float cj = __shfl_sync(0xffffffffu, col, j);
      d[j] = fmaf(-col, cj, d[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < LF_P; ++j) V[P0 + lane][P0 + j] = (j >= lane) ? d[j] : 0.0f;
  __syncwarp();
  // column `lane` of the inverse by back substitution (x[l] = 0 for l > lane)
  float x[LF_P];
#pragma unroll
  for (int r = LF_P - 1; r >= 0; --r) {
    float acc = 0.0f;
#pragma unroll
    for (int l = r + 1; l < LF_P; ++l) acc = fmaf(V[P0 + r][P0 + l], x[l], acc);
    const float vrr = V[P0 + r][P0 + r];
    x[r] = (r == lane) ? 1.0f / vrr : (r < lane ? -acc / vrr : 0.0f);
  }
#pragma unroll
  for (int r = 0; r < LF_P; ++r) X[P0 + r][P0 + lane] = x[r];
}

// Leaf: U_kk (= V_kk^-1, V_kk V_kk^T = A_kk) for the diagonal block at offset o, read from
// the upper triangle of A = A_hi + A_lo.  Writes U (upper, zeros below) and Ut = U^T as
// hi/lo pairs.  A non-positive or non-finite pivot sets ST_NOT_PD (and is replaced by 1
// so the kernel still finishes with finite work).
__global__ void __launch_bounds__(LF_THREADS, 1)
    leaf_chol_inv_kernel(const float* __restrict__ A_hi, const float* __restrict__ A_lo, int n, int o,
                         float* __restrict__ U_hi, float* __restrict__ U_lo, float* __restrict__ Ut_hi,
                         float* __restrict__ Ut_lo, int* __restrict__ status) {
  extern __shared__ float lf_smem[];
  float(*S)[LF_LD] = reinterpret_cast<float(*)[LF_LD]>(lf_smem);
  float(*V)[LF_LD] = reinterpret_cast<float(*)[LF_LD]>(lf_smem + LF_NB * LF_LD);
  float(*X)[LF_LD] = reinterpret_cast<float(*)[LF_LD]>(lf_smem + 2 * LF_NB * LF_LD);
  int* bad = reinterpret_cast<int*>(lf_smem + 3 * LF_NB * LF_LD);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) *bad = 0;
  for (int idx = tid; idx < LF_NB * LF_NB; idx += LF_THREADS) {
    const int i = idx / LF_NB, j = idx % LF_NB;
    const size_t g = static_cast<size_t>(o + i) * n + o + j;
    S[i][j] = (i <= j) ? A_hi[g] + A_lo[g] : 0.0f;
    V[i][j] = 0.0f;
    X[i][j] = 0.0f;
  }
  __syncthreads();

  // ---- reverse right-looking Cholesky, 32-column panels from the bottom-right ----
  for (int p = LF_NB / LF_P - 1; p >= 0; --p) {
    const int P0 = p * LF_P;
    if (warp == 0) leaf_diag_factor(S, V, X, P0, lane, bad);
    __syncthreads();
    // panel: V[i][P0+c] = sum_{k >= c} S[i][P0+k] * Xd[c][k]   for rows i < P0
    for (int item = tid; item < P0 * 8; item += LF_THREADS) {
      const int i = item >> 3, cg = (item & 7) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = cg + e;
        float acc = 0.0f;
        for (int k = c; k < LF_P; ++k) acc = fmaf(S[i][P0 + k], X[P0 + c][P0 + k], acc);
        V[i][P0 + c] = acc;
      }
    }
    __syncthreads();
    // trailing update of the upper triangle: S[i][j] -= sum_c V[i][P0+c] V[j][P0+c], i <= j < P0
    const int nb = P0 / 4;
    const int npairs = nb * (nb + 1) / 2;
    for (int t = tid; t < npairs; t += LF_THREADS) {
      int bj = static_cast<int>((sqrtf(8.0f * t + 1.0f) - 1.0f) * 0.5f);
      while (bj * (bj + 1) / 2 > t) --bj;
      while ((bj + 1) * (bj + 2) / 2 <= t) ++bj;
      const int bi = t - bj * (bj + 1) / 2;
      const int i0 = 4 * bi, j0 = 4 * bj;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
#pragma unroll 4
      for (int c = 0; c < LF_P; ++c) {
        float vi[4], vj[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          vi[a] = V[i0 + a][P0 + c];
          vj[a] = V[j0 + a][P0 + c];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(vi[a], vj[b], acc[a][b]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (i0 + a <= j0 + b) S[i0 + a][j0 + b] -= acc[a][b];
    }
    __syncthreads();
  }

  // ---- U = V^-1: diagonal 32-blocks are in X; off-diagonal blocks by block rows ----
  //   U_ij = -Xd_i * sum_{l=i+1..j} V_il U_lj      (block row i from the bottom)
  for (int bi = LF_NB / LF_P - 2; bi >= 0; --bi) {
    const int I0 = bi * LF_P;
    const int ncols = LF_NB - I0 - LF_P;  // columns right of the diagonal block
    // T[r][c] = sum_{k >= I0+32} V[I0+r][k] X[k][I0+32+c]  -> stored in S (free now)
    for (int item = tid; item < LF_P * ncols / 4; item += LF_THREADS) {
      const int r = item / (ncols / 4), c0 = (item % (ncols / 4)) * 4;
      const int col = I0 + LF_P + c0;
      const int kend = col + 4;  // X is upper: X[k][col..col+3] = 0 for k > col + 3
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int k = I0 + LF_P; k < kend; ++k) {
        const float v = V[I0 + r][k];
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = fmaf(v, X[k][col + e], acc[e]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) S[I0 + r][col + e] = acc[e];
    }
    __syncthreads();
    // X[I0+r][col] = -sum_{k >= r} Xd[r][k] T[k][col]
    for (int item = tid; item < LF_P * ncols / 4; item += LF_THREADS) {
      const int r = item / (ncols / 4), c0 = (item % (ncols / 4)) * 4;
      const int col = I0 + LF_P + c0;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int k = r; k < LF_P; ++k) {
        const float xd = X[I0 + r][I0 + k];
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = fmaf(xd, S[I0 + k][col + e], acc[e]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) X[I0 + r][col + e] = -acc[e];
    }
    __syncthreads();
  }

  // ---- write U (hi/lo) and Ut = U^T (hi/lo) ----
  for (int idx = tid; idx < LF_NB * LF_NB; idx += LF_THREADS) {
    const int i = idx / LF_NB, j = idx % LF_NB;
    const float u = (i <= j) ? X[i][j] : 0.0f;
    const float hi = tf32_round(u);
    const size_t g = static_cast<size_t>(o + i) * n + o + j;
    U_hi[g] = hi;
    U_lo[g] = tf32_round(u - hi);
  }
  for (int idx = tid; idx < LF_NB * LF_NB; idx += LF_THREADS) {
    const int j = idx / LF_NB, i = idx % LF_NB;  // Ut[j][i] = U[i][j]
    const float u = (i <= j) ? X[i][j] : 0.0f;
    const float hi = tf32_round(u);
    const size_t g = static_cast<size_t>(o + j) * n + o + i;
    Ut_hi[g] = hi;
    Ut_lo[g] = tf32_round(u - hi);
  }
  if (tid == 0 && *bad) atomicOr(status, ST_NOT_PD);
}

}  // namespace gptq
