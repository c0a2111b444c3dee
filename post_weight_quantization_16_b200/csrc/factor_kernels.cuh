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
static_assert(LF_NB * LF_NB <= LF_NB * LF_LD, "a staged block must fit in V (and in X)");

__device__ __forceinline__ float tf32_round(float x) {
  uint32_t u = __float_as_uint(x);
  u += 0xFFFu + ((u >> 13) & 1u);
  return __uint_as_float(u & 0xFFFFE000u);
}

// Warp 0: UL Cholesky of the 32 x 32 block S[P0.., P0..] (upper triangle) into V, and its
// inverse X = V^-1 in the same sweep.  Lane i holds row i of the block in registers
// (columns are broadcast with shuffles) and column i of the inverse.  Step c produces
// column c of V and row c of X: X[c][c] = 1/V[c][c], X[c][j] = -(sum_{c<l<=j} V[c][l] X[l][j]) / V[c][c];
// the inverse row uses only earlier steps' results, so it fills the latency of the pivot chain.
__device__ __forceinline__ void leaf_diag_factor(float (*S)[LF_LD], float (*V)[LF_LD], float (*X)[LF_LD], int P0,
                                                 int lane, int* bad) {
  float d[LF_P], x[LF_P];
#pragma unroll
  for (int j = 0; j < LF_P; ++j) {
    d[j] = S[P0 + lane][P0 + j];
    x[j] = 0.0f;
  }
#pragma unroll
  for (int c = LF_P - 1; c >= 0; --c) {
    float piv = __shfl_sync(0xffffffffu, d[c], c);
    if (!(piv > 0.0f) || !isfinite(piv)) {
      if (lane == 0) *bad = 1;
      piv = 1.0f;
    }
    const float rs = rsqrtf(piv);  // 1 / V[c][c]
    const float sv = piv * rs;     // V[c][c]
    const float col = (lane < c) ? d[c] * rs : (lane == c ? sv : 0.0f);
    d[c] = col;
    V[P0 + lane][P0 + c] = col;
#pragma unroll
    for (int j = c - 1; j >= 0; --j) {  // the next pivot column first: it is on the critical path
      const float cj = __shfl_sync(0xffffffffu, col, j);
      d[j] = fmaf(-col, cj, d[j]);
    }
    // row c of the inverse (V[c][l] for l > c were written by earlier steps)
    __syncwarp();
    float acc4[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four partial sums: a short dependent chain
#pragma unroll
    for (int l = c + 1; l < LF_P; ++l) acc4[l & 3] = fmaf(V[P0 + c][P0 + l], x[l], acc4[l & 3]);
    const float acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
    x[c] = (lane == c) ? rs : (lane > c ? -acc * rs : 0.0f);
  }
#pragma unroll
  for (int r = 0; r < LF_P; ++r) X[P0 + r][P0 + lane] = x[r];
  __syncwarp();
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
  griddep_wait();
  griddep_launch_dependents();  // one CTA: the next kernel may take the other SMs right away
  if (tid == 0) *bad = 0;
  // stage A_hi into V's storage and A_lo into X's with asynchronous 16-byte copies, at an
  // unpadded 128-float pitch (the 129-float rows of S are not 16-byte aligned)
  {
    float* th = &V[0][0];
    float* tl = &X[0][0];
    for (int idx = tid; idx < LF_NB * (LF_NB / 4); idx += LF_THREADS) {
      const int i = idx / (LF_NB / 4), j = (idx % (LF_NB / 4)) * 4;
      const size_t g = static_cast<size_t>(o + i) * n + o + j;
      const uint32_t dh = smem_u32(th + i * LF_NB + j), dl = smem_u32(tl + i * LF_NB + j);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dh), "l"(A_hi + g) : "memory");
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dl), "l"(A_lo + g) : "memory");
    }
    asm volatile("cp.async.commit_group;\n cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    for (int idx = tid; idx < LF_NB * LF_NB; idx += LF_THREADS) {
      const int i = idx / LF_NB, j = idx % LF_NB;
      const float v = th[i * LF_NB + j] + tl[i * LF_NB + j];
      S[i][j] = (i <= j) ? v : 0.0f;
    }
    __syncthreads();
    for (int idx = tid; idx < LF_NB * LF_LD; idx += LF_THREADS) {
      (&V[0][0])[idx] = 0.0f;
      (&X[0][0])[idx] = 0.0f;
    }
  }
  __syncthreads();

  // ---- reverse right-looking Cholesky, 32-column panels from the bottom-right ----
  // Lookahead: after the panel solve, warp 0 updates the next diagonal block itself and goes
  // straight on to factor it, while warps 1-3 and 5-7 (warp 4 shares warp 0's scheduler)
  // update the rest of the trailing triangle.
  for (int p = LF_NB / LF_P - 1; p >= 0; --p) {
    const int P0 = p * LF_P;
    if (warp == 0) leaf_diag_factor(S, V, X, P0, lane, bad);
    __syncthreads();
    // panel: V[i][P0+c] = sum_k S[i][P0+k] * Xd[c][k]   for rows i < P0 (Xd upper: zero for k < c);
    // one 4 x 4 tile of (rows, panel columns) per thread
    for (int item = tid; item < (P0 / 4) * (LF_P / 4); item += LF_THREADS) {
      const int i0 = (item / (LF_P / 4)) * 4, c0 = (item % (LF_P / 4)) * 4;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
#pragma unroll 8
      for (int k = 0; k < LF_P; ++k) {
        float sv[4], xv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          sv[a] = S[i0 + a][P0 + k];
          xv[a] = X[P0 + c0 + a][P0 + k];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(sv[a], xv[b], acc[a][b]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) V[i0 + a][P0 + c0 + b] = acc[a][b];
    }
    __syncthreads();
    if (p == 0) break;
    // trailing update of the upper triangle: S[i][j] -= sum_c V[i][P0+c] V[j][P0+c], i <= j < P0,
    // in 4 x 4 tiles (bi <= bj); the tiles of the next diagonal block go to warp 0
    const int nb = P0 / 4, nd = LF_P / 4, d0 = nb - nd;  // next diagonal block = tile rows/cols [d0, nb)
    int t_begin, t_step, t_end;
    if (warp == 0 || warp == 4) {  // the two warps of scheduler 0 update the next diagonal block
      t_begin = (warp == 4 ? 32 : 0) + lane;
      t_step = 64;
      t_end = nd * (nd + 1) / 2;  // tiles inside the next diagonal block
    } else {
      const int wi = (warp < 4) ? warp - 1 : warp - 2;  // 0..5
      t_begin = wi * 32 + lane;
      t_step = 6 * 32;
      t_end = nb * (nb + 1) / 2 - nd * (nd + 1) / 2;  // all other tiles
    }
    for (int t = t_begin; t < t_end; t += t_step) {
      int bi, bj;
      if (warp == 0 || warp == 4) {  // enumerate the upper tiles of the next diagonal block
        int jj = static_cast<int>((sqrtf(8.0f * t + 1.0f) - 1.0f) * 0.5f);
        while (jj * (jj + 1) / 2 > t) --jj;
        while ((jj + 1) * (jj + 2) / 2 <= t) ++jj;
        bi = d0 + (t - jj * (jj + 1) / 2);
        bj = d0 + jj;
      } else {  // enumerate all upper tiles with bj < d0, then the block column bi < d0 <= bj
        const int na = d0 * (d0 + 1) / 2;
        if (t < na) {
          int jj = static_cast<int>((sqrtf(8.0f * t + 1.0f) - 1.0f) * 0.5f);
          while (jj * (jj + 1) / 2 > t) --jj;
          while ((jj + 1) * (jj + 2) / 2 <= t) ++jj;
          bi = t - jj * (jj + 1) / 2;
          bj = jj;
        } else {
          const int u = t - na;
          bi = u / nd;
          bj = d0 + u % nd;
        }
      }
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
    if (warp == 0 || warp == 4) asm volatile("bar.sync 1, 64;" ::: "memory");  // next block updated
  }
  __syncthreads();

  // ---- U = V^-1: diagonal 32-blocks are in X; off-diagonal blocks by block rows ----
  //   U_ij = -Xd_i * sum_{l=i+1..j} V_il U_lj      (block row i from the bottom)
  for (int bi = LF_NB / LF_P - 2; bi >= 0; --bi) {
    const int I0 = bi * LF_P;
    const int ncols = LF_NB - I0 - LF_P;  // columns right of the diagonal block
    // T[r][col] = sum_{k >= I0+32} V[I0+r][k] X[k][col]  -> stored in S (free now);
    // one 4 x 4 tile per thread; X is upper, so X[k][col0..col0+3] = 0 for k > col0 + 3
    const int nct = ncols / 4;
    for (int item = tid; item < (LF_P / 4) * nct; item += LF_THREADS) {
      const int r0 = (item / nct) * 4, col0 = I0 + LF_P + (item % nct) * 4;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
      for (int k = I0 + LF_P; k < col0 + 4; ++k) {
        float vv[4], xv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          vv[a] = V[I0 + r0 + a][k];
          xv[a] = X[k][col0 + a];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(vv[a], xv[b], acc[a][b]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) S[I0 + r0 + a][col0 + b] = acc[a][b];
    }
    __syncthreads();
    // X[I0+r][col] = -sum_{k >= r} Xd[r][k] T[k][col]      (Xd upper: zero for k < r)
    for (int item = tid; item < (LF_P / 4) * nct; item += LF_THREADS) {
      const int r0 = (item / nct) * 4, col0 = I0 + LF_P + (item % nct) * 4;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
      for (int k = r0; k < LF_P; ++k) {
        float xd[4], tv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          xd[a] = X[I0 + r0 + a][I0 + k];
          tv[a] = S[I0 + k][col0 + a];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(xd[a], tv[b], acc[a][b]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) X[I0 + r0 + a][col0 + b] = -acc[a][b];
    }
    __syncthreads();
  }

  // ---- write U (hi/lo) and Ut = U^T (hi/lo), 16-byte stores ----
  for (int idx = tid; idx < LF_NB * (LF_NB / 4); idx += LF_THREADS) {
    const int i = idx / (LF_NB / 4), j = (idx % (LF_NB / 4)) * 4;
    float u[4], ut[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      u[e] = (i <= j + e) ? X[i][j + e] : 0.0f;   // U[i][j+e]
      ut[e] = (j + e <= i) ? X[j + e][i] : 0.0f;  // Ut[i][j+e] = U[j+e][i]
    }
    float uh[4], ul[4], th[4], tl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uh[e] = tf32_round(u[e]);
      ul[e] = tf32_round(u[e] - uh[e]);
      th[e] = tf32_round(ut[e]);
      tl[e] = tf32_round(ut[e] - th[e]);
    }
    const size_t g = static_cast<size_t>(o + i) * n + o + j;
    *reinterpret_cast<float4*>(U_hi + g) = make_float4(uh[0], uh[1], uh[2], uh[3]);
    *reinterpret_cast<float4*>(U_lo + g) = make_float4(ul[0], ul[1], ul[2], ul[3]);
    *reinterpret_cast<float4*>(Ut_hi + g) = make_float4(th[0], th[1], th[2], th[3]);
    *reinterpret_cast<float4*>(Ut_lo + g) = make_float4(tl[0], tl[1], tl[2], tl[3]);
  }
  if (tid == 0 && *bad) atomicOr(status, ST_NOT_PD);
}

}  // namespace gptq
