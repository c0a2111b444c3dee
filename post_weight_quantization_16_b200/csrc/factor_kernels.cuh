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
constexpr int LF_SMEM = 3 * LF_NB * LF_LD * 4 + LF_NB * 4 + 16;  // S, V, X, 1/V[c][c], flag
static_assert(LF_NB * LF_NB <= LF_NB * LF_LD, "a staged block must fit in V (and in X)");

__device__ __forceinline__ float tf32_round(float x) {
  uint32_t u = __float_as_uint(x);
  u += 0xFFFu + ((u >> 13) & 1u);
  return __uint_as_float(u & 0xFFFFE000u);
}

// Warp 0: one 32-column panel of the UL Cholesky, P0 = 32 p.  Lane l carries row P0 + l of
// the diagonal block (and, for NR > 0, row 32 r + l of block row r < NR above it) in
// registers; step c (from the panel's last column down) produces column P0 + c of V for
// those rows, eliminating it from the panel's earlier columns:
//   V[c][c] = sqrt(S[c][c]),   V[i][c] = S[i][c] / V[c][c],   S[i][j] -= V[i][c] V[j][c].
// The pivot chain is kept short: lane c-1's diagonal after column c is its own column value
// squared off its diagonal, so the next pivot is broadcast without waiting for the column
// broadcast.  1 / V[c][c] goes to rsv for the inverse of the diagonal block.
template <int NR>
__device__ __forceinline__ void leaf_sweep(float (*S)[LF_LD], float (*V)[LF_LD], float* rsv, int P0, int lane,
                                           int* bad) {
  float d[NR + 1][LF_P];
#pragma unroll
  for (int j = 0; j < LF_P; ++j) {
    d[0][j] = S[P0 + lane][P0 + j];
#pragma unroll
    for (int r = 0; r < NR; ++r) d[r + 1][j] = S[LF_P * r + lane][P0 + j];
  }
  float pnext = __shfl_sync(0xffffffffu, d[0][LF_P - 1], LF_P - 1);
#pragma unroll
  for (int c = LF_P - 1; c >= 0; --c) {
    float piv = pnext;
    if (!(piv > 0.0f) || !isfinite(piv)) {
      if (lane == 0) *bad = 1;
      piv = 1.0f;
    }
    const float rs = rsqrtf(piv);  // 1 / V[c][c]
    const float sv = piv * rs;     // V[c][c]
    float col[NR + 1];
    col[0] = (lane < c) ? d[0][c] * rs : (lane == c ? sv : 0.0f);
#pragma unroll
    for (int r = 0; r < NR; ++r) col[r + 1] = d[r + 1][c] * rs;
    if (c > 0) pnext = __shfl_sync(0xffffffffu, fmaf(-col[0], col[0], d[0][c - 1]), c - 1);
    V[P0 + lane][P0 + c] = col[0];
#pragma unroll
    for (int r = 0; r < NR; ++r) V[LF_P * r + lane][P0 + c] = col[r + 1];
    if (lane == 0) rsv[P0 + c] = rs;
#pragma unroll
    for (int j = c - 1; j >= 0; --j) {
      const float cj = __shfl_sync(0xffffffffu, col[0], j);  // V[P0 + j][P0 + c]
#pragma unroll
      for (int r = 0; r <= NR; ++r) d[r][j] = fmaf(-col[r], cj, d[r][j]);
    }
  }
  __syncwarp();
}

// One warp, lane l: row 32 r + l above diagonal block P0 (r < P0 / 32), its panel-p part
// from the block's factor (V's diagonal block and 1 / V[c][c] in shared memory):
//   V[i][P0+c] = (S[i][P0+c] - sum_{k>c} V[i][P0+k] V[P0+c][P0+k]) / V[c][c],  c from the last.
// Every lane reads the same V entries (broadcast) and works on its own row.
__device__ __forceinline__ void leaf_rows_above(float (*S)[LF_LD], float (*V)[LF_LD], const float* rsv, int P0,
                                                int row) {
  float d[LF_P];
#pragma unroll
  for (int j = 0; j < LF_P; ++j) d[j] = S[row][P0 + j];
#pragma unroll
  for (int c = LF_P - 1; c >= 0; --c) {
    const float col = d[c] * rsv[P0 + c];
    V[row][P0 + c] = col;
#pragma unroll
    for (int j = c - 1; j >= 0; --j) d[j] = fmaf(-col, V[P0 + j][P0 + c], d[j]);
  }
}

// One warp: the inverse X = V^-1 of diagonal block P0 (upper, 32 x 32), lane j holding column
// j: X[c][c] = 1/V[c][c], X[c][j] = -(sum_{c<l<=j} V[c][l] X[l][j]) / V[c][c], rows from the
// last up.  Written to X's diagonal block (zeros below the diagonal).
__device__ __forceinline__ void leaf_inv_diag(const float (*V)[LF_LD], float (*X)[LF_LD], const float* rsv, int P0,
                                              int lane) {
  float x[LF_P];
#pragma unroll
  for (int c = LF_P - 1; c >= 0; --c) {
    float acc4[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four partial sums: a short dependent chain
#pragma unroll
    for (int l = c + 1; l < LF_P; ++l) acc4[l & 3] = fmaf(V[P0 + c][P0 + l], x[l], acc4[l & 3]);
    const float acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
    const float rs = rsv[P0 + c];
    x[c] = (lane == c) ? rs : (lane > c ? -acc * rs : 0.0f);
  }
#pragma unroll
  for (int r = 0; r < LF_P; ++r) X[P0 + r][P0 + lane] = x[r];
}

// 4 x 4 tile of C[i0.., j0..] = sum_k P[i0 + a][k] Q[j0 + b][k] over k in [k0, k1), rows of
// P and Q in shared memory at pitch LF_LD.
__device__ __forceinline__ void lf_tile_nt(const float (*P)[LF_LD], const float (*Q)[LF_LD], int i0, int j0, int k0,
                                           int k1, float (&acc)[4][4]) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
#pragma unroll 4
  for (int k = k0; k < k1; ++k) {
    float pv[4], qv[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      pv[a] = P[i0 + a][k];
      qv[a] = Q[j0 + a][k];
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(pv[a], qv[b], acc[a][b]);
  }
}

__device__ __forceinline__ void lf_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Rows [R0, R0 + 32) of U = X (zeros left of the diagonal) as a hi/lo pair and as plain fp32,
// 16-byte stores, by threads t = 0 .. nt-1.  (U^T is formed off the critical path.)
__device__ __forceinline__ void leaf_store_rows(const float (*X)[LF_LD], float* __restrict__ U_hi,
                                                float* __restrict__ U_lo, float* __restrict__ U32, int n, int o,
                                                int R0, int t, int nt) {
  for (int idx = t; idx < LF_P * (LF_NB / 4); idx += nt) {
    const int i = R0 + idx / (LF_NB / 4), j = (idx % (LF_NB / 4)) * 4;
    float uh[4], ul[4], u4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float u = (i <= j + e) ? X[i][j + e] : 0.0f;  // U[i][j+e]
      u4[e] = u;
      uh[e] = tf32_round(u);
      ul[e] = tf32_round(u - uh[e]);
    }
    const size_t g = static_cast<size_t>(o + i) * n + o + j;
    *reinterpret_cast<float4*>(U32 + g) = make_float4(u4[0], u4[1], u4[2], u4[3]);
    *reinterpret_cast<float4*>(U_hi + g) = make_float4(uh[0], uh[1], uh[2], uh[3]);
    *reinterpret_cast<float4*>(U_lo + g) = make_float4(ul[0], ul[1], ul[2], ul[3]);
  }
}

// Leaf: U_kk (= V_kk^-1, V_kk V_kk^T = A_kk) for the diagonal block at offset o, read from
// the upper triangle of A = A_hi + A_lo.  Writes U (upper, zeros below) as a hi/lo pair
// (transpose_block_kernel forms U^T on the graph's second branch).  A non-positive or non-finite pivot sets ST_NOT_PD (and is replaced by 1
// so the kernel still finishes with finite work).
//
// Reverse right-looking Cholesky over four 32-column panels, bottom-right first.  The chain
// from one panel to the next is kept short: warp 0 factors diagonal block p in registers,
// warps 1 .. p solve the rows above it (one row a lane) while warp 5 inverts the diagonal
// block, all warps update column block p-1 (lookahead), and warp 0 goes on to block p-1
// while the six warps 1-3, 5-7 finish the trailing update and form block row p of the
// inverse U = V^-1:
//   U_pj = -Xd_p * sum_{l=p+1..j} V_pl U_lj      (Xd_p = the diagonal block's inverse).
__global__ void __launch_bounds__(LF_THREADS, 1)
    leaf_chol_inv_kernel(const float* __restrict__ A_hi, const float* __restrict__ A_lo, int n, int o,
                         float* __restrict__ U_hi, float* __restrict__ U_lo, float* __restrict__ U32,
                         int* __restrict__ status) {
  extern __shared__ float lf_smem[];
  float(*S)[LF_LD] = reinterpret_cast<float(*)[LF_LD]>(lf_smem);
  float(*V)[LF_LD] = reinterpret_cast<float(*)[LF_LD]>(lf_smem + LF_NB * LF_LD);
  float(*X)[LF_LD] = reinterpret_cast<float(*)[LF_LD]>(lf_smem + 2 * LF_NB * LF_LD);
  int* bad = reinterpret_cast<int*>(lf_smem + 3 * LF_NB * LF_LD + LF_NB);  // after rsv
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
  }
  __syncthreads();
  // (every entry of V and X that is read below is written first: no clearing needed)

  float* rsv = &X[0][0] + LF_NB * LF_LD;  // [128] 1 / V[c][c]
  // the six warps 1-3, 5-7 (warp 4 shares warp 0's scheduler and stays out of its way)
  const bool g1 = (warp != 0 && warp != 4);
  const int t1 = tid - 32 * ((warp > 0) + (warp > 4));  // 0..191 within the six warps
  constexpr int NG1 = LF_THREADS - 64;

#pragma unroll 1
  for (int p = LF_NB / LF_P - 1; p >= 0; --p) {
    const int P0 = p * LF_P;
    // panel p: the diagonal block (warp 0, the chain), then the rows above it (warps 1 .. p,
    // one row a lane) while warp 5 inverts the diagonal block
    if (warp == 0) leaf_sweep<0>(S, V, rsv, P0, lane, bad);
    __syncthreads();  // diagonal block p in V; the six warps' work of the step before is done
    if (warp >= 1 && warp <= p) leaf_rows_above(S, V, rsv, P0, LF_P * (warp - 1) + lane);
    if (warp == 5) leaf_inv_diag(V, X, rsv, P0, lane);  // Xd_p
    __syncthreads();  // panel p in V for every row; Xd_p in X
    if (p > 0) {
      // lookahead: column block p-1 of the trailing update, all warps
      //   S[i][j] -= sum_c V[i][P0+c] V[j][P0+c],  j in [P0-32, P0), i <= j
      const int nrt = P0 / 4;  // row tiles 0 .. nrt-1; column tiles of block p-1: 8
      for (int t = tid; t < nrt * 8; t += LF_THREADS) {
        const int bi = t / 8, bj = (P0 - LF_P) / 4 + t % 8;
        if (bi > bj) continue;
        const int i0 = 4 * bi, j0 = 4 * bj;
        float acc[4][4];
        lf_tile_nt(V, V, i0, j0, P0, P0 + LF_P, acc);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b)
            if (i0 + a <= j0 + b) S[i0 + a][j0 + b] -= acc[a][b];
      }
      __syncthreads();  // column block p-1 is up to date: warp 0 may factor it
    }
    // block row p+1 of U is final (since the last step): warp 4, otherwise idle here, writes it
    if (warp == 4 && p + 1 < LF_NB / LF_P) leaf_store_rows(X, U_hi, U_lo, U32, n, o, (p + 1) * LF_P, lane, 32);
    if (g1) {
      {
        // the rest of the trailing update: S[i][j] -= sum_c V[i][P0+c] V[j][P0+c], i <= j < P0-32
        const int nb2 = (P0 - LF_P) / 4;
        const int ntiles = nb2 > 0 ? nb2 * (nb2 + 1) / 2 : 0;
        for (int t = t1; t < ntiles; t += NG1) {
          int bj = 0, tt = t;
          while (tt > bj) {
            tt -= bj + 1;
            ++bj;
          }
          const int i0 = 4 * tt, j0 = 4 * bj;
          float acc[4][4];
          lf_tile_nt(V, V, i0, j0, P0, P0 + LF_P, acc);
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b)
              if (i0 + a <= j0 + b) S[i0 + a][j0 + b] -= acc[a][b];
        }
      }
      // block row p of the inverse, right of the diagonal block:
      //   U_pj = -Xd_p * sum_{l=p+1..j} V_pl U_lj
      // (S's block row p right of its diagonal block is no longer needed and holds T)
      const int ncols = LF_NB - P0 - LF_P;
      if (ncols > 0) {
        const int nct = ncols / 4;
        // T[r][col] = sum_{k >= P0+32} V[P0+r][k] X[k][col]   (X upper: k <= col)
        for (int item = t1; item < (LF_P / 4) * nct; item += NG1) {
          const int r0 = (item / nct) * 4, col0 = P0 + LF_P + (item % nct) * 4;
          float acc[4][4];
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
          for (int k = P0 + LF_P; k < col0 + 4; ++k) {
            float vv[4], xv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              vv[a] = V[P0 + r0 + a][k];
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
            for (int b = 0; b < 4; ++b) S[P0 + r0 + a][col0 + b] = acc[a][b];
        }
        lf_bar_sync(3, NG1);
        // X[P0+r][col] = -sum_{k >= r} Xd[r][k] T[k][col]
        for (int item = t1; item < (LF_P / 4) * nct; item += NG1) {
          const int r0 = (item / nct) * 4, col0 = P0 + LF_P + (item % nct) * 4;
          float acc[4][4];
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
          for (int k = r0; k < LF_P; ++k) {
            float xd[4], tv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              xd[a] = X[P0 + r0 + a][P0 + k];
              tv[a] = S[P0 + k][col0 + a];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
              for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(xd[a], tv[b], acc[a][b]);
          }
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) X[P0 + r0 + a][col0 + b] = -acc[a][b];
        }
      }
    }
  }
  __syncthreads();

  // block row 0 of U (the others went out during the factorization)
  leaf_store_rows(X, U_hi, U_lo, U32, n, o, 0, tid, LF_THREADS);
  if (tid == 0 && *bad) atomicOr(status, ST_NOT_PD);
}

// U^T of one 128 x 128 diagonal block (hi and lo), 32 x 32 tiles through shared memory:
// Ut[o + c][o + r] = U[o + r][o + c].  Grid (4, 4), block (32, 8).
__global__ void __launch_bounds__(256) transpose_block_kernel(const float* __restrict__ U_hi,
                                                              const float* __restrict__ U_lo, int n, int o,
                                                              float* __restrict__ Ut_hi, float* __restrict__ Ut_lo) {
  __shared__ float th[32][33], tl[32][33];
  griddep_wait();
  griddep_launch_dependents();
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int r0 = o + blockIdx.y * 32, c0 = o + blockIdx.x * 32;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const size_t g = static_cast<size_t>(r0 + ty + 8 * k) * n + c0 + tx;
    th[ty + 8 * k][tx] = U_hi[g];
    tl[ty + 8 * k][tx] = U_lo[g];
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const size_t g = static_cast<size_t>(c0 + ty + 8 * k) * n + r0 + tx;
    Ut_hi[g] = th[tx][ty + 8 * k];
    Ut_lo[g] = tl[tx][ty + 8 * k];
  }
}

}  // namespace gptq
