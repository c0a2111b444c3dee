// sgemm_simt.cuh — fp32 CUDA-core GEMM used by the factorization and the lazy trailing
// update:  C = beta * C + alpha * A * op(B)
//   A    : [M x K] row-major (lda)
//   op(B): B [K x N] row-major (ldb)            when TRANS_B == false
//          B^T with B stored [N x K] row-major  when TRANS_B == true
//   C    : [M x N] row-major (ldc)
// UPPER_ONLY skips output tiles that lie entirely below the diagonal of C (for symmetric
// updates where only the upper triangle is consumed).
// Requirements (checked by the host): K % 16 == 0, N % 4 == 0, lda/ldb/ldc % 4 == 0 and
// 16-byte aligned base pointers.  M and N tails are masked.
//
// 128 x 128 x 16 tiles, 256 threads, 8 x 8 outputs per thread, register-prefetched double
// buffering of the shared-memory tiles.
#pragma once

#include <cstdint>

namespace gptq {

constexpr int SG_BM = 128, SG_BN = 128, SG_BK = 16, SG_THREADS = 256;

template <bool TRANS_B>
__global__ void __launch_bounds__(SG_THREADS)
    sgemm_kernel(int M, int N, int K, float alpha, const float* __restrict__ A, int lda,
                 const float* __restrict__ B, int ldb, float beta, float* __restrict__ C, int ldc,
                 int upper_only) {
  const int m0 = blockIdx.y * SG_BM;
  const int n0 = blockIdx.x * SG_BN;
  if (upper_only && m0 >= n0 + SG_BN) return;

  __shared__ __align__(16) float As[2][SG_BK][SG_BM + 4];
  __shared__ __align__(16) float Bs[2][SG_BK][SG_BN + 4];

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  // global -> register staging: A (and B^T) tiles: row = tid/4 (+64), k quad = (tid%4)*4
  const int a_row = tid >> 2, a_k = (tid & 3) * 4;
  // B (row-major K x N) tiles: k = tid/32 (+8), n quad = (tid%32)*4
  const int b_k = tid >> 5, b_n = (tid & 31) * 4;

  float4 ra[2], rb[2];
  auto load_tiles = [&](int k0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = m0 + a_row + 64 * h;
      ra[h] = (row < M) ? *reinterpret_cast<const float4*>(A + static_cast<size_t>(row) * lda + k0 + a_k)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (TRANS_B) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = n0 + a_row + 64 * h;
        rb[h] = (col < N) ? *reinterpret_cast<const float4*>(B + static_cast<size_t>(col) * ldb + k0 + a_k)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    } else {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int kk = k0 + b_k + 8 * h;
        const int col = n0 + b_n;
        rb[h] = (col < N) ? *reinterpret_cast<const float4*>(B + static_cast<size_t>(kk) * ldb + col)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  auto store_tiles = [&](int buf) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = a_row + 64 * h;
      As[buf][a_k + 0][row] = ra[h].x;
      As[buf][a_k + 1][row] = ra[h].y;
      As[buf][a_k + 2][row] = ra[h].z;
      As[buf][a_k + 3][row] = ra[h].w;
    }
    if (TRANS_B) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = a_row + 64 * h;
        Bs[buf][a_k + 0][col] = rb[h].x;
        Bs[buf][a_k + 1][col] = rb[h].y;
        Bs[buf][a_k + 2][col] = rb[h].z;
        Bs[buf][a_k + 3][col] = rb[h].w;
      }
    } else {
#pragma unroll
      for (int h = 0; h < 2; ++h) *reinterpret_cast<float4*>(&Bs[buf][b_k + 8 * h][b_n]) = rb[h];
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int nk = K / SG_BK;
  load_tiles(0);
  store_tiles(0);
  __syncthreads();
  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) load_tiles((kt + 1) * SG_BK);
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4 + 64]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4 + 64]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (kt + 1 < nk) {
      store_tiles(buf ^ 1);
      __syncthreads();
    }
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = m0 + ty * 4 + (i & 3) + 64 * (i >> 2);
    if (row >= M) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int col = n0 + tx * 4 + 64 * h;
      if (col >= N) continue;
      float4* cp = reinterpret_cast<float4*>(C + static_cast<size_t>(row) * ldc + col);
      float4 o;
      o.x = alpha * acc[i][4 * h + 0];
      o.y = alpha * acc[i][4 * h + 1];
      o.z = alpha * acc[i][4 * h + 2];
      o.w = alpha * acc[i][4 * h + 3];
      if (beta != 0.f) {
        const float4 c = *cp;
        o.x = fmaf(beta, c.x, o.x);
        o.y = fmaf(beta, c.y, o.y);
        o.z = fmaf(beta, c.z, o.z);
        o.w = fmaf(beta, c.w, o.w);
      }
      *cp = o;
    }
  }
}

}  // namespace gptq
