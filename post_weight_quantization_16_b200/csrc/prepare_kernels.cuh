// prepare_kernels.cuh — S2/S3 and the data movement around the factorization.
//
//   mirror_upper_kernel   H[r][c] = H[c][r] for r > c (the Hessian kernel writes the upper
//                         triangle only)
//   diag_stats_kernel     dead columns (diag H == 0 -> treated as 1), sort keys, mean diag
//                         ("模型量化实战…" §3.2 prepare: damp = 0.01 * mean(diag H))
//   rank_perm_kernel      desc_act: stable descending order of diag H by rank counting
//                         ("GPTQ量化损失深度解析…": desc_act=True, 按敏感度排序)
//   gather_damp_kernel    A = H[perm][:, perm] + damp * mean(diag) * I  (row staged in smem)
//   init_w_kernel         Wq = fp32(W[:, perm]) with dead columns zeroed
//   g_idx_kernel          g_idx[perm[k]] = k / group_size
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "factor_kernels.cuh"

namespace gptq {

// 64 x 64 tiles, 256 threads: a tile of the upper triangle is staged in shared memory and
// written transposed into the lower triangle (the diagonal tile only below its diagonal).
constexpr int MIR_T = 64;
__global__ void __launch_bounds__(256) mirror_upper_kernel(float* __restrict__ H, int n) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float t[MIR_T][MIR_T + 1];
  const int tr = blockIdx.y, tc = blockIdx.x;
  if (tr > tc) return;
  const int x = threadIdx.x, y = threadIdx.y;  // 32 x 8
  for (int k = y; k < MIR_T; k += 8)
    for (int c = x; c < MIR_T; c += 32) t[k][c] = H[static_cast<size_t>(tr * MIR_T + k) * n + tc * MIR_T + c];
  __syncthreads();
  // block (tc, tr) receives the transpose; on the diagonal tile only the strictly lower part
  for (int k = y; k < MIR_T; k += 8)
    for (int c = x; c < MIR_T; c += 32) {
      const int r = tc * MIR_T + k, col = tr * MIR_T + c;
      if (r > col) H[static_cast<size_t>(r) * n + col] = t[c][k];
    }
}

// One CTA of 1024 threads.
__global__ void diag_stats_kernel(const float* __restrict__ H, int n, float* __restrict__ keys,
                                  uint8_t* __restrict__ dead, double* __restrict__ mean_out) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float d = H[static_cast<size_t>(i) * n + i];
    const bool z = (d == 0.0f);
    // a NaN diagonal sorts last (keys must be totally ordered for the rank permutation)
    const float k = z ? 1.0f : (d == d ? d : -INFINITY);
    keys[i] = k;
    dead[i] = z ? 1 : 0;
    s += static_cast<double>(k);
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) *mean_out = v / static_cast<double>(n);
  }
}

// perm[rank(i)] = i with rank(i) = #{j : key_j > key_i or (key_j == key_i and j < i)}.  One warp
// per element: the lanes count over the keys four at a time (float4, n % 128 == 0), then a warp
// sum.  Grid: ceil(n / 8) CTAs of 256 threads.
__global__ void __launch_bounds__(256) rank_perm_kernel(const float* __restrict__ keys, int n,
                                                        int32_t* __restrict__ perm) {
  griddep_wait();
  griddep_launch_dependents();
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (i >= n) return;
  const float ki = keys[i];
  int rank = 0;
  const float4* k4 = reinterpret_cast<const float4*>(keys);
  for (int q = lane; q < n / 4; q += 32) {
    const float4 v = __ldg(k4 + q);
    const int j = 4 * q;
    rank += (v.x > ki) || (v.x == ki && j < i);
    rank += (v.y > ki) || (v.y == ki && j + 1 < i);
    rank += (v.z > ki) || (v.z == ki && j + 2 < i);
    rank += (v.w > ki) || (v.w == ki && j + 3 < i);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
  if (lane == 0) perm[rank] = i;
}

__global__ void identity_perm_kernel(int n, int32_t* __restrict__ perm) {
  griddep_wait();
  griddep_launch_dependents();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) perm[i] = i;
}

// One CTA (1024 threads) per output row a: the source row perm[a] of the (mirrored) H is
// staged in shared memory, then gathered by perm four columns at a time (16-byte loads of
// perm, 16-byte stores of the hi and lo parts).  n % 4 == 0.
constexpr int GD_THREADS = 1024;
__global__ void __launch_bounds__(GD_THREADS) gather_damp_kernel(const float* __restrict__ H, int n,
                                                                 const int32_t* __restrict__ perm,
                                                                 const float* __restrict__ keys,
                                                                 const double* __restrict__ mean, double damp,
                                                                 float* __restrict__ A_hi, float* __restrict__ A_lo) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ float row_s[];
  const int a = blockIdx.x;
  const int pa = perm[a];
  const float4* src = reinterpret_cast<const float4*>(H + static_cast<size_t>(pa) * n);
  for (int k = threadIdx.x; k < n / 4; k += blockDim.x) reinterpret_cast<float4*>(row_s)[k] = src[k];
  const float dval = static_cast<float>(static_cast<double>(keys[pa]) + damp * (*mean));
  __syncthreads();
  float4* dh = reinterpret_cast<float4*>(A_hi + static_cast<size_t>(a) * n);
  float4* dl = reinterpret_cast<float4*>(A_lo + static_cast<size_t>(a) * n);
  const int4* p4 = reinterpret_cast<const int4*>(perm);
  for (int b4 = threadIdx.x; b4 < n / 4; b4 += blockDim.x) {
    const int4 pb = p4[b4];
    float v[4] = {row_s[pb.x], row_s[pb.y], row_s[pb.z], row_s[pb.w]};
    float hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (4 * b4 + e == a) v[e] = dval;
      hi[e] = tf32_round(v[e]);
      lo[e] = tf32_round(v[e] - hi[e]);
    }
    dh[b4] = make_float4(hi[0], hi[1], hi[2], hi[3]);
    dl[b4] = make_float4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// One CTA per row r: Wq[r][k] = dead[perm[k]] ? 0 : float(W[r][perm[k]]), and the same weights
// kept in fp16 (exact) in W0h when it is given.
__global__ void init_w_kernel(const __half* __restrict__ W, int n, const int32_t* __restrict__ perm,
                              const uint8_t* __restrict__ dead, float* __restrict__ Wq, __half* __restrict__ W0h) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __half wrow_s[];
  const int r = blockIdx.x;
  const __half* src = W + static_cast<size_t>(r) * n;
  for (int k = threadIdx.x; k < n; k += blockDim.x) wrow_s[k] = src[k];
  __syncthreads();
  float* dst = Wq + static_cast<size_t>(r) * n;
  __half* dst0 = W0h ? W0h + static_cast<size_t>(r) * n : nullptr;
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const int p = perm[k];
    const __half w = dead[p] ? __float2half_rn(0.0f) : wrow_s[p];
    dst[k] = __half2float(w);
    if (dst0) dst0[k] = w;
  }
}

// out = hi + lo (the fp32 value of a hi/lo pair)
__global__ void combine_hilo_kernel(const float* __restrict__ hi, const float* __restrict__ lo, size_t count,
                                    float* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    out[i] = hi[i] + lo[i];
}

__global__ void g_idx_kernel(const int32_t* __restrict__ perm, int n, int g, int32_t* __restrict__ g_idx) {
  griddep_wait();
  griddep_launch_dependents();
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < n) g_idx[perm[k]] = k / g;
}

}  // namespace gptq
