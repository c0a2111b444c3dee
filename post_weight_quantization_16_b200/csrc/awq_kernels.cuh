// awq_kernels.cuh — activation-aware channel scaling before round-to-nearest (AWQ), on the
// same calibration activations and weights as the GPTQ path.
//
// ("大模型量化：GPTQ/AWQ/GGUF 原理对比，4-bit 量化对推理精度的影响", AWQ section: the importance
//  of an input channel is its mean |x| over the calibration tokens; the channels above the
//  median importance are multiplied by s before quantization, so they get finer steps; the
//  dequantized weights are divided by the scale again, and the activations by s at inference.)
//
//   channel_abs_sum_kernel  sum_t |X[t][c]| in fp64 (exact for bf16 inputs of ordinary range,
//                           so the result does not depend on the order of the additions)
//   awq_median_kernel       the lower median of the importances by rank counting
//   awq_scale_kernel        scale[c] = s if importance[c] > median else 1
//   awq_rtn_kernel          per row: W' = fp32(W) * scale, min-max group parameters in original
//                           column order, round-to-nearest codes packed LSB-first, optional
//                           dequantized weights (u - z) * s_g / scale
// With s = 1 the last kernel is plain round-to-nearest of W.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sweep_kernels.cuh"

namespace gptq {

constexpr int AWQ_SUM_COLS = 256;  // columns per warp pass (8 bf16 per lane)

// grid (ceil(n / 256), token splits), block (32, 8): lane owns 8 consecutive columns, the 8 warps
// and the grid's y dimension split the tokens; fp64 partial sums are added atomically.
__global__ void __launch_bounds__(256) channel_abs_sum_kernel(const __nv_bfloat16* __restrict__ X, int64_t n_tok,
                                                              int64_t ld, int n, double* __restrict__ sums) {
  const int c0 = blockIdx.x * AWQ_SUM_COLS + threadIdx.x * 8;
  if (c0 >= n) return;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const int64_t step = static_cast<int64_t>(blockDim.y) * gridDim.y;
  for (int64_t t = static_cast<int64_t>(blockIdx.y) * blockDim.y + threadIdx.y; t < n_tok; t += step) {
    const uint4 v = *reinterpret_cast<const uint4*>(X + t * ld + c0);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[2 * k] += fabs(static_cast<double>(__uint_as_float(w[k] << 16)));
      acc[2 * k + 1] += fabs(static_cast<double>(__uint_as_float(w[k] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (acc[k] != 0.0) atomicAdd(sums + c0 + k, acc[k]);
}

// The element of rank (n - 1) / 2 in ascending order (ties by index): the lower median.
__global__ void __launch_bounds__(256) awq_median_kernel(const double* __restrict__ sums, int n,
                                                         double* __restrict__ median) {
  __shared__ double vs[1024];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const double vi = (i < n) ? sums[i] : 0.0;
  int rank = 0;
  for (int j0 = 0; j0 < n; j0 += 1024) {
    __syncthreads();
    for (int t = threadIdx.x; t < 1024; t += blockDim.x) vs[t] = (j0 + t < n) ? sums[j0 + t] : 0.0;
    __syncthreads();
    const int jn = min(1024, n - j0);
    for (int t = 0; t < jn; ++t) {
      const double vj = vs[t];
      rank += (vj < vi) || (vj == vi && j0 + t < i);
    }
  }
  if (i < n && rank == (n - 1) / 2) *median = vi;
}

// importance = sum / n_tok (fp64); scale = s_protect above the median, 1 elsewhere.
__global__ void awq_scale_kernel(const double* __restrict__ sums, int n, int64_t n_tok, const double* __restrict__ median,
                                 float s_protect, float* __restrict__ scale) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const double d = static_cast<double>(n_tok > 0 ? n_tok : 1);
  scale[i] = (sums[i] / d > *median / d) ? s_protect : 1.0f;
}

struct AwqRtnArgs {
  const __half* W;     // [m x n] fp16
  const float* scale;  // [n] channel scale
  int m, n, bits, sym, g, G;
  uint32_t* codes;     // [m x n*bits/32], original column order
  float* scales;       // [m x G]
  float* zeros;        // [m x G]
  float* W_hat;        // [m x n] or nullptr
};

// One CTA (256 threads) per row: the scaled row in shared memory, one warp per group for the
// min-max reduction, then one thread per output word (group boundaries are word boundaries:
// g * bits is a multiple of 32).
__global__ void __launch_bounds__(256) awq_rtn_kernel(AwqRtnArgs a) {
  extern __shared__ float awq_row[];  // n scaled weights, then G scales and G zeros
  float* gs = awq_row + a.n;
  float* gz = gs + a.G;
  const int r = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const __half* src = a.W + static_cast<size_t>(r) * a.n;
  for (int k = tid; k < a.n; k += blockDim.x) awq_row[k] = __fmul_rn(__half2float(src[k]), a.scale[k]);
  __syncthreads();
  QParams qp;
  if (a.sym) {
    qp.lo = -static_cast<float>(1 << (a.bits - 1));
    qp.hi = static_cast<float>((1 << (a.bits - 1)) - 1);
  } else {
    qp.lo = 0.0f;
    qp.hi = static_cast<float>((1 << a.bits) - 1);
  }
  qp.qmax_f = qp.hi;
  qp.zsym = static_cast<float>(1 << (a.bits - 1));
  for (int gi = warp; gi < a.G; gi += blockDim.x / 32) {
    float wmin = INFINITY, wmax = -INFINITY, amax = 0.0f;
    for (int k = gi * a.g + lane; k < (gi + 1) * a.g; k += 32) {
      const float x = awq_row[k];
      wmin = fminf(wmin, x);
      wmax = fmaxf(wmax, x);
      amax = fmaxf(amax, fabsf(x));
    }
    for (int o = 16; o > 0; o >>= 1) {
      wmin = fminf(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
      wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    }
    float s, z;
    group_scale_zero(wmin, wmax, amax, qp, a.sym, s, z);
    if (lane == 0) {
      gs[gi] = s;
      gz[gi] = z;
      a.scales[static_cast<size_t>(r) * a.G + gi] = s;
      a.zeros[static_cast<size_t>(r) * a.G + gi] = z;
    }
  }
  __syncthreads();
  const int words = a.n * a.bits / 32;
  const float rnd = 12582912.0f;  // 1.5 * 2^23: adding and subtracting it rounds half-to-even
  for (int wi = tid; wi < words; wi += blockDim.x) {
    const int b0 = 32 * wi;
    const int k0 = b0 / a.bits, k1 = (b0 + 31) / a.bits;  // codes that touch this word
    const int gi = k0 / a.g;                              // one group per word
    const float s = gs[gi], z = gz[gi];
    const float zs = a.sym ? 0.0f : z;
    const float rs = __frcp_rn(s);
    uint32_t word = 0u;
    for (int k = k0; k <= k1 && k < a.n; ++k) {
      const float x = awq_row[k];
      const float v = __fadd_rn(div_rn(x, s, rs), zs);
      const float q = __fsub_rn(__fadd_rn(fminf(fmaxf(v, qp.lo), qp.hi), rnd), rnd);
      const uint32_t code = static_cast<uint32_t>(static_cast<int>(q - qp.lo));
      const int pos = k * a.bits - b0;
      word |= (pos >= 0) ? (code << pos) : (code >> (-pos));
      if (a.W_hat && k * a.bits >= b0)  // each code's dequantized value written once, by its first word
        a.W_hat[static_cast<size_t>(r) * a.n + k] = __fdiv_rn(__fmul_rn(__fsub_rn(q, zs), s), a.scale[k]);
    }
    a.codes[static_cast<size_t>(r) * words + wi] = word;
  }
}

}  // namespace gptq
