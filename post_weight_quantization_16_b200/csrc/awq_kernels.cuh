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
// With s = 1 the last kernel is plain round-to-nearest of W.  It also serves the round-to-nearest
// quantizer with a clip ratio below 1 ("模型量化实战…" §3.1 LinearQuantizer, clip_ratio): each
// group's range is then a pair of percentiles (of |w| for symmetric codes) instead of its min and
// max, found by selecting the order statistics around the percentile's position.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sweep_kernels.cuh"

namespace gptq {

constexpr int AWQ_SUM_COLS = 256;  // columns per warp pass (8 bf16 per lane)

// |x| of the 8 bf16 values in v added into acc (fp64).
__device__ __forceinline__ void add_abs8(double* acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    acc[2 * k] += fabs(static_cast<double>(__uint_as_float(w[k] << 16)));
    acc[2 * k + 1] += fabs(static_cast<double>(__uint_as_float(w[k] & 0xFFFF0000u)));
  }
}

// grid (ceil(n / 256), token splits), block (32, 8): lane owns 8 consecutive columns, the 8 warps
// and the grid's y dimension split the tokens; each thread keeps four rows' loads in flight
// before adding them; fp64 partial sums are added atomically.
__global__ void __launch_bounds__(256) channel_abs_sum_kernel(const __nv_bfloat16* __restrict__ X, int64_t n_tok,
                                                              int64_t ld, int n, double* __restrict__ sums) {
  const int c0 = blockIdx.x * AWQ_SUM_COLS + threadIdx.x * 8;
  if (c0 >= n) return;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const int64_t step = static_cast<int64_t>(blockDim.y) * gridDim.y;
  int64_t t = static_cast<int64_t>(blockIdx.y) * blockDim.y + threadIdx.y;
  for (; t + 3 * step < n_tok; t += 4 * step) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const uint4*>(X + (t + u * step) * ld + c0);
#pragma unroll
    for (int u = 0; u < 4; ++u) add_abs8(acc, v[u]);
  }
  for (; t < n_tok; t += step) add_abs8(acc, *reinterpret_cast<const uint4*>(X + t * ld + c0));
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
  const float* scale;  // [n] channel scale, or nullptr for 1
  int m, n, bits, sym, g, G;
  uint32_t* codes;     // [m x n*bits/32], original column order
  float* scales;       // [m x G]
  float* zeros;        // [m x G]
  float* W_hat;        // [m x n] or nullptr
  // percentile range (clip != 0): the ranks of the order statistics that bound the lower (0, 1)
  // and upper (2, 3) percentile, and each percentile's interpolation weight t and 1 - t
  int clip;
  int rank[4];
  float t_lo, omt_lo, t_hi, omt_hi;
};

// Order-preserving key of a float: unsigned comparison of keys is the float order (-0 sorts just
// below +0, which the interpolation below cannot tell apart).
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// The percentile between order statistics a <= b at weight t (numpy's linear method in fp32):
// a + (b - a) t below t = 1/2, b - (b - a)(1 - t) from there (exact at both ends).
__device__ __forceinline__ float pct_lerp(float a, float b, float t, float omt) {
  const float d = __fsub_rn(b, a);
  return t < 0.5f ? __fadd_rn(a, __fmul_rn(d, t)) : __fsub_rn(b, __fmul_rn(d, omt));
}

// Keys of the values of ranks r[0..3] (0 = smallest) among v[0..g) (|v| for sym), by bisection on
// the key: the value of rank r has the least key K with at least r + 1 values at or below K, and
// 32 halvings of [0, 2^32) isolate it.  A team of `team` threads (lane `lane` of it) shares the
// counting; `reduce` sums a count over the team.
template <class Reduce>
__device__ __forceinline__ void select_ranks(const float* v, int g, int sym, const int* r, int lane, int team,
                                             Reduce reduce, uint32_t* key) {
  uint32_t lo[4] = {0u, 0u, 0u, 0u}, hi[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
#pragma unroll 1
  for (int it = 0; it < 32; ++it) {
    uint32_t mid[4];
    int cnt[4] = {0, 0, 0, 0};
#pragma unroll
    for (int t = 0; t < 4; ++t) mid[t] = lo[t] + ((hi[t] - lo[t]) >> 1);
    for (int j = lane; j < g; j += team) {
      const float x = v[j];
      const uint32_t k = order_key(sym ? fabsf(x) : x);
#pragma unroll
      for (int t = 0; t < 4; ++t) cnt[t] += (k <= mid[t]) ? 1 : 0;
    }
    reduce(cnt, it);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (cnt[t] >= r[t] + 1)
        hi[t] = mid[t];
      else
        lo[t] = mid[t] + 1u;
    }
  }
#pragma unroll
  for (int t = 0; t < 4; ++t) key[t] = lo[t];
}

// One CTA (256 threads) per row: the scaled row in shared memory, one warp per group for the
// min-max reduction, then one thread per output word (group boundaries are word boundaries:
// g * bits is a multiple of 32).  With a clip ratio, the percentiles' order statistics are
// selected first: one warp per group when the row has at least 8 groups, else the whole CTA
// per group.
__global__ void __launch_bounds__(256) awq_rtn_kernel(AwqRtnArgs a) {
  extern __shared__ float awq_row[];  // n scaled weights, then G scales, G zeros, 4 G order statistics
  __shared__ int red[2 * 8 * 4];      // the CTA-wide selection's per-warp counts (two iterations' worth)
  float* gs = awq_row + a.n;
  float* gz = gs + a.G;
  float* sel = gz + a.G;
  const int r = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const __half* src = a.W + static_cast<size_t>(r) * a.n;
  for (int k = tid; k < a.n; k += blockDim.x)
    awq_row[k] = a.scale ? __fmul_rn(__half2float(src[k]), a.scale[k]) : __half2float(src[k]);
  __syncthreads();
  if (a.clip) {
    uint32_t key[4];
    if (a.G >= 8) {
      auto warp_sum = [](int* cnt, int) {
#pragma unroll
        for (int t = 0; t < 4; ++t)
          for (int o = 16; o > 0; o >>= 1) cnt[t] += __shfl_xor_sync(0xffffffffu, cnt[t], o);
      };
      for (int gi = warp; gi < a.G; gi += blockDim.x / 32) {
        select_ranks(awq_row + gi * a.g, a.g, a.sym, a.rank, lane, 32, warp_sum, key);
        if (lane == 0)
#pragma unroll
          for (int t = 0; t < 4; ++t) sel[4 * gi + t] = key_value(key[t]);
      }
    } else {
      const int nw = blockDim.x / 32;
      auto cta_sum = [&](int* cnt, int it) {
#pragma unroll
        for (int t = 0; t < 4; ++t)
          for (int o = 16; o > 0; o >>= 1) cnt[t] += __shfl_xor_sync(0xffffffffu, cnt[t], o);
        int* rb = red + (it & 1) * 32;
        if (lane == 0)
#pragma unroll
          for (int t = 0; t < 4; ++t) rb[warp * 4 + t] = cnt[t];
        __syncthreads();
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          int s = 0;
          for (int w = 0; w < nw; ++w) s += rb[w * 4 + t];
          cnt[t] = s;
        }
      };
      for (int gi = 0; gi < a.G; ++gi) {
        select_ranks(awq_row + gi * a.g, a.g, a.sym, a.rank, tid, blockDim.x, cta_sum, key);
        if (tid == 0)
#pragma unroll
          for (int t = 0; t < 4; ++t) sel[4 * gi + t] = key_value(key[t]);
      }
    }
    __syncthreads();
  }
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
    if (a.clip) {
      const float* q = sel + 4 * gi;
      wmin = pct_lerp(q[0], q[1], a.t_lo, a.omt_lo);
      wmax = pct_lerp(q[2], q[3], a.t_hi, a.omt_hi);
      amax = wmin;  // symmetric codes: the one percentile, of |w|
    } else {
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
        a.W_hat[static_cast<size_t>(r) * a.n + k] =
            a.scale ? __fdiv_rn(__fmul_rn(__fsub_rn(q, zs), s), a.scale[k]) : __fmul_rn(__fsub_rn(q, zs), s);
    }
    a.codes[static_cast<size_t>(r) * words + wi] = word;
  }
}

}  // namespace gptq
