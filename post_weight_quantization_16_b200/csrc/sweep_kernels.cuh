// sweep_kernels.cuh — S5/S7: one 128-column block of the GPTQ column sweep.
//
// ("大模型量化：GPTQ/AWQ/GGUF 原理对比…" GPTQ section: quantize column by column and push
//  each column's error into the not-yet-quantized columns; "模型量化实战…" §3.2
//  quantize_block: blocks of 128 columns.)
//
// Rows of W are independent once U is known, so each thread owns one row.  The row's 128
// block columns live in registers as eight 16-column sub-blocks R[0..7]; the U block
// (upper 128 x 128) is in shared memory and every U read is a warp-wide broadcast.
// For sub-block sb the thread
//   1. (re)computes the group's min-max scale/zero from the current values when a group
//      starts (groups of 32/64 inside the block; groups >= 128 at block starts),
//   2. quantizes the 16 columns in order, e = (w - q) / U[i,i], and updates the remaining
//      columns of the sub-block,
//   3. applies the 16 errors to the later sub-blocks of the block (a 16 x 16 rank update
//      each), then rotates the registers so the next sub-block is R[0].
// The errors of the whole block go to Err [m x 128]; the columns after the block receive
// them through one GEMM per block (S6) launched by the host.
//
// The integer decisions (code and zero-point) are taken in fp32 with IEEE division and
// round-half-to-even, the precision the pages' own sketches use.
#pragma once

#include <cstdint>

#include "factor_kernels.cuh"

namespace gptq {

constexpr int SW_B = 128;       // sweep block (columns)
constexpr int SW_THREADS = 32;  // rows per CTA
constexpr int SW_SMEM = SW_B * SW_B * 4 + SW_B * 4 + SW_B * 4 + SW_B * SW_THREADS;

struct SweepArgs {
  float* Wq;          // [m x n] fp32 working weights, sweep order
  const float* U;     // [n x n] upper factor (fp32, or the tf32 hi part when U_lo is set)
  const float* U_lo;  // [n x n] tf32 lo part of U, or nullptr
  float* Err;         // [m x 128] scaled errors of the current block (fp32, or hi part)
  float* Err_lo;      // [m x 128] tf32 lo part of the errors, or nullptr
  uint32_t* codes;    // [m x n*bits/32]
  float* scales;      // [m x G]
  float* zeros;       // [m x G]
  float* W_hat;       // [m x n] original order, or nullptr
  const int32_t* perm;
  int m, n, bits, sym, g, G;
};

struct QParams {
  float lo, hi;      // integer code range (signed for sym)
  float qmax_f;      // 2^b - 1 (asym) or 2^(b-1) - 1 (sym)
  float zsym;        // 2^(b-1)
};

__device__ __forceinline__ void group_scale_zero(float wmin, float wmax, float amax, const QParams& qp, int sym,
                                                 float& s, float& z) {
  if (sym) {
    s = fmaxf(__fdiv_rn(amax, qp.qmax_f), 1e-8f);
    z = qp.zsym;
  } else {
    const float xmin = fminf(wmin, 0.0f);
    const float xmax = fmaxf(wmax, 0.0f);
    s = fmaxf(__fdiv_rn(__fsub_rn(xmax, xmin), qp.qmax_f), 1e-8f);
    z = -rintf(__fdiv_rn(xmin, s));
  }
}

template <int GSUB>  // 0: groups of >= 128 columns (params at block starts); 32 or 64: inside the block
__global__ void __launch_bounds__(SW_THREADS)
    sweep_block_kernel(SweepArgs a, int i1) {
  extern __shared__ __align__(16) float sw_smem[];
  float* Us = sw_smem;                                        // [128][128]
  float* rU = Us + SW_B * SW_B;                               // [128] 1 / U[i][i]
  int* perm_s = reinterpret_cast<int*>(rU + SW_B);            // [128]
  uint8_t* code_s = reinterpret_cast<uint8_t*>(perm_s + SW_B);  // [128][32]

  const int lane = threadIdx.x;
  const int n = a.n;
  for (int idx = lane; idx < SW_B * SW_B / 4; idx += SW_THREADS) {
    const int k = idx / (SW_B / 4), j4 = idx % (SW_B / 4);
    const size_t g = static_cast<size_t>(i1 + k) * n + i1 + 4 * j4;
    float4 u = *reinterpret_cast<const float4*>(a.U + g);
    if (a.U_lo) {
      const float4 l = *reinterpret_cast<const float4*>(a.U_lo + g);
      u.x += l.x;
      u.y += l.y;
      u.z += l.z;
      u.w += l.w;
    }
    reinterpret_cast<float4*>(Us)[idx] = u;
  }
  for (int k = lane; k < SW_B; k += SW_THREADS) perm_s[k] = a.perm[i1 + k];
  __syncthreads();
  for (int k = lane; k < SW_B; k += SW_THREADS) rU[k] = 1.0f / Us[k * SW_B + k];
  __syncthreads();

  const int r = blockIdx.x * SW_THREADS + lane;
  const bool valid = r < a.m;
  const int rr = valid ? r : 0;

  QParams qp;
  if (a.sym) {
    qp.lo = -static_cast<float>(1 << (a.bits - 1));
    qp.hi = static_cast<float>((1 << (a.bits - 1)) - 1);
    qp.qmax_f = qp.hi;
  } else {
    qp.lo = 0.0f;
    qp.hi = static_cast<float>((1 << a.bits) - 1);
    qp.qmax_f = qp.hi;
  }
  qp.zsym = static_cast<float>(1 << (a.bits - 1));

  float R[8][16];
  {
    const float4* src = reinterpret_cast<const float4*>(a.Wq + static_cast<size_t>(rr) * n + i1);
#pragma unroll
    for (int t = 0; t < 8; ++t)
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        const float4 v = valid ? src[t * 4 + j4] : make_float4(0.f, 0.f, 0.f, 0.f);
        R[t][4 * j4 + 0] = v.x;
        R[t][4 * j4 + 1] = v.y;
        R[t][4 * j4 + 2] = v.z;
        R[t][4 * j4 + 3] = v.w;
      }
  }

  float s = 1.0f, z = 0.0f;
  if (GSUB == 0) {
    const int gi = i1 / a.g;
    if (i1 % a.g == 0) {
      float wmin = R[0][0], wmax = R[0][0], amax = 0.0f;
#pragma unroll
      for (int t = 0; t < 8; ++t)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          wmin = fminf(wmin, R[t][j]);
          wmax = fmaxf(wmax, R[t][j]);
          amax = fmaxf(amax, fabsf(R[t][j]));
        }
      if (valid) {
        const float* rest = a.Wq + static_cast<size_t>(rr) * n;
        for (int c = i1 + SW_B; c < i1 + a.g; ++c) {
          const float w = rest[c];
          wmin = fminf(wmin, w);
          wmax = fmaxf(wmax, w);
          amax = fmaxf(amax, fabsf(w));
        }
      }
      group_scale_zero(wmin, wmax, amax, qp, a.sym, s, z);
      if (valid) {
        a.scales[static_cast<size_t>(rr) * a.G + gi] = s;
        a.zeros[static_cast<size_t>(rr) * a.G + gi] = z;
      }
    } else if (valid) {
      s = a.scales[static_cast<size_t>(rr) * a.G + gi];
      z = a.zeros[static_cast<size_t>(rr) * a.G + gi];
    }
  }

  float* err_row = a.Err + static_cast<size_t>(rr) * SW_B;
  float* what_row = a.W_hat ? a.W_hat + static_cast<size_t>(rr) * n : nullptr;

#pragma unroll 1
  for (int sb = 0; sb < 8; ++sb) {
    const int c0 = sb * 16;  // first block column of R[0]
    if (GSUB > 0 && (c0 % (GSUB > 0 ? GSUB : 1)) == 0) {
      constexpr int NT = (GSUB > 0 ? GSUB : 16) / 16;
      float wmin = R[0][0], wmax = R[0][0], amax = 0.0f;
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          wmin = fminf(wmin, R[t][j]);
          wmax = fmaxf(wmax, R[t][j]);
          amax = fmaxf(amax, fabsf(R[t][j]));
        }
      group_scale_zero(wmin, wmax, amax, qp, a.sym, s, z);
      if (valid) {
        const int gi = (i1 + c0) / a.g;
        a.scales[static_cast<size_t>(rr) * a.G + gi] = s;
        a.zeros[static_cast<size_t>(rr) * a.G + gi] = z;
      }
    }

    float E[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float w = R[0][k];
      float v = __fdiv_rn(w, s);
      if (!a.sym) v = __fadd_rn(v, z);
      const float q = fminf(fmaxf(rintf(v), qp.lo), qp.hi);
      const float what = a.sym ? __fmul_rn(q, s) : __fmul_rn(__fsub_rn(q, z), s);
      code_s[(c0 + k) * SW_THREADS + lane] = static_cast<uint8_t>(static_cast<int>(q - qp.lo));
      const float e = __fmul_rn(__fsub_rn(w, what), rU[c0 + k]);
      E[k] = e;
      if (what_row && valid) what_row[perm_s[c0 + k]] = what;
      const float* urow = Us + (c0 + k) * SW_B + c0;
#pragma unroll
      for (int j = k + 1; j < 16; ++j) R[0][j] = fmaf(-e, urow[j], R[0][j]);
    }
    if (valid) {
      float4* ep = reinterpret_cast<float4*>(err_row + c0);
      if (a.Err_lo) {
        float4* lp = reinterpret_cast<float4*>(a.Err_lo + static_cast<size_t>(rr) * SW_B + c0);
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          float hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            hi[e] = tf32_round(E[4 * j4 + e]);
            lo[e] = tf32_round(E[4 * j4 + e] - hi[e]);
          }
          ep[j4] = make_float4(hi[0], hi[1], hi[2], hi[3]);
          lp[j4] = make_float4(lo[0], lo[1], lo[2], lo[3]);
        }
      } else {
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) ep[j4] = make_float4(E[4 * j4], E[4 * j4 + 1], E[4 * j4 + 2], E[4 * j4 + 3]);
      }
    }
#pragma unroll
    for (int t = 1; t < 8; ++t) {
      if (sb + t < 8) {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float4* urow = reinterpret_cast<const float4*>(Us + (c0 + k) * SW_B + c0 + 16 * t);
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const float4 u = urow[j4];
            R[t][4 * j4 + 0] = fmaf(-E[k], u.x, R[t][4 * j4 + 0]);
            R[t][4 * j4 + 1] = fmaf(-E[k], u.y, R[t][4 * j4 + 1]);
            R[t][4 * j4 + 2] = fmaf(-E[k], u.z, R[t][4 * j4 + 2]);
            R[t][4 * j4 + 3] = fmaf(-E[k], u.w, R[t][4 * j4 + 3]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 7; ++t)
#pragma unroll
      for (int j = 0; j < 16; ++j) R[t][j] = R[t + 1][j];
  }

  // pack this row's 128 codes (LSB-first bit stream) and store them
  __syncwarp();
  if (valid) {
    const int bits = a.bits;
    const int words = 4 * bits;  // 128 * bits / 32
    const int ldc = n * bits / 32;
    uint32_t* dst = a.codes + static_cast<size_t>(rr) * ldc + (i1 * bits) / 32;
    for (int w = 0; w < words; ++w) {
      const int bit0 = w * 32;
      const int k0 = bit0 / bits, k1 = (bit0 + 31) / bits;
      uint32_t acc = 0;
      for (int k = k0; k <= k1; ++k) {
        const uint32_t c = code_s[k * SW_THREADS + lane];
        const int pos = k * bits - bit0;
        acc |= (pos >= 0) ? (c << pos) : (c >> (-pos));
      }
      dst[w] = acc;
    }
  }
}

}  // namespace gptq
