// sweep_kernels.cuh — S5/S7: one 128-column block of the GPTQ column sweep.
//
// ("大模型量化：GPTQ/AWQ/GGUF 原理对比…" GPTQ section: quantize column by column and push
//  each column's error into the not-yet-quantized columns; "模型量化实战…" §3.2
//  quantize_block: blocks of 128 columns.)
//
// Rows of W are independent once U is known.  A CTA takes 32 rows and keeps their 128
// block columns in shared memory.  The block is walked in eight chunks of 16 columns:
//   * warp 0, the walker, gives each lane one row.  For chunk k it loads the row's 16
//     values, applies the previous chunk's errors to them, then walks the 16 columns:
//     code, dequantized value, e = (w - q) / U[i][i], and w[j] -= e * U[i][j] for the
//     chunk's later columns.  The per-column dependent chain stays in the lane's registers
//     and every U value it needs is the same for all 32 lanes (a broadcast read).
//   * warps 1-3, the updaters, apply chunk k's errors to chunks k+2 .. 7 of the tile while
//     the walker is on chunk k+1 (a rank-16 update in shared memory).
// Named barriers hand each chunk's errors to the updaters and each finished update back to
// the walker.  Group scales/zeros come from a min/max over the group's current values.  The
// U block (128 x 128, hi + lo) is staged in shared memory before the kernel waits on its
// predecessor, so the staging overlaps the previous kernel's tail.  At the end the CTA writes
// the block's errors to Err, the packed code words and the dequantized weights row by row.
// The columns after the block receive the errors through tensor-core products (S6) launched
// by the host: within a super-block of columns right after each block, beyond it once per
// super-block.
//
// The integer decisions (code and zero-point) are taken in fp32 with correctly rounded
// division and round-half-to-even, the precision the pages' own sketches use.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "factor_kernels.cuh"

namespace gptq {

constexpr int SW_B = 128;        // sweep block (columns)
constexpr int SW_ROWS = 32;      // rows per CTA (one walker lane each)
constexpr int SW_CH = 16;        // chunk width
constexpr int SW_NCH = SW_B / SW_CH;
constexpr int SW_THREADS = 128;  // walker warp + three updater warps
constexpr int SW_WLD = 132;      // W tile pitch (floats): 16-byte rows, quarter-warps in distinct banks
constexpr int SW_ELD = 129;      // error / dequantized tile pitch (floats): odd, lane-per-row access
constexpr int SW_CLD = 132;      // code tile pitch (bytes): 33 words, lane-per-row byte stores in distinct banks
// U block | W tile | errors | dequantized values | 1/U[i][i] | perm | group partials | codes
constexpr int SW_SMEM = SW_B * SW_B * 4 + SW_ROWS * SW_WLD * 4 + 2 * SW_ROWS * SW_ELD * 4 + SW_B * 4 + SW_B * 4 +
                        3 * 4 * SW_ROWS * 4 + SW_ROWS * SW_CLD;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n cp.async.wait_group 0;" ::: "memory");
}

struct SweepArgs {
  float* Wq;          // [m x n] fp32 working weights, sweep order
  const float* U;     // [n x n] upper factor (fp32, or the tf32 hi part when U_lo is set)
  const float* U_lo;  // [n x n] tf32 lo part of U, or nullptr
  const __half* W0;   // [m x n] original weights in sweep order, dead columns 0 (slab kernel, d_form)
  int d_form;         // slab kernel: 1 = hand out W0 - Q for the product past the slab, 0 = the errors
  float* Err;         // scaled errors, or W0 - Q (slab kernel, d_form), fp32 or the hi part:
                      // block columns at Err[r * ld_err + err_col0 ..]
  float* Err_lo;      // tf32 lo part of the errors (same layout), or nullptr
  int ld_err, err_col0;
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

// x / s rounded to nearest-even, from r = 1/s rounded to nearest: q0 = x r, then one
// correction with the remainder x - q0 s taken by a fused multiply-add (Markstein's
// correction step, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990).  Three dependent operations instead of a
// full division on the sweep's per-column chain; the tests compare it bit for bit with
// IEEE division over the quantizer's range.
__device__ __forceinline__ float div_rn(float x, float s, float r) {
  const float q0 = __fmul_rn(x, r);
  const float rem = __fmaf_rn(-q0, s, x);
  return __fmaf_rn(rem, r, q0);
}

// Test support: compare div_rn with IEEE division on count (x, s) pairs drawn from a
// counter-based hash (splitmix64 of seed + index).  Even indices take random bit patterns
// (|x| in [2^-60, 2^21), s in [2^-27, 2^11)); odd ones put x / s within a few ulps of a
// half-integer k + 1/2, |k| <= 300, where a code's rounding is decided.
__device__ __forceinline__ uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void div_rn_check_kernel(uint64_t seed, long long count, unsigned long long* mismatches, float* example) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) {
    const uint64_t h1 = splitmix64(seed ^ (static_cast<uint64_t>(i) * 2u));
    const uint64_t h2 = splitmix64(seed ^ (static_cast<uint64_t>(i) * 2u + 1u));
    const uint32_t se = 100u + static_cast<uint32_t>(h2 % 38u);  // biased exponent of s: 2^-27 .. 2^10
    const float s = __uint_as_float((se << 23) | static_cast<uint32_t>(h2 >> 41));
    float x;
    if ((i & 1) == 0) {
      const uint32_t xe = 67u + static_cast<uint32_t>(h1 % 81u);  // 2^-60 .. 2^20
      x = __uint_as_float(((static_cast<uint32_t>(h1 >> 63)) << 31) | (xe << 23) | static_cast<uint32_t>((h1 >> 8) & 0x7FFFFFu));
    } else {
      const int k = static_cast<int>(h1 % 601u) - 300;
      const int d = static_cast<int>((h1 >> 20) % 9u) - 4;  // -4 .. 4 ulps
      x = __fmul_rn(static_cast<float>(k) + 0.5f, s);
      x = __int_as_float(__float_as_int(x) + d);
    }
    const float r = __frcp_rn(s);
    const float a = div_rn(x, s, r);
    const float b = __fdiv_rn(x, s);
    if (__float_as_uint(a) != __float_as_uint(b)) {
      if (atomicAdd(mismatches, 1ull) == 0ull) {
        example[0] = x;
        example[1] = s;
      }
    }
  }
}

__device__ __forceinline__ void named_arrive(int id) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(SW_THREADS) : "memory");
}
__device__ __forceinline__ void named_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(SW_THREADS) : "memory");
}

// GSUB 0: groups of >= 128 columns (parameters at block starts); 32 or 64: groups inside the block
template <int GSUB>
__global__ void __launch_bounds__(SW_THREADS)
    sweep_block_kernel(SweepArgs a, int i1) {
  extern __shared__ __align__(16) float sw_smem[];
  float* Us = sw_smem;                                    // [128][128] U block
  float* Ws = Us + SW_B * SW_B;                           // [32][132] W tile
  float* Es = Ws + SW_ROWS * SW_WLD;                      // [32][129] scaled errors
  float* Hs = Es + SW_ROWS * SW_ELD;                      // [32][129] dequantized values
  float* rU = Hs + SW_ROWS * SW_ELD;                      // [128] 1 / U[i][i]
  int* perm_s = reinterpret_cast<int*>(rU + SW_B);        // [128]
  float* part = reinterpret_cast<float*>(perm_s + SW_B);  // [3][4][32] group min / max / max|.| partials
  uint8_t* codes8 = reinterpret_cast<uint8_t*>(part + 3 * 4 * SW_ROWS);  // [32][132] codes

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n = a.n;
  const int row0 = blockIdx.x * SW_ROWS;

  griddep_launch_dependents();  // the next kernel may start its prologue now; it waits for our completion
  // ---- before the predecessor is waited on: the U block (written long before) ----
  for (int idx = tid; idx < SW_B * (SW_B / 4); idx += SW_THREADS) {
    const int k = idx / (SW_B / 4), j = (idx % (SW_B / 4)) * 4;
    cp_async16(Us + k * SW_B + j, a.U + static_cast<size_t>(i1 + k) * n + i1 + j);
  }
  if (tid < SW_B) perm_s[tid] = a.perm[i1 + tid];
  cp_async_wait_all();
  __syncthreads();
  if (a.U_lo) {
    for (int idx = tid; idx < SW_B * (SW_B / 4); idx += SW_THREADS) {
      const int k = idx / (SW_B / 4), j = (idx % (SW_B / 4)) * 4;
      const float4 l = *reinterpret_cast<const float4*>(a.U_lo + static_cast<size_t>(i1 + k) * n + i1 + j);
      float4* h = reinterpret_cast<float4*>(Us + k * SW_B + j);
      float4 v = *h;
      v.x += l.x;
      v.y += l.y;
      v.z += l.z;
      v.w += l.w;
      *h = v;
    }
    __syncthreads();
  }
  if (tid < SW_B) rU[tid] = 1.0f / Us[tid * SW_B + tid];

  // ---- the W tile (written by the previous kernel) ----
  griddep_wait();
  for (int idx = tid; idx < SW_ROWS * (SW_B / 4); idx += SW_THREADS) {
    const int rl = idx / (SW_B / 4), j = (idx % (SW_B / 4)) * 4;
    const float4 v = (row0 + rl < a.m)
                         ? *reinterpret_cast<const float4*>(a.Wq + static_cast<size_t>(row0 + rl) * n + i1 + j)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(Ws + rl * SW_WLD + j) = v;
  }
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

  // group parameters at the block start (groups of >= 128 columns): each thread reduces a
  // quarter of its row's block columns (and of the group's columns past the block)
  if (GSUB == 0 && i1 % a.g == 0) {
    const int rl = tid & 31, qtr = tid >> 5;
    float wmin = INFINITY, wmax = -INFINITY, amax = 0.0f;
    for (int j = qtr * 32; j < qtr * 32 + 32; ++j) {
      const float x = Ws[rl * SW_WLD + j];
      wmin = fminf(wmin, x);
      wmax = fmaxf(wmax, x);
      amax = fmaxf(amax, fabsf(x));
    }
    if (row0 + rl < a.m) {
      const float* row = a.Wq + static_cast<size_t>(row0 + rl) * n;
      for (int c = i1 + SW_B + qtr; c < i1 + a.g; c += 4) {
        const float x = row[c];
        wmin = fminf(wmin, x);
        wmax = fmaxf(wmax, x);
        amax = fmaxf(amax, fabsf(x));
      }
    }
    part[(0 * 4 + qtr) * SW_ROWS + rl] = wmin;
    part[(1 * 4 + qtr) * SW_ROWS + rl] = wmax;
    part[(2 * 4 + qtr) * SW_ROWS + rl] = amax;
  }
  __syncthreads();

  if (warp == 0) {
    // ================= walker: lane = row =================
    const int rl = lane;
    const bool valid = row0 + rl < a.m;
    float s = 1.0f, z = 0.0f;
    if (GSUB == 0) {
      const int gi = i1 / a.g;
      if (i1 % a.g == 0) {
        float wmin = part[rl], wmax = part[4 * SW_ROWS + rl], amax = part[8 * SW_ROWS + rl];
#pragma unroll
        for (int q = 1; q < 4; ++q) {
          wmin = fminf(wmin, part[q * SW_ROWS + rl]);
          wmax = fmaxf(wmax, part[(4 + q) * SW_ROWS + rl]);
          amax = fmaxf(amax, part[(8 + q) * SW_ROWS + rl]);
        }
        group_scale_zero(wmin, wmax, amax, qp, a.sym, s, z);
        if (valid) {
          a.scales[static_cast<size_t>(row0 + rl) * a.G + gi] = s;
          a.zeros[static_cast<size_t>(row0 + rl) * a.G + gi] = z;
        }
      } else if (valid) {
        s = a.scales[static_cast<size_t>(row0 + rl) * a.G + gi];
        z = a.zeros[static_cast<size_t>(row0 + rl) * a.G + gi];
      }
    }
    // inside the rounding the zero-point enters only for asymmetric codes
    float zs = a.sym ? 0.0f : z;
    float rs = __frcp_rn(s);
    const float rnd = 12582912.0f;  // 1.5 * 2^23: adding and subtracting it rounds half-to-even
    const bool want_what = a.W_hat != nullptr;
    float* wrow = Ws + rl * SW_WLD;
    float ep[SW_CH];  // the previous chunk's errors
#pragma unroll
    for (int t = 0; t < SW_CH; ++t) ep[t] = 0.0f;
    int u_seen = 0;  // updater passes waited for
#pragma unroll 1
    for (int k = 0; k < SW_NCH; ++k) {
      // chunk k has chunks <= k-2 applied once the updaters' pass k-2 is done
      for (; u_seen <= k - 2; ++u_seen) named_sync(3 + (u_seen & 1));
      float w[SW_CH];
#pragma unroll
      for (int j4 = 0; j4 < SW_CH / 4; ++j4) {
        const float4 v = *reinterpret_cast<const float4*>(wrow + k * SW_CH + 4 * j4);
        w[4 * j4 + 0] = v.x;
        w[4 * j4 + 1] = v.y;
        w[4 * j4 + 2] = v.z;
        w[4 * j4 + 3] = v.w;
      }
      if (k > 0) {  // chunk k-1's errors, in the walker's own registers
#pragma unroll
        for (int t = 0; t < SW_CH; ++t) {
          const float4* urow = reinterpret_cast<const float4*>(Us + ((k - 1) * SW_CH + t) * SW_B + k * SW_CH);
#pragma unroll
          for (int j4 = 0; j4 < SW_CH / 4; ++j4) {
            const float4 u = urow[j4];
            w[4 * j4 + 0] = fmaf(-ep[t], u.x, w[4 * j4 + 0]);
            w[4 * j4 + 1] = fmaf(-ep[t], u.y, w[4 * j4 + 1]);
            w[4 * j4 + 2] = fmaf(-ep[t], u.z, w[4 * j4 + 2]);
            w[4 * j4 + 3] = fmaf(-ep[t], u.w, w[4 * j4 + 3]);
          }
        }
      }
      if (GSUB > 0 && ((k * SW_CH) % (GSUB > 0 ? GSUB : SW_CH)) == 0) {
        // a group starts here: its later chunks need the updaters' pass k-1 as well
        for (; u_seen <= k - 1; ++u_seen) named_sync(3 + (u_seen & 1));
        float wmin = w[0], wmax = w[0], amax = 0.0f;
#pragma unroll
        for (int j = 0; j < SW_CH; ++j) {
          wmin = fminf(wmin, w[j]);
          wmax = fmaxf(wmax, w[j]);
          amax = fmaxf(amax, fabsf(w[j]));
        }
        for (int j = (k + 1) * SW_CH; j < k * SW_CH + GSUB; ++j) {
          const float x = wrow[j];
          wmin = fminf(wmin, x);
          wmax = fmaxf(wmax, x);
          amax = fmaxf(amax, fabsf(x));
        }
        group_scale_zero(wmin, wmax, amax, qp, a.sym, s, z);
        zs = a.sym ? 0.0f : z;
        rs = __frcp_rn(s);
        if (valid) {
          const int gi = (i1 + k * SW_CH) / a.g;
          a.scales[static_cast<size_t>(row0 + rl) * a.G + gi] = s;
          a.zeros[static_cast<size_t>(row0 + rl) * a.G + gi] = z;
        }
      }
      // the walk (no shared-memory stores inside it, so its loads can be issued early)
      float qc[SW_CH];
#pragma unroll
      for (int t = 0; t < SW_CH; ++t) {
        const int i = k * SW_CH + t;
        const float x = w[t];
        const float v = __fadd_rn(div_rn(x, s, rs), zs);
        // clamp, then round half-to-even (clamping to integer bounds commutes with rounding)
        const float q = __fsub_rn(__fadd_rn(fminf(fmaxf(v, qp.lo), qp.hi), rnd), rnd);
        const float e = __fmul_rn(__fmaf_rn(-__fsub_rn(q, zs), s, x), rU[i]);
        ep[t] = e;
        qc[t] = q;
        const float4* urow = reinterpret_cast<const float4*>(Us + i * SW_B + k * SW_CH);
#pragma unroll
        for (int j4 = (t + 1) / 4; j4 < SW_CH / 4; ++j4) {
          const float4 u = urow[j4];
          if (4 * j4 + 0 > t) w[4 * j4 + 0] = fmaf(-e, u.x, w[4 * j4 + 0]);
          if (4 * j4 + 1 > t) w[4 * j4 + 1] = fmaf(-e, u.y, w[4 * j4 + 1]);
          if (4 * j4 + 2 > t) w[4 * j4 + 2] = fmaf(-e, u.z, w[4 * j4 + 2]);
          w[4 * j4 + 3] = fmaf(-e, u.w, w[4 * j4 + 3]);
        }
      }
#pragma unroll
      for (int t = 0; t < SW_CH; ++t) {
        const int i = k * SW_CH + t;
        Es[rl * SW_ELD + i] = ep[t];
        codes8[rl * SW_CLD + i] = static_cast<uint8_t>(static_cast<int>(qc[t] - qp.lo));
        if (want_what) Hs[rl * SW_ELD + i] = __fmul_rn(__fsub_rn(qc[t], zs), s);
      }
      if (k + 2 < SW_NCH) named_arrive(1 + (k & 1));  // chunk k's errors are in Es
    }
  } else {
    // ================= updaters: chunks k+2 .. 7 -= E_k U[chunk k, .] =================
    const int ut = tid - 32;  // 0..95
#pragma unroll 1
    for (int k = 0; k + 2 < SW_NCH; ++k) {
      named_sync(1 + (k & 1));
      const int c0 = (k + 2) * SW_CH;
      const int n4 = (SW_B - c0) / 4;  // 4-column groups to update
      for (int item = ut; item < SW_ROWS * n4; item += SW_THREADS - 32) {
        const int rl = item & 31, j = c0 + 4 * (item >> 5);
        float4 acc = *reinterpret_cast<const float4*>(Ws + rl * SW_WLD + j);
#pragma unroll
        for (int t = 0; t < SW_CH; ++t) {
          const float e = Es[rl * SW_ELD + k * SW_CH + t];
          const float4 u = *reinterpret_cast<const float4*>(Us + (k * SW_CH + t) * SW_B + j);
          acc.x = fmaf(-e, u.x, acc.x);
          acc.y = fmaf(-e, u.y, acc.y);
          acc.z = fmaf(-e, u.z, acc.z);
          acc.w = fmaf(-e, u.w, acc.w);
        }
        *reinterpret_cast<float4*>(Ws + rl * SW_WLD + j) = acc;
      }
      named_arrive(3 + (k & 1));
    }
  }

  __syncthreads();
  // errors of the block's rows (hi/lo for the tensor-core update, or fp32), row by row
  for (int idx = tid; idx < SW_ROWS * SW_B; idx += SW_THREADS) {
    const int rl = idx / SW_B, j = idx % SW_B;
    if (row0 + rl >= a.m) continue;
    const float e = Es[rl * SW_ELD + j];
    const size_t eo = static_cast<size_t>(row0 + rl) * a.ld_err + a.err_col0 + j;
    if (a.Err_lo) {
      const float hi = tf32_round(e);
      a.Err[eo] = hi;
      a.Err_lo[eo] = tf32_round(e - hi);
    } else {
      a.Err[eo] = e;
    }
  }
  if (a.W_hat) {  // dequantized weights back to the original column order
    for (int idx = tid; idx < SW_ROWS * SW_B; idx += SW_THREADS) {
      const int rl = idx / SW_B, j = idx % SW_B;
      if (row0 + rl < a.m) a.W_hat[static_cast<size_t>(row0 + rl) * n + perm_s[j]] = Hs[rl * SW_ELD + j];
    }
  }
  // pack each row's 128 codes into its LSB-first bit stream: one 32-bit word per thread
  {
    const int bits = a.bits;
    const int words = 4 * bits;  // 128 * bits / 32
    const int ldc = n * bits / 32;
    for (int idx = tid; idx < SW_ROWS * words; idx += SW_THREADS) {
      const int rl = idx / words, wi = idx % words;
      if (row0 + rl >= a.m) continue;
      const uint8_t* cr = codes8 + rl * SW_CLD;
      const int b0 = 32 * wi;
      uint32_t word = 0u;
      for (int k = b0 / bits; k * bits < b0 + 32; ++k) {
        const int pos = k * bits - b0;
        const uint32_t code = cr[k];
        word |= (pos >= 0) ? (code << pos) : (code >> (-pos));
      }
      a.codes[static_cast<size_t>(row0 + rl) * ldc + (i1 * bits) / 32 + wi] = word;
    }
  }
}

}  // namespace gptq
