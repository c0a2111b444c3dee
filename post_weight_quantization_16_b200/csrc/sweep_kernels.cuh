// sweep_kernels.cuh — S5/S7: one 128-column block of the GPTQ column sweep.
//
// ("大模型量化：GPTQ/AWQ/GGUF 原理对比…" GPTQ section: quantize column by column and push
//  each column's error into the not-yet-quantized columns; "模型量化实战…" §3.2
//  quantize_block: blocks of 128 columns.)
//
// Rows of W are independent once U is known.  Eight lanes of a warp share one row: lane
// l (0..7 within its group) holds the row's block columns 16l .. 16l+15 in registers, so a
// warp sweeps four rows and a 256-thread CTA 32 rows.  For column i the owning lane
// (i / 16) computes the code, the dequantized value and e = (w - q) / U[i][i] and updates
// its own later columns, w[j] -= e * U[i][j], so the per-column dependent chain never
// leaves the lane's registers.  After each 16-column chunk its errors reach the row's later
// lanes in one batch (16 shuffles, then 16 x 16 fused multiply-adds per lane).  Group scales/zeros come from a min/max over the group's
// current values reduced across the row's lanes with shuffles.  The U block (128 x 128) is
// staged in shared memory with asynchronous copies, in a bank-skewed layout so the eight
// 16-column segments a warp reads at once hit different banks.
// The block's errors go to Err; the columns after the block receive them through tensor-core
// products (S6) launched by the host: within a super-block of columns right after each block,
// beyond it once per super-block.
//
// The integer decisions (code and zero-point) are taken in fp32 with correctly rounded
// division and round-half-to-even, the precision the pages' own sketches use.
#pragma once

#include <cstdint>

#include "factor_kernels.cuh"

namespace gptq {

constexpr int SW_B = 128;            // sweep block (columns)
constexpr int SW_LANES = 8;          // lanes per row
constexpr int SW_COLS = SW_B / SW_LANES;  // 16 columns per lane
constexpr int SW_THREADS = 256;
constexpr int SW_ROWS = SW_THREADS / SW_LANES;  // 32 rows per CTA
constexpr int SW_SEG = 20;                      // skewed segment stride (floats) in shared memory
constexpr int SW_ULD = SW_LANES * SW_SEG;       // 160 floats per staged U row
constexpr int SW_SMEM = 2 * SW_B * SW_ULD * 4 + SW_B * 4 + SW_B * 4 + SW_ROWS * 32 * 4;

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
  float* Err;         // scaled errors (fp32, or hi part): block columns at Err[r * ld_err + err_col0 ..]
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

// min / max / max|.| over the eight lanes of a row group
__device__ __forceinline__ void group_reduce(float& wmin, float& wmax, float& amax) {
#pragma unroll
  for (int o = 1; o < SW_LANES; o <<= 1) {
    wmin = fminf(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
    wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
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

template <int GSUB>  // 0: groups of >= 128 columns (params at block starts); 32 or 64: inside the block
__global__ void __launch_bounds__(SW_THREADS)
    sweep_block_kernel(SweepArgs a, int i1) {
  extern __shared__ __align__(16) float sw_smem[];
  float* Us = sw_smem;                                          // [128][160] U block (skewed)
  float* Ul = Us + SW_B * SW_ULD;                               // [128][160] lo part while it lands
  float* rU = Ul + SW_B * SW_ULD;                               // [128] 1 / U[i][i]
  int* perm_s = reinterpret_cast<int*>(rU + SW_B);              // [128]
  uint32_t* cw = reinterpret_cast<uint32_t*>(perm_s + SW_B);    // [32 rows][32 words] packed codes

  griddep_wait();
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int l8 = lane & (SW_LANES - 1);      // segment of the row this lane holds
  const int gbase = lane & ~(SW_LANES - 1);  // first lane of the row's group
  const int rloc = tid / SW_LANES;           // row within the CTA
  const int n = a.n;

  // stage U[i1 + k][i1 + j] at Us[k][SEG * (j / 16) + j % 16]
  for (int idx = tid; idx < SW_B * (SW_B / 4); idx += SW_THREADS) {
    const int k = idx / (SW_B / 4), j = (idx % (SW_B / 4)) * 4;
    const size_t g = static_cast<size_t>(i1 + k) * n + i1 + j;
    const int so = k * SW_ULD + (j / SW_COLS) * SW_SEG + (j % SW_COLS);
    cp_async16(Us + so, a.U + g);
    if (a.U_lo) cp_async16(Ul + so, a.U_lo + g);
  }
  if (tid < SW_B) perm_s[tid] = a.perm[i1 + tid];
  for (int idx = tid; idx < SW_ROWS * 32; idx += SW_THREADS) cw[idx] = 0u;

  const int r = blockIdx.x * SW_ROWS + rloc;
  const bool valid = r < a.m;
  const int rr = valid ? r : 0;

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

  // this lane's 16 columns of the row, while U lands
  float w[SW_COLS];
  {
    const float4* src = reinterpret_cast<const float4*>(a.Wq + static_cast<size_t>(rr) * n + i1 + SW_COLS * l8);
#pragma unroll
    for (int j4 = 0; j4 < SW_COLS / 4; ++j4) {
      const float4 v = valid ? src[j4] : make_float4(0.f, 0.f, 0.f, 0.f);
      w[4 * j4 + 0] = v.x;
      w[4 * j4 + 1] = v.y;
      w[4 * j4 + 2] = v.z;
      w[4 * j4 + 3] = v.w;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (a.U_lo) {
    for (int idx = tid; idx < SW_B * SW_ULD; idx += SW_THREADS) Us[idx] += Ul[idx];
    __syncthreads();
  }
  if (tid < SW_B) rU[tid] = 1.0f / Us[tid * SW_ULD + (tid / SW_COLS) * SW_SEG + (tid % SW_COLS)];
  __syncthreads();

  float s = 1.0f, z = 0.0f;
  if (GSUB == 0) {
    const int gi = i1 / a.g;
    if (i1 % a.g == 0) {
      float wmin = w[0], wmax = w[0], amax = 0.0f;
#pragma unroll
      for (int j = 0; j < SW_COLS; ++j) {
        wmin = fminf(wmin, w[j]);
        wmax = fmaxf(wmax, w[j]);
        amax = fmaxf(amax, fabsf(w[j]));
      }
      if (valid) {  // columns of the group beyond this block (already up to date)
        const float* row = a.Wq + static_cast<size_t>(rr) * n;
        for (int c = i1 + SW_B + l8; c < i1 + a.g; c += SW_LANES) {
          const float x = row[c];
          wmin = fminf(wmin, x);
          wmax = fmaxf(wmax, x);
          amax = fmaxf(amax, fabsf(x));
        }
      }
      group_reduce(wmin, wmax, amax);
      group_scale_zero(wmin, wmax, amax, qp, a.sym, s, z);
      if (valid && l8 == 0) {
        a.scales[static_cast<size_t>(rr) * a.G + gi] = s;
        a.zeros[static_cast<size_t>(rr) * a.G + gi] = z;
      }
    } else if (valid) {
      s = a.scales[static_cast<size_t>(rr) * a.G + gi];
      z = a.zeros[static_cast<size_t>(rr) * a.G + gi];
    }
  }

  uint32_t mycode[SW_COLS];
  float myerr[SW_COLS], mywhat[SW_COLS];
#pragma unroll
  for (int t = 0; t < SW_COLS; ++t) {
    mycode[t] = 0u;
    myerr[t] = 0.0f;
    mywhat[t] = 0.0f;
  }
  // inside the rounding the zero-point enters only for asymmetric codes
  float zs = a.sym ? 0.0f : z;
  float rs = __frcp_rn(s);

#pragma unroll 1
  for (int c = 0; c < SW_LANES; ++c) {  // chunk c = columns 16c .. 16c+15, owned by lane c of each row
    if (GSUB > 0 && ((c * SW_COLS) % (GSUB > 0 ? GSUB : SW_COLS)) == 0) {
      constexpr int NL = (GSUB > 0 ? GSUB : SW_COLS) / SW_COLS;  // lanes covering one group
      const bool in = (l8 >= c) && (l8 < c + NL);
      float wmin = in ? w[0] : INFINITY, wmax = in ? w[0] : -INFINITY, amax = 0.0f;
      if (in) {
#pragma unroll
        for (int j = 0; j < SW_COLS; ++j) {
          wmin = fminf(wmin, w[j]);
          wmax = fmaxf(wmax, w[j]);
          amax = fmaxf(amax, fabsf(w[j]));
        }
      }
      group_reduce(wmin, wmax, amax);
      group_scale_zero(wmin, wmax, amax, qp, a.sym, s, z);
      zs = a.sym ? 0.0f : z;
      rs = __frcp_rn(s);
      if (valid && l8 == 0) {
        const int gi = (i1 + c * SW_COLS) / a.g;
        a.scales[static_cast<size_t>(rr) * a.G + gi] = s;
        a.zeros[static_cast<size_t>(rr) * a.G + gi] = z;
      }
    }
    const bool owner = (l8 == c);
    const float* useg = Us + (c * SW_COLS) * SW_ULD + l8 * SW_SEG;  // U rows of the chunk, this lane's columns
    // The owner walks its 16 columns with nothing but its own registers on the dependent
    // chain; the other lanes run the same instructions with a zero error (no effect).
    float ec[SW_COLS];
#pragma unroll
    for (int t = 0; t < SW_COLS; ++t) {
      const float x = w[t];
      const float v = __fadd_rn(div_rn(x, s, rs), zs);
      const float q = fminf(fmaxf(rintf(v), qp.lo), qp.hi);
      const float qz = __fsub_rn(q, zs);
      const float e = __fmul_rn(__fmaf_rn(-qz, s, x), rU[c * SW_COLS + t]);
      ec[t] = e;
      if (owner) {
        mycode[t] = static_cast<uint32_t>(static_cast<int>(q - qp.lo));
        myerr[t] = e;
        mywhat[t] = __fmul_rn(qz, s);
      }
      const float eo = owner ? e : 0.0f;
      const float4* urow = reinterpret_cast<const float4*>(useg + t * SW_ULD);
#pragma unroll
      for (int j4 = (t + 1) / 4; j4 < SW_COLS / 4; ++j4) {
        const float4 u = urow[j4];
        if (4 * j4 + 0 > t) w[4 * j4 + 0] = fmaf(-eo, u.x, w[4 * j4 + 0]);
        if (4 * j4 + 1 > t) w[4 * j4 + 1] = fmaf(-eo, u.y, w[4 * j4 + 1]);
        if (4 * j4 + 2 > t) w[4 * j4 + 2] = fmaf(-eo, u.z, w[4 * j4 + 2]);
        w[4 * j4 + 3] = fmaf(-eo, u.w, w[4 * j4 + 3]);
      }
    }
    // the chunk's 16 errors reach the row's later lanes in one batch:
    // w[j] -= sum_t e_t U[16c + t][j] for the columns j of lanes l8 > c
    if (c + 1 < SW_LANES) {
      const bool later = l8 > c;
#pragma unroll
      for (int t = 0; t < SW_COLS; ++t) {
        const float eb = __shfl_sync(0xffffffffu, ec[t], gbase + c);
        const float e = later ? eb : 0.0f;
        const float4* urow = reinterpret_cast<const float4*>(useg + t * SW_ULD);
#pragma unroll
        for (int j4 = 0; j4 < SW_COLS / 4; ++j4) {
          const float4 u = urow[j4];
          w[4 * j4 + 0] = fmaf(-e, u.x, w[4 * j4 + 0]);
          w[4 * j4 + 1] = fmaf(-e, u.y, w[4 * j4 + 1]);
          w[4 * j4 + 2] = fmaf(-e, u.z, w[4 * j4 + 2]);
          w[4 * j4 + 3] = fmaf(-e, u.w, w[4 * j4 + 3]);
        }
      }
    }
  }

  griddep_launch_dependents();
  // errors of this lane's 16 columns (hi/lo for the tensor-core update, or fp32)
  if (valid) {
    const size_t eo = static_cast<size_t>(rr) * a.ld_err + a.err_col0 + SW_COLS * l8;
    float4* ep = reinterpret_cast<float4*>(a.Err + eo);
    if (a.Err_lo) {
      float4* lp = reinterpret_cast<float4*>(a.Err_lo + eo);
#pragma unroll
      for (int j4 = 0; j4 < SW_COLS / 4; ++j4) {
        float hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = tf32_round(myerr[4 * j4 + e]);
          lo[e] = tf32_round(myerr[4 * j4 + e] - hi[e]);
        }
        ep[j4] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        lp[j4] = make_float4(lo[0], lo[1], lo[2], lo[3]);
      }
    } else {
#pragma unroll
      for (int j4 = 0; j4 < SW_COLS / 4; ++j4)
        ep[j4] = make_float4(myerr[4 * j4], myerr[4 * j4 + 1], myerr[4 * j4 + 2], myerr[4 * j4 + 3]);
    }
    if (a.W_hat) {
      float* wh = a.W_hat + static_cast<size_t>(rr) * n;
#pragma unroll
      for (int t = 0; t < SW_COLS; ++t) wh[perm_s[SW_COLS * l8 + t]] = mywhat[t];
    }
  }

  // pack the row's 128 codes (LSB-first bit stream): each lane ORs its 16 codes into the
  // row's words in shared memory, then the row's lanes store the words
  const int bits = a.bits;
  uint32_t* rw = cw + rloc * 32;
#pragma unroll
  for (int t = 0; t < SW_COLS; ++t) {
    const int pos = (SW_COLS * l8 + t) * bits;
    const uint32_t code = mycode[t];
    atomicOr(&rw[pos >> 5], code << (pos & 31));
    if ((pos & 31) + bits > 32) atomicOr(&rw[(pos >> 5) + 1], code >> (32 - (pos & 31)));
  }
  __syncwarp();
  if (valid) {
    const int words = 4 * bits;  // 128 * bits / 32
    const int ldc = n * bits / 32;
    uint32_t* dst = a.codes + static_cast<size_t>(rr) * ldc + (i1 * bits) / 32;
    for (int wi = l8; wi < words; wi += SW_LANES) dst[wi] = rw[wi];
  }
}

}  // namespace gptq
