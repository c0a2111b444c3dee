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

#include "sm100_ptx.cuh"

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

namespace gptq {

// CUDA-core fp32 GEMM on hi/lo operands, with the same interface as the tensor-core GEMM
// (gemm_tc.cuh): C = alpha * A * B^T (+ C), A [M x K] and B [N x K] given as hi/lo pairs
// (summed to fp32 on load), the same K-range rules for triangular operands and the same
// outputs.  Used for the factorization's small products, where 64 x 64 tiles spread the
// work over more SMs than the 128 x 256 tensor-core tiles and the fixed cost of a
// tensor-core pipeline would dominate.
struct GemmSimtArgs {
  int M, N, K;
  const float *A_hi, *A_lo;
  int lda;
  const float *B_hi, *B_lo;
  int ldb;
  float alpha;
  int beta, k_lo_mode, k_hi_mode, upper_only;
  float* C;
  int ldc;
  float *Chi, *Clo;
  int ldh;
  float *Cthi, *Ctlo;
  int ldt;
};

constexpr int GS_BK = 32, GS_STAGES = 3, GS_THREADS = 256, GS_LD = GS_BK + 4;

template <int TM, int TN>
constexpr int gs_smem_bytes() {
  return GS_STAGES * 2 * (TM + TN) * GS_LD * 4;
}

__device__ __forceinline__ float tf32_rn_simt(float x) {
  uint32_t u = __float_as_uint(x);
  u += 0xFFFu + ((u >> 13) & 1u);
  return __uint_as_float(u & 0xFFFFE000u);
}

__device__ __forceinline__ void gs_cp_async16(void* smem_dst, const void* gmem_src, bool pred) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  const int sz = pred ? 16 : 0;  // src-size 0 writes zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gmem_src), "r"(sz) : "memory");
}

// TM x TN output tile, 256 threads laid out 16 x 16; thread (tx, ty) owns rows ty + 16 i and
// columns tx + 16 j (strided, so that the shared-memory reads of a warp hit distinct banks).
// K streams through a 3-stage cp.async ring of 32-wide tiles of A_hi, A_lo, B_hi, B_lo
// (K-major, 36-float padded rows); hi + lo are summed as they are read.
template <int TM, int TN>
__global__ void __launch_bounds__(GS_THREADS) gemm_hilo_simt_kernel(GemmSimtArgs p) {
  constexpr int RI = TM / 16, RJ = TN / 16;
  griddep_wait();
  griddep_launch_dependents();
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  if (p.upper_only && m0 >= n0 + TN) return;
  int kb = 0, ke = p.K;
  if (p.k_lo_mode == 1) kb = n0;
  if (p.k_lo_mode == 2) kb = m0;
  if (p.k_lo_mode >= 3) {  // the aligned block of 128 << (mode - 3) columns of the tile (block-diagonal B)
    const int kblk = 128 << (p.k_lo_mode - 3);
    kb = (n0 / kblk) * kblk;
    ke = min(p.K, kb + kblk);
  }
  if (p.k_hi_mode == 1) ke = min(ke, n0 + TN);
  kb = (kb / GS_BK) * GS_BK;
  const int nk = (ke > kb) ? (ke - kb + GS_BK - 1) / GS_BK : 0;

  extern __shared__ __align__(16) float gs_smem[];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  auto stage_ptr = [&](int s) { return gs_smem + s * 2 * (TM + TN) * GS_LD; };

  auto load_stage = [&](int s, int kt) {
    float* Ah = stage_ptr(s);
    float* Al = Ah + TM * GS_LD;
    float* Bh = Al + TM * GS_LD;
    float* Bl = Bh + TN * GS_LD;
    const int k0 = kb + kt * GS_BK;
    for (int idx = tid; idx < TM * (GS_BK / 4); idx += GS_THREADS) {
      const int r = idx / (GS_BK / 4), k4 = (idx % (GS_BK / 4)) * 4;
      const bool ok = (m0 + r) < p.M && (k0 + k4) < ke;
      const size_t o = ok ? static_cast<size_t>(m0 + r) * p.lda + k0 + k4 : 0;
      gs_cp_async16(Ah + r * GS_LD + k4, p.A_hi + o, ok);
      gs_cp_async16(Al + r * GS_LD + k4, p.A_lo + o, ok);
    }
    for (int idx = tid; idx < TN * (GS_BK / 4); idx += GS_THREADS) {
      const int r = idx / (GS_BK / 4), k4 = (idx % (GS_BK / 4)) * 4;
      const bool ok = (n0 + r) < p.N && (k0 + k4) < ke;
      const size_t o = ok ? static_cast<size_t>(n0 + r) * p.ldb + k0 + k4 : 0;
      gs_cp_async16(Bh + r * GS_LD + k4, p.B_hi + o, ok);
      gs_cp_async16(Bl + r * GS_LD + k4, p.B_lo + o, ok);
    }
  };

  float acc[RI][RJ];
#pragma unroll
  for (int i = 0; i < RI; ++i)
#pragma unroll
    for (int j = 0; j < RJ; ++j) acc[i][j] = 0.0f;

  // prologue: GS_STAGES - 1 stages in flight (one commit group per stage, possibly empty)
#pragma unroll
  for (int s = 0; s < GS_STAGES - 1; ++s) {
    if (s < nk) load_stage(s, s);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int kt = 0; kt < nk; ++kt) {
    asm volatile("cp.async.wait_group %0;" ::"n"(GS_STAGES - 2) : "memory");
    __syncthreads();
    // refill the stage consumed one iteration ago
    if (kt + GS_STAGES - 1 < nk) load_stage((kt + GS_STAGES - 1) % GS_STAGES, kt + GS_STAGES - 1);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const float* Ah = stage_ptr(kt % GS_STAGES);
    const float* Al = Ah + TM * GS_LD;
    const float* Bh = Al + TM * GS_LD;
    const float* Bl = Bh + TN * GS_LD;
#pragma unroll
    for (int k4 = 0; k4 < GS_BK; k4 += 4) {
      float4 a[RI], b[RJ];
#pragma unroll
      for (int i = 0; i < RI; ++i) {
        const float4 h = *reinterpret_cast<const float4*>(Ah + (ty + 16 * i) * GS_LD + k4);
        const float4 l = *reinterpret_cast<const float4*>(Al + (ty + 16 * i) * GS_LD + k4);
        a[i] = make_float4(h.x + l.x, h.y + l.y, h.z + l.z, h.w + l.w);
      }
#pragma unroll
      for (int j = 0; j < RJ; ++j) {
        const float4 h = *reinterpret_cast<const float4*>(Bh + (tx + 16 * j) * GS_LD + k4);
        const float4 l = *reinterpret_cast<const float4*>(Bl + (tx + 16 * j) * GS_LD + k4);
        b[j] = make_float4(h.x + l.x, h.y + l.y, h.z + l.z, h.w + l.w);
      }
#pragma unroll
      for (int i = 0; i < RI; ++i)
#pragma unroll
        for (int j = 0; j < RJ; ++j) {
          acc[i][j] = fmaf(a[i].x, b[j].x, acc[i][j]);
          acc[i][j] = fmaf(a[i].y, b[j].y, acc[i][j]);
          acc[i][j] = fmaf(a[i].z, b[j].z, acc[i][j]);
          acc[i][j] = fmaf(a[i].w, b[j].w, acc[i][j]);
        }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");

#pragma unroll
  for (int i = 0; i < RI; ++i) {
    const int r = m0 + ty + 16 * i;
    if (r >= p.M) continue;
#pragma unroll
    for (int j = 0; j < RJ; ++j) {
      const int c = n0 + tx + 16 * j;
      if (c >= p.N) continue;
      const float v = p.alpha * acc[i][j];
      if (p.C) {
        float* cp = p.C + static_cast<size_t>(r) * p.ldc + c;
        *cp = p.beta ? v + *cp : v;
      }
      if (p.Chi) {
        const size_t o = static_cast<size_t>(r) * p.ldh + c;
        const float x = p.beta ? v + (p.Chi[o] + p.Clo[o]) : v;
        const float hi = tf32_rn_simt(x);
        p.Chi[o] = hi;
        p.Clo[o] = tf32_rn_simt(x - hi);
      }
      if (p.Cthi) {
        const size_t o = static_cast<size_t>(c) * p.ldt + r;
        const float hi = tf32_rn_simt(v);
        p.Cthi[o] = hi;
        p.Ctlo[o] = tf32_rn_simt(v - hi);
      }
    }
  }
}

}  // namespace gptq
