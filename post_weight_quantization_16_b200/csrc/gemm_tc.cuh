// gemm_tc.cuh — fp32-faithful GEMM on the sm_100a tensor cores (three tf32 products).
//
//   C = alpha * A * B^T (+ C)      A [M x K] row-major, B [N x K] row-major (both K-major)
//
// Used by the factorization (its Schur-complement, panel and inverse products) and by the
// lazy trailing update of the column sweep (W[:, i2:] -= Err * U[blk, i2:]).  Each operand
// X is stored as two arrays X_hi = rn_tf32(X) and X_lo = rn_tf32(X - X_hi); the product is
// A_hi B_hi + A_hi B_lo + A_lo B_hi, about 2^-21 relative per term, close to fp32.  The
// tensor cores' own accumulation is not round-to-nearest, so every 32-wide K stage is
// accumulated in its own TMEM buffer and then added into fp32 registers with
// round-to-nearest adds (double-buffered TMEM, as in the Hessian kernel).
//
// Tile 128 x BN, BN in {64, 128, 256} chosen per product so that small products still spread
// over many SMs (tcgen05.mma kind::tf32, M=128, N=BN, K=8), persistent CTAs (one per SM) over
// the tiles, a TMA ring of about 192 KB (2, 3 or 4 stages of A_hi, A_lo, B_hi, B_lo; 128-byte
// swizzle; B arrives as 64-row boxes, so one tensor map serves every BN), warp roles:
//   warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps 2-9 epilogue.
// Triangular operands: the K range of a tile can start at its first column (B lower in
// K-major form) or its first row (A upper), or stop after its last column (B upper), so
// the zero halves of triangular factors are skipped; tiles wholly below the diagonal of C
// can be skipped for symmetric updates.
// Outputs (any subset): plain fp32 C (optionally + C), hi/lo pair (optionally + hi+lo), and a
// transposed hi/lo pair (coalesced: the 32 lanes of a warp write 32 consecutive rows).  The
// accumulating plain output of the sweep's trailing update (C += alpha A B^T) can instead go
// out through TMA reduce-add: each epilogue warp stages 32 x 32 boxes in shared memory and
// L2 adds them into C, so the tile never reads C and its stores are whole swizzled boxes.
// A and B are addressed as sub-blocks (row/column offsets) of the whole matrices their tensor
// maps describe, so the maps are encoded once per context.  Rows or columns of a partial
// tile that fall outside the sub-block read neighbouring data whose products land only in
// outputs that are never stored.
#pragma once

#include "sm100_ptx.cuh"

namespace gptq {

constexpr int GT_BM = 128, GT_BK = 32, GT_BOX_N = 64;
constexpr int GT_A_BYTES = GT_BM * GT_BK * 4;  // 16 KB
constexpr int GT_THREADS = 64 + 256;

template <int BN>
struct GtCfg {
  static_assert(BN == 64 || BN == 128 || BN == 256, "tile width");
  static constexpr int B_BYTES = BN * GT_BK * 4;
  static constexpr int STAGE_BYTES = 2 * GT_A_BYTES + 2 * B_BYTES;  // 48, 64 or 96 KB
  static constexpr int STAGES = BN == 256 ? 2 : (BN == 128 ? 3 : 4);
  static constexpr int STG_BYTES = 8 * 32 * 32 * 4;  // one 32 x 32 fp32 staging box per epilogue warp
  static constexpr int SMEM = STAGES * STAGE_BYTES + STG_BYTES + 256 + 1024;
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators
};

// K range of an output tile: from 0, from the tile's first column or first row, or (modes
// GT_KLO_BLK + j) over the kblk = 128 * 2^j columns of the aligned block that holds the tile's
// first column only -- the product with a block-diagonal B of kblk x kblk blocks (tiles at
// most kblk wide; K_HI_COL still cuts the range at the tile's last column).
enum : int { GT_KLO_NONE = 0, GT_KLO_COL = 1, GT_KLO_ROW = 2, GT_KLO_BLK = 3, GT_KLO_BLK_LAST = 6 };
__host__ __device__ constexpr int gt_kblk(int k_lo_mode) {
  return k_lo_mode >= GT_KLO_BLK ? (128 << (k_lo_mode - GT_KLO_BLK)) : 0;
}
enum : int { GT_KHI_NONE = 0, GT_KHI_COL = 1 };

struct GemmTCArgs {
  int M, N, K;
  int a_row0, a_col0;  // offset of A inside the matrix its tensor maps describe
  int b_row0, b_col0;  // offset of B
  float alpha;
  int beta;          // 0 or 1: add the existing C (plain or hi+lo)
  int k_lo_mode, k_hi_mode, upper_only;
  int chunk_stages;  // K stages summed in one TMEM accumulator before the fp32 register add
  float* C;          // plain fp32 output (or nullptr)
  int ldc;
  int c_reduce;        // 1: C += alpha A B^T by TMA reduce-add through the c_map tensor map (beta = 1)
  int c_row0, c_col0;  // offset of C inside the matrix c_map describes
  float* Chi;        // hi/lo output (or nullptr)
  float* Clo;
  int ldh;
  float* Cthi;       // transposed hi/lo output (or nullptr): Ct[c][r]
  float* Ctlo;
  int ldt;
  int* status;
};

__device__ __forceinline__ float tf32_rn(float x) {
  uint32_t u = __float_as_uint(x);
  u += 0xFFFu + ((u >> 13) & 1u);
  return __uint_as_float(u & 0xFFFFE000u);
}

// Number of output tiles the kernel visits: all of them, or with upper_only only the tiles
// that reach the upper triangle (tile (mt, nt) is needed iff mt * BM < (nt + 1) * BN).
__host__ __device__ inline int gt_num_tiles(int M, int N, int upper_only, int bn, int bm = GT_BM) {
  const int mtn = (M + bm - 1) / bm, ntn = (N + bn - 1) / bn;
  if (!upper_only) return mtn * ntn;
  int c = 0;
  for (int nt = 0; nt < ntn; ++nt) c += min(mtn, ((nt + 1) * bn + bm - 1) / bm);
  return c;
}

// Tile t of a product.  Tiles are numbered in order of decreasing K range where the operands
// are triangular (K from the tile's first column: columns ascending; K up to its last column:
// columns descending; K from its first row, or full K: rows ascending), so that the snake
// assignment below pairs long tiles with short ones; with upper_only, column by column over
// the needed tiles (all of full K).
__host__ __device__ inline void gt_tile_at(int M, int N, int K, int k_lo_mode, int k_hi_mode, int upper_only, int bn,
                                           int t, int& m0, int& n0, int& k_begin, int& n_iters, int bm = GT_BM) {
  const int mtn = (M + bm - 1) / bm, ntn = (N + bn - 1) / bn;
  if (!upper_only) {
    if (k_lo_mode == GT_KLO_COL) {
      n0 = (t / mtn) * bn;
      m0 = (t % mtn) * bm;
    } else if (k_hi_mode == GT_KHI_COL) {
      n0 = (ntn - 1 - t / mtn) * bn;
      m0 = (t % mtn) * bm;
    } else {
      m0 = (t / ntn) * bm;
      n0 = (t % ntn) * bn;
    }
  } else {
    int nt = 0;
    for (;; ++nt) {
      const int cnt = min(mtn, ((nt + 1) * bn + bm - 1) / bm);
      if (t < cnt || nt == ntn - 1) break;
      t -= cnt;
    }
    m0 = t * bm;
    n0 = nt * bn;
  }
  int kb = 0, ke = K;
  if (k_lo_mode == GT_KLO_COL) kb = n0;
  if (k_lo_mode == GT_KLO_ROW) kb = m0;
  if (k_lo_mode >= GT_KLO_BLK) {
    const int kblk = gt_kblk(k_lo_mode);
    kb = (n0 / kblk) * kblk;
    ke = min(K, kb + kblk);
  }
  if (k_hi_mode == GT_KHI_COL) ke = min(ke, n0 + bn);
  kb = (kb / GT_BK) * GT_BK;
  k_begin = kb;
  n_iters = (ke > kb) ? (ke - kb + GT_BK - 1) / GT_BK : 0;
}

template <int BN>
__device__ __forceinline__ void gt_tile(const GemmTCArgs& p, int t, int& m0, int& n0, int& k_begin, int& n_iters) {
  gt_tile_at(p.M, p.N, p.K, p.k_lo_mode, p.k_hi_mode, p.upper_only, BN, t, m0, n0, k_begin, n_iters);
}

// Snake assignment of tiles to the G persistent CTAs: round i goes b = 0 .. G-1 on even
// rounds and G-1 .. 0 on odd ones, so a CTA's long first tile meets a short second one.
__host__ __device__ inline int gt_sched(int i, int b, int G) { return i * G + ((i & 1) ? G - 1 - b : b); }

// Epilogue helpers shared by the single-CTA and the CTA-pair kernels.  A warp owns 32 rows (lane
// = row r) and HALF = BN / 2 columns from cbase.
// C (beta = 1) into the accumulators, read while the first stages run.
template <int HALF>
__device__ __forceinline__ void gt_load_c(const GemmTCArgs& p, float (&acc)[HALF], int cbase, int r, bool row_ok) {
  // pre-load C (beta = 1) into the accumulators while the first stages run
#pragma unroll
  for (int cc = 0; cc < HALF / 32; ++cc) {
    const int c0 = cbase + cc * 32;
    const bool ld = p.beta && row_ok && c0 < p.N;
    if (ld && p.C && !p.c_reduce) {
      const float4* cp = reinterpret_cast<const float4*>(p.C + static_cast<size_t>(r) * p.ldc + c0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 c = cp[j];
        acc[cc * 32 + 4 * j + 0] = c.x;
        acc[cc * 32 + 4 * j + 1] = c.y;
        acc[cc * 32 + 4 * j + 2] = c.z;
        acc[cc * 32 + 4 * j + 3] = c.w;
      }
    } else if (ld && p.Chi) {
      const float4* hp = reinterpret_cast<const float4*>(p.Chi + static_cast<size_t>(r) * p.ldh + c0);
      const float4* lp = reinterpret_cast<const float4*>(p.Clo + static_cast<size_t>(r) * p.ldh + c0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 h = hp[j], l = lp[j];
        acc[cc * 32 + 4 * j + 0] = h.x + l.x;
        acc[cc * 32 + 4 * j + 1] = h.y + l.y;
        acc[cc * 32 + 4 * j + 2] = h.z + l.z;
        acc[cc * 32 + 4 * j + 3] = h.w + l.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[cc * 32 + j] = 0.0f;
    }
  }
}

// The tile's columns out: plain, hi/lo, transposed hi/lo, or added into C by TMA reduce boxes
// (32 x 32, staged in the warp's 4 KB buffer stg_warp; wrow0 = the warp's first row).
template <int HALF>
__device__ __forceinline__ void gt_store(const GemmTCArgs& p, const float (&acc)[HALF], int cbase, int r, bool row_ok,
                                   int wrow0, int lane, uint32_t stg_warp, const CUtensorMap& c_map) {
#pragma unroll
  for (int cc = 0; cc < HALF / 32; ++cc) {
    const int c0 = cbase + cc * 32;
    if (c0 >= p.N) continue;  // N % 32 == 0: whole 32-column groups
    if (p.C && p.c_reduce) {
      // stage the warp's 32 x 32 box (128-byte swizzle: 16-byte chunk k of row r at
      // chunk k ^ (r % 8)) and add it into C with one TMA reduce; rows past M add zeros
      const uint32_t stg = stg_warp;
      if (lane == 0) bulk_wait_read0();  // the previous box has left this buffer
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float x0 = row_ok ? acc[cc * 32 + 4 * k + 0] : 0.0f, x1 = row_ok ? acc[cc * 32 + 4 * k + 1] : 0.0f;
        const float x2 = row_ok ? acc[cc * 32 + 4 * k + 2] : 0.0f, x3 = row_ok ? acc[cc * 32 + 4 * k + 3] : 0.0f;
        const uint32_t a = stg + static_cast<uint32_t>(lane * 128 + ((k ^ (lane & 7)) * 16));
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(x0), "f"(x1), "f"(x2), "f"(x3)
                     : "memory");
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_2d(&c_map, stg, p.c_col0 + c0, p.c_row0 + wrow0);
        bulk_commit();
      }
      continue;
    }
    if (!row_ok) continue;
    if (p.C) {
      float4* cp = reinterpret_cast<float4*>(p.C + static_cast<size_t>(r) * p.ldc + c0);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        cp[j] = make_float4(acc[cc * 32 + 4 * j], acc[cc * 32 + 4 * j + 1], acc[cc * 32 + 4 * j + 2],
                            acc[cc * 32 + 4 * j + 3]);
    }
    if (p.Chi) {
      float4* hp = reinterpret_cast<float4*>(p.Chi + static_cast<size_t>(r) * p.ldh + c0);
      float4* lp = reinterpret_cast<float4*>(p.Clo + static_cast<size_t>(r) * p.ldh + c0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = acc[cc * 32 + 4 * j + e];
          hi[e] = tf32_rn(x);
          lo[e] = tf32_rn(x - hi[e]);
        }
        hp[j] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        lp[j] = make_float4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    if (p.Cthi) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float x = acc[cc * 32 + j];
        const float hi = tf32_rn(x);
        const size_t o = static_cast<size_t>(c0 + j) * p.ldt + r;
        p.Cthi[o] = hi;
        p.Ctlo[o] = tf32_rn(x - hi);
      }
    }
  }
}

// Persistent: CTA b handles the tiles gt_sched gives it.  The producer and the MMA issuer run
// ahead across tile boundaries; each K stage lands in one of two TMEM accumulators, which
// the epilogue warps drain into registers that were pre-loaded with C (beta = 1) while the
// tile's first stages were in flight, so a tile ends with stores only.
template <int BN>
__global__ void __launch_bounds__(GT_THREADS, 1)
    gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap a_hi, const __grid_constant__ CUtensorMap a_lo,
                       const __grid_constant__ CUtensorMap b_hi, const __grid_constant__ CUtensorMap b_lo,
                       const __grid_constant__ CUtensorMap c_map, GemmTCArgs p) {
  extern __shared__ uint8_t gt_smem_raw[];
  const uint32_t raw_s = smem_u32(gt_smem_raw);
  uint8_t* smem = gt_smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  using Cfg = GtCfg<BN>;
  constexpr int STAGES = Cfg::STAGES, STAGE_BYTES = Cfg::STAGE_BYTES, B_BYTES = Cfg::B_BYTES;
  const int ntiles = gt_num_tiles(p.M, p.N, p.upper_only, BN);

  const uint32_t stg_base = sbase + STAGES * STAGE_BYTES;  // 1024-aligned staging boxes
  const uint32_t bar_full = stg_base + Cfg::STG_BYTES;
  const uint32_t bar_empty = bar_full + 8 * STAGES;
  const uint32_t bar_tfull = bar_empty + 8 * STAGES;
  const uint32_t bar_tempty = bar_tfull + 16;
  const uint32_t bar_drain = bar_tempty + 16;
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(smem + STAGES * STAGE_BYTES + Cfg::STG_BYTES + 8 * (2 * STAGES + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_tfull + 8 * b, 1);
      mbar_init(bar_tempty + 8 * b, 8 * 32);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a_hi);
    tma_prefetch_desc(&a_lo);
    tma_prefetch_desc(&b_hi);
    tma_prefetch_desc(&b_lo);
    if (p.c_reduce) tma_prefetch_desc(&c_map);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();  // inputs of the previous kernel are complete and visible from here on
  griddep_launch_dependents();  // the next kernel may start its prologue now; it waits for our completion

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (continuous stage ring over all tiles) ----------------
      int it = 0;
      bool ok = true;
      for (int rnd = 0; rnd * static_cast<int>(gridDim.x) < ntiles && ok; ++rnd) {
        const int t = gt_sched(rnd, blockIdx.x, gridDim.x);
        if (t >= ntiles) continue;
        int m0, n0, kb, ni;
        gt_tile<BN>(p, t, m0, n0, kb, ni);
        for (int j = 0; j < ni; ++j, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = static_cast<uint32_t>(it / STAGES) & 1u;
          if (!mbar_wait_bounded(bar_empty + 8 * s, ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar_full + 8 * s;
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          const uint32_t st = sbase + s * STAGE_BYTES;
          const int k = kb + j * GT_BK;
          tma_load_2d(st, &a_hi, fb, p.a_col0 + k, p.a_row0 + m0);
          tma_load_2d(st + GT_A_BYTES, &a_lo, fb, p.a_col0 + k, p.a_row0 + m0);
#pragma unroll
          for (int bx = 0; bx < BN / GT_BOX_N; ++bx) {  // 64-row boxes, stacked at 8 KB
            const uint32_t o8 = bx * (GT_BOX_N * GT_BK * 4);
            tma_load_2d(st + 2 * GT_A_BYTES + o8, &b_hi, fb, p.b_col0 + k, p.b_row0 + n0 + bx * GT_BOX_N);
            tma_load_2d(st + 2 * GT_A_BYTES + B_BYTES + o8, &b_lo, fb, p.b_col0 + k, p.b_row0 + n0 + bx * GT_BOX_N);
          }
        }
      }
      for (int i = max(0, it - STAGES); i < it; ++i)
        mbar_wait_drain(bar_full + 8 * (i % STAGES), static_cast<uint32_t>(i / STAGES) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: one TMEM buffer per chunk of K stages ----------------
      constexpr uint32_t idesc = idesc_make(2u, 2u, 0u, 0u, GT_BM, BN);  // tf32, K-major A and B
      const int cs = p.chunk_stages;
      bool ok = true;
      int it = 0, ch = 0;
      for (int rnd = 0; rnd * static_cast<int>(gridDim.x) < ntiles && ok; ++rnd) {
        const int t = gt_sched(rnd, blockIdx.x, gridDim.x);
        if (t >= ntiles) continue;
        int m0, n0, kb, ni;
        gt_tile<BN>(p, t, m0, n0, kb, ni);
        int b = 0;
        for (int j = 0; j < ni; ++j, ++it) {
          const bool first = (j % cs) == 0;
          if (first) {
            b = ch & 1;
            const uint32_t ph = static_cast<uint32_t>(ch >> 1) & 1u;
            if (!mbar_wait_bounded(bar_tempty + 8 * b, ph ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
          }
          const int s = it % STAGES;
          const uint32_t phs = static_cast<uint32_t>(it / STAGES) & 1u;
          if (!mbar_wait_bounded(bar_full + 8 * s, phs, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN);
          const uint32_t st = sbase + s * STAGE_BYTES;
          const uint32_t sa_hi = st, sa_lo = st + GT_A_BYTES;
          const uint32_t sb_hi = st + 2 * GT_A_BYTES, sb_lo = sb_hi + B_BYTES;
#pragma unroll
          for (int kk = 0; kk < GT_BK / 8; ++kk) {
            const uint32_t off = kk * 32;  // 8 fp32 of K inside the 128-byte swizzle row
            const uint64_t dah = sdesc_sw128(sa_hi + off, 16, 1024), dal = sdesc_sw128(sa_lo + off, 16, 1024);
            const uint64_t dbh = sdesc_sw128(sb_hi + off, 16, 1024), dbl = sdesc_sw128(sb_lo + off, 16, 1024);
            umma_tf32(d_tmem, dal, dbh, idesc, (first && kk == 0) ? 0u : 1u);
            umma_tf32(d_tmem, dah, dbl, idesc, 1u);
            umma_tf32(d_tmem, dah, dbh, idesc, 1u);
          }
          umma_commit(bar_empty + 8 * s);
          if ((j % cs) == cs - 1 || j == ni - 1) {
            umma_commit(bar_tfull + 8 * b);
            ++ch;
          }
        }
      }
      if (!ok) {
        umma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
    }
  } else {
    // ---------------- epilogue ----------------
    const int q = warp & 3;
    const int hh = (warp - 2) >> 2;
    int ch = 0;
    bool all_ok = true;
    for (int rnd = 0; rnd * static_cast<int>(gridDim.x) < ntiles && all_ok; ++rnd) {
      const int t = gt_sched(rnd, blockIdx.x, gridDim.x);
      if (t >= ntiles) continue;
      int m0, n0, kb, ni;
      gt_tile<BN>(p, t, m0, n0, kb, ni);
      const int r = m0 + q * 32 + lane;
      constexpr int HALF = BN / 2;  // columns per epilogue warp
      const int cbase = n0 + hh * HALF;
      const bool row_ok = r < p.M;
      float acc[HALF];
      gt_load_c<HALF>(p, acc, cbase, r, row_ok);
      const int nch = (ni + p.chunk_stages - 1) / p.chunk_stages;
      for (int j = 0; j < nch; ++j, ++ch) {
        const int b = ch & 1;
        const uint32_t ph = static_cast<uint32_t>(ch >> 1) & 1u;
        int ok = 0;
        if (lane == 0) ok = mbar_wait_bounded(bar_tfull + 8 * b, ph, abort_flag) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          all_ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < HALF / 16; ++cc) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(b * BN + hh * HALF + cc * 16),
                             v);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) acc[cc * 16 + jj] = fmaf(p.alpha, __uint_as_float(v[jj]), acc[cc * 16 + jj]);
        }
        tc_fence_before();
        mbar_arrive(bar_tempty + 8 * b);
      }
      if (!all_ok) break;
      gt_store<HALF>(p, acc, cbase, r, row_ok, m0 + q * 32, lane, stg_base + static_cast<uint32_t>(warp - 2) * 4096u,
                     c_map);
    }
  }

  if (warp >= 2 && lane == 0 && p.c_reduce) bulk_wait0();  // this warp's reduces are complete
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, ST_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// The same product on CTA pairs: a cluster of two CTAs per 256 x 256 output tile.  Each CTA
// TMA-loads its own 128 rows of A and its half (128 rows) of B, so a K stage moves a third fewer
// bytes from L2 per flop than the single-CTA 128 x 256 tile; the even CTA issues
// tcgen05.mma.cta_group::2 (M = 256) for the pair and commits to both CTAs' barriers; each CTA's
// epilogue drains its own 128 rows from its own tensor memory, exactly as above.
// ---------------------------------------------------------------------------------------------
constexpr int GP_BN = 256;
constexpr int GP_BM = 2 * GT_BM;                              // rows of a pair tile
constexpr int GP_STAGES = 3;
constexpr int GP_BH_BYTES = (GP_BN / 2) * GT_BK * 4;          // one CTA's half of B, hi or lo: 16 KB
constexpr int GP_STAGE_BYTES = 2 * GT_A_BYTES + 2 * GP_BH_BYTES;  // 64 KB
constexpr int GP_STG_BYTES = 8 * 32 * 32 * 4;
constexpr int GP_SMEM = GP_STAGES * GP_STAGE_BYTES + GP_STG_BYTES + 256 + 1024;
static_assert(GP_SMEM <= 232448, "pair tile fits one CTA's shared memory");

__device__ __forceinline__ void umma_tf32_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n"
      " setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GT_THREADS, 1)
    gemm_tf32x3_pair_kernel(const __grid_constant__ CUtensorMap a_hi, const __grid_constant__ CUtensorMap a_lo,
                            const __grid_constant__ CUtensorMap b_hi, const __grid_constant__ CUtensorMap b_lo,
                            const __grid_constant__ CUtensorMap c_map, GemmTCArgs p) {
  constexpr int BN = GP_BN;
  extern __shared__ uint8_t gp_smem_raw[];
  const uint32_t raw_s = smem_u32(gp_smem_raw);
  uint8_t* smem = gp_smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs; 1: its peer
  const bool leader = rank == 0;
  const int G = static_cast<int>(gridDim.x >> 1), cl = static_cast<int>(blockIdx.x >> 1);
  const int ntiles = gt_num_tiles(p.M, p.N, p.upper_only, BN, GP_BM);

  const uint32_t stg_base = sbase + GP_STAGES * GP_STAGE_BYTES;  // 1024-aligned staging boxes
  const uint32_t bar_full = stg_base + GP_STG_BYTES;
  const uint32_t bar_empty = bar_full + 8 * GP_STAGES;
  const uint32_t bar_tfull = bar_empty + 8 * GP_STAGES;
  const uint32_t bar_tempty = bar_tfull + 16;  // used in the even CTA
  const uint32_t bar_drain = bar_tempty + 16;
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(smem + GP_STAGES * GP_STAGE_BYTES + GP_STG_BYTES + 8 * (2 * GP_STAGES + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < GP_STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);  // even CTA: one expect_tx arrival, the pair's copies' bytes
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_tfull + 8 * b, 1);
      mbar_init(bar_tempty + 8 * b, 2 * 8);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 2 * BN);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a_hi);
    tma_prefetch_desc(&a_lo);
    tma_prefetch_desc(&b_hi);
    tma_prefetch_desc(&b_lo);
    if (p.c_reduce) tma_prefetch_desc(&c_map);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers and tensor memory exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();  // inputs of the previous kernel are complete and visible from here on
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs, each into its own shared memory) ----------------
      // Both halves of a stage complete on the even CTA's full barrier: the even producer expects
      // the bytes of both, the odd CTA's copies count down on it across the pair.
      const uint32_t lead_full = mapa_shared(bar_full, 0);
      int it = 0, issued = 0;
      bool ok = true;
      for (int rnd = 0; rnd * G < ntiles && ok; ++rnd) {
        const int t = gt_sched(rnd, cl, G);
        if (t >= ntiles) continue;
        int m0, n0, kb, ni;
        gt_tile_at(p.M, p.N, p.K, p.k_lo_mode, p.k_hi_mode, p.upper_only, BN, t, m0, n0, kb, ni, GP_BM);
        const int arow = p.a_row0 + m0 + GT_BM * static_cast<int>(rank);
        const int brow = p.b_row0 + n0 + (BN / 2) * static_cast<int>(rank);
        for (int j = 0; j < ni; ++j, ++it) {
          const int s = it % GP_STAGES;
          const uint32_t ph = static_cast<uint32_t>(it / GP_STAGES) & 1u;
          if (!mbar_wait_bounded_cl(bar_empty + 8 * s, ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(bar_full + 8 * s, 2 * GP_STAGE_BYTES);
          const uint32_t fb = lead_full + 8 * s;
          const uint32_t st = sbase + s * GP_STAGE_BYTES;
          const int k = kb + j * GT_BK;
          tma_load_2d_pair(st, &a_hi, fb, p.a_col0 + k, arow);
          tma_load_2d_pair(st + GT_A_BYTES, &a_lo, fb, p.a_col0 + k, arow);
#pragma unroll
          for (int bx = 0; bx < (BN / 2) / GT_BOX_N; ++bx) {  // 64-row boxes, stacked at 8 KB
            const uint32_t o8 = bx * (GT_BOX_N * GT_BK * 4);
            tma_load_2d_pair(st + 2 * GT_A_BYTES + o8, &b_hi, fb, p.b_col0 + k, brow + bx * GT_BOX_N);
            tma_load_2d_pair(st + 2 * GT_A_BYTES + GP_BH_BYTES + o8, &b_lo, fb, p.b_col0 + k, brow + bx * GT_BOX_N);
          }
          issued = it + 1;
        }
      }
      // no TMA write of the pair may still be in flight when either CTA exits: the even CTA
      // waits out the last stages' full barriers; the odd CTA is held by the closing cluster barrier
      if (leader)
        for (int i = max(0, issued - GP_STAGES); i < issued; ++i)
          mbar_wait_drain(bar_full + 8 * (i % GP_STAGES), static_cast<uint32_t>(i / GP_STAGES) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- even CTA: MMA issuer for the pair, one TMEM buffer per chunk ----------------
      constexpr uint32_t idesc = idesc_make(2u, 2u, 0u, 0u, GP_BM, BN);  // tf32, K-major A and B, M = 256
      const int cs = p.chunk_stages;
      bool ok = true;
      int it = 0, ch = 0;
      for (int rnd = 0; rnd * G < ntiles && ok; ++rnd) {
        const int t = gt_sched(rnd, cl, G);
        if (t >= ntiles) continue;
        int m0, n0, kb, ni;
        gt_tile_at(p.M, p.N, p.K, p.k_lo_mode, p.k_hi_mode, p.upper_only, BN, t, m0, n0, kb, ni, GP_BM);
        int b = 0;
        for (int j = 0; j < ni; ++j, ++it) {
          const bool first = (j % cs) == 0;
          if (first) {
            b = ch & 1;
            const uint32_t ph = static_cast<uint32_t>(ch >> 1) & 1u;
            if (!mbar_wait_bounded_cl(bar_tempty + 8 * b, ph ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
          }
          const int s = it % GP_STAGES;
          const uint32_t phs = static_cast<uint32_t>(it / GP_STAGES) & 1u;
          if (!mbar_wait_bounded_cl(bar_full + 8 * s, phs, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN);
          const uint32_t st = sbase + s * GP_STAGE_BYTES;
          const uint32_t sa_hi = st, sa_lo = st + GT_A_BYTES;
          const uint32_t sb_hi = st + 2 * GT_A_BYTES, sb_lo = sb_hi + GP_BH_BYTES;
#pragma unroll
          for (int kk = 0; kk < GT_BK / 8; ++kk) {
            const uint32_t off = kk * 32;  // 8 fp32 of K inside the 128-byte swizzle row
            const uint64_t dah = sdesc_sw128(sa_hi + off, 16, 1024), dal = sdesc_sw128(sa_lo + off, 16, 1024);
            const uint64_t dbh = sdesc_sw128(sb_hi + off, 16, 1024), dbl = sdesc_sw128(sb_lo + off, 16, 1024);
            umma_tf32_pair(d_tmem, dal, dbh, idesc, (first && kk == 0) ? 0u : 1u);
            umma_tf32_pair(d_tmem, dah, dbl, idesc, 1u);
            umma_tf32_pair(d_tmem, dah, dbh, idesc, 1u);
          }
          umma_commit_pair_mc(bar_empty + 8 * s, 0x3);
          if ((j % cs) == cs - 1 || j == ni - 1) {
            umma_commit_pair_mc(bar_tfull + 8 * b, 0x3);
            ++ch;
          }
        }
      }
      if (!ok) {
        // MMAs may still be running: wait for them before the TMEM is released
        umma_commit_pair(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
    }
  } else {
    // ---------------- epilogue (both CTAs): this CTA's 128 rows of each pair tile ----------------
    const int q = warp & 3;
    const int hh = (warp - 2) >> 2;
    const uint32_t lead_tempty = mapa_shared(bar_tempty, 0);
    int ch = 0;
    bool all_ok = true;
    for (int rnd = 0; rnd * G < ntiles && all_ok; ++rnd) {
      const int t = gt_sched(rnd, cl, G);
      if (t >= ntiles) continue;
      int m0, n0, kb, ni;
      gt_tile_at(p.M, p.N, p.K, p.k_lo_mode, p.k_hi_mode, p.upper_only, BN, t, m0, n0, kb, ni, GP_BM);
      const int wrow0 = m0 + GT_BM * static_cast<int>(rank) + q * 32;
      const int r = wrow0 + lane;
      constexpr int HALF = BN / 2;  // columns per epilogue warp
      const int cbase = n0 + hh * HALF;
      const bool row_ok = r < p.M;
      float acc[HALF];
      gt_load_c<HALF>(p, acc, cbase, r, row_ok);
      const int nch = (ni + p.chunk_stages - 1) / p.chunk_stages;
      for (int j = 0; j < nch; ++j, ++ch) {
        const int b = ch & 1;
        const uint32_t ph = static_cast<uint32_t>(ch >> 1) & 1u;
        int ok = 0;
        if (lane == 0) ok = mbar_wait_bounded_cl(bar_tfull + 8 * b, ph, abort_flag) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          all_ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < HALF / 16; ++cc) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(b * BN + hh * HALF + cc * 16),
                             v);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) acc[cc * 16 + jj] = fmaf(p.alpha, __uint_as_float(v[jj]), acc[cc * 16 + jj]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_tempty + 8 * b);
      }
      if (!all_ok) break;
      gt_store<HALF>(p, acc, cbase, r, row_ok, wrow0, lane, stg_base + static_cast<uint32_t>(warp - 2) * 4096u, c_map);
    }
  }

  if (warp >= 2 && lane == 0 && p.c_reduce) bulk_wait0();  // this warp's reduces are complete
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may still read its shared memory or TMEM
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, ST_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * BN);
  }
}

}  // namespace gptq
