// slab_sweep.cuh — S5/S6/S7 within one super-block of columns: the column sweep of every
// 128-column block of the super-block and the lazy update of the super-block's later columns,
// in one launch.
//
// ("大模型量化：GPTQ/AWQ/GGUF 原理对比…" GPTQ section: quantize column by column and push each
//  column's error into the not-yet-quantized columns; "模型量化实战…" §3.2 quantize_block:
//  blocks of 128 columns, the columns after a block updated once per block.)
//
// Rows of W are independent once U is known.  A CTA takes 32 rows and keeps their whole
// super-block (up to 1024 columns, the slab) in shared memory for the launch.  For each
// 128-column block of the slab, in order:
//   * the block's 128 x 128 U block is staged in shared memory;
//   * warp 0, the walker, walks the block in eight chunks of 16 columns exactly as the
//     one-block sweep does (one row per lane, the per-column chain in registers, U values read
//     as broadcasts): code, dequantized value, e = (w - q) / U[i][i], w[j] -= e U[i][j] for the
//     chunk's later columns;
//   * warps 1-7, the updaters, take each finished chunk's errors and apply them, first to the
//     block's chunks two and more ahead (from the staged U block, a lane per row), then to
//     every later column of the slab (a lane per four columns, their 16 U values loaded once,
//     coalesced across the warp, and used for all 32 rows; the errors read as shared-memory
//     broadcasts), in fp32 fused multiply-adds;
//   * for the one product that updates the columns beyond the super-block the block's columns
//     go out as tf32 hi/lo pairs: d = w0 - q (original weight minus dequantized value), or
//     with d_form = 0 the scaled errors e; and its codes are packed.
// The two forms of that product carry the same compensation: the sweep's errors satisfy
// E U = W0 - Q, so the errors of every column before a super-block reach it as
// -E U[., sb] = (W0 - Q) V[., sb] U[sb, sb] (V = U^-1), which needs only the diagonal
// super-block of U; it holds for the super-block as a whole, once every earlier column is in.
// So the per-block product on the later columns of the super-block, and its launch, leave the
// critical path: within a super-block the updates run beside the walker on the same SM.
#pragma once

#include <cstdint>

#include "sweep_kernels.cuh"

namespace gptq {

constexpr int SS_THREADS = 256;            // walker warp + seven updater warps
constexpr int SS_NW = SS_THREADS / 32;
constexpr int SS_MAXW = 1024;              // widest slab (columns)
// slab pitch (floats) for a slab of S columns: lane-per-row float4 access without conflicts
__host__ __device__ constexpr int ss_wld(int S) { return S + 4; }
// U block | slab | errors | the chunk's errors (compact) | 1/U[i][i] | perm | group partials | codes |
// the block's group parameters (s, and the zero-point inside the rounding, per row and group)
__host__ __device__ constexpr int ss_smem_bytes(int S) {
  return SW_B * SW_B * 4 + SW_ROWS * ss_wld(S) * 4 + SW_ROWS * SW_ELD * 4 + 2 * SW_ROWS * SW_CH * 4 + SW_B * 4 +
         SW_B * 4 + 3 * SS_NW * SW_ROWS * 4 + SW_ROWS * SW_CLD + 2 * SW_ROWS * 4 * 4;
}
constexpr int SS_SMEM = ss_smem_bytes(SS_MAXW);

__device__ __forceinline__ void ss_arrive(int id) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(SS_THREADS) : "memory");
}
__device__ __forceinline__ void ss_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(SS_THREADS) : "memory");
}

// GSUB 0: groups of >= 128 columns (parameters at block starts); 32 or 64: groups inside a block.
// Columns [s0, s1) of the rows row0 .. row0 + 31; s1 - s0 <= SS_MAXW, a multiple of 128.
template <int GSUB>
__global__ void __launch_bounds__(SS_THREADS, 1) sweep_slab_kernel(SweepArgs a, int s0, int s1) {
  extern __shared__ __align__(16) float ss_smem[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n = a.n;
  const int row0 = blockIdx.x * SW_ROWS;
  const int S = s1 - s0;
  const int WLD = ss_wld(S);
  float* Us = ss_smem;                                    // [128][128] U block
  float* Ws = Us + SW_B * SW_B;                           // [32][WLD] slab
  float* Es = Ws + SW_ROWS * WLD;                         // [32][129] scaled errors of the block
  float* Ek = Es + SW_ROWS * SW_ELD;                      // [2][32][16] errors of the last two chunks
  float* rU = Ek + 2 * SW_ROWS * SW_CH;                   // [128] 1 / U[i][i]
  int* perm_s = reinterpret_cast<int*>(rU + SW_B);        // [128]
  float* part = reinterpret_cast<float*>(perm_s + SW_B);  // [3][8][32] group min / max / max|.| partials
  uint8_t* codes8 = reinterpret_cast<uint8_t*>(part + 3 * SS_NW * SW_ROWS);  // [32][132] codes
  float* gs_s = reinterpret_cast<float*>(codes8 + SW_ROWS * SW_CLD);          // [32][4] s of the block's groups
  float* gz_s = gs_s + SW_ROWS * 4;                                           // [32][4] zero-point in the rounding

  auto stage_block = [&](int i1) {
    for (int idx = tid; idx < SW_B * (SW_B / 4); idx += SS_THREADS) {
      const int k = idx / (SW_B / 4), j = (idx % (SW_B / 4)) * 4;
      cp_async16(Us + k * SW_B + j, a.U + static_cast<size_t>(i1 + k) * n + i1 + j);
    }
    if (tid < SW_B) perm_s[tid] = a.perm[i1 + tid];
  };

  griddep_launch_dependents();  // the next kernel may start its prologue now; it waits for our completion
  // ---- before the predecessor is waited on: the first U block (written long before) ----
  stage_block(s0);
  // ---- the slab (written by the previous kernels) ----
  griddep_wait();
  for (int idx = tid; idx < SW_ROWS * (S / 4); idx += SS_THREADS) {
    const int rl = idx / (S / 4), j = (idx % (S / 4)) * 4;
    float* dst = Ws + rl * WLD + j;
    if (row0 + rl < a.m)
      cp_async16(dst, a.Wq + static_cast<size_t>(row0 + rl) * n + s0 + j);
    else
      *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  cp_async_wait_all();
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
  const float rnd = 12582912.0f;  // 1.5 * 2^23: adding and subtracting it rounds half-to-even
  const bool want_what = a.W_hat != nullptr;

#pragma unroll 1
  for (int i1 = s0; i1 < s1; i1 += SW_B) {
    const int bo = i1 - s0;                 // the block's first slab column
    const bool slab_rest = i1 + SW_B < s1;  // later slab columns to update
    if (i1 > s0) {
      stage_block(i1);
      cp_async_wait_all();
      __syncthreads();
    }
    if (tid < SW_B) rU[tid] = 1.0f / Us[tid * SW_B + tid];

    // group parameters at the block start (groups of >= 128 columns): warp q reduces the
    // group's columns q, q + 8, ... of its lane's row, in the slab and past it
    if (GSUB == 0 && i1 % a.g == 0) {
      const int rl = lane, q = warp;
      float wmin = INFINITY, wmax = -INFINITY, amax = 0.0f;
      const int in_end = min(S, bo + a.g);
      for (int j = bo + q; j < in_end; j += SS_NW) {
        const float x = Ws[rl * WLD + j];
        wmin = fminf(wmin, x);
        wmax = fmaxf(wmax, x);
        amax = fmaxf(amax, fabsf(x));
      }
      if (row0 + rl < a.m) {
        const float* row = a.Wq + static_cast<size_t>(row0 + rl) * n;
        for (int c = s1 + q; c < i1 + a.g; c += SS_NW) {
          const float x = row[c];
          wmin = fminf(wmin, x);
          wmax = fmaxf(wmax, x);
          amax = fmaxf(amax, fabsf(x));
        }
      }
      part[(0 * SS_NW + q) * SW_ROWS + rl] = wmin;
      part[(1 * SS_NW + q) * SW_ROWS + rl] = wmax;
      part[(2 * SS_NW + q) * SW_ROWS + rl] = amax;
    }
    __syncthreads();

    // the block-end hand-out's original weights (two items of eight columns per thread), loaded
    // now so that their latency hides behind the walk
    uint4 w0pre[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    if (a.d_form && s1 < n) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int it = tid + r * SS_THREADS, rl = it / (SW_B / 8), j0 = (it % (SW_B / 8)) * 8;
        if (row0 + rl < a.m)
          w0pre[r] = __ldg(reinterpret_cast<const uint4*>(a.W0 + static_cast<size_t>(row0 + rl) * n + i1 + j0));
      }
    }

    if (warp == 0) {
      // ================= walker: lane = row =================
      const int rl = lane;
      const bool valid = row0 + rl < a.m;
      float s = 1.0f, z = 0.0f;
      if (GSUB == 0) {
        const int gi = i1 / a.g;
        if (i1 % a.g == 0) {
          float wmin = part[rl], wmax = part[SS_NW * SW_ROWS + rl], amax = part[2 * SS_NW * SW_ROWS + rl];
#pragma unroll
          for (int q = 1; q < SS_NW; ++q) {
            wmin = fminf(wmin, part[q * SW_ROWS + rl]);
            wmax = fmaxf(wmax, part[(SS_NW + q) * SW_ROWS + rl]);
            amax = fmaxf(amax, part[(2 * SS_NW + q) * SW_ROWS + rl]);
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
      if (GSUB == 0) {
        gs_s[rl * 4] = s;
        gz_s[rl * 4] = zs;
      }
      float* wrow = Ws + rl * WLD + bo;
      float ep[SW_CH];  // the previous chunk's errors
#pragma unroll
      for (int t = 0; t < SW_CH; ++t) ep[t] = 0.0f;
      int u_seen = 0;  // updater passes waited for
#pragma unroll 1
      for (int k = 0; k < SW_NCH; ++k) {
        // chunk k has chunks <= k-2 applied once the updaters' pass k-2 is done
        for (; u_seen <= k - 2; ++u_seen) ss_sync(3 + (u_seen & 1));
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
          for (; u_seen <= k - 1; ++u_seen) ss_sync(3 + (u_seen & 1));
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
          gs_s[rl * 4 + (k * SW_CH) / (GSUB > 0 ? GSUB : SW_B)] = s;
          gz_s[rl * 4 + (k * SW_CH) / (GSUB > 0 ? GSUB : SW_B)] = zs;
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
        }
        if (slab_rest) {  // the chunk's errors again, 16-byte aligned per row, for the slab pass
          float4* ek = reinterpret_cast<float4*>(Ek + ((k & 1) * SW_ROWS + rl) * SW_CH);
#pragma unroll
          for (int j4 = 0; j4 < SW_CH / 4; ++j4)
            ek[j4] = make_float4(ep[4 * j4], ep[4 * j4 + 1], ep[4 * j4 + 2], ep[4 * j4 + 3]);
        }
        if (k + 2 < SW_NCH || slab_rest) ss_arrive(1 + (k & 1));  // chunk k's errors are in Es
        if (want_what && valid) {  // dequantized weights, straight to the original column order
#pragma unroll
          for (int t = 0; t < SW_CH; ++t)
            a.W_hat[static_cast<size_t>(row0 + rl) * n + perm_s[k * SW_CH + t]] = __fmul_rn(__fsub_rn(qc[t], zs), s);
        }
      }
      // the passes not yet waited for (their errors reach later blocks of the slab)
      for (; u_seen < SW_NCH; ++u_seen)
        if (u_seen + 2 < SW_NCH || slab_rest) ss_sync(3 + (u_seen & 1));
    } else {
      // ================= updaters: warps 1 .. 7, lane = row =================
      const int uw = warp - 1;  // 0 .. 6
      // the slab pass's geometry (fixed within the block) and this lane's first item
      constexpr int RCH = 8;
      const int cb = bo + SW_B;
      const int nq = slab_rest ? (S - cb) / 4 : 0;
      const int first = uw * 32 + lane;
      const bool have_first = first < (SW_ROWS / RCH) * nq;
#pragma unroll 1
      for (int k = 0; k < SW_NCH; ++k) {
        if (!(k + 2 < SW_NCH || slab_rest)) continue;
        // the first item's 16 U values do not depend on the walker: load them before waiting
        float4 u[SW_CH];
        if (have_first) {
          const float* ub = a.U + static_cast<size_t>(i1 + k * SW_CH) * n + s0 + cb + 4 * (first % nq);
#pragma unroll
          for (int t = 0; t < SW_CH; ++t) u[t] = __ldg(reinterpret_cast<const float4*>(ub + static_cast<size_t>(t) * n));
        }
        ss_sync(1 + (k & 1));
        // (1) the block's chunks k+2 .. 7, from the staged U block
        if (k + 2 < SW_NCH) {
          const int c0 = (k + 2) * SW_CH;
          const int n4 = (SW_B - c0) / 4;
          for (int item = tid - 32; item < SW_ROWS * n4; item += SS_THREADS - 32) {
            const int rl = item & 31, j = c0 + 4 * (item >> 5);
            float4 acc = *reinterpret_cast<const float4*>(Ws + rl * WLD + bo + j);
#pragma unroll
            for (int t = 0; t < SW_CH; ++t) {
              const float e = Es[rl * SW_ELD + k * SW_CH + t];
              const float4 u = *reinterpret_cast<const float4*>(Us + (k * SW_CH + t) * SW_B + j);
              acc.x = fmaf(-e, u.x, acc.x);
              acc.y = fmaf(-e, u.y, acc.y);
              acc.z = fmaf(-e, u.z, acc.z);
              acc.w = fmaf(-e, u.w, acc.w);
            }
            *reinterpret_cast<float4*>(Ws + rl * WLD + bo + j) = acc;
          }
        }
        // (2) the slab's later columns: a lane takes four columns, holds their 16 U values
        // (rows i1 + 16 k .. + 15, coalesced loads across the warp) in registers and walks the
        // 32 rows, the chunk's errors read as shared-memory broadcasts
        if (slab_rest) {
          const float* ub = a.U + static_cast<size_t>(i1 + k * SW_CH) * n + s0 + cb;
          const float4* ek = reinterpret_cast<const float4*>(Ek + (k & 1) * SW_ROWS * SW_CH);
          // items (row chunk of 8 rows, column quad), quads fastest: every updater lane has work
          // however narrow the rest of the slab, and a quad's U values are reused from L1
          for (int item = first; item < (SW_ROWS / RCH) * nq; item += (SS_NW - 1) * 32) {
            const int q = item % nq, r0 = (item / nq) * RCH;
            if (item != first) {
#pragma unroll
              for (int t = 0; t < SW_CH; ++t)
                u[t] = __ldg(reinterpret_cast<const float4*>(ub + static_cast<size_t>(t) * n + 4 * q));
            }
#pragma unroll 2
            for (int r = r0; r < r0 + RCH; ++r) {
              float* wp = Ws + r * WLD + cb + 4 * q;
              float4 acc = *reinterpret_cast<const float4*>(wp);
#pragma unroll
              for (int t4 = 0; t4 < SW_CH / 4; ++t4) {
                const float4 e = ek[r * (SW_CH / 4) + t4];
                const float ev[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                  const float4 uu = u[4 * t4 + tt];
                  acc.x = fmaf(-ev[tt], uu.x, acc.x);
                  acc.y = fmaf(-ev[tt], uu.y, acc.y);
                  acc.z = fmaf(-ev[tt], uu.z, acc.z);
                  acc.w = fmaf(-ev[tt], uu.w, acc.w);
                }
              }
              *reinterpret_cast<float4*>(wp) = acc;
            }
          }
        }
        ss_arrive(3 + (k & 1));
      }
    }

    __syncthreads();
    // the block's columns for the tensor-core update past the super-block (tf32 hi/lo), row by
    // row: d = w0 - q from the codes and the group parameters (the walker's dequantization), eight
    // columns an item, or the scaled errors
    if (s1 < n && a.d_form) {
      static_assert(SW_ROWS * (SW_B / 8) == 2 * SS_THREADS, "two hand-out items per thread");
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int it = tid + r * SS_THREADS;
        const int rl = it / (SW_B / 8), j0 = (it % (SW_B / 8)) * 8;
        if (row0 + rl >= a.m) continue;
        const size_t row = static_cast<size_t>(row0 + rl);
        const int slot = GSUB > 0 ? j0 / (GSUB > 0 ? GSUB : SW_B) : 0;
        const float sc = gs_s[rl * 4 + slot], zc = gz_s[rl * 4 + slot];
        const uint4 wv = w0pre[r];
        const uint32_t cw[2] = {*reinterpret_cast<const uint32_t*>(codes8 + rl * SW_CLD + j0),
                                *reinterpret_cast<const uint32_t*>(codes8 + rl * SW_CLD + j0 + 4)};
        const uint32_t hw[4] = {wv.x, wv.y, wv.z, wv.w};
        float hi[8], lo[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          __half2 h2;
          *reinterpret_cast<uint32_t*>(&h2) = hw[t >> 1];
          const float w0 = (t & 1) ? __high2float(h2) : __low2float(h2);
          const float q = static_cast<float>((cw[t >> 2] >> (8 * (t & 3))) & 0xffu) + qp.lo;
          const float d = __fsub_rn(w0, __fmul_rn(__fsub_rn(q, zc), sc));
          hi[t] = a.Err_lo ? tf32_round(d) : d;
          lo[t] = tf32_round(d - hi[t]);
        }
        const size_t eo = row * a.ld_err + a.err_col0 + bo + j0;
        float4* eh = reinterpret_cast<float4*>(a.Err + eo);
        eh[0] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        eh[1] = make_float4(hi[4], hi[5], hi[6], hi[7]);
        if (a.Err_lo) {
          float4* el = reinterpret_cast<float4*>(a.Err_lo + eo);
          el[0] = make_float4(lo[0], lo[1], lo[2], lo[3]);
          el[1] = make_float4(lo[4], lo[5], lo[6], lo[7]);
        }
      }
    } else if (s1 < n) {
      for (int idx = tid; idx < SW_ROWS * SW_B; idx += SS_THREADS) {
        const int rl = idx / SW_B, j = idx % SW_B;
        if (row0 + rl >= a.m) continue;
        const float e = Es[rl * SW_ELD + j];
        const size_t eo = static_cast<size_t>(row0 + rl) * a.ld_err + a.err_col0 + bo + j;
        if (a.Err_lo) {
          const float hi = tf32_round(e);
          a.Err[eo] = hi;
          a.Err_lo[eo] = tf32_round(e - hi);
        } else {
          a.Err[eo] = e;
        }
      }
    }
    // pack each row's 128 codes into its LSB-first bit stream: one 32-bit word per thread
    {
      const int bits = a.bits;
      const int words = 4 * bits;  // 128 * bits / 32
      const int ldc = n * bits / 32;
      for (int idx = tid; idx < SW_ROWS * words; idx += SS_THREADS) {
        const int rl = idx / words, wi = idx % words;
        if (row0 + rl >= a.m) continue;
        const uint8_t* cr = codes8 + rl * SW_CLD;
        const int b0 = 32 * wi;
        uint32_t word = 0u;
        for (int kk = b0 / bits; kk * bits < b0 + 32; ++kk) {
          const int pos = kk * bits - b0;
          const uint32_t code = cr[kk];
          word |= (pos >= 0) ? (code << pos) : (code >> (-pos));
        }
        a.codes[static_cast<size_t>(row0 + rl) * ldc + (i1 * bits) / 32 + wi] = word;
      }
    }
    __syncthreads();  // the next block restages U and rewrites the errors and codes
  }
}

}  // namespace gptq
