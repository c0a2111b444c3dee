// hessian_tc.cuh — S1: H += 2 X^T X on the sm_100a tensor cores.
//
// ("模型量化实战：从 INT8 PTQ 到 GPTQ 的精度保持与推理加速全解析" §3.2, accumulate_hessian:
//  the calibration Hessian is the running sum of 2 x^T x over the calibration batches.)
//
// X is [n_tok x n] bf16, token-major, exactly as a calibration batch arrives.  H[i][j] is a
// contraction over tokens, so for an output tile H[rows i, cols j] both operands are slices
// of the same X rows: A = X[:, i-block]^T and B = X[:, j-block], both "MN-major" (the
// feature index is contiguous).  TMA loads 64-feature x 64-token boxes with the 128-byte
// swizzle straight into the canonical MN-major layout the tensor core reads, so X is never
// transposed or copied.
//
// Work split: a cluster of two CTAs per 256 x 256 output tile of the upper triangle (tiles
// wholly below the diagonal are never computed); see hessian_syrk_pair_kernel below.  Warp
// roles in each CTA:
//   warp 0      TMA producer (one elected lane), 6-stage ring of 32 KB stages
//   warp 1      tensor-memory allocator; in the even CTA also the MMA issuer (one lane):
//               tcgen05.mma.cta_group::2 kind::f16, M=256, N=256, K=16, bf16 -> fp32 in TMEM
//   warps 2-9   epilogue: TMEM -> registers, fp32 running sums; H += 2 * sums at the end
// The 512 TMEM columns of each CTA hold two 128x256 fp32 accumulators (its rows of the tile).  Each accumulator sums one chunk
// of `chunk_iters` x 64 tokens on the tensor cores; the epilogue then adds that partial sum
// to its register accumulators with round-to-nearest fp32 adds while the other accumulator
// takes the next chunk.  The tensor cores' own accumulation is not round-to-nearest (on a
// long sum of positive terms it drifts low by about 1e-5 relative per 4096 tokens), so
// short chunks keep that drift at the 1e-6 level.
#pragma once

#include "sm100_ptx.cuh"

namespace gptq {

constexpr int HS_BM = 128;                        // tile rows   (features i)
constexpr int HS_BN = 256;                        // tile cols   (features j)
constexpr int HS_BK = 64;                         // tokens per pipeline stage
constexpr int HS_BOX_BYTES = 64 * HS_BK * 2;      // one TMA box: 64 features x 64 tokens, bf16
constexpr int HS_THREADS = 64 + 256;  // producer, MMA, 8 epilogue warps

// ------------------------------------------------------------------------------------------
// The product on CTA pairs.  A cluster of two CTAs owns a 256 x 256 output tile of the
// upper triangle and issues one tcgen05.mma.cta_group::2 (M=256, N=256, K=16) per 16 tokens:
// CTA r loads its own 128 rows of A and its 128-column half of B (32 KB a stage instead of
// 48 KB for the same tensor work per SM), and holds rows 128 r .. 128 r + 127 of the tile in
// its tensor memory and its epilogue registers.  The even CTA issues the MMAs once both
// halves of a stage have landed: both CTAs' copies complete on the even CTA's stage barrier
// (plain per-CTA loads, no multicast).  MMA completion is committed to the stage barriers of
// both CTAs at once; both epilogues report back to the even CTA's accumulator barriers.
constexpr int HP_STAGES = 6;
constexpr int HP_A_BYTES = 128 * HS_BK * 2;       // 16 KB: this CTA's 128 rows
constexpr int HP_B_BYTES = 128 * HS_BK * 2;       // 16 KB: this CTA's half of the 256 columns
constexpr int HP_STAGE_BYTES = HP_A_BYTES + HP_B_BYTES;
constexpr int HP_BAR_BYTES = 8 * (2 * HP_STAGES + 5) + 16;
constexpr int HP_SMEM = HP_STAGES * HP_STAGE_BYTES + HP_BAR_BYTES + 1024;

// Pair tiles: column block bj (256 wide) owns row blocks 0 .. bj (256 high).
__host__ __device__ inline int hp_num_pairs(int n) {
  const int J = (n + 255) / 256;
  return J * (J + 1) / 2;
}

__device__ __forceinline__ void hp_tile_of(int t, int& bi, int& bj) {
  int b = static_cast<int>((sqrtf(8.0f * static_cast<float>(t) + 1.0f) - 1.0f) * 0.5f);
  while (b > 0 && b * (b + 1) / 2 > t) --b;
  while ((b + 1) * (b + 2) / 2 <= t) ++b;
  bj = b;
  bi = t - b * (b + 1) / 2;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(HS_THREADS, 1)
    hessian_syrk_pair_kernel(const __grid_constant__ CUtensorMap xmap, float* __restrict__ H, int n, int n_tok,
                             int chunk_iters, int* __restrict__ status) {
  extern __shared__ uint8_t hs_smem_raw[];
  const uint32_t raw_s = smem_u32(hs_smem_raw);
  uint8_t* smem = hs_smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs; 1: its peer
  const bool leader = rank == 0;

  int bi, bj;
  hp_tile_of(static_cast<int>(blockIdx.x >> 1), bi, bj);
  const int row0 = bi * 256 + 128 * static_cast<int>(rank);  // this CTA's rows (A, TMEM, epilogue)
  const int colb = bj * 256 + 128 * static_cast<int>(rank);  // this CTA's half of B
  const int col0 = bj * 256;                                 // the tile's columns (epilogue)

  const uint32_t bar_full = sbase + HP_STAGES * HP_STAGE_BYTES;
  const uint32_t bar_empty = bar_full + 8 * HP_STAGES;
  const uint32_t bar_tfull = bar_empty + 8 * HP_STAGES;
  const uint32_t bar_tempty = bar_tfull + 16;  // used in the even CTA
  const uint32_t bar_drain = bar_tempty + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + HP_STAGES * HP_STAGE_BYTES + 8 * (2 * HP_STAGES + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int k_iters = (n_tok + HS_BK - 1) / HS_BK;
  const int n_chunks = (k_iters + chunk_iters - 1) / chunk_iters;
  constexpr uint32_t stage_tx = static_cast<uint32_t>(HP_STAGE_BYTES);  // 4 boxes (out-of-range parts zero-filled)

  if (threadIdx.x == 0) {
    for (int s = 0; s < HP_STAGES; ++s) {
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
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&xmap);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers and tensor memory exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();  // inputs of the previous kernel are complete and visible from here on
  griddep_launch_dependents();  // the next kernel may start its prologue now; it waits for our completion

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs, each into its own shared memory) ----------------
      // Both halves of a stage complete on the even CTA's full barrier: the even producer
      // expects the bytes of both, the odd CTA's copies count down on it across the pair.
      const uint32_t lead_full = mapa_shared(bar_full, 0);
      int issued = 0;
      for (int it = 0; it < k_iters; ++it) {
        const int s = it % HP_STAGES;
        const uint32_t ph = static_cast<uint32_t>(it / HP_STAGES) & 1u;
        if (!mbar_wait_bounded_cl(bar_empty + 8 * s, ph ^ 1u, abort_flag)) break;
        if (leader) mbar_arrive_expect_tx(bar_full + 8 * s, 2 * stage_tx);
        const uint32_t fb = lead_full + 8 * s;
        const uint32_t a_s = sbase + s * HP_STAGE_BYTES;
        const uint32_t b_s = a_s + HP_A_BYTES;
        const int tok = it * HS_BK;
        tma_load_2d_pair(a_s, &xmap, fb, row0, tok);
        tma_load_2d_pair(a_s + HS_BOX_BYTES, &xmap, fb, row0 + 64, tok);
        tma_load_2d_pair(b_s, &xmap, fb, colb, tok);
        tma_load_2d_pair(b_s + HS_BOX_BYTES, &xmap, fb, colb + 64, tok);
        issued = it + 1;
      }
      // no TMA write of the pair may still be in flight when either CTA exits: the even CTA
      // waits out the last stages' full barriers (phases its MMA loop already saw complete are
      // passed at once); the odd CTA is held by the closing cluster barrier until then
      if (leader)
        for (int it = max(0, issued - HP_STAGES); it < issued; ++it)
          mbar_wait_drain(bar_full + 8 * (it % HP_STAGES), static_cast<uint32_t>(it / HP_STAGES) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- even CTA: MMA issuer for the pair ----------------
      constexpr uint32_t idesc = idesc_make(1u, 1u, 1u, 1u, 256, HS_BN);  // bf16, MN-major A and B, M=256
      bool ok = true;
      int it = 0;
      for (int c = 0; c < n_chunks && ok; ++c) {
        const int b = c & 1;
        const uint32_t ph = static_cast<uint32_t>(c >> 1) & 1u;
        if (!mbar_wait_bounded_cl(bar_tempty + 8 * b, ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * HS_BN);
        const int it0 = c * chunk_iters;
        const int it_end = min(k_iters, it0 + chunk_iters);
        for (; it < it_end; ++it) {
          const int s = it % HP_STAGES;
          const uint32_t phs = static_cast<uint32_t>(it / HP_STAGES) & 1u;
          if (!mbar_wait_bounded_cl(bar_full + 8 * s, phs, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = sbase + s * HP_STAGE_BYTES;
          const uint32_t b_s = a_s + HP_A_BYTES;
#pragma unroll
          for (int k = 0; k < HS_BK / 16; ++k) {
            // 16 tokens = two 8-row swizzle atoms of 1024 bytes; 64-feature atoms 8 KB apart
            const uint64_t ad = sdesc_sw128(a_s + k * 2048, HS_BOX_BYTES, 1024);
            const uint64_t bd = sdesc_sw128(b_s + k * 2048, HS_BOX_BYTES, 1024);
            umma_f16_pair(d_tmem, ad, bd, idesc, (it > it0 || k > 0) ? 1u : 0u);
          }
          umma_commit_pair_mc(bar_empty + 8 * s, 0x3);
        }
        if (!ok) break;
        umma_commit_pair_mc(bar_tfull + 8 * b, 0x3);
      }
      if (!ok) {
        // MMAs may still be running: wait for them before the TMEM is released
        umma_commit_pair(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
    }
  } else {
    // ---------------- epilogue (both CTAs): TMEM -> registers (fp32) -> H ----------------
    const int q = warp & 3;
    const int hh = (warp - 2) >> 2;
    const int r = row0 + q * 32 + lane;
    const uint32_t lead_tempty = mapa_shared(bar_tempty, 0);
    float acc[HS_BN / 2];
#pragma unroll
    for (int j = 0; j < HS_BN / 2; ++j) acc[j] = 0.0f;
    bool all_ok = true;
    for (int c = 0; c < n_chunks; ++c) {
      const int b = c & 1;
      const uint32_t ph = static_cast<uint32_t>(c >> 1) & 1u;
      int ok = 0;
      if (lane == 0) ok = mbar_wait_bounded_cl(bar_tfull + 8 * b, ph, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        all_ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(b * HS_BN + hh * (HS_BN / 2) + cc * 16),
                           v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[cc * 16 + j] += __uint_as_float(v[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_tempty + 8 * b);
    }
    if (all_ok && r < n) {
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int col = col0 + hh * (HS_BN / 2) + cc * 32;
        if (col < n) {
          float4* dst = reinterpret_cast<float4*>(H + static_cast<size_t>(r) * n + col);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4 h = dst[j];
            h.x = fmaf(2.0f, acc[cc * 32 + 4 * j + 0], h.x);
            h.y = fmaf(2.0f, acc[cc * 32 + 4 * j + 1], h.y);
            h.z = fmaf(2.0f, acc[cc * 32 + 4 * j + 2], h.z);
            h.w = fmaf(2.0f, acc[cc * 32 + 4 * j + 3], h.w);
            dst[j] = h;
          }
        }
      }
    }
  }

  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may still read its shared memory or TMEM
  if (threadIdx.x == 0 && *abort_flag) atomicOr(status, ST_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace gptq
