// dequant_gemm.cuh — the consumer of the packed result: Y = X W16^T on the sm_100a tensor cores.
//
// ("模型量化实战：从 INT8 PTQ 到 GPTQ 的精度保持与推理加速全解析" §4.3: INT4 weights are turned back
//  into FP16 before the matrix product, and what the low-bit storage buys is memory bandwidth.)
//
// A layer kept as the sweep's output (codes packed per row in sweep order, a scale and a
// zero-point per row and group, and the act-order permutation perm) multiplies fp16
// activations X [T x n] (original column order):
//     Y[t][r] = sum_k X[t][perm[k]] * W16[r][k],   W16[r][k] = fp16( fp32(code[r][k] - z) * s )
// with (s, z) the row's parameters of group k / g.  The product runs in sweep order, so the
// activations are gathered by perm once (act-order) and the groups stay contiguous.
//
// One CTA owns 128 weight rows (the MMA's M) and a tile of TN tokens (the MMA's N) over a K
// range (split-K when the grid would not fill the GPU).  Per 128-wide K tile:
//   warp 0      TMA producer (one lane): the rows' packed codes (no swizzle) and the
//               activation tile (two 64-column boxes, 128-byte swizzle) into a stage ring
//   warp 1      TMEM allocator and MMA issuer (one lane): tcgen05.mma kind::f16, M=128, N=TN,
//               K=16, fp16 x fp16 -> fp32 in TMEM
//   warps 2-9   dequantize the stage's codes into an fp16 weight tile (two thread per row, 64
//               columns each), written straight into the swizzled K-major layout the MMA
//               reads (double-buffered), then drain the accumulator at the end
// The dequantized value is formed exactly as the reading states: u - z is exact (small
// integers, via the 2^23 magic constant), times s rounded to nearest in fp32, then rounded to
// nearest fp16 (cvt.rn.f16x2.f32).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace gptq {

constexpr int DQ_BM = 128;                       // weight rows per CTA
constexpr int DQ_BK = 128;                       // K per stage (two 64-column swizzle atoms)
constexpr int DQ_THREADS = 64 + 256;             // producer, MMA, 8 dequant/epilogue warps
constexpr int DQ_A_ATOM = DQ_BM * 64 * 2;        // 16 KB: 128 rows x 64 fp16
constexpr int DQ_A_BYTES = 2 * DQ_A_ATOM;        // 32 KB per dequantized tile
constexpr int DQ_NA_MAX = 4;                     // dequantized tiles in flight: 2, or 4 (decode tiles)
constexpr int DQ_SMEM_BUDGET = 224 * 1024;       // one CTA per SM
constexpr int DQ_SMEM_BUDGET2 = 113 * 1024;      // two CTAs per SM (each also costs the SM 1 KB)

// Launch shape of a tile width and code width: CTAs per SM (minb) and dequantized tiles in flight
// (na).  Few tokens (decode-sized T): the dequantization and the round trip through the MMA set
// the pace, not the MMA's work.  Shape 2 (default there): two CTAs per SM (16 dequantizing warps)
// with two tiles each; shape 4: one CTA with four tiles in flight.  8-bit codes keep one CTA.
struct DqShape {
  int minb, na;
};
__host__ __device__ inline DqShape dq_shape(int tn, int bits, int decode_shape) {
  if (tn <= 32 && decode_shape == 4) return DqShape{1, 4};
  if (tn <= 32 && bits != 8) return DqShape{2, 2};
  return DqShape{1, 2};
}
__host__ __device__ inline int dq_code_bytes(int bits) { return DQ_BM * DQ_BK * bits / 8; }
__host__ __device__ inline int dq_x_atom_bytes(int tn) { return tn * 128; }
__host__ __device__ inline int dq_stage_bytes(int tn, int bits) {
  const int c = (dq_code_bytes(bits) + 1023) / 1024 * 1024;
  return c + 2 * dq_x_atom_bytes(tn);
}
__host__ __device__ inline int dq_stages(int tn, int bits, int minb, int na) {
  const int budget = minb == 2 ? DQ_SMEM_BUDGET2 : DQ_SMEM_BUDGET;
  const int avail = budget - 1024 - 256 - na * DQ_A_BYTES;
  int s = avail / dq_stage_bytes(tn, bits);
  return s < 2 ? 2 : (s > 8 ? 8 : s);
}
__host__ __device__ inline int dq_smem_bytes(int tn, int bits, int minb, int na) {
  return 1024 + na * DQ_A_BYTES + dq_stages(tn, bits, minb, na) * dq_stage_bytes(tn, bits) + 256;
}
__host__ __device__ inline int dq_tmem_cols(int tn) { return tn <= 32 ? 32 : tn; }

struct DqArgs {
  int T, m, n, tn, g, G;
  int k_tiles_per_split;  // K tiles of 128 per CTA (the last split may have fewer)
  int k_tiles;            // n / 128
  float* out;             // Y [T x m] (split 0 only when splits == 1) or partials [splits x T x m]
  const float* scales;    // [m x G]
  const float* zeros;     // [m x G]
  int* status;
};

// Two dequantized values as one fp16 pair: (f0, f1) hold 2^23 + u as fp32 bit patterns;
// f + (-(2^23 + z)) is u - z exactly, times s rounded to nearest in fp32 (the packed fp32x2
// intrinsics: each lane an ordinary correctly rounded operation), then rounded to nearest fp16.
// The low half of the result is f0's value.
__device__ __forceinline__ uint32_t dq_pair(uint32_t f0, uint32_t f1, float2 nzz, float2 ss) {
  const float2 d = __fmul2_rn(__fadd2_rn(make_float2(__uint_as_float(f0), __uint_as_float(f1)), nzz), ss);
  const __half2 h = __floats2half2_rn(d.x, d.y);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Dequantize the 64 codes of one half row (BITS-bit LSB-first stream in `w`) into 8 swizzled
// 16-byte chunks of the fp16 tile.  zm = 2^23 + z.
template <int BITS>
__device__ __forceinline__ void dq_half_row(const uint32_t* w, float s0, float zm0, float s1, float zm1, int g32,
                                            uint32_t dst_row, int r7) {
  const float2 ss0 = make_float2(s0, s0), zz0 = make_float2(-zm0, -zm0), ss1 = make_float2(s1, s1),
               zz1 = make_float2(-zm1, -zm1);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const bool second = g32 && c >= 4;  // columns 32..63 of the half row: the next 32-column group
    const float2 ss = second ? ss1 : ss0, zz = second ? zz1 : zz0;
    uint32_t h2[4];
    if (BITS == 4) {
      // one word holds the chunk's 8 codes: the even ones in the low nibbles of its bytes, the
      // odd ones in the high nibbles; a byte permute puts each under the exponent of 2^23
      const uint32_t ev = w[c] & 0x0F0F0F0Fu, od = (w[c] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
      for (int p = 0; p < 4; ++p)
        h2[p] = dq_pair(__byte_perm(ev, 0x4B000000u, 0x7540u + p), __byte_perm(od, 0x4B000000u, 0x7540u + p), zz, ss);
    } else {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        uint32_t f[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = 8 * c + 2 * p + e;  // column within the half row
          constexpr uint32_t mask = (1u << BITS) - 1u;
          const int bit = j * BITS;
          const int wi = bit >> 5, off = bit & 31;
          uint32_t u = w[wi] >> off;
          if (off + BITS > 32) u |= w[wi + 1] << (32 - off);
          f[e] = 0x4B000000u | (u & mask);
        }
        h2[p] = dq_pair(f[0], f[1], zz, ss);
      }
    }
    const uint32_t a = dst_row + static_cast<uint32_t>(((c ^ r7) << 4));
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(h2[0]), "r"(h2[1]), "r"(h2[2]), "r"(h2[3])
                 : "memory");
  }
}

template <int BITS, int MINB, int NA>
__global__ void __launch_bounds__(DQ_THREADS, MINB)
    dequant_gemm_kernel(const __grid_constant__ CUtensorMap codes_map, const __grid_constant__ CUtensorMap x_map,
                        DqArgs p) {
  extern __shared__ uint8_t dq_smem_raw[];
  const uint32_t raw_s = smem_u32(dq_smem_raw);
  uint8_t* smem = dq_smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  const uint32_t sbase = smem_u32(smem);
  const int tn = p.tn;
  const int stages = dq_stages(tn, BITS, MINB, NA);
  const int stage_bytes = dq_stage_bytes(tn, BITS);
  const int code_bytes = dq_code_bytes(BITS);
  const int code_pad = (code_bytes + 1023) / 1024 * 1024;
  const uint32_t a_base = sbase;                                    // NA dequantized tiles
  const uint32_t st_base = sbase + NA * DQ_A_BYTES;                 // stages: codes | X atom 0 | X atom 1
  const uint32_t bar = st_base + stages * stage_bytes;
  const uint32_t bar_full = bar, bar_empty = bar + 8 * 8, bar_afull = bar + 16 * 8, bar_aempty = bar_afull + 8 * NA,
                 bar_acc = bar_aempty + 8 * NA, bar_drain = bar_acc + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (bar_drain + 8 - sbase));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * DQ_BM;
  const int t0 = blockIdx.y * tn;
  const int kt0 = blockIdx.z * p.k_tiles_per_split;
  const int kt1 = min(p.k_tiles, kt0 + p.k_tiles_per_split);
  const int nk = kt1 - kt0;
  const int tmem_cols = dq_tmem_cols(tn);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int j = 0; j < NA; ++j) {
      mbar_init(bar_afull + 8 * j, 256);
      mbar_init(bar_aempty + 8 * j, 1);
    }
    mbar_init(bar_acc, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(tmem_cols));
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&codes_map);
    tma_prefetch_desc(&x_map);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const uint32_t tx = static_cast<uint32_t>(code_bytes + 2 * dq_x_atom_bytes(tn));
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % stages;
        const uint32_t ph = static_cast<uint32_t>(i / stages) & 1u;
        if (!mbar_wait_bounded(bar_empty + 8 * s, ph ^ 1u, abort_flag)) break;
        const uint32_t fb = bar_full + 8 * s;
        mbar_arrive_expect_tx(fb, tx);
        const uint32_t st = st_base + s * stage_bytes;
        const int kt = kt0 + i;
        tma_load_2d(st, &codes_map, fb, kt * (DQ_BK * BITS / 32), m0);
        tma_load_2d(st + code_pad, &x_map, fb, kt * DQ_BK, t0);
        tma_load_2d(st + code_pad + dq_x_atom_bytes(tn), &x_map, fb, kt * DQ_BK + 64, t0);
        issued = i + 1;
      }
      for (int i = max(0, issued - stages); i < issued; ++i)
        mbar_wait_drain(bar_full + 8 * (i % stages), static_cast<uint32_t>(i / stages) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = idesc_make(0u, 0u, 0u, 0u, DQ_BM, static_cast<uint32_t>(tn));  // f16 x f16, K-major
      bool ok = true;
      for (int i = 0; i < nk && ok; ++i) {
        const int s = i % stages, j = i % NA;
        if (!mbar_wait_bounded(bar_full + 8 * s, static_cast<uint32_t>(i / stages) & 1u, abort_flag) ||
            !mbar_wait_bounded(bar_afull + 8 * j, static_cast<uint32_t>(i / NA) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_t = a_base + j * DQ_A_BYTES;
        const uint32_t x_t = st_base + s * stage_bytes + code_pad;
#pragma unroll
        for (int at = 0; at < 2; ++at)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(a_t + at * DQ_A_ATOM + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(x_t + at * dq_x_atom_bytes(tn) + kk * 32, 16, 1024);
            umma_f16(tmem_base, ad, bd, idesc, (i > 0 || at > 0 || kk > 0) ? 1u : 0u);
          }
        umma_commit(bar_empty + 8 * s);
        umma_commit(bar_aempty + 8 * j);
      }
      if (ok) {
        umma_commit(bar_acc);
      } else {
        umma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
    }
  } else {
    // ---------------- dequantize (two threads per row), then the epilogue ----------------
    const int d = threadIdx.x - 64;
    const int r = d >> 1, h = d & 1;
    const int gr = m0 + r;
    const bool row_ok = gr < p.m;
    const int r7 = r & 7;
    const bool g32 = p.g < 64;
    bool ok = true;
    // group parameters of the next tile, loaded one tile ahead
    auto load_sz = [&](int kt, float& s0, float& zm0, float& s1, float& zm1) {
      const int c0 = kt * DQ_BK + 64 * h;
      const int g0 = c0 / p.g, g1 = (c0 + 32) / p.g;
      if (row_ok) {
        s0 = p.scales[static_cast<size_t>(gr) * p.G + g0];
        zm0 = 8388608.0f + p.zeros[static_cast<size_t>(gr) * p.G + g0];
        s1 = p.scales[static_cast<size_t>(gr) * p.G + g1];
        zm1 = 8388608.0f + p.zeros[static_cast<size_t>(gr) * p.G + g1];
      } else {
        s0 = s1 = 0.0f;
        zm0 = zm1 = 8388608.0f;
      }
    };
    float ns0 = 0.f, nz0 = 0.f, ns1 = 0.f, nz1 = 0.f;
    if (nk > 0) load_sz(kt0, ns0, nz0, ns1, nz1);
    for (int i = 0; i < nk; ++i) {
      const float s0 = ns0, zm0 = nz0, s1 = ns1, zm1 = nz1;
      if (i + 1 < nk) load_sz(kt0 + i + 1, ns0, nz0, ns1, nz1);
      const int s = i % stages, j = i % NA;
      int okw = 1;
      if (lane == 0)
        okw = (mbar_wait_bounded(bar_full + 8 * s, static_cast<uint32_t>(i / stages) & 1u, abort_flag) &&
               mbar_wait_bounded(bar_aempty + 8 * j, (static_cast<uint32_t>(i / NA) & 1u) ^ 1u, abort_flag))
                   ? 1
                   : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) {
        ok = false;
        break;
      }
      // this half row's 2 * BITS code words.  A warp reads 16 rows: with 16-byte loads the
      // first chunk each thread takes is rotated by its row so that the warp's 32 loads fall
      // on distinct bank groups (4-bit: 2 chunks, rotated by row / 2; 8-bit: 4, by row)
      const uint8_t* cw = smem + (st_base - sbase) + s * stage_bytes + r * (16 * BITS) + h * (8 * BITS);
      uint32_t w[2 * BITS];
      if (BITS == 2) {
        const uint4 v = *reinterpret_cast<const uint4*>(cw);
        w[0] = v.x;
        w[1] = v.y;
        w[2] = v.z;
        w[3] = v.w;
      } else if (BITS == 4 || BITS == 8) {
        constexpr int NCH = BITS / 2;  // 16-byte chunks in the half row
        const int rot = (BITS == 4) ? ((r >> 1) & 1) : (r & 3);
        uint4 v[NCH];
#pragma unroll
        for (int q = 0; q < NCH; ++q) v[q] = *reinterpret_cast<const uint4*>(cw + 16 * ((q + rot) & (NCH - 1)));
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          // chunk c was loaded as v[(c - rot) mod NCH] (compile-time indices per rotation)
          const uint4 x = (rot == 0) ? v[c]
                        : (rot == 1) ? v[(c + NCH - 1) & (NCH - 1)]
                        : (rot == 2) ? v[(c + NCH - 2) & (NCH - 1)]
                                     : v[(c + NCH - 3) & (NCH - 1)];
          w[4 * c] = x.x;
          w[4 * c + 1] = x.y;
          w[4 * c + 2] = x.z;
          w[4 * c + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < BITS; ++q) {
          const uint2 v = *reinterpret_cast<const uint2*>(cw + 8 * q);
          w[2 * q] = v.x;
          w[2 * q + 1] = v.y;
        }
      }
      const uint32_t dst_row = a_base + j * DQ_A_BYTES + h * DQ_A_ATOM + (r >> 3) * 1024 + r7 * 128;
      dq_half_row<BITS>(w, s0, zm0, s1, zm1, g32 ? 1 : 0, dst_row, r7);
      fence_proxy_async_smem();
      mbar_arrive(bar_afull + 8 * j);
    }
    // epilogue: warp (q, hh) drains TMEM lanes 32 q .. 32 q + 31 (its rows), 16-column chunks
    // hh, hh + 2, ...; lane = row, so each token's 32 outputs are one coalesced 128-byte store
    const int q = warp & 3, hh = (warp - 2) >> 2;
    int okw = ok ? 1 : 0;
    if (ok && nk > 0) {
      if (lane == 0) okw = mbar_wait_bounded(bar_acc, 0u, abort_flag) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
    }
    if (okw && nk > 0) {
      tc_fence_after();
      const int row = m0 + q * 32 + lane;
      float* out = p.out + static_cast<size_t>(blockIdx.z) * p.T * p.m;
      for (int cc = hh; cc < tn / 16; cc += 2) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(cc * 16), v);
        tmem_ld_wait();
        if (row < p.m) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int t = t0 + cc * 16 + jj;
            if (t < p.T) out[static_cast<size_t>(t) * p.m + row] = __uint_as_float(v[jj]);
          }
        }
      }
      tc_fence_before();
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, ST_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, static_cast<uint32_t>(tmem_cols));
  }
}

// Xp[t][k] = X[t][perm[k]] (fp16), one CTA per token row, the row staged in shared memory.
__global__ void __launch_bounds__(256) permute_x_kernel(const __half* __restrict__ X, int n,
                                                        const int32_t* __restrict__ perm, __half* __restrict__ Xp) {
  extern __shared__ __half px_row[];
  const int t = blockIdx.x;
  const __half* src = X + static_cast<size_t>(t) * n;
  for (int k = threadIdx.x; k < n; k += blockDim.x) px_row[k] = src[k];
  __syncthreads();
  __half* dst = Xp + static_cast<size_t>(t) * n;
  for (int k = threadIdx.x; k < n; k += blockDim.x) dst[k] = px_row[perm[k]];
}

// Y[t][r] = sum over splits s = 0 .. S-1, in that order, of P[s][t][r].
__global__ void splitk_reduce_kernel(const float* __restrict__ P, int splits, size_t count, float* __restrict__ Y) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float acc = P[i];
    for (int s = 1; s < splits; ++s) acc += P[static_cast<size_t>(s) * count + i];
    Y[i] = acc;
  }
}

// The next layer's inputs from a layer's output (sequential quantization): x = act(y), act 0 =
// identity, 1 = ReLU (y if y > 0, else 0), from fp32 or bf16 y, written as bf16 and/or fp16
// (round to nearest even).  Grid-stride, one element per thread and step.
__global__ void activation_convert_kernel(const void* __restrict__ Y, int in_bf16, size_t count, int act,
                                          __nv_bfloat16* __restrict__ out_bf16, __half* __restrict__ out_fp16) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float y = in_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(Y)[i]) : static_cast<const float*>(Y)[i];
    if (act == 1) y = (y > 0.0f) ? y : 0.0f;
    if (out_bf16) out_bf16[i] = __float2bfloat16_rn(y);
    if (out_fp16) out_fp16[i] = __float2half_rn(y);
  }
}

}  // namespace gptq
