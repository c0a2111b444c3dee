/*
 * gptq_testing.h — test hooks of libgptq.  Not part of the method's interface: they expose
 * internal kernels so that the test-suite can check them in isolation.
 */
#ifndef GPTQ_B200_TESTING_H
#define GPTQ_B200_TESTING_H

#include "gptq.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The three-product tf32 tensor-core GEMM of the factorization and of the lazy trailing
 * update (S4, S6):  C = alpha * A * B^T (+ C when beta = 1).
 *   A_hi/A_lo : device fp32 [M x K], leading dimension lda (A = A_hi + A_lo; hi/lo are tf32 values)
 *   B_hi/B_lo : device fp32 [N x K], leading dimension ldb
 *   k_lo_mode : 0 = K from 0; 1 = K from the first column of the output tile (B lower-triangular
 *               in this form); 2 = K from the first row of the tile (A upper-triangular);
 *               3 + j (j = 0..3) = K over the aligned block of kblk = 128 * 2^j columns that
 *               holds the output tile only (B block-diagonal with kblk x kblk blocks; the tile
 *               width is then at most kblk; k_hi_mode 1 still stops K at the tile's last column)
 *   k_hi_mode : 0 = K to the end; 1 = K up to the last column of the tile (B upper-triangular)
 *   upper_only: skip output tiles wholly below the diagonal of C
 *   C         : fp32 output [M x N] (ldc) or NULL; C_hi/C_lo: hi/lo output (ldh) or NULL;
 *   Ct_hi/Ct_lo: transposed hi/lo output [N x M] (ldt) or NULL (beta applies to C and C_hi/C_lo).
 *   chunk_stages: 32-wide K stages summed in one tensor-memory accumulator before the fp32
 *               register add (1 = every stage; the trailing update of the sweep uses 4).
 *   tile_n    : output tile width 64, 128 or 256, 512 for the CTA-pair kernel (256 x 256 tiles on
 *               two CTAs), or 0 for the library's own choice.
 *   c_reduce  : 1 = C += alpha A B^T through TMA reduce-add boxes (needs C and beta = 1; C's
 *               base 16-byte aligned, ldc % 4 == 0), the path of the sweep's trailing update.
 * Requirements: N % 32 == 0, K % 32 == 0, 16-byte aligned bases, leading dimensions % 4 == 0.
 * Synchronizes the stream before returning.  Allocates a 4-byte status word (stream-ordered). */
gptq_status gptq_test_gemm_tf32x3(int M, int N, int K, const float* A_hi, const float* A_lo, int lda, const float* B_hi,
                                  const float* B_lo, int ldb, float alpha, int beta, int k_lo_mode, int k_hi_mode,
                                  int upper_only, float* C, int ldc, float* C_hi, float* C_lo, int ldh, float* Ct_hi,
                                  float* Ct_lo, int ldt, int chunk_stages, int tile_n, int c_reduce, int device,
                                  void* cuda_stream);

/* The sweep's division (S5): x / s from the rounded reciprocal of s plus one fused
 * multiply-add correction, compared bit for bit with IEEE division on `count` (x, s) pairs
 * generated on the device from `seed` (random bit patterns, and quotients within a few ulps
 * of the half-integers where a code's rounding is decided).
 *   mismatches: host, receives the number of pairs whose results differ
 *   example   : host float[2] or NULL; receives (x, s) of one differing pair if any
 * Synchronizes the stream before returning.  Allocates 16 bytes (stream-ordered). */
gptq_status gptq_test_div_rn(uint64_t seed, int64_t count, uint64_t* mismatches, float* example, int device,
                             void* cuda_stream);

/* Failure detection of the device-side waits: enqueue on the context's stream a one-CTA
 * kernel that waits on an mbarrier no thread ever arrives on, with the same bounded wait the
 * tcgen05 kernels use but a limit of limit_ns nanoseconds (1 <= limit_ns <= 10 s).  When the
 * wait gives up the kernel records ST_TIMEOUT in the context's status word and returns, so
 * the next gptq_synchronize (or gptq_prepare) reports GPTQ_ERR_TIMEOUT and the context stays
 * usable.  Asynchronous. */
gptq_status gptq_test_bounded_wait(gptq_ctx* ctx, uint64_t limit_ns);

/* Host-only checks of the tensor-core GEMM's work split (no GPU needed).
 * gptq_test_pick_tile_n: the output tile width (64, 128 or 256) the library picks for an
 *   M x N x K product with the given K-range modes on `sms` persistent CTAs; -1 on bad sizes.
 * gptq_test_tile_schedule: walks the schedule of `ctas` persistent CTAs over the tiles of
 *   width tile_n and returns 0 when every tile is visited exactly once, the tiles are
 *   distinct, aligned and in range (with upper_only: exactly the tiles that reach the upper
 *   triangle, otherwise all of them), and every non-empty K range is aligned and within K; otherwise
 *   the number (1-8) of the first check that failed, or -1 on bad arguments. */
int gptq_test_pick_tile_n(int M, int N, int K, int k_lo_mode, int k_hi_mode, int upper_only, int sms);
/* gptq_test_factor_plan (host only, no GPU): the factorization recursion's nodes for a width
 *   n (multiple of 128, up to 32768) in the order gptq_prepare visits them, as int32 triples
 *   (offset, width, 1 when the node's whole U is formed by gptq_prepare, else 0) into
 *   nodes_out[3 * capacity]; leaves are the 128-wide nodes.  spine_out[spine_capacity] (may be
 *   NULL) receives the widths of the nodes at offset 0 whose U gptq_get_factor completes, in
 *   the order it completes them; *spine_count their number.  Returns the number of nodes, or -1
 *   on bad arguments. */
int gptq_test_factor_plan(int64_t n, int32_t* nodes_out, int capacity, int32_t* spine_out, int spine_capacity,
                          int* spine_count);
int gptq_test_tile_schedule(int M, int N, int K, int k_lo_mode, int k_hi_mode, int upper_only, int tile_n, int ctas);
/* gptq_test_pct_position (host only, no GPU): where gptq_rtn_quantize takes the p-th percentile
 *   (0 <= p <= 100) of k >= 1 sorted values: the ranks *lo and *hi of the two order statistics and
 *   the interpolation weights *t and *omt (= 1 - t), exactly as the call passes them to its kernel.
 *   Returns 0, or -1 on bad arguments. */
int gptq_test_pct_position(double p, int k, int* lo, int* hi, float* t, float* omt);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_TESTING_H */
