// gptq_api.cu — the C ABI declared in include/gptq.h: context, argument checks and the
// launch sequence of the sm_100a kernels on the context's stream.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>
#include <thread>

#include "../../include/gptq.h"
#include "../../include/gptq_testing.h"
#include "awq_kernels.cuh"
#include "dequant_gemm.cuh"
#include "factor_kernels.cuh"
#include "gemm_tc.cuh"
#include "hessian_tc.cuh"
#include "prepare_kernels.cuh"
#include "sgemm_simt.cuh"
#include "slab_sweep.cuh"
#include "sweep_kernels.cuh"

using namespace gptq;

namespace {

enum CtxState { ST_ACCUM = 0, ST_PREPARED = 1 };

constexpr int64_t kMaxN = 32768;
constexpr int kSuperBlock = 1024;  // widest slab: the block-error buffer holds this many columns
// Columns per slab (super-block) of the sweep: the slab kernel's in-slab updates run on the CUDA
// cores and grow with the slab's width, the products past the slab run on the tensor cores and
// grow in number as slabs narrow; measured on B200, 256 columns is fastest up to 8192-wide
// layers, 512 beyond (the 28672-wide layer: 46.9 ms against 48.0 ms for its quantize stage).
int slab_default(int n) { return n > 8192 ? 512 : 256; }
constexpr int64_t kMaxM = int64_t(1) << 24;

}  // namespace

struct gptq_ctx {
  int device = 0;
  cudaStream_t stream = nullptr;
  int64_t n = 0, m_max = 0;
  float* H = nullptr;                          // [n x n] accumulated Hessian (upper triangle until mirrored)
  float *A_hi = nullptr, *A_lo = nullptr;      // [n x n] damped, permuted H; Schur complements.  After the
                                               // factorization: Vs^T = (V blockdiag(U_SS))^T as tf32
                                               // hi/lo in their lower triangles (vs_width = S)
  float *VT_hi = nullptr, *VT_lo = nullptr;    // [n x n] V12 blocks (upper) and T^T blocks (lower)
  float *U_hi = nullptr, *U_lo = nullptr;      // [n x n] U (upper)
  float* U32 = nullptr;                        // [n x n] U as plain fp32 (upper; read by the sweep)
  float *Ut_hi = nullptr, *Ut_lo = nullptr;    // [n x n] U^T
  float* Wq = nullptr;                         // [m_max x n] fp32 working weights
  __half* W0h = nullptr;                       // [m_max x n] the layer's weights in sweep order (dead columns 0)
  float *Err_hi = nullptr, *Err_lo = nullptr;  // [m_max x kSuperBlock] block errors of a super-block
  float* keys = nullptr;
  uint8_t* dead = nullptr;
  int32_t* perm = nullptr;
  double* mean = nullptr;
  int* status = nullptr;      // device status word
  int* status_host = nullptr; // pinned mirror
  int64_t n_tok = 0;
  int state = ST_ACCUM;
  int mirrored = 0;           // H's lower triangle has been filled
  bool u_complete = false;    // U holds every block (the factorization leaves the blocks no step needs)
  int vs_width = 0;           // slab width S of the Vs held in A (0: none since the last prepare)
  int64_t chunk_tokens = 1024;
  int64_t launches = 0;       // kernels launched by this context (instrumentation)
  int num_sms = 148;
  // tensor maps of whole matrices, encoded once: A-operand maps (128-row boxes) and
  // B-operand maps (256-row boxes), hi and lo
  CUtensorMap mA_A[2], mA_VT[2], mA_U[2], mA_Err[2];
  CUtensorMap mB_U[2], mB_VT[2], mB_Ut[2], mB_Vb[2];
  CUtensorMap mC_Wq;  // Wq as the reduce-add target of the trailing update (32 x 32 boxes)
  cudaStream_t capture_stream = nullptr;
  cudaStream_t side_stream = nullptr;     // second branch of the captured factorization graph
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  bool pdl = true;                        // launches overlap their predecessor (programmatic)
  cudaGraphExec_t factor_graph = nullptr;  // the factorization recursion, recorded once
  int64_t factor_graph_launches = 0;
  int gemm_role = 0;                      // which product gemm_tc runs (instrumentation): GR_*
  int factor_chunk = 4;                   // K stages per TMEM accumulator in the factorization's products
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  // per-kernel instrumentation (gptq_set_profiling): the role and algorithmic work of the next
  // launch, and one record (two timing events) per launch while profiling is on
  bool prof = false;
  const char* tag = "other";
  double tag_flops = 0.0, tag_bytes = 0.0;
  struct ProfRec {
    const char* tag;
    double flops, bytes;
    cudaEvent_t e0, e1;
  };
  std::vector<ProfRec> prof_recs;
  bool prof_error = false;
};

namespace {

gptq_status cuda_fail(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return GPTQ_OK;
  if (std::getenv("GPTQ_VERBOSE")) std::fprintf(stderr, "gptq: %s: %s\n", what, cudaGetErrorString(e));
  return GPTQ_ERR_CUDA;
}
#define CK(call)                                         \
  do {                                                   \
    gptq_status _s = cuda_fail((call), #call);           \
    if (_s != GPTQ_OK) return _s;                        \
  } while (0)
#define CKL(what) CK(cudaGetLastError())

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

class DeviceGuard {
 public:
  explicit DeviceGuard(int dev) {
    cudaGetDevice(&prev_);
    cudaSetDevice(dev);
  }
  ~DeviceGuard() { cudaSetDevice(prev_); }

 private:
  int prev_ = 0;
};

int64_t env_int(const char* name, int64_t dflt) {
  const char* v = std::getenv(name);
  if (!v || !*v) return dflt;
  return std::strtoll(v, nullptr, 10);
}

// Bounded host wait for everything enqueued so far on the context's stream.
gptq_status wait_stream(gptq_ctx* c) {
  cudaEvent_t ev;
  CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
  cudaError_t e = cudaEventRecord(ev, c->stream);
  if (e != cudaSuccess) {
    cudaEventDestroy(ev);
    return cuda_fail(e, "cudaEventRecord");
  }
  const int64_t limit_ms = env_int("GPTQ_SYNC_TIMEOUT_MS", 600000);
  const auto t0 = std::chrono::steady_clock::now();
  gptq_status st = GPTQ_OK;
  for (;;) {
    e = cudaEventQuery(ev);
    if (e == cudaSuccess) break;
    if (e != cudaErrorNotReady) {
      st = cuda_fail(e, "cudaEventQuery");
      break;
    }
    const auto ms =
        std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count();
    if (ms > limit_ms) {
      st = GPTQ_ERR_TIMEOUT;
      break;
    }
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
  cudaEventDestroy(ev);
  return st;
}

// Read (and clear) the device status word; waits for the stream.
gptq_status read_status(gptq_ctx* c, int* flags) {
  CK(cudaMemcpyAsync(c->status_host, c->status, sizeof(int), cudaMemcpyDeviceToHost, c->stream));
  gptq_status st = wait_stream(c);
  if (st != GPTQ_OK) return st;
  *flags = *c->status_host;
  if (*flags) CK(cudaMemsetAsync(c->status, 0, sizeof(int), c->stream));
  return GPTQ_OK;
}

gptq_status status_from_flags(int f) {
  if (f & ST_TIMEOUT) return GPTQ_ERR_TIMEOUT;
  if (f & ST_NOT_PD) return GPTQ_ERR_NOT_PD;
  if (f & ST_INTERNAL) return GPTQ_ERR_CUDA;
  return GPTQ_OK;
}

// Launch a kernel on the context's stream with programmatic stream serialization, so that it
// can be scheduled while its predecessor finishes (every kernel waits on griddepcontrol.wait
// before it reads its inputs).
template <typename... KArgs, typename... Args>
cudaError_t launch(gptq_ctx* c, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c->stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (c->pdl && !c->prof) ? 1 : 0;
  ++c->launches;
  const char* tag = c->tag;
  const double fl = c->tag_flops, by = c->tag_bytes;
  c->tag = "other";
  c->tag_flops = c->tag_bytes = 0.0;
  if (!c->prof) return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  gptq_ctx::ProfRec r{tag, fl, by, nullptr, nullptr};
  if (cudaEventCreate(&r.e0) != cudaSuccess || cudaEventCreate(&r.e1) != cudaSuccess) {
    if (r.e0) cudaEventDestroy(r.e0);
    c->prof_error = true;
    cudaGetLastError();
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  }
  cudaEventRecord(r.e0, c->stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  cudaEventRecord(r.e1, c->stream);
  c->prof_recs.push_back(r);
  return e;
}

// Role and algorithmic work of the next launch (instrumentation only).
void tag(gptq_ctx* c, const char* name, double flops, double bytes) {
  c->tag = name;
  c->tag_flops = flops;
  c->tag_bytes = bytes;
}

// Algorithmic flops of C (+)= A B^T with the K ranges and output triangle gemm_tc uses:
// 2 x the nonzero multiply-adds, element (r, c) of C taking k in [kb, ke) with kb = c (B
// lower in K-major form), r (A upper) or 0, ke = c + 1 (B upper) or K; upper_only keeps r <= c.
double gemm_algo_flops(int M, int N, int K, int klo, int khi, int upper) {
  double total = 0.0;
  if (klo >= GT_KLO_BLK) {  // block-diagonal B (upper-triangular blocks with K_HI_COL): the rows
    const int kblk = gt_kblk(klo);  // above the column's block are the ones a caller reads
    for (int col = 0; col < N; ++col) {
      const int64_t b0 = (col / kblk) * kblk;
      const int64_t kc = (khi == GT_KHI_COL) ? col - b0 + 1 : std::min<int64_t>(kblk, K - b0);
      total += static_cast<double>(std::min<int64_t>(M, b0)) * static_cast<double>(kc);
    }
    return 2.0 * total;
  }
  for (int col = 0; col < N; ++col) {
    const int64_t R = upper ? std::min<int64_t>(M, col + 1) : M;
    const int64_t ke = (khi == GT_KHI_COL) ? std::min<int64_t>(K, col + 1) : K;
    if (klo == GT_KLO_ROW) {
      const int64_t q = std::min<int64_t>(R, ke);
      total += static_cast<double>(q * ke - q * (q - 1) / 2);
    } else {
      const int64_t kb = (klo == GT_KLO_COL) ? col : 0;
      total += static_cast<double>(R) * static_cast<double>(std::max<int64_t>(0, ke - kb));
    }
  }
  return 2.0 * total;
}

// 2-D fp32 tensor map of a row-major sub-matrix (rows x cols, leading dimension ld), boxes of
// 32 columns x box_rows rows, 128-byte swizzle.
gptq_status make_map(gptq_ctx* c, CUtensorMap* map, const float* base, int64_t rows, int64_t cols, int64_t ld,
                     int box_rows) {
  if (!aligned16(base) || ld % 4 || cols % GT_BK) return GPTQ_ERR_ARG;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
  const cuuint32_t box[2] = {GT_BK, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = c->encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_ERR_CUDA;
}

// C (+)= alpha * A B^T on the tensor cores, operands as tf32 hi/lo pairs (gemm_tc.cuh).
struct TcOut {
  float* C = nullptr;
  int ldc = 0;
  float* Chi = nullptr;
  float* Clo = nullptr;
  int ldh = 0;
  float* Cthi = nullptr;
  float* Ctlo = nullptr;
  int ldt = 0;
  const CUtensorMap* c_map = nullptr;  // C += ... by TMA reduce-add (beta = 1, plain C)
  int c_row0 = 0, c_col0 = 0;           // offset of C inside the matrix c_map describes
};

// An operand of gemm_tc: the hi/lo tensor maps of a whole matrix and the sub-block offset,
// plus the sub-block's hi/lo pointers and leading dimension (for the CUDA-core path).
struct TcOperand {
  const CUtensorMap* hi;
  const CUtensorMap* lo;
  int row0, col0;
  const float* phi;
  const float* plo;
  int ld;
};

// Roles of the products gemm_tc runs (instrumentation names: kernel:role).
enum : int { GR_V12 = 0, GR_SYRK, GR_T, GR_U12, GR_VB, GR_NEAR, GR_FAR, GR_TEST, GR_COUNT };
const char* const kGemmTcNames[GR_COUNT] = {"gemm_tf32x3:factor_v12",    "gemm_tf32x3:factor_syrk",
                                            "gemm_tf32x3:factor_t",      "gemm_tf32x3:factor_u12",
                                            "gemm_tf32x3:trailing_vs",   "gemm_tf32x3:trailing_near",
                                            "gemm_tf32x3:trailing_far",  "gemm_tf32x3:test"};
const char* const kGemmSimtNames[GR_COUNT] = {"gemm_hilo_simt:factor_v12",    "gemm_hilo_simt:factor_syrk",
                                              "gemm_hilo_simt:factor_t",      "gemm_hilo_simt:factor_u12",
                                              "gemm_hilo_simt:trailing_vs",   "gemm_hilo_simt:trailing_near",
                                              "gemm_hilo_simt:trailing_far",  "gemm_hilo_simt:test"};

// Products with fewer tensor-core tiles (at the narrowest tile) than this run on the CUDA
// cores (fp32, 32 x 32 or 64 x 64 tiles).
constexpr int kMinTcTiles = 32;

cudaError_t set_gemm_tc_attributes() {
  cudaError_t e = cudaFuncSetAttribute(gemm_tf32x3_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       GtCfg<256>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tf32x3_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, GtCfg<128>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tf32x3_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, GtCfg<64>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tf32x3_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GP_SMEM);
  return e;
}

// Tile width of a tensor-core product: the one with the least modelled time.  A tile costs
// (K stages + 2 for the pipeline fill and the epilogue) x (BN + 64): a stage's MMAs grow with
// the tile width, plus a part that does not (issue, barriers, the A operand).  The CTAs take
// tiles in the snake order of gt_sched and the time is that of the busiest CTA.  Products with
// triangular K ranges are simulated tile by tile (they are recorded once, in the factorization
// graph); the others have equal tiles.
int64_t gemm_cost(int M, int N, int K, int klo, int khi, int upper, int bn, int sms) {
  const int ntiles = gt_num_tiles(M, N, upper, bn);
  const int G = std::min(ntiles, sms);
  if (G <= 0) return 0;
  if (klo == GT_KLO_NONE && khi == GT_KHI_NONE) {
    const int64_t waves = (ntiles + G - 1) / G;
    return waves * ((K + GT_BK - 1) / GT_BK + 2) * (bn + 64);
  }
  std::vector<int64_t> load(G, 0);
  for (int t = 0; t < ntiles; ++t) {
    int m0, n0, kb, ni;
    gt_tile_at(M, N, K, klo, khi, upper, bn, t, m0, n0, kb, ni);
    const int r = t / G, q = t % G;
    const int b = (r & 1) ? G - 1 - q : q;
    load[b] += static_cast<int64_t>(ni + 2) * (bn + 64);
  }
  return *std::max_element(load.begin(), load.end());
}

int pick_bn(int M, int N, int K, int klo, int khi, int upper, int sms) {
  int best = 256;
  int64_t best_cost = -1;
  for (int bn : {256, 128, 64}) {
    if (klo >= GT_KLO_BLK && bn > gt_kblk(klo)) continue;  // a tile must not span two blocks of B
    const int64_t cost = gemm_cost(M, N, K, klo, khi, upper, bn, sms);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

gptq_status gemm_tc(gptq_ctx* c, int M, int N, int K, TcOperand A, TcOperand B, float alpha, int beta, int klo,
                    int khi, int upper, const TcOut& o, int chunk_stages = 1, int force_bn = 0) {
  if (M <= 0 || N <= 0) return GPTQ_OK;
  if (N % 32 || K % GT_BK) return GPTQ_ERR_ARG;
  if (klo > GT_KLO_BLK_LAST || (klo >= GT_KLO_BLK && force_bn > gt_kblk(klo))) return GPTQ_ERR_ARG;
  // force_bn 512: the CTA-pair kernel (256 x 256 tiles), for tests
  if (force_bn == 2 * GP_BN && klo >= GT_KLO_BLK) return GPTQ_ERR_ARG;
  const int bn = force_bn == 2 * GP_BN ? GP_BN : (force_bn ? force_bn : pick_bn(M, N, K, klo, khi, upper, c->num_sms));
  const int tc_tiles = gt_num_tiles(M, N, upper, bn);
  if (gt_num_tiles(M, N, upper, 64) < kMinTcTiles && A.phi && B.phi) {
    GemmSimtArgs g;
    g.M = M;
    g.N = N;
    g.K = K;
    g.A_hi = A.phi;
    g.A_lo = A.plo;
    g.lda = A.ld;
    g.B_hi = B.phi;
    g.B_lo = B.plo;
    g.ldb = B.ld;
    g.alpha = alpha;
    g.beta = beta;
    g.k_lo_mode = klo;
    g.k_hi_mode = khi;
    g.upper_only = upper;
    g.C = o.C;
    g.ldc = o.ldc;
    g.Chi = o.Chi;
    g.Clo = o.Clo;
    g.ldh = o.ldh;
    g.Cthi = o.Cthi;
    g.Ctlo = o.Ctlo;
    g.ldt = o.ldt;
    tag(c, kGemmSimtNames[c->gemm_role], gemm_algo_flops(M, N, K, klo, khi, upper), 0.0);
    if (static_cast<int64_t>(M) * N <= 512 * 512) {  // 32 x 32 tiles: more CTAs for the smallest products
      dim3 grid((N + 31) / 32, (M + 31) / 32);
      CK(launch(c, gemm_hilo_simt_kernel<32, 32>, grid, dim3(GS_THREADS), gs_smem_bytes<32, 32>(), g));
    } else {
      dim3 grid((N + 63) / 64, (M + 63) / 64);
      CK(launch(c, gemm_hilo_simt_kernel<64, 64>, grid, dim3(GS_THREADS), gs_smem_bytes<64, 64>(), g));
    }
    CKL("gemm_simt");
    return GPTQ_OK;
  }
  GemmTCArgs a;
  a.chunk_stages = chunk_stages;
  a.M = M;
  a.N = N;
  a.K = K;
  a.a_row0 = A.row0;
  a.a_col0 = A.col0;
  a.b_row0 = B.row0;
  a.b_col0 = B.col0;
  a.alpha = alpha;
  a.beta = beta;
  a.k_lo_mode = klo;
  a.k_hi_mode = khi;
  a.upper_only = upper;
  a.C = o.C;
  a.ldc = o.ldc;
  a.Chi = o.Chi;
  a.Clo = o.Clo;
  a.ldh = o.ldh;
  a.Cthi = o.Cthi;
  a.Ctlo = o.Ctlo;
  a.ldt = o.ldt;
  a.c_reduce = o.c_map ? 1 : 0;
  a.c_row0 = o.c_row0;
  a.c_col0 = o.c_col0;
  a.status = c->status;
  if (o.c_map && (beta != 1 || !o.C)) return GPTQ_ERR_ARG;
  const CUtensorMap& cm = o.c_map ? *o.c_map : *A.hi;  // unused unless c_reduce
  const dim3 grid(std::min(tc_tiles, c->num_sms));
  tag(c, kGemmTcNames[c->gemm_role], gemm_algo_flops(M, N, K, klo, khi, upper), 0.0);
  // Products with wide tiles and work for at least two waves of SM pairs run on CTA pairs
  // (256 x 256 tiles, each CTA loading half of B: a third fewer L2 bytes per flop).  Measured on
  // the 8192 x 28672 layer (same box, alternating runs): the updates past a slab 27.5 ms against
  // 32.8 ms; with four K stages per TMEM chunk the factorization's V12 18.9 ms against 25.6 ms and
  // its SYRK 19.7 ms against 22.6 ms.  GPTQ_GEMM_PAIR: 0 off, 1 dense products only, 2 (default)
  // every eligible product.
  const int pair_tiles = gt_num_tiles(M, N, upper, GP_BN, GP_BM);
  const bool dense = klo == GT_KLO_NONE && khi == GT_KHI_NONE && !upper;
  const int64_t pair_mode = env_int("GPTQ_GEMM_PAIR", 2);
  const bool pair = bn == GP_BN && klo < GT_KLO_BLK &&
                    (force_bn == 2 * GP_BN ||
                     (force_bn == 0 && pair_tiles >= c->num_sms && (pair_mode == 2 || (pair_mode == 1 && dense))));
  if (pair) {
    const dim3 pgrid(2 * std::min(pair_tiles, c->num_sms / 2));
    CK(launch(c, gemm_tf32x3_pair_kernel, pgrid, dim3(GT_THREADS), GP_SMEM, *A.hi, *A.lo, *B.hi, *B.lo, cm, a));
  } else if (bn == 256)
    CK(launch(c, gemm_tf32x3_kernel<256>, grid, dim3(GT_THREADS), GtCfg<256>::SMEM, *A.hi, *A.lo, *B.hi, *B.lo, cm, a));
  else if (bn == 128)
    CK(launch(c, gemm_tf32x3_kernel<128>, grid, dim3(GT_THREADS), GtCfg<128>::SMEM, *A.hi, *A.lo, *B.hi, *B.lo, cm, a));
  else
    CK(launch(c, gemm_tf32x3_kernel<64>, grid, dim3(GT_THREADS), GtCfg<64>::SMEM, *A.hi, *A.lo, *B.hi, *B.lo, cm, a));
  CKL("gemm_tc");
  return GPTQ_OK;
}

// The recursion's products, for the node [o, o+h) = [o, o2) + [o2, o+h) (h1 + h2 columns).
// A, V, T and U share the n x n index space: the node's V12 sits at rows [o, o2), columns
// [o2, o+h) of VT (upper), T^T below the diagonal of VT, U and U^T in their own arrays.
TcOperand fop(CUtensorMap* m, float* hi, float* lo, int n, int r0, int c0) {
  return TcOperand{&m[0], &m[1], r0, c0, hi + static_cast<size_t>(r0) * n + c0, lo + static_cast<size_t>(r0) * n + c0, n};
}
float* at(float* M, int n, int r, int col) { return M + static_cast<size_t>(r) * n + col; }

// T^T = (V12 U22)^T into the lower block [o2.., o..]   (Ut22 rows as B; k <= column)
gptq_status t_product(gptq_ctx* c, int o, int o2, int h1, int h2) {
  const int n = static_cast<int>(c->n);
  TcOut tt;
  tt.Cthi = at(c->VT_hi, n, o2, o);
  tt.Ctlo = at(c->VT_lo, n, o2, o);
  tt.ldt = n;
  c->gemm_role = GR_T;
  return gemm_tc(c, h1, h2, h2, fop(c->mA_VT, c->VT_hi, c->VT_lo, n, o, o2), fop(c->mB_Ut, c->Ut_hi, c->Ut_lo, n, o2, o2),
                 1.f, 0, GT_KLO_NONE, GT_KHI_COL, 0, tt, c->factor_chunk);
}

// U12 = -U11 T  (and Ut21 = U12^T)      (U11 rows as A; k >= row)
gptq_status u12_product(gptq_ctx* c, int o, int o2, int h1, int h2) {
  const int n = static_cast<int>(c->n);
  TcOut u12;
  u12.C = at(c->U32, n, o, o2);
  u12.ldc = n;
  u12.Chi = at(c->U_hi, n, o, o2);
  u12.Clo = at(c->U_lo, n, o, o2);
  u12.ldh = n;
  u12.Cthi = at(c->Ut_hi, n, o2, o);
  u12.Ctlo = at(c->Ut_lo, n, o2, o);
  u12.ldt = n;
  c->gemm_role = GR_U12;
  return gemm_tc(c, h1, h2, h1, fop(c->mA_U, c->U_hi, c->U_lo, n, o, o), fop(c->mB_VT, c->VT_hi, c->VT_lo, n, o2, o),
                 -1.f, 0, GT_KLO_ROW, GT_KHI_NONE, 0, u12, c->factor_chunk);
}

// Width of the left part of a node of h columns: half the leaves; on the recursion's left edge
// (need_u false) a multiple of kSuperBlock, so that every aligned slab of up to kSuperBlock
// columns lies inside one node whose U is computed in full.
int split_left(int h, bool need_u) {
  if (need_u) return h - ((h / LF_NB) / 2) * LF_NB;
  const int h1 = ((h / 2 + kSuperBlock / 2) / kSuperBlock) * kSuperBlock;
  return std::min(std::max(h1, kSuperBlock), h - LF_NB);
}

// The reverse-ordered Cholesky factor V (H = V V^T, V upper) of the diagonal block [o, o+h) of
// A, h a multiple of the 128-column leaf, and U = V^-1 of that block when need_u:
//   V22 = f(A22); V12 = A12 U22^T; A11 -= V12 V12^T; V11 = f(A11); U12 = -U11 V12 U22.
// Every V12 needs the whole U of its node's right part, so right parts are inverted in full;
// the nodes wider than kSuperBlock on the left edge of the recursion (the root, its left
// part, ...) skip T and U12.  The sweep reads V and the diagonal slab blocks of U only (its
// errors satisfy E U = W0 - Q, so the errors of the columns before a slab reach it as
// (W0 - Q) V[., slab] U[slab, slab], see quantize); gptq_get_factor computes the skipped
// blocks when asked (complete_factor).
gptq_status chol_inv(gptq_ctx* c, int o, int h, bool need_u) {
  const int n = static_cast<int>(c->n);
  if (h <= LF_NB) {
    tag(c, "leaf_chol_inv", 2.0 * LF_NB * LF_NB * LF_NB / 3.0, 4.0 * LF_NB * LF_NB * 4);
    CK(launch(c, leaf_chol_inv_kernel, dim3(1), dim3(LF_THREADS), LF_SMEM, c->A_hi, c->A_lo, n, o, c->U_hi, c->U_lo,
              c->U32, c->status));
    CKL("leaf_chol_inv");
    // U^T of the block, needed only by later T products and the block-diagonal product Vb: on
    // the second branch while it exists (the factorization graph), in line otherwise
    const bool branch = c->side_stream != nullptr;
    cudaStream_t main_stream = c->stream;
    if (branch) {
      CK(cudaEventRecord(c->ev_fork, main_stream));
      CK(cudaStreamWaitEvent(c->side_stream, c->ev_fork, 0));
      c->stream = c->side_stream;
      c->pdl = false;
    }
    tag(c, "transpose_block", 0.0, 4.0 * LF_NB * LF_NB * 4);
    const cudaError_t e = launch(c, transpose_block_kernel, dim3(4, 4), dim3(32, 8), 0, c->U_hi, c->U_lo, n, o,
                                 c->Ut_hi, c->Ut_lo);
    if (branch) {
      c->stream = main_stream;
      c->pdl = true;
    }
    CK(e);
    CKL("transpose_block");
    return GPTQ_OK;
  }
  if (h <= kSuperBlock) need_u = true;
  const int h1 = split_left(h, need_u), h2 = h - h1;
  const int o2 = o + h1;
  gptq_status s;
  if ((s = chol_inv(c, o2, h2, true)) != GPTQ_OK) return s;
  // V12 = A12 U22^T                      (U22 rows are the K-major B; k >= column)
  TcOut v12;
  v12.Chi = at(c->VT_hi, n, o, o2);
  v12.Clo = at(c->VT_lo, n, o, o2);
  v12.ldh = n;
  c->gemm_role = GR_V12;
  if ((s = gemm_tc(c, h1, h2, h2, fop(c->mA_A, c->A_hi, c->A_lo, n, o, o2), fop(c->mB_U, c->U_hi, c->U_lo, n, o2, o2),
                   1.f, 0, GT_KLO_COL, GT_KHI_NONE, 0, v12, c->factor_chunk)) != GPTQ_OK)
    return s;
  // A11 -= V12 V12^T                     (upper tiles only)
  TcOut a11;
  a11.Chi = at(c->A_hi, n, o, o);
  a11.Clo = at(c->A_lo, n, o, o);
  a11.ldh = n;
  c->gemm_role = GR_SYRK;
  if ((s = gemm_tc(c, h1, h1, h2, fop(c->mA_VT, c->VT_hi, c->VT_lo, n, o, o2), fop(c->mB_VT, c->VT_hi, c->VT_lo, n, o, o2),
                   -1.f, 1, GT_KLO_NONE, GT_KHI_NONE, 1, a11, c->factor_chunk)) != GPTQ_OK)
    return s;
  if (!need_u) return chol_inv(c, o, h1, false);
  // T is needed only by U12 below, so while the graph is being captured it runs on a second
  // branch, beside the factorization of A11 (which touches only [o, o+h1)^2).
  const bool branch = c->side_stream != nullptr;
  cudaStream_t main_stream = c->stream;
  if (branch) {
    CK(cudaEventRecord(c->ev_fork, main_stream));
    CK(cudaStreamWaitEvent(c->side_stream, c->ev_fork, 0));
    c->stream = c->side_stream;
    c->pdl = false;
  }
  s = t_product(c, o, o2, h1, h2);
  if (branch) {
    c->stream = main_stream;
    c->pdl = true;
    if (s == GPTQ_OK) CK(cudaEventRecord(c->ev_join, c->side_stream));
  }
  if (s != GPTQ_OK) return s;
  if ((s = chol_inv(c, o, h1, true)) != GPTQ_OK) return s;
  // the join: the latest T on the branch (branch launches are in order, so this one too)
  if (branch) CK(cudaStreamWaitEvent(main_stream, c->ev_join, 0));
  return u12_product(c, o, o2, h1, h2);
}

// Vs = V blockdiag(U_SS) for slabs of S columns: every aligned S-column block of V above the
// diagonal times the U block of its columns, in one launch (block-diagonal K ranges), written
// transposed as tf32 hi/lo into the lower triangles of A_hi and A_lo (the K-major operand of
// the product past a slab).  Tiles on the diagonal compute values nothing reads.
gptq_status vs_product(gptq_ctx* c, int S) {
  const int n = static_cast<int>(c->n);
  int mode = GT_KLO_BLK;
  while (gt_kblk(mode) < S) ++mode;
  if (gt_kblk(mode) != S || mode > GT_KLO_BLK_LAST) return GPTQ_ERR_ARG;
  TcOut vo;
  vo.Cthi = c->A_hi;
  vo.Ctlo = c->A_lo;
  vo.ldt = n;
  c->gemm_role = GR_VB;
  // the tile width is fixed (the widest that fits a block): this product is launched from the
  // quantize call, where simulating its many uneven tiles on the host would leave the GPU idle
  return gemm_tc(c, n, n, n, fop(c->mA_VT, c->VT_hi, c->VT_lo, n, 0, 0), fop(c->mB_Ut, c->Ut_hi, c->Ut_lo, n, 0, 0),
                 1.f, 0, mode, GT_KHI_COL, 1, vo, 1, S >= 256 ? 256 : 128);
}

// The U blocks the factorization leaves out: T and U12 of the nodes on the recursion's left
// edge, smallest first (each U12 needs the complete U of its left part).
gptq_status complete_factor(gptq_ctx* c) {
  const int n = static_cast<int>(c->n);
  std::vector<int> hs;
  for (int h = n; h > kSuperBlock; h = split_left(h, false)) hs.push_back(h);
  for (auto it = hs.rbegin(); it != hs.rend(); ++it) {
    const int h = *it, h1 = split_left(h, false), h2 = h - h1;
    gptq_status s;
    if ((s = t_product(c, 0, h1, h1, h2)) != GPTQ_OK) return s;
    if ((s = u12_product(c, 0, h1, h1, h2)) != GPTQ_OK) return s;
  }
  return GPTQ_OK;
}

// The recursion's node plan, host side only, mirroring chol_inv's splits: every node as
// (offset, width, U complete) in the order chol_inv visits them (right part, the node, left
// part); leaves are the 128-wide nodes.  The test hook below hands it to the host tests.
void factor_plan(int o, int h, bool need_u, std::vector<int>& out) {
  if (h <= LF_NB) {
    out.insert(out.end(), {o, h, 1});
    return;
  }
  if (h <= kSuperBlock) need_u = true;
  const int h1 = split_left(h, need_u), h2 = h - h1;
  factor_plan(o + h1, h2, true, out);
  out.insert(out.end(), {o, h, need_u ? 1 : 0});
  factor_plan(o, h1, need_u, out);
}

// Encode the context's whole-matrix tensor maps (once, at create).
gptq_status encode_maps(gptq_ctx* c) {
  const int64_t n = c->n;
  gptq_status s;
  struct M {
    CUtensorMap* m;
    float* p;
    int64_t rows, cols, ld;
    int box;
  } list[] = {
      {&c->mA_A[0], c->A_hi, n, n, n, GT_BM},        {&c->mA_A[1], c->A_lo, n, n, n, GT_BM},
      {&c->mA_VT[0], c->VT_hi, n, n, n, GT_BM},      {&c->mA_VT[1], c->VT_lo, n, n, n, GT_BM},
      {&c->mA_U[0], c->U_hi, n, n, n, GT_BM},        {&c->mA_U[1], c->U_lo, n, n, n, GT_BM},
      {&c->mA_Err[0], c->Err_hi, c->m_max, kSuperBlock, kSuperBlock, GT_BM},
      {&c->mA_Err[1], c->Err_lo, c->m_max, kSuperBlock, kSuperBlock, GT_BM},
      {&c->mB_U[0], c->U_hi, n, n, n, GT_BOX_N},        {&c->mB_U[1], c->U_lo, n, n, n, GT_BOX_N},
      {&c->mB_VT[0], c->VT_hi, n, n, n, GT_BOX_N},      {&c->mB_VT[1], c->VT_lo, n, n, n, GT_BOX_N},
      {&c->mB_Ut[0], c->Ut_hi, n, n, n, GT_BOX_N},      {&c->mB_Ut[1], c->Ut_lo, n, n, n, GT_BOX_N},
      {&c->mB_Vb[0], c->A_hi, n, n, n, GT_BOX_N},       {&c->mB_Vb[1], c->A_lo, n, n, n, GT_BOX_N},
      {&c->mC_Wq, c->Wq, c->m_max, n, n, 32},
  };
  for (auto& e : list)
    if ((s = make_map(c, e.m, e.p, e.rows, e.cols, e.ld, e.box)) != GPTQ_OK) return s;
  return GPTQ_OK;
}

// Run the factorization recursion: recorded as a CUDA graph on first use (on a private
// stream), then replayed on the context's stream.
gptq_status run_factorization(gptq_ctx* c) {
  if (c->prof) {  // instrumented: every launch on its own, timed, on the context's stream
    cudaStream_t side = c->side_stream;
    c->side_stream = nullptr;
    const gptq_status s = chol_inv(c, 0, static_cast<int>(c->n), false);
    c->side_stream = side;
    return s;
  }
  if (!c->factor_graph) {
    if (!c->capture_stream) CK(cudaStreamCreateWithFlags(&c->capture_stream, cudaStreamNonBlocking));
    if (!c->side_stream) CK(cudaStreamCreateWithFlags(&c->side_stream, cudaStreamNonBlocking));
    if (!c->ev_fork) CK(cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming));
    if (!c->ev_join) CK(cudaEventCreateWithFlags(&c->ev_join, cudaEventDisableTiming));
    cudaStream_t user = c->stream;
    const int64_t l0 = c->launches;
    c->stream = c->capture_stream;
    CK(cudaStreamBeginCapture(c->capture_stream, cudaStreamCaptureModeThreadLocal));
    gptq_status s = chol_inv(c, 0, static_cast<int>(c->n), false);
    if (s == GPTQ_OK) {  // join the second branch (the last block's U^T)
      cudaError_t e1 = cudaEventRecord(c->ev_join, c->side_stream);
      if (e1 == cudaSuccess) e1 = cudaStreamWaitEvent(c->capture_stream, c->ev_join, 0);
      if (e1 != cudaSuccess) s = cuda_fail(e1, "join");
    }
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamEndCapture(c->capture_stream, &g);
    c->stream = user;
    if (s != GPTQ_OK || e != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      c->launches = l0;
      return s != GPTQ_OK ? s : cuda_fail(e, "capture");
    }
    e = cudaGraphInstantiate(&c->factor_graph, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) {
      c->factor_graph = nullptr;
      return cuda_fail(e, "instantiate");
    }
    c->factor_graph_launches = c->launches - l0;
    c->launches = l0;
  }
  CK(cudaGraphLaunch(c->factor_graph, c->stream));
  c->launches += c->factor_graph_launches;
  return GPTQ_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 cached = nullptr;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (cached) return cached;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  cached = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cached;
}

void free_prof(gptq_ctx* c) {
  for (auto& r : c->prof_recs) {
    cudaEventDestroy(r.e0);
    cudaEventDestroy(r.e1);
  }
  c->prof_recs.clear();
}

void free_all(gptq_ctx* c) {
  free_prof(c);
  if (c->factor_graph) cudaGraphExecDestroy(c->factor_graph);
  if (c->capture_stream) cudaStreamDestroy(c->capture_stream);
  if (c->side_stream) cudaStreamDestroy(c->side_stream);
  if (c->ev_fork) cudaEventDestroy(c->ev_fork);
  if (c->ev_join) cudaEventDestroy(c->ev_join);
  c->side_stream = nullptr;
  c->ev_fork = c->ev_join = nullptr;
  c->factor_graph = nullptr;
  c->capture_stream = nullptr;
  float** fs[] = {&c->H,     &c->A_hi,  &c->A_lo, &c->VT_hi,  &c->VT_lo,  &c->U_hi, &c->U_lo,
                  &c->U32,   &c->Ut_hi, &c->Ut_lo, &c->Wq,     &c->Err_hi, &c->Err_lo, &c->keys};
  for (float** p : fs)
    if (*p) {
      cudaFree(*p);
      *p = nullptr;
    }
  if (c->W0h) cudaFree(c->W0h);
  c->W0h = nullptr;
  if (c->dead) cudaFree(c->dead);
  if (c->perm) cudaFree(c->perm);
  if (c->mean) cudaFree(c->mean);
  if (c->status) cudaFree(c->status);
  if (c->status_host) cudaFreeHost(c->status_host);
  c->dead = nullptr;
  c->perm = nullptr;
  c->mean = nullptr;
  c->status = nullptr;
  c->status_host = nullptr;
}

bool valid_qparams(const gptq_qparams& qp, int64_t n) {
  if (!(qp.bits == 2 || qp.bits == 3 || qp.bits == 4 || qp.bits == 8)) return false;
  if (!(qp.sym == 0 || qp.sym == 1)) return false;
  const int64_t g = (qp.group_size == -1) ? n : qp.group_size;
  if (g < 32 || g > n || n % g) return false;
  if (!(g % SW_B == 0 || SW_B % g == 0)) return false;
  return true;
}

}  // namespace

extern "C" {

const char* gptq_status_string(gptq_status s) {
  switch (s) {
    case GPTQ_OK: return "ok";
    case GPTQ_ERR_ARG: return "invalid argument";
    case GPTQ_ERR_STATE: return "call not allowed in the current state";
    case GPTQ_ERR_NOT_PD: return "damped Hessian is not positive definite";
    case GPTQ_ERR_OOM: return "workspace does not fit in device memory";
    case GPTQ_ERR_CUDA: return "CUDA error";
    case GPTQ_ERR_TIMEOUT: return "bounded wait timed out";
    case GPTQ_ERR_UNSUPPORTED: return "unsupported request";
  }
  return "unknown status";
}

size_t gptq_workspace_bytes(int64_t n, int64_t m_max) {
  if (n < 128 || n > kMaxN || n % 128 || m_max < 1 || m_max > kMaxM) return 0;
  const size_t nn = static_cast<size_t>(n) * static_cast<size_t>(n);
  size_t b = 10 * nn * sizeof(float);                                             // H, A, VT, U, Ut (hi/lo), U
  b += static_cast<size_t>(m_max) * static_cast<size_t>(n) * (sizeof(float) + 2);   // Wq, W0h
  b += 2 * static_cast<size_t>(m_max) * kSuperBlock * sizeof(float);              // Err hi/lo
  b += static_cast<size_t>(n) * (sizeof(float) + 1 + sizeof(int32_t)) + sizeof(double) + sizeof(int);
  return b;
}

gptq_status gptq_create(gptq_ctx** out, int64_t n, int64_t m_max, int device, void* stream) {
  if (!out) return GPTQ_ERR_ARG;
  *out = nullptr;
  const size_t need = gptq_workspace_bytes(n, m_max);
  if (need == 0 || device < 0) return GPTQ_ERR_ARG;
  const int64_t env_limit = env_int("GPTQ_MAX_WORKSPACE_BYTES", -1);
  if (env_limit >= 0 && static_cast<int64_t>(need) > env_limit) return GPTQ_ERR_OOM;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  size_t free_b = 0, total_b = 0;
  CK(cudaMemGetInfo(&free_b, &total_b));
  if (need > free_b) return GPTQ_ERR_OOM;
  int major = 0, minor = 0;
  CK(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device));
  CK(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device));
  if (major != 10 || minor != 0) return GPTQ_ERR_UNSUPPORTED;  // built for sm_100a only

  gptq_ctx* c = new gptq_ctx();
  c->device = device;
  c->stream = static_cast<cudaStream_t>(stream);
  c->n = n;
  c->m_max = m_max;
  // tokens summed in tensor memory per round-to-nearest register add of the Hessian: measured on
  // B200 (4096 features, 65536 tokens) 1024 runs 4 % faster than 512 with the diagonal's max
  // relative error 2.3e-6 (512: 1.6e-6; 2048: 5.6e-6, the tensor-core sum truncates)
  c->chunk_tokens = 1024;
  // K stages (32 wide) summed in tensor memory before each round-to-nearest register add, in the
  // factorization's products: 4 (as the updates past a slab), measured on B200: the factor's
  // max-abs relative error against float64 1.1e-6 at n = 3200 (6.6e-7 with 1 stage), the 70B
  // layer's factorization products 20 % faster; GPTQ_FACTOR_CHUNK (1, 2 or 4) for tuning
  c->factor_chunk = static_cast<int>(std::min<int64_t>(4, std::max<int64_t>(1, env_int("GPTQ_FACTOR_CHUNK", 4))));
  c->encode = get_encode();
  cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, device);
  const size_t nn = static_cast<size_t>(n) * n;
  cudaError_t e = cudaSuccess;
  auto alloc = [&](void** p, size_t bytes) {
    if (e == cudaSuccess) e = cudaMalloc(p, bytes);
  };
  alloc(reinterpret_cast<void**>(&c->H), nn * 4);
  for (float** p : {&c->A_hi, &c->A_lo, &c->VT_hi, &c->VT_lo, &c->U_hi, &c->U_lo, &c->U32, &c->Ut_hi, &c->Ut_lo})
    alloc(reinterpret_cast<void**>(p), nn * 4);
  alloc(reinterpret_cast<void**>(&c->Wq), static_cast<size_t>(m_max) * n * 4);
  alloc(reinterpret_cast<void**>(&c->W0h), static_cast<size_t>(m_max) * n * 2);
  alloc(reinterpret_cast<void**>(&c->Err_hi), static_cast<size_t>(m_max) * kSuperBlock * 4);
  alloc(reinterpret_cast<void**>(&c->Err_lo), static_cast<size_t>(m_max) * kSuperBlock * 4);
  alloc(reinterpret_cast<void**>(&c->keys), n * 4);
  alloc(reinterpret_cast<void**>(&c->dead), n);
  alloc(reinterpret_cast<void**>(&c->perm), n * 4);
  alloc(reinterpret_cast<void**>(&c->mean), sizeof(double));
  alloc(reinterpret_cast<void**>(&c->status), sizeof(int));
  if (e == cudaSuccess) e = cudaMallocHost(reinterpret_cast<void**>(&c->status_host), sizeof(int));
  if (e != cudaSuccess || !c->encode) {
    cudaGetLastError();
    free_all(c);
    delete c;
    return (e == cudaErrorMemoryAllocation) ? GPTQ_ERR_OOM : GPTQ_ERR_CUDA;
  }
  if (encode_maps(c) != GPTQ_OK) {
    free_all(c);
    delete c;
    return GPTQ_ERR_CUDA;
  }
  e = cudaFuncSetAttribute(hessian_syrk_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, HP_SMEM);
  if (e == cudaSuccess) e = set_gemm_tc_attributes();
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(leaf_chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, LF_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_hilo_simt_kernel<64, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gs_smem_bytes<64, 64>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_hilo_simt_kernel<32, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gs_smem_bytes<32, 32>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(sweep_slab_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, SS_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(sweep_slab_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, SS_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(sweep_slab_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, SS_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(sweep_block_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, SW_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(sweep_block_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, SW_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(sweep_block_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, SW_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gather_damp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kMaxN * 4));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(init_w_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kMaxN * 2));
  if (e == cudaSuccess) e = cudaMemsetAsync(c->H, 0, nn * 4, c->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->status, 0, sizeof(int), c->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);
  if (e != cudaSuccess) {
    cuda_fail(e, "create");
    free_all(c);
    delete c;
    return GPTQ_ERR_CUDA;
  }
  *out = c;
  return GPTQ_OK;
}

gptq_status gptq_set_hessian_chunk(gptq_ctx* c, int64_t tokens) {
  if (!c || tokens < HS_BK || tokens % HS_BK || tokens > (int64_t(1) << 30)) return GPTQ_ERR_ARG;
  c->chunk_tokens = tokens;
  return GPTQ_OK;
}

gptq_status gptq_hessian_accumulate(gptq_ctx* c, const void* X, int64_t n_tok, int64_t ld_x) {
  if (!c) return GPTQ_ERR_ARG;
  if (c->state != ST_ACCUM) return GPTQ_ERR_STATE;
  if (n_tok < 0 || n_tok >= (int64_t(1) << 31)) return GPTQ_ERR_ARG;
  if (n_tok == 0) return GPTQ_OK;
  if (!X || !aligned16(X) || ld_x < c->n || ld_x % 8) return GPTQ_ERR_ARG;
  DeviceGuard dg(c->device);
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(c->n), static_cast<cuuint64_t>(n_tok)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_x) * 2};
  const cuuint32_t box[2] = {64, HS_BK};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = c->encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return GPTQ_ERR_CUDA;
  const int chunk_iters = static_cast<int>(c->chunk_tokens / HS_BK);
  const double nn1 = static_cast<double>(c->n) * (c->n + 1);
  tag(c, "hessian_syrk_pair", static_cast<double>(n_tok) * nn1, 2.0 * n_tok * c->n + 4.0 * nn1);
  CK(launch(c, hessian_syrk_pair_kernel, dim3(2 * hp_num_pairs(static_cast<int>(c->n))), dim3(HS_THREADS), HP_SMEM, map,
            c->H, static_cast<int>(c->n), static_cast<int>(n_tok), chunk_iters, c->status));
  CKL("hessian");
  c->n_tok += n_tok;
  c->mirrored = 0;
  return GPTQ_OK;
}

static gptq_status ensure_mirrored(gptq_ctx* c) {
  if (c->mirrored) return GPTQ_OK;
  const int n = static_cast<int>(c->n);
  tag(c, "prepare:mirror", 0.0, 4.0 * n * n);
  CK(launch(c, mirror_upper_kernel, dim3(n / MIR_T, n / MIR_T), dim3(32, 8), 0, c->H, n));
  CKL("mirror");
  c->mirrored = 1;
  return GPTQ_OK;
}

gptq_status gptq_get_hessian(gptq_ctx* c, float* H_out, int64_t* n_tok_out) {
  if (!c) return GPTQ_ERR_ARG;
  DeviceGuard dg(c->device);
  gptq_status s;
  if ((s = ensure_mirrored(c)) != GPTQ_OK) return s;
  if (H_out)
    CK(cudaMemcpyAsync(H_out, c->H, static_cast<size_t>(c->n) * c->n * 4, cudaMemcpyDeviceToDevice, c->stream));
  if ((s = wait_stream(c)) != GPTQ_OK) return s;
  if (n_tok_out) *n_tok_out = c->n_tok;
  return GPTQ_OK;
}

gptq_status gptq_set_hessian(gptq_ctx* c, const float* H_in, int64_t n_tok) {
  if (!c || !H_in || n_tok < 0) return GPTQ_ERR_ARG;
  if (c->state != ST_ACCUM) return GPTQ_ERR_STATE;
  DeviceGuard dg(c->device);
  CK(cudaMemcpyAsync(c->H, H_in, static_cast<size_t>(c->n) * c->n * 4, cudaMemcpyDeviceToDevice, c->stream));
  c->n_tok = n_tok;
  c->mirrored = 0;  // only the upper triangle is trusted
  return GPTQ_OK;
}

gptq_status gptq_prepare(gptq_ctx* c, double damp, int desc_act, int32_t* perm_out) {
  if (!c) return GPTQ_ERR_ARG;
  if (!(damp >= 0.0) || damp > 1e6 || !(desc_act == 0 || desc_act == 1)) return GPTQ_ERR_ARG;
  DeviceGuard dg(c->device);
  const int n = static_cast<int>(c->n);
  gptq_status s;
  c->state = ST_ACCUM;
  if ((s = ensure_mirrored(c)) != GPTQ_OK) return s;
  tag(c, "prepare:diag_stats", 0.0, 9.0 * n);
  CK(launch(c, diag_stats_kernel, dim3(1), dim3(1024), 0, c->H, n, c->keys, c->dead, c->mean));
  CKL("diag_stats");
  tag(c, "prepare:perm", 0.0, 8.0 * n);
  if (desc_act)
    CK(launch(c, rank_perm_kernel, dim3((n + 7) / 8), dim3(256), 0, c->keys, n, c->perm));
  else
    CK(launch(c, identity_perm_kernel, dim3((n + 255) / 256), dim3(256), 0, n, c->perm));
  CKL("perm");
  tag(c, "prepare:gather_damp", 0.0, 12.0 * n * n);
  CK(launch(c, gather_damp_kernel, dim3(n), dim3(GD_THREADS), static_cast<size_t>(n) * 4, c->H, n, c->perm, c->keys, c->mean, damp,
                                                                        c->A_hi, c->A_lo));
  CKL("gather");
  const size_t nn = static_cast<size_t>(n) * n;
  for (float* p : {c->U_hi, c->U_lo, c->U32, c->Ut_hi, c->Ut_lo}) CK(cudaMemsetAsync(p, 0, nn * 4, c->stream));
  if ((s = run_factorization(c)) != GPTQ_OK) return s;
  c->u_complete = n <= kSuperBlock;
  c->vs_width = 0;
  if (perm_out) CK(cudaMemcpyAsync(perm_out, c->perm, n * 4, cudaMemcpyDeviceToDevice, c->stream));
  int flags = 0;
  if ((s = read_status(c, &flags)) != GPTQ_OK) return s;
  if (flags) return status_from_flags(flags);
  c->state = ST_PREPARED;
  return GPTQ_OK;
}

gptq_status gptq_get_factor(gptq_ctx* c, float* U_out) {
  if (!c || !U_out) return GPTQ_ERR_ARG;
  if (c->state != ST_PREPARED) return GPTQ_ERR_STATE;
  DeviceGuard dg(c->device);
  if (!c->u_complete) {
    gptq_status s;
    if ((s = complete_factor(c)) != GPTQ_OK) return s;
    c->u_complete = true;
  }
  const size_t nn = static_cast<size_t>(c->n) * c->n;
  CK(cudaMemcpyAsync(U_out, c->U32, nn * 4, cudaMemcpyDeviceToDevice, c->stream));
  return GPTQ_OK;
}

gptq_status gptq_get_dead_columns(gptq_ctx* c, uint8_t* dead_out) {
  if (!c || !dead_out) return GPTQ_ERR_ARG;
  if (c->state != ST_PREPARED) return GPTQ_ERR_STATE;
  DeviceGuard dg(c->device);
  CK(cudaMemcpyAsync(dead_out, c->dead, static_cast<size_t>(c->n), cudaMemcpyDeviceToDevice, c->stream));
  return GPTQ_OK;
}

gptq_status gptq_set_profiling(gptq_ctx* c, int on) {
  if (!c || (on != 0 && on != 1)) return GPTQ_ERR_ARG;
  c->prof = on != 0;
  return GPTQ_OK;
}

gptq_status gptq_get_profile(gptq_ctx* c, gptq_kernel_stat* out, int capacity, int* count) {
  if (!c || capacity < 0 || (capacity > 0 && !out)) return GPTQ_ERR_ARG;
  DeviceGuard dg(c->device);
  gptq_status st = wait_stream(c);
  if (st != GPTQ_OK) return st;
  std::vector<gptq_kernel_stat> agg;
  bool bad = c->prof_error;
  for (const auto& r : c->prof_recs) {
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, r.e0, r.e1) != cudaSuccess) {
      bad = true;
      cudaGetLastError();
      continue;
    }
    gptq_kernel_stat* e = nullptr;
    for (auto& a : agg)
      if (std::strncmp(a.name, r.tag, sizeof(a.name)) == 0) e = &a;
    if (!e) {
      gptq_kernel_stat z{};
      std::strncpy(z.name, r.tag, sizeof(z.name) - 1);
      agg.push_back(z);
      e = &agg.back();
    }
    e->launches += 1;
    e->ms += ms;
    e->flops += r.flops;
    e->bytes += r.bytes;
  }
  free_prof(c);
  c->prof_error = false;
  for (int i = 0; i < capacity && i < static_cast<int>(agg.size()); ++i) out[i] = agg[i];
  if (count) *count = static_cast<int>(agg.size());
  return bad ? GPTQ_ERR_CUDA : GPTQ_OK;
}

gptq_status gptq_test_bounded_wait(gptq_ctx* c, uint64_t limit_ns) {
  if (!c || limit_ns < 1 || limit_ns > 10000000000ull) return GPTQ_ERR_ARG;
  DeviceGuard dg(c->device);
  tag(c, "test:bounded_wait", 0.0, 0.0);
  CK(launch(c, bounded_wait_probe_kernel, dim3(1), dim3(32), 0, limit_ns, c->status));
  CKL("bounded_wait_probe");
  return GPTQ_OK;
}

gptq_status gptq_quantize_layer(gptq_ctx* c, const void* W, int64_t m, gptq_qparams qp, uint32_t* codes,
                                float* scales, float* zeros, int32_t* g_idx, float* W_hat) {
  if (!c) return GPTQ_ERR_ARG;
  if (c->state != ST_PREPARED) return GPTQ_ERR_STATE;
  if (!W || !codes || !scales || !zeros || m < 1 || m > c->m_max || !valid_qparams(qp, c->n)) return GPTQ_ERR_ARG;
  if (!aligned16(codes) || (W_hat && !aligned16(W_hat))) return GPTQ_ERR_ARG;
  DeviceGuard dg(c->device);
  const int n = static_cast<int>(c->n);
  const int mi = static_cast<int>(m);
  const int g = (qp.group_size == -1) ? n : qp.group_size;
  tag(c, "quantize:init_w", 0.0, 8.0 * static_cast<double>(m) * n);
  CK(launch(c, init_w_kernel, dim3(mi), dim3(256), static_cast<size_t>(n) * 2, static_cast<const __half*>(W), n, c->perm,
            c->dead, c->Wq, c->W0h));
  CKL("init_w");
  SweepArgs a;
  a.Wq = c->Wq;
  a.U = c->U32;
  a.U_lo = nullptr;
  a.W0 = c->W0h;
  a.Err = c->Err_hi;
  a.Err_lo = c->Err_lo;
  a.codes = codes;
  a.scales = scales;
  a.zeros = zeros;
  a.W_hat = W_hat;
  a.perm = c->perm;
  a.m = mi;
  a.n = n;
  a.bits = qp.bits;
  a.sym = qp.sym;
  a.g = g;
  a.G = n / g;
  a.ld_err = kSuperBlock;
  a.err_col0 = 0;
  const int grid = (mi + SW_ROWS - 1) / SW_ROWS;
  // Two-level lazy update.  Inside a super-block of columns (the slab) the slab kernel carries
  // every column's error forward itself; the columns beyond the slab receive the slab's
  // contribution in one tensor-core product (K = slab width).  The sweep's errors satisfy
  // E U = W0 - Q column by column (W0 the original weights, Q their dequantized values), so the
  // errors of all columns before a slab reach it as -E U[., slab] = D V[., slab] U[slab, slab]
  // with D = W0 - Q.  That product is taken in this form, D Vs with Vs = V blockdiag(U_SS)
  // (computed once per prepared factor and slab width): the factorization then needs U only
  // inside the aligned slab blocks.  The slab's columns are exact once every earlier slab is
  // in, not before, so every group must start and end inside one slab (or be the whole row).
  // Group widths that cannot (wider than kSuperBlock, or not dividing a power-of-two slab)
  // take the form -E U[slab, rest] instead, on the completed U, which also lets groups reach
  // past a slab.  Slab width: slab_default(n), or GPTQ_SLAB_WIDTH (a multiple of 128 up to
  // kSuperBlock) for tuning.
  const int slab = static_cast<int>(
      std::min<int64_t>(kSuperBlock, std::max<int64_t>(SW_B, env_int("GPTQ_SLAB_WIDTH", slab_default(n)) / SW_B * SW_B)));
  int sd = SW_B;  // the widest power-of-two multiple of 128 up to the slab width
  while (sd * 2 <= slab) sd *= 2;
  const bool g_pow2 = g >= SW_B && g <= kSuperBlock && (g & (g - 1)) == 0;
  if (g_pow2 && g > sd) sd = g;
  const bool d_form = g < SW_B || g == n || g_pow2;
  int sb;
  if (d_form) {
    sb = sd;
    if (c->vs_width != sb) {
      gptq_status st;
      if ((st = vs_product(c, sb)) != GPTQ_OK) return st;
      c->vs_width = sb;
    }
  } else {
    sb = ((g <= slab && slab % g == 0) || g % slab == 0) ? slab : SW_B;
    if (!c->u_complete) {
      gptq_status st;
      if ((st = complete_factor(c)) != GPTQ_OK) return st;
      c->u_complete = true;
    }
  }
  a.d_form = d_form ? 1 : 0;
  for (int s0 = 0; s0 < n; s0 += sb) {
    const int s1 = std::min(n, s0 + sb);
    const double S = static_cast<double>(s1 - s0);
    // algorithmic bytes: the slab in, its original weights (d form), its D or errors out
    // (hi/lo) when a product follows, codes, scales/zeros of its groups, the upper half of its
    // U block, the dequantized weights when asked for
    tag(c, "sweep_slab", 0.0,
        4.0 * mi * S + (s1 < n ? (d_form ? 10.0 : 8.0) * mi * S : 0.0) + mi * S * qp.bits / 8.0 +
            8.0 * mi * std::max(1.0, S / g) + 2.0 * S * S + (W_hat ? 4.0 * mi * S : 0.0));
    const size_t smem = static_cast<size_t>(ss_smem_bytes(s1 - s0));
    if (g >= SW_B)
      CK(launch(c, sweep_slab_kernel<0>, dim3(grid), dim3(SS_THREADS), smem, a, s0, s1));
    else if (g == 64)
      CK(launch(c, sweep_slab_kernel<64>, dim3(grid), dim3(SS_THREADS), smem, a, s0, s1));
    else
      CK(launch(c, sweep_slab_kernel<32>, dim3(grid), dim3(SS_THREADS), smem, a, s0, s1));
    CKL("sweep_slab");
    if (s1 < n) {
      // W[:, s1:] += D_slab Vs[s0:s1, s1:], or -= E_slab U[s0:s1, s1:]   (K = s1 - s0; 128-wide
      // TMEM chunks)
      TcOut w;
      w.C = c->Wq + s1;
      w.ldc = n;
      w.c_map = &c->mC_Wq;
      w.c_col0 = s1;
      c->gemm_role = GR_FAR;
      const TcOperand B = d_form ? TcOperand{&c->mB_Vb[0], &c->mB_Vb[1], s1, s0, nullptr, nullptr, 0}
                                 : TcOperand{&c->mB_Ut[0], &c->mB_Ut[1], s1, s0, nullptr, nullptr, 0};
      gptq_status st = gemm_tc(c, mi, n - s1, s1 - s0, TcOperand{&c->mA_Err[0], &c->mA_Err[1], 0, 0, nullptr, nullptr, 0},
                               B, d_form ? 1.f : -1.f, 1, GT_KLO_NONE, GT_KHI_NONE, 0, w, SW_B / GT_BK);
      if (st != GPTQ_OK) return st;
    }
  }
  if (g_idx) {
    tag(c, "quantize:g_idx", 0.0, 8.0 * n);
    CK(launch(c, g_idx_kernel, dim3((n + 255) / 256), dim3(256), 0, c->perm, n, g, g_idx));
    CKL("g_idx");
  }
  return GPTQ_OK;
}

gptq_status gptq_synchronize(gptq_ctx* c) {
  if (!c) return GPTQ_ERR_ARG;
  DeviceGuard dg(c->device);
  int flags = 0;
  gptq_status s = read_status(c, &flags);
  if (s != GPTQ_OK) return s;
  return status_from_flags(flags);
}

gptq_status gptq_reset(gptq_ctx* c) {
  if (!c) return GPTQ_ERR_ARG;
  DeviceGuard dg(c->device);
  CK(cudaMemsetAsync(c->H, 0, static_cast<size_t>(c->n) * c->n * 4, c->stream));
  c->n_tok = 0;
  c->state = ST_ACCUM;
  c->mirrored = 0;
  return GPTQ_OK;
}

int64_t gptq_launch_count(const gptq_ctx* c) { return c ? c->launches : -1; }

gptq_status gptq_test_gemm_tf32x3(int M, int N, int K, const float* A_hi, const float* A_lo, int lda, const float* B_hi,
                                  const float* B_lo, int ldb, float alpha, int beta, int k_lo_mode, int k_hi_mode,
                                  int upper_only, float* C, int ldc, float* C_hi, float* C_lo, int ldh, float* Ct_hi,
                                  float* Ct_lo, int ldt, int chunk_stages, int tile_n, int c_reduce, int device,
                                  void* cuda_stream) {
  if (chunk_stages < 1) return GPTQ_ERR_ARG;
  if (c_reduce && (!C || beta != 1)) return GPTQ_ERR_ARG;
  if (tile_n != 0 && tile_n != 64 && tile_n != 128 && tile_n != 256 && tile_n != 512) return GPTQ_ERR_ARG;
  if (!A_hi || !A_lo || !B_hi || !B_lo || M < 1 || N < 1 || K < GT_BK) return GPTQ_ERR_ARG;
  if (k_lo_mode < 0 || k_lo_mode > GT_KLO_BLK_LAST || k_hi_mode < 0 || k_hi_mode > 1 || (beta != 0 && beta != 1)) return GPTQ_ERR_ARG;
  if ((C_hi == nullptr) != (C_lo == nullptr) || (Ct_hi == nullptr) != (Ct_lo == nullptr)) return GPTQ_ERR_ARG;
  if ((C && (!aligned16(C) || ldc % 4)) || (C_hi && (!aligned16(C_hi) || !aligned16(C_lo) || ldh % 4)))
    return GPTQ_ERR_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  gptq_ctx t;
  t.device = device;
  t.stream = static_cast<cudaStream_t>(cuda_stream);
  t.encode = get_encode();
  if (!t.encode) return GPTQ_ERR_CUDA;
  cudaDeviceGetAttribute(&t.num_sms, cudaDevAttrMultiProcessorCount, device);
  CK(set_gemm_tc_attributes());
  CK(cudaMallocAsync(reinterpret_cast<void**>(&t.status), sizeof(int), t.stream));
  CK(cudaMemsetAsync(t.status, 0, sizeof(int), t.stream));
  TcOut o;
  o.C = C;
  o.ldc = ldc;
  o.Chi = C_hi;
  o.Clo = C_lo;
  o.ldh = ldh;
  o.Cthi = Ct_hi;
  o.Ctlo = Ct_lo;
  o.ldt = ldt;
  CUtensorMap ma[2], mb[2], mc;
  gptq_status s = GPTQ_OK;
  t.gemm_role = GR_TEST;
  if (c_reduce) {
    s = make_map(&t, &mc, C, M, N, ldc, 32);
    o.c_map = &mc;
  }
  if (s == GPTQ_OK) s = make_map(&t, &ma[0], A_hi, M, K, lda, GT_BM);
  if (s == GPTQ_OK) s = make_map(&t, &ma[1], A_lo, M, K, lda, GT_BM);
  if (s == GPTQ_OK) s = make_map(&t, &mb[0], B_hi, N, K, ldb, GT_BOX_N);
  if (s == GPTQ_OK) s = make_map(&t, &mb[1], B_lo, N, K, ldb, GT_BOX_N);
  if (s == GPTQ_OK)
    s = gemm_tc(&t, M, N, K, TcOperand{&ma[0], &ma[1], 0, 0, nullptr, nullptr, 0},
                TcOperand{&mb[0], &mb[1], 0, 0, nullptr, nullptr, 0}, alpha, beta, k_lo_mode, k_hi_mode, upper_only, o,
                chunk_stages, tile_n);
  int flags = 0;
  cudaMemcpyAsync(&flags, t.status, sizeof(int), cudaMemcpyDeviceToHost, t.stream);
  cudaError_t e = cudaStreamSynchronize(t.stream);
  cudaFreeAsync(t.status, t.stream);
  t.status = nullptr;
  if (s != GPTQ_OK) return s;
  if (e != cudaSuccess) return cuda_fail(e, "test gemm");
  return status_from_flags(flags);
}

gptq_status gptq_test_div_rn(uint64_t seed, int64_t count, uint64_t* mismatches, float* example, int device,
                             void* cuda_stream) {
  if (count < 0 || !mismatches) return GPTQ_ERR_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  unsigned long long* d_count = nullptr;
  CK(cudaMallocAsync(reinterpret_cast<void**>(&d_count), 16, st));
  float* d_ex = reinterpret_cast<float*>(d_count + 1);
  cudaMemsetAsync(d_count, 0, 16, st);
  div_rn_check_kernel<<<sms * 8, 256, 0, st>>>(seed, static_cast<long long>(count), d_count, d_ex);
  cudaError_t e = cudaGetLastError();
  unsigned long long h[2] = {0ull, 0ull};
  cudaMemcpyAsync(h, d_count, 16, cudaMemcpyDeviceToHost, st);
  cudaError_t e2 = cudaStreamSynchronize(st);
  cudaFreeAsync(d_count, st);
  cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "test div_rn");
  if (e2 != cudaSuccess) return cuda_fail(e2, "test div_rn");
  *mismatches = h[0];
  if (example) std::memcpy(example, &h[1], 2 * sizeof(float));
  return GPTQ_OK;
}

int gptq_test_pick_tile_n(int M, int N, int K, int k_lo_mode, int k_hi_mode, int upper_only, int sms) {
  if (M < 1 || N < 1 || K < 1 || sms < 1) return -1;
  return pick_bn(M, N, K, k_lo_mode, k_hi_mode, upper_only, sms);
}

int gptq_test_tile_schedule(int M, int N, int K, int k_lo_mode, int k_hi_mode, int upper_only, int tile_n,
                                    int ctas) {
  if (M < 1 || N < 1 || K < 1 || ctas < 1 || (tile_n != 64 && tile_n != 128 && tile_n != 256)) return -1;
  const int ntiles = gt_num_tiles(M, N, upper_only, tile_n);
  const int mtn = (M + GT_BM - 1) / GT_BM, ntn = (N + tile_n - 1) / tile_n;
  std::vector<int> seen(ntiles, 0), cell(static_cast<size_t>(mtn) * ntn, 0);
  for (int b = 0; b < ctas; ++b)
    for (int r = 0; r * ctas < ntiles; ++r) {
      const int t = gt_sched(r, b, ctas);
      if (t < 0) return 1;
      if (t >= ntiles) continue;
      ++seen[t];
    }
  for (int t = 0; t < ntiles; ++t) {
    if (seen[t] != 1) return 2;  // every tile exactly once
    int m0, n0, kb, ni;
    gt_tile_at(M, N, K, k_lo_mode, k_hi_mode, upper_only, tile_n, t, m0, n0, kb, ni);
    if (m0 < 0 || m0 >= mtn * GT_BM || n0 < 0 || n0 >= ntn * tile_n || m0 % GT_BM || n0 % tile_n) return 3;
    if (kb < 0 || kb % GT_BK || ni < 0 || (ni > 0 && kb + ni * GT_BK > ((K + GT_BK - 1) / GT_BK) * GT_BK)) return 4;
    if (upper_only && m0 >= n0 + tile_n) return 5;  // wholly below the diagonal
    if (++cell[static_cast<size_t>(m0 / GT_BM) * ntn + n0 / tile_n] != 1) return 6;  // distinct tiles
  }
  if (!upper_only) {
    for (int v : cell)
      if (v != 1) return 7;  // and all of them
  } else {
    for (int mt = 0; mt < mtn; ++mt)
      for (int nt = 0; nt < ntn; ++nt)
        if ((mt * GT_BM < (nt + 1) * tile_n) != (cell[static_cast<size_t>(mt) * ntn + nt] == 1)) return 8;
  }
  return 0;
}

int gptq_test_factor_plan(int64_t n, int32_t* nodes_out, int capacity, int32_t* spine_out, int spine_capacity,
                          int* spine_count) {
  if (n < LF_NB || n > kMaxN || n % LF_NB || !nodes_out || capacity < 0 || !spine_count) return -1;
  std::vector<int> v;
  factor_plan(0, static_cast<int>(n), false, v);
  const int count = static_cast<int>(v.size() / 3);
  for (int i = 0; i < count && i < capacity; ++i)
    for (int k = 0; k < 3; ++k) nodes_out[3 * i + k] = v[3 * i + k];
  // the nodes gptq_get_factor completes, in its order (complete_factor)
  std::vector<int> hs;
  for (int h = static_cast<int>(n); h > kSuperBlock; h = split_left(h, false)) hs.push_back(h);
  *spine_count = static_cast<int>(hs.size());
  for (int i = 0; i < static_cast<int>(hs.size()) && spine_out && i < spine_capacity; ++i)
    spine_out[i] = hs[hs.size() - 1 - i];
  return count;
}

gptq_status gptq_destroy(gptq_ctx* c) {
  if (!c) return GPTQ_OK;
  gptq_status s;
  {
    DeviceGuard dg(c->device);
    s = wait_stream(c);
    free_all(c);
  }
  delete c;
  return s;
}

}  // extern "C"

// ==========================================================================================
// Allocation-free quantize: gptq_quantize_layer_noalloc
//
// Some callers must not allocate device memory on their own: an engine or plugin host that
// owns a fixed device-memory budget and hands out every byte itself, or code that runs where
// cudaMalloc/cudaFree would stall other work (both synchronize the device) or are not
// permitted at all.  For them this entry point runs the same sweep kernels as
// gptq_quantize_layer, but its scratch (the fp32 working copy of W and the per-block error
// tile) lives in the fixed array below, which the library's module holds on every GPU that
// loads it, until the process exits.
// ==========================================================================================
namespace {
constexpr int64_t kNoAllocMaxWeights = int64_t(1) << 20;  // m * n  (4 MiB of fp32 working weights)
constexpr int64_t kNoAllocMaxRows = 4096;                  // m      (2 MiB of block errors)
constexpr int kNoAllocMaxDevices = 64;
}  // namespace

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocMaxWeights + kNoAllocMaxRows * SW_B];
static __device__ __align__(256) uint8_t g_noalloc_no_dead[kMaxN];  // all zero: no dead columns

namespace {
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kNoAllocMaxDevices] = {};
uint8_t* g_noalloc_nodead_ptr[kNoAllocMaxDevices] = {};

// Once per device, with that device current: resolve the device addresses of the static
// arrays (host code must not use the symbols themselves as addresses) and raise the
// dynamic shared-memory limits of the kernels this path launches.  Allocates nothing.
gptq_status noalloc_setup(int device, float** scratch, uint8_t** nodead) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[device]) {
    void* p = nullptr;
    void* q = nullptr;
    CK(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    CK(cudaGetSymbolAddress(&q, g_noalloc_no_dead));
    CK(cudaFuncSetAttribute(sweep_block_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, SW_SMEM));
    CK(cudaFuncSetAttribute(sweep_block_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, SW_SMEM));
    CK(cudaFuncSetAttribute(sweep_block_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, SW_SMEM));
    CK(cudaFuncSetAttribute(init_w_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            static_cast<int>(kMaxN * 2)));
    g_noalloc_nodead_ptr[device] = static_cast<uint8_t*>(q);
    g_noalloc_ptr[device] = static_cast<float*>(p);
  }
  *scratch = g_noalloc_ptr[device];
  *nodead = g_noalloc_nodead_ptr[device];
  return GPTQ_OK;
}
}  // namespace

extern "C" gptq_status gptq_quantize_layer_noalloc(const void* W, int64_t m, int64_t n, const float* U,
                                                   const int32_t* perm, const uint8_t* dead, gptq_qparams qp,
                                                   uint32_t* codes, float* scales, float* zeros, int32_t* g_idx,
                                                   float* W_hat, int device, void* cuda_stream) {
  if (!W || !U || !perm || !codes || !scales || !zeros) return GPTQ_ERR_ARG;
  if (n < 128 || n > kMaxN || n % 128 || m < 1) return GPTQ_ERR_ARG;
  if (m > kNoAllocMaxRows || m * n > kNoAllocMaxWeights) return GPTQ_ERR_ARG;  // beyond the fixed scratch
  if (!valid_qparams(qp, n)) return GPTQ_ERR_ARG;
  if (!aligned16(U) || !aligned16(codes) || (W_hat && !aligned16(W_hat))) return GPTQ_ERR_ARG;
  if (device < 0 || device >= kNoAllocMaxDevices) return GPTQ_ERR_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  float* scratch = nullptr;
  uint8_t* nodead = nullptr;
  gptq_status s = noalloc_setup(device, &scratch, &nodead);
  if (s != GPTQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const int ni = static_cast<int>(n), mi = static_cast<int>(m);
  const int g = (qp.group_size == -1) ? ni : qp.group_size;
  float* Wq = scratch;                       // [m x n]
  float* Err = scratch + kNoAllocMaxWeights; // [m x 128]
  init_w_kernel<<<mi, 256, static_cast<size_t>(ni) * 2, st>>>(static_cast<const __half*>(W), ni, perm,
                                                             dead ? dead : nodead, Wq, nullptr);
  CKL("noalloc init_w");
  SweepArgs a;
  a.Wq = Wq;
  a.U = U;
  a.U_lo = nullptr;
  a.W0 = nullptr;
  a.d_form = 0;
  a.Err = Err;
  a.Err_lo = nullptr;
  a.ld_err = SW_B;
  a.err_col0 = 0;
  a.codes = codes;
  a.scales = scales;
  a.zeros = zeros;
  a.W_hat = W_hat;
  a.perm = perm;
  a.m = mi;
  a.n = ni;
  a.bits = qp.bits;
  a.sym = qp.sym;
  a.g = g;
  a.G = ni / g;
  const int grid = (mi + SW_ROWS - 1) / SW_ROWS;
  for (int i1 = 0; i1 < ni; i1 += SW_B) {
    if (g >= SW_B)
      sweep_block_kernel<0><<<grid, SW_THREADS, SW_SMEM, st>>>(a, i1);
    else if (g == 64)
      sweep_block_kernel<64><<<grid, SW_THREADS, SW_SMEM, st>>>(a, i1);
    else
      sweep_block_kernel<32><<<grid, SW_THREADS, SW_SMEM, st>>>(a, i1);
    CKL("noalloc sweep");
    const int i2 = i1 + SW_B;
    if (i2 < ni) {
      dim3 gg((ni - i2 + SG_BN - 1) / SG_BN, (mi + SG_BM - 1) / SG_BM);
      sgemm_kernel<false><<<gg, SG_THREADS, 0, st>>>(mi, ni - i2, SW_B, -1.f, Err, SW_B,
                                                     U + static_cast<size_t>(i1) * ni + i2, ni, 1.f, Wq + i2, ni, 0);
      CKL("noalloc trailing");
    }
  }
  if (g_idx) {
    g_idx_kernel<<<(ni + 255) / 256, 256, 0, st>>>(perm, ni, g, g_idx);
    CKL("noalloc g_idx");
  }
  return GPTQ_OK;
}

// ==========================================================================================
// The consumer of the packed result: gptq_dequant_matmul (dequant_gemm.cuh)
// ==========================================================================================
namespace {

constexpr int kDqPlanSms = 148;  // the split-K plan is fixed so that the workspace size is a pure function
constexpr int kMaxDevicesAttr = 64;

struct DqPlan {
  int tn = 0, tiles_m = 0, tiles_t = 0, k_tiles = 0, k_per = 0, splits = 0;
  size_t xp_off = 0, part_off = 0, total = 0;
};

bool dq_plan(int64_t T, int64_t m, int64_t n, int act_order, DqPlan* p) {
  if (T < 1 || T > (int64_t(1) << 24) || m < 1 || m > (int64_t(1) << 24) || n < 128 || n > (int64_t(1) << 20) ||
      n % 128)
    return false;
  p->tn = T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : T <= 128 ? 128 : 256;
  p->tiles_m = static_cast<int>((m + DQ_BM - 1) / DQ_BM);
  p->tiles_t = static_cast<int>((T + p->tn - 1) / p->tn);
  p->k_tiles = static_cast<int>(n / DQ_BK);
  const int64_t base = static_cast<int64_t>(p->tiles_m) * p->tiles_t;
  // fill every SM (two CTAs each when the tile is decode-sized, see dq_shape) with K splits
  const int64_t target = kDqPlanSms * (p->tn <= 32 ? 2 : 1);
  int splits = base >= target ? 1 : static_cast<int>(std::min<int64_t>(p->k_tiles, target / base));
  splits = std::max(1, splits);
  p->k_per = (p->k_tiles + splits - 1) / splits;
  p->splits = (p->k_tiles + p->k_per - 1) / p->k_per;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  size_t off = 256;  // status word
  p->xp_off = off;
  if (act_order) off += up(static_cast<size_t>(T) * n * 2);
  p->part_off = off;
  if (p->splits > 1) off += up(static_cast<size_t>(p->splits) * T * m * 4);
  p->total = off;
  return true;
}

// Raise a kernel's dynamic shared-memory limit once per device (later calls, which may be
// recorded into a graph, then make no attribute call).
std::mutex g_attr_mu;
int g_attr_smem[kMaxDevicesAttr][16] = {};

template <typename K>
cudaError_t ensure_smem_attr(int device, int slot, K kernel, int smem) {
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (device < 0 || device >= kMaxDevicesAttr) return cudaErrorInvalidDevice;
  if (g_attr_smem[device][slot] >= smem) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) g_attr_smem[device][slot] = smem;
  return e;
}

}  // namespace

extern "C" size_t gptq_dequant_matmul_workspace_bytes(int64_t T, int64_t m, int64_t n, int act_order) {
  DqPlan p;
  if (!dq_plan(T, m, n, act_order ? 1 : 0, &p)) return 0;
  return p.total;
}

extern "C" gptq_status gptq_dequant_matmul(const void* X, int64_t T, const uint32_t* codes, const float* scales,
                                           const float* zeros, const int32_t* perm, int64_t m, int64_t n,
                                           gptq_qparams qp, float* Y, void* workspace, size_t workspace_bytes,
                                           int device, void* cuda_stream) {
  if (!X || !codes || !scales || !zeros || !Y || !workspace) return GPTQ_ERR_ARG;
  DqPlan pl;
  if (!dq_plan(T, m, n, perm ? 1 : 0, &pl)) return GPTQ_ERR_ARG;
  if (!valid_qparams(qp, n)) return GPTQ_ERR_ARG;
  if (!aligned16(X) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GPTQ_ERR_ARG;
  if (workspace_bytes < pl.total) return GPTQ_ERR_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode();
  if (!encode) return GPTQ_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  const int ni = static_cast<int>(n), mi = static_cast<int>(m), Ti = static_cast<int>(T);
  const int bits = qp.bits;
  CK(cudaMemsetAsync(status, 0, sizeof(int), st));
  // the activations in sweep order (act-order), else as given
  const __half* Xs = static_cast<const __half*>(X);
  if (perm) {
    __half* Xp = reinterpret_cast<__half*>(ws + pl.xp_off);
    CK(ensure_smem_attr(device, 4, permute_x_kernel, ni * 2));
    permute_x_kernel<<<Ti, 256, static_cast<size_t>(ni) * 2, st>>>(Xs, ni, perm, Xp);
    CKL("permute_x");
    Xs = Xp;
  }
  CUtensorMap cmap, xmap;
  {
    const int64_t words = n * bits / 32;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(words), static_cast<cuuint64_t>(m)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(words) * 4};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(4 * bits), static_cast<cuuint32_t>(DQ_BM)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTQ_ERR_CUDA;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(n) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(pl.tn)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(Xs), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTQ_ERR_CUDA;
  }
  DqArgs a;
  a.T = Ti;
  a.m = mi;
  a.n = ni;
  a.tn = pl.tn;
  a.g = (qp.group_size == -1) ? ni : qp.group_size;
  a.G = ni / a.g;
  a.k_tiles = pl.k_tiles;
  a.k_tiles_per_split = pl.k_per;
  a.out = pl.splits > 1 ? reinterpret_cast<float*>(ws + pl.part_off) : Y;
  a.scales = scales;
  a.zeros = zeros;
  a.status = status;
  // decode-sized tiles: two CTAs per SM with two dequantized tiles each, or (GPTQ_DQ_DECODE=4)
  // one CTA with four
  const DqShape sh = dq_shape(pl.tn, bits, static_cast<int>(env_int("GPTQ_DQ_DECODE", 2)));
  const int smem = dq_smem_bytes(pl.tn, bits, sh.minb, sh.na);
  const dim3 grid(pl.tiles_m, pl.tiles_t, pl.splits);
#define GPTQ_DQ_LAUNCH(B, M, N, SLOT)                                                      \
  do {                                                                                    \
    CK(ensure_smem_attr(device, SLOT, dequant_gemm_kernel<B, M, N>, smem));               \
    dequant_gemm_kernel<B, M, N><<<grid, DQ_THREADS, smem, st>>>(cmap, xmap, a);          \
  } while (0)
  const int shape = sh.minb == 2 ? 0 : (sh.na == 4 ? 1 : 2);
  switch (bits * 4 + shape) {
    case 2 * 4 + 0: GPTQ_DQ_LAUNCH(2, 2, 2, 0); break;
    case 2 * 4 + 1: GPTQ_DQ_LAUNCH(2, 1, 4, 1); break;
    case 2 * 4 + 2: GPTQ_DQ_LAUNCH(2, 1, 2, 2); break;
    case 3 * 4 + 0: GPTQ_DQ_LAUNCH(3, 2, 2, 3); break;
    case 3 * 4 + 1: GPTQ_DQ_LAUNCH(3, 1, 4, 5); break;
    case 3 * 4 + 2: GPTQ_DQ_LAUNCH(3, 1, 2, 6); break;
    case 4 * 4 + 0: GPTQ_DQ_LAUNCH(4, 2, 2, 7); break;
    case 4 * 4 + 1: GPTQ_DQ_LAUNCH(4, 1, 4, 8); break;
    case 4 * 4 + 2: GPTQ_DQ_LAUNCH(4, 1, 2, 9); break;
    case 8 * 4 + 1: GPTQ_DQ_LAUNCH(8, 1, 4, 10); break;
    default: GPTQ_DQ_LAUNCH(8, 1, 2, 11); break;
  }
#undef GPTQ_DQ_LAUNCH
  CKL("dequant_gemm");
  if (pl.splits > 1) {
    splitk_reduce_kernel<<<592, 256, 0, st>>>(a.out, pl.splits, static_cast<size_t>(T) * m, Y);
    CKL("splitk_reduce");
  }
  return GPTQ_OK;
}

extern "C" gptq_status gptq_dequant_matmul_check(void* workspace, int device, void* cuda_stream) {
  if (!workspace) return GPTQ_ERR_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  int flags = 0;
  CK(cudaMemcpyAsync(&flags, workspace, sizeof(int), cudaMemcpyDeviceToHost, st));
  gptq_ctx tmp;
  tmp.stream = st;
  const gptq_status s = wait_stream(&tmp);
  if (s != GPTQ_OK) return s;
  return status_from_flags(flags);
}

// ==========================================================================================
// Many layers in one call: gptq_quantize_layers (two contexts per width, two streams)
// ==========================================================================================
namespace {

struct LayerGroup {
  const gptq_layer_job* first;
  std::vector<int> jobs;
};

bool same_input(const gptq_layer_job& a, const gptq_layer_job& b) {
  return a.X_bf16 == b.X_bf16 && a.n_tok == b.n_tok && a.ld_x == b.ld_x && a.n == b.n;
}

// The slot's context for width n (created on first use with the batch's largest m for that n).
struct Slot {
  cudaStream_t stream = nullptr;
  std::vector<std::pair<int64_t, gptq_ctx*>> ctx;
  gptq_ctx* get(int64_t n) {
    for (auto& e : ctx)
      if (e.first == n) return e.second;
    return nullptr;
  }
};

gptq_status run_group(gptq_ctx* c, const gptq_layer_job* jobs, const LayerGroup& g) {
  // one factorization per distinct (damp, desc_act), each followed by its jobs' quantization
  std::vector<int> done(g.jobs.size(), 0);
  for (size_t i = 0; i < g.jobs.size(); ++i) {
    if (done[i]) continue;
    const gptq_layer_job& a = jobs[g.jobs[i]];
    gptq_status s = gptq_prepare(c, a.damp, a.desc_act, nullptr);
    if (s != GPTQ_OK) return s;
    for (size_t j = i; j < g.jobs.size(); ++j) {
      const gptq_layer_job& b = jobs[g.jobs[j]];
      if (done[j] || b.damp != a.damp || b.desc_act != a.desc_act) continue;
      done[j] = 1;
      if (b.perm_out)
        CK(cudaMemcpyAsync(b.perm_out, c->perm, static_cast<size_t>(c->n) * 4, cudaMemcpyDeviceToDevice, c->stream));
      s = gptq_quantize_layer(c, b.W_fp16, b.m, b.qp, b.codes_out, b.scales_out, b.zeros_out, b.g_idx_out,
                              b.W_hat_out);
      if (s != GPTQ_OK) return s;
    }
  }
  return GPTQ_OK;
}

gptq_status enqueue_hessian(gptq_ctx* c, const gptq_layer_job& a) {
  gptq_status s = gptq_reset(c);
  if (s == GPTQ_OK) s = gptq_hessian_accumulate(c, a.X_bf16, a.n_tok, a.ld_x);
  return s;
}

}  // namespace

struct gptq_pipeline {
  int device = 0;
  cudaStream_t user = nullptr;
  Slot slot[2];
  cudaEvent_t ev = nullptr;
};

namespace {

gptq_status pipeline_free(gptq_pipeline* p) {
  gptq_status st = GPTQ_OK;
  for (auto& sl : p->slot) {
    for (auto& e : sl.ctx) {
      const gptq_status d = gptq_destroy(e.second);
      if (st == GPTQ_OK) st = d;
    }
    sl.ctx.clear();
    if (sl.stream) cudaStreamDestroy(sl.stream);
    sl.stream = nullptr;
  }
  if (p->ev) cudaEventDestroy(p->ev);
  p->ev = nullptr;
  return st;
}

bool valid_job(const gptq_layer_job& j) {
  return j.W_fp16 && j.codes_out && j.scales_out && j.zeros_out && j.m >= 1 && j.n_tok >= 0 &&
         (j.n_tok == 0 || j.X_bf16) && valid_qparams(j.qp, j.n) && gptq_workspace_bytes(j.n, j.m) != 0 &&
         j.damp >= 0.0 && j.damp <= 1e6 && (j.desc_act == 0 || j.desc_act == 1);
}

}  // namespace

extern "C" gptq_status gptq_pipeline_create(gptq_pipeline** out, const int64_t* widths, const int64_t* m_max, int count,
                                            int device, void* cuda_stream) {
  if (!out || !widths || !m_max || count < 1) return GPTQ_ERR_ARG;
  *out = nullptr;
  size_t need = 0;
  for (int i = 0; i < count; ++i) {
    const size_t b = gptq_workspace_bytes(widths[i], m_max[i]);
    if (b == 0) return GPTQ_ERR_ARG;
    for (int j = 0; j < i; ++j)
      if (widths[j] == widths[i]) return GPTQ_ERR_ARG;  // one entry per width
    need += 2 * b;
  }
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  size_t free_b = 0, total_b = 0;
  CK(cudaMemGetInfo(&free_b, &total_b));
  const int64_t env_limit = env_int("GPTQ_MAX_WORKSPACE_BYTES", -1);
  if (need > free_b || (env_limit >= 0 && static_cast<int64_t>(need) > env_limit)) return GPTQ_ERR_OOM;
  gptq_pipeline* p = new gptq_pipeline();
  p->device = device;
  p->user = static_cast<cudaStream_t>(cuda_stream);
  gptq_status st = GPTQ_OK;
  for (auto& sl : p->slot) {
    if (cudaStreamCreateWithFlags(&sl.stream, cudaStreamNonBlocking) != cudaSuccess) {
      st = GPTQ_ERR_CUDA;
      break;
    }
    for (int i = 0; i < count && st == GPTQ_OK; ++i) {
      gptq_ctx* c = nullptr;
      st = gptq_create(&c, widths[i], m_max[i], device, sl.stream);
      if (st == GPTQ_OK) sl.ctx.emplace_back(widths[i], c);
    }
    if (st != GPTQ_OK) break;
  }
  if (st == GPTQ_OK && cudaEventCreateWithFlags(&p->ev, cudaEventDisableTiming) != cudaSuccess) st = GPTQ_ERR_CUDA;
  if (st != GPTQ_OK) {
    pipeline_free(p);
    delete p;
    return st;
  }
  *out = p;
  return GPTQ_OK;
}

extern "C" gptq_status gptq_pipeline_run(gptq_pipeline* p, const gptq_layer_job* jobs, int count) {
  if (!p || !jobs || count < 1) return GPTQ_ERR_ARG;
  for (int i = 0; i < count; ++i) {
    if (!valid_job(jobs[i])) return GPTQ_ERR_ARG;
    gptq_ctx* c = p->slot[0].get(jobs[i].n);
    if (!c || jobs[i].m > c->m_max) return GPTQ_ERR_ARG;  // no context of that width, or too many rows
  }
  // groups of jobs that share their calibration input, in order of first appearance
  std::vector<LayerGroup> groups;
  for (int i = 0; i < count; ++i) {
    LayerGroup* g = nullptr;
    for (auto& e : groups)
      if (same_input(*e.first, jobs[i])) g = &e;
    if (!g) {
      groups.push_back(LayerGroup{&jobs[i], {}});
      g = &groups.back();
    }
    g->jobs.push_back(i);
  }
  DeviceGuard dg(p->device);
  // start after the caller's stream
  CK(cudaEventRecord(p->ev, p->user));
  for (auto& sl : p->slot) CK(cudaStreamWaitEvent(sl.stream, p->ev, 0));
  // Group i runs on slot i % 2: its Hessian and factorization are enqueued behind that slot's
  // earlier work, while the quantization of group i-1, enqueued on the other slot, runs; the
  // host waits only inside each factorization (for its pivot check).
  gptq_status st = GPTQ_OK;
  for (size_t i = 0; i < groups.size() && st == GPTQ_OK; ++i) {
    gptq_ctx* c = p->slot[i & 1].get(groups[i].first->n);
    st = enqueue_hessian(c, *groups[i].first);
    if (st == GPTQ_OK) st = run_group(c, jobs, groups[i]);
  }
  // wait for both slots, collect any device-side failure, and order the caller's stream after
  for (auto& sl : p->slot)
    for (auto& e : sl.ctx) {
      const gptq_status s = gptq_synchronize(e.second);
      if (st == GPTQ_OK) st = s;
    }
  return st;
}

extern "C" gptq_status gptq_pipeline_destroy(gptq_pipeline* p) {
  if (!p) return GPTQ_OK;
  gptq_status st;
  {
    DeviceGuard dg(p->device);
    st = pipeline_free(p);
  }
  delete p;
  return st;
}

extern "C" gptq_status gptq_quantize_layers(const gptq_layer_job* jobs, int count, int device, void* cuda_stream) {
  if (!jobs || count < 1) return GPTQ_ERR_ARG;
  std::vector<int64_t> widths, mm;
  for (int i = 0; i < count; ++i) {
    if (!valid_job(jobs[i])) return GPTQ_ERR_ARG;
    bool found = false;
    for (size_t w = 0; w < widths.size(); ++w)
      if (widths[w] == jobs[i].n) {
        mm[w] = std::max(mm[w], jobs[i].m);
        found = true;
      }
    if (!found) {
      widths.push_back(jobs[i].n);
      mm.push_back(jobs[i].m);
    }
  }
  gptq_pipeline* p = nullptr;
  gptq_status st = gptq_pipeline_create(&p, widths.data(), mm.data(), static_cast<int>(widths.size()), device, cuda_stream);
  if (st != GPTQ_OK) return st;
  st = gptq_pipeline_run(p, jobs, count);
  const gptq_status d = gptq_pipeline_destroy(p);
  return st != GPTQ_OK ? st : d;
}

// ==========================================================================================
// AWQ channel scaling and round-to-nearest on the same inputs (awq_kernels.cuh)
// ==========================================================================================
namespace {
// Position of the p-th percentile among k sorted values, in the fp32 steps of numpy's linear
// method: p rounded to fp32 and divided by 100, h = (k - 1) q, the ranks floor(h) and
// floor(h) + 1 (clamped to k - 1), the weight t = h - floor(h) and 1 - t.
struct PctPos {
  int lo, hi;
  float t, omt;
};
PctPos pct_position(double p, int k) {
  const float q = static_cast<float>(p) / 100.0f;
  volatile float h = static_cast<float>(k - 1) * q;  // rounded once, before the floor
  const float hv = h;
  const int lo = std::max(0, std::min(static_cast<int>(std::floor(hv)), k - 1));
  const float t = hv - static_cast<float>(lo);
  return {lo, std::min(lo + 1, k - 1), t, 1.0f - t};
}

AwqRtnArgs rtn_args(const void* W, int m, int n, const gptq_qparams& qp, const float* channel_scale, uint32_t* codes,
                    float* scales, float* zeros, float* W_hat) {
  AwqRtnArgs a{};
  a.W = static_cast<const __half*>(W);
  a.scale = channel_scale;
  a.m = m;
  a.n = n;
  a.bits = qp.bits;
  a.sym = qp.sym;
  a.g = (qp.group_size == -1) ? n : qp.group_size;
  a.G = n / a.g;
  a.codes = codes;
  a.scales = scales;
  a.zeros = zeros;
  a.W_hat = W_hat;
  a.clip = 0;
  return a;
}

gptq_status launch_rtn(const AwqRtnArgs& a, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(a.n + 6 * a.G) * 4;  // row, scales, zeros, order statistics
  CK(cudaFuncSetAttribute(awq_rtn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
  awq_rtn_kernel<<<a.m, 256, smem, st>>>(a);
  CKL("awq_rtn");
  return GPTQ_OK;
}
}  // namespace

extern "C" size_t gptq_awq_workspace_bytes(int64_t n) {
  if (n < 128 || n > kMaxN || n % 128) return 0;
  return 256 + static_cast<size_t>(n) * sizeof(double);
}

extern "C" gptq_status gptq_awq_quantize(const void* X, int64_t n_tok, int64_t ld_x, const void* W, int64_t m, int64_t n,
                                         float s_protect, gptq_qparams qp, uint32_t* codes, float* scales,
                                         float* zeros, float* channel_scale, float* W_hat, void* workspace,
                                         size_t workspace_bytes, int device, void* cuda_stream) {
  if (!W || !codes || !scales || !zeros || !channel_scale || !workspace) return GPTQ_ERR_ARG;
  if (gptq_awq_workspace_bytes(n) == 0 || workspace_bytes < gptq_awq_workspace_bytes(n)) return GPTQ_ERR_ARG;
  if (m < 1 || m > kMaxM || n_tok < 0 || n_tok >= (int64_t(1) << 40) || (n_tok > 0 && !X)) return GPTQ_ERR_ARG;
  if (!valid_qparams(qp, n) || !(s_protect > 0.0f) || !(s_protect < 1e30f)) return GPTQ_ERR_ARG;
  if ((X && (!aligned16(X) || ld_x < n || ld_x % 8)) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return GPTQ_ERR_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const int ni = static_cast<int>(n), mi = static_cast<int>(m);
  double* median = reinterpret_cast<double*>(workspace);
  double* sums = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + 256);
  CK(cudaMemsetAsync(workspace, 0, gptq_awq_workspace_bytes(n), st));
  if (n_tok > 0) {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
    const int gx = (ni + AWQ_SUM_COLS - 1) / AWQ_SUM_COLS;
    const int gy = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((4 * sms + gx - 1) / gx, (n_tok + 7) / 8)));
    channel_abs_sum_kernel<<<dim3(gx, gy), dim3(32, 8), 0, st>>>(static_cast<const __nv_bfloat16*>(X), n_tok, ld_x, ni,
                                                                 sums);
    CKL("channel_abs_sum");
  }
  awq_median_kernel<<<(ni + 255) / 256, 256, 0, st>>>(sums, ni, median);
  CKL("awq_median");
  awq_scale_kernel<<<(ni + 255) / 256, 256, 0, st>>>(sums, ni, n_tok, median, s_protect, channel_scale);
  CKL("awq_scale");
  return launch_rtn(rtn_args(W, mi, ni, qp, channel_scale, codes, scales, zeros, W_hat), st);
}

// Round-to-nearest with an optional percentile range ("模型量化实战…" §3.1 LinearQuantizer)
extern "C" gptq_status gptq_rtn_quantize(const void* W, int64_t m, int64_t n, gptq_qparams qp, float clip_ratio,
                                         const float* channel_scale, uint32_t* codes, float* scales, float* zeros,
                                         float* W_hat, int device, void* cuda_stream) {
  if (!W || !codes || !scales || !zeros) return GPTQ_ERR_ARG;
  if (n < 128 || n > kMaxN || n % 128 || m < 1 || m > kMaxM) return GPTQ_ERR_ARG;
  if (!valid_qparams(qp, n) || !(clip_ratio > 0.0f && clip_ratio <= 1.0f)) return GPTQ_ERR_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  AwqRtnArgs a = rtn_args(W, static_cast<int>(m), static_cast<int>(n), qp, channel_scale, codes, scales, zeros, W_hat);
  if (clip_ratio < 1.0f) {
    const double c = clip_ratio;
    const PctPos lo = pct_position(qp.sym ? c * 100.0 : (1.0 - c) * 50.0, a.g);
    const PctPos hi = qp.sym ? lo : pct_position(100.0 - (1.0 - c) * 50.0, a.g);
    a.clip = 1;
    a.rank[0] = lo.lo;
    a.rank[1] = lo.hi;
    a.rank[2] = hi.lo;
    a.rank[3] = hi.hi;
    a.t_lo = lo.t;
    a.omt_lo = lo.omt;
    a.t_hi = hi.t;
    a.omt_hi = hi.omt;
  }
  return launch_rtn(a, static_cast<cudaStream_t>(cuda_stream));
}

extern "C" int gptq_test_pct_position(double p, int k, int* lo, int* hi, float* t, float* omt) {
  if (!(p >= 0.0 && p <= 100.0) || k < 1 || !lo || !hi || !t || !omt) return -1;
  const PctPos q = pct_position(p, k);
  *lo = q.lo;
  *hi = q.hi;
  *t = q.t;
  *omt = q.omt;
  return 0;
}

// ==========================================================================================
// Sequential quantization: a layer's output, through its activation, as the next layer's inputs
// ==========================================================================================
extern "C" gptq_status gptq_activation_convert(const void* Y, int in_bf16, int64_t count, int act, void* out_bf16,
                                               void* out_fp16, int device, void* cuda_stream) {
  if (count < 0 || (count > 0 && !Y) || (!out_bf16 && !out_fp16) || (act != 0 && act != 1) ||
      (in_bf16 != 0 && in_bf16 != 1))
    return GPTQ_ERR_ARG;
  if (count == 0) return GPTQ_OK;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  DeviceGuard dg(device);
  activation_convert_kernel<<<4 * 148, 256, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
      Y, in_bf16, static_cast<size_t>(count), act, static_cast<__nv_bfloat16*>(out_bf16), static_cast<__half*>(out_fp16));
  CKL("activation_convert");
  return GPTQ_OK;
}
