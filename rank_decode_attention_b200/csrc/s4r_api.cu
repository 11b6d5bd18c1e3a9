// s4r_api.cu -- the C ABI of libs4r (declared in include/s4r.h): host-side
// validation, workspace layout and kernel launches.  Every step of the decode
// and encode paths runs in the kernels included below; the host only checks
// arguments and enqueues launches on the caller's stream.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "k_attend.cuh"
#include "k_attend_rows.cuh"
#include "k_basis.cuh"
#include "k_encode_simt.cuh"
#include "k_encode_tc.cuh"
#include "k_project.cuh"
#include "k_score_simt.cuh"
#include "k_score_pair.cuh"
#include "k_score_rows.cuh"
#include "k_score_tc.cuh"
#include "k_topk.cuh"

using namespace s4r;

static_assert(S4R_MAX_GROUP <= kAttMaxGroup && S4R_MAX_SINKS <= kAttMaxSinks && S4R_MAX_RANK <= kAttThreads,
              "header limits must fit the attention kernel");

namespace {

constexpr size_t kAlign = 256;
inline size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t esize(s4r_dtype dt) { return dt == S4R_BF16 ? 2 : 4; }

// Byte offsets of the decode workspace regions.
struct Layout {
  size_t status, counters, cq, cqs, qt, tstat, rstat, rowsum, ehist, scores, pooled, total;
};

Layout layout_for(const Shape &s) {
  Layout l{};
  size_t off = 0;
  l.status = off;
  off += kAlign;
  l.counters = off; off += round_up(sizeof(uint32_t) * (size_t)s.batch);
  l.cq = off; off += round_up(sizeof(float) * s.batch * (size_t)s.n_rows * s.rank_k);
  const size_t n_cb = (size_t)ceil_div(s.rank_k, kProjColBlock);
  l.cqs = off; off += round_up((size_t)kCqsCopies * s.batch * n_cb * cqs_block_bytes(s.n_rows));
  l.qt = off; off += round_up(sizeof(float) * s.batch * (size_t)s.n_heads_q * s.rank_k);
  const size_t n_tiles = (size_t)ceil_div(s.cache_rows, kScoreTile);
  l.tstat = off; off += round_up(sizeof(double) * 2 * s.batch * n_tiles * s.n_rows);
  l.rstat = off; off += round_up(sizeof(double) * 2 * s.batch * (size_t)s.n_rows);
  l.rowsum = off; off += round_up(sizeof(double) * s.batch * (size_t)kStcSumSlots * s.n_rows);
  l.ehist = off; off += round_up(sizeof(uint32_t) * s.batch * (size_t)kExpBins);
  l.scores = off; off += round_up(sizeof(float) * s.batch * (size_t)s.cache_rows);
  l.pooled = off; if (s.pool_kernel > 1) off += round_up(sizeof(float) * s.batch * (size_t)s.cache_rows);
  l.total = off;
  return l;
}

// Shape checks shared by workspace sizing and the decode step.
s4r_status make_shape(const s4r_decode_args *a, Shape *s) {
  if (!a) return S4R_ERR_INVALID_ARG;
  if (a->batch < 0 || a->n_heads_q <= 0 || a->n_heads_kv <= 0 || a->head_dim <= 0 ||
      a->rank_k <= 0 || a->rank_v <= 0 || a->n_sink < 0 || a->local_window < 0 ||
      a->top_k < 0 || a->query_window <= 0 || a->pool_kernel < 1 || a->cache_rows < 0)
    return S4R_ERR_INVALID_ARG;
  if (a->n_heads_q % a->n_heads_kv != 0) return S4R_ERR_INVALID_ARG;
  if (a->dtype != S4R_F32 && a->dtype != S4R_BF16) return S4R_ERR_INVALID_ARG;
  if (a->row_mode != S4R_ROWS_CONCAT && a->row_mode != S4R_ROWS_PER_HEAD) return S4R_ERR_INVALID_ARG;
  if (a->pool_kernel % 2 == 0) return S4R_ERR_INVALID_ARG;
  if (a->pool_mode != S4R_POOL_MAX && a->pool_mode != S4R_POOL_AVG) return S4R_ERR_INVALID_ARG;
  const int64_t G = a->n_heads_q / a->n_heads_kv;
  const int64_t Dp = (int64_t)a->n_heads_kv * a->head_dim;
  const int64_t R = (a->row_mode == S4R_ROWS_CONCAT) ? (int64_t)a->query_window * G
                                                    : (int64_t)a->query_window * a->n_heads_q;
  if (a->head_dim % 8 || a->rank_k % 8 || a->rank_v % 8) return S4R_ERR_UNSUPPORTED;
  if (a->head_dim > S4R_MAX_HEAD_DIM || Dp > S4R_MAX_D_MODEL || a->rank_k > S4R_MAX_RANK ||
      a->rank_v > S4R_MAX_RANK || R > S4R_MAX_SCORE_ROWS || G > S4R_MAX_GROUP ||
      a->pool_kernel > S4R_MAX_POOL_KERNEL)
    return S4R_ERR_UNSUPPORTED;
  if (a->cache_rows + a->n_sink > INT32_MAX) return S4R_ERR_UNSUPPORTED;
  if (a->n_sink > S4R_MAX_SINKS || (int64_t)a->top_k + a->local_window > S4R_MAX_SELECTED) return S4R_ERR_UNSUPPORTED;
  s->batch = a->batch;
  s->n_heads_q = a->n_heads_q;
  s->n_heads_kv = a->n_heads_kv;
  s->head_dim = a->head_dim;
  s->rank_k = a->rank_k;
  s->rank_v = a->rank_v;
  s->n_sink = a->n_sink;
  s->local_window = a->local_window;
  s->top_k = a->top_k;
  s->query_window = a->query_window;
  s->pool_kernel = a->pool_kernel;
  s->pool_mode = a->pool_mode;
  s->row_mode = a->row_mode;
  s->d_model = (int32_t)Dp;
  s->group = (int32_t)G;
  s->n_rows = (int32_t)R;
  s->cache_rows = a->cache_rows;
  {
    const int es = a->dtype == S4R_BF16 ? 2 : 4;
    if (att_smem_bytes(*s, es, att_plan(*s, es)) > kAttSmemBudget) return S4R_ERR_UNSUPPORTED;
  }
  return S4R_OK;
}

// Description of the last failure on this host thread (s4r_last_error).
thread_local char g_last_error[256] = "";

s4r_status fail(const char *what, cudaError_t err) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", what, cudaGetErrorName(err), cudaGetErrorString(err));
  return S4R_ERR_CUDA;
}
// Status of the launches enqueued since the previous check, labelled `what`.
s4r_status check_launch(const char *what) {
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? S4R_OK : fail(what, err);
}
s4r_status last_cuda() { return check_launch("kernel launch"); }

// Per-device caches of launch set-up, so that a decode call costs only its
// launches on the host.
constexpr int kMaxDevices = 64;
inline int current_device() {
  int dev = 0;
  return cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices ? dev : -1;
}

// Multiprocessors of the current device (cached).
inline int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  const int dev = current_device();
  if (dev >= 0) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int d = 0, n = 148;
  if (cudaGetDevice(&d) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) {
    cudaGetLastError();
    n = 148;
  }
  if (dev >= 0) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Raise Kernel's dynamic shared-memory limit to `bytes` unless an earlier
// launch on this device already raised it at least that far.
template <auto Kernel>
cudaError_t ensure_smem(size_t bytes) {
  static std::atomic<int> set_to[kMaxDevices];
  const int dev = current_device();
  if (dev >= 0 && set_to[dev].load(std::memory_order_relaxed) >= (int)bytes) return cudaSuccess;
  const cudaError_t err = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (err == cudaSuccess && dev >= 0) {
    int cur = set_to[dev].load(std::memory_order_relaxed);
    while (cur < (int)bytes && !set_to[dev].compare_exchange_weak(cur, (int)bytes)) {
    }
  }
  return err;
}

// Launch attribute that lets a kernel start while the previous kernel in the
// stream drains (its CTAs wait in pdl_wait before reading that kernel's
// output).  Every decode kernel launched with it calls pdl_wait first.
inline cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

// Whether the cooperative scoring launch accepts the attribute above
// (-1 not tried yet, 0 no, 1 yes).
int g_coop_pdl = -1;

// cuTensorMapEncodeTiled, resolved through the runtime (no link-time libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 tensor map, 128-byte swizzle: `inner` contiguous elements per row,
// `outer` rows `row_bytes` apart, box of box_inner x box_outer elements.
bool make_tmap_bf16(CUtensorMap *map, const void *ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor-core encode of bf16 states (rank % 32 == 0) for n_prob (1 or 2)
// problems of the same shape in one persistent launch.
s4r_status encode_tc_launch(int n_prob, const void *const *states, int64_t n, int64_t lds,
                            const void *const *basis, int d, int r, void *const *coeffs, int64_t ldc,
                            cudaStream_t st) {
  CUtensorMap ms[2], mb[2];
  for (int p = 0; p < n_prob; ++p)
    if (!make_tmap_bf16(&ms[p], states[p], (uint64_t)d, (uint64_t)n, (uint64_t)lds * 2, kEncBK, kEncBM) ||
        !make_tmap_bf16(&mb[p], basis[p], (uint64_t)r, (uint64_t)d, (uint64_t)r * 2, 64, kEncBK))
      return S4R_ERR_CUDA;
  if (n_prob == 1) {
    ms[1] = ms[0];
    mb[1] = mb[0];
  }
  EncOut<bf16> o;
  for (int p = 0; p < 2; ++p) {
    o.C[p] = static_cast<bf16 *>(coeffs[p < n_prob ? p : 0]);
    o.ldc[p] = ldc;
  }
  const size_t smem = enc_smem_bytes(r);
  ensure_smem<encode_tc_kernel<bf16>>(smem);
  const unsigned grid = (unsigned)smin<int64_t>(n_prob * ceil_div(n, kEncBM), sm_count());
  encode_tc_kernel<bf16><<<grid, kEncThreads, smem, st>>>(ms[0], mb[0], ms[1], mb[1], o, n_prob, n, d, r);
  return last_cuda();
}

// Which latent-scoring kernel a decode call uses.
struct ScorePlan {
  bool tc = false;   // tensor-core kernel (else fp64 CUDA-core passes)
  bool pair = false; // the fused two-tiles-per-CTA kernel (one problem, one resident wave)
  bool rows = false; // the two-pass kernel for R > 64 rows (per-head rows)
  int R = 0;         // rows per problem (template argument of the TC kernel)
  int grid = 0;      // persistent cooperative grid
  int K = 1;         // consecutive tiles per chunk of the round-robin
  int nB = 1;        // split C_Q operand buffers
  size_t smem = 0;
};

// Whether the tensor-core scoring kernel can run with this much dynamic shared
// memory on the current device: the kernel's limit is raised to it (once per
// size) and one CTA must fit an SM.  Results are cached per device and size.
template <int R>
bool tc_launchable(size_t smem) {
  constexpr int kSizes = 8;
  static std::mutex mu;
  static int known[kMaxDevices][kSizes][2];   // (size, 1 yes / -1 no)
  const int dev = current_device();
  if (ensure_smem<score_tc_kernel<R>>(smem) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (dev >= 0) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kSizes; ++i)
      if (known[dev][i][0] == (int)smem) return known[dev][i][1] > 0;
  }
  int per_sm = 0;
  const bool ok = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_tc_kernel<R>, StcCfg<R>::kThreads, smem) ==
                      cudaSuccess &&
                  per_sm > 0;
  if (!ok) cudaGetLastError();
  if (dev >= 0) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kSizes; ++i)
      if (known[dev][i][0] == 0) {
        known[dev][i][0] = (int)smem;
        known[dev][i][1] = ok ? 1 : -1;
        break;
      }
  }
  return ok;
}

// Whether a pass of the many-rows kernel can be resident (one CTA per SM).
template <int PASS>
bool rows_launchable(size_t smem) {
  if (ensure_smem<score_rows_kernel<PASS>>(smem) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  int per_sm = 0;
  const bool ok =
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_rows_kernel<PASS>, kSrThreads, smem) == cudaSuccess &&
      per_sm > 0;
  if (!ok) cudaGetLastError();
  return ok;
}

// Whether the fused two-tiles-per-CTA kernel can run with `grid` CTAs, all
// resident at once (one per SM: each holds all 512 TMEM columns).
template <int R>
bool pair_launchable(size_t smem, int rank, int grid) {
  if (grid > sm_count()) return false;
  static std::atomic<int> ok_cache[kMaxDevices][S4R_MAX_RANK / 8 + 1];   // per rank: 0 unknown, 1 no, 2 yes
  const int dev = current_device();
  const int slot = rank / 8;
  if (ensure_smem<score_pair_kernel<R>>(smem) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (dev >= 0) {
    const int c = ok_cache[dev][slot].load(std::memory_order_relaxed);
    if (c > 0) return c == 2;
  }
  int per_sm = 0;
  const bool ok = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_pair_kernel<R>, sp_threads(R), smem) ==
                      cudaSuccess &&
                  per_sm > 0;
  if (!ok) cudaGetLastError();
  if (dev >= 0) ok_cache[dev][slot].store(ok ? 2 : 1, std::memory_order_relaxed);
  return ok;
}

// How many clusters of `nc` CTAs of the row-split attention kernel can be
// resident at once with `smem` bytes each (0: not launchable).  Cached per
// device, cluster size and shared-memory size.
int ar_active_clusters(int nc, size_t smem) {
  constexpr int kSizes = 16;
  static std::mutex mu;
  static int known[kMaxDevices][kSizes][3];   // (nc, smem, clusters + 1)
  const int dev = current_device();
  if (ensure_smem<attend_rows_kernel>(smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kSizes; ++i)
      if (known[dev][i][0] == nc && known[dev][i][1] == (int)smem) return known[dev][i][2] - 1;
  }
  int n = 0;
  if (nc > 8 && cudaFuncSetAttribute(attend_rows_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                    cudaSuccess) {
    cudaGetLastError();
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)nc, 1, 1);
    cfg.blockDim = dim3(kArThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)nc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attend_rows_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
  }
  if (dev >= 0) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kSizes; ++i)
      if (known[dev][i][0] == 0) {
        known[dev][i][0] = nc;
        known[dev][i][1] = (int)smem;
        known[dev][i][2] = n + 1;
        break;
      }
  }
  return n;
}

// Plan of the row-split attention kernel (bf16 storage); nc == 0 when the
// shape or the pointers do not suit it and the per-group kernel runs.
// The row-split kernel reads each selected row once for every kv group, which
// pays once a call holds several problems; a single problem is latency-bound
// and runs faster on the per-group kernel's kv groups x ranks CTAs (measured
// on one 32K layer with r = 192: 873 against 847 decode steps/s over 32
// per-layer calls; 128K and per-head rows gain 1%).  Clusters of 16 CTAs
// halve each CTA's rows; they are taken while every problem's cluster can be
// resident at once, else clusters of 8.
ArPlan plan_attend_rows(const Shape &s, const void *ck, const void *cv, const void *bv) {
  ArPlan none{};
  if (s.batch < 2) return none;
  if (!ar_supported(s, 2) || !aligned16(ck) || !aligned16(cv) || !aligned16(bv)) return none;
  for (int nc : {16, 8, 4, 2, 1}) {
    if (s.n_heads_q % nc != 0) continue;
    const ArPlan pl = ar_plan(s, nc);
    const size_t smem = ar_layout(s, pl).total;
    if (!ar_plan_ok(pl) || smem > kArSmemBudget) continue;
    const int n = ar_active_clusters(nc, smem);
    if (n <= 0) continue;
    if (nc == 16 && s.batch > n) continue;
    return pl;
  }
  return none;
}

ScorePlan plan_scoring(const Shape &s, s4r_dtype dt) {
  ScorePlan p;
  if (dt != S4R_BF16 || s.cache_rows == 0 || s.batch == 0) return p;
  if (s.n_rows > 64 && s.n_rows % kSrRc == 0 && s.n_rows <= S4R_MAX_SCORE_ROWS &&
      (int64_t)s.batch * s.cache_rows < INT32_MAX) {
    // many rows (per-head): chunks of 64 rows, two passes over the cache
    const size_t smem = (size_t)sr_smem_bytes(s.rank_k, sr_buffers(s.rank_k));
    if (rows_launchable<1>(smem) && rows_launchable<2>(smem)) {
      p.tc = true;
      p.rows = true;
      p.R = s.n_rows;
      p.smem = smem;
      return p;
    }
  }
  if (s.n_rows != 32 && s.n_rows != 64) return p;
  if ((int64_t)s.batch * s.cache_rows >= INT32_MAX) return p;
  const int R = s.n_rows;
  if (s.batch == 1) {
    // One problem whose tile pairs fit one resident wave: the fused kernel
    // (fewer fixed latencies for a latency-bound single layer).
    const int64_t pairs = ceil_div(ceil_div(s.cache_rows, kStcTile), kSpTiles);
    const size_t psmem = (size_t)sp_smem_bytes(R, s.rank_k);
    if (pairs <= sm_count() &&
        (R == 64 ? pair_launchable<64>(psmem, s.rank_k, (int)pairs) : pair_launchable<32>(psmem, s.rank_k, (int)pairs))) {
      p.tc = true;
      p.pair = true;
      p.R = R;
      p.grid = (int)pairs;
      p.smem = psmem;
      return p;
    }
  }
  // A second operand buffer pays when the CTAs switch problems.
  const int nB = (s.batch > 1 && stc_two_b_fit(R, s.rank_k)) ? 2 : 1;
  const size_t smem = (size_t)stc_smem_bytes(R, s.rank_k, nB);
  if (!(R == 64 ? tc_launchable<64>(smem) : tc_launchable<32>(smem))) return p;
  // One CTA per SM: each holds all 512 TMEM columns.
  const int64_t tiles = (int64_t)s.batch * ceil_div(s.cache_rows, kStcTile);
  p.tc = true;
  p.R = R;
  p.grid = (int)smin<int64_t>(tiles, sm_count());
  // Chunks of one tile balance the CTAs best (at most ceil(tiles / G) each,
  // so the fewest tiles beyond the kept ones); when problems are shorter
  // than the grid, chunks of two keep each CTA on fewer problems, which
  // waits less for problems to complete before kept slots free up.
  // (Measured: 128K 329 -> 352 steps/s, ragged +2%, 32 x 32K in one call +3%
  // with one-tile chunks; 16 x 8K 314 with two-tile chunks, 289 with one, 308 with four.)
  const bool short_problems = ceil_div(s.cache_rows, kStcTile) < (int64_t)p.grid;
  p.K = (tiles > 2 * (int64_t)p.grid && short_problems) ? 2 : 1;
  p.nB = nB;
  p.smem = smem;
  return p;
}

template <int R>
s4r_status launch_score_tc(const ScorePlan &p, const CUtensorMap &tmap, const Shape &s, const int32_t *lengths,
                           const unsigned char *cqs, float *scores, double *rowsum, uint32_t *ehist,
                           unsigned int *counters, uint32_t *status, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid);
  cfg.blockDim = dim3(StcCfg<R>::kThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1] = pdl_attr();
  cfg.attrs = attr;
  cfg.numAttrs = g_coop_pdl == 0 ? 1 : 2;
  cudaError_t err = cudaLaunchKernelEx(&cfg, score_tc_kernel<R>, tmap, s, lengths, cqs, scores, rowsum, ehist,
                                       counters, status, p.K, p.nB);
  if (cfg.numAttrs == 2 && g_coop_pdl < 0) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cap);
    if (err == cudaSuccess) {
      g_coop_pdl = 1;
    } else if (cap == cudaStreamCaptureStatusNone) {
      cudaGetLastError();   // not supported together: launch without it from now on
      g_coop_pdl = 0;
      cfg.numAttrs = 1;
      err = cudaLaunchKernelEx(&cfg, score_tc_kernel<R>, tmap, s, lengths, cqs, scores, rowsum, ehist, counters,
                               status, p.K, p.nB);
    }
  }
  return err == cudaSuccess ? S4R_OK : fail("score_tc_kernel (cooperative launch)", err);
}

template <int R>
s4r_status launch_score_pair(const ScorePlan &p, const CUtensorMap &tmap, const Shape &s, const int32_t *lengths,
                             const unsigned char *cqs, float *scores, double *rowsum, uint32_t *ehist,
                             unsigned int *bar, uint32_t *status, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid);
  cfg.blockDim = dim3(sp_threads(R));
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1] = pdl_attr();
  cfg.attrs = attr;
  cfg.numAttrs = g_coop_pdl == 0 ? 1 : 2;
  cudaError_t err = cudaLaunchKernelEx(&cfg, score_pair_kernel<R>, tmap, s, lengths, cqs, scores, rowsum, ehist, bar,
                                       status);
  if (cfg.numAttrs == 2 && g_coop_pdl < 0) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cap);
    if (err == cudaSuccess) {
      g_coop_pdl = 1;
    } else if (cap == cudaStreamCaptureStatusNone) {
      cudaGetLastError();   // not supported together: launch without it from now on
      g_coop_pdl = 0;
      cfg.numAttrs = 1;
      err = cudaLaunchKernelEx(&cfg, score_pair_kernel<R>, tmap, s, lengths, cqs, scores, rowsum, ehist, bar, status);
    }
  }
  return err == cudaSuccess ? S4R_OK : fail("score_pair_kernel (cooperative launch)", err);
}

template <typename T>
s4r_status decode_launch(const s4r_decode_args *a, const Shape &s, const Layout &ly, cudaStream_t st) {
  unsigned char *ws = static_cast<unsigned char *>(a->workspace);
  uint32_t *status = reinterpret_cast<uint32_t *>(ws + ly.status);
  float *cq = reinterpret_cast<float *>(ws + ly.cq);
  float *qt = reinterpret_cast<float *>(ws + ly.qt);
  double *tstat = reinterpret_cast<double *>(ws + ly.tstat);
  double *rstat = reinterpret_cast<double *>(ws + ly.rstat);
  double *rowsum = reinterpret_cast<double *>(ws + ly.rowsum);
  uint32_t *ehist = reinterpret_cast<uint32_t *>(ws + ly.ehist);
  unsigned char *cqs = ws + ly.cqs;
  unsigned int *counters = reinterpret_cast<unsigned int *>(ws + ly.counters);
  float *scores = a->scores ? a->scores : reinterpret_cast<float *>(ws + ly.scores);
  float *pooled = reinterpret_cast<float *>(ws + ly.pooled);
  const T *q = static_cast<const T *>(a->q);
  const T *ck = static_cast<const T *>(a->coeff_k);
  const T *cv = static_cast<const T *>(a->coeff_v);
  const T *bk = static_cast<const T *>(a->basis_k);
  const T *bv = static_cast<const T *>(a->basis_v);
  const T *sk = static_cast<const T *>(a->sink_k);
  const T *sv = static_cast<const T *>(a->sink_v);

  // 1. query projection
  {
    const unsigned n_rb = (unsigned)ceil_div((int64_t)s.query_window * s.group, kProjRowBlock);
    const unsigned n_rank = (unsigned)proj_cluster(s.n_heads_kv);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_rank, (unsigned)ceil_div(s.rank_k, kProjColBlock), n_rb * (unsigned)s.batch);
    cfg.blockDim = dim3(kProjThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = n_rank;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, project_kernel<T>, s, q, bk, cq, cqs, qt, rowsum, ehist, counters);
    if (err != cudaSuccess) return fail("project_kernel (cluster launch)", err);
    if (check_launch("project_kernel") != S4R_OK) return S4R_ERR_CUDA;
  }
  // 2. latent scoring
  const unsigned n_tiles = (unsigned)ceil_div(s.cache_rows, kScoreTile);
  if (a->profile_events[0])
    cudaEventRecordWithFlags(static_cast<cudaEvent_t>(a->profile_events[0]), st, cudaEventRecordExternal);
  const ScorePlan plan = plan_scoring(s, a->dtype);
  if (plan.tc) {
    CUtensorMap tmap;
    if (!make_tmap_bf16(&tmap, ck, (uint64_t)s.rank_k, (uint64_t)s.batch * s.cache_rows, (uint64_t)s.rank_k * 2, 64,
                        kStcTile)) {
      snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed for the key-coefficient cache");
      return S4R_ERR_CUDA;
    }
    // The fused kernel's grid barrier counts on the problem's counter word.
    if (plan.rows) {
      // pass 1 (row sums), 1 / l, pass 2 (scores); the SIMT path's row
      // statistics region holds 1 / l
      double *inv_l = rstat;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)ceil_div(s.cache_rows, kStcTile), (unsigned)s.batch);
      cfg.blockDim = dim3(kSrThreads);
      cfg.dynamicSmemBytes = plan.smem;
      cfg.stream = st;
      cudaLaunchAttribute attr[1] = {pdl_attr()};
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      cudaError_t err = cudaLaunchKernelEx(&cfg, score_rows_kernel<1>, tmap, s, a->lengths, cqs, rowsum, inv_l, scores,
                                           ehist, status);
      if (err != cudaSuccess) return fail("score_rows_kernel (pass 1)", err);
      cudaLaunchConfig_t fcfg = {};
      fcfg.gridDim = dim3((unsigned)s.batch);
      fcfg.blockDim = dim3(256);
      fcfg.stream = st;
      fcfg.attrs = attr;
      fcfg.numAttrs = 1;
      err = cudaLaunchKernelEx(&fcfg, score_rows_finish, s, (const double *)rowsum, inv_l);
      if (err != cudaSuccess) return fail("score_rows_finish", err);
      err = cudaLaunchKernelEx(&cfg, score_rows_kernel<2>, tmap, s, a->lengths, cqs, rowsum, (const double *)inv_l,
                               scores, ehist, status);
      if (err != cudaSuccess) return fail("score_rows_kernel (pass 2)", err);
      if (check_launch("score_rows_kernel") != S4R_OK) return S4R_ERR_CUDA;
    } else {
    const s4r_status rc =
        plan.pair ? (plan.R == 64 ? launch_score_pair<64>(plan, tmap, s, a->lengths, cqs, scores, rowsum, ehist, counters,
                                                          status, st)
                                  : launch_score_pair<32>(plan, tmap, s, a->lengths, cqs, scores, rowsum, ehist, counters,
                                                          status, st))
        : plan.R == 64 ? launch_score_tc<64>(plan, tmap, s, a->lengths, cqs, scores, rowsum, ehist, counters, status, st)
                       : launch_score_tc<32>(plan, tmap, s, a->lengths, cqs, scores, rowsum, ehist, counters, status, st);
    if (rc != S4R_OK) return rc;
    }
  } else if (n_tiles > 0) {
    const size_t smem = ScoreSmem::bytes(s.rank_k);
    ensure_smem<score_stats_simt<T>>(smem);
    ensure_smem<score_final_simt<T>>(smem);
    score_stats_simt<T><<<dim3(n_tiles, s.batch), kScoreThreads, smem, st>>>(s, a->lengths, ck, cq, tstat);
    score_merge<<<dim3((unsigned)ceil_div(s.n_rows, 8), s.batch), 256, 0, st>>>(s, a->lengths, tstat, rstat);
    score_final_simt<T><<<dim3(n_tiles, s.batch), kScoreThreads, smem, st>>>(s, a->lengths, ck, cq, rstat, scores);
    if (check_launch("score (CUDA-core passes)") != S4R_OK) return S4R_ERR_CUDA;
  }
  if (a->profile_events[1])
    cudaEventRecordWithFlags(static_cast<cudaEvent_t>(a->profile_events[1]), st, cudaEventRecordExternal);
  // 3. selection
  const float *keys = scores;
  if (s.pool_kernel > 1 && s.cache_rows > 0) {
    pool_kernel<<<dim3((unsigned)ceil_div(s.cache_rows, 256), s.batch), 256, 0, st>>>(s, a->lengths, scores, pooled);
    keys = pooled;
  }
  if (s.top_k > 0) {
    if (s.cache_rows <= (int64_t)kTopkCl * kTopkClKeys) {
      const size_t smem = topk_cl_smem_bytes();
      ensure_smem<topk_cluster_kernel>(smem);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(kTopkCl, (unsigned)s.batch);
      cfg.blockDim = dim3(kTopkClThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      cudaLaunchAttribute attr[1] = {pdl_attr()};
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      // The tensor-core scoring kernel also leaves the exponent histogram of
      // the candidates' scores (unpooled keys only).
      const uint32_t *kh = (plan.tc && keys == scores) ? ehist : nullptr;
      const cudaError_t err = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, s, a->lengths, keys, kh, a->idx, status);
      if (err != cudaSuccess) return fail("topk_cluster_kernel (cluster launch)", err);
    } else {
      const size_t smem = topk_smem_bytes(s.cache_rows);
      ensure_smem<topk_kernel>(smem);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)s.batch);
      cfg.blockDim = dim3(kTopkThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      cudaLaunchAttribute attr[1] = {pdl_attr()};
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      const cudaError_t err = cudaLaunchKernelEx(&cfg, topk_kernel, s, a->lengths, keys, a->idx, status);
      if (err != cudaSuccess) return fail("topk_kernel", err);
    }
    if (check_launch("topk_kernel") != S4R_OK) return S4R_ERR_CUDA;
  }
  // 4. rebuild + exact attention: the row-split kernel (one cluster per
  // problem, every head in every CTA) for bf16 storage and two or more
  // problems, else one cluster of CTAs per kv group
  ArPlan ap{};
  if constexpr (std::is_same<T, bf16>::value) ap = plan_attend_rows(s, ck, cv, bv);
  if (ap.nc > 0) {
    if constexpr (std::is_same<T, bf16>::value) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)ap.nc, (unsigned)s.batch);
      cfg.blockDim = dim3(kArThreads);
      cfg.dynamicSmemBytes = ar_layout(s, ap).total;
      cfg.stream = st;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)ap.nc;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      attr[1] = pdl_attr();
      cfg.attrs = attr;
      cfg.numAttrs = 2;
      const cudaError_t err = cudaLaunchKernelEx(&cfg, attend_rows_kernel, s, ap, a->lengths, a->idx, ck, cv, qt, q,
                                                 bv, sk, sv, a->out, status);
      if (err != cudaSuccess) return fail("attend_rows_kernel (cluster launch)", err);
      if (check_launch("attend_rows_kernel") != S4R_OK) return S4R_ERR_CUDA;
    }
  } else {
    AttPlan pl = att_plan(s, (int)sizeof(T), att_ranks(s, sm_count()));
    if (att_smem_bytes(s, (int)sizeof(T), pl) > kAttSmemBudget) pl = att_plan(s, (int)sizeof(T));   // the checked plan
    const size_t smem = att_smem_bytes(s, (int)sizeof(T), pl);
    ensure_smem<attend_kernel<T>>(smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.n_ranks, (unsigned)s.n_heads_kv, (unsigned)s.batch);
    cfg.blockDim = dim3(kAttThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)pl.n_ranks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, attend_kernel<T>, s, pl, a->lengths, a->idx, ck, cv, qt, q, bv, sk,
                                               sv, a->out, status);
    if (err != cudaSuccess) return fail("attend_kernel (cluster launch)", err);
    if (check_launch("attend_kernel") != S4R_OK) return S4R_ERR_CUDA;
  }
  return last_cuda();
}

// ---- prefill bases
struct BasisLayout {
  size_t ctl, rows, inv, M, V, Q, order, sig, Bw, total;
};

s4r_status basis_shape(const s4r_basis_args *a, BasisShape *bs) {
  if (!a) return S4R_ERR_INVALID_ARG;
  if (a->dtype != S4R_F32 && a->dtype != S4R_BF16) return S4R_ERR_INVALID_ARG;
  if (a->n_problems < 0 || a->d_model <= 0 || a->rank <= 0 || a->n_sink < 0 || a->n_sample <= 0 ||
      a->state_rows < 0)
    return S4R_ERR_INVALID_ARG;
  if (a->rank > a->n_sample || a->rank > a->d_model) return S4R_ERR_INVALID_ARG;
  if (a->d_model > S4R_MAX_D_MODEL || a->rank > S4R_MAX_RANK || a->n_sample > S4R_MAX_BASIS_SAMPLE)
    return S4R_ERR_UNSUPPORTED;
  bs->P = a->n_problems;
  bs->D = a->d_model;
  bs->r = a->rank;
  bs->s = a->n_sink;
  bs->T = a->n_sample;
  bs->t_side = a->n_sample <= a->d_model ? 1 : 0;
  const int mm = bs->t_side ? a->n_sample : a->d_model;
  bs->m = (mm + 1) & ~1;
  bs->mp = (mm + 31) & ~31;
  bs->state_rows = a->state_rows;
  return S4R_OK;
}

BasisLayout basis_layout(const BasisShape &bs) {
  BasisLayout l;
  const size_t P = (size_t)bs.P, mp = (size_t)bs.mp;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off += round_up(bytes); return o; };
  l.ctl = take(sizeof(BasisCtl));
  l.rows = take(P * bs.T * sizeof(int64_t));
  l.inv = take(P * bs.T * sizeof(double));
  l.M = take(P * mp * mp * sizeof(double));
  l.V = take(P * mp * mp * sizeof(double));
  l.Q = take(2 * P * (mp / 32) * 32 * 32 * sizeof(double));
  l.order = take(P * bs.r * sizeof(int32_t));
  l.sig = take(P * bs.r * sizeof(double));
  l.Bw = take(P * bs.D * bs.r * sizeof(double));
  l.total = off;
  return l;
}

template <typename T>
s4r_status basis_launch(const s4r_basis_args *a, const BasisShape &bs, const BasisLayout &ly, cudaStream_t st) {
  unsigned char *ws = static_cast<unsigned char *>(a->workspace);
  BasisCtl *ctl = reinterpret_cast<BasisCtl *>(ws + ly.ctl);
  int64_t *rows = reinterpret_cast<int64_t *>(ws + ly.rows);
  double *inv = reinterpret_cast<double *>(ws + ly.inv);
  double *M = reinterpret_cast<double *>(ws + ly.M);
  double *V = reinterpret_cast<double *>(ws + ly.V);
  double *Q = reinterpret_cast<double *>(ws + ly.Q);
  int32_t *order = reinterpret_cast<int32_t *>(ws + ly.order);
  double *sig = reinterpret_cast<double *>(ws + ly.sig);
  double *Bw = reinterpret_cast<double *>(ws + ly.Bw);
  const T *states = static_cast<const T *>(a->states);
  const unsigned P = (unsigned)bs.P;
  basis_prep_kernel<T><<<dim3((unsigned)ceil_div(bs.T, 8), P), 256, 0, st>>>(bs, a->lengths, states, rows, inv, ctl);
  if (check_launch("basis_prep_kernel") != S4R_OK) return S4R_ERR_CUDA;
  const unsigned mt = (unsigned)(bs.mp / 32);
  basis_gram_kernel<T><<<dim3(mt, mt, P), 256, 0, st>>>(bs, states, rows, inv, M, V);
  if (check_launch("basis_gram_kernel") != S4R_OK) return S4R_ERR_CUDA;
  {
    // One cooperative grid for the block Jacobi rounds of every problem.
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, basis_jacobi_kernel, kBjThreads, 0) != cudaSuccess ||
        per_sm < 1)
      return fail("basis_jacobi_kernel occupancy", cudaGetLastError());
    const int64_t npb = bs.mp / 32;
    const int64_t items_a = (int64_t)bs.P * npb;
    const int64_t items_b = (int64_t)bs.P * (npb * (npb - 1) / 2 + npb * ((npb + 1) / 2));
    const int64_t want = items_a > items_b ? items_a : items_b;
    const int64_t cap = (int64_t)per_sm * sm_count();
    const unsigned grid = (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
    BasisShape bsv = bs;
    void *kargs[] = {&bsv, &M, &V, &Q, &ctl};
    const cudaError_t err = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(basis_jacobi_kernel),
                                                        dim3(grid), dim3(kBjThreads), kargs, 0, st);
    if (err != cudaSuccess) return fail("basis_jacobi_kernel (cooperative launch)", err);
  }
  basis_order_kernel<<<P, 1024, 0, st>>>(bs, M, order, sig, a->sigma, ctl);
  if (check_launch("basis_order_kernel") != S4R_OK) return S4R_ERR_CUDA;
  basis_columns_kernel<T><<<dim3((unsigned)ceil_div(bs.r, 32), (unsigned)ceil_div(bs.D, 32), P), 256, 0, st>>>(
      bs, states, rows, inv, V, order, sig, Bw);
  if (check_launch("basis_columns_kernel") != S4R_OK) return S4R_ERR_CUDA;
  basis_output_kernel<T><<<dim3((unsigned)bs.r, P), 256, 0, st>>>(bs, Bw, a->basis_f64,
                                                                   static_cast<T *>(a->basis_out));
  return check_launch("basis_output_kernel");
}

}  // namespace

extern "C" {

size_t s4r_decode_workspace_bytes(const s4r_decode_args *args) {
  Shape s;
  if (make_shape(args, &s) != S4R_OK) return 0;
  return layout_for(s).total;
}

int32_t s4r_decode_kernel_launches(const s4r_decode_args *args) {
  Shape s;
  if (make_shape(args, &s) != S4R_OK) return 0;
  if (s.batch == 0) return 0;
  int32_t n = 1;                                  // projection
  const ScorePlan plan = plan_scoring(s, args->dtype);
  if (plan.rows) n += 3;                          // scoring: pass 1, 1 / l, pass 2
  else if (plan.tc) n += 1;                       // scoring: one tensor-core launch
  else if (s.cache_rows > 0) n += 3;              // scoring: stats, merge, final
  if (s.pool_kernel > 1 && s.cache_rows > 0) n += 1;
  if (s.top_k > 0) n += 1;
  n += 1;                                         // attention (fused combine)
  return n;
}

s4r_status s4r_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
  if (!workspace || workspace_bytes < kAlign || !aligned16(workspace)) return S4R_ERR_INVALID_ARG;
  if (cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return S4R_ERR_CUDA;
  return S4R_OK;
}

s4r_status s4r_decode_step(const s4r_decode_args *a, void *stream) {
  Shape s;
  const s4r_status rc = make_shape(a, &s);
  if (rc != S4R_OK) return rc;
  if (s.batch == 0) return S4R_OK;
  const void *must[] = {a->lengths, a->q, a->coeff_k, a->coeff_v, a->basis_k, a->basis_v, a->out};
  for (const void *p : must)
    if (!p || !aligned16(p)) return S4R_ERR_INVALID_ARG;
  if (s.top_k > 0 && (!a->idx || !aligned16(a->idx))) return S4R_ERR_INVALID_ARG;
  if (s.n_sink > 0 && (!a->sink_k || !a->sink_v || !aligned16(a->sink_k) || !aligned16(a->sink_v)))
    return S4R_ERR_INVALID_ARG;
  if (a->scores && !aligned16(a->scores)) return S4R_ERR_INVALID_ARG;
  const Layout ly = layout_for(s);
  if (!a->workspace || !aligned16(a->workspace) || a->workspace_bytes < ly.total) return S4R_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return a->dtype == S4R_BF16 ? decode_launch<bf16>(a, s, ly, st) : decode_launch<float>(a, s, ly, st);
}

s4r_status s4r_encode(const void *states, int64_t n_tokens, int64_t states_ld, const void *basis,
                      int32_t d_model, int32_t rank, void *coeffs, int64_t coeffs_ld,
                      s4r_dtype dtype, void *stream) {
  if (dtype != S4R_F32 && dtype != S4R_BF16) return S4R_ERR_INVALID_ARG;
  if (n_tokens < 0 || d_model <= 0 || rank <= 0 || states_ld < d_model || coeffs_ld < rank)
    return S4R_ERR_INVALID_ARG;
  if (n_tokens == 0) return S4R_OK;
  if (!states || !basis || !coeffs || !aligned16(states) || !aligned16(basis) || !aligned16(coeffs))
    return S4R_ERR_INVALID_ARG;
  const size_t e = esize(dtype);
  if ((states_ld * e) % 16 || (coeffs_ld * e) % 16 || ((int64_t)rank * e) % 16) return S4R_ERR_INVALID_ARG;
  if (d_model > S4R_MAX_D_MODEL || rank > S4R_MAX_RANK) return S4R_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == S4R_BF16 && rank % 32 == 0)
    return encode_tc_launch(1, &states, n_tokens, states_ld, &basis, d_model, rank, &coeffs, coeffs_ld, st);
  dim3 grid((unsigned)ceil_div(n_tokens, kEncTileM), (unsigned)ceil_div(rank, kEncTileN));
  if (dtype == S4R_BF16)
    encode_simt<bf16><<<grid, 256, 0, st>>>(static_cast<const bf16 *>(states), n_tokens, states_ld,
                                            static_cast<const bf16 *>(basis), d_model, rank,
                                            static_cast<bf16 *>(coeffs), coeffs_ld);
  else
    encode_simt<float><<<grid, 256, 0, st>>>(static_cast<const float *>(states), n_tokens, states_ld,
                                             static_cast<const float *>(basis), d_model, rank,
                                             static_cast<float *>(coeffs), coeffs_ld);
  return last_cuda();
}

s4r_status s4r_encode2(const void *states0, const void *states1, int64_t n_tokens, int64_t states_ld,
                       const void *basis0, const void *basis1, int32_t d_model, int32_t rank,
                       void *coeffs0, void *coeffs1, int64_t coeffs_ld, s4r_dtype dtype, void *stream) {
  if (dtype != S4R_F32 && dtype != S4R_BF16) return S4R_ERR_INVALID_ARG;
  if (n_tokens < 0 || d_model <= 0 || rank <= 0 || states_ld < d_model || coeffs_ld < rank)
    return S4R_ERR_INVALID_ARG;
  if (n_tokens == 0) return S4R_OK;
  const void *st_[2] = {states0, states1}, *bs_[2] = {basis0, basis1};
  void *cs_[2] = {coeffs0, coeffs1};
  for (int p = 0; p < 2; ++p)
    if (!st_[p] || !bs_[p] || !cs_[p] || !aligned16(st_[p]) || !aligned16(bs_[p]) || !aligned16(cs_[p]))
      return S4R_ERR_INVALID_ARG;
  const size_t e = esize(dtype);
  if ((states_ld * e) % 16 || (coeffs_ld * e) % 16 || ((int64_t)rank * e) % 16) return S4R_ERR_INVALID_ARG;
  if (d_model > S4R_MAX_D_MODEL || rank > S4R_MAX_RANK) return S4R_ERR_UNSUPPORTED;
  if (dtype == S4R_BF16 && rank % 32 == 0)
    return encode_tc_launch(2, st_, n_tokens, states_ld, bs_, d_model, rank, cs_, coeffs_ld,
                            static_cast<cudaStream_t>(stream));
  for (int p = 0; p < 2; ++p) {
    const s4r_status rc = s4r_encode(st_[p], n_tokens, states_ld, bs_[p], d_model, rank, cs_[p], coeffs_ld,
                                     dtype, stream);
    if (rc != S4R_OK) return rc;
  }
  return S4R_OK;
}

s4r_status s4r_append(const s4r_append_args *a, void *stream) {
  if (!a) return S4R_ERR_INVALID_ARG;
  if (a->dtype != S4R_F32 && a->dtype != S4R_BF16) return S4R_ERR_INVALID_ARG;
  if (a->batch < 0 || a->d_model <= 0 || a->rank_k <= 0 || a->rank_v <= 0 || a->cache_rows < 0)
    return S4R_ERR_INVALID_ARG;
  if (a->batch == 0) return S4R_OK;
  const void *must[] = {a->state_k, a->state_v, a->basis_k, a->basis_v, a->coeff_k, a->coeff_v, a->lengths};
  for (const void *p : must)
    if (!p || !aligned16(p)) return S4R_ERR_INVALID_ARG;
  if (a->status_workspace && !aligned16(a->status_workspace)) return S4R_ERR_INVALID_ARG;
  if (a->rank_k % 8 || a->rank_v % 8 || a->d_model % 8) return S4R_ERR_UNSUPPORTED;
  if (a->d_model > S4R_MAX_D_MODEL || a->rank_k > S4R_MAX_RANK || a->rank_v > S4R_MAX_RANK)
    return S4R_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *status = static_cast<uint32_t *>(a->status_workspace);
  dim3 grid(a->batch, 2);
  if (a->dtype == S4R_BF16)
    append_kernel<bf16><<<grid, 256, 0, st>>>(
        a->d_model, a->rank_k, a->rank_v, a->cache_rows, static_cast<const bf16 *>(a->state_k),
        static_cast<const bf16 *>(a->state_v), static_cast<const bf16 *>(a->basis_k),
        static_cast<const bf16 *>(a->basis_v), static_cast<bf16 *>(a->coeff_k),
        static_cast<bf16 *>(a->coeff_v), a->lengths, status);
  else
    append_kernel<float><<<grid, 256, 0, st>>>(
        a->d_model, a->rank_k, a->rank_v, a->cache_rows, static_cast<const float *>(a->state_k),
        static_cast<const float *>(a->state_v), static_cast<const float *>(a->basis_k),
        static_cast<const float *>(a->basis_v), static_cast<float *>(a->coeff_k),
        static_cast<float *>(a->coeff_v), a->lengths, status);
  append_bump_lengths<<<(unsigned)ceil_div(a->batch, 256), 256, 0, st>>>(a->batch, a->cache_rows, a->lengths);
  return last_cuda();
}

s4r_status s4r_reconstruct(const void *coeffs, int64_t n_rows_total, const void *basis,
                           int32_t d_model, int32_t rank, const int32_t *rows, int64_t n,
                           float *out, s4r_dtype dtype, void *stream) {
  if (dtype != S4R_F32 && dtype != S4R_BF16) return S4R_ERR_INVALID_ARG;
  if (n < 0 || n_rows_total < 0 || d_model <= 0 || rank <= 0) return S4R_ERR_INVALID_ARG;
  if (n == 0) return S4R_OK;
  if (!coeffs || !basis || !rows || !out || !aligned16(coeffs) || !aligned16(basis) ||
      !aligned16(rows) || !aligned16(out))
    return S4R_ERR_INVALID_ARG;
  if (rank % 8) return S4R_ERR_UNSUPPORTED;
  if (d_model > S4R_MAX_D_MODEL || rank > S4R_MAX_RANK || n > INT32_MAX) return S4R_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid((unsigned)n, (unsigned)ceil_div(d_model, 64));
  if (dtype == S4R_BF16)
    reconstruct_kernel<bf16><<<grid, 256, 0, st>>>(static_cast<const bf16 *>(coeffs), n_rows_total,
                                                   static_cast<const bf16 *>(basis), d_model, rank,
                                                   rows, n, out);
  else
    reconstruct_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(coeffs), n_rows_total,
                                                    static_cast<const float *>(basis), d_model, rank,
                                                    rows, n, out);
  return last_cuda();
}

size_t s4r_basis_workspace_bytes(const s4r_basis_args *args) {
  BasisShape bs;
  if (basis_shape(args, &bs) != S4R_OK) return 0;
  return basis_layout(bs).total;
}

s4r_status s4r_build_basis(const s4r_basis_args *a, void *stream) {
  BasisShape bs;
  const s4r_status rc = basis_shape(a, &bs);
  if (rc != S4R_OK) return rc;
  if (bs.P == 0) return S4R_OK;
  if (!a->lengths || !a->states || !aligned16(a->lengths) || !aligned16(a->states)) return S4R_ERR_INVALID_ARG;
  if (!a->basis_out && !a->basis_f64) return S4R_ERR_INVALID_ARG;
  if ((a->basis_out && !aligned16(a->basis_out)) || (a->basis_f64 && !aligned16(a->basis_f64)) ||
      (a->sigma && !aligned16(a->sigma)))
    return S4R_ERR_INVALID_ARG;
  const BasisLayout ly = basis_layout(bs);
  if (!a->workspace || !aligned16(a->workspace) || a->workspace_bytes < ly.total) return S4R_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return a->dtype == S4R_BF16 ? basis_launch<bf16>(a, bs, ly, st) : basis_launch<float>(a, bs, ly, st);
}

s4r_status s4r_read_device_status(const void *workspace, void *stream) {
  if (workspace && !aligned16(workspace)) return S4R_ERR_INVALID_ARG;
  uint32_t word = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (workspace) {
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return S4R_ERR_CUDA;
  } else if (cudaMemcpyFromSymbolAsync(&word, g_device_status, sizeof(word), 0, cudaMemcpyDeviceToHost, st) !=
             cudaSuccess) {
    return S4R_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return S4R_ERR_CUDA;
  if (word & kDevStatusTimeout) return S4R_ERR_TIMEOUT;
  if (word & kDevStatusCheck) return S4R_ERR_DEVICE;
  return S4R_OK;
}

s4r_status s4r_clear_device_status(void *workspace, void *stream) {
  if (workspace && !aligned16(workspace)) return S4R_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (workspace) {
    if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess) return S4R_ERR_CUDA;
  } else {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) !=
        cudaSuccess)
      return S4R_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return S4R_ERR_CUDA;
  }
  return S4R_OK;
}

s4r_status s4r_debug_waits(int64_t limit_cycles, int32_t unreachable_barrier) {
  const long long limit = limit_cycles > 0 ? (long long)limit_cycles : kWaitCycles;
  const uint32_t unreach = unreachable_barrier ? 1u : 0u;
  cudaError_t err = cudaMemcpyToSymbol(g_wait_limit, &limit, sizeof(limit));
  if (err == cudaSuccess) err = cudaMemcpyToSymbol(g_barrier_unreachable, &unreach, sizeof(unreach));
  return err == cudaSuccess ? S4R_OK : fail("s4r_debug_waits", err);
}

const char *s4r_status_string(s4r_status status) {
  switch (status) {
    case S4R_OK: return "ok";
    case S4R_ERR_INVALID_ARG: return "invalid argument";
    case S4R_ERR_UNSUPPORTED: return "unsupported shape";
    case S4R_ERR_CUDA: return "CUDA error";
    case S4R_ERR_TIMEOUT: return "device wait timed out";
    case S4R_ERR_DEVICE: return "device-side check failed";
    case S4R_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int32_t s4r_version(void) { return 100; }

const char *s4r_last_error(void) { return g_last_error; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without any allocation.
//
// Some callers cannot hand the library a workspace: a host program that
// manages no device memory of its own, or an engine that has given every free
// byte of HBM to its cache pool and must not allocate again while serving.
// For them the decode step can run on a scratch array compiled into the
// library, one per device.  It holds at most S4R_NOALLOC_SCRATCH_BYTES, so
// only shapes whose workspace fits are accepted.  Every call on a device
// shares this one array: two calls that overlap in time (other streams, other
// host threads) overwrite each other's scratch, so callers must order them.
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[S4R_NOALLOC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kNoallocMaxDevices] = {};

// Moves a device-side status the call recorded in the scratch array into the
// library-wide status word of the device, and zeroes the scratch word so the
// next call starts clean.
__global__ void noalloc_fold_status(uint32_t *scratch_status) {
  const uint32_t w = *scratch_status;
  if (w) atomicOr(&g_device_status, w);
  *scratch_status = 0u;
}

// Address of this device's scratch array.  The first call on a device looks
// the symbol up and zeroes the array (synchronously); later calls only read
// the cached pointer.
s4r_status noalloc_scratch(void **out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail("cudaGetDevice", err);
  if (dev < 0 || dev >= kNoallocMaxDevices) {
    snprintf(g_last_error, sizeof(g_last_error), "device ordinal %d beyond the no-alloc table", dev);
    return S4R_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return fail("cudaGetSymbolAddress(no-alloc scratch)", err);
    err = cudaMemset(p, 0, S4R_NOALLOC_SCRATCH_BYTES);
    if (err == cudaSuccess) err = cudaDeviceSynchronize();
    if (err != cudaSuccess) return fail("clearing the no-alloc scratch", err);
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return S4R_OK;
}

}  // namespace

extern "C" s4r_status s4r_decode_step_noalloc(const s4r_decode_args *a, void *stream) {
  Shape s;
  const s4r_status rc = make_shape(a, &s);
  if (rc != S4R_OK) return rc;
  if (s.batch == 0) return S4R_OK;
  const Layout ly = layout_for(s);
  if (ly.total > (size_t)S4R_NOALLOC_SCRATCH_BYTES) {
    snprintf(g_last_error, sizeof(g_last_error),
             "s4r_decode_step_noalloc: these shapes need %zu bytes of scratch, the fixed array holds %zu",
             ly.total, (size_t)S4R_NOALLOC_SCRATCH_BYTES);
    return S4R_ERR_UNSUPPORTED;
  }
  void *scratch = nullptr;
  const s4r_status sr = noalloc_scratch(&scratch);
  if (sr != S4R_OK) return sr;
  s4r_decode_args local = *a;
  local.workspace = scratch;
  local.workspace_bytes = S4R_NOALLOC_SCRATCH_BYTES;
  const s4r_status dr = s4r_decode_step(&local, stream);
  if (dr != S4R_OK) return dr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  noalloc_fold_status<<<1, 1, 0, st>>>(reinterpret_cast<uint32_t *>(static_cast<unsigned char *>(scratch) + ly.status));
  return check_launch("noalloc_fold_status");
}
