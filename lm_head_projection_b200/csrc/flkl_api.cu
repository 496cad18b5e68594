// Host side of the C ABI declared in include/flkl.h: argument validation,
// the pass plan and workspace layout, TMA tensor maps, and the launch
// sequence on the caller's stream.
//
// Launch sequence of one whole call (bf16):
//   k_prepare        N_valid, divisor D, 1/(T D); clears the status word and
//                    the tile counters
//   pass 1 (tc)      z tiles = X W^T in TMEM, fused softmax/KL statistics per
//                    (row, 128-column group); the first chunk's raw logits
//                    kept (fp32, up to a budget)
//   k_combine_split  per-row lse and row loss, gradient coefficients, and the
//                    loss = sum of row losses / D (fixed order)
//   k_grad_cached    pass 2 of chunk 0 from the kept logits: G = (S p - q)/(T D)
//                    -> bf16 staging [BT x Vc], db column partials (a pass-2
//                    GEMM covers the chunk's columns past the budget)
//   per vocabulary chunk c of width Vc, one grouped launch (tc):
//                    dX(c): dX (+)= G_c W[c] (fp32 partial across chunks);
//                    pass 2 of chunk c+1: its z tiles again -> G_{c+1};
//                    dW(c) = G_c^T X (only when dW is asked for)
//   k_db_reduce      db (only when asked for)
// Forward-only and backward-only calls (selective log-probability) run pass
// 1 and the merge, or pass 2 of every chunk by GEMM and the chunk launches.

#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "../../include/flkl.h"
#include "jsd_kernels.cuh"
#include "row_kernels.cuh"
#include "simt_f32.cuh"
#include "tc_gemm.cuh"

namespace flkl {

// Limit of every bounded wait in the library's kernels (flkl_set_wait_limit_ms).
unsigned long long g_wait_limit_ns = 4000ull * 1000000ull;

namespace {

constexpr size_t kStagingBudget = size_t(256) << 20;  // bytes of G staging at most
constexpr size_t kLogitCacheBudget = size_t(256) << 20;  // bytes of the chunk-0 logits cache at most
constexpr long long kPairsPerWave = 74;               // CTA pairs of a 148-SM part
constexpr int kMaxDevices = 64;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

struct Plan {
  bool tc;
  int tile_m, tile_n;
  long long m_tiles, n_tiles;  // pass tiles over [BT] x [V]
  long long n_stat;            // column groups of the pass-1 statistics
  long long Vc, nchunks;
  long long db_groups;
  long long n_counters;  // tile counters of the persistent launches, then combine tickets
  long long comb_rowblocks, comb_splits;  // grid of k_combine_split
  long long zc_cols;     // columns of the first chunk whose logits pass 1 keeps (0: none)
  size_t off_cnt, off_st, off_rows, off_cpart, off_G, off_zc, off_dx, off_db, total;
  size_t g_stride;       // bytes between the two G staging buffers
};

bool make_plan(int64_t BT, int64_t H, int64_t V, int dtype, int compute_dW, int compute_db,
               Plan& p, bool keep_logits = true) {
  (void)compute_dW;
  if (BT < 0 || H < 1 || V < 1) return false;
  if (BT >= (int64_t(1) << 31) || H >= (int64_t(1) << 31) || V >= (int64_t(1) << 31)) return false;
  if (dtype != FLKL_DTYPE_F32 && dtype != FLKL_DTYPE_BF16) return false;
  p.tc = dtype == FLKL_DTYPE_BF16;
  p.tile_m = p.tc ? TC_BM : ST_T;
  p.tile_n = p.tc ? TC_BN : ST_T;
  const size_t elem = p.tc ? 2 : 4;
  p.m_tiles = cdiv(BT, p.tile_m);
  p.n_tiles = cdiv(V, p.tile_n);
  p.n_stat = p.tc ? cdiv(V, TC_EPI_COLS) : p.n_tiles;
  // Chunk width: about V/6 (rounded up to the tile width) and at most the
  // staging budget; never below one tile.  (Measured on the bf16 workloads
  // of H = 4096, V = 128256: 6 chunks 2 – 3 % faster per step than 7 or 8 —
  // fewer launch tails and a wider first chunk, whose logits pass 1 keeps.)
  // On the tensor-core path, when one chunk's pass-2 tiles make only a few
  // waves, the width grows (by at most a half) until they fill whole waves of
  // the CTA pairs of a 148-SM part.
  long long vc = cdiv(cdiv(V, 6), p.tile_n) * p.tile_n;
  if (p.tc && BT > 0) {
    const long long nt0 = vc / p.tile_n;
    if (p.m_tiles * nt0 < 4 * kPairsPerWave) {
      for (long long nt = nt0; nt * 2 <= nt0 * 3; ++nt) {
        if ((p.m_tiles * nt) % kPairsPerWave == 0) {
          vc = nt * p.tile_n;
          break;
        }
      }
    }
  }
  if (BT > 0) {
    long long cap = static_cast<long long>(kStagingBudget / (size_t(BT) * elem));
    cap = (cap / p.tile_n) * p.tile_n;
    vc = std::min(vc, std::max<long long>(cap, p.tile_n));
  }
  vc = std::min(vc, p.n_tiles * p.tile_n);
  p.Vc = vc;
  p.nchunks = cdiv(V, vc);
  p.db_groups = p.tc ? p.m_tiles * (TC_BM / 32) : p.m_tiles;
  size_t off = align256(sizeof(DevCtl));
  // the merge of the statistics: about two blocks per SM of a 148-SM part,
  // at least 16 column groups per split
  p.comb_rowblocks = std::max<long long>(1, cdiv(BT, 32));
  p.comb_splits = std::max<long long>(
      1, std::min<long long>({cdiv(296, p.comb_rowblocks), 16, p.n_stat / 16}));
  p.n_counters = p.nchunks + 2 + p.comb_rowblocks + 1;
  p.off_cnt = off;
  off += align256(size_t(p.n_counters) * 4);
  p.off_st = off;
  off += align256(size_t(5) * p.n_stat * BT * 4);
  p.off_rows = off;
  off += align256(size_t(4) * BT * 4);
  p.off_cpart = off;
  off += align256(size_t(5) * p.comb_splits * BT * 4);
  p.off_G = off;
  // two staging buffers on the tensor-core path: chunk c+1's gradient block
  // is produced while chunk c's is consumed
  p.g_stride = align256(size_t(BT) * vc * elem);
  off += p.g_stride * ((p.tc && p.nchunks > 1) ? 2 : 1);
  // tensor-core path: pass 1 keeps the fp32 logits of the first chunk
  // (32-row blocks), as many of its columns as the budget holds (a multiple
  // of the tile width), so that pass 2 needs no GEMM for them
  const size_t rows32 = size_t(cdiv(BT, 32)) * 32;
  p.zc_cols = 0;
  if (p.tc && BT > 0 && keep_logits)
    p.zc_cols = std::min<long long>(
        vc, static_cast<long long>(kLogitCacheBudget / (rows32 * 4)) / p.tile_n * p.tile_n);
  p.off_zc = off;
  if (p.zc_cols > 0) off += align256(rows32 * size_t(p.zc_cols) * 4);
  p.off_dx = off;
  if (p.nchunks > 1) off += align256(size_t(BT) * H * 4);
  p.off_db = off;
  if (compute_db) off += align256(size_t(p.db_groups) * V * 4);
  p.total = off;
  return true;
}

int g_num_sms[kMaxDevices] = {};
std::mutex g_mu;

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (g_num_sms[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_num_sms[dev] = n > 0 ? n : 148;
  }
  return g_num_sms[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// bf16 2-D tensor map: extents {inner, outer}, row pitch in elements, box
// {64, box_outer}, 128-byte swizzle, zero fill outside the extents.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch,
              uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 3-D "blocked" tensor map over a row-major [outer][inner] matrix whose
// blocked extent is a multiple of 64: dims {64, rows of the other extent,
// blocked extent / 64}, the third dimension stepping 128 bytes.  K-major
// operands block K (box {64, 128, TC_KSUB}); MN-major operands block MN
// (box {64, TC_BK, 2}).  Returns false when the driver refuses the layout.
bool make_blocked_map(CUtensorMap* m, const void* base, uint64_t blocked_extent,
                      uint64_t other_extent, uint64_t pitch, bool mn_major) {
  auto fn = encode_fn();
  if (fn == nullptr || blocked_extent % 64 != 0) return false;
  cuuint64_t dims[3] = {64, other_extent, blocked_extent / 64};
  cuuint64_t strides[2] = {pitch * 2, 128};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(mn_major ? TC_BK : TC_HM),
                       static_cast<cuuint32_t>(mn_major ? 2 : TC_KSUB)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// CTA pairs (clusters of 2) of the GEMM kernel that are resident at once on
// the device, one CTA per SM (a cluster sits inside one GPC), cached per
// device; 0 without a usable device.
int g_tc_pairs[kMaxDevices] = {};

int tc_pairs() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const bool cached = dev >= 0 && dev < kMaxDevices;
  int pairs = cached ? g_tc_pairs[dev] : 0;
  if (pairs == 0) {
    if (cudaFuncSetAttribute(tc_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             TC_SMEM_BYTES) != cudaSuccess)
      return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = TC_SMEM_BYTES;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tc_group_kernel, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();  // clear a failed query; fall back to the SM count
      n = num_sms() / 2;
    }
    pairs = std::max(1, std::min(n, num_sms() / 2));
    if (cached) g_tc_pairs[dev] = pairs;
  }
  return pairs;
}

cudaError_t launch_group(const TcMaps& maps, const TcLaunch& L, cudaStream_t st) {
  const int pairs = tc_pairs();
  if (pairs == 0) return cudaErrorInvalidDevice;
  if (L.total_tiles <= 0) return cudaSuccess;
  // one CTA pair (cluster of 2) per claimed tile, at most the pairs that are
  // resident at once (persistent)
  const int grid = 2 * static_cast<int>(std::min<long long>(L.total_tiles, pairs));
  tc_group_kernel<<<grid, TC_THREADS, TC_SMEM_BYTES, st>>>(maps, L);
  return cudaGetLastError();
}

// One GEMM operand: its tensor map and whether the map is the 3-D blocked
// form (one copy per half-stage) or the plain 2-D form.
struct Operand {
  CUtensorMap map;
  int blocked;
};

// Operand over a row-major [outer][inner] bf16 matrix (pitch in elements),
// K-major (inner = K) or MN-major (inner = M or N).  Uses the blocked 3-D map
// when the inner extent is a multiple of 64, else the 2-D map.
bool make_operand(Operand* o, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch,
                  bool mn_major) {
  if (make_blocked_map(&o->map, base, inner, outer, pitch, mn_major)) {
    o->blocked = 1;
    return true;
  }
  o->blocked = 0;
  return make_map(&o->map, base, inner, outer, pitch, mn_major ? TC_BK : TC_HM);
}

// Appends a problem D[M,N] (K deep) of `kind` to launch L; A and B are its
// operands.  Returns false when L is full.
bool add_problem(TcLaunch& L, TcMaps& maps, int kind, long long M, long long N, long long K,
                 int m_fastest, const Operand& A, const Operand& B, int a_k_off = 0,
                 int b_n_off = 0, int b_k_off = 0) {
  if (L.nprob >= TC_MAX_PROBLEMS) return false;
  TcProblem& P = L.prob[L.nprob];
  P = TcProblem{};
  P.kind = kind;
  P.m_tiles = static_cast<int>(cdiv(M, TC_BM));
  P.n_tiles = static_cast<int>(cdiv(N, TC_BN));
  P.num_kb = static_cast<int>(cdiv(K, TC_BK));
  P.m_fastest = m_fastest;
  P.a_k_off = a_k_off;
  P.b_n_off = b_n_off;
  P.b_k_off = b_k_off;
  P.tile_begin = L.total_tiles;
  P.a_blocked = A.blocked;
  P.b_blocked = B.blocked;
  maps.m[2 * L.nprob] = A.map;
  maps.m[2 * L.nprob + 1] = B.map;
  L.total_tiles += P.m_tiles * P.n_tiles;
  ++L.nprob;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Optional per-launch event recording (flkl_forward_backward_profiled): an
// event before and after every launch, on the launch stream, and the kind of
// each launch.  A null recorder records nothing.
struct Recorder {
  cudaEvent_t* events;  // 2 * capacity events
  int* kinds;           // capacity
  double* flops;        // capacity: GEMM FLOPs of each launch (0 for the others)
  int capacity;
  int count;
  cudaStream_t st;
  void before(int kind, double f) {
    if (count < capacity) {
      kinds[count] = kind;
      flops[count] = f;
      cudaEventRecord(events[2 * count], st);
    }
  }
  void after() {
    if (count < capacity) cudaEventRecord(events[2 * count + 1], st);
    ++count;
  }
};
struct Rec {
  Recorder* r;
  Rec(Recorder* rr, int kind, double flops = 0.0) : r(rr) {
    if (r) r->before(kind, flops);
  }
  ~Rec() {
    if (r) r->after();
  }
};

#define FLKL_CUDA(x)                               \
  do {                                             \
    if ((x) != cudaSuccess) return FLKL_ERR_CUDA;  \
  } while (0)

// Which parts of the path a call runs.  The whole call (forward_backward)
// runs both; the selective log-probability entries run the forward part
// (statistics, per-row log-probabilities into `logp`) and, in a later call on
// the same workspace, the backward part with upstream gradients `dlogp`.
struct Phases {
  bool forward = true;
  bool backward = true;
  float* logp = nullptr;         // forward: per-row output instead of the loss
  const float* dlogp = nullptr;  // backward: per-row upstream gradients
  // data-parallel overlap: event c is recorded on the call's stream once the
  // dW rows of vocabulary chunk c are final (c < n_chunk_events)
  cudaEvent_t* chunk_done = nullptr;
  int n_chunk_events = 0;
  void chunk_finished(long long c, cudaStream_t st) const {
    if (chunk_done != nullptr && c < n_chunk_events) cudaEventRecord(chunk_done[c], st);
  }
};

// Merge of the statistics into row values, then the reduced loss and / or the
// per-row log-probabilities.
cudaError_t finish_rows(const Plan& P, const float* stats, int BT, const int64_t* labels,
                        long long ignore_index, float T, DevCtl* ctl, float* lse2, float* coefS,
                        float* coefQ, float* rowloss, float* loss, float* logp, uint8_t* ws,
                        cudaStream_t st, Recorder* rec) {
  {
    // merge, row values and (with `loss`) the reduced loss in one launch
    Rec r_(rec, 2);
    int* tickets = reinterpret_cast<int*>(ws + P.off_cnt) + (P.nchunks + 2);
    k_combine_split<<<dim3(static_cast<unsigned>(P.comb_rowblocks),
                           static_cast<unsigned>(P.comb_splits)),
                      32 * kCombSplitWarps, 0, st>>>(
        stats, static_cast<int>(P.n_stat), BT, static_cast<int>(P.comb_splits), labels,
        ignore_index, 1.f / T, ctl, reinterpret_cast<float*>(ws + P.off_cpart), tickets, lse2,
        coefS, coefQ, rowloss, loss);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (logp == nullptr) return cudaSuccess;
  Rec r_(rec, 3);
  k_neg_rows<<<static_cast<unsigned>(cdiv(BT, 256)), 256, 0, st>>>(rowloss, BT, logp);
  return cudaGetLastError();
}

// Backward with upstream per-row gradients: replaces the row coefficients.
cudaError_t upstream_coefs(const float* dlogp, const int64_t* target, int BT,
                           long long ignore_index, int V, float T, float* coefS, float* coefQ,
                           cudaStream_t st, Recorder* rec) {
  if (dlogp == nullptr) return cudaSuccess;
  Rec r_(rec, 2);
  k_coef_from_dlogp<<<static_cast<unsigned>(cdiv(BT, 256)), 256, 0, st>>>(
      dlogp, target, BT, ignore_index, V, 1.f / T, coefS, coefQ);
  return cudaGetLastError();
}

flkl_status run_tc(const Plan& P, const __nv_bfloat16* X, const __nv_bfloat16* W,
                   const __nv_bfloat16* b, const __nv_bfloat16* Q, const int64_t* labels,
                   long long ignore_index, int BT, int H, int V, float T, float eps,
                   int compute_dW, int compute_db, int accum_fp32, float* loss,
                   __nv_bfloat16* dX, void* dW, void* db, uint8_t* ws, cudaStream_t st,
                   Recorder* rec, const int64_t* target, const Phases& ph) {
  DevCtl* ctl = reinterpret_cast<DevCtl*>(ws);
  int* counters = reinterpret_cast<int*>(ws + P.off_cnt);
  float* stats = reinterpret_cast<float*>(ws + P.off_st);
  float* rows = reinterpret_cast<float*>(ws + P.off_rows);
  float* lse2 = rows;
  float* coefS = rows + BT;
  float* coefQ = rows + 2 * static_cast<size_t>(BT);
  float* rowloss = rows + 3 * static_cast<size_t>(BT);
  __nv_bfloat16* Gbuf[2] = {reinterpret_cast<__nv_bfloat16*>(ws + P.off_G),
                            reinterpret_cast<__nv_bfloat16*>(ws + P.off_G + P.g_stride)};
  float* dxpart = reinterpret_cast<float*>(ws + P.off_dx);
  float* dbpart = compute_db ? reinterpret_cast<float*>(ws + P.off_db) : nullptr;
  const float LOG2E = 1.4426950408889634f;
  const float t_scale = LOG2E / T;
  const int ldg = static_cast<int>(P.Vc);

  Operand mX_k, mW_k, mX_mn, mW_mn;
  if (!make_operand(&mX_k, X, H, BT, H, false) || !make_operand(&mW_k, W, H, V, H, false) ||
      !make_operand(&mX_mn, X, H, BT, H, true) || !make_operand(&mW_mn, W, H, V, H, true))
    return FLKL_ERR_CUDA;

  auto new_launch = [&](int counter_index) {
    TcLaunch L{};
    L.counter = counters + counter_index;
    L.err_flag = &ctl->err;
    L.wait_limit_ns = g_wait_limit_ns;
    L.stats = EpiStats::Params{Q, b, BT, V, t_scale, eps, stats,
                               static_cast<long long>(P.n_stat) * BT, target, nullptr, 0};
    return L;
  };
  auto chunk_c0 = [&](long long c) { return static_cast<int>(c * P.Vc); };
  auto chunk_w = [&](long long c) {
    return static_cast<int>(std::min<long long>(P.Vc, V - c * P.Vc));
  };
  auto grad_params = [&](long long c) {
    return EpiGrad::Params{Q,       b,    BT,    V,     chunk_c0(c), ldg,   Gbuf[c & 1],
                           t_scale, lse2, coefS, coefQ, dbpart,      target};
  };
  // pass-2 problem of chunk c: logits of the chunk again -> G staging
  auto add_grad = [&](TcLaunch& L, TcMaps& maps, long long c) {
    L.grad = grad_params(c);
    return add_problem(L, maps, KIND_GRAD, BT, chunk_w(c), H, 1, mX_k, mW_k, 0, chunk_c0(c), 0);
  };
  // a whole call keeps the first chunk's logits from pass 1 (when the cache
  // fits); the forward-only and backward-only calls recompute them
  float* zc = reinterpret_cast<float*>(ws + P.off_zc);
  const bool cached = ph.forward && ph.backward && ph.dlogp == nullptr && P.zc_cols > 0;

  if (ph.forward) {
    // pass 1: statistics over all V
    {
      TcLaunch L = new_launch(0);
      TcMaps maps{};
      if (cached) {
        L.stats.zc = zc;
        L.stats.zc_cols = static_cast<int>(P.zc_cols);
      }
      add_problem(L, maps, KIND_STATS, BT, V, H, 1, mX_k, mW_k);
      Rec r_(rec, 1, 2.0 * BT * static_cast<double>(V) * H);
      FLKL_CUDA(launch_group(maps, L, st));
    }
    FLKL_CUDA(finish_rows(P, stats, BT, labels, ignore_index, T, ctl, lse2, coefS, coefQ,
                          rowloss, loss, ph.logp, ws, st, rec));
  }
  if (!ph.backward) return FLKL_OK;
  FLKL_CUDA(upstream_coefs(ph.dlogp, target, BT, ignore_index, V, T, coefS, coefQ, st, rec));
  if (cached) {
    // pass 2 of chunk 0 from the logits cache
    {
      Rec r_(rec, 4);
      const long long warps = cdiv(BT, 32) * (P.zc_cols / 32);
      k_grad_cached<<<static_cast<unsigned>(cdiv(warps, 8)), 256, 0, st>>>(
          grad_params(0), zc, static_cast<int>(P.zc_cols));
      FLKL_CUDA(cudaGetLastError());
    }
    // the chunk's columns past the cache, if any: pass 2 as a GEMM
    const long long rest = chunk_w(0) - P.zc_cols;
    if (rest > 0) {
      TcLaunch L = new_launch(1);
      TcMaps maps{};
      L.grad = grad_params(0);
      L.grad.c0 = static_cast<int>(P.zc_cols);
      L.grad.G = Gbuf[0] + P.zc_cols;
      add_problem(L, maps, KIND_GRAD, BT, rest, H, 1, mX_k, mW_k, 0, static_cast<int>(P.zc_cols),
                  0);
      Rec r_(rec, 4, 2.0 * BT * static_cast<double>(rest) * H);
      FLKL_CUDA(launch_group(maps, L, st));
    }
  } else {
    // pass 2 of chunk 0 alone
    TcLaunch L = new_launch(1);
    TcMaps maps{};
    add_grad(L, maps, 0);
    Rec r_(rec, 4, 2.0 * BT * static_cast<double>(chunk_w(0)) * H);
    FLKL_CUDA(launch_group(maps, L, st));
  }
  // then one launch per chunk c: dX(c) (longest tiles first), pass 2 of
  // chunk c+1 into the other staging buffer, dW(c) (shortest tiles last)
  for (long long c = 0; c < P.nchunks; ++c) {
    const int c0 = chunk_c0(c), Vw = chunk_w(c);
    __nv_bfloat16* G = Gbuf[c & 1];
    Operand mG_k, mG_mn;
    if (!make_operand(&mG_k, G, Vw, BT, ldg, false) || !make_operand(&mG_mn, G, Vw, BT, ldg, true))
      return FLKL_ERR_CUDA;
    TcLaunch L = new_launch(static_cast<int>(2 + c));
    TcMaps maps{};
    const int mode = P.nchunks == 1 ? 0 : (c == 0 ? 1 : (c == P.nchunks - 1 ? 3 : 2));
    L.dx = EpiAccumRows::Params{dxpart, dX, H, BT, H, mode};
    add_problem(L, maps, KIND_DX, BT, H, Vw, 0, mG_k, mW_mn, 0, 0, c0);
    if (c + 1 < P.nchunks) add_grad(L, maps, c + 1);
    if (compute_dW) {
      L.dw = EpiStoreRows::Params{dW, H, Vw, H, c0, accum_fp32};
      // H blocks fastest: consecutive dW tiles share their G block (measured
      // 1.7 % faster on the chunk launches than vocabulary blocks fastest)
      add_problem(L, maps, KIND_DW, Vw, H, BT, 0, mG_mn, mX_mn);
    }
    double f = 2.0 * BT * static_cast<double>(Vw) * H * (1 + (compute_dW ? 1 : 0));
    if (c + 1 < P.nchunks) f += 2.0 * BT * static_cast<double>(chunk_w(c + 1)) * H;
    {
      Rec r_(rec, 9, f);
      FLKL_CUDA(launch_group(maps, L, st));
    }
    ph.chunk_finished(c, st);
  }
  if (compute_db) {
    // the 32-row groups that hold rows (k_grad_cached writes no partials for
    // the all-padding groups of the last row tile; the GEMM epilogues write
    // zeros there)
    Rec r_(rec, 7);
    k_db_reduce<<<static_cast<unsigned>(cdiv(V, 256)), 256, 0, st>>>(
        dbpart, static_cast<int>(cdiv(BT, 32)), V, db, accum_fp32);
    FLKL_CUDA(cudaGetLastError());
  }
  return FLKL_OK;
}

flkl_status run_f32(const Plan& P, const float* X, const float* W, const float* b, const float* Q,
                    const int64_t* labels, long long ignore_index, int BT, int H, int V, float T,
                    float eps, int compute_dW, int compute_db, float* loss, float* dX, float* dW,
                    float* db, uint8_t* ws, cudaStream_t st, Recorder* rec,
                    const int64_t* target, const Phases& ph) {
  DevCtl* ctl = reinterpret_cast<DevCtl*>(ws);
  float* stats = reinterpret_cast<float*>(ws + P.off_st);
  float* rows = reinterpret_cast<float*>(ws + P.off_rows);
  float* lse2 = rows;
  float* coefS = rows + BT;
  float* coefQ = rows + 2 * static_cast<size_t>(BT);
  float* rowloss = rows + 3 * static_cast<size_t>(BT);
  float* G = reinterpret_cast<float*>(ws + P.off_G);
  float* dxpart = reinterpret_cast<float*>(ws + P.off_dx);
  float* dbpart = compute_db ? reinterpret_cast<float*>(ws + P.off_db) : nullptr;
  const float t_scale = 1.4426950408889634f / T;
  const unsigned mt = static_cast<unsigned>(P.m_tiles);

  if (ph.forward) {
    {
      Rec r_(rec, 1, 2.0 * BT * static_cast<double>(V) * H);
      k_simt_stats<<<dim3(static_cast<unsigned>(P.n_tiles), mt), 256, 0, st>>>(
          X, W, b, Q, BT, H, V, t_scale, eps, stats, static_cast<long long>(P.n_tiles) * BT,
          target);
      FLKL_CUDA(cudaGetLastError());
    }
    FLKL_CUDA(finish_rows(P, stats, BT, labels, ignore_index, T, ctl, lse2, coefS, coefQ,
                          rowloss, loss, ph.logp, ws, st, rec));
  }
  if (!ph.backward) return FLKL_OK;
  FLKL_CUDA(upstream_coefs(ph.dlogp, target, BT, ignore_index, V, T, coefS, coefQ, st, rec));

  const int ldg = static_cast<int>(P.Vc);
  for (long long c = 0; c < P.nchunks; ++c) {
    const int c0 = static_cast<int>(c * P.Vc);
    const int Vw = static_cast<int>(std::min<long long>(P.Vc, V - c0));
    {
    Rec r_(rec, 4, 2.0 * BT * static_cast<double>(Vw) * H);
    k_simt_grad<<<dim3(static_cast<unsigned>(cdiv(Vw, ST_T)), mt), 256, 0, st>>>(
        X, W, b, Q, BT, H, V, c0, Vw, t_scale, lse2, coefS, coefQ, G, ldg, dbpart, target);
    FLKL_CUDA(cudaGetLastError());
    }
    if (compute_dW) {
      // dW[c0 + v][h] = sum_r G[r][v] X[r][h]
      Rec r_(rec, 5, 2.0 * BT * static_cast<double>(Vw) * H);
      k_simt_gemm_out<<<dim3(static_cast<unsigned>(cdiv(H, ST_T)),
                             static_cast<unsigned>(cdiv(Vw, ST_T))),
                        256, 0, st>>>(G, 1, ldg, X, 1, H, Vw, H, BT, nullptr, dW, H, c0, 4);
      FLKL_CUDA(cudaGetLastError());
    }
    ph.chunk_finished(c, st);
    const int mode = P.nchunks == 1 ? 0 : (c == 0 ? 1 : (c == P.nchunks - 1 ? 3 : 2));
    // dX[r][h] (+)= sum_v G[r][v] W[c0 + v][h]
    Rec r_(rec, 6, 2.0 * BT * static_cast<double>(Vw) * H);
    k_simt_gemm_out<<<dim3(static_cast<unsigned>(cdiv(H, ST_T)), mt), 256, 0, st>>>(
        G, ldg, 1, W + static_cast<size_t>(c0) * H, 1, H, BT, H, Vw, dxpart, dX, H, 0, mode);
    FLKL_CUDA(cudaGetLastError());
  }
  if (compute_db) {
    Rec r_(rec, 7);
    k_db_reduce<<<static_cast<unsigned>(cdiv(V, 256)), 256, 0, st>>>(
        dbpart, static_cast<int>(P.db_groups), V, db, 1);
    FLKL_CUDA(cudaGetLastError());
  }
  return FLKL_OK;
}

// ------------------------------------------------------------------ JSD
// Fused linear Jensen-Shannon divergence (flkl_jsd_forward_backward): the
// same GEMM kernels, twice per side.  Sequence:
//   statistics passes of the teacher and of the student (log-sum-exps),
//   per vocabulary chunk: both sides' probabilities into staging, then the
//     row sums K = KL(P||M) and l (k_jsd_rows);  loss = sum of kept l / D,
//   per vocabulary chunk again: both sides' probabilities, the gradient block
//     G (k_jsd_grad, written over the student's probabilities, with db column
//     partials), then dX(c) and dW(c).
struct JsdPlan {
  bool tc;
  long long m_tiles, n_tiles, n_stat, Vc, nchunks, db_groups, n_counters;
  size_t off_cnt, off_st, off_rows, off_tgt, off_P, off_Q, off_G, off_dx, off_db, total;
  size_t stage;     // bytes of one staging block (BT x Vc elements)
  size_t off_part;  // tensor-core path: [2][n_stat][BT] fp32 partial sums of the loss sweep
  long long zc_cols;       // tensor-core path: first-chunk logits kept per side (0: none)
  size_t off_zct, off_zcs; // the teacher's and the student's kept logits
};

constexpr int kJsdRows = 10;  // fp32 row arrays in the workspace

bool make_jsd_plan(int64_t BT, int64_t H, int64_t Ht, int64_t V, int dtype, int compute_db,
                   JsdPlan& p) {
  if (BT < 0 || H < 1 || Ht < 1 || V < 1) return false;
  if (BT >= (int64_t(1) << 31) || H >= (int64_t(1) << 31) || Ht >= (int64_t(1) << 31) ||
      V >= (int64_t(1) << 31))
    return false;
  if (dtype != FLKL_DTYPE_F32 && dtype != FLKL_DTYPE_BF16) return false;
  p.tc = dtype == FLKL_DTYPE_BF16;
  const int tile = p.tc ? TC_BN : ST_T;
  const size_t elem = p.tc ? 2 : 4;
  p.m_tiles = cdiv(BT, p.tc ? TC_BM : ST_T);
  p.n_tiles = cdiv(V, tile);
  p.n_stat = p.tc ? cdiv(V, TC_EPI_COLS) : p.n_tiles;
  long long vc = cdiv(cdiv(V, 8), tile) * tile;
  if (BT > 0) {
    long long cap = static_cast<long long>(kStagingBudget / (size_t(BT) * elem));
    cap = (cap / tile) * tile;
    vc = std::min(vc, std::max<long long>(cap, tile));
  }
  vc = std::min(vc, p.n_tiles * tile);
  p.Vc = vc;
  p.nchunks = cdiv(V, vc);
  // db partials per 32-row group: over whole 256-row tiles on the tensor-core path
  p.db_groups = p.tc ? p.m_tiles * (TC_BM / 32) : cdiv(BT, kJsdRowGroup);
  p.n_counters = 2 + 5 * p.nchunks + 2;
  size_t off = align256(sizeof(DevCtl));
  p.off_cnt = off;
  off += align256(size_t(p.n_counters) * 4);
  p.off_st = off;
  off += align256(size_t(5) * p.n_stat * BT * 4);
  p.off_rows = off;
  off += align256(size_t(kJsdRows) * BT * 4);
  p.off_tgt = off;
  off += align256(size_t(BT) * 8);
  const size_t stage = align256(size_t(BT) * vc * elem);
  p.stage = stage;
  if (p.tc) {
    // teacher probabilities of chunks c and c+1 (read by the student pass of
    // chunk c while the teacher pass of chunk c+1 writes; the student pass of
    // the gradient sweep overwrites chunk c's block with its gradient block),
    // and the loss sweep's partial sums
    p.off_Q = off;
    p.off_P = off;
    p.off_G = off;
    off += 2 * stage;
    p.off_part = off;
    off += align256(size_t(2) * p.n_stat * BT * 4);
    // each side's statistics pass keeps the first chunk's logits when the
    // whole chunk fits the budget, so that neither sweep recomputes that
    // chunk's logits
    const size_t zc_bytes = size_t(cdiv(BT, 32)) * 32 * size_t(vc) * 4;
    p.zc_cols = (BT > 0 && zc_bytes <= kLogitCacheBudget) ? vc : 0;
    p.off_zct = off;
    if (p.zc_cols > 0) off += align256(zc_bytes);
    p.off_zcs = off;
    if (p.zc_cols > 0) off += align256(zc_bytes);
  } else {
    p.zc_cols = 0;
    p.off_zct = p.off_zcs = 0;
    // student and teacher probabilities of one chunk; the gradient block
    // overwrites the student's in place
    p.off_P = off;
    p.off_Q = off + stage;
    p.off_G = off;
    p.off_part = 0;
    off += 2 * stage;
  }
  p.off_dx = off;
  if (p.nchunks > 1) off += align256(size_t(BT) * H * 4);
  p.off_db = off;
  if (compute_db) off += align256(size_t(p.db_groups) * V * 4);
  p.total = off;
  return true;
}

struct JsdRows {
  float *lse2_t, *lse2_s, *scrS, *scrQ, *scrL, *K, *L, *rowscale, *ones, *zeros;
};

JsdRows jsd_rows(float* rows, int BT) {
  JsdRows r;
  float** f[kJsdRows] = {&r.lse2_t, &r.lse2_s, &r.scrS, &r.scrQ, &r.scrL,
                         &r.K,      &r.L,      &r.rowscale, &r.ones, &r.zeros};
  for (int i = 0; i < kJsdRows; ++i) *f[i] = rows + static_cast<size_t>(i) * BT;
  return r;
}

cudaError_t jsd_prepare_rows(const JsdRows& R, int64_t* nt, int BT, int V, cudaStream_t st) {
  const unsigned g = static_cast<unsigned>(cdiv(BT, 256));
  // "no target" for the cross-entropy mode of the GEMM epilogues: index V
  k_fill_i64<<<g, 256, 0, st>>>(nt, BT, V);
  k_fill_f32<<<g, 256, 0, st>>>(R.ones, BT, 1.f);
  k_fill_f32<<<g, 256, 0, st>>>(R.zeros, BT, 0.f);
  return cudaGetLastError();
}

flkl_status run_jsd_tc(const JsdPlan& P, const __nv_bfloat16* X, const __nv_bfloat16* W,
                       const __nv_bfloat16* b, const __nv_bfloat16* Xt, const __nv_bfloat16* Wt,
                       const __nv_bfloat16* bt, const int64_t* labels, long long ignore_index,
                       int BT, int H, int Ht, int V, float T, float beta, int compute_dW,
                       int compute_db, int accum_fp32, float* loss, __nv_bfloat16* dX, void* dW,
                       void* db, uint8_t* ws, cudaStream_t st) {
  // Sequence (no probability block of the student ever reaches memory):
  //   statistics passes of the teacher and of the student (log-sum-exps);
  //   loss sweep: teacher probabilities of chunk c+1 into a staging block while
  //     the student pass of chunk c forms p, m and the partial sums of
  //     KL(P||M) and the row loss in its epilogue (reading the staged q);
  //   K and the loss from the partial sums (fixed order);
  //   gradient sweep: the same pairing, the student epilogue writing the
  //     gradient block G of chunk c over the teacher block it reads, then
  //     dX(c) and dW(c) from G.
  DevCtl* ctl = reinterpret_cast<DevCtl*>(ws);
  int* counters = reinterpret_cast<int*>(ws + P.off_cnt);
  float* stats = reinterpret_cast<float*>(ws + P.off_st);
  const JsdRows R = jsd_rows(reinterpret_cast<float*>(ws + P.off_rows), BT);
  int64_t* nt = reinterpret_cast<int64_t*>(ws + P.off_tgt);
  __nv_bfloat16* Qs[2] = {reinterpret_cast<__nv_bfloat16*>(ws + P.off_Q),
                          reinterpret_cast<__nv_bfloat16*>(ws + P.off_Q + P.stage)};
  float* part = reinterpret_cast<float*>(ws + P.off_part);
  float* dxpart = reinterpret_cast<float*>(ws + P.off_dx);
  float* dbpart = compute_db ? reinterpret_cast<float*>(ws + P.off_db) : nullptr;
  const float t_scale = 1.4426950408889634f / T;
  const int ldg = static_cast<int>(P.Vc);
  FLKL_CUDA(jsd_prepare_rows(R, nt, BT, V, st));

  Operand mX_k, mW_k, mX_mn, mW_mn, mXt_k, mWt_k;
  if (!make_operand(&mX_k, X, H, BT, H, false) || !make_operand(&mW_k, W, H, V, H, false) ||
      !make_operand(&mX_mn, X, H, BT, H, true) || !make_operand(&mW_mn, W, H, V, H, true) ||
      !make_operand(&mXt_k, Xt, Ht, BT, Ht, false) || !make_operand(&mWt_k, Wt, Ht, V, Ht, false))
    return FLKL_ERR_CUDA;
  int counter = 0;
  auto new_launch = [&]() {
    TcLaunch L{};
    L.counter = counters + counter++;
    L.err_flag = &ctl->err;
    L.wait_limit_ns = g_wait_limit_ns;
    return L;
  };
  auto chunk_c0 = [&](long long c) { return static_cast<int>(c * P.Vc); };
  auto chunk_w = [&](long long c) {
    return static_cast<int>(std::min<long long>(P.Vc, V - c * P.Vc));
  };
  // the first chunk's logits of each side, kept by its statistics pass
  const bool cached = P.zc_cols > 0;
  float* zct = reinterpret_cast<float*>(ws + P.off_zct);
  float* zcs = reinterpret_cast<float*>(ws + P.off_zcs);
  // log-sum-exp of one side: statistics pass (no teacher) + merge
  auto side_lse = [&](const Operand& mA, const Operand& mB, int Hk, const __nv_bfloat16* bias,
                      float* lse2, float* zc) -> cudaError_t {
    TcLaunch L = new_launch();
    TcMaps maps{};
    L.stats = EpiStats::Params{nullptr, bias, BT, V, t_scale, 0.f, stats,
                               static_cast<long long>(P.n_stat) * BT, nt,
                               cached ? zc : nullptr, static_cast<int>(P.zc_cols)};
    add_problem(L, maps, KIND_STATS, BT, V, Hk, 1, mA, mB);
    cudaError_t e = launch_group(maps, L, st);
    if (e != cudaSuccess) return e;
    k_combine<<<static_cast<unsigned>(cdiv(BT, 32)), 32 * kCombineWarps, 0, st>>>(
        stats, static_cast<int>(P.n_stat), BT, nullptr, ignore_index, 1.f / T, ctl, lse2, R.scrS,
        R.scrQ, R.scrL);
    return cudaGetLastError();
  };
  // teacher probabilities of chunk c into Qs[c & 1] (the pass-2 epilogue with
  // coefficients 1 and 0 and no target)
  auto teacher_params = [&](long long c) {
    return EpiGrad::Params{nullptr, bt,       BT,     V,       chunk_c0(c), ldg, Qs[c & 1],
                           t_scale, R.lse2_t, R.ones, R.zeros, nullptr,     nt};
  };
  auto add_teacher = [&](TcLaunch& L, TcMaps& maps, long long c) {
    L.grad = teacher_params(c);
    add_problem(L, maps, KIND_GRAD, BT, chunk_w(c), Ht, 1, mXt_k, mWt_k, 0, chunk_c0(c), 0);
  };
  // student pass of chunk c, reading Qs[c & 1]
  auto student_params = [&](long long c, int grad) {
    const int c0 = chunk_c0(c);
    EpiJsd::Params j{};
    j.bias = b;
    j.BT = BT;
    j.V = V;
    j.c0 = c0;
    j.ldg = ldg;
    j.Qs = Qs[c & 1];
    j.t_scale = t_scale;
    j.lse2 = R.lse2_s;
    j.beta = beta;
    j.grad = grad;
    j.part = part;
    j.part_plane = static_cast<long long>(P.n_stat) * BT;
    j.G = Qs[c & 1];  // the gradient block replaces the teacher block it is formed from
    j.K = R.K;
    j.rowscale = R.rowscale;
    j.dbpart = grad ? dbpart : nullptr;
    return j;
  };
  auto add_student = [&](TcLaunch& L, TcMaps& maps, long long c, int grad) {
    L.jsd = student_params(c, grad);
    add_problem(L, maps, KIND_JSD, BT, chunk_w(c), H, 1, mX_k, mW_k, 0, chunk_c0(c), 0);
  };
  // the teacher pass of chunk 0 alone, then per chunk c: the student pass of
  // chunk c (longer: with the teacher read) and the teacher pass of chunk c+1
  // (with the kept logits, chunk 0's teacher and student passes are SIMT
  // kernels on them instead of GEMMs)
  const int zcols = static_cast<int>(P.zc_cols);
  auto sweep = [&](int grad) -> flkl_status {
    if (cached) {
      const long long warps = cdiv(BT, 32) * (P.zc_cols / 32);
      k_grad_cached<<<static_cast<unsigned>(cdiv(warps, 8)), 256, 0, st>>>(teacher_params(0),
                                                                          zct, zcols);
      FLKL_CUDA(cudaGetLastError());
    } else {
      TcLaunch L = new_launch();
      TcMaps maps{};
      add_teacher(L, maps, 0);
      FLKL_CUDA(launch_group(maps, L, st));
    }
    for (long long c = 0; c < P.nchunks; ++c) {
      if (c == 0 && cached) {
        const long long warps = cdiv(BT, 32) * (P.zc_cols / TC_EPI_COLS);
        k_jsd_cached<<<static_cast<unsigned>(cdiv(warps, 8)), 256, 0, st>>>(
            student_params(0, grad), zcs, zcols);
        FLKL_CUDA(cudaGetLastError());
        if (P.nchunks > 1) {
          TcLaunch L = new_launch();
          TcMaps maps{};
          add_teacher(L, maps, 1);
          FLKL_CUDA(launch_group(maps, L, st));
        }
      } else {
        TcLaunch L = new_launch();
        TcMaps maps{};
        add_student(L, maps, c, grad);
        if (c + 1 < P.nchunks) add_teacher(L, maps, c + 1);
        FLKL_CUDA(launch_group(maps, L, st));
      }
      if (!grad) continue;
      const int c0 = chunk_c0(c), Vw = chunk_w(c);
      Operand mG_k, mG_mn;
      if (!make_operand(&mG_k, Qs[c & 1], Vw, BT, ldg, false) ||
          !make_operand(&mG_mn, Qs[c & 1], Vw, BT, ldg, true))
        return FLKL_ERR_CUDA;
      TcLaunch L = new_launch();
      TcMaps maps{};
      const int mode = P.nchunks == 1 ? 0 : (c == 0 ? 1 : (c == P.nchunks - 1 ? 3 : 2));
      L.dx = EpiAccumRows::Params{dxpart, dX, H, BT, H, mode};
      add_problem(L, maps, KIND_DX, BT, H, Vw, 0, mG_k, mW_mn, 0, 0, c0);
      if (compute_dW) {
        L.dw = EpiStoreRows::Params{dW, H, Vw, H, c0, accum_fp32};
        add_problem(L, maps, KIND_DW, Vw, H, BT, 1, mG_mn, mX_mn);
      }
      FLKL_CUDA(launch_group(maps, L, st));
    }
    return FLKL_OK;
  };

  FLKL_CUDA(side_lse(mXt_k, mWt_k, Ht, bt, R.lse2_t, zct));
  FLKL_CUDA(side_lse(mX_k, mW_k, H, b, R.lse2_s, zcs));
  k_jsd_init_rows<<<static_cast<unsigned>(cdiv(BT, 256)), 256, 0, st>>>(
      labels, BT, ignore_index, ctl, R.rowscale, R.K, R.L);
  FLKL_CUDA(cudaGetLastError());
  flkl_status s = sweep(0);
  if (s != FLKL_OK) return s;
  k_jsd_sum_parts<<<static_cast<unsigned>(cdiv(BT, 32)), 32 * kJsdSumWarps, 0, st>>>(
      part, static_cast<int>(P.n_stat), BT, R.rowscale, R.K, R.scrL);
  k_loss<<<1, 1024, 0, st>>>(R.scrL, BT, ctl, loss);
  FLKL_CUDA(cudaGetLastError());
  s = sweep(1);
  if (s != FLKL_OK) return s;
  if (compute_db) {
    // the 32-row groups that hold rows (k_jsd_cached writes no partials for
    // the all-padding groups of the last row tile; the GEMM epilogues write
    // zeros there)
    k_db_reduce<<<static_cast<unsigned>(cdiv(V, 256)), 256, 0, st>>>(
        dbpart, static_cast<int>(cdiv(BT, 32)), V, db, accum_fp32);
    FLKL_CUDA(cudaGetLastError());
  }
  return FLKL_OK;
}

flkl_status run_jsd_f32(const JsdPlan& P, const float* X, const float* W, const float* b,
                        const float* Xt, const float* Wt, const float* bt, const int64_t* labels,
                        long long ignore_index, int BT, int H, int Ht, int V, float T, float beta,
                        int compute_dW, int compute_db, float* loss, float* dX, float* dW,
                        float* db, uint8_t* ws, cudaStream_t st) {
  DevCtl* ctl = reinterpret_cast<DevCtl*>(ws);
  float* stats = reinterpret_cast<float*>(ws + P.off_st);
  const JsdRows R = jsd_rows(reinterpret_cast<float*>(ws + P.off_rows), BT);
  int64_t* nt = reinterpret_cast<int64_t*>(ws + P.off_tgt);
  float* Pb = reinterpret_cast<float*>(ws + P.off_P);
  float* Qb = reinterpret_cast<float*>(ws + P.off_Q);
  float* Gb = reinterpret_cast<float*>(ws + P.off_G);
  float* dxpart = reinterpret_cast<float*>(ws + P.off_dx);
  float* dbpart = compute_db ? reinterpret_cast<float*>(ws + P.off_db) : nullptr;
  const float t_scale = 1.4426950408889634f / T;
  const int ldg = static_cast<int>(P.Vc);
  const unsigned mt = static_cast<unsigned>(P.m_tiles);
  FLKL_CUDA(jsd_prepare_rows(R, nt, BT, V, st));
  auto side_lse = [&](const float* A, const float* B, int Hk, const float* bias, float* lse2) {
    k_simt_stats<<<dim3(static_cast<unsigned>(P.n_tiles), mt), 256, 0, st>>>(
        A, B, bias, nullptr, BT, Hk, V, t_scale, 0.f, stats,
        static_cast<long long>(P.n_tiles) * BT, nt);
    k_combine<<<static_cast<unsigned>(cdiv(BT, 32)), 32 * kCombineWarps, 0, st>>>(
        stats, static_cast<int>(P.n_stat), BT, nullptr, ignore_index, 1.f / T, ctl, lse2, R.scrS,
        R.scrQ, R.scrL);
    return cudaGetLastError();
  };
  auto side_probs = [&](const float* A, const float* B, int Hk, const float* bias,
                        const float* lse2, float* out, int c0, int Vw) {
    k_simt_grad<<<dim3(static_cast<unsigned>(cdiv(Vw, ST_T)), mt), 256, 0, st>>>(
        A, B, bias, nullptr, BT, Hk, V, c0, Vw, t_scale, lse2, R.ones, R.zeros, out, ldg,
        nullptr, nt);
    return cudaGetLastError();
  };
  FLKL_CUDA(side_lse(Xt, Wt, Ht, bt, R.lse2_t));
  FLKL_CUDA(side_lse(X, W, H, b, R.lse2_s));
  k_jsd_init_rows<<<static_cast<unsigned>(cdiv(BT, 256)), 256, 0, st>>>(
      labels, BT, ignore_index, ctl, R.rowscale, R.K, R.L);
  FLKL_CUDA(cudaGetLastError());
  for (long long c = 0; c < P.nchunks; ++c) {
    const int c0 = static_cast<int>(c * P.Vc);
    const int Vw = static_cast<int>(std::min<long long>(P.Vc, V - c0));
    FLKL_CUDA(side_probs(Xt, Wt, Ht, bt, R.lse2_t, Qb, c0, Vw));
    FLKL_CUDA(side_probs(X, W, H, b, R.lse2_s, Pb, c0, Vw));
    k_jsd_rows<float><<<static_cast<unsigned>(cdiv(int64_t(BT) * 32, 256)), 256, 0, st>>>(
        Pb, Qb, ldg, BT, Vw, beta, R.K, R.L);
    FLKL_CUDA(cudaGetLastError());
  }
  k_jsd_row_loss<<<static_cast<unsigned>(cdiv(BT, 256)), 256, 0, st>>>(R.L, R.rowscale, BT,
                                                                         R.scrL);
  k_loss<<<1, 1024, 0, st>>>(R.scrL, BT, ctl, loss);
  FLKL_CUDA(cudaGetLastError());
  for (long long c = 0; c < P.nchunks; ++c) {
    const int c0 = static_cast<int>(c * P.Vc);
    const int Vw = static_cast<int>(std::min<long long>(P.Vc, V - c0));
    FLKL_CUDA(side_probs(Xt, Wt, Ht, bt, R.lse2_t, Qb, c0, Vw));
    FLKL_CUDA(side_probs(X, W, H, b, R.lse2_s, Pb, c0, Vw));
    k_jsd_grad<float>
        <<<dim3(static_cast<unsigned>(cdiv(Vw, 256)), static_cast<unsigned>(P.db_groups)), 256,
           0, st>>>(Pb, Qb, ldg, BT, Vw, c0, V, beta, R.K, R.rowscale, Gb, dbpart);
    FLKL_CUDA(cudaGetLastError());
    if (compute_dW) {
      k_simt_gemm_out<<<dim3(static_cast<unsigned>(cdiv(H, ST_T)),
                             static_cast<unsigned>(cdiv(Vw, ST_T))),
                        256, 0, st>>>(Gb, 1, ldg, X, 1, H, Vw, H, BT, nullptr, dW, H, c0, 4);
      FLKL_CUDA(cudaGetLastError());
    }
    const int mode = P.nchunks == 1 ? 0 : (c == 0 ? 1 : (c == P.nchunks - 1 ? 3 : 2));
    k_simt_gemm_out<<<dim3(static_cast<unsigned>(cdiv(H, ST_T)), mt), 256, 0, st>>>(
        Gb, ldg, 1, W + static_cast<size_t>(c0) * H, 1, H, BT, H, Vw, dxpart, dX, H, 0, mode);
    FLKL_CUDA(cudaGetLastError());
  }
  if (compute_db) {
    k_db_reduce<<<static_cast<unsigned>(cdiv(V, 256)), 256, 0, st>>>(
        dbpart, static_cast<int>(P.db_groups), V, db, 1);
    FLKL_CUDA(cudaGetLastError());
  }
  return FLKL_OK;
}

__global__ void k_wait_selftest(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    *status = 0;
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl wc{&abort_flag, status, limit_ns};
    // Nothing arrives on `bar`: the wait must run out and record the status.
    (void)mbar_wait(&bar, 0, wc);
  }
}

}  // namespace
}  // namespace flkl

using namespace flkl;

extern "C" {

int flkl_abi_version(void) { return FLKL_ABI_VERSION; }

size_t flkl_workspace_size(int64_t BT, int64_t H, int64_t V, int dtype, int compute_dW,
                           int compute_db) {
  Plan p;
  if (!make_plan(BT, H, V, dtype, compute_dW, compute_db, p)) return 0;
  return p.total;
}

void flkl_set_wait_limit_ms(unsigned int ms) {
  g_wait_limit_ns = (ms == 0 ? 4000ull : static_cast<unsigned long long>(ms)) * 1000000ull;
}

const char* flkl_status_string(int s) {
  switch (s) {
    case FLKL_OK: return "ok";
    case FLKL_ERR_INVALID_ARG: return "invalid argument";
    case FLKL_ERR_UNSUPPORTED: return "unsupported argument (reduction none, alignment or size)";
    case FLKL_ERR_CUDA: return "CUDA runtime error";
    case FLKL_ERR_TIMEOUT: return "a device-side wait ran out of time";
    case FLKL_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FLKL_ERR_TOO_LARGE: return "sizes need more scratch than the fixed 128 MiB device scratch";
    default: return "unknown status";
  }
}

}  // extern "C"

namespace flkl {
namespace {

flkl_status forward_backward_impl(const void* X, const void* W, const void* b, const void* Q,
                                  const int64_t* shift_labels, int64_t ignore_index, int64_t BT,
                                  int64_t H, int64_t V, int dtype, float temperature, float eps,
                                  int reduction, int compute_dW, int compute_db, int accum_fp32,
                                  float* loss, void* dX, void* dW, void* db, void* workspace,
                                  size_t workspace_bytes, void* stream, Recorder* rec,
                                  const int64_t* target = nullptr,
                                  const int64_t* n_valid_total = nullptr,
                                  const Phases& ph = Phases{}, bool allow_lean = false) {
  // Cross-entropy mode (target set): the teacher is one-hot at target[row],
  // Q is not read and the target doubles as the row mask.
  if (target != nullptr) {
    if (Q != nullptr || shift_labels != nullptr) return FLKL_ERR_INVALID_ARG;
    shift_labels = target;
  }
  // ---- scalar arguments
  if (dtype != FLKL_DTYPE_F32 && dtype != FLKL_DTYPE_BF16) return FLKL_ERR_INVALID_ARG;
  if (reduction == FLKL_REDUCTION_NONE) return FLKL_ERR_UNSUPPORTED;
  if (reduction < FLKL_REDUCTION_BATCHMEAN || reduction > FLKL_REDUCTION_SUM)
    return FLKL_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !(temperature < INFINITY)) return FLKL_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || !(eps < INFINITY)) return FLKL_ERR_INVALID_ARG;
  if (BT < 0 || H < 1 || V < 1) return FLKL_ERR_INVALID_ARG;
  if (BT >= (int64_t(1) << 31) || H >= (int64_t(1) << 31) || V >= (int64_t(1) << 31))
    return FLKL_ERR_UNSUPPORTED;
  const int vec = dtype == FLKL_DTYPE_BF16 ? 8 : 4;
  if (H % vec != 0 || V % vec != 0) return FLKL_ERR_UNSUPPORTED;
  // ---- pointers
  if (W == nullptr) return FLKL_ERR_INVALID_ARG;
  if (ph.forward && loss == nullptr && ph.logp == nullptr) return FLKL_ERR_INVALID_ARG;
  if (BT > 0 && (X == nullptr || (Q == nullptr && target == nullptr))) return FLKL_ERR_INVALID_ARG;
  if (ph.backward) {
    // outputs of the backward part (a forward-only call writes none of them;
    // its flags only size the workspace the backward call will use)
    if (BT > 0 && dX == nullptr) return FLKL_ERR_INVALID_ARG;
    if ((compute_dW != 0) != (dW != nullptr)) return FLKL_ERR_INVALID_ARG;
    if ((compute_db != 0) != (db != nullptr)) return FLKL_ERR_INVALID_ARG;
  }
  if (compute_db && b == nullptr) return FLKL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(b) || !aligned16(Q) || !aligned16(dX) ||
      !aligned16(dW) || !aligned16(db) || (reinterpret_cast<uintptr_t>(shift_labels) & 7u) ||
      (reinterpret_cast<uintptr_t>(loss) & 3u))
    return FLKL_ERR_UNSUPPORTED;
  Plan P;
  if (!make_plan(BT, H, V, dtype, compute_dW, compute_db, P)) return FLKL_ERR_INVALID_ARG;
  // (allow_lean: a workspace that holds all but the first chunk's kept
  // logits runs with that chunk recomputed; the same results)
  if (allow_lean && workspace_bytes < P.total)
    make_plan(BT, H, V, dtype, compute_dW, compute_db, P, false);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < P.total)
    return FLKL_ERR_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int bt = static_cast<int>(BT), h = static_cast<int>(H), v = static_cast<int>(V);

  {
    Rec r_(rec, 0);
    k_prepare<<<1, 1024, 0, st>>>(shift_labels, bt, static_cast<long long>(ignore_index),
                                  reduction, v, temperature, reinterpret_cast<DevCtl*>(ws),
                                  reinterpret_cast<int*>(ws + P.off_cnt),
                                  static_cast<int>(P.n_counters), n_valid_total);
    FLKL_CUDA(cudaGetLastError());
  }

  if (BT == 0) {
    // No rows: loss 0, and zero parameter gradients when asked for.
    Rec r_(rec, 8);
    if (loss != nullptr) k_zero<<<1, 32, 0, st>>>(loss, sizeof(float));
    FLKL_CUDA(cudaGetLastError());
    if (!ph.backward) return FLKL_OK;
    const size_t pe = (dtype == FLKL_DTYPE_F32 || accum_fp32) ? 4 : 2;
    if (compute_dW) {
      const size_t bytes = size_t(V) * H * pe;
      k_zero<<<static_cast<unsigned>(cdiv(bytes, 16 * 256)), 256, 0, st>>>(dW, bytes);
      FLKL_CUDA(cudaGetLastError());
    }
    if (compute_db) {
      const size_t bytes = size_t(V) * pe;
      k_zero<<<static_cast<unsigned>(cdiv(bytes, 16 * 256)), 256, 0, st>>>(db, bytes);
      FLKL_CUDA(cudaGetLastError());
    }
    return FLKL_OK;
  }

  if (P.tc) {
    return run_tc(P, static_cast<const __nv_bfloat16*>(X), static_cast<const __nv_bfloat16*>(W),
                  static_cast<const __nv_bfloat16*>(b), static_cast<const __nv_bfloat16*>(Q),
                  shift_labels, ignore_index, bt, h, v, temperature, eps, compute_dW, compute_db,
                  accum_fp32, loss, static_cast<__nv_bfloat16*>(dX), dW, db, ws, st, rec, target,
                  ph);
  }
  return run_f32(P, static_cast<const float*>(X), static_cast<const float*>(W),
                 static_cast<const float*>(b), static_cast<const float*>(Q), shift_labels,
                 ignore_index, bt, h, v, temperature, eps, compute_dW, compute_db, loss,
                 static_cast<float*>(dX), static_cast<float*>(dW), static_cast<float*>(db), ws,
                 st, rec, target, ph);
}

flkl_status jsd_impl(const void* X, const void* W, const void* b, const void* Xt, const void* Wt,
                     const void* bt, const int64_t* shift_labels, int64_t ignore_index,
                     int64_t BT, int64_t H, int64_t Ht, int64_t V, int dtype, float temperature,
                     float beta, int reduction, int compute_dW, int compute_db, int accum_fp32,
                     float* loss, void* dX, void* dW, void* db, void* workspace,
                     size_t workspace_bytes, void* stream) {
  if (dtype != FLKL_DTYPE_F32 && dtype != FLKL_DTYPE_BF16) return FLKL_ERR_INVALID_ARG;
  if (reduction == FLKL_REDUCTION_NONE) return FLKL_ERR_UNSUPPORTED;
  if (reduction < FLKL_REDUCTION_BATCHMEAN || reduction > FLKL_REDUCTION_SUM)
    return FLKL_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !(temperature < INFINITY)) return FLKL_ERR_INVALID_ARG;
  if (!(beta > 0.f) || !(beta < 1.f)) return FLKL_ERR_INVALID_ARG;
  if (BT < 0 || H < 1 || Ht < 1 || V < 1) return FLKL_ERR_INVALID_ARG;
  if (BT >= (int64_t(1) << 31) || H >= (int64_t(1) << 31) || Ht >= (int64_t(1) << 31) ||
      V >= (int64_t(1) << 31))
    return FLKL_ERR_UNSUPPORTED;
  const int vec = dtype == FLKL_DTYPE_BF16 ? 8 : 4;
  if (H % vec != 0 || Ht % vec != 0 || V % vec != 0) return FLKL_ERR_UNSUPPORTED;
  if (W == nullptr || Wt == nullptr || loss == nullptr) return FLKL_ERR_INVALID_ARG;
  if (BT > 0 && (X == nullptr || Xt == nullptr || dX == nullptr)) return FLKL_ERR_INVALID_ARG;
  if ((compute_dW != 0) != (dW != nullptr)) return FLKL_ERR_INVALID_ARG;
  if ((compute_db != 0) != (db != nullptr)) return FLKL_ERR_INVALID_ARG;
  if (compute_db && b == nullptr) return FLKL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(b) || !aligned16(Xt) || !aligned16(Wt) ||
      !aligned16(bt) || !aligned16(dX) || !aligned16(dW) || !aligned16(db) ||
      (reinterpret_cast<uintptr_t>(shift_labels) & 7u) || (reinterpret_cast<uintptr_t>(loss) & 3u))
    return FLKL_ERR_UNSUPPORTED;
  JsdPlan P;
  if (!make_jsd_plan(BT, H, Ht, V, dtype, compute_db, P)) return FLKL_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < P.total)
    return FLKL_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int bt_ = static_cast<int>(BT), h = static_cast<int>(H), ht = static_cast<int>(Ht),
            v = static_cast<int>(V);
  k_prepare<<<1, 1024, 0, st>>>(shift_labels, bt_, static_cast<long long>(ignore_index),
                                reduction, v, temperature, reinterpret_cast<DevCtl*>(ws),
                                reinterpret_cast<int*>(ws + P.off_cnt),
                                static_cast<int>(P.n_counters), nullptr);
  FLKL_CUDA(cudaGetLastError());
  if (BT == 0) {
    k_zero<<<1, 32, 0, st>>>(loss, sizeof(float));
    const size_t pe = (dtype == FLKL_DTYPE_F32 || accum_fp32) ? 4 : 2;
    if (compute_dW) {
      const size_t bytes = size_t(V) * H * pe;
      k_zero<<<static_cast<unsigned>(cdiv(bytes, 16 * 256)), 256, 0, st>>>(dW, bytes);
    }
    if (compute_db) {
      const size_t bytes = size_t(V) * pe;
      k_zero<<<static_cast<unsigned>(cdiv(bytes, 16 * 256)), 256, 0, st>>>(db, bytes);
    }
    return cudaGetLastError() == cudaSuccess ? FLKL_OK : FLKL_ERR_CUDA;
  }
  if (P.tc)
    return run_jsd_tc(P, static_cast<const __nv_bfloat16*>(X),
                      static_cast<const __nv_bfloat16*>(W), static_cast<const __nv_bfloat16*>(b),
                      static_cast<const __nv_bfloat16*>(Xt),
                      static_cast<const __nv_bfloat16*>(Wt),
                      static_cast<const __nv_bfloat16*>(bt), shift_labels, ignore_index, bt_, h,
                      ht, v, temperature, beta, compute_dW, compute_db, accum_fp32, loss,
                      static_cast<__nv_bfloat16*>(dX), dW, db, ws, st);
  return run_jsd_f32(P, static_cast<const float*>(X), static_cast<const float*>(W),
                     static_cast<const float*>(b), static_cast<const float*>(Xt),
                     static_cast<const float*>(Wt), static_cast<const float*>(bt), shift_labels,
                     ignore_index, bt_, h, ht, v, temperature, beta, compute_dW, compute_db, loss,
                     static_cast<float*>(dX), static_cast<float*>(dW), static_cast<float*>(db),
                     ws, st);
}

// Fixed scratch of flkl_forward_backward_noalloc (see flkl.h): part of the
// library's device image, so it exists on every device that loads the
// library, without any allocation call.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FLKL_NOALLOC_SCRATCH_BYTES];

// Device address of the fixed scratch on the current device.  In host code
// the symbol is only a host-side handle: the address a kernel may use comes
// from cudaGetSymbolAddress.  It is looked up on every call (a host-side
// lookup once the library's device code is loaded on the device), so that a
// device reset, which reloads the device code at a possibly different
// address, never leaves a stale address behind.  The first call on a device
// loads the device code there.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);  // a device must be current
  if (e != cudaSuccess) return e;
  (void)dev;
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  if (p == nullptr) return cudaErrorInvalidSymbol;
  *out = p;
  return cudaSuccess;
}

}  // namespace
}  // namespace flkl

extern "C" {

flkl_status flkl_forward_backward_noalloc(const void* X, const void* W, const void* b,
                                          const void* Q, const int64_t* shift_labels,
                                          int64_t ignore_index, int64_t BT, int64_t H, int64_t V,
                                          int dtype, float temperature, float eps, int reduction,
                                          int compute_dW, int compute_db, int accum_fp32,
                                          float* loss, void* dX, void* dW, void* db,
                                          void* stream) {
  Plan lean;
  if (!make_plan(BT, H, V, dtype, compute_dW, compute_db, lean, false)) {
    // invalid sizes or dtype: let the regular validation name the error
    return forward_backward_impl(X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype,
                                 temperature, eps, reduction, compute_dW, compute_db, accum_fp32,
                                 loss, dX, dW, db, nullptr, 0, stream, nullptr);
  }
  // the scratch holds the regular workspace, or at least the one without
  // the first chunk's kept logits (that chunk is then recomputed)
  if (lean.total > FLKL_NOALLOC_SCRATCH_BYTES) return FLKL_ERR_TOO_LARGE;
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return FLKL_ERR_CUDA;
  return forward_backward_impl(X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype,
                               temperature, eps, reduction, compute_dW, compute_db, accum_fp32,
                               loss, dX, dW, db, scratch, FLKL_NOALLOC_SCRATCH_BYTES, stream,
                               nullptr, nullptr, nullptr, Phases{}, true);
}

flkl_status flkl_forward_backward(const void* X, const void* W, const void* b, const void* Q,
                                  const int64_t* shift_labels, int64_t ignore_index, int64_t BT,
                                  int64_t H, int64_t V, int dtype, float temperature, float eps,
                                  int reduction, int compute_dW, int compute_db, int accum_fp32,
                                  float* loss, void* dX, void* dW, void* db, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return forward_backward_impl(X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype,
                               temperature, eps, reduction, compute_dW, compute_db, accum_fp32,
                               loss, dX, dW, db, workspace, workspace_bytes, stream, nullptr);
}

flkl_status flkl_ce_forward_backward(const void* X, const void* W, const void* b,
                                     const int64_t* target, int64_t ignore_index, int64_t BT,
                                     int64_t H, int64_t V, int dtype, float temperature,
                                     int reduction, int compute_dW, int compute_db, int accum_fp32,
                                     float* loss, void* dX, void* dW, void* db, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (BT > 0 && target == nullptr) return FLKL_ERR_INVALID_ARG;
  return forward_backward_impl(X, W, b, nullptr, nullptr, ignore_index, BT, H, V, dtype,
                               temperature, 0.f, reduction, compute_dW, compute_db, accum_fp32,
                               loss, dX, dW, db, workspace, workspace_bytes, stream, nullptr,
                               BT > 0 ? target : nullptr);
}

flkl_status flkl_scale_cast(const void* src, int src_dtype, void* dst, int dst_dtype,
                            int64_t n, const float* scale, void* stream) {
  const bool ok_dt = (src_dtype == FLKL_DTYPE_F32 || src_dtype == FLKL_DTYPE_BF16) &&
                     (dst_dtype == FLKL_DTYPE_F32 || dst_dtype == FLKL_DTYPE_BF16);
  if (n < 0 || !ok_dt) return FLKL_ERR_INVALID_ARG;
  if (n == 0) return FLKL_OK;
  if (src == nullptr || dst == nullptr) return FLKL_ERR_INVALID_ARG;
  if (src == dst && src_dtype != dst_dtype) return FLKL_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst) || (reinterpret_cast<uintptr_t>(scale) & 3u))
    return FLKL_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long vecs = std::max<long long>(1, n / 8);
  const unsigned grid = static_cast<unsigned>(
      std::min<long long>(cdiv(vecs, 256), static_cast<long long>(num_sms()) * 8));
  const bool sf = src_dtype == FLKL_DTYPE_F32, df = dst_dtype == FLKL_DTYPE_F32;
  if (sf && df)
    k_scale_cast<float, float><<<grid, 256, 0, st>>>(static_cast<const float*>(src),
                                                     static_cast<float*>(dst), n, scale);
  else if (sf)
    k_scale_cast<float, __nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const float*>(src), static_cast<__nv_bfloat16*>(dst), n, scale);
  else if (df)
    k_scale_cast<__nv_bfloat16, float><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(src), static_cast<float*>(dst), n, scale);
  else
    k_scale_cast<__nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(dst), n, scale);
  return cudaGetLastError() == cudaSuccess ? FLKL_OK : FLKL_ERR_CUDA;
}

flkl_status flkl_clock_trace(uint64_t* out, int n_samples, unsigned int interval_ns,
                             void* stream) {
  if (out == nullptr || n_samples < 1 || n_samples > (1 << 24) || interval_ns < 1000u ||
      interval_ns > 100000000u)
    return FLKL_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(out) & 7u) return FLKL_ERR_UNSUPPORTED;
  k_clock_trace<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(out, n_samples, interval_ns);
  return cudaGetLastError() == cudaSuccess ? FLKL_OK : FLKL_ERR_CUDA;
}

flkl_status flkl_count_valid(const int64_t* labels, int64_t BT, int64_t ignore_index,
                             int64_t* count, void* stream) {
  if (count == nullptr || BT < 0) return FLKL_ERR_INVALID_ARG;
  if (BT >= (int64_t(1) << 31)) return FLKL_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(labels) & 7u) || (reinterpret_cast<uintptr_t>(count) & 7u))
    return FLKL_ERR_UNSUPPORTED;
  k_count_valid<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      BT > 0 ? labels : nullptr, static_cast<int>(BT), static_cast<long long>(ignore_index),
      count);
  return cudaGetLastError() == cudaSuccess ? FLKL_OK : FLKL_ERR_CUDA;
}

flkl_status flkl_forward_backward_dp(const void* X, const void* W, const void* b, const void* Q,
                                     const int64_t* shift_labels, int64_t ignore_index,
                                     int64_t BT, int64_t H, int64_t V, int dtype,
                                     float temperature, float eps, int reduction, int compute_dW,
                                     int compute_db, int accum_fp32, float* loss, void* dX,
                                     void* dW, void* db, void* workspace, size_t workspace_bytes,
                                     void* stream, const int64_t* n_valid_total) {
  if (n_valid_total == nullptr || (reinterpret_cast<uintptr_t>(n_valid_total) & 7u))
    return FLKL_ERR_INVALID_ARG;
  return forward_backward_impl(X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype,
                               temperature, eps, reduction, compute_dW, compute_db, accum_fp32,
                               loss, dX, dW, db, workspace, workspace_bytes, stream, nullptr,
                               nullptr, n_valid_total);
}

flkl_status flkl_ce_forward_backward_dp(const void* X, const void* W, const void* b,
                                        const int64_t* target, int64_t ignore_index, int64_t BT,
                                        int64_t H, int64_t V, int dtype, float temperature,
                                        int reduction, int compute_dW, int compute_db,
                                        int accum_fp32, float* loss, void* dX, void* dW, void* db,
                                        void* workspace, size_t workspace_bytes, void* stream,
                                        const int64_t* n_valid_total) {
  if (BT > 0 && target == nullptr) return FLKL_ERR_INVALID_ARG;
  if (n_valid_total == nullptr || (reinterpret_cast<uintptr_t>(n_valid_total) & 7u))
    return FLKL_ERR_INVALID_ARG;
  return forward_backward_impl(X, W, b, nullptr, nullptr, ignore_index, BT, H, V, dtype,
                               temperature, 0.f, reduction, compute_dW, compute_db, accum_fp32,
                               loss, dX, dW, db, workspace, workspace_bytes, stream, nullptr,
                               BT > 0 ? target : nullptr, n_valid_total);
}

int flkl_gemm_ctas(void) { return 2 * tc_pairs(); }

int flkl_vocab_chunks(int64_t BT, int64_t H, int64_t V, int dtype, int compute_dW,
                      int compute_db, int64_t* bounds, int capacity) {
  Plan p;
  if (!make_plan(BT, H, V, dtype, compute_dW, compute_db, p)) return 0;
  if (BT == 0) return 0;  // no launch, no chunk
  if (bounds != nullptr) {
    for (long long c = 0; c <= p.nchunks && c <= capacity; ++c)
      bounds[c] = std::min<long long>(c * p.Vc, V);
  }
  return static_cast<int>(p.nchunks);
}

flkl_status flkl_forward_backward_dp_events(
    const void* X, const void* W, const void* b, const void* Q, const int64_t* shift_labels,
    int64_t ignore_index, int64_t BT, int64_t H, int64_t V, int dtype, float temperature,
    float eps, int reduction, int compute_dW, int compute_db, int accum_fp32, float* loss,
    void* dX, void* dW, void* db, void* workspace, size_t workspace_bytes, void* stream,
    const int64_t* n_valid_total, void** chunk_done, int n_events) {
  if (n_valid_total == nullptr || (reinterpret_cast<uintptr_t>(n_valid_total) & 7u))
    return FLKL_ERR_INVALID_ARG;
  if (n_events < 0 || (n_events > 0 && chunk_done == nullptr)) return FLKL_ERR_INVALID_ARG;
  Phases ph;
  ph.chunk_done = reinterpret_cast<cudaEvent_t*>(chunk_done);
  ph.n_chunk_events = n_events;
  return forward_backward_impl(X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype,
                               temperature, eps, reduction, compute_dW, compute_db, accum_fp32,
                               loss, dX, dW, db, workspace, workspace_bytes, stream, nullptr,
                               nullptr, n_valid_total, ph);
}

flkl_status flkl_ce_forward_backward_dp_events(
    const void* X, const void* W, const void* b, const int64_t* target, int64_t ignore_index,
    int64_t BT, int64_t H, int64_t V, int dtype, float temperature, int reduction,
    int compute_dW, int compute_db, int accum_fp32, float* loss, void* dX, void* dW, void* db,
    void* workspace, size_t workspace_bytes, void* stream, const int64_t* n_valid_total,
    void** chunk_done, int n_events) {
  if (BT > 0 && target == nullptr) return FLKL_ERR_INVALID_ARG;
  if (n_valid_total == nullptr || (reinterpret_cast<uintptr_t>(n_valid_total) & 7u))
    return FLKL_ERR_INVALID_ARG;
  if (n_events < 0 || (n_events > 0 && chunk_done == nullptr)) return FLKL_ERR_INVALID_ARG;
  Phases ph;
  ph.chunk_done = reinterpret_cast<cudaEvent_t*>(chunk_done);
  ph.n_chunk_events = n_events;
  return forward_backward_impl(X, W, b, nullptr, nullptr, ignore_index, BT, H, V, dtype,
                               temperature, 0.f, reduction, compute_dW, compute_db, accum_fp32,
                               loss, dX, dW, db, workspace, workspace_bytes, stream, nullptr,
                               BT > 0 ? target : nullptr, n_valid_total, ph);
}

size_t flkl_jsd_workspace_size(int64_t BT, int64_t H, int64_t Ht, int64_t V, int dtype,
                                int compute_dW, int compute_db) {
  (void)compute_dW;
  JsdPlan p;
  if (!make_jsd_plan(BT, H, Ht, V, dtype, compute_db, p)) return 0;
  return p.total;
}

flkl_status flkl_jsd_forward_backward(const void* X, const void* W, const void* b, const void* Xt,
                                      const void* Wt, const void* bt,
                                      const int64_t* shift_labels, int64_t ignore_index,
                                      int64_t BT, int64_t H, int64_t Ht, int64_t V, int dtype,
                                      float temperature, float beta, int reduction,
                                      int compute_dW, int compute_db, int accum_fp32,
                                      float* loss, void* dX, void* dW, void* db,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  return jsd_impl(X, W, b, Xt, Wt, bt, shift_labels, ignore_index, BT, H, Ht, V, dtype,
                  temperature, beta, reduction, compute_dW, compute_db, accum_fp32, loss, dX, dW,
                  db, workspace, workspace_bytes, stream);
}

flkl_status flkl_selective_logprob_forward(const void* X, const void* W, const void* b,
                                           const int64_t* target, int64_t ignore_index,
                                           int64_t BT, int64_t H, int64_t V, int dtype,
                                           float temperature, int compute_dW, int compute_db,
                                           float* logp, void* workspace, size_t workspace_bytes,
                                           void* stream) {
  if (BT > 0 && (target == nullptr || logp == nullptr)) return FLKL_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(logp) & 3u) return FLKL_ERR_UNSUPPORTED;
  Phases ph;
  ph.backward = false;
  ph.logp = logp;
  return forward_backward_impl(X, W, b, nullptr, nullptr, ignore_index, BT, H, V, dtype,
                               temperature, 0.f, FLKL_REDUCTION_SUM, compute_dW, compute_db, 1,
                               nullptr, nullptr, nullptr, nullptr, workspace, workspace_bytes,
                               stream, nullptr, BT > 0 ? target : nullptr, nullptr, ph);
}

flkl_status flkl_selective_logprob_backward(const void* X, const void* W, const void* b,
                                            const int64_t* target, int64_t ignore_index,
                                            int64_t BT, int64_t H, int64_t V, int dtype,
                                            float temperature, const float* dlogp,
                                            int compute_dW, int compute_db, int accum_fp32,
                                            void* dX, void* dW, void* db, void* workspace,
                                            size_t workspace_bytes, void* stream) {
  if (BT > 0 && (target == nullptr || dlogp == nullptr)) return FLKL_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(dlogp) & 3u) return FLKL_ERR_UNSUPPORTED;
  Phases ph;
  ph.forward = false;
  ph.dlogp = dlogp;
  return forward_backward_impl(X, W, b, nullptr, nullptr, ignore_index, BT, H, V, dtype,
                               temperature, 0.f, FLKL_REDUCTION_SUM, compute_dW, compute_db,
                               accum_fp32, nullptr, dX, dW, db, workspace, workspace_bytes,
                               stream, nullptr, BT > 0 ? target : nullptr, nullptr, ph);
}

flkl_status flkl_forward_backward_profiled(
    const void* X, const void* W, const void* b, const void* Q, const int64_t* shift_labels,
    int64_t ignore_index, int64_t BT, int64_t H, int64_t V, int dtype, float temperature,
    float eps, int reduction, int compute_dW, int compute_db, int accum_fp32, float* loss,
    void* dX, void* dW, void* db, void* workspace, size_t workspace_bytes, void* stream,
    void** events, int* kinds, double* flops, int capacity, int* n_launches,
    const int64_t* ce_target) {
  if (events == nullptr || kinds == nullptr || flops == nullptr || n_launches == nullptr ||
      capacity < 0)
    return FLKL_ERR_INVALID_ARG;
  Recorder r{reinterpret_cast<cudaEvent_t*>(events), kinds, flops, capacity, 0,
             static_cast<cudaStream_t>(stream)};
  if (ce_target != nullptr && BT == 0) ce_target = nullptr;
  if (ce_target == nullptr && Q == nullptr && BT > 0) return FLKL_ERR_INVALID_ARG;
  const flkl_status s = forward_backward_impl(
      X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype, temperature, eps, reduction,
      compute_dW, compute_db, accum_fp32, loss, dX, dW, db, workspace, workspace_bytes, stream, &r,
      ce_target);
  *n_launches = r.count;
  return s;
}

flkl_status flkl_device_status(const void* workspace, void* stream) {
  if (workspace == nullptr) return FLKL_ERR_WORKSPACE;
  int h = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return FLKL_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FLKL_ERR_CUDA;
  return h == 0 ? FLKL_OK : static_cast<flkl_status>(h);
}

flkl_status flkl_wait_selftest(int* status_out, unsigned int limit_ms, void* stream) {
  if (status_out == nullptr) return FLKL_ERR_INVALID_ARG;
  k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      status_out, static_cast<unsigned long long>(limit_ms) * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? FLKL_OK : FLKL_ERR_CUDA;
}

}  // extern "C"
