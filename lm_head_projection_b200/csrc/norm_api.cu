// Host side of the norm-backward entry points declared in include/flkl.h.

#include <algorithm>
#include <mutex>

#include "../../include/flkl.h"
#include "norm_bwd.cuh"

namespace flkl {

extern unsigned long long g_wait_limit_ns;  // flkl_api.cu

namespace {

constexpr int kNormMaxH = 8192;
constexpr int kSmemPerSm = 228 * 1024;  // B200: shared memory per SM
constexpr int kSmemPerCtaReserved = 1024;
constexpr int kMaxCtaSmem = 227 * 1024;
constexpr int kMaxNormDevices = 64;
// With dW / db asked for, each CTA gets at least this many rows (fewer
// partial rows to write and add up).
constexpr int64_t kNormRowsPerCta = 8;

// Status word of the norm kernels (0 or FLKL_ERR_TIMEOUT), read and cleared by
// flkl_norm_device_status.
__device__ int g_norm_status;

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Threads per CTA for a row width (the smallest CTA launch_norm uses).
int norm_threads(int64_t H) { return H <= 4096 ? 128 : 256; }

int sm_count(int dev) {
  static int cache[kMaxNormDevices] = {};
  if (dev < 0 || dev >= kMaxNormDevices) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

int current_device() {
  int d = 0;
  return cudaGetDevice(&d) == cudaSuccess ? d : 0;
}

// Upper bound of the number of CTAs (= partial rows) when dW or db is asked for.
int64_t norm_max_ctas(int64_t rows, int64_t H) {
  return std::min<int64_t>(std::max<int64_t>(1, rows / kNormRowsPerCta),
                           int64_t(sm_count(current_device())) * (2048 / norm_threads(H)));
}

struct NormCfg {
  int stages = 0;
  int ctas_per_sm = 0;
};

// Stages and CTAs per SM of one kernel for one row width: as many CTAs as the
// registers allow, then as many stages (>= min_stages) as their share of
// shared memory holds, fewer CTAs when that many stages do not fit.
template <typename K>
NormCfg pick_config(K kern, int NT, int H, size_t elem, int min_stages) {
  static std::mutex mu;
  struct Entry {
    const void* k;
    int H, dev;
    NormCfg cfg;
  };
  static Entry cache[256];
  static int n_cache = 0;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_cache; ++i)
    if (cache[i].k == reinterpret_cast<const void*>(kern) && cache[i].H == H &&
        cache[i].dev == dev)
      return cache[i].cfg;
  NormCfg c;
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return c;
  const int static_smem = static_cast<int>(fa.sharedSizeBytes);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kMaxCtaSmem - static_smem) != cudaSuccess)
    return c;
  const size_t row = static_cast<size_t>(H) * elem;
  int by_regs = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&by_regs, kern, NT, 3 * row) !=
          cudaSuccess ||
      by_regs < 1)
    return c;
  for (int n = by_regs; n >= 1; --n) {
    const long long budget = kSmemPerSm / n - kSmemPerCtaReserved - static_smem;
    const long long cap = std::min<long long>(budget, kMaxCtaSmem - static_smem);
    const long long st = (cap / static_cast<long long>(row) - 1) / 2;
    if (st >= min_stages) {
      c.stages = static_cast<int>(std::min<long long>(st, kNormMaxStages));
      c.ctas_per_sm = n;
      break;
    }
  }
  if (c.stages >= min_stages) {
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &occ, kern, NT, static_cast<size_t>(row) * (1 + 2 * c.stages)) != cudaSuccess ||
        occ < 1)
      c = NormCfg{};
    else
      c.ctas_per_sm = std::min(c.ctas_per_sm, occ);
  }
  if (n_cache < 256) cache[n_cache++] = Entry{reinterpret_cast<const void*>(kern), H, dev, c};
  return c;
}

template <typename T, int LAYER, int NT, int VPT, int R, bool CW, bool CB>
flkl_status launch_r(NormArgs a, const NormCfg& c, int64_t max_ctas, cudaStream_t st,
                     int* n_ctas) {
  const int64_t grid = std::min<int64_t>({(CW || CB) ? max_ctas : a.rows,
                                          int64_t(sm_count(current_device())) * c.ctas_per_sm,
                                          a.rows});
  a.stages = c.stages;
  *n_ctas = static_cast<int>(grid);
  k_norm_bwd<T, LAYER, NT, VPT, R, CW, CB>
      <<<static_cast<unsigned>(grid), NT, norm_smem_bytes<T>(a.H, c.stages), st>>>(a);
  return cudaGetLastError() == cudaSuccess ? FLKL_OK : FLKL_ERR_CUDA;
}

// R rows per iteration where 2 R stages fit, else one.
template <typename T, int LAYER, int NT, int VPT, int R, bool CW, bool CB>
flkl_status launch_one(const NormArgs& a, int64_t max_ctas, cudaStream_t st, int* n_ctas) {
  const NormCfg c = pick_config(k_norm_bwd<T, LAYER, NT, VPT, R, CW, CB>, NT, a.H, sizeof(T),
                                2 * R);
  if (c.stages >= 2 * R)
    return launch_r<T, LAYER, NT, VPT, R, CW, CB>(a, c, max_ctas, st, n_ctas);
  if constexpr (R > 1) return launch_one<T, LAYER, NT, VPT, 1, CW, CB>(a, max_ctas, st, n_ctas);
  return FLKL_ERR_CUDA;
}

template <typename T, int LAYER, int NT, int VPT, int R>
flkl_status launch_flags(const NormArgs& a, int64_t max_ctas, cudaStream_t st, int* n) {
  if constexpr (LAYER) {
    if (a.part_w && a.part_b)
      return launch_one<T, 1, NT, VPT, R, true, true>(a, max_ctas, st, n);
    if (a.part_b) return launch_one<T, 1, NT, VPT, R, false, true>(a, max_ctas, st, n);
  }
  if (a.part_w) return launch_one<T, LAYER, NT, VPT, R, true, false>(a, max_ctas, st, n);
  return launch_one<T, LAYER, NT, VPT, R, false, false>(a, max_ctas, st, n);
}

// Threads, vectors per thread and rows per iteration by row width.
template <typename T, int LAYER>
flkl_status launch_norm(const NormArgs& a, int64_t max_ctas, cudaStream_t st, int* n) {
  if (a.H <= 2048) return launch_flags<T, LAYER, 128, 2, 1>(a, max_ctas, st, n);
  if (a.H <= 4096) return launch_flags<T, LAYER, 128, 4, 1>(a, max_ctas, st, n);
  return launch_flags<T, LAYER, 256, 4, 1>(a, max_ctas, st, n);
}

int* norm_status_ptr() {
  static int* cache[kMaxNormDevices] = {};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxNormDevices) return nullptr;
  if (cache[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_norm_status) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int*>(p);
  }
  return cache[dev];
}

flkl_status norm_backward(int layer, const void* dY, const void* X, const void* W, int64_t rows,
                          int64_t H, int dtype, float eps, int compute_dW, int compute_db,
                          int accum_fp32, void* dX, void* dW, void* db, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (dtype != FLKL_DTYPE_F32 && dtype != FLKL_DTYPE_BF16) return FLKL_ERR_INVALID_ARG;
  if (rows < 0 || H < 1 || !(eps >= 0.f) || !(eps < INFINITY)) return FLKL_ERR_INVALID_ARG;
  if (H % 8 != 0 || H > kNormMaxH || rows >= (int64_t(1) << 40)) return FLKL_ERR_UNSUPPORTED;
  if (W == nullptr || (rows > 0 && (dY == nullptr || X == nullptr || dX == nullptr)))
    return FLKL_ERR_INVALID_ARG;
  if ((compute_dW != 0) != (dW != nullptr) || (compute_db != 0) != (db != nullptr))
    return FLKL_ERR_INVALID_ARG;
  if (!al16(dY) || !al16(X) || !al16(W) || !al16(dX) || !al16(dW) || !al16(db))
    return FLKL_ERR_UNSUPPORTED;
  const size_t need = flkl_norm_workspace_size(rows, H, compute_dW, compute_db);
  if (need > 0 && (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
                   workspace_bytes < need))
    return FLKL_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t max_ctas = norm_max_ctas(rows, H);
  NormArgs a{};
  a.dY = dY;
  a.X = X;
  a.W = W;
  a.rows = rows;
  a.H = static_cast<int>(H);
  a.eps = eps;
  a.dX = dX;
  a.part_w = compute_dW ? static_cast<float*>(workspace) : nullptr;
  a.part_b = compute_db ? static_cast<float*>(workspace) + (compute_dW ? max_ctas * H : 0)
                        : nullptr;
  a.status = norm_status_ptr();
  a.limit_ns = g_wait_limit_ns;
  if (a.status == nullptr) return FLKL_ERR_CUDA;
  int n_ctas = 0;
  if (rows > 0) {
    const flkl_status s = dtype == FLKL_DTYPE_BF16
        ? (layer ? launch_norm<__nv_bfloat16, 1>(a, max_ctas, st, &n_ctas)
                 : launch_norm<__nv_bfloat16, 0>(a, max_ctas, st, &n_ctas))
        : (layer ? launch_norm<float, 1>(a, max_ctas, st, &n_ctas)
                 : launch_norm<float, 0>(a, max_ctas, st, &n_ctas));
    if (s != FLKL_OK) return s;
  }
  const int out_fp32 = (dtype == FLKL_DTYPE_F32 || accum_fp32) ? 1 : 0;
  const int n_grads = (compute_dW ? 1 : 0) + (compute_db ? 1 : 0);
  if (n_grads > 0) {
    const float* p0 = compute_dW ? a.part_w : a.part_b;
    void* o0 = compute_dW ? dW : db;
    const dim3 grid(static_cast<unsigned>((H + 31) / 32), static_cast<unsigned>(n_grads));
    k_colsum<<<grid, kColsumThreads, 0, st>>>(p0, a.part_b, n_ctas, a.H, o0, db, out_fp32);
    if (cudaGetLastError() != cudaSuccess) return FLKL_ERR_CUDA;
  }
  return FLKL_OK;
}

}  // namespace
}  // namespace flkl

extern "C" {

size_t flkl_norm_workspace_size(int64_t rows, int64_t H, int compute_dW, int compute_db) {
  if (rows < 0 || H < 1 || H > flkl::kNormMaxH) return 0;
  const size_t nb = static_cast<size_t>(flkl::norm_max_ctas(rows, H));
  const size_t n = nb * static_cast<size_t>(H) * 4 * ((compute_dW ? 1 : 0) + (compute_db ? 1 : 0));
  return (n + 255) & ~size_t(255);
}

flkl_status flkl_rms_norm_backward(const void* dY, const void* X, const void* W, int64_t rows,
                                   int64_t H, int dtype, float eps, int compute_dW,
                                   int accum_fp32, void* dX, void* dW, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return flkl::norm_backward(0, dY, X, W, rows, H, dtype, eps, compute_dW, 0, accum_fp32, dX, dW,
                             nullptr, workspace, workspace_bytes, stream);
}

flkl_status flkl_layer_norm_backward(const void* dY, const void* X, const void* W, int64_t rows,
                                     int64_t H, int dtype, float eps, int compute_dW,
                                     int compute_db, int accum_fp32, void* dX, void* dW, void* db,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  return flkl::norm_backward(1, dY, X, W, rows, H, dtype, eps, compute_dW, compute_db,
                             accum_fp32, dX, dW, db, workspace, workspace_bytes, stream);
}

flkl_status flkl_norm_device_status(void* stream) {
  int* p = flkl::norm_status_ptr();
  if (p == nullptr) return FLKL_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int h = 0;
  if (cudaMemcpyAsync(&h, p, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return FLKL_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FLKL_ERR_CUDA;
  if (h != 0 && cudaMemsetAsync(p, 0, sizeof(int), st) != cudaSuccess) return FLKL_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FLKL_ERR_CUDA;
  return h == 0 ? FLKL_OK : static_cast<flkl_status>(h);
}

}  // extern "C"
