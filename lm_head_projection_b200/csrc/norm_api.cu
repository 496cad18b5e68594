// Host side of the norm-backward entry points declared in include/flkl.h.

#include <algorithm>

#include "../../include/flkl.h"
#include "norm_bwd.cuh"

namespace flkl {
namespace {

constexpr int kNormGrid = 4 * 148;  // blocks; fixed so dW/db sum in a fixed order
constexpr int kNormMaxH = 8 * NB_THREADS * 4;

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int norm_blocks(int64_t rows) {
  return static_cast<int>(std::min<int64_t>(rows, kNormGrid));
}

template <typename T, int LAYER, int VPT>
cudaError_t launch_vpt(const void* dY, const void* X, const void* W, int64_t rows, int H,
                       float eps, void* dX, float* pw, float* pb, cudaStream_t st) {
  const int nb = norm_blocks(rows);
  if (nb == 0) return cudaSuccess;
  auto args = [&](auto kern) {
    kern<<<nb, NB_THREADS, 0, st>>>(static_cast<const T*>(dY), static_cast<const T*>(X),
                                    static_cast<const T*>(W), static_cast<long long>(rows), H,
                                    eps, static_cast<T*>(dX), pw, pb);
  };
  if (pw && pb) args(k_norm_bwd<T, LAYER, VPT, true, true>);
  else if (pw) args(k_norm_bwd<T, LAYER, VPT, true, false>);
  else if (pb) args(k_norm_bwd<T, LAYER, VPT, false, true>);
  else args(k_norm_bwd<T, LAYER, VPT, false, false>);
  return cudaGetLastError();
}

template <typename T, int LAYER>
cudaError_t launch_norm(const void* dY, const void* X, const void* W, int64_t rows, int H,
                        float eps, void* dX, float* pw, float* pb, cudaStream_t st) {
  if (H <= 8 * NB_THREADS) return launch_vpt<T, LAYER, 1>(dY, X, W, rows, H, eps, dX, pw, pb, st);
  if (H <= 16 * NB_THREADS) return launch_vpt<T, LAYER, 2>(dY, X, W, rows, H, eps, dX, pw, pb, st);
  return launch_vpt<T, LAYER, 4>(dY, X, W, rows, H, eps, dX, pw, pb, st);
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
  const int nb = norm_blocks(rows);
  float* pw = compute_dW ? static_cast<float*>(workspace) : nullptr;
  float* pb = compute_db ? static_cast<float*>(workspace) + (compute_dW ? size_t(nb) * H : 0)
                         : nullptr;
  const int h = static_cast<int>(H);
  cudaError_t e;
  if (dtype == FLKL_DTYPE_BF16)
    e = layer ? launch_norm<__nv_bfloat16, 1>(dY, X, W, rows, h, eps, dX, pw, pb, st)
              : launch_norm<__nv_bfloat16, 0>(dY, X, W, rows, h, eps, dX, pw, pb, st);
  else
    e = layer ? launch_norm<float, 1>(dY, X, W, rows, h, eps, dX, pw, pb, st)
              : launch_norm<float, 0>(dY, X, W, rows, h, eps, dX, pw, pb, st);
  if (e != cudaSuccess) return FLKL_ERR_CUDA;
  const int out_fp32 = (dtype == FLKL_DTYPE_F32 || accum_fp32) ? 1 : 0;
  const unsigned cb = static_cast<unsigned>((H + 255) / 256);
  if (compute_dW) {
    k_colsum<<<cb, 256, 0, st>>>(pw, nb, h, dW, out_fp32);
    if (cudaGetLastError() != cudaSuccess) return FLKL_ERR_CUDA;
  }
  if (compute_db) {
    k_colsum<<<cb, 256, 0, st>>>(pb, nb, h, db, out_fp32);
    if (cudaGetLastError() != cudaSuccess) return FLKL_ERR_CUDA;
  }
  return FLKL_OK;
}

}  // namespace
}  // namespace flkl

extern "C" {

size_t flkl_norm_workspace_size(int64_t rows, int64_t H, int compute_dW, int compute_db) {
  if (rows < 0 || H < 1 || H > flkl::kNormMaxH) return 0;
  const size_t nb = static_cast<size_t>(flkl::norm_blocks(rows));
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

}  // extern "C"
