// Row and column kernels of the fused linear Jensen-Shannon divergence.
//
// With student P = softmax(z/T), teacher Q = softmax(zt/T) and M = beta P +
// (1 - beta) Q, the loss of row r is
//     l_r = beta KL(P_r || M_r) + (1 - beta) KL(Q_r || M_r)
// and its gradient with respect to the student logits is
//     d l_r / d z_rv = beta p_rv (log(p_rv / m_rv) - K_r) / T,  K_r = KL(P_r || M_r).
// The GEMM kernels write the probabilities of one vocabulary chunk of both
// sides into staging buffers (rows of `ldg` elements); these kernels turn
// them into the row sums K and l (first sweep over the chunks) and into the
// gradient block G of the chunk (second sweep).  0 log 0 is taken as 0.
#pragma once

#include "ptx.cuh"
#include "row_kernels.cuh"

namespace flkl {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void store_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// p log(p / m), 0 when p == 0.
__device__ __forceinline__ float xlog_ratio(float p, float m) {
  return p > 0.f ? p * logf(p / m) : 0.f;
}

// out[i] = value for i < n.
__global__ void k_fill_i64(int64_t* __restrict__ out, int n, long long value) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = value;
}
__global__ void k_fill_f32(float* __restrict__ out, int n, float value) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = value;
}

// Row scale of the gradient: 1 / (T D) on kept rows, 0 on dropped rows (and
// K, L zeroed for the first sweep).
__global__ void k_jsd_init_rows(const int64_t* __restrict__ labels, int BT,
                                long long ignore_index, const DevCtl* __restrict__ ctl,
                                float* __restrict__ rowscale, float* __restrict__ K,
                                float* __restrict__ L) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= BT) return;
  const bool keep = labels == nullptr || labels[r] != ignore_index;
  rowscale[r] = keep ? ctl->scale : 0.f;
  K[r] = 0.f;
  L[r] = 0.f;
}

// First sweep, one warp per row: K[r] += sum_v p log(p/m), L[r] += beta
// sum_v p log(p/m) + (1 - beta) sum_v q log(q/m) over the chunk's Vw columns
// (lane-strided, then a fixed-order warp reduction).
template <typename T>
__global__ void __launch_bounds__(256) k_jsd_rows(const T* __restrict__ P, const T* __restrict__ Qt,
                                                  int ldg, int BT, int Vw, float beta,
                                                  float* __restrict__ K, float* __restrict__ L) {
  const int row = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= BT) return;  // warp-uniform
  const T* p = P + static_cast<size_t>(row) * ldg;
  const T* q = Qt + static_cast<size_t>(row) * ldg;
  float kp = 0.f, kq = 0.f;
  for (int v = lane; v < Vw; v += 32) {
    const float pv = to_f32(p[v]), qv = to_f32(q[v]);
    const float m = beta * pv + (1.f - beta) * qv;
    kp += xlog_ratio(pv, m);
    kq += xlog_ratio(qv, m);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    kp += __shfl_xor_sync(0xffffffffu, kp, o);
    kq += __shfl_xor_sync(0xffffffffu, kq, o);
  }
  if (lane == 0) {
    K[row] += kp;
    L[row] += beta * kp + (1.f - beta) * kq;
  }
}

// K_r = sum over the column groups of the loss sweep's partial sums of
// KL(P_r||M_r), and the row's loss (0 on dropped rows), in a fixed order: one
// block of 32 warps per 32 rows, warp w adding groups w, w + 32, ... (loads
// coalesced over the 32 rows), then warp 0 adding the 32 warp sums in warp
// order.
constexpr int kJsdSumWarps = 32;
__global__ void __launch_bounds__(32 * kJsdSumWarps)
    k_jsd_sum_parts(const float* __restrict__ part, int n_groups, int BT,
                    const float* __restrict__ rowscale, float* __restrict__ K,
                    float* __restrict__ rowloss) {
  __shared__ float sk[kJsdSumWarps][33], sl[kJsdSumWarps][33];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int r = blockIdx.x * 32 + lane;
  const size_t plane = static_cast<size_t>(n_groups) * BT;
  float k = 0.f, l = 0.f;
  if (r < BT) {
#pragma unroll 4
    for (int g = w; g < n_groups; g += kJsdSumWarps) {
      k += part[static_cast<size_t>(g) * BT + r];
      l += part[plane + static_cast<size_t>(g) * BT + r];
    }
  }
  sk[w][lane] = k;
  sl[w][lane] = l;
  __syncthreads();
  if (w == 0 && r < BT) {
    float kk = sk[0][lane], ll = sl[0][lane];
    for (int i = 1; i < kJsdSumWarps; ++i) {
      kk += sk[i][lane];
      ll += sl[i][lane];
    }
    K[r] = kk;
    rowloss[r] = rowscale[r] != 0.f ? ll : 0.f;
  }
}

// Row losses of kept rows (dropped rows 0) for the fixed-order reduction.
__global__ void k_jsd_row_loss(const float* __restrict__ L, const float* __restrict__ rowscale,
                               int BT, float* __restrict__ rowloss) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < BT) rowloss[r] = rowscale[r] != 0.f ? L[r] : 0.f;
}

constexpr int kJsdRowGroup = 32;  // rows per db partial

// Second sweep: G[r][v] = rowscale[r] beta p (log(p/m) - K[r]) for the
// chunk's Vw columns; one thread per column and a group of kJsdRowGroup rows
// (blockIdx.y), stores coalesced along the row; with `dbpart`, the group's
// column sums of G (fp32, rows in order) go to dbpart[group][c0 + v].  G may
// be P itself (each element is read before the same thread overwrites it).
template <typename T>
__global__ void __launch_bounds__(256) k_jsd_grad(const T* P, const T* __restrict__ Qt, int ldg,
                                                  int BT, int Vw, int c0, int V, float beta,
                                                  const float* __restrict__ K,
                                                  const float* __restrict__ rowscale, T* G,
                                                  float* __restrict__ dbpart) {
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= Vw) return;
  const int r0 = blockIdx.y * kJsdRowGroup;
  const int r1 = min(BT, r0 + kJsdRowGroup);
  float colsum = 0.f;
  for (int r = r0; r < r1; ++r) {
    const size_t i = static_cast<size_t>(r) * ldg + v;
    const float pv = to_f32(P[i]), qv = to_f32(Qt[i]);
    const float m = beta * pv + (1.f - beta) * qv;
    const float g = pv > 0.f ? rowscale[r] * beta * pv * (logf(pv / m) - K[r]) : 0.f;
    store_elem(G + i, g);
    colsum += g;
  }
  if (dbpart != nullptr) dbpart[static_cast<size_t>(blockIdx.y) * V + c0 + v] = colsum;
}

}  // namespace flkl
