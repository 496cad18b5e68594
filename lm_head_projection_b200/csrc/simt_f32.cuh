// fp32 path: the same pass structure as the tensor-core path, with 64x64
// SIMT FMA tiles.  Used for fp32 inputs, where bf16/tf32 tensor-core inputs
// would not meet an fp32 tolerance.
#pragma once

#include "ptx.cuh"

namespace flkl {

constexpr int ST_T = 64;   // tile edge
constexpr int ST_KK = 16;  // K step

// acc[i][j] = sum_k A(m0+ty*4+i, k) * B(k, n0+tx*4+j) with
// A(m, k) = A[m*sam + k*sak] (m < M, k < K) and B(k, n) = B[n*sbn + k*sbk].
__device__ __forceinline__ void simt_tile_mma(const float* __restrict__ A, long long sam,
                                              long long sak, const float* __restrict__ B,
                                              long long sbn, long long sbk, int M, int N, int K,
                                              int m0, int n0, float (&acc)[4][4]) {
  __shared__ float As[ST_KK][ST_T + 4];
  __shared__ float Bs[ST_KK][ST_T + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += ST_KK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = tid + r * 256;  // 0..1023 = 64 x 16
      const int mm = e >> 4, kk = e & 15;
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? A[gm * sam + gk * sak] : 0.f;
      const int gn = n0 + mm;
      Bs[kk][mm] = (gn < N && gk < K) ? B[gn * sbn + gk * sbk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < ST_KK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
}

// Pass 1 (fp32): z tile = X W^T + b over 64 vocabulary columns; per-row
// statistics of the tile in the same form as the tensor-core path.  With
// `target` set, the teacher is one-hot at target[row] (Q unused).
__global__ void __launch_bounds__(256) k_simt_stats(const float* __restrict__ X,
                                                    const float* __restrict__ W,
                                                    const float* __restrict__ bias,
                                                    const float* __restrict__ Q, int BT, int H,
                                                    int V, float t_scale, float eps,
                                                    float* __restrict__ st, long long plane,
                                                    const int64_t* __restrict__ target) {
  __shared__ float Zs[ST_T][ST_T + 1];
  const int mb = blockIdx.y, nb = blockIdx.x;
  const int m0 = mb * ST_T, n0 = nb * ST_T;
  float acc[4][4];
  simt_tile_mma(X, H, 1, W, H, 1, BT, V, H, m0, n0, acc);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) Zs[ty * 4 + i][tx * 4 + j] = acc[i][j];
  __syncthreads();
  if (threadIdx.x < ST_T) {
    const int r = threadIdx.x, row = m0 + r;
    if (row < BT) {
      const float qmin = fmaxf(eps, 1.17549435e-38f);
      float m = -INFINITY, A = 0.f, B2 = 0.f, S = 0.f;
      for (int c = 0; c < ST_T && n0 + c < V; ++c) {
        const float z = Zs[r][c] + (bias ? bias[n0 + c] : 0.f);
        m = fmaxf(m, z * t_scale);
      }
      float s = 0.f;
      for (int c = 0; c < ST_T && n0 + c < V; ++c) {
        const float z = Zs[r][c] + (bias ? bias[n0 + c] : 0.f);
        const float q = target != nullptr ? (target[row] == n0 + c ? 1.f : 0.f)
                                          : Q[static_cast<size_t>(row) * V + n0 + c];
        s += exp2f(z * t_scale - m);
        A = fmaf(q, z, A);
        S += q;
        B2 += (q != 0.f) ? q * log2f(fmaxf(q, qmin)) : 0.f;
      }
      const size_t o = static_cast<size_t>(nb) * BT + row;
      st[o] = m;
      st[o + plane] = s;
      st[o + 2 * plane] = A;
      st[o + 3 * plane] = B2;
      st[o + 4 * plane] = S;
    }
  }
}

// Pass 2 (fp32): G = coefS 2^(t - lse2) - coefQ q on the chunk columns
// [c0, c0 + 64*gridDim.x), stored fp32 in the staging buffer; optional
// column sums of the 64-row tile for db.
__global__ void __launch_bounds__(256) k_simt_grad(const float* __restrict__ X,
                                                   const float* __restrict__ W,
                                                   const float* __restrict__ bias,
                                                   const float* __restrict__ Q, int BT, int H,
                                                   int V, int c0, int Vw, float t_scale,
                                                   const float* __restrict__ lse2,
                                                   const float* __restrict__ coefS,
                                                   const float* __restrict__ coefQ,
                                                   float* __restrict__ G, int ldg,
                                                   float* __restrict__ dbpart,
                                                   const int64_t* __restrict__ target) {
  __shared__ float Gs[ST_T][ST_T + 1];
  const int mb = blockIdx.y, nb = blockIdx.x;
  const int m0 = mb * ST_T, n0 = nb * ST_T;  // n0 chunk-relative
  float acc[4][4];
  simt_tile_mma(X, H, 1, W + static_cast<size_t>(c0) * H, H, 1, BT, Vw, H, m0, n0, acc);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i, row = m0 + r;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = tx * 4 + j, col = n0 + c, gcol = c0 + col;
      float g = 0.f;
      if (row < BT && col < Vw) {
        const float t = (acc[i][j] + (bias ? bias[gcol] : 0.f)) * t_scale;
        const float q = target != nullptr ? (target[row] == gcol ? 1.f : 0.f)
                                          : Q[static_cast<size_t>(row) * V + gcol];
        g = coefS[row] * exp2f(t - lse2[row]) - coefQ[row] * q;
        G[static_cast<size_t>(row) * ldg + col] = g;
      }
      Gs[r][c] = g;
    }
  }
  if (dbpart != nullptr) {
    __syncthreads();
    if (threadIdx.x < ST_T) {
      const int c = threadIdx.x, col = n0 + c;
      if (col < Vw) {
        float sum = 0.f;
        for (int r = 0; r < ST_T; ++r) sum += Gs[r][c];
        dbpart[static_cast<size_t>(mb) * V + c0 + col] = sum;
      }
    }
  }
}

// dX (+)= G_c W_c and dW_c = G_c^T X as one strided SIMT GEMM with the
// accumulate modes of the tensor-core path (0 only, 1 first, 2 middle, 3 last,
// 4 plain store with row offset).
__global__ void __launch_bounds__(256) k_simt_gemm_out(const float* __restrict__ A, long long sam,
                                                       long long sak, const float* __restrict__ B,
                                                       long long sbn, long long sbk, int M, int N,
                                                       int K, float* __restrict__ part,
                                                       float* __restrict__ out, int ld,
                                                       int row_off, int mode) {
  const int mb = blockIdx.y, nb = blockIdx.x;
  const int m0 = mb * ST_T, n0 = nb * ST_T;
  float acc[4][4];
  simt_tile_mma(A, sam, sak, B, sbn, sbk, M, N, K, m0, n0, acc);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + ty * 4 + i;
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= N) continue;
      const size_t o = static_cast<size_t>(r) * ld + c;
      float v = acc[i][j];
      if (mode == 2 || mode == 3) v += part[o];
      if (mode == 1 || mode == 2) part[o] = v;
      else if (mode == 4) out[static_cast<size_t>(row_off + r) * ld + c] = v;
      else out[o] = v;
    }
  }
}

}  // namespace flkl
