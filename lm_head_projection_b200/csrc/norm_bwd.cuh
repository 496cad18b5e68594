// RMSNorm / LayerNorm backward with frozen-parameter flags (the LoRA
// normalization change: with a frozen weight or bias the parameter gradient
// is neither accumulated nor reduced, and dx is unchanged).
//
//   RMSNorm:   y = w * x / r,  r = sqrt(mean(x^2) + eps)
//              dx = (g - xhat * mean(g * xhat)) / r,  g = dy * w,  xhat = x / r
//   LayerNorm: y = w * (x - mu) / s + b,  s = sqrt(var(x) + eps)
//              dx = (g - mean(g) - xhat * mean(g * xhat)) / s
//   dW = sum over rows of dy * xhat,  db = sum over rows of dy.
//
// HBM-bound: one 256-thread block per row at a time (persistent over rows),
// each thread keeps VPT vectors of 8 elements of dy, x and w in registers,
// so each input is read once; 16-byte loads and stores.  Block reductions
// are deterministic (warp shuffles, then warps in order).  With dW / db asked
// for, every block accumulates its rows' column sums in registers and writes
// one partial row; a second kernel sums the partial rows in block order.
#pragma once

#include "ptx.cuh"

namespace flkl {

constexpr int NB_THREADS = 256;

template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  __device__ static void load(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    unpack8_bf16(u, f);
  }
  __device__ static void store(__nv_bfloat16* p, const float (&f)[8]) {
    uint4 u;
    u.x = pack_bf16x2(f[0], f[1]);
    u.y = pack_bf16x2(f[2], f[3]);
    u.z = pack_bf16x2(f[4], f[5]);
    u.w = pack_bf16x2(f[6], f[7]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <>
struct Vec8<float> {
  __device__ static void load(const float* p, float (&f)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  __device__ static void store(float* p, const float (&f)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
};

// Sum over the block, the same value returned to every thread; fixed order.
template <int NV>
__device__ __forceinline__ void block_sum(float (&v)[NV], float (*red)[NB_THREADS / 32]) {
#pragma unroll
  for (int k = 0; k < NV; ++k)
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v[k] += __shfl_xor_sync(0xffffffffu, v[k], o);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red[] may still be read from the previous reduction
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < NV; ++k) red[k][w] = v[k];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NB_THREADS / 32; ++i) s += red[k][i];
    v[k] = s;
  }
}

// LAYER: 0 RMSNorm, 1 LayerNorm.  VPT: vectors of 8 per thread (H <= 2048 VPT).
// CW / CB: accumulate dW / db partials (frozen parameters compile them out).
template <typename T, int LAYER, int VPT, bool CW, bool CB>
__global__ void __launch_bounds__(NB_THREADS)
    k_norm_bwd(const T* __restrict__ dY, const T* __restrict__ X, const T* __restrict__ W,
               long long rows, int H, float eps, T* __restrict__ dX, float* __restrict__ part_w,
               float* __restrict__ part_b) {
  __shared__ float red[2][NB_THREADS / 32];
  const float invH = 1.f / static_cast<float>(H);
  float w[VPT][8];
  float accw[CW ? VPT : 1][8], accb[CB ? VPT : 1][8];
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int c = (v * NB_THREADS + threadIdx.x) * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) w[v][i] = 0.f;
    if (c < H) Vec8<T>::load(W + c, w[v]);
  }
#pragma unroll
  for (int v = 0; v < (CW ? VPT : 1); ++v)
#pragma unroll
    for (int i = 0; i < 8; ++i) accw[v][i] = 0.f;
#pragma unroll
  for (int v = 0; v < (CB ? VPT : 1); ++v)
#pragma unroll
    for (int i = 0; i < 8; ++i) accb[v][i] = 0.f;

  for (long long r = blockIdx.x; r < rows; r += gridDim.x) {
    const T* xr = X + static_cast<size_t>(r) * H;
    const T* dyr = dY + static_cast<size_t>(r) * H;
    float x[VPT][8], dy[VPT][8];
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int c = (v * NB_THREADS + threadIdx.x) * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) x[v][i] = dy[v][i] = 0.f;
      if (c < H) {
        Vec8<T>::load(xr + c, x[v]);
        Vec8<T>::load(dyr + c, dy[v]);
      }
    }
    // row statistics (two passes over the registers: mean, then spread)
    float mu = 0.f;
    if (LAYER) {
      float s1[1] = {0.f};
#pragma unroll
      for (int v = 0; v < VPT; ++v)
#pragma unroll
        for (int i = 0; i < 8; ++i) s1[0] += x[v][i];
      block_sum<1>(s1, red);
      mu = s1[0] * invH;
    }
    float s2[1] = {0.f};
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int c = (v * NB_THREADS + threadIdx.x) * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        x[v][i] = (c < H) ? x[v][i] - mu : 0.f;
        s2[0] += x[v][i] * x[v][i];
      }
    }
    block_sum<1>(s2, red);
    const float rinv = rsqrtf(s2[0] * invH + eps);
    // xhat in place; sums of g = dy * w and of g * xhat
    float s3[2] = {0.f, 0.f};
#pragma unroll
    for (int v = 0; v < VPT; ++v)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        x[v][i] *= rinv;
        const float g = dy[v][i] * w[v][i];
        s3[0] += g;
        s3[1] += g * x[v][i];
      }
    block_sum<2>(s3, red);
    const float gm = LAYER ? s3[0] * invH : 0.f;
    const float c2 = s3[1] * invH;
    T* dxr = dX + static_cast<size_t>(r) * H;
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int c = (v * NB_THREADS + threadIdx.x) * 8;
      if (c >= H) continue;
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = (dy[v][i] * w[v][i] - gm - x[v][i] * c2) * rinv;
      Vec8<T>::store(dxr + c, o);
      if constexpr (CW) {
#pragma unroll
        for (int i = 0; i < 8; ++i) accw[v][i] = fmaf(dy[v][i], x[v][i], accw[v][i]);
      }
      if constexpr (CB) {
#pragma unroll
        for (int i = 0; i < 8; ++i) accb[v][i] += dy[v][i];
      }
    }
  }
  // one partial row per block (only for the parameter gradients asked for)
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int c = (v * NB_THREADS + threadIdx.x) * 8;
    if (c >= H) continue;
    if constexpr (CW)
      Vec8<float>::store(part_w + static_cast<size_t>(blockIdx.x) * H + c, accw[v]);
    if constexpr (CB)
      Vec8<float>::store(part_b + static_cast<size_t>(blockIdx.x) * H + c, accb[v]);
  }
}

// out[c] = sum over blocks b (in order) of part[b][c], fp32 or bf16.
__global__ void k_colsum(const float* __restrict__ part, int nblocks, int H, void* out,
                         int out_fp32) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= H) return;
  float s = 0.f;
  for (int b = 0; b < nblocks; ++b) s += part[static_cast<size_t>(b) * H + c];
  if (out_fp32) static_cast<float*>(out)[c] = s;
  else static_cast<__nv_bfloat16*>(out)[c] = __float2bfloat16_rn(s);
}

}  // namespace flkl
