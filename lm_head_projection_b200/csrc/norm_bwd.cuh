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
// HBM-bound, so the design is about keeping bytes in flight: a persistent
// CTA owns rows blockIdx.x, blockIdx.x + gridDim.x, ... and streams each row
// of x and dy into a ring of shared-memory stages with 1-D bulk copies, issued
// up to `stages` rows ahead by one thread; W is copied once.  Each thread owns
// 8 columns and reads them from the staged row twice: pass 1 forms the
// four row sums a LayerNorm needs (of x - K, (x - K)^2, g and g * (x - K),
// with the shift K = x[row][0]: the shifted-data form of the variance), one
// block reduction adds them, and pass 2 writes dx.  Two rows (one where two
// stages of four do not fit) share one __syncthreads, whose barrier also
// frees the previous iteration's stages for the next copies.  Reductions run in a fixed order (deterministic).
// With dW / db asked for, each CTA keeps its column sums in registers and
// writes one fp32 partial row; k_colsum adds the partial rows in CTA order.
// The grid then holds at least kNormRowsPerCta rows per CTA, so that the
// partial rows stay few next to the input rows.
#pragma once

#include "ptx.cuh"

namespace flkl {

constexpr int kNormMaxStages = 8;

struct NormArgs {
  const void* dY;
  const void* X;
  const void* W;
  long long rows;
  int H;
  float eps;
  void* dX;
  float* part_w;
  float* part_b;
  int* status;                  // set to FLKL_ERR_TIMEOUT when a wait gives up
  unsigned long long limit_ns;  // per wait
  int stages;                   // 2 .. kNormMaxStages
};

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
  __device__ static float first(const __nv_bfloat16* p) { return __bfloat162float(*p); }
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
  __device__ static float first(const float* p) { return *p; }
};

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// Dynamic shared memory: W row, then `stages` x (x row, dy row); each row is
// H * sizeof(T) bytes, a multiple of 16.
template <typename T>
__host__ __device__ constexpr size_t norm_smem_bytes(int H, int stages) {
  return static_cast<size_t>(H) * sizeof(T) * (1 + 2 * static_cast<size_t>(stages));
}

// LAYER: 0 RMSNorm, 1 LayerNorm.  NT threads, VPT vectors of 8 columns each
// (H <= 8 * NT * VPT; thread t owns columns 8 (v NT + t) .. + 7).  R rows per
// iteration: their sums share one barrier and their passes interleave, at no
// extra register cost for the dW / db sums; stages >= 2 * R.
// CW / CB: accumulate dW / db (frozen ones compile out).
template <typename T, int LAYER, int NT, int VPT, int R, bool CW, bool CB>
__global__ void __launch_bounds__(NT) k_norm_bwd(const NormArgs a) {
  constexpr int NW = NT / 32;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kNormMaxStages];
  __shared__ uint64_t wbar;
  __shared__ float4 red[2][R][NW];
  __shared__ int abort_flag;

  const int H = a.H;
  const uint32_t row_bytes = static_cast<uint32_t>(H) * sizeof(T);
  const T* w_s = reinterpret_cast<const T*>(smem);
  auto x_stage = [&](int s) { return reinterpret_cast<T*>(smem + row_bytes * (1 + 2 * s)); };
  auto dy_stage = [&](int s) { return reinterpret_cast<T*>(smem + row_bytes * (2 + 2 * s)); };
  const int S = a.stages;
  const long long step = gridDim.x;
  const long long n_mine =
      blockIdx.x < a.rows ? (a.rows - 1 - blockIdx.x) / step + 1 : 0;
  const T* X = static_cast<const T*>(a.X);
  const T* dY = static_cast<const T*>(a.dY);
  auto issue = [&](int s, long long k) {
    const size_t off = static_cast<size_t>(blockIdx.x + k * step) * H;
    mbar_arrive_expect_tx(&full[s], 2 * row_bytes);
    bulk_load_1d(x_stage(s), X + off, row_bytes, &full[s]);
    bulk_load_1d(dy_stage(s), dY + off, row_bytes, &full[s]);
  };
  // Rows issued when the barrier of the iteration starting at row k is
  // reached: 0 .. S-1 at first, then the previous iteration's rows + S at
  // each later barrier.
  auto last_issued = [&](long long k) {
    const long long hi = k == 0 ? static_cast<long long>(S) - 1 : k + S - R - 1;
    return hi < n_mine - 1 ? hi : n_mine - 1;
  };
  // On a timed-out wait: let the copies in flight land, then leave; the
  // status word already holds the error.
  auto drain = [&](long long k0) {
    if (threadIdx.x == 0) {
      for (long long k = k0; k <= last_issued(k0); ++k)
        mbar_drain_wait(&full[k % S], static_cast<uint32_t>((k / S) & 1), a.limit_ns);
      mbar_drain_wait(&wbar, 0, a.limit_ns);
    }
  };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    mbar_init(&wbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&wbar, row_bytes);
    bulk_load_1d(const_cast<T*>(w_s), a.W, row_bytes, &wbar);
    for (int s = 0; s < S && s < n_mine; ++s) issue(s, s);
  }
  const WaitCtl wc{&abort_flag, a.status, a.limit_ns};
  const bool w_ok = mbar_wait(&wbar, 0, wc);
  if (__syncthreads_or(!w_ok)) {
    drain(0);
    return;
  }

  const float invH = 1.f / static_cast<float>(H);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  auto col = [&](int v) { return (v * NT + static_cast<int>(threadIdx.x)) * 8; };
  // W stays in registers unless the dW / db sums need them (then it is read
  // from its shared-memory copy at each use)
  constexpr bool kWReg = !(CW || CB);
  float w[kWReg ? VPT : 1][8], accw[CW ? VPT : 1][8], accb[CB ? VPT : 1][8];
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if constexpr (kWReg) w[v][i] = 0.f;
      if constexpr (CW) accw[v][i] = 0.f;
      if constexpr (CB) accb[v][i] = 0.f;
    }
    if constexpr (kWReg)
      if (col(v) < H) Vec8<T>::load(w_s + col(v), w[v]);
  }
  auto get_w = [&](int v, float (&wv)[8]) {
    if constexpr (kWReg) {
#pragma unroll
      for (int i = 0; i < 8; ++i) wv[i] = w[v][i];
    } else {
      Vec8<T>::load(w_s + col(v), wv);
    }
  };

  for (long long k = 0; k < n_mine; k += R) {
    const int buf = static_cast<int>((k / R) & 1);
    bool got = true;
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (k + r < n_mine)
        got = got && mbar_wait(&full[(k + r) % S], static_cast<uint32_t>(((k + r) / S) & 1), wc);
    // pass 1 over the staged rows: the four sums (shift K = x[row][0])
    float K[R];
    float4 p[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int s = static_cast<int>((k + r) % S);
      const bool live = got && k + r < n_mine;
      K[r] = (LAYER && live) ? Vec8<T>::first(x_stage(s)) : 0.f;
      p[r] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        if (!live || col(v) >= H) continue;
        float x[8], dy[8], wv[8];
        Vec8<T>::load(x_stage(s) + col(v), x);
        Vec8<T>::load(dy_stage(s) + col(v), dy);
        get_w(v, wv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float g = dy[i] * wv[i];
          const float xk = x[i] - K[r];
          if (LAYER) {
            p[r].x += xk;
            p[r].z += g;
          }
          p[r].y = fmaf(xk, xk, p[r].y);
          p[r].w = fmaf(g, xk, p[r].w);
        }
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (LAYER) p[r].x += __shfl_xor_sync(0xffffffffu, p[r].x, o);
        p[r].y += __shfl_xor_sync(0xffffffffu, p[r].y, o);
        if (LAYER) p[r].z += __shfl_xor_sync(0xffffffffu, p[r].z, o);
        p[r].w += __shfl_xor_sync(0xffffffffu, p[r].w, o);
      }
    if (lane == 0)
#pragma unroll
      for (int r = 0; r < R; ++r) red[buf][r][warp] = p[r];
    // one barrier per iteration: the partial sums are visible, every thread is
    // done with the previous iteration's stages, a timed-out wait is seen by all
    if (__syncthreads_or(!got)) {
      drain(k);
      return;
    }
    if (threadIdx.x == 0 && k >= R) {
      fence_proxy_async_shared();
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const long long kp = k - R + r;
        if (kp + S < n_mine) issue(static_cast<int>(kp % S), kp + S);
      }
    }
    // every thread adds the NW warp sums in warp order
    float4 t[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      t[r] = red[buf][r][0];
#pragma unroll
      for (int i = 1; i < NW; ++i) t[r] = f4add(t[r], red[buf][r][i]);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (k + r >= n_mine) continue;
      // row statistics: xhat = x * rinv + bx, dx = g * rinv - xhat * c2r - gmr
      float rinv, bx, c2r, gmr;
      if (LAYER) {
        const float d = t[r].x * invH;  // mean(x) - K
        const float var = fmaxf(t[r].y * invH - d * d, 0.f);
        rinv = rsqrtf(var + a.eps);
        const float gm = t[r].z * invH;
        const float c2 = (t[r].w * invH - d * gm) * rinv;  // mean(g * xhat)
        bx = -(K[r] + d) * rinv;
        c2r = c2 * rinv;
        gmr = gm * rinv;
      } else {
        rinv = rsqrtf(t[r].y * invH + a.eps);
        bx = 0.f;
        c2r = t[r].w * invH * rinv * rinv;
        gmr = 0.f;
      }
      // pass 2 over the staged row: dx and the parameter-gradient sums
      const int s = static_cast<int>((k + r) % S);
      T* dxr = static_cast<T*>(a.dX) + static_cast<size_t>(blockIdx.x + (k + r) * step) * H;
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        if (col(v) >= H) continue;
        float x[8], dy[8], wv[8], o[8];
        Vec8<T>::load(x_stage(s) + col(v), x);
        Vec8<T>::load(dy_stage(s) + col(v), dy);
        get_w(v, wv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float xh = fmaf(x[i], rinv, bx);
          o[i] = fmaf(dy[i] * wv[i], rinv, -fmaf(xh, c2r, gmr));
          if constexpr (CW) accw[v][i] = fmaf(dy[i], xh, accw[v][i]);
          if constexpr (CB) accb[v][i] += dy[i];
        }
        Vec8<T>::store(dxr + col(v), o);
      }
    }
  }
  // one partial row per CTA (only for the parameter gradients asked for)
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    if (col(v) >= H) continue;
    if constexpr (CW)
      Vec8<float>::store(a.part_w + static_cast<size_t>(blockIdx.x) * H + col(v), accw[v]);
    if constexpr (CB)
      Vec8<float>::store(a.part_b + static_cast<size_t>(blockIdx.x) * H + col(v), accb[v]);
  }
}

// out_g[c] = sum over CTAs b of part_g[b][c] (fp32 or bf16) for the one or
// two gradients g = blockIdx.y, in a fixed order: 32 columns per block, warp
// w adds partial rows w, w + 32, ... in order, then warp 0 adds the 32 warp
// sums in order.
constexpr int kColsumThreads = 1024;
__global__ void __launch_bounds__(kColsumThreads)
    k_colsum(const float* __restrict__ part0, const float* __restrict__ part1, int nblocks,
             int H, void* out0, void* out1, int out_fp32) {
  constexpr int NWc = kColsumThreads / 32;
  __shared__ float sl[NWc][33];
  const float* part = blockIdx.y ? part1 : part0;
  void* out = blockIdx.y ? out1 : out0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + lane;
  // 16 loads in flight per thread, then added in order (a missing row adds 0)
  constexpr int U = 16;
  float s = 0.f;
  if (c < H) {
    for (int b0 = warp; b0 < nblocks; b0 += U * NWc) {
      float v[U];
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int b = b0 + j * NWc;
        v[j] = b < nblocks ? part[static_cast<size_t>(b) * H + c] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < U; ++j) s += v[j];
    }
  }
  sl[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && c < H) {
    float t = sl[0][lane];
#pragma unroll
    for (int i = 1; i < NWc; ++i) t += sl[i][lane];
    if (out_fp32) static_cast<float*>(out)[c] = t;
    else static_cast<__nv_bfloat16*>(out)[c] = __float2bfloat16_rn(t);
  }
}

}  // namespace flkl
