// Small SIMT kernels around the GEMMs: valid-row count and divisor, merge of
// the per-tile softmax/KL statistics into per-row log-sum-exp and row loss,
// the deterministic loss sum, and the db column reduction.
#pragma once

#include "ptx.cuh"

namespace flkl {

// Device-side control block at the start of the workspace.
struct DevCtl {
  int err;       // first device error code of the call (0 = none)
  int n_valid;   // rows of this call whose shift label differs from ignore_index
  float D;       // reduction divisor
  float scale;   // 1 / (T * D), 0 when no row is kept
  float invD;    // 1 / D, 0 when no row is kept
};

// One block of 1024 threads.  Counts kept rows (a row is dropped when its
// shift label equals ignore_index), derives the divisor of the reduction
// (batchmean: N_valid, mean: N_valid * V, sum: 1), resets the error flag and
// zeroes the tile counters of the call's persistent launches.  With
// `n_total` (data-parallel use) the divisor counts *n_total kept rows, the
// kept rows of every rank's batch, instead of this call's.
__global__ void __launch_bounds__(1024) k_prepare(const int64_t* __restrict__ labels, int BT,
                                                  long long ignore_index, int reduction, int V,
                                                  float temperature, DevCtl* ctl,
                                                  int* counters, int n_counters,
                                                  const int64_t* __restrict__ n_total) {
  __shared__ int warp_cnt[32];
  for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0;
  int cnt = 0;
  if (labels == nullptr) {
    cnt = (threadIdx.x == 0) ? BT : 0;
  } else {
    for (int i = threadIdx.x; i < BT; i += blockDim.x) cnt += (labels[i] != ignore_index) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) warp_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int n_local = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) n_local += warp_cnt[w];
    const long long n = n_total != nullptr ? *n_total : n_local;
    float D = 1.f;
    if (reduction == 0) D = static_cast<float>(n);
    else if (reduction == 1) D = static_cast<float>(n) * static_cast<float>(V);
    ctl->err = 0;
    ctl->n_valid = n_local;
    ctl->D = D;
    ctl->scale = n > 0 ? 1.f / (temperature * D) : 0.f;
    ctl->invD = n > 0 ? 1.f / D : 0.f;
  }
}

// Kept rows of one batch (labels NULL: all BT rows) into *count (int64).
__global__ void __launch_bounds__(1024) k_count_valid(const int64_t* __restrict__ labels, int BT,
                                                      long long ignore_index, int64_t* count) {
  __shared__ int warp_cnt[32];
  int cnt = 0;
  if (labels == nullptr) {
    cnt = (threadIdx.x == 0) ? BT : 0;
  } else {
    for (int i = threadIdx.x; i < BT; i += blockDim.x) cnt += (labels[i] != ignore_index) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) warp_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long n = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) n += warp_cnt[w];
    *count = n;
  }
}

// Selective log-probability (cross-entropy mode): logp[r] = -rowloss[r], the
// log-probability of row r's target (0 on dropped rows and on targets
// outside [0, V)).
__global__ void k_neg_rows(const float* __restrict__ rowloss, int BT, float* __restrict__ out) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < BT) out[r] = -rowloss[r];
}

// Row coefficients of the selective log-probability backward: for an
// upstream gradient dlogp[r], dz_r = dlogp[r] (onehot(target_r) - p_r) / T,
// which is the pass-2 form G = coefS p - coefQ onehot with coefS = coefQ =
// -dlogp[r] / T; 0 on dropped rows and on targets outside [0, V).
__global__ void k_coef_from_dlogp(const float* __restrict__ dlogp,
                                  const int64_t* __restrict__ target, int BT,
                                  long long ignore_index, int V, float invT,
                                  float* __restrict__ coefS, float* __restrict__ coefQ) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= BT) return;
  const long long y = target[r];
  const bool keep = y != ignore_index && y >= 0 && y < V;
  const float c = keep ? -dlogp[r] * invT : 0.f;
  coefS[r] = c;
  coefQ[r] = c;
}

// Merge of the per-group statistics (m, s, A, B2, S) of each row, in group
// order, into lse2 = log2 sum 2^t and the row loss
//   l_r = ln2 * B2 - A / T + ln2 * lse2 * S
// (= sum_v q (log max(q,eps) - log p)).  Also the per-row coefficients of the
// gradient pass.  Block: 32 warps x 32 rows; warp w merges groups w, w+32, ...
// (loads coalesced over the 32 rows), then warp 0 merges the 32 partials in
// warp order.
constexpr int kCombineWarps = 32;
__global__ void __launch_bounds__(32 * kCombineWarps)
    k_combine(const float* __restrict__ st, int n_tiles, int BT, const int64_t* __restrict__ labels,
              long long ignore_index, float invT, const DevCtl* __restrict__ ctl,
              float* __restrict__ lse2_out, float* __restrict__ coefS, float* __restrict__ coefQ,
              float* __restrict__ rowloss) {
  __shared__ float part[kCombineWarps][5][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int row = blockIdx.x * 32 + lane;
  const size_t plane = static_cast<size_t>(n_tiles) * BT;
  float m = -INFINITY, s = 0.f, A = 0.f, B2 = 0.f, S = 0.f;
  if (row < BT) {
#pragma unroll 4
    for (int t = w; t < n_tiles; t += kCombineWarps) {
      const size_t o = static_cast<size_t>(t) * BT + row;
      const float tm = st[o], ts = st[o + plane];
      A += st[o + 2 * plane];
      B2 += st[o + 3 * plane];
      S += st[o + 4 * plane];
      const float nm = fmaxf(m, tm);
      s = s * exp2f(m - nm) + ts * exp2f(tm - nm);
      m = nm;
    }
  }
  part[w][0][lane] = m;
  part[w][1][lane] = s;
  part[w][2][lane] = A;
  part[w][3][lane] = B2;
  part[w][4][lane] = S;
  __syncthreads();
  if (w == 0 && row < BT) {
    m = part[0][0][lane];
    s = part[0][1][lane];
    A = part[0][2][lane];
    B2 = part[0][3][lane];
    S = part[0][4][lane];
    for (int k = 1; k < kCombineWarps; ++k) {
      const float tm = part[k][0][lane];
      if (tm == -INFINITY) continue;  // warp k saw no group of this row
      const float nm = fmaxf(m, tm);
      s = s * exp2f(m - nm) + part[k][1][lane] * exp2f(tm - nm);
      m = nm;
      A += part[k][2][lane];
      B2 += part[k][3][lane];
      S += part[k][4][lane];
    }
    const float LN2 = 0.693147180559945309f;
    const float lse2 = m + log2f(s);
    const bool keep = labels == nullptr || labels[row] != ignore_index;
    const float sc = ctl->scale;
    lse2_out[row] = lse2;
    coefS[row] = keep ? S * sc : 0.f;
    coefQ[row] = keep ? sc : 0.f;
    rowloss[row] = keep ? (LN2 * B2 - A * invT + LN2 * lse2 * S) : 0.f;
  }
}

// Online merge of one (max, sum) pair of base-2 softmax statistics.
__device__ __forceinline__ void merge_ms(float& m, float& s, float tm, float ts) {
  if (tm == -INFINITY) return;  // nothing to merge (also keeps -inf - -inf out)
  const float nm = fmaxf(m, tm);
  s = s * exp2f(m - nm) + ts * exp2f(tm - nm);
  m = nm;
}

// Row values from the merged statistics of one row.
__device__ __forceinline__ void finish_row(int row, float m, float s, float A, float B2, float S,
                                           const int64_t* __restrict__ labels,
                                           long long ignore_index, float invT, float sc,
                                           float* __restrict__ lse2_out,
                                           float* __restrict__ coefS, float* __restrict__ coefQ,
                                           float* __restrict__ rowloss) {
  const float LN2 = 0.693147180559945309f;
  const float lse2 = m + log2f(s);
  const bool keep = labels == nullptr || labels[row] != ignore_index;
  lse2_out[row] = lse2;
  coefS[row] = keep ? S * sc : 0.f;
  coefQ[row] = keep ? sc : 0.f;
  rowloss[row] = keep ? (LN2 * B2 - A * invT + LN2 * lse2 * S) : 0.f;
}

// The merge of k_combine spread over more blocks, with the loss sum fused:
// grid (ceil(BT/32) row blocks, `splits`); block (row block, split) merges
// groups [split*G/splits, (split+1)*G/splits) of its 32 rows (warp w takes
// every 8th group, then warp 0 merges the 8 warp partials in warp order) into
// part[5][splits][BT].  The last block of a row block to finish (ticket
// tickets[row block]) merges the splits' partials in split order and writes
// the row values; when `loss` is given, the last row block to finish (ticket
// tickets[row blocks]) sums the row losses in a fixed order (fp64) into
// *loss = sum / D.  Every merge and sum has a fixed order, so the results do
// not depend on which block finishes last.  The tickets are zero at launch.
constexpr int kCombSplitWarps = 8;
__global__ void __launch_bounds__(32 * kCombSplitWarps)
    k_combine_split(const float* __restrict__ st, int n_groups, int BT, int splits,
                    const int64_t* __restrict__ labels, long long ignore_index, float invT,
                    const DevCtl* __restrict__ ctl, float* part, int* tickets,
                    float* __restrict__ lse2_out, float* __restrict__ coefS,
                    float* __restrict__ coefQ, float* rowloss, float* loss) {
  __shared__ float sp[kCombSplitWarps][5][32];
  __shared__ double red[32 * kCombSplitWarps];
  __shared__ int is_last;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int row = blockIdx.x * 32 + lane;
  const int split = blockIdx.y;
  const size_t plane = static_cast<size_t>(n_groups) * BT;
  const int g0 = static_cast<int>((static_cast<long long>(split) * n_groups) / splits);
  const int g1 = static_cast<int>((static_cast<long long>(split + 1) * n_groups) / splits);
  float m = -INFINITY, s = 0.f, A = 0.f, B2 = 0.f, S = 0.f;
  if (row < BT) {
#pragma unroll 4
    for (int g = g0 + w; g < g1; g += kCombSplitWarps) {
      const size_t o = static_cast<size_t>(g) * BT + row;
      merge_ms(m, s, st[o], st[o + plane]);
      A += st[o + 2 * plane];
      B2 += st[o + 3 * plane];
      S += st[o + 4 * plane];
    }
  }
  sp[w][0][lane] = m;
  sp[w][1][lane] = s;
  sp[w][2][lane] = A;
  sp[w][3][lane] = B2;
  sp[w][4][lane] = S;
  __syncthreads();
  const size_t pplane = static_cast<size_t>(splits) * BT;
  if (w == 0 && row < BT) {
    m = sp[0][0][lane];
    s = sp[0][1][lane];
    A = sp[0][2][lane];
    B2 = sp[0][3][lane];
    S = sp[0][4][lane];
    for (int k = 1; k < kCombSplitWarps; ++k) {
      merge_ms(m, s, sp[k][0][lane], sp[k][1][lane]);
      A += sp[k][2][lane];
      B2 += sp[k][3][lane];
      S += sp[k][4][lane];
    }
    const size_t o = static_cast<size_t>(split) * BT + row;
    part[o] = m;
    part[o + pplane] = s;
    part[o + 2 * pplane] = A;
    part[o + 3 * pplane] = B2;
    part[o + 4 * pplane] = S;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&tickets[blockIdx.x], 1) == splits - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (w == 0 && row < BT) {
    m = -INFINITY;
    s = A = B2 = S = 0.f;
    for (int k = 0; k < splits; ++k) {
      const size_t o = static_cast<size_t>(k) * BT + row;
      merge_ms(m, s, __ldcg(part + o), __ldcg(part + o + pplane));
      A += __ldcg(part + o + 2 * pplane);
      B2 += __ldcg(part + o + 3 * pplane);
      S += __ldcg(part + o + 4 * pplane);
    }
    finish_row(row, m, s, A, B2, S, labels, ignore_index, invT, ctl->scale, lse2_out, coefS,
               coefQ, rowloss);
  }
  if (loss == nullptr) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&tickets[gridDim.x], 1) == static_cast<int>(gridDim.x) - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  double acc = 0.0;
  for (int i = threadIdx.x; i < BT; i += blockDim.x) acc += static_cast<double>(__ldcg(rowloss + i));
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (static_cast<int>(threadIdx.x) < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = static_cast<float>(red[0] * static_cast<double>(ctl->invD));
}

// loss = (sum of row losses) / D, summed in a fixed order (fp64 partials).
__global__ void __launch_bounds__(1024) k_loss(const float* __restrict__ rowloss, int BT,
                                               const DevCtl* __restrict__ ctl, float* loss) {
  __shared__ double red[1024];
  double acc = 0.0;
  for (int i = threadIdx.x; i < BT; i += blockDim.x) acc += static_cast<double>(rowloss[i]);
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (static_cast<int>(threadIdx.x) < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = static_cast<float>(red[0] * static_cast<double>(ctl->invD));
}

// db[v] = sum over row groups g (in order) of part[g][v].
__global__ void k_db_reduce(const float* __restrict__ part, int groups, int V, void* db,
                            int out_fp32) {
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= V) return;
  float acc = 0.f;
  for (int gi = 0; gi < groups; ++gi) acc += part[static_cast<size_t>(gi) * V + v];
  if (out_fp32) static_cast<float*>(db)[v] = acc;
  else static_cast<__nv_bfloat16*>(db)[v] = __float2bfloat16_rn(acc);
}

// Zero fill (used for empty inputs).
__global__ void k_zero(void* p, size_t bytes) {
  const size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 16;
  if (i + 16 <= bytes) *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p) + i) = make_uint4(0, 0, 0, 0);
  else
    for (size_t j = i; j < bytes; ++j) static_cast<uint8_t*>(p)[j] = 0;
}

// dst = cast(src * s) over n elements, s = *scale (1 when scale is NULL; the
// product is skipped when s == 1).  Grid-stride over 8-element vectors, then
// a scalar tail; src and dst 16-byte aligned, possibly the same buffer (each
// element is read and written by the same thread).
template <class TS>
__device__ __forceinline__ float ld_as_f32(const TS* p, size_t i) {
  if constexpr (sizeof(TS) == 4) return p[i];
  else return __bfloat162float(p[i]);
}
template <class TD>
__device__ __forceinline__ void st_from_f32(TD* p, size_t i, float v) {
  if constexpr (sizeof(TD) == 4) p[i] = v;
  else p[i] = __float2bfloat16_rn(v);
}
template <class TS, class TD>
__global__ void __launch_bounds__(256) k_scale_cast(const TS* src, TD* dst, long long n,
                                                    const float* scale) {
  const float s = scale != nullptr ? *scale : 1.f;
  const bool mul = s != 1.f;
  const long long nv = n / 8;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; v < nv;
       v += stride) {
    float f[8];
    if constexpr (sizeof(TS) == 4) {
      const float4 a = reinterpret_cast<const float4*>(src)[2 * v];
      const float4 b = reinterpret_cast<const float4*>(src)[2 * v + 1];
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
      f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
      unpack8_bf16(reinterpret_cast<const uint4*>(src)[v], f);
    }
    if (mul) {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] *= s;
    }
    if constexpr (sizeof(TD) == 4) {
      reinterpret_cast<float4*>(dst)[2 * v] = make_float4(f[0], f[1], f[2], f[3]);
      reinterpret_cast<float4*>(dst)[2 * v + 1] = make_float4(f[4], f[5], f[6], f[7]);
    } else {
      uint4 u;
      u.x = pack_bf16x2(f[0], f[1]);
      u.y = pack_bf16x2(f[2], f[3]);
      u.z = pack_bf16x2(f[4], f[5]);
      u.w = pack_bf16x2(f[6], f[7]);
      reinterpret_cast<uint4*>(dst)[v] = u;
    }
  }
  for (long long i = nv * 8 + blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
       i < n; i += stride) {
    const float x = ld_as_f32<TS>(src, static_cast<size_t>(i));
    st_from_f32<TD>(dst, static_cast<size_t>(i), mul ? x * s : x);
  }
}

// One thread: (globaltimer, clock64) every interval_ns, n samples.  Each wait
// ends when the global timer passes its target, so the kernel runs for about
// n * interval_ns.
__global__ void k_clock_trace(uint64_t* out, int n, unsigned int interval_ns) {
  const uint64_t t0 = globaltimer_ns();
  for (int i = 0; i < n; ++i) {
    const uint64_t target = t0 + static_cast<uint64_t>(i) * interval_ns;
    uint64_t t = globaltimer_ns();
    while (t < target) t = globaltimer_ns();
    out[2 * i] = t;
    out[2 * i + 1] = static_cast<uint64_t>(clock64());
  }
}

}  // namespace flkl
