// Persistent warp-specialised tcgen05 GEMM for sm_100a with fused epilogues.
//
//   D[M,N] = A[M,K] * B[N,K]^T, bf16 operands, fp32 accumulation in TMEM.
//
// Roles (6 warps, one CTA per SM):
//   warp 0      TMA producer: stages A and B tiles (SWIZZLE_128B) into a
//               4-deep shared-memory ring, one mbarrier pair per stage;
//   warp 1      MMA issuer: owns the TMEM allocation (512 columns = two
//               128x256 fp32 accumulators) and issues tcgen05.mma from one
//               thread; tcgen05.commit frees ring stages and publishes a
//               finished accumulator;
//   warps 2..5  epilogue: each warp reads its 32-lane quarter of the
//               accumulator with tcgen05.ld (one thread = one output row) and
//               runs the fused epilogue, while the MMA warp already fills the
//               other accumulator with the next tile.
//
// Operands may be K-major (rows of K contiguous) or MN-major (K rows of M or N
// contiguous); both are loaded by plain 2-D TMA tile copies, never multicast.
// Every wait is bounded (see mbar_wait); on a timeout the CTA drains its own
// in-flight copies and MMAs, frees TMEM and returns.
#pragma once

#include "ptx.cuh"

namespace flkl {

constexpr int TC_BM = 128;
constexpr int TC_BN = 256;
constexpr int TC_BK = 64;
constexpr int TC_STAGES = 4;
constexpr int TC_THREADS = 192;
constexpr int TC_A_BYTES = TC_BM * TC_BK * 2;  // 16 KiB
constexpr int TC_B_BYTES = TC_BN * TC_BK * 2;  // 32 KiB
constexpr int TC_TMEM_COLS = 512;
constexpr int TC_SMEM_BYTES = TC_STAGES * (TC_A_BYTES + TC_B_BYTES) + 256 + 1024;

struct TcGemmArgs {
  int M, N, K;          // problem extent (rows of D, cols of D, reduction)
  int m_tiles, n_tiles; // ceil(M/128), ceil(N/256)
  int num_kb;           // ceil(K/64)
  int m_fastest;        // tile order: 1 = consecutive tiles walk M
  int a_m_off, a_k_off; // coordinate offsets added to A tile coordinates
  int b_n_off, b_k_off; // coordinate offsets added to B tile coordinates
  int* err_flag;
  unsigned long long wait_limit_ns;
};

__device__ __forceinline__ void tile_coords(const TcGemmArgs& g, int t, int& mb, int& nb) {
  if (g.m_fastest) {
    mb = t % g.m_tiles;
    nb = t / g.m_tiles;
  } else {
    nb = t % g.n_tiles;
    mb = t / g.n_tiles;
  }
}

// Loads one ring stage.  K-major operand tile: one box {64 (K), rows}.
// MN-major operand tile: rows/64 boxes {64 (MN), 64 (K)}, 8 KiB apart.
template <bool MN_MAJOR, int ROWS>
__device__ __forceinline__ void tma_stage(const CUtensorMap* map, uint64_t* bar, uint8_t* dst,
                                          int mn0, int k0) {
  if constexpr (!MN_MAJOR) {
    tma_load_2d(map, bar, dst, k0, mn0);
  } else {
#pragma unroll
    for (int j = 0; j < ROWS / 64; ++j) tma_load_2d(map, bar, dst + j * 8192, mn0 + 64 * j, k0);
  }
}

// Descriptor of the k-th 16-deep slice of a stage.
template <bool MN_MAJOR>
__device__ __forceinline__ uint64_t stage_desc(uint32_t base, int k) {
  if constexpr (!MN_MAJOR) {
    // rows of 128 B (64 bf16 of K), 8-row atoms of 1024 B; K slice = +32 B
    return smem_desc_sw128(base + 32u * k, 16u, 1024u);
  } else {
    // 64-wide MN blocks of 64 K-rows (8 KiB apart = LBO), 8-row K groups of
    // 1024 B (SBO); K slice of 16 rows = +2048 B
    return smem_desc_sw128(base + 2048u * k, 8192u, 1024u);
  }
}

template <class Epi, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const TcGemmArgs g, const typename Epi::Params ep) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + TC_STAGES * TC_A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + TC_STAGES * TC_B_BYTES);
  uint64_t* full = bars;                   // [STAGES] TMA -> MMA
  uint64_t* empty = bars + TC_STAGES;      // [STAGES] MMA -> TMA
  uint64_t* tfull = bars + 2 * TC_STAGES;  // [2] MMA -> epilogue
  uint64_t* tempty = tfull + 2;            // [2] epilogue -> MMA
  uint64_t* drain = tempty + 2;            // MMA drain at exit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TC_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, g.err_flag, g.wait_limit_ns};
  const int num_tiles = g.m_tiles * g.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(g, t, mb, nb);
        const int m0 = mb * TC_BM + g.a_m_off;
        const int n0 = nb * TC_BN + g.b_n_off;
        for (int kb = 0; kb < g.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], TC_A_BYTES + TC_B_BYTES);
          tma_stage<A_MN, TC_BM>(&tmA, &full[stage], sA + stage * TC_A_BYTES, m0,
                                 kb * TC_BK + g.a_k_off);
          tma_stage<B_MN, TC_BN>(&tmB, &full[stage], sB + stage * TC_B_BYTES, n0,
                                 kb * TC_BK + g.b_k_off);
          ++issued;
          if (++stage == TC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: the last min(issued, STAGES) copies must have landed before
      // the CTA may exit (they always complete; the wait is still bounded).
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < TC_STAGES && i < issued; ++i) {
        if (--s < 0) {
          s = TC_STAGES - 1;
          ph ^= 1u;
        }
        const uint32_t addr = smem_u32(&full[s]);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(addr, ph)) {
          if (globaltimer_ns() - t0 > g.wait_limit_ns) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, TC_BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * TC_BN;
        for (int kb = 0; kb < g.num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * TC_A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * TC_B_BYTES);
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k) {
            tc_mma_f16(d_tmem, stage_desc<A_MN>(a_base, k), stage_desc<B_MN>(b_base, k), idesc,
                       (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == TC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      // Drain every MMA this thread issued before TMEM is released.
      tc_commit(drain);
      const uint32_t addr = smem_u32(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(addr, 0)) {
        if (globaltimer_ns() - t0 > g.wait_limit_ns) break;
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------- epilogue
    const int quad = warp & 3;  // TMEM lane quarter this warp may access
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_phase, wc)) break;
      __syncwarp();
      tc_fence_after();
      int mb, nb;
      tile_coords(g, t, mb, nb);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * TC_BN;
      Epi::run(ep, g, taddr, mb, nb, quad, lane);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TC_TMEM_COLS);
  }
}

// ====================================================================
// Epilogues.  `run` is called by each of the 4 epilogue warps for its
// 32-row quarter; lane i owns row (mb*128 + quad*32 + i) of the tile.

// Pass 1: per (row, 256-column tile) softmax and KL statistics.
//   t = (acc + b) * log2(e)/T        (student logits in base-2 units)
//   m = max t, s = sum 2^(t - m)     (online over the tile's 8 column groups)
//   A = sum q z, B2 = sum q log2 max(q, eps), S = sum q
struct EpiStats {
  struct Params {
    const __nv_bfloat16* Q;
    const __nv_bfloat16* bias;  // may be null
    int BT, V;
    float t_scale;  // log2(e) / T
    float eps;
    float* st;      // [5][n_tiles][BT]
    long long st_plane;  // n_tiles * BT
  };
  __device__ __forceinline__ static void run(const Params& p, const TcGemmArgs&, uint32_t taddr,
                                             int mb, int nb, int quad, int lane) {
    const int row = mb * TC_BM + quad * 32 + lane;
    const bool rv = row < p.BT;
    const int n0 = nb * TC_BN;
    const __nv_bfloat16* qrow = p.Q + static_cast<size_t>(rv ? row : 0) * p.V;
    const float qmin = fmaxf(p.eps, 1.17549435e-38f);
    float m = -INFINITY, s = 0.f, A = 0.f, B2 = 0.f, S = 0.f;
#pragma unroll 1
    for (int c = 0; c < TC_BN / 32; ++c) {
      const int col0 = n0 + c * 32;
      if (col0 >= p.V) break;  // warp-uniform
      float q[32], bv[32], z[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = col0 + 8 * j;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (rv && cc < p.V) u = ld_nc_v4(qrow + cc);
        unpack8_bf16(u, q + 8 * j);
        uint4 ub = make_uint4(0, 0, 0, 0);
        if (p.bias != nullptr && cc < p.V) ub = ld_nc_v4(p.bias + cc);
        unpack8_bf16(ub, bv + 8 * j);
      }
      tmem_ld32(taddr + c * 32, z);
      float cm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const bool ok = (col0 + i) < p.V;
        const float zz = z[i] + bv[i];
        z[i] = ok ? zz * p.t_scale : -INFINITY;
        cm = fmaxf(cm, z[i]);
        A = fmaf(q[i], zz, A);
        S += q[i];
        B2 += (q[i] != 0.f) ? q[i] * __log2f(fmaxf(q[i], qmin)) : 0.f;
      }
      const float nm = fmaxf(m, cm);
      float acc = s * exp2f(m - nm);
#pragma unroll
      for (int i = 0; i < 32; ++i) acc += exp2f(z[i] - nm);
      s = acc;
      m = nm;
    }
    if (rv) {
      const size_t o = static_cast<size_t>(nb) * p.BT + row;
      p.st[o] = m;
      p.st[o + p.st_plane] = s;
      p.st[o + 2 * p.st_plane] = A;
      p.st[o + 3 * p.st_plane] = B2;
      p.st[o + 4 * p.st_plane] = S;
    }
  }
};

// Sum 32 per-lane vectors of 32 values across the warp: afterwards v[0] of
// lane l holds the sum over lanes of v[l] (butterfly reduce-scatter, fixed
// order, 31 shuffles).
__device__ __forceinline__ float warp_transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

// Pass 2: G = coefS * 2^(t - lse2) - coefQ * q on the chunk's columns, stored
// as bf16 (round to nearest even) into the staging buffer; optional per
// 32-row column partial sums of the fp32 G (for db).
struct EpiGrad {
  struct Params {
    const __nv_bfloat16* Q;
    const __nv_bfloat16* bias;  // may be null
    int BT, V;
    int c0;          // first vocabulary column of the chunk
    int ldg;         // staging row pitch (elements)
    __nv_bfloat16* G;
    float t_scale;
    const float* lse2;   // [BT] log2-sum-exp2 of t
    const float* coefS;  // [BT] S_r / (T D), 0 on dropped rows
    const float* coefQ;  // [BT] 1 / (T D), 0 on dropped rows
    float* dbpart;       // [row groups of 32][V] or null
  };
  __device__ __forceinline__ static void run(const Params& p, const TcGemmArgs&, uint32_t taddr,
                                             int mb, int nb, int quad, int lane) {
    const int row = mb * TC_BM + quad * 32 + lane;
    const bool rv = row < p.BT;
    const int n0 = nb * TC_BN;  // chunk-relative
    const __nv_bfloat16* qrow = p.Q + static_cast<size_t>(rv ? row : 0) * p.V;
    __nv_bfloat16* grow = p.G + static_cast<size_t>(rv ? row : 0) * p.ldg;
    const float lse2 = rv ? p.lse2[row] : 0.f;
    const float cS = rv ? p.coefS[row] : 0.f;
    const float cQ = rv ? p.coefQ[row] : 0.f;
#pragma unroll 1
    for (int c = 0; c < TC_BN / 32; ++c) {
      const int col0 = n0 + c * 32;
      const int gcol0 = p.c0 + col0;
      if (gcol0 >= p.V) break;  // warp-uniform
      float q[32], bv[32], z[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = gcol0 + 8 * j;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (rv && cc < p.V) u = ld_nc_v4(qrow + cc);
        unpack8_bf16(u, q + 8 * j);
        uint4 ub = make_uint4(0, 0, 0, 0);
        if (p.bias != nullptr && cc < p.V) ub = ld_nc_v4(p.bias + cc);
        unpack8_bf16(ub, bv + 8 * j);
      }
      tmem_ld32(taddr + c * 32, z);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const bool ok = (gcol0 + i) < p.V;
        const float t = (z[i] + bv[i]) * p.t_scale;
        const float gv = cS * exp2f(t - lse2) - cQ * q[i];
        z[i] = ok ? gv : 0.f;
      }
      if (rv) {
        uint4* dst = reinterpret_cast<uint4*>(grow + col0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 u;
          u.x = pack_bf16x2(z[8 * j + 0], z[8 * j + 1]);
          u.y = pack_bf16x2(z[8 * j + 2], z[8 * j + 3]);
          u.z = pack_bf16x2(z[8 * j + 4], z[8 * j + 5]);
          u.w = pack_bf16x2(z[8 * j + 6], z[8 * j + 7]);
          dst[j] = u;
        }
      }
      if (p.dbpart != nullptr) {
        const float colsum = warp_transpose_sum32(z, lane);
        const int gc = gcol0 + lane;
        if (gc < p.V)
          p.dbpart[static_cast<size_t>(mb * 4 + quad) * p.V + gc] = colsum;
      }
    }
  }
};

// dW rows of one chunk: out[c0 + m][n] = acc, fp32 or bf16.
struct EpiStoreRows {
  struct Params {
    void* out;
    int ld;         // elements per output row (H)
    int rows;       // valid rows in this launch (chunk width)
    int cols;       // valid columns (H)
    int row_off;    // first output row (chunk start)
    int out_fp32;
  };
  __device__ __forceinline__ static void run(const Params& p, const TcGemmArgs&, uint32_t taddr,
                                             int mb, int nb, int quad, int lane) {
    const int r = mb * TC_BM + quad * 32 + lane;
    const bool rv = r < p.rows;
    const size_t orow = static_cast<size_t>(p.row_off + (rv ? r : 0)) * p.ld;
#pragma unroll 1
    for (int c = 0; c < TC_BN / 32; ++c) {
      const int col0 = nb * TC_BN + c * 32;
      if (col0 >= p.cols) break;
      float v[32];
      tmem_ld32(taddr + c * 32, v);
      if (!rv) continue;
      if (p.out_fp32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow + col0);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (col0 + 4 * j < p.cols)
            dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow + col0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (col0 + 8 * j < p.cols) {
            uint4 u;
            u.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
            u.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
            u.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
            u.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
            dst[j] = u;
          }
      }
    }
  }
};

// dX accumulation over vocabulary chunks.
//   mode 0 (only chunk):  out = bf16(acc)
//   mode 1 (first):       part = acc
//   mode 2 (middle):      part += acc
//   mode 3 (last):        out = bf16(part + acc)
struct EpiAccumRows {
  struct Params {
    float* part;                 // [rows][ld] fp32
    __nv_bfloat16* out;          // [rows][ld]
    int ld, rows, cols;
    int mode;
  };
  __device__ __forceinline__ static void run(const Params& p, const TcGemmArgs&, uint32_t taddr,
                                             int mb, int nb, int quad, int lane) {
    const int r = mb * TC_BM + quad * 32 + lane;
    const bool rv = r < p.rows;
    const size_t orow = static_cast<size_t>(rv ? r : 0) * p.ld;
#pragma unroll 1
    for (int c = 0; c < TC_BN / 32; ++c) {
      const int col0 = nb * TC_BN + c * 32;
      if (col0 >= p.cols) break;
      float v[32];
      tmem_ld32(taddr + c * 32, v);
      if (!rv) continue;
      float4* pp = reinterpret_cast<float4*>(p.part + orow + col0);
      if (p.mode == 2 || p.mode == 3) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (col0 + 4 * j < p.cols) {
            const float4 o = pp[j];
            v[4 * j] += o.x;
            v[4 * j + 1] += o.y;
            v[4 * j + 2] += o.z;
            v[4 * j + 3] += o.w;
          }
      }
      if (p.mode == 1 || p.mode == 2) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (col0 + 4 * j < p.cols)
            pp[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(p.out + orow + col0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (col0 + 8 * j < p.cols) {
            uint4 u;
            u.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
            u.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
            u.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
            u.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
            dst[j] = u;
          }
      }
    }
  }
};

}  // namespace flkl
