// Persistent warp-specialised tcgen05 GEMM for sm_100a on CTA pairs, with
// fused epilogues.
//
//   D[M,N] = A[M,K] * B[N,K]^T, bf16 operands, fp32 accumulation in TMEM.
//
// A cluster of two CTAs (on two SMs) computes one 256x256 output tile with
// tcgen05.mma.cta_group::2: CTA r stages rows [128r, 128r+128) of the tile's
// A block and rows [128r, 128r+128) of its B block, so each SM streams half
// of B; the even CTA issues the MMAs, which read A and B from both CTAs'
// shared memory and write rows [128r, 128r+128) of D into CTA r's TMEM.
//
// Roles (10 warps per CTA, one CTA per SM):
//   warp 0      TMA producer (both CTAs): a ring of TC_STAGES stages of
//               TC_BK-deep K blocks (3 x 64 KiB per CTA at the default
//               TC_BK = 128); every copy signals the even CTA's `full`
//               barrier;
//   warp 1      TMEM owner (both CTAs, 512 columns = two 256-column fp32
//               accumulators) and, in the even CTA, the MMA issuer;
//               tcgen05.commit arrives on both CTAs' `empty` (stage free)
//               and `tfull` (accumulator ready) barriers;
//   warps 2..9  epilogue (both CTAs): warp w reads lane quarter w%4 of its
//               CTA's accumulator, columns [128h, 128h+128) with h = (w-2)/4,
//               with tcgen05.ld (one thread = one output row) while the MMA
//               fills the other accumulator; the warps then arrive on the
//               even CTA's `tempty` barrier.
//
// Operands may be K-major (rows of K contiguous) or MN-major (K rows of M or N
// contiguous); both are loaded by plain TMA tile copies (one 3-D "blocked"
// copy per operand and stage when the inner extent is a multiple of 64,
// else 2-D copies), never multicast.
// Every wait is bounded (see mbar_wait); on a timeout the CTA stops, drains
// its own in-flight copies and MMAs, frees TMEM and returns.
#pragma once

#include "ptx.cuh"

namespace flkl {

constexpr int TC_BM = 256;            // output tile rows (pair)
constexpr int TC_BN = 256;            // output tile columns
constexpr int TC_HM = 128;            // rows per CTA
// Build-time tunables (-DFLKL_TC_BK=..., -DFLKL_TC_STAGES=...).
#ifndef FLKL_TC_BK
#define FLKL_TC_BK 128
#endif
#ifndef FLKL_TC_STAGES
#define FLKL_TC_STAGES 3
#endif
constexpr int TC_BK = FLKL_TC_BK;     // K depth of a ring stage (a multiple of 64)
constexpr int TC_KSUB = TC_BK / 64;   // 128-byte swizzle atoms along K per stage
constexpr int TC_STAGES = FLKL_TC_STAGES;
static_assert(TC_BK % 64 == 0 && TC_BK <= 256, "stage depth: a multiple of 64, at most 256");
constexpr int TC_EPI_WARPS = 8;       // two per TMEM lane quarter
constexpr int TC_EPI_COLS = 128;      // accumulator columns per epilogue warp
constexpr int TC_THREADS = 64 + 32 * TC_EPI_WARPS;
constexpr int TC_A_BYTES = TC_HM * TC_BK * 2;  // this CTA's A rows (32 KiB at TC_BK = 128)
constexpr int TC_B_BYTES = TC_HM * TC_BK * 2;  // this CTA's half of B (32 KiB at TC_BK = 128)
constexpr int TC_STAGE_BYTES = TC_A_BYTES + TC_B_BYTES;
constexpr int TC_TMEM_COLS = 512;
constexpr int TC_SMEM_BYTES = TC_STAGES * TC_STAGE_BYTES + 256 + 1024;

static_assert(TC_SMEM_BYTES <= 232448, "dynamic shared memory above the sm_100 per-CTA limit");
// Loads this CTA's 128 rows of one operand for one ring stage.  K-major:
// TC_KSUB boxes {64 (K), 128}, 16 KiB apart.  MN-major: two boxes
// {64 (MN), TC_BK (K)}, TC_BK * 128 bytes apart.  When the blocked extent is
// a multiple of 64, a 3-D map whose third dimension steps 64 elements (128
// bytes) along the blocked extent fetches the same bytes in one copy.
__device__ __forceinline__ void tma_half_stage(const CUtensorMap* map, bool mn_major, bool blocked,
                                               uint32_t bar_cluster, uint8_t* dst, int mn0,
                                               int k0) {
  if (blocked) {
    // 3-D map {64, outer, blocks of 64}: the whole half-stage in one copy
    if (!mn_major) tma_load_3d_pair(map, bar_cluster, dst, 0, mn0, k0 >> 6);
    else tma_load_3d_pair(map, bar_cluster, dst, 0, k0, mn0 >> 6);
    return;
  }
  if (!mn_major) {
#pragma unroll
    for (int s = 0; s < TC_KSUB; ++s)
      tma_load_2d_pair(map, bar_cluster, dst + s * 16384, k0 + 64 * s, mn0);
  } else {
    tma_load_2d_pair(map, bar_cluster, dst, mn0, k0);
    tma_load_2d_pair(map, bar_cluster, dst + TC_BK * 128, mn0 + 64, k0);
  }
}

// Descriptor of the k-th 16-deep slice of a stage (the same offsets are used
// in both CTAs of the pair).
__device__ __forceinline__ uint64_t stage_desc(uint32_t base, int k, bool mn_major) {
  if (!mn_major) {
    // 64-deep K sub-blocks of 128 rows x 128 B (16 KiB apart), 8-row atoms of
    // 1024 B; K slice of 16 = +32 B inside the sub-block
    return smem_desc_sw128(base + 16384u * (k >> 2) + 32u * (k & 3), 16u, 1024u);
  } else {
    // 64-wide MN blocks of TC_BK K-rows (TC_BK * 128 B apart = LBO), 8-row K
    // groups of 1024 B (SBO); K slice of 16 rows = +2048 B
    return smem_desc_sw128(base + 2048u * k, TC_BK * 128u, 1024u);
  }
}

// The same descriptors as stage_desc, split for cheap issue: lower word =
// lo_base + (stage address >> 4) + (k & 3) * s1 + (k >> 2) * s2, upper word hi.
struct DescSteps {
  uint32_t lo_base, hi, s1, s2;
};
__device__ __forceinline__ DescSteps desc_steps(bool mn_major) {
  const uint64_t d = mn_major ? smem_desc_sw128(0, TC_BK * 128u, 1024u)
                              : smem_desc_sw128(0, 16u, 1024u);
  DescSteps r;
  r.lo_base = static_cast<uint32_t>(d);
  r.hi = static_cast<uint32_t>(d >> 32);
  r.s1 = mn_major ? (2048u >> 4) : (32u >> 4);     // next 16-deep K slice
  r.s2 = mn_major ? (8192u >> 4) : (16384u >> 4);  // next 64-deep K sub-block
  return r;
}

// ====================================================================
// Epilogues.  `run` is called by each epilogue warp for its 32 rows and 128
// columns of the tile: lane i owns output row (row0 + quad*32 + i), columns
// [n0, n0 + 128).  `prefetch` is called with the same coordinates just before
// the warp waits for that tile's accumulator, so that the rows of Q the tile
// needs are on their way to L2 while the MMAs run.

__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(ptr)));
}


// 32 bf16 of one row (four 16-byte loads), zero beyond `limit` or when !rv.
__device__ __forceinline__ void load_chunk32(const __nv_bfloat16* rowp, bool rv, int col0,
                                             int limit, uint4 (&u)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int cc = col0 + 8 * j;
    u[j] = (rv && cc < limit) ? ld_nc_v4(rowp + cc) : make_uint4(0, 0, 0, 0);
  }
}
// load_chunk32 with coherent loads, for data the same kernel overwrites.
__device__ __forceinline__ void load_chunk32_rw(const __nv_bfloat16* rowp, bool rv, int col0,
                                                int limit, uint4 (&u)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int cc = col0 + 8 * j;
    u[j] = (rv && cc < limit) ? *reinterpret_cast<const uint4*>(rowp + cc)
                              : make_uint4(0, 0, 0, 0);
  }
}
// Same 32 bias values for every lane of the warp (one broadcast request).
__device__ __forceinline__ void load_bias32(const __nv_bfloat16* bias, int col0, int V,
                                            float (&bv)[32]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int cc = col0 + 8 * j;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (bias != nullptr && cc < V) u = *reinterpret_cast<const uint4*>(bias + cc);
    unpack8_bf16(u, bv + 8 * j);
  }
}

// Pass 1: per (row, 128-column group) softmax and KL statistics.
//   t = (acc + b) * log2(e)/T        (student logits in base-2 units)
//   m = max t, s = sum 2^(t - m)     (online over the group's 32-column chunks)
//   A = sum q z, B2 = sum q log2 max(q, eps), S = sum q
struct EpiStats {
  struct Params {
    const __nv_bfloat16* Q;     // teacher [BT][V]; null in cross-entropy mode
    const __nv_bfloat16* bias;  // may be null
    int BT, V;
    float t_scale;  // log2(e) / T
    float eps;
    float* st;      // [5][n_groups][BT], n_groups = ceil(V/128)
    long long st_plane;  // n_groups * BT
    const int64_t* target;  // cross-entropy mode: q = one-hot at target[row]; else null
    // logits cache of the first vocabulary chunk (null: none): the raw
    // accumulators of columns [0, zc_cols) in 32 x 32 blocks, block
    // (row / 32, column / 32) at ((row / 32) * (zc_cols / 32) + column / 32) * 1024,
    // element (column % 32) * 32 + row % 32, so that a warp (lane = row) stores
    // and reads each column of a block as one 128-byte line
    float* zc;
    int zc_cols;
  };
  __device__ __forceinline__ static void prefetch(const Params& p, int row0, int n0, int quad,
                                                  int lane) {
    const int row = row0 + quad * 32 + lane;
    if (p.Q != nullptr && row < p.BT && n0 < p.V) {
      const __nv_bfloat16* q = p.Q + static_cast<size_t>(row) * p.V + n0;
      prefetch_l2(q);
      if (n0 + 64 < p.V) prefetch_l2(q + 64);
    }
  }
  __device__ __forceinline__ static void run(const Params& p, uint32_t taddr, int row0, int n0,
                                             int quad, int lane) {
    const int row = row0 + quad * 32 + lane;
    const bool rv = row < p.BT;
    if (n0 >= p.V) return;  // warp-uniform: this half of the tile is past V
    const bool ce = p.Q == nullptr;  // warp-uniform
    const __nv_bfloat16* qrow = ce ? nullptr : p.Q + static_cast<size_t>(rv ? row : 0) * p.V;
    long long y = (ce && rv) ? p.target[row] : -1;
    if (y >= p.V) y = -1;  // a target outside [0, V) matches no column
    const float qmin = fmaxf(p.eps, 1.17549435e-38f);
    float m = -INFINITY, s = 0.f, A = 0.f, B2 = 0.f, S = 0.f;
    uint4 qa[4], qb[4];
    if (!ce) load_chunk32(qrow, rv, n0, p.V, qa);
#pragma unroll 1
    for (int c = 0; c < TC_EPI_COLS / 32; ++c) {
      const int col0 = n0 + c * 32;
      if (col0 >= p.V) break;  // warp-uniform
      float q[32], bv[32], z[32];
      if (!ce) {
        if (c + 1 < TC_EPI_COLS / 32) load_chunk32(qrow, rv, col0 + 32, p.V, qb);
#pragma unroll
        for (int j = 0; j < 4; ++j) unpack8_bf16(qa[j], q + 8 * j);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) q[i] = (col0 + i == y) ? 1.f : 0.f;
      }
      tmem_ld32(taddr + c * 32, z);
      if (p.zc != nullptr && col0 < p.zc_cols && rv) {  // (the first condition is warp-uniform)
        float* dst = p.zc +
                     (static_cast<size_t>(row >> 5) * (p.zc_cols >> 5) + (col0 >> 5)) * 1024 + lane;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[i * 32] = z[i];
      }
      if (p.bias != nullptr) {  // warp-uniform
        load_bias32(p.bias, col0, p.V, bv);
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] += bv[i];
      }
      float cm = -INFINITY;
      // q = 0 adds q * log2(qmin) = 0 (qmin >= FLT_MIN keeps the logarithm finite)
      if (col0 + 32 <= p.V) {  // warp-uniform: every column of the chunk is a vocabulary entry
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float zz = z[i];
          z[i] = zz * p.t_scale;
          cm = fmaxf(cm, z[i]);
          A = fmaf(q[i], zz, A);
          S += q[i];
          B2 += q[i] * __log2f(fmaxf(q[i], qmin));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const bool ok = (col0 + i) < p.V;
          const float zz = z[i];
          z[i] = ok ? zz * p.t_scale : -INFINITY;
          cm = fmaxf(cm, z[i]);
          A = fmaf(q[i], zz, A);
          S += q[i];
          B2 += q[i] * __log2f(fmaxf(q[i], qmin));
        }
      }
      const float nm = fmaxf(m, cm);
      float acc = s * exp2f(m - nm);
#pragma unroll
      for (int i = 0; i < 32; ++i) acc += exp2f(z[i] - nm);
      s = acc;
      m = nm;
#pragma unroll
      for (int j = 0; j < 4; ++j) qa[j] = qb[j];
    }
    if (rv) {
      const size_t o = static_cast<size_t>(n0 / TC_EPI_COLS) * p.BT + row;
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
    const int64_t* target;  // cross-entropy mode (Q null): one-hot teacher at target[row]
  };
  __device__ __forceinline__ static void prefetch(const Params& p, int row0, int n0, int quad,
                                                  int lane) {
    const int row = row0 + quad * 32 + lane;
    const int gc = p.c0 + n0;
    if (p.Q != nullptr && row < p.BT && gc < p.V) {
      const __nv_bfloat16* q = p.Q + static_cast<size_t>(row) * p.V + gc;
      prefetch_l2(q);
      if (gc + 64 < p.V) prefetch_l2(q + 64);
    }
  }
  // One gradient value from the logit z (bias added): (S p - q) / (T D) with
  // p = 2^(z log2(e) / T - lse2).  Both multiply-adds are explicit so that
  // every caller rounds the same way.
  __device__ __forceinline__ static float value(float z, float t_scale, float lse2, float cS,
                                                float cQ, float q) {
    return __fmaf_rn(cS, exp2f(__fmaf_rn(z, t_scale, -lse2)), -(cQ * q));
  }
  // The gradients of 32 columns of one row (lane = row of a 32-row group)
  // from their logits z (the accumulator, before the bias): bf16 into the
  // staging row and, with db, the group's column sums.  Shared by the
  // epilogue and k_grad_cached, which therefore give the same bits.
  __device__ __forceinline__ static void cols32(const Params& p, float (&z)[32],
                                                const float (&q)[32], int row, bool rv,
                                                int rgroup, int col0, int gcol0, float lse2,
                                                float cS, float cQ, int lane) {
    if (p.bias != nullptr) {  // warp-uniform
      float bv[32];
      load_bias32(p.bias, gcol0, p.V, bv);
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] += bv[i];
    }
    if (gcol0 + 32 <= p.V) {  // warp-uniform: no column past V
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = value(z[i], p.t_scale, lse2, cS, cQ, q[i]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float gv = value(z[i], p.t_scale, lse2, cS, cQ, q[i]);
        z[i] = (gcol0 + i) < p.V ? gv : 0.f;
      }
    }
    if (rv) {
      // this row's 32 gradients of the chunk: two full 32-byte sectors
      uint4* dst = reinterpret_cast<uint4*>(p.G + static_cast<size_t>(row) * p.ldg + col0);
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
      if (gc < p.V) p.dbpart[static_cast<size_t>(rgroup) * p.V + gc] = colsum;
    }
  }
  __device__ __forceinline__ static void run(const Params& p, uint32_t taddr, int row0, int n0,
                                             int quad, int lane) {
    const int row = row0 + quad * 32 + lane;
    const bool rv = row < p.BT;  // n0 is chunk-relative
    if (p.c0 + n0 >= p.V) return;  // warp-uniform
    const bool ce = p.Q == nullptr;  // warp-uniform
    const __nv_bfloat16* qrow = ce ? nullptr : p.Q + static_cast<size_t>(rv ? row : 0) * p.V;
    long long y = (ce && rv) ? p.target[row] : -1;
    if (y >= p.V) y = -1;  // a target outside [0, V) matches no column
    const float lse2 = rv ? p.lse2[row] : 0.f;
    const float cS = rv ? p.coefS[row] : 0.f;
    const float cQ = rv ? p.coefQ[row] : 0.f;
    uint4 qa[4], qb[4];
    if (!ce) load_chunk32(qrow, rv, p.c0 + n0, p.V, qa);
#pragma unroll 1
    for (int c = 0; c < TC_EPI_COLS / 32; ++c) {
      const int col0 = n0 + c * 32;
      const int gcol0 = p.c0 + col0;
      if (gcol0 >= p.V) break;  // warp-uniform
      float q[32], z[32];
      if (!ce) {
        if (c + 1 < TC_EPI_COLS / 32) load_chunk32(qrow, rv, gcol0 + 32, p.V, qb);
#pragma unroll
        for (int j = 0; j < 4; ++j) unpack8_bf16(qa[j], q + 8 * j);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) q[i] = (gcol0 + i == y) ? 1.f : 0.f;
      }
      tmem_ld32(taddr + c * 32, z);
      cols32(p, z, q, row, rv, row0 / 32 + quad, col0, gcol0, lse2, cS, cQ, lane);
#pragma unroll
      for (int j = 0; j < 4; ++j) qa[j] = qb[j];
    }
  }
};

// Fused linear Jensen-Shannon divergence, student side of one vocabulary
// chunk.  With the student probability p = 2^(t - lse2) (t = (acc + b) *
// log2(e)/T, rounded to bf16 as the teacher's is), the teacher probability q
// of the same entry (staged in bf16 by
// an earlier teacher pass, chunk-relative rows of `ldg`) and m = beta p +
// (1 - beta) q:
//   loss mode (grad == 0): per (row, 128-column group) partial sums
//       part[0][g][row] = sum p ln(p/m),
//       part[1][g][row] = beta sum p ln(p/m) + (1 - beta) sum q ln(q/m);
//   gradient mode (grad == 1): G = rowscale * beta * p * (ln(p/m) - K[row])
//       as bf16 into the staging block, with per 32-row column sums for db.
//       G may overwrite the teacher block itself: each thread reads the q of
//       a 32-column chunk (coherent loads) before it stores that chunk's G.
// 0 ln 0 is taken as 0.
struct EpiJsd {
  struct Params {
    const __nv_bfloat16* bias;  // may be null
    int BT, V;
    int c0;          // first vocabulary column of the chunk
    int ldg;         // row pitch (elements) of the staged teacher block and of G
    const __nv_bfloat16* Qs;  // teacher probabilities of the chunk
    float t_scale;
    const float* lse2;   // [BT] student log2-sum-exp2
    float beta;
    int grad;
    float* part;         // loss mode: [2][n_groups][BT]
    long long part_plane;
    __nv_bfloat16* G;    // gradient mode (may be Qs)
    const float* K;      // [BT] KL(P || M) per row
    const float* rowscale;  // [BT] 1 / (T D), 0 on dropped rows
    float* dbpart;       // [row groups of 32][V] or null
  };
  __device__ __forceinline__ static void prefetch(const Params& p, int row0, int n0, int quad,
                                                  int lane) {
    const int row = row0 + quad * 32 + lane;
    if (row < p.BT && p.c0 + n0 < p.V) {
      const __nv_bfloat16* q = p.Qs + static_cast<size_t>(row) * p.ldg + n0;
      prefetch_l2(q);
      prefetch_l2(q + 64);
    }
  }
  // The 32 columns [gcol0, gcol0 + 32) of one row (lane = row of a 32-row
  // group) from the student logits z (the accumulator, before the bias) and
  // the staged teacher probabilities q: loss mode adds p ln(p/m) and
  // q ln(q/m) into kp and kq; gradient mode writes the row's 32 gradients
  // (bf16) at column col0 of G and, with db, the group's column sums.  Shared
  // by the epilogue and k_jsd_cached, which therefore give the same bits.
  __device__ __forceinline__ static void cols32(const Params& p, float (&z)[32],
                                                const float (&q)[32], int row, bool rv,
                                                int rgroup, int col0, int gcol0, float lse2,
                                                float gk, float gs, float& kp, float& kq,
                                                int lane) {
    const float LN2 = 0.693147180559945309f;
    const float beta = p.beta, omb = 1.f - p.beta;
    if (p.bias != nullptr) {  // warp-uniform
      float bv[32];
      load_bias32(p.bias, gcol0, p.V, bv);
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] += bv[i];
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const bool ok = (gcol0 + i) < p.V;
      // p rounded to bf16 like the staged teacher q, so that a teacher equal
      // to the student gives p == q exactly (divergence and gradient 0)
      const float pv =
          ok ? __bfloat162float(__float2bfloat16_rn(exp2f(__fmaf_rn(z[i], p.t_scale, -lse2))))
             : 0.f;
      const float qv = ok ? q[i] : 0.f;
      const float mv = __fmaf_rn(beta, pv, omb * qv);
      const float lm = __log2f(mv);
      // p ln(p/m) and q ln(q/m), 0 when the probability is 0
      const float lp = pv > 0.f ? (__log2f(pv) - lm) * LN2 : 0.f;
      if (!p.grad) {
        kp = __fmaf_rn(pv, lp, kp);
        if (qv > 0.f) kq = __fmaf_rn(qv, (__log2f(qv) - lm) * LN2, kq);
      } else {
        z[i] = pv > 0.f ? gs * pv * (lp - gk) : 0.f;
      }
    }
    if (p.grad) {
      if (rv) {
        uint4* dst = reinterpret_cast<uint4*>(p.G + static_cast<size_t>(row) * p.ldg + col0);
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
        if (gc < p.V) p.dbpart[static_cast<size_t>(rgroup) * p.V + gc] = colsum;
      }
    }
  }
  __device__ __forceinline__ static void run(const Params& p, uint32_t taddr, int row0, int n0,
                                             int quad, int lane) {
    const int row = row0 + quad * 32 + lane;
    const bool rv = row < p.BT;
    if (p.c0 + n0 >= p.V) return;  // warp-uniform
    const __nv_bfloat16* qrow = p.Qs + static_cast<size_t>(rv ? row : 0) * p.ldg;
    const float lse2 = rv ? p.lse2[row] : 0.f;
    const float gk = (p.grad && rv) ? p.K[row] : 0.f;
    const float gs = (p.grad && rv) ? p.rowscale[row] * p.beta : 0.f;
    float kp = 0.f, kq = 0.f;
    uint4 qa[4], qb[4];
    load_chunk32_rw(qrow, rv, n0, p.ldg, qa);
#pragma unroll 1
    for (int c = 0; c < TC_EPI_COLS / 32; ++c) {
      const int col0 = n0 + c * 32;
      const int gcol0 = p.c0 + col0;
      if (gcol0 >= p.V) break;  // warp-uniform
      float q[32], z[32];
      if (c + 1 < TC_EPI_COLS / 32) load_chunk32_rw(qrow, rv, col0 + 32, p.ldg, qb);
#pragma unroll
      for (int j = 0; j < 4; ++j) unpack8_bf16(qa[j], q + 8 * j);
      tmem_ld32(taddr + c * 32, z);
      cols32(p, z, q, row, rv, row0 / 32 + quad, col0, gcol0, lse2, gk, gs, kp, kq, lane);
#pragma unroll
      for (int j = 0; j < 4; ++j) qa[j] = qb[j];
    }
    if (!p.grad && rv) {
      const size_t o = static_cast<size_t>((p.c0 + n0) / TC_EPI_COLS) * p.BT + row;
      p.part[o] = kp;
      p.part[o + p.part_plane] = __fmaf_rn(p.beta, kp, (1.f - p.beta) * kq);
    }
  }
};

// The student pass of the first vocabulary chunk from the logits its
// statistics pass kept (EpiStats::Params::zc, same layout as for
// k_grad_cached): one warp per 32 rows x 128 columns (a statistics group),
// lane = row, the four 32-column blocks in order, EpiJsd::cols32 as in the
// epilogue; loss mode writes the group's partial sums, gradient mode the
// gradient block over the staged teacher block.  8 warps per block.
__global__ void __launch_bounds__(256) k_jsd_cached(const EpiJsd::Params p,
                                                    const float* __restrict__ zc, int zc_cols) {
  const int lane = threadIdx.x & 31;
  const int ngrp = zc_cols / TC_EPI_COLS;
  const long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (w >= static_cast<long long>((p.BT + 31) >> 5) * ngrp) return;  // warp-uniform
  const int rg = static_cast<int>(w / ngrp), n0 = static_cast<int>(w % ngrp) * TC_EPI_COLS;
  if (p.c0 + n0 >= p.V) return;  // warp-uniform
  const int row = rg * 32 + lane;
  const bool rv = row < p.BT;
  const __nv_bfloat16* qrow = p.Qs + static_cast<size_t>(rv ? row : 0) * p.ldg;
  const float lse2 = rv ? p.lse2[row] : 0.f;
  const float gk = (p.grad && rv) ? p.K[row] : 0.f;
  const float gs = (p.grad && rv) ? p.rowscale[row] * p.beta : 0.f;
  float kp = 0.f, kq = 0.f;
#pragma unroll 1
  for (int c = 0; c < TC_EPI_COLS / 32; ++c) {
    const int col0 = n0 + c * 32;
    const int gcol0 = p.c0 + col0;
    if (gcol0 >= p.V) break;  // warp-uniform
    uint4 qa[4];
    load_chunk32_rw(qrow, rv, col0, p.ldg, qa);
    float q[32], z[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack8_bf16(qa[j], q + 8 * j);
    const float* src =
        zc + (static_cast<size_t>(rg) * (zc_cols >> 5) + (col0 >> 5)) * 1024 + lane;
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = rv ? src[i * 32] : 0.f;
    EpiJsd::cols32(p, z, q, row, rv, rg, col0, gcol0, lse2, gk, gs, kp, kq, lane);
  }
  if (!p.grad && rv) {
    const size_t o = static_cast<size_t>((p.c0 + n0) / TC_EPI_COLS) * p.BT + row;
    p.part[o] = kp;
    p.part[o + p.part_plane] = __fmaf_rn(p.beta, kp, (1.f - p.beta) * kq);
  }
}

// dW rows of one chunk: out[c0 + m][n] = acc, fp32 or bf16.
// The store epilogues read the accumulator in the 16-lane fragment layout
// (tmem_ld16x32): for each 32-column chunk and each 16-row half of the warp's
// 32 rows, the threads of a quad hold 8 consecutive columns of a row, so one
// warp store of 8-byte pairs writes 8 rows x 32 bytes (whole sectors).

// dW rows of one chunk: out[c0 + m][n] = acc, fp32 or bf16.
// Pass 2 of the first vocabulary chunk from the logits cache that pass 1
// filled (EpiStats::Params::zc): the same accumulators pass 2 would compute
// again (same operands, same K order), so the same gradients, without the
// GEMM.  One warp per 32 rows x 32 columns, lane = row; 8 warps per block.
__global__ void __launch_bounds__(256) k_grad_cached(const EpiGrad::Params p,
                                                     const float* __restrict__ zc, int zc_cols) {
  const int lane = threadIdx.x & 31;
  const int ncc = zc_cols >> 5;
  const long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (w >= static_cast<long long>((p.BT + 31) >> 5) * ncc) return;  // warp-uniform
  const int rg = static_cast<int>(w / ncc), col0 = static_cast<int>(w % ncc) * 32;
  const int gcol0 = p.c0 + col0;
  if (gcol0 >= p.V) return;  // warp-uniform
  const int row = rg * 32 + lane;
  const bool rv = row < p.BT;
  float z[32], q[32];
  const float* src = zc + static_cast<size_t>(w) * 1024 + lane;
#pragma unroll
  for (int i = 0; i < 32; ++i) z[i] = rv ? src[i * 32] : 0.f;
  if (p.Q != nullptr) {  // warp-uniform
    uint4 qa[4];
    load_chunk32(p.Q + static_cast<size_t>(rv ? row : 0) * p.V, rv, gcol0, p.V, qa);
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack8_bf16(qa[j], q + 8 * j);
  } else {
    long long y = rv ? p.target[row] : -1;
    if (y >= p.V) y = -1;
#pragma unroll
    for (int i = 0; i < 32; ++i) q[i] = (gcol0 + i == y) ? 1.f : 0.f;
  }
  const float lse2 = rv ? p.lse2[row] : 0.f;
  const float cS = rv ? p.coefS[row] : 0.f;
  const float cQ = rv ? p.coefQ[row] : 0.f;
  EpiGrad::cols32(p, z, q, row, rv, rg, col0, gcol0, lse2, cS, cQ, lane);
}

struct EpiStoreRows {
  struct Params {
    void* out;
    int ld;         // elements per output row (H)
    int rows;       // valid rows in this launch (chunk width)
    int cols;       // valid columns (H)
    int row_off;    // first output row (chunk start)
    int out_fp32;
  };
  __device__ __forceinline__ static void prefetch(const Params&, int, int, int, int) {}
  __device__ __forceinline__ static void run(const Params& p, uint32_t taddr, int row0, int n0,
                                             int quad, int lane) {
    const int rq = lane >> 2, cs = (lane & 3) * 2;
#pragma unroll 1
    for (int c = 0; c < TC_EPI_COLS / 32; ++c) {
      const int col0 = n0 + c * 32;
      if (col0 >= p.cols) break;  // warp-uniform
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v[16];
        tmem_ld16x32(taddr + (static_cast<uint32_t>(16 * h) << 16) + c * 32, v);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = row0 + quad * 32 + 16 * h + 8 * e + rq;
          if (r >= p.rows) continue;
          const size_t orow = static_cast<size_t>(p.row_off + r) * p.ld;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int col = col0 + 8 * j;
            if (col >= p.cols) continue;
            const float a = v[4 * j + 2 * e], b = v[4 * j + 2 * e + 1];
            if (p.out_fp32)
              *reinterpret_cast<float2*>(static_cast<float*>(p.out) + orow + col + cs) =
                  make_float2(a, b);
            else
              *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(p.out) + orow + col + cs) =
                  pack_bf16x2(a, b);
          }
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
  __device__ __forceinline__ static void prefetch(const Params& p, int row0, int n0, int quad,
                                                  int lane) {
    const int r = row0 + quad * 32 + lane;
    if ((p.mode == 2 || p.mode == 3) && r < p.rows && n0 < p.cols) {
      const float* q = p.part + static_cast<size_t>(r) * p.ld + n0;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (n0 + 32 * j < p.cols) prefetch_l2(q + 32 * j);
    }
  }
  __device__ __forceinline__ static void run(const Params& p, uint32_t taddr, int row0, int n0,
                                             int quad, int lane) {
    const int rq = lane >> 2, cs = (lane & 3) * 2;
    const bool rd = p.mode == 2 || p.mode == 3, wr_part = p.mode == 1 || p.mode == 2;
#pragma unroll 1
    for (int c = 0; c < TC_EPI_COLS / 32; ++c) {
      const int col0 = n0 + c * 32;
      if (col0 >= p.cols) break;  // warp-uniform
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v[16];
        tmem_ld16x32(taddr + (static_cast<uint32_t>(16 * h) << 16) + c * 32, v);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = row0 + quad * 32 + 16 * h + 8 * e + rq;
          if (r >= p.rows) continue;
          const size_t orow = static_cast<size_t>(r) * p.ld;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int col = col0 + 8 * j;
            if (col >= p.cols) continue;
            float a = v[4 * j + 2 * e], b = v[4 * j + 2 * e + 1];
            float2* pp = reinterpret_cast<float2*>(p.part + orow + col + cs);
            if (rd) {
              const float2 o = *pp;
              a += o.x;
              b += o.y;
            }
            if (wr_part)
              *pp = make_float2(a, b);
            else
              *reinterpret_cast<uint32_t*>(p.out + orow + col + cs) = pack_bf16x2(a, b);
          }
        }
      }
    }
  }
};

// ====================================================================
// Launch descriptor: up to three GEMM problems served by one persistent
// launch.  Their tiles form one sequence [problem 0 tiles, problem 1 tiles,
// ...]; CTA pairs claim tiles in that order from a global counter, so the
// longest tiles (placed first) start first and the shortest fill the end.

enum TcKind : int {
  KIND_STATS = 0,  // z tile -> softmax/KL statistics      A = X (K-major), B = W (K-major)
  KIND_GRAD = 1,   // z tile -> G staging (+ db partials)   A = X (K-major), B = W (K-major)
  KIND_DW = 2,     // dW rows = G^T X                       A = G (MN-major), B = X (MN-major)
  KIND_DX = 3,     // dX (+)= G W                           A = G (K-major), B = W (MN-major)
  KIND_JSD = 4     // student z tile -> JSD partials / G     A = X (K-major), B = W (K-major)
};
__host__ __device__ constexpr bool kind_a_mn(int k) { return k == KIND_DW; }
__host__ __device__ constexpr bool kind_b_mn(int k) { return k == KIND_DW || k == KIND_DX; }

constexpr int TC_MAX_PROBLEMS = 3;
constexpr int TC_SLOTS = 4;  // depth of the tile-id ring

struct TcProblem {
  int kind;
  int a_blocked, b_blocked;  // A / B use 3-D blocked tensor maps
  int m_tiles, n_tiles;   // 256 x 256 tiles
  int num_kb;             // K / 64, rounded up
  int m_fastest;          // tile order inside the problem
  int a_m_off, a_k_off;   // offsets added to A tile coordinates
  int b_n_off, b_k_off;   // offsets added to B tile coordinates
  int tile_begin;         // first tile of the problem in the launch sequence
};

struct TcMaps {
  CUtensorMap m[2 * TC_MAX_PROBLEMS];  // A and B of each problem
};

struct TcLaunch {
  int nprob;
  int total_tiles;
  TcProblem prob[TC_MAX_PROBLEMS];
  int* counter;  // tile counter of this launch, 0 at launch
  int* err_flag;
  unsigned long long wait_limit_ns;
  EpiStats::Params stats;
  EpiGrad::Params grad;
  EpiStoreRows::Params dw;
  EpiAccumRows::Params dx;
  EpiJsd::Params jsd;
};

// Problem and local tile index of sequence position t: the problems' tiles
// follow one another in problem order.
__device__ __forceinline__ int find_problem(const TcLaunch& L, int t, int& local) {
  int pi = 0;
  while (pi + 1 < L.nprob && t >= L.prob[pi + 1].tile_begin) ++pi;
  local = t - L.prob[pi].tile_begin;
  return pi;
}

__device__ __forceinline__ void problem_tile(const TcProblem& P, int local, int& mb, int& nb) {
  if (P.m_fastest) {
    mb = local % P.m_tiles;
    nb = local / P.m_tiles;
  } else {
    nb = local % P.n_tiles;
    mb = local / P.n_tiles;
  }
}

template <class F>
__device__ __forceinline__ void dispatch_epilogue(const TcLaunch& L, int kind, F&& f) {
  switch (kind) {
    case KIND_STATS: f(EpiStats{}, L.stats); break;
    case KIND_GRAD: f(EpiGrad{}, L.grad); break;
    case KIND_DW: f(EpiStoreRows{}, L.dw); break;
    case KIND_JSD: f(EpiJsd{}, L.jsd); break;
    default: f(EpiAccumRows{}, L.dx); break;
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(TC_THREADS, 1)
    tc_group_kernel(const __grid_constant__ TcMaps maps, const __grid_constant__ TcLaunch L) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + TC_STAGES * TC_A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + TC_STAGES * TC_B_BYTES);
  uint64_t* full = bars;                       // [STAGES] TMA -> MMA (even CTA's are used)
  uint64_t* empty = full + TC_STAGES;          // [STAGES] MMA -> TMA (each CTA)
  uint64_t* tfull = empty + TC_STAGES;         // [2] MMA -> epilogue (each CTA)
  uint64_t* tempty = tfull + 2;                // [2] epilogues -> MMA (even CTA's are used)
  uint64_t* drain = tempty + 2;                // MMA drain at exit (even CTA)
  uint64_t* tid_full = drain + 1;              // [SLOTS] tile id published (each CTA)
  uint64_t* tid_empty = tid_full + TC_SLOTS;   // [SLOTS] tile id read (even CTA's are used)
  int* tile_id = reinterpret_cast<int*>(tid_empty + TC_SLOTS);  // [SLOTS]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_id + TC_SLOTS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * TC_EPI_WARPS);  // every epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    for (int k = 0; k < TC_SLOTS; ++k) {
      mbar_init(&tid_full[k], 1);
      // readers of a tile id: the MMA thread, the odd CTA's producer, every epilogue warp
      mbar_init(&tid_empty[k], 2 + 2 * TC_EPI_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < 2 * L.nprob; ++i) tma_prefetch_desc(&maps.m[i]);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TC_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers are initialised before anything targets them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, L.err_flag, L.wait_limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ producer
      int slot = 0, stage = 0, issued = 0;
      uint32_t sph = 0, phase = 0;
      bool ok = true;
      // the even CTA claims one tile ahead, so the atomic's round trip
      // overlaps the loads of the current tile
      int claimed = leader ? atomicAdd(L.counter, 1) : 0;
      while (ok) {
        int t;
        if (leader) {
          // publish the claimed tile to both CTAs of the pair
          if (!mbar_wait(&tid_empty[slot], sph ^ 1u, wc)) break;
          t = claimed;
          if (t < L.total_tiles) claimed = atomicAdd(L.counter, 1);
          tile_id[slot] = t;
          st_shared_cluster_u32(mapa_shared(smem_u32(&tile_id[slot]), 1),
                                static_cast<uint32_t>(t));
          mbar_arrive(&tid_full[slot]);
          mbar_arrive_cluster(mapa_shared(smem_u32(&tid_full[slot]), 1));
        } else {
          if (!mbar_wait_cluster(&tid_full[slot], sph, wc)) break;
          t = tile_id[slot];
          mbar_arrive_cluster(mapa_shared(smem_u32(&tid_empty[slot]), 0));
        }
        if (++slot == TC_SLOTS) {
          slot = 0;
          sph ^= 1u;
        }
        if (t >= L.total_tiles) break;
        int local;
        const int pi = find_problem(L, t, local);
        const TcProblem& P = L.prob[pi];
        const bool a_mn = kind_a_mn(P.kind), b_mn = kind_b_mn(P.kind);
        int mb, nb;
        problem_tile(P, local, mb, nb);
        const int m0 = mb * TC_BM + static_cast<int>(rank) * TC_HM + P.a_m_off;
        const int n0 = nb * TC_BN + static_cast<int>(rank) * TC_HM + P.b_n_off;
        const CUtensorMap* mA = &maps.m[2 * pi];
        const CUtensorMap* mB = &maps.m[2 * pi + 1];
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * TC_STAGE_BYTES);
          tma_half_stage(mA, a_mn, P.a_blocked, fbar, sA + stage * TC_A_BYTES, m0,
                         kb * TC_BK + P.a_k_off);
          tma_half_stage(mB, b_mn, P.b_blocked, fbar, sB + stage * TC_B_BYTES, n0,
                         kb * TC_BK + P.b_k_off);
          ++issued;
          if (++stage == TC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every stage this CTA filled must have been consumed by the
      // pair's MMAs (their commit arrives on `empty`) before the CTA exits.
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < TC_STAGES && i < issued; ++i) {
        if (--s < 0) {
          s = TC_STAGES - 1;
          ph ^= 1u;
        }
        mbar_drain_wait(&empty[s], ph, L.wait_limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------ MMA issuer
      int slot = 0, stage = 0, it = 0;
      uint32_t sph = 0, phase = 0;
      bool ok = true;
      while (ok) {
        if (!mbar_wait(&tid_full[slot], sph, wc)) break;
        const int t = tile_id[slot];
        mbar_arrive(&tid_empty[slot]);
        if (++slot == TC_SLOTS) {
          slot = 0;
          sph ^= 1u;
        }
        if (t >= L.total_tiles) break;
        int local;
        const TcProblem& P = L.prob[find_problem(L, t, local)];
        const bool a_mn = kind_a_mn(P.kind), b_mn = kind_b_mn(P.kind);
        const uint32_t idesc = idesc_bf16_f32(TC_BM, TC_BN, a_mn, b_mn);
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * TC_BN;
        // Descriptors of this tile: a constant upper word (SBO, version,
        // swizzle) and a lower word (LBO | start address >> 4) that only moves
        // by fixed steps between K slices and stages (see stage_desc).
        // (the start-address field holds bits [4, 18) of the CTA's shared
        // address; a shared address may carry the CTA's rank above them)
        const DescSteps da = desc_steps(a_mn), db = desc_steps(b_mn);
        const uint32_t a_lo0 = da.lo_base + ((smem_u32(sA) & 0x3FFFFu) >> 4);
        const uint32_t b_lo0 = db.lo_base + ((smem_u32(sB) & 0x3FFFFu) >> 4);
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_lo = a_lo0 + stage * (TC_A_BYTES >> 4);
          const uint32_t b_lo = b_lo0 + stage * (TC_B_BYTES >> 4);
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k) {
            const uint64_t adesc =
                (static_cast<uint64_t>(da.hi) << 32) | (a_lo + (k & 3) * da.s1 + (k >> 2) * da.s2);
            const uint64_t bdesc =
                (static_cast<uint64_t>(db.hi) << 32) | (b_lo + (k & 3) * db.s1 + (k >> 2) * db.s2);
            tc_mma_pair_f16(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit_pair(&empty[stage], 0x3);
          if (++stage == TC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit_pair(&tfull[acc], 0x3);
        ++it;
      }
      // Drain every MMA this thread issued before TMEM is released.
      tc_commit_pair(drain, 0x1);
      mbar_drain_wait(drain, 0, L.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------- epilogue
    const int quad = warp & 3;         // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;  // which 128 accumulator columns
    const int rbase = static_cast<int>(rank) * TC_HM;
    int slot = 0, it = 0;
    uint32_t sph = 0;
    while (true) {
      if (!mbar_wait_cluster(&tid_full[slot], sph, wc)) break;
      const int t = tile_id[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tid_empty[slot]), 0));
      if (++slot == TC_SLOTS) {
        slot = 0;
        sph ^= 1u;
      }
      if (t >= L.total_tiles) break;
      int local;
      const TcProblem& P = L.prob[find_problem(L, t, local)];
      int mb, nb;
      problem_tile(P, local, mb, nb);
      const int row0 = mb * TC_BM + rbase;
      const int n0 = nb * TC_BN + half * TC_EPI_COLS;
      dispatch_epilogue(L, P.kind, [&](auto epi, const auto& prm) {
        decltype(epi)::prefetch(prm, row0, n0, quad, lane);
      });
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_phase, wc)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * TC_BN +
                             half * TC_EPI_COLS;
      dispatch_epilogue(L, P.kind, [&](auto epi, const auto& prm) {
        decltype(epi)::run(prm, taddr, row0, n0, quad, lane);
      });
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      ++it;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA frees TMEM or leaves while the pair still works
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TC_TMEM_COLS);
  }
}

}  // namespace flkl
