// Stage 2: block pooling, block proxy scores and the two selection modes
// (DynamicRad, Sec. 3.2 and Algorithm 1, selection steps, in block-pooled form).
//
// Two launches:
//
//   pool_kernel    one CTA per (tensor, head, 8 consecutive blocks): each warp
//                  streams one block (B_s x D bf16, 16-byte loads), shuffle-reduces,
//                  and writes the fp32 mean -- qbar row-major [BH, Nb, D], kbar
//                  transposed [BH, D, NbP] through a shared-memory transpose so the
//                  score loads below are coalesced.  HBM-bound.
//   select_kernel  one CTA per (head, 8 consecutive query blocks): the union of the
//                  8 candidate lists is scored once per key block (each kbar value
//                  read feeds 8 dot products, packed f32x2 FMAs), then each warp
//                  selects for its row by a 4-pass radix descent over
//                  order-preserving score keys.
//
// Ranking: (score descending, block index ascending).  Scores compare as
// numbers: -0 is folded into +0 before the key is formed.  Static mode weighs
// every candidate 1 and looks for the first k of the ranking.  Dynamic mode
// weighs candidate J by e_J = exp(s_J - max s) (fp64) quantised to 36-bit
// fixed point, so every mass sum is an exact, order-independent integer sum;
// it looks for the shortest ranking prefix whose weight, added to the forced
// weight, reaches tau * Z.
//
//   scan_*_kernel        kept counts -> CSR row offsets.
//   compact_kernel       per-row kept lists -> col_idx (one warp per row).
#pragma once

#include "common.cuh"

namespace dynrad {

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

constexpr int kSelRows = 8;                   // query blocks per score item (one warp each)
constexpr int kS2Threads = kSelRows * 32;     // 8 warps
constexpr double kMassScale = 68719476736.0;  // 2^36 fixed-point scale of e_J

// Padded block count of the transposed kbar: rows of 128 bytes.
__host__ __device__ constexpr int padded_blocks(int nb) { return (nb + 31) & ~31; }

struct Stage2Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  float* qbar;              // [BH, nb, D]
  float* kbarT;             // [BH, D, nbp]
  const int32_t* cand_row_ptr;
  const int32_t* cand_col;
  const int32_t* forced_lo;
  const int32_t* forced_hi;
  int32_t* counts;          // kept count per row (row_ptr before the scan)
  int32_t* kept_tmp;        // [BH, cand_nnz] kept lists at the candidate offsets
  float* scores_out;        // nullable (caller's export of the scores)
  float* scores;            // [BH, cand_nnz] scores used by the selection
  int32_t* plan_off;        // [groups] first plan entry of each group of 8 rows
  int32_t* plan_cnt;        // [groups] union size of each group
  int32_t* plan_alloc;      // [1] plan entries handed out (zeroed before the plan kernel)
  int32_t* plan_J;          // [cand_nnz] union members (key blocks), per group ascending
  int32_t* plan_pos;        // [cand_nnz][8] score position of (entry, row) in the row's list, or -1
  int rows_bh;              // B * H
  int64_t cand_nnz;
  int N;
  int block;
  int nb;
  int nbp;
  int max_row;              // bound on candidates per row (smem sizing)
  int mode;
  double value;             // rho or tau
  float scale;              // 1 / sqrt(D)
};

// Order-preserving key of a finite float: larger key <=> larger number.
__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u << 1) == 0u) u = 0u;  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__device__ __forceinline__ uint64_t warp_excl_scan_u64(uint64_t v, int lane) {
  uint64_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  return incl - v;
}

// Selection predicate: has the accumulated weight reached the target?
struct Reach {
  bool dynamic;
  uint64_t k;       // static: number of free blocks to keep
  uint64_t base;    // dynamic: forced weight
  double tau_z;     // dynamic: tau * Z (Z < 2^53, so all sums convert exactly)
  __device__ __forceinline__ bool operator()(uint64_t w) const {
    return dynamic ? static_cast<double>(base + w) >= tau_z : w >= k;
  }
};

// Pool item: warp w pools block 8*grp + w of one (tensor, head).
template <int D>
__device__ __forceinline__ void pool_item(const Stage2Params& p, bool is_k, int bh, int grp,
                                          float* tile) {
  constexpr int LPR = D / 8;      // lanes per token row (8 bf16 = 16 B each)
  constexpr int RPI = 32 / LPR;   // token rows per warp iteration
  constexpr int UNROLL = 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = grp * kSelRows + warp;
  const int sub = lane / LPR;
  const int c8 = (lane % LPR) * 8;
  if (blk < p.nb) {
    const int t0 = blk * p.block;
    const int nvalid = min(p.block, p.N - t0);
    const __nv_bfloat16* src = (is_k ? p.k : p.q) + (static_cast<size_t>(bh) * p.N + t0) * D;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    int t = sub;
    for (; t + (UNROLL - 1) * RPI < nvalid; t += UNROLL * RPI) {
      uint4 v[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) v[u] = ldg_stream(src + static_cast<size_t>(t + u * RPI) * D + c8);
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) acc_bf16x8(acc, v[u]);
    }
    for (; t < nvalid; t += RPI) acc_bf16x8(acc, ldg_stream(src + static_cast<size_t>(t) * D + c8));
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
    if (sub == 0) {
      const float inv = static_cast<float>(nvalid);
      if (!is_k) {
        float* dst = p.qbar + (static_cast<int64_t>(bh) * p.nb + blk) * D + c8;
        reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0] / inv, acc[1] / inv, acc[2] / inv, acc[3] / inv);
        reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4] / inv, acc[5] / inv, acc[6] / inv, acc[7] / inv);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) tile[warp * D + c8 + i] = acc[i] / inv;
      }
    }
  }
  if (is_k) {
    // transpose the 8 blocks' means: kbarT[bh][d][8*grp + w], 32-byte runs
    __syncthreads();
    const int nvb = min(kSelRows, p.nb - grp * kSelRows);
    float* dstT = p.kbarT + static_cast<int64_t>(bh) * D * p.nbp + grp * kSelRows;
    for (int i = threadIdx.x; i < kSelRows * D; i += kS2Threads) {
      const int d = i / kSelRows, w = i % kSelRows;
      if (w < nvb) dstT[static_cast<int64_t>(d) * p.nbp + w] = tile[w * D + d];
    }
  }
}

// Pool: one CTA per (tensor, head, 8 consecutive blocks); many CTAs per SM keep
// enough loads in flight to run at HBM bandwidth.
template <int D>
__global__ void __launch_bounds__(kS2Threads, 4) pool_kernel(Stage2Params p) {
  __shared__ __align__(16) float tile[kSelRows * D];
  const int nq = (p.nb + kSelRows - 1) / kSelRows;
  const int grp = blockIdx.x % nq;
  const bool is_k = (blockIdx.x / nq) != 0;
  pool_item<D>(p, is_k, blockIdx.y, grp, tile);
}

// ---------------------------------------------------------------------------
// Scoring, in two kernels.
//
// plan_kernel, one CTA per group of 8 consecutive query blocks, from the
// candidate CSR alone (the same for every head): the union of the 8 candidate
// lists and, for each (union member J, row r), the position of J in row r's
// list -- its rank, from per-row bitmaps and prefix popcounts -- or -1 if row
// r does not list J or needs no score for it.  Union sizes are a fraction of
// the 8 rows' total, so the entries fit in cand_nnz; a counter hands out the
// space.
//
// score_kernel, one CTA per (head, group): every union member's kbar column is
// read once and feeds 8 dot products; the scores go to their positions in the
// per-candidate array [BH, cand_nnz].
// ---------------------------------------------------------------------------
__host__ __device__ constexpr size_t plan_smem_bytes(int nb) {
  // union bitmap + prefix, 8 row bitmaps + prefixes, 8 "needs a score" bitmaps,
  // union list
  return static_cast<size_t>((nb + 31) / 32) * 4 * (2 + 3 * kSelRows) + static_cast<size_t>(nb) * 4 + 64;
}

__global__ void __launch_bounds__(kS2Threads) plan_kernel(Stage2Params p) {
  extern __shared__ __align__(16) uint8_t pl_smem[];
  const int nb = p.nb;
  const int nwords = (nb + 31) >> 5;
  uint32_t* ubits = reinterpret_cast<uint32_t*>(pl_smem);                 // [nwords]
  uint32_t* rbits = ubits + nwords;                                       // [8][nwords]
  int32_t* upre = reinterpret_cast<int32_t*>(rbits + kSelRows * nwords);  // [nwords]
  int32_t* rpre = upre + nwords;                                          // [8][nwords]
  uint32_t* nbits = reinterpret_cast<uint32_t*>(rpre + kSelRows * nwords);  // [8][nwords]
  int32_t* ulist = reinterpret_cast<int32_t*>(nbits + kSelRows * nwords);  // [nb]
  __shared__ int u_total, u_off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = blockIdx.x;
  const int I0 = grp * kSelRows;
  const bool dynamic = p.mode == DYNRAD_DYNAMIC_THRESHOLD;
  // static mode without score export never needs the forced blocks' scores
  const bool skip_forced = !dynamic && p.scores_out == nullptr;

  for (int i = threadIdx.x; i < kSelRows * nwords; i += kS2Threads) {
    rbits[i] = 0u;
    nbits[i] = 0u;
  }
  __syncthreads();
  // row bitmaps (warp r owns row I0 + r): every candidate (for ranks) and the
  // candidates that need a score
  const int I = I0 + warp;
  if (I < nb) {
    const int c_beg = p.cand_row_ptr[I];
    const int n = p.cand_row_ptr[I + 1] - c_beg;
    const int flo = p.forced_lo[I], fhi = p.forced_hi[I];
    // the list is sorted, so lanes sharing a bitmap word are adjacent: OR their
    // bits within the warp, one shared-memory update per word
    for (int c0 = 0; c0 < n; c0 += 32) {
      const int c = c0 + lane;
      const bool in = c < n;
      const int J = in ? p.cand_col[c_beg + c] : 0;
      const int w = in ? (J >> 5) : -1 - lane;
      const uint32_t bit = in ? 1u << (J & 31) : 0u;
      const uint32_t need = (in && (!skip_forced || J < flo || J > fhi)) ? bit : 0u;
      const unsigned grp_lanes = __match_any_sync(0xffffffffu, w);
      const uint32_t all_bits = __reduce_or_sync(grp_lanes, bit);
      const uint32_t need_bits = __reduce_or_sync(grp_lanes, need);
      if (in && lane == __ffs(grp_lanes) - 1) {
        rbits[warp * nwords + w] |= all_bits;
        nbits[warp * nwords + w] |= need_bits;
      }
      __syncwarp();
    }
  }
  __syncthreads();
  // union bitmap
  for (int w = threadIdx.x; w < nwords; w += kS2Threads) {
    uint32_t u = 0;
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) u |= nbits[r * nwords + w];
    ubits[w] = u;
  }
  __syncthreads();
  // prefix popcounts: warp r for row r; warp 0 also for the union
  for (int which = warp; which <= kSelRows; which += kSelRows) {
    const uint32_t* bits = which < kSelRows ? rbits + which * nwords : ubits;
    int32_t* pre = which < kSelRows ? rpre + which * nwords : upre;
    int carry = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int w = w0 + lane;
      const int c = w < nwords ? __popc(bits[w]) : 0;
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (w < nwords) pre[w] = carry + incl - c;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (which == kSelRows && lane == 0) u_total = carry;
  }
  __syncthreads();
  // union list, one word per warp iteration; space for this group's entries
  for (int w = warp; w < nwords; w += kSelRows) {
    const uint32_t bits = ubits[w];
    if ((bits >> lane) & 1u) ulist[upre[w] + __popc(bits & ((1u << lane) - 1u))] = (w << 5) + lane;
  }
  if (threadIdx.x == 0) {
    int off = atomicAdd(p.plan_alloc, u_total);
    if (static_cast<int64_t>(off) + u_total > p.cand_nnz) {   // cannot happen for a valid CSR
      record_error(DYNRAD_ERR_CAPACITY);
      off = -1;
    }
    u_off = off;
    p.plan_off[grp] = off < 0 ? 0 : off;
    p.plan_cnt[grp] = off < 0 ? 0 : u_total;
  }
  __syncthreads();
  const int U = u_total, off = u_off;
  if (off < 0) return;
  for (int u = threadIdx.x; u < U; u += kS2Threads) {
    const int J = ulist[u];
    const int w = J >> 5;
    const uint32_t below = (1u << (J & 31)) - 1u;
    p.plan_J[off + u] = J;
    int32_t pos[kSelRows];
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) {
      const bool has = I0 + r < nb && ((nbits[r * nwords + w] >> (J & 31)) & 1u);
      pos[r] = has ? p.cand_row_ptr[I0 + r] + rpre[r * nwords + w] + __popc(rbits[r * nwords + w] & below) : -1;
    }
    int4* dst = reinterpret_cast<int4*>(p.plan_pos + static_cast<int64_t>(off + u) * kSelRows);
    dst[0] = make_int4(pos[0], pos[1], pos[2], pos[3]);
    dst[1] = make_int4(pos[4], pos[5], pos[6], pos[7]);
  }
}

template <int D>
__global__ void __launch_bounds__(kS2Threads, 3) score_kernel(Stage2Params p) {
  __shared__ __align__(16) float qsT[D * kSelRows];   // [D][8]
  const int nb = p.nb;
  const int bh = blockIdx.y;
  const int grp = blockIdx.x;
  const int I0 = grp * kSelRows;
  for (int i = threadIdx.x; i < kSelRows * D; i += kS2Threads) {
    const int r = i / D, d = i % D;
    qsT[d * kSelRows + r] = (I0 + r < nb) ? p.qbar[(static_cast<int64_t>(bh) * nb + I0 + r) * D + d] : 0.f;
  }
  __syncthreads();
  const int U = p.plan_cnt[grp], off = p.plan_off[grp];
  const float* kT = p.kbarT + static_cast<int64_t>(bh) * D * p.nbp;
  float* out = p.scores + static_cast<int64_t>(bh) * p.cand_nnz;
  for (int u0 = threadIdx.x; u0 < U; u0 += 2 * kS2Threads) {
    const int u1 = u0 + kS2Threads;
    const int J0 = p.plan_J[off + u0];
    const int J1 = u1 < U ? p.plan_J[off + u1] : J0;
    float2 a0[4], a1[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      a0[r] = make_float2(0.f, 0.f);
      a1[r] = make_float2(0.f, 0.f);
    }
#pragma unroll 16
    for (int d = 0; d < D; ++d) {
      const float k0 = __ldg(kT + static_cast<int64_t>(d) * p.nbp + J0);
      const float k1 = __ldg(kT + static_cast<int64_t>(d) * p.nbp + J1);
      const float4 qa = reinterpret_cast<const float4*>(qsT + d * kSelRows)[0];
      const float4 qb = reinterpret_cast<const float4*>(qsT + d * kSelRows)[1];
      const float2 kk0 = make_float2(k0, k0), kk1 = make_float2(k1, k1);
      const float2 q01 = make_float2(qa.x, qa.y), q23 = make_float2(qa.z, qa.w);
      const float2 q45 = make_float2(qb.x, qb.y), q67 = make_float2(qb.z, qb.w);
      a0[0] = __ffma2_rn(q01, kk0, a0[0]);
      a0[1] = __ffma2_rn(q23, kk0, a0[1]);
      a0[2] = __ffma2_rn(q45, kk0, a0[2]);
      a0[3] = __ffma2_rn(q67, kk0, a0[3]);
      a1[0] = __ffma2_rn(q01, kk1, a1[0]);
      a1[1] = __ffma2_rn(q23, kk1, a1[1]);
      a1[2] = __ffma2_rn(q45, kk1, a1[2]);
      a1[3] = __ffma2_rn(q67, kk1, a1[3]);
    }
    // scatter to the rows that need each block's score
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (e == 1 && u1 >= U) break;
      const int u = e == 0 ? u0 : u1;
      const int4* pp = reinterpret_cast<const int4*>(p.plan_pos + static_cast<int64_t>(off + u) * kSelRows);
      const int4 pa = __ldg(pp), pb = __ldg(pp + 1);
      const int pos[kSelRows] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int r = 0; r < kSelRows; ++r) {
        if (pos[r] >= 0) {
          const float2 v = e == 0 ? a0[r >> 1] : a1[r >> 1];
          out[pos[r]] = ((r & 1) ? v.y : v.x) * p.scale;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Selection: one warp per query block; the row's candidates (block, score,
// weight) live in registers, E per lane; a 2 x 256 x u32 bin array in shared
// memory per warp holds the radix histograms.
// ---------------------------------------------------------------------------
constexpr int kSelWarps = 8;

template <int E, bool DYN>
__global__ void __launch_bounds__(kSelWarps * 32, DYN ? (E <= 4 ? 4 : (E <= 8 ? 3 : (E <= 16 ? 2 : 1)))
                                                      : (E <= 8 ? 4 : (E <= 16 ? 3 : 2)))
    select_kernel(Stage2Params p) {
  __shared__ uint32_t bins_all[kSelWarps][512];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* bins = bins_all[warp];
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kSelWarps + warp;
  const int64_t rows = static_cast<int64_t>(p.nb) * p.rows_bh;
  if (row >= rows) return;
  const int64_t bh = row / p.nb;
  const int I = static_cast<int>(row - bh * p.nb);
  const int c_beg = p.cand_row_ptr[I];
  int n = p.cand_row_ptr[I + 1] - c_beg;
  if (n > 32 * E || n < 0) {  // longer than the declared bound: the row stays empty
    if (lane == 0) {
      record_error(DYNRAD_ERR_CAPACITY);
      p.counts[row] = 0;
    }
    return;
  }
  const int flo = p.forced_lo[I], fhi = p.forced_hi[I];
  constexpr bool dynamic = DYN;
  const float* srow = p.scores + bh * p.cand_nnz + c_beg;
  int32_t Jv[DYN ? E : 1];
  uint32_t key[E];
  uint64_t wgt[DYN ? E : 1];
  // weight of element i (static: 1 for every free block)
  auto wof = [&](int i) -> uint64_t {
    if constexpr (DYN) return wgt[i];
    else return 1;
  };
  uint32_t forced = 0, valid = 0;   // bit i: element i of this lane
  float smax = -INFINITY;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int c = lane + 32 * i;
    if constexpr (DYN) {
      Jv[i] = 0;
      wgt[i] = 0;
    }
    key[i] = 0;
    if (c < n) {
      const int J = p.cand_col[c_beg + c];
      const bool f = J >= flo && J <= fhi;
      if constexpr (DYN) Jv[i] = J;
      valid |= 1u << i;
      forced |= (f ? 1u : 0u) << i;
      const float sc = (f && !dynamic) ? 0.f : srow[c];
      key[i] = order_key(sc);
      if (dynamic) smax = fmaxf(smax, sc);
    }
  }
  uint64_t base = 0, ztot = 0;
  int nfree = 0;
  if (dynamic) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, off));
  }
#pragma unroll
  for (int i = 0; i < E; ++i) {
    if ((valid >> i) & 1u) {
      uint64_t w = 1;
      if constexpr (DYN) {
        const double e = exp(static_cast<double>(srow[lane + 32 * i]) - static_cast<double>(smax));
        w = __double2ull_rn(e * kMassScale);
        wgt[i] = ((forced >> i) & 1u) ? 0 : w;
      }
      if ((forced >> i) & 1u) base += w;
      else ++nfree;
      ztot += w;
    }
  }
  base = warp_sum_u64(base);
  ztot = warp_sum_u64(ztot);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) nfree += __shfl_xor_sync(0xffffffffu, nfree, off);
  const uint32_t freev = valid & ~forced;

  Reach reach;
  reach.dynamic = dynamic;
  reach.base = base;
  reach.k = 0;
  reach.tau_z = 0.0;
  bool keep_all = false;
  if (dynamic) {
    if (p.value >= 1.0) keep_all = true;
    else reach.tau_z = __dmul_rn(p.value, static_cast<double>(ztot));
  } else if (nfree > 0) {
    const double kf = floor(__dadd_rn(__dmul_rn(p.value, static_cast<double>(nfree)), 1e-9));
    reach.k = kf < 1.0 ? 1ull : static_cast<uint64_t>(kf);
    if (reach.k > static_cast<uint64_t>(nfree)) reach.k = nfree;
  }

  uint32_t kstar = 0xFFFFFFFFu;  // cut key; free blocks with key > kstar are kept
  uint64_t above = 0;            // weight of free blocks with key > kstar
  const bool cut_none = !keep_all && reach(0);
  if (!keep_all && !cut_none) {
    // the free keys agree above their highest differing bit: start there
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
    for (int i = 0; i < E; ++i)
      if ((freev >> i) & 1u) {
        kmin = min(kmin, key[i]);
        kmax = max(kmax, key[i]);
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
    }
    const int top = (kmin == kmax) ? -1 : 31 - __clz(kmin ^ kmax);  // highest differing bit
    uint32_t pmask = top >= 31 ? 0u : (0xFFFFFFFFu << (top + 1));
    uint32_t prefix = kmax & pmask;
    bool found = true;
    for (int hi = top; hi >= 0 && found; hi -= 8) {
      const int shift = hi >= 7 ? hi - 7 : 0;
      const uint32_t dmask = (1u << (hi - shift + 1)) - 1u;
#pragma unroll
      for (int i = 0; i < 16; ++i) bins[lane * 16 + i] = 0u;
      __syncwarp();
      // weights < 2^36 are split into 18-bit halves; each half's bin sum stays
      // below 2^32 for rows of up to 2^14 candidates
#pragma unroll
      for (int i = 0; i < E; ++i) {
        if (((freev >> i) & 1u) && (key[i] & pmask) == prefix) {
          const uint32_t b = (key[i] >> shift) & dmask;
          const uint64_t w = wof(i);
          atomicAdd(&bins[b], static_cast<uint32_t>(w & 0x3FFFFu));
          if (w >> 18) atomicAdd(&bins[256 + b], static_cast<uint32_t>(w >> 18));
        }
      }
      __syncwarp();
      // lane l owns digits 255-8l ... 248-8l (descending)
      uint64_t loc[8], lsum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t b = 255 - (lane * 8 + i);
        loc[i] = (static_cast<uint64_t>(bins[256 + b]) << 18) + bins[b];
        lsum += loc[i];
      }
      const uint64_t excl = warp_excl_scan_u64(lsum, lane);
      const unsigned hit = __ballot_sync(0xffffffffu, reach(above + excl + lsum));
      if (hit == 0u) {
        found = false;
        break;
      }
      const int src = __ffs(hit) - 1;
      uint32_t digit = 0;
      uint64_t new_above = 0;
      if (lane == src) {
        uint64_t run = above + excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (reach(run + loc[i])) {
            digit = 255u - static_cast<uint32_t>(lane * 8 + i);
            new_above = run;
            break;
          }
          run += loc[i];
        }
      }
      digit = __shfl_sync(0xffffffffu, digit, src);
      above = __shfl_sync(0xffffffffu, new_above, src);
      prefix |= digit << shift;
      pmask |= dmask << shift;
      __syncwarp();
    }
    if (found) kstar = prefix;
    else keep_all = true;  // target not reachable (rounding at tau ~ 1): keep all
  }

  // kept: forced, free with key > kstar, and ties at kstar in ascending order
  // until the target is reached; written ascending
  uint32_t kept = forced;
  if (!cut_none) {
    uint64_t tie_run = 0;
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const bool fr = (freev >> i) & 1u;
      bool k_ = fr && (keep_all || key[i] > kstar);
      const bool tie = !keep_all && fr && key[i] == kstar;
      // ties are few (usually the cut element alone): scan only where they are
      const unsigned tb = __ballot_sync(0xffffffffu, tie);
      if (tb != 0u) {
        uint64_t ex, sum;
        if constexpr (DYN) {
          const uint64_t tw = tie ? wof(i) : 0;
          ex = warp_excl_scan_u64(tw, lane);
          sum = warp_sum_u64(tw);
        } else {   // unit weights: ranks from the ballot
          ex = static_cast<uint64_t>(__popc(tb & lt_mask));
          sum = static_cast<uint64_t>(__popc(tb));
        }
        if (tie && !reach(above + tie_run + ex)) k_ = true;
        tie_run += sum;
      }
      kept |= (k_ ? 1u : 0u) << i;
    }
  }
  int32_t* dst = p.kept_tmp + bh * p.cand_nnz + c_beg;
  int cnt = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const bool k_ = (kept >> i) & 1u;
    const unsigned bal = __ballot_sync(0xffffffffu, k_);
    if (k_) {
      int32_t J;
      if constexpr (DYN) J = Jv[i];
      else J = p.cand_col[c_beg + lane + 32 * i];
      dst[cnt + __popc(bal & ((1u << lane) - 1u))] = J;
    }
    cnt += __popc(bal);
  }
  if (lane == 0) p.counts[row] = cnt;
}

// ---------------------------------------------------------------------------
// counts -> row offsets, and compaction of the kept lists
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 1024;
constexpr int kScanItems = 4;
constexpr int kScanTile = kScanThreads * kScanItems;

__global__ void __launch_bounds__(kScanThreads) scan_partial_kernel(const int32_t* counts,
                                                                    int64_t rows,
                                                                    int64_t* partial) {
  __shared__ int64_t ws[32];
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * kScanTile;
  int64_t s = 0;
  for (int i = threadIdx.x; i < kScanTile; i += kScanThreads) {
    const int64_t r = b0 + i;
    if (r < rows) s += counts[r];
  }
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t t = 0;
    for (int w = 0; w < 32; ++w) t += ws[w];
    partial[blockIdx.x] = t;
  }
}

struct CompactParams {
  int32_t* row_ptr;            // in: counts, out: offsets
  const int64_t* partial;
  int64_t rows;                // B*H*nb
  int nb;
  const int32_t* cand_row_ptr;
  const int32_t* kept_tmp;
  int64_t cand_nnz;
  int32_t* col_idx;
  int64_t col_cap;
};

__global__ void __launch_bounds__(kScanThreads) scan_apply_kernel(CompactParams p) {
  __shared__ int64_t offs[kScanTile + 1];
  __shared__ int64_t ws[32];
  __shared__ int64_t base_s;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * kScanTile;
  // prefix of the tiles before this one
  int64_t pre = 0;
  for (int i = threadIdx.x; i < static_cast<int>(blockIdx.x); i += kScanThreads) pre += p.partial[i];
  for (int off = 16; off > 0; off >>= 1) pre += __shfl_xor_sync(0xffffffffu, pre, off);
  if (lane == 0) ws[warp] = pre;
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t t = 0;
    for (int w = 0; w < 32; ++w) t += ws[w];
    base_s = t;
  }
  __syncthreads();
  // local exclusive scan: thread i owns items [i*4, i*4+4)
  int64_t v[kScanItems], tsum = 0;
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    const int64_t r = b0 + threadIdx.x * kScanItems + j;
    v[j] = r < p.rows ? p.row_ptr[r] : 0;
    tsum += v[j];
  }
  int64_t incl = tsum;
  for (int off = 1; off < 32; off <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  __syncthreads();
  if (lane == 31) ws[warp] = incl;
  __syncthreads();
  int64_t wbefore = 0;
  for (int w = 0; w < warp; ++w) wbefore += ws[w];
  int64_t run = base_s + wbefore + incl - tsum;
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    offs[threadIdx.x * kScanItems + j] = run;
    run += v[j];
  }
  if (threadIdx.x == kScanThreads - 1) offs[kScanTile] = run;
  __syncthreads();
  for (int i = threadIdx.x; i < kScanTile; i += kScanThreads) {
    const int64_t r = b0 + i;
    if (r < p.rows) {
      const int64_t o = offs[i];
      if (o > INT32_MAX) record_error(DYNRAD_ERR_CAPACITY);
      p.row_ptr[r] = o > INT32_MAX ? INT32_MAX : static_cast<int32_t>(o);
    }
  }
  // the grand total, one past the last row, is written by the last tile
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
    const int64_t o = offs[p.rows - b0];
    if (o > INT32_MAX) record_error(DYNRAD_ERR_CAPACITY);
    p.row_ptr[p.rows] = o > INT32_MAX ? INT32_MAX : static_cast<int32_t>(o);
  }
}


// Copies every row's kept list from the candidate-offset scratch to its CSR
// position: one warp per row.
constexpr int kCompactThreads = 256;

__global__ void __launch_bounds__(kCompactThreads) compact_kernel(CompactParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * kCompactThreads + threadIdx.x) >> 5;
  if (r >= p.rows) return;
  const int64_t bh = r / p.nb;
  const int I = static_cast<int>(r - bh * p.nb);
  const int64_t o = p.row_ptr[r];
  const int64_t cnt = static_cast<int64_t>(p.row_ptr[r + 1]) - o;
  const int32_t* src = p.kept_tmp + bh * p.cand_nnz + p.cand_row_ptr[I];
  for (int64_t c = lane; c < cnt; c += 32) {
    const int64_t d = o + c;
    if (d < p.col_cap) p.col_idx[d] = src[c];
    else record_error(DYNRAD_ERR_CAPACITY);
  }
}

}  // namespace dynrad
