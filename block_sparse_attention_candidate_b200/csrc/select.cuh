// Stage 2: block pooling, block proxy scores and the two selection modes
// (DynamicRad, Sec. 3.2 and Algorithm 1, selection steps, in block-pooled form).
//
// One launch, stage2_kernel, whose CTAs take work items from a ticket counter
// (details above the kernel):
//
//   plan    per group of 8 query blocks (all heads): the union of their
//           candidate lists and each member's position in each row's list.
//   pool    per (tensor, head, 8 blocks): each warp streams one block (B_s x D
//           bf16, 16-byte loads), shuffle-reduces, and writes the fp32 mean --
//           qbar row-major [BH, Nb, D], kbar transposed [BH, D, NbP] through a
//           shared-memory transpose so the score loads are coalesced.  HBM-bound.
//   select  per (head, group of 8 query blocks): the union is scored once per
//           key block (each kbar value read feeds 8 dot products, packed f32x2
//           FMAs) into shared memory, each warp selects for its row by a radix
//           descent over order-preserving score keys; the kept lists go to
//           their CSR positions (static mode) or through a scan and a
//           compaction (dynamic mode).
//
// Ranking: (score descending, block index ascending).  Scores compare as
// numbers: -0 is folded into +0 before the key is formed.  Static mode weighs
// every candidate 1 and looks for the first k of the ranking.  Dynamic mode
// weighs candidate J by e_J = exp(s_J - max s) (fp64) quantised to 36-bit
// fixed point, so every mass sum is an exact, order-independent integer sum;
// it looks for the shortest ranking prefix whose weight, added to the forced
// weight, reaches tau * Z.
//
// The scan_* and compact kernels at the end serve the other mask builders.
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

struct Stage2Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  float* qbar;              // [BH, nb, D]
  float* kbar;              // [BH, nb, D]
  const int32_t* cand_row_ptr;
  const int32_t* cand_col;
  const int32_t* forced_lo;
  const int32_t* forced_hi;
  int32_t* row_ptr;         // output CSR [BH * nb + 1] (dynamic mode: the kept counts, scanned afterwards)
  int32_t* col_idx;         // output [col_cap] (static mode)
  int64_t col_cap;
  int32_t* kept_tmp;        // dynamic mode: [BH, cand_nnz] kept lists at the candidate offsets
  float* scores_out;        // nullable (caller's export of the scores)
  int32_t* plan_off;        // [nq] first plan entry of each group of 8 rows
  int32_t* plan_cnt;        // [nq] union size of each group
  int32_t* plan_J;          // [cand_nnz] union members (key blocks), per group ascending
  int32_t* plan_pos;        // [cand_nnz][8] score position of (entry, row) in the row's list, or -1
  int32_t* plan_rows;       // [nq] static mode: kept blocks of the group's 8 rows (the same for every head)
  // per-call counters, zeroed before the launch
  unsigned long long* ticket;   // next work item
  int32_t* plan_alloc;      // plan entries handed out
  int32_t* plan_done;       // plan items finished
  int32_t* pool_done;       // [BH] pool items finished per head
  int rows_bh;              // B * H
  int64_t cand_nnz;
  int N;
  int block;
  int nb;
  int nq;                   // groups of 8 rows
  int max_row;              // bound on candidates per row
  int span_cap;             // score slots of a group in shared memory (8 * max_row, rounded up to 4)
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

// Pool item: warp w pools block 8*grp + w of one (tensor, head) into qbar or
// kbar (both [BH, Nb, D] fp32, row-major).
template <int D>
__device__ __forceinline__ void pool_item(const Stage2Params& p, bool is_k, int bh, int grp) {
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
      float* dst = (is_k ? p.kbar : p.qbar) + (static_cast<int64_t>(bh) * p.nb + blk) * D + c8;
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0] / inv, acc[1] / inv, acc[2] / inv, acc[3] / inv);
      reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4] / inv, acc[5] / inv, acc[6] / inv, acc[7] / inv);
    }
  }
}

// ---------------------------------------------------------------------------
// The stage-2 launch.  One kernel runs three kinds of work item in the order a
// global ticket counter hands them out.  A CTA draws its ticket when it starts,
// so every item with a smaller ticket belongs to a CTA that is running or done:
// waiting on such an item always ends.
//
//   plan    one per group of 8 consecutive query blocks, from the candidate CSR
//           alone (the same for every head): the union of the 8 candidate lists
//           and, for each (member J, row r), the position of J in row r's list
//           (its rank, from per-row bitmaps and prefix popcounts), or -1 if row
//           r does not list J or needs no score for it.  A counter hands out
//           the space; the unions' total is at most cand_nnz.
//   pool    one per (tensor, head, 8 blocks): the fp32 block means (pool_item).
//   select  one per (head, group): the group's candidate scores into shared
//           memory (each union member's kbar column is read once and feeds 8
//           dot products), and one warp per row selects.  Static mode: the
//           kept counts follow from the candidate lists alone (the plan sums
//           them per group), so the kept lists go straight to their CSR
//           positions.  Dynamic mode: the kept lists go to the rows' candidate
//           offsets and the counts to row_ptr; a scan and a compaction follow.
//
// Ticket order: the plan items, then per head h the pool items of h followed
// by the select items of head h - kS2Lag, so the HBM-bound pooling of later
// heads runs beside the ALU-bound selection of earlier ones.  A select item
// waits for the whole plan and for its head's pooling.  Every wait is bounded (kWaitLimitNs); on expiry
// the device status records DYNRAD_ERR_DEVICE and the item carries on.
// ---------------------------------------------------------------------------
constexpr int kS2Lag = 2;   // heads between a head's pooling and its selection, in ticket order

struct S2Item {
  int kind;   // 0 plan, 1 pool, 2 select
  int bh;
  int idx;    // plan / select: group; pool: [0, nq) Q groups, [nq, 2 nq) K groups
};

__host__ __device__ inline int64_t s2_tickets(int nq, int bh_total) {
  return static_cast<int64_t>(nq) * (1 + 3 * static_cast<int64_t>(bh_total));
}

__device__ __forceinline__ S2Item s2_item(int64_t t, int nq, int bh_total) {
  S2Item it{0, 0, 0};
  if (t < nq) {
    it.idx = static_cast<int>(t);
    return it;
  }
  t -= nq;
  const int64_t p2 = 2ll * nq, p3 = 3ll * nq;
  const int64_t lead = bh_total < kS2Lag ? bh_total : kS2Lag;   // heads pooled before any selection
  if (t < lead * p2) {
    it.kind = 1;
    it.bh = static_cast<int>(t / p2);
    it.idx = static_cast<int>(t % p2);
    return it;
  }
  t -= lead * p2;
  const int64_t mixed = bh_total > kS2Lag ? bh_total - kS2Lag : 0;   // pool h, then select h - lag
  if (t < mixed * p3) {
    const int s = static_cast<int>(t / p3), r = static_cast<int>(t % p3);
    if (r < p2) {
      it.kind = 1;
      it.bh = kS2Lag + s;
      it.idx = r;
    } else {
      it.kind = 2;
      it.bh = s;
      it.idx = r - static_cast<int>(p2);
    }
    return it;
  }
  t -= mixed * p3;
  it.kind = 2;
  it.bh = static_cast<int>(mixed + t / nq);
  it.idx = static_cast<int>(t % nq);
  return it;
}

__host__ __device__ constexpr size_t plan_smem_bytes(int nb) {
  // union bitmap + prefix, 8 row bitmaps + prefixes, 8 "needs a score" bitmaps,
  // union list
  return static_cast<size_t>((nb + 31) / 32) * 4 * (2 + 3 * kSelRows) + static_cast<size_t>(nb) * 4 + 64;
}

// Shared memory of a select item: qbar^T [D][8] fp32, 8 per-warp bin arrays of
// 2 x 256 u32, the group's scores [span_cap] fp32 and, in dynamic mode, the
// free candidates' weights [span_cap] u64.
__host__ __device__ constexpr size_t select_smem_bytes(int d, int span_cap, bool dyn) {
  return static_cast<size_t>(d) * kSelRows * 4 + kSelRows * 512 * 4 + static_cast<size_t>(span_cap) * 4 +
         (dyn ? static_cast<size_t>(span_cap) * 8 : 0);
}

__device__ void plan_item(const Stage2Params& p, int grp, uint8_t* smem) {
  const int nb = p.nb;
  const int nwords = (nb + 31) >> 5;
  uint32_t* ubits = reinterpret_cast<uint32_t*>(smem);                    // [nwords]
  uint32_t* rbits = ubits + nwords;                                       // [8][nwords]
  int32_t* upre = reinterpret_cast<int32_t*>(rbits + kSelRows * nwords);  // [nwords]
  int32_t* rpre = upre + nwords;                                          // [8][nwords]
  uint32_t* nbits = reinterpret_cast<uint32_t*>(rpre + kSelRows * nwords);  // [8][nwords]
  int32_t* ulist = reinterpret_cast<int32_t*>(nbits + kSelRows * nwords);  // [nb]
  __shared__ int u_total, u_off, s_rowcnt[kSelRows];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
  int nforced = 0;
  if (I < nb) {
    const int c_beg = p.cand_row_ptr[I];
    const int n = p.cand_row_ptr[I + 1] - c_beg;
    const int flo = p.forced_lo[I], fhi = p.forced_hi[I];
    // lanes sharing a bitmap word OR their bits within the warp: one
    // shared-memory update per word
    for (int c0 = 0; c0 < n; c0 += 32) {
      const int c = c0 + lane;
      const bool in = c < n;
      const int J = in ? p.cand_col[c_beg + c] : 0;
      const bool ok = in && J >= 0 && J < nb;
      const int w = ok ? (J >> 5) : -1 - lane;
      const uint32_t bit = ok ? 1u << (J & 31) : 0u;
      const uint32_t need = (ok && (!skip_forced || J < flo || J > fhi)) ? bit : 0u;
      nforced += __popc(__ballot_sync(0xffffffffu, in && J >= flo && J <= fhi));
      const unsigned grp_lanes = __match_any_sync(0xffffffffu, w);
      const uint32_t all_bits = __reduce_or_sync(grp_lanes, bit);
      const uint32_t need_bits = __reduce_or_sync(grp_lanes, need);
      if (ok && lane == __ffs(grp_lanes) - 1) {
        rbits[warp * nwords + w] |= all_bits;
        nbits[warp * nwords + w] |= need_bits;
      }
      __syncwarp();
    }
  }
  // static mode: the row's kept count follows from the list alone -- the
  // forced blocks plus k of the free ones (0 for a row the selection rejects)
  if (!dynamic && lane == 0) {
    int cnt = 0;
    if (I < nb) {
      const int c_beg = p.cand_row_ptr[I];
      const int n = p.cand_row_ptr[I + 1] - c_beg;
      const int loc = c_beg - p.cand_row_ptr[I0];
      if (!(n < 0 || n > p.max_row || loc < 0 || loc + n > p.span_cap)) {
        const int nfree = n - nforced;
        int k = 0;
        if (nfree > 0) {
          const double kf = floor(__dadd_rn(__dmul_rn(p.value, static_cast<double>(nfree)), 1e-9));
          k = kf < 1.0 ? 1 : (kf > static_cast<double>(nfree) ? nfree : static_cast<int>(kf));
        }
        cnt = nforced + k;
      }
    }
    s_rowcnt[warp] = cnt;
  }
  __syncthreads();
  if (!dynamic && threadIdx.x == 0) {
    int tot = 0;
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) tot += s_rowcnt[r];
    p.plan_rows[grp] = tot;
  }
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
  const int U = u_off < 0 ? 0 : u_total, off = u_off;
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
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) red_release_add_s32(p.plan_done, 1);
}

template <int D>
__device__ __forceinline__ void pool_work(const Stage2Params& p, int bh, int idx) {
  const bool is_k = idx >= p.nq;
  pool_item<D>(p, is_k, bh, is_k ? idx - p.nq : idx);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) red_release_add_s32(p.pool_done + bh, 1);
}

// Selection of one row by one warp, from the row's scores in shared memory
// (srow[c], c in [0, n), list order).  wrow receives the dynamic weights of the
// free candidates.  Returns the kept mask: bit i of lane l is list position
// l + 32 i (n <= 1024).
//
// The cut key k* is found digit by digit over the free candidates' order keys
// (a radix descent, most significant digit first): at each level the free
// keys under the current prefix are binned by their next 8 bits and weighed,
// and the first bin (descending) at which the accumulated weight reaches the
// target extends the prefix.  Bits that all remaining keys share are skipped,
// and the descent stops as soon as the remaining keys are all equal.
template <bool DYN, int E>
__device__ __forceinline__ uint32_t select_row(const Stage2Params& p, int I, int n, int c_beg,
                                               const float* srow, uint64_t* wrow, uint32_t* bins,
                                               int lane) {
  const int ne = (n + 31) >> 5;   // <= E
  const int flo = p.forced_lo[I], fhi = p.forced_hi[I];
  uint32_t forced = 0u, valid = 0u;
#pragma unroll 2
  for (int i = 0; i < ne; ++i) {
    const int c = lane + 32 * i;
    if (c < n) {
      const int J = p.cand_col[c_beg + c];
      valid |= 1u << i;
      if (J >= flo && J <= fhi) forced |= 1u << i;
    }
  }
  const uint32_t freev = valid & ~forced;
  int nfree = __popc(freev);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) nfree += __shfl_xor_sync(0xffffffffu, nfree, off);

  Reach reach;
  reach.dynamic = DYN;
  reach.base = 0;
  reach.k = 0;
  reach.tau_z = 0.0;
  bool keep_all = false;
  if constexpr (DYN) {
    float smax = -INFINITY;
#pragma unroll 2
    for (int i = 0; i < ne; ++i)
      if ((valid >> i) & 1u) smax = fmaxf(smax, srow[lane + 32 * i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, off));
    uint64_t base = 0, ztot = 0;
#pragma unroll 2
    for (int i = 0; i < ne; ++i) {
      if ((valid >> i) & 1u) {
        const int c = lane + 32 * i;
        const double e = exp(static_cast<double>(srow[c]) - static_cast<double>(smax));
        const uint64_t w = __double2ull_rn(e * kMassScale);
        const bool f = (forced >> i) & 1u;
        wrow[c] = f ? 0 : w;
        if (f) base += w;
        ztot += w;
      }
    }
    reach.base = warp_sum_u64(base);
    ztot = warp_sum_u64(ztot);
    if (p.value >= 1.0) keep_all = true;
    else reach.tau_z = __dmul_rn(p.value, static_cast<double>(ztot));
    __syncwarp();
  } else if (nfree > 0) {
    const double kf = floor(__dadd_rn(__dmul_rn(p.value, static_cast<double>(nfree)), 1e-9));
    reach.k = kf < 1.0 ? 1ull : static_cast<uint64_t>(kf);
    if (reach.k > static_cast<uint64_t>(nfree)) reach.k = nfree;
  }
  auto wof = [&](int c) -> uint64_t {
    if constexpr (DYN) return wrow[c];
    else return 1;
  };

  uint32_t kstar = 0xFFFFFFFFu;  // cut key; free blocks with key > kstar are kept
  uint64_t above = 0;            // weight of free blocks with key > kstar
  const bool cut_none = !keep_all && reach(0);
  if (!keep_all && !cut_none) {
    uint32_t prefix = 0u, pmask = 0u;
    while (true) {
      uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll 2
      for (int i = 0; i < ne; ++i) {
        if ((freev >> i) & 1u) {
          const uint32_t k = order_key(srow[lane + 32 * i]);
          if ((k & pmask) == prefix) {
            kmin = min(kmin, k);
            kmax = max(kmax, k);
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
      }
      if (kmin == kmax) {   // one key value left under the prefix: it is the cut
        kstar = kmin;
        break;
      }
      // they agree above their highest differing bit; the next digit ends there
      const int top = 31 - __clz(kmin ^ kmax);
      pmask = top >= 31 ? 0u : (0xFFFFFFFFu << (top + 1));
      prefix = kmax & pmask;
      const int shift = top >= 7 ? top - 7 : 0;
      const uint32_t dmask = (1u << (top - shift + 1)) - 1u;
      // 256 bins of counts (static mode) or, in dynamic mode, of weights
      // < 2^36 split into 18-bit halves in two banks (each half's bin sum stays
      // below 2^32 for rows of up to 2^14 candidates; two 32-bit shared atomics
      // measured faster than one 64-bit one)
      constexpr int kBanks = DYN ? 2 : 1;
#pragma unroll
      for (int i = 0; i < 8 * kBanks; ++i) bins[lane * 8 * kBanks + i] = 0u;
      __syncwarp();
#pragma unroll 2
      for (int i = 0; i < ne; ++i) {
        if ((freev >> i) & 1u) {
          const int c = lane + 32 * i;
          const uint32_t k = order_key(srow[c]);
          if ((k & pmask) == prefix) {
            const uint32_t b = (k >> shift) & dmask;
            if constexpr (DYN) {
              const uint64_t w = wof(c);
              atomicAdd(&bins[b], static_cast<uint32_t>(w & 0x3FFFFu));
              if (w >> 18) atomicAdd(&bins[256 + b], static_cast<uint32_t>(w >> 18));
            } else {
              atomicAdd(&bins[b], 1u);
            }
          }
        }
      }
      __syncwarp();
      // lane l owns digits 255-8l ... 248-8l (descending)
      uint64_t loc[8], lsum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t b = 255 - (lane * 8 + i);
        if constexpr (DYN) loc[i] = (static_cast<uint64_t>(bins[256 + b]) << 18) + bins[b];
        else loc[i] = bins[b];
        lsum += loc[i];
      }
      const uint64_t excl = warp_excl_scan_u64(lsum, lane);
      const unsigned hit = __ballot_sync(0xffffffffu, reach(above + excl + lsum));
      if (hit == 0u) {   // target not reachable (rounding at tau ~ 1): keep all
        keep_all = true;
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
  }

  // kept: forced, free with key > kstar, and ties at kstar in list order
  // until the target is reached
  uint32_t kept = forced;
  if (!cut_none) {
    uint64_t tie_run = 0;
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll 2
    for (int i = 0; i < ne; ++i) {
      const int c = lane + 32 * i;
      const bool fr = (freev >> i) & 1u;
      const uint32_t k = fr ? order_key(srow[c]) : 0u;
      bool k_ = fr && (keep_all || k > kstar);
      const bool tie = !keep_all && fr && k == kstar;
      // ties are few (usually the cut element alone): scan only where they are
      const unsigned tb = __ballot_sync(0xffffffffu, tie);
      if (tb != 0u) {
        uint64_t ex, sum;
        if constexpr (DYN) {
          const uint64_t tw = tie ? wrow[c] : 0;
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
  return kept;
}

template <int D, bool DYN, int E>
__device__ __forceinline__ void select_item(const Stage2Params& p, int bh, int grp, uint8_t* smem) {
  float* qsT = reinterpret_cast<float*>(smem);                          // [D][8]
  uint32_t* bins_all = reinterpret_cast<uint32_t*>(qsT + D * kSelRows);   // [8][512]
  float* sc = reinterpret_cast<float*>(bins_all + kSelRows * 512);        // [span_cap]
  uint64_t* wg = reinterpret_cast<uint64_t*>(sc + p.span_cap);            // [span_cap] (dynamic)
  __shared__ int s_cnt[kSelRows];
  __shared__ long long s_excl;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = p.nb, I0 = grp * kSelRows;
  if (threadIdx.x == 0) {
    wait_at_least(p.plan_done, p.nq);
    wait_at_least(p.pool_done + bh, 2 * p.nq);
  }
  __syncthreads();
  // qbar, kbar and the plan were written earlier in this launch: plain
  // (coherent) loads, no read-only path
  for (int i = threadIdx.x; i < kSelRows * D; i += kS2Threads) {
    const int r = i / D, d = i % D;
    qsT[d * kSelRows + r] = (I0 + r < nb) ? p.qbar[(static_cast<int64_t>(bh) * nb + I0 + r) * D + d] : 0.f;
  }
  __syncthreads();
  if constexpr (!DYN) {
    // static mode: the group's first CSR offset (heads before this one, then
    // groups before this one) comes from the plan's per-group counts, known
    // now; warp 0 sums them here so the loads overlap the scoring
    if (warp == 0) {
      int64_t before = 0, total = 0;
      for (int x = lane; x < p.nq; x += 32) {
        const int64_t c = p.plan_rows[x];
        total += c;
        if (x < grp) before += c;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        before += __shfl_xor_sync(0xffffffffu, before, o);
        total += __shfl_xor_sync(0xffffffffu, total, o);
      }
      if (lane == 0) {
        s_excl = static_cast<int64_t>(bh) * total + before;
        if (bh == p.rows_bh - 1 && grp == p.nq - 1)
          p.row_ptr[static_cast<int64_t>(p.rows_bh) * nb] = static_cast<int32_t>(static_cast<int64_t>(p.rows_bh) * total);
      }
    }
  }
  const int c0 = p.cand_row_ptr[I0];
  {
    // Scoring: a pair of threads per two union members.  Each thread of the
    // pair loads every other 16-byte chunk of both members' kbar rows (the
    // pair covers each 32-byte sector in one instruction), accumulates the 8
    // rows' partial dot products over its chunks, and one shuffle joins the
    // halves; thread 0 of the pair stores the first member's 8 scores, thread
    // 1 the second's.
    constexpr int kChunks = D / 4;             // float4 chunks per kbar row
    constexpr int kMine = kChunks / 2;         // chunks per thread
    constexpr int kUnr = 2;                    // chunks per member in flight
    const int U = p.plan_cnt[grp], off = p.plan_off[grp];
    const float* kb = p.kbar + static_cast<int64_t>(bh) * nb * D;
    float* exp_out = p.scores_out != nullptr ? p.scores_out + static_cast<int64_t>(bh) * p.cand_nnz : nullptr;
    const int half = threadIdx.x & 1, pair = threadIdx.x >> 1;
    constexpr int kPairs = kS2Threads / 2;
    // every thread runs every iteration (the shuffles below need the whole
    // warp); a pair past the union's end reads member 0 and stores nothing
    for (int ub = 0; ub < U; ub += 2 * kPairs) {
      const int u0 = ub + pair, u1 = u0 + kPairs;
      const int J0 = p.plan_J[off + (u0 < U ? u0 : 0)];
      const int J1 = u1 < U ? p.plan_J[off + u1] : J0;
      const float4* r0 = reinterpret_cast<const float4*>(kb + static_cast<int64_t>(J0) * D) + half;
      const float4* r1 = reinterpret_cast<const float4*>(kb + static_cast<int64_t>(J1) * D) + half;
      float2 a0[4], a1[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        a0[r] = make_float2(0.f, 0.f);
        a1[r] = make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int c0_ = 0; c0_ < kMine; c0_ += kUnr) {
        float4 k0v[kUnr], k1v[kUnr];
#pragma unroll
        for (int x = 0; x < kUnr; ++x) {
          k0v[x] = r0[2 * (c0_ + x)];
          k1v[x] = r1[2 * (c0_ + x)];
        }
#pragma unroll
        for (int x = 0; x < kUnr; ++x) {
          const int d0 = 4 * (2 * (c0_ + x) + half);
          const float k0s[4] = {k0v[x].x, k0v[x].y, k0v[x].z, k0v[x].w};
          const float k1s[4] = {k1v[x].x, k1v[x].y, k1v[x].z, k1v[x].w};
#pragma unroll
          for (int dd = 0; dd < 4; ++dd) {
            const float4 qa = reinterpret_cast<const float4*>(qsT + (d0 + dd) * kSelRows)[0];
            const float4 qb = reinterpret_cast<const float4*>(qsT + (d0 + dd) * kSelRows)[1];
            const float2 kk0 = make_float2(k0s[dd], k0s[dd]), kk1 = make_float2(k1s[dd], k1s[dd]);
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
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        a0[r].x += __shfl_xor_sync(0xffffffffu, a0[r].x, 1);
        a0[r].y += __shfl_xor_sync(0xffffffffu, a0[r].y, 1);
        a1[r].x += __shfl_xor_sync(0xffffffffu, a1[r].x, 1);
        a1[r].y += __shfl_xor_sync(0xffffffffu, a1[r].y, 1);
      }
      // thread `half` of the pair scatters member u_half to the rows needing it
      const int u = half == 0 ? u0 : u1;
      if (u < U) {
        const int4* pp = reinterpret_cast<const int4*>(p.plan_pos + static_cast<int64_t>(off + u) * kSelRows);
        const int4 pa = pp[0], pb = pp[1];
        const int pos[kSelRows] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
        for (int r = 0; r < kSelRows; ++r) {
          if (pos[r] >= 0) {
            const float2 v = half == 0 ? a0[r >> 1] : a1[r >> 1];
            const float sv = ((r & 1) ? v.y : v.x) * p.scale;
            const int loc = pos[r] - c0;
            if (loc >= 0 && loc < p.span_cap) sc[loc] = sv;
            if (exp_out != nullptr) exp_out[pos[r]] = sv;
          }
        }
      }
    }
  }
  __syncthreads();
  // selection: warp r for row I0 + r
  const int I = I0 + warp;
  uint32_t kept = 0u;
  int n = 0, c_beg = 0, cnt = 0;
  if (I < nb) {
    c_beg = p.cand_row_ptr[I];
    n = p.cand_row_ptr[I + 1] - c_beg;
    const int loc = c_beg - c0;
    if (n < 0 || n > p.max_row || loc < 0 || loc + n > p.span_cap) {   // beyond the declared bound: empty
      if (lane == 0) record_error(DYNRAD_ERR_CAPACITY);
      n = 0;
    } else if (n > 0) {
      kept = select_row<DYN, E>(p, I, n, c_beg, sc + loc, wg + loc, bins_all + warp * 512, lane);
      const int ne = (n + 31) >> 5;
#pragma unroll 2
      for (int i = 0; i < ne; ++i)
        cnt += __popc(__ballot_sync(0xffffffffu, (kept >> i) & 1u));
    }
  }
  if (lane == 0) s_cnt[warp] = cnt;
  __syncthreads();
  if constexpr (DYN) {
    // kept lists at the rows' candidate offsets and the counts in row_ptr;
    // a scan and a compaction follow
    if (I < nb) {
      const int64_t row = static_cast<int64_t>(bh) * nb + I;
      if (lane == 0) p.row_ptr[row] = cnt;
      int32_t* dst = p.kept_tmp + static_cast<int64_t>(bh) * p.cand_nnz + c_beg;
      const int ne = (n + 31) >> 5;
      int run = 0;
#pragma unroll 2
      for (int i = 0; i < ne; ++i) {
        {
          const bool k_ = (kept >> i) & 1u;
          const unsigned bal = __ballot_sync(0xffffffffu, k_);
          if (k_) dst[run + __popc(bal & ((1u << lane) - 1u))] = p.cand_col[c_beg + lane + 32 * i];
          run += __popc(bal);
        }
      }
    }
  } else {
    // static counts are the same for every head (from the plan): the group's
    // first CSR offset is the heads before this one plus the groups before it
    if (threadIdx.x == 0) {
      int tot = 0;
#pragma unroll
      for (int r = 0; r < kSelRows; ++r) tot += s_cnt[r];
      if (tot != p.plan_rows[grp]) record_error(DYNRAD_ERR_DEVICE);   // cannot happen: same rule
    }
    if (I < nb) {
      int64_t o = s_excl;
      for (int r = 0; r < warp; ++r) o += s_cnt[r];
      if (lane == 0) p.row_ptr[static_cast<int64_t>(bh) * nb + I] = static_cast<int32_t>(o);
      const int ne = (n + 31) >> 5;
      int run = 0;
#pragma unroll 2
      for (int i = 0; i < ne; ++i) {
        {
          const bool k_ = (kept >> i) & 1u;
          const unsigned bal = __ballot_sync(0xffffffffu, k_);
          if (k_) {
            const int64_t d = o + run + __popc(bal & ((1u << lane) - 1u));
            if (d < p.col_cap) p.col_idx[d] = p.cand_col[c_beg + lane + 32 * i];
            else record_error(DYNRAD_ERR_CAPACITY);
          }
          run += __popc(bal);
        }
      }
    }
  }
}

template <int D, bool DYN, int E>
__global__ void __launch_bounds__(kS2Threads, 4) stage2_kernel(Stage2Params p) {
  extern __shared__ __align__(16) uint8_t s2_smem[];
  __shared__ long long s_ticket;
  if (threadIdx.x == 0) s_ticket = atomicAdd(p.ticket, 1ull);
  __syncthreads();
  const S2Item it = s2_item(s_ticket, p.nq, p.rows_bh);
  if (it.kind == 0) plan_item(p, it.idx, s2_smem);
  else if (it.kind == 1) pool_work<D>(p, it.bh, it.idx);
  else select_item<D, DYN, E>(p, it.bh, it.idx, s2_smem);
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
