// Stage 2: block pooling, block proxy scores and the two selection modes
// (DynamicRad, Sec. 3.2 and Algorithm 1 lines 15-22, in block-pooled form).
//
//   pool_kernel          qbar, kbar = fp32 means of Q, K over each block's valid
//                        tokens.  HBM-bound: one warp streams one 64x128 bf16
//                        block with 16-byte loads, shuffle-reduces, writes 512 B.
//   score_select_kernel  one CTA = 8 consecutive query blocks of one head.  The
//                        union of their candidate lists is scored once per key
//                        block (register blocking over the 8 rows: each kbar row
//                        read from L2 feeds 8 dot products), then each warp
//                        selects for its row by a 4-pass radix descent over the
//                        order-preserving 32-bit score keys.
//   scan_*_kernel        kept counts -> CSR row offsets, and compaction of the
//                        per-row kept lists into col_idx.
//
// Ranking: (score descending, block index ascending).  Scores compare as
// numbers: -0 is folded into +0 before the key is formed.  Static mode weighs
// every candidate 1 and looks for the first k of the ranking.  Dynamic mode
// weighs candidate J by e_J = exp(s_J - max s) (fp64) quantised to 36-bit
// fixed point, so every mass sum is an exact, order-independent integer sum;
// it looks for the shortest ranking prefix whose weight, added to the forced
// weight, reaches tau * Z.
#pragma once

#include "common.cuh"

namespace dynrad {

// ---------------------------------------------------------------------------
// pooling
// ---------------------------------------------------------------------------
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

constexpr int kPoolThreads = 256;

// One warp per (tensor in {Q, K}, b*H + h, block).
template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                            const __nv_bfloat16* __restrict__ k,
                                                            float* __restrict__ qbar,
                                                            float* __restrict__ kbar, int N,
                                                            int block, int nb, int64_t rows) {
  constexpr int LPR = D / 8;      // lanes per token row (8 bf16 = 16 B each)
  constexpr int RPI = 32 / LPR;   // token rows per warp iteration
  constexpr int UNROLL = 8;
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * kPoolThreads + threadIdx.x) >> 5;
  if (wid >= 2 * rows) return;
  const bool is_k = wid >= rows;
  const int64_t r = is_k ? wid - rows : wid;
  const int64_t bh = r / nb;
  const int blk = static_cast<int>(r - bh * nb);
  const int t0 = blk * block;
  const int nvalid = min(block, N - t0);
  const __nv_bfloat16* src = (is_k ? k : q) + (static_cast<size_t>(bh) * N + t0) * D;
  const int sub = lane / LPR;
  const int c8 = (lane % LPR) * 8;
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
    float* dst = (is_k ? kbar : qbar) + r * D + c8;
    const float inv = static_cast<float>(nvalid);
    float4 a = make_float4(acc[0] / inv, acc[1] / inv, acc[2] / inv, acc[3] / inv);
    float4 b = make_float4(acc[4] / inv, acc[5] / inv, acc[6] / inv, acc[7] / inv);
    reinterpret_cast<float4*>(dst)[0] = a;
    reinterpret_cast<float4*>(dst)[1] = b;
  }
}

// ---------------------------------------------------------------------------
// scoring + selection
// ---------------------------------------------------------------------------
constexpr int kSelRows = 8;                 // query blocks per CTA (one warp each)
constexpr int kSelThreads = kSelRows * 32;
constexpr double kMassScale = 68719476736.0;  // 2^36 fixed-point scale of e_J

struct SelectParams {
  const float* qbar;
  const float* kbar;
  const int32_t* cand_row_ptr;
  const int32_t* cand_col;
  const int32_t* forced_lo;
  const int32_t* forced_hi;
  int32_t* counts;      // kept count per row (row_ptr before the scan)
  int32_t* kept_tmp;    // [BH, cand_nnz] kept lists at the candidate offsets
  float* scores_out;    // nullable
  int64_t cand_nnz;
  int nb;
  int max_row;          // bound on candidates per row (smem sizing)
  int mode;
  double value;         // rho or tau
  float scale;          // 1 / sqrt(D)
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

// Per-warp selection scratch in shared memory: bins[256] u64, weights[cap] u64,
// keys[cap] u32, flags[cap] u8, rounded to 16 bytes.
__host__ __device__ constexpr size_t sel_warp_bytes(int cap) {
  return (2048 + static_cast<size_t>(cap) * 13 + 15) & ~static_cast<size_t>(15);
}

// Dynamic shared memory of score_select_kernel.
__host__ __device__ constexpr size_t sel_smem_bytes(int D, int nb, int cap) {
  return ((static_cast<size_t>(kSelRows) * D * 4 + static_cast<size_t>((nb + 31) / 32) * 4 +
           static_cast<size_t>((nb + 31) / 32 + 1) * 4 + static_cast<size_t>(nb) * 4 +
           static_cast<size_t>(kSelRows) * nb * 4 + 15) & ~static_cast<size_t>(15)) +
         kSelRows * sel_warp_bytes(cap);
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) score_select_kernel(SelectParams p) {
  extern __shared__ __align__(16) uint8_t sel_smem[];
  const int nb = p.nb;
  const int nwords = (nb + 31) >> 5;
  const int cap = p.max_row;
  // shared layout
  float* qs = reinterpret_cast<float*>(sel_smem);                          // [8][D]
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(qs + kSelRows * D);       // [nwords]
  int32_t* wprefix = reinterpret_cast<int32_t*>(bitmap + nwords);          // [nwords + 1]
  int32_t* ulist = wprefix + nwords + 1;                                   // [nb]
  float* S = reinterpret_cast<float*>(ulist + nb);                         // [8][nb]
  uintptr_t wp = reinterpret_cast<uintptr_t>(S + static_cast<size_t>(kSelRows) * nb);
  wp = (wp + 15) & ~static_cast<uintptr_t>(15);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // per-warp arrays: bins[256] u64, wgt[cap] u64, key[cap] u32, flag[cap] u8
  uint8_t* wbase = reinterpret_cast<uint8_t*>(wp) + static_cast<size_t>(warp) * sel_warp_bytes(cap);
  uint64_t* bins = reinterpret_cast<uint64_t*>(wbase);
  uint64_t* wgt = bins + 256;
  uint32_t* key = reinterpret_cast<uint32_t*>(wgt + cap);
  uint8_t* flag = reinterpret_cast<uint8_t*>(key + cap);

  const int64_t bh = blockIdx.y;
  const int I0 = blockIdx.x * kSelRows;
  const int I = I0 + warp;
  const bool row_ok = I < nb;

  // 1. pooled queries of the 8 rows; clear the union bitmap
  for (int i = threadIdx.x; i < kSelRows * D; i += kSelThreads) {
    const int r = i / D;
    qs[i] = (I0 + r < nb) ? p.qbar[(bh * nb + I0 + r) * D + (i % D)] : 0.f;
  }
  for (int i = threadIdx.x; i < nwords; i += kSelThreads) bitmap[i] = 0u;
  __syncthreads();

  // 2. union of the 8 candidate lists
  int c_beg = 0, n = 0;
  if (row_ok) {
    c_beg = p.cand_row_ptr[I];
    n = p.cand_row_ptr[I + 1] - c_beg;
    if (n > cap || n < 0) {  // longer than the declared bound: the row stays empty
      if (lane == 0) {
        record_error(DYNRAD_ERR_CAPACITY);
        p.counts[bh * nb + I] = 0;
      }
      n = 0;
    }
    for (int c = lane; c < n; c += 32) {
      const int J = p.cand_col[c_beg + c];
      atomicOr(&bitmap[J >> 5], 1u << (J & 31));
    }
  }
  __syncthreads();

  // 3. rank of every union member (word prefix popcounts) and the union list
  if (warp == 0) {
    int carry = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int w = w0 + lane;
      const int c = w < nwords ? __popc(bitmap[w]) : 0;
      int incl = c;
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (w < nwords) wprefix[w] = carry + incl - c;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) wprefix[nwords] = carry;
  }
  __syncthreads();
  const int U = wprefix[nwords];
  for (int w = threadIdx.x; w < nwords; w += kSelThreads) {
    uint32_t bits = bitmap[w];
    int pos = wprefix[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      ulist[pos++] = (w << 5) + b;
    }
  }
  __syncthreads();

  // 4. block scores for every (row, union member); each kbar row feeds 8 rows
  for (int u = threadIdx.x; u < U; u += kSelThreads) {
    const float4* kb = reinterpret_cast<const float4*>(p.kbar + (bh * nb + ulist[u]) * D);
    float acc[kSelRows];
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) acc[r] = 0.f;
#pragma unroll 4
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 kv = __ldg(kb + d4);
#pragma unroll
      for (int r = 0; r < kSelRows; ++r) {
        const float4 qv = reinterpret_cast<const float4*>(qs + r * D)[d4];
        acc[r] = fmaf(qv.x, kv.x, acc[r]);
        acc[r] = fmaf(qv.y, kv.y, acc[r]);
        acc[r] = fmaf(qv.z, kv.z, acc[r]);
        acc[r] = fmaf(qv.w, kv.w, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) S[r * nb + u] = acc[r] * p.scale;
  }
  __syncthreads();
  if (!row_ok || n == 0) {
    if (row_ok && lane == 0) p.counts[bh * nb + I] = 0;
    return;
  }

  // 5. selection for row I (one warp)
  const int flo = p.forced_lo[I], fhi = p.forced_hi[I];
  const int32_t* cols = p.cand_col + c_beg;
  const float* Srow = S + warp * nb;
  auto score_of = [&](int J) -> float {
    const int w = J >> 5;
    return Srow[wprefix[w] + __popc(bitmap[w] & ((1u << (J & 31)) - 1u))];
  };
  const bool dynamic = p.mode == DYNRAD_DYNAMIC_THRESHOLD;
  float smax = -INFINITY;
  for (int c = lane; c < n; c += 32) smax = fmaxf(smax, score_of(cols[c]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, off));
  uint64_t base = 0, ztot = 0;
  int nfree = 0;
  for (int c0 = 0; c0 < n; c0 += 32) {
    const int c = c0 + lane;
    uint64_t w = 0;
    bool forced = false;
    if (c < n) {
      const int J = cols[c];
      const float s = score_of(J);
      if (p.scores_out != nullptr) p.scores_out[bh * p.cand_nnz + c_beg + c] = s;
      forced = J >= flo && J <= fhi;
      if (dynamic) {
        const double e = exp(static_cast<double>(s) - static_cast<double>(smax));
        w = __double2ull_rn(e * kMassScale);
      } else {
        w = 1;
      }
      wgt[c] = forced ? 0 : w;
      key[c] = order_key(s);
      flag[c] = forced ? 1 : 0;
      if (forced) base += w;
      ztot += w;
    }
    nfree += __popc(__ballot_sync(0xffffffffu, c < n && !forced));
  }
  base = warp_sum_u64(base);
  ztot = warp_sum_u64(ztot);

  Reach reach;
  reach.dynamic = dynamic;
  reach.base = base;
  reach.k = 0;
  reach.tau_z = 0.0;
  bool keep_all = false;
  if (dynamic) {
    if (p.value >= 1.0) keep_all = true;
    else reach.tau_z = __dmul_rn(p.value, static_cast<double>(ztot));
  } else {
    if (nfree > 0) {
      const double kf = floor(__dadd_rn(__dmul_rn(p.value, static_cast<double>(nfree)), 1e-9));
      reach.k = kf < 1.0 ? 1ull : static_cast<uint64_t>(kf);
      if (reach.k > static_cast<uint64_t>(nfree)) reach.k = nfree;
    }
  }
  __syncwarp();

  uint32_t kstar = 0xFFFFFFFFu;  // cut key; free blocks with key > kstar are kept
  uint64_t above = 0;            // weight of free blocks with key > kstar
  bool cut_none = !keep_all && reach(0);
  if (!keep_all && !cut_none) {
    uint32_t prefix = 0, pmask = 0;
    bool found = true;
    for (int pass = 0; pass < 4 && found; ++pass) {
      const int shift = 24 - 8 * pass;
#pragma unroll
      for (int i = 0; i < 8; ++i) bins[lane * 8 + i] = 0;
      __syncwarp();
      for (int c = lane; c < n; c += 32) {
        if (flag[c]) continue;
        const uint32_t kk = key[c];
        if ((kk & pmask) == prefix) atomicAdd(reinterpret_cast<unsigned long long*>(&bins[(kk >> shift) & 255u]),
                                              static_cast<unsigned long long>(wgt[c]));
      }
      __syncwarp();
      // lane l owns digits 255-8l ... 248-8l (descending)
      uint64_t loc[8], lsum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        loc[i] = bins[255 - (lane * 8 + i)];
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
      pmask |= 255u << shift;
      __syncwarp();
    }
    if (found) kstar = prefix;
    else keep_all = true;  // target not reachable (rounding at tau ~ 1): keep all
  }

  // 6. mark kept free blocks: key > kstar, and ties at kstar in ascending order
  //    until the target is reached
  if (!cut_none) {
    uint64_t tie_run = 0;
    bool done = false;
    for (int c0 = 0; c0 < n; c0 += 32) {
      const int c = c0 + lane;
      bool kept = false;
      if (c < n && !flag[c]) {
        const uint32_t kk = key[c];
        if (keep_all || kk > kstar) kept = true;
      }
      const bool tie = !keep_all && c < n && !flag[c] && key[c] == kstar;
      const uint64_t tw = tie ? wgt[c] : 0;
      const uint64_t ex = warp_excl_scan_u64(tw, lane);
      if (tie && !done && !reach(above + tie_run + ex)) kept = true;
      tie_run += warp_sum_u64(tw);
      if (!done && reach(above + tie_run)) done = true;
      if (c < n && kept) flag[c] = 1;
    }
  }
  __syncwarp();

  // 7. ordered output of the kept blocks
  int32_t* dst = p.kept_tmp + bh * p.cand_nnz + c_beg;
  int cnt = 0;
  for (int c0 = 0; c0 < n; c0 += 32) {
    const int c = c0 + lane;
    const bool k_ = c < n && flag[c];
    const unsigned bal = __ballot_sync(0xffffffffu, k_);
    if (k_) dst[cnt + __popc(bal & ((1u << lane) - 1u))] = cols[c];
    cnt += __popc(bal);
  }
  if (lane == 0) p.counts[bh * nb + I] = cnt;
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
  // compaction: warp per row
  for (int i = warp; i < kScanTile; i += kScanThreads / 32) {
    const int64_t r = b0 + i;
    if (r >= p.rows) break;
    const int64_t bh = r / p.nb;
    const int I = static_cast<int>(r - bh * p.nb);
    const int64_t o = offs[i];
    const int64_t cnt = offs[i + 1] - o;
    const int32_t* src = p.kept_tmp + bh * p.cand_nnz + p.cand_row_ptr[I];
    for (int64_t c = lane; c < cnt; c += 32) {
      const int64_t d = o + c;
      if (d < p.col_cap) p.col_idx[d] = src[c];
      else record_error(DYNRAD_ERR_CAPACITY);
    }
  }
}

}  // namespace dynrad
