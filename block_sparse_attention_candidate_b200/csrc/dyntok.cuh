// Paper-exact dynamic-threshold mode (DynamicRad, Sec. 3.2 "Dynamic-threshold
// mode", Eqs. 9-11; the fused-head proxy of Appendix B, Eq. 19).
//
// For every candidate token pair (u, v) of an ordered frame pair (i, j) at
// t >= 2, the proxy logit s = (1/H_f) sum_{h < H_f} q_u^h . k_v^h / sqrt(d) over
// the first H_f heads; per frame pair the z-score s~ = (s - mu) / (sigma + eps)
// (Eq. 10, population sigma, eps = 1e-6); the pair is kept when s~ > tau
// (tau_1 near field, L(t) >= B_s; tau_2 far field), i.e. when
// s > mu + tau (sigma + eps); if no pair of the frame pair passes, the pair with
// the largest s is kept (smallest u * N_t + v among equal scores).  Pairs at
// t <= 1 are all kept (tau = -inf).  Kept token links are aggregated to blocks
// with (theta_c, theta_m), united with F_I; one mask per batch element, shared
// by its heads.
//
// Kernels:
//   dyntok_tile_kernel<D, H_f>  one CTA per (frame pair, 128 rows u, batch):
//       the 128 x 64 logit tiles of the band |u - v| <= w, bf16 tensor-core
//       MMAs with fp32 accumulation in a fixed order (identical in both
//       passes).  Pass 0 accumulates sum, sum of squares (fp64) and the packed
//       maximum; pass 1 counts kept links per (query block, key token).
//   dyntok_finalize_kernel  per (batch, frame pair): mu, sigma, the score
//       threshold, and the fallback pair's link.
//   dyntok_aggregate_kernel<BS>  per (batch, query block), one warp per
//       candidate: column counts (plus the t <= 1 links, counted in closed
//       form), (theta_c, theta_m), F_I.
//   expand_csr_kernel       per-batch masks -> rows (b, h, I) for every head.
#pragma once

#include <cuda_bf16.h>

#include "candidates.cuh"
#include "common.cuh"
#include "warp_mma.cuh"

namespace dynrad {

constexpr int kTokRows = 128;     // u rows per CTA
constexpr int kTokCols = 64;      // v columns per staged K tile
constexpr int kTokThreads = 256;  // 8 warps: a 4 x 2 grid of 32 x 32 sub-tiles
constexpr int kTokSlots = kTokRows / 32 + 1;   // query blocks 128 rows can touch (block >= 32)
constexpr double kTokEps = 1e-6;  // eps of Eq. 10

struct DynTokParams {
  GeomDev g;
  const __nv_bfloat16* q;   // [B, H, N, D]
  const __nv_bfloat16* k;
  int B, H, D, hf;
  double tau1, tau2;
  float inv;                // 1 / (hf * sqrt(D))
  double* stats;            // [B][F*F][2]: sum of s, sum of s^2
  unsigned long long* best; // [B][F*F]: (order key of s) << 32 | (0xFFFFFFFF - (u * N_t + v))
  double* thr;              // [B][F*F]: score threshold mu + tau (sigma + eps)
  uint32_t* colcnt;         // [B][nb][N]: kept links of (query block, key token), t >= 2
  const int32_t* cand_row_ptr;
  const int32_t* cand_col;
  const int32_t* forced_lo;
  const int32_t* forced_hi;
  int32_t* counts;          // [B * nb] kept blocks per (batch, row)
  int32_t* kept_tmp;        // [B][cand_nnz]
  int64_t cand_nnz;
  int pass;
};

__device__ __forceinline__ uint32_t tok_order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float tok_key_to_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Row stride (bf16 elements) of the staged Q / K rows: 8 elements of padding
// keep the 8 rows an ldmatrix reads in distinct bank groups.
__host__ __device__ constexpr int tok_row_stride(int x) { return x + 8; }

// Dynamic shared memory of the tile kernel for dot-product length x = H_f * D.
__host__ __device__ constexpr size_t tok_tile_smem(int x) {
  return static_cast<size_t>(tok_row_stride(x)) * (kTokRows + kTokCols) * 2;
}

// The logit tiles are dense 128 x 64 x (H_f * D) products on the warp-level bf16
// tensor-core MMA (m16n8k16, fp32 accumulation), from Q / K rows staged in
// shared memory.  Warp w computes the 32 x 32 sub-tile at rows 32 (w / 2) and
// columns 32 (w % 2): per 16-wide k step two A and two B ldmatrix.x4 feed 8
// MMAs, in one fixed k order in both passes, so both passes see identical
// logits.  A sub-tile with no pair inside the band |u - v| <= w is skipped;
// one wholly inside it skips the per-pair test.  The next K tile is loaded into
// registers while the current one is multiplied.
//
// Pass 1 counts kept links per (query block, key token): for each accumulator
// position a warp ballot over the 8 rows sharing a column gives the column's
// count (split at a query-block boundary when the 8 rows straddle one), and
// one lane per column adds it to the tile's counters.
template <int D, int HF>
__global__ void __launch_bounds__(kTokThreads, D * HF <= 256 ? 2 : 1) dyntok_tile_kernel(DynTokParams p) {
  constexpr int X = D * HF;                        // dot-product length
  constexpr int RS = tok_row_stride(X);
  constexpr int kVec = 8;                          // bf16 per 16-byte copy
  constexpr int VPR = X / kVec;                    // copies per staged row
  constexpr int KV = kTokCols * VPR / kTokThreads; // K-tile copies per thread
  static_assert(kTokCols * VPR % kTokThreads == 0, "K tile copies per thread");
  extern __shared__ __align__(16) __nv_bfloat16 tok_smem[];
  const GeomDev& g = p.g;
  const int F = g.frames, nt = g.nt;
  const int pi = blockIdx.x, b = blockIdx.z;
  const int i = pi / F, j = pi % F;
  const int t = i > j ? i - j : j - i;
  if (t < 2 || !pair_retained(g, t)) return;
  const int w = window_width(g, t);
  const int u0 = blockIdx.y * kTokRows;
  if (u0 >= nt) return;
  __nv_bfloat16* qs = tok_smem;                    // [kTokRows][RS]
  __nv_bfloat16* ks = qs + kTokRows * RS;          // [kTokCols][RS]
  __shared__ double red_d[2][kTokThreads / 32];
  __shared__ unsigned long long red_b[kTokThreads / 32];
  __shared__ uint32_t cnt_tile[kTokSlots][kTokCols];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // query rows of this chunk, fused heads side by side
  for (int e = threadIdx.x; e < kTokRows * VPR; e += kTokThreads) {
    const int r = e / VPR, x = (e % VPR) * kVec, h = x / D, d = x % D;
    const int u = u0 + r;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (u < nt)
      val = *reinterpret_cast<const uint4*>(p.q + ((static_cast<int64_t>(b) * p.H + h) * g.n + i * nt + u) * D + d);
    *reinterpret_cast<uint4*>(qs + r * RS + x) = val;
  }
  const int v_lo = max(u0 - w, 0), v_hi = min(u0 + kTokRows - 1 + w, nt - 1);
  const double thr = p.pass == 1 ? p.thr[static_cast<int64_t>(b) * F * F + pi] : 0.0;
  const int I0 = (i * nt + u0) / g.block;          // first query block of the chunk
  const int wr = warp >> 1, wc = warp & 1;         // sub-tile row / column group
  // ldmatrix row addresses.  A (m16 x k16, mt = 0, 1): rows 32 wr + 16 mt +
  // (lane % 16), k offset 8 (lane / 16).  B (two n8 x k16 tiles per x4, np =
  // 0, 1): rows 32 wc + 16 np + 8 (lane / 16) + (lane % 8), k offset 8 ((lane / 8) % 2).
  uint32_t a_addr[2], b_addr[2];
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    a_addr[m] = smem_u32(qs + (32 * wr + 16 * m + (lane & 15)) * RS + ((lane >> 4) << 3));
    b_addr[m] = smem_u32(ks + (32 * wc + 16 * m + ((lane >> 4) << 3) + (lane & 7)) * RS + (((lane >> 3) & 1) << 3));
  }
  const int g4 = lane >> 2, t4 = lane & 3;         // accumulator fragment coordinates
  const uint32_t col_lanes = 0x11111111u << t4;    // lanes holding this lane's column
  double s1 = 0.0, s2 = 0.0;
  unsigned long long bst = 0ull;
  uint4 pre[KV];
  auto load_k = [&](int v0) {
#pragma unroll
    for (int it = 0; it < KV; ++it) {
      const int e = threadIdx.x + it * kTokThreads;
      const int c = e / VPR, x = (e % VPR) * kVec, h = x / D, d = x % D;
      const int v = v0 + c;
      pre[it] = v <= v_hi ? *reinterpret_cast<const uint4*>(
                                p.k + ((static_cast<int64_t>(b) * p.H + h) * g.n + j * nt + v) * D + d)
                          : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  load_k(v_lo);
  for (int v0 = v_lo; v0 <= v_hi; v0 += kTokCols) {
    __syncthreads();   // previous tile's K rows and counters are consumed
#pragma unroll
    for (int it = 0; it < KV; ++it) {
      const int e = threadIdx.x + it * kTokThreads;
      *reinterpret_cast<uint4*>(ks + (e / VPR) * RS + (e % VPR) * kVec) = pre[it];
    }
    if (p.pass == 1)
      for (int e = threadIdx.x; e < kTokSlots * kTokCols; e += kTokThreads) (&cnt_tile[0][0])[e] = 0u;
    __syncthreads();
    if (v0 + kTokCols <= v_hi) load_k(v0 + kTokCols);
    const int ur0 = u0 + 32 * wr, vc0 = v0 + 32 * wc;
    const int dmin = max(0, max(vc0 - (ur0 + 31), ur0 - (vc0 + 31)));
    if (ur0 < nt && vc0 <= v_hi && dmin <= w) {
      float acc[2][4][4];
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[m][n][e] = 0.f;
#pragma unroll
      for (int k0 = 0; k0 < X; k0 += 16) {
        uint32_t a[2][4], bb[2][4];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          ldsm_x4(a_addr[m] + k0 * 2, a[m][0], a[m][1], a[m][2], a[m][3]);
          ldsm_x4(b_addr[m] + k0 * 2, bb[m][0], bb[m][1], bb[m][2], bb[m][3]);
        }
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int n = 0; n < 4; ++n)
            mma_16816(acc[m][n], a[m][0], a[m][1], a[m][2], a[m][3], bb[n >> 1][2 * (n & 1)],
                      bb[n >> 1][2 * (n & 1) + 1]);
      }
      const int dmax = max(vc0 + 31 - ur0, ur0 + 31 - vc0);
      const bool interior = ur0 + 31 < nt && vc0 + 31 <= v_hi && dmax <= w;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int u = ur0 + 16 * m + 8 * hh + g4;
          // query block slots of this lane's row and of the first of the 8 rows
          const int slot = (i * nt + u) / g.block - I0;
          const int slot0 = (i * nt + ur0 + 16 * m + 8 * hh) / g.block - I0;
#pragma unroll
          for (int n = 0; n < 4; ++n) {
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
              const int v = vc0 + 8 * n + 2 * t4 + cb;
              const int dd = u > v ? u - v : v - u;
              const bool in = interior || (u < nt && v <= v_hi && dd <= w);
              const float s = acc[m][n][2 * hh + cb] * p.inv;
              if (p.pass == 0) {
                if (in) {
                  const double sd = static_cast<double>(s);
                  s1 += sd;
                  s2 += sd * sd;
                  const unsigned long long key = (static_cast<unsigned long long>(tok_order_key(s)) << 32) |
                                                 (0xFFFFFFFFull - static_cast<unsigned long long>(u * nt + v));
                  bst = key > bst ? key : bst;
                }
              } else {
                const bool kept = in && static_cast<double>(s) > thr;
                const uint32_t b_first = __ballot_sync(0xffffffffu, kept && slot == slot0);
                const uint32_t b_next = __ballot_sync(0xffffffffu, kept && slot != slot0);
                if (g4 == 0) {
                  const int c = v - v0;
                  const uint32_t n0 = __popc(b_first & col_lanes), n1 = __popc(b_next & col_lanes);
                  if (n0 != 0u) atomicAdd(&cnt_tile[slot0][c], n0);
                  if (n1 != 0u) atomicAdd(&cnt_tile[slot0 + 1][c], n1);
                }
              }
            }
          }
        }
      }
    }
    if (p.pass == 1) {
      __syncthreads();
      for (int e = threadIdx.x; e < kTokSlots * kTokCols; e += kTokThreads) {
        const int slot = e / kTokCols, c = e % kTokCols;
        const uint32_t n = cnt_tile[slot][c];
        if (n != 0u)
          atomicAdd(&p.colcnt[(static_cast<int64_t>(b) * g.nb + I0 + slot) * g.n + j * nt + v0 + c], n);
      }
    }
  }
  if (p.pass == 0) {
    // CTA reduction, then one atomic per quantity
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, off);
      s2 += __shfl_xor_sync(0xffffffffu, s2, off);
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, bst, off);
      bst = o > bst ? o : bst;
    }
    if (lane == 0) {
      red_d[0][warp] = s1;
      red_d[1][warp] = s2;
      red_b[warp] = bst;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double a1 = 0.0, a2 = 0.0;
      unsigned long long bb = 0ull;
      for (int x = 0; x < kTokThreads / 32; ++x) {
        a1 += red_d[0][x];
        a2 += red_d[1][x];
        bb = red_b[x] > bb ? red_b[x] : bb;
      }
      double* st = p.stats + (static_cast<int64_t>(b) * F * F + pi) * 2;
      atomicAdd(st, a1);
      atomicAdd(st + 1, a2);
      atomicMax(&p.best[static_cast<int64_t>(b) * F * F + pi], bb);
    }
  }
}

// ---------------------------------------------------------------------------
// The same logit tiles on the 5th-generation tensor cores, for dot-product
// lengths H_f * D <= 256 (the usual two fused heads of 128 dimensions).
//
// Persistent CTAs walk work units (frame pair, 128 rows u, batch); a unit is
// its band in 128-column tiles: S = Q_u K_v^T, 128 x 128 x (H_f * D), bf16 operands staged by TMA
// (128-byte swizzle, one 64-column chunk per head half), fp32 accumulation in
// tensor memory, double-buffered so the product of tile j + 1 runs while tile
// j is read out.  The k order of the accumulation is fixed, so both passes see
// identical logits.
//
// Warp roles (320 threads):
//   warps 0-3, 4-7  epilogue: thread t of warpgroup g owns row t (TMEM lane t)
//              and columns 64 g .. 64 g + 63 of every tile.  Pass 0 keeps, per
//              thread, the sum and sum of squares of its row's in-band logits
//              (fp32 over 16 columns, then fp64) and the row's first maximum;
//              pass 1 counts, per key column and query block, the logits above
//              the threshold (a warp ballot per column; lane l adds columns l
//              and 32 + l to shared counters) and adds the tile's counts to
//              colcnt.
//   warp 8     producer: Q once, then the K tiles into a ring of two slots.
//   warp 9     MMA issuer (one thread).
// Every wait is bounded (common.cuh mbar_wait); a wait that runs out records
// DYNRAD_ERR_DEVICE and every role unwinds to the common exit.
// ---------------------------------------------------------------------------
template <int D, int HF>
struct TokTcCfg {
  static constexpr int kX = D * HF;
  static constexpr int kChunks = kX / 64;            // 128-byte column chunks
  static constexpr int kChunksPerHead = D / 64;
  static constexpr int kM = 128, kN = 128;
  static constexpr int kQBytes = kM * kX * 2;
  static constexpr int kKBytes = kN * kX * 2;
  static constexpr int kSlots = 2;
  static constexpr int kSmemData = kQBytes + kSlots * kKBytes;
  static constexpr int kCntWords = 2 * kTokSlots * kN;   // [tile parity][query block][column]
  static constexpr int kSmemCtrl = 512 + kCntWords * 4;   // barriers, reductions, counters
  static constexpr int kSmemTotal = kSmemData + kSmemCtrl + 1024;   // 1024: manual alignment
  static constexpr int kThreads = 320;
  static constexpr uint32_t kTmemCols = 256;         // two 128-column S buffers
  static_assert(kX % 64 == 0 && kX <= 256, "fused dot-product length");
  static_assert(kSmemTotal <= 227 * 1024, "shared memory");
};

// One work unit of the tensor-core tile kernel: (frame pair, 128 query rows,
// batch element).  Units where the pair is not scored (t < 2, or dropped by
// the split rule) have no tiles; every role skips them alike.
struct TokUnit {
  int pi, i, j, u0, b, w, v_lo, v_hi, ntile;
};

__device__ __forceinline__ TokUnit tok_unit(const GeomDev& g, int u, int nchunks, int rows, int cols) {
  TokUnit x;
  const int F = g.frames, nt = g.nt;
  const int per_b = F * F * nchunks;
  x.b = u / per_b;
  const int r = u - x.b * per_b;
  x.pi = r / nchunks;
  x.u0 = (r - x.pi * nchunks) * rows;
  x.i = x.pi / F;
  x.j = x.pi - x.i * F;
  const int t = x.i > x.j ? x.i - x.j : x.j - x.i;
  x.ntile = 0;
  x.w = 0;
  x.v_lo = x.v_hi = 0;
  if (t >= 2 && x.u0 < nt && pair_retained(g, t)) {
    x.w = window_width(g, t);
    x.v_lo = max(x.u0 - x.w, 0);
    x.v_hi = min(x.u0 + rows - 1 + x.w, nt - 1);
    x.ntile = (x.v_hi - x.v_lo + cols) / cols;
  }
  return x;
}

// Persistent: CTA c takes units c, c + gridDim.x, ...; tensor memory, the
// barriers and the K ring live across units, so the next unit's Q and K loads
// run while the current unit's last tiles are read out.
template <int D, int HF>
__global__ void __launch_bounds__(TokTcCfg<D, HF>::kThreads, 1)
    dyntok_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const DynTokParams p) {
  using C = TokTcCfg<D, HF>;
  extern __shared__ uint8_t tok_tc_raw[];
  const GeomDev& g = p.g;
  const int F = g.frames, nt = g.nt;
  const int nchunks = (nt + C::kM - 1) / C::kM;
  const int nunits = p.B * F * F * nchunks;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(tok_tc_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = smem;
  uint8_t* k_smem = smem + C::kQBytes;
  uint8_t* ctrl = smem + C::kSmemData;
  uint64_t* bar = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* q_full = bar;
  uint64_t* q_empty = bar + 1;     // a unit's products are done with Q
  uint64_t* k_full = bar + 2;      // [2]
  uint64_t* k_empty = bar + 4;     // [2]
  uint64_t* s_full = bar + 6;      // [2]
  uint64_t* s_empty = bar + 8;     // [2]
  uint64_t* drain = bar + 10;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(bar + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_s + 1);
  double* red_d = reinterpret_cast<double*>(ctrl + 128);                   // [2 parities][2][8]
  unsigned long long* red_b = reinterpret_cast<unsigned long long*>(ctrl + 384);   // [2 parities][8]
  uint32_t* cnt = reinterpret_cast<uint32_t*>(ctrl + 512);                // [2][kTokSlots][kN]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 8);   // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int e = threadIdx.x; e < C::kCntWords; e += C::kThreads) cnt[e] = 0u;
  if (warp == 9) {
    tmem_alloc(tmem_base_s, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_base_s;

  if (warp == 8) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      int gt = 0, ul = 0;   // K tiles and units issued
      bool ok = true;
      for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
        const TokUnit x = tok_unit(g, u, nchunks, C::kM, C::kN);
        if (x.ntile == 0) continue;
        if (ul > 0 && !mbar_wait(q_empty, (ul - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(q_smem + c * (C::kM * 128), &tm_q, q_full, (c % C::kChunksPerHead) * 64, x.i * nt + x.u0,
                      x.b * p.H + c / C::kChunksPerHead);
        ++ul;
        for (int jt = 0; jt < x.ntile; ++jt) {
          const int sl = gt & 1;
          if (gt >= 2 && !mbar_wait(&k_empty[sl], ((gt >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[sl], C::kKBytes);
          const int v0 = x.v_lo + jt * C::kN;
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(k_smem + sl * C::kKBytes + c * (C::kN * 128), &tm_k, &k_full[sl],
                        (c % C::kChunksPerHead) * 64, x.j * nt + v0, x.b * p.H + c / C::kChunksPerHead);
          ++gt;
        }
      }
      if (!ok) {
        // unwinding: the copies already issued land before shared memory is
        // given back (bounded; ignores the abort flag)
        if (ul > 0) mbar_wait(q_full, (ul - 1) & 1, nullptr);
        for (int k = gt > 2 ? gt - 2 : 0; k < gt; ++k) mbar_wait(&k_full[k & 1], (k >> 1) & 1, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(C::kM, C::kN, false, false);
      auto desc_add = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (bytes >> 4); };
      const uint64_t qdesc0 = smem_desc_sw128(smem_u32(q_smem), 16, 1024);
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(k_smem), 16, 1024);
      int gt = 0, ul = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
        const TokUnit x = tok_unit(g, u, nchunks, C::kM, C::kN);
        if (x.ntile == 0) continue;
        if (!mbar_wait(q_full, ul & 1, abort_flag)) { ok = false; break; }
        for (int jt = 0; jt < x.ntile; ++jt) {
          const int sl = gt & 1;
          if (!mbar_wait(&k_full[sl], (gt >> 1) & 1, abort_flag)) { ok = false; break; }
          if (gt >= 2 && !mbar_wait(&s_empty[sl], ((gt >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bd = desc_add(kdesc0, sl * C::kKBytes);
#pragma unroll
          for (int kk = 0; kk < C::kX / 16; ++kk) {
            const int c = kk >> 2, off = (kk & 3) * 32;
            mma_ss(taddr + sl * C::kN, desc_add(qdesc0, c * (C::kM * 128) + off),
                   desc_add(bd, c * (C::kN * 128) + off), idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&k_empty[sl]);
          mma_commit(&s_full[sl]);
          ++gt;
        }
        if (!ok) break;
        mma_commit(q_empty);   // the unit's products are done with Q
        ++ul;
      }
      // all issued tensor-core work finished before tensor memory is released
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue
    const int grp = warp >> 2;                     // column half
    const int row = (warp & 3) * 32 + lane;        // TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // After a failed wait the warps keep stepping through the units and tiles
    // without work, so every warp reaches the same named barriers.
    bool ok = true;
    int gt = 0, ul = 0;
    for (int uu = blockIdx.x; uu < nunits; uu += gridDim.x) {
      const TokUnit x = tok_unit(g, uu, nchunks, C::kM, C::kN);
      if (x.ntile == 0) continue;
      const int u = x.u0 + row;
      const bool row_ok = u < nt;
      // s > thr in double for a float s is s > thr rounded down to a float
      const float thr_f =
          p.pass == 1 ? __double2float_rd(p.thr[static_cast<int64_t>(x.b) * F * F + x.pi]) : 0.f;
      const int I0 = (x.i * nt + x.u0) / g.block;
      const int slot = (x.i * nt + u) / g.block - I0;                      // this row's query block
      const int slot_first = (x.i * nt + x.u0 + (warp & 3) * 32) / g.block - I0;   // of the warp's first row
      // lanes whose row lies in the warp's first query block (the rest are in the next one)
      const uint32_t lanes_first = __ballot_sync(0xffffffffu, !row_ok || slot == slot_first);
      // in-band columns of this row: v in [v_min, v_max]
      const int v_min = max(u - x.w, x.v_lo), v_max = min(u + x.w, x.v_hi);
      double s1 = 0.0, s2 = 0.0;
      float best = -INFINITY;
      int best_v = -1;
      for (int jt = 0; jt < x.ntile; ++jt, ++gt) {
        const int sl = gt & 1;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sl], (gt >> 1) & 1, abort_flag));
        const int vb = x.v_lo + jt * C::kN + grp * 64;   // column 0 of this thread's half
        const int c_lo = row_ok ? v_min - vb : 1, c_hi = row_ok ? v_max - vb : 0;   // in-band columns
        float sv[64];
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t r[32];
            tmem_ld32(taddr + lane_base + sl * C::kN + grp * 64 + h * 32, r);
#pragma unroll
            for (int q = 0; q < 32; ++q) sv[h * 32 + q] = __uint_as_float(r[q]);
          }
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sl]);
        uint32_t* ct = cnt + sl * (kTokSlots * C::kN);
        if (ok && p.pass == 0) {
          // fp32 partial sums over 16 columns (two chains per sum), added to
          // the fp64 totals once per 16 columns
#pragma unroll
          for (int c16 = 0; c16 < 64; c16 += 16) {
            float a1[2] = {0.f, 0.f}, a2[2] = {0.f, 0.f};
#pragma unroll
            for (int c = c16; c < c16 + 16; ++c) {
              const bool in = c >= c_lo && c <= c_hi;
              const float sc = sv[c] * p.inv;
              const float s = in ? sc : 0.f;
              a1[c & 1] += s;
              a2[c & 1] = fmaf(s, s, a2[c & 1]);
              if (in && sc > best) {   // columns ascend, so the first of equal maxima stays
                best = sc;
                best_v = vb + c;
              }
            }
            s1 += static_cast<double>(a1[0] + a1[1]);
            s2 += static_cast<double>(a2[0] + a2[1]);
          }
        } else if (ok) {
          // lane l collects the counts of columns l and 32 + l from the
          // column ballots, split between the warp's (at most two) query blocks
          uint32_t n_lo[2] = {0u, 0u}, n_hi[2] = {0u, 0u};
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const bool kept = c >= c_lo && c <= c_hi && sv[c] * p.inv > thr_f;
            const uint32_t bal = __ballot_sync(0xffffffffu, kept);
            const uint32_t lo = __popc(bal & lanes_first), hi = __popc(bal & ~lanes_first);
            if (lane == (c & 31)) {
              n_lo[c >> 5] = lo;
              n_hi[c >> 5] = hi;
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int col = grp * 64 + h * 32 + lane;
            if (n_lo[h] != 0u) atomicAdd(&ct[slot_first * C::kN + col], n_lo[h]);
            if (n_hi[h] != 0u) atomicAdd(&ct[(slot_first + 1) * C::kN + col], n_hi[h]);
          }
        }
        if (p.pass == 1) {
          // the warpgroup's 64 columns of this tile are counted: add them to
          // colcnt and clear them for tile gt + 2
          asm volatile("bar.sync %0, 128;" ::"r"(1 + grp) : "memory");
          const int tg = threadIdx.x - grp * 128;
          const int v0 = x.v_lo + jt * C::kN;
          for (int e = tg; e < kTokSlots * 64; e += 128) {
            const int s_ = e / 64, col = grp * 64 + e % 64;
            const uint32_t n = ct[s_ * C::kN + col];
            if (n != 0u) {
              if (ok)
                atomicAdd(&p.colcnt[(static_cast<int64_t>(x.b) * g.nb + I0 + s_) * g.n + x.j * nt + v0 + col], n);
              ct[s_ * C::kN + col] = 0u;
            }
          }
        }
      }
      if (p.pass == 0) {
        // the unit's sums and first maximum: warp, then the 8 epilogue warps
        unsigned long long key = 0ull;
        if (best_v >= 0)
          key = (static_cast<unsigned long long>(tok_order_key(best)) << 32) |
                (0xFFFFFFFFull - static_cast<unsigned long long>(u * nt + best_v));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          s1 += __shfl_xor_sync(0xffffffffu, s1, off);
          s2 += __shfl_xor_sync(0xffffffffu, s2, off);
          const unsigned long long o = __shfl_xor_sync(0xffffffffu, key, off);
          key = o > key ? o : key;
        }
        const int par = ul & 1;
        if (lane == 0) {
          red_d[par * 16 + warp] = s1;
          red_d[par * 16 + 8 + warp] = s2;
          red_b[par * 8 + warp] = key;
        }
        asm volatile("bar.sync 3, 256;" ::: "memory");
        if (threadIdx.x == 0 && ok) {
          double a1 = 0.0, a2 = 0.0;
          unsigned long long bb = 0ull;
          for (int q = 0; q < 8; ++q) {
            a1 += red_d[par * 16 + q];
            a2 += red_d[par * 16 + 8 + q];
            bb = red_b[par * 8 + q] > bb ? red_b[par * 8 + q] : bb;
          }
          double* st = p.stats + (static_cast<int64_t>(x.b) * F * F + x.pi) * 2;
          atomicAdd(st, a1);
          atomicAdd(st + 1, a2);
          atomicMax(&p.best[static_cast<int64_t>(x.b) * F * F + x.pi], bb);
        }
      }
      ++ul;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(taddr, C::kTmemCols);
}

// Per (batch, frame pair): mu, sigma, threshold; the fallback link when no pair
// passes.  stats_out (nullable): [B][F*F][3] mu, sigma, threshold.
__global__ void dyntok_finalize_kernel(DynTokParams p, double* stats_out) {
  const GeomDev& g = p.g;
  const int F = g.frames;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(p.B) * F * F) return;
  const int b = static_cast<int>(idx / (F * F)), pi = static_cast<int>(idx % (F * F));
  const int i = pi / F, j = pi % F;
  const int t = i > j ? i - j : j - i;
  double mu = 0.0, sigma = 0.0, th = -INFINITY;
  if (t >= 2 && pair_retained(g, t)) {
    const int64_t nt = g.nt;
    const int64_t wc0 = window_width(g, t);
    const int64_t wc = wc0 < nt - 1 ? wc0 : nt - 1;
    const double n = static_cast<double>(nt * (2 * wc + 1) - wc * (wc + 1));
    const double* st = p.stats + idx * 2;
    mu = st[0] / n;
    const double var = st[1] / n - mu * mu;
    sigma = var > 0.0 ? sqrt(var) : 0.0;
    const double tau =
        __dmul_rn(span_over_group(g.l0, t), g.gamma) >= static_cast<double>(g.block) ? p.tau1 : p.tau2;
    th = mu + tau * (sigma + kTokEps);
    const unsigned long long bb = p.best[idx];
    const float smax = tok_key_to_float(static_cast<uint32_t>(bb >> 32));
    const int64_t cnt = 0xFFFFFFFFll - static_cast<int64_t>(bb & 0xFFFFFFFFull);
    if (bb == 0ull || cnt >= nt * nt) {       // no pair was scored: cannot happen for finite inputs
      record_error(DYNRAD_ERR_DEVICE);
    } else if (!(static_cast<double>(smax) > th)) {   // no pair passes: keep the best one
      const int u = static_cast<int>(cnt / nt), v = static_cast<int>(cnt % nt);
      const int I = (i * g.nt + u) / g.block;
      atomicAdd(&p.colcnt[(static_cast<int64_t>(b) * g.nb + I) * g.n + j * g.nt + v], 1u);
    }
  }
  p.thr[idx] = th;
  if (stats_out != nullptr) {
    stats_out[idx * 3] = mu;
    stats_out[idx * 3 + 1] = sigma;
    stats_out[idx * 3 + 2] = th;
  }
}

// Per (batch, query block I): keep J if in F_I, or if more than theta_m * n_J
// of J's columns have more than theta_c * n_I kept links from I (the t >= 2
// links counted by the tile kernel, the t <= 1 links -- all of P -- counted
// here per frame).  One warp per candidate, eight at a time; then warp 0 writes
// the kept candidates in list order.
template <int BS>
__global__ void __launch_bounds__(kTokThreads) dyntok_aggregate_kernel(DynTokParams p) {
  extern __shared__ __align__(16) uint8_t ag_raw[];
  const GeomDev& g = p.g;
  int* wt = reinterpret_cast<int*>(ag_raw);                    // [F]
  uint8_t* rt = reinterpret_cast<uint8_t*>(wt + g.frames);     // [F]
  uint8_t* keep = rt + g.frames;                               // [nb] per list position
  __shared__ int seg_frame[BS + 1], seg_count[BS + 1], n_seg;
  constexpr int kTokensPerLane = (BS + 31) / 32;
  const int I = blockIdx.x, b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  build_frame_tables(g, wt, rt);
  const int q0 = I * BS, q1 = min(q0 + BS, g.n), nI = q1 - q0;
  if (threadIdx.x == 0) {
    // the block's query tokens per frame (a block spans one or more frames)
    int ns = 0;
    for (int q = q0; q < q1;) {
      const int f = q / g.nt, end = min(q1, (f + 1) * g.nt);
      seg_frame[ns] = f;
      seg_count[ns] = end - q;
      ++ns;
      q = end;
    }
    n_seg = ns;
  }
  __syncthreads();
  const int c_beg = p.cand_row_ptr[I];
  int nc = p.cand_row_ptr[I + 1] - c_beg;
  if (nc > g.nb || nc < 0) {   // not a valid candidate row
    if (threadIdx.x == 0) record_error(DYNRAD_ERR_CAPACITY);
    nc = nc < 0 ? 0 : g.nb;
  }
  const int flo = p.forced_lo[I], fhi = p.forced_hi[I];
  const uint32_t* cc = p.colcnt + (static_cast<int64_t>(b) * g.nb + I) * g.n;
  const double need_links = g.theta_c * nI;
  for (int c = warp; c < nc; c += kTokThreads / 32) {
    const int J = p.cand_col[c_beg + c];
    bool kp = J >= flo && J <= fhi;
    if (!kp) {
      const int k0 = J * BS, k1 = min(k0 + BS, g.n), nJ = k1 - k0;
      int n_active = 0;
#pragma unroll
      for (int x = 0; x < kTokensPerLane; ++x) {
        const int tk = lane + 32 * x;
        bool active = false;
        if (tk < nJ) {
          const int k = k0 + tk, fj = k / g.nt;
          uint32_t n = cc[k];
          for (int s = 0; s < n_seg; ++s) {   // t <= 1: every pair of P(i, j) is kept
            const int tt = seg_frame[s] > fj ? seg_frame[s] - fj : fj - seg_frame[s];
            if (tt <= 1 && rt[tt]) n += seg_count[s];
          }
          active = static_cast<double>(n) > need_links;
        }
        n_active += __popc(__ballot_sync(0xffffffffu, active));
      }
      kp = static_cast<double>(n_active) > g.theta_m * nJ;
    }
    if (lane == 0) keep[c] = kp ? 1 : 0;
  }
  __syncthreads();
  if (warp == 0) {
    int32_t* kt = p.kept_tmp + static_cast<int64_t>(b) * p.cand_nnz + c_beg;
    int n_kept = 0;
    for (int c0 = 0; c0 < nc; c0 += 32) {
      const int c = c0 + lane;
      const bool k_ = c < nc && keep[c] != 0;
      const unsigned bal = __ballot_sync(0xffffffffu, k_);
      if (k_) kt[n_kept + __popc(bal & ((1u << lane) - 1u))] = p.cand_col[c_beg + c];
      n_kept += __popc(bal);
    }
    if (lane == 0) p.counts[static_cast<int64_t>(b) * g.nb + I] = n_kept;
  }
}

// Rows (b, h, I) of the output from the per-batch CSR src (rows b * nb + I).
__global__ void expand_csr_kernel(const int32_t* src_ptr, const int32_t* src_col, int B, int H, int nb,
                                  int32_t* row_ptr, int32_t* col_idx, int64_t col_cap) {
  const int64_t total = static_cast<int64_t>(H) * src_ptr[static_cast<int64_t>(B) * nb];
  if (total > col_cap || total > INT32_MAX) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(DYNRAD_ERR_CAPACITY);
    return;
  }
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int b = 0; b < B; ++b) {
    const int64_t s0 = src_ptr[static_cast<int64_t>(b) * nb], s1 = src_ptr[static_cast<int64_t>(b + 1) * nb];
    const int64_t nnz_b = s1 - s0;
    const int64_t base = static_cast<int64_t>(H) * s0;   // entries of earlier batch elements
    for (int h = 0; h < H; ++h) {
      const int64_t r0 = (static_cast<int64_t>(b) * H + h) * nb;
      const int64_t o0 = base + h * nnz_b;
      for (int64_t x = tid; x < nb; x += stride)
        row_ptr[r0 + x] = static_cast<int32_t>(o0 + src_ptr[static_cast<int64_t>(b) * nb + x] - s0);
      for (int64_t x = tid; x < nnz_b; x += stride) col_idx[o0 + x] = src_col[s0 + x];
    }
  }
  if (tid == 0) row_ptr[static_cast<int64_t>(B) * H * nb] = static_cast<int32_t>(total);
}

}  // namespace dynrad
