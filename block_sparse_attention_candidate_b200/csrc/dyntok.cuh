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
//   dyntok_tile_kernel<D>   one CTA per (frame pair, 32 rows u, batch): the
//       32 x 64 logit tiles of the band |u - v| <= w, bf16 tensor-core MMAs
//       with fp32 accumulation in a fixed order (identical in both passes).  Pass 0 accumulates sum, sum of
//       squares (fp64) and the packed maximum; pass 1 counts kept links per
//       (query block, key token).
//   dyntok_finalize_kernel  per (batch, frame pair): mu, sigma, the score
//       threshold, and the fallback pair's link.
//   dyntok_aggregate_kernel<BS>  per (batch, query block): column counts (plus
//       the t <= 1 links, counted in closed form), (theta_c, theta_m), F_I.
//   expand_csr_kernel       per-batch masks -> rows (b, h, I) for every head.
#pragma once

#include <cuda_bf16.h>

#include "candidates.cuh"
#include "common.cuh"
#include "warp_mma.cuh"

namespace dynrad {

constexpr int kTokRows = 32;      // u rows per tile
constexpr int kTokCols = 64;      // v columns per tile
constexpr int kTokThreads = 256;
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

// The logit tiles are dense 32 x 64 x (H_f * D) products: warp-level bf16
// tensor-core MMAs (m16n8k16, fp32 accumulation) on Q / K rows staged in shared
// memory.  The kernel is bound by moving the band's K rows through L2, so the
// warp-level instruction suffices.  Warp w computes rows 16 (w / 4) .. +15 and
// columns 16 (w % 4) .. +15 of the tile, in one fixed k order in both passes.
template <int D>
__global__ void __launch_bounds__(kTokThreads) dyntok_tile_kernel(DynTokParams p) {
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
  const int X = p.hf * D;                          // dot-product length
  const int RS = tok_row_stride(X);
  __nv_bfloat16* qs = tok_smem;                    // [kTokRows][RS]
  __nv_bfloat16* ks = qs + kTokRows * RS;          // [kTokCols][RS]
  __shared__ double red_d[2][kTokThreads / 32];
  __shared__ unsigned long long red_b[kTokThreads / 32];
  __shared__ uint32_t cnt_tile[2][kTokCols];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kVec = 8;                          // bf16 per 16-byte copy
  const int vecs_per_row = X / kVec;
  // query rows of this chunk, fused heads side by side
  for (int e = threadIdx.x; e < kTokRows * vecs_per_row; e += kTokThreads) {
    const int r = e / vecs_per_row, x = (e % vecs_per_row) * kVec, h = x / D, d = x % D;
    const int u = u0 + r;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (u < nt)
      val = *reinterpret_cast<const uint4*>(p.q + ((static_cast<int64_t>(b) * p.H + h) * g.n + i * nt + u) * D + d);
    *reinterpret_cast<uint4*>(qs + r * RS + x) = val;
  }
  const int mr = (warp >> 2) * 16;                 // warp's first tile row
  const int nc = (warp & 3) * 16;                  // warp's first tile column
  const int v_lo = max(u0 - w, 0), v_hi = min(u0 + kTokRows - 1 + w, nt - 1);
  const double thr = p.pass == 1 ? p.thr[static_cast<int64_t>(b) * F * F + pi] : 0.0;
  const int I0 = (i * nt + u0) / g.block;          // first query block of the chunk
  // ldmatrix row addresses: A rows mr + (lane % 16), k offset 8 (lane / 16);
  // B rows nc + 8 (lane / 16) + (lane % 8), k offset 8 ((lane / 8) % 2)
  const uint32_t a_addr = smem_u32(qs + (mr + (lane & 15)) * RS + ((lane >> 4) << 3));
  const uint32_t b_addr = smem_u32(ks + (nc + ((lane >> 4) << 3) + (lane & 7)) * RS + (((lane >> 3) & 1) << 3));
  const int g4 = lane >> 2, t4 = lane & 3;         // accumulator fragment coordinates
  double s1 = 0.0, s2 = 0.0;
  unsigned long long bst = 0ull;
  for (int v0 = v_lo; v0 <= v_hi; v0 += kTokCols) {
    __syncthreads();   // previous tile's K rows and counters are consumed
    for (int e = threadIdx.x; e < kTokCols * vecs_per_row; e += kTokThreads) {
      const int c = e / vecs_per_row, x = (e % vecs_per_row) * kVec, h = x / D, d = x % D;
      const int v = v0 + c;
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (v <= v_hi)
        val = *reinterpret_cast<const uint4*>(p.k + ((static_cast<int64_t>(b) * p.H + h) * g.n + j * nt + v) * D + d);
      *reinterpret_cast<uint4*>(ks + c * RS + x) = val;
    }
    if (p.pass == 1 && threadIdx.x < 2 * kTokCols) cnt_tile[threadIdx.x / kTokCols][threadIdx.x % kTokCols] = 0u;
    __syncthreads();
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};   // two n8 tiles
    for (int k0 = 0; k0 < X; k0 += 16) {
      uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
      ldsm_x4(a_addr + k0 * 2, a0, a1, a2, a3);
      ldsm_x4(b_addr + k0 * 2, b0, b1, b2, b3);
      mma_16816(acc[0], a0, a1, a2, a3, b0, b1);
      mma_16816(acc[1], a0, a1, a2, a3, b2, b3);
    }
#pragma unroll
    for (int nt8 = 0; nt8 < 2; ++nt8) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int u = u0 + mr + g4 + ((e >> 1) << 3);
        const int v = v0 + nc + nt8 * 8 + 2 * t4 + (e & 1);
        const int dd = u > v ? u - v : v - u;
        if (u >= nt || v > v_hi || dd > w) continue;
        const float s = acc[nt8][e] * p.inv;
        if (p.pass == 0) {
          s1 += static_cast<double>(s);
          s2 += static_cast<double>(s) * static_cast<double>(s);
          const unsigned long long key = (static_cast<unsigned long long>(tok_order_key(s)) << 32) |
                                         (0xFFFFFFFFull - static_cast<unsigned long long>(u * nt + v));
          bst = key > bst ? key : bst;
        } else if (static_cast<double>(s) > thr) {
          const int slot = (i * nt + u) / g.block - I0;   // 0 or 1 (a chunk spans at most 2 blocks)
          atomicAdd(&cnt_tile[slot][v - v0], 1u);
        }
      }
    }
    if (p.pass == 1) {
      __syncthreads();
      if (threadIdx.x < 2 * kTokCols) {
        const int slot = threadIdx.x / kTokCols, c = threadIdx.x % kTokCols;
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
// here per frame).
template <int BS>
__global__ void __launch_bounds__(kTokThreads) dyntok_aggregate_kernel(DynTokParams p) {
  extern __shared__ __align__(16) uint8_t ag_raw[];
  const GeomDev& g = p.g;
  int* wt = reinterpret_cast<int*>(ag_raw);                    // [F]
  uint8_t* rt = reinterpret_cast<uint8_t*>(wt + g.frames);     // [F]
  __shared__ int seg_frame[BS + 1], seg_count[BS + 1], n_seg, n_kept;
  const int I = blockIdx.x, b = blockIdx.y;
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
    n_kept = 0;
  }
  __syncthreads();
  const int c_beg = p.cand_row_ptr[I], c_end = p.cand_row_ptr[I + 1];
  const int flo = p.forced_lo[I], fhi = p.forced_hi[I];
  const uint32_t* cc = p.colcnt + (static_cast<int64_t>(b) * g.nb + I) * g.n;
  int32_t* kt = p.kept_tmp + static_cast<int64_t>(b) * p.cand_nnz + c_beg;
  for (int c = c_beg; c < c_end; ++c) {
    const int J = p.cand_col[c];
    bool keep = J >= flo && J <= fhi;
    if (!keep) {
      const int k0 = J * BS, k1 = min(k0 + BS, g.n), nJ = k1 - k0;
      bool active = false;
      if (threadIdx.x < nJ) {
        const int k = k0 + threadIdx.x, fj = k / g.nt;
        uint32_t n = cc[k];
        for (int s = 0; s < n_seg; ++s) {   // t <= 1: every pair of P(i, j) is kept
          const int tt = seg_frame[s] > fj ? seg_frame[s] - fj : fj - seg_frame[s];
          if (tt <= 1 && rt[tt]) n += seg_count[s];
        }
        active = static_cast<double>(n) > g.theta_c * nI;
      }
      const int n_active = __syncthreads_count(active);
      keep = static_cast<double>(n_active) > g.theta_m * nJ;
    }
    if (keep && threadIdx.x == 0) kt[n_kept++] = J;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.counts[static_cast<int64_t>(b) * g.nb + I] = n_kept;
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
