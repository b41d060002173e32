// Stage 1: radial candidate block set (DynamicRad, Sec. 3.1, Eqs. 1-7 and
// "Density control within blocks").
//
// Work is integer geometry: one CTA per query block I tests every key block J.
// A block is a run of `block` tokens of the flattened (frame, h, w) order; it
// splits into per-frame segments [u_a, u_b] of in-frame indices.  Two segments
// at frame distance t hold a pair of P (Eq. 7) iff the frame pair is retained
// (Eq. 6) and the intervals [u_a - w(t), u_b + w(t)] and [v_a, v_b] meet.  With
// theta_c or theta_m > 0 the kernel counts, per key token, the linked query
// tokens of I (interval overlaps) and applies the two thresholds.
//
// The fp64 steps (Eq. 2 product, the round-half-up of Eq. 3, the Eq. 5
// quotient, the theta products) use explicitly rounded intrinsics so no FMA
// contraction changes a result: every decision is bit-identical to plain IEEE
// double arithmetic.
#pragma once

#include <cmath>

#include "common.cuh"

namespace dynrad {

struct GeomDev {
  int32_t frames, nt, block, nb, n, force_t;
  int64_t l0;
  double gamma, lambda, theta_c, theta_m, eps;
};

// Correctly rounded double steps.  On the device the explicit intrinsics keep
// nvcc from contracting a multiply-add into an FMA; on the host (x86-64 SSE2
// double, no FMA contraction) the plain operators round the same way.  The host
// forms only size workspaces.
__host__ __device__ __forceinline__ double geo_mul(double a, double b) {
#ifdef __CUDA_ARCH__
  return __dmul_rn(a, b);
#else
  return a * b;
#endif
}
__host__ __device__ __forceinline__ double geo_add(double a, double b) {
#ifdef __CUDA_ARCH__
  return __dadd_rn(a, b);
#else
  return a + b;
#endif
}
__host__ __device__ __forceinline__ double geo_div(double a, double b) {
#ifdef __CUDA_ARCH__
  return __ddiv_rn(a, b);
#else
  return a / b;
#endif
}

// B(t) of Eq. 1 for t >= 1: floor(log2 t) + 1 = bit length of t.
__host__ __device__ __forceinline__ int log_group(int t) {
#ifdef __CUDA_ARCH__
  return 32 - __clz(t);
#else
  return 32 - __builtin_clz(static_cast<unsigned>(t));
#endif
}

// L0 / 2^B(t), exact in double.
__host__ __device__ __forceinline__ double span_over_group(int64_t l0, int t) {
  return ldexp(static_cast<double>(l0), -log_group(t));
}

// w(t) of Eq. 3, clamped to N_t (every |u - v| is below N_t).
__host__ __device__ __forceinline__ int window_width(const GeomDev& g, int t) {
  if (t <= 1) return g.nt;
  const double L = geo_mul(span_over_group(g.l0, t), g.gamma);  // Eq. 2
  const double r = floor(geo_add(L, 0.5));                      // round half up
  long long w = r > 4.0e18 ? (long long)4e18 : (long long)r;
  if (w < g.block) w = g.block;
  return w > g.nt ? g.nt : static_cast<int>(w);
}

// Eq. 6: t mod sf(t) == 0, sf(t) = max(1, floor(B_s / (L_split(t) + eps))).
__host__ __device__ __forceinline__ bool pair_retained(const GeomDev& g, int t) {
  if (t == 0) return true;
  const double ls = geo_mul(span_over_group(g.l0, t), g.lambda);  // Eq. 4
  const double qf = floor(geo_div(static_cast<double>(g.block), geo_add(ls, g.eps)));
  if (qf > static_cast<double>(t)) return false;  // sf > t >= 1: t mod sf = t != 0
  long long sf = static_cast<long long>(qf);
  if (sf < 1) sf = 1;
  return (t % sf) == 0;
}

// Per-frame tables (w(t), retained(t)) for t in [0, frames), built in shared memory.
__device__ __forceinline__ void build_frame_tables(const GeomDev& g, int* wt, uint8_t* rt) {
  for (int t = threadIdx.x; t < g.frames; t += blockDim.x) {
    wt[t] = window_width(g, t);
    rt[t] = pair_retained(g, t) ? 1 : 0;
  }
}

// Always-kept block range of query block I: blocks holding a token whose frame
// lies within force_t (0 or 1) of a frame of I, over retained frame pairs.
__device__ __forceinline__ void forced_range(const GeomDev& g, const uint8_t* rt, int I, int& lo,
                                             int& hi) {
  const int q0 = I * g.block;
  const int q1 = min(q0 + g.block, g.n) - 1;
  int fa = q0 / g.nt, fb = q1 / g.nt;
  if (g.force_t >= 1 && g.frames > 1 && rt[1]) {
    fa = max(fa - 1, 0);
    fb = min(fb + 1, g.frames - 1);
  }
  lo = static_cast<int>((static_cast<int64_t>(fa) * g.nt) / g.block);
  hi = static_cast<int>((static_cast<int64_t>(fb + 1) * g.nt - 1) / g.block);
}

// Does the token-pair set of (I, J) pass the block aggregation?
__device__ bool block_pair_candidate(const GeomDev& g, const int* wt, const uint8_t* rt, int I,
                                     int J) {
  const int q0 = I * g.block, q1 = min(q0 + g.block, g.n) - 1;
  const int k0 = J * g.block, k1 = min(k0 + g.block, g.n) - 1;
  const int fq0 = q0 / g.nt, fq1 = q1 / g.nt;
  const int fk0 = k0 / g.nt, fk1 = k1 / g.nt;
  if (g.theta_c == 0.0 && g.theta_m == 0.0) {
    // some linked pair exists
    for (int fi = fq0; fi <= fq1; ++fi) {
      const int ua = (fi == fq0) ? q0 - fi * g.nt : 0;
      const int ub = (fi == fq1) ? q1 - fi * g.nt : g.nt - 1;
      for (int fj = fk0; fj <= fk1; ++fj) {
        const int t = abs(fi - fj);
        if (!rt[t]) continue;
        const int w = wt[t];
        const int va = (fj == fk0) ? k0 - fj * g.nt : 0;
        const int vb = (fj == fk1) ? k1 - fj * g.nt : g.nt - 1;
        if (va <= ub + w && vb >= ua - w) return true;
      }
    }
    return false;
  }
  const int n_i = q1 - q0 + 1, n_j = k1 - k0 + 1;
  const double col_thr = __dmul_rn(g.theta_c, static_cast<double>(n_i));
  int active = 0;
  for (int kk = k0; kk <= k1; ++kk) {
    const int fj = kk / g.nt, v = kk - fj * g.nt;
    int linked = 0;
    for (int fi = fq0; fi <= fq1; ++fi) {
      const int t = abs(fi - fj);
      if (!rt[t]) continue;
      const int w = wt[t];
      const int ua = (fi == fq0) ? q0 - fi * g.nt : 0;
      const int ub = (fi == fq1) ? q1 - fi * g.nt : g.nt - 1;
      const int lo = max(ua, v - w), hi = min(ub, v + w);
      if (hi >= lo) linked += hi - lo + 1;
    }
    if (static_cast<double>(linked) > col_thr) ++active;
  }
  return static_cast<double>(active) > __dmul_rn(g.theta_m, static_cast<double>(n_j));
}

__device__ __forceinline__ bool is_candidate(const GeomDev& g, const int* wt, const uint8_t* rt,
                                             int I, int J, int flo, int fhi) {
  return (J >= flo && J <= fhi) || block_pair_candidate(g, wt, rt, I, J);
}

constexpr int kCandThreads = 256;

// counts[I] = |C_I|; forced range per row.
__global__ void __launch_bounds__(kCandThreads) cand_count_kernel(GeomDev g, int32_t* counts,
                                                                  int32_t* forced_lo,
                                                                  int32_t* forced_hi) {
  extern __shared__ int smem_tables[];
  int* wt = smem_tables;
  uint8_t* rt = reinterpret_cast<uint8_t*>(wt + g.frames);
  __shared__ int warp_sums[kCandThreads / 32];
  build_frame_tables(g, wt, rt);
  __syncthreads();
  const int I = blockIdx.x;
  int flo, fhi;
  forced_range(g, rt, I, flo, fhi);
  int cnt = 0;
  for (int J = threadIdx.x; J < g.nb; J += blockDim.x) cnt += is_candidate(g, wt, rt, I, J, flo, fhi);
  for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int total = 0;
    for (int w = 0; w < kCandThreads / 32; ++w) total += warp_sums[w];
    counts[I] = total;
    forced_lo[I] = flo;
    forced_hi[I] = fhi;
  }
}

// Writes the candidates of row I in ascending order at cand_row_ptr[I].
__global__ void __launch_bounds__(kCandThreads) cand_fill_kernel(GeomDev g,
                                                                 const int32_t* cand_row_ptr,
                                                                 int32_t* cand_col,
                                                                 int64_t cand_cap) {
  extern __shared__ int smem_tables[];
  int* wt = smem_tables;
  uint8_t* rt = reinterpret_cast<uint8_t*>(wt + g.frames);
  __shared__ int warp_counts[kCandThreads / 32];
  build_frame_tables(g, wt, rt);
  __syncthreads();
  const int I = blockIdx.x;
  int flo, fhi;
  forced_range(g, rt, I, flo, fhi);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t pos = cand_row_ptr[I];
  for (int J0 = 0; J0 < g.nb; J0 += blockDim.x) {
    const int J = J0 + threadIdx.x;
    const bool flag = J < g.nb && is_candidate(g, wt, rt, I, J, flo, fhi);
    const unsigned bal = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) warp_counts[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kCandThreads / 32; ++w) {
      const int c = warp_counts[w];
      if (w < warp) before += c;
      total += c;
    }
    if (flag) {
      const int64_t dst = pos + before + __popc(bal & ((1u << lane) - 1u));
      if (dst < cand_cap) cand_col[dst] = J;
      else record_error(DYNRAD_ERR_CAPACITY);
    }
    pos += total;
    __syncthreads();
  }
}

// Exclusive scan of a[0..n) in place, a[n] = total; single CTA of 1024 threads.
// A total above INT32_MAX is recorded as DYNRAD_ERR_CAPACITY (and saturated).
__global__ void __launch_bounds__(1024) scan_small_kernel(int32_t* a, int n) {
  __shared__ int64_t warp_tot[32];
  __shared__ int64_t carry_s;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + threadIdx.x;
    const int64_t x = i < n ? a[i] : 0;
    int64_t incl = x;
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int64_t wbefore = 0, tot = 0;
    for (int w = 0; w < 32; ++w) {
      if (w < warp) wbefore += warp_tot[w];
      tot += warp_tot[w];
    }
    const int64_t carry = carry_s;
    const int64_t excl = carry + wbefore + incl - x;
    if (i < n) a[i] = excl > INT32_MAX ? INT32_MAX : static_cast<int32_t>(excl);
    __syncthreads();
    if (threadIdx.x == 0) carry_s = carry + tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int64_t t = carry_s;
    if (t > INT32_MAX) record_error(DYNRAD_ERR_CAPACITY);
    a[n] = t > INT32_MAX ? INT32_MAX : static_cast<int32_t>(t);
  }
}

}  // namespace dynrad
