// Paper-exact static-ratio mode (DynamicRad, Sec. 3.2 "Static-ratio mode",
// Eq. 8): per ordered frame pair (i, j) at distance t >= 2 kept by the split
// rule, k = max(1, floor(|P(i, j)| * rho)) token pairs of the candidate set
// P(i, j) of Eq. 7 are sampled -- rho = rho_1 when L(t) >= B_s, rho_2 below --
// and the sampled token links are aggregated to blocks as in Sec. 3.1
// ("Density control within blocks"), united with the near-frame set F_I.
//
// The seeded uniform k-subset: token pair (u, v) of (i, j) has counter
// c = ((i * F + j) * N_t + u) * N_t + v and key = SplitMix64(seed) output
// c + 1, i.e. mix(seed + (c + 1) * 0x9E3779B97F4A7C15) with the SplitMix64
// finaliser (Steele, Lea and Flood, OOPSLA 2014).  mix is a bijection, so keys
// never tie; the sample is the k pairs with the smallest keys, i.e. every pair
// whose key is <= T(i, j), the k-th smallest key.
//
// Kernels:
//   sample_setup_kernel   per frame pair: window, |P| (closed form), rho, k.
//   sample_hist_kernel    one radix pass (11-bit digit, 6 passes for 64 bits):
//                         histogram of the keys that share the digits found.
//   sample_pick_kernel    per frame pair: the digit holding the k-th key.
//   sample_mark_kernel    per query block, one warp per candidate block: its
//                         token-level sampled links, (theta_c, theta_m).
//   replicate_csr_kernel  copies the head-shared CSR for every (batch, head).
#pragma once

#include "candidates.cuh"
#include "common.cuh"

namespace dynrad {

constexpr int kSampleDigitBits = 11;
constexpr int kSampleBins = 1 << kSampleDigitBits;   // 2048
constexpr int kSamplePasses = 6;                     // 5 x 11 + 9 bits
constexpr int kSampleThreads = 256;
constexpr int kSampleRowsPerCta = 32;                // u rows of a frame pair per histogram CTA

__host__ __device__ constexpr int sample_shift(int pass) { return pass < 5 ? 53 - 11 * pass : 0; }
__host__ __device__ constexpr int sample_width(int pass) { return pass < 5 ? 11 : 9; }

struct SamplePair {
  uint64_t n;       // |P(i, j)|
  uint64_t k;       // sample size
  uint64_t prefix;  // key digits found so far (then T)
  uint64_t rank;    // 1-based rank of the k-th key among keys sharing the prefix
  int32_t w;        // window half-width (clamped to N_t)
  int32_t active;   // sampled by key (t >= 2, retained, |P| > 0)
  int32_t pad[2];
};

struct SampleParams {
  GeomDev g;
  double rho1, rho2;
  uint64_t seed;
  SamplePair* pairs;        // [F * F]
  uint32_t* hist;           // [F * F][kSampleBins]
  uint64_t* thresholds;     // [F * F] T(i, j); UINT64_MAX where every pair of P is kept
  const int32_t* cand_row_ptr;
  const int32_t* cand_col;
  const int32_t* forced_lo;
  const int32_t* forced_hi;
  int32_t* counts;          // [nb] kept per row
  int32_t* kept_tmp;        // [cand_nnz] kept lists at the candidate offsets
  int pass;
};

__device__ __forceinline__ uint64_t splitmix64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t sample_key(uint64_t seed, int frames, int nt, int i, int j, int u, int v) {
  const uint64_t c = ((static_cast<uint64_t>(i) * frames + j) * nt + u) * nt + v;
  return splitmix64_mix(seed + (c + 1ull) * 0x9E3779B97F4A7C15ull);
}

__global__ void sample_setup_kernel(SampleParams p) {
  const int F = p.g.frames;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= F * F) return;
  const int i = idx / F, j = idx % F;
  const int t = i > j ? i - j : j - i;
  SamplePair s;
  s.w = window_width(p.g, t);
  const int64_t nt = p.g.nt;
  const int64_t wc = s.w < nt - 1 ? s.w : nt - 1;
  const bool kept = pair_retained(p.g, t);
  // |P| = sum_u (min(u + w, N_t - 1) - max(u - w, 0) + 1) = N_t (2w + 1) - w (w + 1)
  s.n = kept ? static_cast<uint64_t>(nt * (2 * wc + 1) - wc * (wc + 1)) : 0ull;
  double rho = 1.0;
  if (t > 1) rho = __dmul_rn(span_over_group(p.g.l0, t), p.g.gamma) >= static_cast<double>(p.g.block) ? p.rho1
                                                                                                        : p.rho2;
  if (s.n == 0) {
    s.k = 0;
  } else {
    const double kf = floor(__dadd_rn(__dmul_rn(static_cast<double>(s.n), rho), 1e-9));
    uint64_t k = kf < 1.0 ? 1ull : static_cast<uint64_t>(kf);
    s.k = k > s.n ? s.n : k;
  }
  s.active = (t >= 2 && s.n > 0) ? 1 : 0;
  s.prefix = 0ull;
  s.rank = s.k;
  s.pad[0] = s.pad[1] = 0;
  p.pairs[idx] = s;
  p.thresholds[idx] = ~0ull;
}

// Histogram of one 11-bit digit over the keys of frame pair blockIdx.x, rows
// u in [blockIdx.y * 32, +32), that agree with the digits found so far.
__global__ void __launch_bounds__(kSampleThreads) sample_hist_kernel(SampleParams p) {
  __shared__ uint32_t h[kSampleBins];
  __shared__ int32_t rstart[kSampleRowsPerCta + 1];
  const int F = p.g.frames, nt = p.g.nt;
  const int pi = blockIdx.x;
  const SamplePair s = p.pairs[pi];
  if (!s.active) return;
  const int u0 = blockIdx.y * kSampleRowsPerCta;
  if (u0 >= nt) return;
  const int rows = min(kSampleRowsPerCta, nt - u0);
  const int i = pi / F, j = pi % F;
  for (int b = threadIdx.x; b < kSampleBins; b += kSampleThreads) h[b] = 0u;
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int r = 0; r < rows; ++r) {
      rstart[r] = acc;
      const int u = u0 + r;
      acc += min(u + s.w, nt - 1) - max(u - s.w, 0) + 1;
    }
    rstart[rows] = acc;
  }
  __syncthreads();
  const int shift = sample_shift(p.pass), width = sample_width(p.pass);
  const int hi_shift = shift + width;   // digits above this one must match the prefix
  const int total = rstart[rows];
  int r = 0;
  for (int f = threadIdx.x; f < total; f += kSampleThreads) {
    while (r + 1 < rows && rstart[r + 1] <= f) ++r;   // f increases per thread
    const int u = u0 + r;
    const int v = max(u - s.w, 0) + (f - rstart[r]);
    const uint64_t key = sample_key(p.seed, F, nt, i, j, u, v);
    const bool match = hi_shift >= 64 || ((key ^ s.prefix) >> hi_shift) == 0ull;
    if (match) atomicAdd(&h[(key >> shift) & ((1ull << width) - 1ull)], 1u);
  }
  __syncthreads();
  uint32_t* gh = p.hist + static_cast<int64_t>(pi) * kSampleBins;
  for (int b = threadIdx.x; b < kSampleBins; b += kSampleThreads)
    if (h[b] != 0u) atomicAdd(&gh[b], h[b]);
}

// Per frame pair: the digit whose bin holds the rank-th key; clears the bins.
__global__ void __launch_bounds__(kSampleThreads) sample_pick_kernel(SampleParams p) {
  constexpr int kPer = kSampleBins / kSampleThreads;   // 8 bins per thread
  __shared__ uint64_t wsum[kSampleThreads / 32];
  __shared__ int found_bin;
  __shared__ uint64_t found_below;
  const int pi = blockIdx.x;
  SamplePair s = p.pairs[pi];
  if (!s.active) return;
  uint32_t* gh = p.hist + static_cast<int64_t>(pi) * kSampleBins;
  const int width = sample_width(p.pass), shift = sample_shift(p.pass);
  const int nbins = 1 << width;
  uint32_t c[kPer];
  uint64_t local = 0;
#pragma unroll
  for (int x = 0; x < kPer; ++x) {
    const int b = threadIdx.x * kPer + x;
    c[x] = b < nbins ? gh[b] : 0u;
    local += c[x];
  }
  // exclusive prefix of the per-thread sums (bins ascending = keys ascending)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  if (threadIdx.x == 0) found_bin = -1;
  __syncthreads();
  uint64_t base = 0;
  for (int w = 0; w < warp; ++w) base += wsum[w];
  const uint64_t excl = base + incl - local;
  if (s.rank > excl && s.rank <= excl + local) {
    uint64_t run = excl;
#pragma unroll
    for (int x = 0; x < kPer; ++x) {
      if (s.rank <= run + c[x]) {
        found_bin = threadIdx.x * kPer + x;
        found_below = run;
        break;
      }
      run += c[x];
    }
  }
  __syncthreads();
#pragma unroll
  for (int x = 0; x < kPer; ++x) {
    const int b = threadIdx.x * kPer + x;
    if (b < nbins) gh[b] = 0u;
  }
  if (threadIdx.x == 0) {
    if (found_bin < 0) {   // the histogram does not hold rank keys: cannot happen
      record_error(DYNRAD_ERR_DEVICE);
      s.active = 0;
    } else {
      s.prefix |= static_cast<uint64_t>(found_bin) << shift;
      s.rank -= found_below;
    }
    p.pairs[pi] = s;
    if (p.pass == kSamplePasses - 1 && s.active) p.thresholds[pi] = s.prefix;
  }
}

// Per query block I: for each candidate block J (ascending), J is kept if it
// is in F_I or if, over the sampled token links of (I, J), more than
// theta_m * n_J of J's columns are active (a column is active when more than
// theta_c * n_I of I's tokens link to it).  One warp per candidate (eight at a
// time): lanes take J's columns and walk I's tokens; then warp 0 writes the
// kept candidates in list order.
template <int BS>
__global__ void __launch_bounds__(kSampleThreads) sample_mark_kernel(SampleParams p) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  const GeomDev& g = p.g;
  int* wt = reinterpret_cast<int*>(sm_raw);                    // [F]
  uint8_t* rt = reinterpret_cast<uint8_t*>(wt + g.frames);     // [F]
  uint8_t* keep = rt + g.frames;                               // [nb] per list position
  constexpr int kColsPerLane = (BS + 31) / 32;
  const int I = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  build_frame_tables(g, wt, rt);
  __syncthreads();
  const int q0 = I * BS, q1 = min(q0 + BS, g.n);
  const int nI = q1 - q0;
  const int c_beg = p.cand_row_ptr[I];
  int nc = p.cand_row_ptr[I + 1] - c_beg;
  if (nc > g.nb || nc < 0) {   // not a valid candidate row
    if (threadIdx.x == 0) record_error(DYNRAD_ERR_CAPACITY);
    nc = nc < 0 ? 0 : g.nb;
  }
  const int flo = p.forced_lo[I], fhi = p.forced_hi[I];
  const double need_links = g.theta_c * nI;
  for (int c = warp; c < nc; c += kSampleThreads / 32) {
    const int J = p.cand_col[c_beg + c];
    bool kp = J >= flo && J <= fhi;
    if (!kp) {
      const int k0 = J * BS, k1 = min(k0 + BS, g.n), nJ = k1 - k0;
      int n_active = 0;
#pragma unroll
      for (int x = 0; x < kColsPerLane; ++x) {
        const int k = k0 + lane + 32 * x;
        uint32_t cnt = 0;
        if (k < k1) {
          const int j = k / g.nt, v = k % g.nt;
          for (int q = q0; q < q1; ++q) {
            const int i = q / g.nt, u = q % g.nt;
            const int t = i > j ? i - j : j - i;
            const int d = u > v ? u - v : v - u;
            if (!rt[t] || d > wt[t]) continue;   // not in P(i, j)
            if (t >= 2 &&
                sample_key(p.seed, g.frames, g.nt, i, j, u, v) > p.thresholds[static_cast<int64_t>(i) * g.frames + j])
              continue;                          // not sampled
            ++cnt;
          }
        }
        n_active += __popc(__ballot_sync(0xffffffffu, k < k1 && static_cast<double>(cnt) > need_links));
      }
      kp = static_cast<double>(n_active) > g.theta_m * nJ;
    }
    if (lane == 0) keep[c] = kp ? 1 : 0;
  }
  __syncthreads();
  if (warp == 0) {
    int n_kept = 0;
    for (int c0 = 0; c0 < nc; c0 += 32) {
      const int c = c0 + lane;
      const bool k_ = c < nc && keep[c] != 0;
      const unsigned bal = __ballot_sync(0xffffffffu, k_);
      if (k_) p.kept_tmp[c_beg + n_kept + __popc(bal & ((1u << lane) - 1u))] = p.cand_col[c_beg + c];
      n_kept += __popc(bal);
    }
    if (lane == 0) p.counts[I] = n_kept;
  }
}

// Copies replica 0 of the CSR (rows [0, nb), entries [0, nnz)) to replicas
// 1 .. reps-1 and writes the final offset.
__global__ void replicate_csr_kernel(int32_t* row_ptr, int32_t* col_idx, int nb, int reps, int64_t col_cap) {
  const int64_t nnz = row_ptr[nb];
  const int64_t total = static_cast<int64_t>(reps) * nnz;
  if (total > col_cap || total > INT32_MAX) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(DYNRAD_ERR_CAPACITY);
    return;
  }
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int r = 1; r < reps; ++r) {
    for (int64_t x = tid; x < nb; x += stride)
      row_ptr[static_cast<int64_t>(r) * nb + x] = static_cast<int32_t>(r * nnz + row_ptr[x]);
    for (int64_t x = tid; x < nnz; x += stride) col_idx[r * nnz + x] = col_idx[x];
  }
  if (tid == 0) row_ptr[static_cast<int64_t>(reps) * nb] = static_cast<int32_t>(total);
}

}  // namespace dynrad
