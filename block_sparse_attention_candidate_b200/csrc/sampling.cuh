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
// Finding T(i, j) exactly in one pass over the keys.  The keys of a frame pair
// are spread uniformly over [0, 2^64), so the k-th smallest lies near
// (k - 1/2) / |P| * 2^64, within a few sqrt(q (1 - q) / |P|) * 2^64 (q = k / |P|,
// the spread of a uniform order statistic).  One pass counts the keys below a
// window [lo, hi] around that point (7 such deviations plus 64 keys' worth on
// each side, widened to whole multiples of 2^32 so that a key's high word
// classifies it) and copies the keys inside it to a per-pair pool; if the counts
// show that the window holds the k-th key, a radix select over the few
// thousand pooled keys gives T.  Otherwise (never seen with real keys, but
// possible for a pair whose pool reservation did not fit the workspace) the
// select CTA recomputes all of the pair's keys in each radix pass.  Either way
// T is the exact k-th smallest key.
//
// Kernels:
//   sample_setup_kernel    per frame pair: window, |P| (closed form), rho, k,
//                          the key window and its pool reservation.
//   sample_collect_kernel  one pass over every key: counts below the window,
//                          pools the keys inside it.
//   sample_select_kernel   per frame pair: 11-bit radix select of the k-th key
//                          over the pooled keys (or over all keys).
//   sample_mark_kernel     one warp per candidate block (warps claim candidates
//                          in small chunks from a ticket): its token-level
//                          sampled links, (theta_c, theta_m), a keep flag.
//   sample_compact_kernel  one warp per query block: the kept candidates in
//                          list order and the row's count.
//   replicate_csr_kernel   copies the head-shared CSR for every (batch, head).
#pragma once

#include "candidates.cuh"
#include "common.cuh"

namespace dynrad {

constexpr int kSampleDigitBits = 11;
constexpr int kSampleBins = 1 << kSampleDigitBits;   // 2048
constexpr int kSamplePasses = 6;                     // 5 x 11 + 9 bits
constexpr int kSampleThreads = 256;
constexpr int kSampleRowsPerCta = 64;                // u rows of a frame pair per collect CTA
constexpr uint64_t kSplitMixGamma = 0x9E3779B97F4A7C15ull;
constexpr double kSampleWindowDevs = 7.0;            // window half-width in order-statistic deviations
constexpr double kSampleWindowPad = 64.0;            // plus this many keys' worth on each side

__host__ __device__ constexpr int sample_shift(int pass) { return pass < 5 ? 53 - 11 * pass : 0; }
__host__ __device__ constexpr int sample_width(int pass) { return pass < 5 ? 11 : 9; }

// Pool slots reserved for a pair with |P| = n: ceil(e + 8 sqrt(e) + 64), at
// most n, e the expected number of keys in the window.  The host sizes the
// pool with the same function at e's largest value (q = 1/2).
__host__ __device__ inline uint64_t sample_pool_slots(double n, double expect) {
  double c = ceil(expect + 8.0 * sqrt(expect) + 64.0);
  if (c > n) c = n;
  if (c > 2147483647.0) c = 2147483647.0;
  return static_cast<uint64_t>(c);
}

struct SamplePair {
  uint64_t n;       // |P(i, j)|
  uint64_t k;       // sample size
  uint64_t lo, hi;  // key window expected to hold the k-th smallest key
  uint64_t off;     // first pool slot
  uint32_t cap;     // pool slots reserved (0: none; the select recomputes every key)
  int32_t w;        // window half-width (clamped to N_t)
  int32_t active;   // sampled by key (t >= 2, retained, |P| > 0)
  int32_t pad;
};

struct SampleParams {
  GeomDev g;
  double rho1, rho2;
  uint64_t seed;
  SamplePair* pairs;        // [F * F]
  unsigned long long* below;   // [F * F] keys below lo (zeroed before setup)
  unsigned long long* inwin;   // [F * F] keys in [lo, hi] (zeroed before setup)
  unsigned long long* pool_used;  // slots handed out (zeroed before setup)
  uint64_t* pool;           // [pool_cap] pooled window keys
  uint64_t pool_cap;
  uint64_t* thresholds;     // [F * F] T(i, j); UINT64_MAX where every pair of P is kept
  const int32_t* cand_row_ptr;
  const int32_t* cand_col;
  const int32_t* forced_lo;
  const int32_t* forced_hi;
  int64_t cand_nnz;
  uint8_t* keep;            // [cand_nnz] per candidate: kept (1) or not (0)
  unsigned long long* mark_ticket;   // candidates handed out to marking warps (zeroed before setup)
  int32_t* counts;          // [nb] kept per row
  int32_t* kept_tmp;        // [cand_nnz] kept lists at the candidate offsets
};

// The SplitMix64 finaliser up to its last xor-shift; splitmix64_mix is
// y ^ (y >> 31) of this y, whose high 32 bits are yh ^ (yh >> 31), yh = y >> 32.
__device__ __forceinline__ uint64_t splitmix64_premix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  return (z ^ (z >> 27)) * 0x94D049BB133111EBull;
}

__device__ __forceinline__ uint64_t splitmix64_mix(uint64_t z) {
  const uint64_t y = splitmix64_premix(z);
  return y ^ (y >> 31);
}

// The generator state before mixing for counter c: seed + (c + 1) * gamma
// (mod 2^64).  Consecutive v add gamma, consecutive u add N_t * gamma, so the
// scans below step the state instead of recomputing it.
__device__ __forceinline__ uint64_t sample_state(uint64_t seed, int frames, int nt, int i, int j, int u, int v) {
  const uint64_t c = ((static_cast<uint64_t>(i) * frames + j) * nt + u) * nt + v;
  return seed + (c + 1ull) * kSplitMixGamma;
}

__device__ __forceinline__ uint64_t sample_key(uint64_t seed, int frames, int nt, int i, int j, int u, int v) {
  return splitmix64_mix(sample_state(seed, frames, nt, i, j, u, v));
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
  s.lo = 0ull;
  s.hi = ~0ull;
  s.off = 0ull;
  s.cap = 0u;
  s.pad = 0;
  if (s.active) {
    // Any window is correct (the select checks the counts); this one holds
    // the k-th key unless it sits more than 7 deviations from its mean.
    const double n = static_cast<double>(s.n), q = static_cast<double>(s.k) / n;
    const double half = kSampleWindowDevs * sqrt(q * (1.0 - q) / n) + kSampleWindowPad / n;
    const double mid = (static_cast<double>(s.k) - 0.5) / n;
    const double lo_f = mid - half, hi_f = mid + half;
    const double two64 = 18446744073709551616.0;
    if (lo_f > 0.0) s.lo = static_cast<uint64_t>(lo_f * two64);   // lo_f < mid < 1
    if (hi_f < 1.0 - 0x1p-40) s.hi = static_cast<uint64_t>(hi_f * two64);
    // widened to whole 2^32 ranges (at most 2 |P| / 2^32 more keys): the
    // collect pass then classifies a key by its high 32 bits alone
    s.lo &= ~0xFFFFFFFFull;
    s.hi |= 0xFFFFFFFFull;
    const double span = fmin(hi_f, 1.0) - fmax(lo_f, 0.0);
    const uint64_t cap = sample_pool_slots(n, span * n);
    const unsigned long long off = atomicAdd(p.pool_used, static_cast<unsigned long long>(cap));
    if (off + cap <= p.pool_cap) {
      s.off = off;
      s.cap = static_cast<uint32_t>(cap);
    }
  }
  p.pairs[idx] = s;
  p.thresholds[idx] = ~0ull;
}

// One pass over the keys of frame pair blockIdx.x, rows u in
// [blockIdx.y * 64, +64), one warp per row (lanes over v): counts the keys
// below the pair's window and appends the keys inside it to the pair's pool
// slots (in any order).  Each warp gathers its window keys in shared memory
// and claims pool slots for them in one atomic when its buffer fills or its
// rows are done.
__global__ void __launch_bounds__(kSampleThreads) sample_collect_kernel(SampleParams p) {
  constexpr int kBuf = 64;   // window keys buffered per warp
  __shared__ uint64_t wbuf[kSampleThreads / 32][kBuf];
  __shared__ unsigned long long wsum[kSampleThreads / 32];
  const int F = p.g.frames, nt = p.g.nt;
  const int pi = blockIdx.x;
  const SamplePair s = p.pairs[pi];
  if (!s.active || s.cap == 0u) return;   // no pool: the select pass reads every key itself
  const int u0 = blockIdx.y * kSampleRowsPerCta;
  if (u0 >= nt) return;
  const int u1 = min(u0 + kSampleRowsPerCta, nt);
  const int i = pi / F, j = pi % F;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const uint64_t step = 32ull * kSplitMixGamma;
  uint64_t* buf = wbuf[warp];
  uint32_t nbuf = 0;   // warp-uniform
  auto flush = [&]() {
    __syncwarp();
    unsigned long long base = 0;
    if (lane == 0) base = atomicAdd(&p.inwin[pi], static_cast<unsigned long long>(nbuf));
    base = __shfl_sync(0xffffffffu, base, 0);
    for (uint32_t x = lane; x < nbuf; x += 32)
      if (base + x < s.cap) p.pool[s.off + base + x] = buf[x];   // beyond cap: the select falls back
    __syncwarp();
    nbuf = 0;
  };
  // the window is [lo_hi * 2^32, hi_hi * 2^32 + 2^32 - 1]: a key's high word
  // decides below / inside / above
  const uint32_t lo_hi = static_cast<uint32_t>(s.lo >> 32), hi_hi = static_cast<uint32_t>(s.hi >> 32);
  uint32_t below = 0;
  auto visit = [&](uint64_t z, bool valid) {   // called with the whole warp
    const uint64_t y = splitmix64_premix(z);
    const uint32_t yh = static_cast<uint32_t>(y >> 32);
    const uint32_t kh = yh ^ (yh >> 31);   // high word of the key
    below += (valid && kh < lo_hi) ? 1u : 0u;
    const bool in_win = valid && kh >= lo_hi && kh <= hi_hi;
    const unsigned m = __ballot_sync(0xffffffffu, in_win);
    if (m != 0u) {
      if (nbuf + __popc(m) > kBuf) flush();
      if (in_win) buf[nbuf + __popc(m & lt)] = y ^ (y >> 31);
      nbuf += __popc(m);
    }
  };
  for (int u = u0 + warp; u < u1; u += kSampleThreads / 32) {   // warp-uniform
    const int va = max(u - s.w, 0), vb = min(u + s.w, nt - 1);
    const int len = vb - va + 1, full = len >> 5, tail = len & 31;
    uint64_t z = sample_state(p.seed, F, nt, i, j, u, va + lane);
    for (int it = 0; it < full; ++it, z += step) visit(z, true);   // warp-uniform
    if (tail != 0) visit(z, lane < tail);
  }
  if (nbuf != 0u) flush();
  unsigned long long bsum = below;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bsum += __shfl_xor_sync(0xffffffffu, bsum, o);
  if (lane == 0) wsum[warp] = bsum;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long sum = 0;
    for (int x = 0; x < kSampleThreads / 32; ++x) sum += wsum[x];
    if (sum != 0ull) atomicAdd(&p.below[pi], sum);
  }
}

// Per frame pair: T(i, j), the k-th smallest key, by six 11-bit radix passes
// (top digit first) over the pooled window keys when the counts show that the
// window holds it, else over all of the pair's keys, recomputed each pass.
__global__ void __launch_bounds__(kSampleThreads) sample_select_kernel(SampleParams p) {
  constexpr int kPer = kSampleBins / kSampleThreads;   // 8 bins per thread
  __shared__ uint32_t h[kSampleBins];
  __shared__ unsigned long long wsum[kSampleThreads / 32];
  __shared__ int found_bin;
  __shared__ unsigned long long found_below;
  const int F = p.g.frames, nt = p.g.nt;
  const int pi = blockIdx.x;
  const SamplePair s = p.pairs[pi];
  if (!s.active) return;
  const int i = pi / F, j = pi % F;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned long long nb_below = p.below[pi], nb_win = p.inwin[pi];
  const bool pooled = s.cap > 0u && nb_win <= s.cap && s.k > nb_below && s.k - nb_below <= nb_win;
  unsigned long long rank = pooled ? s.k - nb_below : s.k;   // 1-based, among the keys searched
  uint64_t prefix = 0ull;
  for (int pass = 0; pass < kSamplePasses; ++pass) {
    const int shift = sample_shift(pass), width = sample_width(pass);
    const int hi_shift = shift + width;   // digits above this one must match the prefix
    const uint64_t mask = (1ull << width) - 1ull;
    for (int b = threadIdx.x; b < kSampleBins; b += kSampleThreads) h[b] = 0u;
    if (threadIdx.x == 0) found_bin = -1;
    __syncthreads();
    if (pooled) {
      for (uint64_t x = threadIdx.x; x < nb_win; x += kSampleThreads) {
        const uint64_t key = p.pool[s.off + x];
        if (hi_shift >= 64 || ((key ^ prefix) >> hi_shift) == 0ull) atomicAdd(&h[(key >> shift) & mask], 1u);
      }
    } else {
      for (int u = warp; u < nt; u += kSampleThreads / 32) {
        const int v1 = min(u + s.w, nt - 1);
        for (int v = max(u - s.w, 0) + lane; v <= v1; v += 32) {
          const uint64_t key = sample_key(p.seed, F, nt, i, j, u, v);
          if (hi_shift >= 64 || ((key ^ prefix) >> hi_shift) == 0ull) atomicAdd(&h[(key >> shift) & mask], 1u);
        }
      }
    }
    __syncthreads();
    // the bin holding the rank-th key: exclusive prefix of per-thread sums
    // (bins ascending = keys ascending)
    uint32_t c[kPer];
    unsigned long long local = 0;
#pragma unroll
    for (int x = 0; x < kPer; ++x) {
      const int b = threadIdx.x * kPer + x;
      c[x] = b <= static_cast<int>(mask) ? h[b] : 0u;
      local += c[x];
    }
    unsigned long long incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    unsigned long long base = 0;
    for (int x = 0; x < warp; ++x) base += wsum[x];
    const unsigned long long excl = base + incl - local;
    if (rank > excl && rank <= excl + local) {
      unsigned long long run = excl;
#pragma unroll
      for (int x = 0; x < kPer; ++x) {
        if (rank <= run + c[x]) {
          found_bin = threadIdx.x * kPer + x;
          found_below = run;
          break;
        }
        run += c[x];
      }
    }
    __syncthreads();
    const int bin = found_bin;
    const unsigned long long below_bin = found_below;
    if (bin < 0) {   // the keys searched do not hold rank keys: cannot happen
      if (threadIdx.x == 0) record_error(DYNRAD_ERR_DEVICE);
      return;        // T stays UINT64_MAX
    }
    prefix |= static_cast<uint64_t>(bin) << shift;
    rank -= below_bin;
    __syncthreads();   // h, wsum and found_* are rewritten by the next pass
  }
  if (threadIdx.x == 0) p.thresholds[pi] = prefix;
}

// Candidate block J of query block I is kept if it is in F_I or if, over the
// sampled token links of (I, J), more than theta_m * n_J of J's columns are
// active (a column is active when more than theta_c * n_I of I's tokens link
// to it).  One warp per candidate, lanes over J's columns, each walking I's
// tokens; warps claim chunks of kMarkChunk consecutive candidates (flattened
// over all rows) from a ticket, so the uneven cost of candidates (t <= 1 pairs
// are counted in closed form, far pairs token by token) evens out.
constexpr int kMarkChunk = 4;

// Row of flattened candidate c: the I with row_ptr[I] <= c < row_ptr[I + 1].
__device__ __forceinline__ int cand_row_of(const int32_t* row_ptr, int nb, int64_t c) {
  int lo = 0, hi = nb - 1;   // row_ptr[0] = 0 <= c
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<int64_t>(row_ptr[mid]) <= c) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <int BS>
__global__ void __launch_bounds__(kSampleThreads) sample_mark_kernel(SampleParams p) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  const GeomDev& g = p.g;
  int* wt = reinterpret_cast<int*>(sm_raw);                    // [F]
  uint8_t* rt = reinterpret_cast<uint8_t*>(wt + g.frames);     // [F]
  constexpr int kColsPerLane = (BS + 31) / 32;
  const int lane = threadIdx.x & 31;
  build_frame_tables(g, wt, rt);
  __syncthreads();
  const uint64_t ustep = static_cast<uint64_t>(g.nt) * kSplitMixGamma;   // u -> u + 1
  const int64_t nnz = p.cand_nnz;
  for (;;) {
    unsigned long long c0 = 0;
    if (lane == 0) c0 = atomicAdd(p.mark_ticket, static_cast<unsigned long long>(kMarkChunk));
    c0 = __shfl_sync(0xffffffffu, c0, 0);
    if (c0 >= static_cast<unsigned long long>(nnz)) break;   // warp-uniform
    const int64_t c1 = min(static_cast<int64_t>(c0) + kMarkChunk, nnz);
    int I = cand_row_of(p.cand_row_ptr, g.nb, static_cast<int64_t>(c0));
    for (int64_t c = static_cast<int64_t>(c0); c < c1; ++c) {   // warp-uniform
      while (I + 1 < g.nb && static_cast<int64_t>(p.cand_row_ptr[I + 1]) <= c) ++I;
      const int J = p.cand_col[c];
      bool kp = J >= p.forced_lo[I] && J <= p.forced_hi[I];
      if (!kp && J >= 0 && J < g.nb) {
        const int q0 = I * BS, q1 = min(q0 + BS, g.n);
        const double need_links = g.theta_c * (q1 - q0);
        const int k0 = J * BS, k1 = min(k0 + BS, g.n), nJ = k1 - k0;
        int n_active = 0;
#pragma unroll
        for (int x = 0; x < kColsPerLane; ++x) {
          const int k = k0 + lane + 32 * x;
          uint32_t cnt = 0;
          if (k < k1) {
            const int j = k / g.nt, v = k % g.nt;
            // I's tokens in runs of one frame i; in each run only the u within
            // w(t) of v are in P(i, j)
            for (int q = q0; q < q1;) {
              const int i = q / g.nt, ua = q % g.nt;
              const int qe = min(q1, (i + 1) * g.nt);
              const int t = i > j ? i - j : j - i;
              if (rt[t]) {
                const int lo = max(ua, v - wt[t]), hi = min(ua + (qe - q) - 1, v + wt[t]);
                if (lo <= hi) {
                  if (t < 2) {
                    cnt += hi - lo + 1;   // no sampling at t <= 1
                  } else {
                    const uint64_t T = p.thresholds[static_cast<int64_t>(i) * g.frames + j];
                    uint64_t z = sample_state(p.seed, g.frames, g.nt, i, j, lo, v);
                    for (int u = lo; u <= hi; ++u, z += ustep) cnt += splitmix64_mix(z) <= T ? 1u : 0u;
                  }
                }
              }
              q = qe;
            }
          }
          n_active += __popc(__ballot_sync(0xffffffffu, k < k1 && static_cast<double>(cnt) > need_links));
        }
        kp = static_cast<double>(n_active) > g.theta_m * nJ;
      } else if (!kp) {
        if (lane == 0) record_error(DYNRAD_ERR_DEVICE);   // not a block index: dropped
      }
      if (lane == 0) p.keep[c] = kp ? 1 : 0;
    }
  }
}

// One warp per query block I: its kept candidates in list order at the
// row's candidate offsets, and its count.
__global__ void __launch_bounds__(kSampleThreads) sample_compact_kernel(SampleParams p) {
  const int lane = threadIdx.x & 31;
  const int I = (blockIdx.x * kSampleThreads + threadIdx.x) >> 5;
  if (I >= p.g.nb) return;   // whole warps
  const int c_beg = p.cand_row_ptr[I];
  int nc = p.cand_row_ptr[I + 1] - c_beg;
  if (c_beg < 0 || nc < 0 || static_cast<int64_t>(c_beg) + nc > p.cand_nnz) {   // not a candidate row
    if (lane == 0) record_error(DYNRAD_ERR_CAPACITY);
    nc = 0;
  }
  int n_kept = 0;
  for (int c0 = 0; c0 < nc; c0 += 32) {   // warp-uniform
    const int c = c0 + lane;
    const bool k_ = c < nc && p.keep[c_beg + c] != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, k_);
    if (k_) p.kept_tmp[c_beg + n_kept + __popc(bal & ((1u << lane) - 1u))] = p.cand_col[c_beg + c];
    n_kept += __popc(bal);
  }
  if (lane == 0) p.counts[I] = n_kept;
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
