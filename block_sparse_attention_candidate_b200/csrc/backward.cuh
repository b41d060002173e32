// Backward of the block-sparse attention (the gradient the mask-aware
// fine-tuning of DynamicRad Sec. 3.3 needs): dQ, dK, dV from dO, the forward's
// O and LSE, and the same kept-block CSR.
//
//   P = exp(scale Q K^T - LSE) on the kept blocks (0 elsewhere),
//   dV = P^T dO,  dP = dO V^T,  dS = P (dP - D_r),  D_r = rowsum(dO * O),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Kernels (64-row tiles; a block of 64 or 128 tokens is one or two tiles; the
// tiles' products are warp-level bf16 tensor-core MMAs, m16n8k16 with fp32
// accumulation, each warp owning 16 rows of its CTA's tile):
//   bwd_rowdot_kernel     D_r per query row.
//   bwd_tcount_kernel, scan, bwd_tfill_kernel   the transposed CSR: for each
//                         key block, the query blocks that keep it, ascending.
//   bwd_dkv_kernel<D>     one CTA per (head, 64-key tile): walks the key
//                         block's query blocks, recomputes S^T and dP^T, and
//                         accumulates dV and dK in registers (no atomics).
//   bwd_dq_kernel<D>      one CTA per (head, 64-query tile): walks the row's
//                         kept key blocks and accumulates dQ (no atomics).
// P^T / dS^T feed the second products straight from the accumulator
// registers (the m16n8 accumulator pairs are the m16k16 operand pairs).
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "warp_mma.cuh"

namespace dynrad {

constexpr int kBwdTile = 64;
constexpr int kBwdThreads = 128;

struct BwdParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;         // [BH, N] natural log
  float* rowdot;            // [BH, N] D_r
  const int32_t* row_ptr;   // [BH * nb + 1]
  const int32_t* col_idx;
  int32_t* t_ptr;           // [BH * nb + 1] transposed CSR
  int32_t* t_col;
  int64_t t_cap;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int BH, N, nb, block;
  float scale;              // logit scale
};

__global__ void bwd_rowdot_kernel(BwdParams p, int D) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<int64_t>(p.BH) * p.N) return;
  float s = 0.f;
  for (int d = lane; d < D; d += 32)
    s = fmaf(__bfloat162float(p.dout[row * D + d]), __bfloat162float(p.o[row * D + d]), s);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) p.rowdot[row] = s;
}

// one warp per (head, query block): count its key blocks
__global__ void bwd_tcount_kernel(BwdParams p) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= static_cast<int64_t>(p.BH) * p.nb) return;
  const int64_t bh = r / p.nb;
  for (int c = p.row_ptr[r] + lane; c < p.row_ptr[r + 1]; c += 32) {
    const int J = p.col_idx[c];
    if (J >= 0 && J < p.nb) atomicAdd(&p.t_ptr[bh * p.nb + J], 1);
  }
}

__device__ __forceinline__ bool sorted_contains(const int32_t* a, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < x) lo = mid + 1;
    else hi = mid;
  }
  return lo < n && a[lo] == x;
}

// one warp per (head, key block J): the query blocks whose lists hold J, ascending
__global__ void bwd_tfill_kernel(BwdParams p) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= static_cast<int64_t>(p.BH) * p.nb) return;
  const int64_t bh = r / p.nb;
  const int J = static_cast<int>(r - bh * p.nb);
  int64_t out = p.t_ptr[r];
  for (int I0 = 0; I0 < p.nb; I0 += 32) {
    const int I = I0 + lane;
    bool has = false;
    if (I < p.nb) {
      const int64_t row = bh * p.nb + I;
      const int c0 = p.row_ptr[row];
      has = sorted_contains(p.col_idx + c0, p.row_ptr[row + 1] - c0, J);
    }
    const unsigned bal = __ballot_sync(0xffffffffu, has);
    if (has) {
      const int64_t d = out + __popc(bal & ((1u << lane) - 1u));
      if (d < p.t_cap) p.t_col[d] = I;
      else record_error(DYNRAD_ERR_CAPACITY);
    }
    out += __popc(bal);
  }
}

// Stage 64 rows x D of a [BH, N, D] bf16 tensor into shared memory (row
// stride D + 8), zeros past N.
template <int D>
__device__ __forceinline__ void bwd_stage(__nv_bfloat16* dst, const __nv_bfloat16* src, int64_t bh, int N, int r0) {
  constexpr int kVec = D / 8;   // 16-byte pieces per row
  for (int e = threadIdx.x; e < kBwdTile * kVec; e += kBwdThreads) {
    const int r = e / kVec, x = (e % kVec) * 8;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r0 + r < N) val = *reinterpret_cast<const uint4*>(src + (bh * N + r0 + r) * D + x);
    *reinterpret_cast<uint4*>(dst + r * (D + 8) + x) = val;
  }
}

// acc[8][4] (16 rows x 64 columns) += A(16 x D rows of a_s) * B^T, B = 64 rows x D of b_s
template <int D>
__device__ __forceinline__ void bwd_rows_by_rows(float (&acc)[8][4], const __nv_bfloat16* a_s, const __nv_bfloat16* b_s,
                                                 int row0, int lane) {
  constexpr int RS = D + 8;
  const uint32_t a_addr = smem_u32(a_s + (row0 + (lane & 15)) * RS + ((lane >> 4) << 3));
  const uint32_t b_addr = smem_u32(b_s + (((lane >> 4) << 3) + (lane & 7)) * RS + (((lane >> 3) & 1) << 3));
#pragma unroll
  for (int k0 = 0; k0 < D; k0 += 16) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4(a_addr + k0 * 2, a0, a1, a2, a3);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(b_addr + (np * 16 * RS + k0) * 2, b0, b1, b2, b3);
      mma_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
      mma_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
    }
  }
}

// out[D/8][4] (16 rows x D) += X (16 x 64, from accumulator registers) * B, B = 64 rows x D of b_s
template <int D>
__device__ __forceinline__ void bwd_acc_times_rows(float (&out)[D / 8][4], const float (&x)[8][4],
                                                   const __nv_bfloat16* b_s, int lane) {
  constexpr int RS = D + 8;
  const uint32_t b_addr = smem_u32(b_s + ((((lane >> 3) & 1) << 3) + (lane & 7)) * RS + ((lane >> 4) << 3));
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint32_t a0 = pack_bf16x2(x[2 * kk][0], x[2 * kk][1]);
    const uint32_t a1 = pack_bf16x2(x[2 * kk][2], x[2 * kk][3]);
    const uint32_t a2 = pack_bf16x2(x[2 * kk + 1][0], x[2 * kk + 1][1]);
    const uint32_t a3 = pack_bf16x2(x[2 * kk + 1][2], x[2 * kk + 1][3]);
#pragma unroll
    for (int nd = 0; nd < D / 16; ++nd) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_trans(b_addr + (kk * 16 * RS + nd * 16) * 2, b0, b1, b2, b3);
      mma_16816(out[2 * nd], a0, a1, a2, a3, b0, b1);
      mma_16816(out[2 * nd + 1], a0, a1, a2, a3, b2, b3);
    }
  }
}

template <int D>
__device__ __forceinline__ void bwd_store(__nv_bfloat16* dst, const float (&acc)[D / 8][4], float mul, int64_t bh,
                                          int N, int r0, int lane) {
  const int g4 = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + g4 + 8 * h;
      if (r < N)
        *reinterpret_cast<uint32_t*>(dst + (bh * N + r) * D + n * 8 + 2 * t4) =
            pack_bf16x2(acc[n][2 * h] * mul, acc[n][2 * h + 1] * mul);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dkv_kernel(BwdParams p) {
  extern __shared__ __align__(16) __nv_bfloat16 bwd_smem[];
  constexpr int RS = D + 8;
  __nv_bfloat16* ks = bwd_smem;
  __nv_bfloat16* vs = ks + kBwdTile * RS;
  __nv_bfloat16* qs = vs + kBwdTile * RS;
  __nv_bfloat16* dos = qs + kBwdTile * RS;
  __shared__ float lse_s[kBwdTile], dot_s[kBwdTile];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int64_t bh = blockIdx.y;
  const int key0 = blockIdx.x * kBwdTile;
  const int J = key0 / p.block;
  const float c2 = p.scale * 1.4426950408889634f;
  bwd_stage<D>(ks, p.k, bh, p.N, key0);
  bwd_stage<D>(vs, p.v, bh, p.N, key0);
  float acc_dk[D / 8][4], acc_dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc_dk[n][e] = acc_dv[n][e] = 0.f;
  const int tiles_per_block = p.block / kBwdTile;
  const int64_t tr = bh * p.nb + J;
  for (int c = p.t_ptr[tr]; c < p.t_ptr[tr + 1]; ++c) {
    const int I = p.t_col[c];
    for (int qt = 0; qt < tiles_per_block; ++qt) {
      const int q0 = I * p.block + qt * kBwdTile;
      if (q0 >= p.N) break;
      __syncthreads();   // the previous tile's Q / dO are consumed
      bwd_stage<D>(qs, p.q, bh, p.N, q0);
      bwd_stage<D>(dos, p.dout, bh, p.N, q0);
      for (int r = threadIdx.x; r < kBwdTile; r += kBwdThreads) {
        const bool in = q0 + r < p.N;
        lse_s[r] = in ? p.lse[bh * p.N + q0 + r] * 1.4426950408889634f : INFINITY;   // padded rows: P = 0
        dot_s[r] = in ? p.rowdot[bh * p.N + q0 + r] : 0.f;
      }
      __syncthreads();
      float s[8][4], dp[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
      bwd_rows_by_rows<D>(s, ks, qs, warp * 16, lane);    // S^T: keys x queries
      bwd_rows_by_rows<D>(dp, vs, dos, warp * 16, lane);  // dP^T
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + warp * 16 + g4 + 8 * (e >> 1);
          const int qi = n * 8 + 2 * t4 + (e & 1);
          const float pv = key < p.N ? exp2f(s[n][e] * c2 - lse_s[qi]) : 0.f;
          s[n][e] = pv;
          dp[n][e] = pv * (dp[n][e] - dot_s[qi]);
        }
      }
      bwd_acc_times_rows<D>(acc_dv, s, dos, lane);   // dV += P^T dO
      bwd_acc_times_rows<D>(acc_dk, dp, qs, lane);   // dK += dS^T Q
    }
  }
  bwd_store<D>(p.dk, acc_dk, p.scale, bh, p.N, key0 + warp * 16, lane);
  bwd_store<D>(p.dv, acc_dv, 1.0f, bh, p.N, key0 + warp * 16, lane);
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dq_kernel(BwdParams p) {
  extern __shared__ __align__(16) __nv_bfloat16 bwd_smem[];
  constexpr int RS = D + 8;
  __nv_bfloat16* qs = bwd_smem;
  __nv_bfloat16* dos = qs + kBwdTile * RS;
  __nv_bfloat16* ks = dos + kBwdTile * RS;
  __nv_bfloat16* vs = ks + kBwdTile * RS;
  __shared__ float lse_s[kBwdTile], dot_s[kBwdTile];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int64_t bh = blockIdx.y;
  const int q0 = blockIdx.x * kBwdTile;
  const int I = q0 / p.block;
  const float c2 = p.scale * 1.4426950408889634f;
  bwd_stage<D>(qs, p.q, bh, p.N, q0);
  bwd_stage<D>(dos, p.dout, bh, p.N, q0);
  for (int r = threadIdx.x; r < kBwdTile; r += kBwdThreads) {
    const bool in = q0 + r < p.N;
    lse_s[r] = in ? p.lse[bh * p.N + q0 + r] * 1.4426950408889634f : INFINITY;
    dot_s[r] = in ? p.rowdot[bh * p.N + q0 + r] : 0.f;
  }
  float acc_dq[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc_dq[n][e] = 0.f;
  const int tiles_per_block = p.block / kBwdTile;
  const int64_t row = bh * p.nb + I;
  for (int c = p.row_ptr[row]; c < p.row_ptr[row + 1]; ++c) {
    const int J = p.col_idx[c];
    if (J < 0 || J >= p.nb) continue;
    for (int kt = 0; kt < tiles_per_block; ++kt) {
      const int k0 = J * p.block + kt * kBwdTile;
      if (k0 >= p.N) break;
      __syncthreads();
      bwd_stage<D>(ks, p.k, bh, p.N, k0);
      bwd_stage<D>(vs, p.v, bh, p.N, k0);
      __syncthreads();
      float s[8][4], dp[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
      bwd_rows_by_rows<D>(s, qs, ks, warp * 16, lane);    // S: queries x keys
      bwd_rows_by_rows<D>(dp, dos, vs, warp * 16, lane);  // dP
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qi = warp * 16 + g4 + 8 * (e >> 1);
          const int key = k0 + n * 8 + 2 * t4 + (e & 1);
          const float pv = key < p.N ? exp2f(s[n][e] * c2 - lse_s[qi]) : 0.f;
          dp[n][e] = pv * (dp[n][e] - dot_s[qi]);
        }
      }
      bwd_acc_times_rows<D>(acc_dq, dp, ks, lane);   // dQ += dS K
    }
  }
  bwd_store<D>(p.dq, acc_dq, p.scale, bh, p.N, q0 + warp * 16, lane);
}

}  // namespace dynrad
