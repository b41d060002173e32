// Backward of the block-sparse attention (the gradient the mask-aware
// fine-tuning of DynamicRad Sec. 3.3 needs): dQ, dK, dV from dO, the forward's
// O and LSE, and the same kept-block CSR.
//
//   P = exp(scale Q K^T - LSE) on the kept blocks (0 elsewhere),
//   dV = P^T dO,  dP = dO V^T,  dS = P (dP - D_r),  D_r = rowsum(dO * O),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Kernels:
//   bwd_aux_kernel        per query row -lse log2(e) and -D_r, stored per pair of
//                         rows (q even) as {-lse2_q, -lse2_q+1, -D_q, -D_q+1} so
//                         the elementwise pass feeds them straight to paired
//                         FP32 ops; rows padded to a multiple of 64 with
//                         (-inf, 0).
//   bwd_tcount_kernel, scan, bwd_tfill_kernel   the transposed CSR: for each
//                         key block, the query blocks that keep it, ascending.
//   bwd_tc_kernel<D, BS, true>   dK, dV per 128-key tile (tcgen05, TMEM, TMA).
//   bwd_tc_kernel<D, BS, false>  dQ per 128-query tile.
// Each output row is owned by one CTA: no atomics, deterministic.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace dynrad {

struct BwdParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;         // [BH, N] natural log
  float* aux;               // [BH, Np / 2] x {-lse2 (2 rows), -D_r (2 rows)}; rows >= N: (-inf, 0)
  int Np;                   // N rounded up to 64
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

// Position of row i's -lse2 in the pair layout (its -D_r is 2 floats later).
__host__ __device__ __forceinline__ int64_t bwd_aux_index(int64_t bh, int64_t np, int64_t i) {
  return (bh * np + (i & ~static_cast<int64_t>(1))) * 2 + (i & 1);
}

__global__ void bwd_aux_kernel(BwdParams p, int D) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= static_cast<int64_t>(p.BH) * p.Np) return;
  const int64_t bh = r / p.Np;
  const int i = static_cast<int>(r - bh * p.Np);
  float* dst = p.aux + bwd_aux_index(bh, p.Np, i);
  if (i >= p.N) {
    if (lane == 0) {
      dst[0] = -INFINITY;
      dst[2] = 0.f;
    }
    return;
  }
  const int64_t row = bh * p.N + i;
  float s = 0.f;
  for (int d = lane; d < D; d += 32)
    s = fmaf(__bfloat162float(p.dout[row * D + d]), __bfloat162float(p.o[row * D + d]), s);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    dst[0] = -p.lse[row] * 1.4426950408889634f;
    dst[2] = -s;
  }
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


// ----------------------------------------------------------------------------
// Tensor-core gradient kernels.  One template serves both sides:
//   KV = true   one CTA per (head, 128-key tile): resident K, V; streams the
//               Q / dO rows of the query blocks that keep the tile's key
//               blocks; accumulates dV = P^T dO and dK = dS^T Q.
//   KV = false  one CTA per (head, 128-query tile): resident Q, dO; streams the
//               K / V rows of the tile's kept key blocks; accumulates dQ = dS K.
// The tile's rows are R = 128 / BS blocks; their lists (transposed CSR for
// KV, the forward's CSR otherwise) are merged into one ascending walk, and a
// union member's BS rows are streamed as BS / 64 steps of 64 rows (a 32-row
// block as one step whose second half is masked).  A step's
// mask bit r says whether list r holds the member: the tile rows of block r
// get P = 0 otherwise.
//
// Per step j (buffer b = j mod NB; NB = 3 X / Y buffers where tensor memory
// has room, 2 for dK / dV at D = 128):
//   G12  X_b = A0 B0^T, Y_b = A1 B1^T (A = resident tiles, B = the step's
//        tiles; M = 128, N = 64, K = D).  KV: X = S^T, Y = dP^T; else X = S,
//        Y = dP.
//   elementwise (warps 0-7; thread = TMEM lane = tile row; warpgroup g takes
//        the steps j with j mod 2 = g, so two steps' passes overlap):
//        P = 2^(X c - lse2), dS = P (Y - D_r) over the step's 64 columns; P
//        (KV only) and dS are written back as bf16 pairs over the first 32
//        columns of X_b and Y_b (each warp touches only its own 32 lanes).
//   G34  KV: dV += P^T B1, dK += dS^T B0; else dQ += dS B0 (A from tensor
//        memory, B = the step's tile as the MN-major operand; M = 128, N = D,
//        K = 64).
// The MMA thread issues G34(j) and then G12(j + NB) into the same buffer, so
// the tensor core runs the G12 of the next NB - 1 steps while step j's
// elementwise pass runs.
//
// Warp roles (320 threads): warps 0-7 elementwise and epilogue, warp 8
// producer (list walk, TMA loads into a ring of slots, per-query lse2 / D_r of
// the step for KV), warp 9 MMA issuer.  Tensor memory (512 columns): acc0 at 0
// (dV or dQ); KV: acc1 (dK) at D; dQ side: Q at D and dO at 3D / 2 as bf16
// pairs (G12's A operands, written by the elementwise warps); then X_b at
// 2D + 128 b and Y_b at 2D + 128 b + 64.  KV keeps K, V in shared memory (G12
// reads them from there).  Every wait is bounded (common.cuh).
// ----------------------------------------------------------------------------
// 2-D tiled TMA load (non-multicast) of the per-row (-lse2, -D_r) pairs.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

struct BwdStepMeta {
  int32_t row0;     // first streamed row of the step
  uint32_t mask;    // bit r: list r holds the union member
  int32_t end;      // 1: the walk is over
  int32_t pad;
};

template <int D, int BS, bool KV>
struct BwdTcCfg {
  static constexpr int kRows = 128;
  static constexpr int kStep = 64;
  static constexpr int kR = kRows / BS;
  // steps per union member; a 32-row block fills the first half of one step
  static constexpr int kSPB = BS >= kStep ? BS / kStep : 1;
  static constexpr int kChunks = D / 64;
  static constexpr int kResBytes = kRows * D * 2;
  static constexpr int kResChunk = kRows * 128;
  static constexpr int kStepBytes = kStep * D * 2;
  static constexpr int kStepChunk = kStep * 128;
  static constexpr int kSlotBytes = 2 * kStepBytes + 1024;   // two tiles, (lse2, D_r) x 64, meta
  static constexpr int kAuxBytes = KV ? 64 * 8 : 0;
  static constexpr int kSmemCtrl = 1024;
  static constexpr int kBudget = 227 * 1024 - kSmemCtrl - 1024;
  // KV: K, V resident in shared memory (the A operands of G12).  dQ side: Q,
  // dO resident in tensor memory instead, so G12 reads only the step's tiles
  // from shared memory and the freed space holds more slots.
  static constexpr int kResSmem = KV ? 2 * kResBytes : 0;
  static constexpr int kSlotsRaw = (kBudget - kResSmem) / kSlotBytes;
  static constexpr int kSlots = kSlotsRaw > 6 ? 6 : kSlotsRaw;
  static constexpr int kSmemData = kResSmem + kSlots * kSlotBytes;
  static constexpr int kSmemTotal = kSmemData + kSmemCtrl + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kAcc0 = 0;
  static constexpr uint32_t kAcc1 = D;                 // KV: dK
  static constexpr uint32_t kResA0 = D, kResA1 = D + D / 2;   // dQ side: Q, dO as bf16 pairs
  static constexpr uint32_t kXY = 2 * D;
  // X / Y buffers: as many 128-column pairs as tensor memory holds, at most 3
  static constexpr int kBufs = (kTmemCols - kXY) / 128 > 3 ? 3 : static_cast<int>((kTmemCols - kXY) / 128);
  __host__ __device__ static constexpr uint32_t col_x(int b) { return kXY + 128u * b; }
  __host__ __device__ static constexpr uint32_t col_y(int b) { return kXY + 128u * b + 64u; }
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BS == 32 || BS == 64 || BS == 128, "block size");
  static_assert(kBufs >= 2 && kXY + 128u * kBufs <= kTmemCols, "tensor memory");
  // G12(j + kBufs) waits for step j + kBufs's slot, which is freed by G34(j + kBufs - kSlots)
  static_assert(kSlots >= kBufs + 1, "slots for the MMA issue order");
  static_assert(kSmemTotal <= 227 * 1024, "shared memory");
};

template <int D, int BS, bool KV>
__global__ void __launch_bounds__(320, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_res0, const __grid_constant__ CUtensorMap tm_res1,
                  const __grid_constant__ CUtensorMap tm_step0, const __grid_constant__ CUtensorMap tm_step1,
                  const __grid_constant__ CUtensorMap tm_aux, const BwdParams p) {
  using C = BwdTcCfg<D, BS, KV>;
  constexpr int NS = C::kSlots;
  constexpr int NB = C::kBufs;
  extern __shared__ uint8_t bwd_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(bwd_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* res_smem = smem;                        // KV: A0 at 0, A1 at kResBytes
  uint8_t* slot_smem = smem + C::kResSmem;         // step j in slot j % NS
  uint8_t* ctrl = smem + C::kSmemData;
  uint64_t* bar = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* res_full = bar;
  uint64_t* slot_full = bar + 1;          // [NS]
  uint64_t* slot_empty = slot_full + NS;  // [NS]
  uint64_t* s_full = slot_empty + NS;     // [NB]
  uint64_t* p_full = s_full + NB;         // [NB]
  uint64_t* drain = p_full + NB;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_s + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int tile0 = blockIdx.x * C::kRows;   // first resident row
  const int blk0 = blockIdx.x * C::kR;       // first resident block
  const int nb = p.nb;
  const float log2e = 1.4426950408889634f;

  auto slot_tile = [&](int j, int t) -> uint8_t* { return slot_smem + (j % NS) * C::kSlotBytes + t * C::kStepBytes; };
  auto slot_tail = [&](int j) -> uint8_t* { return slot_smem + (j % NS) * C::kSlotBytes + 2 * C::kStepBytes; };

  if (threadIdx.x == 0) {
    mbar_init(res_full, KV ? 1 : 8);   // KV: the TMA transaction; dQ side: one arrival per elementwise warp
    for (int s = 0; s < NS; ++s) {
      mbar_init(&slot_full[s], 32);
      mbar_init(&slot_empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 4);    // one arrival per warp of the step's warpgroup
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
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
    // lane r < R walks list r; `nxt` holds the entry after `cur`, loaded one
    // union member ahead so the walk does not wait on memory
    const int32_t* lst = KV ? p.t_col : p.col_idx;
    int32_t ptr = 0, end = 0, cur = INT32_MAX, nxt = INT32_MAX;
    if (lane < C::kR && blk0 + lane < nb) {
      const int64_t r = static_cast<int64_t>(bh) * nb + blk0 + lane;
      ptr = KV ? p.t_ptr[r] : p.row_ptr[r];
      end = KV ? p.t_ptr[r + 1] : p.row_ptr[r + 1];
      while (ptr < end) {
        const int32_t c = lst[ptr];
        if (c >= 0 && c < nb) { cur = c; break; }
        record_error(DYNRAD_ERR_DEVICE);
        ++ptr;
      }
      if (ptr + 1 < end) nxt = lst[ptr + 1];
    }
    if (lane == 0) {
      prefetch_tensormap(&tm_res0);
      prefetch_tensormap(&tm_res1);
      prefetch_tensormap(&tm_step0);
      prefetch_tensormap(&tm_step1);
      if (KV) prefetch_tensormap(&tm_aux);
      if (KV) {
        mbar_arrive_expect_tx(res_full, 2 * C::kResBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_3d(res_smem + c * C::kResChunk, &tm_res0, res_full, c * 64, tile0, bh);
          tma_load_3d(res_smem + C::kResBytes + c * C::kResChunk, &tm_res1, res_full, c * 64, tile0, bh);
        }
      }
    }
    bool ok = true;
    int j = 0;   // steps published
    auto slot_ready = [&](int i) -> bool {
      bool w = true;
      if (i >= NS && lane == 0) w = mbar_wait(&slot_empty[i % NS], ((i / NS) - 1) & 1, abort_flag);
      return __shfl_sync(0xffffffffu, w, 0);
    };
    for (;;) {
      int32_t m = cur;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = min(m, __shfl_xor_sync(0xffffffffu, m, off));
      const bool mine = lane < C::kR && cur == m && m != INT32_MAX;
      const uint32_t mask = __ballot_sync(0xffffffffu, mine);
      if (mine) {
        // advance past m, skipping malformed entries (out of range or not ascending)
        ++ptr;
        cur = INT32_MAX;
        while (ptr < end) {
          const int32_t c = nxt;
          nxt = ptr + 1 < end ? lst[ptr + 1] : INT32_MAX;
          if (c > m && c < nb) { cur = c; break; }
          record_error(DYNRAD_ERR_DEVICE);
          ++ptr;
        }
      }
      if (m == INT32_MAX) {
        // end markers: two slots with no tiles (each elementwise warpgroup
        // meets one at the first step of its parity past the walk); row0
        // carries the number of real steps
        const int steps = j;
        for (int e = 0; e < 2 && ok; ++e) {
          if (!slot_ready(j)) { ok = false; break; }
          if (lane == 0) {
            BwdStepMeta* mt = reinterpret_cast<BwdStepMeta*>(slot_tail(j) + 512);
            mt->row0 = steps;
            mt->mask = 0u;
            mt->end = 1;
          }
          __syncwarp();
          mbar_arrive(&slot_full[j % NS]);
          ++j;
        }
        break;
      }
      for (int s = 0; s < C::kSPB; ++s) {
        const int row0 = m * BS + s * C::kStep;
        if (row0 >= p.N) break;
        if (!slot_ready(j)) { ok = false; break; }
        uint8_t* tail = slot_tail(j);
        if (lane == 0) {
          BwdStepMeta* mt = reinterpret_cast<BwdStepMeta*>(tail + 512);
          mt->row0 = row0;
          mt->mask = mask;
          mt->end = 0;
          mbar_arrive_expect_tx(&slot_full[j % NS], 2 * C::kStepBytes + C::kAuxBytes);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
            tma_load_3d(slot_tile(j, 0) + c * C::kStepChunk, &tm_step0, &slot_full[j % NS], c * 64, row0, bh);
            tma_load_3d(slot_tile(j, 1) + c * C::kStepChunk, &tm_step1, &slot_full[j % NS], c * 64, row0, bh);
          }
          // (lse2, D_r) of the step's 64 queries: 128 floats at x = 2 row0
          if (KV) tma_load_2d(tail, &tm_aux, &slot_full[j % NS], 2 * row0, bh);
        } else {
          mbar_arrive(&slot_full[j % NS]);
        }
        ++j;
      }
      if (!ok) break;
    }
    if (!ok && lane == 0) {
      for (int i = (j > NS ? j - NS : 0); i < j; ++i) mbar_wait(&slot_full[i % NS], (i / NS) & 1, nullptr);
      if (KV) mbar_wait(res_full, 0, nullptr);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_g12 = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idesc_g34 = idesc_bf16_f32(128, D, false, true);
      const uint32_t res_base = smem_u32(res_smem);
      auto desc_add = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (bytes >> 4); };
      bool ok = mbar_wait(res_full, 0, abort_flag);
      bool started = false;
      // G12 of step j into buffer j % NB; false on abort, more = false at the end marker
      auto issue_g12 = [&](int j, bool& more) -> bool {
        if (!mbar_wait(&slot_full[j % NS], (j / NS) & 1, abort_flag)) return false;
        const BwdStepMeta* mt = reinterpret_cast<const BwdStepMeta*>(slot_tail(j) + 512);
        more = mt->end == 0;
        if (!more) return true;
        tc_fence_after();
        const int b = j % NB;
        // each MMA's descriptor is its batch's first one plus a constant (the
        // 14-bit start-address field cannot carry: shared addresses < 2^18)
        const uint64_t r0 = smem_desc_sw128(res_base, 16, 1024);
        const uint64_t r1 = desc_add(r0, C::kResBytes);
        const uint64_t b0 = smem_desc_sw128(smem_u32(slot_tile(j, 0)), 16, 1024);
        const uint64_t b1 = smem_desc_sw128(smem_u32(slot_tile(j, 1)), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          if (KV)
            mma_ss(taddr + C::col_x(b), desc_add(r0, c * C::kResChunk + off), desc_add(b0, c * C::kStepChunk + off),
                   idesc_g12, kk > 0 ? 1u : 0u);
          else   // A = Q from tensor memory: 16 values of K per 8 columns
            mma_ts(taddr + C::col_x(b), taddr + C::kResA0 + kk * 8, desc_add(b0, c * C::kStepChunk + off), idesc_g12,
                   kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          if (KV)
            mma_ss(taddr + C::col_y(b), desc_add(r1, c * C::kResChunk + off), desc_add(b1, c * C::kStepChunk + off),
                   idesc_g12, kk > 0 ? 1u : 0u);
          else   // A = dO from tensor memory
            mma_ts(taddr + C::col_y(b), taddr + C::kResA1 + kk * 8, desc_add(b1, c * C::kStepChunk + off), idesc_g12,
                   kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[b]);
        return true;
      };
      int issued = 0;       // steps whose G12 has been issued
      bool ended = false;   // the end marker has been read
      for (int i = 0; ok && i < NB && !ended; ++i) {
        bool more = false;
        if (!issue_g12(i, more)) ok = false;
        else if (more) ++issued;
        else ended = true;
      }
      for (int j = 0; ok && j < issued; ++j) {
        const int b = j % NB;
        if (!mbar_wait(&p_full[b], (j / NB) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        // the step tile [64 rows][D] as the MN-major B operand: 64-column
        // chunks kStepChunk bytes apart, 8-row groups 1024 bytes apart
        const uint64_t t0d = smem_desc_sw128(smem_u32(slot_tile(j, 0)), C::kStepChunk, 1024);
        const uint64_t t1d = smem_desc_sw128(smem_u32(slot_tile(j, 1)), C::kStepChunk, 1024);
#pragma unroll
        for (int kk = 0; kk < C::kStep / 16; ++kk) {
          const uint32_t acc = (started || kk > 0) ? 1u : 0u;
          if (KV) {
            mma_ts(taddr + C::kAcc0, taddr + C::col_x(b) + kk * 8, desc_add(t1d, kk * 2048), idesc_g34, acc);
            mma_ts(taddr + C::kAcc1, taddr + C::col_y(b) + kk * 8, desc_add(t0d, kk * 2048), idesc_g34, acc);
          } else {
            mma_ts(taddr + C::kAcc0, taddr + C::col_y(b) + kk * 8, desc_add(t0d, kk * 2048), idesc_g34, acc);
          }
        }
        started = true;
        mma_commit(&slot_empty[j % NS]);
        // G12(j + NB) into buffer b, after G34(j) in issue order; only while
        // every step before it exists (else no slot j + NB comes)
        if (!ended) {
          bool more = false;
          if (!issue_g12(j + NB, more)) { ok = false; break; }
          if (more) ++issued;
          else ended = true;
        }
      }
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- elementwise
    const int t = threadIdx.x & 127;                 // tile row = TMEM lane
    const int g = warp >> 2;                         // warpgroup: steps g, g + 2, ...
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int row = tile0 + t;
    const bool row_in = row < p.N;
    const int rbit = t / BS;
    const float c2 = p.scale * log2e;
    float my_nl2 = -INFINITY, my_ndr = 0.f;   // -lse2, -D_r of this row (dQ side)
    if (!KV && row_in) {
      const float* a = p.aux + bwd_aux_index(bh, p.Np, row);
      my_nl2 = a[0];
      my_ndr = a[2];
    }
    if (!KV) {
      // Q (warpgroup 0) and dO (warpgroup 1) row of this thread into tensor
      // memory as bf16 pairs (element 2c in the low half of column c): the A
      // operands of G12
      const __nv_bfloat16* src = (g == 0 ? p.q : p.dout) + (static_cast<int64_t>(bh) * p.N + row) * D;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v4 = row_in ? reinterpret_cast<const uint4*>(src + c * 64)[i] : make_uint4(0u, 0u, 0u, 0u);
          r[4 * i] = v4.x;
          r[4 * i + 1] = v4.y;
          r[4 * i + 2] = v4.z;
          r[4 * i + 3] = v4.w;
        }
        tmem_st32(taddr + lane_base + (g == 0 ? C::kResA0 : C::kResA1) + c * 32, r);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(res_full);
    }
    bool ok = true;
    int steps = 0;   // real steps of the walk (from the end marker)
    for (int j = g;; j += 2) {
      if (!__all_sync(0xffffffffu, mbar_wait(&slot_full[j % NS], (j / NS) & 1, abort_flag))) { ok = false; break; }
      const uint8_t* tail = slot_tail(j);
      const BwdStepMeta mt = *reinterpret_cast<const BwdStepMeta*>(tail + 512);
      if (mt.end) {
        steps = mt.row0;
        break;
      }
      const int b = j % NB;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[b], (j / NB) & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      // KV: per column pair q, q + 1 the step's {-lse2, -lse2, -D_r, -D_r};
      // padded queries carry -lse2 = -inf, so P = 0 there.  dQ side: per-row
      // constants, keys past N masked on the sequence's last step only.
      const float2 cc = make_float2(c2, c2);
      const bool tail_step = !KV && mt.row0 + 64 > p.N;
      uint32_t pk[32], dk[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // with 32-row blocks the step's second 32 columns belong to the next
        // block (not this member), so that half is masked
        const bool kept = row_in && ((mt.mask >> rbit) & 1u) && (BS >= 64 || h == 0);
        uint32_t xr[32], yr[32];
        tmem_ld32(taddr + lane_base + C::col_x(b) + h * 32, xr);
        tmem_ld32(taddr + lane_base + C::col_y(b) + h * 32, yr);
        tmem_wait_ld();
        const float4* aux_s = reinterpret_cast<const float4*>(tail) + h * 16;
        if (!kept) {   // warp-uniform (the warp's 32 rows share one block) but at the sequence end
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[h * 16 + i] = dk[h * 16 + i] = 0u;
        } else {
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2) {
            const int i = 2 * i2;   // column within the half
            float2 l2, dd;
            if (KV) {
              const float4 a = aux_s[i2];
              l2 = make_float2(a.x, a.y);
              dd = make_float2(a.z, a.w);
            } else {
              l2 = make_float2(my_nl2, my_nl2);
              dd = make_float2(my_ndr, my_ndr);
            }
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(xr[i]), __uint_as_float(xr[i + 1])), cc, l2);
            float2 pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if (tail_step) {
              const int k = mt.row0 + h * 32 + i;
              pv.x = k < p.N ? pv.x : 0.f;
              pv.y = k + 1 < p.N ? pv.y : 0.f;
            }
            const float2 y = __fadd2_rn(make_float2(__uint_as_float(yr[i]), __uint_as_float(yr[i + 1])), dd);
            const float2 ds = __fmul2_rn(pv, y);
            pk[h * 16 + i2] = pack_bf16x2(pv.x, pv.y);
            dk[h * 16 + i2] = pack_bf16x2(ds.x, ds.y);
          }
        }
      }
      // P (KV) and dS as bf16 pairs over the first 32 columns of X_b, Y_b: this
      // warp has read all 64 columns of its own lanes, and no other warp
      // touches them
      if (KV) tmem_st32(taddr + lane_base + C::col_x(b), pk);
      tmem_st32(taddr + lane_base + C::col_y(b), dk);
      tmem_wait_st();
      // every lane's stores are complete and fenced before the warp's one arrival
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(drain, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const bool have = steps > 0;
#pragma unroll
      for (int a = 0; a < (KV ? 2 : 1); ++a) {
        // KV: a = 0 dV (scale 1), a = 1 dK (scale); else dQ (scale).  Warpgroup
        // g writes columns [g D / 2, (g + 1) D / 2).
        const uint32_t col = a == 0 ? C::kAcc0 : C::kAcc1;
        const float mul = (KV && a == 0) ? 1.0f : p.scale;
        __nv_bfloat16* dst = KV ? (a == 0 ? p.dv : p.dk) : p.dq;
        __nv_bfloat16* drow = dst + (static_cast<int64_t>(bh) * p.N + row) * D;
#pragma unroll
        for (int c = g * (D / 64); c < (g + 1) * (D / 64); ++c) {
          uint32_t r[32];
          if (have) {
            tmem_ld32(taddr + lane_base + col + c * 32, r);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = 0u;
          }
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
          if (row_in) {
            uint4* d4 = reinterpret_cast<uint4*>(drow + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(taddr, C::kTmemCols);
}

}  // namespace dynrad
