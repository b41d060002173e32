// Stage 3: block-sparse attention forward on the 5th-generation tensor cores
// (DynamicRad, Sec. 3.3, Eqs. 12-13 with epsilon -> 0).
//
// One CTA computes one tile of 128 query rows (R = 128 / B_s query blocks) of
// one (batch, head).  It walks the ascending union of the R rows' kept-block
// lists; at each step one key block J is loaded and the rows whose own list
// lacks J are masked to -inf.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t of the tile = TMEM lane t.
//              Reads S = Q K^T from TMEM, keeps the running max / sum in fp32
//              (lazy rescale: O is rescaled only when the row max grows by more
//              than 2^8), writes P = exp2(...) as bf16 into TMEM, and finally
//              normalises O and writes O and the log-sum-exp.
//   warp 4     producer: merges the R sorted CSR rows and issues TMA loads of the
//              Q tile and of K_J / V_J (128-byte swizzled, non-multicast) into a
//              STAGES-deep shared-memory ring.
//   warp 5     MMA issuer (one thread): S_j = Q K_j^T (A, B from shared memory)
//              and O += P_j V_j (A = P from tensor memory, B = V from shared
//              memory, MN-major), accumulators in tensor memory.
//
// Tensor memory (512 columns): O [0, D), S0 [128, 128+B_s), S1 [256, 256+B_s),
// P0 [384, 384+B_s/2), P1 [448, 448+B_s/2).  Two S and two P buffers let the
// MMA of step j+1 run while the softmax of step j is in flight.
//
// Every wait is bounded (common.cuh): a wait that runs out records
// DYNRAD_ERR_DEVICE, raises a CTA-wide abort flag, and all roles unwind to the
// common exit where tensor memory is released.
#pragma once

#include "common.cuh"

namespace dynrad {

template <int D, int BS>
struct AttnCfg {
  static constexpr int kM = 128;
  static constexpr int kR = kM / BS;                 // query blocks per tile
  static constexpr int kChunks = D / 64;             // 128-byte column chunks
  static constexpr int kQBytes = kM * D * 2;
  static constexpr int kKVBytes = BS * D * 2;        // one K (or V) block
  static constexpr int kStages = (BS == 128) ? 3 : (BS == 64 ? 4 : 6);
  static constexpr int kSmemData = kQBytes + kStages * 2 * kKVBytes;
  static constexpr int kSmemCtrl = 1024;
  // +1024 for the manual 1024-byte alignment; at least 120 KB so that only one
  // CTA (holding all 512 TMEM columns) lives on an SM at a time
  static constexpr int kSmemTotal =
      (kSmemData + kSmemCtrl + 1024) > 122880 ? (kSmemData + kSmemCtrl + 1024) : 122880;
  static constexpr uint32_t kColO = 0, kColS0 = 128, kColS1 = 256, kColP0 = 384, kColP1 = 448;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BS == 32 || BS == 64 || BS == 128, "block size");
};

struct AttnParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  __nv_bfloat16* o;
  float* lse;
  int N;
  int nb;
  float scale_log2;   // logit scale * log2(e)
};

struct RingEntry {
  int32_t J;          // key block, -1 = end of the walk
  uint32_t mask;      // bit r: query block I0 + r keeps J
};

template <int D, int BS>
__global__ void __launch_bounds__(192, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg<D, BS>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t attn_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = smem;
  uint8_t* kv_smem = smem + C::kQBytes;  // stage s: K at 2s, V at 2s+1
  uint8_t* ctrl = smem + C::kSmemData;
  uint64_t* bar = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* q_full = bar;
  uint64_t* k_full = bar + 1;
  uint64_t* v_full = k_full + S;
  uint64_t* kv_empty = v_full + S;
  uint64_t* s_full = kv_empty + S;   // [2]
  uint64_t* p_full = s_full + 2;     // [2]
  uint64_t* pv_done = p_full + 2;    // [2]
  uint64_t* drain = pv_done + 2;
  RingEntry* ring = reinterpret_cast<RingEntry*>(drain + 1);
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(ring + S);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_s + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int bh = blockIdx.y;
  const int I0 = tile * C::kR;
  const int q_row0 = I0 * BS;
  const int nb = p.nb;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_base_s, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_base_s;

  if (warp == 4) {
    // ------------------------------------------------------------- producer
    int32_t ptr = 0, end = 0, cur = INT32_MAX;
    if (lane < C::kR && I0 + lane < nb) {
      const int64_t row = static_cast<int64_t>(bh) * nb + I0 + lane;
      ptr = p.row_ptr[row];
      end = p.row_ptr[row + 1];
      while (ptr < end) {
        const int32_t c = p.col_idx[ptr];
        if (c >= 0 && c < nb) { cur = c; break; }
        record_error(DYNRAD_ERR_DEVICE);
        ++ptr;
      }
    }
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_3d(q_smem + c * (C::kM * 128), &tm_q, q_full, c * 64, q_row0, bh);
    }
    int j = 0;
    bool ok = true;
    for (;; ++j) {
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
          const int32_t c = p.col_idx[ptr];
          if (c > m && c < nb) { cur = c; break; }
          record_error(DYNRAD_ERR_DEVICE);
          ++ptr;
        }
      }
      const int s = j % S;
      if (j >= S) {
        bool w = true;
        if (lane == 0) w = mbar_wait(&kv_empty[s], ((j / S) - 1) & 1, abort_flag);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
      }
      if (lane == 0) {
        ring[s].J = (m == INT32_MAX) ? -1 : m;
        ring[s].mask = mask;
        if (m == INT32_MAX) {
          mbar_arrive(&k_full[s]);
        } else {
          uint8_t* ks = kv_smem + (2 * s) * C::kKVBytes;
          uint8_t* vs = kv_smem + (2 * s + 1) * C::kKVBytes;
          mbar_arrive_expect_tx(&k_full[s], C::kKVBytes);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(ks + c * (BS * 128), &tm_k, &k_full[s], c * 64, m * BS, bh);
          mbar_arrive_expect_tx(&v_full[s], C::kKVBytes);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(vs + c * (BS * 128), &tm_v, &v_full[s], c * 64, m * BS, bh);
        }
      }
      __syncwarp();
      if (m == INT32_MAX) break;
    }
    if (!ok && lane == 0) {
      // unwinding: let the copies already issued land before shared memory is
      // given back (bounded; ignores the abort flag)
      for (int i = (j > S ? j - S : 0); i < j; ++i) {
        mbar_wait(&k_full[i % S], (i / S) & 1, nullptr);
        mbar_wait(&v_full[i % S], (i / S) & 1, nullptr);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BS, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_base = smem_u32(q_smem);
      const uint32_t kv_base = smem_u32(kv_smem);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      int j = 0;
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(&v_full[i % S], (i / S) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t v_addr = kv_base + (2 * (i % S) + 1) * C::kKVBytes;
        const uint32_t p_col = (i & 1) ? C::kColP1 : C::kColP0;
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk) {
          // V block [BS keys][D] as the MN-major B operand: 64-column chunks
          // BS*128 bytes apart (leading offset), 8-key groups 1024 bytes apart
          const uint64_t bdesc = smem_desc_sw128(v_addr + kk * 2048, BS * 128, 1024);
          mma_ts(taddr + C::kColO, taddr + p_col + kk * 8, bdesc, idesc_pv,
                 (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&kv_empty[i % S]);
        mma_commit(&pv_done[i & 1]);
        return true;
      };
      while (ok) {
        const int s = j % S;
        if (!mbar_wait(&k_full[s], (j / S) & 1, abort_flag)) { ok = false; break; }
        const RingEntry e = ring[s];
        if (e.J < 0) break;
        tc_fence_after();
        const uint32_t k_addr = kv_base + (2 * s) * C::kKVBytes;
        const uint32_t s_col = (j & 1) ? C::kColS1 : C::kColS0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(q_base + c * (C::kM * 128) + off, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(k_addr + c * (BS * 128) + off, 16, 1024);
          mma_ss(taddr + s_col, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[j & 1]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
        ++j;
      }
      if (ok && j >= 1) issue_pv(j - 1);
      // all issued tensor-core work finished before tensor memory is released
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- softmax
    const int t = threadIdx.x;             // tile row = TMEM lane
    const int sub = t / BS;                // query block within the tile
    const int row = q_row0 + t;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_used = -INFINITY;              // running max in log2 units
    float l = 0.f;
    int j = 0;
    bool ok = true;
    for (;; ++j) {
      const int s = j % S;
      if (!mbar_wait(&k_full[s], (j / S) & 1, abort_flag)) { ok = false; break; }
      const RingEntry e = ring[s];
      if (e.J < 0) break;
      if (!mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const bool active = (e.mask >> sub) & 1u;
      const int nvalid = min(BS, p.N - e.J * BS);
      const uint32_t s_col = (j & 1) ? C::kColS1 : C::kColS0;
      float sv[BS];
#pragma unroll
      for (int c = 0; c < BS / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + lane_base + s_col + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(r[i]);
      }
      float mx = -INFINITY;
      if (active) {
#pragma unroll
        for (int i = 0; i < BS; ++i)
          if (i < nvalid) mx = fmaxf(mx, sv[i]);
      }
      const float m_new = active ? fmaxf(m_used, mx * p.scale_log2) : m_used;
      const bool need = active && m_used != -INFINITY && m_new > m_used + 8.0f;
      if (__any_sync(0xffffffffu, need)) {
        // rescale O: the previous P V product must have landed first
        if (!mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const float alpha = need ? ex2_approx(m_used - m_new) : 1.0f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + lane_base + C::kColO + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(taddr + lane_base + C::kColO + c * 32, r);
        }
        tmem_wait_st();
        if (need) {
          l *= alpha;
          m_used = m_new;
        }
      }
      if (active && m_used == -INFINITY) m_used = m_new;
      uint32_t pk[BS / 2];
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < BS; i += 2) {
        const float p0 = (active && i < nvalid) ? ex2_approx(fmaf(sv[i], p.scale_log2, -m_used)) : 0.f;
        const float p1 = (active && i + 1 < nvalid) ? ex2_approx(fmaf(sv[i + 1], p.scale_log2, -m_used)) : 0.f;
        rs += p0 + p1;
        pk[i / 2] = pack_bf16x2(p0, p1);
      }
      l += rs;
      // P buffer j&1 was last read by the P V product of step j-2
      if (j >= 2) {
        if (!mbar_wait(&pv_done[j & 1], ((j - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
      }
      const uint32_t p_col = (j & 1) ? C::kColP1 : C::kColP0;
      if constexpr (BS == 32) {
        tmem_st16(taddr + lane_base + p_col, pk);
      } else {
#pragma unroll
        for (int c = 0; c < BS / 64; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = pk[c * 32 + i];
          tmem_st32(taddr + lane_base + p_col + c * 32, r);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
    }
    const int n_steps = j;
    if (ok) {
      bool have_o = n_steps > 0;
      if (have_o) {
        if (!mbar_wait(&pv_done[(n_steps - 1) & 1], ((n_steps - 1) >> 1) & 1, abort_flag)) have_o = false;
        tc_fence_after();
      }
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        if (have_o) {
          tmem_ld32(taddr + lane_base + C::kColO + c * 32, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0u;
        }
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
        if (row < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
      if (row < p.N)
        p.lse[static_cast<size_t>(bh) * p.N + row] =
            l > 0.f ? m_used * 0.69314718055994531f + __logf(l) : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(taddr, C::kTmemCols);
}

}  // namespace dynrad
