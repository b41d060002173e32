// Stage 3: block-sparse attention forward on the 5th-generation tensor cores
// (DynamicRad, Sec. 3.3, Eqs. 12-13 with epsilon -> 0).
//
// One CTA computes one tile of 128 query rows (R = 128 / B_s query blocks) of
// one (batch, head).  It walks the ascending union of the R rows' kept-block
// lists in key steps of KW = min(B_s, 64) keys (a 128-key block is two steps);
// the rows whose own list lacks the current block are masked to -inf.
//
// Two CTAs share an SM (256 tensor-memory columns and < 113 KB of shared memory
// each), so the softmax of one overlaps the tensor-core work of the other.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t of the tile = TMEM lane t.
//              Loads S = Q K^T from tensor memory, releases it at once (the
//              next Q K^T may overwrite it while the exponentials run), keeps
//              the running max / sum in fp32 (lazy rescale: O is rescaled only
//              when the row max grows by more than 2^8), writes P = 2^(...) as
//              bf16 into tensor memory, and finally normalises O and writes O
//              and the log-sum-exp.
//   warp 4     producer: merges the R sorted CSR rows and issues TMA loads of the
//              Q tile and of the K / V key steps (128-byte swizzled,
//              non-multicast) into a STAGES-deep shared-memory ring.
//   warp 5     MMA issuer (one thread): S = Q K^T (A and B from shared memory)
//              and O += P V (A = P from tensor memory, B = V from shared memory,
//              MN-major); fp32 accumulators in tensor memory.
//
// Tensor memory (256 columns): O [0, D), S [128, 128 + KW), P0 / P1 (KW / 2
// columns each, bf16 pairs) at 192 / 224.  P is double-buffered so the
// softmax of step j+1 need not wait for the P V product of step j.
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
  static constexpr int kKW = BS < 64 ? BS : 64;      // keys per step
  static constexpr int kSub = BS / kKW;              // steps per kept block
  static constexpr int kChunks = D / 64;             // 128-byte column chunks
  static constexpr int kQBytes = kM * D * 2;
  static constexpr int kKVBytes = kKW * D * 2;       // one K (or V) step
  static constexpr int kStagesRaw = (98304 - kQBytes) / (2 * kKVBytes);
  static constexpr int kStages = kStagesRaw < 2 ? 2 : (kStagesRaw > 6 ? 6 : kStagesRaw);
  static constexpr int kSmemData = kQBytes + kStages * 2 * kKVBytes;
  static constexpr int kSmemCtrl = 512;
  static constexpr int kSmemTotal = kSmemData + kSmemCtrl + 1024;  // +1024: manual alignment
  static constexpr uint32_t kColO = 0, kColS = 128, kColP0 = 192, kColP1 = 224;
  static constexpr uint32_t kTmemCols = 256;
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BS == 32 || BS == 64 || BS == 128, "block size");
  static_assert(2 * kSmemTotal <= 227 * 1024, "two CTAs per SM");
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
  int32_t key0;       // first key token of the step, -1 = end of the walk
  uint32_t mask;      // bit r: query block I0 + r keeps the step's block
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int D, int BS>
__global__ void __launch_bounds__(192, 2)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg<D, BS>;
  constexpr int S = C::kStages;
  constexpr int KW = C::kKW;
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
  uint64_t* s_full = kv_empty + S;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;     // [2]
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
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    for (int b = 0; b < 2; ++b) {
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
    int j = 0;  // steps issued
    bool ok = true, done = false;
    while (!done) {
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
      // the kept block's key steps (one, or two halves of a 128-key block);
      // a step entirely past the sequence end is skipped
      const int nsub = (m == INT32_MAX) ? 1 : C::kSub;
      for (int sub = 0; sub < nsub; ++sub) {
        const int key0 = (m == INT32_MAX) ? -1 : m * BS + sub * KW;
        if (key0 >= p.N) continue;
        const int s = j % S;
        if (j >= S) {
          bool w = true;
          if (lane == 0) w = mbar_wait(&kv_empty[s], ((j / S) - 1) & 1, abort_flag);
          w = __shfl_sync(0xffffffffu, w, 0);
          if (!w) { ok = false; done = true; break; }
        }
        if (lane == 0) {
          ring[s].key0 = key0;
          ring[s].mask = mask;
          if (key0 < 0) {
            mbar_arrive(&k_full[s]);
          } else {
            uint8_t* ks = kv_smem + (2 * s) * C::kKVBytes;
            uint8_t* vs = kv_smem + (2 * s + 1) * C::kKVBytes;
            mbar_arrive_expect_tx(&k_full[s], C::kKVBytes);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d(ks + c * (KW * 128), &tm_k, &k_full[s], c * 64, key0, bh);
            mbar_arrive_expect_tx(&v_full[s], C::kKVBytes);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d(vs + c * (KW * 128), &tm_v, &v_full[s], c * 64, key0, bh);
          }
        }
        __syncwarp();
        ++j;
        if (key0 < 0) { done = true; break; }
      }
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
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, KW, false, false);
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
        for (int kk = 0; kk < KW / 16; ++kk) {
          // V step [KW keys][D] as the MN-major B operand: 64-column chunks
          // KW*128 bytes apart (leading offset), 8-key groups 1024 bytes apart
          const uint64_t bdesc = smem_desc_sw128(v_addr + kk * 2048, KW * 128, 1024);
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
        if (e.key0 < 0) break;
        // S is single-buffered: the softmax must have read S_{j-1}
        if (j >= 1 && !mbar_wait(s_free, (j - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = kv_base + (2 * s) * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(q_base + c * (C::kM * 128) + off, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(k_addr + c * (KW * 128) + off, 16, 1024);
          mma_ss(taddr + C::kColS, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
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
    const float c2 = p.scale_log2;
    float m_used = -INFINITY;              // running max in log2 units
    float l = 0.f;
    int j = 0;
    bool ok = true;
    for (;; ++j) {
      const int s = j % S;
      if (!__all_sync(0xffffffffu, mbar_wait(&k_full[s], (j / S) & 1, abort_flag))) { ok = false; break; }
      const RingEntry e = ring[s];
      if (e.key0 < 0) break;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, j & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      float sv[KW];
#pragma unroll
      for (int c = 0; c < KW / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + lane_base + C::kColS + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(r[i]);
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_free);                 // S may be overwritten now
      const bool active = (e.mask >> sub) & 1u;
      const int nvalid = min(KW, p.N - e.key0);
      const bool full = nvalid == KW;
      float mx = -INFINITY;
      if (active) {
        if (full) {
          // four independent max chains, then combined
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < KW; i += 8) {
#pragma unroll
            for (int u = 0; u < 4; ++u) m4[u] = fmax3(m4[u], sv[i + 2 * u], sv[i + 2 * u + 1]);
          }
          mx = fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
        } else {
#pragma unroll
          for (int i = 0; i < KW; ++i)
            if (i < nvalid) mx = fmaxf(mx, sv[i]);
        }
      }
      const float m_new = active ? fmaxf(m_used, mx * c2) : m_used;
      const bool need = active && m_used != -INFINITY && m_new > m_used + 8.0f;
      if (__any_sync(0xffffffffu, need)) {
        // rescale O: the previous P V product must have landed first
        if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
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
      uint32_t pk[KW / 2];
      if (active && full) {
        const float2 cc = make_float2(c2, c2);
        const float2 mm = make_float2(-m_used, -m_used);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < KW; i += 2) {
          const float2 x = __ffma2_rn(make_float2(sv[i], sv[i + 1]), cc, mm);
          const float2 pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          acc[(i >> 1) & 3] = __fadd2_rn(acc[(i >> 1) & 3], pe);
          pk[i / 2] = pack_bf16x2(pe.x, pe.y);
        }
        const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
        const float2 a = __fadd2_rn(a01, a23);
        l += a.x + a.y;
      } else {
        float rs = 0.f;
#pragma unroll
        for (int i = 0; i < KW; i += 2) {
          const float p0 = (active && i < nvalid) ? ex2_approx(fmaf(sv[i], c2, -m_used)) : 0.f;
          const float p1 = (active && i + 1 < nvalid) ? ex2_approx(fmaf(sv[i + 1], c2, -m_used)) : 0.f;
          rs += p0 + p1;
          pk[i / 2] = pack_bf16x2(p0, p1);
        }
        l += rs;
      }
      // P buffer j&1 was last read by the P V product of step j-2
      if (j >= 2) {
        if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[j & 1], ((j - 2) >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      const uint32_t p_col = (j & 1) ? C::kColP1 : C::kColP0;
      if constexpr (KW == 32) {
        tmem_st16(taddr + lane_base + p_col, pk);
      } else {
        tmem_st32(taddr + lane_base + p_col, *reinterpret_cast<const uint32_t(*)[32]>(pk));
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
    }
    const int n_steps = j;
    if (ok) {
      bool have_o = n_steps > 0;
      if (have_o) {
        if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[(n_steps - 1) & 1], ((n_steps - 1) >> 1) & 1,
                                               abort_flag)))
          have_o = false;
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
