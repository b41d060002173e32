// Stage 3: block-sparse attention forward on the 5th-generation tensor cores
// (DynamicRad, Sec. 3.3, Eqs. 12-13 with epsilon -> 0).
//
// One CTA (one per SM) computes 256 query rows of one (batch, head) as two
// 128-row tiles that share one stream of K / V tiles: R = 256 / B_s query
// blocks.  The producer walks the ascending union of the R rows' kept-block
// lists and packs consecutive union blocks into 128-key steps (two 64-key
// blocks, four 32-key blocks, or one 128-key block), so every Q K^T is a
// 128 x 128 x D product -- the shape at which tcgen05 runs at its full rate
// (N = 64 runs at two thirds of it).  A tile none of whose query blocks keeps
// any block of the step skips its tensor-core work for that step; inside an
// active tile the (row, block) pairs outside a row's own list are masked.
//
// Warp roles (320 threads):
//   warps 0-3, 4-7  softmax of tile 0 / tile 1: thread t of the warpgroup owns
//              query row t of its tile = TMEM lane t.  Reads S = Q K^T (128
//              columns) twice -- once for the row max, once for the exponentials,
//              64 columns at a time to bound registers -- keeps the running
//              max / sum in fp32 (lazy rescale: O is
//              rescaled only when the row max grows by more than 2^8), writes
//              P = 2^(...) as bf16 pairs over the first 64 columns of its S
//              buffer, and finally normalises O and writes O and the
//              log-sum-exp.  One exponential pair in four is computed on the FMA
//              pipe (common.cuh exp2_poly2) to unload the MUFU unit.
//   warp 8     producer: merges the R sorted CSR rows, publishes each step's
//              block list, and issues TMA loads of the two Q tiles and of the
//              K and V tiles of every step (128-byte swizzled, non-multicast)
//              into a ring of single-tile slots.
//   warp 9     MMA issuer (one thread), per tile t and step j:
//              O_t += P_t(j) V(j) (A = P from tensor memory, B = V from shared
//              memory, MN-major), then S_t = Q_t K(j+1)^T (A, B from shared
//              memory).  Both go to the tensor core in this issue order, so the
//              Q K^T that overwrites S_t runs after the P V product that reads
//              P_t from the same columns; its completion also tells the softmax
//              that O_t is up to date before a rescale.
//
// Tensor memory (512 columns): O_t at 128 t (D columns), S_t at 256 + 128 t
// (128 columns; P_t over its first 64).
//
// Every wait is bounded (common.cuh): a wait that runs out records
// DYNRAD_ERR_DEVICE, raises a CTA-wide abort flag, and all roles unwind to the
// common exit where tensor memory is released.
#pragma once

#include "common.cuh"

#ifndef DYNRAD_ATTN_POLY_PER8
#define DYNRAD_ATTN_POLY_PER8 2
#endif

namespace dynrad {

// Developer instrumentation, compiled only with -DDYNRAD_ATTN_TRACE: lane 0 of
// every warp of one CTA (the middle query tile of head 0) stamps clock64() at
// fixed points of its first 64 steps into g_attn_trace[warp][step][tile][point],
// read back with dynrad_trace_read().  Off in every normal build.
#ifdef DYNRAD_ATTN_TRACE
__device__ unsigned long long g_attn_trace[10][64][2][8];
#define ATTN_TRACE(j, t, pt)                                                        \
  do {                                                                              \
    if (trace_cta && lane == 0 && (j) < 64) g_attn_trace[warp][(j)][(t)][(pt)] = clock64(); \
  } while (0)
#else
#define ATTN_TRACE(j, t, pt) \
  do {                       \
  } while (0)
#endif

template <int D, int BS>
struct AttnCfg {
  static constexpr int kTiles = 2;                   // 128-row query tiles per CTA
  static constexpr int kM = 128;                     // rows per tile
  static constexpr int kR = kTiles * kM / BS;        // query blocks per CTA
  static constexpr int kRT = kM / BS;                // query blocks per tile
  static constexpr int kKeys = 128;                  // keys per step
  static constexpr int kBPS = kKeys / BS;            // kept blocks per step
  static constexpr int kChunks = D / 64;             // 128-byte column chunks
  static constexpr int kQTileBytes = kM * D * 2;
  static constexpr int kTileBytes = kKeys * D * 2;   // one K or one V tile of a step
  static constexpr int kMetaSlots = 8;
  static constexpr int kSmemCtrl = 1024;
  static constexpr int kSmemBudget = 227 * 1024 - kSmemCtrl - 1024;  // 1024: manual alignment
  static constexpr int kSlotsRaw = (kSmemBudget - kTiles * kQTileBytes) / kTileBytes;
  static constexpr int kSlots = kSlotsRaw < 3 ? 3 : (kSlotsRaw > 8 ? 8 : kSlotsRaw);
  static constexpr int kSmemData = kTiles * kQTileBytes + kSlots * kTileBytes;
  static constexpr int kSmemTotal = kSmemData + kSmemCtrl + 1024;
  static constexpr int kThreads = 320;
  static constexpr uint32_t kTmemCols = 512;
  // pairs of exponentials (of every 8) computed on the FMA pipe
  static constexpr int kPolyPer8 = DYNRAD_ATTN_POLY_PER8;
  static_assert(kPolyPer8 >= 0 && kPolyPer8 <= 8, "FMA-pipe share");
  __host__ __device__ static constexpr uint32_t col_o(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t col_s(int t) { return 256u + 128u * t; }
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BS == 32 || BS == 64 || BS == 128, "block size");
  static_assert(kR <= 32, "one producer lane per query block");
  static_assert(kSmemTotal <= 227 * 1024, "shared memory");
};

struct AttnParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  __nv_bfloat16* o;
  float* lse;
  int N;
  int nb;
  float scale_log2;   // logit scale * log2(e)
  uint64_t wait_ns;   // limit of the pipeline waits (kWaitLimitNs unless shortened for a test)
  int32_t stall_step; // test hook: at this step the MMA warp waits for a barrier nothing
                      // completes, so that wait runs out and the CTA unwinds; -1 = never
};

// One 128-key step: up to 4 kept blocks; nblk = 0 ends the walk.
struct StepMeta {
  int32_t key0[4];    // first key token of each block
  uint32_t mask[4];   // bit r: query block I0 + r keeps that block
  int32_t nblk;
  int32_t pad;
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int D, int BS>
__global__ void __launch_bounds__(AttnCfg<D, BS>::kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg<D, BS>;
  constexpr int NS = C::kSlots;
  constexpr int MS = C::kMetaSlots;
  constexpr int BPS = C::kBPS;
  constexpr uint32_t kTileMask = (1u << C::kRT) - 1u;
  extern __shared__ uint8_t attn_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = smem;                                 // tile t at t * kQTileBytes
  uint8_t* slot_smem = smem + C::kTiles * C::kQTileBytes;  // load i (K_j: 2j, V_j: 2j+1) in slot i % NS
  uint8_t* ctrl = smem + C::kSmemData;
  uint64_t* bar = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* q_full = bar;
  uint64_t* slot_full = bar + 1;
  uint64_t* slot_empty = slot_full + NS;
  uint64_t* meta_full = slot_empty + NS;   // [MS]
  uint64_t* s_full = meta_full + MS;       // [tile]
  uint64_t* p_full = s_full + 2;           // [tile]
  uint64_t* drain = p_full + 2;
  uint64_t* stall = drain + 1;             // never completed (failure-path tests)
  StepMeta* meta = reinterpret_cast<StepMeta*>(stall + 1);
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(meta + MS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_s + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int I0 = blockIdx.x * C::kR;
  const int q_row0 = I0 * BS;
  const int nb = p.nb;
  const uint64_t wlim = p.wait_ns;
#ifdef DYNRAD_ATTN_TRACE
  const bool trace_cta = blockIdx.x == gridDim.x / 2 && blockIdx.y == 0;
#endif

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int m = 0; m < MS; ++m) mbar_init(&meta_full[m], 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);   // one arrival per warp of the tile's warpgroup
    }
    mbar_init(drain, 1);
    mbar_init(stall, 1);
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
      mbar_arrive_expect_tx(q_full, C::kTiles * C::kQTileBytes);
#pragma unroll
      for (int t = 0; t < C::kTiles; ++t)
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(q_smem + t * C::kQTileBytes + c * (C::kM * 128), &tm_q, q_full, c * 64,
                      q_row0 + t * C::kM, bh);
    }
    bool ok = true;
    int li = 0;  // loads issued (K_j = 2j, V_j = 2j + 1, end marker = 2n)
    // waits (bounded) until slot li % NS is free again
    auto slot_ready = [&](int i) -> bool {
      bool w = true;
      if (i >= NS && lane == 0) w = mbar_wait(&slot_empty[i % NS], ((i / NS) - 1) & 1, abort_flag, wlim);
      return __shfl_sync(0xffffffffu, w, 0);
    };
    for (int j = 0;; ++j) {
      // gather the step's blocks: the next BPS union members
      StepMeta st;
      st.nblk = 0;
      st.pad = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        st.key0[b] = 0;
        st.mask[b] = 0u;
      }
#pragma unroll
      for (int b = 0; b < BPS; ++b) {
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
        // once the union is exhausted every later slot is empty too, so slot b
        // holds the b-th block of the step
        st.key0[b] = m != INT32_MAX ? m * BS : 0;
        st.mask[b] = m != INT32_MAX ? mask : 0u;
        st.nblk += m != INT32_MAX ? 1 : 0;
      }
      // publish the step (the walk ends with nblk = 0)
      ATTN_TRACE(j, 0, 0);
      if (!slot_ready(li)) { ok = false; break; }
      ATTN_TRACE(j, 0, 1);
      if (lane == 0) {
        meta[j % MS] = st;
        mbar_arrive(&meta_full[j % MS]);
      }
      if (st.nblk == 0) {
        if (lane == 0) mbar_arrive(&slot_full[li % NS]);  // end marker in the K position
        __syncwarp();
        break;
      }
      // K tile then V tile; blocks missing at the end of the walk repeat the
      // first block so the tile holds finite data (its columns are masked)
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        if (kv == 1 && !slot_ready(li)) { ok = false; break; }
        if (lane == 0) {
          uint8_t* dst = slot_smem + (li % NS) * C::kTileBytes;
          const CUtensorMap* map = kv == 0 ? &tm_k : &tm_v;
          mbar_arrive_expect_tx(&slot_full[li % NS], C::kTileBytes);
#pragma unroll
          for (int b = 0; b < BPS; ++b) {
            const int key0 = b < st.nblk ? st.key0[b] : st.key0[0];
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d(dst + c * (C::kKeys * 128) + b * (BS * 128), map, &slot_full[li % NS], c * 64,
                          key0, bh);
          }
        }
        __syncwarp();
        ++li;
      }
      if (!ok) break;
    }
    if (!ok && lane == 0) {
      // unwinding: let the copies already issued land before shared memory is
      // given back (bounded; ignores the abort flag)
      for (int i = (li > NS ? li - NS : 0); i < li; ++i) mbar_wait(&slot_full[i % NS], (i / NS) & 1, nullptr);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, C::kKeys, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_base = smem_u32(q_smem);
      const uint32_t slot_base = smem_u32(slot_smem);
      bool ok = mbar_wait(q_full, 0, abort_flag, wlim);
      bool started[2] = {false, false};   // O_t holds a P V product
      auto tile_act = [&](const StepMeta& m, int t) -> bool {
        uint32_t any = 0;
#pragma unroll
        for (int b = 0; b < BPS; ++b) any |= (b < m.nblk) ? m.mask[b] : 0u;
        return ((any >> (t * C::kRT)) & kTileMask) != 0u;
      };
      // Shared-memory descriptors: each MMA of a batch adds a constant to the
      // batch's first descriptor (the 14-bit start-address field cannot carry:
      // shared addresses stay below 2^18 bytes), so a batch of 8 issues costs
      // a few integer adds beside the MMAs.
      auto desc_add = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (bytes >> 4); };
      const uint64_t qdesc0 = smem_desc_sw128(q_base, 16, 1024);
      const uint64_t kdesc0 = smem_desc_sw128(slot_base, 16, 1024);
      const uint64_t vdesc0 = smem_desc_sw128(slot_base, C::kKeys * 128, 1024);
      auto issue_qk = [&](int t, int i) {   // S_t = Q_t K^T, K in load slot i
        const uint64_t ad = desc_add(qdesc0, t * C::kQTileBytes);
        const uint64_t bd = desc_add(kdesc0, (i % NS) * C::kTileBytes);
        const uint32_t d = taddr + C::col_s(t);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          mma_ss(d, desc_add(ad, c * (C::kM * 128) + off), desc_add(bd, c * (C::kKeys * 128) + off), idesc_qk,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int i) {   // O_t += P_t V, V in load slot i
        // V tile [128 keys][D] as the MN-major B operand: 64-column chunks
        // 128*128 bytes apart (leading offset), 8-key groups 1024 bytes apart
        const uint64_t bd = desc_add(vdesc0, (i % NS) * C::kTileBytes);
        const uint32_t d = taddr + C::col_o(t), a = taddr + C::col_s(t);
        const uint32_t acc0 = started[t] ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < C::kKeys / 16; ++kk)
          mma_ts(d, a + kk * 8, desc_add(bd, kk * 2048), idesc_pv, kk > 0 ? 1u : acc0);
        started[t] = true;
      };
      // step 0: S_t = Q_t K(0)^T
      int j = 0;
      StepMeta cur_m;
      if (ok && !mbar_wait(&slot_full[0], 0, abort_flag, wlim)) ok = false;
      if (ok) {
        cur_m = meta[0];
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          if (cur_m.nblk > 0 && tile_act(cur_m, t)) issue_qk(t, 0);
          mma_commit(&s_full[t]);
        }
        if (cur_m.nblk > 0) mma_commit(&slot_empty[0]);
      }
      while (ok && cur_m.nblk > 0) {
        if (j == p.stall_step && !mbar_wait(stall, 0, abort_flag, wlim)) { ok = false; break; }
        const int iv = 2 * j + 1, ik = 2 * j + 2;   // V(j) and K(j+1) load indices
        // Every wait of the step except the softmax hand-offs comes first, so
        // that each tile's P V and Q K^T batches go out back to back: V(j),
        // K(j+1) (or the end marker in its place; loaded steps ahead) and the
        // next step's block list.
        ATTN_TRACE(j, 0, 2);
        if (!mbar_wait(&slot_full[iv % NS], (iv / NS) & 1, abort_flag, wlim)) { ok = false; break; }
        if (!mbar_wait(&slot_full[ik % NS], (ik / NS) & 1, abort_flag, wlim)) { ok = false; break; }
        ATTN_TRACE(j, 0, 3);
        const StepMeta next_m = meta[(j + 1) % MS];
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          // O_t += P_t(j) V(j) once the softmax has written P_t(j), then
          // S_t = Q_t K(j+1)^T (after the P V in issue order)
          if (!mbar_wait(&p_full[t], j & 1, abort_flag, wlim)) { ok = false; break; }
          tc_fence_after();
          ATTN_TRACE(j, t, 0);
          if (tile_act(cur_m, t)) issue_pv(t, iv);
          if (next_m.nblk > 0 && tile_act(next_m, t)) issue_qk(t, ik);
          if (t == 1) {
            mma_commit(&slot_empty[iv % NS]);
            if (next_m.nblk > 0) mma_commit(&slot_empty[ik % NS]);
          }
          mma_commit(&s_full[t]);
          ATTN_TRACE(j, t, 1);
        }
        if (!ok) break;
        cur_m = next_m;
        ++j;
      }
      // all issued tensor-core work finished before tensor memory is released
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- softmax
    const int tile = warp >> 2;                    // warpgroup = query tile
    const int t = threadIdx.x - tile * 128;        // row within the tile = TMEM lane
    const int mbit = tile * C::kRT + t / BS;       // this row's bit in the block masks
    const int row = q_row0 + tile * C::kM + t;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t col_s = C::col_s(tile), col_o = C::col_o(tile);
    const float c2 = p.scale_log2;
    float m_used = -INFINITY;              // running max in log2 units
    float l = 0.f;
    bool any_pv = false;                   // a P V product reached O of this tile
    int j = 0;
    bool ok = true;
    for (;; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&meta_full[j % MS], (j / MS) & 1, abort_flag, wlim))) {
        ok = false;
        break;
      }
      const StepMeta st = meta[j % MS];
      // S_t(j) -- or, at the end marker, completion of the last P V product
      ATTN_TRACE(j, tile, 0);
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[tile], j & 1, abort_flag, wlim))) { ok = false; break; }
      tc_fence_after();
      ATTN_TRACE(j, tile, 1);
      if (st.nblk == 0) break;
      uint32_t tile_any = 0, row_bits = 0;
#pragma unroll
      for (int b = 0; b < BPS; ++b) {
        const uint32_t mk = b < st.nblk ? st.mask[b] : 0u;
        tile_any |= mk;
        row_bits |= ((mk >> mbit) & 1u) << b;
      }
      const bool tile_active = ((tile_any >> (tile * C::kRT)) & kTileMask) != 0u;
      if (tile_active) {
        any_pv = true;
        // State of each 64-key half for this row: every key valid (kept block,
        // inside the sequence), none valid (block not kept / no block), or
        // mixed (a sequence tail, or 32-key blocks with different states).
        // Rows of one warp share their query block, so these are warp-uniform.
        uint32_t half_full = 0, half_none = 0;
#pragma unroll
        for (int h = 0; h < C::kKeys / 64; ++h) {
          bool all = true, none = true;
#pragma unroll
          for (int b = 0; b < BPS; ++b) {
            if (b * BS >= (h + 1) * 64 || (b + 1) * BS <= h * 64) continue;  // slot outside the half
            const bool kept = (row_bits >> b) & 1u;
            const int lo = max(h * 64, b * BS) - b * BS, hi = min((h + 1) * 64, (b + 1) * BS) - b * BS;
            const bool inside = st.key0[b] + hi <= p.N;
            const bool any_in = st.key0[b] + lo < p.N;
            all = all && kept && inside;
            none = none && !(kept && any_in);
          }
          half_full |= (all ? 1u : 0u) << h;
          half_none |= (none ? 1u : 0u) << h;
        }
        // pass 1: row max over the valid keys, 64 columns at a time
        float mx = -INFINITY;
#pragma unroll
        for (int h = 0; h < C::kKeys / 64; ++h) {
          if ((half_none >> h) & 1u) continue;
          float sv[64];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t r[32];
            tmem_ld32(taddr + lane_base + col_s + h * 64 + c * 32, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(r[i]);
          }
          tmem_wait_ld();
          if ((half_full >> h) & 1u) {
            float m4[4] = {mx, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < 64; i += 8) {
#pragma unroll
              for (int u = 0; u < 4; ++u) m4[u] = fmax3(m4[u], sv[i + 2 * u], sv[i + 2 * u + 1]);
            }
            mx = fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const int k = h * 64 + i, b = k / BS;
              const bool v = ((row_bits >> b) & 1u) && (st.key0[b] + (k % BS) < p.N);
              if (v) mx = fmaxf(mx, sv[i]);
            }
          }
        }
        ATTN_TRACE(j, tile, 2);
        const bool active = (half_none != (1u << (C::kKeys / 64)) - 1u);
        const float m_new = active ? fmaxf(m_used, mx * c2) : m_used;
        const bool need = active && m_used != -INFINITY && m_new > m_used + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          // rescale O: S_t(j) completing means every earlier P V product has too
          const float alpha = need ? ex2_approx(m_used - m_new) : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(taddr + lane_base + col_o + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(taddr + lane_base + col_o + c * 32, r);
          }
          if (need) {
            l *= alpha;
            m_used = m_new;
          }
        }
        if (active && m_used == -INFINITY) m_used = m_new;
        ATTN_TRACE(j, tile, 3);
        // pass 2: P over the first 64 columns of S_t; keys 64h .. 64h+63 are
        // re-read from columns 64h .. and written as bf16 pairs to columns
        // 32h .., which hold keys already consumed
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        const float2 cc = make_float2(c2, c2);
        const float2 mm = make_float2(-m_used, -m_used);
#pragma unroll
        for (int h = 0; h < C::kKeys / 64; ++h) {
          uint32_t pk[32];
          if ((half_none >> h) & 1u) {
#pragma unroll
            for (int q2 = 0; q2 < 32; ++q2) pk[q2] = 0u;
          } else {
            float sv[64];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              uint32_t r[32];
              tmem_ld32(taddr + lane_base + col_s + h * 64 + c * 32, r);
#pragma unroll
              for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(r[i]);
            }
            tmem_wait_ld();
            if ((half_full >> h) & 1u) {
#pragma unroll
              for (int q2 = 0; q2 < 32; ++q2) {
                const float2 x = __ffma2_rn(make_float2(sv[2 * q2], sv[2 * q2 + 1]), cc, mm);
                // kPolyPer8 pairs in eight on the FMA pipe, the rest on MUFU
                const float2 pe = (q2 & 7) < C::kPolyPer8 ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
                acc[q2 & 3] = __fadd2_rn(acc[q2 & 3], pe);
                pk[q2] = pack_bf16x2(pe.x, pe.y);
              }
            } else {
#pragma unroll
              for (int q2 = 0; q2 < 32; ++q2) {
                const int k = h * 64 + 2 * q2;
                const int b0 = k / BS, b1 = (k + 1) / BS;
                const bool v0 = ((row_bits >> b0) & 1u) && (st.key0[b0] + (k % BS) < p.N);
                const bool v1 = ((row_bits >> b1) & 1u) && (st.key0[b1] + ((k + 1) % BS) < p.N);
                const float p0 = v0 ? ex2_approx(fmaf(sv[2 * q2], c2, -m_used)) : 0.f;
                const float p1 = v1 ? ex2_approx(fmaf(sv[2 * q2 + 1], c2, -m_used)) : 0.f;
                acc[q2 & 3] = __fadd2_rn(acc[q2 & 3], make_float2(p0, p1));
                pk[q2] = pack_bf16x2(p0, p1);
              }
            }
          }
          tmem_st32(taddr + lane_base + col_s + h * 32, pk);
        }
        const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
        const float2 a = __fadd2_rn(a01, a23);
        l += a.x + a.y;
        ATTN_TRACE(j, tile, 4);
        tmem_wait_st();
      }
      // hand P_t over: every lane's stores are complete and fenced before the
      // warp's one arrival
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[tile]);
      ATTN_TRACE(j, tile, 5);
    }
    if (ok) {
      const bool have_o = any_pv;     // the final s_full wait covered the last P V
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        if (have_o) {
          tmem_ld32(taddr + lane_base + col_o + c * 32, r);
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
  if (warp == 9) tmem_dealloc(taddr, C::kTmemCols);
}

}  // namespace dynrad
