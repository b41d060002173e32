// C ABI of the DynamicRad hot path (declared in include/dynrad.h).
//
// Host side only: argument checks, launch configuration, TMA descriptor
// encoding.  Every arithmetic step of the path runs in the kernels included
// below.
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "attention.cuh"
#include "candidates.cuh"
#include "common.cuh"
#include "backward.cuh"
#include "optin.h"
#include "dyntok.cuh"
#include "sampling.cuh"
#include "select.cuh"

using namespace dynrad;

namespace {

constexpr int kMaxFrames = 16384;
constexpr int kMaxBlocks = 16384;        // Nb bound of the scoring kernel's shared memory
constexpr int kMaxRowCandidates = 1024;  // candidates per row (a lane's kept mask covers 32 list positions)

inline cudaStream_t as_stream(dynrad_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DYNRAD_OK : DYNRAD_ERR_CUDA;
}

// Shared geometry validation; fills the device struct.
int check_geom(const dynrad_geom* g, GeomDev* out) {
  if (g == nullptr) return DYNRAD_ERR_INVALID_ARG;
  if (g->frames < 1 || g->height < 1 || g->width < 1 || g->block < 1) return DYNRAD_ERR_INVALID_ARG;
  if (!(g->gamma > 0.0) || !(g->lambda > 0.0) || !(g->eps >= 0.0)) return DYNRAD_ERR_INVALID_ARG;
  if (!std::isfinite(g->gamma) || !std::isfinite(g->lambda) || !std::isfinite(g->eps))
    return DYNRAD_ERR_INVALID_ARG;
  if (!(g->theta_c >= 0.0 && g->theta_c <= 1.0) || !(g->theta_m >= 0.0 && g->theta_m <= 1.0))
    return DYNRAD_ERR_INVALID_ARG;
  if (g->force_t < 0 || g->force_t > 1) return DYNRAD_ERR_INVALID_ARG;
  const int64_t nt = static_cast<int64_t>(g->height) * g->width;
  const int64_t n = nt * g->frames;
  if (nt > INT32_MAX / 4 || n > INT32_MAX / 2) return DYNRAD_ERR_UNSUPPORTED;
  if (g->frames > kMaxFrames) return DYNRAD_ERR_UNSUPPORTED;
  const int64_t nb = (n + g->block - 1) / g->block;
  if (out != nullptr) {
    out->frames = g->frames;
    out->nt = static_cast<int32_t>(nt);
    out->block = g->block;
    out->nb = static_cast<int32_t>(nb);
    out->n = static_cast<int32_t>(n);
    out->force_t = g->force_t;
    int64_t l0 = 1;
    while (l0 < nt) l0 <<= 1;  // Eq. 1: smallest power of two >= N_t
    out->l0 = l0;
    out->gamma = g->gamma;
    out->lambda = g->lambda;
    out->theta_c = g->theta_c;
    out->theta_m = g->theta_m;
    out->eps = g->eps;
  }
  return DYNRAD_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Grants `bytes` of dynamic shared memory to `kernel` on the current device
// (once per device and kernel; see optin.h).
int smem_optin(OptInTable& table, const void* kernel, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DYNRAD_ERR_CUDA;
  const bool ok = table.ensure(dev, bytes, [kernel](int b) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess;
  });
  return ok ? DYNRAD_OK : DYNRAD_ERR_CUDA;
}

// Failure-path test hook of the attention kernel (dynrad_debug_attn_stall):
// the limit of its pipeline waits (0 = the built-in limit) and the step at
// which its MMA warp waits for a barrier nothing completes (-1 = never).
std::atomic<uint64_t> g_attn_wait_ns{0};
std::atomic<int32_t> g_attn_stall_step{-1};

struct SelectWorkspace {
  size_t qbar, kbar, plan_off, plan_cnt, plan_rows, plan_J, plan_pos, kept, partial, counters, zero_end, total;
};

// Counters of one stage-2 launch: ticket (8 bytes), plan_alloc, plan_done, then
// pool_done[bh]; the range [counters, zero_end) is zeroed before each launch.
// kept / partial serve dynamic mode's scan and compaction.
SelectWorkspace select_layout(int64_t bh, int64_t nb, int64_t d, int64_t cand_nnz) {
  SelectWorkspace w;
  const int64_t rows = bh * nb;
  const int64_t groups = (nb + kSelRows - 1) / kSelRows;
  const int64_t tiles = (rows + 1 + kScanTile - 1) / kScanTile;
  w.qbar = 0;
  w.kbar = align256(w.qbar + static_cast<size_t>(rows * d) * 4);
  // scoring plan: per group of 8 rows, the union list and the scatter positions
  // (independent of the head; the unions' total is at most cand_nnz)
  w.plan_off = align256(w.kbar + static_cast<size_t>(rows * d) * 4);
  w.plan_cnt = align256(w.plan_off + static_cast<size_t>(groups) * 4);
  w.plan_rows = align256(w.plan_cnt + static_cast<size_t>(groups) * 4);
  w.plan_J = align256(w.plan_rows + static_cast<size_t>(groups) * 4);
  w.plan_pos = align256(w.plan_J + static_cast<size_t>(cand_nnz) * 4);
  w.kept = align256(w.plan_pos + static_cast<size_t>(cand_nnz) * kSelRows * 4);
  w.partial = align256(w.kept + static_cast<size_t>(bh * cand_nnz) * 4);
  w.counters = align256(w.partial + static_cast<size_t>(tiles) * 8);
  w.zero_end = w.counters + 16 + static_cast<size_t>(bh) * 4;
  w.total = align256(w.zero_end);
  return w;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 3-D map over a [BH, N, D] bf16 tensor: box = 64 columns (128 B) x rows x 1,
// 128-byte swizzle; rows past N of a head read as zeros.
bool encode_map(CUtensorMap* map, const void* base, int D, int N, int BH, int box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D map over the backward's per-row (-lse2, -D_r) array, [BH] x [2 Np] floats:
// box = 128 floats (64 rows, 512 B) x 1.
bool encode_aux_map(CUtensorMap* map, const void* base, int Np, int BH) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(Np) * 2, static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(Np) * 8};
  cuuint32_t box[2] = {128, 1};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BS>
int launch_attn(const void* q, const void* k, const void* v, int BH, int N, const int32_t* row_ptr,
                const int32_t* col_idx, float scale, void* o, float* lse, cudaStream_t st) {
  using C = AttnCfg<D, BS>;
  CUtensorMap mq, mk, mv;
  // K / V boxes are one kept block (BS rows); a slot stacks C::kBPS of them,
  // the unit the kernel's slots and transaction counts are sized for
  static_assert(C::kBPS * BS == C::kKeys, "a step is kBPS blocks");
  if (!encode_map(&mq, q, D, N, BH, C::kM) || !encode_map(&mk, k, D, N, BH, BS) ||
      !encode_map(&mv, v, D, N, BH, BS))
    return DYNRAD_ERR_CUDA;
  static OptInTable optin;   // per instantiation, per device
  const int rc = smem_optin(optin, reinterpret_cast<const void*>(sparse_attn_kernel<D, BS>), C::kSmemTotal);
  if (rc != DYNRAD_OK) return rc;
  AttnParams p;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.N = N;
  p.nb = (N + BS - 1) / BS;
  p.scale_log2 = scale * 1.4426950408889634f;
  const uint64_t wl = g_attn_wait_ns.load(std::memory_order_relaxed);
  p.wait_ns = wl != 0 ? wl : kWaitLimitNs;
  p.stall_step = g_attn_stall_step.load(std::memory_order_relaxed);
  const int tiles = (p.nb + C::kR - 1) / C::kR;
  dim3 grid(tiles, BH);
  sparse_attn_kernel<D, BS><<<grid, C::kThreads, C::kSmemTotal, st>>>(mq, mk, mv, p);
  return launch_status();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int64_t dynrad_num_blocks(const dynrad_geom* geom) {
  GeomDev g;
  if (check_geom(geom, &g) != DYNRAD_OK) return 0;
  return g.nb;
}

const char* dynrad_status_string(int32_t status) {
  switch (status) {
    case DYNRAD_OK: return "ok";
    case DYNRAD_ERR_INVALID_ARG: return "invalid argument";
    case DYNRAD_ERR_UNSUPPORTED: return "unsupported size or parameter";
    case DYNRAD_ERR_CAPACITY: return "output or workspace capacity exceeded";
    case DYNRAD_ERR_CUDA: return "CUDA runtime error";
    case DYNRAD_ERR_DEVICE: return "device-side check or bounded wait failed";
    default: return "unknown status";
  }
}

}  // extern "C"

namespace {
__global__ void exp2_diag_kernel(const float* x, float* poly, float* ref, int64_t n) {
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    poly[i] = r.x;
    poly[i + 1] = r.y;
    ref[i] = exp2f(x[i]);
    ref[i + 1] = exp2f(x[i + 1]);
  } else if (i < n) {
    poly[i] = exp2_poly2(make_float2(x[i], x[i])).x;
    ref[i] = exp2f(x[i]);
  }
}
}  // namespace

extern "C" {

}  // extern "C"

namespace {

// Per query row r, from the log-sum-exps of the dense and the masked attention
// at logit scale c (lse) and 2c (lse2):
//   sum_j a_j^2 over all keys = exp(lse2_dense - 2 lse_dense),
//   the same over kept keys   = exp(lse2_kept - 2 lse_dense),
//   kept mass m               = exp(lse_kept - lse_dense),
// and the row's squared error between the dense softmax row and the masked,
// renormalized one: (1 - 1/m)^2 sum_kept a_j^2 + sum_masked a_j^2.
__global__ void proxy_error_kernel(const float* lse_d, const float* lse_k, const float* lse2_d, const float* lse2_k,
                                   int64_t n, double* out) {
  __shared__ double red[2][8];
  double err = 0.0, tot = 0.0;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; r < n;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const double ld = lse_d[r], l2d = lse2_d[r];
    const double all2 = exp(l2d - 2.0 * ld);
    double kept2 = 0.0, inv_m = 0.0;
    if (isfinite(static_cast<double>(lse_k[r]))) {
      kept2 = exp(static_cast<double>(lse2_k[r]) - 2.0 * ld);
      inv_m = exp(ld - static_cast<double>(lse_k[r]));
    }
    const double f = 1.0 - inv_m;
    err += (kept2 > 0.0 ? f * f * kept2 : 0.0) + fmax(all2 - kept2, 0.0);
    tot += all2;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    err += __shfl_xor_sync(0xffffffffu, err, off);
    tot += __shfl_xor_sync(0xffffffffu, tot, off);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[0][warp] = err;
    red[1][warp] = tot;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double e = 0.0, t = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
      e += red[0][w];
      t += red[1][w];
    }
    atomicAdd(out, e);
    atomicAdd(out + 1, t);
  }
}

}  // namespace

extern "C" {

int dynrad_proxy_error(const float* lse_dense, const float* lse_kept, const float* lse2_dense,
                       const float* lse2_kept, int64_t n, double* out, dynrad_stream_t stream) {
  if (lse_dense == nullptr || lse_kept == nullptr || lse2_dense == nullptr || lse2_kept == nullptr ||
      out == nullptr || n < 1)
    return DYNRAD_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (cudaMemsetAsync(out, 0, 2 * sizeof(double), st) != cudaSuccess) return DYNRAD_ERR_CUDA;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 1184);
  proxy_error_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(lse_dense, lse_kept, lse2_dense, lse2_kept, n,
                                                                   out);
  return launch_status();
}

int dynrad_debug_exp2(const float* x, float* poly_out, float* ref_out, int64_t n, dynrad_stream_t stream) {
  if (x == nullptr || poly_out == nullptr || ref_out == nullptr || n < 0) return DYNRAD_ERR_INVALID_ARG;
  if (n == 0) return DYNRAD_OK;
  const int64_t threads = 256, pairs = (n + 1) / 2;
  exp2_diag_kernel<<<static_cast<unsigned>((pairs + threads - 1) / threads), threads, 0, as_stream(stream)>>>(
      x, poly_out, ref_out, n);
  return launch_status();
}

#ifdef DYNRAD_ATTN_TRACE
// Trace builds only (see attention.cuh): copies the clock stamps to host memory.
int dynrad_trace_read(void* host, size_t bytes) {
  if (host == nullptr) return DYNRAD_ERR_INVALID_ARG;
  const size_t n = bytes < sizeof(g_attn_trace) ? bytes : sizeof(g_attn_trace);
  return cudaMemcpyFromSymbol(host, g_attn_trace, n) == cudaSuccess ? DYNRAD_OK : DYNRAD_ERR_CUDA;
}
#endif

int dynrad_debug_attn_stall(uint64_t wait_ns, int32_t stall_step) {
  if (stall_step < -1) return DYNRAD_ERR_INVALID_ARG;
  g_attn_wait_ns.store(wait_ns, std::memory_order_relaxed);
  g_attn_stall_step.store(stall_step, std::memory_order_relaxed);
  return DYNRAD_OK;
}

int dynrad_device_status(int32_t* status_out, int32_t clear, dynrad_stream_t stream) {
  if (status_out == nullptr) return DYNRAD_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  int32_t v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return DYNRAD_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DYNRAD_ERR_CUDA;
  *status_out = v;
  if (clear) {
    const int32_t zero = 0;
    if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return DYNRAD_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DYNRAD_ERR_CUDA;
  }
  return DYNRAD_OK;
}

int dynrad_build_candidates(const dynrad_geom* geom, int32_t* cand_row_ptr, int32_t* cand_col,
                            int64_t cand_cap, int32_t* forced_lo, int32_t* forced_hi,
                            int64_t* nnz_out, int64_t* max_row_out, dynrad_stream_t stream) {
  GeomDev g;
  int rc = check_geom(geom, &g);
  if (rc != DYNRAD_OK) return rc;
  if (cand_row_ptr == nullptr || forced_lo == nullptr || forced_hi == nullptr) return DYNRAD_ERR_INVALID_ARG;
  if (cand_col == nullptr && nnz_out == nullptr) return DYNRAD_ERR_INVALID_ARG;
  if (cand_col != nullptr && cand_cap < 0) return DYNRAD_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const size_t tab = static_cast<size_t>(g.frames) * 5 + 16;
  cand_count_kernel<<<g.nb, kCandThreads, tab, st>>>(g, cand_row_ptr, forced_lo, forced_hi);
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  scan_small_kernel<<<1, 1024, 0, st>>>(cand_row_ptr, g.nb);
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  if (cand_col != nullptr) {
    cand_fill_kernel<<<g.nb, kCandThreads, tab, st>>>(g, cand_row_ptr, cand_col, cand_cap);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
  }
  if (nnz_out != nullptr || max_row_out != nullptr) {
    std::vector<int32_t> h(static_cast<size_t>(g.nb) + 1);
    if (cudaMemcpyAsync(h.data(), cand_row_ptr, h.size() * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return DYNRAD_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DYNRAD_ERR_CUDA;
    int64_t mx = 0;
    for (int i = 0; i < g.nb; ++i) mx = std::max<int64_t>(mx, h[i + 1] - h[i]);
    if (nnz_out != nullptr) *nnz_out = h[g.nb];
    if (max_row_out != nullptr) *max_row_out = mx;
    if (cand_col != nullptr && h[g.nb] > cand_cap) return DYNRAD_ERR_CAPACITY;
  }
  return DYNRAD_OK;
}

size_t dynrad_select_workspace_bytes(int32_t B, int32_t H, int32_t N, int32_t D, const dynrad_geom* geom,
                                     int64_t cand_nnz) {
  GeomDev g;
  if (check_geom(geom, &g) != DYNRAD_OK || B < 1 || H < 1 || N != g.n || (D != 64 && D != 128) ||
      cand_nnz < 0)
    return 0;
  return select_layout(static_cast<int64_t>(B) * H, g.nb, D, cand_nnz).total;
}

int dynrad_select_blocks(const void* q, const void* k, int32_t B, int32_t H, int32_t N, int32_t D,
                         const dynrad_geom* geom, const int32_t* cand_row_ptr, const int32_t* cand_col,
                         int64_t cand_nnz, int64_t cand_max_row, const int32_t* forced_lo,
                         const int32_t* forced_hi,
                         int32_t mode, double rho_or_tau, int32_t* row_ptr, int32_t* col_idx,
                         int64_t col_cap, float* scores_out, void* workspace, size_t workspace_bytes,
                         dynrad_stream_t stream) {
  GeomDev g;
  int rc = check_geom(geom, &g);
  if (rc != DYNRAD_OK) return rc;
  if (q == nullptr || k == nullptr || cand_row_ptr == nullptr || cand_col == nullptr ||
      forced_lo == nullptr || forced_hi == nullptr || row_ptr == nullptr || col_idx == nullptr ||
      workspace == nullptr)
    return DYNRAD_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N != g.n || cand_nnz < 1 || col_cap < 0 || cand_max_row < 0)
    return DYNRAD_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DYNRAD_ERR_UNSUPPORTED;
  if (mode != DYNRAD_STATIC_RATIO && mode != DYNRAD_DYNAMIC_THRESHOLD) return DYNRAD_ERR_INVALID_ARG;
  if (!(rho_or_tau > 0.0 && rho_or_tau <= 1.0)) return DYNRAD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return DYNRAD_ERR_INVALID_ARG;
  if (g.nb > kMaxBlocks) return DYNRAD_ERR_UNSUPPORTED;
  const int64_t bh = static_cast<int64_t>(B) * H;
  if (bh > 65535) return DYNRAD_ERR_UNSUPPORTED;
  if (bh * cand_nnz > INT32_MAX) return DYNRAD_ERR_UNSUPPORTED;
  const SelectWorkspace w = select_layout(bh, g.nb, D, cand_nnz);
  if (workspace_bytes < w.total) return DYNRAD_ERR_CAPACITY;
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int nq = (g.nb + kSelRows - 1) / kSelRows;
  const bool dyn = mode == DYNRAD_DYNAMIC_THRESHOLD;
  Stage2Params sp;
  sp.q = static_cast<const __nv_bfloat16*>(q);
  sp.k = static_cast<const __nv_bfloat16*>(k);
  sp.qbar = reinterpret_cast<float*>(ws + w.qbar);
  sp.kbar = reinterpret_cast<float*>(ws + w.kbar);
  sp.cand_row_ptr = cand_row_ptr;
  sp.cand_col = cand_col;
  sp.forced_lo = forced_lo;
  sp.forced_hi = forced_hi;
  sp.row_ptr = row_ptr;
  sp.col_idx = col_idx;
  sp.col_cap = col_cap;
  sp.scores_out = scores_out;
  sp.plan_off = reinterpret_cast<int32_t*>(ws + w.plan_off);
  sp.plan_cnt = reinterpret_cast<int32_t*>(ws + w.plan_cnt);
  sp.plan_J = reinterpret_cast<int32_t*>(ws + w.plan_J);
  sp.plan_pos = reinterpret_cast<int32_t*>(ws + w.plan_pos);
  sp.plan_rows = reinterpret_cast<int32_t*>(ws + w.plan_rows);
  sp.ticket = reinterpret_cast<unsigned long long*>(ws + w.counters);
  sp.plan_alloc = reinterpret_cast<int32_t*>(ws + w.counters + 8);
  sp.plan_done = reinterpret_cast<int32_t*>(ws + w.counters + 12);
  sp.pool_done = reinterpret_cast<int32_t*>(ws + w.counters + 16);
  sp.kept_tmp = reinterpret_cast<int32_t*>(ws + w.kept);
  sp.rows_bh = static_cast<int>(bh);
  sp.cand_nnz = cand_nnz;
  sp.N = N;
  sp.block = g.block;
  sp.nb = g.nb;
  sp.nq = nq;
  sp.max_row = (cand_max_row > 0 && cand_max_row < g.nb) ? static_cast<int>(cand_max_row) : g.nb;
  if (sp.max_row > kMaxRowCandidates) return DYNRAD_ERR_UNSUPPORTED;
  sp.span_cap = (kSelRows * sp.max_row + 3) & ~3;
  sp.mode = mode;
  sp.value = rho_or_tau;
  sp.scale = 1.0f / std::sqrt(static_cast<float>(D));
  const int64_t tickets = s2_tickets(nq, static_cast<int>(bh));
  if (tickets > INT32_MAX) return DYNRAD_ERR_UNSUPPORTED;
  size_t smem = std::max(plan_smem_bytes(g.nb), select_smem_bytes(D, sp.span_cap, dyn));
  smem = std::max(smem, static_cast<size_t>(kSelRows) * D * 4);   // pool item's transpose tile
  if (smem > 227 * 1024) return DYNRAD_ERR_UNSUPPORTED;
  // list positions per lane the selection unrolls over
  const int e = sp.max_row <= 128 ? 4 : (sp.max_row <= 256 ? 8 : (sp.max_row <= 512 ? 16 : 32));
  const void* kern = nullptr;
  int kid = 0;
#define DYNRAD_S2_KERNEL(D_, DYN_, E_, ID_)                                      \
  if (D == D_ && dyn == DYN_ && e == E_) {                                       \
    kern = reinterpret_cast<const void*>(stage2_kernel<D_, DYN_, E_>);           \
    kid = ID_;                                                                    \
  }
  DYNRAD_S2_KERNEL(64, false, 4, 0) DYNRAD_S2_KERNEL(64, false, 8, 1)
  DYNRAD_S2_KERNEL(64, false, 16, 2) DYNRAD_S2_KERNEL(64, false, 32, 3)
  DYNRAD_S2_KERNEL(64, true, 4, 4) DYNRAD_S2_KERNEL(64, true, 8, 5)
  DYNRAD_S2_KERNEL(64, true, 16, 6) DYNRAD_S2_KERNEL(64, true, 32, 7)
  DYNRAD_S2_KERNEL(128, false, 4, 8) DYNRAD_S2_KERNEL(128, false, 8, 9)
  DYNRAD_S2_KERNEL(128, false, 16, 10) DYNRAD_S2_KERNEL(128, false, 32, 11)
  DYNRAD_S2_KERNEL(128, true, 4, 12) DYNRAD_S2_KERNEL(128, true, 8, 13)
  DYNRAD_S2_KERNEL(128, true, 16, 14) DYNRAD_S2_KERNEL(128, true, 32, 15)
#undef DYNRAD_S2_KERNEL
  if (kern == nullptr) return DYNRAD_ERR_UNSUPPORTED;
  static OptInTable optin[16];   // per instantiation, per device
  if ((rc = smem_optin(optin[kid], kern, static_cast<int>(smem))) != DYNRAD_OK) return rc;
  if (cudaMemsetAsync(ws + w.counters, 0, w.zero_end - w.counters, st) != cudaSuccess) return DYNRAD_ERR_CUDA;
  {
    void* args[] = {&sp};
    if (cudaLaunchKernel(kern, dim3(static_cast<unsigned>(tickets)), dim3(kS2Threads), args, smem, st) !=
        cudaSuccess)
      return DYNRAD_ERR_CUDA;
  }
  if (dyn) {   // counts -> offsets, then the kept lists to their CSR positions
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    const int64_t rows = bh * g.nb;
    int64_t* partial = reinterpret_cast<int64_t*>(ws + w.partial);
    const int64_t tiles = (rows + 1 + kScanTile - 1) / kScanTile;
    scan_partial_kernel<<<static_cast<unsigned>(tiles), kScanThreads, 0, st>>>(row_ptr, rows, partial);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    CompactParams cp;
    cp.row_ptr = row_ptr;
    cp.partial = partial;
    cp.rows = rows;
    cp.nb = g.nb;
    cp.cand_row_ptr = cand_row_ptr;
    cp.kept_tmp = sp.kept_tmp;
    cp.cand_nnz = cand_nnz;
    cp.col_idx = col_idx;
    cp.col_cap = col_cap;
    scan_apply_kernel<<<static_cast<unsigned>(tiles), kScanThreads, 0, st>>>(cp);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    const int64_t cblocks = (rows * 32 + kCompactThreads - 1) / kCompactThreads;
    compact_kernel<<<static_cast<unsigned>(cblocks), kCompactThreads, 0, st>>>(cp);
  }
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  return DYNRAD_OK;
}

namespace {

struct SampleWorkspace {
  size_t pairs, counters, thresholds, kept, keep, partial, pool, total;
};

// Pool slots for every sampled frame pair at its largest window (q = 1/2):
// sum over distances t >= 2 kept by the split rule of 2 (F - t) ordered pairs.
uint64_t sample_pool_keys(const GeomDev& g) {
  uint64_t total = 0;
  const int64_t nt = g.nt;
  for (int t = 2; t < g.frames; ++t) {
    if (!pair_retained(g, t)) continue;
    const int64_t w = window_width(g, t), wc = w < nt - 1 ? w : nt - 1;
    const double n = static_cast<double>(nt * (2 * wc + 1) - wc * (wc + 1));
    if (n <= 0.0) continue;
    const double e = kSampleWindowDevs * sqrt(n) + 2.0 * kSampleWindowPad;
    total += 2ull * static_cast<uint64_t>(g.frames - t) * (sample_pool_slots(n, e) + 2ull);
  }
  return total;
}

SampleWorkspace sample_layout(const GeomDev& g, int64_t cand_nnz, bool with_pool) {
  SampleWorkspace w;
  const int64_t fp = static_cast<int64_t>(g.frames) * g.frames;
  const int64_t tiles = (g.nb + 1 + kScanTile - 1) / kScanTile;
  w.pairs = 0;
  w.counters = align256(w.pairs + static_cast<size_t>(fp) * sizeof(SamplePair));
  w.thresholds = align256(w.counters + static_cast<size_t>(2 * fp + 2) * 8);
  w.kept = align256(w.thresholds + static_cast<size_t>(fp) * 8);
  w.keep = align256(w.kept + static_cast<size_t>(cand_nnz) * 4);
  w.partial = align256(w.keep + static_cast<size_t>(cand_nnz));
  w.pool = align256(w.partial + static_cast<size_t>(tiles) * 8);
  w.total = with_pool ? align256(w.pool + static_cast<size_t>(sample_pool_keys(g)) * 8) : w.pool;
  return w;
}

}  // namespace

size_t dynrad_sampled_mask_workspace_bytes(const dynrad_geom* geom, int64_t cand_nnz) {
  GeomDev g;
  if (check_geom(geom, &g) != DYNRAD_OK || cand_nnz < 1) return 0;
  return sample_layout(g, cand_nnz, true).total;
}

size_t dynrad_sampled_mask_workspace_min_bytes(const dynrad_geom* geom, int64_t cand_nnz) {
  GeomDev g;
  if (check_geom(geom, &g) != DYNRAD_OK || cand_nnz < 1) return 0;
  return sample_layout(g, cand_nnz, false).total;
}

int dynrad_build_sampled_mask(const dynrad_geom* geom, double rho1, double rho2, uint64_t seed,
                              const int32_t* cand_row_ptr, const int32_t* cand_col, int64_t cand_nnz,
                              const int32_t* forced_lo, const int32_t* forced_hi, int32_t replicas,
                              int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, uint64_t* thresholds_out,
                              void* workspace, size_t workspace_bytes, dynrad_stream_t stream) {
  GeomDev g;
  int rc = check_geom(geom, &g);
  if (rc != DYNRAD_OK) return rc;
  if (cand_row_ptr == nullptr || cand_col == nullptr || forced_lo == nullptr || forced_hi == nullptr ||
      row_ptr == nullptr || col_idx == nullptr || workspace == nullptr)
    return DYNRAD_ERR_INVALID_ARG;
  if (!(rho1 > 0.0 && rho1 <= 1.0) || !(rho2 > 0.0 && rho2 <= 1.0)) return DYNRAD_ERR_INVALID_ARG;
  if (cand_nnz < 1 || replicas < 1 || col_cap < 0) return DYNRAD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DYNRAD_ERR_INVALID_ARG;
  if (g.block != 32 && g.block != 64 && g.block != 128) return DYNRAD_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(replicas) * g.nb + 1 > INT32_MAX) return DYNRAD_ERR_UNSUPPORTED;
  if ((static_cast<int64_t>(g.nt) + kSampleRowsPerCta - 1) / kSampleRowsPerCta > 65535) return DYNRAD_ERR_UNSUPPORTED;
  // the marking keeps a frame table in default shared memory
  if (static_cast<size_t>(g.frames) * 5 + 16 > 48 * 1024) return DYNRAD_ERR_UNSUPPORTED;
  const SampleWorkspace w = sample_layout(g, cand_nnz, false);
  if (workspace_bytes < w.total) return DYNRAD_ERR_CAPACITY;
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int fp = g.frames * g.frames;
  SampleParams sp;
  sp.g = g;
  sp.rho1 = rho1;
  sp.rho2 = rho2;
  sp.seed = seed;
  sp.pairs = reinterpret_cast<SamplePair*>(ws + w.pairs);
  sp.below = reinterpret_cast<unsigned long long*>(ws + w.counters);
  sp.inwin = sp.below + fp;
  sp.pool_used = sp.inwin + fp;
  sp.mark_ticket = sp.pool_used + 1;
  sp.cand_nnz = cand_nnz;
  sp.keep = ws + w.keep;
  sp.pool = reinterpret_cast<uint64_t*>(ws + w.pool);
  sp.pool_cap = (workspace_bytes - w.pool) / 8;   // whatever the caller gave beyond the fixed part
  sp.thresholds = reinterpret_cast<uint64_t*>(ws + w.thresholds);
  sp.cand_row_ptr = cand_row_ptr;
  sp.cand_col = cand_col;
  sp.forced_lo = forced_lo;
  sp.forced_hi = forced_hi;
  sp.counts = row_ptr;
  sp.kept_tmp = reinterpret_cast<int32_t*>(ws + w.kept);
  if (cudaMemsetAsync(sp.below, 0, static_cast<size_t>(2 * fp + 2) * 8, st) != cudaSuccess) return DYNRAD_ERR_CUDA;
  sample_setup_kernel<<<(fp + 255) / 256, 256, 0, st>>>(sp);
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  const dim3 cgrid(fp, (g.nt + kSampleRowsPerCta - 1) / kSampleRowsPerCta);
  sample_collect_kernel<<<cgrid, kSampleThreads, 0, st>>>(sp);
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  sample_select_kernel<<<fp, kSampleThreads, 0, st>>>(sp);
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  // marking: warps claim candidates from a ticket; enough CTAs to fill the SMs
  const size_t msmem = static_cast<size_t>(g.frames) * 5 + 16;
  {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (cand_nnz + kMarkChunk * (kSampleThreads / 32) - 1) / (kMarkChunk * (kSampleThreads / 32));
    const unsigned mgrid = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(want, 6LL * sms)));
    if (g.block == 32) sample_mark_kernel<32><<<mgrid, kSampleThreads, msmem, st>>>(sp);
    else if (g.block == 64) sample_mark_kernel<64><<<mgrid, kSampleThreads, msmem, st>>>(sp);
    else sample_mark_kernel<128><<<mgrid, kSampleThreads, msmem, st>>>(sp);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    const unsigned cgrid2 = static_cast<unsigned>((static_cast<int64_t>(g.nb) * 32 + kSampleThreads - 1) / kSampleThreads);
    sample_compact_kernel<<<cgrid2, kSampleThreads, 0, st>>>(sp);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
  }
  // counts -> offsets -> compacted replica 0 -> replicas
  {
    const int64_t rows = g.nb;
    int64_t* partial = reinterpret_cast<int64_t*>(ws + w.partial);
    const int64_t tiles = (rows + 1 + kScanTile - 1) / kScanTile;
    scan_partial_kernel<<<static_cast<unsigned>(tiles), kScanThreads, 0, st>>>(row_ptr, rows, partial);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    CompactParams cp;
    cp.row_ptr = row_ptr;
    cp.partial = partial;
    cp.rows = rows;
    cp.nb = g.nb;
    cp.cand_row_ptr = cand_row_ptr;
    cp.kept_tmp = sp.kept_tmp;
    cp.cand_nnz = cand_nnz;
    cp.col_idx = col_idx;
    cp.col_cap = col_cap;
    scan_apply_kernel<<<static_cast<unsigned>(tiles), kScanThreads, 0, st>>>(cp);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    const int64_t cblocks = (rows * 32 + kCompactThreads - 1) / kCompactThreads;
    compact_kernel<<<static_cast<unsigned>(cblocks), kCompactThreads, 0, st>>>(cp);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    replicate_csr_kernel<<<264, 256, 0, st>>>(row_ptr, col_idx, g.nb, replicas, col_cap);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
  }
  if (thresholds_out != nullptr &&
      cudaMemcpyAsync(thresholds_out, sp.thresholds, static_cast<size_t>(fp) * 8, cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
    return DYNRAD_ERR_CUDA;
  return DYNRAD_OK;
}

namespace {

struct TokWorkspace {
  size_t stats, best, thr, colcnt, zero_end, kept, src_ptr, src_col, partial, total;
};

TokWorkspace tok_layout(int64_t B, int64_t frames, int64_t nb, int64_t n, int64_t cand_nnz) {
  TokWorkspace w;
  const int64_t fp = B * frames * frames;
  const int64_t rows = B * nb;
  const int64_t tiles = (rows + 1 + kScanTile - 1) / kScanTile;
  w.stats = 0;
  w.best = align256(w.stats + static_cast<size_t>(fp) * 16);
  w.thr = align256(w.best + static_cast<size_t>(fp) * 8);
  w.colcnt = align256(w.thr + static_cast<size_t>(fp) * 8);
  w.zero_end = w.colcnt + static_cast<size_t>(rows) * n * 4;
  w.kept = align256(w.zero_end);
  w.src_ptr = align256(w.kept + static_cast<size_t>(B * cand_nnz) * 4);
  w.src_col = align256(w.src_ptr + static_cast<size_t>(rows + 1) * 4);
  w.partial = align256(w.src_col + static_cast<size_t>(B * cand_nnz) * 4);
  w.total = align256(w.partial + static_cast<size_t>(tiles) * 8);
  return w;
}

constexpr int kTokMaxFusedHeads = 4;

}  // namespace

size_t dynrad_token_mask_workspace_bytes(int32_t B, int32_t N, const dynrad_geom* geom, int64_t cand_nnz) {
  GeomDev g;
  if (check_geom(geom, &g) != DYNRAD_OK || B < 1 || N != g.n || cand_nnz < 1) return 0;
  return tok_layout(B, g.frames, g.nb, g.n, cand_nnz).total;
}

int dynrad_build_token_mask(const void* q, const void* k, int32_t B, int32_t H, int32_t N, int32_t D, int32_t hf,
                            const dynrad_geom* geom, double tau1, double tau2, const int32_t* cand_row_ptr,
                            const int32_t* cand_col, int64_t cand_nnz, const int32_t* forced_lo,
                            const int32_t* forced_hi, int32_t* row_ptr, int32_t* col_idx, int64_t col_cap,
                            double* stats_out, void* workspace, size_t workspace_bytes, dynrad_stream_t stream) {
  GeomDev g;
  int rc = check_geom(geom, &g);
  if (rc != DYNRAD_OK) return rc;
  if (q == nullptr || k == nullptr || cand_row_ptr == nullptr || cand_col == nullptr || forced_lo == nullptr ||
      forced_hi == nullptr || row_ptr == nullptr || col_idx == nullptr || workspace == nullptr)
    return DYNRAD_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N != g.n || cand_nnz < 1 || col_cap < 0) return DYNRAD_ERR_INVALID_ARG;
  if (hf < 1 || hf > H || !std::isfinite(tau1) || !std::isfinite(tau2)) return DYNRAD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k)) return DYNRAD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DYNRAD_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DYNRAD_ERR_UNSUPPORTED;
  if (hf > kTokMaxFusedHeads) return DYNRAD_ERR_UNSUPPORTED;
  if (g.block != 32 && g.block != 64 && g.block != 128) return DYNRAD_ERR_UNSUPPORTED;
  if (g.nt > 65535 || B > 65535) return DYNRAD_ERR_UNSUPPORTED;
  // the aggregation keeps a frame table and one flag per candidate in default shared memory
  if (static_cast<size_t>(g.frames) * 5 + static_cast<size_t>(g.nb) + 16 > 48 * 1024) return DYNRAD_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * g.nb + 1 > INT32_MAX || static_cast<int64_t>(B) * cand_nnz > INT32_MAX)
    return DYNRAD_ERR_UNSUPPORTED;
  const TokWorkspace w = tok_layout(B, g.frames, g.nb, g.n, cand_nnz);
  if (workspace_bytes < w.total) return DYNRAD_ERR_CAPACITY;
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DynTokParams tp;
  tp.g = g;
  tp.q = static_cast<const __nv_bfloat16*>(q);
  tp.k = static_cast<const __nv_bfloat16*>(k);
  tp.B = B;
  tp.H = H;
  tp.D = D;
  tp.hf = hf;
  tp.tau1 = tau1;
  tp.tau2 = tau2;
  tp.inv = 1.0f / (static_cast<float>(hf) * std::sqrt(static_cast<float>(D)));
  tp.stats = reinterpret_cast<double*>(ws + w.stats);
  tp.best = reinterpret_cast<unsigned long long*>(ws + w.best);
  tp.thr = reinterpret_cast<double*>(ws + w.thr);
  tp.colcnt = reinterpret_cast<uint32_t*>(ws + w.colcnt);
  tp.cand_row_ptr = cand_row_ptr;
  tp.cand_col = cand_col;
  tp.forced_lo = forced_lo;
  tp.forced_hi = forced_hi;
  int32_t* src_ptr = reinterpret_cast<int32_t*>(ws + w.src_ptr);
  int32_t* src_col = reinterpret_cast<int32_t*>(ws + w.src_col);
  tp.counts = src_ptr;
  tp.kept_tmp = reinterpret_cast<int32_t*>(ws + w.kept);
  tp.cand_nnz = cand_nnz;
  if (cudaMemsetAsync(ws, 0, w.zero_end, st) != cudaSuccess) return DYNRAD_ERR_CUDA;
  // logit tiles: tcgen05 for H_f * D <= 256, the warp-level MMA kernel above that
  const bool use_tc = hf * D <= 256;
  const void* tk = nullptr;
  size_t tsmem = 0;
  int tthreads = kTokThreads;
  int kid = 0;
#define DYNRAD_TOK_TC(D_, HF_, ID_)                                                     \
  if (D == D_ && hf == HF_) {                                                           \
    tk = reinterpret_cast<const void*>(dyntok_tc_kernel<D_, HF_>);                      \
    tsmem = TokTcCfg<D_, HF_>::kSmemTotal;                                              \
    tthreads = TokTcCfg<D_, HF_>::kThreads;                                             \
    kid = ID_;                                                                          \
  }
#define DYNRAD_TOK_MMA(D_, HF_, ID_)                                                    \
  if (D == D_ && hf == HF_) {                                                           \
    tk = reinterpret_cast<const void*>(dyntok_tile_kernel<D_, HF_>);                    \
    tsmem = tok_tile_smem(D_ * HF_);                                                    \
    kid = ID_;                                                                          \
  }
  DYNRAD_TOK_TC(64, 1, 0) DYNRAD_TOK_TC(64, 2, 1) DYNRAD_TOK_TC(64, 3, 2) DYNRAD_TOK_TC(64, 4, 3)
  DYNRAD_TOK_TC(128, 1, 4) DYNRAD_TOK_TC(128, 2, 5) DYNRAD_TOK_MMA(128, 3, 6) DYNRAD_TOK_MMA(128, 4, 7)
#undef DYNRAD_TOK_TC
#undef DYNRAD_TOK_MMA
  if (tk == nullptr) return DYNRAD_ERR_UNSUPPORTED;
  static OptInTable tok_optin[8];   // per instantiation, per device
  if ((rc = smem_optin(tok_optin[kid], tk, static_cast<int>(tsmem))) != DYNRAD_OK) return rc;
  CUtensorMap mq, mk;
  if (use_tc && (!encode_map(&mq, q, D, N, B * H, 128) || !encode_map(&mk, k, D, N, B * H, 128)))
    return DYNRAD_ERR_CUDA;
  const int fp = g.frames * g.frames;
  dim3 tgrid(fp, (g.nt + kTokRows - 1) / kTokRows, B);
  if (use_tc) {   // persistent: one CTA per SM over the (frame pair, 128 rows, batch) units
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
      return DYNRAD_ERR_CUDA;
    const int64_t units = static_cast<int64_t>(B) * fp * ((g.nt + 127) / 128);
    if (units > INT32_MAX) return DYNRAD_ERR_UNSUPPORTED;
    tgrid = dim3(static_cast<unsigned>(std::min<int64_t>(units, sms)), 1, 1);
  }
  for (int pass = 0; pass < 2; ++pass) {
    tp.pass = pass;
    void* args_tc[] = {&mq, &mk, &tp};
    void* args_mma[] = {&tp};
    if (cudaLaunchKernel(tk, tgrid, dim3(tthreads), use_tc ? args_tc : args_mma, tsmem, st) != cudaSuccess)
      return DYNRAD_ERR_CUDA;
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    if (pass == 0) {
      const int64_t m = static_cast<int64_t>(B) * fp;
      dyntok_finalize_kernel<<<static_cast<unsigned>((m + 255) / 256), 256, 0, st>>>(tp, stats_out);
      if ((rc = launch_status()) != DYNRAD_OK) return rc;
    }
  }
  const size_t asmem = static_cast<size_t>(g.frames) * 5 + static_cast<size_t>(g.nb) + 16;
  const dim3 agrid(g.nb, B);
  if (g.block == 32) dyntok_aggregate_kernel<32><<<agrid, kTokThreads, asmem, st>>>(tp);
  else if (g.block == 64) dyntok_aggregate_kernel<64><<<agrid, kTokThreads, asmem, st>>>(tp);
  else dyntok_aggregate_kernel<128><<<agrid, kTokThreads, asmem, st>>>(tp);
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  {
    const int64_t rows = static_cast<int64_t>(B) * g.nb;
    int64_t* partial = reinterpret_cast<int64_t*>(ws + w.partial);
    const int64_t tiles = (rows + 1 + kScanTile - 1) / kScanTile;
    scan_partial_kernel<<<static_cast<unsigned>(tiles), kScanThreads, 0, st>>>(src_ptr, rows, partial);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    CompactParams cp;
    cp.row_ptr = src_ptr;
    cp.partial = partial;
    cp.rows = rows;
    cp.nb = g.nb;
    cp.cand_row_ptr = cand_row_ptr;
    cp.kept_tmp = tp.kept_tmp;
    cp.cand_nnz = cand_nnz;
    cp.col_idx = src_col;
    cp.col_cap = static_cast<int64_t>(B) * cand_nnz;
    scan_apply_kernel<<<static_cast<unsigned>(tiles), kScanThreads, 0, st>>>(cp);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    const int64_t cblocks = (rows * 32 + kCompactThreads - 1) / kCompactThreads;
    compact_kernel<<<static_cast<unsigned>(cblocks), kCompactThreads, 0, st>>>(cp);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    expand_csr_kernel<<<264, 256, 0, st>>>(src_ptr, src_col, B, H, g.nb, row_ptr, col_idx, col_cap);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
  }
  return DYNRAD_OK;
}

}  // extern "C"

namespace {

struct BwdWorkspace {
  size_t aux, t_ptr, t_col, partial, total;
};

BwdWorkspace bwd_layout(int64_t bh, int64_t n, int64_t nb, int64_t col_cap) {
  BwdWorkspace w;
  const int64_t rows = bh * nb;
  const int64_t tiles = (rows + 1 + kScanTile - 1) / kScanTile;
  const int64_t np = (n + 63) / 64 * 64;
  w.aux = 0;
  w.t_ptr = align256(w.aux + static_cast<size_t>(bh * np) * 8);
  w.t_col = align256(w.t_ptr + static_cast<size_t>(rows + 1) * 4);
  w.partial = align256(w.t_col + static_cast<size_t>(col_cap) * 4);
  w.total = align256(w.partial + static_cast<size_t>(tiles) * 8);
  return w;
}

template <int D, int BS, bool KV>
int launch_bwd_tc(const BwdParams& bp, const CUtensorMap& r0, const CUtensorMap& r1, const CUtensorMap& s0,
                  const CUtensorMap& s1, const CUtensorMap& aux, cudaStream_t st) {
  using C = BwdTcCfg<D, BS, KV>;
  static OptInTable optin;   // per instantiation, per device
  const int rc0 = smem_optin(optin, reinterpret_cast<const void*>(bwd_tc_kernel<D, BS, KV>), C::kSmemTotal);
  if (rc0 != DYNRAD_OK) return rc0;
  const dim3 grid((bp.N + C::kRows - 1) / C::kRows, bp.BH);
  bwd_tc_kernel<D, BS, KV><<<grid, 320, C::kSmemTotal, st>>>(r0, r1, s0, s1, aux, bp);
  return launch_status();
}

// dK / dV (resident K, V; streamed Q, dO), then dQ (resident Q, dO; streamed K, V)
template <int D, int BS>
int launch_backward(const BwdParams& bp, cudaStream_t st) {
  CUtensorMap k128, v128, q64, do64, q128, do128, k64, v64, aux;
  if (!encode_map(&k128, bp.k, D, bp.N, bp.BH, 128) || !encode_map(&v128, bp.v, D, bp.N, bp.BH, 128) ||
      !encode_map(&q64, bp.q, D, bp.N, bp.BH, 64) || !encode_map(&do64, bp.dout, D, bp.N, bp.BH, 64) ||
      !encode_map(&q128, bp.q, D, bp.N, bp.BH, 128) || !encode_map(&do128, bp.dout, D, bp.N, bp.BH, 128) ||
      !encode_map(&k64, bp.k, D, bp.N, bp.BH, 64) || !encode_map(&v64, bp.v, D, bp.N, bp.BH, 64) ||
      !encode_aux_map(&aux, bp.aux, bp.Np, bp.BH))
    return DYNRAD_ERR_CUDA;
  const int rc = launch_bwd_tc<D, BS, true>(bp, k128, v128, q64, do64, aux, st);
  if (rc != DYNRAD_OK) return rc;
  return launch_bwd_tc<D, BS, false>(bp, q128, do128, k64, v64, aux, st);
}

}  // namespace

extern "C" {

size_t dynrad_attn_backward_workspace_bytes(int32_t B, int32_t H, int32_t N, int32_t block, int64_t col_cap) {
  if (B < 1 || H < 1 || N < 1 || block < 1 || col_cap < 0) return 0;
  const int64_t nb = (static_cast<int64_t>(N) + block - 1) / block;
  return bwd_layout(static_cast<int64_t>(B) * H, N, nb, col_cap).total;
}

int dynrad_attn_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, int32_t B, int32_t H, int32_t N, int32_t D, int32_t block,
                         const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap, float scale, void* dq,
                         void* dk, void* dv, void* workspace, size_t workspace_bytes, dynrad_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || dout == nullptr || lse == nullptr ||
      row_ptr == nullptr || col_idx == nullptr || dq == nullptr || dk == nullptr || dv == nullptr ||
      workspace == nullptr)
    return DYNRAD_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || col_cap < 0) return DYNRAD_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || !std::isfinite(scale)) return DYNRAD_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DYNRAD_ERR_UNSUPPORTED;
  if (block != 32 && block != 64 && block != 128) return DYNRAD_ERR_UNSUPPORTED;
  for (const void* ptr : {q, k, v, o, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
    if (!aligned16(ptr)) return DYNRAD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DYNRAD_ERR_INVALID_ARG;
  const int64_t bh = static_cast<int64_t>(B) * H;
  if (bh > 65535) return DYNRAD_ERR_UNSUPPORTED;
  const int64_t nb = (static_cast<int64_t>(N) + block - 1) / block;
  if (bh * nb + 1 > INT32_MAX) return DYNRAD_ERR_UNSUPPORTED;
  const BwdWorkspace w = bwd_layout(bh, N, nb, col_cap);
  if (workspace_bytes < w.total) return DYNRAD_ERR_CAPACITY;
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdParams bp;
  bp.q = static_cast<const __nv_bfloat16*>(q);
  bp.k = static_cast<const __nv_bfloat16*>(k);
  bp.v = static_cast<const __nv_bfloat16*>(v);
  bp.o = static_cast<const __nv_bfloat16*>(o);
  bp.dout = static_cast<const __nv_bfloat16*>(dout);
  bp.lse = lse;
  bp.aux = reinterpret_cast<float*>(ws + w.aux);
  bp.Np = (N + 63) / 64 * 64;
  bp.row_ptr = row_ptr;
  bp.col_idx = col_idx;
  bp.t_ptr = reinterpret_cast<int32_t*>(ws + w.t_ptr);
  bp.t_col = reinterpret_cast<int32_t*>(ws + w.t_col);
  bp.t_cap = col_cap;
  bp.dq = static_cast<__nv_bfloat16*>(dq);
  bp.dk = static_cast<__nv_bfloat16*>(dk);
  bp.dv = static_cast<__nv_bfloat16*>(dv);
  bp.BH = static_cast<int>(bh);
  bp.N = N;
  bp.nb = static_cast<int>(nb);
  bp.block = block;
  bp.scale = scale == 0.0f ? 1.0f / std::sqrt(static_cast<float>(D)) : scale;
  int rc;
  const int64_t rows = bh * nb;
  // (lse2, D_r) per query row, then the transposed CSR
  const int64_t nrows = bh * bp.Np;
  bwd_aux_kernel<<<static_cast<unsigned>((nrows * 32 + 255) / 256), 256, 0, st>>>(bp, D);
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  if (cudaMemsetAsync(bp.t_ptr, 0, static_cast<size_t>(rows + 1) * 4, st) != cudaSuccess) return DYNRAD_ERR_CUDA;
  const unsigned wblocks = static_cast<unsigned>((rows * 32 + 255) / 256);
  bwd_tcount_kernel<<<wblocks, 256, 0, st>>>(bp);
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  {
    int64_t* partial = reinterpret_cast<int64_t*>(ws + w.partial);
    const int64_t tiles = (rows + 1 + kScanTile - 1) / kScanTile;
    scan_partial_kernel<<<static_cast<unsigned>(tiles), kScanThreads, 0, st>>>(bp.t_ptr, rows, partial);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
    CompactParams cp;
    cp.row_ptr = bp.t_ptr;
    cp.partial = partial;
    cp.rows = rows;
    cp.nb = static_cast<int>(nb);
    cp.cand_row_ptr = nullptr;
    cp.kept_tmp = nullptr;
    cp.cand_nnz = 0;
    cp.col_idx = nullptr;
    cp.col_cap = 0;
    scan_apply_kernel<<<static_cast<unsigned>(tiles), kScanThreads, 0, st>>>(cp);
    if ((rc = launch_status()) != DYNRAD_OK) return rc;
  }
  bwd_tfill_kernel<<<wblocks, 256, 0, st>>>(bp);
  if ((rc = launch_status()) != DYNRAD_OK) return rc;
  if (D == 128) {
    if (block == 32) return launch_backward<128, 32>(bp, st);
    return block == 64 ? launch_backward<128, 64>(bp, st) : launch_backward<128, 128>(bp, st);
  }
  if (block == 32) return launch_backward<64, 32>(bp, st);
  return block == 64 ? launch_backward<64, 64>(bp, st) : launch_backward<64, 128>(bp, st);
}

int dynrad_sparse_attn(const void* q, const void* k, const void* v, int32_t B, int32_t H, int32_t N,
                       int32_t D, int32_t block, const int32_t* row_ptr, const int32_t* col_idx, float scale,
                       void* o, float* lse, dynrad_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || row_ptr == nullptr || col_idx == nullptr ||
      o == nullptr || lse == nullptr)
    return DYNRAD_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return DYNRAD_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || !std::isfinite(scale)) return DYNRAD_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DYNRAD_ERR_UNSUPPORTED;
  if (block != 32 && block != 64 && block != 128) return DYNRAD_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return DYNRAD_ERR_INVALID_ARG;
  const int64_t bh = static_cast<int64_t>(B) * H;
  if (bh > 65535) return DYNRAD_ERR_UNSUPPORTED;
  const int64_t nb = (static_cast<int64_t>(N) + block - 1) / block;
  if (static_cast<int64_t>(N) * D * 2 >= (int64_t(1) << 40)) return DYNRAD_ERR_UNSUPPORTED;
  if ((nb + 128 / block - 1) / (128 / block) > INT32_MAX) return DYNRAD_ERR_UNSUPPORTED;
  const float sc = scale == 0.0f ? 1.0f / std::sqrt(static_cast<float>(D)) : scale;
  cudaStream_t st = as_stream(stream);
  const int bhi = static_cast<int>(bh);
  if (D == 128) {
    if (block == 32) return launch_attn<128, 32>(q, k, v, bhi, N, row_ptr, col_idx, sc, o, lse, st);
    if (block == 64) return launch_attn<128, 64>(q, k, v, bhi, N, row_ptr, col_idx, sc, o, lse, st);
    return launch_attn<128, 128>(q, k, v, bhi, N, row_ptr, col_idx, sc, o, lse, st);
  }
  if (block == 32) return launch_attn<64, 32>(q, k, v, bhi, N, row_ptr, col_idx, sc, o, lse, st);
  if (block == 64) return launch_attn<64, 64>(q, k, v, bhi, N, row_ptr, col_idx, sc, o, lse, st);
  return launch_attn<64, 128>(q, k, v, bhi, N, row_ptr, col_idx, sc, o, lse, st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Stage 2 without a caller-provided workspace.
//
// Some callers cannot call cudaMalloc: a host library embedded in an
// application whose caching allocator owns all device memory, or code that must
// not risk the device-wide synchronisation a cudaMalloc / cudaFree may cause.
// For them the selection scratch lives in this file-scope device array.  Every
// GPU that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(32) << 20;  // 32 MiB

static __device__ __align__(256) unsigned char g_select_scratch[kStaticScratchBytes];

// Device address of g_select_scratch per device ordinal (the array's name in
// host code is only a stand-in), resolved on the first call on that device and
// again whenever the calling thread's context on it is another one than the
// address was resolved in (a cudaDeviceReset, or a caller that made its own
// context, loads the module anew).  Contexts are told apart by their unique
// id, which, unlike the handle, is never reused.
struct ScratchAddr {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;
};
std::mutex g_scratch_mu;
ScratchAddr g_scratch_addr[256];

// Unique id of the calling thread's current context; 0 when there is none yet
// or the driver does not provide the calls.
unsigned long long current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(f);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace

extern "C" size_t dynrad_static_scratch_bytes(void) { return kStaticScratchBytes; }

extern "C" int dynrad_select_blocks_static_scratch(
    const void* q, const void* k, int32_t B, int32_t H, int32_t N, int32_t D, const dynrad_geom* geom,
    const int32_t* cand_row_ptr, const int32_t* cand_col, int64_t cand_nnz, int64_t cand_max_row,
    const int32_t* forced_lo, const int32_t* forced_hi, int32_t mode, double rho_or_tau, int32_t* row_ptr,
    int32_t* col_idx, int64_t col_cap, float* scores_out, dynrad_stream_t stream) {
  const size_t need = dynrad_select_workspace_bytes(B, H, N, D, geom, cand_nnz);
  if (need == 0) return DYNRAD_ERR_INVALID_ARG;
  if (need > kStaticScratchBytes) return DYNRAD_ERR_CAPACITY;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return DYNRAD_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchAddr& e = g_scratch_addr[dev];
    const unsigned long long ctx = current_context_id();
    if (e.addr == nullptr || ctx == 0 || ctx != e.ctx_id) {
      // with this device current: the symbol lookup binds its context if needed
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr) return DYNRAD_ERR_CUDA;
      e.addr = p;
      e.ctx_id = current_context_id();
    }
    scratch = e.addr;
  }
  // The scratch needs no clearing: every byte the selection reads in it is
  // written earlier in the same call.
  return dynrad_select_blocks(q, k, B, H, N, D, geom, cand_row_ptr, cand_col, cand_nnz, cand_max_row, forced_lo,
                              forced_hi, mode, rho_or_tau, row_ptr, col_idx, col_cap, scores_out, scratch, need,
                              stream);
}
