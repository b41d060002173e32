// The whole path from and to host memory, with the host<->device copies
// overlapped with the kernels (a runtime convenience; the paper has no
// counterpart).
//
// The B*H (batch, head) rows of the layer are cut into chunks.  Four queues
// run at once: a copy-in stream moves the chunks' Q, K, V into the device
// workspace; two compute queues (the caller's stream and a second one) take
// the (chunk, run) items in turn and run stages 2 and 3 of each as soon as its
// chunk's inputs are in, each queue with its own kept CSR and selection
// workspace, so one item's kernels start while the previous item's attention
// kernel drains its last wave; and a copy-out stream returns each item's O and
// LSE as soon as its attention kernel is done.  PCIe is full duplex, so with
// enough chunks the copies hide behind the kernels except for the first
// chunk's copy-in and the last chunk's copy-out, which the schedule keeps small
// (chunks of 1 and 2 rows at both ends).
//
// Every stage is independent per (batch, head) row (the candidate set is
// shared geometry, the selection and the attention never mix rows), so a
// chunk's results are the same bits the device-resident calls produce for
// those rows.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <utility>
#include <vector>

#include "dynrad.h"

namespace {

constexpr int kMaxHostRuns = 16;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct HostLayout {
  size_t q = 0, k = 0, v = 0;   // full [B*H, N, D] inputs
  std::vector<size_t> o, lse;   // per run, full outputs
  size_t row_ptr[2] = {0, 0}, col[2] = {0, 0};  // per compute queue: a chunk's kept CSR (largest run)
  size_t sel[2] = {0, 0};                       // per compute queue: a chunk's selection workspace
  size_t sel_bytes = 0, col_cap = 0;
  size_t total = 0;
};

// Returns false on an argument error.
bool host_layout(int32_t B, int32_t H, int32_t N, int32_t D, const dynrad_host_run* runs, int32_t n_runs,
                 int32_t chunk_bh, HostLayout* out) {
  if (B < 1 || H < 1 || N < 1 || (D != 64 && D != 128) || runs == nullptr || n_runs < 1 ||
      n_runs > kMaxHostRuns || chunk_bh < 1)
    return false;
  const int64_t bh = static_cast<int64_t>(B) * H;
  const int64_t chunk = std::min<int64_t>(chunk_bh, bh);
  const size_t qkv = static_cast<size_t>(bh) * N * D * 2;
  HostLayout L;
  size_t off = 0;
  L.q = off;
  off += align256(qkv);
  L.k = off;
  off += align256(qkv);
  L.v = off;
  off += align256(qkv);
  int64_t max_nb = 0, max_col = 0;
  size_t max_sel = 0;
  for (int r = 0; r < n_runs; ++r) {
    const dynrad_host_run& run = runs[r];
    const int64_t nb = dynrad_num_blocks(&run.geom);
    if (nb <= 0 || run.cand_nnz < 1) return false;
    const size_t sel = dynrad_select_workspace_bytes(1, static_cast<int32_t>(chunk), N, D, &run.geom, run.cand_nnz);
    if (sel == 0) return false;
    max_nb = std::max(max_nb, nb);
    max_col = std::max(max_col, chunk * run.cand_nnz);
    max_sel = std::max(max_sel, sel);
    L.o.push_back(off);
    off += align256(qkv);
    L.lse.push_back(off);
    off += align256(static_cast<size_t>(bh) * N * 4);
  }
  for (int x = 0; x < 2; ++x) {
    L.row_ptr[x] = off;
    off += align256(static_cast<size_t>(chunk * max_nb + 1) * 4);
    L.col[x] = off;
    off += align256(static_cast<size_t>(max_col) * 4);
    L.sel[x] = off;
    off += align256(max_sel);
  }
  L.col_cap = static_cast<size_t>(max_col);
  L.sel_bytes = max_sel;
  L.total = off;
  *out = L;
  return true;
}

// Streams and events made for one call; released when the call returns (the
// runtime defers the release of objects with work still pending).
struct CallObjects {
  cudaStream_t in = nullptr, out = nullptr, comp = nullptr;
  std::vector<cudaEvent_t> events;
  ~CallObjects() {
    for (cudaEvent_t e : events) cudaEventDestroy(e);
    for (cudaStream_t s : {in, out, comp})
      if (s != nullptr) cudaStreamDestroy(s);
  }
  cudaEvent_t event() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    events.push_back(e);
    return e;
  }
};

// Joins the side streams back into the caller's stream when the call returns,
// on every path once they exist: whatever was queued on them (copies into the
// workspace from the caller's host buffers, kernels, copies out to them) is
// then ordered before anything the caller queues next, even after an error
// return.  If an event cannot be made, it falls back to waiting on the host.
struct JoinOnReturn {
  cudaStream_t main;
  CallObjects* co;
  ~JoinOnReturn() {
    for (cudaStream_t side : {co->in, co->comp, co->out}) {
      if (side == nullptr) continue;
      cudaEvent_t e = co->event();
      if (e == nullptr || cudaEventRecord(e, side) != cudaSuccess || cudaStreamWaitEvent(main, e, 0) != cudaSuccess)
        cudaStreamSynchronize(side);
    }
  }
};

}  // namespace

extern "C" {

size_t dynrad_host_path_workspace_bytes(int32_t B, int32_t H, int32_t N, int32_t D, const dynrad_host_run* runs,
                                        int32_t n_runs, int32_t chunk_bh) {
  HostLayout L;
  if (!host_layout(B, H, N, D, runs, n_runs, chunk_bh, &L)) return 0;
  return L.total;
}

int dynrad_host_path(const void* q_host, const void* k_host, const void* v_host, int32_t B, int32_t H, int32_t N,
                     int32_t D, const dynrad_host_run* runs, int32_t n_runs, int32_t chunk_bh, float scale,
                     void* workspace, size_t workspace_bytes, dynrad_stream_t stream) {
  if (q_host == nullptr || k_host == nullptr || v_host == nullptr || workspace == nullptr)
    return DYNRAD_ERR_INVALID_ARG;
  HostLayout L;
  if (!host_layout(B, H, N, D, runs, n_runs, chunk_bh, &L)) return DYNRAD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DYNRAD_ERR_INVALID_ARG;
  if (workspace_bytes < L.total) return DYNRAD_ERR_CAPACITY;
  for (int r = 0; r < n_runs; ++r) {
    const dynrad_host_run& run = runs[r];
    if (run.o_host == nullptr || run.lse_host == nullptr || run.cand_row_ptr == nullptr ||
        run.cand_col == nullptr || run.forced_lo == nullptr || run.forced_hi == nullptr)
      return DYNRAD_ERR_INVALID_ARG;
    if (dynrad_num_blocks(&run.geom) <= 0 || run.geom.frames * run.geom.height * run.geom.width != N)
      return DYNRAD_ERR_INVALID_ARG;
  }
  if (!(scale >= 0.0f) || !std::isfinite(scale)) return DYNRAD_ERR_INVALID_ARG;

  cudaStream_t main = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t bh = static_cast<int64_t>(B) * H;
  const int64_t chunk = std::min<int64_t>(chunk_bh, bh);
  // Chunk schedule: (first row, rows).  Only the first chunk's copy-in and the
  // last chunk's copy-out are not hidden behind kernels, so with room for it
  // the schedule starts and ends with chunks of 1 and 2 rows.
  std::vector<std::pair<int64_t, int64_t>> sched;
  {
    const bool ramp = chunk >= 4 && bh >= 2 * chunk + 6;
    int64_t r = 0;
    const int64_t edge[2] = {1, 2};
    if (ramp)
      for (int64_t e : edge) sched.push_back({r, e}), r += e;
    const int64_t mid_end = ramp ? bh - 3 : bh;
    while (r < mid_end) {
      const int64_t n = std::min(chunk, mid_end - r);
      sched.push_back({r, n});
      r += n;
    }
    if (ramp)
      for (int i = 1; i >= 0; --i) sched.push_back({r, edge[i]}), r += edge[i];
  }
  const int64_t n_chunks = static_cast<int64_t>(sched.size());
  const size_t row_in = static_cast<size_t>(N) * D * 2;   // bytes of one row of Q, K, V or O
  const size_t row_lse = static_cast<size_t>(N) * 4;

  CallObjects co;
  // declared after co: joins the side streams before co releases them
  JoinOnReturn join{main, &co};
  if (cudaStreamCreateWithFlags(&co.in, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&co.out, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&co.comp, cudaStreamNonBlocking) != cudaSuccess)
    return DYNRAD_ERR_CUDA;
  // the side streams start after everything already queued on the caller's
  // stream (an earlier call may still read this workspace)
  cudaEvent_t start = co.event();
  if (start == nullptr || cudaEventRecord(start, main) != cudaSuccess ||
      cudaStreamWaitEvent(co.in, start, 0) != cudaSuccess || cudaStreamWaitEvent(co.out, start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(co.comp, start, 0) != cudaSuccess)
    return DYNRAD_ERR_CUDA;

  // copy-in of every chunk, in order
  std::vector<cudaEvent_t> in_done(static_cast<size_t>(n_chunks));
  const void* src[3] = {q_host, k_host, v_host};
  const size_t dst[3] = {L.q, L.k, L.v};
  for (int64_t c = 0; c < n_chunks; ++c) {
    const int64_t r0 = sched[c].first, rows = sched[c].second;
    for (int t = 0; t < 3; ++t) {
      if (cudaMemcpyAsync(ws + dst[t] + r0 * row_in, static_cast<const uint8_t*>(src[t]) + r0 * row_in,
                          rows * row_in, cudaMemcpyHostToDevice, co.in) != cudaSuccess)
        return DYNRAD_ERR_CUDA;
    }
    in_done[c] = co.event();
    if (in_done[c] == nullptr || cudaEventRecord(in_done[c], co.in) != cudaSuccess) return DYNRAD_ERR_CUDA;
  }

  // (chunk, run) items alternate between the two compute queues, each with
  // its own kept CSR and selection workspace; copy-out per item
  const cudaStream_t queue[2] = {main, co.comp};
  int64_t item = 0;
  for (int64_t c = 0; c < n_chunks; ++c) {
    const int64_t r0 = sched[c].first, rows = sched[c].second;
    const uint8_t* qc = ws + L.q + r0 * row_in;
    const uint8_t* kc = ws + L.k + r0 * row_in;
    const uint8_t* vc = ws + L.v + r0 * row_in;
    for (int r = 0; r < n_runs; ++r, ++item) {
      const dynrad_host_run& run = runs[r];
      const int x = static_cast<int>(item & 1);
      const cudaStream_t s = queue[x];
      const dynrad_stream_t ss = reinterpret_cast<dynrad_stream_t>(s);
      int32_t* row_ptr = reinterpret_cast<int32_t*>(ws + L.row_ptr[x]);
      int32_t* col = reinterpret_cast<int32_t*>(ws + L.col[x]);
      if (cudaStreamWaitEvent(s, in_done[c], 0) != cudaSuccess) return DYNRAD_ERR_CUDA;
      int rc = dynrad_select_blocks(qc, kc, 1, static_cast<int32_t>(rows), N, D, &run.geom, run.cand_row_ptr,
                                    run.cand_col, run.cand_nnz, run.cand_max_row, run.forced_lo, run.forced_hi,
                                    run.mode, run.rho_or_tau, row_ptr, col, static_cast<int64_t>(L.col_cap),
                                    nullptr, ws + L.sel[x], L.sel_bytes, ss);
      if (rc != DYNRAD_OK) return rc;
      uint8_t* oc = ws + L.o[r] + r0 * row_in;
      float* lc = reinterpret_cast<float*>(ws + L.lse[r] + r0 * row_lse);
      rc = dynrad_sparse_attn(qc, kc, vc, 1, static_cast<int32_t>(rows), N, D, run.geom.block, row_ptr, col,
                              scale, oc, lc, ss);
      if (rc != DYNRAD_OK) return rc;
      cudaEvent_t done = co.event();
      if (done == nullptr || cudaEventRecord(done, s) != cudaSuccess ||
          cudaStreamWaitEvent(co.out, done, 0) != cudaSuccess)
        return DYNRAD_ERR_CUDA;
      if (cudaMemcpyAsync(static_cast<uint8_t*>(run.o_host) + r0 * row_in, oc, rows * row_in,
                          cudaMemcpyDeviceToHost, co.out) != cudaSuccess ||
          cudaMemcpyAsync(reinterpret_cast<uint8_t*>(run.lse_host) + r0 * row_lse, lc, rows * row_lse,
                          cudaMemcpyDeviceToHost, co.out) != cudaSuccess)
        return DYNRAD_ERR_CUDA;
    }
  }
  // the caller's stream continues once the last copy-out is done (join)
  return DYNRAD_OK;
}

}  // extern "C"
