// api.cu - the C ABI of libmoe_b200 (declared in include/moe.h): argument
// checks, workspace layout and the order of the layer's launches.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <vector>

#include "device.cuh"
#include "kernels.h"

namespace moe {

int num_sms() {
  static std::atomic<int> cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    n = n > 0 ? n : 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

cudaError_t smem_attr_once(const void* func, int bytes, std::atomic<int>* done) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const bool tracked = dev >= 0 && dev < kMaxDevices;
  if (tracked && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess && tracked) done[dev].store(1, std::memory_order_release);
  return err;
}

bool device_ok() {
  static std::atomic<int> cache[kMaxDevices] = {};  // 0 unknown, 1 ok, -1 not sm_100
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  int ok = cache[dev].load(std::memory_order_relaxed);
  if (ok == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    ok = (major == 10 && minor == 0) ? 1 : -1;
    cache[dev].store(ok, std::memory_order_relaxed);
  }
  return ok == 1;
}

moe_status check_dims(const moe_dims* d) {
  if (!d) return MOE_ERR_INVALID_ARG;
  if (d->T < 0 || d->E < 1 || d->K < 1 || d->K > d->E || d->P < 1 || d->E % d->P != 0 || d->H < 8 ||
      d->F < 8 || d->d_model < 0)
    return MOE_ERR_INVALID_ARG;
  if (d->H % 8 != 0 || d->F % 8 != 0 || d->d_model % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (d->E > MOE_MAX_E || d->K > MOE_MAX_K) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (d->group_limit < 0 || d->group_limit > d->P ||
      (d->group_limit > 0 && d->K > static_cast<long long>(d->group_limit) * (d->E / d->P)))
    return MOE_ERR_INVALID_ARG;
  if (d->group_limit > 0 && d->P > MOE_MAX_LIMITED_GROUPS) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (d->F_shared < 0) return MOE_ERR_INVALID_ARG;
  if (d->F_shared % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (d->fp8_dispatch != 0 && d->fp8_dispatch != 1) return MOE_ERR_INVALID_ARG;
  if (d->fp8_dispatch && d->H % 16 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (d->T * static_cast<long long>(d->K) > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

namespace {

// Workspace: the count/scan state (ScanWorkspace: [0] status word, [64, 160) the count/scan
// ticket, done counter and failure flag, [256 ...) look-back flags, expert totals and per-block
// rows), whose bytes [160 + 16 s, 176 + 16 s) hold the GEMM tile schedule of call site s
// (s < 6); then the gating partials.
constexpr size_t kWsHeader = 256;
enum SchedSlot : int { kSchedGating = 0, kSchedGateUp, kSchedDown, kSchedDense, kSchedSharedGateUp, kSchedSharedDown };

// The split gating reduction keeps its partial logits after the histograms.  The workspace
// is sized for a 148-SM B200; a device with fewer SMs uses fewer splits.
constexpr int kSizingSms = 148;

size_t scan_bytes(const moe_dims* d) { return scan_ws_bytes(d->T * static_cast<long long>(d->K), d->E); }

int gating_split_count(const moe_dims* d) {
  return std::min(gating_splits(d->T, d->H, d->E, num_sms()), gating_splits(d->T, d->H, d->E, kSizingSms));
}

size_t ws_bytes_for(const moe_dims* d) {
  const int S = gating_splits(d->T, d->H, d->E, kSizingSms);
  const size_t partials = S > 1 ? static_cast<size_t>(S) * d->T * d->E * sizeof(float) : 0;
  return scan_bytes(d) + partials;
}

float* ws_partials(void* ws, const moe_dims* d) {
  return reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + scan_bytes(d));
}

int* ws_status(void* ws) { return reinterpret_cast<int*>(ws); }
int* ws_sched(void* ws, SchedSlot s) { return reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(ws) + 160 + 16 * s); }

ScanWorkspace scan_ws(void* ws, const moe_dims* d) {
  return scan_workspace(ws, d->T * static_cast<long long>(d->K), d->E);
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                      \
  do {                                     \
    const moe_status _s = (expr);          \
    if (_s != MOE_OK) return _s;           \
  } while (0)

#define MOE_CUDA(expr)                                        \
  do {                                                        \
    if ((expr) != cudaSuccess) return MOE_ERR_CUDA;           \
  } while (0)

moe_status common_checks(const moe_dims* d) {
  MOE_TRY(check_dims(d));
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  return MOE_OK;
}

moe_status check_ws(const void* ws, size_t ws_bytes, const moe_dims* d) {
  if (!ws) return MOE_ERR_WORKSPACE;
  if (ws_bytes < ws_bytes_for(d)) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// The grouped GEMMs use only the workspace header (status word and tile-schedule counters).
moe_status check_ws_header(const void* ws, size_t ws_bytes) {
  if (!ws || ws_bytes < kWsHeader || reinterpret_cast<uintptr_t>(ws) % 256 != 0) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_bytes(const moe_dims* d) {
  if (check_dims(d) != MOE_OK) return 0;
  return ws_bytes_for(d);
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kWsHeader) return MOE_ERR_WORKSPACE;
  MOE_CUDA(cudaMemsetAsync(ws, 0, ws_bytes, as_stream(stream)));
  return MOE_OK;
}

moe_status moe_read_device_status(const void* ws, int32_t* status, void* stream) {
  if (!ws || !status) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(cudaStreamSynchronize(as_stream(stream)));
  MOE_CUDA(cudaMemcpy(status, ws, sizeof(int32_t), cudaMemcpyDeviceToHost));
  return MOE_OK;
}

const char* moe_status_str(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE_BAD_INDEX: return "device-side index out of range";
    case MOE_ERR_NO_DEVICE: return "no sm_100 device is current";
  }
  return "unknown status";
}

moe_status moe_pack_router(const float* w_g, const moe_dims* d, void* w_g_split, void* stream) {
  MOE_TRY(common_checks(d));
  if (!w_g || !w_g_split) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_pack_router(w_g, d->H, d->E, w_g_split, as_stream(stream)));
}

moe_status moe_gating(const void* x, const void* w_g_split, const float* bias, const moe_dims* d, float* logits,
                      void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(common_checks(d));
  MOE_TRY(check_ws(ws, ws_bytes, d));
  if (d->T == 0) return MOE_OK;
  if (!x || !w_g_split || !logits) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_g_split)) return MOE_ERR_INVALID_ARG;
  const int S = gating_split_count(d);
  if (S <= 1)
    return cuda_status(gemm_gating(x, w_g_split, bias, d->T, d->H, d->E, logits, 1, ws_status(ws),
                                   ws_sched(ws, kSchedGating), as_stream(stream)));
  float* partials = ws_partials(ws, d);
  MOE_CUDA(gemm_gating(x, w_g_split, bias, d->T, d->H, d->E, partials, S, ws_status(ws), ws_sched(ws, kSchedGating),
                       as_stream(stream)));
  return cuda_status(launch_sum_partials(partials, S, d->T * static_cast<long long>(d->E), logits, as_stream(stream)));
}

moe_status moe_route(const float* logits, const moe_dims* d, int32_t* topk_ids, float* topk_w, void* stream) {
  MOE_TRY(common_checks(d));
  if (d->T == 0) return MOE_OK;
  if (!logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_route(logits, 1, nullptr, d->T, d->E, d->K, d->renormalize, d->P, d->group_limit,
                                  topk_ids, topk_w, as_stream(stream)));
}

moe_status moe_count_scan(const int32_t* topk_ids, const moe_dims* d, int32_t* counts, int32_t* offsets,
                          int32_t* part_counts, int32_t* part_offsets, int32_t* row_of_assign,
                          int32_t* assign_of_row, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(common_checks(d));
  MOE_TRY(check_ws(ws, ws_bytes, d));
  if (!counts || !offsets || !part_counts || !part_offsets || (d->T > 0 && (!topk_ids || !row_of_assign ||
                                                                           !assign_of_row)))
    return MOE_ERR_INVALID_ARG;
  const long long TK = d->T * static_cast<long long>(d->K);
  MOE_CUDA(launch_count_scan(topk_ids, TK, d->E, d->P, row_of_assign, counts, offsets, part_counts, part_offsets,
                             nullptr, scan_ws(ws, d), as_stream(stream)));
  return cuda_status(launch_scan_finalize(topk_ids, TK, d->E, offsets, row_of_assign, assign_of_row,
                                          as_stream(stream)));
}

moe_status moe_permute(const void* x, const int32_t* row_of_assign, const int32_t* topk_ids, const float* topk_w,
                       const moe_dims* d, void* xp, int32_t* meta_token, int32_t* meta_slot, float* meta_w,
                       int32_t* meta_local_expert, void* stream) {
  MOE_TRY(common_checks(d));
  if (d->T == 0) return MOE_OK;
  if (!x || !row_of_assign || !xp || (meta_w && !topk_w) || (meta_local_expert && !topk_ids))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xp)) return MOE_ERR_INVALID_ARG;
  // the rows are given: the kernel only reads row_of_assign
  return cuda_status(launch_permute(x, const_cast<int32_t*>(row_of_assign), topk_ids, topk_w, d->T, d->H, d->E, d->K,
                                    d->P, xp, meta_token, meta_slot, meta_w, meta_local_expert, nullptr, nullptr,
                                    as_stream(stream)));
}

void moe_set_pair_min_rows(int32_t rows) { set_pair_min_rows(rows); }

moe_status moe_quantize_fp8_rows(const void* x, int64_t rows, int32_t cols, void* q, float* scales, void* stream) {
  if (rows < 0 || cols < 16) return MOE_ERR_INVALID_ARG;
  if (cols % 16 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  if (rows == 0) return MOE_OK;
  if (!x || !q || !scales || !aligned16(x) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_quantize_fp8_rows(x, rows, cols, q, scales, as_stream(stream)));
}

moe_status moe_permute_fp8(const void* x, const int32_t* row_of_assign, const int32_t* topk_ids,
                           const float* topk_w, const moe_dims* d, void* xq, float* xs, int32_t* meta_token,
                           int32_t* meta_slot, float* meta_w, int32_t* meta_local_expert, void* stream) {
  MOE_TRY(common_checks(d));
  if (d->H % 16 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (d->T == 0) return MOE_OK;
  if (!x || !row_of_assign || !xq || !xs || (meta_w && !topk_w) || (meta_local_expert && !topk_ids))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_permute_fp8(x, const_cast<int32_t*>(row_of_assign), topk_ids, topk_w, d->T, d->H, d->E,
                                        d->K, d->P, xq, xs, meta_token, meta_slot, meta_w, meta_local_expert, nullptr,
                                        nullptr, as_stream(stream)));
}

moe_status moe_grouped_gate_up_fp8(const void* xq, const float* xs, const int32_t* offsets, const void* wq_gate,
                                   const void* wq_up, const float* s_gate, const float* s_up, const moe_dims* d,
                                   void* h, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(common_checks(d));
  MOE_TRY(check_ws_header(ws, ws_bytes));
  if (d->H % 16 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (d->T == 0) return MOE_OK;
  if (!xq || !xs || !offsets || !wq_gate || !wq_up || !s_gate || !s_up || !h) return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(wq_gate) || !aligned16(wq_up) || !aligned16(h)) return MOE_ERR_INVALID_ARG;
  return cuda_status(gemm_gate_up_fp8(xq, xs, offsets, wq_gate, wq_up, s_gate, s_up, d->E,
                                      d->T * static_cast<long long>(d->K), d->H, d->F, h, ws_status(ws),
                                      ws_sched(ws, kSchedGateUp), as_stream(stream)));
}

moe_status moe_grouped_gate_up(const void* xp, const int32_t* offsets, const void* w_gate, const void* w_up,
                               const moe_dims* d, void* h, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(common_checks(d));
  MOE_TRY(check_ws_header(ws, ws_bytes));
  if (d->T == 0) return MOE_OK;
  if (!xp || !offsets || !w_gate || !w_up || !h) return MOE_ERR_INVALID_ARG;
  if (!aligned16(xp) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(h)) return MOE_ERR_INVALID_ARG;
  return cuda_status(gemm_gate_up(xp, offsets, w_gate, w_up, d->E, d->T * static_cast<long long>(d->K), d->H,
                                  d->F, h, ws_status(ws), ws_sched(ws, kSchedGateUp), as_stream(stream)));
}

moe_status moe_grouped_gate_up_gather(const void* x, const int32_t* assign_of_row, const int32_t* offsets,
                                      const void* w_gate, const void* w_up, const moe_dims* d, void* h, void* ws,
                                      size_t ws_bytes, void* stream) {
  MOE_TRY(common_checks(d));
  MOE_TRY(check_ws_header(ws, ws_bytes));
  if (d->T == 0) return MOE_OK;
  if (!x || !assign_of_row || !offsets || !w_gate || !w_up || !h) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(h)) return MOE_ERR_INVALID_ARG;
  return cuda_status(gemm_gate_up(x, offsets, w_gate, w_up, d->E, d->T * static_cast<long long>(d->K), d->H, d->F, h,
                                  ws_status(ws), ws_sched(ws, kSchedGateUp), as_stream(stream), assign_of_row, d->K,
                                  d->T));
}

moe_status moe_grouped_down(const void* h, const int32_t* offsets, const void* w_down, const moe_dims* d, void* y,
                            void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(common_checks(d));
  MOE_TRY(check_ws_header(ws, ws_bytes));
  if (d->T == 0) return MOE_OK;
  if (!h || !offsets || !w_down || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_down) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  return cuda_status(gemm_down(h, offsets, w_down, d->E, d->T * static_cast<long long>(d->K), d->H, d->F, y,
                               ws_status(ws), ws_sched(ws, kSchedDown), as_stream(stream)));
}

moe_status moe_grouped_ffn(const void* xp, const int32_t* offsets, const void* w_gate, const void* w_up,
                           const void* w_down, const moe_dims* d, void* h, void* y, void* ws, size_t ws_bytes,
                           void* stream) {
  MOE_TRY(moe_grouped_gate_up(xp, offsets, w_gate, w_up, d, h, ws, ws_bytes, stream));
  return moe_grouped_down(h, offsets, w_down, d, y, ws, ws_bytes, stream);
}

moe_status moe_combine(const void* y, const int32_t* row_of_assign, const float* topk_w, const void* shared,
                       const moe_dims* d, void* out, void* stream) {
  MOE_TRY(common_checks(d));
  if (d->T == 0) return MOE_OK;
  if (!y || !row_of_assign || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(out) || !aligned16(shared)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine(y, row_of_assign, topk_w, shared, d->T, d->H, d->K, out, as_stream(stream)));
}

moe_status moe_skew_stats(const int32_t* counts, const moe_dims* d, float* d_ratio, void* stream) {
  MOE_TRY(common_checks(d));
  if (!counts || !d_ratio) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_skew(counts, d->E, d_ratio, as_stream(stream)));
}

double moe_p95(const float* ratios, int n) {
  if (!ratios || n <= 0) return NAN;
  std::vector<float> v(ratios, ratios + n);
  std::sort(v.begin(), v.end());
  const int r = std::max(1, static_cast<int>(std::ceil(0.95 * n - 1e-9)));
  return static_cast<double>(v[r - 1]);
}

moe_status moe_dense(const void* a, const void* w, int64_t M, int32_t N, int32_t Kd, void* out, void* ws,
                     size_t ws_bytes, void* stream) {
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  if (!a || !w || !out || !ws || M < 0 || N < 8 || Kd < 8) return MOE_ERR_INVALID_ARG;
  if (N % 8 != 0 || Kd % 8 != 0 || M > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < kWsHeader || reinterpret_cast<uintptr_t>(ws) % 256 != 0) return MOE_ERR_WORKSPACE;
  if (!aligned16(a) || !aligned16(w) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (M == 0) return MOE_OK;
  return cuda_status(gemm_dense(a, w, M, N, Kd, out, ws_status(ws), ws_sched(ws, kSchedDense), as_stream(stream)));
}

moe_status moe_layer_forward(const void* x, const moe_layer_weights* w, const moe_dims* d,
                             const moe_layer_buffers* b, void* ws, size_t ws_bytes, void* const* stage_events,
                             void* stream) {
  MOE_TRY(common_checks(d));
  MOE_TRY(check_ws(ws, ws_bytes, d));
  if (d->T == 0) {
    // No tokens: only the per-expert outputs exist, all zero (count/scan of no assignments).
    if (!b || !b->counts || !b->offsets || !b->part_counts || !b->part_offsets) return MOE_ERR_INVALID_ARG;
    cudaStream_t s0 = as_stream(stream);
    for (int i = 0; stage_events && i < MOE_NUM_STAGE_EVENTS; ++i)
      if (stage_events[i]) MOE_CUDA(cudaEventRecord(reinterpret_cast<cudaEvent_t>(stage_events[i]), s0));
    return cuda_status(launch_count_scan(nullptr, 0, d->E, d->P, nullptr, b->counts, b->offsets, b->part_counts,
                                         b->part_offsets, b->skew, scan_ws(ws, d), s0));
  }
  if (!x || !w || !b) return MOE_ERR_INVALID_ARG;
  const bool latent = d->d_model > 0;
  const bool fp8 = d->fp8_dispatch != 0;
  if (!w->w_g_split || !w->w_down) return MOE_ERR_INVALID_ARG;
  if (!fp8 && (!w->w_gate || !w->w_up)) return MOE_ERR_INVALID_ARG;
  if (fp8 && (!w->w_gate_q || !w->w_up_q || !w->s_gate || !w->s_up || !b->xq || !b->xs)) return MOE_ERR_INVALID_ARG;
  if (fp8 && (!aligned16(w->w_gate_q) || !aligned16(w->w_up_q) || !aligned16(b->xq))) return MOE_ERR_INVALID_ARG;
  if (latent && (!w->w_dp || !w->w_upp || !b->z || !b->final_out)) return MOE_ERR_INVALID_ARG;
  const bool shared = d->F_shared > 0;
  if (shared && (!w->w_shared_gate || !w->w_shared_up || !w->w_shared_down || !b->h_shared || !b->y_shared))
    return MOE_ERR_INVALID_ARG;
  if (shared && b->aux_stream && (!b->fork_event || !b->join_event)) return MOE_ERR_INVALID_ARG;
  if (!b->logits || !b->topk_ids || !b->topk_w || !b->counts || !b->offsets || !b->part_counts ||
      !b->part_offsets || !b->row_of_assign || !b->assign_of_row || !b->h || !b->y || !b->out)
    return MOE_ERR_INVALID_ARG;
  // bf16 dispatch without an xp buffer: the gate/up GEMM reads each row's token in place
  const bool gather = !fp8 && !b->xp;
  // every bf16 row buffer is read or written in 16-byte pieces
  for (const void* p : {x, static_cast<const void*>(b->xp), static_cast<const void*>(b->h), static_cast<const void*>(b->y),
                        static_cast<const void*>(b->out), static_cast<const void*>(b->z),
                        static_cast<const void*>(b->final_out), static_cast<const void*>(b->h_shared),
                        static_cast<const void*>(b->y_shared)})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  auto mark = [&](int i) -> moe_status {
    if (stage_events && stage_events[i])
      return cuda_status(cudaEventRecord(reinterpret_cast<cudaEvent_t>(stage_events[i]), s));
    return MOE_OK;
  };
  int* status = ws_status(ws);
  const long long T = d->T, TK = d->T * static_cast<long long>(d->K);
  MOE_TRY(mark(0));
  const void* routed = x;
  if (latent) {
    if (T > 0) MOE_CUDA(gemm_dense(x, w->w_dp, T, d->H, d->d_model, b->z, status, ws_sched(ws, kSchedDense), s));
    routed = b->z;
  }
  MOE_TRY(mark(1));
  // Shared expert: a dense SwiGLU over every token, beside the routed path.
  cudaStream_t sh = s;
  if (shared && T > 0) {
    if (b->aux_stream) {
      sh = as_stream(b->aux_stream);
      MOE_CUDA(cudaEventRecord(reinterpret_cast<cudaEvent_t>(b->fork_event), s));
      MOE_CUDA(cudaStreamWaitEvent(sh, reinterpret_cast<cudaEvent_t>(b->fork_event), 0));
    }
    MOE_CUDA(gemm_gate_up(routed, nullptr, w->w_shared_gate, w->w_shared_up, 1, T, d->H, d->F_shared, b->h_shared,
                          status, ws_sched(ws, kSchedSharedGateUp), sh));
    MOE_CUDA(gemm_down(b->h_shared, nullptr, w->w_shared_down, 1, T, d->H, d->F_shared, b->y_shared, status,
                       ws_sched(ws, kSchedSharedDown), sh));
    if (b->aux_stream) MOE_CUDA(cudaEventRecord(reinterpret_cast<cudaEvent_t>(b->join_event), sh));
  }
  // Gating with a split reduction leaves partial logits in the workspace; the route kernel adds
  // them in split order and writes the logits buffer.
  const int nsplit = gating_split_count(d);
  float* gate_out = nsplit > 1 ? ws_partials(ws, d) : b->logits;
  if (T > 0)
    MOE_CUDA(gemm_gating(routed, w->w_g_split, w->bias, T, d->H, d->E, gate_out, nsplit, status,
                         ws_sched(ws, kSchedGating), s));
  MOE_TRY(mark(2));
  MOE_CUDA(launch_route(gate_out, nsplit, b->logits, T, d->E, d->K, d->renormalize, d->P, d->group_limit, b->topk_ids,
                        b->topk_w, s));
  MOE_TRY(mark(3));
  // count/scan leaves each assignment's rank within its expert in row_of_assign; the permute
  // turns it into the row (offsets[e] + rank) and writes assign_of_row (and, without a
  // gather, copies the rows)
  MOE_CUDA(launch_count_scan(b->topk_ids, TK, d->E, d->P, b->row_of_assign, b->counts, b->offsets, b->part_counts,
                             b->part_offsets, b->skew, scan_ws(ws, d), s));
  MOE_TRY(mark(4));
  if (fp8)
    MOE_CUDA(launch_permute_fp8(routed, b->row_of_assign, b->topk_ids, b->topk_w, T, d->H, d->E, d->K, d->P, b->xq,
                                b->xs, b->meta_token, b->meta_slot, b->meta_w, b->meta_local_expert, b->offsets,
                                b->assign_of_row, s));
  else
    MOE_CUDA(launch_permute(routed, b->row_of_assign, b->topk_ids, b->topk_w, T, d->H, d->E, d->K, d->P, b->xp,
                            b->meta_token, b->meta_slot, b->meta_w, b->meta_local_expert, b->offsets,
                            b->assign_of_row, s));
  MOE_TRY(mark(5));
  if (T > 0) {
    if (fp8)
      MOE_CUDA(gemm_gate_up_fp8(b->xq, b->xs, b->offsets, w->w_gate_q, w->w_up_q, w->s_gate, w->s_up, d->E, TK, d->H,
                                d->F, b->h, status, ws_sched(ws, kSchedGateUp), s));
    else
      MOE_CUDA(gemm_gate_up(gather ? routed : b->xp, b->offsets, w->w_gate, w->w_up, d->E, TK, d->H, d->F, b->h,
                            status, ws_sched(ws, kSchedGateUp), s, gather ? b->assign_of_row : nullptr, d->K, T));
  }
  MOE_TRY(mark(6));
  if (T > 0)
    MOE_CUDA(gemm_down(b->h, b->offsets, w->w_down, d->E, TK, d->H, d->F, b->y, status, ws_sched(ws, kSchedDown), s));
  MOE_TRY(mark(7));
  if (shared && T > 0 && b->aux_stream)
    MOE_CUDA(cudaStreamWaitEvent(s, reinterpret_cast<cudaEvent_t>(b->join_event), 0));
  MOE_CUDA(launch_combine(b->y, b->row_of_assign, b->topk_w, shared ? b->y_shared : nullptr, T, d->H, d->K,
                          b->out, s));
  MOE_TRY(mark(8));
  if (latent && T > 0)
    MOE_CUDA(gemm_dense(b->out, w->w_upp, T, d->d_model, d->H, b->final_out, status, ws_sched(ws, kSchedDense), s));
  MOE_TRY(mark(9));
  return MOE_OK;
}

moe_status moe_layer_forward_host(const void* x_host, void* x_dev, const moe_layer_weights* w, const moe_dims* d,
                                  const moe_layer_buffers* b, void* ws, size_t ws_bytes, void* out_host,
                                  void* stream) {
  MOE_TRY(common_checks(d));
  if (d->T == 0) return moe_layer_forward(x_dev, w, d, b, ws, ws_bytes, nullptr, stream);
  if (!x_host || !x_dev || !out_host || !b) return MOE_ERR_INVALID_ARG;
  const bool latent = d->d_model > 0;
  const size_t d_in = latent ? d->d_model : d->H;
  cudaStream_t s = as_stream(stream);
  MOE_CUDA(cudaMemcpyAsync(x_dev, x_host, static_cast<size_t>(d->T) * d_in * 2, cudaMemcpyHostToDevice, s));
  MOE_TRY(moe_layer_forward(x_dev, w, d, b, ws, ws_bytes, nullptr, stream));
  const void* res = latent ? b->final_out : b->out;
  MOE_CUDA(cudaMemcpyAsync(out_host, res, static_cast<size_t>(d->T) * d_in * 2, cudaMemcpyDeviceToHost, s));
  return MOE_OK;
}

}  // extern "C"
