// kernels.h - launchers of libmoe_b200's kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/moe.h"

namespace moe {

enum Epi : int { kEpiSwiGLU = 0, kEpiBF16 = 1, kEpiF32 = 2, kEpiSwiGLUFp8 = 4 };

struct GemmArgs {
  const int32_t* offsets;  // [G + 1] device row offsets of the groups, or nullptr: one group of M rows
  int G;
  int M;
  int N;                   // output features
  int Kd;                  // reduction length
  void* out;
  long long ldo;           // output row stride in elements
  const float* bias;       // kEpiF32 only: [N] or nullptr
  int* status;             // device status word (MOE_DEV_* bits)
  const float* scale_a0;   // kEpiSwiGLUFp8: per-feature scales of the gate weights [G][N]
  const float* scale_a1;   //                per-feature scales of the up weights [G][N]
  const float* scale_b;    //                per-row scales of the token operand [M]
  int* sched;              // two device ints {next tile, finished CTAs}, zero between launches
  int ksplit;              // kEpiF32: reduction split into this many partial outputs (0 or 1: none)
  long long split_stride;  // elements between the partial outputs of consecutive splits
  // CTA-pair kEpiSwiGLU only: token operand gathered in place.  Row r of the operand is row
  // gather[r] / gather_div of gather_x ([gather_rows][Kd] bf16) instead of row r of a permuted
  // copy; nullptr: rows are read as they lie.
  const int32_t* gather;
  int gather_div;
  int gather_rows;
  const void* gather_x;
};

int num_sms();             // SM count of the current device (cached per device)
bool device_ok();          // the current device is an sm_100 (cached per device)
moe_status check_dims(const moe_dims* d);  // the shape checks every entry point makes

// Raises `func`'s dynamic shared-memory limit to `bytes` on the current device, once per
// device: a function attribute belongs to the device's context, so a process that drives
// several GPUs sets it on each.  `done` is the caller's per-device flag table
// (kMaxDevices entries, zero-initialised).
constexpr int kMaxDevices = 64;
cudaError_t smem_attr_once(const void* func, int bytes, std::atomic<int>* done);

// Launches `kernel` with programmatic stream serialization, so that it may begin while
// the previous kernel on the stream drains (the kernel calls pdl_wait before reading).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
int gemm_smem_bytes(int epi);
// Average rows per group from which the grouped GEMMs use the CTA-pair kernel (< 0: never).
void set_pair_min_rows(int rows);

// With `gather` (assign_of_row of the layer's count/scan), the token operand's row r is row
// gather[r] / K of x ([x_rows][H]), read in place; otherwise x holds the permuted rows.
cudaError_t gemm_gate_up(const void* x, const int32_t* offsets, const void* w_gate, const void* w_up, int E,
                         long long rows, int H, int F, void* h, int* status, int* sched, cudaStream_t stream,
                         const int32_t* gather = nullptr, int K = 1, long long x_rows = 0);
// h = silu(s_x s_g (xq Wg_q^T)) * (s_x s_u (xq Wu_q^T)) on E4M3 operands.
cudaError_t gemm_gate_up_fp8(const void* xq, const float* xs, const int32_t* offsets, const void* wq_gate,
                             const void* wq_up, const float* s_gate, const float* s_up, int E, long long rows, int H,
                             int F, void* h, int* status, int* sched, cudaStream_t stream);
cudaError_t gemm_down(const void* h, const int32_t* offsets, const void* w_down, int E, long long rows, int H,
                      int F, void* y, int* status, int* sched, cudaStream_t stream);
cudaError_t gemm_dense(const void* a, const void* w, long long M, int N, int Kd, void* out, int* status,
                       int* sched, cudaStream_t stream);
// logits (ksplit <= 1), or ksplit partial sums at logits + s * T * E whose sum in order
// s = 0, 1, ... is the logits (bias in partial 0).  gating_splits picks ksplit.
cudaError_t gemm_gating(const void* x, const void* w_split, const float* bias, long long T, int H, int E,
                        float* logits, int ksplit, int* status, int* sched, cudaStream_t stream);
int gating_splits(long long T, int H, int E, int sms);
cudaError_t launch_sum_partials(const float* partials, int nsplit, long long n, float* out, cudaStream_t stream);

// With nsplit > 1 the logits are the in-order sum of nsplit partial planes (T * E apart) starting
// at `logits`; the kernel writes that sum to `logits_out` as well.
cudaError_t launch_route(const float* logits, int nsplit, float* logits_out, long long T, int E, int K,
                         int renormalize, int P, int group_limit, int32_t* ids, float* w, cudaStream_t stream);

// Count/scan state inside a workspace (or the library's own scratch):
//   [0] status word, [64] ticket, [96] done counter, [128] failure flag (the bytes 160-255
//   belong to the GEMMs' tile schedules), [256] kScanMaxBlocks look-back flags, then
//   agg[nb][E] and inc[nb][E] (each 256-byte aligned).  The ticket, done counter, failure
//   flag and flags are zero between calls (the last block of every call clears them; the
//   workspace starts zeroed).
constexpr int kScanMaxBlocks = 128;
inline size_t round256(size_t n) { return (n + 255) / 256 * 256; }
struct ScanWorkspace {
  static constexpr size_t kFixedBytes = 256 + kScanMaxBlocks * sizeof(int);
  int* status;
  int* ticket;
  int* done;
  int* fail;
  int* flags;   // [kScanMaxBlocks]
  int* agg;     // [nb][E] per-block counts
  int* inc;     // [nb][E] per-block inclusive prefixes over blocks
};
int scan_blocks(long long TK);                      // blocks (chunks) of one count/scan call
size_t scan_ws_bytes(long long TK, int E);          // bytes of the state above
ScanWorkspace scan_workspace(void* base, long long TK, int E);
// One pass: ranks[a] = rank of assignment a among the assignments of its expert (stable), or -1
// for an id outside [0, E); counts, offsets (offsets[E] = -1 after a device-side failure),
// partition counts/offsets and the skew ratio (nullable).
cudaError_t launch_count_scan(const int32_t* ids, long long TK, int E, int P, int32_t* ranks, int32_t* counts,
                              int32_t* offsets, int32_t* part_counts, int32_t* part_offsets, float* skew,
                              const ScanWorkspace& ws, cudaStream_t stream);
// row_of_assign (holding the ranks) becomes offsets[ids[a]] + rank in place; assign_of_row its inverse.
cudaError_t launch_scan_finalize(const int32_t* ids, long long TK, int E, const int32_t* offsets,
                                 int32_t* row_of_assign, int32_t* assign_of_row, cudaStream_t stream);
cudaError_t launch_skew(const int32_t* counts, int E, float* ratio, cudaStream_t stream);

// With rank_offsets != nullptr, row_of_assign holds count_scan's ranks: the row of assignment a
// is rank_offsets[ids[a]] + rank, written back to row_of_assign[a] (and assign_of_row[row] = a).
cudaError_t launch_permute(const void* x, int32_t* row_of_assign, const int32_t* ids, const float* w,
                           long long T, int H, int E, int K, int P, void* xp, int32_t* meta_token,
                           int32_t* meta_slot, float* meta_w, int32_t* meta_local, const int32_t* rank_offsets,
                           int32_t* assign_of_row, cudaStream_t stream);
cudaError_t launch_quantize_fp8_rows(const void* x, long long rows, int cols, void* q, float* scales,
                                     cudaStream_t stream);
cudaError_t launch_permute_fp8(const void* x, int32_t* row_of_assign, const int32_t* ids, const float* w,
                               long long T, int H, int E, int K, int P, void* xq, float* xs, int32_t* meta_token,
                               int32_t* meta_slot, float* meta_w, int32_t* meta_local, const int32_t* rank_offsets,
                               int32_t* assign_of_row, cudaStream_t stream);
cudaError_t launch_combine(const void* y, const int32_t* row_of_assign, const float* w, const void* shared,
                           long long T, int H, int K, void* out, cudaStream_t stream);
cudaError_t launch_pack_router(const float* w_g, int H, int E, void* w_split, cudaStream_t stream);

}  // namespace moe
