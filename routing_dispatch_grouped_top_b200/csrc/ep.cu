// ep.cu - expert-parallel dispatch and return across GPUs (NVLink peer stores).
//
// With expert parallelism the experts are split evenly over R ranks (rank d owns experts
// [d El, (d + 1) El), El = E / R), and the router's choices become a network schedule: each
// rank counts what every destination receives, reserves the rows there, sends the
// activations, and the expert outputs come back to be weighted and summed at their tokens
// (WideEP essay, "The router writes a network schedule"; "Top-k multiplies traffic.
// Locality subtracts it." for the T x K x H x b bytes each way; EP8 places 32 of 256
// experts per GPU in the InferenceX v2 review, claim IX2-0384).
//
// Layout.  Rank d receives its rows expert-major, then source-major, then in the source's
// own stable order: the rows of local expert l from source s start at
//   recv_offsets[l] + sum_{s' < s} C[s'][d El + l],  recv_offsets[l] = sum_{l' < l} sum_s C[s][d El + l'],
// where C[s][e] is source s's count for expert e (all-gathered before the dispatch).  This
// is exactly the single-GPU expert-major layout of all ranks' tokens concatenated in rank
// order, restricted to rank d's experts; the grouped GEMM runs on it with recv_offsets.
//
// Kernels (all bounds-checked; every wait bounded):
//   ep_plan_kernel     send_base[e] (where this rank's rows of expert e start in the owner's
//                      receive buffer) and recv_offsets[El + 1], from C on the device;
//   ep_dispatch_kernel 16-byte peer stores of each token row to the K owners' receive
//                      buffers, plus (source rank, source row) per row; the last block then
//                      publishes the call's epoch in every peer's signal pad (release, system
//                      scope) after a system-scope fence of every block's stores;
//   ep_wait_kernel     acquire-loads this rank's signal pad until every source has published
//                      the epoch (2 s limit, then MOE_DEV_TIMEOUT);
//   ep_return_kernel   peer stores of each received row's expert output to its source's
//                      return buffer, at the source's own row (so the source's combine runs
//                      unchanged on row_of_assign), then the same signal.
// Peer pointers arrive by value in a kernel parameter (no device pointer table), and no
// load or store here uses TMA or multicast.
#include <algorithm>
#include <cstring>

#include "device.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kEpThreads = 256;
constexpr int kPlanThreads = 1024;

struct EpArgs {
  void* recv_x[MOE_EP_MAX_RANKS];
  int32_t* recv_meta[MOE_EP_MAX_RANKS];
  void* ret_y[MOE_EP_MAX_RANKS];
  int32_t* signal[MOE_EP_MAX_RANKS];
};

__device__ __forceinline__ void st_release_sys(int32_t* p, int v) {
  asm volatile("st.release.sys.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire_sys(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.sys.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// After a block's peer stores: every thread fences its own stores at system scope, the block
// counts itself done, and the last block (after an acquiring fence) publishes `epoch` in slot
// [phase][rank] of every peer's signal pad with release stores, then rewinds the counter.
__device__ void signal_when_done(const EpArgs& peers, int R, int rank, int phase, int epoch, int* done) {
  __threadfence_system();
  __syncthreads();
  if (threadIdx.x == 0 && atomicAdd(done, 1) == static_cast<int>(gridDim.x) - 1) {
    __threadfence_system();
    for (int d = 0; d < R; ++d) st_release_sys(peers.signal[d] + phase * R + rank, epoch);
    atomicExch(done, 0);
  }
}

// send_base[E], recv_offsets[El + 1] from C [R][E].
__global__ void __launch_bounds__(kPlanThreads) ep_plan_kernel(const int32_t* __restrict__ C, int R, int E, int rank,
                                                               int32_t* __restrict__ send_base,
                                                               int32_t* __restrict__ recv_offsets) {
  __shared__ int s_col[MOE_MAX_E + 1], s_pre[MOE_MAX_E], s_warp[kPlanThreads / 32];
  pdl_wait();  // the count matrix comes from the all-gather
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int El = E / R;
  // column sums over the sources, and this rank's predecessors' part of them
  for (int e = tid; e < E; e += kPlanThreads) {
    int col = 0, pre = 0;
    for (int s = 0; s < R; ++s) {
      const int c = __ldg(C + static_cast<long long>(s) * E + e);
      col += c;
      if (s < rank) pre += c;
    }
    s_col[e] = col;
    s_pre[e] = pre;
  }
  __syncthreads();
  // exclusive scan of the column sums over the experts (E <= 1024: one per thread)
  const int v = tid < E ? s_col[tid] : 0;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
  for (int w = 0; w < kPlanThreads / 32; ++w) {
    if (w < warp) wbase += s_warp[w];
    total += s_warp[w];
  }
  __syncthreads();
  if (tid < E) s_col[tid] = wbase + incl - v;  // exclusive prefix
  if (tid == 0) s_col[E] = total;
  __syncthreads();
  for (int e = tid; e < E; e += kPlanThreads) {
    const int owner0 = (e / El) * El;
    send_base[e] = s_col[e] - s_col[owner0] + s_pre[e];
    if (e / El == rank) recv_offsets[e - owner0] = s_col[e] - s_col[owner0];
  }
  if (tid == 0) recv_offsets[El] = s_col[(rank + 1) * El] - s_col[rank * El];
}

// Token rows to their owners.  Item space (token, 16-byte vector) as in the permute; the
// K copies of a vector go to the K assignments' owners.  Then (rank, row) per assignment.
__global__ void __launch_bounds__(kEpThreads) ep_dispatch_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ roa, const int32_t* __restrict__ ids,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ send_base, long long T, int vpr, int E, int K,
    int R, int rank, long long cap, const __grid_constant__ EpArgs peers, int epoch, int* status, int* done) {
  pdl_wait();
  pdl_launch_dependents();
  const int El = E / R;
  const long long TK = T * K;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  bool bad = false;
  for (long long it = tid; it < T * vpr; it += stride) {
    const long long t = it / vpr;
    const int vec = static_cast<int>(it - t * vpr);
    const uint4 v = __ldg(x + it);
    for (int k = 0; k < K; ++k) {
      const long long a = t * K + k;
      const int e = __ldg(ids + a);
      const int r = __ldg(roa + a);
      if (e < 0 || e >= E || r < 0 || r >= TK) {
        bad = true;
        continue;
      }
      const long long row = static_cast<long long>(__ldg(send_base + e)) + (r - __ldg(offsets + e));
      if (row < 0 || row >= cap) {
        bad = true;
        continue;
      }
      reinterpret_cast<uint4*>(peers.recv_x[e / El])[row * vpr + vec] = v;
    }
  }
  for (long long a = tid; a < TK; a += stride) {
    const int e = __ldg(ids + a);
    const int r = __ldg(roa + a);
    if (e < 0 || e >= E || r < 0 || r >= TK) continue;
    const long long row = static_cast<long long>(__ldg(send_base + e)) + (r - __ldg(offsets + e));
    if (row < 0 || row >= cap) continue;
    reinterpret_cast<int2*>(peers.recv_meta[e / El])[row] = make_int2(rank, r);
  }
  if (bad) report(status, MOE_DEV_BAD_INDEX);
  signal_when_done(peers, R, rank, 0, epoch, done);
}

// Received rows' outputs back to their sources, at the source's own row.
__global__ void __launch_bounds__(kEpThreads) ep_return_kernel(
    const uint4* __restrict__ y, const int2* __restrict__ meta, const int32_t* __restrict__ recv_offsets, int El,
    long long cap, long long src_rows, int vpr, int R, int rank, const __grid_constant__ EpArgs peers, int epoch,
    int* status, int* done) {
  pdl_wait();
  pdl_launch_dependents();
  const long long n = min(static_cast<long long>(__ldg(recv_offsets + El)), cap);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  bool bad = false;
  for (long long it = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; it < n * vpr; it += stride) {
    const long long j = it / vpr;
    const int vec = static_cast<int>(it - j * vpr);
    const int2 m = __ldg(meta + j);
    if (m.x < 0 || m.x >= R || m.y < 0 || m.y >= src_rows) {
      bad = true;
      continue;
    }
    reinterpret_cast<uint4*>(peers.ret_y[m.x])[static_cast<long long>(m.y) * vpr + vec] = __ldg(y + it);
  }
  if (bad) report(status, MOE_DEV_BAD_INDEX);
  signal_when_done(peers, R, rank, 1, epoch, done);
}

// Until every source has published at least `epoch` in this rank's pad, slot [phase][s].
__global__ void ep_wait_kernel(const int32_t* signal, int R, int phase, int epoch, int* status) {
  pdl_wait();
  pdl_launch_dependents();
  for (int s = threadIdx.x; s < R; s += blockDim.x) {
    const int32_t* p = signal + phase * R + s;
    if (ld_acquire_sys(p) >= epoch) continue;
    const uint64_t t0 = global_timer_ns();
    unsigned int i = 0;
    while (ld_acquire_sys(p) < epoch) {
      if ((++i & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
        report(status, MOE_DEV_TIMEOUT);
        break;
      }
    }
  }
}

// The plan on the host, from the same definition (used to check the device plan and by
// callers that hold the count matrix on the host).
void ep_plan_host(const int32_t* C, int R, int E, int rank, int32_t* send_base, int32_t* recv_offsets) {
  const int El = E / R;
  long long run = 0;
  long long owner_start = 0;
  for (int e = 0; e < E; ++e) {
    if (e % El == 0) owner_start = run;
    long long col = 0, pre = 0;
    for (int s = 0; s < R; ++s) {
      col += C[static_cast<long long>(s) * E + e];
      if (s < rank) pre += C[static_cast<long long>(s) * E + e];
    }
    send_base[e] = static_cast<int32_t>(run - owner_start + pre);
    if (e / El == rank) recv_offsets[e % El] = static_cast<int32_t>(run - owner_start);
    run += col;
    if (e / El == rank && e % El == El - 1) recv_offsets[El] = static_cast<int32_t>(run - owner_start);
  }
}

moe_status ep_checks(const moe_dims* d, int R, int rank) {
  const moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (R < 1 || rank < 0 || rank >= R || d->E % R != 0) return MOE_ERR_INVALID_ARG;
  if (R > MOE_EP_MAX_RANKS) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

bool fill_peers(const moe_ep_peers* p, int R, EpArgs* a) {
  std::memset(a, 0, sizeof(*a));
  for (int d = 0; d < R; ++d) {
    if (!p->recv_x[d] || !p->recv_meta[d] || !p->ret_y[d] || !p->signal[d]) return false;
    if ((reinterpret_cast<uintptr_t>(p->recv_x[d]) | reinterpret_cast<uintptr_t>(p->ret_y[d])) & 15u) return false;
    a->recv_x[d] = p->recv_x[d];
    a->recv_meta[d] = p->recv_meta[d];
    a->ret_y[d] = p->ret_y[d];
    a->signal[d] = p->signal[d];
  }
  return true;
}

int ep_blocks(long long items) {
  const long long want = (items + kEpThreads - 1) / kEpThreads;
  return static_cast<int>(std::max<long long>(1, std::min<long long>(want, 8LL * num_sms())));
}

// Workspace of the EP calls: [0] status word, [64] dispatch done counter, [128] return done counter.
constexpr size_t kEpWsBytes = 256;
int* ep_status(void* ws) { return static_cast<int*>(ws); }
int* ep_done(void* ws, int phase) { return reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + 64 * (1 + phase)); }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_ep_workspace_bytes(void) { return kEpWsBytes; }

moe_status moe_ep_plan_host(const int32_t* counts_all, int32_t R, int32_t rank, const moe_dims* d,
                            int32_t* send_base, int32_t* recv_offsets) {
  const moe_status st = ep_checks(d, R, rank);
  if (st != MOE_OK) return st;
  if (!counts_all || !send_base || !recv_offsets) return MOE_ERR_INVALID_ARG;
  ep_plan_host(counts_all, R, d->E, rank, send_base, recv_offsets);
  return MOE_OK;
}

moe_status moe_ep_plan(const int32_t* counts_all, int32_t R, int32_t rank, const moe_dims* d, int32_t* send_base,
                       int32_t* recv_offsets, void* stream) {
  const moe_status st = ep_checks(d, R, rank);
  if (st != MOE_OK) return st;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  if (!counts_all || !send_base || !recv_offsets) return MOE_ERR_INVALID_ARG;
  return launch_pdl(ep_plan_kernel, dim3(1), dim3(kPlanThreads), 0, reinterpret_cast<cudaStream_t>(stream),
                    counts_all, static_cast<int>(R), d->E, static_cast<int>(rank), send_base, recv_offsets) ==
                         cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status moe_ep_dispatch(const void* x, const int32_t* row_of_assign, const int32_t* topk_ids,
                           const int32_t* offsets, const int32_t* send_base, const moe_dims* d, int32_t R,
                           int32_t rank, int64_t cap, const moe_ep_peers* peers, int32_t epoch, void* ep_ws,
                           void* stream) {
  const moe_status st = ep_checks(d, R, rank);
  if (st != MOE_OK) return st;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  if (!peers || !ep_ws || cap < 0 || epoch < 1) return MOE_ERR_INVALID_ARG;
  if (d->T > 0 && (!x || !row_of_assign || !topk_ids || !offsets || !send_base)) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) & 15u) return MOE_ERR_INVALID_ARG;
  EpArgs a;
  if (!fill_peers(peers, R, &a)) return MOE_ERR_INVALID_ARG;
  const int vpr = d->H / 8;
  const long long items = std::max<long long>(d->T * vpr, d->T * static_cast<long long>(d->K));
  return launch_pdl(ep_dispatch_kernel, dim3(ep_blocks(items)), dim3(kEpThreads), 0,
                    reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const uint4*>(x), row_of_assign,
                    topk_ids, offsets, send_base, static_cast<long long>(d->T), vpr, d->E, d->K, static_cast<int>(R),
                    static_cast<int>(rank), static_cast<long long>(cap), a, static_cast<int>(epoch),
                    ep_status(ep_ws), ep_done(ep_ws, 0)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status moe_ep_wait(const int32_t* signal, int32_t R, int32_t phase, int32_t epoch, void* ep_ws, void* stream) {
  if (!signal || !ep_ws || R < 1 || R > MOE_EP_MAX_RANKS || phase < 0 || phase > 1 || epoch < 1)
    return MOE_ERR_INVALID_ARG;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  return launch_pdl(ep_wait_kernel, dim3(1), dim3(64), 0, reinterpret_cast<cudaStream_t>(stream), signal,
                    static_cast<int>(R), static_cast<int>(phase), static_cast<int>(epoch), ep_status(ep_ws)) ==
                         cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status moe_ep_return(const void* y_recv, const int32_t* recv_meta, const int32_t* recv_offsets, const moe_dims* d,
                         int32_t R, int32_t rank, int64_t cap, const moe_ep_peers* peers, int32_t epoch, void* ep_ws,
                         void* stream) {
  const moe_status st = ep_checks(d, R, rank);
  if (st != MOE_OK) return st;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  if (!peers || !ep_ws || cap < 0 || epoch < 1 || !recv_offsets || (cap > 0 && (!y_recv || !recv_meta)))
    return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(y_recv) & 15u) return MOE_ERR_INVALID_ARG;
  EpArgs a;
  if (!fill_peers(peers, R, &a)) return MOE_ERR_INVALID_ARG;
  const int vpr = d->H / 8;
  return launch_pdl(ep_return_kernel, dim3(ep_blocks(cap * vpr)), dim3(kEpThreads), 0,
                    reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const uint4*>(y_recv),
                    reinterpret_cast<const int2*>(recv_meta), recv_offsets, d->E / static_cast<int>(R),
                    static_cast<long long>(cap), d->T * static_cast<long long>(d->K), vpr, static_cast<int>(R),
                    static_cast<int>(rank), a, static_cast<int>(epoch), ep_status(ep_ws), ep_done(ep_ws, 1)) ==
                         cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status moe_ep_ipc_export(const void* dev_ptr, void* handle, uint64_t* offset) {
  if (!dev_ptr || !handle || !offset) return MOE_ERR_INVALID_ARG;
  CUdeviceptr base = 0;
  size_t size = 0;
  // the handle names the whole allocation; the pointer is an offset into it
  using RangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
  static RangeFn range = nullptr;
  if (!range) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return MOE_ERR_CUDA;
    range = reinterpret_cast<RangeFn>(p);
  }
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return MOE_ERR_CUDA;
  std::memcpy(handle, &h, sizeof(h));
  *offset = static_cast<uint64_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return MOE_OK;
}

moe_status moe_ep_ipc_import(const void* handle, uint64_t offset, void** base, void** dev_ptr) {
  if (!handle || !base || !dev_ptr) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return MOE_ERR_CUDA;
  *base = p;
  *dev_ptr = static_cast<uint8_t*>(p) + offset;
  return MOE_OK;
}

moe_status moe_ep_ipc_close(void* base) {
  if (!base) return MOE_ERR_INVALID_ARG;
  return cudaIpcCloseMemHandle(base) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
