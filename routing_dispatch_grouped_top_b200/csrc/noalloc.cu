// noalloc.cu - count/scan for callers that cannot allocate device memory.
//
// moe_count_scan needs scratch (a status word, the ticket and done counters and flags of its
// look-back scan, and two rows of per-expert counts per block) and takes it from a
// caller-owned workspace.  Some callers cannot provide one: a plugin running
// inside a host framework that owns every device allocation, or a real-time loop that
// must not allocate (cudaMalloc/cudaFree can also synchronize the device) once it is
// running.  For them moe_count_scan_noalloc runs the same kernels on a fixed scratch array
// that lives in this library's own device memory, so the call allocates nothing.  The
// scratch is a file-scope device array of MOE_NOALLOC_SCRATCH_BYTES; every GPU that loads
// the library holds it until the process exits.
#include <mutex>

#include "device.cuh"
#include "kernels.h"

namespace moe {
namespace {

// Same layout as the count/scan state of a caller workspace (ScanWorkspace).
static __device__ __align__(256) unsigned char g_scan_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// Device address of g_scan_scratch on the current device.  In host code the name
// g_scan_scratch is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
void* scratch_address() {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scan_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_count_scan_noalloc(const int32_t* topk_ids, const moe_dims* d, int32_t* counts,
                                             int32_t* offsets, int32_t* part_counts, int32_t* part_offsets,
                                             int32_t* row_of_assign, int32_t* assign_of_row, void* stream) {
  using namespace moe;
  const moe_status st = check_dims(d);  // the same shape checks (and codes) as moe_count_scan
  if (st != MOE_OK) return st;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  if (!counts || !offsets || !part_counts || !part_offsets ||
      (d->T > 0 && (!topk_ids || !row_of_assign || !assign_of_row)))
    return MOE_ERR_INVALID_ARG;
  const long long TK = d->T * static_cast<long long>(d->K);
  if (scan_ws_bytes(TK, d->E) > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED_SHAPE;
  uint8_t* base = static_cast<uint8_t*>(scratch_address());
  if (!base) return MOE_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The scratch keeps the previous call's contents.  The kernel leaves its counters and
  // look-back flags at zero, but a previous call whose kernel failed to launch or to finish
  // would not have: clear them (and the status word) on every call.
  if (cudaMemsetAsync(base, 0, ScanWorkspace::kFixedBytes, s) != cudaSuccess) return MOE_ERR_CUDA;
  const ScanWorkspace ws = scan_workspace(base, TK, d->E);
  if (launch_count_scan(topk_ids, TK, d->E, d->P, row_of_assign, counts, offsets, part_counts, part_offsets, nullptr,
                        ws, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_scan_finalize(topk_ids, TK, d->E, offsets, row_of_assign, assign_of_row, s) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
