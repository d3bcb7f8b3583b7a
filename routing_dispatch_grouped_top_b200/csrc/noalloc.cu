// noalloc.cu - count/scan for callers that cannot allocate device memory.
//
// moe_count_scan needs scratch (a status word, the grid-barrier words of its
// cooperative kernel and one expert histogram per block) and takes it from a
// caller-owned workspace.  Some callers cannot provide one: a plugin running inside
// a host framework that owns every device allocation, or a real-time loop that must
// not allocate (cudaMalloc/cudaFree can also synchronize the device) once it is
// running.  For them moe_count_scan_noalloc runs the same kernel on a fixed scratch
// array that lives in this library's own device memory, so the call allocates
// nothing.  The scratch is a file-scope device array of MOE_NOALLOC_SCRATCH_BYTES;
// every GPU that loads the library holds it until the process exits.
#include <mutex>

#include "device.cuh"
#include "kernels.h"

namespace moe {
namespace {

// Layout (same as a caller workspace): [0] status word, [64] grid-barrier count,
// [128] grid-barrier generation, [256 ...) per-block expert histograms.
constexpr size_t kHeaderBytes = 256;
static __device__ __align__(256) unsigned char g_scan_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// Device address of g_scan_scratch on the current device.  In host code the name
// g_scan_scratch is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
void* scratch_address() {
  static void* addr[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scan_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

bool device_is_sm100() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
  return major == 10 && minor == 0;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_count_scan_noalloc(const int32_t* topk_ids, const moe_dims* d, int32_t* counts,
                                             int32_t* offsets, int32_t* part_counts, int32_t* part_offsets,
                                             int32_t* row_of_assign, int32_t* assign_of_row, void* stream) {
  using namespace moe;
  if (moe_workspace_bytes(d) == 0) return MOE_ERR_INVALID_ARG;  // shape checks of the other calls
  if (!counts || !offsets || !part_counts || !part_offsets ||
      (d->T > 0 && (!topk_ids || !row_of_assign || !assign_of_row)))
    return MOE_ERR_INVALID_ARG;
  const long long TK = d->T * static_cast<long long>(d->K);
  const int blocks = scan_max_blocks(TK);
  if (kHeaderBytes + static_cast<size_t>(blocks) * d->E * sizeof(int) > MOE_NOALLOC_SCRATCH_BYTES)
    return MOE_ERR_UNSUPPORTED_SHAPE;  // histograms would not fit the fixed scratch
  if (!device_is_sm100()) return MOE_ERR_NO_DEVICE;
  uint8_t* base = static_cast<uint8_t*>(scratch_address());
  if (!base) return MOE_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The scratch keeps the previous call's contents: the status and barrier words must
  // start at zero (the histograms are fully rewritten by every call).
  if (cudaMemsetAsync(base, 0, kHeaderBytes, s) != cudaSuccess) return MOE_ERR_CUDA;
  ScanWorkspace ws;
  ws.status = reinterpret_cast<int*>(base);
  ws.bar_count = reinterpret_cast<unsigned int*>(base + 64);
  ws.bar_gen = reinterpret_cast<unsigned int*>(base + 128);
  ws.block_counts = reinterpret_cast<int*>(base + kHeaderBytes);
  ws.max_blocks = blocks;
  const cudaError_t e = launch_count_scan(topk_ids, TK, d->E, d->P, counts, offsets, part_counts, part_offsets,
                                          row_of_assign, assign_of_row, nullptr, ws, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
