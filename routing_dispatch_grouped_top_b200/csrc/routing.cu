// routing.cu - router top-K, per-expert count + stable scan, skew statistics.
//
// The router keeps the K best-scoring experts of each token, and the dispatcher
// counts what every expert receives and reserves its rows (WideEP essay, "The
// router writes a network schedule").  Counts are per token-expert assignment
// and the skew statistic is the busiest expert's load over the mean load
// ("Three Parameter Counts...", "What the utilization dashboard smooths away").
#include <cuda/atomic>

#include <algorithm>

#include "device.cuh"
#include "kernels.h"

namespace moe {

namespace {

// ---------------------------------------------------------------------------
// Top-K: one warp per token.  Lane l owns experts e = l + 32 i (i < VPL).  Each
// logit becomes a 32-bit order key: the order-preserving image of the float
// (-0.0 folded into +0.0), 1 for NaN (below every number) and 0 for an empty or
// retired slot.  The warp keeps the keys of its token in shared memory and each
// lane its best (key, i), ties to the lower i.  A round takes the warp maximum of
// the lanes' best keys and, among the lanes holding it, the lowest expert id
// (two warp reductions), so equal values prefer the lower expert id.  The winner's
// slot is cleared and its owner's best is rebuilt by the whole warp: lane j reads
// the owner's slot j, two more reductions give the new best.  Slot w + 32 j is
// only ever read or written by lane j during the rounds.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t order_key(float v) {
  if (v != v) return 1u;    // NaN ranks below every number, above an empty slot
  if (v == 0.0f) v = 0.0f;  // -0.0 == +0.0
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // -inf -> 0x007fffff > 1
}

__device__ __forceinline__ float key_value(uint32_t k) {
  if (k <= 1u) return __uint_as_float(0x7fc00000u);
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Warps per block: the per-warp key rows grow with VPL.
constexpr int route_warps(int vpl) { return vpl <= 8 ? 8 : 4; }

template <int VPL>
__global__ void __launch_bounds__(32 * route_warps(VPL)) route_kernel(
    const float* __restrict__ logits, int nsplit, float* __restrict__ logits_out, long long T, int E, int K,
    int renormalize, int P, int M, int32_t* __restrict__ ids, float* __restrict__ w) {
  constexpr int W = route_warps(VPL);
  constexpr unsigned kFull = 0xffffffffu;
  __shared__ alignas(16) uint32_t s_key[W][32 * VPL];
  // node-limited routing: each group's best key and expert, and the groups kept (per warp)
  __shared__ uint32_t s_gh[W][MOE_MAX_LIMITED_GROUPS];
  __shared__ int s_ge[W][MOE_MAX_LIMITED_GROUPS];
  __shared__ unsigned char s_kept[W][MOE_MAX_LIMITED_GROUPS];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const bool limited = M > 0 && M < P;
  const int epp = E / P;
  uint32_t* sk = s_key[wib];
  pdl_wait();  // logits come from the previous kernel
  pdl_launch_dependents();
  const long long warps = static_cast<long long>(gridDim.x) * W;
  for (long long t = static_cast<long long>(blockIdx.x) * W + wib; t < T; t += warps) {
    const float* row = logits + t * E;
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      v[i] = (e < E) ? __ldg(row + e) : 0.0f;
    }
    if (nsplit > 1) {
      // Split gating reduction: partial sums added in split order.  The loads of
      // kSplitBatch splits are issued before their additions so that their
      // latencies overlap (fewer splits per batch when each lane already holds
      // many experts); the additions keep the order p = 1, 2, ...
      constexpr int kSplitBatch = VPL <= 4 ? 4 : (VPL <= 8 ? 2 : 1);
      const long long plane = T * E;
      for (int p0 = 1; p0 < nsplit; p0 += kSplitBatch) {
        float part[kSplitBatch][VPL];
#pragma unroll
        for (int q = 0; q < kSplitBatch; ++q) {
#pragma unroll
          for (int i = 0; i < VPL; ++i) {
            const int e = lane + 32 * i;
            part[q][i] = (p0 + q < nsplit && e < E) ? __ldg(row + (p0 + q) * plane + e) : 0.0f;
          }
        }
#pragma unroll
        for (int q = 0; q < kSplitBatch; ++q) {
          if (p0 + q < nsplit) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) v[i] += part[q][i];
          }
        }
      }
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) logits_out[t * E + e] = v[i];
      }
    }
    uint32_t hk[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      hk[i] = (lane + 32 * i < E) ? order_key(v[i]) : 0u;
      sk[lane + 32 * i] = hk[i];
    }
    __syncwarp();
    if (limited) {
      // A group ranks by its best expert under the same order (higher key, then lower id).
      // Lane l owns groups l, l + 32, ... and scans their experts from shared memory; then
      // M rounds of the two warp reductions keep the best groups.
      uint32_t* gh = s_gh[wib];
      int* ge = s_ge[wib];
      for (int g = lane; g < P; g += 32) {
        const int e0 = g * epp;
        uint32_t bh = 0u;
        int be = e0;
        if ((epp & 3) == 0) {  // 16-byte aligned runs of 4 keys (e0 % 4 == 0)
          const uint4* q = reinterpret_cast<const uint4*>(sk + e0);
          for (int c = 0; c < (epp >> 2); ++c) {
            const uint4 h4 = q[c];
            const int e = e0 + 4 * c;
            if (h4.x > bh) bh = h4.x, be = e;
            if (h4.y > bh) bh = h4.y, be = e + 1;
            if (h4.z > bh) bh = h4.z, be = e + 2;
            if (h4.w > bh) bh = h4.w, be = e + 3;
          }
        } else {
          for (int e = e0; e < e0 + epp; ++e) {
            const uint32_t h = sk[e];
            if (h > bh) bh = h, be = e;
          }
        }
        gh[g] = bh;
        ge[g] = be;
        s_kept[wib][g] = 0;
      }
      for (int m = 0; m < M; ++m) {
        uint32_t bh = 0u;
        int be = 0x7fffffff;
        for (int g = lane; g < P; g += 32) {
          const uint32_t h = gh[g];
          if (h > bh || (h == bh && ge[g] < be)) bh = h, be = ge[g];
        }
        const uint32_t top = __reduce_max_sync(kFull, bh);
        const int e = __reduce_min_sync(kFull, bh == top ? be : 0x7fffffff);
        const int g = e / epp;  // every group not yet kept holds a candidate (key >= 1)
        if (lane == (g & 31)) {
          s_kept[wib][g] = 1;
          gh[g] = 0u;
        }
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !s_kept[wib][e / epp]) hk[i] = 0u, sk[e] = 0u;  // dropped groups leave the race
      }
      __syncwarp();
    }
    // Every real candidate has key >= 1; empty slots have 0.  K <= number of candidates.
    uint32_t bh = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (hk[i] > bh) bh = hk[i], bi = i;
    }
    int my_id = 0;
    uint32_t my_key = 0u;
    for (int k = 0; k < K; ++k) {
      const uint32_t m = __reduce_max_sync(kFull, bh);
      const int e = __reduce_min_sync(kFull, bh == m ? lane + 32 * bi : 0x7fffffff);
      if (lane == k) my_id = e, my_key = m;
      // retire e; the owner's best is rebuilt over its remaining slots
      const int owner = e & 31;
      uint32_t x = 0u;
      if (lane < VPL) {
        x = sk[owner + 32 * lane];
        if (owner + 32 * lane == e) sk[e] = x = 0u;
      }
      const uint32_t nm = __reduce_max_sync(kFull, x);
      const int ni = __reduce_min_sync(kFull, (lane < VPL && x == nm) ? lane : 0x7fffffff);
      if (lane == owner) bh = nm, bi = ni;
    }
    __syncwarp();  // the next token's keys overwrite this token's slots
    const float my_val = key_value(my_key);
    // Weights: exp(l_k - l_top) / (sum over the K selected, or over all E).
    const float top = __shfl_sync(kFull, my_val, 0);
    const float num = (lane < K) ? expf(my_val - top) : 0.0f;
    float den = 0.0f;
    if (renormalize) {
      den = num;
    } else {
      // the lane reads back only the logits it summed itself (same e = lane + 32 i)
      const float* r = nsplit > 1 ? logits_out + t * E : row;
      for (int e = lane; e < E; e += 32) den += expf(r[e] - top);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(kFull, den, o);
    if (lane < K) {
      ids[t * K + lane] = my_id;
      w[t * K + lane] = num / den;
    }
  }
}

template <int VPL>
cudaError_t launch_route_vpl(const float* logits, int nsplit, float* logits_out, long long T, int E, int K,
                             int renorm, int P, int M, int32_t* ids, float* w, cudaStream_t s) {
  constexpr int W = route_warps(VPL);
  const long long blocks = std::min<long long>((T + W - 1) / W, 64LL * num_sms());
  return launch_pdl(route_kernel<VPL>, dim3(static_cast<unsigned>(std::max<long long>(blocks, 1))), dim3(32 * W), 0,
                    s, logits, nsplit, logits_out, T, E, K, renorm, P, M, ids, w);
}

// out[i] = sum_{p < nsplit} partials[p * n + i], added in order p = 0, 1, ...
__global__ void sum_partials_kernel(const float* __restrict__ partials, int nsplit, long long n,
                                    float* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float v = partials[i];
    for (int p = 1; p < nsplit; ++p) v += partials[p * n + i];
    out[i] = v;
  }
}

// ---------------------------------------------------------------------------
// Count + scan + stable rank, one cooperative launch.
//  phase 1: block b histograms its contiguous slice of assignments -> block_counts[b][e]
//  grid barrier (bounded wait; all blocks are co-resident by the cooperative launch)
//  phase 2: offsets[e] = sum of all counts of experts < e; base[b][e] = offsets[e] +
//           counts of expert e in blocks < b.  Block 0 writes counts, offsets,
//           partition counts/offsets and the skew ratio.
//  phase 3: block b walks its slice in order, 256 assignments at a time; the rank of
//           an assignment among equal ids = earlier warps' counts (shared) + its rank
//           inside the warp (__match_any_sync); row = base + rank.
// ---------------------------------------------------------------------------

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kScanMinChunk = 1024;

__device__ bool grid_barrier(unsigned int* count, unsigned int* gen, unsigned int nblocks, int* status,
                             int* s_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    cuda::atomic_ref<unsigned int, cuda::thread_scope_device> c(*count), g(*gen);
    const unsigned int my_gen = g.load(cuda::memory_order_acquire);
    const unsigned int arrived = c.fetch_add(1u, cuda::memory_order_acq_rel);
    int ok = 1;
    if (arrived == nblocks - 1) {
      c.store(0u, cuda::memory_order_relaxed);
      g.fetch_add(1u, cuda::memory_order_release);
    } else {
      const uint64_t t0 = global_timer_ns();
      unsigned int i = 0;
      while (g.load(cuda::memory_order_acquire) == my_gen) {
        if ((++i & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
          report(status, MOE_DEV_TIMEOUT);
          ok = 0;
          break;
        }
      }
    }
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

__global__ void __launch_bounds__(kScanThreads) count_scan_kernel(
    const int32_t* __restrict__ ids, int TK, int E, int P, int chunk, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ part_counts, int32_t* __restrict__ part_offsets,
    int32_t* __restrict__ row_of_assign, int32_t* __restrict__ assign_of_row, float* __restrict__ skew,
    int* block_counts, unsigned int* bar_count, unsigned int* bar_gen, int* status) {
  extern __shared__ int sm[];
  int* s_hist = sm;                    // [E]   this block's histogram, then its running base
  int* s_off = s_hist + E;             // [E+1] global exclusive offsets
  int* s_wcnt = s_off + E + 1;         // [kScanWarps][E] per-warp counts of one 256-slice
  __shared__ int s_ok, s_bad, s_red[kScanWarps], s_max[kScanWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x;
  const int lo = min(TK, b * chunk), hi = min(TK, lo + chunk);

  for (int e = tid; e < E; e += kScanThreads) s_hist[e] = 0;
  for (int i = tid; i < kScanWarps * E; i += kScanThreads) s_wcnt[i] = 0;
  if (tid == 0) s_bad = 0;
  pdl_wait();  // the expert ids come from the route kernel
  pdl_launch_dependents();
  __syncthreads();

  // phase 1
  for (int a = lo + tid; a < hi; a += kScanThreads) {
    const int e = __ldg(ids + a);
    if (e >= 0 && e < E) atomicAdd(&s_hist[e], 1);
    else s_bad = 1;
  }
  __syncthreads();
  if (s_bad && tid == 0) report(status, MOE_DEV_BAD_INDEX);
  for (int e = tid; e < E; e += kScanThreads) block_counts[static_cast<long long>(b) * E + e] = s_hist[e];

  if (!grid_barrier(bar_count, bar_gen, gridDim.x, status, &s_ok)) return;

  // phase 2: column sums over blocks.  The block_counts rows start 16-byte aligned (the
  // workspace is 256-byte aligned), so with E % 4 == 0 a thread sums four experts per
  // 16-byte load and keeps eight loads in flight.
  int my_max = 0;
  const int nb = static_cast<int>(gridDim.x);
  if ((E & 3) == 0) {
    const int E4 = E >> 2;
    for (int q = tid; q < E4; q += kScanThreads) {
      const int4* col = reinterpret_cast<const int4*>(block_counts) + q;
      int4 before = make_int4(0, 0, 0, 0), total = make_int4(0, 0, 0, 0);
#pragma unroll 8
      for (int bb = 0; bb < nb; ++bb) {
        const int4 c = __ldcg(col + static_cast<long long>(bb) * E4);
        if (bb < b) before.x += c.x, before.y += c.y, before.z += c.z, before.w += c.w;
        total.x += c.x, total.y += c.y, total.z += c.z, total.w += c.w;
      }
      const int e = 4 * q;
      s_hist[e] = before.x, s_hist[e + 1] = before.y, s_hist[e + 2] = before.z, s_hist[e + 3] = before.w;
      s_off[e] = total.x, s_off[e + 1] = total.y, s_off[e + 2] = total.z, s_off[e + 3] = total.w;
      my_max = max(my_max, max(max(total.x, total.y), max(total.z, total.w)));
    }
  } else {
    for (int e = tid; e < E; e += kScanThreads) {
      int before = 0, total = 0;
#pragma unroll 8
      for (int bb = 0; bb < nb; ++bb) {
        const int c = __ldcg(block_counts + static_cast<long long>(bb) * E + e);
        before += (bb < b) ? c : 0;
        total += c;
      }
      s_hist[e] = before;
      s_off[e] = total;
      my_max = max(my_max, total);
    }
  }
  __syncthreads();
  // exclusive scan of s_off[0..E) in place (E <= 1024: 4 per thread)
  {
    const int per = (E + kScanThreads - 1) / kScanThreads;
    const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
    int local = 0;
    for (int e = e0; e < e1; ++e) local += s_off[e];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_red[warp] = incl;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, o));
    if (lane == 0) s_max[warp] = my_max;
    __syncthreads();
    int wbase = 0, total = 0, mx = 0;
    for (int w = 0; w < kScanWarps; ++w) {
      if (w < warp) wbase += s_red[w];
      total += s_red[w];
      mx = max(mx, s_max[w]);
    }
    int run = wbase + incl - local;
    __syncthreads();
    for (int e = e0; e < e1; ++e) {
      const int c = s_off[e];
      s_off[e] = run;
      run += c;
    }
    if (tid == 0) s_off[E] = total;
    __syncthreads();
    if (b == 0) {
      for (int e = tid; e <= E; e += kScanThreads) {
        offsets[e] = s_off[e];
        if (e < E) counts[e] = s_off[e + 1] - s_off[e];
      }
      const int epp = E / P;
      for (int p = tid; p <= P; p += kScanThreads) {
        part_offsets[p] = s_off[p * epp];
        if (p < P) part_counts[p] = s_off[(p + 1) * epp] - s_off[p * epp];
      }
      if (tid == 0 && skew) skew[0] = total > 0 ? static_cast<float>(mx) * static_cast<float>(E) / total : 0.0f;
    }
  }
  for (int e = tid; e < E; e += kScanThreads) s_hist[e] += s_off[e];
  __syncthreads();

  // phase 3
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += kScanThreads) {
    const int a = base + tid;
    int e = -1;
    if (a < hi) {
      e = __ldg(ids + a);
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(same) - 1;
    const int rank_in_warp = __popc(same & lt_mask);
    if (e >= 0 && lane == leader) s_wcnt[warp * E + e] = __popc(same);
    __syncthreads();
    if (a < hi && e < 0) row_of_assign[a] = -1;  // an invalid id gets no row
    if (e >= 0) {
      int r = s_hist[e] + rank_in_warp;
      for (int w = 0; w < warp; ++w) r += s_wcnt[w * E + e];
      row_of_assign[a] = r;
      assign_of_row[r] = a;
    }
    __syncthreads();
    if (e >= 0 && lane == leader) {
      atomicAdd(&s_hist[e], __popc(same));
      s_wcnt[warp * E + e] = 0;
    }
    __syncthreads();
  }
}

__global__ void skew_kernel(const int32_t* __restrict__ counts, int E, float* ratio) {
  __shared__ int s_max[32], s_sum[32];
  int mx = 0, sum = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = counts[e];
    mx = max(mx, c);
    sum += c;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = mx, s_sum[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    mx = 0, sum = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) mx = max(mx, s_max[w]), sum += s_sum[w];
    ratio[0] = sum > 0 ? static_cast<float>(mx) * static_cast<float>(E) / sum : 0.0f;
  }
}

size_t scan_smem_bytes(int E) { return static_cast<size_t>(E * 2 + 1 + kScanWarps * E) * sizeof(int); }

}  // namespace

cudaError_t launch_sum_partials(const float* partials, int nsplit, long long n, float* out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const long long blocks = std::min<long long>((n + 255) / 256, 8LL * num_sms());
  return launch_pdl(sum_partials_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, partials, nsplit, n,
                    out);
}

cudaError_t launch_route(const float* logits, int nsplit, float* logits_out, long long T, int E, int K, int renorm,
                         int P, int M, int32_t* ids,
                         float* w, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int vpl = (E + 31) / 32;
  if (vpl <= 1) return launch_route_vpl<1>(logits, nsplit, logits_out, T, E, K, renorm, P, M, ids, w, s);
  if (vpl <= 2) return launch_route_vpl<2>(logits, nsplit, logits_out, T, E, K, renorm, P, M, ids, w, s);
  if (vpl <= 4) return launch_route_vpl<4>(logits, nsplit, logits_out, T, E, K, renorm, P, M, ids, w, s);
  if (vpl <= 8) return launch_route_vpl<8>(logits, nsplit, logits_out, T, E, K, renorm, P, M, ids, w, s);
  if (vpl <= 16) return launch_route_vpl<16>(logits, nsplit, logits_out, T, E, K, renorm, P, M, ids, w, s);
  return launch_route_vpl<32>(logits, nsplit, logits_out, T, E, K, renorm, P, M, ids, w, s);
}

int scan_max_blocks(long long TK) {
  const long long b = (TK + kScanMinChunk - 1) / kScanMinChunk;
  return static_cast<int>(std::max<long long>(1, std::min<long long>(b, 1024)));
}

cudaError_t launch_count_scan(const int32_t* ids, long long TK, int E, int P, int32_t* counts, int32_t* offsets,
                              int32_t* part_counts, int32_t* part_offsets, int32_t* row_of_assign,
                              int32_t* assign_of_row, float* skew, const ScanWorkspace& ws, cudaStream_t s) {
  const size_t smem = scan_smem_bytes(E);
  static std::atomic<int> attr_done[kMaxDevices] = {};
  const cudaError_t attr = smem_attr_once(reinterpret_cast<const void*>(count_scan_kernel),
                                          static_cast<int>(scan_smem_bytes(MOE_MAX_E)), attr_done);
  if (attr != cudaSuccess) return attr;
  int occ = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, count_scan_kernel, kScanThreads, smem);
  if (err != cudaSuccess) return err;
  const long long resident = static_cast<long long>(std::max(occ, 1)) * num_sms();
  int blocks = static_cast<int>(std::min<long long>({static_cast<long long>(ws.max_blocks), resident,
                                                     std::max<long long>(1, (TK + kScanMinChunk - 1) / kScanMinChunk)}));
  blocks = std::max(blocks, 1);
  long long chunk = (TK + blocks - 1) / blocks;
  chunk = (chunk + kScanThreads - 1) / kScanThreads * kScanThreads;
  int TKi = static_cast<int>(TK), chunki = static_cast<int>(std::max<long long>(chunk, kScanThreads));
  int* block_counts = ws.block_counts;
  unsigned int* bc = ws.bar_count;
  unsigned int* bg = ws.bar_gen;
  int* status = ws.status;
  // Cooperative (the grid barrier needs every block resident) and programmatic: the blocks may
  // start while the route kernel drains and wait for it in griddepcontrol.wait.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(kScanThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr2[2];
  attr2[0].id = cudaLaunchAttributeCooperative;
  attr2[0].val.cooperative = 1;
  attr2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr2[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr2;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, count_scan_kernel, ids, TKi, E, P, chunki, counts, offsets, part_counts,
                            part_offsets, row_of_assign, assign_of_row, skew, block_counts, bc, bg, status);
}

cudaError_t launch_skew(const int32_t* counts, int E, float* ratio, cudaStream_t s) {
  skew_kernel<<<1, 256, 0, s>>>(counts, E, ratio);
  return cudaGetLastError();
}

}  // namespace moe
