// routing.cu - router top-K, per-expert count + stable scan, skew statistics.
//
// The router keeps the K best-scoring experts of each token, and the dispatcher
// counts what every expert receives and reserves its rows (WideEP essay, "The
// router writes a network schedule").  Counts are per token-expert assignment
// and the skew statistic is the busiest expert's load over the mean load
// ("Three Parameter Counts...", "What the utilization dashboard smooths away").
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
// Count + scan + stable rank in one pass: block-local histograms and a decoupled look-back
// scan over the blocks.
//
// count_scan_kernel splits the assignments into nb chunks, one block per chunk, the chunk
// chosen by a ticket the block takes when it starts (so a block only waits for blocks that
// are already running):
//   1. block histogram of its chunk, kept per warp (warp w owns a contiguous slice);
//   2. the block publishes its per-expert counts (flag AGG) and looks back over its
//      predecessors: one warp reads 32 flags at a time, and the counts of the blocks up to
//      the nearest one that has published an inclusive prefix (flag INC) are added to that
//      prefix; then it publishes its own inclusive prefix (flag INC);
//   3. rank of assignment a (expert e) within its expert = the counts of e in earlier
//      blocks + in earlier warps of this block + the number of earlier assignments of e in
//      this warp (__match_any_sync): the stable order (increasing a) inside each expert.
//      The rank is written to row_of_assign[a]; the row is offsets[e] + rank;
//   4. the last block to finish takes the totals from the last chunk's inclusive prefix,
//      scans them into offsets (and counts, partitions, skew), then clears the flags and
//      rewinds the ticket and done counters for the next call.
// The offsets exist only once every block is done, so the ranks become rows afterwards:
// in the layer's permute (which reads them anyway), or in scan_finalize_kernel.  Every
// wait is bounded: a block that gives up sets MOE_DEV_TIMEOUT and ranks nothing, and a call
// that met an invalid id or a wait that ran out leaves offsets[E] = -1.
// ---------------------------------------------------------------------------

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kScanMinChunk = 1024;  // per block: 4 assignments per thread; short look-back chains
constexpr int kLookWindow = 32;
constexpr int kLookBatch = 8;  // look-back rows loaded together
constexpr int kIdBatch = 4;    // ids per lane loaded together
constexpr int kPerThreadE = MOE_MAX_E / kScanThreads;  // experts a thread scans and looks back for
constexpr int kFlagAgg = 1, kFlagInc = 2;

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Exclusive scan of vals[0..n) (n <= 1024) in shared memory by the whole block; returns the
// total and the maximum, out[n] = total.
__device__ void block_exclusive_scan(const int* vals, int n, int* out, int* s_red, int* s_max, int& total,
                                     int& mx) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + kScanThreads - 1) / kScanThreads;
  const int e0 = min(n, tid * per), e1 = min(n, e0 + per);
  int local = 0, my_max = 0;
  for (int e = e0; e < e1; ++e) {
    const int c = vals[e];
    local += c;
    my_max = max(my_max, c);
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, o));
  __syncthreads();  // vals may alias out
  if (lane == 31) s_red[warp] = incl;
  if (lane == 0) s_max[warp] = my_max;
  __syncthreads();
  int wbase = 0;
  total = 0, mx = 0;
  for (int w = 0; w < kScanWarps; ++w) {
    if (w < warp) wbase += s_red[w];
    total += s_red[w];
    mx = max(mx, s_max[w]);
  }
  int run = wbase + incl - local;
  int c_buf[kPerThreadE];
  for (int e = e0; e < e1; ++e) c_buf[e - e0] = vals[e];
  __syncthreads();
  for (int e = e0; e < e1; ++e) {
    out[e] = run;
    run += c_buf[e - e0];
  }
  if (tid == 0) out[n] = total;
  __syncthreads();
}

__global__ void __launch_bounds__(kScanThreads) count_scan_kernel(
    const int32_t* __restrict__ ids, int TK, int E, int P, int chunk, int nb, int32_t* __restrict__ rank_out,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ part_counts,
    int32_t* __restrict__ part_offsets, float* __restrict__ skew, const ScanWorkspace ws) {
  extern __shared__ int sm[];
  int* s_run = sm;                        // [kScanWarps][E] warp counts, then each warp's next rank
  int* s_agg = s_run + kScanWarps * E;    // [E] this block's counts; the last block: totals
  int* s_off = s_agg + E;                 // [E + 1] the last block: exclusive scan of the totals
  __shared__ int s_b, s_bad, s_ok, s_last, s_nwin, s_incpos, s_red[kScanWarps], s_max[kScanWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kScanWarps * E; i += kScanThreads) s_run[i] = 0;
  pdl_wait();  // the ids come from the previous kernel
  pdl_launch_dependents();
  if (tid == 0) {
    s_b = atomicAdd(ws.ticket, 1);
    s_bad = 0;
    s_ok = s_b < nb;  // a ticket beyond the grid: the previous call on this workspace did not finish
    if (!s_ok) report(ws.status, MOE_DEV_TIMEOUT);
  }
  __syncthreads();
  const int b = s_b;
  const bool active = s_ok;  // block-uniform
  const int lo = min(TK, b * chunk), hi = min(TK, lo + chunk);
  const int sub = ((chunk + kScanWarps - 1) / kScanWarps + 31) & ~31;
  const int wlo = min(hi, lo + warp * sub), whi = min(hi, wlo + sub);
  const unsigned lt_mask = (1u << lane) - 1u;
  int excl[kPerThreadE];
#pragma unroll
  for (int j = 0; j < kPerThreadE; ++j) excl[j] = 0;

  // a warp slice of at most 32 * kIdBatch ids is loaded once and kept for the ranking pass
  const bool keep = whi - wlo <= 32 * kIdBatch;
  int kept[kIdBatch];
#pragma unroll
  for (int u = 0; u < kIdBatch; ++u) kept[u] = -1;
  if (active) {
    // 1. counts of this warp's slice (kIdBatch ids per lane in flight at once)
    for (int base = wlo; base < whi; base += 32 * kIdBatch) {
      int ev[kIdBatch];
#pragma unroll
      for (int u = 0; u < kIdBatch; ++u) {
        const int a = base + 32 * u + lane;
        ev[u] = a < whi ? __ldg(ids + a) : -1;
        kept[u] = ev[u];
      }
#pragma unroll
      for (int u = 0; u < kIdBatch; ++u) {
        int e = ev[u];
        if (base + 32 * u + lane < whi && (e < 0 || e >= E)) s_bad = 1;
        if (e < 0 || e >= E) e = -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(same) - 1) s_run[warp * E + e] += __popc(same);
        __syncwarp();
      }
    }
    __syncthreads();
    // per expert: counts of the earlier warps of the block, and the block's count, published
    int* my_row = (b == 0 ? ws.inc : ws.agg) + static_cast<long long>(b) * E;
    for (int e = tid; e < E; e += kScanThreads) {
      int run = 0;
#pragma unroll
      for (int w = 0; w < kScanWarps; ++w) {
        const int c = s_run[w * E + e];
        s_run[w * E + e] = run;
        run += c;
      }
      s_agg[e] = run;
      __stcg(my_row + e, run);
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      st_release(ws.flags + b, b == 0 ? kFlagInc : kFlagAgg);
    }
    // 2. look back over the predecessors, kLookWindow blocks at a time
    int top = b - 1;
    while (top >= 0) {
      if (warp == 0) {
        const int p = top - lane;
        int f = 0;
        bool ok = true;
        if (p >= 0) {
          f = ld_acquire(ws.flags + p);
          if (f == 0) {
            const uint64_t t0 = global_timer_ns();
            unsigned int i = 0;
            while ((f = ld_acquire(ws.flags + p)) == 0) {
              if ((++i & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
                ok = false;
                break;
              }
            }
          }
        }
        const unsigned okm = __ballot_sync(0xffffffffu, ok);
        const unsigned incm = __ballot_sync(0xffffffffu, p >= 0 && f == kFlagInc);
        if (lane == 0) {
          if (okm != 0xffffffffu) {
            s_ok = 0;
            report(ws.status, MOE_DEV_TIMEOUT);
          }
          // lanes before the first INC carry counts (AGG); block 0 is INC, so a window that
          // reaches it always ends in an INC
          s_incpos = incm ? __ffs(incm) - 1 : -1;
          s_nwin = incm ? __ffs(incm) : min(kLookWindow, top + 1);
        }
      }
      __syncthreads();
      if (!s_ok) break;
      const int n = s_nwin, ip = s_incpos;
#pragma unroll
      for (int j = 0; j < kPerThreadE; ++j) {
        const int e = tid + j * kScanThreads;
        if (e < E) {
          // the window's rows in batches of independent loads (one round trip per batch)
          int acc = 0;
          for (int i0 = 0; i0 < n; i0 += kLookBatch) {
            int v[kLookBatch];
#pragma unroll
            for (int u = 0; u < kLookBatch; ++u) {
              const int i = i0 + u;
              v[u] = i < n ? __ldcg(((i == ip) ? ws.inc : ws.agg) + static_cast<long long>(top - i) * E + e) : 0;
            }
#pragma unroll
            for (int u = 0; u < kLookBatch; ++u) acc += v[u];
          }
          excl[j] += acc;
        }
      }
      if (ip >= 0) break;
      top -= kLookWindow;
      __syncthreads();  // s_nwin and s_incpos are rewritten
    }
    __syncthreads();
  }
  if (active && s_ok) {
    if (b > 0) {
      for (int j = 0; j < kPerThreadE; ++j) {
        const int e = tid + j * kScanThreads;
        if (e < E) __stcg(ws.inc + static_cast<long long>(b) * E + e, excl[j] + s_agg[e]);
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        st_release(ws.flags + b, kFlagInc);
      }
    }
    // 3. each warp's first rank per expert, then the ranks of its slice in order
#pragma unroll
    for (int j = 0; j < kPerThreadE; ++j) {
      const int e = tid + j * kScanThreads;
      if (e < E) {
#pragma unroll
        for (int w = 0; w < kScanWarps; ++w) s_run[w * E + e] += excl[j];
      }
    }
    __syncthreads();
    for (int base = wlo; base < whi; base += 32 * kIdBatch) {
      int ev[kIdBatch];
#pragma unroll
      for (int u = 0; u < kIdBatch; ++u) {
        const int a = base + 32 * u + lane;
        ev[u] = keep ? kept[u] : (a < whi ? __ldg(ids + a) : -1);
      }
#pragma unroll
      for (int u = 0; u < kIdBatch; ++u) {
        const int a = base + 32 * u + lane;
        const int e = (ev[u] < 0 || ev[u] >= E) ? -1 : ev[u];
        const unsigned same = __match_any_sync(0xffffffffu, e);
        if (a < whi) rank_out[a] = e < 0 ? -1 : s_run[warp * E + e] + __popc(same & lt_mask);  // -1: no row
        __syncwarp();
        if (e >= 0 && lane == __ffs(same) - 1) s_run[warp * E + e] += __popc(same);
        __syncwarp();
      }
    }
  }

  // 4. the last block writes the per-expert outputs and rewinds the workspace for the next call
  __syncthreads();
  if (tid == 0) {
    if (s_bad) report(ws.status, MOE_DEV_BAD_INDEX);
    if (s_bad || !s_ok) atomicOr(ws.fail, 1);
    __threadfence();
    s_last = atomicAdd(ws.done, 1) == nb - 1;
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    // totals: the inclusive prefix of the last chunk (every block published it before counting done)
    const int* totals = ws.inc + static_cast<long long>(nb - 1) * E;
    for (int e = tid; e < E; e += kScanThreads) s_agg[e] = TK > 0 ? __ldcg(totals + e) : 0;
    __syncthreads();
    int total = 0, mx = 0;
    block_exclusive_scan(s_agg, E, s_off, s_red, s_max, total, mx);
    const bool failed = *reinterpret_cast<volatile int*>(ws.fail) != 0;  // every block's flag is in
    for (int e = tid; e <= E; e += kScanThreads) {
      offsets[e] = (e == E && failed) ? -1 : s_off[e];
      if (e < E) counts[e] = s_off[e + 1] - s_off[e];
    }
    const int epp = E / P;
    for (int p = tid; p <= P; p += kScanThreads) {
      part_offsets[p] = s_off[p * epp];
      if (p < P) part_counts[p] = s_off[(p + 1) * epp] - s_off[p * epp];
    }
    if (tid == 0 && skew) skew[0] = total > 0 ? static_cast<float>(mx) * static_cast<float>(E) / total : 0.0f;
    for (int p = tid; p < kScanMaxBlocks; p += kScanThreads) ws.flags[p] = 0;
    __syncthreads();
    if (tid == 0) {
      *ws.fail = 0;
      *ws.ticket = 0;
      *ws.done = 0;
    }
  }
}

// row_of_assign[a] = offsets[ids[a]] + rank (in place), assign_of_row[row] = a.
__global__ void __launch_bounds__(kScanThreads) scan_finalize_kernel(const int32_t* __restrict__ ids, long long TK,
                                                                     int E, const int32_t* __restrict__ offsets,
                                                                     int32_t* __restrict__ row_of_assign,
                                                                     int32_t* __restrict__ assign_of_row) {
  pdl_wait();  // the ranks and offsets come from count_scan_kernel
  pdl_launch_dependents();
  for (long long a = static_cast<long long>(blockIdx.x) * kScanThreads + threadIdx.x; a < TK;
       a += static_cast<long long>(gridDim.x) * kScanThreads) {
    const int r = row_of_assign[a];
    const int e = __ldg(ids + a);
    int row = -1;
    if (r >= 0 && e >= 0 && e < E) {
      const long long v = static_cast<long long>(__ldg(offsets + e)) + r;
      if (v >= 0 && v < TK) row = static_cast<int>(v);
    }
    row_of_assign[a] = row;
    if (row >= 0) assign_of_row[row] = static_cast<int>(a);
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

size_t scan_smem_bytes(int E) { return static_cast<size_t>(kScanWarps * E + E + E + 1) * sizeof(int); }

}  // namespace

cudaError_t launch_sum_partials(const float* partials, int nsplit, long long n, float* out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const long long blocks = std::min<long long>((n + 255) / 256, 8LL * num_sms());
  return launch_pdl(sum_partials_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, partials, nsplit, n,
                    out);
}

cudaError_t launch_route(const float* logits, int nsplit, float* logits_out, long long T, int E, int K, int renorm,
                         int P, int M, int32_t* ids, float* w, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int vpl = (E + 31) / 32;
#define MOE_ROUTE(V) launch_route_vpl<V>(logits, nsplit, logits_out, T, E, K, renorm, P, M, ids, w, s)
  if (vpl <= 1) return MOE_ROUTE(1);
  if (vpl <= 2) return MOE_ROUTE(2);
  if (vpl <= 4) return MOE_ROUTE(4);
  if (vpl <= 8) return MOE_ROUTE(8);
  if (vpl <= 16) return MOE_ROUTE(16);
  return MOE_ROUTE(32);
#undef MOE_ROUTE
}

int scan_blocks(long long TK) {
  const long long b = (TK + kScanMinChunk - 1) / kScanMinChunk;
  return static_cast<int>(std::max<long long>(1, std::min<long long>(b, kScanMaxBlocks)));
}

size_t scan_ws_bytes(long long TK, int E) {
  const size_t rows = static_cast<size_t>(scan_blocks(TK)) * E * sizeof(int);
  return ScanWorkspace::kFixedBytes + 2 * round256(rows);
}

ScanWorkspace scan_workspace(void* base, long long TK, int E) {
  uint8_t* p = static_cast<uint8_t*>(base);
  ScanWorkspace w;
  w.status = reinterpret_cast<int*>(p);
  w.ticket = reinterpret_cast<int*>(p + 64);
  w.done = reinterpret_cast<int*>(p + 96);
  w.fail = reinterpret_cast<int*>(p + 128);
  w.flags = reinterpret_cast<int*>(p + 256);
  const size_t rows = round256(static_cast<size_t>(scan_blocks(TK)) * E * sizeof(int));
  w.agg = reinterpret_cast<int*>(p + ScanWorkspace::kFixedBytes);
  w.inc = reinterpret_cast<int*>(p + ScanWorkspace::kFixedBytes + rows);
  return w;
}

cudaError_t launch_count_scan(const int32_t* ids, long long TK, int E, int P, int32_t* ranks, int32_t* counts,
                              int32_t* offsets, int32_t* part_counts, int32_t* part_offsets, float* skew,
                              const ScanWorkspace& ws, cudaStream_t s) {
  static std::atomic<int> attr_done[kMaxDevices] = {};
  const cudaError_t attr = smem_attr_once(reinterpret_cast<const void*>(count_scan_kernel),
                                          static_cast<int>(scan_smem_bytes(MOE_MAX_E)), attr_done);
  if (attr != cudaSuccess) return attr;
  const int nb = scan_blocks(TK);
  const long long chunk = (TK + nb - 1) / nb;
  return launch_pdl(count_scan_kernel, dim3(nb), dim3(kScanThreads), scan_smem_bytes(E), s, ids,
                    static_cast<int>(TK), E, P, static_cast<int>(chunk), nb, ranks, counts, offsets, part_counts,
                    part_offsets, skew, ws);
}

cudaError_t launch_scan_finalize(const int32_t* ids, long long TK, int E, const int32_t* offsets,
                                 int32_t* row_of_assign, int32_t* assign_of_row, cudaStream_t s) {
  if (TK == 0) return cudaSuccess;
  const long long blocks = std::min<long long>((TK + kScanThreads - 1) / kScanThreads, 4LL * num_sms());
  return launch_pdl(scan_finalize_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kScanThreads), 0, s, ids, TK, E,
                    offsets, row_of_assign, assign_of_row);
}

cudaError_t launch_skew(const int32_t* counts, int E, float* ratio, cudaStream_t s) {
  skew_kernel<<<1, 256, 0, s>>>(counts, E, ratio);
  return cudaGetLastError();
}

}  // namespace moe
