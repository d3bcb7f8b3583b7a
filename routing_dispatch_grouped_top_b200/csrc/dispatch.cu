// dispatch.cu - permute (dispatch into expert-contiguous rows + routing
// metadata), combine (unpermute + weighted sum) and the one-time router split.
//
// The dispatcher gathers each destination's activations into one contiguous
// block with routing metadata per row, and the combine step returns every
// expert output to its token and sums them with the routing weights (WideEP
// essay, "The router writes a network schedule").  On one GPU no fabric is
// crossed, but the permute still moves T x K x H x b bytes through HBM and the
// combine about as many back (same essay: its regime table and "Top-k
// multiplies traffic").
//
// Both copy kernels are HBM-bound.  They work on 16-byte vectors (8 bf16): the
// item space is (token, vector) flattened, so consecutive threads touch
// consecutive 16-byte pieces of one row (coalesced on both sides), and each
// thread keeps several independent items in flight.
#include <cuda_fp8.h>

#include <algorithm>

#include "device.cuh"
#include "kernels.h"

namespace moe {

namespace {

#ifndef MOE_COPY_UNROLL
#define MOE_COPY_UNROLL 4
#endif
// Grid of the copy kernels: up to this many 256-thread blocks per SM.  Measured on B200 (Qwen3 /
// DeepSeek-R1 layers): 8 -> 16 raised permute from 74 to 80 % and combine from 79 to 84 % of the
// HBM copy bandwidth; 4, 32, and 2 or 8 loads in flight per thread were no better.
#ifndef MOE_COPY_BLOCKS_PER_SM
#define MOE_COPY_BLOCKS_PER_SM 16
#endif
#ifndef MOE_COMBINE_KC
#define MOE_COMBINE_KC 4
#endif
constexpr int kCopyThreads = 256;
constexpr int kUnroll = MOE_COPY_UNROLL;   // independent 16-byte loads in flight per thread

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Row of assignment a for the copy kernels: row_of_assign[a] as given, or, with rank_off
// (the layer path), count/scan's rank of a within its expert turned into rank_off[e] + rank and
// written back, with assign_of_row[row] = a.  Only the thread that owns a reads or writes
// row_of_assign[a].  -1 for an assignment without a valid row.
__device__ __forceinline__ int assignment_row(int32_t* roa, const int32_t* __restrict__ ids, long long a, long long TK,
                                             int E, const int32_t* __restrict__ rank_off, int32_t* aor) {
  int r = roa[a];
  if (rank_off) {
    const int e = __ldg(ids + a);
    int row = -1;
    if (r >= 0 && e >= 0 && e < E) {
      const long long v = static_cast<long long>(__ldg(rank_off + e)) + r;
      if (v >= 0 && v < TK) row = static_cast<int>(v);
    }
    roa[a] = row;
    if (row >= 0) aor[row] = static_cast<int>(a);
    r = row;
  }
  return (r >= 0 && r < TK) ? r : -1;
}

// One warp per token: lanes k < K find the rows of the token's K assignments (and write their
// metadata), then the warp copies the token's row of 16-byte vectors to those K rows, kUnroll
// loads in flight per lane; consecutive lanes touch consecutive vectors (coalesced both ways).
// Without xp (the gate/up GEMM gathers the rows itself) only the rows and metadata are made.
__global__ void __launch_bounds__(kCopyThreads) permute_kernel(
    const uint4* __restrict__ x, int32_t* roa, const int32_t* __restrict__ ids, const float* __restrict__ w,
    long long T, int vpr, int E, int K, int P, uint4* __restrict__ xp, int32_t* __restrict__ meta_token,
    int32_t* __restrict__ meta_slot, float* __restrict__ meta_w, int32_t* __restrict__ meta_local,
    const int32_t* __restrict__ rank_off, int32_t* __restrict__ aor) {
  pdl_wait();  // the ranks or rows come from the count/scan kernel
  pdl_launch_dependents();
  constexpr int kWarps = kCopyThreads / 32;
  const int lane = threadIdx.x & 31;
  const long long TK = T * K;
  const int epp = E / P;
  const long long nwarps = static_cast<long long>(gridDim.x) * kWarps;
  for (long long t = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5); t < T; t += nwarps) {
    const uint4* src = x + t * vpr;
    uint4 v[kUnroll];  // the first vectors are on their way while the rows are looked up
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (xp && lane + 32 * u < vpr) v[u] = ld_stream(src + lane + 32 * u);
    int row = -1;
    if (lane < K) {
      const long long a = t * K + lane;
      row = assignment_row(roa, ids, a, TK, E, rank_off, aor);
      if (row >= 0) {
        if (meta_token) meta_token[row] = static_cast<int>(t);
        if (meta_slot) meta_slot[row] = lane;
        if (meta_w) meta_w[row] = __ldg(w + a);
        if (meta_local) meta_local[row] = __ldg(ids + a) % epp;
      }
    }
    if (!xp) continue;
    for (int v0 = lane; v0 < vpr; v0 += 32 * kUnroll) {
      if (v0 != lane) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
          if (v0 + 32 * u < vpr) v[u] = ld_stream(src + v0 + 32 * u);
      }
      for (int k = 0; k < K; ++k) {
        const int rk = __shfl_sync(0xffffffffu, row, k);
        if (rk < 0) continue;
        uint4* dst = xp + static_cast<long long>(rk) * vpr + v0;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
          if (v0 + 32 * u < vpr) dst[32 * u] = v[u];
      }
    }
  }
}

template <int KC>
__global__ void __launch_bounds__(kCopyThreads) combine_kernel(const uint4* __restrict__ y,
                                                               const int32_t* __restrict__ roa,
                                                               const float* __restrict__ w,
                                                               const uint4* __restrict__ shared, long long T,
                                                               int vpr, int K, uint4* __restrict__ out) {
  pdl_wait();  // y comes from the down-projection GEMM
  pdl_launch_dependents();
  const long long n_items = T * vpr;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long it = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; it < n_items; it += stride) {
    const long long t = it / vpr;
    const int vec = static_cast<int>(it - t * vpr);
    const int32_t* r = roa + t * K;
    const float* wt = w + t * K;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
    if (shared) {  // shared expert output, weight 1
      const uint4 sv = ld_stream(shared + it);
      const __nv_bfloat162* ps = reinterpret_cast<const __nv_bfloat162*>(&sv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(ps[j]);
        acc[2 * j] = f.x;
        acc[2 * j + 1] = f.y;
      }
    }
    // slots in order; KC rows fetched before they are summed
    for (int k0 = 0; k0 < K; k0 += KC) {
      uint4 yv[KC];
      float wk[KC];
#pragma unroll
      for (int u = 0; u < KC; ++u) {
        yv[u] = make_uint4(0u, 0u, 0u, 0u);
        wk[u] = 0.0f;
        if (k0 + u < K) {
          const int row = __ldg(r + k0 + u);
          if (static_cast<unsigned long long>(row) < static_cast<unsigned long long>(T * K)) {
            yv[u] = ld_stream(y + static_cast<long long>(row) * vpr + vec);
            wk[u] = __ldg(wt + k0 + u);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < KC; ++u) {
        if (k0 + u < K) {
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&yv[u]);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p[j]);
            acc[2 * j] = fmaf(wk[u], f.x, acc[2 * j]);
            acc[2 * j + 1] = fmaf(wk[u], f.y, acc[2 * j + 1]);
          }
        }
      }
    }
    uint4 o;
    __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int j = 0; j < 4; ++j) po[j] = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
    out[it] = o;
  }
}

// W_g [H][E] fp32 -> [3][E][H] bf16 planes hi, mid, lo (hi = rn(w), mid = rn(w - hi),
// lo = rn(w - hi - mid); both differences are exact in fp32).
__global__ void pack_router_kernel(const float* __restrict__ w_g, int H, int E, __nv_bfloat16* __restrict__ out) {
  __shared__ float tile[32][33];
  const int h0 = blockIdx.y * 32, e0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int h = h0 + i, e = e0 + threadIdx.x;
    tile[i][threadIdx.x] = (h < H && e < E) ? w_g[static_cast<long long>(h) * E + e] : 0.0f;
  }
  __syncthreads();
  const long long plane = static_cast<long long>(E) * H;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int e = e0 + i, h = h0 + threadIdx.x;
    if (e < E && h < H) {
      const float v = tile[threadIdx.x][i];
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      const float r1 = v - __bfloat162float(hi);
      const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
      const float r2 = r1 - __bfloat162float(mid);
      const long long o = static_cast<long long>(e) * H + h;
      out[o] = hi;
      out[plane + o] = mid;
      out[2 * plane + o] = __float2bfloat16_rn(r2);
    }
  }
}

// ---------------------------------------------------------------------------
// FP8 (E4M3) rows with one fp32 scale per row.  Low-precision dispatch narrows each row sent
// to the experts and sends its scale with it (WideEP essay, "Top-k multiplies traffic.
// Locality subtracts it.").  s = amax / 448 (1 for an all-zero row), code = E4M3 of x / s
// (IEEE fp32 division, round to nearest even, saturating): both are decided in fp32.
// One block per row: the first pass reduces |x| to amax, the second (an L1/L2 hit)
// converts 8 values per 16-byte vector into one 8-byte store per destination row.
// ---------------------------------------------------------------------------
constexpr int kQuantThreads = 128;
constexpr float kE4M3Max = 448.0f;

__device__ __forceinline__ float block_max(float v, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float m = s_red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) m = fmaxf(m, s_red[w]);
  __syncthreads();  // s_red is reused by the next row
  return m;
}

__device__ __forceinline__ uint2 quantize8(const uint4 v, float s) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(p[j]);
    const uint32_t lo = __nv_cvt_float_to_fp8(__fdiv_rn(f.x, s), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float_to_fp8(__fdiv_rn(f.y, s), __NV_SATFINITE, __NV_E4M3);
    w[j >> 1] |= (lo | (hi << 8)) << (16 * (j & 1));
  }
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ float row_amax(const uint4* __restrict__ xr, int vpr) {
  float m = 0.0f;
  for (int v = threadIdx.x; v < vpr; v += kQuantThreads) {
    const uint4 u = xr[v];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(p[j]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  return m;
}

// Rows of x [rows][vpr * 8] -> q [rows][vpr * 8] codes, scales [rows].
__global__ void __launch_bounds__(kQuantThreads) quantize_fp8_rows_kernel(const uint4* __restrict__ x, long long rows,
                                                                           int vpr, uint2* __restrict__ q,
                                                                           float* __restrict__ scales) {
  __shared__ float s_red[kQuantThreads / 32];
  for (long long r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint4* xr = x + r * vpr;
    const float amax = block_max(row_amax(xr, vpr), s_red);
    const float s = amax > 0.0f ? __fdiv_rn(amax, kE4M3Max) : 1.0f;
    for (int v = threadIdx.x; v < vpr; v += kQuantThreads) q[r * vpr + v] = quantize8(xr[v], s);
    if (threadIdx.x == 0) scales[r] = s;
  }
}

// FP8 dispatch: token t quantized once, its codes and scale stored at the rows of its K
// assignments; routing metadata as in permute_kernel.
__global__ void __launch_bounds__(kQuantThreads) permute_fp8_kernel(
    const uint4* __restrict__ x, int32_t* roa, const int32_t* __restrict__ ids, const float* __restrict__ w,
    long long T, int vpr, int E, int K, int P, uint2* __restrict__ xq, float* __restrict__ xs,
    int32_t* __restrict__ meta_token, int32_t* __restrict__ meta_slot, float* __restrict__ meta_w,
    int32_t* __restrict__ meta_local, const int32_t* __restrict__ rank_off, int32_t* __restrict__ aor) {
  pdl_wait();  // row_of_assign comes from the count/scan kernel
  pdl_launch_dependents();
  __shared__ float s_red[kQuantThreads / 32];
  __shared__ int s_row[MOE_MAX_K];
  const long long TK = T * K;
  const int epp = E / P;
  for (long long t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < K) {
      const long long a = t * K + threadIdx.x;
      const int r = assignment_row(roa, ids, a, TK, E, rank_off, aor);
      const bool ok = r >= 0;
      s_row[threadIdx.x] = r;
      if (ok) {
        if (meta_token) meta_token[r] = static_cast<int>(t);
        if (meta_slot) meta_slot[r] = threadIdx.x;
        if (meta_w) meta_w[r] = __ldg(w + a);
        if (meta_local) meta_local[r] = __ldg(ids + a) % epp;
      }
    }
    const uint4* xr = x + t * vpr;
    const float amax = block_max(row_amax(xr, vpr), s_red);  // its barriers also publish s_row
    const float s = amax > 0.0f ? __fdiv_rn(amax, kE4M3Max) : 1.0f;
    if (threadIdx.x < K && s_row[threadIdx.x] >= 0) xs[s_row[threadIdx.x]] = s;
    for (int v = threadIdx.x; v < vpr; v += kQuantThreads) {
      const uint2 c = quantize8(xr[v], s);
      for (int k = 0; k < K; ++k) {
        const int r = s_row[k];
        if (r >= 0) xq[static_cast<long long>(r) * vpr + v] = c;
      }
    }
    __syncthreads();  // s_row is rewritten for the next token
  }
}

int copy_blocks(long long items) {
  const long long want = (items + kCopyThreads - 1) / kCopyThreads;
  return static_cast<int>(
      std::max<long long>(1, std::min<long long>(want, static_cast<long long>(MOE_COPY_BLOCKS_PER_SM) * num_sms())));
}

}  // namespace

cudaError_t launch_permute(const void* x, int32_t* roa, const int32_t* ids, const float* w, long long T, int H,
                           int E, int K, int P, void* xp, int32_t* meta_token, int32_t* meta_slot, float* meta_w,
                           int32_t* meta_local, const int32_t* rank_off, int32_t* aor, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int vpr = H / 8;
  const long long blocks = std::min<long long>((T + kCopyThreads / 32 - 1) / (kCopyThreads / 32),
                                               static_cast<long long>(MOE_COPY_BLOCKS_PER_SM) * num_sms());
  return launch_pdl(permute_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kCopyThreads), 0, s,
                    reinterpret_cast<const uint4*>(x), roa, ids, w, T, vpr, E, K, P, reinterpret_cast<uint4*>(xp),
                    meta_token, meta_slot, meta_w, meta_local, rank_off, aor);
}

cudaError_t launch_quantize_fp8_rows(const void* x, long long rows, int cols, void* q, float* scales,
                                     cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<long long>(rows, 16LL * num_sms()));
  quantize_fp8_rows_kernel<<<blocks, kQuantThreads, 0, s>>>(reinterpret_cast<const uint4*>(x), rows, cols / 8,
                                                            reinterpret_cast<uint2*>(q), scales);
  return cudaGetLastError();
}

cudaError_t launch_permute_fp8(const void* x, int32_t* roa, const int32_t* ids, const float* w, long long T,
                               int H, int E, int K, int P, void* xq, float* xs, int32_t* meta_token,
                               int32_t* meta_slot, float* meta_w, int32_t* meta_local, const int32_t* rank_off,
                               int32_t* aor, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<long long>(T, 16LL * num_sms()));
  return launch_pdl(permute_fp8_kernel, dim3(blocks), dim3(kQuantThreads), 0, s, reinterpret_cast<const uint4*>(x),
                    roa, ids, w, T, H / 8, E, K, P, reinterpret_cast<uint2*>(xq), xs, meta_token, meta_slot, meta_w,
                    meta_local, rank_off, aor);
}

cudaError_t launch_combine(const void* y, const int32_t* roa, const float* w, const void* shared, long long T, int H,
                           int K, void* out, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int vpr = H / 8;
  const int blocks = copy_blocks(T * vpr);
  if (K <= 2)
    return launch_pdl(combine_kernel<2>, dim3(blocks), dim3(kCopyThreads), 0, s, reinterpret_cast<const uint4*>(y),
                      roa, w, reinterpret_cast<const uint4*>(shared), T, vpr, K, reinterpret_cast<uint4*>(out));
  return launch_pdl(combine_kernel<MOE_COMBINE_KC>, dim3(blocks), dim3(kCopyThreads), 0, s,
                    reinterpret_cast<const uint4*>(y), roa, w, reinterpret_cast<const uint4*>(shared), T, vpr, K,
                    reinterpret_cast<uint4*>(out));
}

cudaError_t launch_pack_router(const float* w_g, int H, int E, void* w_split, cudaStream_t s) {
  dim3 grid((E + 31) / 32, (H + 31) / 32), block(32, 8);
  pack_router_kernel<<<grid, block, 0, s>>>(w_g, H, E, reinterpret_cast<__nv_bfloat16*>(w_split));
  return cudaGetLastError();
}

}  // namespace moe
