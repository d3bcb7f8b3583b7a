// grouped_gemm.cu - persistent, warp-specialised tcgen05 GEMM over groups of
// rows with device-resident row offsets (the experts' matrix multiplies of a
// routed MoE layer), plus its dense single-group uses (gating, latent
// projections).
//
// "The receiver groups tokens by local expert and launches expert matrix
// multiplies" (WideEP essay, "The router writes a network schedule"); "Grouped
// GEMM ... runs several expert matrices in one launch and cuts launch overhead
// even when row counts differ" ("Three Parameter Counts...", "Which
// optimizations need a task-level gate").
//
// Orientation: the weight rows (output features) are the MMA's M side (128 per
// tile) and an expert's tokens are its N side (a multiple of 16, at most NT per
// tile), both K-major in shared memory.  A group of `cnt` rows is cut into
// ceil(cnt / NT) balanced chunks whose N is rounded up to 16, so a ragged
// expert wastes at most 15 token columns per chunk and an expert without rows
// costs nothing.  The instruction descriptor carries N, so it is chosen per
// tile at run time.
//
// Roles (192 threads, one CTA per SM, persistent over a static tile order):
//   warp 0      TMA producer: weight tile(s) 128 x 64 and token boxes 32 x 64,
//               128-byte swizzle, into a STAGES-deep ring of shared memory;
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer;
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator (each warp reads
//               the TMEM lane quadrant warp % 4), activation, masked stores.
// Accumulators are double-buffered in TMEM so the epilogue of tile i overlaps
// the main loop of tile i + 1.  Tiles are ordered group-major, then weight tile,
// then token chunk: CTAs working at the same time share weight and token tiles
// through L2, so each expert's weights cross HBM about once.
#include <algorithm>
#include <mutex>

#include "device.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kBM = 128;                  // output features per tile (MMA M)
constexpr int kBK = 64;                   // K per stage: one 128-byte swizzle atom of bf16
constexpr int kABytes = kBM * kBK * 2;    // 16 KB per weight tile
constexpr int kBoxB = 32;                 // token rows per TMA box of the B operand
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kMaxGroups = MOE_MAX_E;

template <int EPI>
struct Cfg;
// SwiGLU: gate and up tiles share one token tile; two accumulators per tile.
template <>
struct Cfg<kEpiSwiGLU> {
  static constexpr int NA = 2, NT = 128, STAGES = 4;
  static constexpr bool SEP = true;
};
// Plain bf16 output (down projection, latent projections).
template <>
struct Cfg<kEpiBF16> {
  static constexpr int NA = 1, NT = 256, STAGES = 4;
  static constexpr bool SEP = false;
};
// fp32 output: three bf16 weight planes accumulated into one fp32 accumulator.
template <>
struct Cfg<kEpiF32> {
  static constexpr int NA = 3, NT = 128, STAGES = 3;
  static constexpr bool SEP = false;
};

template <int EPI>
struct Layout {
  using C = Cfg<EPI>;
  static constexpr int kBBytes = C::NT * 128;
  static constexpr int kStageBytes = C::NA * kABytes + kBBytes;
  static constexpr int kAccCols = C::SEP ? C::NA * C::NT : C::NT;
  static constexpr uint32_t kTmemCols = 2 * kAccCols;
  static constexpr int kBarBytes = 8 * (2 * C::STAGES + 5) + 16;
  static constexpr int kTableBytes = 2 * (kMaxGroups + 1) * 4;
  static constexpr int kSmemBytes = 1024 + C::STAGES * kStageBytes + kBarBytes + kTableBytes;
  static_assert(kTmemCols == 256 || kTmemCols == 512, "TMEM allocation must be a power of two");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Tile {
  int g, n0, row0, nvalid, nround;
};

// Tile t -> (group, weight tile, token chunk).  s_pre[g] = first tile of group g.
__device__ __forceinline__ Tile decode_tile(int t, const int* s_pre, const int* s_off, int G, int NT) {
  int lo = 0, hi = G;  // s_pre[lo] <= t < s_pre[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_pre[mid] <= t) lo = mid;
    else hi = mid;
  }
  const int local = t - s_pre[lo];
  const int cnt = s_off[lo + 1] - s_off[lo];
  const int nch = (cnt + NT - 1) / NT;
  const int ft = local / nch;
  const int c = local - ft * nch;
  const int sz = (((cnt + nch - 1) / nch) + 15) & ~15;
  Tile r;
  r.g = lo;
  r.n0 = ft * kBM;
  r.row0 = s_off[lo] + c * sz;
  r.nvalid = min(sz, cnt - c * sz);
  r.nround = (r.nvalid + 15) & ~15;
  return r;
}

// s_pre[g] = sum_{g' < g} ceil(cnt_g' / NT) * NFT for g = 0..G (block-wide scan).
__device__ void build_tile_table(int* s_pre, const int* s_off, int G, int NT, int NFT, int* s_warp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seg = (G + kThreads - 1) / kThreads;
  const int b = min(G, tid * seg), e = min(G, b + seg);
  int local = 0;
  for (int g = b; g < e; ++g) local += ((s_off[g + 1] - s_off[g] + NT - 1) / NT) * NFT;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int w = 0; w < kThreads / 32; ++w) {
      const int v = s_warp[w];
      s_warp[w] = run;
      run += v;
    }
    s_pre[G] = run;
  }
  __syncthreads();
  int run = s_warp[warp] + incl - local;
  for (int g = b; g < e; ++g) {
    s_pre[g] = run;
    run += ((s_off[g + 1] - s_off[g] + NT - 1) / NT) * NFT;
  }
  __syncthreads();
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB,
                        const GemmArgs args) {
  using C = Cfg<EPI>;
  using L = Layout<EPI>;
  constexpr int NA = C::NA, NT = C::NT, STAGES = C::STAGES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * L::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_off = reinterpret_cast<int*>(smem + STAGES * L::kStageBytes + L::kBarBytes);
  int* s_pre = s_off + (kMaxGroups + 1);
  __shared__ int s_warp_sums[kThreads / 32];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = args.offsets ? args.G : 1;
  const int NFT = (args.N + kBM - 1) / kBM;
  const int KB = (args.Kd + kBK - 1) / kBK;

  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  for (int i = threadIdx.x; i <= G; i += kThreads)
    s_off[i] = args.offsets ? __ldg(args.offsets + i) : (i == 0 ? 0 : args.M);
  __syncthreads();
  // Offsets must be non-decreasing inside [0, M]; otherwise no tile runs.
  for (int i = threadIdx.x; i <= G; i += kThreads) {
    const bool bad = s_off[i] < 0 || s_off[i] > args.M || (i > 0 && s_off[i] < s_off[i - 1]);
    if (bad) s_bad = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0) report(args.status, MOE_DEV_BAD_INDEX);
    for (int i = threadIdx.x; i <= G; i += kThreads) s_off[i] = 0;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiThreads);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA0);
    tma_prefetch_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  build_tile_table(s_pre, s_off, G, NT, NFT, s_warp_sums);  // ends with __syncthreads
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pre[G];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t pend_phase[STAGES];
      bool pend[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) pend[s] = false, pend_phase[s] = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        const Tile tl = decode_tile(t, s_pre, s_off, G, NT);
        const int nbox = (tl.nround + kBoxB - 1) / kBoxB;
        const uint32_t bytes = NA * kABytes + nbox * kBoxB * 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          uint8_t* st = ring + stage * L::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], bytes);
          const int kx = kb * kBK;
#pragma unroll
          for (int i = 0; i < NA; ++i) {
            const CUtensorMap* m = (i == 0) ? &tmA0 : ((i == 1) ? &tmA1 : &tmA2);
            const int z = (EPI == kEpiF32) ? i : tl.g;
            tma_load_3d(st + i * kABytes, m, &full[stage], kx, tl.n0, z);
          }
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(st + NA * kABytes + b * kBoxB * 128, &tmB, &full[stage], kx, tl.row0 + b * kBoxB);
          pend[stage] = true;
          pend_phase[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
#pragma unroll
        for (int s = 0; s < STAGES; ++s)
          if (pend[s]) mbar_drain(&full[s], pend_phase[s], 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        const Tile tl = decode_tile(t, s_pre, s_off, G, NT);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, args.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(kBM, tl.nround);
        const uint32_t d0 = tmem_base + acc * L::kAccCols;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * L::kStageBytes);
          const uint32_t sb = sa + NA * kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bdesc = sw128_kmajor_desc(sb + kk * 32);
#pragma unroll
            for (int i = 0; i < NA; ++i) {
              const uint64_t adesc = sw128_kmajor_desc(sa + i * kABytes + kk * 32);
              const uint32_t d = d0 + (C::SEP ? i * NT : 0);
              const uint32_t accumulate = (kb > 0 || kk > 0 || (!C::SEP && i > 0)) ? 1u : 0u;
              umma_bf16(d, adesc, bdesc, idesc, accumulate);
            }
          }
          umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {  // wait for the MMAs already issued before TMEM is released
        umma_commit(drain);
        mbar_drain(drain, 0, 200000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lanes [32q, 32q + 32) are visible to this warp
    uint32_t acc = 0, acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile tl = decode_tile(t, s_pre, s_off, G, NT);
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, args.status)) break;
      tc_fence_after();
      const int f = tl.n0 + q * 32 + lane;
      const bool f_ok = f < args.N;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * L::kAccCols;
      for (int j0 = 0; j0 < tl.nvalid; j0 += 32) {
        uint32_t r0[32];
        tmem_ld_32cols(tbase + j0, r0);
        const int jn = min(32, tl.nvalid - j0);
        const long long row0 = static_cast<long long>(tl.row0) + j0;
        if constexpr (EPI == kEpiSwiGLU) {
          uint32_t r1[32];
          tmem_ld_32cols(tbase + NT + j0, r1);
          tmem_wait_ld();
          __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(args.out);
          if (f_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < jn) {
                const float g = __uint_as_float(r0[j]);
                const float u = __uint_as_float(r1[j]);
                const float h = g / (1.0f + __expf(-g)) * u;
                out[(row0 + j) * args.ldo + f] = __float2bfloat16_rn(h);
              }
            }
          }
        } else if constexpr (EPI == kEpiBF16) {
          tmem_wait_ld();
          __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(args.out);
          if (f_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < jn) out[(row0 + j) * args.ldo + f] = __float2bfloat16_rn(__uint_as_float(r0[j]));
          }
        } else {
          tmem_wait_ld();
          float* out = reinterpret_cast<float*>(args.out);
          if (f_ok) {
            const float b = args.bias ? __ldg(args.bias + f) : 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < jn) out[(row0 + j) * args.ldo + f] = __uint_as_float(r0[j]) + b;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor [d2][d1][d0] (d0 contiguous), box {64, box1, 1}, 128-byte swizzle.
bool map_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kBK), box1, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_bf16_2d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint32_t box1) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {d0 * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box1};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI>
cudaError_t launch(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2, const CUtensorMap& b,
                   const GemmArgs& args, long long tile_bound, cudaStream_t stream) {
  using L = Layout<EPI>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(grouped_gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  if (tile_bound <= 0) return cudaSuccess;
  const int grid = static_cast<int>(std::min<long long>(num_sms(), tile_bound));
  grouped_gemm_kernel<EPI><<<grid, kThreads, L::kSmemBytes, stream>>>(a0, a1, a2, b, args);
  return cudaGetLastError();
}

long long tile_bound(long long rows, int groups, int NT, int N) {
  const long long nft = (N + kBM - 1) / kBM;
  return ((rows + NT - 1) / NT + (groups > 1 ? groups : 0)) * nft;
}

}  // namespace

int gemm_smem_bytes(int epi) {
  switch (epi) {
    case kEpiSwiGLU: return Layout<kEpiSwiGLU>::kSmemBytes;
    case kEpiBF16: return Layout<kEpiBF16>::kSmemBytes;
    default: return Layout<kEpiF32>::kSmemBytes;
  }
}

// h = silu(xp Wg^T) * (xp Wu^T) per expert group.
cudaError_t gemm_gate_up(const void* xp, const int32_t* offsets, const void* w_gate, const void* w_up, int E,
                         long long rows, int H, int F, void* h, int* status, cudaStream_t stream) {
  CUtensorMap a0, a1, b;
  if (!map_bf16_3d(&a0, w_gate, H, F, E, kBM) || !map_bf16_3d(&a1, w_up, H, F, E, kBM) ||
      !map_bf16_2d(&b, xp, H, rows, kBoxB))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, E, static_cast<int>(rows), F, H, h, F, nullptr, status};
  return launch<kEpiSwiGLU>(a0, a1, a1, b, args, tile_bound(rows, E, Cfg<kEpiSwiGLU>::NT, F), stream);
}

// y = h Wd^T per expert group.
cudaError_t gemm_down(const void* h, const int32_t* offsets, const void* w_down, int E, long long rows, int H,
                      int F, void* y, int* status, cudaStream_t stream) {
  CUtensorMap a0, b;
  if (!map_bf16_3d(&a0, w_down, F, H, E, kBM) || !map_bf16_2d(&b, h, F, rows, kBoxB))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, E, static_cast<int>(rows), H, F, y, H, nullptr, status};
  return launch<kEpiBF16>(a0, a0, a0, b, args, tile_bound(rows, E, Cfg<kEpiBF16>::NT, H), stream);
}

// out[M][N] = a[M][Kd] w[N][Kd]^T, bf16 out.
cudaError_t gemm_dense(const void* a, const void* w, long long M, int N, int Kd, void* out, int* status,
                       cudaStream_t stream) {
  CUtensorMap a0, b;
  if (!map_bf16_3d(&a0, w, Kd, N, 1, kBM) || !map_bf16_2d(&b, a, Kd, M, kBoxB)) return cudaErrorInvalidValue;
  GemmArgs args{nullptr, 1, static_cast<int>(M), N, Kd, out, N, nullptr, status};
  return launch<kEpiBF16>(a0, a0, a0, b, args, tile_bound(M, 1, Cfg<kEpiBF16>::NT, N), stream);
}

// logits[T][E] = x[T][H] (hi + mid + lo)^T (+ bias), fp32 out; w_split is [3][E][H] bf16.
cudaError_t gemm_gating(const void* x, const void* w_split, const float* bias, long long T, int H, int E,
                        float* logits, int* status, cudaStream_t stream) {
  CUtensorMap a0, b;
  if (!map_bf16_3d(&a0, w_split, H, E, 3, kBM) || !map_bf16_2d(&b, x, H, T, kBoxB)) return cudaErrorInvalidValue;
  GemmArgs args{nullptr, 1, static_cast<int>(T), E, H, logits, E, bias, status};
  return launch<kEpiF32>(a0, a0, a0, b, args, tile_bound(T, 1, Cfg<kEpiF32>::NT, E), stream);
}

}  // namespace moe
