// grouped_gemm.cu - persistent, warp-specialised tcgen05 GEMM over groups of
// rows with device-resident row offsets (the experts' matrix multiplies of a
// routed MoE layer), plus its dense single-group uses (gating, latent
// projections).
//
// Each expert multiplies the rows routed to it (WideEP essay, "The router
// writes a network schedule"); a grouped GEMM serves all experts in a single
// launch whatever their row counts, without changing those counts ("Three
// Parameter Counts...", "Which optimizations need a task-level gate").
//
// Orientation: the weight rows (output features) are the MMA's M side (128 per
// tile) and an expert's tokens are its N side (a multiple of 16, at most NT per
// tile), both K-major in shared memory.  A group of `cnt` rows is cut into
// ceil(cnt / NT) balanced chunks whose N is rounded up to 16, so a ragged
// expert wastes at most 15 token columns per chunk and an expert without rows
// costs nothing.  The instruction descriptor carries N, so it is chosen per
// tile at run time.
//
// Roles (persistent, one CTA per SM; two kernels, single-CTA and CTA-pair):
//   warp 0      TMA producer: claims the next tile of the launch from a counter in
//               the workspace (the last CTA rewinds it), publishes its id through a
//               ring of tile ids in shared memory, and streams weight boxes of 128 or
//               256 rows and token boxes of 8..256 rows (128-byte swizzle) into a
//               STAGES-deep ring of shared memory;
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer;
//   warps 2..   epilogue: tcgen05.ld of the fp32 accumulator (warp w reads the TMEM
//               lane quadrant w % 4; with eight warps two share a quadrant and take
//               alternate 32-token chunks), activation, and bf16 rows written through a
//               per-warp shared-memory transpose as 16-byte pieces (the pair kernel's bf16
//               epilogue stores each full 32 x 32 chunk with one TMA tile store instead);
//   (pair, SwiGLU) four gather warps, one per stage, that copy the token rows with 16-byte
//               cp.async through the rows' source indices when the operand is gathered in
//               place instead of read from a permuted copy.
// Tiles are numbered group-major, then weight tile, then token chunk, and claimed in
// that order: CTAs working at the same time share weight and token tiles through L2,
// so each expert's weights cross HBM about once, and SMs that draw short tiles take
// more of them.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "device.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kBM = 128;                  // output features per tile (MMA M)
constexpr int kBK = 64;                   // K per stage: one 128-byte swizzle atom of bf16
constexpr int kABytes = kBM * kBK * 2;    // 16 KB per weight tile
// The token operand of a tile (nround rows, a multiple of 16) is fetched with one TMA box
// per set bit of nround: boxes of 256, 128, 64, 32 and 16 rows (single CTA), or of 128 down to 8
// rows for each CTA's half of a CTA-pair tile.
constexpr int kNumBoxes = 6;
struct BoxMaps {
  CUtensorMap box[kNumBoxes];  // box[i] is (256 >> i) rows x 64 columns
};
constexpr int kMaxThreads = 320;         // single-CTA kernel with 8 epilogue warps
constexpr int kMaxPairThreads = 448;     // CTA-pair kernel with 8 epilogue and 4 gather warps
constexpr int kMaxGroups = MOE_MAX_E;
constexpr int kRing = 8;                 // tile ids in flight from the producer to the MMA and epilogue warps

template <int EPI>
struct Cfg;
// SwiGLU: gate and up tiles share one token tile; two accumulators per tile.
// NA weight tiles of 128 rows per stage share one token tile of NT rows.  SEP: each
// weight tile has its own accumulator (SwiGLU: gate and up; wide bf16 tiles: rows
// 0-127 and 128-255 of the output features); otherwise all accumulate into one.
// FEAT output features per tile.  Accumulators are double-buffered in TMEM when two fit
// in its 512 columns (the epilogue of one tile then overlaps the next tile's main loop).
//
// Measured on B200: the MMA itself runs at its full rate (128 cycles per 128 x 256 x 16
// bf16 MMA, with a commit every 8), and the shared-memory fill per MMA cycle is what these
// kernels trade against the TMEM budget: 256-token tiles (two 128-row weight tiles and a
// 256-row token tile per stage, single-buffered accumulators) beat 128-token tiles with
// double-buffered accumulators on every layer workload once the epilogue stores were
// vectorised (Qwen3 gate/up 253 -> 214 us).
// Build-time tuning: token columns of the separate-weight SwiGLU tiles (128: double-buffered
// accumulators, 4 stages; 256: single-buffered, 3 stages) and epilogue warps (4 or 8: two
// warps per TMEM lane quadrant split a tile's token chunks).
#ifndef MOE_SWIGLU_NT
#define MOE_SWIGLU_NT 256
#endif
#ifndef MOE_EPI_WARPS
#define MOE_EPI_WARPS 8
#endif
template <>
struct Cfg<kEpiSwiGLU> {
  static constexpr int NA = 2, NT = MOE_SWIGLU_NT, STAGES = NT == 256 ? 3 : 4, FEAT = 128, EW = MOE_EPI_WARPS;
  static constexpr bool SEP = true;
};
// SwiGLU on E4M3 operands (FP8 dispatch): the same tile as the bf16 SwiGLU, each stage
// carrying 128 K-elements (one 128-byte swizzle atom of 8-bit codes) instead of 64, so a
// stage holds twice the MMA work.
template <>
struct Cfg<kEpiSwiGLUFp8> {
  static constexpr int NA = 2, NT = MOE_SWIGLU_NT, STAGES = NT == 256 ? 3 : 4, FEAT = 128, EW = MOE_EPI_WARPS;
  static constexpr bool SEP = true;
};
// Plain bf16 output (down projection, latent projections).
#ifndef MOE_BF16_NT
#define MOE_BF16_NT 256
#endif
template <>
struct Cfg<kEpiBF16> {
  static constexpr int NA = 2, NT = MOE_BF16_NT, STAGES = NT == 256 ? 3 : 4, FEAT = 256, EW = MOE_EPI_WARPS;
  static constexpr bool SEP = true;
};
// fp32 output: three bf16 weight planes accumulated into one fp32 accumulator.
template <>
struct Cfg<kEpiF32> {
  static constexpr int NA = 3, NT = 128, STAGES = 3, FEAT = 128, EW = 4;
  static constexpr bool SEP = false;
};

template <int EPI>
struct Layout {
  using C = Cfg<EPI>;
  static constexpr int kThr = 64 + 32 * C::EW;  // producer warp, MMA warp, epilogue warps
  static_assert(C::EW == 4 || C::EW == 8, "one or two epilogue warps per TMEM lane quadrant");
  static_assert(kThr <= kMaxThreads, "block size");
  static constexpr int kBBytes = C::NT * 128;
  static constexpr int kStageBytes = C::NA * kABytes + kBBytes;
  static constexpr int kAccCols = C::SEP ? C::NA * C::NT : C::NT;
  static constexpr int kNumAcc = (2 * kAccCols <= 512) ? 2 : 1;
  static constexpr uint32_t kTmemCols = kNumAcc * kAccCols;
  // bf16 outputs: one 32 x 32 transpose tile per epilogue warp
  static constexpr int kExchBytes = EPI == kEpiF32 ? 0 : C::EW * 32 * 32 * 2;
  // barriers: full/empty per stage, tmem full/empty x2, drain, tile ring full/empty; then the
  // TMEM address, the abort flag and the ring's tile ids
  static constexpr int kBarBytes = (8 * (2 * C::STAGES + 5 + 2 * kRing) + 8 + 4 * kRing + 15) / 16 * 16;
  static constexpr int kTableBytes = 2 * (kMaxGroups + 1) * 4;
  static constexpr int kSmemBytes = 1024 + C::STAGES * kStageBytes + kExchBytes + kBarBytes + kTableBytes;
  static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512, "TMEM allocation must be a power of two");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Tile {
  int g, n0, row0, nvalid, nround;
};

// K elements per stage: one 128-byte swizzle atom per operand row.
template <int EPI>
constexpr int stage_k() {
  return EPI == kEpiSwiGLUFp8 ? 128 : kBK;
}

// silu(g) * u = g u / (1 + e^-g) with the fast exponential and divide (2 MUFU ops):
// for g -> -inf the denominator overflows and the result is 0, for g -> +inf it is g u.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g * u, 1.0f + __expf(-g)); }

// bf16 outputs leave through a per-warp 32 x 32 transpose in shared memory: the thread of
// feature fbase + lane holds v[j] for tokens row0 + j, a token row wants 32 consecutive
// features, so each lane then writes whole 16-byte pieces of rows (four per 32-token chunk)
// instead of 32 scattered 2-byte values.  Rows j >= jn and features >= N are not written.
__device__ __forceinline__ void store_rows32(__nv_bfloat16* stg, int lane, const float (&v)[32],
                                             __nv_bfloat16* out, long long ldo, int N, int fbase, long long row0,
                                             int jn) {
#pragma unroll
  for (int j = 0; j < 32; ++j) stg[j * 32 + lane] = __float2bfloat16_rn(v[j]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = 8 * i + (lane >> 2), c = 8 * (lane & 3);
    if (j < jn && fbase + c < N)
      *reinterpret_cast<uint4*>(out + (row0 + j) * ldo + fbase + c) = *reinterpret_cast<const uint4*>(stg + j * 32 + c);
  }
  __syncwarp();
}

// store_rows32 through a TMA tile store: the 32 x 32 chunk (tokens x features) is staged as 32
// rows of 64 bytes and one lane stores it as one box of `map` (the output, box 32 x 32, no
// swizzle), which completes in the background: the warp goes on (and hands TMEM back) while the
// rows drain.  A chunk with fewer than 32 valid rows takes store_rows32's 16-byte stores, since
// the box would also write the first rows of the next group.  The staging tile is reused only
// after the previous chunk's store has read it.
__device__ __forceinline__ void store_rows32_tma(__nv_bfloat16* stg, int lane, const float (&v)[32],
                                                 const CUtensorMap* map, __nv_bfloat16* out, long long ldo, int N,
                                                 int fbase, long long row0, int jn) {
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
  if (jn < 32) {
    store_rows32(stg, lane, v, out, ldo, N, fbase, row0, jn);
    return;
  }
  if (fbase >= N) return;
#pragma unroll
  for (int j = 0; j < 32; ++j) stg[j * 32 + lane] = __float2bfloat16_rn(v[j]);
  fence_proxy_async_shared();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, stg, fbase, static_cast<int>(row0));
    bulk_commit_group();
  }
}

// Tile t -> (group, weight tile, token chunk).  s_pre[g] = first tile of group g.  A group of
// cnt rows is cut into ceil(cnt / NT) balanced chunks of a multiple of ROUND rows; a weight
// tile covers FEAT output features.
template <int NT, int ROUND, int FEAT>
__device__ __forceinline__ Tile decode_tile(int t, const int* s_pre, const int* s_off, int G) {
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
  const int sz = (((cnt + nch - 1) / nch) + ROUND - 1) & ~(ROUND - 1);
  Tile r;
  r.g = lo;
  r.n0 = ft * FEAT;
  r.row0 = s_off[lo] + c * sz;
  r.nvalid = min(sz, cnt - c * sz);
  r.nround = (r.nvalid + ROUND - 1) & ~(ROUND - 1);
  return r;
}

// s_pre[g] = sum_{g' < g} ceil(cnt_g' / NT) * NFT for g = 0..G (block-wide scan).
__device__ void build_tile_table(int* s_pre, const int* s_off, int G, int NT, int NFT, int* s_warp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = blockDim.x;
  const int seg = (G + nthreads - 1) / nthreads;
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
    for (int w = 0; w < nthreads / 32; ++w) {
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

// Source row of token operand row r when the operand is gathered in place (GemmArgs::gather).
// An entry that names no source row is reported (bad index) and row 0 is read instead.
__device__ __forceinline__ int gather_source(const GemmArgs& args, int r) {
  const int a = __ldg(args.gather + r);
  const int src = a >= 0 ? a / args.gather_div : -1;
  if (static_cast<unsigned>(src) >= static_cast<unsigned>(args.gather_rows)) {
    report(args.status, MOE_DEV_BAD_INDEX);
    return 0;
  }
  return src;
}

template <int EPI>
__global__ void __launch_bounds__(kMaxThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ BoxMaps tmB,
                        const GemmArgs args) {
  using C = Cfg<EPI>;
  using L = Layout<EPI>;
  constexpr int NA = C::NA, NT = C::NT, STAGES = C::STAGES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* exch = reinterpret_cast<float*>(smem + STAGES * L::kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * L::kStageBytes + L::kExchBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* rfull = drain + 1;       // tile ring: the producer publishes each tile id it takes
  uint64_t* rempty = rfull + kRing;  // released by the MMA thread and every epilogue warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rempty + kRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring_tile = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(smem + STAGES * L::kStageBytes + L::kExchBytes + L::kBarBytes);
  int* s_pre = s_off + (kMaxGroups + 1);
  __shared__ int s_warp_sums[kMaxThreads / 32];
  (void)exch;
  constexpr int kEpiThr = 32 * C::EW;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = args.offsets ? args.G : 1;
  const int NFT = (args.N + C::FEAT - 1) / C::FEAT;
  constexpr int KS = stage_k<EPI>();
  const int KB = (args.Kd + KS - 1) / KS;

  // Set-up that reads no global input runs before the wait on the previous kernel.
  __shared__ int s_bad;
  if (threadIdx.x == 0) {
    s_bad = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiThr);
    }
    mbar_init(drain, 1);
    for (int r = 0; r < kRing; ++r) {
      mbar_init(&rfull[r], 1);
      mbar_init(&rempty[r], 1 + C::EW);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA0);
    for (int i = 0; i < kNumBoxes; ++i) tma_prefetch_map(&tmB.box[i]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  pdl_wait();  // offsets and the token operand come from earlier kernels
  pdl_launch_dependents();
  __syncthreads();
  for (int i = threadIdx.x; i <= G; i += L::kThr)
    s_off[i] = args.offsets ? __ldg(args.offsets + i) : (i == 0 ? 0 : args.M);
  __syncthreads();
  // Offsets must be non-decreasing inside [0, M]; otherwise no tile runs.
  for (int i = threadIdx.x; i <= G; i += L::kThr) {
    const bool bad = s_off[i] < 0 || s_off[i] > args.M || (i > 0 && s_off[i] < s_off[i - 1]);
    if (bad) s_bad = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0) report(args.status, MOE_DEV_BAD_INDEX);
    for (int i = threadIdx.x; i <= G; i += L::kThr) s_off[i] = 0;
  }
  __syncthreads();
  build_tile_table(s_pre, s_off, G, NT, NFT, s_warp_sums);  // ends with __syncthreads
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Split reduction (fp32 gating only): tile t covers output tile t / S and K-steps
  // [ks KB / S, (ks + 1) KB / S) of split ks = t % S; the host keeps S <= KB.
  const int S = (EPI == kEpiF32 && args.ksplit > 1) ? args.ksplit : 1;
  const int total = s_pre[G] * S;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t pend_phase[STAGES];
      bool pend[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) pend[s] = false, pend_phase[s] = 0;
      bool ok = true;
      uint32_t rs = 0, rphase = 0;
      for (;;) {
        // Dynamic schedule: the next unclaimed tile of the launch (tiles differ in their token
        // count, so a fixed round-robin leaves some SMs with much more work than others).
        if (!mbar_wait(&rempty[rs], rphase ^ 1u, abort_flag, args.status)) {
          ok = false;
          break;
        }
        const int t = atomicAdd(&args.sched[0], 1);
        ring_tile[rs] = t < total ? t : -1;
        mbar_arrive(&rfull[rs]);
        if (++rs == kRing) {
          rs = 0;
          rphase ^= 1u;
        }
        if (t >= total) break;
        const int tb = t / S, ks = t - tb * S;
        const Tile tl = decode_tile<NT, 16, C::FEAT>(tb, s_pre, s_off, G);
        const uint32_t bytes = NA * kABytes + tl.nround * 128;
        for (int kb = ks * KB / S; kb < (ks + 1) * KB / S; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          uint8_t* st = ring + stage * L::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], bytes);
          const int kx = kb * KS;
          if constexpr (EPI == kEpiBF16) {
            // both 128-row weight tiles in one 256-row box
            tma_load_3d(st, &tmA0, &full[stage], kx, tl.n0, tl.g);
          } else {
#pragma unroll
            for (int i = 0; i < NA; ++i) {
              const CUtensorMap* m = (i == 0) ? &tmA0 : ((i == 1) ? &tmA1 : &tmA2);
              tma_load_3d(st + i * kABytes, m, &full[stage], kx, tl.n0, (EPI == kEpiF32) ? i : tl.g);
            }
          }
          int r = 0;
#pragma unroll
          for (int i = 0; i < kNumBoxes; ++i) {
            const int rows = 256 >> i;
            if (tl.nround & rows) {
              tma_load_2d(st + NA * kABytes + r * 128, &tmB.box[i], &full[stage], kx, tl.row0 + r);
              r += rows;
            }
          }
          pend[stage] = true;
          pend_phase[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
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
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0, rs = 0, rphase = 0;
      bool ok = true;
      for (;;) {
        if (!mbar_wait(&rfull[rs], rphase, abort_flag, args.status)) {
          ok = false;
          break;
        }
        const int t = ring_tile[rs];
        mbar_arrive(&rempty[rs]);
        if (++rs == kRing) {
          rs = 0;
          rphase ^= 1u;
        }
        if (t < 0) break;
        const int tb = t / S, ks = t - tb * S;
        const int kb_lo = ks * KB / S, kb_hi = (ks + 1) * KB / S;
        const Tile tl = decode_tile<NT, 16, C::FEAT>(tb, s_pre, s_off, G);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, args.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc =
            (EPI == kEpiSwiGLUFp8) ? idesc_e4m3_f32(kBM, tl.nround) : idesc_bf16_f32(kBM, tl.nround);
        const uint32_t d0 = tmem_base + acc * L::kAccCols;
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * L::kStageBytes);
          const uint32_t sb = sa + NA * kABytes;
          // four MMAs per 128-byte atom: K = 16 bf16 or 32 E4M3 elements (32 bytes) each
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = sw128_kmajor_desc(sb + kk * 32);
#pragma unroll
            for (int i = 0; i < NA; ++i) {
              const uint64_t adesc = sw128_kmajor_desc(sa + i * kABytes + kk * 32);
              const uint32_t d = d0 + (C::SEP ? i * NT : 0);
              const uint32_t accumulate = (kb > kb_lo || kk > 0 || (!C::SEP && i > 0)) ? 1u : 0u;
              if constexpr (EPI == kEpiSwiGLUFp8) umma_e4m3(d, adesc, bdesc, idesc, accumulate);
              else umma_bf16(d, adesc, bdesc, idesc, accumulate);
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
        if (++acc == L::kNumAcc) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {  // wait for the MMAs already issued before TMEM is released
        umma_commit(drain);
        mbar_drain(drain, 0, 200000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lanes [32q, 32q + 32) are visible to this warp
    // With 8 epilogue warps, two share each lane quadrant and take alternate 32-token chunks.
    constexpr int kSplit = C::EW / 4;
    const int part = (warp - 2) >> 2;
    uint32_t acc = 0, acc_phase = 0, rs = 0, rphase = 0;
    for (;;) {
      if (!mbar_wait(&rfull[rs], rphase, abort_flag, args.status)) break;
      const int t = ring_tile[rs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&rempty[rs]);
      if (++rs == kRing) {
        rs = 0;
        rphase ^= 1u;
      }
      if (t < 0) break;
      const int tb = t / S, ks = t - tb * S;
      const Tile tl = decode_tile<NT, 16, C::FEAT>(tb, s_pre, s_off, G);
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, args.status)) break;
      tc_fence_after();
      const int f = tl.n0 + q * 32 + lane;
      const bool f_ok = f < args.N;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * L::kAccCols;
      __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(exch) + (warp - 2) * 32 * 32;  // transpose tile
      __nv_bfloat16* outb = reinterpret_cast<__nv_bfloat16*>(args.out);
      auto store_rows = [&](const float (&v)[32], int fbase, long long row0, int jn) {
        store_rows32(stg, lane, v, outb, args.ldo, args.N, fbase, row0, jn);
      };
      (void)store_rows;
      float sg = 1.0f, su = 1.0f;
      (void)part;  // FP8: per-feature weight scales of this thread's output feature
      if constexpr (EPI == kEpiSwiGLUFp8) {
        if (f_ok) {
          const long long fi = static_cast<long long>(tl.g) * args.N + f;
          sg = __ldg(args.scale_a0 + fi);
          su = __ldg(args.scale_a1 + fi);
        }
      }
      for (int j0 = 32 * part; j0 < tl.nvalid; j0 += 32 * kSplit) {
        uint32_t r0[32];
        tmem_ld_32cols(tbase + j0, r0);
        const int jn = min(32, tl.nvalid - j0);
        const long long row0 = static_cast<long long>(tl.row0) + j0;
        if constexpr (EPI == kEpiSwiGLU || EPI == kEpiSwiGLUFp8) {
          uint32_t r1[32];
          tmem_ld_32cols(tbase + NT + j0, r1);
          float sx = 1.0f;  // FP8: row scale of token j0 + lane, handed to the other lanes below
          if constexpr (EPI == kEpiSwiGLUFp8) sx = lane < jn ? __ldg(args.scale_b + row0 + lane) : 0.0f;
          tmem_wait_ld();
          float h[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float g = __uint_as_float(r0[j]), u = __uint_as_float(r1[j]);
            if constexpr (EPI == kEpiSwiGLUFp8) {
              const float sj = __shfl_sync(0xffffffffu, sx, j);
              g *= sj * sg;
              u *= sj * su;
            }
            h[j] = silu_mul(g, u);
          }
          store_rows(h, tl.n0 + q * 32, row0, jn);
        } else if constexpr (EPI == kEpiBF16) {
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r0[j]);
          store_rows(v, tl.n0 + q * 32, row0, jn);
          if constexpr (C::SEP) {  // wide tile: second accumulator = features n0 + 128 ..
            uint32_t r1[32];
            tmem_ld_32cols(tbase + NT + j0, r1);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r1[j]);
            store_rows(v, tl.n0 + kBM + q * 32, row0, jn);
          }
        } else {
          tmem_wait_ld();
          float* out = reinterpret_cast<float*>(args.out) + ks * args.split_stride;
          if (f_ok) {
            const float b = (args.bias && ks == 0) ? __ldg(args.bias + f) : 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < jn) out[(row0 + j) * args.ldo + f] = __uint_as_float(r0[j]) + b;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == L::kNumAcc) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
  // The last CTA to finish rewinds the schedule for the next launch on this slot (every CTA
  // has claimed its last tile before it counts itself done).
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&args.sched[1], 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(&args.sched[0], 0);
      atomicExch(&args.sched[1], 0);
    }
  }
}

// ---------------------------------------------------------------------------
// CTA-pair kernel (cta_group::2).  The two SMs of a cluster share one tile of 256 (SwiGLU)
// or 512 (bf16) output features x N <= 256 tokens.  Each CTA stages its own 128 rows of
// each of the two weight operands and half of the token rows; the pair MMA (M = 256,
// issued by the leader, rank 0) reads both token halves, so a token tile crosses L2 once
// per pair and each SM fills 48 KB of shared memory per K-step instead of the single-CTA
// tile's 64 KB for the same MMA work per SM.
//   SwiGLU: CTA r holds gate and up rows [n0 + 128 r, +128): gate and up accumulate in
//           separate TMEM columns of the same lanes, so no exchange between warps; the two
//           accumulators fill TMEM, so the epilogue of a tile runs between main loops.
//   bf16:   CTA r holds rows [n0 + 128 r, +128) and [n0 + 256 + 128 r, +128) (NA = 2).
// Both CTAs' TMA loads of a stage complete on the leader's "full" barrier; the leader's
// commits release both CTAs' "empty" and "tmem full" barriers; both CTAs' epilogue warps
// release the leader's "tmem empty" barrier.  The leader's producer claims tiles from the
// launch's counter and publishes each id to both CTAs through a ring in shared memory (the
// peer's slot written over the cluster), which both CTAs' consumers release.
// ---------------------------------------------------------------------------
template <int EPI>
struct PairLayout {
  static constexpr int NT = 256;                                // tokens per pair tile (MMA N)
  static constexpr int NA = 2;                                  // weight operands (accumulators)
  static constexpr int STAGES = 4;
  static constexpr int EW = 8;                                  // epilogue warps per CTA
  // bf16 SwiGLU: one warp per stage that fills the stage's token rows when they are gathered
  static constexpr int GW = EPI == kEpiSwiGLU ? STAGES : 0;
  static constexpr int kThr = 64 + 32 * (EW + GW);
  static constexpr int FEAT = (EPI == kEpiBF16) ? 512 : 256;   // output features per pair tile
  // token rows per tile rounded to ROUND (MMA N): 16 for bf16 operands (N = 16..256 in steps of
  // 16 for a CTA pair), 32 for E4M3 operands
  static constexpr int ROUND = EPI == kEpiSwiGLUFp8 ? 32 : 16;
  static constexpr int kAPair = NA * kABytes;                   // this CTA's 128-row weight boxes (one atom)
  static constexpr int kBBytes = (NT / 2) * 128;                // this CTA's token rows (one atom)
  static constexpr int kStageBytes = kAPair + kBBytes;
  static constexpr uint32_t kAccCols = NA * NT;                 // one tile's accumulators
  static constexpr int kNumAcc = 1;                             // TMEM buffers
  static constexpr uint32_t kTmemCols = kNumAcc * kAccCols;
  static constexpr int kStgBytes = EW * 32 * 32 * 2;
  static constexpr int kBarBytes = (8 * (2 * STAGES + 5 + 2 * kRing) + 8 + 4 * kRing + 15) / 16 * 16;
  static constexpr int kTableBytes = 2 * (kMaxGroups + 1) * 4;
  static constexpr int kSrcBytes = GW * (NT / 2) * 4;          // each gather warp's source rows of a tile
  static constexpr int kSmemBytes =
      1024 + STAGES * kStageBytes + kStgBytes + kBarBytes + kTableBytes + kSrcBytes;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kThr <= kMaxPairThreads, "block size");
};

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairLayout<EPI>::kThr, 1)
    pair_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                     const __grid_constant__ BoxMaps tmB, const __grid_constant__ CUtensorMap tmO,
                     const GemmArgs args) {
  using L = PairLayout<EPI>;
  constexpr int NT = L::NT, NA = L::NA, STAGES = L::STAGES, EW = L::EW;
  constexpr int KS = stage_k<EPI>();
  static_assert(EPI == kEpiSwiGLU || EPI == kEpiSwiGLUFp8 || EPI == kEpiBF16, "pair epilogues");
  static_assert(L::kTmemCols == 512, "TMEM allocation");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  __nv_bfloat16* stg_all = reinterpret_cast<__nv_bfloat16*>(smem + STAGES * L::kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * L::kStageBytes + L::kStgBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* rfull = drain + 1;
  uint64_t* rempty = rfull + kRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rempty + kRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring_tile = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(smem + STAGES * L::kStageBytes + L::kStgBytes + L::kBarBytes);
  int* s_pre = s_off + (kMaxGroups + 1);
  int* s_src = s_pre + (kMaxGroups + 1);
  __shared__ int s_warp_sums[kMaxPairThreads / 32];
  __shared__ int s_bad;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  // Gathered token rows (bf16 SwiGLU): the gather warps copy each stage's token rows with
  // 16-byte cp.async through assign_of_row instead of the producer's token boxes; a stage is
  // then full after the producer's weight bytes and one gather warp of each CTA.
  const bool gather = L::GW > 0 && args.gather != nullptr;
  const int G = args.offsets ? args.G : 1;
  const int NFT = (args.N + L::FEAT - 1) / L::FEAT;
  const int KB = (args.Kd + KS - 1) / KS;  // K-steps (a K atom beyond Kd reads the zero fill)

  // Set-up that reads no global input runs before the wait on the previous kernel.
  if (threadIdx.x == 0) {
    s_bad = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], gather ? 3 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * EW);  // every epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    for (int r = 0; r < kRing; ++r) {
      mbar_init(&rfull[r], 1);
      // leader MMA + leader epilogue, peer producer + peer epilogue (+ both CTAs' gather warps)
      mbar_init(&rempty[r], 2 + 2 * EW + (gather ? 2 * L::GW : 0));
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA0);
    tma_prefetch_map(&tmA1);
    for (int i = 0; i < kNumBoxes; ++i) tma_prefetch_map(&tmB.box[i]);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::kTmemCols);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  pdl_wait();  // offsets and the token operand come from earlier kernels
  pdl_launch_dependents();
  __syncthreads();
  for (int i = threadIdx.x; i <= G; i += L::kThr)
    s_off[i] = args.offsets ? __ldg(args.offsets + i) : (i == 0 ? 0 : args.M);
  __syncthreads();
  for (int i = threadIdx.x; i <= G; i += L::kThr) {
    const bool bad = s_off[i] < 0 || s_off[i] > args.M || (i > 0 && s_off[i] < s_off[i - 1]);
    if (bad) s_bad = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0 && rank == 0) report(args.status, MOE_DEV_BAD_INDEX);
    for (int i = threadIdx.x; i <= G; i += L::kThr) s_off[i] = 0;
  }
  __syncthreads();
  build_tile_table(s_pre, s_off, G, NT, NFT, s_warp_sums);  // ends with __syncthreads
  cluster_sync();  // both CTAs' barriers exist before any access over the cluster
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pre[G];
  const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
  const uint32_t rempty_leader = mapa_shared(smem_u32(rempty), 0);
  const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      const uint32_t rfull_peer = mapa_shared(smem_u32(rfull), 1);
      const uint32_t ring_peer = mapa_shared(smem_u32(const_cast<int*>(ring_tile)), 1);
      uint32_t stage = 0, phase = 0, rs = 0, rphase = 0;
      uint32_t pend_phase[STAGES];
      bool pend[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) pend[s] = false, pend_phase[s] = 0;
      bool ok = true;
      for (;;) {
        int t;
        if (rank == 0) {
          if (!mbar_wait_cluster(&rempty[rs], rphase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          const int claimed = atomicAdd(&args.sched[0], 1);
          t = claimed < total ? claimed : -1;
          ring_tile[rs] = t;
          st_shared_cluster(ring_peer + 4 * rs, t);
          mbar_arrive(&rfull[rs]);
          mbar_arrive_cluster(rfull_peer + 8 * rs);
        } else {
          if (!mbar_wait_cluster(&rfull[rs], rphase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          t = ring_tile[rs];
          mbar_arrive_cluster(rempty_leader + 8 * rs);
        }
        if (++rs == kRing) {
          rs = 0;
          rphase ^= 1u;
        }
        if (t < 0) break;
        const Tile tl = decode_tile<NT, L::ROUND, L::FEAT>(t, s_pre, s_off, G);
        const int half = tl.nround >> 1;  // token rows staged by each CTA (a multiple of ROUND / 2)
        const int rbase = tl.row0 + static_cast<int>(rank) * half;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          const uint32_t bar = full_leader + stage * 8;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2u * (L::kAPair + (gather ? 0 : half * 128)));
          uint8_t* st = ring + stage * L::kStageBytes;
          const int kx = kb * KS;
          if constexpr (EPI == kEpiBF16) {
            tma_load_3d_pair(st, &tmA0, bar, kx, tl.n0 + 128 * static_cast<int>(rank), tl.g);
            tma_load_3d_pair(st + kABytes, &tmA0, bar, kx, tl.n0 + 256 + 128 * static_cast<int>(rank), tl.g);
          } else {
            const int fr = tl.n0 + 128 * static_cast<int>(rank);
            tma_load_3d_pair(st, &tmA0, bar, kx, fr, tl.g);            // gate rows
            tma_load_3d_pair(st + kABytes, &tmA1, bar, kx, fr, tl.g);  // up rows
          }
          if (!gather) {
            int r = 0;
#pragma unroll
            for (int i = 1; i < kNumBoxes; ++i) {  // boxes of 128, 64, 32, 16, 8 rows
              const int rows = 256 >> i;
              if (half & rows) {
                tma_load_2d_pair(st + L::kAPair + r * 128, &tmB.box[i], bar, kx, rbase + r);
                r += rows;
              }
            }
          }
          pend[stage] = true;
          pend_phase[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (!ok) {
        if (rank == 0) {
#pragma unroll
          for (int s = 0; s < STAGES; ++s)
            if (pend[s]) mbar_drain(&full[s], pend_phase[s], 200000000ull);
        } else {  // the peer's copies complete on the leader's barrier: give them time to land
          const uint64_t t0 = global_timer_ns();
          while (global_timer_ns() - t0 < 2000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      const uint32_t empty_peer = mapa_shared(smem_u32(empty), 1);
      const uint32_t tfull_peer = mapa_shared(smem_u32(tfull), 1);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0, rs = 0, rphase = 0;
      bool ok = true;
      for (;;) {
        if (!mbar_wait_cluster(&rfull[rs], rphase, abort_flag, args.status)) {
          ok = false;
          break;
        }
        const int t = ring_tile[rs];
        mbar_arrive(&rempty[rs]);
        if (++rs == kRing) {
          rs = 0;
          rphase ^= 1u;
        }
        if (t < 0) break;
        const Tile tl = decode_tile<NT, L::ROUND, L::FEAT>(t, s_pre, s_off, G);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, args.status)) {
          ok = false;
          break;
        }
        const uint32_t d0 = tmem_base + acc * L::kAccCols;
        tc_fence_after();
        const uint32_t idesc =
            (EPI == kEpiSwiGLUFp8) ? idesc_e4m3_f32(256, tl.nround) : idesc_bf16_f32(256, tl.nround);
        for (int kb = 0; kb < KB; ++kb) {
          // gathered rows: the peer's gather warp wrote its rows with plain stores and arrived
          // with cluster-scope release, so this wait acquires at cluster scope
          if (!(gather ? mbar_wait_cluster(&full[stage], phase, abort_flag, args.status)
                       : mbar_wait(&full[stage], phase, abort_flag, args.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * L::kStageBytes);
          const uint32_t sb = sa + L::kAPair;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = sw128_kmajor_desc(sb + kk * 32);
#pragma unroll
            for (int i = 0; i < NA; ++i) {
              const uint64_t adesc = sw128_kmajor_desc(sa + i * kABytes + kk * 32);
              const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
              if constexpr (EPI == kEpiSwiGLUFp8) umma_e4m3_pair(d0 + i * NT, adesc, bdesc, idesc, accum);
              else umma_bf16_pair(d0 + i * NT, adesc, bdesc, idesc, accum);
            }
          }
          umma_commit_pair(smem_u32(&empty[stage]));  // both CTAs' stage buffers are free again
          umma_commit_pair(empty_peer + stage * 8);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(smem_u32(&tfull[acc]));
        umma_commit_pair(tfull_peer + acc * 8);
        if (++acc == L::kNumAcc) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {
        umma_commit_pair(smem_u32(drain));
        mbar_drain(drain, 0, 200000000ull);
      }
    }
  } else if (warp < 2 + EW) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;               // TMEM lanes [32q, 32q + 32)
    const int part = (warp - 2) >> 2;     // two warps per lane quadrant take alternate chunks
    __nv_bfloat16* stg = stg_all + (warp - 2) * 32 * 32;
    __nv_bfloat16* outb = reinterpret_cast<__nv_bfloat16*>(args.out);
    uint32_t acc = 0, acc_phase = 0, rs = 0, rphase = 0;
    for (;;) {
      if (!mbar_wait_cluster(&rfull[rs], rphase, abort_flag, args.status)) break;
      const int t = ring_tile[rs];
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&rempty[rs]);
        else mbar_arrive_cluster(rempty_leader + 8 * rs);
      }
      if (++rs == kRing) {
        rs = 0;
        rphase ^= 1u;
      }
      if (t < 0) break;
      const Tile tl = decode_tile<NT, L::ROUND, L::FEAT>(t, s_pre, s_off, G);
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, args.status)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * L::kAccCols;
      const int fa = tl.n0 + 128 * static_cast<int>(rank) + 32 * q;  // this warp's first feature
      float sg = 1.0f, su = 1.0f;
      if constexpr (EPI == kEpiSwiGLUFp8) {
        if (fa + lane < args.N) {
          const long long fi = static_cast<long long>(tl.g) * args.N + fa + lane;
          sg = __ldg(args.scale_a0 + fi);
          su = __ldg(args.scale_a1 + fi);
        }
      }
      for (int j0 = 32 * part; j0 < tl.nvalid; j0 += 64) {
        const int jn = min(32, tl.nvalid - j0);
        const long long row0 = static_cast<long long>(tl.row0) + j0;
        uint32_t r0[32], r1[32];
        tmem_ld_32cols(tbase + j0, r0);
        tmem_ld_32cols(tbase + NT + j0, r1);
        float sx = 1.0f;
        if constexpr (EPI == kEpiSwiGLUFp8) sx = lane < jn ? __ldg(args.scale_b + row0 + lane) : 0.0f;
        tmem_wait_ld();
        float v[32];
        if constexpr (EPI == kEpiBF16) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r0[j]);
          store_rows32_tma(stg, lane, v, &tmO, outb, args.ldo, args.N, fa, row0, jn);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r1[j]);
          store_rows32_tma(stg, lane, v, &tmO, outb, args.ldo, args.N, fa + 256, row0, jn);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float g = __uint_as_float(r0[j]), u = __uint_as_float(r1[j]);
            if constexpr (EPI == kEpiSwiGLUFp8) {
              const float sj = __shfl_sync(0xffffffffu, sx, j);
              g *= sj * sg;
              u *= sj * su;
            }
            v[j] = silu_mul(g, u);
          }
          store_rows32(stg, lane, v, outb, args.ldo, args.N, fa, row0, jn);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&tempty[acc]);
        else mbar_arrive_cluster(tempty_leader + acc * 8);
      }
      if (++acc == L::kNumAcc) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if constexpr (EPI == kEpiBF16) {
      if (lane == 0) bulk_wait_all();  // the tile stores are complete before the CTA exits
    }
  } else if (gather) {
    // ------------------------------------------------------------ token-row gather (both CTAs)
    // Warp gw fills the token rows of stage gw, i.e. K-steps gw, gw + STAGES, ... of the CTA's
    // sequence (the producer's stage counter).  Per tile it looks up the source row of each of
    // this CTA's rows once; per K-step each lane copies one 16-byte piece of four rows' 128-byte
    // K slices into the 128-byte-swizzled layout the producer's token boxes would have written
    // (piece c of row r at r * 128 + (c ^ (r % 8)) * 16), waits for its copies, fences them
    // against the tensor core's async-proxy reads and the warp arrives on the leader's barrier.
    const int gw = warp - 2 - EW;
    int* srow = s_src + gw * (NT / 2);
    const __nv_bfloat16* xsrc = reinterpret_cast<const __nv_bfloat16*>(args.gather_x);
    const uint32_t full_arrive = rank == 0 ? smem_u32(&full[gw]) : full_leader + gw * 8;
    const int c = lane & 7;  // this lane's 16-byte piece of a row's K slice
    constexpr int kGatherRows = NT / 2 / 4;  // rows per lane: four rows per warp-wide copy
    constexpr int kGatherBatch = 8;
    uint32_t rs = 0, rphase = 0, kstep = 0;
    for (;;) {
      int t = 0, got = 1;
      if (lane == 0) {
        got = mbar_wait_cluster(&rfull[rs], rphase, abort_flag, args.status);
        if (got) {
          t = ring_tile[rs];
          if (rank == 0) mbar_arrive(&rempty[rs]);
          else mbar_arrive_cluster(rempty_leader + 8 * rs);
        }
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      t = __shfl_sync(0xffffffffu, t, 0);
      if (++rs == kRing) {
        rs = 0;
        rphase ^= 1u;
      }
      if (t < 0) break;
      const Tile tl = decode_tile<NT, L::ROUND, L::FEAT>(t, s_pre, s_off, G);
      const int half = tl.nround >> 1;
      // this CTA's rows are tile rows rank * half + i; rows past the valid ones repeat row 0
      // (computed, never stored)
      for (int i = lane; i < half; i += 32) {
        const int j = static_cast<int>(rank) * half + i;
        srow[i] = gather_source(args, tl.row0 + (j < tl.nvalid ? j : 0));
      }
      __syncwarp();
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++kstep) {
        if (static_cast<int>(kstep % STAGES) != gw) continue;
        got = 1;
        if (lane == 0) got = mbar_wait(&empty[gw], ((kstep / STAGES) & 1u) ^ 1u, abort_flag, args.status);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        const uint32_t dst = smem_u32(ring + gw * L::kStageBytes + L::kAPair);
        const int k0 = kb * KS + 8 * c;  // first K element of this lane's piece
        const uint32_t nbytes = k0 < args.Kd ? 16u : 0u;  // past the reduction: zero fill
        const __nv_bfloat16* xk = xsrc + (nbytes ? k0 : 0);
        // this lane's rows lane / 8 + 4 i: their source rows read in batches, then the copies
#pragma unroll
        for (int i0 = 0; i0 < kGatherRows; i0 += kGatherBatch) {
          int sr[kGatherBatch];
#pragma unroll
          for (int u = 0; u < kGatherBatch; ++u) sr[u] = srow[min((lane >> 3) + 4 * (i0 + u), half - 1)];
#pragma unroll
          for (int u = 0; u < kGatherBatch; ++u) {
            const int r = (lane >> 3) + 4 * (i0 + u);
            if (r < half)
              cp_async_16(dst + r * 128 + ((c ^ (r & 7)) << 4), xk + static_cast<long long>(sr[u]) * args.Kd, nbytes);
          }
        }
        cp_async_wait_all();
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive(&full[gw]);
          else mbar_arrive_cluster(full_arrive);
        }
      }
      if (!ok) break;
      __syncwarp();  // srow is rewritten for the next tile
    }
  }

  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still touch its barriers or smem
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
  if (threadIdx.x == 0) {  // the last CTA rewinds the schedule for the next launch on this slot
    __threadfence();
    if (atomicAdd(&args.sched[1], 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(&args.sched[0], 0);
      atomicExch(&args.sched[1], 0);
    }
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

// Tensor [d2][d1][d0] (d0 contiguous) of bf16 (elem = 2) or 8-bit codes (elem = 1), box
// {128 bytes of d0, box1, 1}, 128-byte swizzle.
bool map_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1,
                 int elem = 2) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * elem, d0 * d1 * elem};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem), box1, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
             const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_bf16_2d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint32_t box1, int elem = 2) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {d0 * elem};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem), box1};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
             const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_token_boxes(BoxMaps* m, const void* base, uint64_t d0, uint64_t rows, int elem = 2) {
  for (int i = 0; i < kNumBoxes; ++i)
    if (!map_bf16_2d(&m->box[i], base, d0, rows, 256u >> i, elem)) return false;
  return true;
}

template <int EPI>
cudaError_t launch(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2, const BoxMaps& b,
                   const GemmArgs& args, long long tile_bound, cudaStream_t stream) {
  using L = Layout<EPI>;
  static std::atomic<int> attr_done[kMaxDevices] = {};
  const cudaError_t attr_err =
      smem_attr_once(reinterpret_cast<const void*>(grouped_gemm_kernel<EPI>), L::kSmemBytes, attr_done);
  if (attr_err != cudaSuccess) return attr_err;
  if (tile_bound <= 0) return cudaSuccess;
  const int grid = static_cast<int>(std::min<long long>(num_sms(), tile_bound));
  return launch_pdl(grouped_gemm_kernel<EPI>, dim3(grid), dim3(L::kThr), L::kSmemBytes, stream, a0, a1, a2, b, args);
}

// Output map of the pair kernel's tile stores: out [M][N] bf16 (row stride ldo), box 32 x 32.
bool map_out_tiles(CUtensorMap* m, const GemmArgs& args) {
  EncodeTiledFn enc = encoder();
  if (!enc || args.N <= 0 || args.M <= 0) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(args.N), static_cast<cuuint64_t>(args.M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(args.ldo) * 2};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, args.out, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI>
cudaError_t launch_pair(const CUtensorMap& a0, const CUtensorMap& a1, const BoxMaps& b, const GemmArgs& args,
                        long long tile_bound, cudaStream_t stream) {
  using L = PairLayout<EPI>;
  static std::atomic<int> attr_done[kMaxDevices] = {};
  const cudaError_t attr_err =
      smem_attr_once(reinterpret_cast<const void*>(pair_gemm_kernel<EPI>), L::kSmemBytes, attr_done);
  if (attr_err != cudaSuccess) return attr_err;
  if (tile_bound <= 0) return cudaSuccess;
  const int pairs = static_cast<int>(std::min<long long>(num_sms() / 2, tile_bound));
  CUtensorMap o;
  if (!map_out_tiles(&o, args)) return cudaErrorInvalidValue;
  return launch_pdl(pair_gemm_kernel<EPI>, dim3(2 * pairs), dim3(L::kThr), L::kSmemBytes, stream, a0, a1, b, o,
                    args);
}

long long tile_bound(long long rows, int groups, int NT, int N, int feat) {
  const long long nft = (N + feat - 1) / feat;
  return ((rows + NT - 1) / NT + (groups > 1 ? groups : 0)) * nft;
}

}  // namespace

int gemm_smem_bytes(int epi) {
  switch (epi) {
    case kEpiSwiGLU: return Layout<kEpiSwiGLU>::kSmemBytes;
    case kEpiBF16: return Layout<kEpiBF16>::kSmemBytes;
    case kEpiSwiGLUFp8: return Layout<kEpiSwiGLUFp8>::kSmemBytes;
    default: return Layout<kEpiF32>::kSmemBytes;
  }
}

// The CTA-pair kernel serves groups of at least MOE_PAIR_MIN_ROWS rows on average (its
// token tiles are cut in multiples of 16 (E4M3: 32) rows and split between the two SMs); smaller
// groups (decode) and the fp32 gating use the single-CTA kernel.  MOE_GEMM_PAIR=0 builds
// the single-CTA kernel only.
#ifndef MOE_GEMM_PAIR
#define MOE_GEMM_PAIR 1
#endif
#ifndef MOE_PAIR_MIN_ROWS
#define MOE_PAIR_MIN_ROWS 64
#endif
static std::atomic<int> g_pair_min_rows{MOE_PAIR_MIN_ROWS};
static bool use_pair(long long rows, int groups) {
  const int min_rows = g_pair_min_rows.load(std::memory_order_relaxed);
  return MOE_GEMM_PAIR && min_rows >= 0 && num_sms() >= 2 &&
         rows >= static_cast<long long>(min_rows) * std::max(groups, 1);
}

void set_pair_min_rows(int rows) { g_pair_min_rows.store(rows, std::memory_order_relaxed); }

// h = silu(xp Wg^T) * (xp Wu^T) per expert group; xp is x itself, or x's rows gathered
// through `gather` (row r of xp = row gather[r] / K of x) by the GEMM's own loads.
cudaError_t gemm_gate_up(const void* x, const int32_t* offsets, const void* w_gate, const void* w_up, int E,
                         long long rows, int H, int F, void* h, int* status, int* sched, cudaStream_t stream,
                         const int32_t* gather, int K, long long x_rows) {
  GemmArgs args{offsets, E, static_cast<int>(rows), F, H, h, F, nullptr, status, nullptr, nullptr, nullptr, sched};
  CUtensorMap a0, a1;
  BoxMaps b;
  if (gather) {
    // gathered rows: the CTA-pair kernel's gather warps copy them, whatever the row count
    if (K < 1 || x_rows < 1 || x_rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (!MOE_GEMM_PAIR || num_sms() < 2) return cudaErrorNotSupported;
    args.gather = gather;
    args.gather_div = K;
    args.gather_rows = static_cast<int>(x_rows);
    args.gather_x = x;
  }
  // the token maps are not read when the rows are gathered, but stay valid maps
  if (!map_token_boxes(&b, x, H, gather ? x_rows : rows)) return cudaErrorInvalidValue;
  if (!map_bf16_3d(&a0, w_gate, H, F, E, kBM) || !map_bf16_3d(&a1, w_up, H, F, E, kBM)) return cudaErrorInvalidValue;
  if (gather || use_pair(rows, E))
    return launch_pair<kEpiSwiGLU>(a0, a1, b, args,
                                   tile_bound(rows, E, PairLayout<kEpiSwiGLU>::NT, F, PairLayout<kEpiSwiGLU>::FEAT),
                                   stream);
  return launch<kEpiSwiGLU>(a0, a1, a1, b, args, tile_bound(rows, E, Cfg<kEpiSwiGLU>::NT, F, Cfg<kEpiSwiGLU>::FEAT), stream);
}

// FP8 dispatch: gate/up on E4M3 codes; g and u are scaled by the row's and the feature's
// scales in the epilogue (both factor out of the K sum), h is bf16 as in gemm_gate_up.
cudaError_t gemm_gate_up_fp8(const void* xq, const float* xs, const int32_t* offsets, const void* wq_gate,
                             const void* wq_up, const float* s_gate, const float* s_up, int E, long long rows, int H,
                             int F, void* h, int* status, int* sched, cudaStream_t stream) {
  GemmArgs args{offsets, E, static_cast<int>(rows), F, H, h, F, nullptr, status, s_gate, s_up, xs, sched};
  CUtensorMap a0, a1;
  BoxMaps b;
  if (!map_token_boxes(&b, xq, H, rows, 1) || !map_bf16_3d(&a0, wq_gate, H, F, E, kBM, 1) ||
      !map_bf16_3d(&a1, wq_up, H, F, E, kBM, 1))
    return cudaErrorInvalidValue;
  if (use_pair(rows, E))
    return launch_pair<kEpiSwiGLUFp8>(
        a0, a1, b, args, tile_bound(rows, E, PairLayout<kEpiSwiGLUFp8>::NT, F, PairLayout<kEpiSwiGLUFp8>::FEAT), stream);
  return launch<kEpiSwiGLUFp8>(a0, a1, a1, b, args,
                               tile_bound(rows, E, Cfg<kEpiSwiGLUFp8>::NT, F, Cfg<kEpiSwiGLUFp8>::FEAT), stream);
}

// y = h Wd^T per expert group.
cudaError_t gemm_down(const void* h, const int32_t* offsets, const void* w_down, int E, long long rows, int H,
                      int F, void* y, int* status, int* sched, cudaStream_t stream) {
  GemmArgs args{offsets, E, static_cast<int>(rows), H, F, y, H, nullptr, status, nullptr, nullptr, nullptr, sched};
  CUtensorMap a0;
  BoxMaps b;
  const bool pair = use_pair(rows, E);
  if (!map_bf16_3d(&a0, w_down, F, H, E, pair ? kBM : 256) || !map_token_boxes(&b, h, F, rows))
    return cudaErrorInvalidValue;
  if (pair)
    return launch_pair<kEpiBF16>(a0, a0, b, args,
                                 tile_bound(rows, E, PairLayout<kEpiBF16>::NT, H, PairLayout<kEpiBF16>::FEAT), stream);
  return launch<kEpiBF16>(a0, a0, a0, b, args, tile_bound(rows, E, Cfg<kEpiBF16>::NT, H, Cfg<kEpiBF16>::FEAT), stream);
}

// out[M][N] = a[M][Kd] w[N][Kd]^T, bf16 out.
cudaError_t gemm_dense(const void* a, const void* w, long long M, int N, int Kd, void* out, int* status,
                       int* sched, cudaStream_t stream) {
  CUtensorMap a0;
  BoxMaps b;
  const bool pair = use_pair(M, 1);
  if (!map_bf16_3d(&a0, w, Kd, N, 1, pair ? kBM : 256) || !map_token_boxes(&b, a, Kd, M))
    return cudaErrorInvalidValue;
  GemmArgs args{nullptr, 1, static_cast<int>(M), N, Kd, out, N, nullptr, status, nullptr, nullptr, nullptr, sched};
  if (pair)
    return launch_pair<kEpiBF16>(a0, a0, b, args, tile_bound(M, 1, PairLayout<kEpiBF16>::NT, N, PairLayout<kEpiBF16>::FEAT),
                                 stream);
  return launch<kEpiBF16>(a0, a0, a0, b, args, tile_bound(M, 1, Cfg<kEpiBF16>::NT, N, Cfg<kEpiBF16>::FEAT), stream);
}

// logits[T][E] = x[T][H] (hi + mid + lo)^T (+ bias), fp32 out; w_split is [3][E][H] bf16.
// Splits of the gating reduction: enough work units to fill the SMs when the output has few
// tiles (Qwen3 layer: 32 tiles of 128 tokens x 128 experts over 148 SMs -> 4 splits; a
// DeepSeek-R1 decode step: 2 tiles -> 28 splits), at least 4 K-steps per split, at most 32.
int gating_splits(long long T, int H, int E, int sms) {
  const long long units = ((T + 127) / 128) * ((E + 127) / 128);
  const int KB = (H + kBK - 1) / kBK;
  if (units <= 0) return 1;
  long long s = sms / units;
  s = std::min<long long>(s, std::min(32, KB / 4));
  return static_cast<int>(std::max<long long>(1, s));
}

cudaError_t gemm_gating(const void* x, const void* w_split, const float* bias, long long T, int H, int E,
                        float* logits, int ksplit, int* status, int* sched, cudaStream_t stream) {
  CUtensorMap a0;
  BoxMaps b;
  if (!map_bf16_3d(&a0, w_split, H, E, 3, kBM) || !map_token_boxes(&b, x, H, T)) return cudaErrorInvalidValue;
  const int S = std::max(1, ksplit);
  GemmArgs args{nullptr, 1, static_cast<int>(T), E, H, logits, E, bias, status, nullptr, nullptr, nullptr, sched,
                S, T * E};
  return launch<kEpiF32>(a0, a0, a0, b, args, tile_bound(T, 1, Cfg<kEpiF32>::NT, E, kBM) * S, stream);
}

}  // namespace moe
