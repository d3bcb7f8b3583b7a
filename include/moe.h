/*
 * moe.h - C ABI of the B200 (sm_100a) routed Mixture-of-Experts layer.
 *
 * One routed MoE layer on one GPU, following the pipeline of the "WideEP: Wide
 * Expert Parallelism and Kimi K3" essay, section "The router writes a network
 * schedule": the router scores every expert and keeps the top K per token; the
 * dispatcher counts the assignments bound for each destination, reserves their
 * rows and gathers the activations into one contiguous block per destination,
 * with routing metadata per row; each expert multiplies its block; the combine
 * step brings every output back to its token and sums the K of them with the
 * routing weights.  The essay's table of communication regimes says that local
 * (same-GPU) assignments avoid the fabric but still pay the permute's HBM
 * traffic, and points to fused layouts and grouped GEMM: that is the regime of
 * this library.  Logical expert-parallel partitions are only a buffer layout;
 * nothing is transferred between GPUs.
 *
 * Notation (the pages' statement of the problem): T tokens, E experts, top-K,
 * H dispatch width, F expert FFN width, b = 2 bytes per bf16 activation,
 * P logical partitions, TK = T*K assignments.  Assignment a = t*K + k is slot k
 * of token t.
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers unless the name ends in _host.  bf16 data is
 *    passed as raw IEEE bfloat16 (void*), row-major, densely packed.  Activation,
 *    weight and output matrices (bf16 or E4M3 rows) must start on a 16-byte boundary:
 *    the kernels move them in 16-byte pieces (MOE_ERR_INVALID_ARG otherwise).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only
 *    enqueues work and returns; none synchronizes with the host except
 *    moe_read_device_status.
 *  - The caller owns every buffer, including the workspace.  The library never
 *    allocates device memory and keeps no per-call state; it caches only device
 *    properties and the driver's tensor-map encoder.
 *  - Output shapes are static (TK rows, no capacity factor, no dropped tokens).
 *  - Argument and shape errors are returned synchronously and enqueue nothing.
 *    Launch failures return MOE_ERR_CUDA.  Conditions detected on the device
 *    (an expert id outside [0, E), a wait that exceeded its time limit) are
 *    OR-ed into the status word inside the workspace and read back with
 *    moe_read_device_status; no kernel traps or asserts.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Layer shape.  d_model = 0 except for the latent layer, whose tokens arrive at
 * width d_model and are projected down to H before routing ("Latent MoE" page,
 * sections "Definition" and "Current Synthesis"). */
typedef struct moe_dims {
  int64_t T;
  int32_t H;
  int32_t E;
  int32_t K;
  int32_t F;
  int32_t P;            /* logical partitions, E % P == 0 (1 = no partitioning) */
  int32_t renormalize;  /* 1: weights = softmax over the K selected logits;
                           0: weights = softmax over all E at the selected ids */
  int32_t d_model;      /* 0, or the model width of a latent layer */
  int32_t group_limit;  /* 0, or M: node-limited routing, each token takes its K experts from
                           its M best partitions (a partition ranks by its best expert);
                           needs P <= MOE_MAX_LIMITED_GROUPS and K <= M * E / P */
  int32_t F_shared;     /* 0, or the width of a shared expert that every token passes through
                           (a multiple of 8) */
  int32_t fp8_dispatch; /* 0, or 1: the layer dispatches E4M3 rows with per-token scales and
                           runs gate/up on E4M3 weights (moe_permute_fp8,
                           moe_grouped_gate_up_fp8); needs H % 16 == 0 */
} moe_dims;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* null pointer, T < 0, K > E, E % P != 0, ... */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* valid but outside this build's limits    */
  MOE_ERR_WORKSPACE = 3,          /* workspace missing or too small           */
  MOE_ERR_CUDA = 4,               /* a CUDA runtime / driver call failed      */
  MOE_ERR_DEVICE_TIMEOUT = 5,     /* a device-side wait ran out of time       */
  MOE_ERR_DEVICE_BAD_INDEX = 6,   /* an expert id or row index out of range   */
  MOE_ERR_NO_DEVICE = 7           /* no sm_100 device current                 */
} moe_status;

/* Device status bits OR-ed into the workspace status word. */
#define MOE_DEV_BAD_INDEX 0x1
#define MOE_DEV_TIMEOUT   0x2

/* Limits of this build (checked; larger shapes return MOE_ERR_UNSUPPORTED_SHAPE). */
#define MOE_MAX_E 1024
#define MOE_MAX_K 32
#define MOE_MAX_LIMITED_GROUPS 256

/* ------------------------------------------------------------------------- */
/* Workspace                                                                 */
/* ------------------------------------------------------------------------- */

/* Bytes of workspace the calls that take `ws` need for `d` (a multiple of 256).
 * One workspace may serve every call of one layer shape, on one stream at a
 * time.  Returns 0 for an invalid shape. */
size_t moe_workspace_bytes(const moe_dims* d);

/* Clears the whole workspace (an async memset of ws_bytes on `stream`): the status word,
 * the count/scan state (its block ticket, done counter, look-back flags and expert totals)
 * and the grouped GEMMs' tile-schedule counters.  The kernels leave that state at zero
 * after every call, so this is needed once after allocating the workspace, and again after
 * a device-side error has been reported or a call failed part-way. */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronizes `stream`, then copies the workspace status word to *status
 * (0 = no device-side error; otherwise MOE_DEV_* bits).  Off the hot path. */
moe_status moe_read_device_status(const void* ws, int32_t* status, void* stream);

const char* moe_status_str(moe_status s);

/* ------------------------------------------------------------------------- */
/* S0  Gating logits                                                         */
/* The sending rank scores each token against every expert (WideEP essay,   */
/* "The router writes a network schedule"); the gating network is non-expert */
/* work every rank replicates (InferenceX v2 review, claim IX2-0406).        */
/* ------------------------------------------------------------------------- */

/* One-time weight preparation: splits the fp32 router W_g [H][E] into three
 * bf16 planes hi, mid, lo with W_g = hi + mid + lo to float32 accuracy and
 * stores them transposed as w_g_split [3][E][H] (bf16, 6*E*H bytes, caller
 * allocated).  Not part of the per-token path. */
moe_status moe_pack_router(const float* w_g, const moe_dims* d, void* w_g_split, void* stream);

/* logits[t][e] = sum_h x[t][h] * W_g[h][e] (+ bias[e]), fp32 out [T][E].
 * x: [T][H] bf16.  w_g_split: from moe_pack_router.  bias: [E] fp32 or NULL.
 * Tensor-core products of the exact bf16 x with the three bf16 planes,
 * accumulated in fp32.  When [T][E] has few 128 x 128 tiles the reduction over H is
 * split (up to 32 parts) into partial logits in the workspace, added in split order;
 * the workspace of moe_workspace_bytes(d) bytes holds them. */
moe_status moe_gating(const void* x, const void* w_g_split, const float* bias,
                      const moe_dims* d, float* logits, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* S1  Router top-K + routing weights                                        */
/* Per-token choice of the K best-scoring experts (WideEP essay, "The       */
/* router writes a network schedule").                                       */
/* ------------------------------------------------------------------------- */

/* logits: [T][E] fp32.  Out: topk_ids [T][K] int32 and topk_w [T][K] fp32, slot
 * 0 the best.  Order: larger logit first; equal logits (-0.0 == +0.0) go to the
 * lower expert id; NaN ranks below every number.  Weights: exp(l_k - l_max)
 * normalised over the K selected (renormalize = 1) or over all E.
 * With d->group_limit = M > 0 (node-limited routing, DeepSeek-V3's bound on how many
 * nodes a token's experts span: "Three Parameter Counts...", "Halving top-k is a
 * network change first"), the K experts are the best among the experts of the token's
 * M best partitions, a partition ranking by its best expert under the same order. */
moe_status moe_route(const float* logits, const moe_dims* d, int32_t* topk_ids,
                     float* topk_w, void* stream);

/* ------------------------------------------------------------------------- */
/* S2  Count destinations, allocate slots                                    */
/* Counting what each expert receives and reserving its rows (WideEP essay, */
/* "The router writes a network schedule"); counts are of token-expert       */
/* assignments, so a token routed to K experts counts K times ("Three        */
/* Parameter Counts...", "What the utilization dashboard smooths away").     */
/* ------------------------------------------------------------------------- */

/* topk_ids: [T][K] int32.  Out (all int32):
 *   counts[E], offsets[E+1] (exclusive scan, offsets[E] = TK),
 *   part_counts[P], part_offsets[P+1] (partition p owns experts
 *     [p*E/P, (p+1)*E/P); part_offsets[p] = offsets[p*E/P]),
 *   row_of_assign[TK]: row of assignment a in the expert-major buffer, a stable
 *     counting sort (rows of one expert keep increasing a),
 *   assign_of_row[TK]: its inverse.
 * Two launches: one pass over the assignments in up to 128 chunks (1024 or more
 * assignments each), block-local histograms
 * with a decoupled look-back scan across the chunks (each chunk's counts are published and
 * added up by its successors; no grid-wide barrier), which ranks every assignment within
 * its expert and leaves the offsets; then the ranks become rows.  Uses the workspace
 * (per-chunk count rows, look-back flags and counters).
 * An id outside [0, E) sets MOE_DEV_BAD_INDEX and gets row -1; a look-back wait that runs
 * out (2 s) sets MOE_DEV_TIMEOUT.  Either way offsets[E] is set to -1 (a bad-offsets
 * marker that the grouped GEMMs refuse) and the other outputs are unspecified. */
moe_status moe_count_scan(const int32_t* topk_ids, const moe_dims* d, int32_t* counts,
                          int32_t* offsets, int32_t* part_counts, int32_t* part_offsets,
                          int32_t* row_of_assign, int32_t* assign_of_row,
                          void* ws, size_t ws_bytes, void* stream);

/* Bytes of device memory that moe_count_scan_noalloc keeps as its scratch.  Every GPU
 * that loads this library holds them until the process exits. */
#define MOE_NOALLOC_SCRATCH_BYTES (1u << 20)

/* moe_count_scan without a caller workspace (the source pages have no counterpart for
 * this call; it exists for callers that cannot allocate device memory: a plugin inside
 * a host framework that owns every device allocation, or a real-time loop that may not
 * call cudaMalloc/cudaFree, which can also synchronize the device, once it runs).
 * Same arguments, results and status codes as moe_count_scan minus the workspace.  The
 * scratch is a fixed device array inside the library holding the count/scan state: 768
 * bytes of counters and look-back flags and two int32 rows of E per chunk (ceil(T*K / 1024)
 * chunks, at most 128), at most MOE_NOALLOC_SCRATCH_BYTES in all; larger shapes return
 * MOE_ERR_UNSUPPORTED_SHAPE (only E = 1024 with T*K > 130 048 exceeds it).  The call
 * allocates nothing: it clears the scratch's counters and flags with an async memset on
 * `stream`, then launches the count/scan kernel and the kernel that turns ranks into rows.
 * The first call on a device looks up the scratch's device address once (with that device
 * current); make that first call before any stream capture.  All calls share the one
 * scratch and it keeps the last call's contents, so calls that overlap on the GPU (other
 * streams, other host threads) race: serialize them.  Device-side conditions have no status
 * word to go to (no workspace): an id outside [0, E) shows up as row -1 in row_of_assign,
 * and a call that met one, or whose look-back wait ran out, leaves offsets[E] = -1. */
moe_status moe_count_scan_noalloc(const int32_t* topk_ids, const moe_dims* d, int32_t* counts,
                                  int32_t* offsets, int32_t* part_counts, int32_t* part_offsets,
                                  int32_t* row_of_assign, int32_t* assign_of_row, void* stream);

/* ------------------------------------------------------------------------- */
/* S3  Permute into destination-contiguous rows + routing metadata           */
/* Gathering each destination's activations into one contiguous block with */
/* per-row routing metadata (WideEP essay, "The router writes a network     */
/* schedule"); the block holds T x K x H x b bytes (same essay, "Top-k      */
/* multiplies traffic"; "Three Parameter Counts...", "Halving top-k is a    */
/* network change first").                                                  */
/* ------------------------------------------------------------------------- */

/* xp[row_of_assign[t*K+k]][:] = x[t][:] for every (t, k); x [T][H] bf16,
 * xp [TK][H] bf16 (exactly T*K*H*2 bytes, no padding).  Metadata per row r
 * (each pointer may be NULL to skip it): meta_token[r] = t, meta_slot[r] = k,
 * meta_w[r] = topk_w[t][k], meta_local_expert[r] = e - p*E/P for the row's
 * expert e in partition p.  topk_ids is read only for meta_local_expert,
 * topk_w only for meta_w (either may be NULL when its output is NULL).
 * H must be a multiple of 8 (16-byte rows). */
moe_status moe_permute(const void* x, const int32_t* row_of_assign, const int32_t* topk_ids,
                       const float* topk_w, const moe_dims* d, void* xp,
                       int32_t* meta_token, int32_t* meta_slot, float* meta_w,
                       int32_t* meta_local_expert, void* stream);

/* ------------------------------------------------------------------------- */
/* S4 + S5  Expert SwiGLU FFN as grouped GEMMs over variable row counts      */
/* Each expert multiplies the rows routed to it (WideEP essay, "The router  */
/* writes a network schedule"); one grouped launch serves every expert,      */
/* whatever its row count ("Three Parameter Counts...", "Which               */
/* optimizations need a task-level gate").                                   */
/* ------------------------------------------------------------------------- */

/* For every expert e and row r in [offsets[e], offsets[e+1]):
 *   h[r][f] = bf16( silu(sum_k xp[r][k] w_gate[e][f][k]) * (sum_k xp[r][k] w_up[e][f][k]) )
 *   y[r][j] = bf16( sum_f h[r][f] w_down[e][j][f] )
 * xp [TK][H], w_gate/w_up [E][F][H], w_down [E][H][F] (nn.Linear layout),
 * h [TK][F], y [TK][H]; all bf16.  offsets: device [E+1] from moe_count_scan;
 * it is read on the device, so launch shapes never depend on the counts.
 * Experts with no rows cost nothing.  H and F must be multiples of 8.  Offsets
 * that decrease or leave [0, TK] set MOE_DEV_BAD_INDEX and the call computes
 * nothing.  The GEMM calls use only the workspace's 256-byte header (status word and
 * tile-schedule counters); any workspace of moe_workspace_bytes(d) bytes serves
 * (moe_dense needs 256 bytes). */
moe_status moe_grouped_ffn(const void* xp, const int32_t* offsets, const void* w_gate,
                           const void* w_up, const void* w_down, const moe_dims* d,
                           void* h, void* y, void* ws, size_t ws_bytes, void* stream);

/* Process-wide tuning of the grouped GEMMs (not part of the method): groups with at least
 * `rows` rows on average (default 64) run on the CTA-pair kernel, in which the two SMs of a
 * cluster share each token tile (tcgen05 cta_group::2); smaller groups, and every call when
 * `rows` < 0, run on the single-CTA kernel.  Both give the same results up to fp32
 * accumulation order.  Takes effect for launches enqueued after the call. */
void moe_set_pair_min_rows(int32_t rows);

/* The two halves of moe_grouped_ffn as separate launches (S4 and S5). */
moe_status moe_grouped_gate_up(const void* xp, const int32_t* offsets, const void* w_gate,
                               const void* w_up, const moe_dims* d, void* h, void* ws,
                               size_t ws_bytes, void* stream);
moe_status moe_grouped_down(const void* h, const int32_t* offsets, const void* w_down,
                            const moe_dims* d, void* y, void* ws, size_t ws_bytes, void* stream);

/* moe_grouped_gate_up without the permuted copy: row r of the operand is row
 * assign_of_row[r] / K of x ([T][H] bf16, the unpermuted activations), copied into the
 * GEMM's shared-memory stages by its own gather warps (16-byte cp.async, CTA-pair kernel
 * at every row count), so h equals moe_grouped_gate_up(xp, ...) bit for bit for
 * xp = moe_permute(x).  assign_of_row [TK] from moe_count_scan.  An entry outside
 * [0, T*K) is reported as MOE_ERR_DEVICE_BAD_INDEX (row 0 of x is read in its place).
 * Saves the T*K*H*2-byte xp buffer and its write and read; on B200 the row-by-row
 * operand fetch makes the GEMM slower than reading xp (about 1.5x at prefill sizes). */
moe_status moe_grouped_gate_up_gather(const void* x, const int32_t* assign_of_row, const int32_t* offsets,
                                      const void* w_gate, const void* w_up, const moe_dims* d, void* h,
                                      void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* FP8 dispatch: E4M3 rows with one fp32 scale per row, gate/up on E4M3,     */
/* bf16 down projection and combine.  The rows sent to the experts may be  */
/* narrowed to a low-precision format with their scales alongside and the   */
/* result widened again (WideEP essay, "Top-k multiplies traffic. Locality  */
/* subtracts it."); the change alters values, so it belongs to the bucket   */
/* that needs a task-level evaluation before release ("Three Parameter      */
/* Counts...", "Which optimizations need a task-level gate").                */
/* Format: E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits; largest */
/* finite 448; no infinities; 0x7F / 0xFF are NaN).                          */
/* ------------------------------------------------------------------------- */

/* Per-row quantization of x [rows][cols] bf16:
 *   scales[r] = amax_r / 448 (fp32 division; 1 when row r is all zero),
 *   q[r][c]   = E4M3 code of fp32(x[r][c]) / scales[r] (fp32 division, round to nearest
 *               even, saturating to +-448).
 * q [rows][cols] uint8, scales [rows] fp32.  cols must be a multiple of 16.  One-time
 * preparation of the gate and up weights ([E*F] rows of H each). */
moe_status moe_quantize_fp8_rows(const void* x, int64_t rows, int32_t cols, void* q, float* scales,
                                 void* stream);

/* FP8 dispatch: each token t is quantized once as by moe_quantize_fp8_rows and its codes and
 * scale land at the rows r = row_of_assign[t*K+k] of its K assignments: xq[r][:] (uint8
 * [TK][H]) and xs[r] (fp32 [TK]), T*K*H + 4*T*K bytes in all (half the bf16 payload plus
 * the scales).  Metadata as moe_permute.  H must be a multiple of 16. */
moe_status moe_permute_fp8(const void* x, const int32_t* row_of_assign, const int32_t* topk_ids,
                           const float* topk_w, const moe_dims* d, void* xq, float* xs,
                           int32_t* meta_token, int32_t* meta_slot, float* meta_w,
                           int32_t* meta_local_expert, void* stream);

/* Gate/up + SwiGLU on E4M3 rows.  For every expert e and row r in [offsets[e], offsets[e+1]):
 *   g = xs[r] * s_gate[e][f] * sum_k val(xq[r][k]) * val(wq_gate[e][f][k]),
 *   u = xs[r] * s_up[e][f]   * sum_k val(xq[r][k]) * val(wq_up[e][f][k]),
 *   h[r][f] = bf16( silu(g) * u ),
 * E4M3 x E4M3 tensor-core products accumulated in fp32.  xq [TK][H] uint8, xs [TK] fp32 (from
 * moe_permute_fp8); wq_gate, wq_up [E][F][H] uint8 and s_gate, s_up [E][F] fp32 (from
 * moe_quantize_fp8_rows on the bf16 weights); h [TK][F] bf16, consumed by moe_grouped_down.
 * H a multiple of 16.  Offsets are checked as in moe_grouped_ffn. */
moe_status moe_grouped_gate_up_fp8(const void* xq, const float* xs, const int32_t* offsets,
                                   const void* wq_gate, const void* wq_up, const float* s_gate,
                                   const float* s_up, const moe_dims* d, void* h, void* ws,
                                   size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* S6  Combine: unpermute + weighted sum                                     */
/* Every expert output goes back to its token and the K outputs are summed */
/* with the routing weights (WideEP essay, "The router writes a network     */
/* schedule").                                                               */
/* ------------------------------------------------------------------------- */

/* out[t][:] = bf16( sum_{k<K} topk_w[t][k] * y[row_of_assign[t*K+k]][:] + shared[t][:] ),
 * accumulated in fp32 in slot order.  y [TK][H] bf16, out [T][H] bf16; shared: [T][H] bf16
 * output of a shared expert (added with weight 1: a shared expert sees every token and
 * takes no routing weight, "Three Parameter Counts...", "What the utilization dashboard
 * smooths away"), or NULL. */
moe_status moe_combine(const void* y, const int32_t* row_of_assign, const float* topk_w,
                       const void* shared, const moe_dims* d, void* out, void* stream);

/* ------------------------------------------------------------------------- */
/* S7  Skew statistics                                                       */
/* Load skew = the busiest expert's load over the mean load, followed at    */
/* its 95th percentile over steps ("Three Parameter Counts...", "What the   */
/* utilization dashboard smooths away").                                     */
/* ------------------------------------------------------------------------- */

/* *d_ratio (device fp32) = max_e counts[e] / (sum_e counts[e] / E); 0 if no rows. */
moe_status moe_skew_stats(const int32_t* counts, const moe_dims* d, float* d_ratio, void* stream);

/* Host helper: 95th percentile of n per-step ratios by nearest rank (the
 * ceil(0.95 n)-th smallest).  Returns NaN for n <= 0. */
double moe_p95(const float* ratios, int n);

/* ------------------------------------------------------------------------- */
/* S8  Latent projections ("Latent MoE" page: dispatch on a reduced width)   */
/* ------------------------------------------------------------------------- */

/* out[m][n] = bf16( sum_k a[m][k] * w[n][k] ): a [M][Kd] bf16, w [N][Kd] bf16
 * (nn.Linear layout), out [M][N] bf16.  Used for z = x W_dp^T (d_model -> H)
 * before routing and final = out W_up^T (H -> d_model) after combine.
 * Kd and N must be multiples of 8. */
moe_status moe_dense(const void* a, const void* w, int64_t M, int32_t N, int32_t Kd,
                     void* out, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* Whole layer                                                               */
/* ------------------------------------------------------------------------- */

typedef struct moe_layer_weights {
  const void*  w_g_split;   /* [3][E][H] bf16 from moe_pack_router          */
  const float* bias;        /* [E] fp32 router bias, or NULL                 */
  const void*  w_gate;      /* [E][F][H] bf16                                */
  const void*  w_up;        /* [E][F][H] bf16                                */
  const void*  w_down;      /* [E][H][F] bf16                                */
  const void*  w_dp;        /* latent only: [H][d_model] bf16, else NULL     */
  const void*  w_upp;       /* latent only: [d_model][H] bf16, else NULL     */
  const void*  w_shared_gate; /* shared expert (F_shared > 0): [F_shared][H] bf16    */
  const void*  w_shared_up;   /* [F_shared][H] bf16                                  */
  const void*  w_shared_down; /* [H][F_shared] bf16                                  */
  const void*  w_gate_q;    /* fp8_dispatch: [E][F][H] E4M3 codes of w_gate   */
  const void*  w_up_q;      /* fp8_dispatch: [E][F][H] E4M3 codes of w_up     */
  const float* s_gate;      /* fp8_dispatch: [E][F] fp32 scales of w_gate_q   */
  const float* s_up;        /* fp8_dispatch: [E][F] fp32 scales of w_up_q     */
} moe_layer_weights;

typedef struct moe_layer_buffers {
  void*    z;               /* latent only: [T][H] bf16 (routed activations) */
  float*   logits;          /* [T][E] fp32                                   */
  int32_t* topk_ids;        /* [T][K]                                        */
  float*   topk_w;          /* [T][K]                                        */
  int32_t* counts;          /* [E]                                           */
  int32_t* offsets;         /* [E+1]                                         */
  int32_t* part_counts;     /* [P]                                           */
  int32_t* part_offsets;    /* [P+1]                                         */
  int32_t* row_of_assign;   /* [TK]                                          */
  int32_t* assign_of_row;   /* [TK]                                          */
  void*    xp;              /* [TK][H] bf16, or NULL: see moe_layer_forward   */
  int32_t* meta_token;      /* [TK] or NULL                                  */
  int32_t* meta_slot;       /* [TK] or NULL                                  */
  float*   meta_w;          /* [TK] or NULL                                  */
  int32_t* meta_local_expert; /* [TK] or NULL                                */
  void*    h;               /* [TK][F] bf16                                  */
  void*    y;               /* [TK][H] bf16                                  */
  void*    out;             /* [T][H] bf16 (combine output)                  */
  void*    final_out;       /* latent only: [T][d_model] bf16                */
  float*   skew;            /* [1] fp32 max/mean expert load                 */
  void*    h_shared;        /* shared expert: [T][F_shared] bf16             */
  void*    y_shared;        /* shared expert output: [T][H] bf16             */
  void*    aux_stream;      /* NULL, or a cudaStream_t on which the shared expert
                               runs alongside the routed path                */
  void*    fork_event;      /* with aux_stream: two cudaEvent_t created by the */
  void*    join_event;      /* caller (timing disabled is fine)              */
  void*    xq;              /* fp8_dispatch: [TK][H] uint8 dispatched codes (xp unused) */
  float*   xs;              /* fp8_dispatch: [TK] fp32 row scales            */
} moe_layer_buffers;

/* Number of stage boundaries recorded when stage events are given. */
#define MOE_NUM_STAGE_EVENTS 10

/* With d->T = 0 only counts, offsets, part_counts, part_offsets (all set to zero) and skew
 * (set to 0) are written; the other pointers may be NULL.
 * Runs every step on `stream` in pipeline order: [latent down-projection] ->
 * gating -> route -> count/scan -> permute -> gate/up+SwiGLU -> down -> combine
 * -> [latent up-projection] -> skew statistics.  With d->fp8_dispatch the permute is
 * moe_permute_fp8 (into b->xq, b->xs; b->xp may be NULL) and gate/up runs on
 * w->w_gate_q / w->w_up_q with their scales.  With bf16 dispatch and b->xp NULL no
 * permuted copy is made: the permute step only writes the rows (row_of_assign,
 * assign_of_row) and the metadata, and the gate/up GEMM copies each row's token
 * straight from the routed activations (row r is token assign_of_row[r] / K, as in
 * moe_grouped_gate_up_gather); h, y and out are bit-identical to the run with xp.  With d->F_shared > 0 the shared
 * expert (gate/up+SwiGLU and down over all T tokens of the routed activations) runs
 * on b->aux_stream, forked after the routed activations are ready and joined before
 * the combine, or on `stream` when aux_stream is NULL.  x: [T][d_in] bf16 with
 * d_in = d_model for a latent layer, else H.  stage_events: NULL, or an array of
 * MOE_NUM_STAGE_EVENTS cudaEvent_t (created by the caller) recorded at: start,
 * after latent-down, gating, route, count/scan, permute, gate/up, down,
 * combine, latent-up/skew (end).  Events of absent stages are still recorded. */
moe_status moe_layer_forward(const void* x, const moe_layer_weights* w, const moe_dims* d,
                             const moe_layer_buffers* b, void* ws, size_t ws_bytes,
                             void* const* stage_events, void* stream);

/* The same layer with HOST activations: copies x_host (pinned, [T][d_in] bf16)
 * into x_dev, runs moe_layer_forward, and copies the final output ([T][d_out]
 * bf16, d_out = d_model for a latent layer, else H) back to out_host, all
 * enqueued on `stream` (the host data must stay valid until the stream reaches
 * the copies). */
moe_status moe_layer_forward_host(const void* x_host, void* x_dev, const moe_layer_weights* w,
                                  const moe_dims* d, const moe_layer_buffers* b, void* ws,
                                  size_t ws_bytes, void* out_host, void* stream);

/* ------------------------------------------------------------------------- */
/* Expert-parallel exchange across GPUs (one process per GPU, R ranks)       */
/* The experts are split evenly over the ranks (WideEP essay, "896 experts  */
/* across 64 ranks"; EP8 = 32 of 256 experts per GPU in the InferenceX v2   */
/* review, claim IX2-0384); each rank routes its own tokens, counts what    */
/* every destination receives, reserves the rows there and sends the        */
/* activations; the experts' outputs come back to be weighted and summed    */
/* (WideEP essay, "The router writes a network schedule"), about T*K*H*b    */
/* bytes each way ("Top-k multiplies traffic. Locality subtracts it.").      */
/*                                                                           */
/* Protocol, per layer call with an epoch number that every rank increases  */
/* in step (1, 2, ...):                                                      */
/*   1. each rank: route and moe_count_scan of its T tokens with P = R (the */
/*      partitions are the ranks: rank d owns experts [d*El, (d+1)*El),     */
/*      El = E / R); every rank has the same T;                             */
/*   2. all-gather of the E per-expert counts of every rank into C [R][E]   */
/*      (the caller's collective, e.g. NCCL on the same stream);            */
/*   3. moe_ep_plan (C on the device), moe_ep_dispatch;                     */
/*   4. moe_ep_wait(phase 0); grouped gate/up and down on the received rows  */
/*      (moe_grouped_ffn with recv_offsets, E = El local experts);           */
/*   5. moe_ep_return; moe_ep_wait(phase 1); moe_combine on ret_y with the   */
/*      rank's own row_of_assign and weights.                                */
/* Rank d's receive buffer holds its experts' rows expert-major, then by    */
/* source rank, then in the source's stable order: the single-GPU layout of */
/* all ranks' tokens concatenated in rank order, restricted to its experts. */
/* The transfers are plain 16-byte stores into the peers' memory (CUDA IPC   */
/* mappings, NVLink), no TMA and no multicast; each kernel's last block     */
/* publishes the epoch in every peer's signal pad with system-scope release */
/* stores, and moe_ep_wait acquires them (2 s limit, then MOE_DEV_TIMEOUT). */
/* Buffers: recv_x [cap][H] bf16 and recv_meta [cap][2] int32 (source rank, */
/* source row) with cap = R*T*K (every assignment of every rank may land on */
/* one rank: no capacity factor, no dropped tokens), ret_y [T*K][H] bf16,    */
/* signal [2][R] int32 zeroed once; all four are read or written by peers.   */
/* ------------------------------------------------------------------------- */

#define MOE_EP_MAX_RANKS 64
#define MOE_EP_IPC_HANDLE_BYTES 64

/* Device addresses, valid in the calling process, of every rank's exchange buffers
 * (entries [0, R); this rank's own buffers at index rank). */
typedef struct moe_ep_peers {
  void*    recv_x[MOE_EP_MAX_RANKS];
  int32_t* recv_meta[MOE_EP_MAX_RANKS];
  void*    ret_y[MOE_EP_MAX_RANKS];
  int32_t* signal[MOE_EP_MAX_RANKS];
} moe_ep_peers;

/* Bytes of the EP workspace (status word and the two kernels' done counters), zeroed once
 * with moe_workspace_init; one per rank, one stream at a time. */
size_t moe_ep_workspace_bytes(void);

/* From C [R][E] (device int32): send_base[E], the row of rank d = e / El's receive buffer at
 * which this rank's rows of expert e start, and recv_offsets[El + 1], this rank's received
 * rows per local expert (the grouped GEMM's offsets).  One block on `stream`. */
moe_status moe_ep_plan(const int32_t* counts_all, int32_t R, int32_t rank, const moe_dims* d,
                       int32_t* send_base, int32_t* recv_offsets, void* stream);
/* The same plan computed on the host from a host copy of C (host pointers, no GPU). */
moe_status moe_ep_plan_host(const int32_t* counts_all, int32_t R, int32_t rank, const moe_dims* d,
                            int32_t* send_base, int32_t* recv_offsets);

/* For every assignment a = t*K + k with expert e: row = send_base[e] + row_of_assign[a] -
 * offsets[e] of rank e / El receives x[t] (recv_x) and (rank, row_of_assign[a])
 * (recv_meta); then slot [0][rank] of every rank's signal pad gets `epoch`.  x [T][H] bf16;
 * offsets from moe_count_scan.  A row outside [0, cap) is skipped and sets
 * MOE_DEV_BAD_INDEX in the EP workspace. */
moe_status moe_ep_dispatch(const void* x, const int32_t* row_of_assign, const int32_t* topk_ids,
                           const int32_t* offsets, const int32_t* send_base, const moe_dims* d,
                           int32_t R, int32_t rank, int64_t cap, const moe_ep_peers* peers,
                           int32_t epoch, void* ep_ws, void* stream);

/* Waits on the device until slots [phase][0..R) of this rank's signal pad hold at least
 * `epoch` (phase 0: every source has dispatched; phase 1: every owner has returned). */
moe_status moe_ep_wait(const int32_t* signal, int32_t R, int32_t phase, int32_t epoch, void* ep_ws,
                       void* stream);

/* For every received row j < recv_offsets[El]: y_recv[j] goes to row recv_meta[j].row of
 * rank recv_meta[j].rank's ret_y; then slot [1][rank] of every signal pad gets `epoch`.
 * y_recv [cap][H] bf16 (the grouped FFN's output on recv_x). */
moe_status moe_ep_return(const void* y_recv, const int32_t* recv_meta, const int32_t* recv_offsets,
                         const moe_dims* d, int32_t R, int32_t rank, int64_t cap,
                         const moe_ep_peers* peers, int32_t epoch, void* ep_ws, void* stream);

/* CUDA IPC plumbing for the peer addresses: export a handle (MOE_EP_IPC_HANDLE_BYTES) of the
 * allocation holding dev_ptr and dev_ptr's offset in it; import opens a peer's handle in this
 * process (*base, to close later) and returns base + offset; close releases an import. */
moe_status moe_ep_ipc_export(const void* dev_ptr, void* handle, uint64_t* offset);
moe_status moe_ep_ipc_import(const void* handle, uint64_t offset, void** base, void** dev_ptr);
moe_status moe_ep_ipc_close(void* base);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
