"""Plain CPU oracle for one routed Mixture-of-Experts layer (fp64 arithmetic).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, table or
helper with the CUDA library; both sides only consume the same seeded inputs.

Every function is the plain definition of one step, written with numpy in
float64 (library primitives such as ``matmul`` and a stable ``argsort`` serve as
steps; nothing is blocked, fused or reordered).  Sources, cited by page title
and section:

* [WideEP/router]  "WideEP: Wide Expert Parallelism and Kimi K3" essay
  (manishklach.github.io/writings/wideep-kimi-expert-parallelism), section
  "The router writes a network schedule": the pipeline of a routed layer
  (score experts and keep the top k; count each destination's assignments and
  reserve their slots; gather activations per destination with routing
  metadata; run each expert on its rows; send outputs back, undo the
  permutation and weight them).
* [WideEP/bytes]  same essay, section "Top-k multiplies traffic. Locality
  subtracts it.": one dispatch carries about T x k x H x B activation bytes
  and the combine about as many.
* [WideEP/regimes]  same essay, table of communication regimes: assignments
  that stay on the same GPU cross no fabric but still cost a permute in HBM.
* [WideEP/placement]  same essay, section "896 experts across 64 ranks": an
  even split of the experts over the ranks (896 / 64 = 14 per rank).
* [ParamCounts/network]  "Three Parameter Counts, and Only One Tells You Whether
  the Model Fits" (clarity-us-archive, 2026-09-24 science edition), section
  "Halving top-k is a network change first": the dispatch payload is bounded by
  T x K x H x b.
* [ParamCounts/dashboard]  same article, section "What the utilization
  dashboard smooths away": count per expert every token-expert assignment, and
  watch the busiest expert's load over the mean load at its 95th percentile.
* [ParamCounts/gate]  same article, section "Which optimizations need a
  task-level gate": a grouped GEMM serves experts with different row counts in
  one launch and leaves the expert selection unchanged.
* [LatentMoE]  "Latent MoE" concept page (podcastatlas.ai wiki), sections
  "Definition" and "Current Synthesis": experts receive a narrower, projected
  hidden state.
* [ParamCounts/layout]  "Three Parameter Counts...", section "Halving top-k is
  a network change first": in DeepSeek-V3 the set of nodes (expert groups) a
  token's experts may come from is capped by the trained router itself.

Readings where the pages are silent:

* Top-k order: a beats b iff value(a) > value(b), or the values compare equal
  and id(a) < id(b).  -0.0 equals +0.0; NaN ranks below every number (also
  below -inf) and NaNs tie-break by id.  Slots are stored best first.
* Routing weights: softmax over the K selected logits (equal to softmax over all
  E followed by renormalising the top-K); with ``renormalize=False`` the weight
  is the plain softmax over all E at the selected experts.
* Order of rows inside one expert: stable (assignment a = t*K + k ascending).
* Shared expert [ParamCounts/dashboard: a shared expert in the DeepSeekMoE manner
  processes all tokens, independent of routing; InferenceX review claim IX2-0406 lists the shared
  expert among the replicated non-expert weights]: a SwiGLU FFN of its own width on
  every token, rounded like a routed expert, added with weight 1 in the combine:
  out[t] = bf16( sum_k w[t,k] y[row(t,k)] + s[t] ).
* Node-limited routing: the groups are the P partitions; a group ranks by its best
  expert under the top-k order; each token keeps its M best groups and takes its K
  experts from those groups only.
* Partition p owns experts [p*E/P, (p+1)*E/P); metadata per row is
  (token, slot, weight, expert - p*E/P).
* Expert FFN: SwiGLU, h = silu(x Wg^T) * (x Wu^T), y = h Wd^T with nn.Linear
  weight layout (Wg, Wu: [E][F][H]; Wd: [E][H][F]).  h and y are rounded to
  bf16 (round to nearest, ties to even), the storage points of the layer.
* Combine: out[t] = bf16( sum_k w[t,k] * y[row(t,k)] ), summed in slot order.
* Latent layer: z = bf16(x Wdp^T) is routed and dispatched; the final output is
  bf16(out Wup^T).
* FP8 dispatch [WideEP/bytes: low-precision dispatch quantizes the outbound
  activation, carries its scales, computes in the other format and returns at higher
  precision; DeepEP's published examples dispatch in FP8 and combine in BF16]: the
  format is E4M3 (bias 7, 3 mantissa bits, largest finite 448, no infinities, code
  0x7F/0xFF = NaN) with one fp32 scale per row, s = amax(|row|) / 448 (1 for an
  all-zero row) and code = round-to-nearest-even(x / s) saturated to +-448, the
  scale and the quotient both taken in fp32 (the float decides an integer code, so
  it is decided in the kernel's precision).  Activations are quantized per token (the
  K dispatched copies share the token's codes and scale), gate and up weights per
  output feature.  g = s_x s_wg sum_k q_x q_wg (likewise u) from the codes; h, the
  down projection (bf16 weights) and the combine are as in the bf16 layer.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_bits_to_f64", "f64_to_bf16_bits", "gating_logits", "route",
    "count_scan", "permute", "grouped_ffn", "ffn_rows", "combine",
    "skew_ratio", "p95_nearest_rank", "dense_bf16", "layer_forward", "route_limited",
    "dispatch_bytes", "expert_weight_bytes", "experts_per_partition",
    "E4M3_MAX", "e4m3_to_f64", "f32_to_e4m3", "quantize_rows_fp8", "dispatch_fp8", "ffn_rows_fp8",
    "grouped_ffn_fp8", "quantize_experts_fp8", "dispatch_bytes_fp8",
    "checkpoint_bytes",
]


# ----------------------------------------------------------------------------
# bf16 storage format (8 exponent bits, 7 stored mantissa bits)
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as float64."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even), directly.

    For a finite v with binade 2^e (e = floor(log2|v|), at least -126 so that
    the subnormal range keeps its fixed spacing), the bf16 spacing is 2^(e-7);
    v is scaled by that power of two (exact), rounded half-to-even by
    ``np.rint`` and scaled back.  The result is then an exactly representable
    bf16 value whose float32 form carries the bf16 pattern in its top 16 bits.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.float64)
    finite = np.isfinite(v)
    vf = v[finite]
    _, ex = np.frexp(vf)                 # vf = m * 2**ex, 0.5 <= |m| < 1
    e = np.maximum(ex - 1, -126)         # binade exponent, clamped to normal min
    ulp = np.ldexp(1.0, e - 7)
    out[finite] = np.rint(vf / ulp) * ulp
    out[~finite] = v[~finite]
    with np.errstate(over="ignore"):
        f32 = out.astype(np.float32)     # exact for every bf16 value; overflow -> inf
    bits = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(v)
    bits[nan] = np.uint16(0x7FC0)
    return bits


# ----------------------------------------------------------------------------
# Step S0: gating logits   [WideEP/router]: the sending rank scores every expert per token
# ----------------------------------------------------------------------------

def gating_logits(x_bits, w_g, bias=None) -> np.ndarray:
    """logits[t, e] = fp32( sum_h x[t, h] * W_g[h, e] ) (+ bias[e] added in fp32).

    x_bits: [T, H] bf16 bits; w_g: [H, E] float32; bias: [E] float32 or None.
    """
    x = bf16_bits_to_f64(x_bits)
    l64 = x @ np.asarray(w_g, dtype=np.float64)
    l32 = l64.astype(np.float32)
    if bias is not None:
        l32 = (l32 + np.asarray(bias, dtype=np.float32)).astype(np.float32)
    return l32


# ----------------------------------------------------------------------------
# Step S1: top-K selection + routing weights   [WideEP/router]
# ----------------------------------------------------------------------------

def route(logits, K: int, renormalize: bool = True):
    """Top-K expert ids per token and their routing weights.

    Ids are ordered best first under: larger value wins; equal values (with
    -0.0 == +0.0) go to the lower id; NaN is below every number.  Weights are
    computed in float64 from the float32 logits and rounded to float32:
    renormalised: w_k = exp(l_k - m) / sum_{j<K} exp(l_j - m), m = top logit;
    plain:        w_k = exp(l_k - m) / sum_{e<E} exp(l_e - m).
    """
    l = np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    if not (1 <= K <= E):
        raise ValueError("need 1 <= K <= E")
    v = l.astype(np.float64) + 0.0          # -0.0 + 0.0 == +0.0
    is_nan = np.isnan(v)
    key_val = np.where(is_nan, 0.0, -v)     # ascending sort of -v = descending v
    ids_e = np.broadcast_to(np.arange(E), (T, E))
    # lexsort: last key is primary.  Order: non-NaN first, then larger value, then lower id.
    order = np.lexsort((ids_e, key_val, is_nan.astype(np.int8)), axis=1)
    ids = order[:, :K].astype(np.int32)
    sel = np.take_along_axis(v, ids, axis=1)
    m = sel[:, :1]
    with np.errstate(invalid="ignore", over="ignore"):
        if renormalize:
            num = np.exp(sel - m)
            w = num / num.sum(axis=1, keepdims=True)
        else:
            mall = np.max(np.where(is_nan, -np.inf, v), axis=1, keepdims=True)
            num = np.exp(sel - mall)
            w = num / np.exp(v - mall).sum(axis=1, keepdims=True)
    return ids, w.astype(np.float32)


def _expert_order(v64):
    """Per token, expert ids best first (larger value; ties -> lower id; NaN last)."""
    T, E = v64.shape
    is_nan = np.isnan(v64)
    key_val = np.where(is_nan, 0.0, -v64)
    ids_e = np.broadcast_to(np.arange(E), (T, E))
    return np.lexsort((ids_e, key_val, is_nan.astype(np.int8)), axis=1)


def route_limited(logits, K: int, P: int, M: int, renormalize: bool = True):
    """Node-limited top-K: the K experts come from the token's M best groups.

    Group p holds experts [p*E/P, (p+1)*E/P).  A group ranks by its best expert under
    the top-k order of ``route``; the M groups whose best experts come first are kept
    and the K best experts among their experts are selected.  Weights as in ``route``
    (over the K selected, or over all E when not renormalising).  [ParamCounts/layout]
    """
    l = np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    if E % P or not (1 <= M <= P) or K > M * (E // P):
        raise ValueError("need E % P == 0, 1 <= M <= P and K <= M * E / P")
    epp = E // P
    v = l.astype(np.float64) + 0.0
    order = _expert_order(v)                      # [T, E] expert ids, best first
    group_of = order // epp
    ids = np.empty((T, K), np.int64)
    for t in range(T):
        kept, seen = [], set()
        for g in group_of[t]:                     # groups in the order of their best expert
            if g not in seen:
                seen.add(g)
                kept.append(g)
                if len(kept) == M:
                    break
        allowed = np.isin(group_of[t], kept)
        ids[t] = order[t][allowed][:K]
    ids = ids.astype(np.int32)
    sel = np.take_along_axis(v, ids, axis=1)
    with np.errstate(invalid="ignore", over="ignore"):
        if renormalize:
            num = np.exp(sel - sel[:, :1])
            w = num / num.sum(axis=1, keepdims=True)
        else:
            mall = np.max(np.where(np.isnan(v), -np.inf, v), axis=1, keepdims=True)
            w = np.exp(sel - mall) / np.exp(v - mall).sum(axis=1, keepdims=True)
    return ids, w.astype(np.float32)


# ----------------------------------------------------------------------------
# Step S2: count destinations, allocate slots   [WideEP/router], [ParamCounts/dashboard]
# ----------------------------------------------------------------------------

def count_scan(topk_ids, E: int, P: int = 1):
    """Per-expert counts, exclusive offsets and the stable expert-major permutation.

    Assignment a = t*K + k goes to row
        row_of_assign[a] = offsets[id[a]] + #{a' < a : id[a'] == id[a]},
    i.e. a stable counting sort by expert; assign_of_row is its inverse.
    Partition p owns experts [p*E/P, (p+1)*E/P) ([WideEP/placement]), so its
    rows are [offsets[p*E/P], offsets[(p+1)*E/P]).
    """
    ids = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    if E % P != 0:
        raise ValueError("E must be a multiple of P")
    if ids.size and (ids.min() < 0 or ids.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.bincount(ids, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    assign_of_row = np.argsort(ids, kind="stable")
    row_of_assign = np.empty_like(assign_of_row)
    row_of_assign[assign_of_row] = np.arange(ids.size)
    epp = E // P
    part_offsets = offsets[::epp].copy()
    part_counts = np.diff(part_offsets)
    return dict(
        counts=counts,
        offsets=offsets.astype(np.int32),
        part_counts=part_counts.astype(np.int32),
        part_offsets=part_offsets.astype(np.int32),
        row_of_assign=row_of_assign.astype(np.int32),
        assign_of_row=assign_of_row.astype(np.int32),
    )


# ----------------------------------------------------------------------------
# Step S3: permute + routing metadata   [WideEP/router], [WideEP/regimes]
# ----------------------------------------------------------------------------

def permute(x_bits, row_of_assign, topk_ids, topk_w, E: int, P: int = 1):
    """xp[row_of_assign[t*K+k]] = x[t]; per-row metadata (token, slot, weight, local expert)."""
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    ids = np.asarray(topk_ids, dtype=np.int64)
    T, K = ids.shape
    roa = np.asarray(row_of_assign, dtype=np.int64).reshape(-1)
    a = np.arange(T * K)
    t = a // K
    k = a % K
    xp = np.empty((T * K, x_bits.shape[1]), dtype=np.uint16)
    xp[roa] = x_bits[t]
    epp = E // P
    e = ids.reshape(-1)
    meta_token = np.empty(T * K, np.int32)
    meta_slot = np.empty(T * K, np.int32)
    meta_w = np.empty(T * K, np.float32)
    meta_local = np.empty(T * K, np.int32)
    meta_token[roa] = t
    meta_slot[roa] = k
    meta_w[roa] = np.asarray(topk_w, dtype=np.float32).reshape(-1)
    meta_local[roa] = e - (e // epp) * epp
    return xp, dict(token=meta_token, slot=meta_slot, w=meta_w, local_expert=meta_local)


# ----------------------------------------------------------------------------
# Steps S4/S5: expert SwiGLU FFN over each expert's rows   [WideEP/router], [ParamCounts/gate]
# ----------------------------------------------------------------------------

def _silu(g):
    return g / (1.0 + np.exp(-g))


def ffn_rows(xp_rows_bits, w_gate_e_bits, w_up_e_bits, w_down_e_bits):
    """SwiGLU expert FFN of one expert for the given rows.

    g = x Wg^T, u = x Wu^T (float64), h = bf16(silu(g) * u), y = bf16(h Wd^T).
    Shapes: x [n, H]; Wg, Wu [F, H]; Wd [H, F]; all bf16 bits.  Returns (h, y) bits.
    """
    x = bf16_bits_to_f64(xp_rows_bits)
    wg = bf16_bits_to_f64(w_gate_e_bits)
    wu = bf16_bits_to_f64(w_up_e_bits)
    wd = bf16_bits_to_f64(w_down_e_bits)
    g = x @ wg.T
    u = x @ wu.T
    h_bits = f64_to_bf16_bits(_silu(g) * u)
    y_bits = f64_to_bf16_bits(bf16_bits_to_f64(h_bits) @ wd.T)
    return h_bits, y_bits


def grouped_ffn(xp_bits, offsets, w_gate_bits, w_up_bits, w_down_bits):
    """Apply expert e's FFN to rows [offsets[e], offsets[e+1]) of xp, for every e."""
    xp_bits = np.asarray(xp_bits, dtype=np.uint16)
    off = np.asarray(offsets, dtype=np.int64)
    E = off.size - 1
    rows = xp_bits.shape[0]
    F = w_gate_bits.shape[1]
    H = w_down_bits.shape[1]
    h = np.zeros((rows, F), dtype=np.uint16)
    y = np.zeros((rows, H), dtype=np.uint16)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            h[lo:hi], y[lo:hi] = ffn_rows(xp_bits[lo:hi], w_gate_bits[e], w_up_bits[e], w_down_bits[e])
    return h, y


# ----------------------------------------------------------------------------
# FP8 dispatch: E4M3 codes with one fp32 scale per row   [WideEP/bytes]
# ----------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_to_f64(codes) -> np.ndarray:
    """Value of each E4M3 code: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0;
    exponent 0 is subnormal (m * 2^-9); exponent 15 with mantissa 7 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return np.where(c & 0x80, -mag, mag)


def f32_to_e4m3(v) -> np.ndarray:
    """Nearest E4M3 code of each fp32 value (ties to an even mantissa), saturating to +-448
    (infinities included); NaN gives 0x7F."""
    v32 = np.asarray(v, dtype=np.float32)
    finite = np.isfinite(v32)
    a = np.where(finite, np.abs(v32).astype(np.float64), 0.0)
    frac, ex = np.frexp(a)                       # a = frac * 2^ex, frac in [0.5, 1)
    unb = ex.astype(np.int64) - 1                # a = (2 frac) * 2^unb
    q = np.rint((2.0 * frac - 1.0) * 8.0)        # mantissa steps, ties to even
    carry = q == 8.0
    unb = np.where(carry, unb + 1, unb)
    q = np.where(carry, 0.0, q)
    normal_code = (unb + 7) * 8 + q.astype(np.int64)
    sub_code = np.rint(np.minimum(a, 2.0 ** -6) / 2.0 ** -9).astype(np.int64)  # 8 steps of 2^-9 = code 8, the smallest normal
    mag = np.where(a >= 2.0 ** -6, normal_code, sub_code)
    mag = np.minimum(np.where(finite, mag, 0x7E), 0x7E)   # 0x7E = 448; anything larger saturates
    mag = np.where(np.isnan(v32), 0x7F, mag)
    sign = np.where(np.signbit(v32) & ~np.isnan(v32), 0x80, 0)
    return (mag | sign).astype(np.uint8)


def quantize_rows_fp8(x_bits):
    """Per-row E4M3 quantization of bf16 rows: (codes uint8 [R][C], scales fp32 [R]).
    s = fp32(amax) / 448 in fp32 (1 for an all-zero row); code = f32_to_e4m3(fp32(x) / s)."""
    x = bf16_bits_to_f64(x_bits).astype(np.float32)          # exact
    amax = np.abs(x).max(axis=-1) if x.shape[-1] else np.zeros(x.shape[:-1], np.float32)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = f32_to_e4m3((x / s[..., None]).astype(np.float32))
    return q, s


def dispatch_fp8(z_bits, row_of_assign, K: int):
    """FP8 dispatch buffer: every token quantized once, its codes and scale placed at the
    rows of its K assignments (xq[row_of_assign[t*K+k]] = q[t], xs[...] = s[t])."""
    q, s = quantize_rows_fp8(z_bits)
    T = q.shape[0]
    roa = np.asarray(row_of_assign, dtype=np.int64).reshape(-1)
    t = np.arange(T * K) // K
    xq = np.empty((T * K, q.shape[1]), dtype=np.uint8)
    xs = np.empty(T * K, dtype=np.float32)
    xq[roa] = q[t]
    xs[roa] = s[t]
    return xq, xs


def quantize_experts_fp8(w_bits):
    """Gate or up weights [E][F][H] quantized per output feature: codes [E][F][H], scales [E][F]."""
    w = np.asarray(w_bits, dtype=np.uint16)
    q, s = quantize_rows_fp8(w.reshape(-1, w.shape[-1]))
    return q.reshape(w.shape), s.reshape(w.shape[:-1])


def ffn_rows_fp8(xq, xs, wg_q, wg_s, wu_q, wu_s, w_down_e_bits):
    """SwiGLU expert FFN on E4M3 rows: g = s_x s_wg (q_x q_wg^T), u likewise (float64),
    h = bf16(silu(g) * u), y = bf16(h Wd^T) with bf16 Wd.  Returns (h, y) bits."""
    x = e4m3_to_f64(xq)
    sx = np.asarray(xs, dtype=np.float32).astype(np.float64)[:, None]
    g = (x @ e4m3_to_f64(wg_q).T) * sx * np.asarray(wg_s, np.float32).astype(np.float64)[None, :]
    u = (x @ e4m3_to_f64(wu_q).T) * sx * np.asarray(wu_s, np.float32).astype(np.float64)[None, :]
    h_bits = f64_to_bf16_bits(_silu(g) * u)
    y_bits = f64_to_bf16_bits(bf16_bits_to_f64(h_bits) @ bf16_bits_to_f64(w_down_e_bits).T)
    return h_bits, y_bits


def grouped_ffn_fp8(xq, xs, offsets, wg_q, wg_s, wu_q, wu_s, w_down_bits):
    """ffn_rows_fp8 of expert e on rows [offsets[e], offsets[e+1]), for every e."""
    off = np.asarray(offsets, dtype=np.int64)
    rows, F, H = xq.shape[0], wg_q.shape[1], w_down_bits.shape[1]
    h = np.zeros((rows, F), dtype=np.uint16)
    y = np.zeros((rows, H), dtype=np.uint16)
    for e in range(off.size - 1):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            h[lo:hi], y[lo:hi] = ffn_rows_fp8(xq[lo:hi], xs[lo:hi], wg_q[e], wg_s[e], wu_q[e], wu_s[e],
                                              w_down_bits[e])
    return h, y


def dispatch_bytes_fp8(T: int, K: int, H: int) -> int:
    """FP8 dispatch payload: T K H one-byte codes plus one 4-byte scale per dispatched row."""
    return T * K * H + 4 * T * K


# ----------------------------------------------------------------------------
# Step S6: combine = unpermute + weighted sum   [WideEP/router], [WideEP/bytes]
# ----------------------------------------------------------------------------

def combine(y_bits, row_of_assign, topk_w, shared_bits=None):
    """out[t] = bf16( sum_{k<K} w[t,k] * y[row_of_assign[t*K+k]] (+ s[t]) ), summed in slot order;
    s is the shared expert's output when given."""
    w = np.asarray(topk_w, dtype=np.float32).astype(np.float64)
    T, K = w.shape
    y = bf16_bits_to_f64(y_bits)
    roa = np.asarray(row_of_assign, dtype=np.int64).reshape(T, K)
    acc = np.zeros((T, y.shape[1]), dtype=np.float64)
    if shared_bits is not None:
        acc = acc + bf16_bits_to_f64(shared_bits)
    for k in range(K):
        acc = acc + w[:, k:k + 1] * y[roa[:, k]]
    return f64_to_bf16_bits(acc)


# ----------------------------------------------------------------------------
# Step S7: skew statistics   [ParamCounts/dashboard]
# ----------------------------------------------------------------------------

def skew_ratio(counts) -> float:
    """max expert load / mean expert load, mean = (sum of counts) / E."""
    c = np.asarray(counts, dtype=np.float64)
    total = c.sum()
    if total == 0:
        return 0.0
    return float(c.max() / (total / c.size))


def p95_nearest_rank(values) -> float:
    """95th percentile by nearest rank: the ceil(0.95 n)-th smallest value."""
    v = np.sort(np.asarray(values, dtype=np.float64))
    if v.size == 0:
        return float("nan")
    r = max(1, math.ceil(0.95 * v.size))
    return float(v[r - 1])


# ----------------------------------------------------------------------------
# Step S8: latent projections   [LatentMoE]
# ----------------------------------------------------------------------------

def dense_bf16(x_bits, w_bits):
    """bf16( x W^T ) with nn.Linear layout: x [T, D_in], W [D_out, D_in]."""
    return f64_to_bf16_bits(bf16_bits_to_f64(x_bits) @ bf16_bits_to_f64(w_bits).T)


# ----------------------------------------------------------------------------
# Whole layer
# ----------------------------------------------------------------------------

def layer_forward(x_bits, w_g, w_gate_bits, w_up_bits, w_down_bits, K: int, P: int = 1,
                  renormalize: bool = True, bias=None, w_dp_bits=None, w_upp_bits=None,
                  logits=None, group_limit: int = 0, shared=None, fp8: bool = False):
    """All steps in pipeline order.  Returns a dict with every intermediate.

    ``shared`` = (W_gate_s [Fs][d], W_up_s [Fs][d], W_down_s [d][Fs]) bf16 bits adds a shared
    expert on the routed activations (x, or z for a latent layer).

    If ``logits`` is given it replaces the oracle's own gating output (used by
    the routing tests, which hand both sides the same float32 logits).

    ``fp8`` dispatches E4M3 codes with per-token scales and runs gate/up on E4M3 weights
    quantized per output feature (results "xq", "xs", "wg_q", "wg_s", "wu_q", "wu_s").
    """
    res = {}
    z = x_bits
    if w_dp_bits is not None:
        z = dense_bf16(x_bits, w_dp_bits)
        res["z"] = z
    l = gating_logits(z, w_g, bias) if logits is None else np.asarray(logits, np.float32)
    res["logits"] = l
    E = l.shape[1]
    if group_limit:
        ids, w = route_limited(l, K, P, group_limit, renormalize)
    else:
        ids, w = route(l, K, renormalize)
    res["topk_ids"], res["topk_w"] = ids, w
    cs = count_scan(ids, E, P)
    res.update(cs)
    xp, meta = permute(z, cs["row_of_assign"], ids, w, E, P)
    res["xp"] = xp
    res["meta"] = meta
    if fp8:
        xq, xs = dispatch_fp8(z, cs["row_of_assign"], K)
        wg_q, wg_s = quantize_experts_fp8(w_gate_bits)
        wu_q, wu_s = quantize_experts_fp8(w_up_bits)
        res.update(xq=xq, xs=xs, wg_q=wg_q, wg_s=wg_s, wu_q=wu_q, wu_s=wu_s)
        h, y = grouped_ffn_fp8(xq, xs, cs["offsets"], wg_q, wg_s, wu_q, wu_s, w_down_bits)
    else:
        h, y = grouped_ffn(xp, cs["offsets"], w_gate_bits, w_up_bits, w_down_bits)
    res["h"], res["y"] = h, y
    s_bits = None
    if shared is not None:
        res["h_shared"], s_bits = ffn_rows(z, *shared)
        res["y_shared"] = s_bits
    out = combine(y, cs["row_of_assign"], w, s_bits)
    res["out"] = out
    if w_upp_bits is not None:
        res["final"] = dense_bf16(out, w_upp_bits)
    res["skew"] = skew_ratio(cs["counts"])
    return res


# ----------------------------------------------------------------------------
# Sizing identities   [WideEP/bytes], [ParamCounts/network], [WideEP/placement]
# ----------------------------------------------------------------------------

def dispatch_bytes(T: int, K: int, H: int, b: int) -> int:
    """Activation bytes one dispatch moves with no padding: T x K x H x b."""
    return T * K * H * b


def expert_weight_bytes(E: int, H: int, F: int, b: int) -> int:
    """Bytes of E SwiGLU experts (gate, up: H x F each; down: F x H)."""
    return 3 * H * F * E * b


def experts_per_partition(E: int, P: int) -> int:
    """Experts owned by each of P evenly placed partitions."""
    if E % P:
        raise ValueError("E must be a multiple of P")
    return E // P


def checkpoint_bytes(params: float, b: int) -> float:
    """Total parameters x bytes per parameter."""
    return params * b
