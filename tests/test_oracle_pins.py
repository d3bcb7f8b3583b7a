"""Pins of the CPU oracle to facts fixed outside itself (CPU only).

Each test checks the oracle against a closed form, an invariant the pages state,
brute force on tiny inputs, an independent library routine, or a figure the
pages print (tests/golden/).  A plausible slip in the oracle (a dropped term, a
swapped operand, a wrong index, a missed rounding point) fails one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from routing_dispatch_grouped_top_b200 import inputs
from routing_dispatch_grouped_top_b200.config import DEEPSEEK_R1_DECODE, TINY

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf(vals):
    return oracle.f64_to_bf16_bits(np.asarray(vals, dtype=np.float64))


def val(bits):
    return oracle.bf16_bits_to_f64(bits)


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------

def test_bf16_rounding_hand_values():
    # 1 + 2^-8 is the midpoint of 1.0 and 1.0078125: ties go to the even pattern 0x3F80.
    assert bf([1.0 + 2 ** -8])[0] == 0x3F80
    assert bf([1.0 + 3 * 2 ** -8])[0] == 0x3F82       # midpoint of 0x3F81/0x3F82 -> even
    assert bf([1.0 + 1.5 * 2 ** -8])[0] == 0x3F81
    assert bf([-2.0])[0] == 0xC000
    assert bf([65504.0])[0] == 0x4780                  # rounds up to 65536
    assert bf([3 * 2.0 ** -133])[0] == 0x0003          # subnormal spacing 2^-133
    assert bf([np.inf])[0] == 0x7F80 and bf([-np.inf])[0] == 0xFF80


def test_bf16_rounding_matches_torch_on_float32_values():
    # Every float32 value is exact in float64, so direct f64->bf16 rounding must
    # agree with torch's float32->bf16 conversion (an independent implementation).
    g = torch.Generator().manual_seed(0)
    f = torch.cat([torch.randn(200000, generator=g) * 10.0 ** torch.randint(-30, 30, (200000,), generator=g),
                   torch.tensor([0.0, -0.0, 1e-40, -3e-39, 3.3e38])]).to(torch.float32)
    ref = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = bf(f.numpy().astype(np.float64))
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------------------
# S0 gating logits
# ---------------------------------------------------------------------------

def test_logits_one_hot_rows_select_router_rows():
    H, E = 16, 5
    w_g = np.random.default_rng(1).standard_normal((H, E)).astype(np.float32)
    x = np.zeros((H, H)); x[np.arange(H), np.arange(H)] = 1.0
    l = oracle.gating_logits(bf(x), w_g)
    assert np.array_equal(l, w_g)                      # row h of W_g, not a column
    bias = np.arange(E, dtype=np.float32) * 0.25
    lb = oracle.gating_logits(bf(x), w_g, bias)
    assert np.array_equal(lb, (w_g + bias).astype(np.float32))


def test_logits_exact_small_integer_sum():
    x = bf([[1.0, 2.0, -3.0]])
    w_g = np.array([[1.0, 0.5], [2.0, 0.25], [1.0, -1.0]], np.float32)
    assert np.array_equal(oracle.gating_logits(x, w_g), np.array([[2.0, 4.0]], np.float32))


# ---------------------------------------------------------------------------
# S1 top-k selection (brute force over all subsets) and weights (closed forms)
# ---------------------------------------------------------------------------

def _beats(va, a, vb, b):
    """a ranks above b: larger value; equal values -> lower id; NaN below all."""
    na, nb = math.isnan(va), math.isnan(vb)
    if na or nb:
        if na and nb:
            return a < b
        return nb
    if va != vb:
        return va > vb
    return a < b


def _brute_topk(row, K):
    E = len(row)
    winners = []
    for S in itertools.combinations(range(E), K):
        rest = [j for j in range(E) if j not in S]
        if all(_beats(row[i], i, row[j], j) for i in S for j in rest):
            winners.append(S)
    assert len(winners) == 1
    S = list(winners[0])
    # order inside the set: best first (insertion sort with the same relation)
    out = []
    for i in S:
        pos = 0
        while pos < len(out) and _beats(row[out[pos]], out[pos], row[i], i):
            pos += 1
        out.insert(pos, i)
    return out


@pytest.mark.parametrize("gen", ["random", "quantized", "special"])
@pytest.mark.parametrize("E,K", [(5, 2), (7, 3), (8, 8), (8, 1), (6, 4)])
def test_topk_matches_brute_force(gen, E, K):
    T = 40
    if gen == "random":
        l = inputs.random_logits(T, E, seed=E * 10 + K)
    elif gen == "quantized":
        l = inputs.quantized_logits(T, E, levels=3, seed=E * 10 + K)
    else:
        l = inputs.special_logits(T, E, seed=E * 10 + K)
    l = l.numpy()
    ids, _ = oracle.route(l, K)
    for t in range(T):
        assert list(ids[t]) == _brute_topk([float(v) for v in l[t]], K), (t, l[t])


def test_topk_all_equal_logits_gives_lowest_ids():
    ids, w = oracle.route(np.full((3, 9), 0.5, np.float32), 4)
    assert (ids == np.arange(4)).all()
    assert np.allclose(w, 0.25, atol=0)


def test_topk_signed_zero_is_a_tie():
    l = np.array([[-0.0, 0.0, -1.0]], np.float32)
    ids, _ = oracle.route(l, 1)
    assert ids[0, 0] == 0                              # -0.0 == +0.0 -> lower id


def test_weights_closed_form_renormalised():
    # logits ln1, ln2, ln3 (+ a loser): renormalised top-3 weights are 3/6, 2/6, 1/6.
    l = np.array([[0.0, math.log(2.0), math.log(3.0), -50.0]], np.float32)
    ids, w = oracle.route(l, 3, renormalize=True)
    assert list(ids[0]) == [2, 1, 0]
    e = np.exp(l[0, [2, 1, 0]].astype(np.float64))
    assert np.allclose(w[0], [0.5, 1 / 3, 1 / 6], atol=2e-7)
    assert abs(float(w.sum()) - 1.0) < 1e-6
    assert e[0] > e[1] > e[2]


def test_weights_closed_form_plain_softmax():
    # logits ln1..ln4, K = 2 without renormalising: weights 4/10 and 3/10.
    l = np.log(np.array([[1.0, 2.0, 3.0, 4.0]])).astype(np.float32)
    ids, w = oracle.route(l, 2, renormalize=False)
    assert list(ids[0]) == [3, 2]
    assert np.allclose(w[0], [0.4, 0.3], atol=2e-7)


def test_weights_sum_to_one_and_K_equal_E_is_full_softmax_order():
    l = inputs.random_logits(64, 12, seed=3).numpy()
    ids, w = oracle.route(l, 12)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6)
    for t in range(64):
        assert sorted(ids[t]) == list(range(12))       # K = E selects every expert
        assert np.all(np.diff(w[t]) <= 0)              # weights follow the slot order
    # K = E with renormalisation equals the plain softmax over E (same weights).
    _, w2 = oracle.route(l, 12, renormalize=False)
    assert np.allclose(w, w2, atol=1e-7)


# ---------------------------------------------------------------------------
# S2 counting / scan / permutation
# ---------------------------------------------------------------------------

def _count_definition(ids_flat, E):
    """Row of each assignment straight from the counting definition, in loops."""
    counts = [0] * E
    for e in ids_flat:
        counts[e] += 1
    off = [0]
    for c in counts:
        off.append(off[-1] + c)
    seen = [0] * E
    rows = []
    for e in ids_flat:
        rows.append(off[e] + seen[e])
        seen[e] += 1
    return counts, off, rows


@pytest.mark.parametrize("T,E,K,P,zipf", [(37, 8, 2, 2, None), (64, 16, 4, 4, 1.1), (5, 32, 3, 8, None),
                                          (1, 4, 4, 1, None), (100, 6, 1, 3, 2.0)])
def test_count_scan_matches_counting_definition(T, E, K, P, zipf):
    ids = inputs.random_topk_ids(T, E, K, seed=T + E, zipf_s=zipf).numpy()
    cs = oracle.count_scan(ids, E, P)
    counts, off, rows = _count_definition(list(ids.reshape(-1)), E)
    assert list(cs["counts"]) == counts
    assert list(cs["offsets"]) == off
    assert list(cs["row_of_assign"]) == rows
    # invariants: counts sum to T*K (every token contributes K rows)
    assert cs["counts"].sum() == T * K and cs["offsets"][-1] == T * K
    # bijection
    roa, aor = cs["row_of_assign"], cs["assign_of_row"]
    assert np.array_equal(aor[roa], np.arange(T * K)) and np.array_equal(roa[aor], np.arange(T * K))
    # partitions: part_offsets[p] = offsets[p*E/P]; rows of partition p hold its experts
    epp = E // P
    assert np.array_equal(cs["part_offsets"], cs["offsets"][::epp])
    flat = ids.reshape(-1)
    for p in range(P):
        lo, hi = cs["part_offsets"][p], cs["part_offsets"][p + 1]
        assert cs["part_counts"][p] == hi - lo
        e_rows = flat[aor[lo:hi]]
        assert np.all((e_rows >= p * epp) & (e_rows < (p + 1) * epp))


def test_rows_per_token_figure():
    fig = json.load(open(os.path.join(GOLDEN, "sizing_figures.json")))["rows_per_token"]
    ids = inputs.random_topk_ids(50, 8, fig["K"], seed=5).numpy()
    cs = oracle.count_scan(ids, 8)
    assert cs["counts"].sum() == 50 * fig["rows_per_token"]


# ---------------------------------------------------------------------------
# S3 permute
# ---------------------------------------------------------------------------

def test_permute_roundtrip_bytes_and_metadata():
    T, H, E, K, P = 29, 24, 8, 3, 4
    x = inputs.to_bits(inputs.random_bf16((T, H), seed=1))
    ids = inputs.random_topk_ids(T, E, K, seed=2).numpy()
    w = inputs.random_weights(T, K, seed=3).numpy()
    cs = oracle.count_scan(ids, E, P)
    xp, meta = oracle.permute(x, cs["row_of_assign"], ids, w, E, P)
    # dispatch bytes = T x K x H x b, no padding
    assert xp.nbytes == oracle.dispatch_bytes(T, K, H, 2) == T * K * H * 2
    # unpermute(permute(x)) = x for every slot
    roa = cs["row_of_assign"].reshape(T, K)
    for k in range(K):
        assert np.array_equal(xp[roa[:, k]], x)
    # metadata reproduces the route
    assert np.array_equal(xp, x[meta["token"]])
    assert np.array_equal(ids[meta["token"], meta["slot"]] % (E // P), meta["local_expert"])
    assert np.array_equal(w[meta["token"], meta["slot"]], meta["w"])
    # rows are expert-contiguous: expert of row r is non-decreasing
    e_of_row = ids[meta["token"], meta["slot"]]
    assert np.all(np.diff(e_of_row) >= 0)


# ---------------------------------------------------------------------------
# S4/S5 SwiGLU expert FFN (closed forms on structured weights)
# ---------------------------------------------------------------------------

def _sel(rows, cols, pairs, scale=1.0):
    w = np.zeros((rows, cols))
    for r, c in pairs:
        w[r, c] = scale
    return bf(w)


def test_ffn_silu_known_value_and_rounding_points():
    # x = [1, 1]; gate selects x0, up selects x1 -> a = silu(1) * 1 = sigma(1).
    # sigma(1) = 0.7310585786300049 (logistic at 1); bf16 -> 0.73046875.
    x = bf([[1.0, 1.0]])
    wg = _sel(1, 2, [(0, 0)])
    wu = _sel(1, 2, [(0, 1)])
    wd = bf([[1.0078125], [1.0]])                    # W_down [H=2][F=1]
    h, y = oracle.ffn_rows(x, wg, wu, wd)
    assert val(h)[0, 0] == 0.73046875
    # y rounds h to bf16 first: 0.73046875 * 1.0078125 = 0.7361755... -> 0.734375.
    # (Rounding only once, sigma(1) * 1.0078125 = 0.73677... would give 0.73828125.)
    assert val(y)[0, 0] == 0.734375 and val(y)[0, 1] == 0.73046875


def test_ffn_silu_odd_part_identity_and_gate_up_order():
    # silu(v) - silu(-v) = v exactly in real arithmetic; with u = 1 the rows for x and -x
    # give h(v) - h(-v) = v up to two bf16 roundings.  With gate <-> up swapped the
    # second row below would be silu(1)*4 instead of silu(4)*1.
    v = np.array([0.5, 1.5, 3.0, 6.0, 0.0])
    x = bf(np.stack([np.concatenate([v, [1.0]]), np.concatenate([-v, [1.0]])]))
    H = 6
    wg = _sel(5, H, [(i, i) for i in range(5)])
    wu = _sel(5, H, [(i, 5) for i in range(5)])
    wd = _sel(H, 5, [(i, i) for i in range(5)])
    h, _ = oracle.ffn_rows(x, wg, wu, wd)
    hv = val(h)
    assert np.all(np.abs((hv[0] - hv[1]) - v) <= 2 ** -7 * np.maximum(np.abs(v), 1))
    assert hv[0, 4] == 0.0
    # order check: gate = 4, up = 1 vs gate = 1, up = 4
    x2 = bf([[4.0, 1.0]])
    h2, _ = oracle.ffn_rows(x2, _sel(1, 2, [(0, 0)]), _sel(1, 2, [(0, 1)]), _sel(2, 1, [(0, 0)]))
    # silu(4) = 4 * sigma(4) with sigma(4) in (0.98, 0.99); silu(1)*4 would be ~2.92
    assert 3.9 < val(h2)[0, 0] < 3.96


def test_ffn_transposition_non_square():
    # H = 3, F = 2: gate row f reads x[(f+1) % 3], up row f reads x[f]; down maps h_f -> y_{2-f}.
    x = bf([[2.0, -1.0, 0.5]])
    wg = _sel(2, 3, [(0, 1), (1, 2)], scale=0.0)        # gate = 0 -> silu(0) = 0 everywhere
    wu = _sel(2, 3, [(0, 0), (1, 1)])
    wd = _sel(3, 2, [(2, 0), (1, 1)])
    h, y = oracle.ffn_rows(x, wg, wu, wd)
    assert np.all(val(h) == 0.0) and np.all(val(y) == 0.0)
    big = 16.0                                          # silu(16) = 16 * (1 - 1.1e-7) -> bf16 16
    x = bf([[big, big, big]])
    wu = _sel(2, 3, [(0, 0), (1, 1)], scale=0.5)        # u = 8 for both features
    wg = _sel(2, 3, [(0, 1), (1, 2)])                  # g = 16
    wd = _sel(3, 2, [(2, 0), (1, 1)], scale=0.25)
    h, y = oracle.ffn_rows(x, wg, wu, wd)
    assert np.array_equal(val(h), [[128.0, 128.0]])
    assert np.array_equal(val(y), [[0.0, 32.0, 32.0]])  # output 0 gets nothing: Wd[0,:] = 0


def test_grouped_ffn_uses_each_experts_weights_on_its_rows():
    E, H, F = 4, 2, 1
    counts = [3, 0, 2, 1]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    xp = bf(np.full((6, H), 16.0))
    wg = np.stack([_sel(F, H, [(0, 0)]) for _ in range(E)])
    wu = np.stack([_sel(F, H, [(0, 1)], scale=e + 1.0) for e in range(E)])
    wd = np.stack([_sel(H, F, [(0, 0)]) for _ in range(E)])
    h, y = oracle.grouped_ffn(xp, off, wg, wu, wd)
    expect = [16.0 * 16 * 1] * 3 + [16.0 * 16 * 3] * 2 + [16.0 * 16 * 4]
    assert np.array_equal(val(h)[:, 0], expect)
    assert np.array_equal(val(y)[:, 0], expect) and np.all(val(y)[:, 1] == 0)


# ---------------------------------------------------------------------------
# S6 combine
# ---------------------------------------------------------------------------

def test_combine_identity_experts_returns_x():
    # Identity experts (y = xp): combine gives (sum_k w) * x = x when renormalised.
    T, H, E, K = 33, 40, 8, 4
    x = inputs.to_bits(inputs.random_bf16((T, H), seed=11))
    l = inputs.random_logits(T, E, seed=12).numpy()
    ids, w = oracle.route(l, K, renormalize=True)
    cs = oracle.count_scan(ids, E)
    xp, _ = oracle.permute(x, cs["row_of_assign"], ids, w, E)
    out = oracle.combine(xp, cs["row_of_assign"], w)
    assert np.array_equal(out, x)
    # without renormalisation: out = bf16(sum_k w * x)
    ids2, w2 = oracle.route(l, K, renormalize=False)
    cs2 = oracle.count_scan(ids2, E)
    xp2, _ = oracle.permute(x, cs2["row_of_assign"], ids2, w2, E)
    out2 = val(oracle.combine(xp2, cs2["row_of_assign"], w2))
    s = w2.astype(np.float64).sum(axis=1, keepdims=True)
    assert np.allclose(out2, val(x) * s, rtol=2 ** -8, atol=0)


def test_combine_weighted_slots_closed_form():
    y = bf([[1.0, 2.0], [4.0, 8.0], [16.0, 32.0]])
    roa = np.array([2, 0, 1, 2], np.int32)           # token 0 -> rows 2,0; token 1 -> rows 1,2
    w = np.array([[0.25, 0.75], [0.5, 0.125]], np.float32)
    out = val(oracle.combine(y, roa, w))
    assert np.array_equal(out, [[0.25 * 16 + 0.75 * 1, 0.25 * 32 + 0.75 * 2],
                                [0.5 * 4 + 0.125 * 16, 0.5 * 8 + 0.125 * 32]])


# ---------------------------------------------------------------------------
# S7 skew statistics
# ---------------------------------------------------------------------------

def test_skew_ratio_and_p95():
    assert oracle.skew_ratio([4, 4, 4, 4]) == 1.0
    assert oracle.skew_ratio([16, 0, 0, 0]) == 4.0
    assert oracle.skew_ratio([3, 1, 0, 0]) == 3.0
    assert oracle.skew_ratio([0, 0]) == 0.0
    assert oracle.p95_nearest_rank(np.arange(1, 101)) == 95.0
    assert oracle.p95_nearest_rank(np.arange(20, 0, -1)) == 19.0
    assert oracle.p95_nearest_rank([7.0]) == 7.0


def test_zipf_decode_workload_reaches_p95_skew_4():
    # The skewed decode router is calibrated to a p95 max/mean load near 4.
    cfg = DEEPSEEK_R1_DECODE
    w_g, bias = inputs.make_router(cfg)
    ratios = []
    for s in range(64):
        l = oracle.gating_logits(inputs.to_bits(inputs.make_tokens(cfg, "cpu", s)), w_g.numpy(), bias.numpy())
        ids, _ = oracle.route(l, cfg.K)
        ratios.append(oracle.skew_ratio(oracle.count_scan(ids, cfg.E)["counts"]))
    assert 3.75 <= oracle.p95_nearest_rank(ratios) <= 4.25


# ---------------------------------------------------------------------------
# S8 latent projections
# ---------------------------------------------------------------------------

def test_dense_projection_layout():
    x = bf([[1.0, 2.0, 3.0, 4.0]])
    w = _sel(2, 4, [(0, 3), (1, 0)], scale=0.5)       # [D_out=2][D_in=4]
    assert np.array_equal(val(oracle.dense_bf16(x, w)), [[2.0, 0.5]])


def test_layer_forward_tiny_is_consistent():
    cfg = TINY
    d = inputs.make_layer(cfg)
    r = oracle.layer_forward(inputs.to_bits(d["x"]), d["w_g"].numpy(), inputs.to_bits(d["w_gate"]),
                             inputs.to_bits(d["w_up"]), inputs.to_bits(d["w_down"]), cfg.K, cfg.P)
    assert r["counts"].sum() == cfg.TK
    assert r["xp"].shape == (cfg.TK, cfg.H) and r["out"].shape == (cfg.T, cfg.H)
    # row-by-row evaluation of one token equals the grouped evaluation
    t = 5
    acc = np.zeros(cfg.H)
    for k in range(cfg.K):
        e = r["topk_ids"][t, k]
        _, yk = oracle.ffn_rows(inputs.to_bits(d["x"])[t:t + 1], inputs.to_bits(d["w_gate"][e]),
                                inputs.to_bits(d["w_up"][e]), inputs.to_bits(d["w_down"][e]))
        acc += float(r["topk_w"][t, k]) * val(yk)[0]
    assert np.array_equal(oracle.f64_to_bf16_bits(acc), r["out"][t])


def test_latent_layer_routes_and_dispatches_z_and_projects_the_combined_output():
    # "Latent MoE" (Definition, Current Synthesis): the experts see the narrower projected state z.
    # With a permutation W_dp (not an involution), z = x[:, perm] exactly: the router must rank
    # z W_g (routing on x gives other experts here) and the dispatched rows must be rows of z.
    # With W_upp rows that add two columns of their input, final = bf16(out[:, a] + out[:, b]) of
    # the combined output (one rounding); a projection applied to the expert rows before the
    # combine rounds differently somewhere.
    rng = np.random.default_rng(5)
    T, D, E, K, F = 64, 8, 6, 2, 16
    x = bf(rng.standard_normal((T, D)))
    perm = np.array([3, 0, 6, 1, 7, 2, 5, 4])
    w_dp = np.zeros((D, D))
    w_dp[np.arange(D), perm] = 1.0
    w_g = rng.standard_normal((D, E)).astype(np.float32)
    wg = bf(rng.standard_normal((E, F, D)) * 0.5)
    wu = bf(rng.standard_normal((E, F, D)) * 0.5)
    wd = bf(rng.standard_normal((E, D, F)) * 0.25)
    a_idx, b_idx = np.arange(D), (np.arange(D) + 3) % D
    w_upp = np.zeros((D, D))
    w_upp[np.arange(D), a_idx] = 1.0
    w_upp[np.arange(D), b_idx] = 1.0
    r = oracle.layer_forward(x, w_g, wg, wu, wd, K, 1, w_dp_bits=bf(w_dp), w_upp_bits=bf(w_upp))
    z = x[:, perm]
    assert np.array_equal(r["z"], z)

    def topk_by_definition(l):
        return np.array([sorted(range(E), key=lambda e: (-float(l[t, e]), e))[:K] for t in range(T)])

    want = topk_by_definition((val(z) @ w_g.astype(np.float64)).astype(np.float32))
    assert np.array_equal(r["topk_ids"], want)
    assert not np.array_equal(topk_by_definition((val(x) @ w_g.astype(np.float64)).astype(np.float32)), want)
    roa = r["row_of_assign"].reshape(T, K)
    for t in range(T):
        for k in range(K):
            assert np.array_equal(r["xp"][roa[t, k]], z[t])
    out = val(r["out"])
    assert np.array_equal(r["final"], bf(out[:, a_idx] + out[:, b_idx]))
    y, w = val(r["y"]), r["topk_w"].astype(np.float64)
    early = np.zeros((T, D))
    for t in range(T):
        for k in range(K):
            row = y[roa[t, k]]
            early[t] += w[t, k] * val(bf(row[a_idx] + row[b_idx]))
    assert not np.array_equal(bf(early), r["final"])


# ---------------------------------------------------------------------------
# Figures the pages print
# ---------------------------------------------------------------------------

def test_sizing_figures_from_pages():
    g = json.load(open(os.path.join(GOLDEN, "sizing_figures.json")))
    c = g["checkpoint"]
    nbytes = oracle.checkpoint_bytes(c["params"], c["bytes_per_param"])
    assert nbytes / 1e9 == pytest.approx(c["bytes_decimal_GB"])
    assert round(nbytes / 2 ** 30, 1) == c["GiB"]
    for row in g["experts_per_partition"]:
        assert oracle.experts_per_partition(row["E"], row["P"]) == row["per_partition"]
    a = g["activated_share"]
    assert round(100.0 * a["K"] / a["E"], 1) == a["percent"]
    u = g["unselected_experts"]
    assert u["E"] - u["K"] == u["unselected"]
    cs = g["cold_share_ep8"]
    assert 100.0 * (cs["local_experts"] - cs["K"]) / cs["local_experts"] == cs["cold_percent"]
    th = g["topk_halving"]
    assert oracle.dispatch_bytes(4096, th["K_to"], 2048, 2) / oracle.dispatch_bytes(4096, th["K_from"], 2048, 2) == th["ratio"]


# ---------------------------------------------------------------------------
# Node-limited routing (a variant of S1)
# ---------------------------------------------------------------------------

def _brute_limited(row, K, P, M):
    """Every choice of M groups, every K-subset of their experts: the selection is the
    unique K-set that beats every other expert of the kept groups, where the kept groups
    are the M whose best experts beat the best experts of the others."""
    E = len(row)
    epp = E // P

    def best(g):
        b = g * epp
        for j in range(g * epp, (g + 1) * epp):
            if _beats(row[j], j, row[b], b):
                b = j
        return b

    bests = [best(g) for g in range(P)]
    kept = None
    for G in itertools.combinations(range(P), M):
        rest = [g for g in range(P) if g not in G]
        if all(_beats(row[bests[a]], bests[a], row[bests[b]], bests[b]) for a in G for b in rest):
            assert kept is None
            kept = G
    allowed = [j for j in range(E) if j // epp in kept]
    return sorted_topk(row, allowed, K)


def sorted_topk(row, allowed, K):
    out = []
    for i in allowed:
        pos = 0
        while pos < len(out) and _beats(row[out[pos]], out[pos], row[i], i):
            pos += 1
        out.insert(pos, i)
    return out[:K]


@pytest.mark.parametrize("gen", ["random", "quantized", "special"])
@pytest.mark.parametrize("E,P,M,K", [(8, 4, 2, 3), (12, 6, 1, 2), (9, 3, 2, 4), (8, 8, 3, 3), (6, 2, 2, 5)])
def test_route_limited_matches_brute_force(gen, E, P, M, K):
    T = 30
    l = {"random": inputs.random_logits, "quantized": lambda T, E, seed: inputs.quantized_logits(T, E, 3, seed),
         "special": inputs.special_logits}[gen](T, E, seed=E * P + M).numpy()
    ids, _ = oracle.route_limited(l, K, P, M)
    for t in range(T):
        assert list(ids[t]) == _brute_limited([float(v) for v in l[t]], K, P, M), (t, l[t])


def test_route_limited_special_cases():
    l = inputs.random_logits(50, 16, seed=4).numpy()
    # all groups kept -> plain top-K
    assert np.array_equal(oracle.route_limited(l, 5, 4, 4)[0], oracle.route(l, 5)[0])
    # one expert per group and M >= K -> plain top-K
    assert np.array_equal(oracle.route_limited(l, 3, 16, 5)[0], oracle.route(l, 3)[0])
    # M = 1: all K experts in one group (the group of the best expert)
    ids, w = oracle.route_limited(l, 3, 4, 1)
    best = oracle.route(l, 1)[0][:, 0]
    assert np.all(ids // 4 == (best // 4)[:, None])
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6)
    # hand example: groups {0,1} {2,3} {4,5}; best group is {4,5} (logit 9); then {0,1} (5)
    row = np.array([[5.0, 1.0, 4.0, 4.5, 9.0, 0.0]], np.float32)
    ids, _ = oracle.route_limited(row, 3, 3, 2)
    assert list(ids[0]) == [4, 0, 1]          # 3 and 2 are excluded although 4.5 > 1.0


# ---------------------------------------------------------------------------
# Shared expert (added in the combine)
# ---------------------------------------------------------------------------

def test_combine_with_shared_expert_closed_form():
    y = bf([[1.0, 2.0], [4.0, 8.0]])
    roa = np.array([1, 0], np.int32)                # token 0 -> rows 1, 0
    w = np.array([[0.25, 0.75]], np.float32)
    s = bf([[0.5, -6.0]])
    out = val(oracle.combine(y, roa, w, s))
    assert np.array_equal(out, [[0.25 * 4 + 0.75 * 1 + 0.5, 0.25 * 8 + 0.75 * 2 - 6.0]])


def test_layer_shared_expert_is_a_dense_swiglu_added_to_every_token():
    cfg = TINY
    d = inputs.make_layer(cfg)
    xs = inputs.to_bits(d["x"])
    args = (xs, d["w_g"].numpy(), inputs.to_bits(d["w_gate"]), inputs.to_bits(d["w_up"]),
            inputs.to_bits(d["w_down"]), cfg.K, cfg.P)
    Fs = 64
    sh = (inputs.to_bits(inputs.random_bf16((Fs, cfg.H), seed=7, std=cfg.H ** -0.5)),
          inputs.to_bits(inputs.random_bf16((Fs, cfg.H), seed=8, std=cfg.H ** -0.5)),
          inputs.to_bits(inputs.random_bf16((cfg.H, Fs), seed=9, std=Fs ** -0.5)))
    plain = oracle.layer_forward(*args)
    with_s = oracle.layer_forward(*args, shared=sh)
    # routing and the routed experts are untouched
    for k in ("topk_ids", "row_of_assign", "xp", "h", "y"):
        assert np.array_equal(plain[k], with_s[k])
    # the shared expert equals a dense SwiGLU of every token
    _, s_dense = oracle.ffn_rows(xs, *sh)
    assert np.array_equal(with_s["y_shared"], s_dense)
    # zero shared weights leave the output unchanged
    zero = tuple(np.zeros_like(a) for a in sh)
    assert np.array_equal(oracle.layer_forward(*args, shared=zero)["out"], plain["out"])


# ---------------------------------------------------------------------------
# FP8 dispatch (E4M3 codes, one fp32 scale per row)
# ---------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_and_hand_values():
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_to_f64(codes)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()   # torch's own decoder
    assert np.array_equal(np.isnan(v), np.isnan(t))
    assert np.array_equal(v[~np.isnan(v)], t[~np.isnan(t)])
    hand = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
            0xB8: -1.0, 0x7E: 448.0, 0xFE: -448.0, 0x77: 240.0, 0x40: 2.0}
    for c, x in hand.items():
        assert oracle.e4m3_to_f64(np.array([c], np.uint8))[0] == x, hex(c)
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and np.isnan(v).sum() == 2
    assert np.signbit(v[0x80]) and v[0x80] == 0.0


def test_e4m3_encode_roundtrip_ties_to_even_and_saturation():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    v = oracle.e4m3_to_f64(codes)
    assert np.array_equal(oracle.f32_to_e4m3(v.astype(np.float32)), codes)
    # midpoints between neighbouring positive codes go to the code with the even mantissa
    pos = np.arange(0, 0x7F, dtype=np.uint8)
    pv = oracle.e4m3_to_f64(pos)
    mid = ((pv[:-1] + pv[1:]) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (pv[:-1] + pv[1:]) / 2)   # midpoints are fp32-exact
    got = oracle.f32_to_e4m3(mid)
    want = np.where(pos[:-1] % 2 == 0, pos[:-1], pos[1:])
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.f32_to_e4m3(-mid), want | 0x80)
    # just off the midpoints the nearest code wins
    up = np.nextafter(mid, np.float32(np.inf))
    dn = np.nextafter(mid, np.float32(0))
    assert np.array_equal(oracle.f32_to_e4m3(up), pos[1:])
    assert np.array_equal(oracle.f32_to_e4m3(dn), pos[:-1])
    # saturation to +-448; NaN stays NaN
    big = np.array([448.0, 449.0, 463.99, 464.0, 480.0, 1e6, 3.0e38, np.inf], np.float32)
    assert np.all(oracle.f32_to_e4m3(big) == 0x7E)
    assert np.all(oracle.f32_to_e4m3(-big) == 0xFE)
    assert oracle.f32_to_e4m3(np.array([np.nan], np.float32))[0] == 0x7F
    # below half the smallest subnormal: zero; the sign survives
    assert oracle.f32_to_e4m3(np.array([2.0 ** -11, -2.0 ** -11], np.float32)).tolist() == [0x00, 0x80]


def test_e4m3_encode_matches_torch_on_random_values():
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    v = np.clip(v, -447.0, 447.0).astype(np.float32)
    t = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()   # torch's own encoder
    assert np.array_equal(oracle.f32_to_e4m3(v), t)


def test_quantize_rows_fp8_scale_amax_and_error_bound():
    rng = np.random.default_rng(5)
    x = bf(rng.standard_normal((40, 96)) * np.exp(rng.uniform(-6, 6, (40, 1))))
    x[3] = bf(np.zeros(96))
    q, s = oracle.quantize_rows_fp8(x)
    xv = val(x)
    assert s.dtype == np.float32 and q.dtype == np.uint8
    assert s[3] == 1.0 and np.all(q[3] == 0)
    amax = np.abs(xv).max(axis=1)
    nz = amax > 0
    assert np.array_equal(s[nz], (amax[nz].astype(np.float32) / np.float32(448.0)))
    # the largest element of each row lands on +-448
    i = np.abs(xv).argmax(axis=1)
    assert np.all(oracle.e4m3_to_f64(q[np.arange(40), i])[nz] == np.sign(xv[np.arange(40), i])[nz] * 448.0)
    # dequantization error: half a step of 3 mantissa bits, or half a subnormal step
    err = np.abs(xv - oracle.e4m3_to_f64(q) * s[:, None].astype(np.float64))
    bound = 2.0 ** -4 * np.abs(xv) * (1 + 2.0 ** -20) + 2.0 ** -10 * s[:, None]
    assert np.all(err <= bound)
    # scaling a row by a power of two scales s and leaves the codes unchanged
    q2, s2 = oracle.quantize_rows_fp8(bf(xv * 2.0 ** 7))
    assert np.array_equal(q2, q) and np.array_equal(s2[nz], s[nz] * np.float32(2 ** 7))


def _exact_fp8_rows(rng, R, C):
    """bf16 rows that per-row E4M3 quantization represents exactly: codes times 2^a_r, with one
    element per row at +-448 so that the scale comes out as 2^a_r."""
    codes = rng.integers(0, 0x7E, size=(R, C)).astype(np.uint8) | (rng.integers(0, 2, (R, C)) * 0x80).astype(np.uint8)
    codes[np.arange(R), rng.integers(0, C, R)] = np.where(rng.integers(0, 2, R) > 0, 0x7E, 0xFE)
    a = rng.integers(-14, -6, R).astype(np.float64)
    x = oracle.e4m3_to_f64(codes) * np.exp2(a)[:, None]
    bits = bf(x)
    assert np.array_equal(val(bits), x)
    return bits, codes, np.exp2(a).astype(np.float32)


def test_quantize_rows_fp8_recovers_exact_codes_and_scales():
    rng = np.random.default_rng(8)
    bits, codes, scale = _exact_fp8_rows(rng, 17, 50)
    q, s = oracle.quantize_rows_fp8(bits)
    assert np.array_equal(q, codes) and np.array_equal(s, scale)


def test_ffn_rows_fp8_equals_bf16_ffn_on_exactly_representable_inputs():
    # per-token and per-feature scales differ, T != F: a scale on the wrong axis changes g and u
    rng = np.random.default_rng(9)
    T, H, F = 7, 64, 24
    x, qx, sx = _exact_fp8_rows(rng, T, H)
    wg, qg, sg = _exact_fp8_rows(rng, F, H)
    wu, qu, su = _exact_fp8_rows(rng, F, H)
    wd = bf(rng.standard_normal((H, F)) / np.sqrt(F))
    h8, y8 = oracle.ffn_rows_fp8(qx, sx, qg, sg, qu, su, wd)
    h, y = oracle.ffn_rows(x, wg, wu, wd)
    assert np.array_equal(h8, h) and np.array_equal(y8, y)
    # a swapped pair of scales is visible
    h_bad, _ = oracle.ffn_rows_fp8(qx, sx, qg, su, qu, sg, wd)
    assert not np.array_equal(h_bad, h)


def test_dispatch_fp8_rows_and_bytes():
    rng = np.random.default_rng(2)
    T, K, E, H = 30, 3, 8, 40
    z = bf(rng.standard_normal((T, H)))
    ids = np.stack([rng.permutation(E)[:K] for _ in range(T)])
    cs = oracle.count_scan(ids, E, 1)
    xq, xs = oracle.dispatch_fp8(z, cs["row_of_assign"], K)
    q, s = oracle.quantize_rows_fp8(z)
    roa = cs["row_of_assign"].reshape(T, K)
    for t in range(T):
        for k in range(K):
            assert np.array_equal(xq[roa[t, k]], q[t]) and xs[roa[t, k]] == s[t]
    assert xq.nbytes + xs.nbytes == oracle.dispatch_bytes_fp8(T, K, H) == oracle.dispatch_bytes(T, K, H, 1) + 4 * T * K
    assert 2 * oracle.dispatch_bytes(T, K, H, 1) == oracle.dispatch_bytes(T, K, H, 2)   # FP8 halves the payload


def test_layer_fp8_equals_bf16_layer_on_exactly_representable_inputs():
    rng = np.random.default_rng(4)
    T, H, F, E, K = 24, 64, 32, 6, 2
    x, _, _ = _exact_fp8_rows(rng, T, H)
    wg = np.stack([_exact_fp8_rows(rng, F, H)[0] for _ in range(E)])
    wu = np.stack([_exact_fp8_rows(rng, F, H)[0] for _ in range(E)])
    wd = bf(rng.standard_normal((E, H, F)) / np.sqrt(F))
    w_g = (rng.standard_normal((H, E)) / np.sqrt(H)).astype(np.float32)
    r16 = oracle.layer_forward(x, w_g, wg, wu, wd, K)
    r8 = oracle.layer_forward(x, w_g, wg, wu, wd, K, fp8=True)
    assert np.array_equal(r8["topk_ids"], r16["topk_ids"])
    for k in ("h", "y", "out"):
        assert np.array_equal(r8[k], r16[k]), k
    assert np.array_equal(oracle.e4m3_to_f64(r8["xq"]) * r8["xs"][:, None], val(r16["xp"]))
