"""End-to-end parity of moe_layer_forward (C ABI) with the CPU oracle.

Small layers are compared output by output against the whole oracle.  The full
workloads (the sizes bench.py times, same launch path) are checked on sampled
tokens that the oracle evaluates one by one, and on properties that hold at any
size (counting sort = bijection, expert-sorted and stable; xp rows are copies of
x rows; partition ranges).

Routing is compared token by token against the oracle's own logits.  Where
the K-th and (K+1)-th oracle logits are closer than (a multiple of) the observed
GPU-vs-oracle logit error, both selections are correct and the GPU's is only
checked for validity; where two selected logits are that close, only their slot
order is open.  Every other token must get exactly the oracle's ids, and when
every token is unambiguous all integer outputs are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from routing_dispatch_grouped_top_b200 import binding as B
from routing_dispatch_grouped_top_b200 import build, inputs
from routing_dispatch_grouped_top_b200.config import (DEEPSEEK_R1_DECODE, DEEPSEEK_R1_PREFILL, LATENT_896E,
                                                      QWEN3_30B_A3B_PREFILL, TINY)
from parity import check_bf16, check_logits, topk_margin

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    B.lib()


def bits(t):
    return inputs.to_bits(t)


@pytest.fixture(params=["single_cta", "cta_pair"])
def gemm_kernel(request):
    """Runs a layer once with every grouped GEMM on the single-CTA kernel and once on the
    CTA-pair kernel (default rule: pair from 64 rows per expert)."""
    B.set_pair_min_rows(-1 if request.param == "single_cta" else 0)
    yield request.param
    B.set_pair_min_rows(64)


def cpu(t):
    return t.detach().cpu().numpy()


def run_gpu_layer(cfg, inp, aux=False, gather=False):
    d = B.dims_of(cfg)
    w = B.pack_layer_weights(d, inp["w_g"], inp["bias"], inp["w_gate"], inp["w_up"], inp["w_down"], inp["w_dp"],
                             inp["w_upp"], shared=inp["shared"])
    bufs = B.alloc_layer_buffers(d, gather=gather)
    if aux:
        B.attach_aux_stream(bufs, torch.cuda.Stream())
    ws = B.make_workspace(d)
    B.moe_layer_forward(inp["x"], w, d, bufs, ws)
    assert B.read_device_status(ws) == 0
    return bufs


def routing_split(ref_logits, got_logits, K):
    """(set_safe, order_safe, err): tokens whose selected set / slot order is fixed
    despite the largest GPU-vs-oracle logit difference err."""
    err = float(np.abs(np.asarray(got_logits, np.float64) - ref_logits).max()) if ref_logits.size else 0.0
    boundary, order = topk_margin(ref_logits, K)
    thr = 4.0 * err + 1e-7
    return boundary > thr, order > thr, err


def check_routing(got_ids, ref_ids, ref_logits, set_safe, order_safe, err, K):
    assert np.array_equal(got_ids[order_safe], ref_ids[order_safe])
    assert np.array_equal(np.sort(got_ids[set_safe], axis=1), np.sort(ref_ids[set_safe], axis=1))
    for t in np.nonzero(~set_safe)[0]:   # ambiguous tokens: the GPU's choice must be a valid top-K
        kth = np.sort(ref_logits[t])[::-1][K - 1]
        assert len(set(got_ids[t].tolist())) == K
        assert np.all(ref_logits[t][got_ids[t]] >= kth - 2.0 * err - 1e-7)


def gpu_slot(got_ids_row, e):
    """Slot k at which the GPU routed this token to expert e."""
    k = np.nonzero(got_ids_row == e)[0]
    assert k.size == 1
    return int(k[0])


def check_count_scan_properties(ids, E, P, res):
    """Properties that fix the stable counting sort at any size (checked with torch on the GPU)."""
    ids = ids.reshape(-1).long()
    TK = ids.numel()
    counts = torch.bincount(ids, minlength=E)
    assert torch.equal(res["counts"].long(), counts)
    off = torch.zeros(E + 1, dtype=torch.long, device=ids.device)
    off[1:] = torch.cumsum(counts, 0)
    assert torch.equal(res["offsets"].long(), off)
    roa, aor = res["row_of_assign"].long(), res["assign_of_row"].long()
    ar = torch.arange(TK, device=ids.device)
    assert torch.equal(aor[roa], ar) and torch.equal(roa[aor], ar)       # bijection
    e_of_row = ids[aor]
    assert bool((e_of_row[1:] >= e_of_row[:-1]).all())                     # expert-major
    same = e_of_row[1:] == e_of_row[:-1]
    assert bool((aor[1:][same] > aor[:-1][same]).all())                    # stable inside an expert
    epp = E // P
    assert torch.equal(res["part_offsets"].long(), off[::epp])
    assert torch.equal(res["part_counts"].long(), off[epp::epp] - off[:-1:epp])


# ---------------------------------------------------------------------------
# Small layers against the whole oracle
# ---------------------------------------------------------------------------

SMALL = [
    TINY,
    TINY.with_(name="tiny_T100_P2_plain_softmax", T=100, P=2, renormalize=False),
    QWEN3_30B_A3B_PREFILL.with_(name="qwen3_shape_T256_H512_F384", T=256, H=512, F=384),
    DEEPSEEK_R1_PREFILL.with_(name="r1_shape_T64_H1024_F256_E64_P8", T=64, H=1024, F=256, E=64),
    DEEPSEEK_R1_DECODE.with_(name="r1_decode_shape_T32_H1024_F512", T=32, H=1024, F=512),
    LATENT_896E.with_(name="latent_shape_T48_D1024_H256_E112_P8", T=48, d_model=1024, H=256, E=112, F=128, P=8),
    TINY.with_(name="one_token", T=1),
    DEEPSEEK_R1_PREFILL.with_(name="r1_shape_node_limited_T96_H512_F256_M4", T=96, H=512, F=256, group_limit=4),
    DEEPSEEK_R1_PREFILL.with_(name="r1_shape_shared_expert_T80_H512_F256_E32_Fs384", T=80, H=512, F=256, E=32,
                              F_shared=384),
    LATENT_896E.with_(name="latent_shared_expert_T40_D512_H256_E64_Fs128", T=40, d_model=512, H=256, E=64, F=128,
                      P=8, F_shared=128),
    QWEN3_30B_A3B_PREFILL.with_(name="qwen3_shape_fp8_dispatch_T256_H512_F384", T=256, H=512, F=384,
                                fp8_dispatch=True),
    DEEPSEEK_R1_PREFILL.with_(name="r1_shape_fp8_dispatch_T64_H1024_F256_E64", T=64, H=1024, F=256, E=64,
                              fp8_dispatch=True),
    LATENT_896E.with_(name="latent_fp8_dispatch_T48_D1024_H256_E112_P8", T=48, d_model=1024, H=256, E=112, F=128,
                      P=8, fp8_dispatch=True),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_layer_matches_oracle(cfg, gemm_kernel):
    inp = inputs.make_layer(cfg, DEV)
    # the shared expert on its own stream in one layer and in line in the other
    g = run_gpu_layer(cfg, inp, aux=cfg.name.startswith("r1_shape_shared"))
    torch.cuda.synchronize()
    cpu_in = {k: (v.cpu() if isinstance(v, torch.Tensor) else None) for k, v in inp.items()}
    shared = None if inp["shared"] is None else tuple(bits(t) for t in inp["shared"])
    r = oracle.layer_forward(bits(cpu_in["x"]), cpu_in["w_g"].numpy(), bits(cpu_in["w_gate"]),
                             bits(cpu_in["w_up"]), bits(cpu_in["w_down"]), cfg.K, cfg.P, cfg.renormalize,
                             bias=None if cpu_in["bias"] is None else cpu_in["bias"].numpy(),
                             w_dp_bits=None if cpu_in["w_dp"] is None else bits(cpu_in["w_dp"]),
                             w_upp_bits=None if cpu_in["w_upp"] is None else bits(cpu_in["w_upp"]),
                             group_limit=cfg.group_limit, shared=shared, fp8=cfg.fp8_dispatch)
    latent = bool(cfg.d_model)
    if latent:
        # The latent layer's z is held to the bf16 bound against the oracle's own z; the steps
        # after it then start from the GPU's z, and the final projection from the GPU's out,
        # so every later output is compared element by element without inheriting z's (or
        # out's) bf16 rounding flips.
        check_bf16("z", bits(g["z"]), r["z"])
        r = oracle.layer_forward(bits(g["z"]), cpu_in["w_g"].numpy(), bits(cpu_in["w_gate"]), bits(cpu_in["w_up"]),
                                 bits(cpu_in["w_down"]), cfg.K, cfg.P, cfg.renormalize,
                                 bias=None if cpu_in["bias"] is None else cpu_in["bias"].numpy(),
                                 group_limit=cfg.group_limit, shared=shared, fp8=cfg.fp8_dispatch)
        check_bf16("final", bits(g["final_out"]), oracle.dense_bf16(bits(g["out"]), bits(cpu_in["w_upp"])))
    if shared is not None:
        check_bf16("h_shared", bits(g["h_shared"]), r["h_shared"])
        check_bf16("y_shared", bits(g["y_shared"]), r["y_shared"])
    check_logits("logits", cpu(g["logits"]), r["logits"])
    set_safe, order_safe, err = routing_split(r["logits"], cpu(g["logits"]), cfg.K)
    gid, gw = cpu(g["topk_ids"]), cpu(g["topk_w"])
    if cfg.group_limit:
        # node-limited routing: margins of plain top-K do not bound the group choice;
        # at this size every token is expected to be unambiguous
        assert np.array_equal(gid, r["topk_ids"])
        set_safe = order_safe = np.ones(cfg.T, bool)
    else:
        check_routing(gid, r["topk_ids"], r["logits"], set_safe, order_safe, err, cfg.K)
    w_tol = 2e-6 + err           # weights follow their own side's logits
    check_count_scan_properties(g["topk_ids"], cfg.E, cfg.P, g)
    if order_safe.all():
        for k in ("counts", "offsets", "part_counts", "part_offsets", "row_of_assign", "assign_of_row"):
            assert np.array_equal(cpu(g[k]), r[k]), k
        if cfg.fp8_dispatch:
            assert np.array_equal(cpu(g["xq"]), r["xq"])
            assert np.array_equal(cpu(g["xs"]).view(np.uint32), r["xs"].view(np.uint32))
        else:
            assert np.array_equal(bits(g["xp"]), r["xp"])
        for key, mk in (("meta_token", "token"), ("meta_slot", "slot"), ("meta_local_expert", "local_expert")):
            assert np.array_equal(cpu(g[key]), r["meta"][mk]), key
        np.testing.assert_allclose(cpu(g["meta_w"]), r["meta"]["w"], atol=w_tol, rtol=0)
        check_bf16("h", bits(g["h"]), r["h"])
        check_bf16("y", bits(g["y"]), r["y"])
    # per (token, expert) of tokens with an unambiguous expert set: weight, h, y at each side's own row
    T, K = cfg.T, cfg.K
    ga, ra = cpu(g["row_of_assign"]).reshape(T, K), r["row_of_assign"].reshape(T, K)
    st = np.nonzero(set_safe)[0]
    grow, rrow = [], []
    for t in st:
        for k in range(K):
            kg = gpu_slot(gid[t], r["topk_ids"][t, k])
            assert abs(float(gw[t, kg]) - float(r["topk_w"][t, k])) <= w_tol
            grow.append(ga[t, kg])
            rrow.append(ra[t, k])
    if st.size:
        check_bf16("h(assign)", bits(g["h"])[grow], r["h"][rrow])
        check_bf16("y(assign)", bits(g["y"])[grow], r["y"][rrow])
        check_bf16("out", bits(g["out"])[st], r["out"][st])
    assert float(g["skew"].item()) == pytest.approx(oracle.skew_ratio(cpu(g["counts"])), rel=1e-6)


def test_layer_with_no_tokens_enqueues_nothing_and_reports_ok():
    cfg = TINY.with_(name="no_tokens", T=0)
    d = B.dims_of(cfg)
    inp = inputs.make_layer(TINY, DEV)
    w = B.pack_layer_weights(d, inp["w_g"], inp["bias"], inp["w_gate"], inp["w_up"], inp["w_down"])
    bufs = B.alloc_layer_buffers(d)
    ws = B.make_workspace(d)
    B.moe_layer_forward(torch.empty((0, cfg.H), dtype=torch.bfloat16, device=DEV), w, d, bufs, ws)
    assert B.read_device_status(ws) == 0
    assert torch.equal(bufs["offsets"].cpu(), torch.zeros(cfg.E + 1, dtype=torch.int32))
    assert float(bufs["skew"].item()) == 0.0


def test_layer_with_a_single_expert_is_one_dense_ffn():
    # E = K = 1: every token goes to the one expert with weight 1, so the layer is that expert's FFN
    cfg = TINY.with_(name="single_expert", T=200, E=1, K=1, P=1)
    inp = inputs.make_layer(cfg, DEV)
    g = run_gpu_layer(cfg, inp)
    assert torch.equal(g["topk_ids"].cpu(), torch.zeros((cfg.T, 1), dtype=torch.int32))
    assert torch.all(g["topk_w"] == 1.0)
    assert torch.equal(g["row_of_assign"].cpu(), torch.arange(cfg.T, dtype=torch.int32))
    h, y = oracle.ffn_rows(bits(inp["x"]), bits(inp["w_gate"][0]), bits(inp["w_up"][0]), bits(inp["w_down"][0]))
    check_bf16("out", bits(g["out"]), y)


def test_layer_forward_host_io_matches_device_call():
    cfg = TINY.with_(T=200, name="tiny_T200")
    inp = inputs.make_layer(cfg, DEV)
    g = run_gpu_layer(cfg, inp)
    d = B.dims_of(cfg)
    w = B.pack_layer_weights(d, inp["w_g"], inp["bias"], inp["w_gate"], inp["w_up"], inp["w_down"])
    bufs = B.alloc_layer_buffers(d)
    ws = B.make_workspace(d)
    xh = inp["x"].cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(inp["x"])
    B.moe_layer_forward_host(xh, xd, w, d, bufs, ws, oh)
    torch.cuda.synchronize()
    assert torch.equal(oh.view(torch.int16), g["out"].cpu().view(torch.int16))


def test_layer_stage_events_are_recorded():
    cfg = TINY
    inp = inputs.make_layer(cfg, DEV)
    d = B.dims_of(cfg)
    w = B.pack_layer_weights(d, inp["w_g"], inp["bias"], inp["w_gate"], inp["w_up"], inp["w_down"])
    bufs = B.alloc_layer_buffers(d)
    ws = B.make_workspace(d)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(B.MOE_NUM_STAGE_EVENTS)]
    B.moe_layer_forward(inp["x"], w, d, bufs, ws, stage_events=ev)
    torch.cuda.synchronize()
    times = [ev[i].elapsed_time(ev[i + 1]) for i in range(len(ev) - 1)]
    assert all(t >= 0 for t in times) and sum(times) > 0


# ---------------------------------------------------------------------------
# Full workloads: sampled tokens + size-independent properties
# ---------------------------------------------------------------------------

LAYER_KEYS = ("logits", "topk_ids", "topk_w", "counts", "offsets", "part_counts", "part_offsets", "row_of_assign",
              "assign_of_row", "meta_token", "meta_slot", "meta_w", "meta_local_expert", "h", "y", "out", "z",
              "final_out", "h_shared", "y_shared", "skew")


def assert_same_layer_outputs(a, b):
    for k in LAYER_KEYS:
        if a.get(k) is not None:
            assert torch.equal(a[k].view(torch.uint8), b[k].view(torch.uint8)), k


@pytest.mark.parametrize("cfg", [c for c in SMALL if not c.fp8_dispatch], ids=lambda c: c.name)
def test_layer_gathering_rows_in_place_equals_the_permuted_copy(cfg, gemm_kernel):
    # without an xp buffer the gate/up GEMM gathers each row's token itself: every output of the
    # layer must be bit for bit the one of the run with the permuted copy (checked above
    # against the oracle)
    inp = inputs.make_layer(cfg, DEV)
    copy = run_gpu_layer(cfg, inp)
    gath = run_gpu_layer(cfg, inp, gather=True)
    torch.cuda.synchronize()
    assert gath["xp"] is None
    assert_same_layer_outputs(copy, gath)


FULL = [QWEN3_30B_A3B_PREFILL, DEEPSEEK_R1_PREFILL, DEEPSEEK_R1_DECODE, LATENT_896E,
        DEEPSEEK_R1_PREFILL.with_(name=DEEPSEEK_R1_PREFILL.name + "_fp8_dispatch", fp8_dispatch=True)]
HOST_EXPERT_BUDGET = 2.5e9   # bytes of expert weights copied to the host for the oracle


@pytest.mark.slow
@pytest.mark.parametrize("cfg", FULL, ids=lambda c: c.name)
def test_full_size_sampled(cfg):
    torch.cuda.empty_cache()
    inp = inputs.make_layer(cfg, DEV)
    g = run_gpu_layer(cfg, inp)
    if not cfg.fp8_dispatch:
        # the same layer without the permuted copy (bench.py --gather) must give these outputs
        gath = run_gpu_layer(cfg, inp, gather=True)
        torch.cuda.synchronize()
        assert_same_layer_outputs(g, gath)
        del gath
    T, K, E, H, F = cfg.T, cfg.K, cfg.E, cfg.H, cfg.F
    latent = bool(cfg.d_model)
    # properties at full size
    check_count_scan_properties(g["topk_ids"], E, cfg.P, g)
    routed = g["z"] if latent else inp["x"]
    roa = g["row_of_assign"].long()
    tok = torch.arange(T * K, device=DEV) // K
    fp8 = cfg.fp8_dispatch
    if fp8:   # every copy of a token carries the same codes and scale
        first = roa.view(T, K)[:, :1].expand(T, K).reshape(-1)
        assert torch.equal(g["xq"][roa], g["xq"][first]) and torch.equal(g["xs"][roa], g["xs"][first])
        assert g["xq"].numel() + 4 * g["xs"].numel() == oracle.dispatch_bytes_fp8(T, K, H)
    else:
        assert torch.equal(g["xp"][roa].view(torch.int16), routed[tok].view(torch.int16))
        assert g["xp"].numel() * 2 == oracle.dispatch_bytes(T, K, H, 2)
    assert torch.equal(g["meta_token"][roa].long(), tok)
    # sampled tokens through the oracle
    rng = np.random.default_rng(cfg.T + cfg.E)
    cand = rng.permutation(T)[:256]
    x_rows = bits(inp["x"][torch.from_numpy(cand).to(DEV)])
    w_g = inp["w_g"].cpu().numpy()
    bias = None if inp["bias"] is None else inp["bias"].cpu().numpy()
    if latent:
        # z against the oracle's own z; the later steps start from the GPU's z (so they do
        # not inherit its bf16 rounding flips) and the final projection from the GPU's out
        check_bf16("z(sampled)", bits(g["z"])[cand], oracle.dense_bf16(x_rows, bits(inp["w_dp"])))
        z_rows = bits(g["z"])[cand]
    else:
        z_rows = x_rows
    lref = oracle.gating_logits(z_rows, w_g, bias)
    lgot = cpu(g["logits"])[cand]
    check_logits("logits(sampled)", lgot, lref)
    ids_ref, w_ref = oracle.route(lref, K, cfg.renormalize)
    set_safe, order_safe, err = routing_split(lref, lgot, K)
    gid_s = cpu(g["topk_ids"])[cand]
    check_routing(gid_s, ids_ref, lref, set_safe, order_safe, err, K)
    # FFN + combine for sampled tokens with an unambiguous expert set, within a host-memory budget
    per_expert = 3 * H * F * 2
    max_experts = max(K, int(HOST_EXPERT_BUDGET // per_expert))
    if cfg.fp8_dispatch:
        max_experts = min(max_experts, 2 * K)    # the oracle quantizes each expert's weights on the host
    chosen, experts = [], set()
    for i in np.nonzero(set_safe)[0]:
        need = experts | set(ids_ref[i].tolist())
        if len(need) > max_experts and chosen:
            break
        chosen.append(i)
        experts = need
        if len(chosen) >= 64:
            break
    assert chosen, "no unambiguous sampled token"
    wcache = {e: (bits(inp["w_gate"][e]), bits(inp["w_up"][e]), bits(inp["w_down"][e])) for e in sorted(experts)}
    if fp8:   # the oracle quantizes the sampled tokens and the experts' gate/up weights itself
        zq, zs = oracle.quantize_rows_fp8(z_rows)
        rows0 = torch.from_numpy(cpu(g["row_of_assign"]).reshape(T, K)[cand, 0].astype(np.int64)).to(DEV)
        assert np.array_equal(cpu(g["xq"][rows0]), zq)
        assert np.array_equal(cpu(g["xs"][rows0]).view(np.uint32), zs.view(np.uint32))
        wq = {}
        for e, (wg_, wu_, wd_) in wcache.items():
            (qg, sg), (qu, su) = oracle.quantize_rows_fp8(wg_), oracle.quantize_rows_fp8(wu_)
            wq[e] = (qg, sg, qu, su, wd_)
    ga = cpu(g["row_of_assign"]).reshape(T, K)
    gh, gy, gout = [], [], []
    rh, ry, rout = [], [], []
    for i in chosen:
        t = cand[i]
        acc = np.zeros(H)
        for k in range(K):
            e = int(ids_ref[i, k])
            if fp8:
                h_, y_ = oracle.ffn_rows_fp8(zq[i:i + 1], zs[i:i + 1], *wq[e])
            else:
                h_, y_ = oracle.ffn_rows(z_rows[i:i + 1], *wcache[e])
            rh.append(h_[0])
            ry.append(y_[0])
            acc += float(w_ref[i, k]) * oracle.bf16_bits_to_f64(y_)[0]
            row = ga[t, gpu_slot(gid_s[i], e)]
            gh.append(bits(g["h"][row]))
            gy.append(bits(g["y"][row]))
        rout.append(oracle.f64_to_bf16_bits(acc))
        gout.append(bits(g["out"][t]))
    check_bf16("h(sampled)", np.stack(gh), np.stack(rh))
    check_bf16("y(sampled)", np.stack(gy), np.stack(ry))
    check_bf16("out(sampled)", np.stack(gout), np.stack(rout))
    if latent:
        fin = oracle.dense_bf16(np.stack(gout), bits(inp["w_upp"]))
        check_bf16("final(sampled)", bits(g["final_out"])[cand[chosen]], fin)
    assert float(g["skew"].item()) == pytest.approx(oracle.skew_ratio(cpu(g["counts"])), rel=1e-6)
    del g, inp
    torch.cuda.empty_cache()
