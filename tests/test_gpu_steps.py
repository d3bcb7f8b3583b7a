"""GPU parity of each step, called through the C ABI, against the CPU oracle.

Both sides get the same seeded inputs from routing_dispatch_grouped_top_b200.inputs;
nothing the GPU computes is fed to the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from routing_dispatch_grouped_top_b200 import binding as B
from routing_dispatch_grouped_top_b200 import build, inputs
from parity import WEIGHT_ABS, check_bf16, check_logits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    B.lib()


def bits(t):
    return inputs.to_bits(t)


PAIR_DEFAULT_MIN_ROWS = 64


@pytest.fixture(params=["single_cta", "cta_pair"])
def gemm_kernel(request):
    """Runs a GEMM test once on the single-CTA kernel and once on the CTA-pair kernel."""
    B.set_pair_min_rows(-1 if request.param == "single_cta" else 0)
    yield request.param
    B.set_pair_min_rows(PAIR_DEFAULT_MIN_ROWS)


def cpu(t):
    return t.detach().cpu().numpy()


# ---------------------------------------------------------------------------
# S1 route
# ---------------------------------------------------------------------------

ROUTE_CASES = [  # T, E, K, renormalize, generator
    (300, 8, 2, True, "random"), (257, 128, 8, True, "random"), (100, 256, 8, False, "random"),
    (77, 896, 16, True, "random"), (64, 33, 5, True, "quantized"), (50, 1024, 32, True, "random"),
    (129, 64, 6, True, "special"), (40, 1000, 7, False, "quantized"), (1, 5, 5, True, "random"),
    (0, 16, 4, True, "random"), (4096, 128, 8, True, "random"), (64, 64, 8, True, "nan_heavy"),
    (40, 896, 16, False, "nan_heavy"), (33, 1024, 32, True, "nan_heavy"), (10, 1, 1, True, "random"),
    (17, 32, 32, True, "quantized"), (9, 64, 32, False, "special"), (5, 1024, 32, True, "quantized"),
]


@pytest.mark.parametrize("T,E,K,renorm,gen", ROUTE_CASES)
def test_route_matches_oracle(T, E, K, renorm, gen):
    seed = T * 7 + E
    if gen == "random":
        l = inputs.random_logits(T, E, seed=seed, scale=2.0)
    elif gen == "quantized":
        l = inputs.quantized_logits(T, E, levels=5, seed=seed)
    elif gen == "nan_heavy":
        l = inputs.nan_heavy_logits(T, E, seed=seed)
    else:
        l = inputs.special_logits(T, E, seed=seed)
    d = B.dims(T=T, H=8, E=E, K=K, F=8, renormalize=renorm)
    ids = torch.full((T, K), -7, dtype=torch.int32, device=DEV)
    w = torch.empty((T, K), dtype=torch.float32, device=DEV)
    B.moe_route(l.to(DEV), d, ids, w)
    torch.cuda.synchronize()
    if T == 0:
        return
    rid, rw = oracle.route(l.numpy(), K, renorm)
    assert np.array_equal(cpu(ids), rid)
    if gen in ("special", "nan_heavy"):
        sel = np.take_along_axis(l.numpy(), rid, axis=1)
        ok_rows = np.all(np.isfinite(sel), axis=1) & np.all(np.isfinite(l.numpy()) | renorm, axis=1)
        np.testing.assert_allclose(cpu(w)[ok_rows], rw[ok_rows], atol=WEIGHT_ABS, rtol=0)
    else:
        np.testing.assert_allclose(cpu(w), rw, atol=WEIGHT_ABS, rtol=0)
        if renorm:
            assert np.allclose(cpu(w).sum(axis=1), 1.0, atol=1e-6)


LIMITED_CASES = [  # T, E, K, P, M, renormalize, generator
    (300, 256, 8, 8, 4, True, "random"), (200, 896, 16, 64, 8, True, "random"), (100, 16, 3, 4, 2, True, "quantized"),
    (129, 64, 6, 16, 3, False, "special"), (77, 1024, 8, 256, 4, True, "random"), (50, 32, 4, 32, 4, True, "random"),
    (64, 48, 5, 6, 1, True, "quantized"), (60, 256, 8, 8, 4, True, "nan_heavy"),
    (40, 12, 3, 4, 3, True, "quantized"), (30, 60, 9, 20, 3, True, "special"), (25, 128, 16, 8, 7, True, "nan_heavy"),
]


@pytest.mark.parametrize("T,E,K,P,M,renorm,gen", LIMITED_CASES)
def test_route_limited_matches_oracle(T, E, K, P, M, renorm, gen):
    seed = T + E + M
    l = {"random": lambda: inputs.random_logits(T, E, seed=seed, scale=2.0),
         "quantized": lambda: inputs.quantized_logits(T, E, levels=4, seed=seed),
         "special": lambda: inputs.special_logits(T, E, seed=seed),
         "nan_heavy": lambda: inputs.nan_heavy_logits(T, E, seed=seed)}[gen]()
    d = B.dims(T=T, H=8, E=E, K=K, F=8, P=P, renormalize=renorm, group_limit=M)
    ids = torch.full((T, K), -7, dtype=torch.int32, device=DEV)
    w = torch.empty((T, K), dtype=torch.float32, device=DEV)
    B.moe_route(l.to(DEV), d, ids, w)
    torch.cuda.synchronize()
    rid, rw = oracle.route_limited(l.numpy(), K, P, M, renorm)
    assert np.array_equal(cpu(ids), rid)
    if gen not in ("special", "nan_heavy"):
        np.testing.assert_allclose(cpu(w), rw, atol=WEIGHT_ABS, rtol=0)


def test_route_limited_argument_checks():
    with pytest.raises(B.MoEError):
        B.moe_route(torch.zeros((4, 16), device=DEV), B.dims(T=4, H=8, E=16, K=5, F=8, P=4, group_limit=1),
                    torch.empty((4, 5), dtype=torch.int32, device=DEV), torch.empty((4, 5), device=DEV))


# ---------------------------------------------------------------------------
# S2 count + scan
# ---------------------------------------------------------------------------

SCAN_CASES = [  # T, E, K, P, zipf
    (64, 8, 2, 1, None), (300, 16, 4, 4, None), (1, 4, 4, 2, None), (0, 8, 2, 1, None),
    (128, 256, 8, 8, 1.1), (4096, 128, 8, 1, None), (8192, 256, 8, 8, None), (4096, 896, 16, 64, None),
    (3000, 1024, 3, 16, 2.0), (5000, 7, 7, 7, None), (20000, 64, 6, 4, 1.1),
    # 128 chunks of 2048 assignments, four experts per thread in the look-back; all ids on one expert
    (32768, 1024, 8, 8, 1.1), (32768, 64, 8, 4, None), (4000, 1, 1, 1, None),
]


def run_count_scan(ids, E, P):
    T, K = ids.shape
    d = B.dims(T=T, H=8, E=E, K=K, F=8, P=P)
    ws = B.make_workspace(d)
    TK = T * K
    mk = lambda n: torch.full((n,), -3, dtype=torch.int32, device=DEV)  # noqa: E731
    out = dict(counts=mk(E), offsets=mk(E + 1), part_counts=mk(P), part_offsets=mk(P + 1),
               row_of_assign=mk(max(TK, 1)), assign_of_row=mk(max(TK, 1)))
    B.moe_count_scan(ids.to(DEV).contiguous(), d, out["counts"], out["offsets"], out["part_counts"],
                     out["part_offsets"], out["row_of_assign"], out["assign_of_row"], ws)
    status = B.read_device_status(ws)
    res = {k: cpu(v) for k, v in out.items()}
    res["row_of_assign"] = res["row_of_assign"][:TK]
    res["assign_of_row"] = res["assign_of_row"][:TK]
    return res, status


@pytest.mark.parametrize("T,E,K,P,zipf", SCAN_CASES)
def test_count_scan_matches_oracle(T, E, K, P, zipf):
    ids = inputs.random_topk_ids(T, E, K, seed=T + E + K, zipf_s=zipf) if T else torch.zeros((0, K), dtype=torch.int32)
    got, status = run_count_scan(ids, E, P)
    assert status == 0
    ref = oracle.count_scan(ids.numpy(), E, P)
    for k in ("counts", "offsets", "part_counts", "part_offsets", "row_of_assign", "assign_of_row"):
        assert np.array_equal(got[k], ref[k]), k


def test_count_scan_repeated_calls_reuse_workspace():
    ids = inputs.random_topk_ids(2000, 64, 4, seed=3)
    d = B.dims(T=2000, H=8, E=64, K=4, F=8, P=4)
    ws = B.make_workspace(d)
    ref = oracle.count_scan(ids.numpy(), 64, 4)
    idd = ids.to(DEV)
    bufs = [torch.empty(n, dtype=torch.int32, device=DEV) for n in (64, 65, 4, 5, 8000, 8000)]
    for _ in range(5):
        B.moe_count_scan(idd, d, *bufs, ws)
    assert B.read_device_status(ws) == 0
    assert np.array_equal(cpu(bufs[4]), ref["row_of_assign"])


def test_count_scan_flags_out_of_range_ids():
    ids = inputs.random_topk_ids(100, 16, 2, seed=1)
    ids[17, 1] = 16
    ids[50, 0] = -2
    got, status = run_count_scan(ids, 16, 1)
    assert status & B.DEV_BAD_INDEX
    flat = ids.numpy().reshape(-1)
    assert got["counts"].sum() == int(((flat >= 0) & (flat < 16)).sum())
    assert got["row_of_assign"][17 * 2 + 1] == -1 and got["row_of_assign"][100] == -1
    assert got["offsets"][16] == -1          # the call is marked failed


def test_count_scan_lookback_wait_times_out_and_reports():
    # A block ticket counter that starts at 1 (set on the host): no block draws ticket 0, so
    # the first chunk's flag is never published and every look-back that reaches it must
    # give up after its bounded wait, report MOE_DEV_TIMEOUT and mark the call failed.
    T, E, K = 4000, 32, 4
    ids = inputs.random_topk_ids(T, E, K, seed=9)
    d = B.dims(T=T, H=8, E=E, K=K, F=8)
    ws = B.make_workspace(d)
    ws[64:68] = torch.tensor([1, 0, 0, 0], dtype=torch.uint8, device=DEV)
    bufs = [torch.empty(n, dtype=torch.int32, device=DEV) for n in (E, E + 1, 1, 2, T * K, T * K)]
    B.moe_count_scan(ids.to(DEV), d, *bufs, ws)
    assert B.read_device_status(ws) & B.DEV_TIMEOUT
    assert int(bufs[1][E]) == -1
    # the kernels rewound their state: the context stays usable and the next call works
    B.workspace_init(ws)
    B.moe_count_scan(ids.to(DEV), d, *bufs, ws)
    assert B.read_device_status(ws) == 0
    want = oracle.count_scan(ids.numpy(), E)
    assert np.array_equal(cpu(bufs[4]), want["row_of_assign"])
    assert np.array_equal(cpu(bufs[1]), want["offsets"])


def test_count_scan_state_is_rewound_without_reinit():
    # after a normal call the kernels leave ticket, flags and totals at zero: many calls of
    # different sizes on one workspace (sized for the largest) stay exact
    E, K, P = 64, 4, 4
    d = B.dims(T=9000, H=8, E=E, K=K, F=8, P=P)
    ws = B.make_workspace(d)
    for i, T in enumerate((9000, 1, 300, 64, 9000, 0, 257)):
        ids = inputs.random_topk_ids(T, E, K, seed=40 + i) if T else torch.zeros((0, K), dtype=torch.int32)
        di = B.dims(T=T, H=8, E=E, K=K, F=8, P=P)
        bufs = [torch.full((n,), -7, dtype=torch.int32, device=DEV) for n in (E, E + 1, P, P + 1, T * K, T * K)]
        B.moe_count_scan(ids.to(DEV), di, *bufs, ws)
        want = oracle.count_scan(ids.numpy(), E, P)
        for k, a in zip(("counts", "offsets", "part_counts", "part_offsets", "row_of_assign", "assign_of_row"), bufs):
            assert np.array_equal(cpu(a), want[k]), (T, k)
    assert B.read_device_status(ws) == 0


# ---------------------------------------------------------------------------
# S3 permute
# ---------------------------------------------------------------------------

PERMUTE_CASES = [(300, 256, 16, 4, 4), (1, 8, 4, 1, 1), (64, 7168, 256, 8, 8), (1000, 2048, 128, 8, 1),
                 (33, 72, 6, 6, 3), (0, 64, 8, 2, 1)]


@pytest.mark.parametrize("T,H,E,K,P", PERMUTE_CASES)
def test_permute_matches_oracle(T, H, E, K, P):
    x = inputs.random_bf16((T, H), seed=T + H)
    ids = inputs.random_topk_ids(T, E, K, seed=T + E) if T else torch.zeros((0, K), dtype=torch.int32)
    w = inputs.random_weights(T, K, seed=5)
    cs = oracle.count_scan(ids.numpy(), E, P)
    roa = torch.from_numpy(cs["row_of_assign"])
    d = B.dims(T=T, H=H, E=E, K=K, F=8, P=P)
    TK = T * K
    xp = torch.zeros((TK, H), dtype=torch.bfloat16, device=DEV)
    meta = [torch.full((TK,), -1, dtype=dt, device=DEV) for dt in (torch.int32, torch.int32, torch.float32, torch.int32)]
    B.moe_permute(x.to(DEV), roa.to(DEV), ids.to(DEV), w.to(DEV), d, xp, *meta)
    torch.cuda.synchronize()
    rxp, rmeta = oracle.permute(bits(x), cs["row_of_assign"], ids.numpy(), w.numpy(), E, P)
    assert np.array_equal(bits(xp), rxp)
    assert xp.numel() * xp.element_size() == oracle.dispatch_bytes(T, K, H, 2)
    for got, key in zip(meta, ("token", "slot", "w", "local_expert")):
        assert np.array_equal(cpu(got), rmeta[key]), key


def test_permute_then_combine_of_identity_experts_returns_x():
    # Identity experts (y = xp): combine(permute(x)) = (sum of weights) * x = x.
    T, H, E, K = 500, 1024, 32, 8
    x = inputs.random_bf16((T, H), seed=1).to(DEV)
    l = inputs.random_logits(T, E, seed=2).to(DEV)
    d = B.dims(T=T, H=H, E=E, K=K, F=8)
    ws = B.make_workspace(d)
    b = B.alloc_layer_buffers(d)
    B.moe_route(l, d, b["topk_ids"], b["topk_w"])
    B.moe_count_scan(b["topk_ids"], d, b["counts"], b["offsets"], b["part_counts"], b["part_offsets"],
                     b["row_of_assign"], b["assign_of_row"], ws)
    B.moe_permute(x, b["row_of_assign"], b["topk_ids"], b["topk_w"], d, b["xp"])
    B.moe_combine(b["xp"], b["row_of_assign"], b["topk_w"], d, b["out"])
    torch.cuda.synchronize()
    assert torch.equal(b["out"].view(torch.int16), x.view(torch.int16))


# ---------------------------------------------------------------------------
# S4/S5 grouped SwiGLU FFN
# ---------------------------------------------------------------------------

FFN_CASES = [  # E, H, F, rows, zipf, zero_frac
    (8, 256, 512, 300, None, 0.25), (4, 200, 200, 260, None, 0.0), (16, 2048, 768, 2000, 1.1, 0.2),
    (3, 64, 136, 1, None, 0.0), (32, 512, 256, 700, 2.0, 0.3), (1, 1024, 384, 513, None, 0.0),
    (64, 128, 128, 64, None, 0.5),
]


def ffn_inputs(E, H, F, rows, zipf, zero_frac, seed=0):
    counts = inputs.random_counts(E, rows, seed=seed + E + rows, zipf_s=zipf, zero_frac=zero_frac)
    off = np.zeros(E + 1, np.int32)
    off[1:] = np.cumsum(counts.numpy())
    xp = inputs.random_bf16((rows, H), seed=seed + 1)
    wg = inputs.random_bf16((E, F, H), seed=seed + 2, std=H ** -0.5)
    wu = inputs.random_bf16((E, F, H), seed=seed + 3, std=H ** -0.5)
    wd = inputs.random_bf16((E, H, F), seed=seed + 4, std=F ** -0.5)
    return off, xp, wg, wu, wd


@pytest.mark.parametrize("E,H,F,rows,zipf,zf", FFN_CASES)
def test_grouped_ffn_matches_oracle(E, H, F, rows, zipf, zf, gemm_kernel):
    off, xp, wg, wu, wd = ffn_inputs(E, H, F, rows, zipf, zf)
    d = B.dims(T=rows, H=H, E=E, K=1, F=F)
    ws = B.make_workspace(d)
    h = torch.zeros((rows, F), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros((rows, H), dtype=torch.bfloat16, device=DEV)
    offd = torch.from_numpy(off).to(DEV)
    B.moe_grouped_ffn(xp.to(DEV), offd, wg.to(DEV), wu.to(DEV), wd.to(DEV), d, h, y, ws)
    assert B.read_device_status(ws) == 0
    rh, ry = oracle.grouped_ffn(bits(xp), off, bits(wg), bits(wu), bits(wd))
    check_bf16("h", bits(h), rh)
    check_bf16("y", bits(y), ry)


GATHER_CASES = [  # T, H, E, K, F, zipf
    (300, 256, 8, 2, 512, None), (130, 200, 4, 2, 200, None), (2000, 2048, 16, 8, 768, 1.1),
    (1, 64, 3, 1, 136, None), (64, 128, 64, 1, 128, None), (700, 512, 32, 4, 256, 2.0),
]


def gather_inputs(T, H, E, K, F, zipf, seed=0):
    ids = inputs.random_topk_ids(T, E, K, seed=seed + T, zipf_s=zipf)
    cs = oracle.count_scan(ids.numpy(), E, 1)
    x = inputs.random_bf16((T, H), seed=seed + 1)
    wg = inputs.random_bf16((E, F, H), seed=seed + 2, std=H ** -0.5)
    wu = inputs.random_bf16((E, F, H), seed=seed + 3, std=H ** -0.5)
    return cs, x, wg, wu


@pytest.mark.parametrize("T,H,E,K,F,zipf", GATHER_CASES)
def test_grouped_gate_up_gather_equals_the_permuted_copy_bit_for_bit(T, H, E, K, F, zipf, gemm_kernel):
    # row r of the gathered operand is token assign_of_row[r] // K: the same bytes reach the same
    # MMAs in the same order as with the permuted copy, so h is identical, not just close
    cs, x, wg, wu = gather_inputs(T, H, E, K, F, zipf)
    TK = T * K
    d = B.dims(T=T, H=H, E=E, K=K, F=F)
    ws = B.make_workspace(d)
    aor = torch.from_numpy(cs["assign_of_row"]).to(DEV)
    off = torch.from_numpy(cs["offsets"]).to(DEV)
    xp = x[torch.from_numpy(cs["assign_of_row"] // K)]
    h_copy = torch.full((TK, F), -1.0, dtype=torch.bfloat16, device=DEV)
    h_gather = torch.full((TK, F), -2.0, dtype=torch.bfloat16, device=DEV)
    B.moe_grouped_gate_up(xp.to(DEV), off, wg.to(DEV), wu.to(DEV), d, h_copy, ws)
    B.moe_grouped_gate_up_gather(x.to(DEV), aor, off, wg.to(DEV), wu.to(DEV), d, h_gather, ws)
    torch.cuda.synchronize()
    assert B.read_device_status(ws) == 0
    assert torch.equal(h_gather.view(torch.int16), h_copy.view(torch.int16))
    rh, _ = oracle.grouped_ffn(bits(xp), cs["offsets"], bits(wg), bits(wu), np.zeros((E, 8, F), np.uint16))
    check_bf16("h", bits(h_gather), rh)


def test_grouped_gate_up_gather_reports_a_row_outside_the_tokens_then_recovers():
    T, H, E, K, F = 200, 256, 4, 2, 128
    cs, x, wg, wu = gather_inputs(T, H, E, K, F, None, seed=5)
    d = B.dims(T=T, H=H, E=E, K=K, F=F)
    off = torch.from_numpy(cs["offsets"]).to(DEV)
    xd, wgd, wud = x.to(DEV), wg.to(DEV), wu.to(DEV)
    h = torch.zeros((T * K, F), dtype=torch.bfloat16, device=DEV)
    for bad in (T * K + 7, -3):
        ws = B.make_workspace(d)
        aor = cs["assign_of_row"].copy()
        aor[17] = bad                      # names no token: reported, row 0 read instead
        B.moe_grouped_gate_up_gather(xd, torch.from_numpy(aor).to(DEV), off, wgd, wud, d, h, ws)
        torch.cuda.synchronize()
        assert B.read_device_status(ws) & B.DEV_BAD_INDEX
    ws = B.make_workspace(d)
    B.moe_grouped_gate_up_gather(xd, torch.from_numpy(cs["assign_of_row"]).to(DEV), off, wgd, wud, d, h, ws)
    torch.cuda.synchronize()
    assert B.read_device_status(ws) == 0
    xp = x[torch.from_numpy(cs["assign_of_row"] // K)]
    rh, _ = oracle.grouped_ffn(bits(xp), cs["offsets"], bits(wg), bits(wu), np.zeros((E, 8, F), np.uint16))
    check_bf16("h", bits(h), rh)


# ---------------------------------------------------------------------------
# FP8 dispatch: E4M3 codes with per-row scales, gate/up on E4M3
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(300, 256), (64, 7168), (7, 16), (129, 2064), (1, 48), (0, 32)])
def test_quantize_fp8_rows_matches_oracle_bit_exact(rows, cols):
    x = inputs.random_bf16((rows, cols), seed=rows + cols)
    if rows:
        # rows over many magnitudes, one all-zero row, one row of a single nonzero element
        x = x * torch.exp(torch.linspace(-20.0, 12.0, rows)).to(torch.bfloat16)[:, None]
        x[rows // 2] = 0
        x[-1, :] = 0
        x[-1, cols // 3] = -3.0
    q = torch.full((rows, cols), 0x55, dtype=torch.uint8, device=DEV)
    sc = torch.full((rows,), -1.0, dtype=torch.float32, device=DEV)
    B.moe_quantize_fp8_rows(x.to(DEV), q, sc)
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_rows_fp8(bits(x))
    assert np.array_equal(cpu(q), rq)
    assert np.array_equal(cpu(sc).view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("T,H,E,K,P", [(300, 256, 16, 4, 4), (1, 16, 4, 1, 1), (64, 7168, 256, 8, 8),
                                       (1000, 2048, 128, 8, 1), (33, 80, 6, 6, 3), (0, 64, 8, 2, 1)])
def test_permute_fp8_matches_oracle_bit_exact(T, H, E, K, P):
    x = inputs.random_bf16((T, H), seed=T + H)
    ids = inputs.random_topk_ids(T, E, K, seed=T + E) if T else torch.zeros((0, K), dtype=torch.int32)
    w = inputs.random_weights(T, K, seed=5)
    cs = oracle.count_scan(ids.numpy(), E, P)
    roa = torch.from_numpy(cs["row_of_assign"])
    d = B.dims(T=T, H=H, E=E, K=K, F=8, P=P, fp8_dispatch=True)
    TK = T * K
    xq = torch.full((TK, H), 0x55, dtype=torch.uint8, device=DEV)
    xs = torch.full((TK,), -1.0, dtype=torch.float32, device=DEV)
    meta = [torch.full((TK,), -1, dtype=dt, device=DEV) for dt in (torch.int32, torch.int32, torch.float32, torch.int32)]
    B.moe_permute_fp8(x.to(DEV), roa.to(DEV), ids.to(DEV), w.to(DEV), d, xq, xs, *meta)
    torch.cuda.synchronize()
    rq, rs = oracle.dispatch_fp8(bits(x), cs["row_of_assign"], K)
    assert np.array_equal(cpu(xq), rq)
    assert np.array_equal(cpu(xs).view(np.uint32), rs.view(np.uint32))
    assert xq.numel() + 4 * xs.numel() == oracle.dispatch_bytes_fp8(T, K, H)
    _, rmeta = oracle.permute(bits(x), cs["row_of_assign"], ids.numpy(), w.numpy(), E, P)
    for got, key in zip(meta, ("token", "slot", "w", "local_expert")):
        assert np.array_equal(cpu(got), rmeta[key]), key


FP8_FFN_CASES = [  # E, H, F, rows, zipf, zero_frac
    (8, 256, 512, 300, None, 0.25), (4, 208, 200, 260, None, 0.0), (16, 2048, 768, 2000, 1.1, 0.2),
    (3, 64, 136, 1, None, 0.0), (32, 512, 256, 700, 2.0, 0.3), (1, 1024, 384, 513, None, 0.0),
    (8, 7168, 256, 300, None, 0.0),
]


@pytest.mark.parametrize("E,H,F,rows,zipf,zf", FP8_FFN_CASES)
def test_grouped_gate_up_fp8_matches_oracle(E, H, F, rows, zipf, zf, gemm_kernel):
    counts = inputs.random_counts(E, rows, seed=E + rows, zipf_s=zipf, zero_frac=zf)
    off = np.zeros(E + 1, np.int32)
    off[1:] = np.cumsum(counts.numpy())
    xq = inputs.random_e4m3_codes((rows, H), seed=1)
    xs = inputs.random_scales(rows, seed=2)
    wgq = inputs.random_e4m3_codes((E, F, H), seed=3)
    wuq = inputs.random_e4m3_codes((E, F, H), seed=4)
    # weight scales ~ 1/(64 sqrt(H)) keep g and u of order one
    sg = inputs.random_scales(E * F, seed=5, lo=0.5 / (64 * H ** 0.5), hi=2.0 / (64 * H ** 0.5)).reshape(E, F)
    su = inputs.random_scales(E * F, seed=6, lo=0.5 / (64 * H ** 0.5), hi=2.0 / (64 * H ** 0.5)).reshape(E, F)
    d = B.dims(T=rows, H=H, E=E, K=1, F=F, fp8_dispatch=True)
    ws = B.make_workspace(d)
    h = torch.zeros((rows, F), dtype=torch.bfloat16, device=DEV)
    B.moe_grouped_gate_up_fp8(xq.to(DEV), xs.to(DEV), torch.from_numpy(off).to(DEV), wgq.to(DEV), wuq.to(DEV),
                              sg.to(DEV), su.to(DEV), d, h, ws)
    assert B.read_device_status(ws) == 0
    wd = np.zeros((E, 8, F), np.uint16)      # h only: the down projection is the bf16 kernel
    rh = np.zeros((rows, F), np.uint16)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            rh[lo:hi], _ = oracle.ffn_rows_fp8(xq.numpy()[lo:hi], xs.numpy()[lo:hi], wgq.numpy()[e], sg.numpy()[e],
                                               wuq.numpy()[e], su.numpy()[e], wd[e])
    check_bf16("h", bits(h), rh)


def test_grouped_gemm_schedule_rewinds_across_many_launches(gemm_kernel):
    # every launch claims tiles from the workspace's per-call-site counter and the last CTA
    # rewinds it: 40 launches in a row on one workspace give the same result every time
    off, xp, wg, wu, wd = ffn_inputs(16, 512, 384, 3000, 1.1, 0.1, seed=3)
    d = B.dims(T=3000, H=512, E=16, K=1, F=384)
    ws = B.make_workspace(d)
    offd, xpd, wgd, wud, wdd = (torch.from_numpy(off).to(DEV), xp.to(DEV), wg.to(DEV), wu.to(DEV), wd.to(DEV))
    h = torch.zeros((3000, 384), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros((3000, 512), dtype=torch.bfloat16, device=DEV)
    B.moe_grouped_ffn(xpd, offd, wgd, wud, wdd, d, h, y, ws)
    first = y.clone()
    for _ in range(40):
        y.zero_()
        B.moe_grouped_ffn(xpd, offd, wgd, wud, wdd, d, h, y, ws)
    torch.cuda.synchronize()
    assert B.read_device_status(ws) == 0
    assert torch.equal(y.view(torch.int16), first.view(torch.int16))
    sched = ws[160:256].view(torch.int32).cpu()
    assert int(sched.abs().sum()) == 0          # every counter rewound to zero


def test_grouped_gemms_run_on_a_header_only_workspace():
    # the GEMM calls use only the 256-byte workspace header (status, tile-schedule counters)
    off, xp, wg, wu, wd = ffn_inputs(4, 256, 128, 300, None, 0.0, seed=7)
    d = B.dims(T=300, H=256, E=4, K=1, F=128)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    B.workspace_init(ws)
    h = torch.zeros((300, 128), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros((300, 256), dtype=torch.bfloat16, device=DEV)
    B.moe_grouped_ffn(xp.to(DEV), torch.from_numpy(off).to(DEV), wg.to(DEV), wu.to(DEV), wd.to(DEV), d, h, y, ws)
    assert B.read_device_status(ws) == 0
    rh, ry = oracle.grouped_ffn(bits(xp), off, bits(wg), bits(wu), bits(wd))
    check_bf16("y", bits(y), ry)
    with pytest.raises(B.MoEError):
        B.moe_grouped_ffn(xp.to(DEV), torch.from_numpy(off).to(DEV), wg.to(DEV), wu.to(DEV), wd.to(DEV), d, h, y,
                          ws[:128])


def test_grouped_down_alone_matches_oracle(gemm_kernel):
    E, H, F, rows = 12, 1024, 512, 900
    counts = inputs.random_counts(E, rows, seed=4, zero_frac=0.2)
    off = np.concatenate([[0], np.cumsum(counts.numpy())]).astype(np.int32)
    hin = inputs.random_bf16((rows, F), seed=5, std=0.5)
    wd = inputs.random_bf16((E, H, F), seed=6, std=F ** -0.5)
    d = B.dims(T=rows, H=H, E=E, K=1, F=F)
    ws = B.make_workspace(d)
    y = torch.zeros((rows, H), dtype=torch.bfloat16, device=DEV)
    B.moe_grouped_down(hin.to(DEV), torch.from_numpy(off).to(DEV), wd.to(DEV), d, y, ws)
    assert B.read_device_status(ws) == 0
    ry = np.zeros((rows, H), np.uint16)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        if hi > lo:
            ry[lo:hi] = oracle.f64_to_bf16_bits(oracle.bf16_bits_to_f64(bits(hin)[lo:hi]) @
                                                oracle.bf16_bits_to_f64(bits(wd)[e]).T)
    check_bf16("y", bits(y), ry)


def test_grouped_gemm_rejects_bad_offsets_without_touching_memory():
    E, H, F, rows = 4, 128, 128, 64
    off, xp, wg, wu, wd = ffn_inputs(E, H, F, rows, None, 0.0)
    off_bad = off.copy()
    off_bad[2] = rows + 5000                          # beyond the buffer
    d = B.dims(T=rows, H=H, E=E, K=1, F=F)
    ws = B.make_workspace(d)
    h = torch.zeros((rows, F), dtype=torch.bfloat16, device=DEV)
    B.moe_grouped_gate_up(xp.to(DEV), torch.from_numpy(off_bad).to(DEV), wg.to(DEV), wu.to(DEV), d, h, ws)
    assert B.read_device_status(ws) & B.DEV_BAD_INDEX
    assert int(h.view(torch.int16).abs().sum()) == 0


# ---------------------------------------------------------------------------
# S6 combine
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("with_shared", [False, True], ids=["routed", "plus_shared"])
@pytest.mark.parametrize("T,H,K", [(300, 256, 2), (77, 7168, 8), (1000, 2048, 16), (5, 8, 1), (64, 512, 32)])
def test_combine_matches_oracle(T, H, K, with_shared):
    y = inputs.random_bf16((T * K, H), seed=T + H)
    roa = inputs.random_bijection(T * K, seed=K)
    w = inputs.random_weights(T, K, seed=T)
    s = inputs.random_bf16((T, H), seed=T + 3, std=0.5) if with_shared else None
    d = B.dims(T=T, H=H, E=max(K, 2), K=K, F=8)
    out = torch.zeros((T, H), dtype=torch.bfloat16, device=DEV)
    B.moe_combine(y.to(DEV), roa.to(DEV), w.to(DEV), d, out, shared=None if s is None else s.to(DEV))
    torch.cuda.synchronize()
    ref = oracle.combine(bits(y), roa.numpy(), w.numpy(), None if s is None else bits(s))
    check_bf16("out", bits(out), ref)


# ---------------------------------------------------------------------------
# S7 skew
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("E,total,zipf", [(8, 128, None), (256, 1024, 1.1), (896, 65536, None), (4, 0, None)])
def test_skew_matches_oracle(E, total, zipf):
    c = inputs.random_counts(E, total, seed=E, zipf_s=zipf)
    d = B.dims(T=max(total, 1), H=8, E=E, K=1, F=8)
    r = torch.zeros(1, dtype=torch.float32, device=DEV)
    B.moe_skew_stats(c.to(DEV), d, r)
    torch.cuda.synchronize()
    assert float(r.item()) == pytest.approx(oracle.skew_ratio(c.numpy()), rel=1e-6)


# ---------------------------------------------------------------------------
# S0 gating and S8 dense projections
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,H,E,bias", [(300, 256, 8, False), (200, 2048, 128, False), (130, 7168, 256, True),
                                        (97, 2048, 896, False), (5, 64, 1000, True)])
def test_gating_matches_oracle(T, H, E, bias):
    x = inputs.random_bf16((T, H), seed=T)
    w_g = (torch.randn((H, E), generator=torch.Generator().manual_seed(H + E)) * H ** -0.5).float()
    b = (torch.randn(E, generator=torch.Generator().manual_seed(E)) * 0.5).float() if bias else None
    d = B.dims(T=T, H=H, E=E, K=1, F=8)
    ws = B.make_workspace(d)
    split = torch.empty((3, E, H), dtype=torch.bfloat16, device=DEV)
    B.moe_pack_router(w_g.to(DEV), d, split)
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    B.moe_gating(x.to(DEV), split, b.to(DEV) if bias else None, d, logits, ws)
    assert B.read_device_status(ws) == 0
    ref = oracle.gating_logits(bits(x), w_g.numpy(), b.numpy() if bias else None)
    check_logits("logits", cpu(logits), ref)


@pytest.mark.parametrize("M,Kd,N", [(300, 1024, 256), (64, 7168, 2048), (257, 2048, 7168), (3, 72, 40)])
def test_dense_projection_matches_oracle(M, Kd, N, gemm_kernel):
    a = inputs.random_bf16((M, Kd), seed=M)
    w = inputs.random_bf16((N, Kd), seed=N, std=Kd ** -0.5)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    B.moe_dense(a.to(DEV), w.to(DEV), out, ws)
    assert B.read_device_status(ws) == 0
    check_bf16("dense", bits(out), oracle.dense_bf16(bits(a), bits(w)))
