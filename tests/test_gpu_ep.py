"""Expert-parallel exchange kernels on one GPU: R ranks emulated in one process.

Every rank's buffers live on the one GPU and the peer table holds their addresses, so the
dispatch and return kernels' peer stores land in the other ranks' buffers exactly as they
would over NVLink.  The ranks' launches go to one stream in protocol order (all dispatches
before any wait on them, all returns before any wait on them), so every wait finds its flags
already published and nothing waits for a kernel that has not run.

Checked against the oracle's counting sort of all ranks' routing concatenated in rank order:
the device plan equals the host plan; each rank's received block is bit for bit that layout's
rows of its experts, with (source rank, source row) metadata; the returned rows are bit copies
of the owners' expert outputs; the expert outputs and the combined outputs are within the bf16
tolerance of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import check_bf16
from routing_dispatch_grouped_top_b200 import binding as B
from routing_dispatch_grouped_top_b200 import build, ep, inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    B.lib()


def bits(t):
    return inputs.to_bits(t)


def make_ranks(R, T, H, E, K, F, seed=0):
    El = E // R
    w_g = inputs.random_bf16((H, E), seed=seed + 1, std=H ** -0.5).float().to(DEV)
    wg = inputs.random_bf16((E, F, H), seed=seed + 2, std=H ** -0.5).to(DEV)
    wu = inputs.random_bf16((E, F, H), seed=seed + 3, std=H ** -0.5).to(DEV)
    wd = inputs.random_bf16((E, H, F), seed=seed + 4, std=F ** -0.5).to(DEV)
    ranks = [ep.EPRank(T, H, E, K, F, R, r, w_g, wg[r * El:(r + 1) * El].contiguous(),
                       wu[r * El:(r + 1) * El].contiguous(), wd[r * El:(r + 1) * El].contiguous())
             for r in range(R)]
    peers = ep.emulated_peers(ranks)
    for r in ranks:
        r.peers = peers
    return ranks, (w_g, wg, wu, wd)


def run_protocol(ranks, xs):
    for r, x in zip(ranks, xs):
        r.route(x)
    C = torch.stack([r.counts for r in ranks])
    for r in ranks:
        r.counts_all.copy_(C)
    for r, x in zip(ranks, xs):
        r.dispatch(x)
    for r in ranks:
        r.experts()
    for r in ranks:
        r.give_back()
    outs = [r.combine().clone() for r in ranks]
    torch.cuda.synchronize()
    for r in ranks:
        assert B.read_device_status(r.ep_ws) == 0
        assert B.read_device_status(r.ws) == 0 and B.read_device_status(r.gemm_ws) == 0
    return outs, C.cpu().numpy()


@pytest.mark.parametrize("R,T,H,E,K,F", [(4, 64, 512, 16, 4, 256), (2, 200, 256, 8, 2, 128), (8, 48, 1024, 64, 8, 192)])
def test_ep_exchange_matches_the_oracle_layout_and_outputs(R, T, H, E, K, F):
    ranks, (w_g, wg, wu, wd) = make_ranks(R, T, H, E, K, F)
    El = E // R
    for call in range(2):   # the second call reuses every buffer with a higher epoch
        xs = [inputs.random_bf16((T, H), seed=1000 * call + r).to(DEV) for r in range(R)]
        outs, C = run_protocol(ranks, xs)
        ids = np.concatenate([r.topk_ids.cpu().numpy() for r in ranks])
        wts = np.concatenate([r.topk_w.cpu().numpy() for r in ranks])
        cs = oracle.count_scan(ids, E, R)
        X = np.concatenate([bits(x) for x in xs])
        xp = X[cs["assign_of_row"] // K]
        off = cs["offsets"]
        h_ref, _ = oracle.grouped_ffn(xp, off, bits(wg), bits(wu), bits(wd))
        wd_b = bits(wd)
        for d, r in enumerate(ranks):
            sb, ro = B.moe_ep_plan_host(C, R, d, r.d)
            assert np.array_equal(r.send_base.cpu().numpy(), sb)
            assert np.array_equal(r.recv_offsets.cpu().numpy(), ro)
            lo, hi = off[d * El], off[(d + 1) * El]
            assert np.array_equal(ro, off[d * El:(d + 1) * El + 1] - lo)
            n = hi - lo
            assert np.array_equal(bits(r.recv_x[:n]), xp[lo:hi])
            src = cs["assign_of_row"][lo:hi] // (T * K)
            meta = r.recv_meta[:n].cpu().numpy()
            assert np.array_equal(meta[:, 0], src)
            src_roa = [rk.row_of_assign.cpu().numpy() for rk in ranks]
            assert np.array_equal(meta[:, 1], [src_roa[a // (T * K)][a % (T * K)] for a in cs["assign_of_row"][lo:hi]])
            # h against the oracle's; y against the oracle's down projection of the GPU's own h (a
            # rounding flip of a large h element would otherwise move y by more than its own rounding)
            h_gpu = bits(r.h_recv[:n])
            check_bf16(f"h_recv[{d}]", h_gpu, h_ref[lo:hi])
            ro_ = r.recv_offsets.cpu().numpy()
            y_exp = np.concatenate([oracle.dense_bf16(h_gpu[ro_[l]:ro_[l + 1]], wd_b[d * El + l]) for l in range(El)])
            check_bf16(f"y_recv[{d}]", bits(r.y_recv[:n]), y_exp)
        # returned rows are bit copies of the owners' outputs; combine at each source
        y_recv = [bits(r.y_recv) for r in ranks]
        for s, r in enumerate(ranks):
            ret = bits(r.ret_y)
            roa = r.row_of_assign.cpu().numpy()
            for a in range(T * K):
                row_g = cs["row_of_assign"][s * T * K + a]     # the assignment's row in the global layout
                d = int(np.searchsorted(off, row_g, side="right") - 1) // El
                assert np.array_equal(ret[roa[a]], y_recv[d][row_g - off[d * El]])
            # the combine of the returned rows (bit copies checked above) at the source's own rows
            check_bf16(f"out[{s}]", bits(outs[s]), oracle.combine(ret, roa, wts[s * T:(s + 1) * T]))


def test_ep_wait_for_an_epoch_nobody_publishes_times_out_and_reports():
    # a signal slot that nothing sets: the bounded wait must give up, report MOE_DEV_TIMEOUT
    # and leave the context usable
    ep_ws = B.ep_workspace(DEV)
    signal = torch.zeros(2 * 3, dtype=torch.int32, device=DEV)
    signal[:3] = 5
    B.moe_ep_wait(signal, 3, 0, 5, ep_ws)           # published: returns at once
    torch.cuda.synchronize()
    assert B.read_device_status(ep_ws) == 0
    B.moe_ep_wait(signal, 3, 0, 6, ep_ws)           # epoch 6 never published
    assert B.read_device_status(ep_ws) & B.DEV_TIMEOUT
    x = torch.ones(4, device=DEV)
    assert float((x * 2).sum()) == 8.0
