"""Expert-parallel exchange plan and protocol on CPU: gloo ranks, world sizes 2 and 4.

Each rank routes its own seeded tokens with the oracle, the per-expert counts are
all-gathered over gloo, and the library's host plan (moe_ep_plan_host, no GPU) says where
every row lands.  The rows then travel as the dispatch kernel moves them (to row send_base[e]
+ row_of_assign[a] - offsets[e] of the owner, with (source rank, source row)), the owner runs
the oracle FFN of its experts on what it received, and the outputs travel back to the source
rows named in the metadata, where the oracle combine sums them.  Everything must equal the
oracle layer run on all ranks' tokens concatenated in rank order, bit for bit: the received
blocks are that layer's expert-major rows of the owner's experts, and the combined outputs
are its outputs.
"""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
T, H, E, K, F = 24, 32, 8, 3, 16


def rank_inputs(R):
    sys.path.insert(0, ROOT)
    from routing_dispatch_grouped_top_b200 import inputs
    xs = [inputs.to_bits(inputs.random_bf16((T, H), seed=100 + r)) for r in range(R)]
    w_g = inputs.random_logits(H, E, seed=7).numpy() * (H ** -0.5)
    wg = inputs.to_bits(inputs.random_bf16((E, F, H), seed=8, std=H ** -0.5))
    wu = inputs.to_bits(inputs.random_bf16((E, F, H), seed=9, std=H ** -0.5))
    wd = inputs.to_bits(inputs.random_bf16((E, H, F), seed=10, std=F ** -0.5))
    return xs, w_g.astype(np.float32), wg, wu, wd


def _worker(rank, R, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from routing_dispatch_grouped_top_b200 import binding as B
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=R)
    try:
        El = E // R
        xs, w_g, wg, wu, wd = rank_inputs(R)
        x = xs[rank]
        # 1. route and count/scan this rank's tokens (partitions = ranks)
        ids, w = oracle.route(oracle.gating_logits(x, w_g), K)
        cs = oracle.count_scan(ids, E, R)
        # 2. all-gather of the counts
        counts = torch.from_numpy(cs["counts"].astype(np.int32))
        allc = [torch.zeros(E, dtype=torch.int32) for _ in range(R)]
        dist.all_gather(allc, counts)
        C = torch.stack(allc).numpy()
        # 3. the library's plan and the dispatch's row moves
        d = B.dims(T=T, H=H, E=E, K=K, F=F, P=R)
        send_base, recv_off = B.moe_ep_plan_host(C, R, rank, d)
        msgs = [[] for _ in range(R)]
        for a in range(T * K):
            e = int(ids.reshape(-1)[a])
            r = int(cs["row_of_assign"][a])
            row = int(send_base[e]) + r - int(cs["offsets"][e])
            msgs[e // El].append((row, x[a // K].copy(), (rank, r)))
        got = [None] * R
        dist.all_gather_object(got, msgs)
        cap = R * T * K
        recv_x = np.zeros((cap, H), np.uint16)
        recv_meta = np.full((cap, 2), -1, np.int64)
        seen = set()
        for src in range(R):
            for row, xr, meta in got[src][rank]:
                assert 0 <= row < cap and row not in seen
                seen.add(row)
                recv_x[row], recv_meta[row] = xr, meta
        n = int(recv_off[El])
        assert seen == set(range(n))                      # the rows fill [0, n) exactly
        # 4. the owner's experts on the received rows
        _, y_recv = oracle.grouped_ffn(recv_x[:n], recv_off, wg[rank * El:(rank + 1) * El],
                                       wu[rank * El:(rank + 1) * El], wd[rank * El:(rank + 1) * El])
        # 5. outputs back to their sources' rows, combine there
        back = [[] for _ in range(R)]
        for j in range(n):
            s, r = recv_meta[j]
            back[int(s)].append((int(r), y_recv[j].copy()))
        got = [None] * R
        dist.all_gather_object(got, back)
        ret_y = np.zeros((T * K, H), np.uint16)
        filled = set()
        for src in range(R):
            for r, yr in got[src][rank]:
                ret_y[r] = yr
                filled.add(r)
        assert filled == set(range(T * K))
        out = oracle.combine(ret_y, cs["row_of_assign"], w)
        q.put((rank, recv_x[:n], recv_off, recv_meta[:n], out))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("R", [2, 4])
def test_ep_exchange_equals_the_single_gpu_layer(R):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + 10 * R + os.getpid() % 500
    procs = [ctx.Process(target=_worker, args=(r, R, port, q)) for r in range(R)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(R):
        rank, *vals = q.get(timeout=180)
        res[rank] = vals
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    xs, w_g, wg, wu, wd = rank_inputs(R)
    ref = oracle.layer_forward(np.concatenate(xs), w_g, wg, wu, wd, K, R)
    El = E // R
    off = ref["offsets"]
    for d in range(R):
        recv_x, recv_off, recv_meta, out = res[d]
        lo, hi = off[d * El], off[(d + 1) * El]
        assert np.array_equal(recv_off, off[d * El:(d + 1) * El + 1] - lo)
        assert np.array_equal(recv_x, ref["xp"][lo:hi])              # the received block, bit for bit
        a_glob = ref["assign_of_row"][lo:hi]                           # its source rank and source row
        assert np.array_equal(recv_meta[:, 0], a_glob // (T * K))
        src_roa = [oracle.count_scan(oracle.route(oracle.gating_logits(xs[s], w_g), K)[0], E, R)["row_of_assign"]
                   for s in range(R)]
        assert np.array_equal(recv_meta[:, 1], [src_roa[ag // (T * K)][ag % (T * K)] for ag in a_glob])
        assert np.array_equal(out, ref["out"][d * T:(d + 1) * T])    # the round trip, bit for bit
