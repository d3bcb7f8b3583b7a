"""The scratch-free count/scan entry point, for callers that cannot allocate device memory.

moe_count_scan_noalloc runs the count/scan kernels on a fixed scratch array inside the
library instead of a caller workspace.  It must give exactly what the oracle's counting
sort gives (and so what moe_count_scan gives), call after call (its scratch keeps the
previous call's contents), mark a call that met an invalid id without spoiling the next
one, and refuse shapes whose state would not fit the scratch.  This file is collected last
on purpose.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from routing_dispatch_grouped_top_b200 import binding as B
from routing_dispatch_grouped_top_b200 import build, inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
KEYS = ("counts", "offsets", "part_counts", "part_offsets", "row_of_assign", "assign_of_row")


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    B.lib()


def outputs(E, P, TK, fill):
    return [torch.full((n,), fill, dtype=torch.int32, device=DEV) for n in (E, E + 1, P, P + 1, TK, TK)]


@pytest.mark.parametrize("T,E,K,P,zipf", [(4096, 896, 16, 64, None), (300, 16, 4, 4, 1.1), (128, 256, 8, 8, 1.1),
                                          (8192, 256, 8, 8, None), (1, 8, 2, 1, None)])
def test_noalloc_count_scan_matches_oracle_and_workspace_call_twice(T, E, K, P, zipf):
    d = B.dims(T=T, H=8, E=E, K=K, F=8, P=P)
    ws = B.make_workspace(d)
    TK = T * K
    ref = outputs(E, P, TK, -5)
    for call in range(2):
        # a different routing on each call: the second call must not see the first one's state
        ids = inputs.random_topk_ids(T, E, K, seed=T + call, zipf_s=zipf)
        B.moe_count_scan(ids.to(DEV), d, *ref, ws)
        got = outputs(E, P, TK, -9)
        B.moe_count_scan_noalloc(ids.to(DEV), d, *got)
        torch.cuda.synchronize()
        assert B.read_device_status(ws) == 0
        want = oracle.count_scan(ids.numpy(), E, P)
        for k, a, b in zip(KEYS, got, ref):
            assert np.array_equal(a.cpu().numpy(), want[k]), k
            assert torch.equal(a, b), k


def test_noalloc_count_scan_marks_an_invalid_id_then_recovers():
    T, E, K = 600, 32, 4
    TK = T * K
    d = B.dims(T=T, H=8, E=E, K=K, F=8)
    ids = inputs.random_topk_ids(T, E, K, seed=21)
    bad = ids.clone()
    bad[123, 2] = E                      # one id out of range
    got = outputs(E, 1, TK, -9)
    B.moe_count_scan_noalloc(bad.to(DEV), d, *got)
    torch.cuda.synchronize()
    roa = got[4].cpu().numpy()
    assert roa[123 * K + 2] == -1        # no row for it
    assert int(got[1][E]) == -1          # and the call is marked failed
    valid = np.delete(roa, 123 * K + 2)
    assert np.array_equal(np.sort(valid), np.arange(TK - 1))   # the other assignments still get distinct rows
    # the next call on the shared scratch is clean
    got = outputs(E, 1, TK, -9)
    B.moe_count_scan_noalloc(ids.to(DEV), d, *got)
    torch.cuda.synchronize()
    want = oracle.count_scan(ids.numpy(), E, 1)
    for k, a in zip(KEYS, got):
        assert np.array_equal(a.cpu().numpy(), want[k]), k


def test_noalloc_count_scan_rejects_shapes_beyond_its_scratch():
    # E = 1024 with more than 127 chunks of 1024 assignments needs more than the 1 MiB scratch
    d = B.dims(T=32768, H=8, E=1024, K=8, F=8)
    st = B.lib().moe_count_scan_noalloc(None, C.byref(d), None, None, None, None, None, None, None)
    assert st == 1   # null outputs are refused first
    bufs = outputs(1024, 1, 32768 * 8, 0)
    with pytest.raises(B.MoEError) as e:
        B.moe_count_scan_noalloc(torch.zeros((32768, 8), dtype=torch.int32, device=DEV), d, *bufs)
    assert e.value.status == 2   # MOE_ERR_UNSUPPORTED_SHAPE
    T = 127 * 1024 // 8          # 127 chunks: fits
    ok = B.dims(T=T, H=8, E=1024, K=8, F=8)
    ids = inputs.random_topk_ids(T, 1024, 8, seed=3)
    bufs = outputs(1024, 1, T * 8, 0)
    B.moe_count_scan_noalloc(ids.to(DEV), ok, *bufs)
    torch.cuda.synchronize()
    want = oracle.count_scan(ids.numpy(), 1024, 1)
    for k, a in zip(KEYS, bufs):
        assert np.array_equal(a.cpu().numpy(), want[k]), k
