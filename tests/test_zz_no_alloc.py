"""The scratch-free count/scan entry point, for callers that cannot allocate device memory.

moe_count_scan_noalloc runs the count/scan kernel on a fixed scratch array inside the
library instead of a caller workspace.  It must give exactly what moe_count_scan gives,
call after call (its scratch keeps the previous call's contents), and refuse shapes
whose histograms would not fit the scratch.  This file is collected last on purpose.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from routing_dispatch_grouped_top_b200 import binding as B
from routing_dispatch_grouped_top_b200 import build, inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    build.build()
    B.lib()


def outputs(E, P, TK, fill):
    return [torch.full((n,), fill, dtype=torch.int32, device=DEV) for n in (E, E + 1, P, P + 1, TK, TK)]


@pytest.mark.parametrize("T,E,K,P,zipf", [(4096, 896, 16, 64, None), (300, 16, 4, 4, 1.1), (128, 256, 8, 8, 1.1)])
def test_noalloc_count_scan_matches_workspace_call_twice(T, E, K, P, zipf):
    d = B.dims(T=T, H=8, E=E, K=K, F=8, P=P)
    ws = B.make_workspace(d)
    TK = T * K
    ref = outputs(E, P, TK, -5)
    for call in range(2):
        # a different routing on each call: the second call must not see the first one's state
        ids = inputs.random_topk_ids(T, E, K, seed=T + call, zipf_s=zipf).to(DEV)
        B.moe_count_scan(ids, d, *ref, ws)
        got = outputs(E, P, TK, -9)
        B.moe_count_scan_noalloc(ids, d, *got)
        torch.cuda.synchronize()
        assert B.read_device_status(ws) == 0
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_noalloc_count_scan_rejects_shapes_beyond_its_scratch():
    # E = 1024 fits 255 block histograms in 1 MiB: T*K = 256 * 1024 needs 256 of them.
    d = B.dims(T=32768, H=8, E=1024, K=8, F=8)
    st = B.lib().moe_count_scan_noalloc(None, C.byref(d), None, None, None, None, None, None, None)
    assert st == 1   # null outputs are refused first
    bufs = outputs(1024, 1, 32768 * 8, 0)
    with pytest.raises(B.MoEError) as e:
        B.moe_count_scan_noalloc(torch.zeros((32768, 8), dtype=torch.int32, device=DEV), d, *bufs)
    assert e.value.status == 2   # MOE_ERR_UNSUPPORTED_SHAPE
    ok = B.dims(T=32640, H=8, E=1024, K=8, F=8)  # 255 blocks: fits
    ids = inputs.random_topk_ids(32640, 1024, 8, seed=3).to(DEV)
    bufs = outputs(1024, 1, 32640 * 8, 0)
    B.moe_count_scan_noalloc(ids, ok, *bufs)
    torch.cuda.synchronize()
    assert int(bufs[0].sum()) == 32640 * 8
    assert np.array_equal(np.sort(bufs[4].cpu().numpy()), np.arange(32640 * 8))
