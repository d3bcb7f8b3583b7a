"""The C-ABI library loads and exports what include/moe.h declares (CPU only: no compute calls)."""
import ctypes as C
import math
import os
import re

import numpy as np
import pytest

import oracle
from routing_dispatch_grouped_top_b200 import binding, build
from routing_dispatch_grouped_top_b200.config import ALL

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(moe_[a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 18
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(binding.EXPORTED)


def test_workspace_bytes_host_only(lib):
    for cfg in ALL.values():
        d = binding.dims_of(cfg)
        n = binding.workspace_bytes(d)
        assert n > 0 and n % 256 == 0
    bad = binding.dims(T=4, H=64, E=8, K=9, F=64)        # K > E
    assert binding.workspace_bytes(bad) == 0
    assert binding.workspace_bytes(binding.dims(T=4, H=64, E=9, K=2, F=64, P=2)) == 0   # E % P != 0


def test_argument_errors_are_synchronous(lib):
    bad = binding.dims(T=4, H=64, E=8, K=9, F=64)
    st = lib.moe_route(None, C.byref(bad), None, None, None)
    assert st == 1 and lib.moe_status_str(st) == b"invalid argument"
    odd = binding.dims(T=4, H=60, E=8, K=2, F=64)        # H not a multiple of 8
    assert lib.moe_route(None, C.byref(odd), None, None, None) == 2
    big = binding.dims(T=4, H=64, E=2048, K=2, F=64)
    assert lib.moe_route(None, C.byref(big), None, None, None) == 2
    for s in range(8):
        assert lib.moe_status_str(s)


def test_option_fields_are_validated_on_the_host(lib):
    ok = dict(T=8, H=64, E=8, K=2, F=64, P=4)
    assert binding.workspace_bytes(binding.dims(**ok, fp8_dispatch=True)) > 0
    fp8_odd = binding.dims(T=8, H=72, E=8, K=2, F=64, fp8_dispatch=True)     # E4M3 rows need H % 16 == 0
    assert lib.moe_route(None, C.byref(fp8_odd), None, None, None) == 2
    bad_flag = binding.dims(**ok)
    bad_flag.fp8_dispatch = 2
    assert lib.moe_route(None, C.byref(bad_flag), None, None, None) == 1
    assert binding.workspace_bytes(binding.dims(**ok, group_limit=5)) == 0      # M > P
    assert binding.workspace_bytes(binding.dims(**dict(ok, K=5), group_limit=1)) == 0  # K > M * E / P
    assert binding.workspace_bytes(binding.dims(**ok, F_shared=12)) == 0       # F_shared % 8 != 0


def test_gating_partials_enlarge_the_workspace(lib):
    # a layer whose router output has few tiles splits the gating reduction and keeps the
    # partial logits in the workspace (Qwen3 layer: 4 splits of T x E fp32)
    from routing_dispatch_grouped_top_b200.config import QWEN3_30B_A3B_PREFILL as q
    d = binding.dims_of(q)
    d_r1 = binding.dims_of(ALL["deepseek_r1_prefill_T8192_H7168_E256_K8_F2048_P8"])
    assert binding.workspace_bytes(d) >= 4 * q.T * q.E * 4
    assert binding.workspace_bytes(d_r1) < q.T * q.E * 4 * 4   # 128 router tiles: no split


@pytest.mark.parametrize("n", [1, 2, 19, 20, 21, 100, 101])
def test_p95_host_helper_matches_oracle(lib, n):
    r = np.random.default_rng(n).uniform(1, 6, n).astype(np.float32)
    assert binding.moe_p95(list(r)) == pytest.approx(oracle.p95_nearest_rank(r), abs=0)
    assert math.isnan(lib.moe_p95(None, 0))


def test_noalloc_count_scan_returns_the_same_shape_codes(lib):
    # the scratch-free call checks shapes exactly like moe_count_scan (checked before any device use)
    for d, code in ((binding.dims(T=4, H=64, E=1025, K=2, F=64), 2),      # E > MOE_MAX_E
                    (binding.dims(T=4, H=64, E=64, K=33, F=64), 2),       # K > MOE_MAX_K
                    (binding.dims(T=1 << 30, H=64, E=64, K=8, F=64), 2),  # T*K beyond int32
                    (binding.dims(T=4, H=64, E=8, K=9, F=64), 1)):        # K > E
        a = lib.moe_count_scan(None, C.byref(d), None, None, None, None, None, None, None, 0, None)
        b = lib.moe_count_scan_noalloc(None, C.byref(d), None, None, None, None, None, None, None)
        assert a == b == code
