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


@pytest.mark.parametrize("n", [1, 2, 19, 20, 21, 100, 101])
def test_p95_host_helper_matches_oracle(lib, n):
    r = np.random.default_rng(n).uniform(1, 6, n).astype(np.float32)
    assert binding.moe_p95(list(r)) == pytest.approx(oracle.p95_nearest_rank(r), abs=0)
    assert math.isnan(lib.moe_p95(None, 0))
