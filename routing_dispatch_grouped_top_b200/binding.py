"""Thin ctypes binding over libmoe_b200.so (the C ABI in include/moe.h).

Argument marshalling only: every function checks dtype/device/shape of the torch
tensors it is handed, passes raw device pointers and the current CUDA stream,
and raises :class:`MoEError` on a non-zero status.  All arithmetic happens in the
library's kernels; there is no fallback when the library or a GPU is missing.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_B200_LIB may name another build of the same library (e.g. a tuning variant).
LIB_PATH = os.environ.get("MOE_B200_LIB") or os.path.join(_HERE, "libmoe_b200.so")

MOE_NUM_STAGE_EVENTS = 10
STAGE_NAMES = ["latent_down", "gating", "route", "count_scan", "permute", "gate_up", "down", "combine",
               "latent_up"]
DEV_BAD_INDEX = 0x1
DEV_TIMEOUT = 0x2


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: status {status} ({msg})")
        self.status = status


class moe_dims(C.Structure):
    _fields_ = [("T", C.c_int64), ("H", C.c_int32), ("E", C.c_int32), ("K", C.c_int32), ("F", C.c_int32),
                ("P", C.c_int32), ("renormalize", C.c_int32), ("d_model", C.c_int32), ("group_limit", C.c_int32),
                ("F_shared", C.c_int32), ("fp8_dispatch", C.c_int32)]


_W_FIELDS = ("w_g_split", "bias", "w_gate", "w_up", "w_down", "w_dp", "w_upp", "w_shared_gate",
             "w_shared_up", "w_shared_down", "w_gate_q", "w_up_q", "s_gate", "s_up")


class moe_layer_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _W_FIELDS]


_BUF_FIELDS = ("z", "logits", "topk_ids", "topk_w", "counts", "offsets", "part_counts", "part_offsets",
               "row_of_assign", "assign_of_row", "xp", "meta_token", "meta_slot", "meta_w", "meta_local_expert",
               "h", "y", "out", "final_out", "skew", "h_shared", "y_shared", "aux_stream", "fork_event", "join_event",
               "xq", "xs")


class moe_layer_buffers(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _BUF_FIELDS]


MOE_EP_MAX_RANKS = 64
MOE_EP_IPC_HANDLE_BYTES = 64


class moe_ep_peers(C.Structure):
    _fields_ = [("recv_x", C.c_void_p * MOE_EP_MAX_RANKS), ("recv_meta", C.c_void_p * MOE_EP_MAX_RANKS),
                ("ret_y", C.c_void_p * MOE_EP_MAX_RANKS), ("signal", C.c_void_p * MOE_EP_MAX_RANKS)]


_VP, _SZ, _I32, _I64 = C.c_void_p, C.c_size_t, C.c_int32, C.c_int64
_DP = C.POINTER(moe_dims)
_SIGS = {
    "moe_workspace_bytes": (_SZ, [_DP]),
    "moe_workspace_init": (C.c_int, [_VP, _SZ, _VP]),
    "moe_read_device_status": (C.c_int, [_VP, C.POINTER(C.c_int32), _VP]),
    "moe_status_str": (C.c_char_p, [C.c_int]),
    "moe_pack_router": (C.c_int, [_VP, _DP, _VP, _VP]),
    "moe_gating": (C.c_int, [_VP, _VP, _VP, _DP, _VP, _VP, _SZ, _VP]),
    "moe_route": (C.c_int, [_VP, _DP, _VP, _VP, _VP]),
    "moe_count_scan": (C.c_int, [_VP, _DP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_count_scan_noalloc": (C.c_int, [_VP, _DP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_permute": (C.c_int, [_VP, _VP, _VP, _VP, _DP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_grouped_ffn": (C.c_int, [_VP, _VP, _VP, _VP, _VP, _DP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_grouped_gate_up": (C.c_int, [_VP, _VP, _VP, _VP, _DP, _VP, _VP, _SZ, _VP]),
    "moe_grouped_gate_up_gather": (C.c_int, [_VP, _VP, _VP, _VP, _VP, _DP, _VP, _VP, _SZ, _VP]),
    "moe_grouped_down": (C.c_int, [_VP, _VP, _VP, _DP, _VP, _VP, _SZ, _VP]),
    "moe_set_pair_min_rows": (None, [_I32]),
    "moe_quantize_fp8_rows": (C.c_int, [_VP, _I64, _I32, _VP, _VP, _VP]),
    "moe_permute_fp8": (C.c_int, [_VP, _VP, _VP, _VP, _DP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_grouped_gate_up_fp8": (C.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _DP, _VP, _VP, _SZ, _VP]),
    "moe_combine": (C.c_int, [_VP, _VP, _VP, _VP, _DP, _VP, _VP]),
    "moe_skew_stats": (C.c_int, [_VP, _DP, _VP, _VP]),
    "moe_p95": (C.c_double, [C.POINTER(C.c_float), C.c_int]),
    "moe_dense": (C.c_int, [_VP, _VP, _I64, _I32, _I32, _VP, _VP, _SZ, _VP]),
    "moe_layer_forward": (C.c_int, [_VP, C.POINTER(moe_layer_weights), _DP, C.POINTER(moe_layer_buffers), _VP,
                                    _SZ, C.POINTER(_VP), _VP]),
    "moe_layer_forward_host": (C.c_int, [_VP, _VP, C.POINTER(moe_layer_weights), _DP,
                                         C.POINTER(moe_layer_buffers), _VP, _SZ, _VP, _VP]),
    "moe_ep_workspace_bytes": (_SZ, []),
    "moe_ep_plan": (C.c_int, [_VP, _I32, _I32, _DP, _VP, _VP, _VP]),
    "moe_ep_plan_host": (C.c_int, [_VP, _I32, _I32, _DP, _VP, _VP]),
    "moe_ep_dispatch": (C.c_int, [_VP, _VP, _VP, _VP, _VP, _DP, _I32, _I32, _I64, C.POINTER(moe_ep_peers), _I32,
                                  _VP, _VP]),
    "moe_ep_wait": (C.c_int, [_VP, _I32, _I32, _I32, _VP, _VP]),
    "moe_ep_return": (C.c_int, [_VP, _VP, _VP, _DP, _I32, _I32, _I64, C.POINTER(moe_ep_peers), _I32, _VP, _VP]),
    "moe_ep_ipc_export": (C.c_int, [_VP, _VP, C.POINTER(C.c_uint64)]),
    "moe_ep_ipc_import": (C.c_int, [_VP, C.c_uint64, C.POINTER(_VP), C.POINTER(_VP)]),
    "moe_ep_ipc_close": (C.c_int, [_VP]),
}
EXPORTED = tuple(_SIGS)

_lib_handle: Optional[C.CDLL] = None


def lib() -> C.CDLL:
    """Loads libmoe_b200.so (raises if it has not been built)."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m routing_dispatch_grouped_top_b200.build`")
        h = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib_handle = h
    return _lib_handle


def _check(fn: str, status: int):
    if status != 0:
        raise MoEError(fn, status, lib().moe_status_str(status).decode())


def dims(T, H, E, K, F, P=1, renormalize=True, d_model=0, group_limit=0, F_shared=0,
         fp8_dispatch=False) -> moe_dims:
    return moe_dims(int(T), int(H), int(E), int(K), int(F), int(P), int(bool(renormalize)), int(d_model or 0),
                    int(group_limit or 0), int(F_shared or 0), int(bool(fp8_dispatch)))


def dims_of(cfg, T=None) -> moe_dims:
    return dims(cfg.T if T is None else T, cfg.H, cfg.E, cfg.K, cfg.F, cfg.P, cfg.renormalize, cfg.d_model or 0,
                cfg.group_limit or 0, cfg.F_shared or 0, cfg.fp8_dispatch)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor", numel=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {numel}")
    return t.data_ptr()


# ---------------------------------------------------------------------------
# Workspace
# ---------------------------------------------------------------------------

def workspace_bytes(d: moe_dims) -> int:
    return int(lib().moe_workspace_bytes(C.byref(d)))


def make_workspace(d: moe_dims, device="cuda") -> torch.Tensor:
    """Allocates and initialises a workspace (uint8 tensor, 256-byte aligned)."""
    n = workspace_bytes(d)
    if n == 0:
        raise ValueError("invalid layer shape")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check("moe_workspace_init", lib().moe_workspace_init(ws.data_ptr(), n, _stream(None)))
    return ws


def workspace_init(ws: torch.Tensor, stream=None):
    _check("moe_workspace_init", lib().moe_workspace_init(_ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def read_device_status(ws: torch.Tensor, stream=None) -> int:
    st = C.c_int32(0)
    _check("moe_read_device_status", lib().moe_read_device_status(_ptr(ws, torch.uint8, "ws"), C.byref(st),
                                                                  _stream(stream)))
    return int(st.value)


# ---------------------------------------------------------------------------
# Steps
# ---------------------------------------------------------------------------

def moe_pack_router(w_g: torch.Tensor, d: moe_dims, w_g_split: torch.Tensor, stream=None):
    _check("moe_pack_router", lib().moe_pack_router(_ptr(w_g, torch.float32, "w_g", d.H * d.E), C.byref(d),
                                                    _ptr(w_g_split, torch.bfloat16, "w_g_split", 3 * d.E * d.H),
                                                    _stream(stream)))


def moe_gating(x, w_g_split, bias, d: moe_dims, logits, ws, stream=None):
    _check("moe_gating", lib().moe_gating(_ptr(x, torch.bfloat16, "x", d.T * d.H),
                                          _ptr(w_g_split, torch.bfloat16, "w_g_split", 3 * d.E * d.H),
                                          _ptr(bias, torch.float32, "bias", d.E), C.byref(d),
                                          _ptr(logits, torch.float32, "logits", d.T * d.E),
                                          _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_route(logits, d: moe_dims, topk_ids, topk_w, stream=None):
    _check("moe_route", lib().moe_route(_ptr(logits, torch.float32, "logits", d.T * d.E), C.byref(d),
                                        _ptr(topk_ids, torch.int32, "topk_ids", d.T * d.K),
                                        _ptr(topk_w, torch.float32, "topk_w", d.T * d.K), _stream(stream)))


def moe_count_scan(topk_ids, d: moe_dims, counts, offsets, part_counts, part_offsets, row_of_assign,
                   assign_of_row, ws, stream=None):
    TK = d.T * d.K
    _check("moe_count_scan", lib().moe_count_scan(
        _ptr(topk_ids, torch.int32, "topk_ids", TK), C.byref(d), _ptr(counts, torch.int32, "counts", d.E),
        _ptr(offsets, torch.int32, "offsets", d.E + 1), _ptr(part_counts, torch.int32, "part_counts", d.P),
        _ptr(part_offsets, torch.int32, "part_offsets", d.P + 1),
        _ptr(row_of_assign, torch.int32, "row_of_assign", TK),
        _ptr(assign_of_row, torch.int32, "assign_of_row", TK), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream)))


def moe_count_scan_noalloc(topk_ids, d: moe_dims, counts, offsets, part_counts, part_offsets, row_of_assign,
                           assign_of_row, stream=None):
    """moe_count_scan for callers that cannot allocate: the library's own fixed scratch
    replaces the workspace (see include/moe.h for its limit and sharing rules)."""
    TK = d.T * d.K
    _check("moe_count_scan_noalloc", lib().moe_count_scan_noalloc(
        _ptr(topk_ids, torch.int32, "topk_ids", TK), C.byref(d), _ptr(counts, torch.int32, "counts", d.E),
        _ptr(offsets, torch.int32, "offsets", d.E + 1), _ptr(part_counts, torch.int32, "part_counts", d.P),
        _ptr(part_offsets, torch.int32, "part_offsets", d.P + 1),
        _ptr(row_of_assign, torch.int32, "row_of_assign", TK),
        _ptr(assign_of_row, torch.int32, "assign_of_row", TK), _stream(stream)))


def moe_permute(x, row_of_assign, topk_ids, topk_w, d: moe_dims, xp, meta_token=None, meta_slot=None,
                meta_w=None, meta_local_expert=None, stream=None):
    TK = d.T * d.K
    _check("moe_permute", lib().moe_permute(
        _ptr(x, torch.bfloat16, "x", d.T * d.H), _ptr(row_of_assign, torch.int32, "row_of_assign", TK),
        _ptr(topk_ids, torch.int32, "topk_ids", TK), _ptr(topk_w, torch.float32, "topk_w", TK), C.byref(d),
        _ptr(xp, torch.bfloat16, "xp", TK * d.H), _ptr(meta_token, torch.int32, "meta_token", TK),
        _ptr(meta_slot, torch.int32, "meta_slot", TK), _ptr(meta_w, torch.float32, "meta_w", TK),
        _ptr(meta_local_expert, torch.int32, "meta_local_expert", TK), _stream(stream)))


def set_pair_min_rows(rows: int):
    """Average rows per group from which the grouped GEMMs use the CTA-pair kernel (< 0: never)."""
    lib().moe_set_pair_min_rows(int(rows))


def moe_quantize_fp8_rows(x, q, scales, stream=None):
    """Per-row E4M3 codes (uint8, x's shape) and fp32 scales of the bf16 rows of x."""
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    if tuple(q.shape) != tuple(x.shape) or scales.numel() < rows:
        raise ValueError("shape mismatch")
    _check("moe_quantize_fp8_rows", lib().moe_quantize_fp8_rows(
        _ptr(x, torch.bfloat16, "x"), rows, cols, _ptr(q, torch.uint8, "q"), _ptr(scales, torch.float32, "scales"),
        _stream(stream)))


def quantize_fp8(x, stream=None):
    """(codes, scales) of x [..., cols] bf16, allocated here."""
    q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    s = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    moe_quantize_fp8_rows(x, q, s, stream)
    return q, s


def moe_permute_fp8(x, row_of_assign, topk_ids, topk_w, d: moe_dims, xq, xs, meta_token=None, meta_slot=None,
                    meta_w=None, meta_local_expert=None, stream=None):
    TK = d.T * d.K
    _check("moe_permute_fp8", lib().moe_permute_fp8(
        _ptr(x, torch.bfloat16, "x", d.T * d.H), _ptr(row_of_assign, torch.int32, "row_of_assign", TK),
        _ptr(topk_ids, torch.int32, "topk_ids", TK), _ptr(topk_w, torch.float32, "topk_w", TK), C.byref(d),
        _ptr(xq, torch.uint8, "xq", TK * d.H), _ptr(xs, torch.float32, "xs", TK),
        _ptr(meta_token, torch.int32, "meta_token", TK), _ptr(meta_slot, torch.int32, "meta_slot", TK),
        _ptr(meta_w, torch.float32, "meta_w", TK), _ptr(meta_local_expert, torch.int32, "meta_local_expert", TK),
        _stream(stream)))


def moe_grouped_gate_up_fp8(xq, xs, offsets, wq_gate, wq_up, s_gate, s_up, d: moe_dims, h, ws, stream=None):
    TK = d.T * d.K
    _check("moe_grouped_gate_up_fp8", lib().moe_grouped_gate_up_fp8(
        _ptr(xq, torch.uint8, "xq", TK * d.H), _ptr(xs, torch.float32, "xs", TK),
        _ptr(offsets, torch.int32, "offsets", d.E + 1), _ptr(wq_gate, torch.uint8, "wq_gate", d.E * d.F * d.H),
        _ptr(wq_up, torch.uint8, "wq_up", d.E * d.F * d.H), _ptr(s_gate, torch.float32, "s_gate", d.E * d.F),
        _ptr(s_up, torch.float32, "s_up", d.E * d.F), C.byref(d), _ptr(h, torch.bfloat16, "h", TK * d.F),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_grouped_ffn(xp, offsets, w_gate, w_up, w_down, d: moe_dims, h, y, ws, stream=None):
    TK = d.T * d.K
    _check("moe_grouped_ffn", lib().moe_grouped_ffn(
        _ptr(xp, torch.bfloat16, "xp", TK * d.H), _ptr(offsets, torch.int32, "offsets", d.E + 1),
        _ptr(w_gate, torch.bfloat16, "w_gate", d.E * d.F * d.H), _ptr(w_up, torch.bfloat16, "w_up", d.E * d.F * d.H),
        _ptr(w_down, torch.bfloat16, "w_down", d.E * d.F * d.H), C.byref(d), _ptr(h, torch.bfloat16, "h", TK * d.F),
        _ptr(y, torch.bfloat16, "y", TK * d.H), _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_grouped_gate_up(xp, offsets, w_gate, w_up, d: moe_dims, h, ws, stream=None):
    TK = d.T * d.K
    _check("moe_grouped_gate_up", lib().moe_grouped_gate_up(
        _ptr(xp, torch.bfloat16, "xp", TK * d.H), _ptr(offsets, torch.int32, "offsets", d.E + 1),
        _ptr(w_gate, torch.bfloat16, "w_gate", d.E * d.F * d.H), _ptr(w_up, torch.bfloat16, "w_up", d.E * d.F * d.H),
        C.byref(d), _ptr(h, torch.bfloat16, "h", TK * d.F), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream)))


def moe_grouped_gate_up_gather(x, assign_of_row, offsets, w_gate, w_up, d: moe_dims, h, ws, stream=None):
    """moe_grouped_gate_up on the unpermuted x [T][H]: row r is token assign_of_row[r] // K."""
    TK = d.T * d.K
    _check("moe_grouped_gate_up_gather", lib().moe_grouped_gate_up_gather(
        _ptr(x, torch.bfloat16, "x", d.T * d.H), _ptr(assign_of_row, torch.int32, "assign_of_row", TK),
        _ptr(offsets, torch.int32, "offsets", d.E + 1), _ptr(w_gate, torch.bfloat16, "w_gate", d.E * d.F * d.H),
        _ptr(w_up, torch.bfloat16, "w_up", d.E * d.F * d.H), C.byref(d), _ptr(h, torch.bfloat16, "h", TK * d.F),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_grouped_down(h, offsets, w_down, d: moe_dims, y, ws, stream=None):
    TK = d.T * d.K
    _check("moe_grouped_down", lib().moe_grouped_down(
        _ptr(h, torch.bfloat16, "h", TK * d.F), _ptr(offsets, torch.int32, "offsets", d.E + 1),
        _ptr(w_down, torch.bfloat16, "w_down", d.E * d.F * d.H), C.byref(d), _ptr(y, torch.bfloat16, "y", TK * d.H),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_combine(y, row_of_assign, topk_w, d: moe_dims, out, shared=None, stream=None):
    TK = d.T * d.K
    _check("moe_combine", lib().moe_combine(
        _ptr(y, torch.bfloat16, "y", TK * d.H), _ptr(row_of_assign, torch.int32, "row_of_assign", TK),
        _ptr(topk_w, torch.float32, "topk_w", TK), _ptr(shared, torch.bfloat16, "shared", d.T * d.H), C.byref(d),
        _ptr(out, torch.bfloat16, "out", d.T * d.H), _stream(stream)))


def moe_skew_stats(counts, d: moe_dims, d_ratio, stream=None):
    _check("moe_skew_stats", lib().moe_skew_stats(_ptr(counts, torch.int32, "counts", d.E), C.byref(d),
                                                  _ptr(d_ratio, torch.float32, "d_ratio", 1), _stream(stream)))


def moe_p95(ratios: Sequence[float]) -> float:
    arr = (C.c_float * len(ratios))(*[float(r) for r in ratios])
    return float(lib().moe_p95(arr, len(ratios)))


def moe_dense(a, w, out, ws, stream=None):
    M, Kd = a.shape
    N = w.shape[0]
    if w.shape[1] != Kd or tuple(out.shape) != (M, N):
        raise ValueError("shape mismatch")
    _check("moe_dense", lib().moe_dense(_ptr(a, torch.bfloat16, "a"), _ptr(w, torch.bfloat16, "w"), M, N, Kd,
                                        _ptr(out, torch.bfloat16, "out"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                        _stream(stream)))


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------

def alloc_layer_buffers(d: moe_dims, device="cuda", meta=True, gather=False) -> dict:
    """Device buffers for every output of moe_layer_forward (torch allocations).  gather=True
    leaves out xp: the layer's gate/up GEMM then reads the token rows in place."""
    T, TK = d.T, d.T * d.K
    i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
    e = lambda shape, dt: torch.empty(shape, dtype=dt, device=device)  # noqa: E731
    b = dict(z=e((T, d.H), bf) if d.d_model else None, logits=e((T, d.E), f32), topk_ids=e((T, d.K), i32),
             topk_w=e((T, d.K), f32), counts=e((d.E,), i32), offsets=e((d.E + 1,), i32), part_counts=e((d.P,), i32),
             part_offsets=e((d.P + 1,), i32), row_of_assign=e((TK,), i32), assign_of_row=e((TK,), i32),
             xp=None if d.fp8_dispatch or gather else e((TK, d.H), bf), meta_token=e((TK,), i32) if meta else None,
             meta_slot=e((TK,), i32) if meta else None, meta_w=e((TK,), f32) if meta else None,
             meta_local_expert=e((TK,), i32) if meta else None, h=e((TK, d.F), bf), y=e((TK, d.H), bf),
             out=e((T, d.H), bf), final_out=e((T, d.d_model), bf) if d.d_model else None, skew=e((1,), f32),
             h_shared=e((T, d.F_shared), bf) if d.F_shared else None,
             y_shared=e((T, d.H), bf) if d.F_shared else None,
             xq=e((TK, d.H), torch.uint8) if d.fp8_dispatch else None,
             xs=e((TK,), f32) if d.fp8_dispatch else None)
    return b


def attach_aux_stream(buffers: dict, stream: torch.cuda.Stream) -> dict:
    """Lets the shared expert run on ``stream`` beside the routed path (events created here)."""
    buffers["aux_stream"] = stream
    buffers["fork_event"] = torch.cuda.Event()
    buffers["join_event"] = torch.cuda.Event()
    for ev in (buffers["fork_event"], buffers["join_event"]):
        ev.record(stream)               # torch creates the CUDA event on its first record
    return buffers


def _handle(v):
    if v is None:
        return None
    if isinstance(v, torch.Tensor):
        return v.data_ptr()
    if isinstance(v, torch.cuda.Stream):
        return v.cuda_stream
    if isinstance(v, torch.cuda.Event):
        return v.cuda_event
    raise TypeError(type(v))


def _buffers_struct(b: dict) -> moe_layer_buffers:
    return moe_layer_buffers(*[_handle(b.get(n)) for n in _BUF_FIELDS])


def _weights_struct(w: dict) -> moe_layer_weights:
    return moe_layer_weights(*[(w[n].data_ptr() if w.get(n) is not None else None) for n in _W_FIELDS])


def pack_layer_weights(d: moe_dims, w_g, bias, w_gate, w_up, w_down, w_dp=None, w_upp=None, stream=None,
                       shared=None) -> dict:
    """One-time weight preparation: router split into three bf16 planes; with
    ``d.fp8_dispatch`` the gate and up weights are also quantized to E4M3 per output feature."""
    split = torch.empty((3, d.E, d.H), dtype=torch.bfloat16, device=w_g.device)
    moe_pack_router(w_g.contiguous(), d, split, stream)
    for name, t, n in (("w_gate", w_gate, d.E * d.F * d.H), ("w_up", w_up, d.E * d.F * d.H),
                       ("w_down", w_down, d.E * d.F * d.H)):
        _ptr(t, torch.bfloat16, name, n)
    if d.d_model:
        _ptr(w_dp, torch.bfloat16, "w_dp", d.H * d.d_model)
        _ptr(w_upp, torch.bfloat16, "w_upp", d.H * d.d_model)
    if bias is not None:
        _ptr(bias, torch.float32, "bias", d.E)
    sg, su, sd = shared if shared is not None else (None, None, None)
    if d.F_shared:
        for name, t in (("w_shared_gate", sg), ("w_shared_up", su), ("w_shared_down", sd)):
            _ptr(t, torch.bfloat16, name, d.F_shared * d.H)
    q = dict(w_gate_q=None, s_gate=None, w_up_q=None, s_up=None)
    if d.fp8_dispatch:
        q["w_gate_q"], q["s_gate"] = quantize_fp8(w_gate, stream)
        q["w_up_q"], q["s_up"] = quantize_fp8(w_up, stream)
    return dict(w_g_split=split, bias=bias, w_gate=w_gate, w_up=w_up, w_down=w_down, w_dp=w_dp, w_upp=w_upp,
                w_shared_gate=sg, w_shared_up=su, w_shared_down=sd, **q)


def moe_layer_forward(x, weights: dict, d: moe_dims, buffers: dict, ws, stage_events=None, stream=None):
    d_in = d.d_model or d.H
    ev = None
    if stage_events is not None:
        if len(stage_events) != MOE_NUM_STAGE_EVENTS:
            raise ValueError(f"need {MOE_NUM_STAGE_EVENTS} events")
        for e in stage_events:          # torch creates the CUDA event on its first record
            if e is not None and not e.cuda_event:
                e.record(torch.cuda.current_stream() if stream is None else stream)
        ev = (C.c_void_p * MOE_NUM_STAGE_EVENTS)(*[(e.cuda_event if e is not None else None)
                                                   for e in stage_events])
    wst, bst = _weights_struct(weights), _buffers_struct(buffers)
    _check("moe_layer_forward", lib().moe_layer_forward(
        _ptr(x, torch.bfloat16, "x", d.T * d_in), C.byref(wst), C.byref(d), C.byref(bst),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), ev, _stream(stream)))


def moe_layer_forward_host(x_host, x_dev, weights: dict, d: moe_dims, buffers: dict, ws, out_host, stream=None):
    """Host-in / host-out layer: x_host and out_host are pinned CPU tensors."""
    d_in = d.d_model or d.H
    if x_host.is_cuda or out_host.is_cuda or not x_host.is_pinned() or not out_host.is_pinned():
        raise ValueError("x_host and out_host must be pinned host tensors")
    if x_host.numel() < d.T * d_in or out_host.numel() < d.T * d_in:
        raise ValueError("host buffers too small")
    wst, bst = _weights_struct(weights), _buffers_struct(buffers)
    _check("moe_layer_forward_host", lib().moe_layer_forward_host(
        x_host.data_ptr(), _ptr(x_dev, torch.bfloat16, "x_dev", d.T * d_in), C.byref(wst), C.byref(d),
        C.byref(bst), _ptr(ws, torch.uint8, "ws"), ws.numel(), out_host.data_ptr(), _stream(stream)))


# ---------------------------------------------------------------------------
# Expert-parallel exchange (include/moe.h, "Expert-parallel exchange across GPUs")
# ---------------------------------------------------------------------------

def ep_workspace(device="cuda") -> torch.Tensor:
    ws = torch.empty(int(lib().moe_ep_workspace_bytes()), dtype=torch.uint8, device=device)
    workspace_init(ws)
    return ws


def ep_peers(recv_x: Sequence[int], recv_meta: Sequence[int], ret_y: Sequence[int], signal: Sequence[int]) -> moe_ep_peers:
    """Peer table from per-rank device addresses (ints valid in this process)."""
    R = len(recv_x)
    if not (len(recv_meta) == len(ret_y) == len(signal) == R) or R > MOE_EP_MAX_RANKS:
        raise ValueError("one address per rank for each buffer")
    p = moe_ep_peers()
    for i in range(R):
        p.recv_x[i], p.recv_meta[i], p.ret_y[i], p.signal[i] = recv_x[i], recv_meta[i], ret_y[i], signal[i]
    return p


def moe_ep_plan(counts_all, R: int, rank: int, d: moe_dims, send_base, recv_offsets, stream=None):
    El = d.E // R
    _check("moe_ep_plan", lib().moe_ep_plan(
        _ptr(counts_all, torch.int32, "counts_all", R * d.E), R, rank, C.byref(d),
        _ptr(send_base, torch.int32, "send_base", d.E), _ptr(recv_offsets, torch.int32, "recv_offsets", El + 1),
        _stream(stream)))


def moe_ep_plan_host(counts_all, R: int, rank: int, d: moe_dims):
    """(send_base [E], recv_offsets [E/R + 1]) from a host int32 array C [R][E]; no GPU."""
    import numpy as np
    c = np.ascontiguousarray(np.asarray(counts_all, dtype=np.int32).reshape(R, d.E))
    send_base = np.zeros(d.E, np.int32)
    recv_off = np.zeros(d.E // R + 1, np.int32)
    _check("moe_ep_plan_host", lib().moe_ep_plan_host(
        c.ctypes.data_as(C.c_void_p), R, rank, C.byref(d), send_base.ctypes.data_as(C.c_void_p),
        recv_off.ctypes.data_as(C.c_void_p)))
    return send_base, recv_off


def moe_ep_dispatch(x, row_of_assign, topk_ids, offsets, send_base, d: moe_dims, R: int, rank: int, cap: int,
                    peers: moe_ep_peers, epoch: int, ep_ws, stream=None):
    TK = d.T * d.K
    _check("moe_ep_dispatch", lib().moe_ep_dispatch(
        _ptr(x, torch.bfloat16, "x", d.T * d.H), _ptr(row_of_assign, torch.int32, "row_of_assign", TK),
        _ptr(topk_ids, torch.int32, "topk_ids", TK), _ptr(offsets, torch.int32, "offsets", d.E + 1),
        _ptr(send_base, torch.int32, "send_base", d.E), C.byref(d), R, rank, cap, C.byref(peers), epoch,
        _ptr(ep_ws, torch.uint8, "ep_ws"), _stream(stream)))


def moe_ep_wait(signal, R: int, phase: int, epoch: int, ep_ws, stream=None):
    _check("moe_ep_wait", lib().moe_ep_wait(_ptr(signal, torch.int32, "signal", 2 * R), R, phase, epoch,
                                            _ptr(ep_ws, torch.uint8, "ep_ws"), _stream(stream)))


def moe_ep_return(y_recv, recv_meta, recv_offsets, d: moe_dims, R: int, rank: int, cap: int, peers: moe_ep_peers,
                  epoch: int, ep_ws, stream=None):
    _check("moe_ep_return", lib().moe_ep_return(
        _ptr(y_recv, torch.bfloat16, "y_recv", cap * d.H), _ptr(recv_meta, torch.int32, "recv_meta", 2 * cap),
        _ptr(recv_offsets, torch.int32, "recv_offsets", d.E // R + 1), C.byref(d), R, rank, cap, C.byref(peers),
        epoch, _ptr(ep_ws, torch.uint8, "ep_ws"), _stream(stream)))


def ep_ipc_export(t: torch.Tensor):
    """(handle bytes, offset) naming tensor t's device memory for another process."""
    h = (C.c_uint8 * MOE_EP_IPC_HANDLE_BYTES)()
    off = C.c_uint64(0)
    _check("moe_ep_ipc_export", lib().moe_ep_ipc_export(_ptr(t, name="tensor"), h, C.byref(off)))
    return bytes(h), int(off.value)


def ep_ipc_import(handle: bytes, offset: int):
    """(base, address) of a peer's exported memory opened in this process."""
    h = (C.c_uint8 * MOE_EP_IPC_HANDLE_BYTES).from_buffer_copy(handle)
    base, ptr = C.c_void_p(), C.c_void_p()
    _check("moe_ep_ipc_import", lib().moe_ep_ipc_import(h, offset, C.byref(base), C.byref(ptr)))
    return int(base.value), int(ptr.value)


def ep_ipc_close(base: int):
    _check("moe_ep_ipc_close", lib().moe_ep_ipc_close(base))
