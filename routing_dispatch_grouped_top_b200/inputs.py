"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle.

This module draws random numbers and lays them out; it holds none of the
layer's arithmetic (no routing, counting, permuting, FFN or combine).

Recipe (the pages name no dataset; these stand in for real activations):
* x ~ N(0, 1) in bf16, [T, d_in] (d_in = H, or the model width of the latent layer).
* Router weight W_g ~ N(0, 1/H) in fp32, [H, E] (a random Gaussian router, near-
  balanced loads).
* Expert weights in bf16 with the nn.Linear layout: W_gate, W_up ~ N(0, 1/H),
  [E][F][H]; W_down ~ N(0, 1/F), [E][H][F].
* Latent layer: W_dp ~ N(0, 1/d_model), [H][d_model]; W_up_proj ~ N(0, 1/H),
  [d_model][H].
* Shared expert (optional): like a routed expert of width F_shared.
* Skewed decode router: popularity p_r proportional to r^(-s) over ranks
  r = 1..E, ranks assigned to experts by a seeded random permutation pi, and a
  logit bias bias_e = beta * ln(p_pi(e) * E).  beta is a fixed constant,
  ZIPF_BETA, found by bisection with the CPU oracle's router (see
  ``oracle/calibrate_zipf_beta.py``) so that the p95 over 64 decode steps of
  max/mean expert load is about 4.
"""
from __future__ import annotations

import numpy as np
import torch

from .config import MoEConfig

# beta for s = 1.1, E = 256, K = 8, T = 128 (written by oracle/calibrate_zipf_beta.py).
ZIPF_BETA = {(1.1, 256, 8, 128): 0.1031}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, std, g, device, dtype):
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)


def make_tokens(cfg: MoEConfig, device="cpu", step: int = 0) -> torch.Tensor:
    """x [T, d_in] bf16 for decode/prefill step ``step``."""
    g = _gen(device, 1_000_003 * (cfg.seed + 1) + 7919 * step)
    return _randn((cfg.T, cfg.d_in), 1.0, g, device, torch.bfloat16)


def make_router(cfg: MoEConfig, device="cpu"):
    """(W_g [H, E] fp32, bias [E] fp32 or None)."""
    g = _gen(device, 17 + cfg.seed)
    w_g = _randn((cfg.H, cfg.E), cfg.H ** -0.5, g, device, torch.float32)
    bias = None
    if cfg.zipf_s is not None:
        beta = ZIPF_BETA.get((cfg.zipf_s, cfg.E, cfg.K, cfg.T), ZIPF_BETA[(1.1, 256, 8, 128)])
        bias = zipf_bias(cfg.E, cfg.zipf_s, beta, seed=cfg.seed, device=device)
    return w_g, bias


def zipf_bias(E: int, s: float, beta: float, seed: int = 0, device="cpu") -> torch.Tensor:
    g = _gen("cpu", 31 + seed)
    perm = torch.randperm(E, generator=g)
    r = torch.arange(1, E + 1, dtype=torch.float64)
    p = r ** (-s)
    p = p / p.sum()
    bias = beta * torch.log(p[perm] * E)
    return bias.to(torch.float32).to(device)


def make_experts(cfg: MoEConfig, device="cpu"):
    """(W_gate [E,F,H], W_up [E,F,H], W_down [E,H,F]) bf16, generated one expert at a time."""
    g = _gen(device, 101 + cfg.seed)
    E, F, H = cfg.E, cfg.F, cfg.H
    w_gate = torch.empty((E, F, H), dtype=torch.bfloat16, device=device)
    w_up = torch.empty((E, F, H), dtype=torch.bfloat16, device=device)
    w_down = torch.empty((E, H, F), dtype=torch.bfloat16, device=device)
    for e in range(E):
        w_gate[e] = _randn((F, H), H ** -0.5, g, device, torch.bfloat16)
        w_up[e] = _randn((F, H), H ** -0.5, g, device, torch.bfloat16)
        w_down[e] = _randn((H, F), F ** -0.5, g, device, torch.bfloat16)
    return w_gate, w_up, w_down


def make_latent(cfg: MoEConfig, device="cpu"):
    """(W_dp [H, d_model], W_up_proj [d_model, H]) bf16, or (None, None)."""
    if not cfg.d_model:
        return None, None
    g = _gen(device, 211 + cfg.seed)
    w_dp = _randn((cfg.H, cfg.d_model), cfg.d_model ** -0.5, g, device, torch.bfloat16)
    w_upp = _randn((cfg.d_model, cfg.H), cfg.H ** -0.5, g, device, torch.bfloat16)
    return w_dp, w_upp


def make_shared_expert(cfg: MoEConfig, device="cpu"):
    """(W_gate_s, W_up_s [F_shared][H], W_down_s [H][F_shared]) bf16, or None."""
    if not cfg.F_shared:
        return None
    g = _gen(device, 307 + cfg.seed)
    Fs, H = cfg.F_shared, cfg.H
    return (_randn((Fs, H), H ** -0.5, g, device, torch.bfloat16), _randn((Fs, H), H ** -0.5, g, device, torch.bfloat16),
            _randn((H, Fs), Fs ** -0.5, g, device, torch.bfloat16))


def make_layer(cfg: MoEConfig, device="cpu", step: int = 0) -> dict:
    w_g, bias = make_router(cfg, device)
    w_gate, w_up, w_down = make_experts(cfg, device)
    w_dp, w_upp = make_latent(cfg, device)
    return dict(x=make_tokens(cfg, device, step), w_g=w_g, bias=bias, w_gate=w_gate,
                w_up=w_up, w_down=w_down, w_dp=w_dp, w_upp=w_upp, shared=make_shared_expert(cfg, device))


# ---------------------------------------------------------------------------
# Stand-alone stage inputs (each stage is tested on inputs drawn directly)
# ---------------------------------------------------------------------------

def random_logits(T: int, E: int, seed: int = 0, scale: float = 1.0) -> torch.Tensor:
    g = _gen("cpu", seed)
    return torch.randn((T, E), generator=g, dtype=torch.float32) * scale


def special_logits(T: int, E: int, seed: int = 0) -> torch.Tensor:
    """Logits rich in ties, signed zeros, infinities and NaNs (values from a small set)."""
    g = _gen("cpu", seed)
    pool = torch.tensor([0.0, -0.0, 1.0, 1.0, -1.0, 2.5, float("inf"), float("-inf"),
                         float("nan"), 0.5, 0.5, -2.0], dtype=torch.float32)
    idx = torch.randint(0, pool.numel(), (T, E), generator=g)
    return pool[idx]


def nan_heavy_logits(T: int, E: int, frac: float = 0.8, seed: int = 0) -> torch.Tensor:
    """Gaussian logits with a fraction `frac` replaced by NaN and every fifth row all NaN,
    so that the top-K reaches into (and ties among) NaNs."""
    g = _gen("cpu", seed)
    l = torch.randn((T, E), generator=g, dtype=torch.float32)
    drop = torch.rand((T, E), generator=g) < frac
    drop[::5] = True
    return torch.where(drop, torch.full_like(l, float("nan")), l)


def quantized_logits(T: int, E: int, levels: int = 4, seed: int = 0) -> torch.Tensor:
    """Logits drawn from a few integer levels: every row is full of exact ties."""
    g = _gen("cpu", seed)
    return torch.randint(0, levels, (T, E), generator=g).to(torch.float32)


def random_topk_ids(T: int, E: int, K: int, seed: int = 0, zipf_s=None) -> torch.Tensor:
    """K distinct expert ids per token, uniform or with rank-Zipf popularity."""
    g = _gen("cpu", seed)
    if zipf_s is None:
        p = torch.ones(E, dtype=torch.float64)
    else:
        p = torch.arange(1, E + 1, dtype=torch.float64) ** (-zipf_s)
        p = p[torch.randperm(E, generator=g)]
    ids = torch.multinomial(p.expand(T, E).contiguous(), K, replacement=False, generator=g)
    return ids.to(torch.int32)


def random_bijection(n: int, seed: int = 0) -> torch.Tensor:
    g = _gen("cpu", seed)
    return torch.randperm(n, generator=g).to(torch.int32)


def random_weights(T: int, K: int, seed: int = 0) -> torch.Tensor:
    g = _gen("cpu", seed)
    return torch.rand((T, K), generator=g, dtype=torch.float32)


def random_bf16(shape, seed: int = 0, std: float = 1.0, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    return _randn(shape, std, g, device, torch.bfloat16)


def random_e4m3_codes(shape, seed: int = 0, spread: float = 64.0) -> torch.Tensor:
    """uint8 E4M3 bit patterns of N(0, spread^2) draws clamped to +-448 (torch's own float8
    conversion); no NaN codes."""
    g = _gen("cpu", seed)
    v = (torch.randn(shape, generator=g) * spread).clamp_(-448.0, 448.0)
    return v.to(torch.float8_e4m3fn).view(torch.uint8)


def random_scales(n: int, seed: int = 0, lo: float = 2.0 ** -9, hi: float = 2.0 ** -5) -> torch.Tensor:
    """fp32 row scales, log-uniform in [lo, hi]."""
    g = _gen("cpu", seed)
    return torch.exp(torch.empty(n).uniform_(float(np.log(lo)), float(np.log(hi)), generator=g)).to(torch.float32)


def random_counts(E: int, total: int, seed: int = 0, zipf_s=None, zero_frac: float = 0.0):
    """Per-expert row counts summing to ``total`` (some forced to zero if zero_frac > 0)."""
    g = _gen("cpu", seed)
    if zipf_s is None:
        p = torch.ones(E, dtype=torch.float64)
    else:
        p = torch.arange(1, E + 1, dtype=torch.float64) ** (-zipf_s)
        p = p[torch.randperm(E, generator=g)]
    if zero_frac > 0:
        mask = torch.rand(E, generator=g, dtype=torch.float64) < zero_frac
        mask[0] = False
        p = torch.where(mask, torch.zeros_like(p), p)
    draws = torch.multinomial(p, total, replacement=True, generator=g) if total else torch.zeros(0, dtype=torch.long)
    return torch.bincount(draws, minlength=E).to(torch.int32)


# ---------------------------------------------------------------------------
# Format conversion (bf16 tensors <-> the uint16 bit arrays the oracle takes)
# ---------------------------------------------------------------------------

def to_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(a: np.ndarray, device="cpu") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def to_np(t):
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return to_bits(t)
    return t.detach().cpu().numpy()
