"""Seeded synthetic inputs for the RDA core.

This module serves both the CUDA path and the oracle.  It holds none of the
method's arithmetic: it only draws random values, normalises q and k (the
workloads ask for L2-normalised keys and queries), squashes the gate draws into
their ranges and casts to the requested dtypes.

Draw order, all in fp64 from one ``numpy.random.Generator(PCG64(seed))``:
(varlen only: sequence lengths first), q, k, v, beta, log_alpha, initial state.

Distributions (the workloads this library is measured on):

- q, k ~ N(0, 1), each L2-normalised over the head dimension per (token, head);
- v ~ N(0, 1);
- beta = sigmoid(N(0, 1));
- log_alpha = -softplus(N(0, 1) + 2) * 0.1  (alpha roughly 0.60 .. 0.99), or,
  for the long-context workload, alpha ~ U(0.90, 0.9999) and log_alpha = ln(alpha);
- initial state ~ N(0, 0.01), read as variance 0.01 (standard deviation 0.1).

q, k, v are cast to the workload dtype (bf16 or fp32, round to nearest even);
log_alpha, beta and states stay fp32.  Everything is returned as CPU torch
tensors; callers move them to a device.
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

S0_STD = 0.1  # "N(0, 0.01)" read as variance 0.01


def _normal(rng, shape):
    return rng.standard_normal(shape)


def _l2norm_last(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _softplus(x):
    return np.log1p(np.exp(-np.abs(x))) + np.maximum(x, 0.0)


def _to(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype)


def draw_log_alpha(rng, shape, decay: str):
    if decay == "softplus":
        return -_softplus(_normal(rng, shape) + 2.0) * 0.1
    if decay == "uniform":
        return np.log(rng.uniform(0.90, 0.9999, size=shape))
    if decay == "strong":   # the decay's lower bound region: log alpha in [-5, -4]
        return rng.uniform(-5.0, -4.0, size=shape)
    raise ValueError(f"unknown decay distribution {decay!r}")


@dataclass
class Inputs:
    """A fixed-length batch: q, k [B,T,H,Dk]; v [B,T,H,Dv]; gates [B,T,H]."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    log_alpha: torch.Tensor
    beta: torch.Tensor
    initial_state: Optional[torch.Tensor]
    gamma: Optional[torch.Tensor] = None
    meta: dict = field(default_factory=dict)

    def to(self, device):
        f = lambda t: None if t is None else t.to(device)
        return Inputs(f(self.q), f(self.k), f(self.v), f(self.log_alpha), f(self.beta),
                      f(self.initial_state), f(self.gamma), dict(self.meta))


def fixed_inputs(B, T, H, Dk, Dv, dtype=torch.bfloat16, seed=0, s0=True, decay="softplus",
                 gamma=False, channel=False) -> Inputs:
    """Draws one fixed-length batch (see module docstring for the recipe).
    With ``channel`` log_alpha is drawn per key channel, ``[B,T,H,Dk]``."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _l2norm_last(_normal(rng, (B, T, H, Dk)))
    k = _l2norm_last(_normal(rng, (B, T, H, Dk)))
    v = _normal(rng, (B, T, H, Dv))
    beta = _sigmoid(_normal(rng, (B, T, H)))
    la = draw_log_alpha(rng, (B, T, H, Dk) if channel else (B, T, H), decay)
    st = _normal(rng, (B, H, Dk, Dv)) * S0_STD if s0 else None
    ga = None
    if gamma:
        # A write gate sigma(b + d) / sigma(b) for random b, d: positive, around 1.
        braw = _normal(rng, (B, T, H))
        d = _normal(rng, (B, T, H)) * 0.5
        ga = _to(_sigmoid(braw + d) / _sigmoid(braw), torch.float32)
    return Inputs(_to(q, dtype), _to(k, dtype), _to(v, dtype), _to(la, torch.float32),
                  _to(beta, torch.float32), None if st is None else _to(st, torch.float32), ga,
                  dict(B=B, T=T, H=H, Dk=Dk, Dv=Dv, dtype=dtype, seed=seed, decay=decay,
                       channel=channel))


@dataclass
class VarlenInputs:
    """Packed sequences: q, k [total,H,Dk]; v [total,H,Dv]; gates [total,H]."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    log_alpha: torch.Tensor
    beta: torch.Tensor
    cu_seqlens: torch.Tensor       # int32 [N+1]
    initial_states: Optional[torch.Tensor]
    gamma: Optional[torch.Tensor] = None
    meta: dict = field(default_factory=dict)

    def to(self, device):
        f = lambda t: None if t is None else t.to(device)
        return VarlenInputs(f(self.q), f(self.k), f(self.v), f(self.log_alpha), f(self.beta),
                            f(self.cu_seqlens), f(self.initial_states), f(self.gamma),
                            dict(self.meta))


def varlen_inputs(lengths=None, H=16, Dk=128, Dv=128, dtype=torch.bfloat16, seed=5,
                  num_seqs=64, min_len=128, max_len=8192, s0=True, decay="softplus",
                  gamma=False, channel=False) -> VarlenInputs:
    """Draws packed sequences.  Lengths are drawn first (integers, both ends
    inclusive) unless given; then per-token tensors are drawn sequence by
    sequence in the module's order, so peak host memory stays bounded."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if lengths is None:
        lengths = rng.integers(min_len, max_len, size=num_seqs, endpoint=True)
    lengths = np.asarray(lengths, dtype=np.int64)
    N = len(lengths)
    cu = np.zeros(N + 1, np.int64)
    cu[1:] = np.cumsum(lengths)
    total = int(cu[-1])
    q = torch.empty((total, H, Dk), dtype=dtype)
    k = torch.empty((total, H, Dk), dtype=dtype)
    v = torch.empty((total, H, Dv), dtype=dtype)
    la = torch.empty((total, H, Dk) if channel else (total, H), dtype=torch.float32)
    be = torch.empty((total, H), dtype=torch.float32)
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        L = b - a
        q[a:b] = _to(_l2norm_last(_normal(rng, (L, H, Dk))), dtype)
        k[a:b] = _to(_l2norm_last(_normal(rng, (L, H, Dk))), dtype)
        v[a:b] = _to(_normal(rng, (L, H, Dv)), dtype)
        be[a:b] = _to(_sigmoid(_normal(rng, (L, H))), torch.float32)
        la[a:b] = _to(draw_log_alpha(rng, (L, H, Dk) if channel else (L, H), decay), torch.float32)
    st = _to(_normal(rng, (N, H, Dk, Dv)) * S0_STD, torch.float32) if s0 else None
    ga = None
    if gamma:
        braw = _normal(rng, (total, H))
        d = _normal(rng, (total, H)) * 0.5
        ga = _to(_sigmoid(braw + d) / _sigmoid(braw), torch.float32)
    return VarlenInputs(q, k, v, la, be, torch.from_numpy(cu.astype(np.int32)), st, ga,
                        dict(N=N, total=total, H=H, Dk=Dk, Dv=Dv, dtype=dtype, seed=seed,
                             lengths=lengths.tolist()))


@dataclass
class DecodeInputs:
    """``steps`` single-token steps for B sequences: q, k [steps,B,H,Dk];
    v [steps,B,H,Dv]; gates [steps,B,H]; state [B,H,Dk,Dv]."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    log_alpha: torch.Tensor
    beta: torch.Tensor
    state: torch.Tensor
    meta: dict = field(default_factory=dict)

    def to(self, device):
        f = lambda t: None if t is None else t.to(device)
        return DecodeInputs(f(self.q), f(self.k), f(self.v), f(self.log_alpha), f(self.beta),
                            f(self.state), dict(self.meta))


def decode_inputs(B=256, H=16, Dk=128, Dv=128, steps=128, dtype=torch.bfloat16, seed=4,
                  decay="softplus", channel=False) -> DecodeInputs:
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _l2norm_last(_normal(rng, (steps, B, H, Dk)))
    k = _l2norm_last(_normal(rng, (steps, B, H, Dk)))
    v = _normal(rng, (steps, B, H, Dv))
    beta = _sigmoid(_normal(rng, (steps, B, H)))
    la = draw_log_alpha(rng, (steps, B, H, Dk) if channel else (steps, B, H), decay)
    st = _normal(rng, (B, H, Dk, Dv)) * S0_STD
    return DecodeInputs(_to(q, dtype), _to(k, dtype), _to(v, dtype), _to(la, torch.float32),
                        _to(beta, torch.float32), _to(st, torch.float32),
                        dict(B=B, H=H, Dk=Dk, Dv=Dv, steps=steps, dtype=dtype, seed=seed))


@dataclass
class RawLayerInputs:
    """The projections' outputs an RDA layer hands to the steps before the core,
    and the parameters of those steps: q_raw, k_raw [.., H, Dk]; v_raw [.., H, Dv]
    (fixed length ``[B,T,..]`` or packed ``[total,..]`` with cu_seqlens); conv
    taps [H*D, 3]; beta_raw, delta [.., H]; log_alpha_raw [.., H] or [.., H, Dk];
    conv_window [N, 3, H*(2Dk+Dv)] (bf16); and, for the step after the core, an
    output gate g [.., H, Dv] and the norm weight [Dv]."""
    q_raw: torch.Tensor
    k_raw: torch.Tensor
    v_raw: torch.Tensor
    w_q: torch.Tensor
    w_k: torch.Tensor
    w_v: torch.Tensor
    beta_raw: torch.Tensor
    delta: torch.Tensor
    log_alpha_raw: torch.Tensor
    conv_window: torch.Tensor
    g: torch.Tensor
    norm_weight: torch.Tensor
    cu_seqlens: Optional[torch.Tensor] = None
    meta: dict = field(default_factory=dict)

    def to(self, device):
        f = lambda t: None if t is None else t.to(device)
        return RawLayerInputs(*(f(getattr(self, k)) for k in (
            "q_raw", "k_raw", "v_raw", "w_q", "w_k", "w_v", "beta_raw", "delta", "log_alpha_raw",
            "conv_window", "g", "norm_weight", "cu_seqlens")), dict(self.meta))


def raw_layer_inputs(B=None, T=None, H=2, Dk=128, Dv=128, dtype=torch.bfloat16, seed=0,
                     lengths=None, channel=False) -> RawLayerInputs:
    """Fixed length (B, T) or packed (``lengths``).  q/k/v projections, beta_raw
    and g ~ N(0, 1); delta ~ N(0, 0.25); conv taps ~ N(0, 1/3); the log decay
    before its clamp ~ U(-6, 0.2) (both ends of the clamp are reached); the
    carried window ~ N(0, 1); the norm weight ~ 1 + N(0, 0.01)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if lengths is not None:
        lengths = np.asarray(lengths, np.int64)
        cu = np.concatenate([[0], np.cumsum(lengths)])
        lead, N = (int(cu[-1]),), len(lengths)
    else:
        cu, lead, N = None, (B, T), B
    q = _normal(rng, lead + (H, Dk))
    k = _normal(rng, lead + (H, Dk))
    v = _normal(rng, lead + (H, Dv))
    w_q = _normal(rng, (H * Dk, 3)) / np.sqrt(3.0)
    w_k = _normal(rng, (H * Dk, 3)) / np.sqrt(3.0)
    w_v = _normal(rng, (H * Dv, 3)) / np.sqrt(3.0)
    br = _normal(rng, lead + (H,))
    de = _normal(rng, lead + (H,)) * 0.5
    la = rng.uniform(-6.0, 0.2, size=lead + ((H, Dk) if channel else (H,)))
    win = _normal(rng, (N, 3, H * (2 * Dk + Dv)))
    g = _normal(rng, lead + (H, Dv))
    nw = 1.0 + _normal(rng, (Dv,)) * 0.1
    f32 = lambda x: _to(x, torch.float32)
    return RawLayerInputs(_to(q, dtype), _to(k, dtype), _to(v, dtype), f32(w_q), f32(w_k), f32(w_v),
                          f32(br), f32(de), f32(la), _to(win, torch.bfloat16), _to(g, dtype), f32(nw),
                          None if cu is None else torch.from_numpy(cu.astype(np.int32)),
                          dict(B=B, T=T, H=H, Dk=Dk, Dv=Dv, dtype=dtype, seed=seed, channel=channel,
                               lengths=None if lengths is None else lengths.tolist()))


# The measured workloads.  Seeds are the workload numbers (the mini shape, H = 40, is 6).
WORKLOADS = {
    "fp32_parity_b1_t256_h2_d64": dict(kind="fixed", B=1, T=256, H=2, Dk=64, Dv=64,
                                       dtype=torch.float32, seed=1, s0=False, decay="softplus"),
    "nano_prefill_b1_t4096_h16_d128": dict(kind="fixed", B=1, T=4096, H=16, Dk=128, Dv=128,
                                           dtype=torch.bfloat16, seed=2, s0=True,
                                           decay="softplus"),
    "long_prefill_b1_t32768_h16_d128": dict(kind="fixed", B=1, T=32768, H=16, Dk=128, Dv=128,
                                            dtype=torch.bfloat16, seed=3, s0=False,
                                            decay="uniform"),
    "mini_prefill_b1_t4096_h40_d128": dict(kind="fixed", B=1, T=4096, H=40, Dk=128, Dv=128,
                                           dtype=torch.bfloat16, seed=6, s0=True,
                                           decay="softplus"),
    "decode_b256_h16_d128_128steps": dict(kind="decode", B=256, H=16, Dk=128, Dv=128,
                                          steps=128, dtype=torch.bfloat16, seed=4),
    "varlen_64seqs_128to8192_h16_d128": dict(kind="varlen", num_seqs=64, min_len=128,
                                             max_len=8192, H=16, Dk=128, Dv=128,
                                             dtype=torch.bfloat16, seed=5, s0=True),
    # per-key-channel decay at the nano shape: log alpha [B,T,H,Dk], each element
    # drawn like the scalar decay
    "nano_prefill_channel_b1_t4096_h16_d128": dict(kind="fixed", B=1, T=4096, H=16, Dk=128,
                                                   Dv=128, dtype=torch.bfloat16, seed=7, s0=True,
                                                   decay="softplus", channel=True),
}


def workload(name, **override):
    """Draws the named workload's inputs (CPU tensors)."""
    cfg = dict(WORKLOADS[name])
    cfg.update(override)
    kind = cfg.pop("kind")
    if kind == "fixed":
        return fixed_inputs(**cfg)
    if kind == "decode":
        return decode_inputs(**cfg)
    if kind == "varlen":
        return varlen_inputs(**cfg)
    raise ValueError(kind)
