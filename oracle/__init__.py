"""Plain, slow, fp64 CPU oracle for the RDA core (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA path never does, and nothing
here imports the CUDA path.

Contents
--------
- :func:`forward`, :func:`varlen`, :func:`decode_step`: the token-sequential
  fp64 recurrence (C, ``rda_oracle.c``), the definition of what the core
  computes.
- :mod:`oracle.chunked`: an independent fp64 chunked (UT/WY) evaluator, used
  only to pin "chunked equals sequential".
- :mod:`oracle.exact`: exact rational brute force and the hand-expanded closed
  form, for tiny cases.

All array arguments are numpy arrays; they are promoted to float64 exactly
(bf16 and fp32 values are exactly representable in fp64).  Layouts follow the
library: q, k ``[B,T,H,Dk]``; v, out ``[B,T,H,Dv]``; log_alpha, beta, gamma
``[B,T,H]``; states ``[B,H,Dk,Dv]`` holding S transposed (element [i][j] is
S[j][i] of the math-orientation state S, Dv x Dk).
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None


def load_library(path):
    """Loads a compiled oracle library and declares its C signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int32)
    lib.rda_oracle_forward.argtypes = [ctypes.c_int] * 5 + [dp] * 9 + [ctypes.c_double, ctypes.c_int]
    lib.rda_oracle_forward_channel.argtypes = [ctypes.c_int] * 5 + [dp] * 9 + [ctypes.c_double, ctypes.c_int]
    lib.rda_oracle_varlen.argtypes = [ctypes.c_int, ip] + [ctypes.c_int] * 3 + [dp] * 9 + [ctypes.c_double, ctypes.c_int]
    lib.rda_oracle_decode_step.argtypes = [ctypes.c_int] * 4 + [dp] * 8 + [ctypes.c_double, ctypes.c_int]
    lib.rda_oracle_varlen_channel.argtypes = lib.rda_oracle_varlen.argtypes
    lib.rda_oracle_decode_step_channel.argtypes = lib.rda_oracle_decode_step.argtypes
    lib.rda_oracle_max_threads.argtypes = []
    for f in (lib.rda_oracle_forward, lib.rda_oracle_forward_channel, lib.rda_oracle_varlen,
              lib.rda_oracle_varlen_channel, lib.rda_oracle_decode_step,
              lib.rda_oracle_decode_step_channel, lib.rda_oracle_max_threads):
        f.restype = ctypes.c_int
    return lib


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = load_library(_build.build())
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: promote exactly on the CPU
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().rda_oracle_max_threads())


def forward(q, k, v, log_alpha, beta, gamma=None, initial_state=None, scale=1.0,
            num_threads=0, lib=None):
    """Token-sequential fp64 recurrence over a fixed-length batch.

    ``log_alpha`` is ``[B,T,H]`` (one decay per token and head) or ``[B,T,H,Dk]``
    (one per key channel: column i of the state decays by alpha_i).
    Returns ``(out [B,T,H,Dv], final_state [B,H,Dk,Dv])`` as float64 arrays.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be, ga, s0 = _f64(log_alpha), _f64(beta), _f64(gamma), _f64(initial_state)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    assert k.shape == q.shape and v.shape == (B, T, H, Dv)
    per_channel = la.ndim == 4
    assert la.shape == ((B, T, H, Dk) if per_channel else (B, T, H)) and be.shape == (B, T, H)
    if ga is not None:
        assert ga.shape == (B, T, H)
    if s0 is not None:
        assert s0.shape == (B, H, Dk, Dv)
    out = np.zeros((B, T, H, Dv), np.float64)
    sf = np.zeros((B, H, Dk, Dv), np.float64)
    L = _load(lib)
    fn = L.rda_oracle_forward_channel if per_channel else L.rda_oracle_forward
    rc = fn(B, T, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(ga), _ptr(s0),
            _ptr(sf), _ptr(out), float(scale), int(num_threads))
    if rc != 0:
        raise ValueError("oracle.forward: bad arguments")
    return out, sf


def varlen(q, k, v, log_alpha, beta, cu_seqlens, gamma=None, initial_states=None,
           scale=1.0, num_threads=0):
    """Token-sequential fp64 recurrence over packed sequences.

    q, k ``[total,H,Dk]``; v ``[total,H,Dv]``; log_alpha, beta, gamma
    ``[total,H]`` (log_alpha ``[total,H,Dk]`` for per-key-channel decay);
    cu_seqlens int ``[N+1]``; initial_states ``[N,H,Dk,Dv]``.
    Returns ``(out [total,H,Dv], final_states [N,H,Dk,Dv])``.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be, ga, s0 = _f64(log_alpha), _f64(beta), _f64(gamma), _f64(initial_states)
    cu = np.ascontiguousarray(np.asarray(
        cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int32))
    total, H, Dk = q.shape
    Dv = v.shape[-1]
    N = cu.shape[0] - 1
    assert cu[0] == 0 and cu[-1] == total
    out = np.zeros((total, H, Dv), np.float64)
    sf = np.zeros((N, H, Dk, Dv), np.float64)
    assert la.shape == ((total, H, Dk) if la.ndim == 3 else (total, H))
    L = _load()
    fn = L.rda_oracle_varlen_channel if la.ndim == 3 else L.rda_oracle_varlen
    rc = fn(N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), H, Dk, Dv,
            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(ga),
            _ptr(s0), _ptr(sf), _ptr(out), float(scale), int(num_threads))
    if rc != 0:
        raise ValueError("oracle.varlen: bad arguments")
    return out, sf


def decode_step(q, k, v, log_alpha, beta, state, gamma=None, scale=1.0, num_threads=0,
                lib=None):
    """One decode step: returns ``(out [B,H,Dv], new_state [B,H,Dk,Dv])``.

    ``log_alpha`` is ``[B,H]``, or ``[B,H,Dk]`` for per-key-channel decay.
    ``state`` is not modified; a float64 copy is updated and returned.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be, ga = _f64(log_alpha), _f64(beta), _f64(gamma)
    st = _f64(state).copy()
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    out = np.zeros((B, H, Dv), np.float64)
    assert la.shape == ((B, H, Dk) if la.ndim == 3 else (B, H))
    L = _load(lib)
    fn = L.rda_oracle_decode_step_channel if la.ndim == 3 else L.rda_oracle_decode_step
    rc = fn(B, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(ga), _ptr(st),
            _ptr(out), float(scale), int(num_threads))
    if rc != 0:
        raise ValueError("oracle.decode_step: bad arguments")
    return out, st


__all__ = ["forward", "varlen", "decode_step", "max_threads"]
