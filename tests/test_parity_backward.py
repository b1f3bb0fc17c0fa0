"""GPU parity of the backward pass (rda_backward) against the fp64 gradient
oracle (``oracle.backward``: autograd of the token loop), through the C ABI.

The backward is evaluated in fp32 whatever the input dtype (bf16 inputs are
exact in fp32), so every gradient is held to relative L2 1e-4 over the whole
tensor: fp32 rounding through T reverse steps and the order of the atomic sums
over value columns stay well inside it.
"""
import numpy as np
import pytest
import torch

import rda_gen
from oracle import backward as bw
from parity_util import rel_l2, to_np

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _check(inp, d_out, d_sf, scale=1.0):
    import gated_delta_rule_rda_b200 as rda
    d = inp.to("cuda")
    g = rda.rda_backward(d.q, d.k, d.v, d.log_alpha, d.beta, d_out.to("cuda"), write_gate=d.gamma,
                         initial_state=d.initial_state, d_final_state=None if d_sf is None else d_sf.to("cuda"),
                         scale=scale)
    torch.cuda.synchronize()
    ref = bw.backward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, d_out, gamma=inp.gamma,
                      initial_state=inp.initial_state, d_final_state=d_sf, scale=scale)
    pairs = [("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("d_log_alpha", "d_log_alpha"), ("d_beta", "d_beta")]
    if inp.gamma is not None:
        pairs.append(("d_write_gate", "d_gamma"))
    if inp.initial_state is not None:
        pairs.append(("d_initial_state", "d_initial_state"))
    for got, want in pairs:
        x = to_np(g[got])
        assert np.all(np.isfinite(x)), got
        e = rel_l2(x, ref[want])
        assert e <= TOL, f"{got}: rel-L2 {e:.3e}"
    return g


def _grads(inp, seed, dtype):
    gen = torch.Generator().manual_seed(seed)
    d_out = torch.randn(inp.v.shape, generator=gen).to(dtype)
    d_sf = torch.randn(inp.q.shape[0], inp.q.shape[2], inp.q.shape[3], inp.v.shape[3], generator=gen)
    return d_out, d_sf


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 15, 16, 17, 100])
def test_backward_lengths(cuda_device, dtype, T):
    inp = rda_gen.fixed_inputs(2, T, 2, 128, 128, dtype=dtype, seed=500 + T, s0=True, gamma=True)
    d_out, d_sf = _grads(inp, 501 + T, dtype)
    _check(inp, d_out, d_sf, scale=0.75)


@pytest.mark.parametrize("Dk,Dv", [(128, 64), (64, 128), (64, 64)])
def test_backward_shapes(cuda_device, Dk, Dv):
    inp = rda_gen.fixed_inputs(1, 70, 3, Dk, Dv, dtype=torch.float32, seed=510 + Dk + Dv, s0=True, gamma=False)
    d_out, d_sf = _grads(inp, 511, torch.float32)
    _check(inp, d_out, d_sf)


def test_backward_upstream_parts(cuda_device):
    """Only d_out (no final-state gradient), and only the final-state gradient."""
    inp = rda_gen.fixed_inputs(1, 50, 2, 128, 128, dtype=torch.float32, seed=520, s0=False, gamma=False)
    d_out, d_sf = _grads(inp, 521, torch.float32)
    _check(inp, d_out, None)
    _check(inp, torch.zeros_like(d_out), d_sf)


def test_backward_medium(cuda_device):
    """bf16, B=1, T=512, H=4, D=128, nonzero initial state, write gate."""
    inp = rda_gen.fixed_inputs(1, 512, 4, 128, 128, dtype=torch.bfloat16, seed=530, s0=True, gamma=True)
    d_out, d_sf = _grads(inp, 531, torch.bfloat16)
    _check(inp, d_out, d_sf)


def test_backward_zero_length(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    q = torch.empty(2, 0, 3, 128, device="cuda")
    v = torch.empty(2, 0, 3, 64, device="cuda")
    gts = torch.empty(2, 0, 3, device="cuda")
    d_sf = torch.randn(2, 3, 128, 64, device="cuda")
    g = rda.rda_backward(q, q, v, gts, gts, v, initial_state=torch.zeros(2, 3, 128, 64, device="cuda"),
                         d_final_state=d_sf)
    torch.cuda.synchronize()
    assert torch.equal(g["d_initial_state"], d_sf)
