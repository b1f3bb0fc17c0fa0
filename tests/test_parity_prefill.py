"""GPU parity of fixed-length prefill against the fp64 oracle (through the C ABI).

Relative L2 over the whole returned tensor: <= 1e-5 for fp32 inputs, <= 1e-2
for bf16 inputs (fp32 state and accumulation), outputs and final states both.
"""
import numpy as np
import pytest
import torch

import rda_gen
from parity_util import TOL, gpu_fixed, oracle_fixed, rel_l2

pytestmark = pytest.mark.gpu


def _check(inp, scale=1.0, tol=None):
    """Whole returned tensors against the oracle; the worst head's rel-L2 is
    reported in the assertion message as a diagnostic."""
    tol = tol or TOL[inp.q.dtype]
    out, sf = gpu_fixed(inp, scale)
    ro, rs = oracle_fixed(inp, scale)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(sf))
    eo, es = rel_l2(out, ro), rel_l2(sf, rs)
    H = ro.shape[2]
    worst_o = max(rel_l2(out[:, :, h], ro[:, :, h]) for h in range(H))
    worst_s = max(rel_l2(sf[:, h], rs[:, h]) for h in range(H))
    assert eo <= tol and es <= tol, (f"rel-L2 out {eo:.3e} state {es:.3e} (tol {tol:g}); "
                                     f"worst head out {worst_o:.3e} state {worst_s:.3e}")
    return eo, es


def test_fp32_parity_workload(cuda_device):
    """fp32, B=1, T=256, H=2, Dk=Dv=64, zero initial state."""
    _check(rda_gen.workload("fp32_parity_b1_t256_h2_d64"))


@pytest.mark.parametrize("B,T,H,Dk,Dv", [(2, 1, 3, 64, 64), (1, 63, 2, 128, 64), (2, 130, 1, 64, 128),
                                         (1, 200, 2, 128, 128), (3, 65, 2, 128, 128)])
def test_fp32_shapes(cuda_device, B, T, H, Dk, Dv):
    inp = rda_gen.fixed_inputs(B, T, H, Dk, Dv, dtype=torch.float32, seed=B * 1000 + T, s0=True,
                               gamma=True)
    _check(inp, scale=0.5)


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 128, 129, 200, 320])
@pytest.mark.parametrize("Dv", [64, 128])
def test_bf16_ragged_lengths(cuda_device, T, Dv):
    inp = rda_gen.fixed_inputs(2, T, 3, 128, Dv, dtype=torch.bfloat16, seed=T + Dv, s0=True)
    _check(inp)


@pytest.mark.parametrize("s0,gamma,scale", [(False, False, 1.0), (True, True, 0.125), (False, True, 2.0)])
def test_bf16_options(cuda_device, s0, gamma, scale):
    inp = rda_gen.fixed_inputs(1, 300, 4, 128, 128, dtype=torch.bfloat16, seed=77, s0=s0, gamma=gamma)
    _check(inp, scale=scale)


def test_bf16_dk64(cuda_device):
    inp = rda_gen.fixed_inputs(2, 150, 2, 64, 64, dtype=torch.bfloat16, seed=5, s0=True)
    _check(inp)


def test_bf16_strong_decay(cuda_device):
    """log alpha = -5 everywhere (the bound the pages give for the decay)."""
    inp = rda_gen.fixed_inputs(1, 256, 2, 128, 128, dtype=torch.bfloat16, seed=8, s0=True)
    inp.log_alpha.fill_(-5.0)
    _check(inp)


def test_bf16_no_decay_unit_beta(cuda_device):
    """alpha = 1, beta = 1: the state never forgets; long-memory stress."""
    inp = rda_gen.fixed_inputs(1, 512, 2, 128, 128, dtype=torch.bfloat16, seed=9, s0=True)
    inp.log_alpha.fill_(0.0)
    inp.beta.fill_(1.0)
    _check(inp)


def test_nano_prefill_workload(cuda_device):
    """bf16, B=1, T=4096, H=16, Dk=Dv=128, nonzero initial state -- all heads."""
    _check(rda_gen.workload("nano_prefill_b1_t4096_h16_d128"))


def test_long_context_workload(cuda_device):
    """bf16, B=1, T=32768, H=16, D=128, alpha ~ U(0.90, 0.9999): every head."""
    _check(rda_gen.workload("long_prefill_b1_t32768_h16_d128"))


def test_zero_length_copies_state(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    s0 = torch.randn(2, 3, 128, 64, device="cuda")
    q = torch.empty(2, 0, 3, 128, device="cuda", dtype=torch.bfloat16)
    v = torch.empty(2, 0, 3, 64, device="cuda", dtype=torch.bfloat16)
    g = torch.empty(2, 0, 3, device="cuda")
    out, sf = rda.rda_prefill_chunked(q, q, v, g, g, initial_state=s0)
    torch.cuda.synchronize()
    assert out.shape == (2, 0, 3, 64) and torch.equal(sf, s0)
    _, sf0 = rda.rda_prefill_chunked(q, q, v, g, g)
    torch.cuda.synchronize()
    assert torch.count_nonzero(sf0) == 0


def test_split_prefill_carries_state(cuda_device):
    """prefill(x[:T1]) then prefill(x[T1:]) from the carried state == prefill(x)."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(1, 333, 2, 128, 128, dtype=torch.bfloat16, seed=12, s0=True).to("cuda")
    full_o, full_s = rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                             initial_state=inp.initial_state)
    for T1 in (64, 100):
        sl = lambda t, a, b: t[:, a:b].contiguous()
        o1, s1 = rda.rda_prefill_chunked(sl(inp.q, 0, T1), sl(inp.k, 0, T1), sl(inp.v, 0, T1),
                                         sl(inp.log_alpha, 0, T1), sl(inp.beta, 0, T1),
                                         initial_state=inp.initial_state)
        o2, s2 = rda.rda_prefill_chunked(sl(inp.q, T1, 333), sl(inp.k, T1, 333), sl(inp.v, T1, 333),
                                         sl(inp.log_alpha, T1, 333), sl(inp.beta, T1, 333),
                                         initial_state=s1)
        torch.cuda.synchronize()
        assert rel_l2(torch.cat([o1, o2], 1).double().cpu(), full_o.double().cpu()) < 1e-2
        assert rel_l2(s2.double().cpu(), full_s.double().cpu()) < 1e-2


def test_in_place_final_state(cuda_device):
    """final_state may alias initial_state."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(1, 130, 2, 128, 128, dtype=torch.bfloat16, seed=13, s0=True)
    ro, rs = oracle_fixed(inp)
    d = inp.to("cuda")
    st = d.initial_state.clone()
    out, _ = rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, initial_state=st,
                                     final_state=st)
    torch.cuda.synchronize()
    assert rel_l2(st.double().cpu().numpy(), rs) < 1e-2
    assert rel_l2(out.double().cpu().numpy(), ro) < 1e-2


@pytest.mark.parametrize("Dv", [64, 128])
def test_bf16_long_odd_chunk_count(cuda_device, Dv):
    """38 chunks (an odd count) with a ragged tail, B > 1, write gate, and the
    final state written over the initial one."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(2, 64 * 37 + 5, 3, 128, Dv, dtype=torch.bfloat16, seed=40 + Dv, s0=True,
                               gamma=True)
    ro, rs = oracle_fixed(inp, scale=0.5)
    d = inp.to("cuda")
    st = d.initial_state.clone()
    out, _ = rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, write_gate=d.gamma,
                                     initial_state=st, final_state=st, scale=0.5)
    torch.cuda.synchronize()
    assert rel_l2(out.double().cpu().numpy(), ro) <= 1e-2
    assert rel_l2(st.double().cpu().numpy(), rs) <= 1e-2


@pytest.mark.parametrize("B,H", [(2, 12), (3, 13)])
def test_bf16_many_heads(cuda_device, B, H):
    """Many (sequence, head) pairs: the scan runs more CTAs than there are SMs,
    with value slices of 16 columns (B=2, H=12) and of 32 columns (B=3, H=13)."""
    inp = rda_gen.fixed_inputs(B, 130, H, 128, 128, dtype=torch.bfloat16, seed=B * 100 + H, s0=True,
                               gamma=True)
    _check(inp, scale=0.75)


def test_mini_shape_workload(cuda_device):
    """bf16, B=1, T=4096, H=40 (the mini model's head count), D=128: every head."""
    _check(rda_gen.workload("mini_prefill_b1_t4096_h40_d128"))
