"""GPU parity of the multi-token decode (T new tokens per sequence, one pass
over the state) against the fp64 oracle's token-sequential recurrence, through
the C ABI.  Relative L2 over the whole returned tensors: <= 1e-5 for fp32
inputs, <= 1e-2 for bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
import rda_gen
from parity_util import TOL, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _run(inp, scale=1.0):
    import gated_delta_rule_rda_b200 as rda
    d = inp.to("cuda")
    state = d.initial_state.clone()
    out = rda.rda_decode_tokens(d.q, d.k, d.v, d.log_alpha, d.beta, state, write_gate=d.gamma,
                                scale=scale)
    torch.cuda.synchronize()
    return to_np(out), to_np(state)


def _check(inp, scale=1.0):
    out, st = _run(inp, scale)
    ro, rs = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, gamma=inp.gamma,
                            initial_state=inp.initial_state, scale=scale)
    tol = TOL[inp.q.dtype]
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(st))
    eo, es = rel_l2(out, ro), rel_l2(st, rs)
    assert eo <= tol and es <= tol, f"rel-L2 out {eo:.3e} state {es:.3e} (tol {tol:g})"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8])
def test_tokens_d128(cuda_device, dtype, T):
    inp = rda_gen.fixed_inputs(5, T, 4, 128, 128, dtype=dtype, seed=300 + T, s0=True, gamma=True)
    _check(inp, scale=0.5)


@pytest.mark.parametrize("Dk,Dv", [(64, 64), (64, 128), (128, 64)])
def test_tokens_shapes(cuda_device, Dk, Dv):
    inp = rda_gen.fixed_inputs(3, 3, 2, Dk, Dv, dtype=torch.float32, seed=Dk + Dv, s0=True)
    _check(inp)


def test_tokens_strong_decay(cuda_device):
    """log alpha = -5 on all 8 tokens: the old state's weight falls to e^-40."""
    inp = rda_gen.fixed_inputs(2, 8, 3, 128, 128, dtype=torch.float32, seed=311, s0=True)
    inp.log_alpha.fill_(-5.0)
    _check(inp)


def test_tokens_no_decay_unit_beta(cuda_device):
    inp = rda_gen.fixed_inputs(2, 8, 3, 128, 128, dtype=torch.float32, seed=312, s0=True)
    inp.log_alpha.fill_(0.0)
    inp.beta.fill_(1.0)
    _check(inp)


def test_one_token_matches_decode_step(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(4, 1, 3, 128, 128, dtype=torch.bfloat16, seed=313, s0=True, gamma=True)
    d = inp.to("cuda")
    s1, s2 = d.initial_state.clone(), d.initial_state.clone()
    o1 = rda.rda_decode_tokens(d.q, d.k, d.v, d.log_alpha, d.beta, s1, write_gate=d.gamma)
    o2 = rda.rda_decode_step(d.q[:, 0].contiguous(), d.k[:, 0].contiguous(), d.v[:, 0].contiguous(),
                             d.log_alpha[:, 0].contiguous(), d.beta[:, 0].contiguous(), s2,
                             write_gate=d.gamma[:, 0].contiguous())
    torch.cuda.synchronize()
    assert rel_l2(to_np(o1[:, 0]), to_np(o2)) < 1e-2
    assert rel_l2(to_np(s1), to_np(s2)) < 1e-5


def test_chained_calls_equal_one_prefill(cuda_device):
    """Two calls of 8 tokens carry the state like a 16-token prefill."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(2, 16, 2, 128, 128, dtype=torch.float32, seed=314, s0=True)
    d = inp.to("cuda")
    st = d.initial_state.clone()
    outs = []
    for t0 in (0, 8):
        sl = lambda x: x[:, t0:t0 + 8].contiguous()
        outs.append(rda.rda_decode_tokens(sl(d.q), sl(d.k), sl(d.v), sl(d.log_alpha), sl(d.beta), st))
    torch.cuda.synchronize()
    ro, rs = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                            initial_state=inp.initial_state)
    assert rel_l2(to_np(torch.cat(outs, 1)), ro) <= 1e-5
    assert rel_l2(to_np(st), rs) <= 1e-5


def test_zero_tokens_is_a_no_op(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    st = torch.randn(2, 3, 128, 128, device="cuda")
    ref = st.clone()
    q = torch.empty(2, 0, 3, 128, device="cuda", dtype=torch.bfloat16)
    g = torch.empty(2, 0, 3, device="cuda")
    out = rda.rda_decode_tokens(q, q, q, g, g, st)
    torch.cuda.synchronize()
    assert out.shape == (2, 0, 3, 128) and torch.equal(st, ref)
