"""GPU parity of packed (varlen) prefill and of the decode step against the
fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import rda_gen
from parity_util import TOL, gpu_varlen, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("host_schedule", [True, False])
def test_varlen_edge_lengths(cuda_device, dtype, host_schedule):
    lengths = [0, 1, 63, 64, 65, 130, 7, 0, 200]
    vin = rda_gen.varlen_inputs(lengths=lengths, H=3, Dk=128, Dv=128, dtype=dtype, seed=21,
                                gamma=True)
    out, sf = gpu_varlen(vin, scale=0.5, host_schedule=host_schedule)
    ro, rs = oracle.varlen(vin.q, vin.k, vin.v, vin.log_alpha, vin.beta, vin.cu_seqlens,
                           gamma=vin.gamma, initial_states=vin.initial_states, scale=0.5)
    tol = TOL[dtype]
    assert rel_l2(out, ro) <= tol and rel_l2(sf, rs) <= tol
    # each sequence on its own, including the empty ones (state passes through)
    cu = vin.cu_seqlens.numpy()
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        assert rel_l2(sf[n], rs[n]) <= tol
        if b > a:
            assert rel_l2(out[a:b], ro[a:b]) <= tol
    assert np.array_equal(sf[0], to_np(vin.initial_states[0]))


def test_varlen_dk64_dv64(cuda_device):
    vin = rda_gen.varlen_inputs(lengths=[5, 64, 100], H=2, Dk=64, Dv=64, dtype=torch.bfloat16, seed=22)
    out, sf = gpu_varlen(vin)
    ro, rs = oracle.varlen(vin.q, vin.k, vin.v, vin.log_alpha, vin.beta, vin.cu_seqlens,
                           initial_states=vin.initial_states)
    assert rel_l2(out, ro) <= 1e-2 and rel_l2(sf, rs) <= 1e-2


def test_varlen_without_states(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    vin = rda_gen.varlen_inputs(lengths=[70, 3], H=2, Dk=128, Dv=64, dtype=torch.bfloat16, seed=23,
                                s0=False)
    d = vin.to("cuda")
    out, sf = rda.rda_prefill_varlen(d.q, d.k, d.v, d.log_alpha, d.beta, d.cu_seqlens,
                                     return_final_states=False)
    torch.cuda.synchronize()
    assert sf is None
    ro, _ = oracle.varlen(vin.q, vin.k, vin.v, vin.log_alpha, vin.beta, vin.cu_seqlens)
    assert rel_l2(to_np(out), ro) <= 1e-2


def test_varlen_workload(cuda_device):
    """64 sequences of length U[128, 8192] packed, 16 heads: every output and
    every final state against the oracle (the worst sequence is reported)."""
    vin = rda_gen.workload("varlen_64seqs_128to8192_h16_d128")
    out, sf = gpu_varlen(vin)
    ro, rs = oracle.varlen(vin.q, vin.k, vin.v, vin.log_alpha, vin.beta, vin.cu_seqlens,
                           initial_states=vin.initial_states)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(sf))
    cu = vin.cu_seqlens.numpy()
    worst = max((max(rel_l2(out[cu[n]:cu[n + 1]], ro[cu[n]:cu[n + 1]]), rel_l2(sf[n], rs[n])), n)
                for n in range(len(cu) - 1))
    eo, es = rel_l2(out, ro), rel_l2(sf, rs)
    assert eo <= 1e-2 and es <= 1e-2 and worst[0] <= 1e-2, \
        f"rel-L2 out {eo:.3e} states {es:.3e}; worst sequence {worst[1]}: {worst[0]:.3e}"


# ------------------------------------------------------------------ decode

def _gpu_decode_steps(din, steps, scale=1.0, gamma=None):
    import gated_delta_rule_rda_b200 as rda
    d = din.to("cuda")
    st = d.state.clone()
    outs = []
    for t in range(steps):
        g = None if gamma is None else gamma[t].to("cuda")
        outs.append(rda.rda_decode_step(d.q[t], d.k[t], d.v[t], d.log_alpha[t], d.beta[t], st,
                                        write_gate=g, scale=scale))
    torch.cuda.synchronize()
    return np.stack([to_np(o) for o in outs]), to_np(st)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("Dk,Dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
def test_decode_small(cuda_device, dtype, Dk, Dv):
    din = rda_gen.decode_inputs(B=5, H=3, Dk=Dk, Dv=Dv, steps=6, dtype=dtype, seed=Dk + Dv)
    gamma = torch.rand(6, 5, 3) + 0.5
    out, st = _gpu_decode_steps(din, 6, scale=0.75, gamma=gamma)
    s = din.state
    ref = []
    for t in range(6):
        o, s = oracle.decode_step(din.q[t], din.k[t], din.v[t], din.log_alpha[t], din.beta[t], s,
                                  gamma=gamma[t], scale=0.75)
        ref.append(o)
    tol = TOL[dtype]
    assert rel_l2(out, np.stack(ref)) <= tol and rel_l2(st, s) <= tol


def test_decode_workload(cuda_device):
    """B=256, H=16, D=128, 128 steps: every sequence's outputs and final state."""
    din = rda_gen.workload("decode_b256_h16_d128_128steps")
    out, st = _gpu_decode_steps(din, 128)
    s = din.state
    ref = []
    for t in range(128):
        o, s = oracle.decode_step(din.q[t], din.k[t], din.v[t], din.log_alpha[t], din.beta[t], s)
        ref.append(o)
    ref = np.stack(ref)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(st))
    eo, es = rel_l2(out, ref), rel_l2(st, s)
    worst = max(max(rel_l2(out[:, b], ref[:, b]), rel_l2(st[b], s[b])) for b in range(out.shape[1]))
    assert eo <= 1e-2 and es <= 1e-2 and worst <= 1e-2, \
        f"rel-L2 out {eo:.3e} state {es:.3e}; worst sequence {worst:.3e}"


def test_decode_continues_prefill(cuda_device):
    """prefill(T tokens) then 5 decode steps == prefill(T + 5 tokens)."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(2, 205, 2, 128, 128, dtype=torch.bfloat16, seed=31, s0=True).to("cuda")
    full_o, full_s = rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                             initial_state=inp.initial_state)
    T0 = 200
    c = lambda t: t[:, :T0].contiguous()
    _, st = rda.rda_prefill_chunked(c(inp.q), c(inp.k), c(inp.v), c(inp.log_alpha), c(inp.beta),
                                    initial_state=inp.initial_state)
    outs = []
    for t in range(T0, 205):
        s = lambda x: x[:, t].contiguous()
        outs.append(rda.rda_decode_step(s(inp.q), s(inp.k), s(inp.v), s(inp.log_alpha), s(inp.beta), st))
    torch.cuda.synchronize()
    got = torch.stack(outs, 1).double().cpu().numpy()
    assert rel_l2(got, full_o[:, T0:].double().cpu().numpy()) < 1e-2
    assert rel_l2(st.double().cpu().numpy(), full_s.double().cpu().numpy()) < 1e-2
