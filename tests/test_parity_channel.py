"""GPU parity of the per-key-channel decay entry points against the fp64
oracle (log alpha with one value per key dimension), through the C ABI.
bf16 with Dk = 128 runs the chunked tensor-core path (decayed Grams split
around reference tokens, decayed K and Q images); fp32 and Dk = 64 run the
token-sequential kernel.

Relative L2 over the whole returned tensors: <= 1e-5 for fp32 inputs, <= 1e-2
for bf16 inputs, outputs and final states both.
"""
import numpy as np
import pytest
import torch

import oracle
import rda_gen
from parity_util import TOL, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _gpu(inp, scale=1.0):
    import gated_delta_rule_rda_b200 as rda
    d = inp.to("cuda")
    B, T, H, Dk = d.q.shape
    ws = rda.new_workspace(rda.rda_prefill_channel_workspace_bytes(B, T, H, Dk, d.v.shape[-1], 0), "cuda")
    out, sf = rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, write_gate=d.gamma,
                                      initial_state=d.initial_state, scale=scale, workspace=ws)
    torch.cuda.synchronize()
    assert rda.rda_read_device_error(ws) == 0
    return to_np(out), to_np(sf)


def _check(inp, scale=1.0):
    assert inp.log_alpha.dim() == 4
    out, sf = _gpu(inp, scale)
    ro, rs = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, gamma=inp.gamma,
                            initial_state=inp.initial_state, scale=scale)
    tol = TOL[inp.q.dtype]
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(sf))
    eo, es = rel_l2(out, ro), rel_l2(sf, rs)
    assert eo <= tol and es <= tol, f"rel-L2 out {eo:.3e} state {es:.3e} (tol {tol:g})"


@pytest.mark.parametrize("B,T,H,Dk,Dv", [(2, 1, 3, 64, 64), (1, 65, 2, 128, 64), (2, 130, 1, 64, 128),
                                         (1, 200, 2, 128, 128)])
def test_channel_fp32_shapes(cuda_device, B, T, H, Dk, Dv):
    inp = rda_gen.fixed_inputs(B, T, H, Dk, Dv, dtype=torch.float32, seed=300 + T, s0=True,
                               gamma=True, channel=True)
    _check(inp, scale=0.5)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_channel_bf16_ragged(cuda_device, T):
    inp = rda_gen.fixed_inputs(2, T, 3, 128, 128, dtype=torch.bfloat16, seed=310 + T, s0=True,
                               channel=True)
    _check(inp)


@pytest.mark.parametrize("B,T,H,Dv", [(1, 1, 1, 64), (3, 129, 2, 64), (1, 320, 4, 128)])
def test_channel_bf16_chunked_shapes(cuda_device, B, T, H, Dv):
    inp = rda_gen.fixed_inputs(B, T, H, 128, Dv, dtype=torch.bfloat16, seed=305 + T + Dv, s0=True,
                               gamma=True, channel=True)
    _check(inp, scale=0.5)


def test_channel_bf16_mixed_channels(cuda_device):
    """Within every token, key dims that do not decay (log alpha 0) next to dims
    at the bound (-5) and in between: the split factors of the Grams span their
    whole range."""
    inp = rda_gen.fixed_inputs(2, 200, 2, 128, 128, dtype=torch.bfloat16, seed=315, s0=True,
                               gamma=True, channel=True)
    la = inp.log_alpha.clone()
    la[..., 0::4] = 0.0
    la[..., 1::4] = -5.0
    inp.log_alpha = la
    _check(inp)


def test_channel_bf16_equal_channels_match_scalar(cuda_device):
    """Both chunked paths: per-channel with log alpha repeated over the key dims
    against the scalar call (different roundings of the same quantities)."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(2, 300, 2, 128, 128, dtype=torch.bfloat16, seed=325, s0=True, gamma=True)
    d = inp.to("cuda")
    la_ch = d.log_alpha[..., None].expand(-1, -1, -1, 128).contiguous()
    o_s, s_s = rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, write_gate=d.gamma,
                                       initial_state=d.initial_state)
    o_c, s_c = rda.rda_prefill_chunked(d.q, d.k, d.v, la_ch, d.beta, write_gate=d.gamma,
                                       initial_state=d.initial_state)
    torch.cuda.synchronize()
    assert rel_l2(to_np(o_c), to_np(o_s)) <= 1e-2 and rel_l2(to_np(s_c), to_np(s_s)) <= 1e-2


def test_channel_workspace_checked(cuda_device):
    """The chunked per-channel path needs its own (larger) workspace."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(1, 128, 2, 128, 128, dtype=torch.bfloat16, seed=335, channel=True).to("cuda")
    small = rda.rda_prefill_workspace_bytes(1, 128, 2, 128, 128, 0)
    assert rda.rda_prefill_channel_workspace_bytes(1, 128, 2, 128, 128, 0) > small
    with pytest.raises(RuntimeError, match="RDA_ERR_WORKSPACE"):
        rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                workspace=rda.new_workspace(small, "cuda"))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_channel_strong_decay(cuda_device, dtype):
    """Every log alpha in [-5, -4] (the bound the pages give for the decay)."""
    inp = rda_gen.fixed_inputs(1, 256, 2, 128, 128, dtype=dtype, seed=320, s0=True,
                               decay="strong", channel=True)
    _check(inp)


def test_channel_equal_channels_match_scalar(cuda_device):
    """Equal channels are the scalar rule: the per-channel call with log alpha
    repeated over the key dims matches the scalar call (fp32, both token-sequential)."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(2, 150, 2, 128, 64, dtype=torch.float32, seed=330, s0=True, gamma=True)
    d = inp.to("cuda")
    la_ch = d.log_alpha[..., None].expand(-1, -1, -1, 128).contiguous()
    o_s, s_s = rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, write_gate=d.gamma,
                                       initial_state=d.initial_state, scale=0.75)
    o_c, s_c = rda.rda_prefill_chunked(d.q, d.k, d.v, la_ch, d.beta, write_gate=d.gamma,
                                       initial_state=d.initial_state, scale=0.75)
    torch.cuda.synchronize()
    assert rel_l2(to_np(o_c), to_np(o_s)) <= 1e-6 and rel_l2(to_np(s_c), to_np(s_s)) <= 1e-6


def test_channel_nano_workload(cuda_device):
    """bf16, B=1, T=4096, H=16, D=128, nonzero initial state, per-channel decay."""
    _check(rda_gen.workload("nano_prefill_channel_b1_t4096_h16_d128"))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_channel_varlen_edge_lengths(cuda_device, dtype):
    import gated_delta_rule_rda_b200 as rda
    lengths = [0, 1, 63, 64, 65, 130, 7, 0, 200]
    vin = rda_gen.varlen_inputs(lengths=lengths, H=3, Dk=128, Dv=64, dtype=dtype, seed=340,
                                gamma=True, channel=True)
    d = vin.to("cuda")
    out, sf = rda.rda_prefill_varlen(d.q, d.k, d.v, d.log_alpha, d.beta, d.cu_seqlens,
                                     write_gate=d.gamma, initial_states=d.initial_states, scale=0.5,
                                     cu_seqlens_host=vin.cu_seqlens)
    torch.cuda.synchronize()
    ro, rs = oracle.varlen(vin.q, vin.k, vin.v, vin.log_alpha, vin.beta, vin.cu_seqlens,
                           gamma=vin.gamma, initial_states=vin.initial_states, scale=0.5)
    tol = TOL[dtype]
    assert rel_l2(to_np(out), ro) <= tol and rel_l2(to_np(sf), rs) <= tol
    assert np.array_equal(to_np(sf)[0], to_np(vin.initial_states[0]))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("Dk,Dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
def test_channel_decode_steps(cuda_device, dtype, Dk, Dv):
    import gated_delta_rule_rda_b200 as rda
    din = rda_gen.decode_inputs(B=5, H=3, Dk=Dk, Dv=Dv, steps=6, dtype=dtype, seed=350 + Dk + Dv,
                                channel=True)
    gamma = torch.rand(6, 5, 3) + 0.5
    d = din.to("cuda")
    st = d.state.clone()
    outs = []
    for t in range(6):
        outs.append(rda.rda_decode_step(d.q[t], d.k[t], d.v[t], d.log_alpha[t], d.beta[t], st,
                                        write_gate=gamma[t].to("cuda"), scale=0.75))
    torch.cuda.synchronize()
    s = din.state
    ref = []
    for t in range(6):
        o, s = oracle.decode_step(din.q[t], din.k[t], din.v[t], din.log_alpha[t], din.beta[t], s,
                                  gamma=gamma[t], scale=0.75)
        ref.append(o)
    tol = TOL[dtype]
    got = np.stack([to_np(o) for o in outs])
    assert rel_l2(got, np.stack(ref)) <= tol and rel_l2(to_np(st), s) <= tol


def test_channel_decode_continues_prefill(cuda_device):
    """Per-channel prefill of T tokens then 5 per-channel decode steps equals the
    per-channel prefill of T + 5 tokens (fp32)."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(2, 105, 2, 128, 128, dtype=torch.float32, seed=360, s0=True,
                               channel=True).to("cuda")
    full_o, full_s = rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                             initial_state=inp.initial_state)
    c = lambda t: t[:, :100].contiguous()
    _, st = rda.rda_prefill_chunked(c(inp.q), c(inp.k), c(inp.v), c(inp.log_alpha), c(inp.beta),
                                    initial_state=inp.initial_state)
    outs = []
    for t in range(100, 105):
        s = lambda x: x[:, t].contiguous()
        outs.append(rda.rda_decode_step(s(inp.q), s(inp.k), s(inp.v), s(inp.log_alpha), s(inp.beta), st))
    torch.cuda.synchronize()
    got = torch.stack(outs, 1)
    assert rel_l2(to_np(got), to_np(full_o[:, 100:])) <= 1e-5
    assert rel_l2(to_np(st), to_np(full_s)) <= 1e-5


def test_channel_bf16_decode_continues_chunked_prefill(cuda_device):
    """bf16, Dk = 128: the chunked per-channel prefill of T tokens, then 5
    per-channel decode steps from its final state, equals the chunked prefill of
    T + 5 tokens (the state the chunked path hands over is the rule's state)."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(2, 135, 2, 128, 128, dtype=torch.bfloat16, seed=365, s0=True,
                               gamma=True, channel=True).to("cuda")
    full_o, full_s = rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                             write_gate=inp.gamma, initial_state=inp.initial_state)
    c = lambda t: t[:, :130].contiguous()
    _, st = rda.rda_prefill_chunked(c(inp.q), c(inp.k), c(inp.v), c(inp.log_alpha), c(inp.beta),
                                    write_gate=c(inp.gamma), initial_state=inp.initial_state)
    outs = []
    for t in range(130, 135):
        s = lambda x: x[:, t].contiguous()
        outs.append(rda.rda_decode_step(s(inp.q), s(inp.k), s(inp.v), s(inp.log_alpha), s(inp.beta), st,
                                        write_gate=s(inp.gamma)))
    torch.cuda.synchronize()
    got = torch.stack(outs, 1)
    assert rel_l2(to_np(got), to_np(full_o[:, 130:])) <= 1e-2
    assert rel_l2(to_np(st), to_np(full_s)) <= 1e-2


def test_channel_bf16_no_initial_state(cuda_device):
    """The chunked per-channel path from a zero state (no initial state given)."""
    inp = rda_gen.fixed_inputs(2, 193, 2, 128, 128, dtype=torch.bfloat16, seed=370, s0=False,
                               gamma=True, channel=True)
    assert inp.initial_state is None
    _check(inp)


def test_channel_bf16_in_place_final_state(cuda_device):
    """final_state may alias initial_state on the chunked per-channel path, over
    an odd number of chunks with a ragged tail."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(2, 64 * 9 + 7, 3, 128, 64, dtype=torch.bfloat16, seed=375, s0=True,
                               channel=True)
    ro, rs = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, initial_state=inp.initial_state)
    d = inp.to("cuda")
    st = d.initial_state.clone()
    out, _ = rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, initial_state=st, final_state=st)
    torch.cuda.synchronize()
    assert rel_l2(to_np(st), rs) <= 1e-2 and rel_l2(to_np(out), ro) <= 1e-2
