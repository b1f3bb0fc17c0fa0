"""GPU parity of the steps around the core (rda_prep_inputs,
rda_output_gate_norm) against the fp64 oracle in ``oracle.prepost``, and of
prep -> core -> post against the oracles chained, through the C ABI.

Tolerances: q, k, v, out in bf16 are held to rel-L2 1e-2 (their rounding alone
is ~2e-3), in fp32 to 1e-5; beta, the write gate and the log decay (fp32 outputs)
to 1e-5; the carried bf16 window is compared exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import rda_gen
from oracle import prepost as pp
from parity_util import rel_l2, to_np

pytestmark = pytest.mark.gpu


def _flat(t, lead):
    return t.reshape((-1,) + tuple(t.shape[lead:]))


def _oracle_prep(inp, act, fixed):
    lead = 2 if fixed else 1
    if fixed:
        B, T = inp.q_raw.shape[:2]
        cu = np.arange(B + 1) * T
    else:
        cu = inp.cu_seqlens.numpy()
    return pp.prep_inputs(_flat(inp.q_raw, lead), _flat(inp.k_raw, lead), _flat(inp.v_raw, lead), inp.w_q,
                          inp.w_k, inp.w_v, _flat(inp.beta_raw, lead), _flat(inp.log_alpha_raw, lead), cu,
                          delta=_flat(inp.delta, lead), conv_window=inp.conv_window, act=act)


def _gpu_prep(inp, act, fixed, window=True, in_place=False):
    import gated_delta_rule_rda_b200 as rda
    d = inp.to("cuda")
    win_in = d.conv_window if window else None
    win_out = win_in if in_place else torch.full_like(d.conv_window, float("nan"))
    kw = {} if fixed else dict(cu_seqlens=d.cu_seqlens, max_seqlen=int(max(inp.meta["lengths"] + [0])))
    r = rda.rda_prep_inputs(d.q_raw, d.k_raw, d.v_raw, d.w_q, d.w_k, d.w_v, d.beta_raw, d.log_alpha_raw,
                            delta=d.delta, conv_window_in=win_in, conv_window_out=win_out, conv_act=act, **kw)
    torch.cuda.synchronize()
    return r, win_out


def _compare(r, win_out, ref, lead, dtype):
    tol = 1e-2 if dtype == torch.bfloat16 else 1e-5
    for name in ("q", "k", "v"):
        e = rel_l2(to_np(_flat(r[name], lead)), ref[name])
        assert e <= tol, f"{name}: rel-L2 {e:.3e}"
    for name, got in (("beta", r["beta"]), ("gamma", r["write_gate"]), ("log_alpha", r["log_alpha"])):
        e = rel_l2(to_np(_flat(got, lead)), ref[name])
        assert e <= 1e-5, f"{name}: rel-L2 {e:.3e}"
    assert np.array_equal(to_np(win_out), ref["conv_window"])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("Dk,Dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("act", [pp.ACT_SILU, pp.ACT_NONE])
def test_prep_fixed(cuda_device, dtype, Dk, Dv, act):
    inp = rda_gen.raw_layer_inputs(B=2, T=150, H=3, Dk=Dk, Dv=Dv, dtype=dtype, seed=400 + Dk + Dv + act,
                                   channel=(Dk == 128))
    r, win = _gpu_prep(inp, act, fixed=True)
    ref = _oracle_prep(inp, act, fixed=True)
    if dtype == torch.float32:
        # the carried window is bf16: compare with the rounded raw inputs
        ref["conv_window"] = ref["conv_window"].astype(np.float32).astype(np.float64)
        ref["conv_window"] = to_np(torch.from_numpy(ref["conv_window"]).to(torch.bfloat16))
    _compare(r, win, ref, 2, dtype)


def test_prep_packed_edge_lengths(cuda_device):
    lengths = [0, 1, 2, 3, 64, 65, 130, 0, 200]
    inp = rda_gen.raw_layer_inputs(H=2, Dk=128, Dv=128, dtype=torch.bfloat16, seed=410, lengths=lengths,
                                   channel=False)
    r, win = _gpu_prep(inp, pp.ACT_SILU, fixed=False)
    _compare(r, win, _oracle_prep(inp, pp.ACT_SILU, fixed=False), 1, torch.bfloat16)


def test_prep_without_window_and_in_place_window(cuda_device):
    inp = rda_gen.raw_layer_inputs(B=3, T=70, H=2, Dk=128, Dv=64, dtype=torch.bfloat16, seed=420)
    r, _ = _gpu_prep(inp, pp.ACT_SILU, fixed=True, window=False)
    inp0 = rda_gen.raw_layer_inputs(B=3, T=70, H=2, Dk=128, Dv=64, dtype=torch.bfloat16, seed=420)
    inp0.conv_window.zero_()
    ref = _oracle_prep(inp0, pp.ACT_SILU, fixed=True)
    assert rel_l2(to_np(_flat(r["q"], 2)), ref["q"]) <= 1e-2
    r2, win = _gpu_prep(inp, pp.ACT_SILU, fixed=True, in_place=True)
    _compare(r2, win, _oracle_prep(inp, pp.ACT_SILU, fixed=True), 2, torch.bfloat16)


def test_prep_split_calls_carry_the_window(cuda_device):
    """Two calls carrying the window equal one call, bit for bit (bf16)."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.raw_layer_inputs(B=2, T=200, H=2, Dk=128, Dv=128, dtype=torch.bfloat16, seed=430).to("cuda")
    args = lambda a, b: [x[:, a:b].contiguous() for x in (inp.q_raw, inp.k_raw, inp.v_raw)] + \
        [inp.w_q, inp.w_k, inp.w_v] + [x[:, a:b].contiguous() for x in (inp.beta_raw, inp.log_alpha_raw)]
    whole_win = torch.empty_like(inp.conv_window)
    whole = rda.rda_prep_inputs(*args(0, 200), delta=inp.delta, conv_window_in=inp.conv_window,
                                conv_window_out=whole_win)
    for cut in (1, 2, 64, 101):
        w1 = torch.empty_like(inp.conv_window)
        w2 = torch.empty_like(inp.conv_window)
        a = rda.rda_prep_inputs(*args(0, cut), delta=inp.delta[:, :cut].contiguous(),
                                conv_window_in=inp.conv_window, conv_window_out=w1)
        b = rda.rda_prep_inputs(*args(cut, 200), delta=inp.delta[:, cut:].contiguous(),
                                conv_window_in=w1, conv_window_out=w2)
        torch.cuda.synchronize()
        for name in ("q", "k", "v", "beta", "log_alpha"):
            assert torch.equal(torch.cat([a[name], b[name]], 1), whole[name]), (cut, name)
        assert torch.equal(w2, whole_win)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("Dv", [64, 128])
@pytest.mark.parametrize("act", [pp.ACT_SIGMOID, pp.ACT_SILU])
def test_output_gate_norm(cuda_device, dtype, Dv, act):
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.raw_layer_inputs(B=2, T=77, H=3, Dk=128, Dv=Dv, dtype=dtype, seed=440 + Dv + act)
    o = inp.v_raw
    d = inp.to("cuda")
    out = rda.rda_output_gate_norm(d.v_raw, d.g, d.norm_weight, eps=1e-5, gate_act=act)
    torch.cuda.synchronize()
    ref = pp.output_gate_norm(o, inp.g, inp.norm_weight, eps=1e-5, act=act)
    tol = 1e-2 if dtype == torch.bfloat16 else 1e-5
    assert rel_l2(to_np(out), ref) <= tol


def test_layer_prep_core_post_end_to_end(cuda_device):
    """prep -> chunked core -> output norm and gate, against the three oracles
    chained (bf16, nonzero state and window, per-head decay, write gate)."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.raw_layer_inputs(B=1, T=300, H=2, Dk=128, Dv=128, dtype=torch.bfloat16, seed=450)
    s0 = torch.randn(1, 2, 128, 128, generator=torch.Generator().manual_seed(451)) * 0.1
    d = inp.to("cuda")
    r = rda.rda_prep_inputs(d.q_raw, d.k_raw, d.v_raw, d.w_q, d.w_k, d.w_v, d.beta_raw, d.log_alpha_raw,
                            delta=d.delta, conv_window_in=d.conv_window,
                            conv_window_out=torch.empty_like(d.conv_window))
    o, sf = rda.rda_prefill_chunked(r["q"], r["k"], r["v"], r["log_alpha"], r["beta"],
                                    write_gate=r["write_gate"], initial_state=s0.to("cuda"))
    y = rda.rda_output_gate_norm(o, d.g, d.norm_weight)
    torch.cuda.synchronize()
    ref = _oracle_prep(inp, pp.ACT_SILU, fixed=True)
    sh = lambda x: x.reshape((1, 300) + x.shape[1:])
    ro, rs = oracle.forward(sh(ref["q"]), sh(ref["k"]), sh(ref["v"]), sh(ref["log_alpha"]), sh(ref["beta"]),
                            gamma=sh(ref["gamma"]), initial_state=s0)
    ry = pp.output_gate_norm(ro, inp.g, inp.norm_weight)
    assert rel_l2(to_np(y), ry) <= 1e-2 and rel_l2(to_np(sf), rs) <= 1e-2
