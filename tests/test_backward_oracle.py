"""Pins of the gradient oracle (``oracle.backward``), independent of autograd:

- its forward equals the C token-sequential oracle (itself pinned by exact
  rational arithmetic), so the differentiated function is the defined one;
- every gradient matches central finite differences of that forward in fp64
  on tiny cases (random directions), with and without the write gate and the
  initial state;
- with beta = 0 nothing is written: dv and the write gate's gradient vanish;
- the gradients are linear in (d_out, d_final_state).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bw


def _case(seed, B=1, T=5, H=2, Dk=3, Dv=2, gamma=True, s0=True):
    rng = np.random.default_rng(seed)
    c = dict(q=rng.standard_normal((B, T, H, Dk)), k=rng.standard_normal((B, T, H, Dk)) / np.sqrt(Dk),
             v=rng.standard_normal((B, T, H, Dv)), log_alpha=-rng.uniform(0.01, 1.0, (B, T, H)),
             beta=rng.uniform(0.1, 0.9, (B, T, H)))
    c["gamma"] = rng.uniform(0.5, 1.5, (B, T, H)) if gamma else None
    c["initial_state"] = rng.standard_normal((B, H, Dk, Dv)) * 0.5 if s0 else None
    d = dict(d_out=rng.standard_normal((B, T, H, Dv)), d_final_state=rng.standard_normal((B, H, Dk, Dv)))
    return c, d


def test_forward_matches_c_oracle():
    c, _ = _case(1, B=2, T=9, H=2, Dk=4, Dv=3)
    o, s = bw.forward_torch(*(torch.as_tensor(c[n]) for n in ("q", "k", "v", "log_alpha", "beta")),
                            gamma=torch.as_tensor(c["gamma"]), initial_state=torch.as_tensor(c["initial_state"]),
                            scale=0.7)
    ro, rs = oracle.forward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], gamma=c["gamma"],
                            initial_state=c["initial_state"], scale=0.7)
    np.testing.assert_allclose(o.numpy(), ro, rtol=0, atol=1e-13)
    np.testing.assert_allclose(s.numpy(), rs, rtol=0, atol=1e-13)


def _loss(c, d, scale):
    o, s = oracle.forward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], gamma=c["gamma"],
                          initial_state=c["initial_state"], scale=scale)
    return float(np.sum(o * d["d_out"]) + np.sum(s * d["d_final_state"]))


@pytest.mark.parametrize("gamma,s0", [(True, True), (False, False)])
def test_gradients_match_finite_differences(gamma, s0):
    c, d = _case(2, gamma=gamma, s0=s0)
    g = bw.backward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], d["d_out"], gamma=c["gamma"],
                    initial_state=c["initial_state"], d_final_state=d["d_final_state"], scale=1.3)
    rng = np.random.default_rng(3)
    names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("log_alpha", "d_log_alpha"), ("beta", "d_beta")]
    if gamma:
        names.append(("gamma", "d_gamma"))
    if s0:
        names.append(("initial_state", "d_initial_state"))
    eps = 1e-6
    for x, gx in names:
        u = rng.standard_normal(c[x].shape)
        cp, cm = dict(c), dict(c)
        cp[x] = c[x] + eps * u
        cm[x] = c[x] - eps * u
        fd = (_loss(cp, d, 1.3) - _loss(cm, d, 1.3)) / (2 * eps)
        an = float(np.sum(g[gx] * u))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), f"{x}: fd {fd!r} analytic {an!r}"


def test_zero_strength_writes_nothing():
    c, d = _case(4)
    c["beta"] = np.zeros_like(c["beta"])
    g = bw.backward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], d["d_out"], gamma=c["gamma"],
                    initial_state=c["initial_state"], d_final_state=d["d_final_state"])
    assert np.all(g["dv"] == 0) and np.all(g["d_gamma"] == 0)


def test_gradients_are_linear_in_the_upstream_gradients():
    c, d = _case(5)
    args = (c["q"], c["k"], c["v"], c["log_alpha"], c["beta"])
    g1 = bw.backward(*args, d["d_out"], gamma=c["gamma"], initial_state=c["initial_state"],
                     d_final_state=d["d_final_state"])
    g2 = bw.backward(*args, 2.0 * d["d_out"], gamma=c["gamma"], initial_state=c["initial_state"],
                     d_final_state=2.0 * d["d_final_state"])
    for n in ("dq", "dk", "dv", "d_log_alpha", "d_beta", "d_gamma", "d_initial_state"):
        np.testing.assert_allclose(g2[n], 2.0 * g1[n], rtol=1e-12, atol=1e-13)
