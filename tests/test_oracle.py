"""Pins the fp64 oracle to things other than itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle -- a dropped term, a
wrong sign or index, a transposed operand, decaying at the wrong moment --
fails at least one of them; ``test_oracle_mutants.py`` plants such slips and
checks that they are caught.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import chunked, exact
import rda_gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "exact_tiny.json")


def _rand(seed, B, T, H, Dk, Dv, s0=True, gamma=False, decay="softplus"):
    inp = rda_gen.fixed_inputs(B, T, H, Dk, Dv, dtype=torch.float64, seed=seed, s0=s0,
                               decay=decay, gamma=gamma)
    f = lambda t: None if t is None else t.double().numpy()
    return dict(q=f(inp.q), k=f(inp.k), v=f(inp.v), log_alpha=f(inp.log_alpha),
                beta=f(inp.beta), gamma=f(inp.gamma), initial_state=f(inp.initial_state))


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------- 1. exact pins

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: f"seed{c['seed']}")
def test_golden_exact_rational(case):
    """fp64 oracle vs exact rational results stored by tests/golden/make_golden.py."""
    F = lambda m: np.array([[float(Fraction(x)) for x in r] for r in m])
    T, Dk, Dv = case["T"], case["Dk"], case["Dv"]
    q = F(case["q"]).reshape(1, T, 1, Dk)
    k = F(case["k"]).reshape(1, T, 1, Dk)
    v = F(case["v"]).reshape(1, T, 1, Dv)
    la = np.array([a * math.log(2.0) for a in case["alpha_log2"]]).reshape(1, T, 1)
    be = np.array([float(Fraction(x)) for x in case["beta"]]).reshape(1, T, 1)
    ga = (None if case["gamma"] is None
          else np.array([float(Fraction(x)) for x in case["gamma"]]).reshape(1, T, 1))
    s0 = None if case["S0"] is None else F(case["S0"]).T.reshape(1, 1, Dk, Dv)
    out, sf = oracle.forward(q, k, v, la, be, gamma=ga, initial_state=s0)
    want_out = F(case["out"])
    want_S = F(case["S_final"])
    assert np.max(np.abs(out[0, :, 0, :] - want_out)) <= 1e-14 * max(1.0, np.abs(want_out).max())
    assert np.max(np.abs(sf[0, 0].T - want_S)) <= 1e-14 * max(1.0, np.abs(want_S).max())


@pytest.mark.parametrize("seed", range(4))
def test_exact_sequential_equals_closed_form(seed):
    """The token loop equals the hand-expanded product form, exactly."""
    rng = np.random.default_rng(100 + seed)
    T, Dk, Dv = 4 + seed, 3, 2 + seed % 2
    fr = lambda: Fraction(int(rng.integers(-6, 7)), 4)
    q = [[fr() for _ in range(Dk)] for _ in range(T)]
    k = [[fr() for _ in range(Dk)] for _ in range(T)]
    v = [[fr() for _ in range(Dv)] for _ in range(T)]
    alpha = [Fraction(int(rng.integers(1, 5)), 4) for _ in range(T)]
    beta = [Fraction(int(rng.integers(0, 5)), 4) for _ in range(T)]
    gamma = [Fraction(int(rng.integers(1, 9)), 4) for _ in range(T)]
    S0 = [[fr() for _ in range(Dk)] for _ in range(Dv)]
    _, S = exact.sequential(q, k, v, alpha, beta, S0=S0, gamma=gamma)
    assert S == exact.closed_form(k, v, alpha, beta, S0=S0, gamma=gamma)


def test_exact_matches_oracle_random_dyadic():
    """Fresh random tiny case: fp64 oracle within 1e-14 of exact arithmetic."""
    rng = np.random.default_rng(7)
    T, Dk, Dv = 8, 4, 4
    qn = rng.integers(-8, 9, (T, Dk)) / 8
    kn = rng.integers(-8, 9, (T, Dk)) / 8
    vn = rng.integers(-8, 9, (T, Dv)) / 8
    m = rng.integers(0, 3, T)
    bn = rng.integers(0, 5, T) / 4
    s0n = rng.integers(-8, 9, (Dv, Dk)) / 8
    fr = lambda x: Fraction(x).limit_denominator(1 << 20)
    outs, S = exact.sequential([[fr(x) for x in r] for r in qn], [[fr(x) for x in r] for r in kn],
                               [[fr(x) for x in r] for r in vn], [Fraction(1, 2 ** int(x)) for x in m],
                               [fr(x) for x in bn], S0=[[fr(x) for x in r] for r in s0n])
    out, sf = oracle.forward(qn.reshape(1, T, 1, Dk), kn.reshape(1, T, 1, Dk), vn.reshape(1, T, 1, Dv),
                             (-m * math.log(2.0)).reshape(1, T, 1), bn.reshape(1, T, 1),
                             initial_state=s0n.T.reshape(1, 1, Dk, Dv))
    want = np.array([[float(x) for x in r] for r in outs])
    assert np.allclose(out[0, :, 0], want, rtol=0, atol=1e-13)
    assert np.allclose(sf[0, 0].T, np.array([[float(x) for x in r] for r in S]), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- 2. special cases

def test_beta0_alpha1_state_unchanged():
    d = _rand(1, 2, 17, 3, 8, 5)
    d["beta"][:] = 0.0
    d["log_alpha"][:] = 0.0
    out, sf = oracle.forward(**d)
    assert np.array_equal(sf, d["initial_state"])
    # o_t = S0 q_t with S0 (math) = initial_state^T
    want = np.einsum("bhij,bthi->bthj", d["initial_state"], d["q"])
    assert np.allclose(out, want, rtol=1e-14, atol=1e-15)


def test_beta0_pure_decay():
    d = _rand(2, 1, 23, 2, 6, 6)
    d["beta"][:] = 0.0
    out, sf = oracle.forward(**d)
    total = np.exp(d["log_alpha"].sum(axis=1))            # [B,H]
    assert np.allclose(sf, d["initial_state"] * total[:, :, None, None], rtol=1e-13, atol=1e-16)


def test_orthonormal_keys_recall():
    """alpha=1, beta=1, orthonormal keys, S0=0: S_T k_i = v_i for every i."""
    Dk, Dv, T = 16, 7, 12
    rng = np.random.default_rng(3)
    Qm, _ = np.linalg.qr(rng.standard_normal((Dk, Dk)))
    keys = Qm[:, :T].T                                       # T orthonormal rows
    vals = rng.standard_normal((T, Dv))
    q = rng.standard_normal((1, T, 1, Dk))
    out, sf = oracle.forward(q, keys.reshape(1, T, 1, Dk), vals.reshape(1, T, 1, Dv),
                             np.zeros((1, T, 1)), np.ones((1, T, 1)))
    S = sf[0, 0].T                                            # Dv x Dk
    for i in range(T):
        assert np.allclose(S @ keys[i], vals[i], rtol=0, atol=1e-13)


def test_current_key_exactness():
    """beta_t=1, |k_t|=1, q_t=k_t gives o_t = gamma_t v_t for any alpha and history."""
    d = _rand(4, 2, 40, 3, 8, 6, gamma=True)
    d["beta"][:] = 1.0
    d["q"] = d["k"].copy()
    out, _ = oracle.forward(**d)
    want = d["v"] * d["gamma"][..., None]
    assert np.allclose(out, want, rtol=0, atol=1e-12)


def test_scalar_case_first_order_recurrence():
    """Dk = Dv = 1: s_T = s_0 prod(m) + sum_t b_t v_t k_t prod_{s>t} m_s."""
    rng = np.random.default_rng(5)
    T = 30
    k = rng.uniform(-1, 1, T)
    v = rng.standard_normal(T)
    q = rng.standard_normal(T)
    b = rng.uniform(0, 1, T)
    la = -rng.uniform(0, 0.5, T)
    s0 = 0.7
    m = np.exp(la) * (1 - b * k * k)
    sT = s0 * np.prod(m) + sum(b[t] * v[t] * k[t] * np.prod(m[t + 1:]) for t in range(T))
    # outputs: o_t = q_t * s_t, s_t from the same closed form truncated at t
    s_t = [s0 * np.prod(m[:t + 1]) + sum(b[i] * v[i] * k[i] * np.prod(m[i + 1:t + 1])
                                         for i in range(t + 1)) for t in range(T)]
    out, sf = oracle.forward(q.reshape(1, T, 1, 1), k.reshape(1, T, 1, 1), v.reshape(1, T, 1, 1),
                             la.reshape(1, T, 1), b.reshape(1, T, 1),
                             initial_state=np.array(s0).reshape(1, 1, 1, 1))
    assert abs(sf.item() - sT) < 1e-13
    assert np.allclose(out.ravel(), q * np.array(s_t), rtol=1e-12, atol=1e-14)


def test_scale_multiplies_output_only():
    d = _rand(6, 1, 20, 2, 8, 8)
    o1, s1 = oracle.forward(**d)
    o2, s2 = oracle.forward(**d, scale=0.25)
    assert np.array_equal(s1, s2)
    assert np.allclose(o2, 0.25 * o1, rtol=1e-15, atol=0)


# ---------------------------------------------------------------- 3. chunked == sequential

@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 256])
def test_chunked_equals_sequential(T):
    d = _rand(10 + T, 1, T, 2, 16, 12, gamma=True)
    out, sf = oracle.forward(**d)
    out_c, sf_c = chunked.forward(**d, chunk=64)
    assert _rel(out_c, out) < 1e-12
    assert _rel(sf_c, sf) < 1e-12


def test_chunked_equals_sequential_strong_decay():
    """log alpha = -5 everywhere (the clamp value): chunk decays reach e^-320."""
    d = _rand(21, 1, 200, 2, 16, 16)
    d["log_alpha"][:] = -5.0
    out, sf = oracle.forward(**d)
    out_c, sf_c = chunked.forward(**d, chunk=64)
    assert np.all(np.isfinite(out_c)) and np.all(np.isfinite(sf_c))
    assert _rel(out_c, out) < 1e-12
    assert _rel(sf_c, sf) < 1e-12


def test_chunked_equals_sequential_long_context_decay():
    d = _rand(22, 1, 300, 1, 32, 32, decay="uniform")
    out, sf = oracle.forward(**d)
    out_c, sf_c = chunked.forward(**d, chunk=64)
    assert _rel(out_c, out) < 1e-12 and _rel(sf_c, sf) < 1e-12


# ---------------------------------------------------------------- 4. structural invariants

def test_linearity_in_v_and_s0():
    d = _rand(30, 1, 50, 2, 8, 6, s0=False)
    d2 = _rand(31, 1, 50, 2, 8, 6, s0=False)
    o1, s1 = oracle.forward(**d)
    dsum = dict(d)
    dsum["v"] = d["v"] + 3.0 * d2["v"]
    o2, s2 = oracle.forward(**{**d, "v": d2["v"]})
    o3, s3 = oracle.forward(**dsum)
    assert np.allclose(o3, o1 + 3.0 * o2, rtol=1e-12, atol=1e-12)
    assert np.allclose(s3, s1 + 3.0 * s2, rtol=1e-12, atol=1e-12)
    # linear in S0 when V = 0
    z = dict(d)
    z["v"] = np.zeros_like(d["v"])
    A = np.random.default_rng(1).standard_normal((1, 2, 8, 6))
    Bm = np.random.default_rng(2).standard_normal((1, 2, 8, 6))
    oa, sa = oracle.forward(**{**z, "initial_state": A})
    ob, sb = oracle.forward(**{**z, "initial_state": Bm})
    oab, sab = oracle.forward(**{**z, "initial_state": A - 2 * Bm})
    assert np.allclose(oab, oa - 2 * ob, rtol=1e-12, atol=1e-12)
    assert np.allclose(sab, sa - 2 * sb, rtol=1e-12, atol=1e-12)


def test_value_column_independence():
    d = _rand(32, 1, 70, 2, 8, 6)
    out, sf = oracle.forward(**d)
    for j in range(6):
        dj = dict(d)
        dj["v"] = d["v"][..., j:j + 1]
        dj["initial_state"] = d["initial_state"][..., j:j + 1]
        oj, sj = oracle.forward(**dj)
        assert np.array_equal(oj[..., 0], out[..., j])
        assert np.array_equal(sj[..., 0], sf[..., j])


@pytest.mark.parametrize("T1", [1, 37, 64, 99])
def test_split_and_carry_state(T1):
    d = _rand(33, 2, 100, 2, 8, 8, gamma=True)
    out, sf = oracle.forward(**d)
    a = {k: (v[:, :T1] if k != "initial_state" and v is not None else v) for k, v in d.items()}
    o1, s1 = oracle.forward(**a)
    b = {k: (v[:, T1:] if k != "initial_state" and v is not None else v) for k, v in d.items()}
    b["initial_state"] = s1
    o2, s2 = oracle.forward(**b)
    assert np.allclose(np.concatenate([o1, o2], axis=1), out, rtol=1e-13, atol=1e-14)
    assert np.allclose(s2, sf, rtol=1e-13, atol=1e-14)


def test_decode_steps_equal_prefill():
    d = _rand(34, 3, 12, 2, 8, 8)
    out, sf = oracle.forward(**d)
    st = d["initial_state"]
    for t in range(12):
        o, st = oracle.decode_step(d["q"][:, t], d["k"][:, t], d["v"][:, t], d["log_alpha"][:, t],
                                   d["beta"][:, t], st)
        assert np.allclose(o, out[:, t], rtol=1e-13, atol=1e-14)
    assert np.allclose(st, sf, rtol=1e-13, atol=1e-14)


def test_varlen_equals_per_sequence_loop():
    vin = rda_gen.varlen_inputs(lengths=[5, 0, 64, 1, 70], H=2, Dk=8, Dv=6, dtype=torch.float64,
                                seed=9, gamma=True)
    f = lambda t: t.double().numpy()
    out, sf = oracle.varlen(f(vin.q), f(vin.k), f(vin.v), f(vin.log_alpha), f(vin.beta),
                            vin.cu_seqlens.numpy(), gamma=f(vin.gamma),
                            initial_states=f(vin.initial_states))
    cu = vin.cu_seqlens.numpy()
    for n in range(5):
        a, b = cu[n], cu[n + 1]
        o, s = oracle.forward(f(vin.q)[None, a:b], f(vin.k)[None, a:b], f(vin.v)[None, a:b],
                              f(vin.log_alpha)[None, a:b], f(vin.beta)[None, a:b],
                              gamma=f(vin.gamma)[None, a:b],
                              initial_state=f(vin.initial_states)[n:n + 1])
        assert np.array_equal(o[0], out[a:b])
        assert np.array_equal(s[0], sf[n])
    # a zero-length sequence returns its initial state
    assert np.array_equal(sf[1], f(vin.initial_states)[1])


def test_non_expansion_bound():
    """alpha<=1, beta in [0,1], |k|=1: |S_t|_F <= |S_{t-1}|_F + beta_t |v_t|."""
    d = _rand(35, 1, 60, 1, 8, 8)
    st = d["initial_state"]
    for t in range(60):
        prev = np.linalg.norm(st)
        _, st = oracle.decode_step(d["q"][:, t], d["k"][:, t], d["v"][:, t],
                                   d["log_alpha"][:, t], d["beta"][:, t], st)
        bound = prev + d["beta"][0, t, 0] * np.linalg.norm(d["v"][0, t, 0])
        assert np.linalg.norm(st) <= bound * (1 + 1e-14)


def test_workload_generator_shapes_and_ranges():
    inp = rda_gen.workload("fp32_parity_b1_t256_h2_d64")
    assert inp.q.dtype == torch.float32 and inp.q.shape == (1, 256, 2, 64)
    assert inp.initial_state is None
    n = inp.k.double().norm(dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-6)
    assert float(inp.beta.min()) > 0 and float(inp.beta.max()) < 1
    a = inp.log_alpha.double().exp()
    assert float(a.min()) > 0.5 and float(a.max()) < 1.0
    again = rda_gen.workload("fp32_parity_b1_t256_h2_d64")
    assert torch.equal(again.v, inp.v)


# ---------------------------------------------------------------- per-key-channel decay (next row 2)

@pytest.mark.parametrize("seed", range(3))
def test_exact_per_channel_sequential_equals_closed_form(seed):
    """Per-channel decay: the token loop equals the product form with
    M_s = diag(alpha_s) (I - beta_s k_s k_s^T), exactly."""
    rng = np.random.default_rng(200 + seed)
    T, Dk, Dv = 4 + seed, 3, 2 + seed % 2
    fr = lambda: Fraction(int(rng.integers(-6, 7)), 4)
    q = [[fr() for _ in range(Dk)] for _ in range(T)]
    k = [[fr() for _ in range(Dk)] for _ in range(T)]
    v = [[fr() for _ in range(Dv)] for _ in range(T)]
    alpha = [[Fraction(int(rng.integers(1, 5)), 4) for _ in range(Dk)] for _ in range(T)]
    beta = [Fraction(int(rng.integers(0, 5)), 4) for _ in range(T)]
    gamma = [Fraction(int(rng.integers(1, 9)), 4) for _ in range(T)]
    S0 = [[fr() for _ in range(Dk)] for _ in range(Dv)]
    _, S = exact.sequential(q, k, v, alpha, beta, S0=S0, gamma=gamma)
    assert S == exact.closed_form(k, v, alpha, beta, S0=S0, gamma=gamma)


def test_per_channel_oracle_matches_exact_dyadic():
    """fp64 per-channel oracle within 1e-13 of exact arithmetic (dyadic inputs,
    per-channel alpha = 2^-m)."""
    rng = np.random.default_rng(11)
    T, Dk, Dv = 7, 4, 3
    qn = rng.integers(-8, 9, (T, Dk)) / 8
    kn = rng.integers(-8, 9, (T, Dk)) / 8
    vn = rng.integers(-8, 9, (T, Dv)) / 8
    m = rng.integers(0, 3, (T, Dk))
    bn = rng.integers(0, 5, T) / 4
    gn = rng.integers(1, 9, T) / 4
    s0n = rng.integers(-8, 9, (Dv, Dk)) / 8
    fr = lambda x: Fraction(x).limit_denominator(1 << 20)
    outs, S = exact.sequential([[fr(x) for x in r] for r in qn], [[fr(x) for x in r] for r in kn],
                               [[fr(x) for x in r] for r in vn],
                               [[Fraction(1, 2 ** int(x)) for x in r] for r in m],
                               [fr(x) for x in bn], S0=[[fr(x) for x in r] for r in s0n],
                               gamma=[fr(x) for x in gn], scale=Fraction(1, 2))
    out, sf = oracle.forward(qn.reshape(1, T, 1, Dk), kn.reshape(1, T, 1, Dk), vn.reshape(1, T, 1, Dv),
                             (-m * math.log(2.0)).reshape(1, T, 1, Dk), bn.reshape(1, T, 1),
                             gamma=gn.reshape(1, T, 1), initial_state=s0n.T.reshape(1, 1, Dk, Dv),
                             scale=0.5)
    assert np.allclose(out[0, :, 0], np.array([[float(x) for x in r] for r in outs]), rtol=0, atol=1e-13)
    assert np.allclose(sf[0, 0].T, np.array([[float(x) for x in r] for r in S]), rtol=0, atol=1e-13)


def test_per_channel_with_equal_channels_is_the_scalar_rule():
    """Every channel at the token's decay: bit-identical to the scalar oracle."""
    d = _rand(21, 2, 37, 3, 8, 5, gamma=True)
    o1, s1 = oracle.forward(**d, scale=0.75)
    d2 = dict(d)
    d2["log_alpha"] = np.repeat(d["log_alpha"][..., None], 8, axis=-1)
    o2, s2 = oracle.forward(**d2, scale=0.75)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def test_per_channel_pure_decay_scales_key_columns():
    """beta = 0: column i of the (math) state, i.e. row i of the stored
    [Dk, Dv] state, decays by prod_t alpha_t[i]; Dk != Dv so rows and columns
    cannot be confused."""
    d = _rand(22, 1, 19, 2, 6, 4)
    d["beta"][:] = 0.0
    rng = np.random.default_rng(5)
    la = -rng.uniform(0.0, 0.3, (1, 19, 2, 6))
    d["log_alpha"] = la
    _, sf = oracle.forward(**d)
    total = np.exp(la.sum(axis=1))                          # [B,H,Dk]
    assert np.allclose(sf, d["initial_state"] * total[:, :, :, None], rtol=1e-13, atol=1e-16)


@pytest.mark.parametrize("T,decay_hi", [(70, 0.5), (130, 5.0), (64, 2.0)])
def test_per_channel_chunked_equals_sequential(T, decay_hi):
    """The independent per-channel chunked derivation (oracle/chunked.py) equals
    the token-sequential per-channel oracle, ragged T and decays up to
    log alpha = -5 per channel included."""
    d = _rand(30 + T, 1, T, 2, 8, 5, gamma=True)
    rng = np.random.default_rng(T)
    d["log_alpha"] = -rng.uniform(0.0, decay_hi, (1, T, 2, 8))
    o, s = oracle.forward(**d, scale=0.5)
    oc, sc = chunked.forward(**d, scale=0.5, chunk=16)
    assert _rel(oc, o) <= 1e-12 and _rel(sc, s) <= 1e-12


def test_per_channel_varlen_equals_per_sequence_loop():
    rng = np.random.default_rng(41)
    lens = [5, 0, 70, 33]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total, H, Dk, Dv = int(cu[-1]), 2, 8, 5
    nrm = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q, k = nrm(rng.standard_normal((total, H, Dk))), nrm(rng.standard_normal((total, H, Dk)))
    v = rng.standard_normal((total, H, Dv))
    la = -rng.uniform(0.0, 0.5, (total, H, Dk))
    be, ga = rng.uniform(0, 1, (total, H)), rng.uniform(0.5, 1.5, (total, H))
    s0 = rng.standard_normal((len(lens), H, Dk, Dv)) * 0.3
    out, sf = oracle.varlen(q, k, v, la, be, cu, gamma=ga, initial_states=s0, scale=0.5)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        o1, s1 = oracle.forward(q[None, a:b], k[None, a:b], v[None, a:b], la[None, a:b], be[None, a:b],
                                gamma=ga[None, a:b], initial_state=s0[n:n + 1], scale=0.5)
        assert np.array_equal(out[a:b], o1[0]) and np.array_equal(sf[n], s1[0])


def test_per_channel_decode_steps_equal_prefill():
    d = _rand(43, 3, 9, 2, 8, 5, gamma=True)
    rng = np.random.default_rng(43)
    d["log_alpha"] = -rng.uniform(0.0, 0.6, (3, 9, 2, 8))
    o_ref, s_ref = oracle.forward(**d)
    st = d["initial_state"]
    for t in range(9):
        o, st = oracle.decode_step(d["q"][:, t], d["k"][:, t], d["v"][:, t], d["log_alpha"][:, t],
                                   d["beta"][:, t], st, gamma=d["gamma"][:, t])
        assert np.array_equal(o, o_ref[:, t])
    assert np.array_equal(st, s_ref)
