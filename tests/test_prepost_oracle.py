"""Pins of the pre/post-processing oracle (``oracle.prepost``) against what
the pages and the mathematics fix, independent of the oracle's own code:

- the causal 3-tap convolution equals numpy's full convolution (a library
  routine) truncated to the causal part, and a hand-expanded tiny case exactly;
- the carried window makes a split call equal the whole call, exactly, and
  holds the last three raw inputs (short sequences shift the old window);
- the gates satisfy their closed forms: beta * gamma = sigmoid(beta_raw +
  delta), delta = 0 gives gamma = 1, the log decay is clamped to [-5, 0];
- the output norm: a constant vector maps to the norm weight times the gate,
  and the norm is scale invariant;
- planted slips (reversed taps, a dropped history, a gate without the division,
  a norm over the wrong axis) each fail one of these.
"""
import numpy as np
import pytest
from scipy.special import expit

from oracle import prepost as pp


def _rng(seed):
    return np.random.default_rng(seed)


def test_conv_equals_library_convolution():
    rng = _rng(1)
    L, C = 37, 5
    x = rng.standard_normal((L, C))
    w = rng.standard_normal((C, 3))
    y, _ = pp.short_conv(x, w)
    for c in range(C):
        # y_t = w0 x_{t-2} + w1 x_{t-1} + w2 x_t  <=>  full convolution with (w2, w1, w0)
        ref = np.convolve(x[:, c], w[c, ::-1])[:L]
        np.testing.assert_allclose(y[:, c], ref, rtol=0, atol=1e-13)


def test_conv_hand_expanded_with_window():
    # integers: every product and sum is exact in fp64
    s0, s1, s2 = 3.0, -5.0, 7.0
    a, b, c = 2.0, -1.0, 4.0
    x = np.array([[11.0], [-13.0], [17.0], [19.0]])
    y, win = pp.short_conv(x, np.array([[a, b, c]]), window=np.array([[s0], [s1], [s2]]))
    x0, x1, x2, x3 = x[:, 0]
    expect = [a * s1 + b * s2 + c * x0,
              a * s2 + b * x0 + c * x1,
              a * x0 + b * x1 + c * x2,
              a * x1 + b * x2 + c * x3]
    assert y[:, 0].tolist() == expect
    assert win[:, 0].tolist() == [x1, x2, x3]


def test_conv_short_sequence_shifts_window():
    win0 = np.array([[1.0], [2.0], [3.0]])
    y, win = pp.short_conv(np.array([[9.0]]), np.array([[0.0, 0.0, 1.0]]), window=win0)
    assert y[0, 0] == 9.0 and win[:, 0].tolist() == [2.0, 3.0, 9.0]
    _, win2 = pp.short_conv(np.array([[5.0], [6.0]]), np.array([[1.0, 0.0, 0.0]]), window=win0)
    assert win2[:, 0].tolist() == [3.0, 5.0, 6.0]


@pytest.mark.parametrize("act", [pp.ACT_NONE, pp.ACT_SILU])
def test_conv_split_equals_whole(act):
    rng = _rng(2)
    x = rng.standard_normal((50, 6))
    w = rng.standard_normal((6, 3))
    win = rng.standard_normal((3, 6))
    y, wend = pp.short_conv(x, w, win, act)
    for cut in (1, 2, 3, 17, 49):
        y1, w1 = pp.short_conv(x[:cut], w, win, act)
        y2, w2 = pp.short_conv(x[cut:], w, w1, act)
        assert np.array_equal(np.concatenate([y1, y2]), y) and np.array_equal(w2, wend)


def test_silu_closed_form():
    x = np.linspace(-8, 8, 101)
    np.testing.assert_allclose(pp.activation(x, pp.ACT_SILU), x * expit(x), rtol=1e-15, atol=1e-15)


def _prep_case(seed=3, lengths=(5, 1, 9), H=2, Dk=4, Dv=3, channel=False, window=True, delta=True):
    rng = _rng(seed)
    total = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    C = H * (2 * Dk + Dv)
    return dict(q_raw=rng.standard_normal((total, H, Dk)), k_raw=rng.standard_normal((total, H, Dk)),
                v_raw=rng.standard_normal((total, H, Dv)), w_q=rng.standard_normal((H * Dk, 3)),
                w_k=rng.standard_normal((H * Dk, 3)), w_v=rng.standard_normal((H * Dv, 3)),
                beta_raw=rng.standard_normal((total, H)),
                log_alpha_raw=rng.uniform(-7, 0.5, (total, H, Dk) if channel else (total, H)),
                cu_seqlens=cu, delta=rng.standard_normal((total, H)) if delta else None,
                conv_window=rng.standard_normal((len(lengths), 3, C)) if window else None)


def test_prep_norms_and_directions():
    case = _prep_case()
    r = pp.prep_inputs(**case, act=pp.ACT_SILU)
    np.testing.assert_allclose(np.linalg.norm(r["q"], axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(r["k"], axis=-1), 1.0, rtol=1e-14)
    # sequence 0, head 1: q is the normalised conv output of its own channels
    H, Dk = 2, 4
    y, _ = pp.short_conv(case["q_raw"][0:5].reshape(5, -1), case["w_q"], case["conv_window"][0][:, :H * Dk],
                         pp.ACT_SILU)
    y = y.reshape(5, H, Dk)[:, 1]
    np.testing.assert_allclose(r["q"][0:5, 1], y / np.linalg.norm(y, axis=-1, keepdims=True), rtol=1e-14)
    # v is the conv output, not normalised; the new window holds the last raw inputs
    assert r["conv_window"].shape == (3, 3, H * (2 * Dk + 3))
    assert np.array_equal(r["conv_window"][2, :, :H * Dk], case["q_raw"][-3:].reshape(3, -1))


def test_prep_empty_sequence_passes_window_through():
    case = _prep_case(lengths=(4, 0, 2))
    r = pp.prep_inputs(**case)
    assert np.array_equal(r["conv_window"][1], case["conv_window"][1])
    # a 2-token sequence keeps the newest old row and its two inputs
    H, Dk = 2, 4
    assert np.array_equal(r["conv_window"][2, 0, :H * Dk], case["conv_window"][2, 2, :H * Dk])
    assert np.array_equal(r["conv_window"][2, 1:, :H * Dk], case["q_raw"][4:6].reshape(2, -1))


def test_prep_sequences_do_not_leak():
    """A sequence's outputs depend only on its own tokens and its own window."""
    case = _prep_case()
    r = pp.prep_inputs(**case)
    case2 = dict(case)
    case2["q_raw"] = case["q_raw"].copy()
    case2["q_raw"][5] += 100.0                    # sequence 1's only token
    r2 = pp.prep_inputs(**case2)
    assert np.array_equal(r["q"][:5], r2["q"][:5]) and np.array_equal(r["q"][6:], r2["q"][6:])


def test_prep_gates_closed_forms():
    case = _prep_case(channel=True)
    r = pp.prep_inputs(**case)
    np.testing.assert_allclose(r["beta"], expit(case["beta_raw"]), rtol=1e-15)
    np.testing.assert_allclose(r["beta"] * r["gamma"], expit(case["beta_raw"] + case["delta"]), rtol=1e-14)
    la = case["log_alpha_raw"]
    assert np.array_equal(r["log_alpha"], np.where(la < -5, -5.0, np.where(la > 0, 0.0, la)))
    case0 = _prep_case(delta=True)
    case0["delta"] = np.zeros_like(case0["delta"])
    np.testing.assert_allclose(pp.prep_inputs(**case0)["gamma"], 1.0, rtol=1e-15)
    assert pp.prep_inputs(**_prep_case(delta=False))["gamma"] is None


def test_output_gate_norm_closed_forms():
    rng = _rng(4)
    w = rng.standard_normal(6)
    g = rng.standard_normal((3, 2, 6))
    o = np.full((3, 2, 6), 2.5)
    y = pp.output_gate_norm(o, g, w, eps=0.0, act=pp.ACT_SIGMOID)
    np.testing.assert_allclose(y, w * expit(g), rtol=1e-14)
    o = rng.standard_normal((3, 2, 6))
    np.testing.assert_allclose(pp.output_gate_norm(7.0 * o, g, w, eps=0.0), pp.output_gate_norm(o, g, w, eps=0.0),
                               rtol=1e-13)
    y = pp.output_gate_norm(o, g, np.ones(6), eps=0.0, act=pp.ACT_SILU) / (g * expit(g))
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-13)


# ---------------------------------------------------------------- planted slips

def _conv_reversed(x, w, window=None, act=pp.ACT_NONE):
    return pp.short_conv(x, w[:, ::-1], window, act)


def _conv_no_history(x, w, window=None, act=pp.ACT_NONE):
    return pp.short_conv(x, w, None, act)


def test_mutant_reversed_taps_is_caught():
    rng = _rng(5)
    x = rng.standard_normal((20, 2))
    w = rng.standard_normal((2, 3))
    y, _ = _conv_reversed(x, w)
    assert not np.allclose(y[:, 0], np.convolve(x[:, 0], w[0, ::-1])[:20])


def test_mutant_dropped_history_is_caught():
    rng = _rng(6)
    x = rng.standard_normal((10, 2))
    w = rng.standard_normal((2, 3))
    win = rng.standard_normal((3, 2))
    y, _ = pp.short_conv(x, w, win)
    y1, w1 = pp.short_conv(x[:4], w, win)
    y2, _ = _conv_no_history(x[4:], w, w1)
    assert not np.array_equal(np.concatenate([y1, y2]), y)


def test_mutant_gate_without_division_is_caught():
    rng = _rng(7)
    b, d = rng.standard_normal(10), rng.standard_normal(10)
    wrong = expit(b + d)                         # the gate without / sigmoid(b)
    assert not np.allclose(expit(b) * wrong, expit(b + d))


def test_mutant_norm_over_heads_is_caught():
    rng = _rng(8)
    o, g, w = rng.standard_normal((3, 2, 6)), rng.standard_normal((3, 2, 6)), np.ones(6)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=(-2, -1), keepdims=True))
    wrong = o * r * w * expit(g)
    y = wrong / expit(g)
    assert not np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0)
