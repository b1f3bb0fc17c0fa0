"""Exact rational brute force of the RDA core for tiny cases (T <= 8, D <= 4).

Test infrastructure only.  Two independent exact evaluations:

- :func:`sequential`: the recurrence as the article "Raon-1 nano: half of a
  3.1B model is a lookup table, and a 99M model keeps one too" describes it in
  section "The other 1.5B: a hybrid built to forget" -- decay the state, form
  ``error = v - S k`` with the decayed state, write ``beta * error * k^T`` --
  followed by the read ``o = S q``.
- :func:`closed_form`: the hand-expanded product form of the gated delta rule
  ``S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T``::

      S_T = S_0 M_1 M_2 ... M_T + sum_t beta_t v_t k_t^T M_{t+1} ... M_T,
      M_s = alpha_s (I - beta_s k_s k_s^T),

  products ordered left to right in s.

Here alpha is given directly (a rational), not as its logarithm: one per token,
or one per token and key channel (a list of Dk rationals), in which case the
decay multiplies column i of S (key dim i) by alpha_i and ``M_s`` becomes
``diag(alpha_s) (I - beta_s k_s k_s^T)``.  Matrices are lists of lists of
``fractions.Fraction``; S is Dv x Dk (math orientation).
"""
from fractions import Fraction


def _zeros(r, c):
    return [[Fraction(0)] * c for _ in range(r)]


def _eye(n):
    m = _zeros(n, n)
    for i in range(n):
        m[i][i] = Fraction(1)
    return m


def _matmul(a, b):
    n, m, p = len(a), len(b), len(b[0])
    return [[sum((a[i][l] * b[l][j] for l in range(m)), Fraction(0)) for j in range(p)]
            for i in range(n)]


def _add(a, b):
    return [[x + y for x, y in zip(ra, rb)] for ra, rb in zip(a, b)]


def _outer(u, w):
    return [[x * y for y in w] for x in u]


def _scal(c, a):
    return [[c * x for x in r] for r in a]


def _matvec(a, x):
    return [sum((a[i][l] * x[l] for l in range(len(x))), Fraction(0)) for i in range(len(a))]


def _per_channel(a):
    return isinstance(a, (list, tuple))


def sequential(q, k, v, alpha, beta, S0=None, gamma=None, scale=Fraction(1)):
    """Exact token-sequential recurrence for one head.

    q, k: T lists of Dk Fractions; v: T lists of Dv; beta, gamma: T Fractions;
    alpha: T Fractions, or T lists of Dk Fractions (per key channel).  Returns
    ``(outs, S)`` with outs a T-list of Dv-lists and S the final Dv x Dk state.
    """
    T, Dk, Dv = len(k), len(k[0]), len(v[0])
    S = [row[:] for row in S0] if S0 is not None else _zeros(Dv, Dk)
    outs = []
    for t in range(T):
        if _per_channel(alpha[t]):                                 # decay
            S = [[S[j][i] * alpha[t][i] for i in range(Dk)] for j in range(Dv)]
        else:
            S = _scal(alpha[t], S)
        g = gamma[t] if gamma is not None else Fraction(1)
        pred = _matvec(S, k[t])
        err = [g * v[t][j] - pred[j] for j in range(Dv)]           # error
        S = _add(S, _scal(beta[t], _outer(err, k[t])))              # write
        outs.append([scale * x for x in _matvec(S, q[t])])         # read
    return outs, S


def closed_form(k, v, alpha, beta, S0=None, gamma=None):
    """Final state by the hand-expanded product form (no token loop state)."""
    T, Dk, Dv = len(k), len(k[0]), len(v[0])

    def M(s):
        P = _add(_eye(Dk), _scal(-beta[s], _outer(k[s], k[s])))
        if _per_channel(alpha[s]):
            D = _zeros(Dk, Dk)
            for i in range(Dk):
                D[i][i] = alpha[s][i]
            return _matmul(D, P)
        return _scal(alpha[s], P)

    def prod(lo):
        P = _eye(Dk)
        for s in range(lo, T):
            P = _matmul(P, M(s))
        return P

    total = _matmul(S0, prod(0)) if S0 is not None else _zeros(Dv, Dk)
    for t in range(T):
        g = gamma[t] if gamma is not None else Fraction(1)
        vt = [g * x for x in v[t]]
        total = _add(total, _matmul(_scal(beta[t], _outer(vt, k[t])), prod(t + 1)))
    return total
