"""Independent fp64 chunked (UT / WY) evaluator of the RDA core.

Test infrastructure only.  It exists to pin "a chunked evaluation equals the
token-sequential one" before any GPU code relies on the chunked form.  It
shares nothing with ``rda_oracle.c`` except the problem statement.

Derivation (math orientation: S is Dv x Dk, o = S q).  The gated delta rule
of the article "Raon-1 nano: half of a 3.1B model is a lookup table, and a 99M
model keeps one too", section "The other 1.5B: a hybrid built to forget"
(decay, then error against the decayed state, then write with strength beta)
gives, for tokens r = 1..C of one chunk entered with state S0 and with
g_r = sum_{s<=r} log alpha_s:

    S_r = e^{g_r} S0 + sum_{i<=r} e^{g_r - g_i} u_i k_i^T

where the "pseudo-values" u_i satisfy

    u_i = beta_i (v_i - e^{g_i} S0 k_i - sum_{j<i} e^{g_i - g_j} (k_j^T k_i) u_j).

Stacking rows (U: C x Dv, K: C x Dk, V: C x Dv, Q: C x Dk):

    (I + A) U = diag(beta) (V - diag(e^g) K S0^T),
    A = strictly_lower( diag(beta) (K K^T) o Gamma ),  Gamma_ri = e^{g_r - g_i}
    O = diag(e^g) Q S0^T + ((Q K^T) o Gamma_incl) U        (causal, diagonal kept)
    S_C = e^{g_C} S0 + U^T diag(e^{g_C - g}) K.

The unit lower-triangular system is solved with a library triangular solve.

Per-key-channel decay (log alpha per token and key dim; column d of S decays by
alpha_d): with G_r = sum_{s<=r} log alpha_s a vector over the key dims, the
same steps give

    S_r = S0 diag(e^{G_r}) + sum_{i<=r} u_i (k_i o e^{G_r - G_i})^T,
    u_i = beta_i (v_i - S0 (e^{G_i} o k_i) - sum_{j<i} (sum_d k_j[d] k_i[d] e^{G_i[d] - G_j[d]}) u_j),

so A_ri = beta_r sum_d k_r[d] k_i[d] e^{G_r[d] - G_i[d]} (i < r), the right-hand
side uses K o e^G, O = (Q o e^G) S0^T + P U with P_ri = sum_d q_r[d] k_i[d]
e^{G_r[d] - G_i[d]} (i <= r), and S_C = S0 diag(e^{G_C}) + U^T (K o e^{G_C - G}).
The decay Gram is no longer a product of a matrix and a rank-one mask, which is
what a kernel for this variant has to organise.
"""
import numpy as np
from scipy.linalg import solve_triangular


def _chunk(S0, Q, K, V, la, be, scale):
    """One chunk of one head.  S0 is Dv x Dk (math orientation)."""
    C = K.shape[0]
    g = np.cumsum(la)                                # g_r, r = 1..C
    diff = g[:, None] - g[None, :]                   # g_r - g_i
    lower_incl = np.tril(np.ones((C, C), dtype=bool))
    Gamma = np.where(lower_incl, np.exp(np.where(lower_incl, diff, 0.0)), 0.0)
    A = np.tril(be[:, None] * (K @ K.T) * Gamma, -1)
    rhs = be[:, None] * (V - np.exp(g)[:, None] * (K @ S0.T))
    U = solve_triangular(np.eye(C) + A, rhs, lower=True, unit_diagonal=True)
    O = np.exp(g)[:, None] * (Q @ S0.T) + ((Q @ K.T) * Gamma) @ U
    S_end = np.exp(g[-1]) * S0 + U.T @ (np.exp(g[-1] - g)[:, None] * K)
    return scale * O, S_end


def _chunk_channel(S0, Q, K, V, la, be, scale):
    """One chunk of one head with per-key-channel decay (la: C x Dk)."""
    C = K.shape[0]
    G = np.cumsum(la, axis=0)                        # G_r, C x Dk
    lower_incl = np.tril(np.ones((C, C), dtype=bool))
    diff = np.where(lower_incl[:, :, None], G[:, None, :] - G[None, :, :], 0.0)   # r, i, d
    E = np.where(lower_incl[:, :, None], np.exp(diff), 0.0)
    KK = np.einsum("rd,id,rid->ri", K, K, E)
    QK = np.einsum("rd,id,rid->ri", Q, K, E)
    A = np.tril(be[:, None] * KK, -1)
    rhs = be[:, None] * (V - (K * np.exp(G)) @ S0.T)
    U = solve_triangular(np.eye(C) + A, rhs, lower=True, unit_diagonal=True)
    O = (Q * np.exp(G)) @ S0.T + QK @ U
    S_end = S0 * np.exp(G[-1])[None, :] + U.T @ (K * np.exp(G[-1][None, :] - G))
    return scale * O, S_end


def forward(q, k, v, log_alpha, beta, gamma=None, initial_state=None, scale=1.0,
            chunk=64):
    """Chunked evaluation; same arguments and returns as :func:`oracle.forward`
    (``log_alpha`` ``[B,T,H]``, or ``[B,T,H,Dk]`` for per-key-channel decay)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    la = np.asarray(log_alpha, np.float64)
    be = np.asarray(beta, np.float64)
    B, T, H, Dk = q.shape
    step = _chunk_channel if la.ndim == 4 else _chunk
    Dv = v.shape[-1]
    if gamma is not None:
        v = v * np.asarray(gamma, np.float64)[..., None]
    out = np.zeros((B, T, H, Dv))
    sf = np.zeros((B, H, Dk, Dv))
    for b in range(B):
        for h in range(H):
            S = (np.zeros((Dv, Dk)) if initial_state is None
                 else np.asarray(initial_state, np.float64)[b, h].T.copy())
            for t0 in range(0, T, chunk):
                t1 = min(T, t0 + chunk)
                O, S = step(S, q[b, t0:t1, h], k[b, t0:t1, h], v[b, t0:t1, h],
                            la[b, t0:t1, h], be[b, t0:t1, h], scale)
                out[b, t0:t1, h] = O
            sf[b, h] = S.T
    return out, sf
