"""The per-key-channel decayed Grams the chunked kernels form, checked in fp64
on the CPU against their definition (no GPU, no oracle code).

With one decay per key dim the chunk's Gram entries are
    X[t] . (K[s] o e^{G[t] - G[s]}),   s <= t   (X = K for A, Q for P),
where G is the cumulative log decay of the chunk.  The kernels split each entry
of row block rb (rows 16 rb .. 16 rb + 15) around the block's first token
r = 16 rb: e^{G[t] - G[r]} scales the row operand and e^{G[r] - G[s]} the column
operand, so each 16 x 16 block is a plain product.  This file checks that the
split reproduces the definition, and the bounds the kernels rely on: row factors
<= 1, column factors <= 1 below the diagonal block and at most e^{15 x 5} on it
for log alpha in [-5, 0] (finite in fp32 and bf16).
"""
import numpy as np
import pytest


def _chunk(seed, mode):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((64, 128))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    Q = rng.standard_normal((64, 128))
    Q /= np.linalg.norm(Q, axis=1, keepdims=True)
    if mode == "bound":
        la = np.full((64, 128), -5.0)
    elif mode == "mixed":
        la = -rng.uniform(0.0, 5.0, (64, 128))
        la[:, 0::4] = 0.0
        la[:, 1::4] = -5.0
    else:
        la = -rng.uniform(0.01, 0.4, (64, 128))
    return K, Q, np.cumsum(la, axis=0)


def _direct(X, K, G, strict):
    n = X.shape[0]
    out = np.zeros((n, n))
    for t in range(n):
        for s in range(t if strict else t + 1):
            out[t, s] = np.sum(X[t] * K[s] * np.exp(G[t] - G[s]))
    return out


def _split(X, K, G, strict):
    out = np.zeros((64, 64))
    for rb in range(4):
        r = 16 * rb
        rows = slice(16 * rb, 16 * rb + 16)
        row_op = X[rows] * np.exp(G[rows] - G[r])          # factors <= 1
        col_op = K[: 16 * rb + 16] * np.exp(G[r] - G[: 16 * rb + 16])
        block = row_op @ col_op.T                            # [16, 16 (rb + 1)]
        t = np.arange(16 * rb, 16 * rb + 16)[:, None]
        s = np.arange(16 * rb + 16)[None, :]
        keep = s < t if strict else s <= t
        out[rows, : 16 * rb + 16] = np.where(keep, block, 0.0)
    return out


@pytest.mark.parametrize("mode", ["plain", "mixed", "bound"])
def test_split_equals_definition(mode):
    K, Q, G = _chunk(1, mode)
    for X, strict in ((K, True), (Q, False)):
        d = _direct(X, K, G, strict)
        sp = _split(X, K, G, strict)
        assert np.max(np.abs(sp - d)) <= 1e-12 * max(1.0, np.max(np.abs(d)))


@pytest.mark.parametrize("mode", ["plain", "mixed", "bound"])
def test_split_factor_bounds(mode):
    _, _, G = _chunk(2, mode)
    for rb in range(4):
        r = 16 * rb
        row_f = np.exp(G[16 * rb:16 * rb + 16] - G[r])
        assert np.all(row_f <= 1.0 + 1e-15)
        off = np.exp(G[r] - G[: 16 * rb])
        assert off.size == 0 or np.all(off <= 1.0 + 1e-15)
        diag = np.exp(G[r] - G[16 * rb:16 * rb + 16])
        assert np.all(diag <= np.exp(15 * 5.0) * (1 + 1e-12))
        assert np.all(np.isfinite(diag.astype(np.float32)))


def test_split_survives_bf16_operands():
    """The kernels round the scaled operands to bf16 (fp32 accumulation): the
    Grams stay within bf16-level error of the definition, also at the bound."""
    K, Q, G = _chunk(3, "bound")

    def bf16(x):
        a = np.asarray(x, np.float32).view(np.uint32)
        a = ((a + 0x7FFF + ((a >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
        return a.view(np.float32).astype(np.float64)

    for X, strict in ((K, True), (Q, False)):
        d = _direct(X, K, G, strict)
        out = np.zeros((64, 64))
        for rb in range(4):
            r = 16 * rb
            rows = slice(16 * rb, 16 * rb + 16)
            row_op = bf16(X[rows] * np.exp(G[rows] - G[r]))
            col_op = bf16(K[: 16 * rb + 16] * np.exp(G[r] - G[: 16 * rb + 16]))
            block = row_op @ col_op.T
            t = np.arange(16 * rb, 16 * rb + 16)[:, None]
            s = np.arange(16 * rb + 16)[None, :]
            keep = s < t if strict else s <= t
            out[rows, : 16 * rb + 16] = np.where(keep, block, 0.0)
        assert np.linalg.norm(out - d) <= 1e-2 * np.linalg.norm(d)
