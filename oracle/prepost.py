"""Plain fp64 oracle of the steps either side of the RDA core (test
infrastructure only, like the rest of this package).

Sources (page title and section):

- *tiny-random/raon-1-mini README*, "Printing the model": the RDA layer runs
  q, k, v through short convolutions (``q_conv1d``, ``k_conv1d``, ``v_conv1d``)
  after their projections, has a write-strength projection (``b_proj``), a
  write-gate projection (``rda_w_proj``), an output-gate projection
  (``g_proj``) and an RMSNorm over the head dimension on the output
  (``o_norm``, eps 1e-5) before ``o_proj``.
- *Raon-1 nano: half of a 3.1B model is a lookup table...*, "The cache is small
  if the runtime keeps it small": each layer carries a three-token convolution
  window next to its state; "The other 1.5B": beta is the write strength, the
  write gate is sigma(beta_raw + delta) / sigma(beta_raw), and the decay is
  bounded below by -5 in log space.
- The blog post on Raon-1 mini (vLLM pull-request section): the convolution
  history is kept in BF16.

Readings where the pages are silent (each is an argument or stated here):

- The convolution is causal and depthwise with 3 taps per channel:
  ``y_t = w[0] x_{t-2} + w[1] x_{t-1} + w[2] x_t``.  The carried window holds
  the last 3 raw inputs of each channel (oldest first), which is the size the
  nano article gives (3 tokens x 6,144 channels x 2 bytes per layer, with the
  1 MiB state: 19.5 MB for 18 layers); a call reads the 2 newest of them.
- Its activation is an argument: none, or SiLU (x sigmoid(x)), the form used by
  Kimi Delta Attention, which the pages name as what RDA modifies.
- q and k are L2-normalised per head after the convolution (the workloads'
  inputs are L2-normalised q and k); v is not.
- beta = sigmoid(beta_raw); write gate = sigmoid(beta_raw + delta) /
  sigmoid(beta_raw) (delta absent: 1); log alpha = clip(log_alpha_raw, -5, 0).
- The output is RMSNorm(o) * w_norm * act(g) per head, act = sigmoid or SiLU
  (an argument).

Layouts follow the library: per-token tensors ``[total_T, H, D]``; the conv
window ``[N, 3, C]`` with the channels of q, k and v concatenated
(C = H Dk + H Dk + H Dv); conv weights ``[channels, 3]``.
"""
import numpy as np

ACT_NONE, ACT_SILU, ACT_SIGMOID = 0, 1, 2


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def activation(x, act):
    if act == ACT_NONE:
        return x
    if act == ACT_SILU:
        return x * sigmoid(x)
    if act == ACT_SIGMOID:
        return sigmoid(x)
    raise ValueError(act)


def short_conv(x, w, window=None, act=ACT_NONE):
    """One sequence.  x [L, C]; w [C, 3] (taps for t-2, t-1, t); window [3, C]
    of the last raw inputs before x (oldest first), None for zeros.
    Returns (y [L, C], new window [3, C])."""
    x, w = _f64(x), _f64(w)
    L, C = x.shape
    win = np.zeros((3, C)) if window is None else _f64(window)
    hist = np.concatenate([win, x], axis=0)          # [3 + L, C]
    y = np.empty((L, C))
    for t in range(L):                                # row 3 + t is x_t
        y[t] = w[:, 0] * hist[t + 1] + w[:, 1] * hist[t + 2] + w[:, 2] * hist[t + 3]
    return activation(y, act), hist[-3:].copy()


def l2_normalize(x, axis=-1):
    return x / np.sqrt(np.sum(x * x, axis=axis, keepdims=True))


def prep_inputs(q_raw, k_raw, v_raw, w_q, w_k, w_v, beta_raw, log_alpha_raw, cu_seqlens,
                delta=None, conv_window=None, act=ACT_SILU):
    """Everything the core takes, from the projections' outputs.

    q_raw, k_raw [total, H, Dk]; v_raw [total, H, Dv]; w_* [H*D, 3]; beta_raw,
    delta [total, H]; log_alpha_raw [total, H] or [total, H, Dk]; cu_seqlens
    [N+1]; conv_window [N, 3, C] or None.  Returns a dict with q, k, v, beta,
    gamma (None without delta), log_alpha and the new conv_window [N, 3, C].
    """
    q_raw, k_raw, v_raw = _f64(q_raw), _f64(k_raw), _f64(v_raw)
    total, H, Dk = q_raw.shape
    Dv = v_raw.shape[-1]
    cq, ck, cv = H * Dk, H * Dk, H * Dv
    cu = np.asarray(cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, np.int64)
    N = len(cu) - 1
    win = None if conv_window is None else _f64(conv_window)
    q = np.empty((total, H, Dk))
    k = np.empty((total, H, Dk))
    v = np.empty((total, H, Dv))
    new_win = np.zeros((N, 3, cq + ck + cv))
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        wn = None if win is None else win[n]
        parts = []
        for raw, w, lo, hi, D in ((q_raw, w_q, 0, cq, Dk), (k_raw, w_k, cq, cq + ck, Dk),
                                  (v_raw, w_v, cq + ck, cq + ck + cv, Dv)):
            y, nw = short_conv(raw[a:b].reshape(b - a, hi - lo), w, None if wn is None else wn[:, lo:hi], act)
            parts.append(y.reshape(b - a, H, D))
            new_win[n, :, lo:hi] = nw
        q[a:b] = l2_normalize(parts[0])
        k[a:b] = l2_normalize(parts[1])
        v[a:b] = parts[2]
    br = _f64(beta_raw)
    beta = sigmoid(br)
    gamma = None if delta is None else sigmoid(br + _f64(delta)) / beta
    log_alpha = np.clip(_f64(log_alpha_raw), -5.0, 0.0)
    return dict(q=q, k=k, v=v, beta=beta, gamma=gamma, log_alpha=log_alpha, conv_window=new_win)


def output_gate_norm(o, g, w_norm, eps=1e-5, act=ACT_SIGMOID):
    """RMSNorm over the head dimension times the activated output gate.
    o, g [tokens, H, Dv]; w_norm [Dv]."""
    o, g, w = _f64(o), _f64(g), _f64(w_norm)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o * r * w * activation(g, act)


__all__ = ["short_conv", "prep_inputs", "output_gate_norm", "l2_normalize", "sigmoid", "activation",
           "ACT_NONE", "ACT_SILU", "ACT_SIGMOID"]
