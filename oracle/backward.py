"""Plain fp64 oracle of the gradients of the RDA core (test infrastructure
only, like the rest of this package).

The forward here is the gated delta rule written token by token in plain
PyTorch ops on the CPU, in the order the nano article's section "The other
1.5B: a hybrid built to forget" gives (decay the state, form the error between
the value and the decayed state's prediction for the key, write it with
strength beta, read with the query; the write gate rescales the value), and the
gradients are PyTorch autograd of that loop.  The pages say nothing about
training: these are the gradients of the defined function, nothing more.

For a loss L = <d_out, out> + <d_final_state, final_state> the gradients of
q, k, v, log_alpha, beta, the write gate and the initial state are returned.
Layouts follow the library (states ``[B,H,Dk,Dv]``, S transposed).
"""
import numpy as np
import torch


def _t(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64)
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def forward_torch(q, k, v, log_alpha, beta, gamma=None, initial_state=None, scale=1.0):
    """fp64 token loop; returns (out [B,T,H,Dv], final_state [B,H,Dk,Dv])."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S = torch.zeros(B, H, Dv, Dk, dtype=torch.float64) if initial_state is None \
        else initial_state.transpose(-1, -2)
    outs = []
    for t in range(T):
        a = torch.exp(log_alpha[:, t])[..., None, None]                  # [B,H,1,1]
        vt = v[:, t] if gamma is None else gamma[:, t][..., None] * v[:, t]
        kt, qt = k[:, t], q[:, t]                                         # [B,H,Dk]
        S = a * S                                                         # decay
        e = vt - torch.einsum("bhjd,bhd->bhj", S, kt)                     # error
        S = S + beta[:, t][..., None, None] * torch.einsum("bhj,bhd->bhjd", e, kt)   # write
        outs.append(scale * torch.einsum("bhjd,bhd->bhj", S, qt))        # read
    return torch.stack(outs, 1), S.transpose(-1, -2)


def backward(q, k, v, log_alpha, beta, d_out, gamma=None, initial_state=None, d_final_state=None,
             scale=1.0):
    """Gradients of <d_out, out> + <d_final_state, final_state>.  Returns a dict
    with dq, dk, dv, d_log_alpha, d_beta, d_gamma (None without gamma) and
    d_initial_state (None without an initial state), as float64 numpy arrays."""
    xs = {"q": _t(q), "k": _t(k), "v": _t(v), "log_alpha": _t(log_alpha), "beta": _t(beta)}
    if gamma is not None:
        xs["gamma"] = _t(gamma)
    if initial_state is not None:
        xs["initial_state"] = _t(initial_state)
    for x in xs.values():
        x.requires_grad_(True)
    out, sf = forward_torch(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["beta"], xs.get("gamma"),
                            xs.get("initial_state"), scale)
    loss = (out * _t(d_out)).sum()
    if d_final_state is not None:
        loss = loss + (sf * _t(d_final_state)).sum()
    names = list(xs)
    grads = torch.autograd.grad(loss, [xs[n] for n in names], allow_unused=True)
    g = {n: (None if gr is None else gr.numpy()) for n, gr in zip(names, grads)}
    for n in names:
        if g[n] is None:
            g[n] = np.zeros(tuple(xs[n].shape))
    return {"dq": g["q"], "dk": g["k"], "dv": g["v"], "d_log_alpha": g["log_alpha"], "d_beta": g["beta"],
            "d_gamma": g.get("gamma"), "d_initial_state": g.get("initial_state")}


__all__ = ["forward_torch", "backward"]
