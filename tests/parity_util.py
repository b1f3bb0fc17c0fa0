"""Helpers for the GPU parity tests: run the CUDA path through the C-ABI
binding, run the oracle on the same inputs, compare by relative L2."""
import numpy as np
import torch

import oracle

# Tolerances on relative L2 error over a whole returned tensor: fp32 inputs
# are held to 1e-5; bf16 inputs (fp32 state and accumulation) to 1e-2.
TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}


def rel_l2(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def to_np(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def gpu_fixed(inp, scale=1.0, device="cuda"):
    import gated_delta_rule_rda_b200 as rda
    d = inp.to(device)
    ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(*d.q.shape[:3], d.q.shape[3],
                                                           d.v.shape[3], 0), device)
    out, sf = rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, write_gate=d.gamma,
                                      initial_state=d.initial_state, scale=scale, workspace=ws)
    torch.cuda.synchronize()
    assert rda.rda_read_device_error(ws) == 0
    return to_np(out), to_np(sf)


def oracle_fixed(inp, scale=1.0):
    return oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, gamma=inp.gamma,
                          initial_state=inp.initial_state, scale=scale)


def gpu_varlen(vin, scale=1.0, host_schedule=True, device="cuda"):
    import gated_delta_rule_rda_b200 as rda
    d = vin.to(device)
    out, sf = rda.rda_prefill_varlen(d.q, d.k, d.v, d.log_alpha, d.beta, d.cu_seqlens,
                                     write_gate=d.gamma, initial_states=d.initial_states,
                                     scale=scale,
                                     cu_seqlens_host=vin.cu_seqlens if host_schedule else None)
    torch.cuda.synchronize()
    return to_np(out), to_np(sf)
