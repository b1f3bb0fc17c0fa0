"""The allocation-free prefill entry point, called through the C ABI.

`rda_prefill_chunked_noalloc` serves callers that cannot give the library any
scratch memory (programs that own all device memory and allow no allocation
after start-up).  It runs the same prefill on a fixed device array; these
checks compare it with `rda_prefill_chunked` on two calls in a row.  This file
is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import rda_gen
from parity_util import rel_l2

pytestmark = pytest.mark.gpu


def _noalloc(lib, d, scale, out, sf):
    B, T, H, Dk = d.q.shape
    Dv = d.v.shape[-1]
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return lib.rda_prefill_chunked_noalloc(p(d.q), p(d.k), p(d.v), p(d.log_alpha), p(d.beta),
                                           p(d.gamma), p(d.initial_state), p(sf), p(out), 1,
                                           B, T, H, Dk, Dv, float(scale),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    for call, (T, seed, gamma) in enumerate([(1000, 61, False), (1600, 62, True)]):
        inp = rda_gen.fixed_inputs(1, T, 8, 128, 128, dtype=torch.bfloat16, seed=seed, s0=True,
                                   gamma=gamma).to("cuda")
        ref_o, ref_s = rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                               write_gate=inp.gamma, initial_state=inp.initial_state,
                                               scale=0.75)
        out = torch.full_like(ref_o, float("nan"))
        sf = torch.full_like(ref_s, float("nan"))
        assert _noalloc(rda.lib, inp, 0.75, out, sf) == 0, f"call {call}"
        torch.cuda.synchronize()
        o, s = out.double().cpu().numpy(), sf.double().cpu().numpy()
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(s))
        assert rel_l2(o, ref_o.double().cpu().numpy()) <= 1e-2, f"call {call}"
        assert rel_l2(s, ref_s.double().cpu().numpy()) <= 1e-2, f"call {call}"


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    big = rda_gen.fixed_inputs(1, 8192, 16, 128, 128, dtype=torch.bfloat16, seed=63, s0=False).to("cuda")
    out = torch.empty_like(big.v)
    sf = torch.empty(1, 16, 128, 128, device="cuda")
    assert _noalloc(rda.lib, big, 1.0, out, sf) == 4          # RDA_ERR_WORKSPACE, nothing launched
    with pytest.raises(rda.RdaError, match="WORKSPACE"):
        rda.rda_prefill_chunked_noalloc(big.q, big.k, big.v, big.log_alpha, big.beta)
