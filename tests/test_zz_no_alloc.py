"""The allocation-free prefill entry point, called through the C ABI.

`rda_prefill_chunked_noalloc` serves callers that cannot give the library any
scratch memory (programs that own all device memory and allow no allocation
after start-up).  It runs the same kernels as `rda_prefill_chunked` on a fixed
device array instead of a caller workspace, so its results must equal that
call's bit for bit; these checks compare the two on two calls in a row, check
that a call leaves the device's free memory unchanged, and check the size
limit.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import rda_gen

pytestmark = pytest.mark.gpu

RDA_ERR_INVALID_ARG = 1
RDA_ERR_WORKSPACE = 4


def _noalloc(lib, d, scale, out, sf, dtype_code=1, q=None):
    B, T, H, Dk = d.q.shape
    Dv = d.v.shape[-1]
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    qp = p(d.q) if q is None else q
    return lib.rda_prefill_chunked_noalloc(qp, p(d.k), p(d.v), p(d.log_alpha), p(d.beta),
                                           p(d.gamma), p(d.initial_state), p(sf), p(out), dtype_code,
                                           B, T, H, Dk, Dv, float(scale),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _reference(rda, inp, scale):
    return rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, write_gate=inp.gamma,
                                   initial_state=inp.initial_state, scale=scale)


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    for call, (T, seed, gamma) in enumerate([(1000, 61, False), (1600, 62, True)]):
        inp = rda_gen.fixed_inputs(1, T, 8, 128, 128, dtype=torch.bfloat16, seed=seed, s0=True,
                                   gamma=gamma).to("cuda")
        ref_o, ref_s = _reference(rda, inp, 0.75)
        out = torch.full_like(ref_o, float("nan"))
        sf = torch.full_like(ref_s, float("nan"))
        assert _noalloc(rda.lib, inp, 0.75, out, sf) == 0, f"call {call}"
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o), f"call {call}: outputs differ"
        assert torch.equal(sf, ref_s), f"call {call}: final states differ"


def test_noalloc_call_allocates_no_device_memory(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(1, 700, 4, 128, 128, dtype=torch.bfloat16, seed=64, s0=True).to("cuda")
    out = torch.empty_like(inp.v)
    sf = torch.empty_like(inp.initial_state)
    assert _noalloc(rda.lib, inp, 1.0, out, sf) == 0      # first call: the library is loaded
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert _noalloc(rda.lib, inp, 1.0, out, sf) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    big = rda_gen.fixed_inputs(1, 8192, 16, 128, 128, dtype=torch.bfloat16, seed=63, s0=False).to("cuda")
    out = torch.empty_like(big.v)
    sf = torch.empty(1, 16, 128, 128, device="cuda")
    assert _noalloc(rda.lib, big, 1.0, out, sf) == RDA_ERR_WORKSPACE    # nothing launched
    with pytest.raises(rda.RdaError, match="WORKSPACE"):
        rda.rda_prefill_chunked_noalloc(big.q, big.k, big.v, big.log_alpha, big.beta)
    # an argument error is reported as such, before anything is enqueued
    assert _noalloc(rda.lib, big, 1.0, out, sf, q=ctypes.c_void_p(0)) == \
        RDA_ERR_INVALID_ARG


def test_noalloc_fp32_beyond_the_bf16_limit(cuda_device):
    """fp32 inputs take the token-sequential path, which needs only the error
    word: a size the bf16 path rejects still runs, and equals the workspace
    entry point."""
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(1, 8192, 16, 128, 128, dtype=torch.float32, seed=65, s0=True).to("cuda")
    ref_o, ref_s = _reference(rda, inp, 1.0)
    out = torch.full_like(ref_o, float("nan"))
    sf = torch.full_like(ref_s, float("nan"))
    assert _noalloc(rda.lib, inp, 1.0, out, sf, dtype_code=0) == 0
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(sf, ref_s)
