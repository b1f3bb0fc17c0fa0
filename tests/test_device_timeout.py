"""The device-side timeout path of the chunked prefill, made to run out on
purpose through the test-only fault injection `rda_debug_set_wait_fault`.

The state scan is told never to fill one chunk's operands and its waits are
bounded at 20 ms.  The kernel must then record RDA_ERR_TIMEOUT in the
workspace error word and return through its abort and drain paths (no trap,
no fault, no unbounded wait); the context must stay usable, so a normal call
on the same stream and workspace afterwards is correct and leaves the word
clear.
"""
import numpy as np
import pytest
import torch

import rda_gen
from parity_util import oracle_fixed, rel_l2, to_np

pytestmark = pytest.mark.gpu

RDA_ERR_TIMEOUT = 6


def _call(rda, d, ws):
    return rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, initial_state=d.initial_state,
                                   workspace=ws)


@pytest.mark.parametrize("drop_chunk", [0, 2])
def test_scan_wait_runs_out_and_context_stays_usable(cuda_device, drop_chunk):
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(1, 320, 2, 128, 128, dtype=torch.bfloat16, seed=91, s0=True)
    ro, rs = oracle_fixed(inp)
    d = inp.to("cuda")
    ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(1, 320, 2, 128, 128, 0), "cuda")
    try:
        rda.rda_debug_set_wait_fault(drop_chunk=drop_chunk, wait_limit_ns=20_000_000)
        out, sf = _call(rda, d, ws)
        torch.cuda.synchronize()
    finally:
        rda.rda_debug_set_wait_fault()
    assert rda.rda_read_device_error(ws) == RDA_ERR_TIMEOUT
    # the chunks before the stalled one were finished and stored
    done = 64 * drop_chunk
    if done:
        assert rel_l2(to_np(out)[:, :done], ro[:, :done]) <= 1e-2

    # the same stream and workspace, without the fault: correct, error word clear
    out2, sf2 = _call(rda, d, ws)
    torch.cuda.synchronize()
    assert rda.rda_read_device_error(ws) == 0
    o2, s2 = to_np(out2), to_np(sf2)
    assert np.all(np.isfinite(o2)) and np.all(np.isfinite(s2))
    assert rel_l2(o2, ro) <= 1e-2 and rel_l2(s2, rs) <= 1e-2


def test_varlen_scan_wait_runs_out(cuda_device):
    """The same through the packed entry point: every sequence long enough to
    reach the dropped chunk stalls; the next normal call is correct."""
    import oracle
    import gated_delta_rule_rda_b200 as rda
    from parity_util import gpu_varlen
    vin = rda_gen.varlen_inputs(lengths=[200, 30, 140], H=2, Dk=128, Dv=128, dtype=torch.bfloat16,
                                seed=92)
    d = vin.to("cuda")
    total = vin.q.shape[0]
    ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(1, total, 2, 128, 128, 3), "cuda")
    try:
        rda.rda_debug_set_wait_fault(drop_chunk=1, wait_limit_ns=20_000_000)
        rda.rda_prefill_varlen(d.q, d.k, d.v, d.log_alpha, d.beta, d.cu_seqlens,
                               initial_states=d.initial_states, workspace=ws)
        torch.cuda.synchronize()
    finally:
        rda.rda_debug_set_wait_fault()
    assert rda.rda_read_device_error(ws) == RDA_ERR_TIMEOUT
    out, sf = gpu_varlen(vin)
    ro, rs = oracle.varlen(vin.q, vin.k, vin.v, vin.log_alpha, vin.beta, vin.cu_seqlens,
                           initial_states=vin.initial_states)
    assert rel_l2(out, ro) <= 1e-2 and rel_l2(sf, rs) <= 1e-2


def test_channel_scan_wait_runs_out(cuda_device):
    """The per-key-channel chunked prefill (its scan has the same bounded waits,
    fed from the K~ and Q~ images): the stalled chunk records the timeout, the
    chunks before it are stored, and the next normal call is correct."""
    import oracle
    import gated_delta_rule_rda_b200 as rda
    inp = rda_gen.fixed_inputs(1, 320, 2, 128, 128, dtype=torch.bfloat16, seed=93, s0=True, channel=True)
    ro, rs = oracle.forward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, initial_state=inp.initial_state)
    d = inp.to("cuda")
    ws = rda.new_workspace(rda.rda_prefill_channel_workspace_bytes(1, 320, 2, 128, 128, 0), "cuda")
    try:
        rda.rda_debug_set_wait_fault(drop_chunk=2, wait_limit_ns=20_000_000)
        out, _ = _call(rda, d, ws)
        torch.cuda.synchronize()
    finally:
        rda.rda_debug_set_wait_fault()
    assert rda.rda_read_device_error(ws) == RDA_ERR_TIMEOUT
    assert rel_l2(to_np(out)[:, :128], ro[:, :128]) <= 1e-2
    out2, sf2 = _call(rda, d, ws)
    torch.cuda.synchronize()
    assert rda.rda_read_device_error(ws) == 0
    assert rel_l2(to_np(out2), ro) <= 1e-2 and rel_l2(to_np(sf2), rs) <= 1e-2
