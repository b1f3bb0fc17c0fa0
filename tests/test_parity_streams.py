"""Prefill calls on several streams, from several host threads, and replayed
from a captured CUDA graph.

One prefill call enqueues its kernels on the caller's stream only.  These
checks run calls that overlap on the GPU (each with its own workspace) and
compare every result bit for bit with the same call run alone:
the kernels are deterministic, so any cross-call interference shows as a
mismatch.  The single-call results are themselves checked against the fp64
oracle.
"""
import threading

import numpy as np
import pytest
import torch

import rda_gen
from parity_util import oracle_fixed, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _inputs(n):
    return [rda_gen.fixed_inputs(1, 300 + 64 * i, 4, 128, 128, dtype=torch.bfloat16, seed=500 + i,
                                 s0=True, gamma=(i % 2 == 1)).to("cuda") for i in range(n)]


def _call(rda, d, ws, stream=None):
    return rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, write_gate=d.gamma,
                                   initial_state=d.initial_state, workspace=ws, stream=stream)


def _alone(rda, ins):
    res = []
    for d in ins:
        ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(*d.q.shape[:3], 128, 128, 0), "cuda")
        o, s = _call(rda, d, ws)
        torch.cuda.synchronize()
        res.append((o.clone(), s.clone()))
    return res


def test_overlapping_calls_on_two_streams(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    ins = _inputs(4)
    ref = _alone(rda, ins)
    # the single-call results against the oracle (one of them; the others are bit-compared)
    ro, rs = oracle_fixed(ins[1].to("cpu"))
    assert rel_l2(to_np(ref[1][0]), ro) <= 1e-2 and rel_l2(to_np(ref[1][1]), rs) <= 1e-2
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    wss = [rda.new_workspace(rda.rda_prefill_workspace_bytes(*d.q.shape[:3], 128, 128, 0), "cuda")
           for d in ins]
    outs = [None] * len(ins)
    for rep in range(3):
        for i, d in enumerate(ins):
            with torch.cuda.stream(streams[i % 2]):
                outs[i] = _call(rda, d, wss[i])
        torch.cuda.synchronize()
        for i in range(len(ins)):
            assert torch.equal(outs[i][0], ref[i][0]) and torch.equal(outs[i][1], ref[i][1]), (rep, i)


def test_calls_from_two_host_threads(cuda_device):
    import gated_delta_rule_rda_b200 as rda
    ins = _inputs(2)
    ref = _alone(rda, ins)
    errors = []

    def worker(i):
        try:
            torch.cuda.set_device(0)
            st = torch.cuda.Stream()
            d = ins[i]
            ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(*d.q.shape[:3], 128, 128, 0), "cuda")
            for _ in range(20):
                with torch.cuda.stream(st):
                    o, s = _call(rda, d, ws)
                st.synchronize()
                if not (torch.equal(o, ref[i][0]) and torch.equal(s, ref[i][1])):
                    errors.append(i)
                    return
        except Exception as e:  # noqa: BLE001 -- reported below
            errors.append(repr(e))

    ts = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors


def test_graph_capture_and_replay(cuda_device):
    """A captured call (kernel launches only, no host work inside) replays to
    the eager result."""
    import gated_delta_rule_rda_b200 as rda
    d = _inputs(1)[0]
    ref = _alone(rda, [d])[0]
    ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(*d.q.shape[:3], 128, 128, 0), "cuda")
    out = torch.empty_like(ref[0])
    sf = torch.empty_like(ref[1])
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):      # first call outside capture (one-time setup: kernel attributes)
        rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, write_gate=d.gamma,
                                initial_state=d.initial_state, out=out, final_state=sf, workspace=ws)
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta, write_gate=d.gamma,
                                initial_state=d.initial_state, out=out, final_state=sf, workspace=ws)
    for _ in range(3):
        out.zero_()
        sf.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref[0]) and torch.equal(sf, ref[1])
    del g
