"""The C-ABI library loads, exports every symbol include/rda.h declares, and
rejects bad arguments on the host before anything is launched (CPU only:
no call here reaches a CUDA runtime function)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rda.h")

import gated_delta_rule_rda_b200 as rda  # noqa: E402  (fails loudly if librda.so is missing)

OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE = 0, 1, 2, 3, 4


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rda_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for want in ["rda_prefill_chunked", "rda_prefill_varlen", "rda_decode_step", "rda_decode_tokens",
                 "rda_prefill_chunked_channel", "rda_prefill_varlen_channel", "rda_decode_step_channel",
                 "rda_prefill_chunked_noalloc", "rda_debug_set_wait_fault",
                 "rda_prep_inputs", "rda_output_gate_norm", "rda_backward",
                 "rda_backward_workspace_bytes",
                 "rda_prefill_workspace_bytes", "rda_prefill_channel_workspace_bytes",
                 "rda_read_device_error", "rda_status_string",
                 "rda_version"]:
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(rda.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, f"librda.so lacks {missing}"


def test_status_strings_and_version():
    for code in range(7):
        s = rda.lib.rda_status_string(code).decode()
        assert s.startswith(rda.STATUS_NAMES[code])
    assert rda.lib.rda_status_string(99).decode() == "RDA_ERR_UNKNOWN"
    assert re.match(r"^\d+\.\d+\.\d+$", rda.version())


def test_workspace_query():
    # the chunked path keeps about 40 KiB of prep results per (chunk, head)
    assert rda.rda_prefill_workspace_bytes(1, 4096, 16, 128, 128, 0) >= 64 * 16 * 40 * 1024
    assert rda.rda_prefill_workspace_bytes(1, 4096, 16, 64, 64, 0) >= 256
    assert rda.rda_prefill_workspace_bytes(1, 100, 16, 128, 128, 64) >= 256 + 64 * 4
    assert rda.rda_prefill_workspace_bytes(1, 100, 16, 96, 128, 0) == 0
    assert rda.rda_prefill_workspace_bytes(-1, 100, 16, 128, 128, 0) == 0
    # per-key-channel decay: the decayed K and Q images (32 KiB per chunk and head) on top
    ch = rda.rda_prefill_channel_workspace_bytes(1, 4096, 16, 128, 128, 0)
    assert ch >= rda.rda_prefill_workspace_bytes(1, 4096, 16, 128, 128, 0) + 64 * 16 * 32 * 1024
    assert rda.rda_prefill_channel_workspace_bytes(1, 4096, 16, 64, 64, 0) == \
        rda.rda_prefill_workspace_bytes(1, 4096, 16, 64, 64, 0)
    assert rda.rda_prefill_channel_workspace_bytes(1, 100, 16, 96, 128, 0) == 0
    # packed batches: the schedule and the chunk offsets on top, more than the fixed-length figure
    assert rda.rda_prefill_channel_workspace_bytes(1, 4096, 16, 128, 128, 8) > \
        rda.rda_prefill_channel_workspace_bytes(1, 4096, 16, 128, 128, 0)
    assert rda.rda_prefill_channel_workspace_bytes(1, 4096, 16, 128, 128, 8) > \
        rda.rda_prefill_workspace_bytes(1, 4096, 16, 128, 128, 8)


# Fake device addresses: never dereferenced, because validation fails first.
A16 = 0x10000
A256 = 0x20000


def _chunked(**kw):
    args = dict(q=A16, k=A16, v=A16, la=A16, be=A16, wg=None, s0=None, sf=None, out=A16,
                dtype=1, B=1, T=64, H=2, Dk=128, Dv=128, scale=1.0, ws=A256, wsb=1 << 40, stream=None)
    args.update(kw)
    return rda.lib.rda_prefill_chunked(*[args[k] for k in ["q", "k", "v", "la", "be", "wg", "s0", "sf",
                                                           "out", "dtype", "B", "T", "H", "Dk", "Dv",
                                                           "scale", "ws", "wsb", "stream"]])


def test_chunked_rejects_bad_arguments():
    assert _chunked(dtype=7) == UNSUPPORTED
    assert _chunked(Dk=96) == UNSUPPORTED
    assert _chunked(Dv=32) == UNSUPPORTED
    assert _chunked(H=0) == INVALID
    assert _chunked(T=-1) == INVALID
    assert _chunked(B=-2) == INVALID
    assert _chunked(q=None) == INVALID
    assert _chunked(out=None) == INVALID
    assert _chunked(be=None) == INVALID
    assert _chunked(k=A16 + 8) == MISALIGNED
    assert _chunked(out=A16 + 2) == MISALIGNED
    assert _chunked(s0=A16 + 4) == MISALIGNED
    assert _chunked(ws=None) == WORKSPACE
    assert _chunked(wsb=16) == WORKSPACE
    assert _chunked(ws=A256 + 16) == MISALIGNED
    assert _chunked(B=1, T=1 << 20, H=64) == INVALID   # a tensor of 2^33 elements


def _varlen(**kw):
    args = dict(q=A16, k=A16, v=A16, la=A16, be=A16, wg=None, cu=A16, cuh=None, N=2, total=100,
                s0=None, sf=None, out=A16, dtype=1, H=2, Dk=128, Dv=128, scale=1.0, ws=A256,
                wsb=1 << 40, stream=None)
    args.update(kw)
    return rda.lib.rda_prefill_varlen(*[args[k] for k in ["q", "k", "v", "la", "be", "wg", "cu", "cuh",
                                                          "N", "total", "s0", "sf", "out", "dtype",
                                                          "H", "Dk", "Dv", "scale", "ws", "wsb",
                                                          "stream"]])


def test_varlen_rejects_bad_arguments():
    assert _varlen(cu=None) == INVALID
    assert _varlen(N=-1) == INVALID
    assert _varlen(Dk=32) == UNSUPPORTED
    assert _varlen(wsb=256) == WORKSPACE          # schedule needs room beyond the error word
    assert _varlen(dtype=0, Dk=64, wsb=256) == WORKSPACE
    bad = (ctypes.c_int32 * 3)(0, 60, 50)         # total mismatch
    assert _varlen(cuh=ctypes.cast(bad, ctypes.c_void_p)) == INVALID
    dec = (ctypes.c_int32 * 3)(0, 60, 40)         # decreasing
    assert _varlen(total=40, cuh=ctypes.cast(dec, ctypes.c_void_p)) == INVALID
    first = (ctypes.c_int32 * 3)(5, 60, 100)      # must start at 0
    assert _varlen(cuh=ctypes.cast(first, ctypes.c_void_p)) == INVALID
    assert _varlen(N=0) == OK                      # nothing to do, nothing launched


def _decode(**kw):
    args = dict(q=A16, k=A16, v=A16, la=A16, be=A16, wg=None, st=A16, out=A16, dtype=1, B=4, H=2,
                Dk=128, Dv=128, scale=1.0, stream=None)
    args.update(kw)
    return rda.lib.rda_decode_step(*[args[k] for k in ["q", "k", "v", "la", "be", "wg", "st", "out",
                                                       "dtype", "B", "H", "Dk", "Dv", "scale",
                                                       "stream"]])


def test_decode_rejects_bad_arguments():
    assert _decode(st=None) == INVALID
    assert _decode(st=A16 + 4) == MISALIGNED
    assert _decode(Dv=256) == UNSUPPORTED
    assert _decode(dtype=-1) == UNSUPPORTED
    assert _decode(B=-1) == INVALID
    assert _decode(B=0) == OK


def test_read_device_error_rejects_null():
    assert rda.lib.rda_read_device_error(None, None, None) == INVALID


def test_python_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        rda.rda_prefill_chunked(q, q, q, torch.zeros(1, 4, 1), torch.zeros(1, 4, 1))


def _tokens(**kw):
    args = dict(q=A16, k=A16, v=A16, la=A16, be=A16, wg=None, st=A16, out=A16, dtype=1, B=4, T=4, H=2,
                Dk=128, Dv=128, scale=1.0, stream=None)
    args.update(kw)
    return rda.lib.rda_decode_tokens(*[args[k] for k in ["q", "k", "v", "la", "be", "wg", "st", "out",
                                                         "dtype", "B", "T", "H", "Dk", "Dv", "scale",
                                                         "stream"]])


def test_decode_tokens_rejects_bad_arguments():
    assert _tokens(T=9) == UNSUPPORTED              # at most 8 tokens per call
    assert _tokens(T=-1) == INVALID
    assert _tokens(st=None) == INVALID
    assert _tokens(st=A16 + 4) == MISALIGNED
    assert _tokens(q=A16 + 2) == MISALIGNED
    assert _tokens(Dk=96) == UNSUPPORTED
    assert _tokens(dtype=3) == UNSUPPORTED
    assert _tokens(T=0) == OK                       # nothing to do, nothing launched
    assert _tokens(B=0) == OK
