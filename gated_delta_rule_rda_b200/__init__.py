"""Python binding of the RDA core C-ABI library (``librda.so``).

Argument marshalling only: every step of the recurrence runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  There is
no CPU fallback: importing this package fails loudly when ``librda.so`` has not
been built, and every call requires CUDA tensors.

Functions mirror the C entry points of ``include/rda.h``:

- :func:`rda_prefill_chunked` -- fixed-length prefill ``[B,T,H,D]`` (a log alpha
  ``[B,T,H,Dk]`` selects the per-key-channel decay);
- :func:`rda_prefill_varlen` -- packed sequences with ``cu_seqlens``;
- :func:`rda_decode_step` -- one token per sequence, state updated in place;
- :func:`rda_decode_tokens` -- 1..8 tokens per sequence in one pass over the state;
- :func:`rda_prep_inputs`, :func:`rda_output_gate_norm` -- the steps either side of
  the core (short convolutions, q/k norms, gates; output RMSNorm times the gate);
- :func:`rda_backward` -- the gradients of the core;
- :func:`rda_read_device_error`, :func:`rda_prefill_workspace_bytes`,
  :func:`rda_prefill_channel_workspace_bytes`.

The raw ctypes handle is :data:`lib` (``lib.rda_prefill_chunked(...)`` takes
plain pointers and sizes, including host-pointer use for the varlen schedule).
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librda.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m gated_delta_rule_rda_b200.build` "
        "(or __graft_entry__.build()); there is no fallback implementation")

lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t

lib.rda_status_string.argtypes = [_i]
lib.rda_status_string.restype = ctypes.c_char_p
lib.rda_version.argtypes = []
lib.rda_version.restype = ctypes.c_char_p
lib.rda_prefill_workspace_bytes.argtypes = [_i] * 6
lib.rda_prefill_workspace_bytes.restype = _sz
lib.rda_prefill_channel_workspace_bytes.argtypes = [_i] * 6
lib.rda_prefill_channel_workspace_bytes.restype = _sz
lib.rda_prefill_chunked.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _vp, _sz, _vp]
lib.rda_prefill_chunked.restype = _i
lib.rda_prefill_varlen.argtypes = [_vp] * 8 + [_i, _i, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _sz, _vp]
lib.rda_prefill_varlen.restype = _i
lib.rda_decode_step.argtypes = [_vp] * 8 + [_i] * 5 + [_f, _vp]
lib.rda_decode_step.restype = _i
lib.rda_decode_tokens.argtypes = [_vp] * 8 + [_i] * 6 + [_f, _vp]
lib.rda_decode_tokens.restype = _i
lib.rda_read_device_error.argtypes = [_vp, ctypes.POINTER(_i), _vp]
lib.rda_read_device_error.restype = _i
lib.rda_prefill_chunked_channel.argtypes = lib.rda_prefill_chunked.argtypes
lib.rda_prefill_chunked_channel.restype = _i
lib.rda_prefill_varlen_channel.argtypes = lib.rda_prefill_varlen.argtypes
lib.rda_prefill_varlen_channel.restype = _i
lib.rda_decode_step_channel.argtypes = lib.rda_decode_step.argtypes
lib.rda_decode_step_channel.restype = _i
lib.rda_prefill_chunked_noalloc.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _vp]
lib.rda_prefill_chunked_noalloc.restype = _i
lib.rda_prep_inputs.argtypes = [_vp] * 8 + [_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i] + [_vp] * 6 + \
    [_i, _i, _i, _i, _i, _vp]
lib.rda_prep_inputs.restype = _i
lib.rda_output_gate_norm.argtypes = [_vp, _vp, _vp, _f, _i, _vp, _i, ctypes.c_longlong, _i, _i, _vp]
lib.rda_output_gate_norm.restype = _i
lib.rda_backward_workspace_bytes.argtypes = [_i] * 5
lib.rda_backward_workspace_bytes.restype = _sz
lib.rda_backward.argtypes = [_vp] * 16 + [_i] * 6 + [_f, _vp, _sz, _vp]
lib.rda_backward.restype = _i
lib.rda_debug_set_wait_fault.argtypes = [_i, ctypes.c_ulonglong]
lib.rda_debug_set_wait_fault.restype = None

RDA_OK = 0
RDA_F32 = 0
RDA_BF16 = 1
RDA_ACT_NONE, RDA_ACT_SILU, RDA_ACT_SIGMOID = 0, 1, 2
STATUS_NAMES = {0: "RDA_OK", 1: "RDA_ERR_INVALID_ARG", 2: "RDA_ERR_UNSUPPORTED",
                3: "RDA_ERR_MISALIGNED", 4: "RDA_ERR_WORKSPACE", 5: "RDA_ERR_CUDA",
                6: "RDA_ERR_TIMEOUT"}


class RdaError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {lib.rda_status_string(code).decode()}")


def _check(code, where):
    if code != RDA_OK:
        raise RdaError(code, where)


def version() -> str:
    return lib.rda_version().decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RDA_F32
    if t.dtype == torch.bfloat16:
        return RDA_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("rda: tensors must be CUDA tensors (no CPU path exists)")
            if not t.is_contiguous():
                raise ValueError("rda: tensors must be contiguous")


def _need_f32(*ts):
    for t in ts:
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"rda: gates and states must be float32, got {t.dtype}")


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def rda_prefill_workspace_bytes(B, T, H, Dk, Dv, num_seqs=0) -> int:
    return int(lib.rda_prefill_workspace_bytes(B, T, H, Dk, Dv, num_seqs))


def rda_prefill_channel_workspace_bytes(B, T, H, Dk, Dv, num_seqs=0) -> int:
    return int(lib.rda_prefill_channel_workspace_bytes(B, T, H, Dk, Dv, num_seqs))


def new_workspace(nbytes, device) -> torch.Tensor:
    """A workspace of ``nbytes`` (256-byte aligned by the caching allocator)
    whose device error word (first 256 bytes) starts cleared."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def rda_prefill_chunked(q, k, v, log_alpha, beta, write_gate=None, initial_state=None,
                        scale=1.0, out=None, final_state=None, return_final_state=True,
                        workspace=None, stream=None):
    """Fixed-length prefill.  q, k ``[B,T,H,Dk]``; v ``[B,T,H,Dv]``; gates fp32
    ``[B,T,H]`` (log_alpha ``[B,T,H,Dk]`` for per-key-channel decay, which calls
    ``rda_prefill_chunked_channel``); initial_state fp32 ``[B,H,Dk,Dv]`` or None.

    Returns ``(out [B,T,H,Dv], final_state [B,H,Dk,Dv] or None)``.
    """
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    _need_cuda(q, k, v, log_alpha, beta, write_gate, initial_state, out, final_state, workspace)
    _need_f32(log_alpha, beta, write_gate, initial_state, final_state)
    dt = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("rda: q, k and v must share a dtype")
    channel = log_alpha.dim() == 4
    if k.shape != q.shape or v.shape[:3] != (B, T, H) or beta.shape != (B, T, H) \
            or log_alpha.shape != ((B, T, H, Dk) if channel else (B, T, H)):
        raise ValueError("rda: inconsistent shapes")
    if out is None:
        out = torch.empty((B, T, H, Dv), dtype=q.dtype, device=q.device)
    if final_state is None and return_final_state:
        final_state = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        wb = rda_prefill_channel_workspace_bytes if channel else rda_prefill_workspace_bytes
        workspace = new_workspace(wb(B, T, H, Dk, Dv, 0), q.device)
    fn = lib.rda_prefill_chunked_channel if channel else lib.rda_prefill_chunked
    code = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
              _ptr(write_gate), _ptr(initial_state), _ptr(final_state),
              _ptr(out), dt, B, T, H, Dk, Dv, float(scale),
              _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, fn.__name__)
    return out, final_state


def rda_prefill_varlen(q, k, v, log_alpha, beta, cu_seqlens, write_gate=None,
                       initial_states=None, scale=1.0, out=None, final_states=None,
                       return_final_states=True, cu_seqlens_host=None, workspace=None,
                       stream=None):
    """Packed prefill.  q, k ``[total,H,Dk]``; v ``[total,H,Dv]``; gates
    ``[total,H]`` (log_alpha ``[total,H,Dk]`` for per-key-channel decay);
    cu_seqlens int32 CUDA ``[N+1]``; cu_seqlens_host optional
    int32 CPU mirror (enables longest-first scheduling).

    Returns ``(out [total,H,Dv], final_states [N,H,Dk,Dv] or None)``.
    """
    total, H, Dk = q.shape
    Dv = v.shape[-1]
    N = cu_seqlens.numel() - 1
    _need_cuda(q, k, v, log_alpha, beta, cu_seqlens, write_gate, initial_states, out,
               final_states, workspace)
    _need_f32(log_alpha, beta, write_gate, initial_states, final_states)
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("rda: cu_seqlens must be int32")
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((total, H, Dv), dtype=q.dtype, device=q.device)
    if final_states is None and return_final_states:
        final_states = torch.empty((N, H, Dk, Dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        wb = rda_prefill_channel_workspace_bytes if log_alpha.dim() == 3 else rda_prefill_workspace_bytes
        workspace = new_workspace(wb(1, total, H, Dk, Dv, N), q.device)
    host_ptr = None
    if cu_seqlens_host is not None:
        cu_seqlens_host = cu_seqlens_host.to(torch.int32).contiguous()
        if cu_seqlens_host.is_cuda:
            raise ValueError("rda: cu_seqlens_host must be a CPU tensor")
        host_ptr = ctypes.c_void_p(cu_seqlens_host.data_ptr())
    fn = lib.rda_prefill_varlen_channel if log_alpha.dim() == 3 else lib.rda_prefill_varlen
    code = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
              _ptr(write_gate), _ptr(cu_seqlens), host_ptr, N, total,
              _ptr(initial_states), _ptr(final_states), _ptr(out), dt, H, Dk,
              Dv, float(scale), _ptr(workspace), workspace.numel(),
              _stream(stream))
    _check(code, fn.__name__)
    return out, final_states


def rda_decode_step(q, k, v, log_alpha, beta, state, write_gate=None, scale=1.0, out=None,
                    stream=None):
    """One decode step.  q, k ``[B,H,Dk]``; v ``[B,H,Dv]``; gates fp32 ``[B,H]``
    (log_alpha ``[B,H,Dk]`` for per-key-channel decay);
    state fp32 ``[B,H,Dk,Dv]`` updated in place.  Returns ``out [B,H,Dv]``."""
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    _need_cuda(q, k, v, log_alpha, beta, state, write_gate, out)
    _need_f32(log_alpha, beta, state, write_gate)
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, Dv), dtype=q.dtype, device=q.device)
    fn = lib.rda_decode_step_channel if log_alpha.dim() == 3 else lib.rda_decode_step
    code = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
              _ptr(write_gate), _ptr(state), _ptr(out), dt, B, H, Dk, Dv,
              float(scale), _stream(stream))
    _check(code, fn.__name__)
    return out


def rda_decode_tokens(q, k, v, log_alpha, beta, state, write_gate=None, scale=1.0, out=None,
                      stream=None):
    """T (<= 8) decode steps in one pass over the state.  q, k ``[B,T,H,Dk]``;
    v ``[B,T,H,Dv]``; gates fp32 ``[B,T,H]``; state fp32 ``[B,H,Dk,Dv]`` updated
    in place.  Returns ``out [B,T,H,Dv]``."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    _need_cuda(q, k, v, log_alpha, beta, state, write_gate, out)
    _need_f32(log_alpha, beta, state, write_gate)
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, T, H, Dv), dtype=q.dtype, device=q.device)
    code = lib.rda_decode_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                 _ptr(write_gate), _ptr(state), _ptr(out), dt, B, T, H, Dk, Dv,
                                 float(scale), _stream(stream))
    _check(code, "rda_decode_tokens")
    return out


def rda_prefill_chunked_noalloc(q, k, v, log_alpha, beta, write_gate=None, initial_state=None,
                                scale=1.0, out=None, final_state=None, stream=None):
    """rda_prefill_chunked without a workspace: for callers that cannot give
    the library scratch memory.  Uses the library's fixed 64 MiB device array
    (see include/rda.h); larger problems raise RdaError (RDA_ERR_WORKSPACE)."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    _need_cuda(q, k, v, log_alpha, beta, write_gate, initial_state, out, final_state)
    _need_f32(log_alpha, beta, write_gate, initial_state, final_state)
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, T, H, Dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    code = lib.rda_prefill_chunked_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                           _ptr(write_gate), _ptr(initial_state), _ptr(final_state),
                                           _ptr(out), dt, B, T, H, Dk, Dv, float(scale),
                                           _stream(stream))
    _check(code, "rda_prefill_chunked_noalloc")
    return out, final_state


def rda_prep_inputs(q_raw, k_raw, v_raw, conv_w_q, conv_w_k, conv_w_v, beta_raw, log_alpha_raw,
                    cu_seqlens=None, delta=None, conv_window_in=None, conv_window_out=None,
                    conv_act=RDA_ACT_SILU, max_seqlen=None, stream=None):
    """The steps before the core (short conv, q/k L2 norm, gates, log-decay clamp).

    Fixed length: q_raw, k_raw ``[B,T,H,Dk]``, v_raw ``[B,T,H,Dv]``, beta_raw, delta
    ``[B,T,H]``, log_alpha_raw ``[B,T,H]`` or ``[B,T,H,Dk]``.  Packed: the same
    without B, plus ``cu_seqlens`` (int32 CUDA) and ``max_seqlen``.  Conv
    windows are bf16 ``[N,3,H*(2Dk+Dv)]``.  Returns a dict with q, k, v, beta,
    write_gate (None without delta) and log_alpha.
    """
    packed = cu_seqlens is not None
    H, Dk = q_raw.shape[-2:]
    Dv = v_raw.shape[-1]
    if packed:
        total = q_raw.shape[0]
        N = cu_seqlens.numel() - 1
        T = 0
        if max_seqlen is None:
            raise ValueError("rda: packed sequences need max_seqlen")
    else:
        N, T = q_raw.shape[:2]
        total = N * T
        max_seqlen = T
    channel = log_alpha_raw.dim() == q_raw.dim()
    _need_cuda(q_raw, k_raw, v_raw, conv_w_q, conv_w_k, conv_w_v, beta_raw, log_alpha_raw,
               cu_seqlens, delta, conv_window_in, conv_window_out)
    _need_f32(conv_w_q, conv_w_k, conv_w_v, beta_raw, log_alpha_raw, delta)
    for w in (conv_window_in, conv_window_out):
        if w is not None and w.dtype != torch.bfloat16:
            raise TypeError("rda: the conv window is bfloat16")
    dt = _dtype_code(q_raw)
    q, k, v = torch.empty_like(q_raw), torch.empty_like(k_raw), torch.empty_like(v_raw)
    beta = torch.empty_like(beta_raw)
    gamma = None if delta is None else torch.empty_like(beta_raw)
    la = torch.empty_like(log_alpha_raw)
    code = lib.rda_prep_inputs(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_w_q), _ptr(conv_w_k),
                               _ptr(conv_w_v), _ptr(conv_window_in), _ptr(conv_window_out),
                               _ptr(beta_raw), _ptr(delta), _ptr(log_alpha_raw), int(channel),
                               _ptr(cu_seqlens), N, T, int(max_seqlen), total,
                               _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gamma), _ptr(la),
                               dt, H, Dk, Dv, int(conv_act), _stream(stream))
    _check(code, "rda_prep_inputs")
    return dict(q=q, k=k, v=v, beta=beta, write_gate=gamma, log_alpha=la)


def rda_output_gate_norm(o, g, norm_weight, eps=1e-5, gate_act=RDA_ACT_SIGMOID, out=None,
                         stream=None):
    """RMSNorm of the core's output over the head dimension times act(g).
    o, g ``[..., H, Dv]`` (same dtype); norm_weight fp32 ``[Dv]``."""
    _need_cuda(o, g, norm_weight, out)
    _need_f32(norm_weight)
    if g.shape != o.shape or g.dtype != o.dtype:
        raise ValueError("rda: o and g must match")
    H, Dv = o.shape[-2:]
    tokens = o.numel() // (H * Dv)
    if out is None:
        out = torch.empty_like(o)
    code = lib.rda_output_gate_norm(_ptr(o), _ptr(g), _ptr(norm_weight), float(eps), int(gate_act),
                                    _ptr(out), _dtype_code(o), tokens, H, Dv, _stream(stream))
    _check(code, "rda_output_gate_norm")
    return out


def rda_backward(q, k, v, log_alpha, beta, d_out, write_gate=None, initial_state=None,
                 d_final_state=None, scale=1.0, workspace=None, stream=None):
    """Gradients of ``<d_out, out> + <d_final_state, final_state>`` for a
    fixed-length prefill (shapes as :func:`rda_prefill_chunked`).  Returns a
    dict of fp32 tensors dq, dk, dv, d_log_alpha, d_beta, d_write_gate (None
    without a write gate) and d_initial_state."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    _need_cuda(q, k, v, log_alpha, beta, d_out, write_gate, initial_state, d_final_state, workspace)
    _need_f32(log_alpha, beta, write_gate, initial_state, d_final_state)
    dt = _dtype_code(q)
    if d_out.dtype != q.dtype or d_out.shape != v.shape:
        raise ValueError("rda: d_out must match out")
    f = lambda *shape: torch.empty(shape, dtype=torch.float32, device=q.device)
    g = dict(dq=f(B, T, H, Dk), dk=f(B, T, H, Dk), dv=f(B, T, H, Dv), d_log_alpha=f(B, T, H),
             d_beta=f(B, T, H), d_write_gate=None if write_gate is None else f(B, T, H),
             d_initial_state=f(B, H, Dk, Dv))
    if workspace is None:
        workspace = new_workspace(int(lib.rda_backward_workspace_bytes(B, T, H, Dk, Dv)), q.device)
    code = lib.rda_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(write_gate),
                            _ptr(initial_state), _ptr(d_out), _ptr(d_final_state), _ptr(g["dq"]),
                            _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["d_log_alpha"]), _ptr(g["d_beta"]),
                            _ptr(g["d_write_gate"]), _ptr(g["d_initial_state"]), dt, B, T, H, Dk, Dv,
                            float(scale), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "rda_backward")
    return g


def rda_debug_set_wait_fault(drop_chunk=-1, wait_limit_ns=0):
    """Testing only: bound of the device-side waits and an injected stall of the
    scan (see include/rda.h); ``rda_debug_set_wait_fault()`` turns it off."""
    lib.rda_debug_set_wait_fault(int(drop_chunk), int(wait_limit_ns))


def rda_read_device_error(workspace, stream=None) -> int:
    code = _i(0)
    _check(lib.rda_read_device_error(_ptr(workspace), ctypes.byref(code), _stream(stream)),
           "rda_read_device_error")
    return int(code.value)


__all__ = ["rda_prefill_chunked", "rda_prefill_varlen", "rda_decode_step", "rda_decode_tokens",
           "rda_prep_inputs", "rda_output_gate_norm", "rda_backward",
           "rda_prefill_chunked_noalloc",
           "rda_read_device_error", "rda_debug_set_wait_fault", "rda_prefill_workspace_bytes",
           "rda_prefill_channel_workspace_bytes", "new_workspace", "version",
           "RdaError", "lib", "LIB_PATH"]
