"""Benchmark of the RDA core on B200: prefill tokens/s and decode state GB/s.

One JSON line on stdout (rank 0).  A "step" is one call of the prefill entry
point over the nano-shaped workload (bf16 q/k/v, B=1, T=4096, H=16,
Dk=Dv=128, 64-token chunks, nonzero fp32 initial state, final state returned)
with its inputs resident in HBM; L2 is flushed (a 256 MiB write) between
timed steps and each step is timed alone with CUDA events on the launching
stream.  ``e2e`` times the same call with host (pinned) inputs and outputs,
copies included, as a two-slot pipeline (one step's copies overlap the next
step's compute and copies; every step moves all of its own bytes).  ``decode`` times 128 consecutive decode steps over
B=256 sequences (state 256 MiB, larger than L2).

Multi-GPU (torchrun): the path does not shard within one problem; every rank
runs its own replica (weak scaling), timing is the max over ranks.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only), on a
bounded sample of the same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RDA prefill tokens/s (H=16,D=128) and decode state GB/s on 1 B200 vs roofline"
WORKLOAD = "nano_prefill_b1_t4096_h16_d128"
# kernels one fixed-length bf16 prefill call enqueues (prep with the output
# operands, state scan with the outputs)
LAUNCHES_PER_PREFILL = 2
CHUNK = 64


# ------------------------------------------------------------------ algorithmic counts

def prefill_flops_per_token_head(Dk=128, Dv=128, C=CHUNK):
    """QK^T, KK^T, T.(beta K): 2 C Dk each; T.(beta V), P.U: 2 C Dv each;
    W.S, Q.S, K^T.U: 2 Dk Dv each; the UT solve: C^2/3 per token."""
    return 6 * C * Dk + 4 * C * Dv + 6 * Dk * Dv + C * C / 3.0


def prefill_bytes_per_token_head(Dk=128, Dv=128, elem=2):
    """q, k, v read and o written in the I/O dtype; log alpha and beta (fp32) read."""
    return (2 * Dk + Dv) * elem + Dv * elem + 8


def state_bytes(H, Dk, Dv):
    return H * Dk * Dv * 4


def decode_bytes_per_seq_head(Dk=128, Dv=128, elem=2):
    """State read + written once (fp32) plus the token's q, k, v, o and gates."""
    return 2 * Dk * Dv * 4 + prefill_bytes_per_token_head(Dk, Dv, elem)


# ------------------------------------------------------------------ helpers

def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi in the background."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id, interval_ms=20):
        self.samples = []
        self.proc = None
        self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", f"-lms={interval_ms}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                self.samples.append((time.time(), float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                pass

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if len(inside) < 3:  # short windows: widen to the nearest samples around it
            inside = [s for s in self.samples if t0 - 0.25 <= s[0] <= t1 + 0.25] or self.samples[-5:]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({self.REASONS[i] for s in inside for i, r in enumerate(s[3])
                          if r.lower().startswith("active")})
        return {"sm_mhz": statistics.median(s[1] for s in inside),
                "sm_max_mhz": max(s[2] for s in inside), "reasons": reasons,
                "samples": len(inside)}


def captured_traffic():
    """DRAM bytes per step from a committed ncu capture, only while the kernel
    source it was taken on is unchanged (sha256 match); else None."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, rec["source"])
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
        if digest != rec["source_sha256"]:
            return None
        return float(rec["dram_bytes_per_step"])
    except Exception:
        return None


def gpu_id_for(device):
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        return str(device.index or 0)


# ------------------------------------------------------------------ our arm

def as_graph(fn):
    """Captures the calls `fn` makes on the current stream into a CUDA graph and
    returns its replay.  The timed regions replay graphs so that they measure
    the kernels, not the host's argument marshalling between a start event and
    the launch; the same kernels run with the same arguments.  `fn` runs twice
    eagerly first (the library sets kernel attributes on a first call, outside
    capture)."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    return graph.replay

def max_over_ranks(value, device):
    """The largest of every rank's `value` over the default process group (the
    job's time is its slowest rank's); `value` itself without one."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms):
    """Units per second of the whole job: every rank processes `units_per_rank`
    in `ms` (the max over ranks)."""
    return units_per_rank * world / (ms * 1e-3)


def run_ours(args, rank, world, device):
    import torch
    import gated_delta_rule_rda_b200 as rda
    import rda_gen

    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    dist = None
    if world > 1:
        import torch.distributed as dist

    inp = rda_gen.workload(WORKLOAD)
    B, T, H, Dk = inp.q.shape
    Dv = inp.v.shape[-1]
    d = inp.to(device)
    out = torch.empty((B, T, H, Dv), dtype=d.q.dtype, device=device)
    sf = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=device)
    ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(B, T, H, Dk, Dv, 0), device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def step():
        rda.rda_prefill_chunked(d.q, d.k, d.v, d.log_alpha, d.beta,
                                initial_state=d.initial_state, out=out, final_state=sf,
                                workspace=ws)

    sampler = ClockSampler(gpu_id_for(device)) if rank == 0 else None
    step_eager = step
    step = as_graph(step_eager)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for s, e in ev:
        flush.zero_()
        s.record(stream)
        step()
        e.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if dist:
        dist.barrier()
    step_ms = [s.elapsed_time(e) for s, e in ev]
    ms_per_step = sum(step_ms) / len(step_ms)
    ms_per_step = max_over_ranks(ms_per_step, device)
    assert rda.rda_read_device_error(ws) == 0, "device error word set during the benchmark"

    # ---- e2e: host (pinned) inputs and outputs, copies inside the timed region.
    # Two pipeline slots on two streams, each with its own device buffers and
    # workspace: step i copies its inputs in, runs the prefill and copies the
    # output and final state back on slot i % 2, so one step's copies overlap
    # the neighbouring step's (PCIe is full duplex).  Every step still moves all
    # of its own bytes both ways.
    host_in = [t.pin_memory() for t in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state)]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    slots = []
    for _ in range(2):
        slots.append({
            "stream": torch.cuda.Stream(device),
            "dev_in": [torch.empty_like(t, device=device) for t in host_in],
            "out": torch.empty((B, T, H, Dv), dtype=inp.q.dtype, device=device),
            "sf": torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=device),
            "ws": ws if not slots else rda.new_workspace(ws.numel(), device),
            "host_out": torch.empty((B, T, H, Dv), dtype=inp.q.dtype).pin_memory(),
            "host_sf": torch.empty((B, H, Dk, Dv), dtype=torch.float32).pin_memory(),
        })
    d2h = (slots[0]["host_out"].numel() * slots[0]["host_out"].element_size() +
           slots[0]["host_sf"].numel() * slots[0]["host_sf"].element_size())

    def e2e_step(i):
        sl = slots[i % 2]
        with torch.cuda.stream(sl["stream"]):
            for hd, dd in zip(host_in, sl["dev_in"]):
                dd.copy_(hd, non_blocking=True)
            q, k, v, la, be, s0 = sl["dev_in"]
            rda.rda_prefill_chunked(q, k, v, la, be, initial_state=s0, out=sl["out"], final_state=sl["sf"],
                                    workspace=sl["ws"])
            sl["host_out"].copy_(sl["out"], non_blocking=True)
            sl["host_sf"].copy_(sl["sf"], non_blocking=True)

    e2e_steps = max(4, min(args.steps, 50))
    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for sl in slots:
        sl["stream"].wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    for sl in slots:
        stream.wait_stream(sl["stream"])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, device)
    # the pipelined result must match the device-resident run
    assert torch.equal(slots[0]["host_out"], out.cpu()) and torch.equal(slots[1]["host_sf"], sf.cpu()), \
        "end-to-end result differs from the device-resident step"
    del slots

    # ---- decode: 128 consecutive steps over B=256 (state larger than L2)
    dec = None
    if not args.no_decode:
        din = rda_gen.workload("decode_b256_h16_d128_128steps").to(device)
        st = din.state.clone()
        dout = torch.empty((din.q.shape[1], H, Dv), dtype=din.q.dtype, device=device)
        nsteps = din.q.shape[0]

        def dec_rep():
            for t in range(nsteps):
                rda.rda_decode_step(din.q[t], din.k[t], din.v[t], din.log_alpha[t], din.beta[t],
                                    st, out=dout)
        dec_rep()
        torch.cuda.synchronize()
        reps = 3
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist:
            dist.barrier()
        d0.record(stream)
        for _ in range(reps):
            dec_rep()
        d1.record(stream)
        torch.cuda.synchronize()
        dms = d0.elapsed_time(d1) / (reps * nsteps)
        dms = max_over_ranks(dms, device)
        Bd = din.q.shape[1]
        bytes_step = Bd * H * decode_bytes_per_seq_head(Dk, Dv, 2)
        hbm, _, _, src = load_peaks()
        gbs = bytes_step / (dms * 1e-3) / 1e9
        dec = {"workload": "decode_b256_h16_d128_128steps", "ms_per_decode_step": dms,
               "state_gbs": gbs * world, "bytes_per_step": bytes_step,
               "hbm_frac": gbs / hbm, "peak_gbs": hbm, "peak_source": src,
               "tokens_per_s": Bd * world / (dms * 1e-3)}
        del din, st

    extra = {}
    if args.all:
        extra = other_workloads(device, stream, rank, world)

    clocks = None
    if sampler:
        sampler.stop()
        clocks = sampler.summary(t_wall0, t_wall1)

    hbm, tf, tf_sus, src = load_peaks()
    tokens = B * T
    alg_bytes = tokens * H * prefill_bytes_per_token_head(Dk, Dv, 2) + 2 * B * state_bytes(H, Dk, Dv)
    alg_flops = tokens * H * prefill_flops_per_token_head(Dk, Dv)
    gbs = alg_bytes / (ms_per_step * 1e-3) / 1e9
    tflops = alg_flops / (ms_per_step * 1e-3) / 1e12
    return {
        "metric": METRIC,
        "value": whole_job_rate(tokens, world, ms_per_step),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "T": T, "H": H, "Dk": Dk, "Dv": Dv,
                   "chunk": CHUNK, "state": "fp32, nonzero initial, final returned",
                   "l2": "flushed between timed steps (256 MiB write)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm, "traffic": captured_traffic(), "peak_source": src,
                     "algorithmic_bytes_per_launch": alg_bytes,
                     "tensor": {"achieved_tflops": tflops, "peak_tflops": tf,
                                "frac": tflops / tf, "algorithmic_flops_per_launch": alg_flops}},
        "e2e": {"value": whole_job_rate(tokens, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipeline": "2 slots on 2 streams: copies of one step overlap the next step's"},
        "gpu_launches": args.steps * LAUNCHES_PER_PREFILL,
        "clocks": clocks,
        "decode": dec,
        **extra,
    }


def other_workloads(device, stream, rank, world, reps=5):
    """Long-context and packed (varlen) prefill: event-timed, L2 flushed between
    repetitions (both inputs are larger than L2 anyway)."""
    import torch
    import gated_delta_rule_rda_b200 as rda
    import rda_gen
    res = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def timed(fn, graph=True):
        if graph:
            fn = as_graph(fn)
        for _ in range(2):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            fn()
            e.record(stream)
            ts.append((s, e))
        torch.cuda.synchronize()
        return max_over_ranks(sorted(a.elapsed_time(b) for a, b in ts)[len(ts) // 2], device)

    inp = rda_gen.workload("long_prefill_b1_t32768_h16_d128").to(device)
    B, T, H, Dk = inp.q.shape
    ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(B, T, H, Dk, Dk, 0), device)
    out = torch.empty_like(inp.v)
    sf = torch.empty((B, H, Dk, Dk), device=device)
    ms = timed(lambda: rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                               out=out, final_state=sf, workspace=ws))
    nbytes = B * T * H * prefill_bytes_per_token_head() + B * state_bytes(H, Dk, Dk)
    res["long_prefill"] = {"workload": "long_prefill_b1_t32768_h16_d128", "ms": ms,
                           "tokens_per_s": world * B * T / (ms * 1e-3),
                           "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / load_peaks()[0]}
    del inp, ws, out, sf
    vin = rda_gen.workload("varlen_64seqs_128to8192_h16_d128")
    d = vin.to(device)
    total, H, Dk = vin.q.shape
    N = vin.cu_seqlens.numel() - 1
    ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(1, total, H, Dk, Dk, N), device)
    out = torch.empty_like(d.v)
    sf = torch.empty((N, H, Dk, Dk), device=device)
    ms = timed(lambda: rda.rda_prefill_varlen(d.q, d.k, d.v, d.log_alpha, d.beta, d.cu_seqlens,
                                              initial_states=d.initial_states, out=out,
                                              final_states=sf, cu_seqlens_host=vin.cu_seqlens,
                                              workspace=ws), graph=False)
    nbytes = total * H * prefill_bytes_per_token_head() + 2 * N * state_bytes(H, Dk, Dk)
    res["varlen_prefill"] = {"workload": "varlen_64seqs_128to8192_h16_d128", "tokens": total,
                             "ms": ms, "tokens_per_s": world * total / (ms * 1e-3),
                             "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / load_peaks()[0]}
    del d, vin, ws, out, sf

    # mini shape (H = 40) prefill, same kernels
    inp = rda_gen.workload("mini_prefill_b1_t4096_h40_d128").to(device)
    B, T, H, Dk = inp.q.shape
    ws = rda.new_workspace(rda.rda_prefill_workspace_bytes(B, T, H, Dk, Dk, 0), device)
    out = torch.empty_like(inp.v)
    sf = torch.empty((B, H, Dk, Dk), device=device)
    ms = timed(lambda: rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                               initial_state=inp.initial_state, out=out,
                                               final_state=sf, workspace=ws))
    nbytes = B * T * H * prefill_bytes_per_token_head() + 2 * B * state_bytes(H, Dk, Dk)
    res["mini_prefill"] = {"workload": "mini_prefill_b1_t4096_h40_d128", "ms": ms,
                           "tokens_per_s": world * B * T / (ms * 1e-3),
                           "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / load_peaks()[0]}
    del inp, ws, out, sf

    # per-key-channel decay at the nano shape (chunked tensor-core path)
    inp = rda_gen.workload("nano_prefill_channel_b1_t4096_h16_d128").to(device)
    B, T, H, Dk = inp.q.shape
    ws = rda.new_workspace(rda.rda_prefill_channel_workspace_bytes(B, T, H, Dk, Dk, 0), device)
    out = torch.empty_like(inp.v)
    sf = torch.empty((B, H, Dk, Dk), device=device)
    ms = timed(lambda: rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                               initial_state=inp.initial_state, out=out,
                                               final_state=sf, workspace=ws))
    nbytes = B * T * H * (prefill_bytes_per_token_head() + 4 * (Dk - 1)) + 2 * B * state_bytes(H, Dk, Dk)
    res["channel_prefill"] = {"workload": "nano_prefill_channel_b1_t4096_h16_d128", "ms": ms,
                              "tokens_per_s": world * B * T / (ms * 1e-3),
                              "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / load_peaks()[0]}
    del inp, ws, out, sf

    # per-key-channel decode step at the decode shape: one step's inputs, 128 calls
    din = rda_gen.decode_inputs(B=256, H=16, Dk=128, Dv=128, steps=1, seed=8, channel=True).to(device)
    st = din.state.clone()
    dout = torch.empty((256, 16, 128), dtype=din.q.dtype, device=device)

    def ch_rep():
        for _ in range(128):
            rda.rda_decode_step(din.q[0], din.k[0], din.v[0], din.log_alpha[0], din.beta[0], st, out=dout)
    ms = timed(ch_rep) / 128
    bytes_step = 256 * 16 * (decode_bytes_per_seq_head(128, 128, 2) + 4 * 127)
    res["channel_decode"] = {"workload": "decode_b256_h16_d128, per-key-channel decay", "ms_per_step": ms,
                             "state_gbs": world * bytes_step / (ms * 1e-3) / 1e9,
                             "hbm_frac": bytes_step / (ms * 1e-3) / 1e9 / load_peaks()[0]}
    del din, st, dout

    # backward pass at the nano shape (token-sequential fp32, checkpoints every 16 tokens)
    inp = rda_gen.workload(WORKLOAD).to(device)
    B, T, H, Dk = inp.q.shape
    gen = torch.Generator(device="cpu").manual_seed(11)
    d_out = torch.randn(inp.v.shape, generator=gen).to(device=device, dtype=inp.v.dtype)
    d_sf = torch.randn((B, H, Dk, Dk), generator=gen).to(device)
    bws = rda.new_workspace(int(rda.lib.rda_backward_workspace_bytes(B, T, H, Dk, Dk)), device)
    ms = timed(lambda: rda.rda_backward(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, d_out,
                                        initial_state=inp.initial_state, d_final_state=d_sf, workspace=bws))
    res["backward"] = {"workload": WORKLOAD + ", gradients of <d_out, out> + <d_final_state, final_state>",
                       "ms": ms, "tokens_per_s": world * B * T / (ms * 1e-3)}
    del inp, d_out, d_sf, bws

    # the steps around the core at the nano shape: short conv + norms + gates, and
    # the output norm x gate
    raw = rda_gen.raw_layer_inputs(B=1, T=4096, H=16, Dk=128, Dv=128, dtype=torch.bfloat16, seed=9).to(device)
    win_out = torch.empty_like(raw.conv_window)
    ms_pre = timed(lambda: rda.rda_prep_inputs(raw.q_raw, raw.k_raw, raw.v_raw, raw.w_q, raw.w_k, raw.w_v,
                                               raw.beta_raw, raw.log_alpha_raw, delta=raw.delta,
                                               conv_window_in=raw.conv_window, conv_window_out=win_out))
    # bytes: q, k, v read and written (bf16), three fp32 gates read and written
    pre_bytes = 4096 * 16 * (2 * (3 * 128 * 2) + 2 * 3 * 4)
    post_out = torch.empty_like(raw.v_raw)
    ms_post = timed(lambda: rda.rda_output_gate_norm(raw.v_raw, raw.g, raw.norm_weight, out=post_out))
    post_bytes = 4096 * 16 * 3 * 128 * 2
    res["prep_inputs"] = {"workload": "nano shape, B=1 T=4096 H=16 D=128 bf16", "ms": ms_pre,
                          "hbm_frac": pre_bytes / (ms_pre * 1e-3) / 1e9 / load_peaks()[0]}
    res["output_gate_norm"] = {"workload": "nano shape, B=1 T=4096 H=16 Dv=128 bf16", "ms": ms_post,
                               "hbm_frac": post_bytes / (ms_post * 1e-3) / 1e9 / load_peaks()[0]}
    del raw, win_out, post_out

    # multi-token decode: the decode workload's first 128 tokens as calls of T tokens
    din = rda_gen.workload("decode_b256_h16_d128_128steps")
    st = din.state.to(device)
    Bd, H, Dk, Dv = st.shape
    res["decode_tokens"] = {}
    for T in (1, 2, 4, 8):
        blocks = [[x[t0:t0 + T].transpose(0, 1).contiguous().to(device)
                   for x in (din.q, din.k, din.v, din.log_alpha, din.beta)] for t0 in range(0, 128, T)]
        dout = torch.empty((Bd, T, H, Dv), dtype=din.q.dtype, device=device)

        def tok_rep():
            for q, k, v, la, be in blocks:
                rda.rda_decode_tokens(q, k, v, la, be, st, out=dout)
        ms = timed(tok_rep) / len(blocks)
        bytes_call = Bd * H * (2 * state_bytes(1, Dk, Dv) + T * prefill_bytes_per_token_head())
        gbs = bytes_call / (ms * 1e-3) / 1e9
        res["decode_tokens"][f"T{T}"] = {
            "workload": f"decode_b256_h16_d128_128steps, {T} tokens per call", "ms_per_call": ms,
            "tokens_per_s": world * Bd * T / (ms * 1e-3), "state_gbs": world * gbs,
            "hbm_frac": gbs / load_peaks()[0]}
        del blocks
    return res


# ------------------------------------------------------------------ oracle timing

_ORACLE_INPUTS = []


def oracle_sample_rate(T_sample, threads):
    """Times the oracle on the first T_sample tokens of the workload, all 16
    heads; returns (tokens/s, seconds, cores used)."""
    import oracle
    import rda_gen
    if not _ORACLE_INPUTS:
        _ORACLE_INPUTS.append(rda_gen.workload(WORKLOAD))
    inp = _ORACLE_INPUTS[0]
    sl = lambda t: t[:, :T_sample]
    H = inp.q.shape[2]
    t0 = time.perf_counter()
    oracle.forward(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.log_alpha), sl(inp.beta),
                   initial_state=inp.initial_state, num_threads=threads)
    dt = time.perf_counter() - t0
    return T_sample / dt, dt, min(threads, H)


def host_cores():
    """Cores this process may run on (``nproc``)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(target_s=12.0, single_core_T=1024):
    """The oracle on the whole workload, repeated until about target_s seconds
    of CPU work have run; tokens/s of the mean repetition.  Also the oracle on
    one core over the first `single_core_T` tokens (all heads)."""
    import oracle
    threads = oracle.max_threads()
    T = 4096
    _, dt, cores = oracle_sample_rate(T, threads)
    reps = max(1, int(target_s / max(dt, 1e-3)))
    total = dt
    for _ in range(reps - 1):
        _, d, _ = oracle_sample_rate(T, threads)
        total += d
    rate = T * reps / total
    rate1, dt1, _ = oracle_sample_rate(single_core_T, 1)
    return {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "host_nproc": host_cores(), "omp_threads_available": threads,
            "sample": f"fp64 token-sequential oracle over the full {WORKLOAD} workload "
                      f"(T=4096, all 16 heads, OpenMP over the 16 heads: {cores} threads busy on a "
                      f"{host_cores()}-core host), {reps} repetitions, {total:.1f} s",
            "single_core": {"value": rate1, "unit": "tokens/s", "cores": 1,
                            "sample": f"same oracle on one thread, first {single_core_T} tokens of "
                                      f"{WORKLOAD} (all 16 heads), {dt1:.1f} s"}}


def run_reference(args):
    import oracle
    threads = oracle.max_threads()
    rate, _, _ = oracle_sample_rate(16, threads)
    per_step_s = min(3.0, 120.0 / max(1, args.steps + args.warmup))
    T_sample = int(min(4096, max(16, rate * per_step_s)))
    for _ in range(args.warmup):
        oracle_sample_rate(T_sample, threads)
    times = []
    cores = 1
    for _ in range(args.steps):
        _, dt, cores = oracle_sample_rate(T_sample, threads)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = T_sample / (ms * 1e-3)
    sample = (f"fp64 token-sequential oracle, first {T_sample} tokens of {WORKLOAD} per step "
              f"(all 16 heads)")
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "B": 1, "T": 4096, "H": 16, "Dk": 128, "Dv": 128,
                   "chunk": CHUNK, "sample_T": T_sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "host_nproc": host_cores(), "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def profile_decode_tokens(T, steps, warmup):
    """Only the multi-token decode (decode workload shape, T tokens per call):
    a short, self-contained run for a profiler.  Prints ms per call."""
    import torch
    import gated_delta_rule_rda_b200 as rda
    import rda_gen
    din = rda_gen.workload("decode_b256_h16_d128_128steps")
    device = torch.device("cuda", 0)
    st = din.state.to(device)
    q, k, v, la, be = [x[0:T].transpose(0, 1).contiguous().to(device)
                       for x in (din.q, din.k, din.v, din.log_alpha, din.beta)]
    out = torch.empty((st.shape[0], T, st.shape[1], st.shape[3]), dtype=din.q.dtype, device=device)
    for _ in range(warmup):
        rda.rda_decode_tokens(q, k, v, la, be, st, out=out)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        rda.rda_decode_tokens(q, k, v, la, be, st, out=out)
    e.record()
    torch.cuda.synchronize()
    print(json.dumps({"decode_tokens_T": T, "ms_per_call": s.elapsed_time(e) / steps}), flush=True)


def profile_prefill(steps, warmup, workload=WORKLOAD):
    """Only the nano prefill (or the per-key-channel one): `warmup` + `steps`
    eager calls, L2 flushed before each (a short, self-contained run for a
    profiler)."""
    import torch
    import gated_delta_rule_rda_b200 as rda
    import rda_gen
    inp = rda_gen.workload(workload).to("cuda")
    B, T, H, Dk = inp.q.shape
    Dv = inp.v.shape[-1]
    wb = rda.rda_prefill_channel_workspace_bytes if inp.log_alpha.dim() == 4 else rda.rda_prefill_workspace_bytes
    ws = rda.new_workspace(wb(B, T, H, Dk, Dv, 0), "cuda")
    out = torch.empty_like(inp.v)
    sf = torch.empty(B, H, Dk, Dv, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(warmup + steps):
        flush.zero_()
        rda.rda_prefill_chunked(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, initial_state=inp.initial_state,
                                out=out, final_state=sf, workspace=ws)
    torch.cuda.synchronize()
    assert rda.rda_read_device_error(ws) == 0
    print(json.dumps({"profile_prefill_calls": warmup + steps}), flush=True)


def profile_prepost(steps, warmup):
    """Only the steps around the core at the nano shape (bf16 B1 T4096 H16 D128):
    `warmup` + `steps` calls of each, L2 flushed before each pair."""
    import torch
    import gated_delta_rule_rda_b200 as rda
    import rda_gen
    raw = rda_gen.raw_layer_inputs(B=1, T=4096, H=16, Dk=128, Dv=128, dtype=torch.bfloat16, seed=9).to("cuda")
    win_out = torch.empty_like(raw.conv_window)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(warmup + steps):
        flush.zero_()
        rda.rda_prep_inputs(raw.q_raw, raw.k_raw, raw.v_raw, raw.w_q, raw.w_k, raw.w_v, raw.beta_raw,
                            raw.log_alpha_raw, delta=raw.delta, conv_window_in=raw.conv_window,
                            conv_window_out=win_out)
        rda.rda_output_gate_norm(raw.v_raw, raw.g, raw.norm_weight)
    torch.cuda.synchronize()
    print(json.dumps({"profile_prepost_calls": warmup + steps}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--all", action="store_true",
                    help="also time the long-context and packed (varlen) prefill workloads")
    ap.add_argument("--profile-decode-tokens", type=int, default=0, metavar="T",
                    help="run only the multi-token decode with T tokens per call (for a profiler)")
    ap.add_argument("--profile-prefill-channel", action="store_true",
                    help="run only warmup + steps per-key-channel nano prefill calls, L2 flushed (for a profiler)")
    ap.add_argument("--profile-prefill", action="store_true",
                    help="run only warmup + steps nano prefill calls, L2 flushed (for a profiler)")
    ap.add_argument("--profile-prepost", action="store_true",
                    help="run only warmup + steps calls of the steps around the core (for a profiler)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.profile_decode_tokens:
        profile_decode_tokens(args.profile_decode_tokens, args.steps, args.warmup)
        return
    if args.profile_prefill:
        profile_prefill(args.steps, args.warmup)
        return
    if args.profile_prefill_channel:
        profile_prefill(args.steps, args.warmup, "nano_prefill_channel_b1_t4096_h16_d128")
        return
    if args.profile_prepost:
        profile_prepost(args.steps, args.warmup)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    import torch
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(device)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    try:
        line = run_ours(args, rank, world, device)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
