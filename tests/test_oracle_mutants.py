"""Plants plausible slips in a copy of the C oracle and checks that the pins
catch every one of them (CPU only).

Each mutant is the oracle source with one textual edit, compiled into a
temporary directory; the real oracle source is never touched.
"""
import json
import math
import os
import subprocess
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import chunked, exact

SRC = os.path.join(os.path.dirname(oracle.__file__), "rda_oracle.c")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "exact_tiny.json")


def _compile(src_text, out_dir, name):
    c = os.path.join(out_dir, name + ".c")
    so = os.path.join(out_dir, name + ".so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", c, "-o", so, "-lm"],
                   check=True)
    return oracle.load_library(so)


def _battery(lib):
    """Runs the pins against ``lib``; returns the names of the pins that fail."""
    failed = []
    # golden exact rationals
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    F = lambda m: np.array([[float(Fraction(x)) for x in r] for r in m])
    for c in cases:
        T, Dk, Dv = c["T"], c["Dk"], c["Dv"]
        ga = None if c["gamma"] is None else np.array([float(Fraction(x)) for x in c["gamma"]]).reshape(1, T, 1)
        s0 = None if c["S0"] is None else F(c["S0"]).T.reshape(1, 1, Dk, Dv)
        out, sf = oracle.forward(F(c["q"]).reshape(1, T, 1, Dk), F(c["k"]).reshape(1, T, 1, Dk),
                                 F(c["v"]).reshape(1, T, 1, Dv),
                                 np.array([a * math.log(2.0) for a in c["alpha_log2"]]).reshape(1, T, 1),
                                 np.array([float(Fraction(x)) for x in c["beta"]]).reshape(1, T, 1),
                                 gamma=ga, initial_state=s0, lib=lib)
        if not (np.allclose(out[0, :, 0], F(c["out"]), rtol=0, atol=1e-12)
                and np.allclose(sf[0, 0].T, F(c["S_final"]), rtol=0, atol=1e-12)):
            failed.append(f"golden{c['seed']}")
    # chunked (independent derivation) equals sequential, with gamma, S0 and scale != 1
    rng = np.random.default_rng(0)
    B, T, H, Dk, Dv = 1, 70, 2, 8, 5
    nrm = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    d = dict(q=nrm(rng.standard_normal((B, T, H, Dk))), k=nrm(rng.standard_normal((B, T, H, Dk))),
             v=rng.standard_normal((B, T, H, Dv)), log_alpha=-rng.uniform(0.01, 0.5, (B, T, H)),
             beta=rng.uniform(0.05, 1, (B, T, H)), gamma=rng.uniform(0.5, 1.5, (B, T, H)),
             initial_state=rng.standard_normal((B, H, Dk, Dv)) * 0.3)
    o, s = oracle.forward(**d, scale=0.5, lib=lib)
    oc, sc = chunked.forward(**d, scale=0.5, chunk=16)
    if not (np.allclose(o, oc, rtol=1e-10, atol=1e-12) and np.allclose(s, sc, rtol=1e-10, atol=1e-12)):
        failed.append("chunked")
    # current-key exactness
    d2 = dict(d)
    d2["beta"] = np.ones_like(d["beta"])
    d2["q"] = d["k"]
    o2, _ = oracle.forward(**d2, lib=lib)
    if not np.allclose(o2, d["v"] * d["gamma"][..., None], rtol=0, atol=1e-12):
        failed.append("current_key")
    # beta = 0, alpha = 1
    d3 = dict(d)
    d3["beta"] = np.zeros_like(d["beta"])
    d3["log_alpha"] = np.zeros_like(d["log_alpha"])
    o3, s3 = oracle.forward(**d3, lib=lib)
    if not np.array_equal(s3, d["initial_state"]):
        failed.append("beta0")
    # per-key-channel decay against exact arithmetic (dyadic inputs, alpha = 2^-m per channel)
    rng = np.random.default_rng(11)
    T, Dk, Dv = 7, 4, 3
    qn, kn = rng.integers(-8, 9, (T, Dk)) / 8, rng.integers(-8, 9, (T, Dk)) / 8
    vn = rng.integers(-8, 9, (T, Dv)) / 8
    m = rng.integers(0, 3, (T, Dk))
    bn = rng.integers(0, 5, T) / 4
    s0n = rng.integers(-8, 9, (Dv, Dk)) / 8
    fr = lambda x: Fraction(x).limit_denominator(1 << 20)
    outs, S = exact.sequential([[fr(x) for x in r] for r in qn], [[fr(x) for x in r] for r in kn],
                               [[fr(x) for x in r] for r in vn],
                               [[Fraction(1, 2 ** int(x)) for x in r] for r in m],
                               [fr(x) for x in bn], S0=[[fr(x) for x in r] for r in s0n])
    o4, s4 = oracle.forward(qn.reshape(1, T, 1, Dk), kn.reshape(1, T, 1, Dk), vn.reshape(1, T, 1, Dv),
                            (-m * math.log(2.0)).reshape(1, T, 1, Dk), bn.reshape(1, T, 1),
                            initial_state=s0n.T.reshape(1, 1, Dk, Dv), lib=lib)
    if not (np.allclose(o4[0, :, 0], np.array([[float(x) for x in r] for r in outs]), rtol=0, atol=1e-12)
            and np.allclose(s4[0, 0].T, np.array([[float(x) for x in r] for r in S]), rtol=0, atol=1e-12)):
        failed.append("per_channel_exact")
    return failed


def _swap_update_and_read(src):
    a = src.index("    /* 3. write")
    b = src.index("    /* 4. read")
    e = src.index("}\n\nstatic void load_state")
    return src[:a] + src[b:e] + src[a:b] + src[e:]


MUTANTS = {
    "error_sign": lambda s: s.replace("e[j] = gamma * v[j] - pred;", "e[j] = gamma * v[j] + pred;"),
    "no_decay": lambda s: s.replace("S[(long)j * Dk + i] *= a;", "S[(long)j * Dk + i] *= 1.0;"),
    "double_decay": lambda s: s.replace("S[(long)j * Dk + i] *= a;", "S[(long)j * Dk + i] *= a * a;"),
    "beta_dropped": lambda s: s.replace("const double be = beta * e[j];", "const double be = e[j];"),
    "gamma_dropped": lambda s: s.replace("e[j] = gamma * v[j] - pred;", "e[j] = v[j] - pred;"),
    "read_with_k": lambda s: s.replace("acc += S[(long)j * Dk + i] * q[i];",
                                       "acc += S[(long)j * Dk + i] * k[i];"),
    "predict_with_q": lambda s: s.replace("pred += S[(long)j * Dk + i] * k[i];",
                                          "pred += S[(long)j * Dk + i] * q[i];"),
    "write_with_q": lambda s: s.replace("S[(long)j * Dk + i] += be * k[i];",
                                        "S[(long)j * Dk + i] += be * q[i];"),
    "state_not_transposed": lambda s: s.replace("S[(long)j * Dk + i] = src[(long)i * Dv + j];",
                                                "S[(long)j * Dk + i] = src[(long)j * Dk + i];"),
    "scale_dropped": lambda s: s.replace("o[(long)j * o_stride] = scale * acc;",
                                         "o[(long)j * o_stride] = acc;"),
    "read_before_write": _swap_update_and_read,
    "gate_index_shift": lambda s: s.replace("log_alpha[row], beta[row],",
                                            "log_alpha[row], beta[row > h ? row - 1 : row],"),
    # per-key-channel decay
    "channel_decay_dropped": lambda s: s.replace("S[(long)j * Dk + i] *= exp(la_ch[i]);",
                                                 "S[(long)j * Dk + i] *= 1.0;"),
    "channel_index_reversed": lambda s: s.replace("*= exp(la_ch[i]);", "*= exp(la_ch[Dk - 1 - i]);"),
    "channel_stride_per_token": lambda s: s.replace("la_ch ? la_ch + row * Dk : NULL",
                                                    "la_ch ? la_ch + row : NULL"),
}


def test_real_oracle_passes_battery(tmp_path):
    with open(SRC) as f:
        lib = _compile(f.read(), str(tmp_path), "real")
    assert _battery(lib) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    with open(SRC) as f:
        src = f.read()
    mutated = MUTANTS[name](src)
    assert mutated != src, f"mutant {name} did not apply"
    lib = _compile(mutated, str(tmp_path), name)
    assert _battery(lib), f"mutant {name} passed every pin"
