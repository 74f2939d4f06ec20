"""The oracle's pins catch plausible mistakes (CPU only).

Each case copies the oracle's C source, plants one mistake (a dropped term, a wrong sign, a gate
in the wrong place, a swapped operand), builds the copy into a temporary library and runs the pin
checks against it.  At least one check must fail for every mutant; the unmodified source must pass
all of them.  Nothing here touches a GPU.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import chunkwise
from tests.test_oracle_pins import rand_inputs, GOLDEN

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

MUTANTS = {
    "gate_not_on_correction": ("a * (Si[j] - b * ki * kS[j])", "a * Si[j] - b * ki * kS[j]"),
    "gate_also_on_write": ("+ b * ki * v[j]", "+ a * b * ki * v[j]"),
    "wrong_sign_of_correction": ("Si[j] - b * ki * kS[j]", "Si[j] + b * ki * kS[j]"),
    "beta_missing_on_write": ("+ b * ki * v[j]", "+ ki * v[j]"),
    "readout_with_key_not_query": ("const double qi = q[i];", "const double qi = k[i];"),
    "gate_linearised": ("exp(log_alpha)", "(1.0 + log_alpha)"),
    "beta_missing_on_correction": ("Si[j] - b * ki * kS[j]", "Si[j] - ki * kS[j]"),
}


def _build(tmp_path, name, src_text):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src_text)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so),
                    str(c), "-lm"], check=True)
    return str(so)


def _checks():
    """Return the list of pin names that fail with the currently loaded oracle library."""
    import json
    failed = []
    # hand-worked example
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_2x2.json")))
    with np.errstate(divide="ignore"):
        la = np.log(np.array(g["alpha"]))
    out, Sf = oracle.forward(np.array(g["q"])[None, :, None], np.array(g["k"])[None, :, None],
                             np.array(g["v"])[None, :, None], la[None, :, None],
                             np.array(g["beta"])[None, :, None], np.array(g["S0"])[None, None])
    if not (np.allclose(out[0, :, 0], g["out"], atol=1e-12)
            and np.allclose(Sf[0, 0], g["S_final"], atol=1e-12)):
        failed.append("hand_worked")
    # chunkwise form agreement
    rng = np.random.default_rng(0)
    q, k, v, la, beta, S0 = rand_inputs(rng, 1, 70, 2, 6, 4, beta_scale=2.0)
    o_s, s_s = oracle.forward(q, k, v, la, beta, S0)
    o_c, s_c = chunkwise.forward_chunkwise(q, k, v, la, beta, S0, chunk=16)
    if not (np.allclose(o_s, o_c, atol=1e-10) and np.allclose(s_s, s_c, atol=1e-10)):
        failed.append("chunkwise")
    # beta = 0 closed form
    beta0 = np.zeros_like(beta)
    out, Sf = oracle.forward(q, k, v, la, beta0, S0)
    G = np.cumsum(la, axis=1)
    if not np.allclose(out, np.exp(G)[..., None] * np.einsum("bhij,bthi->bthj", S0, q),
                       atol=1e-12):
        failed.append("beta_zero")
    # Householder with v = 0 keeps the norm
    d = 5
    S = rng.standard_normal((1, 1, d, d))
    kk = rng.standard_normal(d)
    kk /= np.linalg.norm(kk)
    z = np.zeros((1, 1, d))
    _, S1 = oracle.decode_step(z, kk[None, None], z, np.zeros((1, 1)), np.full((1, 1), 2.0), S)
    if not np.isclose(np.linalg.norm(S1), np.linalg.norm(S), rtol=1e-12):
        failed.append("householder")
    return failed


@pytest.fixture
def swap_lib():
    import ctypes
    saved = oracle._lib

    def use(path):
        oracle._lib = None
        lib = ctypes.CDLL(path)
        # reuse the argument declarations of the real library
        real = saved or oracle._load()
        for fn in ("gdn_oracle_forward", "gdn_oracle_decode_step", "gdn_oracle_max_threads"):
            getattr(lib, fn).argtypes = getattr(real, fn).argtypes
            getattr(lib, fn).restype = getattr(real, fn).restype
        oracle._lib = lib

    yield use
    oracle._lib = saved


def test_unmodified_oracle_passes_all_checks(tmp_path, swap_lib):
    swap_lib(_build(tmp_path, "clean", open(SRC).read()))
    assert _checks() == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, swap_lib, name):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert old in text, f"mutation site for {name} not found"
    swap_lib(_build(tmp_path, name, text.replace(old, new)))
    failed = _checks()
    assert failed, f"mutant {name} passed every pin"
