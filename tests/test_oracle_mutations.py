"""Plant plausible mistakes in copies of the oracle and check the pins catch them.

No GPU. Each mutation rewrites one line of the oracle's C source into a temp
directory, compiles it, and runs a compact set of the pins from
``test_oracle_pins.py`` against the broken copy. At least one pin must fail
for every mutation; the unmodified oracle must pass all of them.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from test_oracle_pins import dense_affine_prefix, one_head, rand_head

SRC = os.path.join(os.path.dirname(oracle.__file__), "ckda_oracle.c")

MUTATIONS = {
    "correction_sign": ("row[c] += bk * (v[c] - p[c]);",
                        "row[c] += bk * (v[c] + p[c]);"),
    "dropped_beta": ("const double bk = beta * k[r];",
                     "const double bk = k[r];"),
    "dropped_gate": ("for (c = 0; c < dv; ++c) row[c] *= a;",
                     "for (c = 0; c < dv; ++c) row[c] *= 1.0;"),
    "reversed_gate_channel": ("const double a = alpha[r];",
                              "const double a = alpha[dk - 1 - r];"),
    "readout_with_key": ("      const double qr = q[r];",
                         "      const double qr = k[r];"),
    "read_with_query": ("    const double kr = k[r];",
                        "    const double kr = q[r];"),
    "no_readout_scale": ("for (c = 0; c < dv; ++c) o[c] = scale * p[c];",
                         "for (c = 0; c < dv; ++c) o[c] = p[c];"),
}


def _compile(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path = tmp_path / ("m_%s.c" % name)
    path.write_text(src.replace(old, new))
    so = tmp_path / ("m_%s.so" % name)
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC",
                           "-shared", "-o", str(so), str(path)])
    return oracle._bind(str(so))


def _pins(lib):
    """A compact subset of the oracle pins, run against ``lib``."""
    # dense affine composition, random CKDA inputs, scale != 1
    rng = np.random.default_rng(0)
    q, k, v, a, b = rand_head(rng, 8, 4, 3, "ckda")
    s0 = rng.standard_normal((4, 3))
    o, S = one_head(q, k, v, a, b, s0=s0, scale=0.7, lib=lib)
    o_ref, S_ref = dense_affine_prefix(q, k, v, a, b, s0, scale=0.7)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, atol=1e-12)
    # lesson trace: gate [0.9, 0.2] on memory [10, 10] -> [9, 2]
    _, S = one_head(np.eye(2)[:1], np.eye(2)[:1], np.zeros((1, 1)),
                    np.array([[0.9, 0.2]]), [0.0], s0=[[10.0], [10.0]], lib=lib)
    np.testing.assert_allclose(S[:, 0], [9.0, 2.0], atol=1e-12)
    # rotation from one reflection in the gate plus one beta=2 step
    phi = math.pi / 5
    kk = np.array([[math.cos(phi), math.sin(phi)]])
    _, S = one_head(np.eye(2)[:1], kk, np.zeros((1, 2)),
                    np.array([[-1.0, 1.0]]), [2.0], s0=np.eye(2), lib=lib)
    th = 2 * phi
    np.testing.assert_allclose(
        S, [[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]],
        atol=1e-12)


def test_unmodified_oracle_passes(tmp_path):
    _pins(oracle._load())


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    lib = _compile(tmp_path, name, old, new)
    with pytest.raises(AssertionError):
        _pins(lib)
