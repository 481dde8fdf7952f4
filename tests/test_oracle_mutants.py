"""Mutation check of the oracle's pins: each plausible slip planted in a copy of the oracle's C
source (a dropped term, a wrong sign or index, a transposed block) must fail at least one pin.

The mutants are compiled on the CPU into a temporary directory and never touch the real
oracle.  Every mutation keeps all memory accesses in bounds.
"""
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
from tests import _pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "fir_oracle.c")

# (name, original text, replacement); the original must occur exactly once.
MUTANTS = [
    ("anticausal_index", "(b * L + (t - j)) * D + c;\n                s += hg[j] * (k[src] * v[src]);", "(b * L + (t - j + (t + j < L ? 2 * j : 0))) * D + c;\n                s += hg[j] * (k[src] * v[src]);"),
    ("reversed_taps", "s += hg[j] * (k[src] * v[src]);", "s += hg[l_h - 1 - j] * (k[src] * v[src]);"),
    ("dropped_v_gate", "s += hg[j] * (k[src] * v[src]);", "s += hg[j] * k[src];"),
    ("dropped_k_gate", "s += hg[j] * (k[src] * v[src]);", "s += hg[j] * v[src];"),
    ("dropped_q_gate", "y[row * D + c] = q[row * D + c] * s;", "y[row * D + c] = s;"),
    ("wrong_group", "const double *hg = h + (c / d_g) * l_h;\n            double s = 0.0;", "const double *hg = h + (c % (D / d_g)) * l_h;\n            double s = 0.0;"),
    ("dropped_last_tap", "for (int64_t j = 0; j <= jmax; ++j) {", "for (int64_t j = 0; j < jmax; ++j) {"),
    ("ignores_batch", "(b * L + (t - j)) * D + c;\n                s += hg[j] * (k[src] * v[src]);", "((t - j)) * D + c;\n                s += hg[j] * (k[src] * v[src]);"),
    ("transposed_block", "const int64_t idx = m * l_b + i - j;", "const int64_t idx = m * l_b + j - i;"),
    ("block_sign", "const int64_t src_chunk = n - m;", "const int64_t src_chunk = n + m - 2 * m * (n >= m);"),
    ("block_index", "const int64_t idx = m * l_b + i - jj;  /* H_m[i][jj] */", "const int64_t idx = m * l_b + jj - i;"),
    ("block_drops_history", "if (src_chunk < 0) continue;", "if (src_chunk < 0 || m > 0) continue;"),
    ("gate_added", "s += hg[j] * (k[src] * v[src]);", "s += hg[j] * (k[src] + v[src]);"),
    ("bwd_dx_drops_q", "dx += hg[j] * (dy[src] * q[src]);", "dx += hg[j] * dy[src];"),
    ("bwd_dk_wrong_factor", "dk[e] = dx * v[e];", "dk[e] = dx * k[e];"),
    ("bwd_dq_wrong_factor", "dq[e] = dy[e] * z;", "dq[e] = q[e] * z;"),
    ("bwd_dh_no_lag", "s += (dy[e] * q[e]) * (k[src] * v[src]);", "s += (dy[e] * q[e]) * (k[e] * v[e]);"),
    ("rows_reversed_taps", "acc += hg[tap] * (k[at] * v[at]);", "acc += hg[l_h - 1 - tap] * (k[at] * v[at]);"),
    ("rows_drops_last_tap", "for (int64_t tap = 0; tap <= last; ++tap) {", "for (int64_t tap = 0; tap < last; ++tap) {"),
    ("bwd_dx_drops_tap0", "for (int64_t j = 0; j < l_h && t + j < L; ++j) {", "for (int64_t j = 1; j < l_h && t + j < L; ++j) {"),
]


def _build_mutant(tmp, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation site %r not unique in the oracle source" % name
    path = os.path.join(tmp, name + ".c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(tmp, name + ".so")
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", lib, path], check=True)
    return oracle.OracleLib(lib)


@pytest.fixture(scope="module")
def tmpdir_mut():
    d = tempfile.mkdtemp(prefix="oracle_mut_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmpdir_mut):
    mut = _build_mutant(tmpdir_mut, name, old, new)
    caught = []
    for pin in _pins.ALL_PINS:
        try:
            pin(mut)
        except Exception:  # any failure of a pin counts as catching the mutant
            caught.append(pin.__name__)
    assert caught, "mutant %s passes every pin" % name
