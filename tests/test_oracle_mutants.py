"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each mutant is a one-place edit of oracle/kda_oracle.c: a plausible bug of
the kind the pins are meant to catch (a dropped term, a wrong sign, a
transposed operand, an off-by-one, a read of the pre-update state).  The test
compiles each mutant into a temporary library and checks that at least one
pin fails on it.  The oracle source itself is never modified.
"""
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
import oracle_pins as P  # noqa: E402

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)
SRC = os.path.join(ROOT, "oracle", "kda_oracle.c")

STEP = "        kda_step(S, dk, dv, c->k + th * dk, c->v + th * dv, c->g + th * dk, c->beta[th], u);\n"
READ = "        if (c->o) kda_readout(S, dk, dv, c->q + th * dk, c->o + th * dv);\n"
SNAP = ("        if (c->snaps && c->stride > 0 && pos % c->stride == 0) {\n"
        "            const int64_t idx = c->cu_snap[r] + pos / c->stride - 1;\n"
        "            memcpy(c->snaps + ((size_t)idx * H + h) * ss, S, ss * sizeof(double));\n"
        "        }\n")

MUTANTS = {
    "delta_sign": ("u[j] = beta * (v[j] - u[j]);  /* delta", "u[j] = beta * (v[j] + u[j]);  /* delta"),
    "dropped_decay": ("for (j = 0; j < dv; ++j) row[j] *= a;", "for (j = 0; j < dv; ++j) row[j] *= 1.0;"),
    "half_gate": ("const double a = exp(g[i]);\n        double *row",
                  "const double a = exp(0.5 * g[i]);\n        double *row"),
    "dropped_beta": ("u[j] = beta * (v[j] - u[j]);  /* delta", "u[j] = (v[j] - u[j]);  /* delta"),
    "transposed_readout": ("o[j] += row[j] * q[i];", "o[j] += S[(size_t)j * dv + i] * q[j];"),
    "transposed_write": ("row[j] += k[i] * u[j];", "row[j] += k[j % dk] * u[i % dv];"),
    "preupdate_output": (STEP + READ, READ + STEP),
    "snapshot_before_update": (STEP + READ + SNAP, SNAP + STEP + READ),
    "snapshot_ignores_request_offset": ("c->cu_snap[r] + pos / c->stride - 1", "pos / c->stride - 1"),
    "combine_transposed_M": ("acc += M[(size_t)i * dk + l] * cur[(size_t)l * dv + j];",
                             "acc += M[(size_t)l * dk + i] * cur[(size_t)l * dv + j];"),
    "transition_dropped_beta": ("M[(size_t)i * dk + j] -= bt * kt[i] * w[j];",
                                "M[(size_t)i * dk + j] -= kt[i] * w[j];"),
    "decode_ignores_slot": ("c->slot ? c->slot[n] : n", "n"),
    "bwd_dropped_read_term": ("for (j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += k[i] * du[j];",
                              "for (j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += 0.0 * du[j];"),
    "bwd_du_sign": ("du[j] = -beta * dd[j];", "du[j] = beta * dd[j];"),
    "bwd_dg_without_alpha": ("dg[i] = a * s;", "dg[i] = s;"),
    "bwd_dq_dropped_write": ("dq[i] = s + k[i] * dq_tail;", "dq[i] = s;"),
    "bwd_dk_transposed_state": ("for (j = 0; j < dv; ++j) s += Sp[(size_t)i * dv + j] * du[j];",
                                "for (j = 0; j < dv; ++j) s += Sp[(size_t)(j % dk) * dv + i % dv] * du[j];"),
    "bwd_wrong_checkpoint": ("memcpy(blk, ck + (size_t)b * ss, ss * sizeof(double));",
                             "memcpy(blk, ck + (size_t)(b > 0 ? b - 1 : 0) * ss, ss * sizeof(double));"),
    "readout_uses_key": ("kda_readout(S, dk, dv, c->q + th * dk, c->o + th * dv);\n    free(u);",
                         "kda_readout(S, dk, dv, c->k + th * dk, c->o + th * dv);\n    free(u);"),
}


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="kda_oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, workdir):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation target for {name} must occur exactly once"
    msrc = os.path.join(workdir, f"{name}.c")
    with open(msrc, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(workdir, f"lib_{name}.so")
    oracle.build(src=msrc, out=so)
    script = (
        "import sys; sys.path[:0] = [%r, %r]\n"
        "import oracle, oracle_pins as P\n"
        "lib = oracle.load(%r)\n"
        "for pin in P.ALL_PINS:\n"
        "    try:\n"
        "        pin(lib)\n"
        "    except Exception:\n"
        "        print('FAILED', pin.__name__)\n"
    ) % (ROOT, TESTS, so)
    res = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, f"mutant {name} crashed the pins: {res.stderr[-500:]}"
    assert "FAILED" in res.stdout, f"mutant {name} survived every pin"


def test_unmutated_source_builds_and_passes(workdir):
    so = os.path.join(workdir, "lib_clean.so")
    oracle.build(out=so)
    lib = oracle.load(so)
    for pin in P.ALL_PINS:
        pin(lib)



# Mistakes planted in the fused gate activation (Python side of the oracle): each
# must fail at least one of the gate-logit pins.
_GATE_PINS = [P.pin_gate_logit_map, P.pin_gate_logit_decay, P.pin_gate_logit_backward]


def _sig(x):
    import numpy as np
    return 1.0 / (1.0 + np.exp(-oracle._f64(x)))


_GATE_MUTANTS = {
    "flipped_logit": ("gate_from_logits", lambda x: -5.0 * _sig(-oracle._f64(x))),
    "wrong_scale": ("gate_from_logits", lambda x: -4.0 * _sig(x)),
    "slope_dropped_factor": ("gate_logit_slope", lambda x: -5.0 * _sig(x)),
    "slope_sign": ("gate_logit_slope", lambda x: 5.0 * _sig(x) * (1.0 - _sig(x))),
}


@pytest.mark.parametrize("name", sorted(_GATE_MUTANTS))
def test_gate_mutant_is_caught(name, monkeypatch, oracle_lib):
    attr, fn = _GATE_MUTANTS[name]
    monkeypatch.setattr(oracle, attr, fn)
    caught = False
    for pin in _GATE_PINS:
        try:
            pin(oracle_lib)
        except AssertionError:
            caught = True
            break
    assert caught, f"gate mutant {name} passed every gate pin"
