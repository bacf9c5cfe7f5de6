"""Planted mistakes in the oracle: each one must fail a pin.

The pins in test_oracle_pins.py, test_tconv_oracle.py and test_nvfp4_oracle.py
tie the float64 oracle to brute force, closed forms, hand-worked examples,
library routines and invariants.  This file checks that they would notice a
plausible mistake: it builds altered copies of the oracle's C source (a sign,
an index, a dropped or misplaced term, a transposed operand, a wrong field of a
number format), runs the pins against each copy in a child process, and
expects at least one pin to fail.  The golden regression fixture is left out of
those runs, since it was written by the oracle itself and would flag any change.

The mistakes are planted in the oracle on the CPU only; no GPU code is built.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = "tests/test_oracle_pins.py"
CONV = "tests/test_tconv_oracle.py"
FP4 = "tests/test_nvfp4_oracle.py"

# name -> (pin file to run first, [(original text, planted text), ...]); every
# original text occurs exactly once in the oracle's C source.
MISTAKES = {
    "rope-rotation-transposed": (PINS, [
        ("out[off + 2 * j] = x0 * c - x1 * s;", "out[off + 2 * j] = x0 * c + x1 * s;"),
        ("out[off + 2 * j + 1] = x0 * s + x1 * c;", "out[off + 2 * j + 1] = -x0 * s + x1 * c;")]),
    "rope-frequency-exponent-halved": (PINS, [
        ("pow(theta, -2.0 * (double)j / (double)da)", "pow(theta, -(double)j / (double)da)")]),
    "rope-axes-reversed": (PINS, [("(double)p[a] * freq", "(double)p[2 - a] * freq")]),
    "rope-half-split-pairs": (PINS, [
        ("x0 = u[off + 2 * j], x1 = u[off + 2 * j + 1];", "x0 = u[off + j], x1 = u[off + j + da / 2];"),
        ("out[off + 2 * j] = x0 * c - x1 * s;", "out[off + j] = x0 * c - x1 * s;"),
        ("out[off + 2 * j + 1] = x0 * s + x1 * c;", "out[off + j + da / 2] = x0 * s + x1 * c;")]),
    "phi-identity": (PINS, [("return x > 0.0 ? x : 0.0;", "return x;")]),
    "phi-absolute-value": (PINS, [("return x > 0.0 ? x : 0.0;", "return x > 0.0 ? x : -x;")]),
    "mask-excludes-own-block": (PINS, [("if (kblk[m] > qblk[n]) continue;", "if (kblk[m] >= qblk[n]) continue;")]),
    "mask-admits-later-blocks": (PINS, [("if (kblk[m] > qblk[n]) continue;", "if (kblk[m] > qblk[n] + 1) continue;")]),
    "rope-also-in-denominator": (PINS, [
        ("s += qp[i] * kp[i];", "s += qr[i] * kr[i];"),
        ("z[i] += ph[i];", "z[i] += rt[i];"),
        ("den += ph[i] * z[i];", "den += rt[i] * z[i];")]),
    "no-rope-in-numerator": (PINS, [
        ("w += qr[i] * kr[i];", "w += qp[i] * kp[i];"),
        ("S[(size_t)i * d + j] += rt[i] * (double)vm[j];", "S[(size_t)i * d + j] += ph[i] * (double)vm[j];"),
        ("s += rt[i] * S[(size_t)i * d + j];", "s += ph[i] * S[(size_t)i * d + j];")]),
    "eps-dropped": (PINS, [
        ("/ (den[r] + eps);", "/ (den[r] + 0.0 * eps);"),
        ("den += eps;", "den += 0.0 * eps;")]),
    "eps-outside-the-division": (PINS, [
        ("/ (den[r] + eps);", "/ den[r] + eps;"),
        ("den += eps;", "den += 0.0 * eps;"),
        ("o[j] = s / den;", "o[j] = s / den + eps;")]),
    "state-transposed": (PINS, [
        ("S[(size_t)i * d + j] += rt[i] * (double)vm[j];", "S[(size_t)j * d + i] += rt[i] * (double)vm[j];")]),
    "grid-y-and-x-swapped": (PINS, [
        ("pos[3 * n + 1] = y;", "pos[3 * n + 1] = x;"),
        ("pos[3 * n + 2] = x;", "pos[3 * n + 2] = y;")]),
    "grid-block-relative-to-call": (PINS, [("blk[n] = (t0 + t) / F;", "blk[n] = t / F;")]),
    "tconv-taps-reversed": (CONV, [
        ("w[3 * c] * xp + w[3 * c + 1] * xc + w[3 * c + 2] * xn",
         "w[3 * c + 2] * xp + w[3 * c + 1] * xc + w[3 * c] * xn")]),
    "tconv-next-frame-crosses-blocks": (CONV, [("(ta + 1) / F == ta / F", "1")]),
    "tconv-cache-ignored": (CONV, [("else if (ta > 0 && prev != NULL)", "else if (0)")]),
    "tconv-bias-dropped": (CONV, [("(bias ? bias[c] : 0.0)", "0.0")]),
    "e2m1-exponent-bias": (FP4, [("ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e)")]),
    "e2m1-subnormal-step": (FP4, [("e == 0 ? 0.5 * m :", "e == 0 ? 1.0 * m :")]),
    "e4m3-exponent-bias": (FP4, [("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)")]),
    "nvfp4-nibble-order": (FP4, [
        ("(i & 1) ? (byte >> 4) & 15 : byte & 15", "(i & 1) ? byte & 15 : (byte >> 4) & 15")]),
    "nvfp4-scale-per-32": (FP4, [("scale[r * (d / 16) + i / 16]", "scale[r * (d / 16) + i / 32]")]),
    "nvfp4-global-scale-dropped": (FP4, [(") * global;", ") * 1.0;")]),
}


def _plant(src, edits):
    for old, new in edits:
        assert src.count(old) == 1, f"{old!r} occurs {src.count(old)} times in the oracle source"
        src = src.replace(old, new)
    return src


def _run_pins(lib, first):
    files = [first] + [f for f in (PINS, CONV, FP4) if f != first]
    env = dict(os.environ, BLIN_ORACLE_MUTANT_LIB=lib, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
           "--deselect", f"{PINS}::test_golden_fixture_unchanged", *files]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout + r.stderr


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    src = open(oracle._SRC).read()
    jobs = {"unaltered": (PINS, [])}
    jobs.update(MISTAKES)
    libs = {}
    for name, (first, edits) in jobs.items():
        folder = tmp_path_factory.mktemp(name)
        c_file = folder / "oracle.c"
        c_file.write_text(_plant(src, edits))
        lib = str(folder / "oracle.so")
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", lib, str(c_file),
                               "-lm"])
        libs[name] = (lib, first)
    workers = max(2, min(8, len(os.sched_getaffinity(0))))  # each child imports torch: keep the count modest
    with ThreadPoolExecutor(max_workers=workers) as ex:
        futs = {name: ex.submit(_run_pins, lib, first) for name, (lib, first) in libs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_unaltered_copy_passes_every_pin(outcomes):
    rc, out = outcomes["unaltered"]
    assert rc == 0, out[-3000:]


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_mistake_fails_a_pin(outcomes, name):
    rc, out = outcomes[name]
    failed = [line.split()[1] for line in out.splitlines() if line.startswith("FAILED ")]
    assert rc == 1 and failed, f"no pin caught {name}:\n{out[-3000:]}"
    print(f"{name}: caught by {failed[0]}")
