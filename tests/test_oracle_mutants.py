"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check
that at least one pin catches each of them.  This is evidence that the pins in
tests/oracle_pins.py constrain every step of the oracle, not just some."""
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)

# Runs every pin against one compiled library in a child process (a mutant may
# crash) and prints the names of the pins that failed.
_CHILD = """
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle
from oracle_pins import ALL_PINS
o = oracle.Oracle({lib!r})
for pin in ALL_PINS:
    try:
        pin(o)
    except (AssertionError, ValueError, IndexError):
        print("CAUGHT", pin.__name__)
"""

SRC = os.path.join(os.path.dirname(oracle.__file__), "slr_oracle.c")

# (name, text to replace, replacement, expected number of occurrences)
MUTANTS = [
    ("tie_to_higher_index", "(kq == kp && q < p)", "(kq == kp && q > p)", 2),
    ("signed_key", " & 0x7FFFu;", ";", 4),
    ("smallest_magnitude", "if (rank < 2) kept[n++] = p;", "if (rank >= 2) kept[n++] = p;", 2),
    ("kept_order_swapped", "*idx0 = kept[0];\n    *idx1 = kept[1];", "*idx0 = kept[1];\n    *idx1 = kept[0];", 2),
    ("nibble_fields_swapped", "(unsigned)a | ((unsigned)b << 2)", "(unsigned)b | ((unsigned)a << 2)", 2),
    ("nibble_position_swapped", "nib << (4 * (g % 2))", "nib << (4 * ((g + 1) % 2))", 2),
    ("lowrank_sign", "row[j] += lr;", "row[j] -= lr;", 1),
    ("lowrank_dropped", "row[j] += lr;", "(void)lr;", 1),
    ("V_transposed", "V[k * d_in + j]", "V[j * r + k]", 2),
    ("U_wrong_row", "U[i * r + k]", "U[k]", 1),
    ("X_wrong_row", "xr[j] = bf16_bits_to_double(X[m * d_in + j]);", "xr[j] = bf16_bits_to_double(X[j]);", 1),
    ("bound_signed", "fabs(xr[j]) * fabs(row[j])", "xr[j] * row[j]", 1),
    ("sparse_vals_swapped", "row[4 * g + a] = bf16_bits_to_double(vals[i * (d_in / 2) + 2 * g + 0]);",
     "row[4 * g + a] = bf16_bits_to_double(vals[i * (d_in / 2) + 2 * g + 1]);", 1),
    ("scaled_tie_to_higher_index", "(key[q] == key[p] && q < p)", "(key[q] == key[p] && q > p)", 1),
    ("scaled_signed_scale", "aw * fabsf(s)", "aw * s", 1),
    ("scaled_nan_lowest", "if (isnan(prod)) return 0x7FFFFFFFu;", "if (isnan(prod)) return 0u;", 1),
    ("scaled_wrong_column", "scale[4 * g + p]", "scale[p]", 1),
    ("scaled_scale_ignored", "key[p] = scaled_key(w[p], scale[4 * g + p]);",
     "key[p] = scaled_key(w[p], 1.0f);", 1),
    ("norm_no_sqrt", "out[j] = sqrt(acc);", "out[j] = acc;", 1),
    ("norm_abs_sum", "acc += x * x;", "acc += fabs(x);", 1),
    ("pack28_meta_shift", "(uint8_t)(kept[0] | (kept[1] << 3))", "(uint8_t)(kept[0] | (kept[1] << 2))", 1),
    ("pack28_vals_swapped", "vals[i * (d_in / 4) + 2 * g + 0] = w[kept[0]];", "vals[i * (d_in / 4) + 2 * g + 0] = w[kept[1]];", 1),
    ("pack28_group_stride", "const uint16_t *w = W + i * ldw + 8 * g;", "const uint16_t *w = W + i * ldw + 4 * g;", 1),
    ("unpack28_meta_field", "(int)((byte >> 3) & 7u)", "(int)((byte >> 4) & 7u)", 1),
    ("norm_wrong_column", "double x = bf16_bits_to_double(X[m * d_in + j]);",
     "double x = bf16_bits_to_double(X[m * d_in]);", 1),
]


@pytest.mark.parametrize("name,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, count, tmp_path):
    text = open(SRC).read()
    assert text.count(old) == count, f"mutation site for {name} not found"
    src = tmp_path / f"{name}.c"
    src.write_text(text.replace(old, new))
    lib = oracle.compile_source(str(src), str(tmp_path / f"lib{name}.so"))
    proc = subprocess.run([sys.executable, "-c", _CHILD.format(root=ROOT, tests=TESTS, lib=lib)],
                          capture_output=True, text=True, timeout=300)
    caught = [l.split()[1] for l in proc.stdout.splitlines() if l.startswith("CAUGHT")]
    # A crash of the mutant also counts as detection, but say so.
    assert caught or proc.returncode != 0, f"no pin caught mutant {name}: {proc.stderr[-500:]}"


# Planted mistakes in the alternating-minimisation oracle (numpy): each copy is
# imported from a temporary file and must fail at least one AM pin.
AM_SRC = os.path.join(os.path.dirname(oracle.__file__), "datafree_am.py")
AM_MUTANTS = [
    ("am_tie_to_higher", "            if q < p:\n", "            if q > p:\n", 1),
    ("am_keep_three", "return (beaten < 2).reshape", "return (beaten < 3).reshape", 1),
    ("am_truncation_one_more", "return (Uz[:, :r] * sz[:r]) @ Vz[:r, :]", "return (Uz[:, :r + 1] * sz[:r + 1]) @ Vz[:r + 1, :]", 1),
    ("am_smallest_singular", "return (Uz[:, :r] * sz[:r]) @ Vz[:r, :]", "return (Uz[:, -r:] * sz[-r:]) @ Vz[-r:, :]", 1),
    ("am_threshold_signed", "g = np.abs(R).reshape", "g = R.reshape", 1),
    ("am_p2_uses_w", "L = truncated_svd(Wf - S, r)", "L = truncated_svd(Wf, r)", 1),
    ("am_p1_ignores_l", "S = hard_threshold_2to4(Wf - L)\n        objs", "S = hard_threshold_2to4(Wf)\n        objs", 1),
]


@pytest.mark.parametrize("name,old,new,count", AM_MUTANTS, ids=[m[0] for m in AM_MUTANTS])
def test_am_mutant_is_caught(name, old, new, count, tmp_path):
    import importlib.util
    import sys as _sys
    _sys.path.insert(0, TESTS)
    from oracle_pins import AM_PINS
    text = open(AM_SRC).read()
    assert text.count(old) == count, f"mutation site for {name} not found"
    path = tmp_path / f"{name}.py"
    path.write_text(text.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"am_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    caught = []
    for pin in AM_PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError, np.linalg.LinAlgError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"


LORA_SRC = os.path.join(os.path.dirname(oracle.__file__), "lora_backward.py")
LORA_MUTANTS = [
    ("lora_v_rows_reversed", "T = Xf @ Vf.T", "T = Xf @ Vf[::-1].T", 1),
    ("lora_dv_sign", "dV = G.T @ Xf", "dV = -(G.T @ Xf)", 1),
    ("lora_du_uses_u", "dU = dYf.T @ T", "dU = dYf.T @ (T + 0.5 * (dYf @ Uf))", 1),
    ("lora_bound_signed", "B_dU = np.abs(dYf).T @ (np.abs(Xf) @ np.abs(Vf).T)", "B_dU = np.abs(dYf).T @ (np.abs(Xf) @ Vf.T)", 1),
]


@pytest.mark.parametrize("name,old,new,count", LORA_MUTANTS, ids=[m[0] for m in LORA_MUTANTS])
def test_lora_mutant_is_caught(name, old, new, count, tmp_path):
    import importlib.util
    import sys as _sys
    _sys.path.insert(0, TESTS)
    from oracle_pins import LORA_PINS
    text = open(LORA_SRC).read()
    assert text.count(old) == count, f"mutation site for {name} not found"
    path = tmp_path / f"{name}.py"
    path.write_text(text.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"lora_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    caught = []
    for pin in LORA_PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"
