"""Planted mistakes in the dynamic low-rank oracle (oracle/lowrank.py):
each test loads a copy of the module with one plausible mistake and runs
every pin of test_lowrank_oracle_pins.py against it; at least one must fail.
The unchanged copy must pass them all. CPU only."""
import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lowrank.py")
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import test_lowrank_oracle_pins as pins  # noqa: E402

# (name, text in the source, replacement): the first occurrence is replaced
MISTAKES = [
    ("scaled_by_inverse_scales", "Ws = W * s[None, :]",
     "Ws = W / s[None, :]"),
    ("projection_of_scaled_weight", "return round_bf16(Q), round_bf16(Q.T @ W)",
     "return round_bf16(Q), round_bf16(Q.T @ (W * np.asarray(s)[None, :]))"),
    ("one_iteration_short", "for _ in range(int(iters)):",
     "for _ in range(int(iters) - 1):"),
    ("transpose_step_on_the_unscaled_weight",
     "Z = orthonormalize(Ws.T @ Q)", "Z = orthonormalize(W.T @ Q)"),
    ("single_gram_schmidt_pass", "for _ in range(2):\n            for i in kept:",
     "for _ in range(1):\n            for i in kept:"),
    ("drop_relative_to_first_column",
     "ref = float(np.max(np.linalg.norm(Y, axis=0))) if l else 0.0",
     "ref = float(np.linalg.norm(Y[:, 0])) if l else 0.0"),
    ("no_drop_rule", "if ref > 0.0 and nv > tol * ref:", "if nv > 0.0:"),
    ("absolute_drop_threshold", "if ref > 0.0 and nv > tol * ref:",
     "if ref > 0.0 and nv > tol:"),
    ("projection_instead_of_residual", "return round_bf16(W - B @ A)",
     "return round_bf16(B @ A)"),
    ("residual_rounded_through_fp32",
     "return round_bf16(W - B @ A)",
     "return round_bf16((W - B @ A).astype(np.float32).astype(np.float64))"),
    ("bf16_with_seven_significant_bits", "step_exp = e - 8", "step_exp = e - 7"),
    ("bf16_rounding_half_up",
     "np.rint(np.ldexp(x, -step_exp))", "np.floor(np.ldexp(x, -step_exp) + 0.5)"),
    ("no_subnormal_floor", "e = np.maximum(e, -125)", "e = e"),
    ("near_ties_without_the_chain_bound",
     "bound = (r + 1) * 2.0 ** -24 * (np.abs(W) + np.abs(B) @ np.abs(A))",
     "bound = 0.0 * np.abs(W)"),
    ("near_ties_at_representable_values",
     "dist = np.abs(frac - 0.5) * step", "dist = np.minimum(frac, 1 - frac) * step"),
]


def load_variant(name, text):
    path = os.path.join(ROOT, "_build", "lowrank_variants", f"{name}.py")
    os.makedirs(os.path.dirname(path), exist_ok=True)
    with open(path, "w") as f:
        f.write(text)
    spec = importlib.util.spec_from_file_location(f"lowrank_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def failing_pins(mod):
    failed = []
    for pin in pins.PINS:
        try:
            pin(mod)
        except Exception:  # an assertion, or arithmetic that breaks outright
            failed.append(pin.__name__)
    return failed


def test_unchanged_copy_passes_the_pins():
    assert failing_pins(load_variant("unchanged", open(SRC).read())) == []


@pytest.mark.parametrize("name,old,new", MISTAKES,
                         ids=[m[0] for m in MISTAKES])
def test_each_planted_mistake_fails_a_pin(name, old, new):
    src = open(SRC).read()
    assert old in src, f"{name}: the planted text no longer occurs"
    failed = failing_pins(load_variant(name, src.replace(old, new, 1)))
    assert failed, f"{name}: every pin passed"
