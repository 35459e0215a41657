"""Plants plausible mistakes in a copy of the oracle (CPU only) and checks
that the pin suite catches every one of them.

Each mutant is a one-line source edit of ``oracle/muon_oracle.py``: a dropped
term, a flipped sign, a wrong index or operand order, a missing transpose.
The edited copy is compiled into a throw-away module; the real oracle is not
touched.  (Running the iteration on the tall orientation instead of the wide
one is not a mistake: an odd matrix polynomial satisfies
X p(X^T X) = p(X X^T) X, so that edit changes only the cost.)
"""
import types
from pathlib import Path

import pytest

from oracle_pins import ALL_PINS

SRC = (Path(__file__).resolve().parent.parent / "oracle" / "muon_oracle.py").read_text()

MUTANTS = {
    "b_sign": ("Bp = b * A + c * (A @ A)", "Bp = -b * A + c * (A @ A)"),
    "drop_c_term": ("Bp = b * A + c * (A @ A)", "Bp = b * A"),
    "drop_aX": ("X = a * X + Bp @ X", "X = Bp @ X"),
    "operand_order": ("X = a * X + Bp @ X", "X = a * X + (X @ Bp if X.shape[0] == X.shape[1] else Bp @ X.T @ X)"),
    "wrong_gram_side": ("A = X @ X.T\n", "A = (X.T @ X)[: X.shape[0], : X.shape[0]]\n"),
    "coeff_swap": ("NS_B = -4.7750\nNS_C = 2.0315", "NS_B = 2.0315\nNS_C = -4.7750"),
    "steps_off_by_one": ("for _ in range(steps):\n        A = X @ X.T",
                         "for _ in range(max(steps - 1, 0)):\n        A = X @ X.T"),
    "gram_missing_QT": ("A = Q @ G @ Q.T", "A = Q @ G"),
    "gram_no_identity": ("Q = (a * I + b * A + c * (A @ A)) @ Q", "Q = (b * A + c * (A @ A)) @ Q"),
    "gram_final_transposed": ("return Q @ X0", "return Q.T @ Q @ X0"),
    "norm_squared": ("return X / (np.sqrt(np.sum(X * X)) + eps)", "return X / (np.sum(X * X) + eps)"),
    "no_normalise": ("return X / (np.sqrt(np.sum(X * X)) + eps)", "return X"),
    "momentum_old_buffer": ("U = G + mu * B_new if nesterov else B_new", "U = G + mu * B if nesterov else B_new"),
    "momentum_lerp": ("B_new = mu * B + G", "B_new = mu * B + (1 - mu) * G"),
    "momentum_no_grad": ("U = G + mu * B_new if nesterov else B_new", "U = mu * B_new if nesterov else B_new"),
    "scale_uses_min": ("RMS_FACTOR * math.sqrt(max(rows, cols))", "RMS_FACTOR * math.sqrt(min(rows, cols))"),
    "scale_factor": ("RMS_FACTOR = 0.2", "RMS_FACTOR = 0.25"),
    "decay_after_update": ("return (1.0 - lr * wd) * W - lr * rms_scale(rows, cols) * O",
                           "return (1.0 - lr * wd) * (W - lr * rms_scale(rows, cols) * O)"),
    "update_sign": ("return (1.0 - lr * wd) * W - lr * rms_scale(rows, cols) * O",
                    "return (1.0 - lr * wd) * W + lr * rms_scale(rows, cols) * O"),
    "decay_sign": ("return (1.0 - lr * wd) * W - lr", "return (1.0 + lr * wd) * W - lr"),
    "no_transpose_back": ("O = XK.T if transposed else XK", "O = XK.reshape(U.shape)"),
}


def _mutant(name):
    old, new = MUTANTS[name]
    assert SRC.count(old) >= 1, f"mutation anchor for {name} not found"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    exec(compile(SRC.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    mod = _mutant(name)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(mod)
        except Exception as e:  # AssertionError, or a shape error the mistake causes
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin catches mutant {name}"
