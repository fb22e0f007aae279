"""Each plausible mistake planted in a copy of the oracle (on the CPU) must
make at least one pin fail: a dropped term, a wrong sign, a swapped
coefficient, a transposed operand, a wrong index, a missing step."""

import importlib.util
import os
import types

import pytest

import pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "muon_oracle.py")

MUTANTS = {
    "b_sign": ("NS_B = -4.7750", "NS_B = 4.7750"),
    "drop_c_term": ("poly = b * gram + c * (gram @ gram)", "poly = b * gram"),
    "swap_a_c": ("x = a * x + poly @ x", "x = c * x + poly @ x"),
    "transposed_gram": ("gram = x @ x.T", "gram = x.T @ x if x.shape[0] == x.shape[1] else x @ x.T"),
    "poly_times_gram": ("x = a * x + poly @ x", "x = a * x + poly @ gram @ x"),
    "no_normalise": ("x = x / (np.linalg.norm(x) + eps)", "x = x"),
    "spectral_normalise": ("x = x / (np.linalg.norm(x) + eps)", "x = x / (np.abs(x).max() + eps)"),
    "no_transpose_back": ("return x.T if transposed else x\n", "return x\n"),
    "no_nesterov": ("u = (1.0 - beta) * g + beta * new_buf", "u = new_buf.copy()"),
    "classic_momentum": ("new_buf = beta * np.asarray(buf, dtype=np.float64) + (1.0 - beta) * g",
                         "new_buf = beta * np.asarray(buf, dtype=np.float64) + g"),
    "scale_inverted": ("return math.sqrt(max(1.0, rows / cols))", "return math.sqrt(max(1.0, cols / rows))"),
    "coupled_decay": ("return w * (1.0 - lr * weight_decay) - lr * scale * np.asarray(o, dtype=np.float64)",
                      "return w * (1.0 - weight_decay) - lr * scale * np.asarray(o, dtype=np.float64)"),
    "adamw_no_bias_corr": ("m_hat = m / (1.0 - p[\"beta1\"] ** step)", "m_hat = m"),
    "adamw_eps_inside": ("np.sqrt(v_hat) + p[\"eps\"]", "np.sqrt(v_hat + p[\"eps\"])"),
    "moment_not_mean": ("return (x.T @ x) / x.shape[0]", "return (x.T @ x)"),
    "moment_transposed": ("return (x.T @ x) / x.shape[0]", "return (x @ x.T) / x.shape[0]"),
    "moment_not_inverted": ("return np.linalg.inv(s + damping * np.eye(s.shape[0]))",
                            "return s + damping * np.eye(s.shape[0])"),
    "block_index": ("out[:, k * d:(k + 1) * d] = g[:, k * d:(k + 1) * d] @ s_inv",
                    "out[:, k * d:(k + 1) * d] = g[:, k * d:(k + 1) * d] @ blocks[0]"),
    "no_damping": ("np.linalg.inv(s + damping * np.eye(s.shape[0]))", "np.linalg.inv(s + 0 * np.eye(s.shape[0]))"),
    "one_step_less": ("for _ in range(steps):", "for _ in range(max(steps - 1, 0)):"),
}


def load_mutant(old, new):
    src = open(SRC).read()
    assert old in src, f"mutation anchor not found: {old!r}"
    src = src.replace(old, new, 1)
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src, "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    mod = load_mutant(*MUTANTS[name])
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(mod)
        except Exception as e:  # AssertionError or a shape error
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
