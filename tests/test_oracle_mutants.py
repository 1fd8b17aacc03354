"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that
at least one pin catches each: the pins are strong enough to trust the oracle."""
import importlib.util
import os
import sys
import types

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import oracle_pins  # noqa: E402
from oracle import mla_oracle  # noqa: E402

SRC = open(mla_oracle.__file__).read()

# (description, exact source text, replacement)
MUTANTS = [
    ("rope sign flipped", "x0 * cos - x1 * sin", "x0 * cos + x1 * sin"),
    ("rope frequency exponent halved", "-2.0 * i / d_rope", "-1.0 * i / d_rope"),
    ("rope on split halves instead of interleaved pairs",
     "x0 = x[..., 0::2]\n    x1 = x[..., 1::2]", "x0 = x[..., : d // 2]\n    x1 = x[..., d // 2 :]"),
    ("cache rope keys one position late", "rope(k[b, :L], np.arange(L), base)",
     "rope(k[b, :L], np.arange(L) + 1, base)"),
    ("query position always the last slot", "p = L - n_q + j                                 # query position",
     "p = L - 1"),
    ("softmax scale dropped", "s = (K @ q) * scale", "s = (K @ q)"),
    ("scale without the rope width", "s = (K @ q) * scale", "s = (K @ q) * scale * 1.25"),
    ("query rope not rotated", "rope(q_rope[b, j, h], p + pos_offset, base)", "q_rope[b, j, h]"),
    ("rope term dropped from the key", "K = np.concatenate([K_nope[: p + 1], k_r[: p + 1]], axis=1)",
     "K = np.concatenate([K_nope[: p + 1], 0 * k_r[: p + 1]], axis=1)"),
    ("value from the key weights", "V = c @ W_uv[h]", "V = c @ W_uv[h][::-1]"),
    ("key weights transposed per head", "K_nope = c @ W_uk[h]", "K_nope = c @ W_uk[(h + 1) % W_uk.shape[0]]"),
    ("softmax not normalised", "return e / np.sum(e)", "return e"),
    ("one key too many", "out[b, j, h] = w @ V[: p + 1]", "out[b, j, h] = w @ V[1 : p + 2]"),
    ("append rope key not rotated", "rows[:, d_c:] = rope(y[:, d_c:], np.asarray(positions), base)",
     "rows[:, d_c:] = y[:, d_c:]"),
    ("append split taken from the wrong end", "y = _f64(x) @ _f64(W_dkv)", "y = np.roll(_f64(x) @ _f64(W_dkv), 3, axis=1)"),
    ("appended row written one slot late", "c[b, pos[b, i]] = r[:d_c]", "c[b, pos[b, i] - 1] = r[:d_c]"),
    ("mha cache count without the value", "return heads * (qk_dim + v_dim)", "return heads * qk_dim"),
    ("rms over the sum instead of the mean", "np.mean(c * c, axis=-1, keepdims=True)",
     "np.sum(c * c, axis=-1, keepdims=True)"),
    ("rms norm applied to the rope key too", "rows[:, :d_c] = rms_norm(y[:, :d_c], rms_gamma, eps)",
     "rows[:, :d_c] = rms_norm(y[:, :d_c], rms_gamma, eps)\n        rows[:, d_c:] = y[:, d_c:] / np.sqrt(np.mean(y[:, d_c:] ** 2, axis=-1, keepdims=True) + eps)\n        y = rows"),
    ("rms norm without gamma", "return _f64(gamma) * c / rms", "return c / rms"),
    ("output heads concatenated value-major", "return out.reshape(T, H * v) @ _f64(W_O)",
     "return out.transpose(0, 2, 1).reshape(T, H * v) @ _f64(W_O)"),
    ("output projection with the weight transposed per block", "return out.reshape(T, H * v) @ _f64(W_O)",
     "return out.reshape(T, H * v) @ _f64(W_O)[::-1]"),
    ("sparse selection ignores the count", "rows = sel[b, j, : int(n_sel[b, j])]", "rows = sel[b, j]"),
    ("sparse rows taken one slot late", "c = _f64(c_kv[b, rows])                             # [k][d_c]",
     "c = _f64(c_kv[b, rows + 1])                         # [k][d_c]"),
    ("sparse query rotated at the wrong position", "q = np.concatenate([q_nope[b, j, h], rope(q_rope[b, j, h], p, base)])",
     "q = np.concatenate([q_nope[b, j, h], rope(q_rope[b, j, h], p + 1, base)])"),
    ("rms epsilon outside the square root", "np.sqrt(np.mean(c * c, axis=-1, keepdims=True) + eps)",
     "np.sqrt(np.mean(c * c, axis=-1, keepdims=True)) + eps"),
]


def _mutant(old, new):
    assert SRC.count(old) == 1, f"mutation target not unique/absent: {old!r}"
    mod = types.ModuleType("mla_oracle_mutant")
    mod.__file__ = mla_oracle.__file__
    exec(compile(SRC.replace(old, new), "mla_oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(desc, old, new):
    mod = _mutant(old, new)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mod)
        except Exception as e:  # noqa: BLE001 -- any failure counts as caught
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant: {desc}"
