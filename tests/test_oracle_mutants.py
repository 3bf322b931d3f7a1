"""Planted mistakes in copies of the oracle must each fail some pin.

Every mutant is the oracle's source with one plausible mistake (a dropped
term, a wrong sign, index or rounding mode, a transposed layout).  The copy is
loaded as a separate module on the CPU; the real oracle is never modified.
"""
import importlib.util
import os

import pytest

from oracle_pins import ALL_CHECKS

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "varq_oracle.py")

MUTANTS = {
    "rint_to_floor": ("q = np.rint((xb - mn[:, :, None, :]) / s_safe[:, :, None, :])",
                      "q = np.floor((xb - mn[:, :, None, :]) / s_safe[:, :, None, :])"),
    "cell_rint_to_floor": ("q = np.rint(np.float32(x - mn) / s)", "q = np.floor(np.float32(x - mn) / s)"),
    "ties_away_from_zero": ("q = np.rint((xb - mn[:, :, None, :]) / s_safe[:, :, None, :])",
                            "q = np.floor((xb - mn[:, :, None, :]) / s_safe[:, :, None, :] + np.float32(0.5))"),
    "scale_over_2_pow_b": ("s = (mx - mn) / qmax                       # two fp32 roundings",
                           "s = (mx - mn) / (qmax + 1)"),
    "reciprocal_multiply": ("q = np.rint((xb - mn[:, :, None, :]) / s_safe[:, :, None, :])",
                            "q = np.rint((xb - mn[:, :, None, :]) * (np.float32(1) / s_safe[:, :, None, :]))"),
    "pack_msb_first": ("words |= slots[:, :, :, j, :] << np.uint32(j * bits)",
                       "words |= slots[:, :, :, j, :] << np.uint32((cpw - 1 - j) * bits)"),
    "pack_power_of_two_slots": ("return 32 // bits", "return 1 << ((32 // bits).bit_length() - 1)"),
    "meta_halves_swapped": ("return lo | (hi << 16)", "return hi | (lo << 16)"),
    "dequant_drops_min": ("exact = codes.astype(np.float64) * s16[:, :, tb, :] + m16[:, :, tb, :]",
                          "exact = codes.astype(np.float64) * s16[:, :, tb, :]"),
    "dequant_block_off_by_one": ('np.arange(n_tokens), side="right") - 1',
                                 'np.arange(n_tokens), side="left") - 1'),
    "bf16_truncates": ("r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)",
                       "r = (u >> 16).astype(np.uint16)"),
    "softmax_max_over_wrong_axis": ("m = s.max(axis=1, keepdims=True)", "m = s.max(axis=0, keepdims=True)"),
    "attention_no_scale": ("s = (q @ k.T) * scale", "s = (q @ k.T)"),
    "rope_sign": ("out[..., 0::2] = a * c - b * s", "out[..., 0::2] = a * c + b * s"),
    "rope_pairs_halves": ("a = k[..., 0::2]\n    b = k[..., 1::2]",
                          "a = k[..., :k.shape[-1] // 2]\n    b = k[..., k.shape[-1] // 2:]"),
    "meta_two_bytes": ("meta = nb * 32.0", "meta = nb * 16.0"),
    "schedule_row_column_swapped": ("    row = in_frame // grid_w\n    col = in_frame % grid_w",
                                    "    row = in_frame % grid_w\n    col = in_frame // grid_w"),
    "schedule_frequency_exponent": ("float(base) ** (-j / n)", "float(base) ** (-2 * j / n)"),
    "schedule_frame_local": ("frame = t // frame_tokens", "frame = (t // frame_tokens) % 3"),
    "reduction_per_block_padding": ("words = words_per_row(t, bits) if whole_words else t / cpw",
                                    "words = words_per_row(t, bits) + nb - 1"),
}


def _load_mutant(name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutant {name}: anchor not found exactly once"
    mod_src = src.replace(old, new)
    spec = importlib.util.spec_from_loader(f"varq_oracle_mutant_{name}", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(mod_src, f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    mod = _load_mutant(name, old, new)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(mod)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"no pin catches mutant {name}"
