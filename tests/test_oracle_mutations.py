"""Every plausible single mistake planted in a copy of the oracle fails a pin.

Each case edits the oracle's source text in memory (never on disk), loads the
edited copy as a fresh module and runs all pins of tests/oracle_pins.py on it.
A mutation that no pin catches would mean the pins leave that part of the
oracle unchecked.
"""

import os
import types

import pytest

from oracle_pins import PINS

SRC_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "oracle", "attention.py")

MUTATIONS = {
    "causal_excludes_diagonal": ("ok = ok & (j <= i)", "ok = ok & (j < i)"),
    "causal_reversed": ("ok = ok & (j <= i)", "ok = ok & (j >= i)"),
    "key_pad_off_by_one": ("ok = (j < key_len) & (i >= 0)", "ok = (j <= key_len) & (i >= 0)"),
    "key_pad_ignored": ("ok = (j < key_len) & (i >= 0)", "ok = (j >= 0) & (i >= 0)"),
    "scale_dropped": ("s = scale * (q_rows @ k.T)", "s = (q_rows @ k.T)"),
    "scale_squared": ("s = scale * (q_rows @ k.T)", "s = scale * scale * (q_rows @ k.T)"),
    "gqa_head_modulo": ("hk = hq // group  #", "hk = hq % Hk  #"),
    "rows_head_modulo": ("        hk = hq // group\n        ok = allowed_keys([i]",
                         "        hk = hq % k.shape[1]\n        ok = allowed_keys([i]"),
    "max_not_subtracted": ("np.exp(s - m_safe[:, None])", "np.exp(s)"),
    "exp_sign_flipped": ("np.exp(s - m_safe[:, None])", "np.exp(m_safe[:, None] - s)"),
    "normalisation_dropped": ("o[has] = (p[has] @ v) / l[has][:, None]", "o[has] = (p[has] @ v)"),
    "lse_without_max": ("lse[has] = m[has] + np.log(l[has])", "lse[has] = np.log(l[has])"),
    "lse_log2": ("lse[has] = m[has] + np.log(l[has])", "lse[has] = m[has] + np.log2(l[has])"),
    "empty_row_lse_zero": ("lse = np.full(p.shape[0], -np.inf, dtype=np.float64)",
                           "lse = np.zeros(p.shape[0], dtype=np.float64)"),
    "flowchart_alpha_dropped_on_o": ("o_new = alpha[:, None] * o_old + p @ v_tile",
                                     "o_new = o_old + p @ v_tile"),
    "flowchart_alpha_dropped_on_l": ("l_new = alpha * l_old + p.sum(axis=1)",
                                     "l_new = l_old + p.sum(axis=1)"),
    "equations_local_factor_dropped": ("a_loc[:, None] * (p_loc @ v_tile)", "(p_loc @ v_tile)"),
    "equations_l_local_factor_dropped": ("a_loc * p_loc.sum(axis=1)", "p_loc.sum(axis=1)"),
    "online_stale_max": ("m_new = np.maximum(m_old, s.max(axis=1))", "m_new = s.max(axis=1)"),
    "v_rows_reversed": ("rows] = _finish(p, m, l, v[b, hk])", "rows] = _finish(p, m, l, v[b, hk][::-1])"),
    "k_rows_reversed": ("s = scores(q[b, hq, rows], k[b, hk], scale, ok,",
                        "s = scores(q[b, hq, rows], k[b, hk][::-1], scale, ok,"),
    "key_range_hi_inclusive": ("in_range = (j >= key_lo) & (j < key_hi)",
                               "in_range = (j >= key_lo) & (j <= key_hi)"),
    "key_range_lo_exclusive": ("in_range = (j >= key_lo) & (j < key_hi)",
                               "in_range = (j > key_lo) & (j < key_hi)"),
    "merge_max_not_subtracted": ("np.exp(np.where(np.isfinite(lse_s), lse_s, 0.0) - m_safe)",
                                 "np.exp(np.where(np.isfinite(lse_s), lse_s, 0.0))"),
    "merge_unweighted": ("num += w[..., None] * o_s", "num += o_s"),
    "merge_unnormalised": ("o[has] = num[has] / den[has][..., None]", "o[has] = num[has]"),
    "merge_lse_without_max": ("lse[has] = m[has] + np.log(den[has])", "lse[has] = np.log(den[has])"),
    "bias_scaled": ("s = s + bias_rows", "s = s + scale * bias_rows"),
    "bias_dropped": ("s = s + bias_rows", "s = s + 0.0 * bias_rows"),
    "bias_transposed": ("None if plane is None else plane[rows])", "None if plane is None else plane.T[rows])"),
    "bias_head_ignored": ("hq if bias.shape[1] > 1 else 0]", "0]"),
    "bias_batch_ignored": ("b if bias.shape[0] > 1 else 0,", "0,"),
    "bias_rows_wrong_row": ("_as_f64(plane[[i]])", "_as_f64(plane[[0]])"),
    "bwd_dsum_dropped": ("ds = p * (dp - dsum[:, None])", "ds = p * dp"),
    "bwd_dq_unscaled": ("dq[b, hq] = scale * (ds @ k[b, hk])", "dq[b, hq] = (ds @ k[b, hk])"),
    "bwd_dk_untransposed": ("dk[b, hk] += scale * (ds.T @ q[b, hq])", "dk[b, hk] += scale * (ds @ q[b, hq])"),
    "bwd_dv_untransposed": ("dv[b, hk] += p.T @ do[b, hq]", "dv[b, hk] += p @ do[b, hq]"),
    "bwd_gqa_overwrites": ("dv[b, hk] += p.T @ do[b, hq]", "dv[b, hk] = p.T @ do[b, hq]"),
    "bwd_lse_ignored": ("np.exp(s[has] - lse[b, hq][has][:, None])", "np.exp(s[has])"),
    "bwd_dp_wrong_v": ("dp = do[b, hq] @ v[b, hk].T", "dp = do[b, hq] @ v[b, hk][::-1].T"),
}


def load_mutant(old, new):
    src = open(SRC_PATH, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name):
    mutant = load_mutant(*MUTATIONS[name])
    caught = []
    for pin in PINS:
        try:
            pin(mutant)
        except Exception:  # an assertion or a crash both count as caught
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {name}"


def test_unmutated_copy_passes_every_pin():
    mod = load_mutant("import numpy as np", "import numpy as np")
    for pin in PINS:
        pin(mod)
