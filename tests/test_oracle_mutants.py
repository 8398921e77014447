"""Plant plausible mistakes in (copies of) the oracle and check that the pins catch each.

Each mutant replaces one exact statement of ``oracle/wkv6_oracle.c`` (the statement must
occur exactly once, so the test tracks the source), is compiled to a temporary shared
object with gcc, and must fail at least one pin of ``tests/pins.py``.  CPU only.
"""
import pathlib

import pytest

import oracle as oracle_pkg
from tests import pins

SRC = pathlib.Path(oracle_pkg.__file__).parent / "wkv6_oracle.c"

MUTANTS = {
    # decay transform wrong: single exponential, or sign flipped inside
    "decay_single_exp": ("w[i] = exp(-exp(ot[i]));", "w[i] = exp(-ot[i]);"),
    "decay_sign": ("w[i] = exp(-exp(ot[i]));", "w[i] = exp(-exp(-ot[i]));"),
    # bonus term: u dropped, or the whole bonus dropped
    "bonus_without_u": ("bonus += rt[i] * u[i] * kt[i];", "bonus += rt[i] * kt[i];"),
    "bonus_dropped": ("yt[j] = acc + bonus * vt[j];", "yt[j] = acc;"),
    # decay applied to value columns instead of key rows
    "decay_on_columns": ("S[i * D + j] = w[i] * S[i * D + j] + kt[i] * vt[j];",
                         "S[i * D + j] = w[j] * S[i * D + j] + kt[i] * vt[j];"),
    # outer product transposed
    "outer_transposed": ("S[i * D + j] = w[i] * S[i * D + j] + kt[i] * vt[j];",
                         "S[i * D + j] = w[i] * S[i * D + j] + kt[j] * vt[i];"),
    # new outer product decayed by the current token
    "decay_after_add": ("S[i * D + j] = w[i] * S[i * D + j] + kt[i] * vt[j];",
                        "S[i * D + j] = w[i] * (S[i * D + j] + kt[i] * vt[j]);"),
    # readout through the transposed state
    "readout_transposed": ("acc += rt[i] * S[i * D + j];", "acc += rt[i] * S[j * D + i];"),
    # readout from the state after this token's update (off by one in time)
    "readout_after_update": ("acc += rt[i] * S[i * D + j];",
                             "acc += rt[i] * (w[i] * S[i * D + j] + kt[i] * vt[j]);"),
    # initial state ignored
    "state_in_ignored": ("S[i * D + j] = s_in ? s_in[i * D + j] : 0.0;", "S[i * D + j] = 0.0;"),
    # LayerNorm: unbiased variance, eps outside the square root, beta dropped, mean not removed
    "ln_unbiased_var": ("var /= (double)C;", "var /= (double)(C - 1);"),
    "ln_eps_outside": ("double inv = 1.0 / sqrt(var + eps);", "double inv = 1.0 / (sqrt(var) + eps);"),
    "ln_beta_dropped": ("orow[c] = (xr[c] - mean) * inv * g + bb;", "orow[c] = (xr[c] - mean) * inv * g;"),
    "ln_mean_kept": ("orow[c] = (xr[c] - mean) * inv * g + bb;", "orow[c] = xr[c] * inv * g + bb;"),
    # Finch-C2 exact form
    "c2_key_not_normalised": ("const double kn = kt[i] * (1.0 - w[i]);", "const double kn = kt[i];"),
    "c2_key_scaled_by_w": ("const double kn = kt[i] * (1.0 - w[i]);", "const double kn = kt[i] * w[i];"),
    "c2_second_value_dropped": ("yt[j] = acc + ut[j];", "yt[j] = acc;"),
    "c2_second_value_on_state": ("S[i * D + j] = w[i] * S[i * D + j] + kn * vt[j];",
                                 "S[i * D + j] = w[i] * S[i * D + j] + kn * vt[j] + ut[j];"),
    "c2_decay_after_update": ("S[i * D + j] = w[i] * S[i * D + j] + kn * vt[j];",
                              "S[i * D + j] = w[i] * (S[i * D + j] + kn * vt[j]);"),
    # per-head GroupNorm and gate
    "gn_unbiased_var": ("s2 /= (double)D;", "s2 /= (double)(D - 1);"),
    "gn_gamma_not_per_head": ("const double ga = gamma ? gamma[h * D + c] : 1.0;",
                              "const double ga = gamma ? gamma[c] : 1.0;"),
    "gn_gate_on_input": ("out[base + c] = ((x[base + c] - mu) * rs * ga + be) * gt;",
                         "out[base + c] = ((x[base + c] * gt - mu) * rs * ga + be);"),
    "gn_gate_before_beta": ("out[base + c] = ((x[base + c] - mu) * rs * ga + be) * gt;",
                            "out[base + c] = (x[base + c] - mu) * rs * ga * gt + be;"),
    # backward pass
    "bwd_dr_from_state_after": ("gr += Sprev[i * D + j] * dyt[j];",
                                "gr += Sall[(t + 1) * DD + i * D + j] * dyt[j];"),
    "bwd_dk_bonus_dropped": ("dkt[i] = gk + rt[i] * u[i] * vdy;", "dkt[i] = gk;"),
    "bwd_domega_without_w": ("dot[i] = gw * (-exp(ot[i]) * wi);", "dot[i] = gw * (-exp(ot[i]));"),
    "bwd_carry_on_columns": ("G[i * D + j] = wi * G[i * D + j] + rt[i] * dyt[j];",
                             "G[i * D + j] = exp(-exp(ot[j])) * G[i * D + j] + rt[i] * dyt[j];"),
    "bwd_carry_without_readout": ("G[i * D + j] = wi * G[i * D + j] + rt[i] * dyt[j];",
                                  "G[i * D + j] = wi * G[i * D + j];"),
    "bwd_dv_transposed": ("g += G[i * D + j] * kt[i];", "g += G[j * D + i] * kt[i];"),
    "bwd_du_without_r": ("du_acc[i] += rt[i] * kt[i] * vdy;", "du_acc[i] += kt[i] * vdy;"),
    # Finch-C2 backward
    "c2bwd_dk_without_1mw": ("dkt[i] = gkn * (1.0 - wi);", "dkt[i] = gkn;"),
    "c2bwd_domega_without_key_term": ("dot[i] = (gw - gkn * kt[i]) * (-exp(ot[i]) * wi);",
                                      "dot[i] = gw * (-exp(ot[i]) * wi);"),
    "c2bwd_dv_raw_key": ("g += G[i * D + j] * (kt[i] * (1.0 - exp(-exp(ot[i]))));",
                         "g += G[i * D + j] * kt[i];"),
    # GOLD compression and TokenCat decompression
    "gold_compress_transposed": ("acc += x[n * D + i] * w_kd[(long)j * D + i];",
                                 "acc += x[n * D + i] * w_kd[(long)i * Dc + j];"),
    "gold_cat_drops_c": ("cat[D + j] = c[n * Dc + j];", "cat[D + j] = 0.0;"),
    "gold_rms_eps_outside": ("const double inv_rms = 1.0 / sqrt(ms + eps);",
                             "const double inv_rms = 1.0 / (sqrt(ms) + eps);"),
    "gold_rms_mean_over_cat": ("ms /= (double)D;", "ms /= (double)K;"),
    "gold_gamma_ignored": ("kd[n * D + o] = z[o] * inv_rms * (gamma ? gamma[o] : 1.0);",
                           "kd[n * D + o] = z[o] * inv_rms;"),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    before, after = MUTANTS[name]
    text = SRC.read_text()
    assert text.count(before) == 1, f"mutant {name}: statement not found exactly once"
    mutated = tmp_path / f"{name}.c"
    mutated.write_text(text.replace(before, after))
    so = oracle_pkg.build(mutated, tmp_path / f"lib{name}.so")
    failed = pins.run_all(oracle_pkg.Oracle(so))
    assert failed, f"mutant {name} passes every pin"


def test_unmutated_oracle_passes_all_pins(oracle):
    assert pins.run_all(oracle) == []
