"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of oracle/sf_oracle.c (a dropped term, a wrong sign, an
off-by-one, a transposed operand, a wrong rounding), builds it on the CPU, swaps it in for the
real oracle and runs the pins of test_oracle_pins.py until one fails. A mistake that no pin
catches fails this test. Nothing here touches the CUDA path.
"""
import ctypes
import inspect
import os
import subprocess

import pytest

import oracle.oracle as ormod
from tests import test_oracle_pins as pins

MUTANTS = {
    "charge_gain_not_halved": ("charge[r] = 0.5f * charge[r] + 0.5f * share;",
                               "charge[r] = 0.5f * charge[r] + share;"),
    "charge_no_decay": ("charge[r] = 0.5f * charge[r] + 0.5f * share;",
                        "charge[r] = charge[r] + 0.5f * share;"),
    "threshold_strict": ("if (charge[r] >= thr)", "if (charge[r] > thr)"),
    "share_wrong_denominator": ("h[r] / hmax;", "h[r] / (hmax + 1.0f);"),
    "tracker_signed_max": ("float a = fabsf(orc_bf16_to_f32(Y[(size_t)t * R + r]));",
                           "float a = orc_bf16_to_f32(Y[(size_t)t * R + r]);"),
    "tracker_nan_wins": ("            if (isnan(a)) {\n                ++nonfinite;\n                continue;\n            }",
                         "            if (isnan(a)) {\n                ++nonfinite;\n                a = largest;\n            }"),
    "tracker_inf_kept": ("                a = largest;\n            }\n            if (a > m)",
                         "            }\n            if (a > m)"),
    "dw_transposed_operand": ("(double)orc_bf16_to_f32(dX[(size_t)t * R + r])",
                              "(double)orc_bf16_to_f32(dX[(size_t)r * T + t])"),
    "dw_ignores_row_mask": ("continue;                               /* inactive row of an active tile */",
                            ";"),
    "embed_keeps_inactive_tokens": ("if (r < 0 || r >= V || !((words[r / 32] >> (r % 32)) & 1))",
                                    "if (r < 0 || r >= V)"),
    "update_step_sign": ("float Wn = fmaf(-lr, u, W);", "float Wn = fmaf(lr, u, W);"),
    "update_no_bias_correction_t": ("for (int i = 0; i < t; ++i)\n        p *= (double)beta;",
                                    "for (int i = 1; i < t; ++i)\n        p *= (double)beta;"),
    "update_partner_dropped": ("float gt = fmaf(c_partner, gb, c_self * ga);",
                               "float gt = c_self * ga;"),
    "update_partner_sign": ("float gt = fmaf(c_partner, gb, c_self * ga);",
                            "float gt = fmaf(-c_partner, gb, c_self * ga);"),
    "update_v_not_squared": ("one_minus_b2 * (gt * gt)", "one_minus_b2 * fabsf(gt)"),
    "update_eps_inside_sqrt": ("/ (sqrtf(v1 * bc2) + eps)", "/ sqrtf(v1 * bc2 + eps)"),
    "update_decay_coupled_sign": ("Wn = fmaf(-lr * wd, W, Wn);", "Wn = fmaf(lr * wd, W, Wn);"),
    "update_clip_one_sided": ("ga = fminf(fmaxf(ga, -clip), clip);", "ga = fminf(ga, clip);"),
    "quant_truncates": ("float k = rintf(W[c] / sc);", "float k = truncf(W[c] / sc);"),
    "quant_scale_255": ("float sc = amax / 127.0f;", "float sc = amax / 128.0f;"),
    "quant_residual_dropped": ("delta[c] = fmaf(-sc, k, W[c]);", "delta[c] = 0.0f;"),
    "f16_round_down": ("float sig = rintf(ldexpf(a, 10 - E));",
                       "float sig = floorf(ldexpf(a, 10 - E));"),
    "bf16_round_up_ties": ("if (drop > 0x8000u || (drop == 0x8000u && (keep & 1u)))",
                           "if (drop >= 0x8000u)"),
    "moments_kept_on_deactivation": ("if (was == now)\n            continue;",
                                     "if (was == now || was)\n            continue;"),
    "restore_forgets_scale": ("        s[r] = cs[k];\n", "\n"),
    "restore_moments_to_inactive_rows": ("            if (active) {\n                m[i] = cm[j];",
                                         "            if (1) {\n                m[i] = cm[j];"),
    "restore_live_not_rebuilt": ("live[i] = orc_f32_to_bf16(fmaf(cs[k], (float)cq[j], cdelta[j]));",
                                 "(void)live;"),
    "restore_live_without_residual": ("live[i] = orc_f32_to_bf16(fmaf(cs[k], (float)cq[j], cdelta[j]));",
                                      "live[i] = orc_f32_to_bf16(cs[k] * (float)cq[j]);"),
}

PIN_TESTS = [f for name, f in inspect.getmembers(pins, inspect.isfunction)
             if name.startswith("test_")]
# cheapest first, so that most mutants die quickly
PIN_TESTS.sort(key=lambda f: ("format" in f.__name__ or "f16" in f.__name__ or "bf16" in f.__name__,
                              f.__code__.co_firstlineno))


def _build_mutant(tmp_path, name, old, new):
    src = open(ormod._SRC).read()
    assert src.count(old) >= 1, f"mutation {name} does not apply"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new, 1))
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", *ormod.CFLAGS, str(path), "-o", str(so), "-lm"])
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_kill_mutant(name, tmp_path):
    so = _build_mutant(tmp_path, name, *MUTANTS[name])
    real = ormod.lib()
    mutant = ctypes.CDLL(so)
    ormod._declare(mutant)
    ormod._lib = mutant
    killed_by = None
    try:
        for fn in PIN_TESTS:
            try:
                fn()
            except Exception:  # any failure of a pin counts as catching the mistake
                killed_by = fn.__name__
                break
    finally:
        ormod._lib = real
    assert killed_by is not None, f"no pin catches mutant {name}"
