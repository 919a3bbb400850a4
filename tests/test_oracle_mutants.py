"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a temporary copy of
oracle/ia_oracle.c: a dropped conjugate, a missing or misplaced b, a wrong
decay or sign, a transposed index, an off-by-one in the causal order or the
mode frequencies, a wrong derivative. It builds the copy with the oracle's
own flags and runs every pin of test_oracle_pins.py against it. Each mutant
must fail at least one pin. An unmutated copy, built and run the same way,
must pass them all, so a failure comes from the planted mistake and not from
the harness. The mutants live only in pytest's temporary directory; the
oracle's source and library are never modified.
"""
import os
import shutil

import pytest

import test_oracle_pins as P

ORACLE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")

# (name, exact source text, replacement): every occurrence in ia_oracle.c is replaced
MUTANTS = [
    # forward recurrence and readout
    ("readout without conjugate",
     "nf += creal(conj(a[m]) * G[(long)m * d_v + f]);",
     "nf += creal(a[m] * G[(long)m * d_v + f]);"),
    ("readout reads Gamma transposed",
     "nf += creal(conj(a[m]) * G[(long)m * d_v + f]);",
     "nf += creal(conj(a[m]) * G[(long)f * M + m]);"),
    ("key drive without b",
     "Um[f] = lam[m] * Um[f] + bb[m] * fkt[f];",
     "Um[f] = lam[m] * Um[f] + fkt[f];"),
    ("query reads the state before the update",
     "        Um[f] = lam[m] * Um[f] + bb[m] * fkt[f];\n        am += Um[f] * fqt[f];",
     "        am += Um[f] * fqt[f];\n        Um[f] = lam[m] * Um[f] + bb[m] * fkt[f];"),
    ("value state decays with conj(lambda)",
     "Gm[f] = lam[m] * Gm[f] + bb[m] * vt[f];",
     "Gm[f] = conj(lam[m]) * Gm[f] + bb[m] * vt[f];"),
    ("eta driven by 1 instead of b",
     "eta[m] = lam[m] * eta[m] + bb[m];",
     "eta[m] = lam[m] * eta[m] + 1.0;"),
    # parameters and feature map (shared with the C brute force)
    ("feature map without the +1",
     "return x > 0.0 ? x + 1.0 : exp(x); }",
     "return x > 0.0 ? x : exp(x); }"),
    ("zero-order hold without 1/A",
     "*bm = (*l - 1.0) / a;",
     "*bm = *l - 1.0;"),
    ("decay exp(-Delta A)",
     "*l = cexp(delta * a);",
     "*l = cexp(-delta * a);"),
    ("S4D-Lin frequencies shifted by one",
     "return -0.5 + I * (kPi * (double)m);",
     "return -0.5 + I * (kPi * (double)(m + 1));"),
    # reverse mode
    ("xi' copied from xi",
     "return x > 0.0 ? 1.0 : exp(x); }",
     "return x > 0.0 ? x + 1.0 : exp(x); }"),
    ("adjoint carried back with lambda instead of conj(lambda)",
     "cd cl = conj(lam[m]);",
     "cd cl = lam[m];"),
    ("dDelta without the b term",
     "part[bh * M + m] = creal(conj(glam[m]) * Am[m] * lam[m] + conj(gb_[m]) * lam[m]);",
     "part[bh * M + m] = creal(conj(glam[m]) * Am[m] * lam[m]);"),
    # trainable A and per-(head, mode) Delta
    ("per-mode Delta read from the head's first mode",
     "return dpm ? delta[(long)h * M + m] : delta[h];",
     "return dpm ? delta[(long)h * M] : delta[h];"),
    ("dA without the b term",
     "partA[bh * M + m] = conj(dl * lam[m]) * glam[m] + conj((dl * lam[m] - bb[m]) / Am[m]) * gb_[m];",
     "partA[bh * M + m] = conj(dl * lam[m]) * glam[m];"),
    ("dA with dlambda/dA taken as A lambda",
     "partA[bh * M + m] = conj(dl * lam[m]) * glam[m] + conj((dl * lam[m] - bb[m]) / Am[m]) * gb_[m];",
     "partA[bh * M + m] = conj(Am[m] * lam[m]) * glam[m] + conj((dl * lam[m] - bb[m]) / Am[m]) * gb_[m];"),
    ("db/dA without the -b term",
     "partA[bh * M + m] = conj(dl * lam[m]) * glam[m] + conj((dl * lam[m] - bb[m]) / Am[m]) * gb_[m];",
     "partA[bh * M + m] = conj(dl * lam[m]) * glam[m] + conj(dl * lam[m] / Am[m]) * gb_[m];"),
    # optional parts of the layer
    ("RMSNorm without the square root",
     "double r = 1.0 / sqrt(ss / (double)D + eps);",
     "double r = 1.0 / (ss / (double)D + eps);"),
    ("RMSNorm bias added before the gain",
     "z[f] = z[f] * r * g + c;",
     "z[f] = (z[f] * r + c) * g;"),
    ("per-token step read from the previous token",
     "for (int m = 0; m < M; ++m) zoh(delta_t[bh * N + t], Am[m], &lam[m], &bb[m]);",
     "for (int m = 0; m < M; ++m) zoh(delta_t[bh * N + (t > 0 ? t - 1 : 0)], Am[m], &lam[m], &bb[m]);"),
    ("readout matrix applied transposed",
     "acc += ld_c(W + 2 * (((long)h * M + m) * M + mp)) * a[mp];",
     "acc += ld_c(W + 2 * (((long)h * M + mp) * M + m)) * a[mp];"),
    ("readout matrix conjugated",
     "acc += ld_c(W + 2 * (((long)h * M + m) * M + mp)) * a[mp];",
     "acc += conj(ld_c(W + 2 * (((long)h * M + m) * M + mp))) * a[mp];"),
    ("per-mode dDelta summed into the head's first mode",
     "dDelta[dpm ? (bh % H) * M + m : bh % H] += part[bh * M + m];",
     "dDelta[dpm ? (bh % H) * M : bh % H] += part[bh * M + m];"),
    ("dk without conj(b)",
     "s += creal(conj(bb[m]) * G[m * d_xi + f]);",
     "s += creal(bb[m] * G[m * d_xi + f]);"),
    ("dden with the wrong sign",
     "dden -= dOt[f] * ot[f];",
     "dden += dOt[f] * ot[f];"),
    ("lambda adjoint paired with S_t instead of S_(t-1)",
     "const cd* Sp = blk + (size_t)(t - t0) * SL;",
     "const cd* Sp = blk + (size_t)(t - t0 + 1) * SL;"),
    ("local U adjoint with xi(k) instead of xi(q)",
     "G[m * d_xi + f] += ga[m] * fqt[f];",
     "G[m * d_xi + f] += ga[m] * fkt[f];"),
]

PINS = [
    ("p1 brute force", P.test_p1_brute_force_matches_recurrence, {}),
    ("p2 eta closed form", P.test_p2_eta_closed_form, {}),
    ("p2 zoh quadrature", P.test_p2_params_zoh, {}),
    ("p3 first token", P.test_p3_first_token_returns_v1, {}),
    ("p4 affine values", P.test_p4_constant_and_affine_values, {}),
    ("p5 feature scaling", P.test_p5_feature_scaling_leaves_o, {}),
    ("p6 mode additivity", P.test_p6_mode_additivity, {}),
    ("p10 ema", P.test_p10_single_real_mode_is_normalised_ema, {}),
    ("p11 cumulative mean", P.test_p11_small_step_limit_is_cumulative_mean, {}),
    ("p12 prefill then decode", P.test_p12_prefill_then_decode_equals_longer_prefill, {}),
    ("p13 split prefill", P.test_p13_split_prefill_equals_single_prefill, {}),
    ("golden ema", P.test_golden_hand_derived, {"name": "m1_real_ema.json"}),
    ("golden rotating", P.test_golden_hand_derived, {"name": "m1_rotating_mode.json"}),
    ("p8 finite differences", P.test_p8_finite_differences, {}),
    ("p9 tangent/adjoint", P.test_p9_tangent_adjoint_dot_product, {}),
    ("dDelta batch sum", P.test_backward_batch_sum_of_ddelta, {}),
    ("p1 mpmath", P.test_p1_mpmath_brute_force, {}),
    ("p1 per-mode Delta brute force", P.test_p1_per_mode_delta_brute_force, {}),
    ("p1 per-mode Delta mpmath", P.test_p1_per_mode_delta_mpmath, {}),
    ("p8 modes and A", P.test_p8_finite_differences_per_mode_delta_and_A, {}),
    ("p9 modes and A", P.test_p9_dot_product_per_mode_delta_and_A, {}),
    ("ex all off", P.test_extended_forward_with_everything_off_is_the_layer, {}),
    ("selective mpmath", P.test_selective_steps_mpmath, {}),
    ("selective constant", P.test_selective_constant_steps_reduce_to_per_head_delta, {}),
    ("selective skip", P.test_selective_zero_step_skips_the_token, {}),
    ("readout mpmath", P.test_readout_matrix_mpmath_and_identity, {}),
    ("readout linear", P.test_readout_matrix_linear_and_scale_free, {}),
    ("norm bias", P.test_input_norm_bias_alone_gives_the_bias, {}),
    ("norm scale", P.test_input_norm_is_scale_free, {}),
    ("bidirectional", P.test_bidirectional_time_reversal_and_first_token, {}),
]


def _failing_pins(oracle_mod, stop_at_first):
    failed = []
    for name, fn, kw in PINS:
        try:
            fn(oracle_mod, **kw)
        except (AssertionError, FloatingPointError, ValueError, RuntimeError, ZeroDivisionError,
                OverflowError):
            failed.append(name)
            if stop_at_first:
                break
    return failed


def _with_library(oracle_mod, monkeypatch, tmp_path, tag, edit):
    """Build a copy of the oracle source (edited by `edit`) and point the oracle module at it."""
    src_dir = tmp_path / tag
    src_dir.mkdir()
    shutil.copy(os.path.join(ORACLE_DIR, "ia_oracle.h"), src_dir / "ia_oracle.h")
    text = open(os.path.join(ORACLE_DIR, "ia_oracle.c")).read()
    (src_dir / "ia_oracle.c").write_text(edit(text))
    lib = oracle_mod.compile_source(str(src_dir / "ia_oracle.c"), str(src_dir / ("libia_oracle_%s.so" % tag)))
    monkeypatch.setattr(oracle_mod, "build", lambda force=False: lib)
    monkeypatch.setattr(oracle_mod, "_LIB", lib)
    monkeypatch.setattr(oracle_mod, "_lib", None)


def test_unmutated_copy_passes_every_pin(oracle_mod, monkeypatch, tmp_path):
    _with_library(oracle_mod, monkeypatch, tmp_path, "control", lambda t: t)
    assert _failing_pins(oracle_mod, stop_at_first=False) == []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_every_planted_mistake_fails_a_pin(oracle_mod, monkeypatch, tmp_path, name, old, new):
    def edit(text):
        # a slip in a formula that the plain and the extended forward both
        # spell out is planted in both (a slip in only one of them is caught
        # by the pin that compares the two with the options off)
        assert text.count(old) >= 1, "mutation site missing: " + old
        return text.replace(old, new)
    _with_library(oracle_mod, monkeypatch, tmp_path, "mutant", edit)
    assert _failing_pins(oracle_mod, stop_at_first=True), "no pin catches: " + name
