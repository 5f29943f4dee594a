"""Planted mistakes in the CPU oracle: each case edits one oracle function's
own source text (a dropped term, a wrong sign, index or operand, an
off-by-one), swaps the edited function in for the original on the CPU, and
runs the pins of test_oracle_pins that should notice.  At least one of them
must fail.  This tests the pins, not the oracle: a plausible slip anywhere in
the oracle would have failed a pin.  The unedited oracle passes every listed
pin (the control case).

Not covered: which of two clipping candidates with exactly equal float32
error sums the mse refresh keeps (the first, in ratio order).  Such ties
between different grids do not arise on realistic inputs; the kernels follow
the same rule and the bit-exact GPU tests compare them on real sums.
"""
import inspect
import textwrap

import pytest

import test_oracle_pins as pins
from oracle import admmq_oracle as O
from oracle import projection_fp32 as P

# the edited code may overflow or divide by zero on the way to a failed pin
pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _edited(mod, name, old, new):
    """The function `name` of `mod` compiled from its source with `old`
    replaced by `new` (exactly one occurrence), in a copy of the module's
    namespace so that it calls the module's other functions."""
    src = textwrap.dedent(inspect.getsource(getattr(mod, name)))
    assert src.count(old) == 1, (name, old, src.count(old))
    ns = dict(vars(mod))
    exec(compile(src.replace(old, new), f"<planted mistake in {name}>", "exec"), ns)
    return ns[name]


# pin shorthands: (pin function, its arguments)
GRAM = (pins.test_gram_and_damping, ())
OBJ = (pins.test_objective_equals_output_error, ())
SCALING = (pins.test_scaling_unit_diagonal_and_invariance, ())
WUPD = (pins.test_w_update_matches_linear_solve, ())
COLLINEAR = (pins.test_collinear_example_gptq_and_admm, ())
BEATS = (pins.test_admm_beats_rtn_and_gptq_with_lsq_refresh, ())
CONVERGE = tuple((pins.test_admm_converges_to_common_limit, (g,)) for g in ("minmax", "lsq", "frozen"))
DIAG_RTN = (pins.test_diagonal_hessian_frozen_grid_gives_rtn, ())
BRUTE = (pins.test_tiny_layers_against_brute_force, (0,))
WORKED = (pins.test_worked_example_compensation_values, ())
WORKED_GPTQ = (pins.test_worked_example_through_gptq_algorithm, ())
GPTQ_FIRST = (pins.test_gptq_first_step_is_closed_form_compensation, ())
GPTQ_BLOCK = (pins.test_gptq_block_size_invariance, (0,))
BABAI = (pins.test_back_to_front_gptq_equals_babai, (0,))
BOUND = (pins.test_babai_error_bound_theorem5, (0,))
MINMAX_HAND = (pins.test_minmax_grid_hand_example, ())
MINMAX_ZERO = (pins.test_minmax_grid_all_zero_group, ())
MINMAX_SIGNED = (pins.test_minmax_grid_one_signed_groups, ())
NEAREST = (pins.test_projection_is_nearest_grid_point, (3,))
MSE_HAND = (pins.test_mse_clip_hand_example, ())
MSE_EXACT = (pins.test_mse_clip_exact_grid_keeps_minmax, ())
MSE_F64 = (pins.test_mse_clip_search_against_float64, (3,))
LSQ_EXACT = (pins.test_lsq_refit_recovers_exact_grid, ())
LSQ_DOWN = (pins.test_lsq_refit_does_not_increase_weighted_error, ())
LSQ_STAGES = (pins.test_lsq_refit_stages_against_lstsq, ())
LSQ_MIN = (pins.test_lsq_refit_scale_is_a_weighted_minimum, ())
TF32 = (pins.test_tf32_split_reconstructs_float32, ())
F16 = (pins.test_f16_split_encoding, ())
F16_ROWS = (pins.test_f16_row_scales, ())
MIXED = (pins.test_mixed_split_encoding, ())
EPI = tuple((pins.test_epilogue_step_follows_the_d_and_dual_updates, (mode, 3, 32, 5, 96))
            for mode in ("minmax", "lsq", "frozen"))
INIT = (pins.test_init_step_is_rtn_in_memory_layout, (3, 32, 6, 96))
PACK = (pins.test_pack_hand_examples, ())
RESCALE = (pins.test_dual_rescaling_keeps_the_unscaled_dual, ())
RESCALE_F32 = (pins.test_epilogue_step_dual_scale, ())
FIT_W = tuple((pins.test_grid_fitted_on_w, (mode,)) for mode in ("minmax", "lsq", "mse"))
PACK_BIG = (pins.test_pack_matches_big_integer_route, (3,))

# name: (module, function, old text, new text, pins that should notice)
MISTAKES = {
    # Hessian, damping, scaling, objective
    "gram_drops_last_chunk": (O, "gram", "range(0, X.shape[0], chunk)",
                              "range(0, X.shape[0] - chunk, chunk)", [GRAM]),
    "damping_mean_of_all_entries": (O, "damping", "np.mean(np.diag(G))", "np.mean(G)", [GRAM]),
    "damping_added_everywhere": (O, "damping", "G + lam * np.eye(G.shape[0])", "G + lam", [GRAM, OBJ]),
    "scaling_wrong_power": (O, "diagonal_scaling", "1.0 / np.sqrt(np.diag(H))", "np.sqrt(np.diag(H))",
                            [SCALING]),
    "scaling_one_sided": (O, "diagonal_scaling", "sigma[:, None] * H * sigma[None, :]",
                          "sigma[:, None] * H", [SCALING]),
    "objective_without_half": (O, "objective", "return 0.5 * float(", "return float(", [OBJ]),
    "objective_sum_not_difference": (O, "objective", "np.asarray(W, dtype=np.float64) - np.asarray",
                                     "np.asarray(W, dtype=np.float64) + np.asarray", [OBJ]),
    # grids in the [d_in][d_out] layout
    "groups_along_output_axis": (O, "_groups", "np.ascontiguousarray(A.T)", "np.ascontiguousarray(A)",
                                 [INIT] + list(EPI)),
    "frozen_grid_refitted": (O, "project", "s, z = sp, zp", "s, z = p32.fit_minmax(yg, L)",
                             list(EPI) + [DIAG_RTN]),
    # W-update and the ADMM loop
    "w_update_dual_sign": (O, "w_update", "rho * (Dt - Vt)", "rho * (Dt + Vt)", [WUPD]),
    "w_update_transposed_basis": (O, "w_update", "Q @ ((Q.T @", "Q.T @ ((Q @", [WUPD]),
    "w_update_no_rho_in_denominator": (O, "w_update", "/ (lam + rho)[:, None]", "/ lam[:, None]",
                                       [WUPD]),
    "admm_dual_sign": (O, "admm_q", "Vt = Vt + Wt - Dt_new", "Vt = Vt - Wt + Dt_new",
                       list(CONVERGE) + [BEATS, COLLINEAR]),
    "admm_projects_without_dual": (O, "admm_q", "Y = sigma[:, None] * (Wt + Vt)",
                                   "Y = sigma[:, None] * Wt", list(CONVERGE) + [BEATS, COLLINEAR]),
    "admm_scales_target_wrong_way": (O, "admm_q", "Wt_hat = W_hat / sigma[:, None]",
                                     "Wt_hat = W_hat * sigma[:, None]", [BEATS, COLLINEAR, DIAG_RTN]),
    "admm_unscales_d_wrong_way": (O, "admm_q", "Dt_new = D / sigma[:, None]", "Dt_new = D * sigma[:, None]",
                                  list(CONVERGE) + [BEATS, COLLINEAR]),
    "admm_drops_hessian_in_target": (O, "admm_q", "B = Ht @ Wt_hat", "B = Wt_hat",
                                     [BEATS, COLLINEAR, DIAG_RTN]),
    # GPTQ and Babai
    "compensation_sign": (O, "compensation", "return d * Hinv", "return -d * Hinv", [WORKED, GPTQ_FIRST]),
    "gptq_error_sign": (O, "gptq", "(Wp[:, j] - Qp[:, j]) / R[j, j]", "(Qp[:, j] - Wp[:, j]) / R[j, j]",
                        [WORKED_GPTQ, GPTQ_FIRST, COLLINEAR]),
    "gptq_drops_block_update": (O, "gptq", "Wp[:, b:] -= E @ R[a:b, b:]", "pass", [GPTQ_BLOCK]),
    "gptq_transposed_factor_row": (O, "gptq", "R[j, j:b])", "R[j:b, j])", [WORKED_GPTQ, GPTQ_BLOCK, BABAI]),
    "babai_front_to_back": (O, "babai_nearest_plane", "range(d - 1, -1, -1)", "range(d)", [BABAI]),
    "babai_row_not_column": (O, "babai_nearest_plane", "s[k] * R[:, k]", "s[k] * R[k, :]", [BABAI, BOUND]),
    "babai_bound_constant": (O, "babai_error_bound", "0.25 *", "0.025 *", [BOUND]),
    "pack_reversed_bits": (O, "pack", "pos = k * bits + b\n", "pos = k * bits + (bits - 1 - b)\n",
                           [PACK, PACK_BIG]),
    # float32 grid fit and rounding
    "zero_point_sign": (P, "_range_grid", "np.rint(_f(np.negative(mn) / s_safe))",
                        "np.rint(_f(mn / s_safe))", [MINMAX_HAND, NEAREST]),
    "scale_divides_by_levels": (P, "_range_grid", "/ f32(L))", "/ f32(L + 1))", [MINMAX_HAND]),
    "all_zero_group_divides_by_zero": (P, "_range_grid", "s_safe = np.where(zero_range, f32(1), s).astype(f32)",
                                       "s_safe = s", [MINMAX_ZERO]),
    "brute_force_drops_hessian": (O, "brute_force_column", "v = 0.5 * np.sum((e @ H) * e, axis=1)",
                                  "v = 0.5 * np.sum(e * e, axis=1)", [BRUTE]),
    "range_without_zero": (P, "_group_range", "np.minimum(yg.min(axis=1), f32(0))", "yg.min(axis=1)",
                           [MINMAX_HAND, MINMAX_SIGNED, NEAREST]),
    "clamp_one_level_short": (P, "round_to_grid", "f32(0), f32(L))", "f32(0), f32(L - 1))",
                              [MINMAX_HAND, NEAREST]),
    "floor_not_nearest": (P, "round_to_grid", "np.rint(", "np.floor(", [MINMAX_HAND, NEAREST]),
    "dequantize_adds_zero": (P, "dequantize", "_f(q) - _f(z)", "_f(q) + _f(z)", [MINMAX_HAND, NEAREST]),
    "mse_absolute_error": (P, "fit_mse", "d2 = _f(d * d)", "d2 = _f(np.abs(d))",
                           [MSE_HAND, MSE_EXACT, MSE_F64]),
    "mse_no_clipping": (P, "fit_mse", "_range_grid(_f(a * mn), _f(a * mx), L)", "_range_grid(mn, mx, L)",
                        [MSE_HAND, MSE_F64]),
    "lsq_cross_sum_drops_code": (P, "fit_lsq", "Sqy = _f(Sqy + _f(wq * yi))", "Sqy = _f(Sqy + _f(w * yi))",
                                 [LSQ_EXACT, LSQ_DOWN]),
    "lsq_variance_uses_mean_y": (P, "fit_lsq", "var = _f(Sqq - _f(Sq * qm))", "var = _f(Sqq - _f(Sq * ym))",
                                 [LSQ_EXACT, LSQ_DOWN]),
    "lsq_zero_point_sign": (P, "fit_lsq", "_f(qm - _f(ym /", "_f(qm + _f(ym /",
                            [LSQ_EXACT, LSQ_DOWN, LSQ_STAGES]),
    "lsq_second_fit_drops_factor_2": (P, "fit_lsq", "_f(f32(2) * zc)", "zc", [LSQ_STAGES, LSQ_MIN]),
    "lsq_second_fit_wrong_cross_term": (P, "fit_lsq", "num = _f(Sqy - _f(zc * Sy))",
                                        "num = _f(Sqy - _f(zc * Sq))", [LSQ_STAGES, LSQ_MIN]),
    "lsq_zero_point_floor": (P, "fit_lsq", "np.clip(np.rint(_f(qm", "np.clip(np.floor(_f(qm",
                             [LSQ_STAGES]),
    "lsq_keeps_first_slope": (P, "fit_lsq", "s = np.where(ok, s2, s0)", "s = np.where(ok, s1, s0)",
                              [LSQ_STAGES, LSQ_MIN]),
    "lsq_unweighted_mean": (P, "fit_lsq", "Sw = _f(Sw + w)", "Sw = _f(Sw + f32(1))", [LSQ_STAGES]),
    # operand encodings
    "tf32_truncates": (P, "tf32_round", "((b + 0xFFF + lsb) >> 13) << 13", "(b >> 13) << 13", [TF32]),
    "f16_low_part_unscaled": (P, "split_f16", "_f(xs - hi.astype(np.float32))",
                              "_f(x - hi.astype(np.float32))", [F16]),
    "f16_row_scale_octave_low": (P, "row_scales_f16", "np.clip(10 - k, -60, 60)", "np.clip(9 - k, -60, 60)",
                                 [F16_ROWS]),
    "mixed_halves_swapped": (P, "split_mix", '(hb, lb) if side == "A" else (lb, hb)',
                             '(lb, hb) if side == "A" else (hb, lb)', [MIXED]),
    # the fused step in memory layout
    "epilogue_dual_sign": (P, "epilogue_step", "V_new = _f(t - Dt)", "V_new = _f(t + Dt)", list(EPI)),
    "epilogue_unscales_with_sigma": (P, "epilogue_step", "Dt = _f(D * _f(rsig)[None, :])",
                                     "Dt = _f(D * _f(sigma)[None, :])", list(EPI)),
    "epilogue_p_sign": (P, "epilogue_step", "P = _f(Dt - V_new)", "P = _f(V_new - Dt)", list(EPI)),
    "epilogue_projects_without_dual": (P, "epilogue_step", "y = _f(_f(sigma)[None, :] * t)",
                                       "y = _f(_f(sigma)[None, :] * W_acc)", list(EPI)),
    "epilogue_residual_against_v": (P, "epilogue_step", "np.sum((W_acc.astype(np.float64) - Dt) ** 2)",
                                    "np.sum((V.astype(np.float64) - Dt) ** 2)", list(EPI)),
    "rescale_factor_inverted": (O, "admm_q", "Vt = Vt * (rho / (rho0 * gamma ** (t + 1)))",
                                "Vt = Vt * ((rho0 * gamma ** (t + 1)) / rho)", [RESCALE]),
    "epilogue_rescales_p_not_v": (P, "epilogue_step", "V_new = _f(V_new * f32(dual_scale))",
                                  "V_new = V_new", [RESCALE_F32]),
    "fit_target_ignored": (O, "project", "fg = yg if Y_fit is None else", "fg = yg if True else",
                           list(FIT_W)),
    "epilogue_fits_with_dual": (P, "epilogue_step", "_f(_f(sigma)[None, :] * W_acc), group) if fit_on_w",
                                "_f(_f(sigma)[None, :] * t), group) if fit_on_w", list(FIT_W)),
    "init_forgets_scaling": (P, "init_step", "Dt = _f(D * _f(rsig)[None, :])", "Dt = _f(D)", [INIT]),
    "rows_grouped_by_column": (P, "_rows_to_groups", "A.reshape(m * (d // g), g)",
                               "np.ascontiguousarray(A.T).reshape(m * (d // g), g)", list(EPI) + [INIT]),
}


def _failures(targets):
    failed = []
    for fn, args in targets:
        try:
            fn(*args)
        except Exception as e:  # an assertion, or the edited code crashing
            failed.append(f"{fn.__name__}{args}: {type(e).__name__}")
    return failed


def test_control_unedited_oracle_passes_every_listed_pin():
    targets = {(fn, args) for *_, t in MISTAKES.values() for fn, args in t}
    assert _failures(sorted(targets, key=lambda x: (x[0].__name__, x[1]))) == []


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_pins_catch_planted_mistake(name, monkeypatch):
    mod, fn, old, new, targets = MISTAKES[name]
    monkeypatch.setattr(mod, fn, _edited(mod, fn, old, new))
    assert _failures(targets), f"no pin noticed {name}"
