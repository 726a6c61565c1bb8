"""The oracle's pins have teeth: each test plants one plausible mistake in
an oracle function (a dropped term, a wrong sign, coefficient or index, a
stale operand, a missing step) on the CPU, and checks that at least one of
the pins written for that function now fails.

A mutant is the oracle function's own source with one edit, compiled in a
copy of its module's namespace and patched in for the duration of the test;
the pins look the function up on the module at call time, so they see it.
Every edit must match the source exactly once, so a change to the oracle
that removes the edited text fails here loudly instead of passing."""
import inspect
import textwrap

import pytest

from oracle import apply, dion, dion3, momentum, ns
from tests import test_oracle_dion as tdion
from tests import test_oracle_dion3 as td3
from tests import test_oracle_ns as tns


def _mutant(module, fname, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(module, fname)))
    assert src.count(old) == 1, f"{module.__name__}.{fname}: edit must match once: {old!r}"
    env = dict(vars(module))
    exec(compile(src.replace(old, new), f"<mutant of {module.__name__}.{fname}>", "exec"), env)
    return env[fname]


# pins (the existing oracle tests, called with fixed arguments)
CLOSED_FORM = lambda: tns.test_closed_form_through_svd((32, 80), 1.0)  # noqa: E731
CLOSED_FORM_SAFETY = lambda: tns.test_closed_form_through_svd((32, 80), 1.01)  # noqa: E731
CLOSED_FORM_TALL = lambda: tns.test_closed_form_through_svd((80, 32), 1.0)  # noqa: E731
GRAM_EQ = lambda: tns.test_gram_equals_standard_fp64((64, 256), (), 1.0)  # noqa: E731
GRAM_EQ_RESTART = lambda: tns.test_gram_equals_standard_fp64((64, 256), (3,), 1.0)  # noqa: E731
SAFETY = tns.test_safety_factor_is_input_rescaling
NORMALIZATION = tns.test_normalization_and_scale_invariance
SINGLE_ROW = tns.test_zero_iterations_and_single_row
EQUIVARIANCE = tns.test_permutation_and_transpose_equivariance
BRUTE_TOPK = lambda: td3.test_select_rows_brute_force(64, 0.125)  # noqa: E731
TIES = td3.test_select_rows_exact_ties
NUM_SELECTED = td3.test_num_selected_edges
GATHER = td3.test_gather_normalize_unit_frobenius
EF3 = td3.test_error_feedback_conservation
EMA = td3.test_ema_closed_form_three_steps
KEYS = td3.test_accum_and_row_keys
APPLY = td3.test_apply_update_weight_decay
QR = lambda: tdion.test_householder_qr((300, 40))  # noqa: E731
COLNORM = tdion.test_colnorm_unit_columns
EF_DION = lambda: tdion.test_error_feedback_conservation(dion.COLNORM)  # noqa: E731
EF_ORTH = lambda: tdion.test_error_feedback_conservation(dion.QR)  # noqa: E731
NU_T = tdion.test_nu_t_bounds
BETA = tdion.test_beta_reading_reduces_to_dion_at_one
ERANK = tdion.test_effective_rank_closed_forms

MUTANTS = [
    # Newton-Schulz and Gram Newton-Schulz
    ("ns_drops_square_term", ns, "newton_schulz",
     "        B = b * A + c * (A @ A)\n", "        B = b * A\n", [CLOSED_FORM]),
    ("ns_sign_of_update", ns, "newton_schulz",
     "        X = a * X + B @ X", "        X = a * X - B @ X", [CLOSED_FORM]),
    ("ns_no_transpose_back", ns, "newton_schulz",
     "    return X.T if transposed else X", "    return X", [CLOSED_FORM_TALL, EQUIVARIANCE]),
    ("gram_single_h_on_a", ns, "gram_newton_schulz",
     "            A = H @ (H @ A)", "            A = H @ A", [GRAM_EQ, CLOSED_FORM]),
    ("gram_h_linear_in_a", ns, "gram_newton_schulz",
     "        H = a * eye + b * A + c * (A @ A)", "        H = a * eye + b * A + c * A",
     [GRAM_EQ, CLOSED_FORM]),
    ("gram_restart_keeps_q", ns, "gram_newton_schulz",
     "            A = X0 @ X0.T\n            Q = _identity_like(k, A)\n",
     "            A = X0 @ X0.T\n", [GRAM_EQ_RESTART]),
    ("gram_restart_keeps_a", ns, "gram_newton_schulz",
     "            X0 = Q @ X0\n            A = X0 @ X0.T\n", "            X0 = Q @ X0\n",
     [GRAM_EQ_RESTART]),
    ("gram_output_without_q", ns, "gram_newton_schulz",
     "    out = Q @ X0", "    out = X0", [GRAM_EQ, CLOSED_FORM]),
    ("safety_wrong_power", ns, "scaled_coeffs",
     "c / (s * s * s * s * s)", "c / (s * s * s)", [CLOSED_FORM_SAFETY, SAFETY]),
    ("norm_is_max_abs", ns, "frobenius_normalize",
     "    fro = float(np.sqrt(np.sum(X * X)))", "    fro = float(np.max(np.abs(X)))",
     [NORMALIZATION, CLOSED_FORM]),
    ("norm_drops_eps", ns, "frobenius_normalize",
     "    factor = 1.0 / (fro + eps)", "    factor = 1.0 / fro", [SINGLE_ROW, CLOSED_FORM]),
    # momentum, Dion3 selection, error feedback, weight update
    ("ema_damps_gradient", momentum, "momentum_update",
     "new = mu64 * M64 + G64", "new = mu64 * M64 + (1.0 - mu64) * G64", [EMA]),
    ("keys_are_l1", momentum, "row_sqnorms",
     'return np.einsum("ij,ij->i", B64, B64)', "return np.sum(np.abs(B64), axis=1)", [KEYS]),
    ("select_smallest", dion3, "select_rows",
     "np.lexsort((np.arange(m), -keys))", "np.lexsort((np.arange(m), keys))", [BRUTE_TOPK]),
    ("ties_to_higher_index", dion3, "select_rows",
     "np.lexsort((np.arange(m), -keys))", "np.lexsort((-np.arange(m), -keys))", [TIES]),
    ("k_rounds_down", dion3, "num_selected",
     "math.ceil(float(rho) * m - 1e-9)", "math.floor(float(rho) * m + 1e-9)", [NUM_SELECTED]),
    ("norm_over_all_rows", dion3, "gather_normalize",
     "np.asarray(keys, dtype=np.float64)[idx]", "np.asarray(keys, dtype=np.float64)", [GATHER]),
    ("ef_leaves_wrong_share", dion3, "ef_write",
     "out[idx] = float(np.float32(mu)) * out[idx]",
     "out[idx] = (1.0 - float(np.float32(mu))) * out[idx]", [EF3]),
    ("update_sign", apply, "apply_update",
     "W64[idx] = decay * W64[idx] - lr * scale * O64",
     "W64[idx] = decay * W64[idx] + lr * scale * O64", [APPLY]),
    ("no_weight_decay", apply, "apply_update",
     "    decay = 1.0 - lr * wd", "    decay = 1.0", [APPLY]),
    # Householder QR, ColNorm and the Dion / Orth-Dion step
    ("qr_without_sign_fix", dion, "householder_qr",
     "    signs = np.where(np.diag(R) < 0, -1.0, 1.0)", "    signs = np.ones(r)", [QR]),
    ("colnorm_squared_norm", dion, "colnorm",
     "    return R / (norms + eps)[None, :]", "    return R / (norms * norms + eps)[None, :]",
     [COLNORM]),
    ("p_not_orthonormalized", dion, "dion_step",
     "    P = orth(B @ np.asarray(Q_prev, dtype=np.float64))",
     "    P = B @ np.asarray(Q_prev, dtype=np.float64)", [EF_DION]),
    ("r_from_unorthonormalized_p", dion, "dion_step",
     "    R = B.T @ P\n", "    R = B.T @ (B @ np.asarray(Q_prev, dtype=np.float64))\n",
     [EF_DION]),
    ("ef_coefficient_mu", dion, "dion_step",
     "    M_new = beta * B - (beta - mu) * (P @ R.T)", "    M_new = beta * B - mu * (P @ R.T)",
     [EF_DION]),
    ("beta_not_on_b", dion, "dion_step",
     "    M_new = beta * B - (beta - mu) * (P @ R.T)", "    M_new = B - (beta - mu) * (P @ R.T)",
     [BETA]),
    ("update_with_stale_q", dion, "dion_step",
     "    O = P @ Q_new.T", "    O = P @ np.asarray(Q_prev, dtype=np.float64).T", [EF_ORTH]),
    ("orth_dion_uses_colnorm", dion, "dion_step",
     "        Q_new = orth(R)", "        Q_new = colnorm(R, eps)", [NU_T]),
    ("erank_of_sigma_not_energy", dion, "effective_rank",
     "    s2 = np.asarray(sigma, dtype=np.float64) ** 2",
     "    s2 = np.asarray(sigma, dtype=np.float64)", [ERANK]),
]


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # mutants may overflow
@pytest.mark.parametrize("name,module,fname,old,new,pins", MUTANTS,
                         ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(name, module, fname, old, new, pins, monkeypatch):
    for pin in pins:  # the pins hold for the oracle as it is
        pin()
    monkeypatch.setattr(module, fname, _mutant(module, fname, old, new))
    failed = []
    for pin in pins:
        try:
            pin()
        except Exception as exc:  # an assertion, or a shape error of the mutant
            failed.append(type(exc).__name__)
    assert failed, f"no pin catches the planted mistake {name}"
