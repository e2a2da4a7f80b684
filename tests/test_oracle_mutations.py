"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the
pins in test_oracle_pins.py catch every one of them.

Each mutation edits one spot of wkv_oracle.c (a dropped term, a wrong sign, a
wrong index, a missing factor), compiles the copy with gcc, and runs the pins
that should notice.  The unmodified source must pass the same pins.
"""
import pytest

import oracle
from tests import test_oracle_pins as pins

# (id, original text, replacement, occurrence, pins that must fail on the mutant)
MUTATIONS = [
    ("fwd_drop_bonus", "if (bonus) m += u[h * N + i] * kt[i] * vt[j];", "if (bonus) m += 0.0 * u[h * N + i];", 0,
     [pins.test_golden_wkv6_forward, lambda o: pins.test_wkv6_single_token_closed_form(o)]),
    ("fwd_wrong_decay", "for (int j = 0; j < N; ++j) S[i * N + j] = d * S[i * N + j] + kt[i] * vt[j];",
     "for (int j = 0; j < N; ++j) S[i * N + j] = d * d * S[i * N + j] + kt[i] * vt[j];", 0,
     [pins.test_golden_wkv6_forward, lambda o: pins.test_wkv6_recurrence_matches_pair_sums(o, 1, 7, 1, 64, False)]),
    ("fwd_transposed_readout", "for (int i = 0; i < N; ++i) acc += rt[i] * M[i * N + j];",
     "for (int i = 0; i < N; ++i) acc += rt[i] * M[j * N + i];", 0,
     [pins.test_golden_wkv6_forward, lambda o: pins.test_wkv6_recurrence_matches_pair_sums(o, 2, 7, 2, 4, False)]),
    ("bidir_bonus_twice", "wkv6_head_sweep(T, C, N, b, h, 1, 0,", "wkv6_head_sweep(T, C, N, b, h, 1, 1,", 0,
     [pins.test_golden_wkv6_forward, pins.test_wkv6_bidir_is_causal_plus_anticausal_minus_bonus]),
    ("bidir_missing_reverse", "wkv6_head_sweep(T, C, N, b, h, 1, 0,", "wkv6_head_sweep(T, C, N, b, h, 0, 0,", 0,
     [pins.test_wkv6_bidir_reversal_symmetry]),
    ("bwd_dw_missing_decay_factor", "dwt[i] += exp(wt[i]) * accw;", "dwt[i] += accw;", 0,
     [lambda o: pins.test_wkv6_backward_finite_differences(o, False)]),
    ("bwd_adjoint_without_decay", "A[i * N + j] = rt[i] * gt[j] + d * A[i * N + j];",
     "A[i * N + j] = rt[i] * gt[j] + A[i * N + j];", 0,
     [lambda o: pins.test_wkv6_backward_finite_differences(o, False)]),
    ("bwd_anticausal_adjoint_sign", "A[i * N + j] = rt[i] * gt[j] + d * A[i * N + j];",
     "A[i * N + j] = rt[i] * gt[j] - d * A[i * N + j];", 1,
     [lambda o: pins.test_wkv6_backward_finite_differences(o, True)]),
    ("bwd_du_missing_vdy", "du[h * N + i] += rt[i] * kt[i] * vdy;", "du[h * N + i] += rt[i] * kt[i];", 0,
     [lambda o: pins.test_golden_wkv6_backward(o, "causal"),
      lambda o: pins.test_wkv6_backward_euler_identities(o, False)]),
    ("bwd_dk_drops_bonus", "dkt[i] += acck + u[h * N + i] * rt[i] * vdy;", "dkt[i] += acck;", 0,
     [lambda o: pins.test_wkv6_backward_matches_pair_form(o, False, 9, 4)]),
    ("state_initial_transposed", "if (s_init) memcpy(S, s_init, sizeof(double) * (size_t)N * N);",
     "if (s_init) { for (int i = 0; i < N; ++i) for (int j = 0; j < N; ++j) S[i * N + j] = s_init[j * N + i]; }",
     0, [lambda o: pins.test_wkv6_state_matches_pair_form(o, 1, 7, 2, 8)]),
    ("state_out_is_initial", "if (sT) memcpy(sT + off, S, sizeof(double) * NN);",
     "if (sT) memcpy(sT + off, s0 ? s0 + off : S, sizeof(double) * NN);", 0,
     [lambda o: pins.test_wkv6_state_matches_pair_form(o, 2, 3, 1, 4), lambda o: pins.test_wkv6_state_split_equals_whole(o, 13)]),
    ("wkv4_bwd_dk_drops_y", "dk[IDX(b, s, c)] += g * e * (vs - yt);", "dk[IDX(b, s, c)] += g * e * vs;", 0,
     [lambda o: pins.test_wkv4_backward_finite_differences(o, 2, 5, 3), pins.test_wkv4_backward_invariants]),
    ("wkv4_bwd_dw_weight", "dw[c] -= (t - 1 - s) * g * e * (vs - yt);", "dw[c] -= (t - s) * g * e * (vs - yt);", 0,
     [lambda o: pins.test_wkv4_backward_finite_differences(o, 2, 5, 3)]),
    ("wkv4_bwd_bonus_dv_missing", "dv[IDX(b, t, c)] += g * ett;", "dv[IDX(b, t, c)] += 0.0 * ett;", 0,
     [pins.test_wkv4_backward_invariants]),
    ("wkv4_decay_sign", "e1 = exp(p - w[c] - q);", "e1 = exp(p + w[c] - q);", 0,
     [pins.test_wkv4_geometric_closed_form, pins.test_golden_wkv4_forward]),
    ("wkv4_missing_bonus", "e2 = exp(u[c] + kt - q);", "e2 = exp(kt - q);", 0,
     [pins.test_golden_wkv4_forward, lambda o: pins.test_wkv4_recurrence_matches_ratio_of_sums(o, 2, 5, 3)]),
    ("wkv5_decay_sign", "const double d = exp(-w[h * N + i]);", "const double d = exp(w[h * N + i]);", 0,
     [pins.test_wkv5_geometric_closed_form, lambda o: pins.test_wkv5_is_wkv6_with_constant_decay(o, 2, 7, 2, 4)]),
    ("wkv5_readout_before_bonus", "acc += rt[i] * (S[i * N + j] + u[h * N + i] * kt[i] * vt[j]);",
     "acc += rt[i] * S[i * N + j];", 0, [pins.test_wkv5_geometric_closed_form]),
    ("wkv5_bwd_dw_sign", "dw[h * N + i] -= exp(-wh[i]) * accw;", "dw[h * N + i] += exp(-wh[i]) * accw;", 0,
     [pins.test_wkv5_backward_finite_differences, pins.test_wkv5_backward_matches_summed_wkv6_pair_form]),
    ("wkv5_bwd_adjoint_without_decay", "A[i * N + j] = rt[i] * gt[j] + exp(-wh[i]) * A[i * N + j];",
     "A[i * N + j] = rt[i] * gt[j] + A[i * N + j];", 0, [pins.test_wkv5_backward_finite_differences]),
    ("fused_no_mean", "for (int i = 0; i < N; ++i) mu += yh[i];", "for (int i = 0; i < N; ++i) mu += 0.0 * yh[i];", 0,
     [pins.test_fused_rows_are_normalised_per_head, lambda o: pins.test_fused_matches_library_group_norm(o, False)]),
    ("fused_gate_before_bias", "out[row * C + c] = ((yh[i] - mu) * inv * gn_w[c] + gn_b[c]) * g[row * C + c];",
     "out[row * C + c] = (yh[i] - mu) * inv * gn_w[c] * g[row * C + c] + gn_b[c];", 0,
     [pins.test_fused_scale_invariance_and_affine_order]),
    ("fused_decay_sign", "ew[e] = -exp(w_base[e % C] + ww[e]);", "ew[e] = -exp(w_base[e % C] - ww[e]);", 0,
     [pins.test_fused_prologue_moves_constant_between_base_and_lora]),
    ("fused_var_without_eps", "const double inv = 1.0 / sqrt(var + eps);", "const double inv = 1.0 / sqrt(var);", 0,
     [lambda o: pins.test_fused_matches_library_group_norm(o, True)]),
    ("wkv4_no_shift_update", "                p = q;\n", "", 0,
     [lambda o: pins.test_wkv4_recurrence_matches_ratio_of_sums(o, 1, 40, 4), pins.test_wkv4_large_keys_stay_finite]),
]


def _replace_nth(src, old, new, n):
    pos = -1
    for _ in range(n + 1):
        pos = src.index(old, pos + 1)
    return src[:pos] + new + src[pos + len(old):]


@pytest.mark.parametrize("mid,old,new,nth,checks", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, oracle_mod, mid, old, new, nth, checks):
    src = oracle.source()
    assert src.count(old) >= nth + 1, f"mutation site for {mid} not found"
    mutant = oracle.compile_variant(_replace_nth(src, old, new, nth), str(tmp_path / f"{mid}.so"))
    for check in checks:
        check(oracle_mod)                    # the real oracle passes
        with pytest.raises(AssertionError):  # the mutant fails
            check(mutant)
