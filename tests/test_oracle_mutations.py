"""Each pin set must catch a plausible mistake planted in the oracle.

A mutation is a textual edit of oracle/sla_oracle.py, executed as a separate
module on the CPU; the real oracle is untouched.  Every mutation must make at
least one pin fail.
"""
import os
import types

import pytest

from tests.oracle_pins import ALL_PINS

SRC = open(os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "sla_oracle.py")).read()

MUTATIONS = {
    "phi_drops_plus_one": ("np.where(x > 0, x + 1.0, np.exp", "np.where(x > 0, x, np.exp"),
    "sparse_no_sqrt_d": ("(q[rows] @ k[keys].T) / math.sqrt(d)", "(q[rows] @ k[keys].T)"),
    "linear_H_transposed": ("Hm = pk.T @ v[keys]", "Hm = (pk.T @ v[keys]).T"),
    "linear_no_denominator": ("(pq @ Hm) / (pq @ Z)[:, None]", "(pq @ Hm)"),
    "alpha_swapped": ("a * o_s + (1.0 - a) * o_l", "(1.0 - a) * o_s + a * o_l"),
    "pool_divides_by_block_size": ("return acc / counts.astype(F32)[None, None, :, None]",
                                   "return acc / F32(b)"),
    "project_uses_W_transpose": ("fma32(xbar32[..., e:e + 1], w32[e, :], acc)", "fma32(xbar32[..., e:e + 1], w32[:, e], acc)"),
    "fma_rounds_twice": ("    s = np.where((e != 0) & even, step, s)\n", ""),
    "score_mul_then_add": ("acc = fma32(qt32[..., :, c, None], kt32[..., None, :, c], acc)",
                           "acc = (acc + qt32[..., :, c, None] * kt32[..., None, :, c]).astype(F32)"),
    "ties_prefer_higher_index": ('return np.argsort(-scores, axis=-1, kind="stable")',
                                 'return scores.shape[-1] - 1 - np.argsort(-scores[..., ::-1], axis=-1, kind="stable")'),
    "negligible_taken_from_top": ("order[..., n_kv - k_l:]", "order[..., k_h:k_h + k_l]"),
    "sla_proj_transposed": ("o_s + o_l @ wp", "o_s + o_l @ wp.T"),
    "sla_linear_includes_negligible": ("np.nonzero(lab == 0)", "np.nonzero(lab <= 0)"),
    "keep_count_truncates": ("ratio * n_kv + 0.5", "ratio * n_kv"),
    "e4m3_truncates": ("q = np.rint((f - 1.0) * 8.0)", "q = np.floor((f - 1.0) * 8.0)"),
    "unselected_uses_kept": ("uns = [j for j in range(n_kv) if j not in set(sel)]",
                             "uns = [j for j in range(n_kv)]"),
    "fp8_no_k_smoothing": ("kp32 = (ks - mu).astype(F32)", "kp32 = ks.astype(F32)"),
    "fp8_p_not_rescaled": ("p8 = _e4m3_q((p * 448.0).astype(F32), codec) / 448.0",
                           "p8 = _e4m3_q((p * 448.0).astype(F32), codec)"),
    "fp8_tile_drops_blocks": ("sel[g0:g0 + kv_tile]", "sel[g0:g0 + 1]"),
    "fp8_tile_width_ignored": ("for g0 in range(0, len(sel), kv_tile):", "for g0 in range(0, len(sel), kv_tile):\n                kv_tile = 1"),
    "fp8_key_scale_of_row_block": ("kdq = k8[keys] * sk[tok_q[keys]][:, None]",
                                   "kdq = k8[keys] * sk[tok_q[rows[0]]]"),
    "soft_topk_tau_ignored": ("x = np.asarray(scores, dtype=np.float64) / tau",
                              "x = np.asarray(scores, dtype=np.float64)"),
    "soft_topk_bisection_backwards": ("lo = np.where(below, mid, lo)\n        hi = np.where(below, hi, mid)",
                                      "lo = np.where(below, lo, mid)\n        hi = np.where(below, mid, hi)"),
    "sigmoid_sign_flipped": ("out[pos] = 1.0 / (1.0 + np.exp(-z[pos]))", "out[pos] = 1.0 / (1.0 + np.exp(z[pos]))"),
    "bwd_softmax_drops_D": ("ds = p * (dp - D)", "ds = p * dp"),
    "bwd_dq_no_sqrt_d": ("dq = ds @ k[keys] / math.sqrt(d)", "dq = ds @ k[keys]"),
    "bwd_dk_uses_k": ("dk = ds.T @ q[rows] / math.sqrt(d)", "dk = ds.T @ k[keys] / math.sqrt(d)"),
    "bwd_dv_from_unnormalised_p": ("dv = p.T @ do_s", "dv = np.exp(s - s.max(axis=1, keepdims=True)).T @ do_s"),
    "bwd_denominator_sign": ("dden = -(do_l * o).sum(axis=1) / den", "dden = (do_l * o).sum(axis=1) / den"),
    "bwd_phi_k_drops_dZ": ("dpk = v[keys] @ dH.T + dZ[None, :]", "dpk = v[keys] @ dH.T"),
    "bwd_phi_q_drops_Z_term": ("dpq = dnum @ Hm.T + dden[:, None] * Z[None, :]", "dpq = dnum @ Hm.T"),
    "bwd_dH_transposed": ("dv = pk @ dH\n", "dv = pk @ dH.T\n"),
    "bwd_elu_derivative_one": ("return dphi * np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))", "return dphi"),
    "bwd_softmax_phi_jacobian_sign": ("return p * (dphi - (dphi * p).sum(axis=-1, keepdims=True))",
                                      "return p * (dphi + (dphi * p).sum(axis=-1, keepdims=True))"),
    "bwd_alpha_not_applied": ("sparse_branch_backward(qs, ks, vs, rows, ts, a * g)",
                              "sparse_branch_backward(qs, ks, vs, rows, ts, g)"),
    "bwd_dalpha_sign": ("dalpha[b, h, i] = (g * (o_s - o_l)).sum()", "dalpha[b, h, i] = (g * (o_l - o_s)).sum()"),
    "bwd_sla_proj_not_transposed": ("g @ wp.T, phi_kind)", "g @ wp, phi_kind)"),
    "bwd_sla_dwproj_transposed": ("dwp += o_l.T @ g", "dwp += g.T @ o_l"),
    "int8_rounds_half_up": ("np.clip(np.rint(np.asarray(x32, dtype=F64)), -127.0, 127.0)",
                            "np.clip(np.floor(np.asarray(x32, dtype=F64) + 0.5), -127.0, 127.0)"),
    "int8_saturates_at_128": ("np.clip(np.rint(np.asarray(x32, dtype=F64)), -127.0, 127.0)",
                              "np.clip(np.rint(np.asarray(x32, dtype=F64)), -128.0, 128.0)"),
    "int8_variant_keeps_448": ("qk_codec=int8_round, qk_max=127.0)", "qk_codec=int8_round, qk_max=448.0)"),
    "quant_blocks_ignores_qmax": ("inv = F32(qmax) / amax", "inv = F32(448.0) / amax"),
}


def _mutant(old, new):
    assert SRC.count(old) >= 1, old  # applied wherever the line occurs
    mod = types.ModuleType("sla_oracle_mutant")
    exec(compile(SRC.replace(old, new), "sla_oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name):
    mod = _mutant(*MUTATIONS[name])
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutation {name}"
