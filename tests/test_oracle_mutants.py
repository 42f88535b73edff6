"""Every plausible slip in the oracle must be caught by at least one pin.

Each mutant is a copy of oracle/gdla_oracle.c with one planted mistake (a
dropped term, a wrong sign, a wrong or transposed index, an off-by-one mask),
compiled on the CPU into a scratch directory.  The test runs the pins of
tests/oracle_pins.py against it and requires at least one of them to fail.
Every mutant keeps all memory accesses in bounds.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    "sign_of_noise_term": ("- l * hn[", "+ l * hn["),
    "dropped_lambda": ("- l * hn[", "- hn["),
    "repeat_tiled_not_interleaved": ("const int n = h / g;", "const int n = h % Hn;"),
    "kv_head_tiled": ("int kvh = h / group;", "int kvh = h % Hkv;"),
    "window_off_by_one": ("if (window > 0 && i - window + 1 > 0) *lo = i - window + 1;",
                          "if (window > 0 && i - window > 0) *lo = i - window;"),
    "causal_excludes_diagonal": ("*hi = i;", "*hi = i > 0 ? i - 1 : 0;"),
    "dropped_gate": ("= gv * diff;", "= diff;"),
    "dropped_scale": ("s[j - lo] = scale * dot;", "s[j - lo] = dot;"),
    "dropped_normaliser": ("o[c] = acc[c] / denom;", "o[c] = acc[c];"),
    "values_read_from_keys": ("acc[c] += p * load_elem(v, v_dt, voff + c);",
                              "acc[c] += p * load_elem(k, k_dt, voff + c);"),
    "gate_index_transposed": ("(int64_t)h * d + c);", "(int64_t)c * Hs + h);"),
    "lambda_head_reversed": ("load_elem(lam, lam_dt, row * Hs + h);",
                             "load_elem(lam, lam_dt, row * Hs + (Hs - 1 - h));"),
    "rms_dropped_eps": ("sqrt(ss / (double)d_latent + eps)", "sqrt(ss / (double)d_latent)"),
    "rms_sum_not_mean": ("sqrt(ss / (double)d_latent + eps)", "sqrt(ss + eps)"),
    "expand_w_transposed": ("(int64_t)k * ncol + col)", "col * d_latent + k)"),
    "expand_k_v_swapped": ("if (x < dk)\n        k_out", "if (x >= dk)\n        k_out"),
    "rope_term_dropped": ("        for (int c = 0; c < dr; ++c)\n          dot +=",
                          "        for (int c = 0; c < 0; ++c)\n          dot +="),
    "rope_key_of_the_query_token": ("load_elem(kr, kr_dt, (b * T + j) * (int64_t)dr + c);",
                                    "load_elem(kr, kr_dt, (b * T + i) * (int64_t)dr + c);"),
    "rope_query_of_head_zero": ("const int64_t qroff = ((q_compact ? ri : row) * H + h)",
                                "const int64_t qroff = ((q_compact ? ri : row) * H + 0)"),
    "rope_sign": ("          dot += load_elem(qr, qr_dt, qroff + c) *",
                  "          dot -= load_elem(qr, qr_dt, qroff + c) *"),
    "decode_rope_key_of_first_cached_token": ("kr_b = ORACLE_AT(kr, kr_dt, ((int64_t)b * L_max + first) * dr);",
                                              "kr_b = ORACLE_AT(kr, kr_dt, ((int64_t)b * L_max) * dr);"),
    "bwd_softmax_jacobian_without_delta": ("const double ds = p[j - lo] * (dp[j - lo] - delta);",
                                           "const double ds = p[j - lo] * dp[j - lo];"),
    "bwd_dlambda_sign": ("dl -= ddd * hnv;", "dl += ddd * hnv;"),
    "bwd_dhn_without_lambda": ("dhn[(row * Hn + n) * d + c] -= l * ddd;",
                               "dhn[(row * Hn + n) * d + c] -= ddd;"),
    "bwd_dk_unscaled": ("dk[koff + c] += scale * ds *", "dk[koff + c] += ds *"),
    "bwd_dv_from_ds": ("dv[koff + c] += p[j - lo] * dh[qoff + c];",
                       "dv[koff + c] += ds * dh[qoff + c];"),
    "bwd_dgate_from_signal_only": ("dgate[oc] = go * dd;",
                                   "dgate[oc] = go * hs[(row * Hs + h) * d + c];"),
    "decode_query_is_first_token": ("const int64_t row = L - 1;", "const int64_t row = 0;"),
    "decode_window_slice_drops_oldest_key": ("(window > 0 && Lb > window) ? Lb - window : 0",
                                             "(window > 0 && Lb >= window) ? Lb - window + 1 : 0"),
    "decode_cache_stride_by_length": ("((int64_t)b * L_max + first) * d_latent",
                                      "((int64_t)b * Lb + first) * d_latent"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(oracle.SOURCE).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    if name == "expand_k_v_swapped":
        # keep the store indices in range after swapping the branches
        mutated = mutated.replace("k_out[(t * n_kv_heads + h) * dk + x] = acc;",
                                  "k_out[(t * n_kv_heads + h) * dk + (x - dk)] = acc;", 1)
        mutated = mutated.replace("v_out[(t * n_kv_heads + h) * dv + (x - dk)] = acc;",
                                  "v_out[(t * n_kv_heads + h) * dv + x] = acc;", 1)
    path = os.path.join(str(tmp_path), "mutant.c")
    with open(path, "w") as f:
        f.write(mutated)
    lib = oracle.compile_source(path, os.path.join(str(tmp_path), "libmutant.so"))
    o = oracle.Oracle(lib)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except AssertionError:
            caught.append(pin.__name__)
            break
    assert caught, f"no pin catches the planted mistake '{name}'"
